// bias_project.cuh -- the N x N products of the low-rank factoriser of a
// materialised bias ("FlashBias: Fast Computation of Attention with Bias",
// Abstract: a low-rank bias keeps attention fast; the factoriser produces the
// factors U, W of a dense per-head bias):
//
//     out[h] = B[h] X[h]      or      out[h] = B[h]^T X[h],
//
// B [H, N, N] fp32, X [H, N, k] fp32 with k <= 80 (rank plus oversampling),
// out [H, N, k] fp32, accumulated in fp32.  Each product reads the bias once
// (4 N^2 bytes per head) for 2 N^2 k flops, i.e. k / 2 flop per byte.  This
// is a SIMT fp32 kernel: it reads B once, coalesced, keeps chunks of X and
// the accumulators on chip, and is bound by the fp32 FMA rate for k above
// about 20 (the factoriser runs once per model, not per attention step, and
// keeps fp32 accuracy in its subspace iteration).
#pragma once
#include <cstdint>

#include "sm100.cuh"

namespace rfb {

constexpr int kProjRows = 128;    // output rows per CTA
constexpr int kProjChunk = 32;    // reduction step
constexpr int kProjMaxK = 80;     // columns of X (padded in shared memory)
constexpr int kProjThreads = 256; // 16 x 16: 8 output rows x 5 columns per thread

// One CTA: output rows [r0, r0 + 128) of head blockIdx.y.  Reduction over the
// N rows (TRANS: the first index of B) or columns (otherwise) of B in chunks
// of 32, each chunk of B staged transposed-or-not so that the inner loop reads
// Bs[out row][reduction index].
template <bool TRANS>
__global__ void __launch_bounds__(kProjThreads) bias_project_kernel(const float* __restrict__ B,
                                                                   const float* __restrict__ X,
                                                                   float* __restrict__ out, int N,
                                                                   int k) {
  __shared__ float Bs[kProjRows][kProjChunk + 1];
  __shared__ float Xs[kProjChunk][kProjMaxK];
  grid_dep_wait();
  const int h = blockIdx.y;
  const int r0 = blockIdx.x * kProjRows;
  const float* Bh = B + static_cast<size_t>(h) * N * N;
  const float* Xh = X + static_cast<size_t>(h) * N * k;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[8][5];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < 5; ++b) acc[a][b] = 0.f;
  for (int j0 = 0; j0 < N; j0 += kProjChunk) {
    // B chunk: rows = output rows r0.., cols = reduction j0.. (not TRANS);
    // TRANS reads B[j0 + jj][r0 + rr] (rows of B contiguous in rr).
    for (int t = threadIdx.x; t < kProjRows * kProjChunk; t += kProjThreads) {
      float v = 0.f;
      if constexpr (TRANS) {
        const int jj = t / kProjRows, rr = t % kProjRows;
        if (j0 + jj < N && r0 + rr < N) v = Bh[static_cast<size_t>(j0 + jj) * N + r0 + rr];
        Bs[rr][jj] = v;
      } else {
        const int rr = t / kProjChunk, jj = t % kProjChunk;
        if (r0 + rr < N && j0 + jj < N) v = Bh[static_cast<size_t>(r0 + rr) * N + j0 + jj];
        Bs[rr][jj] = v;
      }
    }
    for (int t = threadIdx.x; t < kProjChunk * kProjMaxK; t += kProjThreads) {
      const int jj = t / kProjMaxK, c = t % kProjMaxK;
      Xs[jj][c] = (j0 + jj < N && c < k) ? Xh[static_cast<size_t>(j0 + jj) * k + c] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int jj = 0; jj < kProjChunk; ++jj) {
      float a[8], b[5];
#pragma unroll
      for (int u = 0; u < 8; ++u) a[u] = Bs[ty * 8 + u][jj];
#pragma unroll
      for (int v = 0; v < 5; ++v) b[v] = Xs[jj][tx * 5 + v];
#pragma unroll
      for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int v = 0; v < 5; ++v) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
    }
    __syncthreads();
  }
  float* oh = out + static_cast<size_t>(h) * N * k;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int row = r0 + ty * 8 + u;
    if (row >= N) continue;
#pragma unroll
    for (int v = 0; v < 5; ++v) {
      const int c = tx * 5 + v;
      if (c < k) oh[static_cast<size_t>(row) * k + c] = acc[u][v];
    }
  }
}

}  // namespace rfb
