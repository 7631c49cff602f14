// bwd_kernels.cuh -- backward of O = softmax(s Q K^T + U W^T) V on sm_100a.
//
// Chain rule through the same definition (dP = dO V^T, D_i = sum_j P_ij dP_ij,
// dS = P o (dP - D)):
//     dQ = s dS K     dU = dS W     dK = s dS^T Q     dW = dS^T U     dV = P^T dO.
// With U' = U / s staged on chip the bias side rides the same contractions as
// the content side ("Rank-Factorized Implicit Neural Bias", Abstract:
// concatenation turns the bias into part of one dot product):
//     S^T/s = [K | W] . [Q | U']^T         (one accumulation, recompute of P)
//     [dK | dW] = s dS^T . [Q | U']        (dW = s dS^T U' = dS^T U)
//     [dQ | dU] = dS . [K | W] with per-column scales (s | 1).
//
// Three kernels:
//   bwd_pre  : D_i = rowsum(dO o O) (equal to sum_j P_ij dP_ij because O = P V)
//              and LSE_i log2(e), both stored negated, U' = bf16(U / s), and
//              zeroes the fp32 dQ|dU accumulator.
//   bwd_main : one CTA per (head, 128-key tile); K, W, V stay in shared memory,
//              dV, dK, dW accumulate in TMEM across all 128-query tiles.  Per
//              query tile: S^T and dP^T by tcgen05 into TMEM; two compute
//              warpgroups (64 query columns each) form P^T and dS^T, write P^T
//              back into TMEM in place (bf16) and dS^T into swizzled shared
//              memory; dV (+=) reads its A operand P^T from TMEM, dK and dW
//              (+=) read dS^T from shared memory, so that the next tile's
//              dP^T can be issued as soon as the softmax has read dP^T and
//              its S^T as soon as dV is done (the tensor pipe stays fed);
//              the partial dQ|dU tile goes to TMEM columns of its own (when
//              they fit), which four reduction warps of their own stage in
//              128-byte-swizzled shared memory and add into the fp32
//              accumulator with TMA bulk tensor reductions, each warp its own
//              32 query rows, while the softmax warps go on with the next
//              tile.  Each query half (one warpgroup's 64 columns) has
//              barriers of its own: S^T / dP^T of a half (N = 64 MMAs) and its
//              dV / dK / dW MMAs are issued as soon as that half is ready, so
//              one half's MMAs overlap the other half's softmax.  All MMAs are
//              issued by one converged warp.
//   bwd_post : dQ = bf16(acc[:, :d]), dU = bf16(acc[:, d:d+r]) (with shared
//              factors dU and dW are instead summed over the windows by
//              sum_bias_grads_kernel in bwd_window.cuh).
#pragma once
#include "fwd_kernels.cuh"

namespace rfb {

constexpr float kLog2e = 1.4426950408889634f;

struct BwdArgs {
  const __nv_bfloat16* o;     // [BH, N, D]
  const float* lse;           // [BH, N]
  const __nv_bfloat16* dout;  // [BH, N, D]
  const __nv_bfloat16* u;     // [BH, N, r]   bias factor U
  __nv_bfloat16* uprime;      // [BH, N, r]   U' = bf16(U / s), written by bwd_pre
  // [BH, Npad, 16] bf16 per query row: -LSE_i / s and -D_i, each as three
  // bf16 parts (columns 0-2 and 3-5; hi + mid + lo carries fp32 precision),
  // zeros elsewhere.  The score MMAs add them to S^T / s and dP^T through a
  // constant operand of ones, so the softmax needs no per-query loads.
  __nv_bfloat16* aug;
  float* acc;                 // [BH, N, D + r] fp32 dQ | dU accumulator
  __nv_bfloat16* dq;          // [BH, N, D]
  __nv_bfloat16* dk;          // [BH, N, D]
  __nv_bfloat16* dv;          // [BH, N, D]
  __nv_bfloat16* du;          // [BH, N, r]
  __nv_bfloat16* dw;          // [BH, N, r]  (per-window factors)
  float* dw_part;             // [BH, N, r]  fp32 dW of each window-head (shared factors)
  int* err;
  int BH, N, Npad, D, r;
  int bias_heads;             // BH (per-window factors) or H (shared; bias head = bh % H)
  float scale;       // s
  float scale_log2;  // s log2(e)
  float inv_scale;   // 1/s
  uint64_t timeout_ns;  // limit of each main-loop wait
  int fail_site;        // test hook: wait site that gives up at once (-1: none)
  // Shifted-window mask of image windows (N = 64, tokens in raster order
  // inside each 8 x 8 window; 0 = no mask): window-head bh is window
  // (bh / mask_heads) of a map of mask_nwy x mask_nwx windows per image.
  int mask_shift, mask_nwx, mask_nwy, mask_heads;
};

// Image windows <-> window tensors.  Window-head bh = ((b * nwy + wy) * nwx +
// wx) * heads + h, token n = 8 ty + tx (raster order inside the window) is the
// map token (b, (8 wy + ty + shift) mod img_h, (8 wx + tx + shift) mod img_w)
// of head h: the window cut of the map rolled by (-shift, -shift).  Moves
// `ntensor` bf16 tensors (and optionally the fp32 LSE) between the map layout
// [B, img_h, img_w, heads, d] and the window layout [BH, 64, d], in either
// direction; every position is written exactly once.
struct ImgMoveArgs {
  const __nv_bfloat16* src[5];
  __nv_bfloat16* dst[5];
  const float* lse_src;  // NULL: no LSE to move
  float* lse_dst;
  int ntensor, BH, img_h, img_w, heads, d, shift;
  int to_windows;  // 1: maps -> windows, 0: windows -> maps
};

__global__ void __launch_bounds__(256) img_move_kernel(const ImgMoveArgs a) {
  grid_dep_wait();
  const int G = a.d / 8;  // 16-byte pieces per token row
  const long long total = static_cast<long long>(a.BH) * 64 * G;
  const int nwx = a.img_w / 8, nwy = a.img_h / 8;
  for (long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int g = static_cast<int>(t % G);
    const long long wrow = t / G;  // bh * 64 + n
    const int n = static_cast<int>(wrow % 64);
    const int bh = static_cast<int>(wrow / 64);
    const int h = bh % a.heads, bw = bh / a.heads;
    const int wx = bw % nwx, wy = (bw / nwx) % nwy, b = bw / (nwx * nwy);
    const int y = (wy * 8 + (n >> 3) + a.shift) % a.img_h;
    const int x = (wx * 8 + (n & 7) + a.shift) % a.img_w;
    const long long mrow = ((static_cast<long long>(b) * a.img_h + y) * a.img_w + x) * a.heads + h;
    const long long srow = a.to_windows ? mrow : wrow, drow = a.to_windows ? wrow : mrow;
    for (int i = 0; i < a.ntensor; ++i) {
      const uint4 v = reinterpret_cast<const uint4*>(a.src[i] + srow * a.d)[g];
      reinterpret_cast<uint4*>(a.dst[i] + drow * a.d)[g] = v;
    }
    if (g == 0 && a.lse_src != nullptr) a.lse_dst[drow] = a.lse_src[srow];
  }
}

// x as the sum of three bf16 values (each returned as the float it rounds to):
// hi = bf16(x), mid = bf16(x - hi), lo = bf16(x - hi - mid); the remainder is
// below 2^-24 |x|, as for fp32.
__device__ __forceinline__ void split3_bf16(float x, float (&p)[3]) {
  p[0] = __bfloat162float(__float2bfloat16_rn(x));
  const float r1 = x - p[0];
  p[1] = __bfloat162float(__float2bfloat16_rn(r1));
  p[2] = __bfloat162float(__float2bfloat16_rn(r1 - p[1]));
}

// ------------------------------------------------------------------ bwd_pre
// Thread group of G = D/8 lanes per row (16-byte loads); rows grid-strided.
__global__ void __launch_bounds__(256) bwd_pre_kernel(const BwdArgs a) {
  grid_dep_wait();
  const int G = a.D / 8;
  const int rows_per_block = 256 / G;
  const int sub = threadIdx.x % G;
  const long total_rows = static_cast<long>(a.BH) * a.Npad;
  for (long row = static_cast<long>(blockIdx.x) * rows_per_block + threadIdx.x / G; row < total_rows;
       row += static_cast<long>(gridDim.x) * rows_per_block) {
    const int bh = static_cast<int>(row / a.Npad);
    const int i = static_cast<int>(row % a.Npad);
    float dsum = 0.f, lse = 0.f;
    if (i < a.N) {
      const size_t base = (static_cast<size_t>(bh) * a.N + i) * a.D + sub * 8;
      const uint4 ov = *reinterpret_cast<const uint4*>(a.o + base);
      const uint4 gv = *reinterpret_cast<const uint4*>(a.dout + base);
      const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w};
      const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        dsum = fmaf(__uint_as_float(ow[e] << 16), __uint_as_float(gw[e] << 16), dsum);
        dsum = fmaf(__uint_as_float(ow[e] & 0xFFFF0000u), __uint_as_float(gw[e] & 0xFFFF0000u), dsum);
      }
      lse = a.lse[static_cast<size_t>(bh) * a.N + i];
    }
    for (int off = G / 2; off > 0; off >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off, G);
    if (sub == 0) {
      // Padding rows (i >= N) get zeros; their scores are masked anyway.
      uint32_t w[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
      if (i < a.N) {
        float c[3], dd[3];
        split3_bf16(-lse * a.inv_scale, c);
        split3_bf16(-dsum, dd);
        w[0] = pack_bf16x2(c[0], c[1]);
        w[1] = pack_bf16x2(c[2], dd[0]);
        w[2] = pack_bf16x2(dd[1], dd[2]);
      }
      uint4* dst = reinterpret_cast<uint4*>(a.aug + static_cast<size_t>(row) * 16);
      dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
      dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
  }
  // Zero the dQ | dU accumulator.
  const size_t n4 = static_cast<size_t>(a.BH) * a.N * (a.D + a.r) / 4;
  float4* acc4 = reinterpret_cast<float4*>(a.acc);
  for (size_t t = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < n4;
       t += static_cast<size_t>(gridDim.x) * blockDim.x)
    acc4[t] = make_float4(0.f, 0.f, 0.f, 0.f);
  // U' = bf16(U / s), staged once here instead of once per (key tile, query tile).
  const size_t n8 = static_cast<size_t>(a.bias_heads) * a.N * a.r / 8;
  for (size_t t = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < n8;
       t += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint4 v = reinterpret_cast<const uint4*>(a.u)[t];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      o[e] = pack_bf16x2(__uint_as_float(w[e] << 16) * a.inv_scale,
                         __uint_as_float(w[e] & 0xFFFF0000u) * a.inv_scale);
    reinterpret_cast<uint4*>(a.uprime)[t] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// ----------------------------------------------------------------- bwd_post
__global__ void __launch_bounds__(256) bwd_post_kernel(const BwdArgs a) {
  grid_dep_wait();
  const int DA = a.D + a.r;
  const int groups = DA / 8;
  const long total = static_cast<long>(a.BH) * a.N * groups;
  for (long t = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<long>(gridDim.x) * blockDim.x) {
    const long row = t / groups;
    const int c = static_cast<int>(t % groups) * 8;
    const float4* src = reinterpret_cast<const float4*>(a.acc + row * DA + c);
    const float4 x = src[0], y = src[1];
    uint4 v;
    v.x = pack_bf16x2(x.x, x.y);
    v.y = pack_bf16x2(x.z, x.w);
    v.z = pack_bf16x2(y.x, y.y);
    v.w = pack_bf16x2(y.z, y.w);
    if (c < a.D)
      *reinterpret_cast<uint4*>(a.dq + row * a.D + c) = v;
    else if (a.bias_heads == a.BH)
      *reinterpret_cast<uint4*>(a.du + row * a.r + (c - a.D)) = v;
  }
}

template <int D, int RP>
struct BwdCfg {
  static constexpr int QB = kTile * D * 2;
  static constexpr int UB = kTile * RP * 2;
  // With d = 64, U' and W are staged 64 columns wide (128-byte rows, zero
  // padded beyond r) so that [Q | U'] and [K | W] each form one MN-major B
  // operand of two 128-byte swizzle atoms: dK | dW and dQ | dU each come from a
  // single MMA chain (N = d + r_pad).
  static constexpr bool MERGE_KW = (D == 64) && (RP > 0);
  static constexpr int UW = MERGE_KW ? 64 : RP;     // staged width of U' and W
  static constexpr int UQB = kTile * UW * 2;        // bytes of a staged U' or W tile
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = QB;
  static constexpr int OFF_W = 2 * QB;
  static constexpr int KVB = 2 * QB + UQB;
  // Two constant K-major A tiles [128 x 16] bf16 (32-byte rows and swizzle):
  // ones in columns 0-2 (they add the -LSE / s parts of the query rows' aug
  // rows to S^T / s) and in columns 3-5 (the -D parts, to dP^T).
  static constexpr int OFF_ONES = KVB;
  static constexpr int ONEB = kTile * 32;
  // stage: Q, dO, U', the 128 query rows' aug rows (32 bytes each)
  static constexpr int S_Q = 0, S_DO = QB, S_U = 2 * QB, S_AUG = 2 * QB + UQB;
  static constexpr int STAGE = 2 * QB + UQB + kTile * 32;
  static constexpr int PB = kTile * kTile * 2;  // one dS tile (bf16)
  static constexpr int NCH = (D + RP + 31) / 32;  // dQ | dU chunks of 32 columns
  // TMEM columns.  When dQ | dU fit in columns of their own (DEFER), the next
  // tile's S^T / dP^T MMAs are issued before tile i's dQ | dU MMAs and the
  // reduction of tile i overlaps the next tile's softmax, so the dS tile in
  // shared memory is double buffered.  Otherwise dQ | dU reuse the S^T
  // columns and each tile runs its phases in order.
  static constexpr int T_S = 0, T_DP = 128, T_DV = 256, T_DK = 256 + D, T_DW = 256 + 2 * D;
  static constexpr bool DEFER = (256 + 2 * D + RP + NCH * 32) <= 512;
  static constexpr int T_DQ = DEFER ? 256 + 2 * D + RP : 0;
  static constexpr int NDS = DEFER ? 2 : 1;
  // The dQ | dU chunks are staged for their TMA reductions in the two 64-query
  // blocks (16 KB each) of the tile's dS buffer, free once dQ's MMAs have
  // read it: chunk c in block c & 1, chunks 2 and 3 once the copies of
  // chunks 0 and 1 have read theirs.
  // The dynamic shared memory is declared 1024-byte aligned (no slack); 256
  // bytes are kept for the barriers.
  static constexpr int NS_FIT = (232448 - 256 - KVB - 2 * ONEB - NDS * PB) / STAGE;
  static constexpr int NS = NS_FIT > 3 ? 3 : NS_FIT;
  static constexpr int OFF_STAGE = KVB + 2 * ONEB;
  static constexpr int OFF_DS = OFF_STAGE + NS * STAGE;
  static constexpr int OFF_BAR = OFF_DS + NDS * PB;
  // kv_full q_full[NS] q_empty[NS] sdp_full[2] ds_full[2] dq_full dq_free drain a_done[2]
  // ds_free[2][2]
  static constexpr int NBAR = 2 * NS + 14;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16;
  static_assert(NS >= 2, "shared memory budget");
  static_assert(OFF_STAGE % 1024 == 0 && STAGE % 1024 == 0, "stage alignment");
  static_assert(SMEM <= 232448, "shared memory budget exceeded");
  static_assert(T_DW + RP <= 512 && NCH * 32 <= 128, "TMEM budget");
};

// warps 0-7 softmax (two warpgroups), 8 TMA, 9 MMA, 10-13 dQ | dU reduction
constexpr int kBwdThreads = 448;

template <int D, int RP>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                    const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mU,
                    const __grid_constant__ CUtensorMap mW, const __grid_constant__ CUtensorMap mDO,
                    const __grid_constant__ CUtensorMap mAcc,
                    const __grid_constant__ CUtensorMap mAug, const BwdArgs args) {
  using C = BwdCfg<D, RP>;
  constexpr int NS = C::NS;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  const uint32_t sb = smem_u32(smem);
  if (sb & 1023u) {  // the swizzled operand tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicCAS(args.err, 0, kErrAlignment | (98 << 8));
    return;
  }
  const uint32_t bar0 = sb + C::OFF_BAR;
  const uint32_t kv_full = bar0;
  auto q_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto q_empty = [&](int s) { return bar0 + 8u * (1 + NS + s); };
  // Query half h (columns 64h .. 64h + 63 of a tile, warpgroup h): its S^T and
  // dP^T are in TMEM, its P^T / dS^T are written, its dV MMAs (which read P^T
  // from TMEM) are done.
  auto sdp_full = [&](int h) { return bar0 + 8u * (1 + 2 * NS + h); };
  auto ds_full = [&](int h) { return bar0 + 8u * (3 + 2 * NS + h); };
  const uint32_t dq_full = bar0 + 8u * (5 + 2 * NS);
  const uint32_t dq_free = bar0 + 8u * (6 + 2 * NS);
  const uint32_t drain_bar = bar0 + 8u * (7 + 2 * NS);
  auto a_done = [&](int h) { return bar0 + 8u * (8 + 2 * NS + h); };
  // Block k (queries 64k .. 64k + 63) of dS buffer b: the reductions staged
  // in it have been read, so warpgroup k may write the next dS^T there.
  auto ds_free = [&](int b, int k) { return bar0 + 8u * (10 + 2 * NS + 2 * b + k); };
  auto ds_buf = [&](int i) { return sb + C::OFF_DS + (C::NDS == 2 ? (i & 1) : 0) * C::PB; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + C::NBAR * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = static_cast<int>(warp_id());
  const int lane = static_cast<int>(lane_id());
  const int N = args.N;
  const int bh = blockIdx.y;
  const int k0 = blockIdx.x * kTile;
  const int nq = (N + kTile - 1) / kTile;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(kv_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(q_full(s), 1);
      mbar_init(q_empty(s), 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(sdp_full(h), 1);
      mbar_init(ds_full(h), 4);   // one arrival per warp of the half's warpgroup
      mbar_init(a_done(h), 1);
    }
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 4);        // one arrival per reduction warp
    for (int b = 0; b < 2; ++b)
      for (int k = 0; k < 2; ++k) mbar_init(ds_free(b, k), 4);
    mbar_init(drain_bar, 1);
    fence_mbar_init();
  }
  {
    // The ones tiles: row r of tile t holds bf16 1.0 in columns 3t .. 3t + 2
    // (first 16-byte chunk of the row, stored at its 32-byte-swizzle place).
    const uint4 one_l = make_uint4(0x3F803F80u, 0x00003F80u, 0u, 0u);
    const uint4 one_d = make_uint4(0u, 0x3F800000u, 0x3F803F80u, 0u);
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    for (int idx = threadIdx.x; idx < 2 * kTile * 2; idx += kBwdThreads) {
      const int t = idx / (2 * kTile), r = (idx / 2) % kTile, c = idx & 1;
      uint4* dst = reinterpret_cast<uint4*>(smem + C::OFF_ONES + t * C::ONEB + swz_offset(r, c, 32));
      *dst = c != 0 ? zero : (t == 0 ? one_l : one_d);
    }
    fence_async_smem();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch(&mQ);
    tma_prefetch(&mK);
    tma_prefetch(&mV);
    tma_prefetch(&mDO);
    tma_prefetch(&mAcc);
    tma_prefetch(&mAug);
    if constexpr (RP > 0) {
      tma_prefetch(&mU);
      tma_prefetch(&mW);
    }
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitGuard g{abort_flag, args.err, args.timeout_ns, args.fail_site};
  grid_dep_wait();

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_expect_tx(kv_full, C::KVB);
      tma_load_3d(sb + C::OFF_K, &mK, kv_full, 0, k0, bh);
      tma_load_3d(sb + C::OFF_V, &mV, kv_full, 0, k0, bh);
      if constexpr (RP > 0) tma_load_3d(sb + C::OFF_W, &mW, kv_full, 0, k0, bh % args.bias_heads);
      int i = 0;
      for (; i < nq; ++i) {
        const int s = i % NS;
        if (i >= NS && !wait_bounded(q_empty(s), ((i / NS) + 1) & 1, g, 31)) break;
        const uint32_t st = sb + C::OFF_STAGE + s * C::STAGE;
        mbar_expect_tx(q_full(s), C::STAGE);
        tma_load_3d(st + C::S_Q, &mQ, q_full(s), 0, i * kTile, bh);
        tma_load_3d(st + C::S_DO, &mDO, q_full(s), 0, i * kTile, bh);
        if constexpr (RP > 0)
          tma_load_3d(st + C::S_U, &mU, q_full(s), 0, i * kTile, bh % args.bias_heads);
        tma_load_3d(st + C::S_AUG, &mAug, q_full(s), 0, i * kTile, bh);
      }
      wait_drain(kv_full, 0);
      for (int j = (i > NS ? i - NS : 0); j < i; ++j)
        wait_drain(q_full(j % NS), (j / NS) & 1);
    }
  } else if (warp == 9) {
    // ------------------------------------------------ MMA issue (whole warp)
    constexpr uint32_t idS = idesc_bf16_f32(128, 64, false, false);
    // Operand descriptors are built once (resident operands) or once per tile
    // (stage operands) and stepped through the K-steps with constant adds.
    const uint64_t dK = desc_kmajor(sb + C::OFF_K, D * 2);
    const uint64_t dV = desc_kmajor(sb + C::OFF_V, D * 2);
    const uint64_t dW = desc_kmajor(sb + C::OFF_W, C::UW * 2);
    const uint64_t dOnesL = desc_kmajor(sb + C::OFF_ONES, 32);
    const uint64_t dOnesD = desc_kmajor(sb + C::OFF_ONES + C::ONEB, 32);
    // [K | W] as the MN-major B operand of dQ | dU (W beside K for d = 64).
    const uint64_t dKWmn = C::MERGE_KW ? desc_mnmajor(sb + C::OFF_K, 128, C::OFF_W - C::OFF_K)
                                       : desc_mnmajor(sb + C::OFF_K, D * 2, 128 * D * 2);
    const uint64_t dWmn = desc_mnmajor(sb + C::OFF_W, RP > 0 ? RP * 2 : 32, 128 * (RP > 0 ? RP : 16) * 2);
    // Query half h of tile i:  S^T / s = K Q_h^T + W U'_h^T  and  dP^T = V dO_h^T
    // into TMEM columns 64h .. 64h + 63 of the S^T / dP^T accumulators.
    auto issue_sdp = [&](int i, int h) -> bool {
      const int s = i % NS;
      const uint32_t st = sb + C::OFF_STAGE + s * C::STAGE;
      if (!wait_warp(q_full(s), (i / NS) & 1, g, 33)) return false;
      if (!C::DEFER && i > 0 && !wait_warp(dq_free, (i - 1) & 1, g, 34)) return false;
      tc_fence_after();
      const uint32_t tS = tmem + C::T_S + h * 64, tP = tmem + C::T_DP + h * 64;
      const uint64_t dQ = desc_kmajor(st + C::S_Q + h * 64 * (D * 2), D * 2);
      const uint64_t dO = desc_kmajor(st + C::S_DO + h * 64 * (D * 2), D * 2);
      const uint64_t dU = desc_kmajor(st + C::S_U + h * 64 * (C::UW * 2), C::UW * 2);
      // dP^T first: the softmax has read the previous dP^T of this half (its
      // dS^T goes to shared memory only), so these columns are free.
      // The query rows' aug rows: + (-D) through the second ones tile.
      const uint64_t aug = desc_kmajor(st + C::S_AUG + h * 64 * 32, 32);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        umma_bf16(tP, desc_add(dV, kk * 32), desc_add(dO, kk * 32), idS, kk > 0 ? 1u : 0u);
      umma_bf16(tP, dOnesD, aug, idS, 1u);
      // P^T of the previous tile lives in the S^T columns: the dV MMAs reading
      // it must be done before S^T is overwritten (dK / dW and the dP^T above
      // are still queued behind them, so the tensor pipe does not run dry).
      if (i > 0 && !wait_warp(a_done(h), (i - 1) & 1, g, 41)) return false;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        umma_bf16(tS, desc_add(dK, kk * 32), desc_add(dQ, kk * 32), idS, kk > 0 ? 1u : 0u);
#pragma unroll
      for (int kk = 0; kk < RP / 16; ++kk)
        umma_bf16(tS, desc_add(dW, kk * 32), desc_add(dU, kk * 32), idS, 1u);
      umma_bf16(tS, dOnesL, aug, idS, 1u);  // + (-LSE / s)
      umma_commit(sdp_full(h));
      return true;
    };
    // dV += P^T dO over the 64 queries of half h with A = P^T read from TMEM
    // (packed bf16 over the S^T columns 64h .. 64h + 31), then a_done(h); then
    // dK += dS^T Q, dW += dS^T U' with A = dS^T from its swizzled shared-memory
    // block h (K-major: 128 key rows of 64 queries).
    auto issue_grad_kv = [&](int i, int h) {
      const uint32_t st = sb + C::OFF_STAGE + (i % NS) * C::STAGE;
      constexpr uint32_t idD = idesc_bf16_f32(128, D, false, true);
      constexpr uint32_t idR = idesc_bf16_f32(128, RP > 0 ? RP : 16, false, true);
      const uint64_t dOmn = desc_mnmajor(st + C::S_DO, D * 2, 128 * D * 2);
#pragma unroll
      for (int kk = 4 * h; kk < 4 * h + 4; ++kk) {
        const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
        umma_bf16_ts(tmem + C::T_DV, tmem + C::T_S + h * 64 + (kk & 3) * 8,
                     desc_add(dOmn, kk * 16 * (D * 2)), idD, acc);
      }
      umma_commit(a_done(h));
      const uint64_t dsa = desc_kmajor(ds_buf(i) + h * (kTile * 128), 128);
      // [Q | U'] as the MN-major B operand (U' beside Q for d = 64)
      const uint64_t dQUmn = C::MERGE_KW ? desc_mnmajor(st + C::S_Q, 128, C::S_U - C::S_Q)
                                         : desc_mnmajor(st + C::S_Q, D * 2, 128 * D * 2);
      const uint64_t dUmn = desc_mnmajor(st + C::S_U, RP > 0 ? RP * 2 : 32, 128 * (RP > 0 ? RP : 16) * 2);
#pragma unroll
      for (int kk = 4 * h; kk < 4 * h + 4; ++kk) {
        const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
        const uint64_t ad = desc_add(dsa, (kk & 3) * 32);
        if constexpr (C::MERGE_KW) {
          // [dK | dW] += dS^T [Q | U']: one B operand, atoms Q (64 cols) and U'
          // (C::S_U - C::S_Q bytes further), N = D + RP.
          constexpr uint32_t idKW = idesc_bf16_f32(128, D + RP, false, true);
          umma_bf16(tmem + C::T_DK, ad, desc_add(dQUmn, kk * 16 * 128), idKW, acc);
        } else {
          umma_bf16(tmem + C::T_DK, ad, desc_add(dQUmn, kk * 16 * (D * 2)), idD, acc);
          if constexpr (RP > 0)
            umma_bf16(tmem + C::T_DW, ad, desc_add(dUmn, kk * 16 * (RP * 2)), idR, acc);
        }
      }
    };
    // dQ = dS K and dU = dS W (A = the dS^T tile read transposed): one chain
    // over [K | W] (N = D + RP) when W is staged beside K, else interleaved.
    auto issue_grad_q = [&](int i) {
      const uint64_t dsm = desc_mnmajor(ds_buf(i), 128, 128 * 128);
      constexpr uint32_t idD = idesc_bf16_f32(128, D, true, true);
      constexpr uint32_t idR = idesc_bf16_f32(128, RP > 0 ? RP : 16, true, true);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t ad = desc_add(dsm, kk * 16 * 128);
        if constexpr (C::MERGE_KW) {
          constexpr uint32_t idQU = idesc_bf16_f32(128, D + RP, true, true);
          umma_bf16(tmem + C::T_DQ, ad, desc_add(dKWmn, kk * 16 * 128), idQU, kk > 0 ? 1u : 0u);
        } else {
          umma_bf16(tmem + C::T_DQ, ad, desc_add(dKWmn, kk * 16 * (D * 2)), idD, kk > 0 ? 1u : 0u);
          if constexpr (RP > 0)
            umma_bf16(tmem + C::T_DQ + D, ad, desc_add(dWmn, kk * 16 * (RP * 2)), idR,
                      kk > 0 ? 1u : 0u);
        }
      }
      umma_commit(dq_full);
    };
    bool ok = wait_warp(kv_full, 0, g, 32);
    if (ok && nq > 0) ok = issue_sdp(0, 0) && issue_sdp(0, 1);
    for (int i = 0; ok && i < nq; ++i) {
      if constexpr (C::DEFER) {
        // Half by half: its dV / dK / dW MMAs, then its scores of the next tile,
        // so that one warpgroup's softmax overlaps the other half's MMAs; this
        // tile's dQ | dU last (their reduction happens after the next softmax).
        for (int h = 0; ok && h < 2; ++h) {
          if (!wait_warp(ds_full(h), i & 1, g, 35)) { ok = false; break; }
          tc_fence_after();
          issue_grad_kv(i, h);
          if (h == 1) umma_commit(q_empty(i % NS));  // Q, dO, U' of this tile are read
          if (i + 1 < nq && !issue_sdp(i + 1, h)) ok = false;
        }
        if (!ok) break;
        if (i > 0 && !wait_warp(dq_free, (i - 1) & 1, g, 36)) break;
        tc_fence_after();
        issue_grad_q(i);
      } else {
        if (!wait_warp(ds_full(0), i & 1, g, 35) || !wait_warp(ds_full(1), i & 1, g, 35)) break;
        tc_fence_after();
        issue_grad_kv(i, 0);
        issue_grad_kv(i, 1);
        umma_commit(q_empty(i % NS));
        // dQ | dU overwrite the S^T columns that dV / dK / dW read P^T from.
        if (!wait_warp(a_done(1), i & 1, g, 42)) break;
        tc_fence_after();
        issue_grad_q(i);
        if (i + 1 < nq && !(issue_sdp(i + 1, 0) && issue_sdp(i + 1, 1))) break;
      }
    }
    umma_commit(drain_bar);
    wait_drain(drain_bar, 0);
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------- softmax warps (two warpgroups)
    const int wg = warp >> 2;                  // 0: queries 0-63, 1: queries 64-127
    const int row = threadIdx.x & 127;         // TMEM lane == key row (S^T) == query row (dQ)
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const bool key_ok = (k0 + row) < N;
    const uint64_t sl2x2 = f2_pack(args.scale_log2, args.scale_log2);
    // Shifted-window mask: in the last window row (column) of a shifted map the
    // top and bottom (left and right) 4-token halves are different regions, so
    // key k and query q interact only if ((k ^ q) & mask_bits) == 0 (bit 5 of
    // the raster index selects the half of rows, bit 2 the half of columns).
    int mask_bits = 0;
    if (args.mask_shift > 0) {
      const int bw = bh / args.mask_heads;
      const int wx = bw % args.mask_nwx, wy = (bw / args.mask_nwx) % args.mask_nwy;
      mask_bits = (wy == args.mask_nwy - 1 ? 32 : 0) | (wx == args.mask_nwx - 1 ? 4 : 0);
    }
    // P^T = 2^((S^T / s - LSE / s) s log2e), dS^T = P^T o (dP^T - D) for
    // this warpgroup's 64 query columns of tile i (the MMAs have subtracted
    // LSE / s and D already); P^T goes back into TMEM in place (packed bf16,
    // columns wg*64 + [0, 32)), dS^T into shared memory.
    auto softmax = [&](int i) -> bool {
      if (!wait_warp(sdp_full(wg), i & 1, g, 38)) return false;
      tc_fence_after();
      const int qvalid = N - i * kTile;
      const uint32_t dsb = ds_buf(i);
#pragma unroll 1
      for (int c = wg * 64; c < wg * 64 + 64; c += 32) {
        uint32_t xy[64];
        tmem_ld32x2(tmem + lane_base + C::T_S + c, tmem + lane_base + C::T_DP + c, xy);
        // Padding keys / queries: a score of -inf gives P = 0 and dS = 0.
        if (!key_ok || c + 32 > qvalid) {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (!key_ok || c + e >= qvalid) xy[e] = 0xFF800000u;
        }
        if (mask_bits != 0) {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if ((((k0 + row) ^ (i * kTile + c + e)) & mask_bits) != 0) xy[e] = 0xFF800000u;
        }
        uint32_t pk[16], dk[16];
#pragma unroll
        // S^T / s already holds - LSE / s and dP^T already holds - D.
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const uint64_t x2 = static_cast<uint64_t>(xy[e + 1]) << 32 | xy[e];
          const uint64_t y2 = static_cast<uint64_t>(xy[32 + e + 1]) << 32 | xy[32 + e];
          const float2 arg = f2_unpack(f2_mul(x2, sl2x2));
          const float p0 = fast_exp2(arg.x), p1 = fast_exp2(arg.y);
          const float2 ds = f2_unpack(f2_mul(f2_pack(p0, p1), y2));
          pk[e >> 1] = pack_bf16x2(p0, p1);
          dk[e >> 1] = pack_bf16x2(ds.x, ds.y);
        }
        const int pcol = wg * 64 + (c - wg * 64) / 2;
        tmem_st16_nowait(tmem + lane_base + C::T_S + pcol, pk);
        // This dS buffer last staged the reductions of tile i - NDS: they must
        // have been read before dS^T overwrites them.
        if (c == wg * 64 && i >= C::NDS &&
            !wait_warp(ds_free(i % C::NDS, wg), ((i / C::NDS) + 1) & 1, g, 43))
          return false;
#pragma unroll
        for (int e = 0; e < 32; e += 8)
          st_shared_v4(dsb + sw128_offset(row, c + e, 128), dk[e / 2], dk[e / 2 + 1],
                       dk[e / 2 + 2], dk[e / 2 + 3]);
      }
      tmem_st_wait();
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ds_full(wg));
      return true;
    };
    bool ok = true;
    for (int i = 0; ok && i < nq; ++i) ok = softmax(i);
    // The MMA warp's final commit: every dV, dK, dW MMA has completed.
    if (ok && nq > 0) ok = wait_warp(drain_bar, 0, g, 44);
    if (ok && nq > 0) {
      tc_fence_after();
      const size_t r0 = static_cast<size_t>(bh) * N + k0 + row;
      if (wg == 0) {
        uint32_t gv[D];
        tmem_ld_cols<D>(tmem + lane_base + C::T_DV, gv);
        if (key_ok) store_o_row<D>(args.dv + r0 * D, gv, 1.0f);
        if constexpr (RP > 0) {
          uint32_t gw[RP];
          tmem_ld_cols<RP>(tmem + lane_base + C::T_DW, gw);
          if (key_ok && args.dw_part != nullptr) {
            // Shared factors: this window-head's fp32 dW rows, summed over the
            // windows afterwards.
            float4* dst = reinterpret_cast<float4*>(args.dw_part + r0 * args.r);
            const float f = args.scale;
#pragma unroll
            for (int c = 0; c < RP; c += 4)
              if (c < args.r)
                dst[c >> 2] = make_float4(__uint_as_float(gw[c]) * f, __uint_as_float(gw[c + 1]) * f,
                                          __uint_as_float(gw[c + 2]) * f,
                                          __uint_as_float(gw[c + 3]) * f);
          } else if (key_ok) {
            uint4* dst = reinterpret_cast<uint4*>(args.dw + r0 * args.r);
            const float f = args.scale;
#pragma unroll
            for (int c = 0; c < RP; c += 8) {
              if (c < args.r) {
                uint4 v;
                v.x = pack_bf16x2(__uint_as_float(gw[c]) * f, __uint_as_float(gw[c + 1]) * f);
                v.y = pack_bf16x2(__uint_as_float(gw[c + 2]) * f, __uint_as_float(gw[c + 3]) * f);
                v.z = pack_bf16x2(__uint_as_float(gw[c + 4]) * f, __uint_as_float(gw[c + 5]) * f);
                v.w = pack_bf16x2(__uint_as_float(gw[c + 6]) * f, __uint_as_float(gw[c + 7]) * f);
                dst[c >> 3] = v;
              }
            }
          }
        }
      } else {
        uint32_t gk[D];
        tmem_ld_cols<D>(tmem + lane_base + C::T_DK, gk);
        if (key_ok) store_o_row<D>(args.dk + r0 * D, gk, args.scale);
      }
    }
  } else {
    // --------------------------------- dQ | dU reduction warps (10 - 13)
    // Partial dQ | dU of tile j (TMEM lane = query row): each warp takes its 32
    // query rows of every 32-column chunk, scales the dQ columns by s, stages
    // the chunk 128-byte swizzled and adds it into the fp32 accumulator with a
    // TMA bulk tensor reduction (32 x 32 box) issued by its lane 0.  The
    // chunks are staged in the two 64-query blocks of the tile's dS buffer
    // (read by dQ's MMAs already, dq_full): with three chunks, chunk 0 in block
    // 0 and chunks 1, 2 in block 1 (block 0 is released after one copy);
    // otherwise chunk c in block c & 1.  Warpgroup k overwrites block k NDS
    // tiles later, once that block's copies have read it (ds_free).  Rows
    // entirely past N issue no copy.
    const int rw = warp & 3;                     // TMEM lane quarter
    const uint32_t lane_base = static_cast<uint32_t>(rw * 32) << 16;
    const int row = rw * 32 + lane;              // query row within the tile
    const int wq = rw * 32;
    for (int j = 0; j < nq; ++j) {
      if (!wait_warp(dq_full, j & 1, g, 39)) break;
      tc_fence_after();
#pragma unroll
      for (int ch = 0; ch < C::NCH; ++ch) {
        uint32_t z[32];
        tmem_ld32(tmem + lane_base + C::T_DQ + ch * 32, z);
        if (ch == C::NCH - 1) {
          // dQ | dU of this tile are in registers: the next dQ MMAs may start.
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(dq_free);
        }
        const int blk = C::NCH == 3 ? (ch > 0 ? 1 : 0) : (ch & 1);
        const uint32_t buf = ds_buf(j) + blk * (kTile * 128);
        if (ch >= 2) {
          // The block's previous copy must have read it: with three chunks
          // that is chunk 1's, the last committed (and then block 0 is free
          // too), with four chunk ch - 2's, the one before the last.
          if (lane == 0) {
            if (C::NCH == 3) bulk_wait_read<0>();
            else bulk_wait_read<1>();
          }
          __syncwarp();
          if (C::NCH == 3 && lane == 0) mbar_arrive(ds_free(j % C::NDS, 0));
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float v4[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int col = ch * 32 + q * 4 + t;
            v4[t] = __uint_as_float(z[q * 4 + t]) * (col < D ? args.scale : 1.0f);
          }
          st_shared_v4(buf + row * 128 + ((q ^ (row & 7)) << 4), __float_as_uint(v4[0]),
                       __float_as_uint(v4[1]), __float_as_uint(v4[2]), __float_as_uint(v4[3]));
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (j * kTile + wq < N)
            tma_reduce_add_3d(&mAcc, buf + wq * 128, ch * 32, j * kTile + wq, bh);
          bulk_commit();
        }
      }
      // Release each block once the copies out of it have read it.
      const int b = j % C::NDS;
      if constexpr (C::NCH == 3) {
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_free(b, 1));
      } else if constexpr (C::NCH == 1) {
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(ds_free(b, 0));
          mbar_arrive(ds_free(b, 1));
        }
      } else {
        // the last two copies came from blocks 0 and 1, in that order
        if (lane == 0) bulk_wait_read<1>();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_free(b, 0));
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_free(b, 1));
      }
    }
    if (lane == 0) bulk_wait_all();  // reductions complete before the CTA exits
  }

  // This CTA's work is done: the next grid may start launching (a long
  // kernel gains nothing from letting it in earlier).
  grid_dep_launch_next();
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace rfb
