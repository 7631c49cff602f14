// bwd_window.cuh -- backward of O = softmax(s Q K^T + U W^T) V for windows of
// at most 128 tokens (head size 32, bias rank up to 16), the shape of
// SwinIR-style window attention.
//
// The same chain rule as bwd_kernels.cuh (dS = P o (dP - D), dQ = s dS K,
// dK = s dS^T Q, dV = P^T dO, dU = dS W, dW = dS^T U), but a whole window fits
// in one 128-row tile, so every gradient is complete after one pass over the
// tile: no fp32 accumulator in global memory, no row-statistics pre-pass and no
// cast pass.  Windows of <= 64 tokens are packed two per tile (rows 0-63 and
// 64-127) with a block-diagonal P, as in the window forward.
//
// One persistent CTA per SM walks through tiles:
//   warp 4      TMA producer: Q, K, V, dO, O and the factors U, W of a tile
//               (U, W staged 32 columns wide, zero padded, so that [Q | U'] and
//               [K | W] are single MMA operands), a ring of input stages; the
//               tile's copies are spread over the warp's lanes;
//   warp 5      MMA issue: S^T/s = K Q^T + W U'^T and dP^T = V dO^T into TMEM,
//               then dV = P^T dO, [dK | dW] = dS^T [Q | U'] (A operands read
//               from TMEM) and [dQ | dU] = dS [K | W] (A = the dS^T tile in
//               shared memory, read transposed);
//   warp 6      U' = U / s in each stage;
//   warps 0-3   per tile: -LSE log2(e) and -D = -rowsum(dO o O) of the
//               tile's query rows into shared memory; P^T and dS^T (thread =
//               key row = TMEM lane) written back into TMEM in place and dS^T
//               into shared memory; then the gradients out of TMEM, dQ, dK, dV
//               staged in the (now free) rows of the dS tile and written by TMA
//               stores, one per warp; dU, dW rows stored directly (per-window
//               factors) or as fp32 rows per window-head that a second kernel
//               sums over the windows (factors shared by all windows).
// With IMG the tensors are channels-last feature maps and the tiles are the
// windows of the map rolled by -shift, gathered and scattered by the TMA
// addressing (4 x 4-token quadrant boxes, tokens in quadrant-major order
// inside a window), with the shifted-window mask.
#pragma once
#include "bwd_kernels.cuh"

namespace rfb {

struct BwdWinArgs {
  const float* lse;   // [BH, N] (IMG: [B, img_h, img_w, heads])
  __nv_bfloat16* du;  // per-window factors: [BH, N, r] bf16
  __nv_bfloat16* dw;
  float* du_part;     // shared factors: [BH, N, r] fp32 rows of each window-head
  float* dw_part;     // (NULL with per-window factors)
  int* err;
  int BH, N, r;
  int bias_heads;     // BH (per window-head) or H (shared: bias head = bh % H)
  int shared;         // 1: factors shared by all windows ([H, N, r], one copy per window)
  int img_h, img_w, img_heads, shift;  // IMG only
  float scale, scale_log2, inv_scale;
  uint64_t timeout_ns;
  int fail_site;
};

template <int RP, int NP, bool IMG>
struct BwdWinCfg {
  static_assert(RP == 0 || RP == 16, "bias rank up to 16");
  static_assert(!IMG || NP == 64, "image windows are 8 x 8");
  static constexpr int D = 32;
  static constexpr int NW = kTile / NP;   // windows per tile
  static constexpr int TB = kTile * D * 2;  // one [128, 32] bf16 tile, 64-byte rows
  static constexpr int S_Q = 0, S_K = TB, S_V = 2 * TB, S_DO = 3 * TB, S_O = 4 * TB;
  static constexpr int S_U = 5 * TB, S_W = 6 * TB;
  static constexpr int STAGE = (RP > 0 ? 7 : 5) * TB;
  static constexpr int DSB = kTile * kTile * 2;  // the dS^T tile: two 64-query blocks
  static constexpr int VEC = 2 * 2 * kTile * 4;  // (-LSE log2 e, -D) x 2 tile parities
  static constexpr int NS_FIT = (232448 - 1024 - DSB - VEC - 256) / STAGE;
  static constexpr int NS = NS_FIT > 4 ? 4 : NS_FIT;
  static constexpr int OFF_DS = NS * STAGE;
  static constexpr int OFF_VEC = OFF_DS + DSB;
  static constexpr int OFF_BAR = OFF_VEC + VEC;
  // in_full[NS] u_ready[NS] in_empty[NS] sdp_full ds_full grad_full grad_free
  // vec_full[2] drain
  static constexpr int NBAR = 3 * NS + 7;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
  // TMEM columns: S^T, dP^T (P^T / dS^T packed in place), dV, [dK | dW], [dQ | dU].
  static constexpr int T_S = 0, T_DP = 128, T_DV = 256, T_DK = 256 + D, T_DQ = 256 + 2 * D + RP;
  static_assert(T_DQ + D + RP <= 512, "TMEM budget");
  static_assert(NS >= 2, "shared memory budget");
  static_assert(SMEM <= 232448, "shared memory budget exceeded");
};

constexpr int kBwdWinThreads = 224;  // warps 0-3 compute, 4 TMA, 5 MMA, 6 U' scaling

template <int NC>
__device__ __forceinline__ void tmem_ld_any(uint32_t taddr, uint32_t (&r)[NC]) {
  static_assert(NC == 16 || NC == 32 || NC == 48, "column count");
  if constexpr (NC == 48) {
    tmem_ld32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
    tmem_ld16(taddr + 32, *reinterpret_cast<uint32_t(*)[16]>(&r[32]));
  } else if constexpr (NC == 32) {
    tmem_ld32(taddr, r);
  } else {
    tmem_ld16(taddr, r);
  }
}

// One row of 32 bf16 values (from fp32 bits times f) into a 64-byte-row tile
// with 64-byte swizzle (the tile starts on a 1024-byte boundary).
__device__ __forceinline__ void stage_row32(uint32_t tile, int row, const uint32_t* v, float f) {
#pragma unroll
  for (int c = 0; c < 4; ++c)
    st_shared_v4(tile + swz_offset(row, c, 64),
                 pack_bf16x2(__uint_as_float(v[8 * c + 0]) * f, __uint_as_float(v[8 * c + 1]) * f),
                 pack_bf16x2(__uint_as_float(v[8 * c + 2]) * f, __uint_as_float(v[8 * c + 3]) * f),
                 pack_bf16x2(__uint_as_float(v[8 * c + 4]) * f, __uint_as_float(v[8 * c + 5]) * f),
                 pack_bf16x2(__uint_as_float(v[8 * c + 6]) * f, __uint_as_float(v[8 * c + 7]) * f));
}

template <int RP, int NP, bool IMG>
__global__ void __launch_bounds__(kBwdWinThreads, 1)
    bwd_window_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                      const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mDO,
                      const __grid_constant__ CUtensorMap mO, const __grid_constant__ CUtensorMap mU,
                      const __grid_constant__ CUtensorMap mW, const __grid_constant__ CUtensorMap mDQ,
                      const __grid_constant__ CUtensorMap mDK, const __grid_constant__ CUtensorMap mDV,
                      const BwdWinArgs args) {
  using C = BwdWinCfg<RP, NP, IMG>;
  constexpr int D = C::D, NS = C::NS, NW = C::NW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_1024(smem_raw);
  const uint32_t sb = smem_u32(smem);
  const uint32_t bar0 = sb + C::OFF_BAR;
  auto in_full = [&](int s) { return bar0 + 8u * s; };
  auto u_ready = [&](int s) { return bar0 + 8u * (NS + s); };
  auto in_empty = [&](int s) { return bar0 + 8u * (2 * NS + s); };
  const uint32_t sdp_full = bar0 + 8u * (3 * NS);
  const uint32_t ds_full = bar0 + 8u * (3 * NS + 1);
  const uint32_t grad_full = bar0 + 8u * (3 * NS + 2);
  const uint32_t grad_free = bar0 + 8u * (3 * NS + 3);
  auto vec_full = [&](int p) { return bar0 + 8u * (3 * NS + 4 + p); };
  const uint32_t drain_bar = bar0 + 8u * (3 * NS + 6);
  const uint32_t dsb = sb + C::OFF_DS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + C::NBAR * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = static_cast<int>(warp_id());
  const int lane = static_cast<int>(lane_id());
  const int N = args.N;
  const int num_tiles = (args.BH + NW - 1) / NW;
  // Image windows: window-head bh = ((b * nwy + wy) * nwx + wx) * heads + h.
  const int nwx = IMG ? args.img_w / 8 : 1, nwy = IMG ? args.img_h / 8 : 1;
  auto window_of = [&](int bh, int& b, int& wy, int& wx, int& h) {
    h = bh % args.img_heads;
    const int bw = bh / args.img_heads;
    wx = bw % nwx;
    wy = (bw / nwx) % nwy;
    b = bw / (nwx * nwy);
  };
  // v mod size for 0 <= v < 2 size (a window's rows and columns, shifted).
  auto wrap = [](int v, int size) { return v >= size ? v - size : v; };

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < NS; ++s) {
      mbar_init(in_full(s), 1);
      mbar_init(u_ready(s), 1);
      mbar_init(in_empty(s), 1);
    }
    mbar_init(sdp_full, 1);
    mbar_init(ds_full, 4);      // one arrival per compute warp
    mbar_init(grad_full, 1);
    mbar_init(grad_free, 4);    // one arrival per compute warp
    mbar_init(vec_full(0), 4);
    mbar_init(vec_full(1), 4);
    mbar_init(drain_bar, 1);
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch(&mQ);
    tma_prefetch(&mK);
    tma_prefetch(&mV);
    tma_prefetch(&mDO);
    tma_prefetch(&mO);
    tma_prefetch(&mDQ);
    tma_prefetch(&mDK);
    tma_prefetch(&mDV);
    if constexpr (RP > 0) {
      tma_prefetch(&mU);
      tma_prefetch(&mW);
    }
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitGuard g{abort_flag, args.err, args.timeout_ns, args.fail_site};
  grid_dep_wait();
  grid_dep_launch_next();

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    // The whole warp runs the loop: lane 0 waits for the stage and posts the
    // expected bytes, then the lanes share the tile's copies (with image
    // windows a tile takes 4 quadrant copies per tensor and window).
    int it = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++it) {
      const int s = it % NS;
      if (it >= NS && !wait_warp(in_empty(s), ((it / NS) + 1) & 1, g, 51)) break;
      const uint32_t st = sb + s * C::STAGE;
      if (lane == 0) mbar_expect_tx(in_full(s), C::STAGE);
      __syncwarp();
      const int w0 = t * NW;
      if constexpr (IMG) {
        // Four 4 x 4 quadrants per window of the rolled map; a missing last
        // window repeats the previous one (nothing of it is stored).  Copy
        // j = (window i, quadrant qd, tensor c) goes to lane j % 32.
        constexpr int NT = RP > 0 ? 7 : 5;
        for (int j = lane; j < NW * 4 * NT; j += 32) {
          const int i = j / (4 * NT), qd = (j / NT) % 4, c = j % NT;
          int b, wy, wx, h;
          window_of(min(w0 + i, args.BH - 1), b, wy, wx, h);
          const uint32_t off = i * (NP * D * 2) + qd * (16 * D * 2);
          if (c >= 5) {
            tma_load_4d(st + (c == 5 ? C::S_U : C::S_W) + off, c == 5 ? &mU : &mW, in_full(s), 0,
                        4 * (qd & 1), 4 * (qd >> 1), h);
          } else {
            const int y = wrap(wy * 8 + 4 * (qd >> 1) + args.shift, args.img_h);
            const int x = wrap(wx * 8 + 4 * (qd & 1) + args.shift, args.img_w);
            const CUtensorMap* mp = c == 0 ? &mQ : c == 1 ? &mK : c == 2 ? &mV : c == 3 ? &mDO : &mO;
            const uint32_t so = c == 0 ? C::S_Q : c == 1 ? C::S_K : c == 2 ? C::S_V : c == 3 ? C::S_DO : C::S_O;
            tma_load_5d(st + so + off, mp, in_full(s), 0, h, x, y, b);
          }
        }
      } else if (lane == 0) {
        tma_load_3d(st + C::S_Q, &mQ, in_full(s), 0, 0, w0);
        tma_load_3d(st + C::S_K, &mK, in_full(s), 0, 0, w0);
        tma_load_3d(st + C::S_V, &mV, in_full(s), 0, 0, w0);
        tma_load_3d(st + C::S_DO, &mDO, in_full(s), 0, 0, w0);
        tma_load_3d(st + C::S_O, &mO, in_full(s), 0, 0, w0);
        if constexpr (RP > 0) {
          if (!args.shared) {
            tma_load_3d(st + C::S_U, &mU, in_full(s), 0, 0, w0);
            tma_load_3d(st + C::S_W, &mW, in_full(s), 0, 0, w0);
          } else {
            // Shared factors: one copy per window (its bias head).
#pragma unroll
            for (int i = 0; i < NW; ++i) {
              const int z = (w0 + i) % args.bias_heads;
              tma_load_3d(st + C::S_U + i * (NP * D * 2), &mU, in_full(s), 0, 0, z);
              tma_load_3d(st + C::S_W + i * (NP * D * 2), &mW, in_full(s), 0, 0, z);
            }
          }
        }
      }
    }
    if (lane == 0)
      for (int j = (it > NS ? it - NS : 0); j < it; ++j) wait_drain(in_full(j % NS), (j / NS) & 1);
  } else if (warp == 5) {
    // --------------------------------------------------------- MMA issue
    constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);
    constexpr uint32_t idV = idesc_bf16_f32(128, D, false, true);
    constexpr uint32_t idKW = idesc_bf16_f32(128, D + RP, false, true);
    constexpr uint32_t idQU = idesc_bf16_f32(128, D + RP, true, true);
    int it = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++it) {
      const int s = it % NS;
      const uint32_t st = sb + s * C::STAGE;
      if (!wait_warp(RP > 0 ? u_ready(s) : in_full(s), (it / NS) & 1, g, 52)) break;
      // The previous tile's gradient MMAs read P^T / dS^T from the S^T / dP^T
      // columns that these MMAs overwrite.
      if (it > 0 && !wait_warp(grad_full, (it - 1) & 1, g, 53)) break;
      tc_fence_after();
      // Each operand's descriptor once, stepped through the K-steps by adds.
      const uint64_t dK = desc_kmajor(st + C::S_K, 64), dQ = desc_kmajor(st + C::S_Q, 64);
      const uint64_t dV = desc_kmajor(st + C::S_V, 64), dO = desc_kmajor(st + C::S_DO, 64);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        umma_bf16(tmem + C::T_S, desc_add(dK, kk * 32), desc_add(dQ, kk * 32), idS,
                  kk > 0 ? 1u : 0u);
        umma_bf16(tmem + C::T_DP, desc_add(dV, kk * 32), desc_add(dO, kk * 32), idS,
                  kk > 0 ? 1u : 0u);
      }
      if constexpr (RP > 0) {
        const uint64_t dW = desc_kmajor(st + C::S_W, 64), dU = desc_kmajor(st + C::S_U, 64);
#pragma unroll
        for (int kk = 0; kk < RP / 16; ++kk)
          umma_bf16(tmem + C::T_S, desc_add(dW, kk * 32), desc_add(dU, kk * 32), idS, 1u);
      }
      umma_commit(sdp_full);
      if (!wait_warp(ds_full, it & 1, g, 54)) break;
      // The previous tile's gradients have been read out of TMEM.
      if (it > 0 && !wait_warp(grad_free, (it - 1) & 1, g, 55)) break;
      tc_fence_after();
      const uint64_t dOmn = desc_mnmajor(st + C::S_DO, 64, C::TB);
      const uint64_t dQUmn = desc_mnmajor(st + C::S_Q, 64, C::S_U - C::S_Q);
      const uint64_t dSmn = desc_mnmajor(dsb, 128, 128 * 128);
      const uint64_t dKWmn = desc_mnmajor(st + C::S_K, 64, C::S_W - C::S_K);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t acc = kk > 0 ? 1u : 0u;
        // dV = P^T dO
        umma_bf16_ts(tmem + C::T_DV, tmem + C::T_S + kk * 8, desc_add(dOmn, kk * 16 * 64), idV, acc);
        // [dK | dW] = dS^T [Q | U']
        umma_bf16_ts(tmem + C::T_DK, tmem + C::T_DP + kk * 8, desc_add(dQUmn, kk * 16 * 64), idKW,
                     acc);
        // [dQ | dU] = dS [K | W]
        umma_bf16(tmem + C::T_DQ, desc_add(dSmn, kk * 16 * 128), desc_add(dKWmn, kk * 16 * 64), idQU,
                  acc);
      }
      umma_commit(grad_full);
      umma_commit(in_empty(s));
    }
    umma_commit(drain_bar);
    wait_drain(drain_bar, 0);
    __syncwarp();
  } else if (warp == 6) {
    // ------------------------------------------------- U' = U / s in place
    if constexpr (RP > 0) {
      int it = 0;
      for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++it) {
        const int s = it % NS;
        if (!wait_warp(in_full(s), (it / NS) & 1, g, 50)) break;
        scale_tile_bf16(sb + s * C::STAGE + C::S_U, C::TB, args.inv_scale);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(u_ready(s));
      }
    }
  } else {
    // ------------------------------------------------------ compute warps
    const int row = threadIdx.x;  // TMEM lane = tile row (key row of S^T, query row of dQ)
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const int wl = row / NP;       // window within the tile
    const int n = row % NP;        // token within the window
    const int c0 = wl * NP;        // first column of the window's block
    const float sl2 = args.scale_log2;
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    // this warp's rows of the dS tile double as its output staging: dQ, dK in
    // block 0, dV in block 1 (32 rows x 64 bytes each)
    const uint32_t stg_q = dsb + warp * 4096, stg_k = stg_q + 2048, stg_v = dsb + 16384 + warp * 4096;
    // lanes issuing this warp's output stores (each waits for its own copies)
    constexpr int kStoreLanes = IMG ? 6 : 3;
    // LSE of this thread's query row of tile tt (0 for padding rows); loaded
    // one tile ahead so that its global-memory latency overlaps a whole tile.
    // With image windows it also decodes the row's window into nb, nwy_,
    // nwx_, nh, which the next tile then uses (rows of a missing window keep
    // stale values: they are masked and not stored).
    int nb = 0, nwy_ = 0, nwx_ = 0, nh = 0;
    auto load_lse = [&](int tt) -> float {
      const int wn = tt * NW + wl;
      if (tt >= num_tiles || wn >= args.BH || n >= N) return 0.f;
      size_t r = static_cast<size_t>(wn) * N + n;
      if constexpr (IMG) {
        window_of(wn, nb, nwy_, nwx_, nh);
        const int qq = n >> 4;
        const int y = wrap(nwy_ * 8 + 4 * (qq >> 1) + ((n >> 2) & 3) + args.shift, args.img_h);
        const int x = wrap(nwx_ * 8 + 4 * (qq & 1) + (n & 3) + args.shift, args.img_w);
        r = ((static_cast<size_t>(nb) * args.img_h + y) * args.img_w + x) * args.img_heads + nh;
      }
      return args.lse[r];
    };
    float lse_next = load_lse(blockIdx.x);
    int it = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++it) {
      const int s = it % NS;
      const uint32_t st = sb + s * C::STAGE;
      const int win = t * NW + wl;
      const bool valid = win < args.BH && n < N;
      // this row's window, decoded by load_lse(t)
      const int b = nb, wy = nwy_, wx = nwx_, h = nh;
      const float lse_cur = lse_next;
      lse_next = load_lse(t + gridDim.x);
      // ---- -LSE log2(e) and -D of this query row
      if (!wait_warp(in_full(s), (it / NS) & 1, g, 56)) break;
      float nl2 = 0.f, nd = 0.f;
      if (valid) {
        nl2 = -lse_cur * kLog2e;
        float acc = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 ov = ld_shared_v4(st + C::S_O + swz_offset(row, c, 64));
          const uint4 gv = ld_shared_v4(st + C::S_DO + swz_offset(row, c, 64));
          const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w};
          const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc = fmaf(__uint_as_float(ow[e] << 16), __uint_as_float(gw[e] << 16), acc);
            acc = fmaf(__uint_as_float(ow[e] & 0xFFFF0000u), __uint_as_float(gw[e] & 0xFFFF0000u), acc);
          }
        }
        nd = -acc;
      }
      const uint32_t vec = sb + C::OFF_VEC + (it & 1) * (2 * kTile * 4);
      asm volatile("st.shared.f32 [%0], %1;" ::"r"(vec + row * 4), "f"(nl2) : "memory");
      asm volatile("st.shared.f32 [%0], %1;" ::"r"(vec + kTile * 4 + row * 4), "f"(nd) : "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(vec_full(it & 1));
      // ---- P^T, dS^T of this key row against its window's queries
      if (!wait_warp(sdp_full, it & 1, g, 57)) break;
      if (!wait_warp(vec_full(it & 1), (it >> 1) & 1, g, 58)) break;
      if (it > 0) {
        // this warp's TMA stores of the previous tile read the rows written next
        if (lane < kStoreLanes) bulk_wait_read<0>();
        __syncwarp();
      }
      tc_fence_after();
      int mask_bits = 0;
      if constexpr (IMG) {
        // shifted-window mask (quadrant-major tokens: bit 5 = quadrant row,
        // bit 4 = quadrant column): in the last window row / column of the
        // rolled map the two halves are different regions
        if (args.shift > 0)
          mask_bits = (wy == nwy - 1 ? 32 : 0) | (wx == nwx - 1 ? 16 : 0);
      }
#pragma unroll 1
      for (int cc = 0; cc < NP; cc += 32) {
        uint32_t xy[64];
        tmem_ld32x2(tmem + lane_base + C::T_S + c0 + cc, tmem + lane_base + C::T_DP + c0 + cc, xy);
        // Padding keys / queries and masked pairs: a score of -inf gives P = 0, dS = 0.
        if (!valid || N < cc + 32 || mask_bits != 0) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int q = cc + e;
            if (!valid || q >= N || ((n ^ q) & mask_bits) != 0) xy[e] = 0xFF800000u;
          }
        }
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const uint4 nl = ld_shared_v4(vec + (c0 + cc + e) * 4);
          const uint4 nv = ld_shared_v4(vec + kTile * 4 + (c0 + cc + e) * 4);
#pragma unroll
          for (int u = 0; u < 4; u += 2) {
            const uint64_t nl2x = (u == 0) ? (static_cast<uint64_t>(nl.y) << 32 | nl.x)
                                           : (static_cast<uint64_t>(nl.w) << 32 | nl.z);
            const uint64_t ndx = (u == 0) ? (static_cast<uint64_t>(nv.y) << 32 | nv.x)
                                          : (static_cast<uint64_t>(nv.w) << 32 | nv.z);
            const uint64_t x2 = static_cast<uint64_t>(xy[e + u + 1]) << 32 | xy[e + u];
            const uint64_t y2 = static_cast<uint64_t>(xy[32 + e + u + 1]) << 32 | xy[32 + e + u];
            const float2 arg = f2_unpack(f2_fma(x2, sl2x2, nl2x));
            const float p0 = fast_exp2(arg.x), p1 = fast_exp2(arg.y);
            const float2 ds = f2_unpack(f2_mul(f2_pack(p0, p1), f2_add(y2, ndx)));
            pk[(e + u) >> 1] = pack_bf16x2(p0, p1);
            dk[(e + u) >> 1] = pack_bf16x2(ds.x, ds.y);
          }
        }
        tmem_st16_nowait(tmem + lane_base + C::T_S + (c0 + cc) / 2, pk);
        tmem_st16_nowait(tmem + lane_base + C::T_DP + (c0 + cc) / 2, dk);
#pragma unroll
        for (int e = 0; e < 32; e += 8)
          st_shared_v4(dsb + sw128_offset(row, c0 + cc + e, 128), dk[e / 2], dk[e / 2 + 1],
                       dk[e / 2 + 2], dk[e / 2 + 3]);
      }
      if constexpr (NW == 2) {
        // The other window's block stays zero (block-diagonal P^T and dS^T).
        const int co = (1 - wl) * NP;
        uint32_t zero[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) zero[e] = 0u;
#pragma unroll
        for (int cc = 0; cc < NP; cc += 32) {
          tmem_st16_nowait(tmem + lane_base + C::T_S + (co + cc) / 2, zero);
          tmem_st16_nowait(tmem + lane_base + C::T_DP + (co + cc) / 2, zero);
        }
#pragma unroll
        for (int e = 0; e < NP; e += 8)
          st_shared_v4(dsb + sw128_offset(row, co + e, 128), 0u, 0u, 0u, 0u);
      }
      tmem_st_wait();
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ds_full);
      // ---- gradients of this tile
      if (!wait_warp(grad_full, it & 1, g, 59)) break;
      tc_fence_after();
      uint32_t gv[D], gk[D + RP], gq[D + RP];
      tmem_ld_any<D>(tmem + lane_base + C::T_DV, gv);
      tmem_ld_any<D + RP>(tmem + lane_base + C::T_DK, gk);
      tmem_ld_any<D + RP>(tmem + lane_base + C::T_DQ, gq);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(grad_free);
      // dQ = s dS K (query rows), dK = s dS^T Q, dV = P^T dO (key rows): staged
      // in this warp's rows of the dS tile, which the gradient MMAs have read.
      stage_row32(stg_q, lane, gq, args.scale);
      stage_row32(stg_k, lane, gk, args.scale);
      stage_row32(stg_v, lane, gv, 1.0f);
      fence_async_smem();
      __syncwarp();
      if (lane < kStoreLanes) {
        // lane L stores tensor L % 3 (dQ, dK, dV) (with image windows, the
        // quadrant L / 3 of the warp's two)
        const int r0 = warp * 32;
        const int wwin = t * NW + r0 / NP, n0 = r0 % NP;
        const int c = lane % 3;
        const CUtensorMap* mp = c == 0 ? &mDQ : c == 1 ? &mDK : &mDV;
        const uint32_t src = c == 0 ? stg_q : c == 1 ? stg_k : stg_v;
        if (wwin < args.BH && n0 < N) {
          if constexpr (IMG) {
            // the warp's rows lie in this thread's window (b, wy, wx, h)
            const int k = lane / 3;
            const int qd = (n0 >> 4) + k;
            const int y = wrap(wy * 8 + 4 * (qd >> 1) + args.shift, args.img_h);
            const int x = wrap(wx * 8 + 4 * (qd & 1) + args.shift, args.img_w);
            tma_store_5d(mp, src + k * 1024, 0, h, x, y, b);
          } else {
            tma_store_3d(mp, src, 0, n0, wwin);
          }
        }
        bulk_commit();
      }
      // dU = dS W (query row), dW = dS^T U = s dS^T U' (key row).
      if constexpr (RP > 0) {
        if (valid) {
          size_t ur = static_cast<size_t>(win) * N + n;
          if constexpr (IMG) {
            // factor row = the token's raster position in its window
            const int qq = n >> 4;
            const int ty = 4 * (qq >> 1) + ((n >> 2) & 3), tx = 4 * (qq & 1) + (n & 3);
            ur = static_cast<size_t>(win) * 64 + ty * 8 + tx;
          }
          const float f = args.scale;
          if (args.du_part != nullptr) {
            float4* pu = reinterpret_cast<float4*>(args.du_part + ur * args.r);
            float4* pw = reinterpret_cast<float4*>(args.dw_part + ur * args.r);
#pragma unroll
            for (int c = 0; c < RP; c += 4) {
              if (c < args.r) {
                pu[c >> 2] = make_float4(__uint_as_float(gq[D + c]), __uint_as_float(gq[D + c + 1]),
                                         __uint_as_float(gq[D + c + 2]), __uint_as_float(gq[D + c + 3]));
                pw[c >> 2] = make_float4(__uint_as_float(gk[D + c]) * f, __uint_as_float(gk[D + c + 1]) * f,
                                         __uint_as_float(gk[D + c + 2]) * f,
                                         __uint_as_float(gk[D + c + 3]) * f);
              }
            }
          } else {
            uint4* pu = reinterpret_cast<uint4*>(args.du + ur * args.r);
            uint4* pw = reinterpret_cast<uint4*>(args.dw + ur * args.r);
#pragma unroll
            for (int c = 0; c < RP; c += 8) {
              if (c < args.r) {
                pu[c >> 3] = make_uint4(
                    pack_bf16x2(__uint_as_float(gq[D + c]), __uint_as_float(gq[D + c + 1])),
                    pack_bf16x2(__uint_as_float(gq[D + c + 2]), __uint_as_float(gq[D + c + 3])),
                    pack_bf16x2(__uint_as_float(gq[D + c + 4]), __uint_as_float(gq[D + c + 5])),
                    pack_bf16x2(__uint_as_float(gq[D + c + 6]), __uint_as_float(gq[D + c + 7])));
                pw[c >> 3] = make_uint4(
                    pack_bf16x2(__uint_as_float(gk[D + c]) * f, __uint_as_float(gk[D + c + 1]) * f),
                    pack_bf16x2(__uint_as_float(gk[D + c + 2]) * f, __uint_as_float(gk[D + c + 3]) * f),
                    pack_bf16x2(__uint_as_float(gk[D + c + 4]) * f, __uint_as_float(gk[D + c + 5]) * f),
                    pack_bf16x2(__uint_as_float(gk[D + c + 6]) * f, __uint_as_float(gk[D + c + 7]) * f));
              }
            }
          }
        }
      }
    }
    // The TMA stores must have finished before the CTA exits.
    if (lane < kStoreLanes) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Shared factors: dU[h] = sum over the windows b of the fp32 rows of window-head
// b H + h (likewise dW), rounded to bf16 once.  One block per factor row
// (h, n); its threads split the windows (each sums every G-th window of one
// 4-column group in fp32), then the partial sums are added in a fixed order.
// du_src / dw_src rows are du_stride / dw_stride floats apart.
__global__ void __launch_bounds__(256) sum_bias_grads_kernel(const float* du_src, int du_stride,
                                                           const float* dw_src, int dw_stride,
                                                           __nv_bfloat16* du, __nv_bfloat16* dw,
                                                           int B, int H, int N, int r) {
  __shared__ float4 part[256];
  grid_dep_wait();
  const int hrow = blockIdx.x;            // h * N + n
  const int nv = r / 2;                   // float4 columns: r / 4 of dU, then r / 4 of dW
  const int G = blockDim.x / nv;          // window groups
  const int col = threadIdx.x % nv, grp = threadIdx.x / nv;
  const bool is_w = col >= nv / 2;
  const int c = (is_w ? col - nv / 2 : col) * 4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (grp < G) {
    const float* src = is_w ? dw_src : du_src;
    const long stride = is_w ? dw_stride : du_stride;
    for (int b = grp; b < B; b += G) {
      const float4 v = *reinterpret_cast<const float4*>(src + (static_cast<long>(b) * H * N + hrow) * stride + c);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
  }
  part[threadIdx.x] = acc;
  __syncthreads();
  if (threadIdx.x < nv) {
    float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k = 0; k < G; ++k) {
      const float4 v = part[threadIdx.x + k * nv];
      sum.x += v.x;
      sum.y += v.y;
      sum.z += v.z;
      sum.w += v.w;
    }
    uint2 o;
    o.x = pack_bf16x2(sum.x, sum.y);
    o.y = pack_bf16x2(sum.z, sum.w);
    *reinterpret_cast<uint2*>((is_w ? dw : du) + static_cast<long>(hrow) * r + c) = o;
  }
}

}  // namespace rfb
