// fwd_kernels.cuh -- forward of attention with an additive rank-factorised bias,
//
//     O = softmax(s Q K^T + U W^T) V,   LSE_i = log sum_j exp(S_ij),
//
// on sm_100a.  The bias is never materialised: following "Rank-Factorized
// Implicit Neural Bias" (Abstract: the low-rank bias factors are concatenated
// with the content channels so the element-wise bias addition becomes part of
// the dot product), the score tile is ONE tcgen05 accumulation over the
// concatenated contraction [Q | U'] . [K | W]^T, with U' = U / s staged on chip,
// so that the accumulator holds S / s and the softmax applies s log2(e).
// "FlashBias" (Abstract) is the reason this matters: a low-rank bias keeps the
// fused attention pipeline intact.
//
// Two kernels:
//   * fwd_window_kernel  (N <= 128): persistent CTAs; each 128-row tile packs
//     128/NP whole windows (NP = 64 or 128 rows per window).  One S tile per
//     tile, single-pass softmax, block-diagonal P (off-window blocks stay 0).
//     Warps 0-3 and 4-7 softmax + epilogue of even and odd tiles (thread = row
//     = TMEM lane; a tile's epilogue runs after the warpgroup's next
//     exponentials, O leaves by TMA stores), warp 8 TMA producer (a tile's
//     copies spread over its lanes), warp 9 score MMAs, warp 10 PV MMAs,
//     warp 11 U' scaling; P goes back into TMEM (packed bf16) for the PV MMA.
//   * fwd_long_kernel    (N > 128): persistent CTAs over units (head, two
//     128-query tiles); each unit loops over 128-key tiles with an online
//     softmax (lazy rescale of O in TMEM).  Warps 0-15 are four softmax
//     warpgroups, one per (query tile, 64-key half), exchanging half-row
//     maxima through shared memory; warp 16 TMA; warps 17 / 18 MMA issue for
//     query tile 0 / 1 (with d = 32 the next unit's first scores are issued
//     before the current unit ends); P goes back into TMEM as packed bf16
//     and the PV MMA reads it from there.  With d = 32 the row sums of P come
//     out of the PV MMA (a block of ones beside V), not from the softmax.
// Operands are staged by TMA with the swizzle that matches their row width.
#pragma once
#include "sm100.cuh"

namespace rfb {

constexpr int kTile = 128;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2eF = 1.4426950408889634f;

struct FwdArgs {
  __nv_bfloat16* o;  // [BH, N, D]
  float* lse;        // [BH, N]
  int* err;          // device error word
  int BH;
  int N;
  // Heads of the U / W tensors: BH (factors per window and head) or H (one
  // pair per head, shared by all windows).  Window-head bh uses bias head
  // bh % bias_heads (bh = b H + h).
  int bias_heads;
  // Image-window mode of the window kernel (feature maps [B, img_h, img_w,
  // img_heads, D], 8 x 8 windows of the map rolled by -shift): window-head
  // bh = ((b * (img_h / 8) + wy) * (img_w / 8) + wx) * img_heads + h.
  int img_h, img_w, img_heads, shift;
  // Window kernel: how U / W reach shared memory.  kBiasTile: one copy per
  // tile (per-window factors); kBiasWindow: one copy per window (shared
  // factors); kBiasResident: all bias heads loaded once per CTA (shared
  // factors that fit), followed by copies of heads 0 .. NW-2 so that any NW
  // consecutive windows' heads are contiguous.
  int bias_mode;
  float scale_log2;  // s * log2(e)
  float inv_scale;   // 1 / s  (U' = bf16(U / s))
  uint64_t timeout_ns;  // limit of each main-loop wait
  int fail_site;        // test hook: wait site that gives up at once (-1: none)
};

__device__ __forceinline__ uint8_t* align_1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Bounded wait that ignores the abort flag: used only on the exit path to let
// in-flight copies and MMAs land before the CTA frees its resources.
__device__ __forceinline__ void wait_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kDrainTimeoutNs) return;
  }
}

template <int NC>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[NC]) {
  if constexpr (NC == 16) tmem_ld16(taddr, r);
  else if constexpr (NC == 32) tmem_ld32(taddr, r);
  else if constexpr (NC == 64) tmem_ld64(taddr, r);
  else tmem_ld128(taddr, r);
}
template <int NC>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t (&r)[NC]) {
  if constexpr (NC == 16) tmem_st16(taddr, r);
  else if constexpr (NC == 32) tmem_st32(taddr, r);
  else tmem_st64(taddr, r);
}

// Write one normalised output row (D bf16 values, 16-byte stores).
template <int D>
__device__ __forceinline__ void store_o_row(__nv_bfloat16* dst, const uint32_t (&ov)[D], float inv) {
  uint4* p = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int c = 0; c < D; c += 8) {
    uint4 v;
    v.x = pack_bf16x2(__uint_as_float(ov[c + 0]) * inv, __uint_as_float(ov[c + 1]) * inv);
    v.y = pack_bf16x2(__uint_as_float(ov[c + 2]) * inv, __uint_as_float(ov[c + 3]) * inv);
    v.z = pack_bf16x2(__uint_as_float(ov[c + 4]) * inv, __uint_as_float(ov[c + 5]) * inv);
    v.w = pack_bf16x2(__uint_as_float(ov[c + 6]) * inv, __uint_as_float(ov[c + 7]) * inv);
    p[c >> 3] = v;
  }
}

// Sets raw scores at positions >= valid to -inf (only the last key tile of a
// row is ragged, so this runs at most once per row).
template <int NC>
__device__ __forceinline__ void mask_tail(uint32_t (&sv)[NC], int valid) {
#pragma unroll
  for (int c = 0; c < NC; ++c)
    if (c >= valid) sv[c] = 0xFF800000u;
}

// Row maximum with 8 independent partial maxima (short dependency chains),
// two new values per three-input max.
template <int NC>
__device__ __forceinline__ float row_max(const uint32_t (&sv)[NC]) {
  float m[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) m[e] = __uint_as_float(sv[e]);
  int c = 8;
#pragma unroll
  for (; c + 16 <= NC; c += 16)
#pragma unroll
    for (int e = 0; e < 8; ++e)
      m[e] = fmax3(m[e], __uint_as_float(sv[c + e]), __uint_as_float(sv[c + 8 + e]));
  if (c < NC) {
#pragma unroll
    for (int e = 0; e < 8; ++e) m[e] = fmaxf(m[e], __uint_as_float(sv[c + e]));
  }
  return fmax3(fmax3(m[0], m[1], m[2]), fmax3(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
}

// p_j = 2^(s_j * sl2 - m) for the NC scores of this thread's row, written as
// packed bf16 pairs into its TMEM lane (column p_tm + c / 2 holds keys c and
// c + 1), where the PV MMA reads them as its A operand; returns sum_j p_j
// (fp32; the arguments and four partial sums in packed f32x2 arithmetic, one
// instruction per pair).  Masked scores are -inf and give p = 0.  SOFT_PAIRS
// of every 4 pairs of exponentials use the software exp2 (FMA / integer pipes)
// instead of the MUFU unit.  The stores are not awaited (tmem_st_wait()).
template <int NC, int SOFT_PAIRS = 0>
__device__ __forceinline__ float exp_row_to_tmem(const uint32_t (&sv)[NC], float sl2, float m,
                                                 uint32_t p_tm) {
  constexpr int HW = 8 - 2 * SOFT_PAIRS;
  const uint64_t sl2x2 = f2_pack(sl2, sl2);
  const uint64_t nm2 = f2_pack(-m, -m);
  uint64_t l2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
  for (int c0 = 0; c0 < NC; c0 += 32) {
    uint32_t pk[16];
#pragma unroll
    for (int c = c0; c < c0 + 32; c += 8) {
      float p[8];
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        const uint64_t x2 = static_cast<uint64_t>(sv[c + e + 1]) << 32 | sv[c + e];
        const float2 a = f2_unpack(f2_fma(x2, sl2x2, nm2));
        if (e < HW) {
          p[e] = fast_exp2(a.x);
          p[e + 1] = fast_exp2(a.y);
        } else {
          soft_exp2_x2(a.x, a.y, p[e], p[e + 1]);
        }
        l2[e >> 1] = f2_add(l2[e >> 1], f2_pack(p[e], p[e + 1]));
        pk[(c - c0 + e) >> 1] = pack_bf16x2(p[e], p[e + 1]);
      }
    }
    tmem_st16_nowait(p_tm + (c0 >> 1), pk);
  }
  const float2 a = f2_unpack(f2_add(l2[0], l2[1])), b = f2_unpack(f2_add(l2[2], l2[3]));
  return (a.x + a.y) + (b.x + b.y);
}

// Issue the score MMAs  S(tmem) = Q.K^T + U'.W^T  for one 128x128 tile.
template <int D, int RP>
__device__ __forceinline__ void issue_scores(uint32_t s_tmem, uint32_t q, uint32_t k, uint32_t u,
                                             uint32_t w) {
  constexpr uint32_t id = idesc_bf16_f32(128, 128, false, false);
  const uint64_t dq = desc_kmajor(q, D * 2), dk = desc_kmajor(k, D * 2);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk)
    umma_bf16(s_tmem, desc_add(dq, kk * 32), desc_add(dk, kk * 32), id, kk > 0 ? 1u : 0u);
  if constexpr (RP > 0) {
    const uint64_t du = desc_kmajor(u, RP * 2), dw = desc_kmajor(w, RP * 2);
#pragma unroll
    for (int kk = 0; kk < RP / 16; ++kk)
      umma_bf16(s_tmem, desc_add(du, kk * 32), desc_add(dw, kk * 32), id, 1u);
  }
}

// Issue O(tmem) (+)= P . V for a 128-key tile with P read from TMEM (packed
// bf16, 8 columns per 16 keys), V MN-major in shared memory.
template <int D>
__device__ __forceinline__ void issue_pv_ts(uint32_t o_tmem, uint32_t p_tmem, uint32_t v,
                                            bool accumulate) {
  constexpr uint32_t id = idesc_bf16_f32(128, D, false, true);
  const uint64_t dv = desc_mnmajor(v, D * 2, 128 * D * 2);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    umma_bf16_ts(o_tmem, p_tmem + kk * 8, desc_add(dv, kk * 16 * (D * 2)), id,
                 (accumulate || kk > 0) ? 1u : 0u);
}

// O'(tmem) (+)= P . [V | 1] (N = D + 16): the second MN block of B is a
// constant block of ones `ones_off` bytes after V, so columns D .. D + 15 of
// O' accumulate the row sums of P.
template <int D>
__device__ __forceinline__ void issue_pv_ts_ones(uint32_t o_tmem, uint32_t p_tmem, uint32_t v,
                                                 uint32_t ones_off, bool accumulate) {
  constexpr uint32_t id = idesc_bf16_f32(128, D + 16, false, true);
  const uint64_t dv = desc_mnmajor(v, D * 2, ones_off);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    umma_bf16_ts(o_tmem, p_tmem + kk * 8, desc_add(dv, kk * 16 * (D * 2)), id,
                 (accumulate || kk > 0) ? 1u : 0u);
}

// ============================================================ window regime
constexpr int kBiasTile = 0, kBiasWindow = 1, kBiasResident = 2;

// IMG: windows gathered from feature maps (8 x 8 windows, NP = 64), factors
// always resident, so a stage holds only Q, K, V.
template <int D, int RP, int NP, bool IMG = false>
struct WinCfg {
  static_assert(!IMG || NP == 64, "image windows are 8 x 8");
  static constexpr int NW = kTile / NP;       // windows packed per tile
  static constexpr int QB = kTile * D * 2;    // bytes of a Q / K / V tile
  static constexpr int UB = kTile * RP * 2;   // bytes of a U / W tile
  static constexpr int STAGE = 3 * QB + (IMG ? 0 : 2 * UB);
  // O of a tile is staged per softmax warpgroup (swizzled like the O tensor
  // map) and written by TMA stores, one per warp and 32 rows.
  static constexpr int OB = kTile * D * 2;
  // Image windows keep every head's factors resident: leave 32 KB for them.
  static constexpr int NS_FIT = (224 * 1024 - 2 * OB - (IMG ? 32 * 1024 : 0)) / STAGE;
  static constexpr int NS = NS_FIT > 6 ? 6 : NS_FIT;
  static constexpr int OFF_OST = NS * STAGE;
  static constexpr int OFF_BAR = OFF_OST + 2 * OB;
  // TMEM columns: S_a at 128 a, O_a at 256 + D a, P_a (packed bf16) at 384 + 64 a.
  static constexpr int T_O = 256, T_P = 384;
  // in_full[NS] u_ready[NS] in_empty[NS] s_full[2] s_empty[2] p_full[2] o_full[2]
  // acc_empty[2] drain res_full res_ready
  static constexpr int NBAR = 3 * NS + 13;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
  // Resident shared factors start after the barriers; one head's U or W rows.
  static constexpr int OFF_RES = (OFF_BAR + NBAR * 8 + 16 + 1023) / 1024 * 1024;
  static constexpr int HB = NP * RP * 2;
  static constexpr int res_bytes(int heads) { return 2 * (heads + NW - 1) * HB; }
  static_assert(NS >= 2, "not enough shared memory for two input stages");
  static_assert(SMEM <= 232448, "shared memory budget exceeded");
  static_assert(QB % 1024 == 0 && UB % 1024 == 0, "tile alignment");
};

// Warps 0-3 / 4-7 softmax + epilogue of even / odd tiles, 8 TMA, 9 score MMAs,
// 10 PV MMAs, 11 U' scaling.  Registers as in the long kernel: launched with 168
// per thread, control warpgroup down to 56, softmax warpgroups up to 208.
constexpr int kWinThreads = 384;
constexpr uint32_t kWinSoftmaxRegs = 208, kWinControlRegs = 56;
static_assert(2 * 128 * kWinSoftmaxRegs + 128 * kWinControlRegs <= kWinThreads * 168,
              "register split exceeds the launch budget");

// With IMG the Q / K / V / O maps are 5-D over the feature maps (D, heads, W,
// H, B) with a 4 x 4-token box, and U / W 4-D (r, 8, 8, heads) with a 4 x 4
// box: each window is copied as four 4 x 4 quadrants, so inside the kernel its
// tokens are in quadrant-major order (row 16 q + 4 (y % 4) + x % 4, q = 2 (y /
// 4) + x / 4) for Q, K, V, U and W alike; O and LSE go back to map positions.
// Otherwise mO is the 3-D map of O [BH, N, D] with a 32-row box.
template <int D, int RP, int NP, bool IMG = false>
__global__ void __launch_bounds__(kWinThreads, 1)
    fwd_window_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                      const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mU,
                      const __grid_constant__ CUtensorMap mW, const __grid_constant__ CUtensorMap mO,
                      const FwdArgs args) {
  using C = WinCfg<D, RP, NP, IMG>;
  constexpr int NS = C::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_1024(smem_raw);
  const uint32_t sb = smem_u32(smem);
  const uint32_t bar0 = sb + C::OFF_BAR;
  auto in_full = [&](int s) { return bar0 + 8u * s; };
  auto u_ready = [&](int s) { return bar0 + 8u * (NS + s); };  // U' scaled in stage s
  auto in_empty = [&](int s) { return bar0 + 8u * (2 * NS + s); };
  auto s_full = [&](int a) { return bar0 + 8u * (3 * NS + a); };
  auto s_empty = [&](int a) { return bar0 + 8u * (3 * NS + 2 + a); };
  auto p_full = [&](int a) { return bar0 + 8u * (3 * NS + 4 + a); };
  auto o_full = [&](int a) { return bar0 + 8u * (3 * NS + 6 + a); };
  auto acc_empty = [&](int a) { return bar0 + 8u * (3 * NS + 8 + a); };
  const uint32_t drain_bar = bar0 + 8u * (3 * NS + 10);
  const uint32_t res_full = bar0 + 8u * (3 * NS + 11);   // resident factors landed
  const uint32_t res_ready = bar0 + 8u * (3 * NS + 12);  // resident U' scaled
  const bool resident = RP > 0 && (IMG || args.bias_mode == kBiasResident);
  // Image windows: map coordinates of window-head bh.
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
  const int res_heads = args.bias_heads + C::NW - 1;
  const uint32_t res_u = sb + C::OFF_RES, res_w = res_u + res_heads * C::HB;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + C::NBAR * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = static_cast<int>(warp_id());
  const int lane = static_cast<int>(lane_id());
  const int num_tiles = (args.BH + C::NW - 1) / C::NW;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < NS; ++s) {
      mbar_init(in_full(s), 1);
      mbar_init(u_ready(s), 1);
      mbar_init(in_empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(s_full(a), 1);
      mbar_init(s_empty(a), 4);   // one arrival per softmax warp
      mbar_init(p_full(a), 4);
      mbar_init(o_full(a), 1);
      mbar_init(acc_empty(a), 4);
    }
    mbar_init(drain_bar, 2);
    mbar_init(res_full, 1);
    mbar_init(res_ready, 8);  // one arrival per softmax warp
    fence_mbar_init();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch(&mQ);
    tma_prefetch(&mK);
    tma_prefetch(&mV);
    tma_prefetch(&mO);
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
  grid_dep_launch_next();

  if (warp >= 8) {
   // Control warpgroup: all four warps shrink their budget at this point.
   warpgroup_reg_dealloc<kWinControlRegs>();
   if (warp == 8) {
    // ------------------------------------------------------------ producer
    // The whole warp runs the loop: lane 0 posts the expected bytes and issues
    // the resident factors' copies; the lanes share a tile's copies (with
    // image windows 4 quadrant copies per tensor and window).
    if (resident && lane == 0) {
      // Every bias head once (head hh % H at slot hh), for the whole kernel.
      mbar_expect_tx(res_full, C::res_bytes(args.bias_heads));
      for (int hh = 0; hh < res_heads; ++hh) {
        const int z = hh % args.bias_heads;
        if constexpr (IMG) {
#pragma unroll
          for (int qd = 0; qd < 4; ++qd) {
            const uint32_t off = hh * C::HB + qd * (16 * RP * 2);
            tma_load_4d(res_u + off, &mU, res_full, 0, 4 * (qd & 1), 4 * (qd >> 1), z);
            tma_load_4d(res_w + off, &mW, res_full, 0, 4 * (qd & 1), 4 * (qd >> 1), z);
          }
        } else {
          tma_load_3d(res_u + hh * C::HB, &mU, res_full, 0, 0, z);
          tma_load_3d(res_w + hh * C::HB, &mW, res_full, 0, 0, z);
        }
      }
    }
    const uint32_t stage_tx = resident ? 3 * C::QB : C::STAGE;
    int it = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++it) {
      const int s = it % NS;
      if (it >= NS && !wait_warp(in_empty(s), ((it / NS) + 1) & 1, g, 1)) break;
      const uint32_t st = sb + s * C::STAGE;
      if (lane == 0) mbar_expect_tx(in_full(s), stage_tx);
      __syncwarp();
      const int w0 = t * C::NW;
      if constexpr (IMG) {
        // Each window as four 4 x 4 quadrants of the rolled map, taken from
        // the unrolled map at (row + shift, column + shift) mod size.  A
        // missing last window repeats the previous one (not stored).  Copy
        // j = (window i, quadrant qd, tensor c) goes to lane j % 32.
        for (int jj = lane; jj < C::NW * 4 * 3; jj += 32) {
          const int i = jj / 12, qd = (jj / 3) % 4, c = jj % 3;
          int b, wy, wx, h;
          window_of(min(w0 + i, args.BH - 1), b, wy, wx, h);
          const int y = wrap(wy * 8 + 4 * (qd >> 1) + args.shift, args.img_h);
          const int x = wrap(wx * 8 + 4 * (qd & 1) + args.shift, args.img_w);
          const uint32_t off = i * (NP * D * 2) + qd * (16 * D * 2);
          tma_load_5d(st + c * C::QB + off, c == 0 ? &mQ : c == 1 ? &mK : &mV, in_full(s), 0, h, x,
                      y, b);
        }
      } else if (lane == 0) {
        tma_load_3d(st, &mQ, in_full(s), 0, 0, w0);
        tma_load_3d(st + C::QB, &mK, in_full(s), 0, 0, w0);
        tma_load_3d(st + 2 * C::QB, &mV, in_full(s), 0, 0, w0);
        if constexpr (RP > 0 && !IMG) {
          if (resident) {
            // factors already resident
          } else if (args.bias_mode == kBiasTile) {
            tma_load_3d(st + 3 * C::QB, &mU, in_full(s), 0, 0, w0);
            tma_load_3d(st + 3 * C::QB + C::UB, &mW, in_full(s), 0, 0, w0);
          } else {
            // Shared factors: one copy per window (its bias head), since
            // consecutive windows' bias heads wrap around at H.
#pragma unroll
            for (int i = 0; i < C::NW; ++i) {
              const int z = (w0 + i) % args.bias_heads;
              tma_load_3d(st + 3 * C::QB + i * (C::UB / C::NW), &mU, in_full(s), 0, 0, z);
              tma_load_3d(st + 3 * C::QB + C::UB + i * (C::UB / C::NW), &mW, in_full(s), 0, 0, z);
            }
          }
        }
      }
    }
    // Let the last copies land before the CTA can exit.
    if (lane == 0) {
      if (resident) wait_drain(res_full, 0);
      for (int j = (it > NS ? it - NS : 0); j < it; ++j)
        wait_drain(in_full(j % NS), (j / NS) & 1);
    }
   } else if (warp == 9) {
    // --------------------------------------------------- score MMA issue
    bool ok = true;
    if (resident) ok = wait_warp(res_ready, 0, g, 9);
    int it = 0;
    for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x, ++it) {
      const int s = it % NS, a = it & 1;
      // Inputs landed (and, with per-tile factors, U' scaled in place).
      const uint32_t ready = (RP > 0 && !resident) ? u_ready(s) : in_full(s);
      if (!wait_warp(ready, (it / NS) & 1, g, 2)) { ok = false; break; }
      // S_a is free once the softmax of tile it - 2 has loaded it.
      if (it >= 2 && !wait_warp(s_empty(a), ((it >> 1) + 1) & 1, g, 4)) { ok = false; break; }
      tc_fence_after();
      const uint32_t st = sb + s * C::STAGE;
      // Resident factors: the NW windows' heads are contiguous from head w0 % H.
      const uint32_t hoff = resident ? ((t * C::NW) % args.bias_heads) * C::HB : 0u;
      const uint32_t ua = resident ? res_u + hoff : st + 3 * C::QB;
      const uint32_t wa = resident ? res_w + hoff : st + 3 * C::QB + C::UB;
      issue_scores<D, RP>(tmem + a * 128, st, st + C::QB, ua, wa);
      umma_commit(s_full(a));
    }
    (void)ok;
    umma_commit(drain_bar);
    wait_drain(drain_bar, 0);
    __syncwarp();
   } else if (warp == 10) {
    // ------------------------------------------------------ PV MMA issue
    int it = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++it) {
      const int s = it % NS, a = it & 1;
      if (!wait_warp(p_full(a), (it >> 1) & 1, g, 3)) break;
      // O_a is free once the epilogue of tile it - 2 has read it.
      if (it >= 2 && !wait_warp(acc_empty(a), ((it >> 1) + 1) & 1, g, 7)) break;
      tc_fence_after();
      issue_pv_ts<D>(tmem + C::T_O + a * D, tmem + C::T_P + a * 64, sb + s * C::STAGE + 2 * C::QB,
                     false);
      umma_commit(o_full(a));
      umma_commit(in_empty(s));
    }
    umma_commit(drain_bar);
    wait_drain(drain_bar, 0);
    __syncwarp();
   } else {
    // ------------------------------------------------- U' = U / s in place
    if (RP > 0 && resident) {
      // The softmax warpgroups scale the resident U (they are idle until the
      // first scores).
    } else if constexpr (RP > 0) {
      int it = 0;
      for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++it) {
        const int s = it % NS;
        if (!wait_warp(in_full(s), (it / NS) & 1, g, 8)) break;
        scale_tile_bf16(sb + s * C::STAGE + 3 * C::QB, C::UB, args.inv_scale);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(u_ready(s));
      }
    }
   }
  } else {
    // ------------------------------------------------- softmax + epilogue
    warpgroup_reg_alloc<kWinSoftmaxRegs>();
    // Warpgroup a (= warp / 4) takes the tiles with it % 2 == a, i.e. exactly
    // the tiles that use S, O and P buffer a, so the two warpgroups work on
    // consecutive tiles at the same time.
    const int a = warp >> 2;
    const int row = threadIdx.x & 127;  // TMEM lane == tile row
    const int wl = row / NP;            // window inside the tile
    const int n = row % NP;             // token inside the window
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t p_tm = tmem + lane_base + C::T_P + a * 64;
    const int N = args.N;
    const float sl2 = args.scale_log2;
    constexpr int kStoreLanes = IMG ? 2 : 1;  // lanes issuing the warp's O stores
    if (resident) {
      // U' = U / s for the resident factors, 16 bytes per thread per step.
      if (wait_warp(res_full, 0, g, 10)) {
        const uint32_t bytes = res_heads * C::HB;
        for (uint32_t off = threadIdx.x * 16u; off < bytes; off += 256u * 16u) {
          uint4 v = ld_shared_v4(res_u + off);
          uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            wv[e] = pack_bf16x2(__uint_as_float(wv[e] << 16) * args.inv_scale,
                                __uint_as_float(wv[e] & 0xFFFF0000u) * args.inv_scale);
          st_shared_v4(res_u + off, wv[0], wv[1], wv[2], wv[3]);
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(res_ready);
      }
    }
    // P_a starts at zero: each row only ever writes its own window's block of
    // NP / 2 columns, so the other blocks stay zero (block-diagonal P).
    {
      uint32_t zero[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) zero[e] = 0u;
#pragma unroll
      for (int c = 0; c < 64; c += 16) tmem_st16_nowait(p_tm + c, zero);
      tmem_st_wait();
    }
    // Epilogue of tile t (iteration it of the CTA), whose PV has landed
    // (o_full awaited): O_a is read (acc_empty frees it for the next PV), the
    // O rows go into this warpgroup's staging tile (the TMA store that read
    // the warp's rows two tiles ago must have finished reading them), one TMA
    // store per warp writes its 32 rows, and LSE is written directly.
    // (IMG: wb, wwy, wwx, wh = the row's window, decoded once per tile; the
    // warp's rows all lie in that window too.)
    auto epilogue = [&](int t, int it, float m, float l, int wb, int wwy, int wwx, int wh) {
      tc_fence_after();
      uint32_t ov[D];
      tmem_ld_cols<D>(tmem + lane_base + C::T_O + a * D, ov);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty(a));
      const uint32_t ost = sb + C::OFF_OST + a * C::OB;
      if (it >= 2) {
        if (lane < kStoreLanes) bulk_wait_read<0>();
        __syncwarp();
      }
      {
        const float inv = 1.0f / l;
#pragma unroll
        for (int c = 0; c < D; c += 8)
          st_shared_v4(ost + swz_offset(row, c >> 3, D * 2),
                       pack_bf16x2(__uint_as_float(ov[c + 0]) * inv, __uint_as_float(ov[c + 1]) * inv),
                       pack_bf16x2(__uint_as_float(ov[c + 2]) * inv, __uint_as_float(ov[c + 3]) * inv),
                       pack_bf16x2(__uint_as_float(ov[c + 4]) * inv, __uint_as_float(ov[c + 5]) * inv),
                       pack_bf16x2(__uint_as_float(ov[c + 6]) * inv, __uint_as_float(ov[c + 7]) * inv));
      }
      fence_async_smem();
      __syncwarp();
      if (lane < kStoreLanes) {
        const int r0 = (warp & 3) * 32;           // the warp's first tile row
        const int wwin = t * C::NW + r0 / NP;     // its window
        const int n0 = r0 % NP;                   // its first token in the window
        if (wwin < args.BH && n0 < N) {
          if constexpr (IMG) {
            // lane k stores quadrant k of the warp's two
            const int qd = (n0 >> 4) + lane;
            const int y = wrap(wwy * 8 + 4 * (qd >> 1) + args.shift, args.img_h);
            const int x = wrap(wwx * 8 + 4 * (qd & 1) + args.shift, args.img_w);
            tma_store_5d(&mO, ost + (r0 + 16 * lane) * (D * 2), 0, wh, x, y, wb);
          } else {
            tma_store_3d(&mO, ost + r0 * (D * 2), 0, n0, wwin);
          }
        }
        bulk_commit();
      }
      const int win = t * C::NW + wl;
      if (win < args.BH && n < N) {
        size_t r = static_cast<size_t>(win) * N + n;
        if constexpr (IMG) {
          // the token's place in the unrolled map
          const int qq = n >> 4;
          const int y = wrap(wwy * 8 + 4 * (qq >> 1) + ((n >> 2) & 3) + args.shift, args.img_h);
          const int x = wrap(wwx * 8 + 4 * (qq & 1) + (n & 3) + args.shift, args.img_w);
          r = ((static_cast<size_t>(wb) * args.img_h + y) * args.img_w + x) * args.img_heads + wh;
        }
        args.lse[r] = (m + __log2f(l)) * kLn2;
      }
    };
    // Each tile's epilogue runs after the next tile's exponentials (of this
    // warpgroup), so the tile's PV overlaps them instead of being waited for.
    bool ok = true, pending = false;
    int pt = 0, pit = 0;       // the tile whose epilogue is pending
    float pm = 0.f, pl = 1.f;  // its row maximum and row sum
    int pb = 0, pwy = 0, pwx = 0, ph = 0;  // its window
    int it = a;
    for (int t = blockIdx.x + a * gridDim.x; t < num_tiles; t += 2 * gridDim.x, it += 2) {
      if (!wait_warp(s_full(a), (it >> 1) & 1, g, 5)) { ok = false; break; }
      tc_fence_after();
      uint32_t sv[NP];
      tmem_ld_cols<NP>(tmem + lane_base + a * 128 + wl * NP, sv);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_empty(a));
      if (N < NP) mask_tail<NP>(sv, N);
      int wb = 0, wwy = 0, wwx = 0, wh = 0;  // this row's window (image windows)
      if constexpr (IMG) {
        window_of(min(t * C::NW + wl, args.BH - 1), wb, wwy, wwx, wh);
        // Shifted-window mask: in the last window row (column) of the rolled
        // map the two quadrant rows (columns) come from opposite edges of the
        // unrolled map; keys of another region are excluded.
        if (args.shift > 0) {
          const int qq = n >> 4;
          const bool split_y = wwy == nwy - 1, split_x = wwx == nwx - 1;
          if (split_y || split_x) {  // windows inside the map need no mask
#pragma unroll
            for (int kq = 0; kq < 4; ++kq) {
              const bool ok_key = (!split_y || (kq >> 1) == (qq >> 1)) &&
                                  (!split_x || (kq & 1) == (qq & 1));
              if (!ok_key) {
#pragma unroll
                for (int e = 0; e < 16; ++e) sv[kq * 16 + e] = 0xFF800000u;
              }
            }
          }
        }
      }
      const float m = row_max<NP>(sv) * sl2;
      // P_a and O_a: the pending tile's PV must have read P_a and written O_a.
      if (pending && !wait_warp(o_full(a), (pit >> 1) & 1, g, 6)) { ok = false; break; }
      tc_fence_after();
      const float l = exp_row_to_tmem<NP>(sv, sl2, m, p_tm + wl * (NP / 2));
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full(a));
      // The pending tile's O is read now, so this tile's PV may start.
      if (pending) epilogue(pt, pit, pm, pl, pb, pwy, pwx, ph);
      pending = true;
      pt = t;
      pit = it;
      pm = m;
      pl = l;
      pb = wb;
      pwy = wwy;
      pwx = wwx;
      ph = wh;
    }
    if (ok && pending && wait_warp(o_full(a), (pit >> 1) & 1, g, 6))
      epilogue(pt, pit, pm, pl, pb, pwy, pwx, ph);
    // The O stores must have finished before the CTA exits.
    if (lane < kStoreLanes) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ============================================================== long regime
// DENSE: the materialised-bias comparator (no factors; each K/V stage also
// holds the two query tiles' 128 x 128 bf16 bias tiles, each as two 64-column
// 128-byte-swizzled halves).
template <int D, int RP, bool DENSE = false>
struct LongCfg {
  static_assert(!DENSE || RP == 0, "the dense-bias comparator takes no factors");
  static constexpr int QB = kTile * D * 2;
  static constexpr int UB = kTile * RP * 2;
  static constexpr int BT = DENSE ? kTile * kTile * 2 : 0;  // one query tile's bias tile
  static constexpr int OFF_BIAS = 2 * QB + UB;                // within a stage
  static constexpr int STAGE = 2 * QB + UB + 2 * BT;        // K, V, W, bias tiles
  // Two query tiles per unit: Q0 U0 Q1 U1, in QSETS sets so that the next
  // unit's tiles load while the current unit runs -- for d = 32, where the
  // K/V ring keeps its six stages; with d = 64 a second set would cost a K/V
  // stage, which measured slower.  Then the K/V stages.  P lives in TMEM.
  static constexpr int QSETS = (D == 32 && !DENSE) ? 2 : 1;
  static constexpr int OFF_Q = 0;  // set b, tile t at OFF_Q + (2 b + t) (QB + UB), U right after Q
  static constexpr int OFF_STAGE = QSETS * 2 * (QB + UB);
  // With d = 32 the row sums come out of the PV MMA: B is [V | 1] (a constant
  // 128 x 32 block of ones as a second MN block, N = d + 16), so column d of
  // the O accumulator collects sum_j bf16(p_j) and the softmax adds nothing.
  static constexpr bool LCOL = (D == 32);
  static constexpr int OD = LCOL ? D + 16 : D;  // O accumulator columns per query tile
  static constexpr int ONES = LCOL ? kTile * 64 : 0;
  // Shared-memory exchange between the two key-half warpgroups of a query
  // tile: half-row maxima [t][h][128] (and, at the end of a unit, key half
  // 1's row sums in the [t][0] slots).
  static constexpr int XCH = 2 * 2 * kTile * 4;
  static constexpr int NS_FIT = (232448 - 256 - OFF_STAGE - ONES - XCH) / STAGE;
  static constexpr int NS = NS_FIT > 6 ? 6 : NS_FIT;
  static constexpr int OFF_ONES = OFF_STAGE + NS * STAGE;  // 1024-byte aligned
  static constexpr int OFF_MAX = OFF_ONES + ONES;
  static constexpr int OFF_BAR = OFF_MAX + XCH;
  // TMEM columns: S_t at 128 t, O_t at 256 + OD t, P_t (packed bf16) at 384 + 64 t.
  static constexpr int T_O = 256, T_P = 384;
  static_assert(T_O + 2 * OD <= T_P, "TMEM budget");
  static_assert(OFF_ONES % 1024 == 0, "ones block alignment");
  // q_full kv_full[NS] kv_empty[NS] s_full[2] s_empty[2] mx_full[2] p_full[2]
  // pv_done[2] drain q_empty o_empty[2] sum_full[2] q_full' q_empty' (second set)
  static constexpr int NBAR = 2 * NS + 19;
  // The dynamic shared memory is declared 1024-byte aligned and used without
  // slack (checked on entry).
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16;
  static_assert(NS >= 2, "not enough shared memory for two KV stages");
  static_assert(SMEM <= 232448, "shared memory budget exceeded");
};

// Warps 0-15: four softmax warpgroups, warpgroup g = 2 t + h takes query tile t
// and key half h (keys 64 h .. 64 h + 63 of every 128-key tile); warp 16 TMA
// producer; warps 17 / 18 MMA issue for query tiles 0 / 1.  A query tile's
// exponentials are shared by two warps on every scheduler, which keeps the
// exponential unit busier than one warp can; the other query tile's
// warpgroups meanwhile load scores, take maxima and wait for their MMAs.
constexpr int kLongThreads = 608;
// Pairs of every 4 softmax exponentials computed in software in the long
// forward (the MUFU unit is its limit).
constexpr int kLongSoftPairs = 1;

// Long regime: a persistent CTA per SM works through units (head, pair of
// 128-query tiles), each a loop over 128-key tiles.  Each query tile t has an
// MMA-issuing warp, an S buffer (TMEM columns 128 t), an O accumulator, a P
// buffer and two softmax warpgroups, one per key half of every tile; the two
// exchange their half-row maxima through shared memory so that both apply the
// same running maximum (online softmax with a lazy rescale of O, done by the
// key-half-0 warpgroup), and each keeps the row sums of its half.  The next
// tile's scores are issued as soon as both halves have loaded S, so they
// overlap the exponentials; each K/V tile serves 256 query rows.  Barrier
// phases run on across units.  With DENSE (the comparator) mU is the map of the
// dense bias [bias heads, N, N] (box 64 x 128) and mW is unused.
template <int D, int RP, bool DENSE = false>
__global__ void __launch_bounds__(kLongThreads, 1)
    fwd_long_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                    const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mU,
                    const __grid_constant__ CUtensorMap mW, const FwdArgs args) {
  using C = LongCfg<D, RP, DENSE>;
  constexpr int NS = C::NS;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  const uint32_t sb = smem_u32(smem);
  if (sb & 1023u) {  // the swizzled operand tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicCAS(args.err, 0, kErrAlignment | (97 << 8));
    return;
  }
  const uint32_t bar0 = sb + C::OFF_BAR;
  // Q / U' set b loaded, and read by the unit's last score MMAs.
  auto q_full = [&](int b) { return b == 0 ? bar0 : bar0 + 8u * (17 + 2 * NS); };
  auto kv_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto kv_empty = [&](int s) { return bar0 + 8u * (1 + NS + s); };
  auto s_full = [&](int t) { return bar0 + 8u * (1 + 2 * NS + t); };
  auto s_empty = [&](int t) { return bar0 + 8u * (3 + 2 * NS + t); };
  auto mx_full = [&](int t) { return bar0 + 8u * (5 + 2 * NS + t); };
  auto p_full = [&](int t) { return bar0 + 8u * (7 + 2 * NS + t); };
  auto pv_done = [&](int t) { return bar0 + 8u * (9 + 2 * NS + t); };
  const uint32_t drain_bar = bar0 + 8u * (11 + 2 * NS);
  // The unit's last score MMAs are done (Q / U' may be replaced); tile t's
  // epilogue has read O (the next unit's first PV may overwrite it); the key
  // half-1 row sums of tile t are in shared memory.
  auto q_empty = [&](int b) { return bar0 + 8u * (b == 0 ? 12 + 2 * NS : 18 + 2 * NS); };
  auto o_empty = [&](int t) { return bar0 + 8u * (13 + 2 * NS + t); };
  auto sum_full = [&](int t) { return bar0 + 8u * (15 + 2 * NS + t); };
  auto q_addr = [&](int b, int t) { return sb + C::OFF_Q + (2 * b + t) * (C::QB + C::UB); };
  auto u_addr = [&](int b, int t) { return q_addr(b, t) + C::QB; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + C::NBAR * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = static_cast<int>(warp_id());
  const int lane = static_cast<int>(lane_id());
  const int N = args.N;
  const int nkv = (N + kTile - 1) / kTile;
  const int npairs = (N + 2 * kTile - 1) / (2 * kTile);
  const int nunits = npairs * args.BH;
  // Units of this CTA: blockIdx.x, blockIdx.x + gridDim.x, ...  (consecutive
  // units share a head, so concurrent CTAs read the same K / V from L2).
  const int first = blockIdx.x, stride = gridDim.x;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int b = 0; b < 2; ++b) {
      mbar_init(q_full(b), 1);
      mbar_init(q_empty(b), 2);  // one commit per query tile's MMA warp
    }
    for (int s = 0; s < NS; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 2);  // one arrival per query tile's MMA warp
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(s_full(t), 1);
      // one arrival per warp (lane 0, after __syncwarp), both key halves
      mbar_init(s_empty(t), 8);
      mbar_init(mx_full(t), 8);
      mbar_init(p_full(t), 8);
      mbar_init(pv_done(t), 1);
      mbar_init(o_empty(t), 4);
      mbar_init(sum_full(t), 4);
    }
    mbar_init(drain_bar, 2);
    fence_mbar_init();
  }
  if constexpr (C::LCOL) {
    // bf16 1.0 everywhere (so the swizzle pattern of the block is immaterial);
    // the fence makes the stores visible to the tensor core (async proxy).
    uint4* ones = reinterpret_cast<uint4*>(smem + C::OFF_ONES);
    for (int i = threadIdx.x; i < C::ONES / 16; i += kLongThreads)
      ones[i] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    fence_async_smem();
  }
  if (warp == 16 && lane == 0) {
    tma_prefetch(&mQ);
    tma_prefetch(&mK);
    tma_prefetch(&mV);
    if constexpr (RP > 0 || DENSE) tma_prefetch(&mU);
    if constexpr (RP > 0) tma_prefetch(&mW);
  }
  if (warp == 17) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitGuard g{abort_flag, args.err, args.timeout_ns, args.fail_site};
  grid_dep_wait();

  if (warp == 16) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int it = 0, uc = 0;  // K/V tiles and units loaded so far
      bool ok = true;
      for (int u = first; ok && u < nunits; u += stride, ++uc) {
        const int bh = u / npairs, q0 = (u % npairs) * 2 * kTile;
        const int qb = uc % C::QSETS;
        if (uc >= C::QSETS &&
            !wait_bounded(q_empty(qb), ((uc / C::QSETS) - 1) & 1, g, 10))
          break;
        mbar_expect_tx(q_full(qb), 2 * (C::QB + C::UB));
        for (int t = 0; t < 2; ++t) {
          tma_load_3d(q_addr(qb, t), &mQ, q_full(qb), 0, q0 + t * kTile, bh);
          if constexpr (RP > 0)
            tma_load_3d(u_addr(qb, t), &mU, q_full(qb), 0, q0 + t * kTile, bh % args.bias_heads);
        }
        for (int j = 0; j < nkv; ++j, ++it) {
          const int s = it % NS;
          if (it >= NS && !wait_bounded(kv_empty(s), ((it / NS) + 1) & 1, g, 11)) {
            ok = false;
            break;
          }
          const uint32_t st = sb + C::OFF_STAGE + s * C::STAGE;
          mbar_expect_tx(kv_full(s), C::STAGE);
          tma_load_3d(st, &mK, kv_full(s), 0, j * kTile, bh);
          tma_load_3d(st + C::QB, &mV, kv_full(s), 0, j * kTile, bh);
          if constexpr (RP > 0)
            tma_load_3d(st + 2 * C::QB, &mW, kv_full(s), 0, j * kTile, bh % args.bias_heads);
          if constexpr (DENSE) {
            // bias[q0 + 128 t + row, 128 j + col] for both query tiles, in two
            // 64-column halves each
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
              for (int c = 0; c < 2; ++c)
                tma_load_3d(st + C::OFF_BIAS + t * C::BT + c * (C::BT / 2), &mU, kv_full(s),
                            j * kTile + c * 64, q0 + t * kTile, bh % args.bias_heads);
          }
        }
      }
      // No copy may still be in flight when the CTA exits.
      for (int k = (uc > C::QSETS ? uc - C::QSETS : 0); k < uc; ++k)
        wait_drain(q_full(k % C::QSETS), (k / C::QSETS) & 1);
      for (int i = (it > NS ? it - NS : 0); i < it; ++i) wait_drain(kv_full(i % NS), (i / NS) & 1);
    }
  } else if (warp == 17 || warp == 18) {
    // ---------------------------- MMA issue for query tile t (whole warp)
    const int t = warp - 17;
    int it = 0, jt = 0;  // K/V tiles, S tiles of this query tile
    bool ok = true;
    // Q_t / U'_t of this CTA's unit number ucn: loaded, and U' = U / s scaled
    // in place by this warp.
    auto prep_unit = [&](int ucn) -> bool {
      const int b = ucn % C::QSETS;
      if (!wait_warp(q_full(b), (ucn / C::QSETS) & 1, g, 12)) return false;
      if constexpr (RP > 0) {
        scale_tile_bf16(u_addr(b, t), C::UB, args.inv_scale);
        fence_async_smem();
      }
      __syncwarp();
      return true;
    };
    // S_t = Q_t K^T + U'_t W^T for K/V tile `itj` with Q / U' set qb, once
    // both halves have loaded the previous scores (s_empty).
    auto do_s = [&](int itj, int jtj, int qb) -> bool {
      const int s = itj % NS;
      if (!wait_warp(kv_full(s), (itj / NS) & 1, g, 13)) return false;
      if (jtj >= 1 && !wait_warp(s_empty(t), (jtj - 1) & 1, g, 14)) return false;
      tc_fence_after();
      const uint32_t st = sb + C::OFF_STAGE + s * C::STAGE;
      issue_scores<D, RP>(tmem + t * 128, q_addr(qb, t), st, u_addr(qb, t), st + 2 * C::QB);
      umma_commit(s_full(t));
      return true;
    };
    auto do_pv = [&](int itj, int jtj, bool first_of_unit) -> bool {
      const int s = itj % NS;
      if (!wait_warp(p_full(t), jtj & 1, g, 15)) return false;
      tc_fence_after();
      const uint32_t v = sb + C::OFF_STAGE + s * C::STAGE + C::QB;
      if constexpr (C::LCOL)
        issue_pv_ts_ones<D>(tmem + C::T_O + t * C::OD, tmem + C::T_P + t * 64, v,
                            sb + C::OFF_ONES - v, !first_of_unit);
      else
        issue_pv_ts<D>(tmem + C::T_O + t * D, tmem + C::T_P + t * 64, v, !first_of_unit);
      umma_commit(pv_done(t));
      umma_commit(kv_empty(s));
      return true;
    };
    if constexpr (C::QSETS == 2) {
      // One sequence over this CTA's tiles (unit uc, key tile j): the next
      // tile's scores are issued as soon as the softmax has loaded the
      // current ones, across unit boundaries too -- the next unit's Q / U'
      // are in the other set -- so a unit's first scores are ready when its
      // softmax starts.  The next unit's Q / U' are awaited (and U' scaled)
      // at key tile prep_j: the producer loads them after the current unit's
      // last K / V tile, whose stage the PV of tile nkv - 1 - NS releases, so
      // prep_j must come after that PV is issued (j >= nkv - NS), else the two
      // warps would wait for each other.
      const int nu = first < nunits ? (nunits - first + stride - 1) / stride : 0;
      const int prep_j = nkv / 2 > nkv - NS ? nkv / 2 : nkv - NS;
      if (nu > 0 && nkv > 0) {
        // Query tile 1 starts once tile 0's first P is written, so that the
        // two tiles' exponentials start offset.
        ok = prep_unit(0) && (t == 0 || wait_warp(p_full(0), 0, g, 15)) && do_s(0, 0, 0);
        int prepared = 1;  // units whose Q / U' are ready
        for (int uc = 0, j = 0; ok;) {
          const bool last_j = j + 1 == nkv;
          const bool has_next = !last_j || uc + 1 < nu;
          if (uc + 1 < nu && prepared == uc + 1 && j == prep_j) {
            if (!(ok = prep_unit(uc + 1))) break;
            ++prepared;
          }
          if (has_next && !(ok = do_s(it + 1, jt + 1, (last_j ? uc + 1 : uc) % 2))) break;
          if (last_j) umma_commit(q_empty(uc % 2));  // the unit's scores are all issued
          // The previous unit's epilogue must have read O before it is overwritten.
          if (j == 0 && uc > 0 && !(ok = wait_warp(o_empty(t), (uc - 1) & 1, g, 18))) break;
          if (!(ok = do_pv(it, jt, j == 0))) break;
          ++it;
          ++jt;
          if (!has_next) break;
          if (last_j) {
            ++uc;
            j = 0;
          } else {
            ++j;
          }
        }
      }
    } else {
      int uc = 0;
      for (int u = first; ok && u < nunits; u += stride, ++uc) {
        const int qb = uc % C::QSETS;
        if (!prep_unit(uc)) break;
        // Query tile 1 starts each unit once tile 0's first P is written, so
        // that the two tiles' exponentials start offset.
        ok = (t == 0 || wait_warp(p_full(0), jt & 1, g, 15)) && do_s(it, jt, qb);
        for (int j = 0; ok && j < nkv; ++j) {
          if (j + 1 < nkv) {
            if (!do_s(it + 1, jt + 1, qb)) { ok = false; break; }
          } else {
            umma_commit(q_empty(qb));  // the unit's last scores read Q_t / U'_t
          }
          // The previous unit's epilogue must have read O before it is overwritten.
          if (j == 0 && uc > 0 && !wait_warp(o_empty(t), (uc - 1) & 1, g, 18)) { ok = false; break; }
          if (!do_pv(it, jt, j == 0)) { ok = false; break; }
          ++it;
          ++jt;
        }
      }
    }
    umma_commit(drain_bar);
    wait_drain(drain_bar, 0);
    __syncwarp();
  } else if (warp < 16) {
    // ---------------------------------------- softmax, query tile t, key half h
    const int wg = warp >> 2;
    const int t = wg >> 1, h = wg & 1;
    const int row = threadIdx.x & 127;   // TMEM lane == query row within the tile
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t s_tm = tmem + lane_base + t * 128 + 64 * h;      // this half's scores
    const uint32_t o_tm = tmem + lane_base + C::T_O + t * C::OD;
    const uint32_t p_tm = tmem + lane_base + C::T_P + t * 64 + 32 * h;  // this half's P
    // half-row maxima [t][h][row]; key half 1's row sums go to the [t][0] slot
    // at the end of a unit (half 0 no longer writes it until its epilogue is
    // done, and half 1 has read half 0's last maximum).
    auto max_addr = [&](int hh) { return sb + C::OFF_MAX + (t * 2 + hh) * (kTile * 4) + row * 4; };
    const uint32_t sum_addr = max_addr(0);
    // Scores are accumulator * sl2 in log2 units; the comparator adds its bias
    // to the scaled scores first and then uses a unit factor.
    const float sl2 = DENSE ? 1.0f : args.scale_log2;
    int jt = 0, uc = 0;  // S tiles of this query tile so far, units
    bool ok = true;
    for (int u = first; ok && u < nunits; u += stride, ++uc) {
      const int bh = u / npairs, q0 = (u % npairs) * 2 * kTile;
      float m_run = -INFINITY, l = 0.f;  // l: this half's row sum (d = 64)
      for (int j = 0; j < nkv; ++j, ++jt) {
        if (!wait_warp(s_full(t), jt & 1, g, 16)) { ok = false; break; }
        tc_fence_after();
        uint32_t sv[64];
        tmem_ld_cols<64>(s_tm, sv);
        tc_fence_before();
        if constexpr (DENSE) {
          // s_j = acc_j s log2(e) + bias_j log2(e), the bias row from this K/V
          // tile's stage (its copy is awaited here too; it landed with K / V).
          const int s = jt % NS;
          if (!wait_warp(kv_full(s), (jt / NS) & 1, g, 20)) { ok = false; break; }
          const uint32_t bt = sb + C::OFF_STAGE + s * C::STAGE + C::OFF_BIAS + t * C::BT +
                              h * (C::BT / 2);
          const float sl = args.scale_log2;
#pragma unroll
          for (int c = 0; c < 64; c += 8) {
            const uint4 bv = ld_shared_v4(bt + row * 128 + (((c >> 3) ^ (row & 7)) << 4));
            const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              sv[c + 2 * e] = __float_as_uint(fmaf(__uint_as_float(sv[c + 2 * e]), sl,
                                                   __uint_as_float(bw[e] << 16) * kLog2eF));
              sv[c + 2 * e + 1] = __float_as_uint(
                  fmaf(__uint_as_float(sv[c + 2 * e + 1]), sl,
                       __uint_as_float(bw[e] & 0xFFFF0000u) * kLog2eF));
            }
          }
        }
        const int kvalid = N - j * kTile - 64 * h;  // keys of this half that exist
        if (kvalid < 64) mask_tail<64>(sv, kvalid);
        // Row maximum over both halves: publish this half's, read the other's.
        // The next scores (and with them the next maxima) wait for s_empty,
        // which both halves signal only after reading, so one slot suffices.
        const float mh = row_max<64>(sv) * sl2;
        asm volatile("st.shared.f32 [%0], %1;" ::"r"(max_addr(h)), "f"(mh) : "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(mx_full(t));
        if (!wait_warp(mx_full(t), jt & 1, g, 21)) { ok = false; break; }
        float mo;
        asm volatile("ld.shared.f32 %0, [%1];" : "=f"(mo) : "r"(max_addr(h ^ 1)) : "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(s_empty(t));
        const float m_new = fmax3(m_run, mh, mo);
        // Lazy rescale: keep the running max unless it grew by more than 2^8
        // (both halves take the same decision from the same values).
        const bool need = m_new > m_run + 8.0f;
        float alpha = 1.f;
        if (need) {
          alpha = fast_exp2(m_run - m_new);
          l *= alpha;
          m_run = m_new;
        }
        const bool fix_o = h == 0 && __any_sync(0xffffffffu, need && j > 0);
        // P_t and O_t: the previous PV must have finished.
        if (jt >= 1 && !wait_warp(pv_done(t), (jt - 1) & 1, g, 17)) { ok = false; break; }
        tc_fence_after();
        if constexpr (C::LCOL) exp_row_to_tmem<64, kLongSoftPairs>(sv, sl2, m_run, p_tm);
        else l += exp_row_to_tmem<64, kLongSoftPairs>(sv, sl2, m_run, p_tm);
        if (fix_o) {
          uint32_t ov[D];
          tmem_ld_cols<D>(o_tm, ov);
#pragma unroll
          for (int c = 0; c < D; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
          tmem_st_cols<D>(o_tm, ov);
          if constexpr (C::LCOL) {  // the row-sum columns
            uint32_t lv[16];
            tmem_ld_cols<16>(o_tm + D, lv);
#pragma unroll
            for (int c = 0; c < 16; ++c) lv[c] = __float_as_uint(__uint_as_float(lv[c]) * alpha);
            tmem_st_cols<16>(o_tm + D, lv);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full(t));
      }
      if (!ok || nkv == 0) break;
      if constexpr (!C::LCOL) {
        if (h == 1) {
          // Key half 1 hands its row sums to half 0, which writes the output.
          asm volatile("st.shared.f32 [%0], %1;" ::"r"(sum_addr), "f"(l) : "memory");
          __syncwarp();
          if (lane == 0) mbar_arrive(sum_full(t));
          continue;
        }
      } else {
        if (h == 1) continue;
      }
      if (!wait_warp(pv_done(t), (jt - 1) & 1, g, 19)) break;
      if constexpr (!C::LCOL) {
        if (!wait_warp(sum_full(t), uc & 1, g, 22)) break;
        float l1;
        asm volatile("ld.shared.f32 %0, [%1];" : "=f"(l1) : "r"(sum_addr) : "memory");
        l += l1;
      }
      tc_fence_after();
      const int q = q0 + t * kTile + row;
      uint32_t ov[D];
      tmem_ld_cols<D>(o_tm, ov);
      if constexpr (C::LCOL) {
        uint32_t lv[16];
        tmem_ld_cols<16>(o_tm + D, lv);
        l = __uint_as_float(lv[0]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_empty(t));
      if (q < N) {
        const size_t r = static_cast<size_t>(bh) * N + q;
        store_o_row<D>(args.o + r * D, ov, 1.0f / l);
        args.lse[r] = (m_run + __log2f(l)) * kLn2;
      }
    }
  }

  // This CTA's work is done: the next grid may start launching (a long
  // kernel gains nothing from letting it in earlier).
  grid_dep_launch_next();
  tc_fence_before();
  __syncthreads();
  if (warp == 17) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace rfb
