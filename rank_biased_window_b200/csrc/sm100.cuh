// sm100.cuh -- thin inline-PTX wrappers for the Blackwell (sm_100a) pieces the
// attention kernels use: mbarriers, TMA tile loads, bulk copies, tcgen05 MMA
// with TMEM accumulators, and the shared-memory / instruction descriptors.
//
// Descriptor bit layouts follow the public PTX ISA description of the
// tcgen05 shared-memory matrix descriptor and the kind::f16 instruction
// descriptor.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "tmem_io.cuh"

namespace rfb {

// Status codes written into the device error word (kept equal to the C-ABI codes).
constexpr int kErrAlignment = 3;
constexpr int kErrDeviceTimeout = 6;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t lane_id() { return threadIdx.x & 31u; }
__device__ __forceinline__ uint32_t warp_id() {
  return __shfl_sync(0xffffffffu, threadIdx.x >> 5, 0);
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0u;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Every wait in these kernels is bounded.  On expiry the waiter raises the
// CTA's abort flag (shared memory) and the global error word, and returns
// false; every later bounded wait in the CTA then returns false at once, so
// all roles leave their loops and reach the common exit, where TMEM is freed.
// A test hook can name one wait site (fail_site, else -1) whose first wait in
// each CTA gives up at once, as if its limit had expired, so that the abort
// path of the real kernels can be exercised without a fault.
struct WaitGuard {
  volatile int* abort_flag;   // shared memory, one per CTA
  int* err_word;              // global memory
  uint64_t timeout_ns;
  int fail_site;
};

// Limit of the exit-path waits (wait_drain): in-flight copies and MMAs always
// finish, so these keep the full limit whatever the main-loop limit is.
constexpr uint64_t kDrainTimeoutNs = 2000000000ull;

__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, const WaitGuard& g,
                                             int site) {
  if (site == g.fail_site) {
    *g.abort_flag = 1;
    atomicCAS(g.err_word, 0, kErrDeviceTimeout | (site << 8));
    return false;
  }
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t n = 1;; ++n) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((n & 63u) == 0u) {
      if (*g.abort_flag) return false;
      if (global_timer_ns() - t0 > g.timeout_ns) {
        *g.abort_flag = 1;
        atomicCAS(g.err_word, 0, kErrDeviceTimeout | (site << 8));
        return false;
      }
    }
  }
}

// Warp-uniform variant: every lane of the warp calls it; the result is true only
// if every lane saw the phase complete, so warp-collective tcgen05.ld/st that
// follow are executed by all lanes or by none.
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, const WaitGuard& g,
                                          int site) {
  const bool ok = wait_bounded(bar, parity, g, site);
  return __all_sync(0xffffffffu, ok);
}

// --------------------------------------------- programmatic dependent launch
// Every kernel of this library is launched with programmatic stream
// serialisation: it may start while the grid before it in the stream is still
// running, so each one waits here before its first global-memory access (the
// wait returns once that grid has completed and its writes are visible; at
// once when there is none).  The short persistent kernels (window forward and
// backward) then let the grid after them start launching at once, which
// overlaps that grid's launch and set-up with their own tiles (its CTAs find
// room on an SM only as this grid's CTAs exit); the long ones do so when a
// CTA's work is done.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch_next() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------ proxies
// Make generic-proxy writes to shared memory (threads writing P, dS, U') visible
// to the async proxy (tcgen05.mma operand reads).
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// -------------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "r"(c4)
      : "memory");
}
// Plain (non-tensor) bulk copy global -> shared; addresses 16-byte aligned,
// size a multiple of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Bulk tensor reduction shared -> global (element-wise add, dtype from the map),
// tracked with the bulk async-group mechanism of the issuing thread.
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* map, uint32_t src, int c0,
                                                  int c1, int c2) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.bulk_group [%0, {%2, %3, %4}], [%1];" ::
          "l"(reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
// Bulk tensor stores shared -> global (tile mode), tracked with the bulk
// async-group mechanism of the issuing thread.  Elements outside the tensor
// are not written.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int c0, int c1,
                                             int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tma_store_5d(const CUtensorMap* map, uint32_t src, int c0, int c1,
                                             int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5, %6}], [%1];" ::
          "l"(reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until every committed bulk group of this thread has finished reading
// its shared-memory source (the buffer may then be overwritten).
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until at most N committed bulk groups of this thread are still reading
// their shared-memory sources.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until every committed bulk group of this thread has completed.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// ------------------------------------------------------------ tcgen05 / TMEM
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// The MMA-issue helpers below are called by a whole, converged warp: one lane
// is elected inside the asm and issues.  (Issuing from a lone lane inside a
// divergent branch costs several times more per instruction.)

// D[tmem] (+)= A[smem] * B[smem], bf16 inputs, fp32 accumulate, one CTA.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]: A (K-major, M = 128 lanes) is read from TMEM,
// two bf16 per 32-bit column (element (m, k) in lane m, column k/2, the even k
// in the low half); B from shared memory as above.
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on an mbarrier when all previously issued tcgen05 ops of this
// thread have completed.
// (Whole warp calls; one elected lane commits.)
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          bar)
      : "memory");
}

// Shared-memory matrix descriptor swizzle codes.
enum : uint32_t { kSwNone = 0, kSw128 = 2, kSw64 = 4, kSw32 = 6 };

__host__ __device__ constexpr uint32_t swizzle_code(int row_bytes) {
  return row_bytes == 128 ? kSw128 : row_bytes == 64 ? kSw64 : row_bytes == 32 ? kSw32 : kSwNone;
}

// Descriptor: start address, leading / stride byte offsets (16-byte units),
// version 1 (bits 46-47), base offset 0, swizzle mode in bits 61-63.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                              uint32_t swz) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(swz & 7u) << 61;
  return d;
}

// K-major operand: rows of `row_bytes` (32/64/128 B, one swizzle atom wide),
// 8-row groups `8*row_bytes` apart.  K-step kk (16 bf16 = 32 B) of a tile whose
// K extent fits in one row is at byte offset 32*kk.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t saddr, int row_bytes) {
  return smem_desc(saddr, 16u, 8u * static_cast<uint32_t>(row_bytes), swizzle_code(row_bytes));
}
// MN-major operand: each K row holds `row_bytes` of contiguous MN elements,
// 8-row K groups `8*row_bytes` apart (SBO); MN blocks of one swizzle atom are
// `mn_block_bytes` apart (LBO).  K-step kk (16 rows) is at byte offset
// 16*row_bytes*kk.
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t saddr, int row_bytes,
                                                 uint32_t mn_block_bytes) {
  return smem_desc(saddr, mn_block_bytes, 8u * static_cast<uint32_t>(row_bytes),
                   swizzle_code(row_bytes));
}

// The descriptor of the operand `bytes` (a multiple of 16) further on in
// shared memory: one add to the address field, which cannot carry (shared
// memory ends below 256 KB).  Lets a kernel build each operand's descriptor
// once and step through its K-steps with constant adds.
__device__ __forceinline__ uint64_t desc_add(uint64_t desc, uint32_t bytes) {
  return desc + (bytes >> 4);
}

// kind::f16 instruction descriptor: D fp32, A and B bf16, dense.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn_major,
                                                      bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         ((b_mn_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// Byte offset of element (row, col) in a K-major bf16 tile stored as column
// blocks of 64 elements (128 B rows, 128-byte swizzle), `rows` rows per block.
__device__ __forceinline__ uint32_t sw128_offset(int row, int col, int rows) {
  const int blk = col >> 6;
  const int chunk = (col & 63) >> 3;
  return static_cast<uint32_t>(blk * rows * 128 + row * 128 + ((chunk ^ (row & 7)) << 4) +
                               ((col & 7) << 1));
}

// Byte offset of 16-byte chunk `chunk` of row `row` in a tile of rows
// `row_bytes` wide (32, 64 or 128), stored with the matching TMA swizzle
// (the tile starts on a 1024-byte boundary): the chunk index is XORed with
// address bits 7 and up.
__device__ __forceinline__ uint32_t swz_offset(int row, int chunk, int row_bytes) {
  const int line = (row * row_bytes) >> 7;  // 128-byte line of the row
  const int x = row_bytes == 128 ? (line & 7) : row_bytes == 64 ? (line & 3) : (line & 1);
  return static_cast<uint32_t>(row * row_bytes + ((chunk ^ x) << 4));
}

// -------------------------------------------------------------- numerics
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Per-warpgroup register budget changes (all four warps of a warpgroup execute
// the same one).  The budgets of all warpgroups must add up to no more than the
// registers the CTA was launched with.
template <uint32_t R>
__device__ __forceinline__ void warpgroup_reg_alloc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R));
}
template <uint32_t R>
__device__ __forceinline__ void warpgroup_reg_dealloc() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R));
}

// max(a, b, c) in one instruction (three-input max.f32 of sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Packed fp32 pairs (Blackwell f32x2 arithmetic): lo in the low 32 bits.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 f2_unpack(uint64_t v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// Software 2^x for a pair of inputs on the FMA and integer pipes (relieves the
// MUFU unit, which is the limit of the softmax).  x = n + f with n = round(x)
// obtained by adding 1.5 * 2^23 (Cody and Waite's additive range reduction,
// base 2) and f in [-1/2, 1/2]; 2^f by a degree-3 polynomial with minimum
// relative error (coefficients from gen_exp2_poly.py: max relative error
// 7.6e-5, far below bf16's 2^-9 rounding of P); 2^n added to the exponent
// field.  Inputs are clamped at -125 (results below 2^-125 are not needed by
// the softmax: they are masked or negligible).  x <= 126 is assumed.
__device__ __forceinline__ void soft_exp2_x2(float a, float b, float& ra, float& rb) {
  constexpr float kC0 = 0.9999275803565979f, kC1 = 0.6932516098022461f;
  constexpr float kC2 = 0.24261537194252014f, kC3 = 0.05522261559963226f;
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  const uint64_t x2 = f2_pack(fmaxf(a, -125.0f), fmaxf(b, -125.0f));
  const uint64_t r2 = f2_pack(kRound, kRound);
  const uint64_t t2 = f2_add(x2, r2);
  const uint64_t fr = f2_sub(x2, f2_sub(t2, r2));
  uint64_t p = f2_fma(f2_pack(kC3, kC3), fr, f2_pack(kC2, kC2));
  p = f2_fma(p, fr, f2_pack(kC1, kC1));
  p = f2_fma(p, fr, f2_pack(kC0, kC0));
  const float2 pf = f2_unpack(p), tf = f2_unpack(t2);
  // t's low mantissa bits hold n (two's complement); shifting them into the
  // exponent field adds n to p's exponent.
  ra = __uint_as_float(__float_as_uint(pf.x) + (__float_as_uint(tf.x) << 23));
  rb = __uint_as_float(__float_as_uint(pf.y) + (__float_as_uint(tf.y) << 23));
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ void red_add_v4(float* gaddr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(gaddr), "f"(a), "f"(b),
               "f"(c), "f"(d)
               : "memory");
}

// Named barrier among `nthreads` threads (ids 1..15; 0 is __syncthreads).
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Scale every bf16 element of a shared-memory tile in place by `f` (one warp,
// `bytes` a multiple of 512).  The element layout does not matter.
__device__ __forceinline__ void scale_tile_bf16(uint32_t base, uint32_t bytes, float f) {
  for (uint32_t off = lane_id() * 16u; off < bytes; off += 512u) {
    uint4 v = ld_shared_v4(base + off);
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float lo = __uint_as_float(w[i] << 16) * f;
      const float hi = __uint_as_float(w[i] & 0xFFFF0000u) * f;
      w[i] = pack_bf16x2(lo, hi);
    }
    st_shared_v4(base + off, w[0], w[1], w[2], w[3]);
  }
}

}  // namespace rfb
