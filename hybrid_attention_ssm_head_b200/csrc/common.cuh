// Device helpers shared by the sm_100a kernels: bf16 conversion, mbarrier,
// TMA (cp.async.bulk.tensor, no multicast), tcgen05 (TMEM alloc, MMA, commit,
// loads/stores) and bounded waits that report an error word instead of hanging.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hymba.h"

namespace hymba {

// ---------------------------------------------------------------------------
// Error word.  Every translation unit has its own; the host folds them into
// hymba_stream_status().  Codes: 1 = bounded wait timed out.
// ---------------------------------------------------------------------------
#define HYMBA_DEVICE_ERROR_WORD(name) static __device__ unsigned int name = 0u

constexpr unsigned kErrTimeout = 1u;
// Every mbarrier wait gives up after a limit in SM clock cycles that the launching host
// code passes to the kernel (wait_limit_cycles(): 1e9 cycles, about 0.5 s at 2 GHz, unless
// set otherwise).  Legitimate waits in these kernels last microseconds.

// ---------------------------------------------------------------------------
// Small math helpers
// ---------------------------------------------------------------------------
template <typename T> struct Store;
template <> struct Store<float> {
  static __device__ __forceinline__ float to_f(float v) { return v; }
  static __device__ __forceinline__ float from_f(float v) { return v; }
};
template <> struct Store<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 v) {
    return __uint_as_float(uint32_t(*reinterpret_cast<const unsigned short *>(&v)) << 16);
  }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

// The MUFU approximations with subnormal inputs and results flushed to zero: one
// instruction each (the non-flushing forms add range fix-ups around the MUFU).
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2_ftz(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_ftz(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// x * sigmoid(x) = x / (1 + 2^(-x log2 e)); 0 for x -> -inf (the reciprocal of +inf).
__device__ __forceinline__ float silu_f(float x) { return x * rcp_ftz(1.0f + ex2_ftz(-kLog2e * x)); }
// bf16 -> fp32 is a 16-bit shift of the bits (exact): an integer-pipe operation.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
// Two fp32 fused multiply-adds in one instruction (d = a * b + c, elementwise).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(d)
      : "l"(*reinterpret_cast<uint64_t *>(&a)), "l"(*reinterpret_cast<uint64_t *>(&b)),
        "l"(*reinterpret_cast<uint64_t *>(&c)));
  return *reinterpret_cast<float2 *>(&d);
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;"
      : "=l"(d)
      : "l"(*reinterpret_cast<uint64_t *>(&a)), "l"(*reinterpret_cast<uint64_t *>(&b)));
  return *reinterpret_cast<float2 *>(&d);
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;"
      : "=l"(d)
      : "l"(*reinterpret_cast<uint64_t *>(&a)), "l"(*reinterpret_cast<uint64_t *>(&b)));
  return *reinterpret_cast<float2 *>(&d);
}
__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;"
      : "=l"(d)
      : "l"(*reinterpret_cast<uint64_t *>(&a)), "l"(*reinterpret_cast<uint64_t *>(&b)));
  return *reinterpret_cast<float2 *>(&d);
}
// max of three in one instruction
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// 2^x on the FMA pipe, two lanes per instruction (Cody-Waite style reduction):
// j = rint(x) through the 1.5 * 2^23 rounding constant, f = x - j in [-1/2, 1/2],
// 2^f by a polynomial of degree DEG, j added into the exponent field.  The
// coefficients are relative-error minimax fits of 2^f on [-1/2, 1/2] made for this
// library (fp32 Horner evaluation: max relative error 7.5e-5 at degree 3, 2.4e-7 at
// degree 5, the size of the MUFU's own error).  x is clamped below at -125 so the
// exponent stays in range (the result is then 2^-125 instead of smaller); no upper
// clamp, valid for x < 128.
template <int DEG>
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  static_assert(DEG == 3 || DEG == 5, "fitted degrees");
  x.x = fmaxf(x.x, -125.f);
  x.y = fmaxf(x.y, -125.f);
  const float2 rnd = make_float2(12582912.f, 12582912.f);
  const float2 t = fadd2(x, rnd);
  const float2 f = fsub2(x, fsub2(t, rnd));
  float2 p;
  if constexpr (DEG == 5) {
    p = ffma2(make_float2(1.3276470e-3f, 1.3276470e-3f), f, make_float2(9.6755419e-3f, 9.6755419e-3f));
    p = ffma2(p, f, make_float2(5.5507135e-2f, 5.5507135e-2f));
    p = ffma2(p, f, make_float2(2.4022120e-1f, 2.4022120e-1f));
    p = ffma2(p, f, make_float2(6.9314694e-1f, 6.9314694e-1f));
    p = ffma2(p, f, make_float2(1.0000001f, 1.0000001f));
  } else {
    p = ffma2(make_float2(5.5171657e-2f, 5.5171657e-2f), f, make_float2(2.4261114e-1f, 2.4261114e-1f));
    p = ffma2(p, f, make_float2(6.9326097e-1f, 6.9326097e-1f));
    p = ffma2(p, f, make_float2(9.9992806e-1f, 9.9992806e-1f));
  }
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}
// log(1 + e^x) with the fast exp/log: x above 20 returns x; below -8 returns e^x
// (relative error e^x / 2 < 2e-4); in between log(1 + e^x) with 1 + e^x >= 1 + 3e-4,
// so the fp32 rounding of the sum costs at most ~2e-4 relative.
__device__ __forceinline__ float softplus_f(float x) {
  const float e = ex2_ftz(kLog2e * fminf(x, 20.0f));
  const float l = kLn2 * lg2_ftz(1.0f + e);
  return x > 20.0f ? x : (x < -8.0f ? e : l);  // selects, no divergence
}
// Full-precision variant for the fp32 storage path.
__device__ __forceinline__ float softplus_accurate(float x) {
  return x > 20.0f ? x : log1pf(expf(x));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// ---------------------------------------------------------------------------
// Attention mask predicate (A-shape: meta prefix + sliding window, or causal).
// One definition, used by the attention kernels and by the bitmap dump.
// ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ bool mask_allowed(long long i, long long j, int n_meta,
                                                      int window, int is_global) {
  if (j > i) return false;
  if (is_global) return true;
  return j < n_meta || (i - j) < window;
}
// 0 = no visible pair, 1 = all pairs visible, 2 = mixed, for rows [i0,i1] x cols [j0,j1].
__host__ __device__ __forceinline__ int mask_tile_class(long long i0, long long i1, long long j0,
                                                        long long j1, int n_meta, int window,
                                                        int is_global) {
  if (j0 > i1) return 0;
  if (!is_global && j0 >= n_meta && (i0 - j1) >= window) return 0;
  bool causal_full = j1 <= i0;
  bool win_full = is_global || j1 < n_meta || (i1 - j0) < window;
  return (causal_full && win_full) ? 1 : 2;
}

// Class of 128-row query tile qt (query positions q_off + 128 qt ...) against 128-key
// tile kt of a sequence of L positions: rows past the sequence are ignored (their
// outputs are never stored); keys past it are not (they are zero-filled by TMA and must
// stay masked).
__host__ __device__ __forceinline__ int seq_tile_class(int qt, int kt, int L, int q_off, int n_meta,
                                                       int window, int is_global) {
  const long long i0 = (long long)q_off + (long long)qt * 128;
  if (i0 >= L) return 0;
  const long long i1 = (i0 + 127 < L - 1) ? i0 + 127 : L - 1;
  const long long j0 = (long long)kt * 128, j1 = j0 + 127;
  return mask_tile_class(i0, i1, j0, j1, n_meta, window, is_global);
}

// ---------------------------------------------------------------------------
// Shared-memory addresses, mbarriers, fences
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte asynchronous global -> shared copies (LDGSTS), committed and waited by group.
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
// try_wait with a suspend-time hint: a waiting thread sleeps until the phase
// completes (or the hint expires) instead of spinning, so waiting warps do not take
// issue slots from the warps computing beside them.
constexpr uint32_t kSuspendHintNs = 1000000u;
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "n"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}
// Waits for the phase with the given parity to complete.  Gives up after `limit`
// cycles, records kErrTimeout in *err and returns false.
// Also gives up at once when another CTA has already recorded a timeout, so a
// broken pipeline ends after one limit instead of one limit per wave of CTAs.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, unsigned int *err,
                                          long long limit) {
  if (mbar_try_wait(bar, parity)) return true;
  long long t0 = clock64();
  unsigned spins = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((++spins & 3u) == 0 && *reinterpret_cast<volatile unsigned *>(err) != 0u) return false;
    if (clock64() - t0 > limit) {
      atomicOr(err, kErrTimeout);
      return false;
    }
  }
}

// Drain wait for the abort path: waits (bounded) for copies or MMAs already
// issued by this CTA, even when another CTA has recorded an error.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t *bar, uint32_t parity, unsigned int *err,
                                                long long limit) {
  long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > limit) {
      atomicOr(err, kErrTimeout);
      return false;
    }
  }
  return true;
}

// ---------------------------------------------------------------------------
// TMA (tiled tensor copies global -> shared, completion on an mbarrier).
// No cluster multicast anywhere in this library.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}
// Shared -> global tile store by TMA (bulk async group); rows or columns past the
// tensor's extent are not written.  The coordinates must not be negative.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map, const void *src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// the issuing thread's bulk stores have finished reading shared memory
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// ... and their global writes are complete
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
// Hint: bring one tile of a 2-D tensor map into L2 (no shared memory, no completion).
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap *map, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y)
               : "memory");
}
// ---------------------------------------------------------------------------
// Programmatic dependent launch.  A kernel launched with the programmatic-serialisation
// attribute may begin while the kernel before it in the stream is still running.
// pdl_wait() returns once the preceding grids have completed and their writes are visible
// (at once for a normal launch).  Every CTA of such a kernel calls pdl_wait() before
// pdl_trigger(), which lets the next kernel start its own prologue, so when a kernel starts,
// every kernel but its direct predecessors has completed.  Before pdl_wait() a kernel
// therefore reads only weights, its own shared memory and barriers, and data that no
// direct predecessor writes (a decode kernel's own state from the previous step); it
// writes global memory only after pdl_wait().
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------------------
// tcgen05: tensor memory and the 5th-generation MMA (cta_group::1)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
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
// D(tmem) (+)= A(smem desc) * B(smem desc)^T, kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// bf16 MMA with the A operand in tensor memory (M = 128 lanes, K = 16 per instruction:
// eight 32-bit columns, each holding two consecutive bf16 of a row) and B in shared memory.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Same with kind::tf32 (fp32 operands in shared memory, tf32 multiply, fp32 accumulate).
__device__ __forceinline__ void mma_tf32_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` once every previously issued tcgen05.mma of this thread completed.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Instruction descriptor, kind::f16 / kind::tf32: fp32 accumulator, M = 128.
// Bits: [4,6) D format (1 = f32), [7,10) A format, [10,13) B format
// (kind::f16: 1 = bf16; kind::tf32: 2 = tf32), bit 15 A major, bit 16 B major
// (0 = K-major, 1 = MN-major), [17,23) N >> 3, [24,29) M >> 4.
__host__ __device__ constexpr uint32_t make_idesc(int n, int ab_format, int a_mn_major,
                                                  int b_mn_major) {
  return (1u << 4) | (uint32_t(ab_format) << 7) | (uint32_t(ab_format) << 10) |
         (uint32_t(a_mn_major) << 15) | (uint32_t(b_mn_major) << 16) |
         (uint32_t(n >> 3) << 17) | (uint32_t(128 >> 4) << 24);
}

// Shared-memory matrix descriptor for a 128-byte-swizzled tile (the layout TMA
// writes with CU_TENSOR_MAP_SWIZZLE_128B).  Fields: [0,14) start >> 4,
// [16,30) leading byte offset >> 4, [32,46) stride byte offset >> 4,
// [46,48) version 1, [61,64) layout 2 = 128B swizzle.
//  K-major operand: rows of 128 B, 8-row groups 1024 B apart -> lbo unused (1), sbo 1024.
//  MN-major operand: 64-element (128 B) atoms along MN lbo apart; 8-row K groups sbo apart.
__device__ __forceinline__ uint64_t make_sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= uint64_t((saddr >> 4) & 0x3FFFu);
  d |= uint64_t((lbo >> 4) & 0x3FFFu) << 16;
  d |= uint64_t((sbo >> 4) & 0x3FFFu) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(2) << 61;
  return d;
}

// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp receives lane
// (warp%4)*32 + t, columns [col, col+32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Thread-block clusters: rank, cluster-wide barrier, distributed shared memory
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Every thread of every CTA of the cluster arrives (release) and waits (acquire).
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// The shared::cluster address of this CTA's shared-memory address saddr in CTA `rank`.
__device__ __forceinline__ uint32_t map_shared_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ float ld_shared_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ float4 ld_shared_cluster_v4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ int warp_id() { return threadIdx.x >> 5; }
__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }
__device__ __forceinline__ bool elect_lane0() { return (threadIdx.x & 31) == 0; }

// 16-byte vector store of 8 bf16 (generic address).
__device__ __forceinline__ void st_global_v4(void *p, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}
// 32 bytes (one whole sector) per thread: the address must be 32-byte aligned
__device__ __forceinline__ void st_global_v8(void *p, uint32_t a, uint32_t b, uint32_t c, uint32_t d,
                                             uint32_t e, uint32_t f, uint32_t g, uint32_t h) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a), "r"(b),
               "r"(c), "r"(d), "r"(e), "r"(f), "r"(g), "r"(h)
               : "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

}  // namespace hymba
