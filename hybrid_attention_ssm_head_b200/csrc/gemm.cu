// Dense projections of the hybrid-head layer (W_in_proj, x_proj, dt_proj, W_out_proj):
//   out[m, n] = epilogue( sum_k A[m, k] * B[n, k] )
//
// Tensor-core path: persistent, warp-specialised tcgen05 kernel.
//   warp 0   : TMA producer (one lane) filling a ring of STAGES shared-memory
//              stages, each a 128 x 128-byte A tile and a BN x 128-byte B tile,
//              both 128-byte swizzled (K-major).
//   warp 1   : TMEM allocator and MMA issuer (one lane): per 128-byte K block,
//              4 x tcgen05.mma (M=128, N=BN, K=32 bytes) into one of two fp32
//              accumulators in tensor memory, then tcgen05.commit frees the stage.
//   warps 2-17: epilogue, one thread per accumulator row (four warps per TMEM
//              lane quarter, every fourth 16-column chunk): tcgen05.ld, bias /
//              softplus, per-segment SiLU and rotary embedding, fp32 -> bf16, routed
//              stores (one GEMM writes Q, K, V, x_ssm and the gate SiLU(z) to their own
//              buffers).  The second accumulator lets the epilogue of tile i overlap
//              the MMAs of tile i+1.
// Tiles are visited N-fastest so the CTAs in flight share A rows in L2.
// Decode-sized products (<= 256 rows) use the weight-streaming kernel further down.
// fp32 path: a plain CUDA-core tiled kernel with the same epilogue.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tmap.h"

namespace hymba {

HYMBA_DEVICE_ERROR_WORD(g_err_gemm);

// ---------------------------------------------------------------------------
// Epilogue stores
// ---------------------------------------------------------------------------
__device__ __forceinline__ int find_seg(const Epilogue &e, int n) {
  int s = 0;
#pragma unroll 1
  while (s + 1 < e.nseg && n >= e.seg[s].col1) ++s;
  return s;
}

// Column `local` of a segment -> (group, offset in group) without a division on the
// common layouts: one group, or a power-of-two group width.
// Destination row of product row m for the segments with a row remap.
__device__ __forceinline__ long long remap_row(const Epilogue &e, long long m) {
  if (e.rmap_rows <= 0) return m;
  const unsigned q = (unsigned)m / (unsigned)e.rmap_rows, r = (unsigned)m - q * (unsigned)e.rmap_rows;
  return (long long)q * e.rmap_stride + r + e.rmap_off;
}

__device__ __forceinline__ long long seg_offset(const EpiSeg &g, long long m, int local) {
  int grp, lin;
  if (g.inner >= g.col1 - g.col0) {
    grp = 0;
    lin = local;
  } else if ((g.inner & (g.inner - 1)) == 0) {
    const int sh = __ffs(g.inner) - 1;
    grp = local >> sh;
    lin = local & (g.inner - 1);
  } else {
    grp = local / g.inner;
    lin = local - grp * g.inner;
  }
  return m * g.ld_row + (long long)grp * g.ld_group + lin;
}

// Bias and activation of the fp32 CUDA-core path (full-precision softplus).
__device__ __forceinline__ float epi_act(const Epilogue &e, int n, float v) {
  if (e.bias) v += __ldg(e.bias + n);
  if (e.act == 1) v = softplus_accurate(v);
  return v;
}

// Position of product row m for the rotary embedding.
__device__ __forceinline__ int rope_pos(const Epilogue &e, long long m) {
  if (!e.rope_tab) return 0;
  return (int)((unsigned)m % (unsigned)e.rope_rows) + e.rope_off;
}
// Rotates the column pairs of v[0..2*NP) (columns n, n+1, ... of segment g, n even) by the
// rotary angles of position pos.
template <int NP>
__device__ __forceinline__ void rope_rotate(const Epilogue &e, const EpiSeg &g, int n, int pos, float *v) {
  const int hp = e.rope_hd >> 1;
  const int pair0 = ((n - g.col0) & (e.rope_hd - 1)) >> 1;
  const float2 *cs = e.rope_tab + (long long)pos * hp + pair0;
#pragma unroll
  for (int i = 0; i < NP; ++i) {
    const float2 c = __ldg(cs + i);
    const float a = v[2 * i], b = v[2 * i + 1];
    v[2 * i] = a * c.x - b * c.y;
    v[2 * i + 1] = fmaf(a, c.y, b * c.x);
  }
}

// The segment's own activation.
__device__ __forceinline__ float seg_act(const EpiSeg &g, float v) { return g.act == 2 ? silu_f(v) : v; }

// Residual of column `local` of segment g at product row m.
__device__ __forceinline__ float resid_at(const EpiSeg &g, long long m, int local) {
  const long long o = m * g.ld_resid + local;
  if (g.f32) return __ldg(reinterpret_cast<const float *>(g.resid) + o);
  return bf16_lo((uint32_t)__ldg(reinterpret_cast<const unsigned short *>(g.resid) + o));
}
// Residual of 8 consecutive columns (16-byte aligned, bf16 or fp32).
__device__ __forceinline__ void resid8(const EpiSeg &g, long long m, int local, float (&r)[8]) {
  const long long o = m * g.ld_resid + local;
  if (g.f32) {
    const float4 *p = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(g.resid) + o);
    const float4 a = __ldg(p), b = __ldg(p + 1);
    r[0] = a.x; r[1] = a.y; r[2] = a.z; r[3] = a.w; r[4] = b.x; r[5] = b.y; r[6] = b.z; r[7] = b.w;
  } else {
    const uint4 w = __ldg(reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(g.resid) + o));
    const uint32_t q[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      r[2 * i] = bf16_lo(q[i]);
      r[2 * i + 1] = bf16_hi(q[i]);
    }
  }
}

// m: the product row; mk: its remapped row (used by segments with rmap).
template <int EPI>
__device__ __forceinline__ void epi_store_scalar(const Epilogue &e, long long m, long long mk, int n,
                                                 float v) {
  const EpiSeg &g = e.seg[find_seg(e, n)];
  const long long off = seg_offset(g, g.rmap ? mk : m, n - g.col0);
  v = seg_act(g, v);
  if constexpr ((EPI & kEpiResid) != 0) {
    if (g.resid) v += resid_at(g, m, n - g.col0);
  }
  if (g.f32) {
    reinterpret_cast<float *>(g.ptr)[off] = v;
  } else {
    reinterpret_cast<__nv_bfloat16 *>(g.ptr)[off] = __float2bfloat16_rn(v);
  }
}

// Stores 8 consecutive columns n..n+7 of row m (values already activated).
// EPI (kEpi* flags): the features this instantiation carries; the plain one (one segment,
// no routing) keeps fewer registers live.  The 8-column path takes what the 16-column
// fast path cannot (segment edges, unaligned destinations); it does no gated SiLU (the
// host keeps such segments on whole 16-column chunks).
template <int EPI>
__device__ __forceinline__ void epi_store8(const Epilogue &e, long long m, long long mk, int rp, int n,
                                           int N, const float (&v_raw)[8]) {
  if (n >= N) return;
  const EpiSeg &g = e.seg[find_seg(e, n)];
  float v_in[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) v_in[i] = v_raw[i];
  if constexpr ((EPI & kEpiRoute) != 0) {
    if (g.rope && n + 8 <= g.col1) rope_rotate<4>(e, g, n, rp, v_in);
  }
  int local = n - g.col0;
  bool vec = g.vec_ok && (n + 8 <= N) && (n + 8 <= g.col1) && (local % 8 == 0) &&
             ((local % g.inner) + 8 <= g.inner);
  if (vec) {
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = seg_act(g, v_in[i]);
    if constexpr ((EPI & kEpiResid) != 0) {
      if (g.resid) {
        float rr[8];
        resid8(g, m, local, rr);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] += rr[i];
      }
    }
    const long long off = seg_offset(g, g.rmap ? mk : m, local);
    if (g.f32) {
      float *p = reinterpret_cast<float *>(g.ptr) + off;
      st_global_v4(p, __float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]),
                   __float_as_uint(v[3]));
      st_global_v4(p + 4, __float_as_uint(v[4]), __float_as_uint(v[5]), __float_as_uint(v[6]),
                   __float_as_uint(v[7]));
    } else {
      __nv_bfloat16 *p = reinterpret_cast<__nv_bfloat16 *>(g.ptr) + off;
      st_global_v4(p, pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                   pack_bf16x2(v[6], v[7]));
    }
    return;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (n + i < N) epi_store_scalar<EPI>(e, m, mk, n + i, v_in[i]);
}

// Bias of columns n0..n0+15 (zero past N).
__device__ __forceinline__ void epi_bias16(const Epilogue &e, int n0, int N, float (&b)[16]) {
  if (n0 + 16 <= N) {
    const float4 *bp = reinterpret_cast<const float4 *>(e.bias + n0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 b4 = __ldg(bp + q);
      b[4 * q] = b4.x;
      b[4 * q + 1] = b4.y;
      b[4 * q + 2] = b4.z;
      b[4 * q + 3] = b4.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) b[i] = n0 + i < N ? __ldg(e.bias + n0 + i) : 0.f;
  }
}

// 16 consecutive product columns n0..n0+15 of row m from raw fp32 accumulator bits,
// plus the bias (when the epilogue has one).  One segment lookup per chunk on the
// common path.
template <int EPI>
__device__ __forceinline__ void epi_store16(const Epilogue &e, long long m, long long mk, int rp, int n0,
                                            int N, const uint32_t (&r)[16], const float (&bias)[16]) {
  if constexpr ((EPI & kEpiSoftplus) != 0) {
    // dt_proj: one plain segment, bias and softplus of every column (checked on the host)
    const EpiSeg &g = e.seg[0];
    if (n0 + 16 <= N && g.vec_ok && !g.f32) {
      float o[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) o[i] = softplus_f(__uint_as_float(r[i]) + bias[i]);
      __nv_bfloat16 *p = reinterpret_cast<__nv_bfloat16 *>(g.ptr) + m * g.ld_row + (n0 - g.col0);
      if (g.vec32) {
        st_global_v8(p, pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                     pack_bf16x2(o[6], o[7]), pack_bf16x2(o[8], o[9]), pack_bf16x2(o[10], o[11]),
                     pack_bf16x2(o[12], o[13]), pack_bf16x2(o[14], o[15]));
      } else {
        st_global_v4(p, pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                     pack_bf16x2(o[6], o[7]));
        st_global_v4(p + 8, pack_bf16x2(o[8], o[9]), pack_bf16x2(o[10], o[11]), pack_bf16x2(o[12], o[13]),
                     pack_bf16x2(o[14], o[15]));
      }
      return;
    }
  }
  float v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
  const bool full = n0 + 16 <= N;
  if (e.bias) {
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] += bias[i];
  }
  if (e.act == 1) {
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = softplus_f(v[i]);
  }
  // common case: the 16 columns lie in one segment and one group, 16-byte aligned rows
  const int sidx = find_seg(e, n0);
  const EpiSeg &g = e.seg[sidx];
  const int local = n0 - g.col0;
  if (full && g.vec_ok && n0 + 16 <= g.col1 &&
      (g.inner >= g.col1 - g.col0 || ((g.inner & 15) == 0 && (local & 15) == 0))) {
    if constexpr ((EPI & kEpiGlu) != 0) {
      if (g.act == 3) {
        // gated SiLU: product columns (2i, 2i+1) -> output column local/2 + i
        float o[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = silu_f(v[2 * i]) * v[2 * i + 1];
        const long long off = m * g.ld_row + (local >> 1);
        if (g.f32) {
          float *p = reinterpret_cast<float *>(g.ptr) + off;
          st_global_v4(p, __float_as_uint(o[0]), __float_as_uint(o[1]), __float_as_uint(o[2]), __float_as_uint(o[3]));
          st_global_v4(p + 4, __float_as_uint(o[4]), __float_as_uint(o[5]), __float_as_uint(o[6]),
                       __float_as_uint(o[7]));
        } else {
          st_global_v4(reinterpret_cast<__nv_bfloat16 *>(g.ptr) + off, pack_bf16x2(o[0], o[1]),
                       pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
        }
        return;
      }
    }
    if (g.act) {
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = seg_act(g, v[i]);
    }
    if constexpr ((EPI & kEpiRoute) != 0) {
      if (g.rope) rope_rotate<8>(e, g, n0, rp, v);
    }
    if constexpr ((EPI & kEpiResid) != 0) {
      if (g.resid) {
        float rr[8];
        resid8(g, m, local, rr);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] += rr[i];
        resid8(g, m, local + 8, rr);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[8 + i] += rr[i];
      }
    }
    const long long off = seg_offset(g, ((EPI & kEpiRoute) && g.rmap) ? mk : m, local);
    if (g.f32) {
      float *p = reinterpret_cast<float *>(g.ptr) + off;
      if (g.vec32) {
#pragma unroll
        for (int q = 0; q < 2; ++q)
          st_global_v8(p + 8 * q, __float_as_uint(v[8 * q]), __float_as_uint(v[8 * q + 1]),
                       __float_as_uint(v[8 * q + 2]), __float_as_uint(v[8 * q + 3]),
                       __float_as_uint(v[8 * q + 4]), __float_as_uint(v[8 * q + 5]),
                       __float_as_uint(v[8 * q + 6]), __float_as_uint(v[8 * q + 7]));
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          st_global_v4(p + 4 * q, __float_as_uint(v[4 * q]), __float_as_uint(v[4 * q + 1]),
                       __float_as_uint(v[4 * q + 2]), __float_as_uint(v[4 * q + 3]));
      }
    } else {
      __nv_bfloat16 *p = reinterpret_cast<__nv_bfloat16 *>(g.ptr) + off;
      if (g.vec32) {
        st_global_v8(p, pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                     pack_bf16x2(v[6], v[7]), pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]),
                     pack_bf16x2(v[12], v[13]), pack_bf16x2(v[14], v[15]));
      } else {
        st_global_v4(p, pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                     pack_bf16x2(v[6], v[7]));
        st_global_v4(p + 8, pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]),
                     pack_bf16x2(v[12], v[13]), pack_bf16x2(v[14], v[15]));
      }
    }
    return;
  }
  float a[8], b[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    a[i] = v[i];
    b[i] = v[8 + i];
  }
  epi_store8<EPI>(e, m, mk, rp, n0, N, a);
  epi_store8<EPI>(e, m, mk, rp, n0 + 8, N, b);
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05 GEMM
// ---------------------------------------------------------------------------
template <int BN, int ELEM>
struct TcCfg {
  static constexpr int BM = 128;
  static constexpr int BK = 128 / ELEM;  // elements in one 128-byte swizzle row
  static constexpr int A_BYTES = BM * 128;
  static constexpr int B_BYTES = BN * 128;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (196 * 1024) / STAGE_BYTES > 8 ? 8 : (196 * 1024) / STAGE_BYTES;
  static constexpr int TMEM_COLS = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128
                                   : (2 * BN <= 256) ? 256 : 512;
  static constexpr uint32_t IDESC = make_idesc(BN, ELEM == 2 ? 1 : 2, 0, 0);
  static constexpr int SCHED = 8;  // tile ids in flight from the producer to the MMA and epilogue warps
  static constexpr int BAR_BYTES = (2 * STAGES + 5 + 2 * SCHED) * 8 + SCHED * 4 + 16;  // + static smem: Epilogue
  static constexpr int SMEM = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "tcgen05 M=128 needs N % 16 == 0, N <= 256");
};

// Tile order: with a work counter (tile_ctr), the producer takes the next tile with an
// atomic add and hands its id to the MMA warp and the epilogue warps through a ring of
// SCHED slots in shared memory (so a CTA that starts late, e.g. behind other kernels'
// CTAs on its SM, takes fewer tiles); without one, CTA b takes tiles b, b + grid, ...
template <int BN, int ELEM, int EPI>
__global__ void __launch_bounds__(576, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   int M, int N, int K, Epilogue epi, long long wlim, int stall, unsigned *tile_ctr) {
  pdl_wait();
  pdl_trigger();
  using C = TcCfg<BN, ELEM>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t *sA = smem;
  uint8_t *sB = smem + C::STAGES * C::A_BYTES;
  uint64_t *full = reinterpret_cast<uint64_t *>(sB + C::STAGES * C::B_BYTES);
  uint64_t *empty = full + C::STAGES;
  uint64_t *tfull = empty + C::STAGES;
  uint64_t *tempty = tfull + 2;
  uint64_t *never = tempty + 2;  // nothing arrives on it: the wait of a stalled MMA warp
  uint64_t *sfull = never + 1;       // [SCHED] a tile id is in the slot
  uint64_t *sempty = sfull + C::SCHED;  // [SCHED] the MMA warp and the 16 epilogue warps have read it
  int *stile = reinterpret_cast<int *>(sempty + C::SCHED);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(stile + C::SCHED);
  const bool dyn = tile_ctr != nullptr;
  // Segment table in shared memory: per-column routing then indexes smem, not
  // kernel parameters.
  __shared__ Epilogue s_epi;
  if (threadIdx.x == 0) s_epi = epi;

  const int warp = warp_id();
  const int lane = lane_id();
  const int m_tiles = (M + C::BM - 1) / C::BM;
  const int n_tiles = (N + BN - 1) / BN;
  const int kblocks = (K + C::BK - 1) / C::BK;
  const long long units = (long long)m_tiles * n_tiles;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 512);
    }
    mbar_init(never, 1);
    for (int i = 0; i < C::SCHED; ++i) {
      mbar_init(&sfull[i], 1);
      mbar_init(&sempty[i], 17);
    }
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      bool ok = true;
      int si = 0;
      uint32_t sph = 0;
      for (long long u = dyn ? (long long)atomicAdd(tile_ctr, 1u) : blockIdx.x; ok;
           u = dyn ? (long long)atomicAdd(tile_ctr, 1u) : u + gridDim.x) {
        if (dyn) {  // publish the tile id (or the end) to the MMA and epilogue warps
          if (!mbar_wait(&sempty[si], sph ^ 1u, &g_err_gemm, wlim)) {
            ok = false;
            break;
          }
          stile[si] = u < units ? (int)u : -1;
          mbar_arrive(&sfull[si]);
          if (++si == C::SCHED) {
            si = 0;
            sph ^= 1u;
          }
        }
        if (u >= units) break;
        const int mt = int(u / n_tiles), nt = int(u % n_tiles);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, &g_err_gemm, wlim)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          tma_load_2d(sA + stage * C::A_BYTES, &tmA, &full[stage], kb * C::BK, mt * C::BM);
          tma_load_2d(sB + stage * C::B_BYTES, &tmB, &full[stage], kb * C::BK, nt * BN);
          ++issued[stage];
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // Leave no copy in flight into shared memory that is about to be released.
        for (int s = 0; s < C::STAGES; ++s)
          if (issued[s]) mbar_wait_drain(&full[s], (issued[s] - 1) & 1u, &g_err_gemm, wlim);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      // A stalled launch (the bounded-wait test) waits for an arrival that never comes
      // instead of issuing its first MMA; it then takes the abort path below.
      bool ok = !stall || mbar_wait(never, 0, &g_err_gemm, wlim);
      int si = 0;
      uint32_t sph = 0;
      for (long long u = blockIdx.x; ok; u += gridDim.x) {
        if (dyn) {
          if (!mbar_wait(&sfull[si], sph, &g_err_gemm, wlim)) {
            ok = false;
            break;
          }
          u = stile[si];
          mbar_arrive(&sempty[si]);
          if (++si == C::SCHED) {
            si = 0;
            sph ^= 1u;
          }
          if (u < 0) break;
        }
        if (u >= units) break;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, &g_err_gemm, wlim)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + uint32_t(acc * BN);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, &g_err_gemm, wlim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t ad = make_sdesc(a_addr + k * 32, 16, 1024);
            const uint64_t bd = make_sdesc(b_addr + k * 32, 16, 1024);
            if (ELEM == 2)
              mma_bf16_ss(d_tmem, ad, bd, C::IDESC, (kb > 0 || k > 0) ? 1u : 0u);
            else
              mma_tf32_ss(d_tmem, ad, bd, C::IDESC, (kb > 0 || k > 0) ? 1u : 0u);
          }
          mma_commit(&empty[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&tfull[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok) {
        // Drain issued MMAs before tensor memory is released.
        mma_commit(&tfull[acc]);
        mbar_wait_drain(&tfull[acc], acc_phase, &g_err_gemm, wlim);
      }
    }
  } else {
    // ---------------- epilogue: warps 2..9, one thread per accumulator row ----------------
    // Warps w, w+4, w+8, w+12 share a TMEM lane quarter and take every fourth
    // 16-column chunk.
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int sub = (warp - 2) >> 2;
    const int row = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    int si = 0;
    uint32_t sph = 0;
    for (long long u = blockIdx.x;; u += gridDim.x) {
      if (dyn) {
        if (!mbar_wait(&sfull[si], sph, &g_err_gemm, wlim)) break;
        u = stile[si];
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[si]);
        if (++si == C::SCHED) {
          si = 0;
          sph ^= 1u;
        }
        if (u < 0) break;
      }
      if (u >= units) break;
      const int mt = int(u / n_tiles), nt = int(u % n_tiles);
      constexpr int NCH = (BN + 63) / 64;
      if (!mbar_wait(&tfull[acc], acc_phase, &g_err_gemm, wlim)) break;
      tc_fence_after();
      const long long m = (long long)mt * C::BM + row;
      const long long mk = (EPI & kEpiRoute) ? remap_row(s_epi, m) : m;
      const int rp = (EPI & kEpiRoute) ? rope_pos(s_epi, m) : 0;
      const uint32_t t_row = tmem_base + (uint32_t(quarter * 32) << 16) + uint32_t(acc * BN);
      // this warp's chunks in rounds of at most two loads; the accumulator is handed back
      // to the MMA warp after the last round's loads, before its activation math and stores
      constexpr int BATCH = NCH > 2 ? 2 : NCH;
#pragma unroll
      for (int k0 = 0; k0 < NCH; k0 += BATCH) {
        uint32_t r[BATCH][16];
#pragma unroll
        for (int k = 0; k < BATCH; ++k) {
          const int c = sub * 16 + 64 * (k0 + k);
          if (k0 + k < NCH && c < BN) tmem_ld16(t_row + c, r[k]);  // uniform per warp
        }
        // the softplus epilogue's bias: its loads overlap the tensor-memory loads
        float pbias[(EPI & kEpiSoftplus) ? BATCH : 1][16];
        if constexpr ((EPI & kEpiSoftplus) != 0) {
#pragma unroll
          for (int k = 0; k < BATCH; ++k) {
            const int n0 = nt * BN + sub * 16 + 64 * (k0 + k);
            if (k0 + k < NCH && n0 < N) epi_bias16(s_epi, n0, N, pbias[k]);
          }
        }
        tmem_wait_ld();
        if (k0 + BATCH >= NCH) {
          tc_fence_before();
          mbar_arrive(&tempty[acc]);
        }
#pragma unroll
        for (int k = 0; k < BATCH; ++k) {
          const int c = sub * 16 + 64 * (k0 + k);
          const int n0 = nt * BN + c;
          if (k0 + k < NCH && c < BN && n0 < N && m < M) {
            if constexpr ((EPI & kEpiSoftplus) != 0) {
              epi_store16<EPI>(s_epi, m, mk, rp, n0, N, r[k], pbias[k]);
            } else {
              float bias[16];
              if (s_epi.bias) epi_bias16(s_epi, n0, N, bias);
              epi_store16<EPI>(s_epi, m, mk, rp, n0, N, r[k], bias);
            }
          }
        }
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// SM count of the current device (queried per launch: devices may differ between calls)
static int num_sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// ---------------------------------------------------------------------------
// Weight-streaming GEMM for a few activation rows (the decode step):
//   out[b, n] = epi( sum_k X[b, k] W[n, k] ),   b < B <= 256 (one tile of rows)
// computed transposed on the tensor cores, D[n, b] = W[n, :] . X[b, :], with the weights
// as the M = 128 operand: a cluster of CL CTAs shares one 128-row weight tile, each CTA
// streaming a disjoint 1/CL of K, so every weight byte is read from HBM once by one SM
// while the few activation rows come from L2.  The CL partial accumulators are reduced
// through distributed shared memory: every CTA puts its partial tile in its own shared
// memory, then CTA r sums the CL partials of weight rows [r*128/CL, (r+1)*128/CL) for all
// activation rows and stores them through the routed epilogue (one thread per activation
// row, 16 output columns per store).  No atomics, no second pass.
//   warp 0, one lane : TMA producer (weight tile and activation rows, 4-stage ring)
//   warp 1, one lane : tcgen05.mma (M = 128, N = BN) into tensor memory
//   all four warps   : tensor memory -> shared partial tile; the cluster reduction with
//                      16-byte distributed-shared-memory loads into a local tile of the
//                      CTA's rows, then the epilogue from there
// ---------------------------------------------------------------------------
namespace wsg {
constexpr int BM = 128, BK = 64, STAGES = 3;  // 3 stages: 5.43 ms per decode step, 4: 5.49, 2: 5.52
constexpr int W_BYTES = BM * 128;
template <int BN, int CL>
struct Cfg {
  static constexpr int X_BYTES = BN * 128;
  static constexpr int STAGE = W_BYTES + X_BYTES;
  // floats per partial row: a multiple of 4 (16-byte rows pieces) that is 16 bytes past a
  // multiple of 128 bytes, so eight rows' 16-byte stores fall in eight different bank groups
  static constexpr int PSTRIDE = BN + 4;
  static constexpr int P_BYTES = BM * PSTRIDE * 4;
  // clusters of 4 or more: the CTA's BM / CL reduced rows after the partial tile
  static constexpr int R_BYTES = CL >= 4 ? (BM / CL) * PSTRIDE * 4 : 0;
  static constexpr int BODY = STAGE * STAGES > P_BYTES + R_BYTES ? STAGE * STAGES : P_BYTES + R_BYTES;
  static constexpr int SMEM = BODY + (2 * STAGES + 1) * 8 + 16 + 1024;
  static constexpr uint32_t IDESC = make_idesc(BN, 1, 0, 0);
};
}  // namespace wsg

template <int BN, int CL>
__global__ void __launch_bounds__(128, 1)
    gemm_ws_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, int Nout,
                   int B, int K, Epilogue epi, long long wlim) {
  using C = wsg::Cfg<BN, CL>;
  using namespace wsg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::BODY);
  uint64_t *empty = full + STAGES;
  uint64_t *done = empty + STAGES;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
  float *part = reinterpret_cast<float *>(smem);  // [BM][PSTRIDE], over the stages once the MMAs are done
  __shared__ Epilogue s_epi;
  const int warp = warp_id(), lane = lane_id(), tid = threadIdx.x;
  const uint32_t rank = cluster_ctarank();
  const int mt = blockIdx.y;
  const int kblocks = (K + BK - 1) / BK;
  const int kb_per = (kblocks + CL - 1) / CL;
  const int kb0 = min(kblocks, (int)rank * kb_per), kb1 = min(kblocks, kb0 + kb_per);
  if (tid == 0) {
    s_epi = epi;
    for (int st = 0; st < STAGES; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], 1);
    }
    mbar_init(done, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
  }
  __syncthreads();
  // The weights are no kernel's output: the first stages' weight tiles are requested, and
  // the rest of this CTA's weight slice is hinted into L2, before the wait for the
  // preceding kernel (whose tail they overlap under a programmatic launch).
  const int npre = min(STAGES, kb1 - kb0);
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < npre; ++i) {
      mbar_arrive_expect_tx(&full[i], C::STAGE);
      tma_load_2d(smem + i * C::STAGE, &tmW, &full[i], (kb0 + i) * BK, mt * BM);
    }
    for (int kb = kb0 + npre; kb < kb1; ++kb) tma_prefetch_l2_2d(&tmW, kb * BK, mt * BM);
  }
  pdl_wait();
  pdl_trigger();
  if (epi.zero) {  // an accumulator the next kernel adds into
    const long long nth = (long long)gridDim.x * gridDim.y * blockDim.x;
    for (long long i = ((long long)blockIdx.y * gridDim.x + blockIdx.x) * blockDim.x + tid; i < epi.zero_n; i += nth)
      epi.zero[i] = 0.f;
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer ----------------
    int st = 0;
    uint32_t ph = 0, issued[STAGES] = {};
    bool ok = true;
    for (int kb = kb0; kb < kb1; ++kb) {
      if (kb - kb0 < npre) {  // the weight tile of this (fresh) stage is already on its way
        tma_load_2d(smem + st * C::STAGE + W_BYTES, &tmX, &full[st], kb * BK, 0);
      } else {
        if (!mbar_wait(&empty[st], ph ^ 1u, &g_err_gemm, wlim)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[st], C::STAGE);
        tma_load_2d(smem + st * C::STAGE, &tmW, &full[st], kb * BK, mt * BM);
        tma_load_2d(smem + st * C::STAGE + W_BYTES, &tmX, &full[st], kb * BK, 0);
      }
      ++issued[st];
      if (++st == STAGES) {
        st = 0;
        ph ^= 1u;
      }
    }
    if (!ok)  // no copy may still be landing in the stages that the partial tile reuses
      for (int x = 0; x < STAGES; ++x)
        if (issued[x]) mbar_wait_drain(&full[x], (issued[x] - 1) & 1u, &g_err_gemm, wlim);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    int st = 0;
    uint32_t ph = 0;
    for (int kb = kb0; kb < kb1; ++kb) {
      if (!mbar_wait(&full[st], ph, &g_err_gemm, wlim)) break;
      tc_fence_after();
      const uint32_t a = smem_u32(smem + st * C::STAGE), b = a + W_BYTES;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_bf16_ss(tmem, make_sdesc(a + 32 * k, 16, 1024), make_sdesc(b + 32 * k, 16, 1024), C::IDESC,
                    (kb > kb0 || k > 0) ? 1u : 0u);
      mma_commit(&empty[st]);
      if (++st == STAGES) {
        st = 0;
        ph ^= 1u;
      }
    }
    mma_commit(done);  // arrives once every MMA issued above has finished (at once if none)
  }
  __syncwarp();
  const bool acc_ok = mbar_wait(done, 0, &g_err_gemm, wlim) && kb1 > kb0;
  __syncthreads();  // the producer has drained: the stages are free for the partial tile
  tc_fence_after();
  {
    // tensor memory -> this CTA's partial tile, part[row of W][activation row], 16 bytes
    // per store
    const int f = warp * 32 + lane;
    const uint32_t t_row = tmem + (uint32_t(warp * 32) << 16);
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      uint32_t r[32];
      tmem_ld32(t_row + c, r);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; j += 4)
        *reinterpret_cast<float4 *>(part + f * C::PSTRIDE + c + j) =
            acc_ok ? make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]), __uint_as_float(r[j + 2]),
                                 __uint_as_float(r[j + 3]))
                   : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  tc_fence_before();
  cluster_sync();  // every partial tile of the cluster is written
  constexpr int F = BM / CL;  // weight rows this CTA reduces and stores
  // Clusters of 4 or more: the sums of this CTA's rows first go to a local tile [F][PSTRIDE]
  // (each of the CL-fold 16-byte loads feeds four sums); smaller clusters sum the few remote
  // values inside the store loop, whose loads then overlap the stores.
  float *red = part + BM * C::PSTRIDE;
  if constexpr (CL >= 4) {
    // the CL partials of rows rank*F .. rank*F + F - 1: 16-byte loads, consecutive threads
    // on consecutive pieces of a row (activation rows past the batch are not summed)
    const uint32_t pbase = smem_u32(part);
    const int quads = (min(B, BN) + 3) / 4;
#pragma unroll 4  // several rows' loads in flight at once
    for (int it = tid; it < F * quads; it += 128) {
      const int fl = it / quads, q = it - fl * quads;
      const uint32_t off = (uint32_t)((((int)rank * F + fl) * C::PSTRIDE + 4 * q) * 4);
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int c = 0; c < CL; ++c) {
        const float4 v = ld_shared_cluster_v4(map_shared_rank(pbase, (uint32_t)c) + off);
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      *reinterpret_cast<float4 *>(red + fl * C::PSTRIDE + 4 * q) = acc;
    }
  }
  __syncthreads();
  {
#pragma unroll 1
    for (int b = tid; b < B && b < BN; b += 128) {
      const long long m = b;
      const long long mk = remap_row(s_epi, m);
      const int rp = rope_pos(s_epi, m);
#pragma unroll 1
      for (int j = 0; j < F; j += 16) {
        const int f0 = (int)rank * F + j;
        const int n0 = mt * BM + f0;
        if (n0 >= Nout) break;
        uint32_t bits[16];
        if constexpr (CL >= 4) {
#pragma unroll
          for (int i = 0; i < 16; ++i) bits[i] = __float_as_uint(red[(j + i) * C::PSTRIDE + b]);
        } else {
          float acc[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) acc[i] = 0.f;
#pragma unroll
          for (int c = 0; c < CL; ++c) {
            const uint32_t remote = map_shared_rank(smem_u32(part), (uint32_t)c);
#pragma unroll
            for (int i = 0; i < 16; ++i)
              acc[i] += ld_shared_cluster_f32(remote + (uint32_t)(((f0 + i) * C::PSTRIDE + b) * 4));
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) bits[i] = __float_as_uint(acc[i]);
        }
        float bias[16];
        if (s_epi.bias) epi_bias16(s_epi, n0, Nout, bias);
        epi_store16<kEpiRoute | kEpiResid | kEpiGlu>(s_epi, m, mk, rp, n0, Nout, bits, bias);
      }
    }
  }
  cluster_sync();  // no CTA leaves while the others still read its partial tile
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, BN);
  }
}

template <int BN, int CL>
static hymba_status launch_ws(const GemmArgs &g, cudaStream_t s) {
  using C = wsg::Cfg<BN, CL>;
  static DeviceOnce attr_set;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr_set.done(dev)) {
    if (cudaFuncSetAttribute(gemm_ws_kernel<BN, CL>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
        cudaSuccess) {
      set_error("cudaFuncSetAttribute(weight-streaming gemm smem %d) failed", C::SMEM);
      return HYMBA_ERR_CUDA;
    }
    attr_set.mark(dev);
  }
  CUtensorMap tw, tx;
  // W = the product's B operand [N, K]; X = its A operand [M, K] (the activation rows)
  const uint64_t dw[2] = {(uint64_t)g.K, (uint64_t)g.N}, sw[1] = {(uint64_t)g.ldb * 2};
  const uint32_t bw[2] = {(uint32_t)wsg::BK, (uint32_t)wsg::BM};
  const uint64_t dx[2] = {(uint64_t)g.K, (uint64_t)g.M}, sx[1] = {(uint64_t)g.lda * 2};
  const uint32_t bx[2] = {(uint32_t)wsg::BK, (uint32_t)BN};
  if (!make_tmap(&tw, g.B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dw, sw, bw)) return HYMBA_ERR_CUDA;
  if (!make_tmap(&tx, g.A, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dx, sx, bx)) return HYMBA_ERR_CUDA;
  const int m_tiles = (g.N + wsg::BM - 1) / wsg::BM;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CL, m_tiles, 1);
  cfg.blockDim = dim3(128, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[3];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = launch_attrs(attr, 1);
  cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_ws_kernel<BN, CL>, tw, tx, g.N, g.M, g.K, g.epi,
                                     wait_limit_cycles());
  note_launch(1);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("weight-streaming gemm launch failed: %s", cudaGetErrorString(e));
    return HYMBA_ERR_CUDA;
  }
  return HYMBA_OK;
}

template <int BN>
static hymba_status launch_ws_cl(const GemmArgs &g, int cl, cudaStream_t s) {
  switch (cl) {
    case 8: return launch_ws<BN, 8>(g, s);
    case 4: return launch_ws<BN, 4>(g, s);
    case 2: return launch_ws<BN, 2>(g, s);
    default: return launch_ws<BN, 1>(g, s);
  }
}

// Decode-sized products (at most 256 activation rows, bf16, no split-K or atomic epilogue).
hymba_status gemm_ws(const GemmArgs &g, cudaStream_t s) {
  if (g.elem != 2 || g.M < 1 || g.M > 256 || g.stall) {
    set_error("gemm_ws: unsupported product (bf16, at most 256 rows)");
    return HYMBA_ERR_UNSUPPORTED;
  }
  // cluster size: enough CTAs to put most SMs on the weight stream, at most one K block each
  const int m_tiles = (g.N + wsg::BM - 1) / wsg::BM;
  const int kblocks = (g.K + wsg::BK - 1) / wsg::BK;
  int cl = 1;
  // (two CTAs per SM, i.e. clusters of 4 for the headline in_proj, measured 5.02 against
  // 4.81 ms per decode step)
  while (cl < 8 && m_tiles * cl * 2 <= num_sms() + num_sms() / 8 && kblocks >= cl * 2) cl *= 2;
  if (g.M <= 32) return launch_ws_cl<32>(g, cl, s);
  if (g.M <= 64) return launch_ws_cl<64>(g, cl, s);
  if (g.M <= 128) return launch_ws_cl<128>(g, cl, s);
  return launch_ws_cl<256>(g, cl, s);
}

// The epilogue features a product needs (kEpi* flags).
static int epi_flags(const Epilogue &e) {
  int f = 0;
  if (e.act == 1 && e.bias && e.nseg == 1 && !e.seg[0].f32 && !e.seg[0].act && !e.seg[0].resid &&
      !e.seg[0].rmap && !e.seg[0].rope && e.seg[0].inner >= e.seg[0].col1 - e.seg[0].col0)
    f |= kEpiSoftplus;
  if (e.nseg > 1 || e.rmap_rows > 0 || e.rope_tab) f |= kEpiRoute;
  for (int i = 0; i < e.nseg; ++i) {
    if (e.seg[i].rmap || e.seg[i].rope) f |= kEpiRoute;
    if (e.seg[i].resid) f |= kEpiResid;
    if (e.seg[i].act == 3) f |= kEpiGlu;
  }
  return f;
}

template <int BN, int ELEM, int EPI>
static hymba_status launch_tc(const GemmArgs &g, cudaStream_t s) {
  using C = TcCfg<BN, ELEM>;
  static DeviceOnce attr_set;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr_set.done(dev)) {
    if (cudaFuncSetAttribute(gemm_tc_kernel<BN, ELEM, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM) != cudaSuccess) {
      set_error("cudaFuncSetAttribute(gemm smem %d) failed", C::SMEM);
      return HYMBA_ERR_CUDA;
    }
    attr_set.mark(dev);
  }
  CUtensorMapDataType dt = ELEM == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  CUtensorMap ta, tb;
  uint64_t da[2] = {(uint64_t)g.K, (uint64_t)g.M}, sa[1] = {(uint64_t)g.lda * ELEM};
  uint32_t ba[2] = {(uint32_t)C::BK, (uint32_t)C::BM};
  uint64_t db[2] = {(uint64_t)g.K, (uint64_t)g.N}, sb[1] = {(uint64_t)g.ldb * ELEM};
  uint32_t bb[2] = {(uint32_t)C::BK, (uint32_t)BN};
  if (!make_tmap(&ta, g.A, dt, 2, da, sa, ba)) return HYMBA_ERR_CUDA;
  if (!make_tmap(&tb, g.B, dt, 2, db, sb, bb)) return HYMBA_ERR_CUDA;
  const long long tiles = (long long)((g.M + 127) / 128) * ((g.N + BN - 1) / BN);
  const int grid = (int)std::min<long long>(tiles, num_sms());
  launch_kernel(gemm_tc_kernel<BN, ELEM, EPI>, dim3(grid), dim3(576), (size_t)C::SMEM, s, ta, tb, g.M, g.N, g.K,
                g.epi, wait_limit_cycles(), g.stall, g.tile_ctr);
  note_launch(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("gemm_tc launch failed: %s", cudaGetErrorString(e));
    return HYMBA_ERR_CUDA;
  }
  return HYMBA_OK;
}

hymba_status gemm_tc(const GemmArgs &g, cudaStream_t s) {
  // Tile width: prefer wide tiles for large M, narrow ones when M is one tile
  // (decode) so that more CTAs stream the weights.
  const bool small_m = g.M <= 128;
  if (g.elem == 2) {
    const int f = epi_flags(g.epi) & ~kEpiSoftplus;  // a bf16 softplus takes the generic epilogue
    if (f == kEpiRoute) {  // the input projection
      if (small_m) return launch_tc<64, 2, kEpiRoute>(g, s);
      return launch_tc<256, 2, kEpiRoute>(g, s);
    }
    if (f == kEpiResid) {  // a projection back into the residual stream (the 160-wide tile spills)
      if (small_m) return launch_tc<64, 2, kEpiResid>(g, s);
      return launch_tc<128, 2, kEpiResid>(g, s);
    }
    if (f == kEpiGlu) {  // the MLP's gated up projection
      if (small_m) return launch_tc<64, 2, kEpiGlu>(g, s);
      return launch_tc<256, 2, kEpiGlu>(g, s);
    }
    if (f != 0) {
      set_error("gemm_tc: unsupported combination of epilogue features %d", f);
      return HYMBA_ERR_UNSUPPORTED;
    }
    if (g.N <= 144) return launch_tc<144, 2, 0>(g, s);
    if (small_m) return launch_tc<64, 2, 0>(g, s);
    if (g.N % 256 == 0 || g.N > 4096) return launch_tc<256, 2, 0>(g, s);
    if (g.N % 160 == 0) return launch_tc<160, 2, 0>(g, s);
    return launch_tc<128, 2, 0>(g, s);
  }
  if (g.elem == 4) {
    if (small_m) return launch_tc<64, 4, 0>(g, s);
    // dt_proj (bias + softplus, one plain bf16 segment): 128-wide tiles, two 16-column chunks
    // per epilogue warp, the bias loaded while the accumulator is read
    if (epi_flags(g.epi) == kEpiSoftplus && g.N % 128 == 0) return launch_tc<128, 4, kEpiSoftplus>(g, s);
    if (g.N % 160 == 0) return launch_tc<160, 4, 0>(g, s);
    return launch_tc<128, 4, 0>(g, s);
  }
  set_error("gemm_tc: unsupported element size %d", g.elem);
  return HYMBA_ERR_UNSUPPORTED;
}

// ---------------------------------------------------------------------------
// fp32 CUDA-core GEMM (64 x 64 tile, 16-deep K slices, 4 x 4 outputs per thread)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
    gemm_simt_f32_kernel(const float *__restrict__ A, long long lda, const float *__restrict__ B,
                         long long ldb, int M, int N, int K, Epilogue epi) {
  pdl_wait();
  pdl_trigger();
  __shared__ float As[16][64 + 4];
  __shared__ float Bs[16][64 + 4];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const long long m0 = (long long)blockIdx.y * 64;
  const int n0 = blockIdx.x * 64;
  const int kend = K;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < kend; k0 += 16) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = tid + i * 256;
      const int r = idx >> 4, kk = idx & 15;
      const long long gm = m0 + r;
      const int gn = n0 + r, gk = k0 + kk;
      As[kk][r] = (gm < M && gk < kend) ? A[gm * lda + gk] : 0.f;
      Bs[kk][r] = (gn < N && gk < kend) ? B[(long long)gn * ldb + gk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][ty * 4 + i];
        b[i] = Bs[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const long long m = m0 + ty * 4 + i;
    if (m >= M) continue;
    float v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      v[j] = n < N ? epi_act(epi, n, acc[i][j]) : acc[i][j];
    }
    // rotary pairs (2i, 2i+1) are both in this thread's four columns
#pragma unroll
    for (int j = 0; j < 4; j += 2) {
      const int n = n0 + tx * 4 + j;
      if (n + 1 < N) {
        const EpiSeg &g = epi.seg[find_seg(epi, n)];
        if (g.rope && n + 1 < g.col1) rope_rotate<1>(epi, g, n, rope_pos(epi, m), v + j);
      }
    }
    // gated SiLU pairs (both columns in this thread) write one output column each
    bool done_pair[2] = {false, false};
#pragma unroll
    for (int j = 0; j < 4; j += 2) {
      const int n = n0 + tx * 4 + j;
      if (n + 1 < N) {
        const EpiSeg &g = epi.seg[find_seg(epi, n)];
        if (g.act == 3 && n + 1 < g.col1) {
          reinterpret_cast<float *>(g.ptr)[m * g.ld_row + ((n - g.col0) >> 1)] = silu_f(v[j]) * v[j + 1];
          done_pair[j >> 1] = true;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < N && !done_pair[j >> 1]) epi_store_scalar<kEpiRoute | kEpiResid>(epi, m, remap_row(epi, m), n, v[j]);
    }
  }
}

hymba_status gemm_simt_f32(const GemmArgs &g, cudaStream_t s) {
  dim3 grid((g.N + 63) / 64, (g.M + 63) / 64);
  launch_kernel(gemm_simt_f32_kernel, grid, dim3(256), 0, s, reinterpret_cast<const float *>(g.A), g.lda,
                reinterpret_cast<const float *>(g.B), g.ldb, g.M, g.N, g.K, g.epi);
  note_launch(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("gemm_simt_f32 launch failed: %s", cudaGetErrorString(e));
    return HYMBA_ERR_CUDA;
  }
  return HYMBA_OK;
}

unsigned take_error_gemm() {
  unsigned v = 0, z = 0;
  cudaMemcpyFromSymbol(&v, g_err_gemm, sizeof(v));
  if (v) cudaMemcpyToSymbol(g_err_gemm, &z, sizeof(z));
  return v;
}

}  // namespace hymba
