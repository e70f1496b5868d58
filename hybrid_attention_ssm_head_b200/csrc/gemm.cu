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
//              softplus, fp32 -> bf16, routed stores (one GEMM writes Q, K, V,
//              x_ssm and z to their own buffers).  The second accumulator lets
//              the epilogue of tile i overlap the MMAs of tile i+1.
// Tiles are visited N-fastest so the CTAs in flight share A rows in L2.
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

__device__ __forceinline__ void epi_store_scalar(const Epilogue &e, long long m, int n, float v) {
  const EpiSeg &g = e.seg[find_seg(e, n)];
  const long long off = seg_offset(g, m, n - g.col0);
  if (e.atomic) {
    atomicAdd(reinterpret_cast<float *>(g.ptr) + off, v);
  } else if (g.f32) {
    reinterpret_cast<float *>(g.ptr)[off] = v;
  } else {
    reinterpret_cast<__nv_bfloat16 *>(g.ptr)[off] = __float2bfloat16_rn(v);
  }
}

// Stores 8 consecutive columns n..n+7 of row m (values already activated).
__device__ __forceinline__ void epi_store8(const Epilogue &e, long long m, int n, int N,
                                           const float (&v)[8]) {
  if (n >= N) return;
  const EpiSeg &g = e.seg[find_seg(e, n)];
  int local = n - g.col0;
  bool vec = !e.atomic && g.vec_ok && (n + 8 <= N) && (n + 8 <= g.col1) && (local % 8 == 0) &&
             ((local % g.inner) + 8 <= g.inner);
  if (vec) {
    const long long off = seg_offset(g, m, local);
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
    if (n + i < N) epi_store_scalar(e, m, n + i, v[i]);
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
__device__ __forceinline__ void epi_store16(const Epilogue &e, long long m, int n0, int N,
                                            const uint32_t (&r)[16], const float (&bias)[16]) {
  float v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
  const bool full = n0 + 16 <= N;
  if (!e.atomic) {
    if (e.bias) {
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] += bias[i];
    }
    if (e.act == 1) {
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = softplus_f(v[i]);
    }
  }
  // common case: the 16 columns lie in one segment and one group, 16-byte aligned rows
  const int sidx = find_seg(e, n0);
  const EpiSeg &g = e.seg[sidx];
  const int local = n0 - g.col0;
  if (full && !e.atomic && g.vec_ok && n0 + 16 <= g.col1 &&
      (g.inner >= g.col1 - g.col0 || ((g.inner & 15) == 0 && (local & 15) == 0))) {
    const long long off = seg_offset(g, m, local);
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
  epi_store8(e, m, n0, N, a);
  epi_store8(e, m, n0 + 8, N, b);
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
  static constexpr int BAR_BYTES = (2 * STAGES + 4) * 8 + 16;  // + static smem: Epilogue
  static constexpr int SMEM = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "tcgen05 M=128 needs N % 16 == 0, N <= 256");
};

template <int BN, int ELEM>
__global__ void __launch_bounds__(576, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   int M, int N, int K, int ksplit, Epilogue epi) {
  using C = TcCfg<BN, ELEM>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t *sA = smem;
  uint8_t *sB = smem + C::STAGES * C::A_BYTES;
  uint64_t *full = reinterpret_cast<uint64_t *>(sB + C::STAGES * C::B_BYTES);
  uint64_t *empty = full + C::STAGES;
  uint64_t *tfull = empty + C::STAGES;
  uint64_t *tempty = tfull + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);
  // Segment table in shared memory: per-column routing then indexes smem, not
  // kernel parameters.
  __shared__ Epilogue s_epi;
  if (threadIdx.x == 0) s_epi = epi;

  const int warp = warp_id();
  const int lane = lane_id();
  const int m_tiles = (M + C::BM - 1) / C::BM;
  const int n_tiles = (N + BN - 1) / BN;
  const int kblocks = (K + C::BK - 1) / C::BK;
  const int kb_per = (kblocks + ksplit - 1) / ksplit;
  const long long units = (long long)m_tiles * n_tiles * ksplit;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 512);
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
  if (epi.zero && warp >= 2) {
    for (long long i = (long long)blockIdx.x * 512 + (threadIdx.x - 64); i < epi.zero_n;
         i += (long long)gridDim.x * 512)
      epi.zero[i] = 0.f;
  }

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      bool ok = true;
      for (long long u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const int ks = int(u % ksplit);
        const long long tile = u / ksplit;
        const int mt = int(tile / n_tiles), nt = int(tile % n_tiles);
        const int kb0 = ks * kb_per, kb1 = min(kblocks, kb0 + kb_per);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, &g_err_gemm)) {
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
          if (issued[s]) mbar_wait_drain(&full[s], (issued[s] - 1) & 1u, &g_err_gemm);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (long long u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const int ks = int(u % ksplit);
        const int kb0 = ks * kb_per, kb1 = min(kblocks, kb0 + kb_per);
        if (kb0 >= kb1) continue;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, &g_err_gemm)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + uint32_t(acc * BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, &g_err_gemm)) {
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
              mma_bf16_ss(d_tmem, ad, bd, C::IDESC, (kb > kb0 || k > 0) ? 1u : 0u);
            else
              mma_tf32_ss(d_tmem, ad, bd, C::IDESC, (kb > kb0 || k > 0) ? 1u : 0u);
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
        mbar_wait_drain(&tfull[acc], acc_phase, &g_err_gemm);
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
    for (long long u = blockIdx.x; u < units; u += gridDim.x) {
      const int ks = int(u % ksplit);
      const long long tile = u / ksplit;
      const int kb0 = ks * kb_per, kb1 = min(kblocks, kb0 + kb_per);
      if (kb0 >= kb1) continue;
      const int mt = int(tile / n_tiles), nt = int(tile % n_tiles);
      constexpr int NCH = (BN + 63) / 64;
      if (!mbar_wait(&tfull[acc], acc_phase, &g_err_gemm)) break;
      tc_fence_after();
      const long long m = (long long)mt * C::BM + row;
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
            float bias[16];
            if (s_epi.bias) epi_bias16(s_epi, n0, N, bias);
            epi_store16(s_epi, m, n0, N, r[k], bias);
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

template <int BN, int ELEM>
static hymba_status launch_tc(const GemmArgs &g, cudaStream_t s) {
  using C = TcCfg<BN, ELEM>;
  static DeviceOnce attr_set;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr_set.done(dev)) {
    if (cudaFuncSetAttribute(gemm_tc_kernel<BN, ELEM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
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
  const long long tiles = (long long)((g.M + 127) / 128) * ((g.N + BN - 1) / BN) * g.ksplit;
  const int grid = (int)std::min<long long>(tiles, num_sms());
  gemm_tc_kernel<BN, ELEM><<<grid, 576, C::SMEM, s>>>(ta, tb, g.M, g.N, g.K, g.ksplit, g.epi);
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
    if (g.N <= 144) return launch_tc<144, 2>(g, s);
    if (small_m) return launch_tc<64, 2>(g, s);
    if (g.N % 256 == 0 || g.N > 4096) return launch_tc<256, 2>(g, s);
    if (g.N % 160 == 0) return launch_tc<160, 2>(g, s);
    return launch_tc<128, 2>(g, s);
  }
  if (g.elem == 4) {
    if (small_m) return launch_tc<64, 4>(g, s);
    if (g.N % 160 == 0) return launch_tc<160, 4>(g, s);
    return launch_tc<128, 4>(g, s);
  }
  set_error("gemm_tc: unsupported element size %d", g.elem);
  return HYMBA_ERR_UNSUPPORTED;
}

// ---------------------------------------------------------------------------
// fp32 CUDA-core GEMM (64 x 64 tile, 16-deep K slices, 4 x 4 outputs per thread)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
    gemm_simt_f32_kernel(const float *__restrict__ A, long long lda, const float *__restrict__ B,
                         long long ldb, int M, int N, int K, int kb_per, Epilogue epi) {
  __shared__ float As[16][64 + 4];
  __shared__ float Bs[16][64 + 4];
  const int tid = threadIdx.x;
  if (epi.zero) {
    const long long nb = (long long)gridDim.x * gridDim.y * gridDim.z;
    const long long bid = blockIdx.x + (long long)gridDim.x * (blockIdx.y + (long long)gridDim.y * blockIdx.z);
    for (long long i = bid * 256 + tid; i < epi.zero_n; i += nb * 256) epi.zero[i] = 0.f;
  }
  const int tx = tid & 15, ty = tid >> 4;
  const long long m0 = (long long)blockIdx.y * 64;
  const int n0 = blockIdx.x * 64;
  const int kbeg = blockIdx.z * kb_per * 16;
  const int kend = min(K, kbeg + kb_per * 16);
  float acc[4][4] = {};
  for (int k0 = kbeg; k0 < kend; k0 += 16) {
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
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < N) {
        float v = acc[i][j];
        if (!epi.atomic) v = epi_act(epi, n, v);
        epi_store_scalar(epi, m, n, v);
      }
    }
  }
}

hymba_status gemm_simt_f32(const GemmArgs &g, cudaStream_t s) {
  const int kblocks = (g.K + 15) / 16;
  const int kb_per = (kblocks + g.ksplit - 1) / g.ksplit;
  dim3 grid((g.N + 63) / 64, (g.M + 63) / 64, g.ksplit);
  gemm_simt_f32_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const float *>(g.A), g.lda,
                                            reinterpret_cast<const float *>(g.B), g.ldb, g.M, g.N,
                                            g.K, kb_per, g.epi);
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
