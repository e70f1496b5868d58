// Attention heads of the hybrid-head layer (Hymba §2.1 Eq. 1 with the 1/sqrt(d)
// scale of the authors' OpenReview reply Q2), GQA with query groups (Appendix E
// Table 11), under the A-shape mask (meta tokens always visible + sliding
// window; OpenReview reply Q1) or the causal mask of the global layers (§2.2).
//
// Prefill, bf16, d_qk = 64, d_v = 128: one CTA owns two 128-row query tiles of
// one (batch, head) and streams the visible 128-key tiles of their kv head.
//   warp 0     : TMA producer: Q tiles once, K and V tiles into 2-stage rings.
//   warp 1     : TMEM allocation and MMA issue.  Per key tile and query tile:
//                S = Q K^T (tcgen05, M=128, N=128, K=64) and O += P V
//                (M=128, N=128, K=128; V read MN-major from its natural layout).
//   warps 2-5, 6-9 : one softmax warpgroup per query tile, one thread per row:
//                row max over S (tcgen05.ld), lazy rescaling of O in TMEM only
//                when the max grows by more than 2^8, exp2, P (bf16) written to
//                shared memory in the 128-byte swizzled K-major layout.
// The two query tiles ping-pong: while one warpgroup computes softmax the
// tensor core runs the other tile's MMAs.  Key tiles with no visible pair are
// never loaded; fully visible tiles skip the per-element mask.
//
// fp32 path and decode: CUDA-core kernels (small or bandwidth-bound work).
#include <algorithm>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tmap.h"

namespace hymba {

HYMBA_DEVICE_ERROR_WORD(g_err_attn);

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------------------
// tcgen05 prefill attention
// ---------------------------------------------------------------------------
namespace fa {
constexpr int QT = 128;          // query rows per tile
constexpr int KT = 128;          // keys per tile
constexpr int NQ = 2;            // query tiles per CTA
constexpr int Q_BYTES = QT * 128;        // 64 bf16 per row
constexpr int K_BYTES = KT * 128;
constexpr int V_BYTES = KT * 256;        // two 64-column boxes
constexpr int P_BYTES = QT * 256;        // two 64-key swizzle atoms
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + NQ * Q_BYTES;
constexpr int OFF_V = OFF_K + 2 * K_BYTES;
constexpr int OFF_P = OFF_V + 2 * V_BYTES;
constexpr int OFF_BAR = OFF_P + NQ * P_BYTES;
constexpr int NBAR = 1 + 2 + 2 + 2 + 2 + NQ * 3 + 1;
constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
constexpr int THREADS = 64 + NQ * 128;
constexpr uint32_t IDESC_S = make_idesc(128, 1, 0, 0);
constexpr uint32_t IDESC_PV = make_idesc(128, 1, 0, 1);
}  // namespace fa

// Class of the (query tile, key tile) pair as the prefill kernel sees it.
__device__ __forceinline__ int fa_tile_class(int qtile, int kt, int L, int n_meta, int window,
                                             int is_global) {
  return seq_tile_class(qtile, kt, L, n_meta, window, is_global);
}
__device__ __forceinline__ bool fa_streamed(int qa, int kt, int L, int m, int w, int g) {
  return fa_tile_class(qa, kt, L, m, w, g) != 0 || fa_tile_class(qa + 1, kt, L, m, w, g) != 0;
}

__global__ void __launch_bounds__(fa::THREADS, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, __nv_bfloat16 *__restrict__ out,
                       int L, int H, int Hkv, int n_meta, int window, int is_global, float scale_log2,
                       int npairs) {
  using namespace fa;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  uint64_t *q_full = bars + 0;
  uint64_t *k_full = bars + 1, *k_empty = bars + 3;
  uint64_t *v_full = bars + 5, *v_empty = bars + 7;
  uint64_t *s_full = bars + 9;            // [NQ]
  uint64_t *p_full = bars + 9 + NQ;       // [NQ]
  uint64_t *o_done = bars + 9 + 2 * NQ;   // [NQ]
  uint64_t *drain = bars + 9 + 3 * NQ;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NBAR);

  const int warp = warp_id(), lane = lane_id();
  // block -> (head fastest, then query-tile pair, then batch): the heads of one
  // kv group run together and share K/V tiles through L2.
  const int h = blockIdx.x % H;
  const int rest = blockIdx.x / H;
  const int pair = rest % npairs;
  const int b = rest / npairs;
  const int g = h / (H / Hkv);
  const int qa = 2 * pair;
  const int kt_last = min(qa + 1, (L - 1) / KT);

  if (warp == 0 && lane == 0) {
    mbar_init(q_full, 1);
    mbar_init(drain, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int q = 0; q < NQ; ++q) {
      mbar_init(&s_full[q], 1);
      mbar_init(&p_full[q], 4);
      mbar_init(&o_done[q], 1);
    }
    fence_barrier_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM columns: S of tile q at 256q, O of tile q at 256q + 128.

  // Number of streamed key tiles (same count in every role).
  int nstream = 0;
  for (int kt = 0; kt <= kt_last; ++kt)
    if (fa_streamed(qa, kt, L, n_meta, window, is_global)) ++nstream;

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      uint32_t k_issued[2] = {0, 0}, v_issued[2] = {0, 0};
      mbar_arrive_expect_tx(q_full, NQ * Q_BYTES);
      for (int q = 0; q < NQ; ++q)
        tma_load_3d(smem + OFF_Q + q * Q_BYTES, &tmQ, q_full, h * 64, (qa + q) * QT, b);
      int j = 0;
      for (int kt = 0; kt <= kt_last && ok; ++kt) {
        if (!fa_streamed(qa, kt, L, n_meta, window, is_global)) continue;
        const int st = j & 1;
        const uint32_t ph = (uint32_t(j) >> 1) & 1u;
        if (!mbar_wait(&k_empty[st], ph ^ 1u, &g_err_attn)) { ok = false; break; }
        mbar_arrive_expect_tx(&k_full[st], K_BYTES);
        tma_load_3d(smem + OFF_K + st * K_BYTES, &tmK, &k_full[st], g * 64, kt * KT, b);
        ++k_issued[st];
        if (!mbar_wait(&v_empty[st], ph ^ 1u, &g_err_attn)) { ok = false; break; }
        mbar_arrive_expect_tx(&v_full[st], V_BYTES);
        uint8_t *vdst = smem + OFF_V + st * V_BYTES;
        tma_load_3d(vdst, &tmV, &v_full[st], g * 128, kt * KT, b);
        tma_load_3d(vdst + V_BYTES / 2, &tmV, &v_full[st], g * 128 + 64, kt * KT, b);
        ++v_issued[st];
        ++j;
      }
      if (!ok) {
        mbar_wait(q_full, 0, &g_err_attn);
        for (int s = 0; s < 2; ++s) {
          if (k_issued[s]) mbar_wait(&k_full[s], (k_issued[s] - 1) & 1u, &g_err_attn);
          if (v_issued[s]) mbar_wait(&v_full[s], (v_issued[s] - 1) & 1u, &g_err_attn);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && nstream > 0) {
      bool ok = mbar_wait(q_full, 0, &g_err_attn);
      const uint32_t q_addr0 = smem_u32(smem + OFF_Q);
      const uint32_t p_addr0 = smem_u32(smem + OFF_P);
      auto issue_S = [&](int q, int st) {
        const uint32_t qa_ = q_addr0 + q * Q_BYTES;
        const uint32_t ka = smem_u32(smem + OFF_K + st * K_BYTES);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_bf16_ss(tmem + 256 * q, make_sdesc(qa_ + 32 * k, 16, 1024),
                      make_sdesc(ka + 32 * k, 16, 1024), IDESC_S, k > 0 ? 1u : 0u);
        mma_commit(&s_full[q]);
      };
      auto issue_PV = [&](int q, int st, bool acc_prev) {
        const uint32_t pa = p_addr0 + q * P_BYTES;
        const uint32_t va = smem_u32(smem + OFF_V + st * V_BYTES);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ad = make_sdesc(pa + (kk >> 2) * (P_BYTES / 2) + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = make_sdesc(va + kk * 2048, V_BYTES / 2, 1024);
          mma_bf16_ss(tmem + 256 * q + 128, ad, bd, IDESC_PV, (acc_prev || kk > 0) ? 1u : 0u);
        }
        mma_commit(&o_done[q]);
      };
      if (ok) ok = mbar_wait(&k_full[0], 0, &g_err_attn);
      if (ok) {
        tc_fence_after();
        for (int q = 0; q < NQ; ++q) issue_S(q, 0);
        mma_commit(&k_empty[0]);
      }
      for (int j = 0; j < nstream && ok; ++j) {
        const int st = j & 1;
        const uint32_t ph = (uint32_t(j) >> 1) & 1u;
        for (int q = 0; q < NQ && ok; ++q) {
          if (!mbar_wait(&p_full[q], uint32_t(j) & 1u, &g_err_attn)) { ok = false; break; }
          if (q == 0 && !mbar_wait(&v_full[st], ph, &g_err_attn)) { ok = false; break; }
          tc_fence_after();
          issue_PV(q, st, j > 0);
          if (q == NQ - 1) mma_commit(&v_empty[st]);
          if (j + 1 < nstream) {
            const int st1 = (j + 1) & 1;
            const uint32_t ph1 = (uint32_t(j + 1) >> 1) & 1u;
            if (q == 0 && !mbar_wait(&k_full[st1], ph1, &g_err_attn)) { ok = false; break; }
            tc_fence_after();
            issue_S(q, st1);
            if (q == NQ - 1) mma_commit(&k_empty[st1]);
          }
        }
      }
      if (!ok) {
        // Drain issued MMAs before tensor memory is released.
        mma_commit(drain);
        mbar_wait(drain, 0, &g_err_attn);
      }
    }
  } else {
    // ---------------- softmax warpgroups ----------------
    const int q = (warp - 2) >> 2;        // query tile of this warpgroup
    const int quarter = warp & 3;         // TMEM lane quarter
    const int r = quarter * 32 + lane;    // row within the tile
    const long long i = (long long)(qa + q) * QT + r;  // query position
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const uint32_t tS = tmem + 256 * q + lane_off;
    const uint32_t tO = tS + 128;
    const uint32_t p_base = smem_u32(smem + OFF_P + q * P_BYTES);
    const int qtile = qa + q;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    int j = 0;
    for (int kt = 0; kt <= kt_last && ok; ++kt) {
      if (!fa_streamed(qa, kt, L, n_meta, window, is_global)) continue;
      const int cls = fa_tile_class(qtile, kt, L, n_meta, window, is_global);
      const long long key0 = (long long)kt * KT;
      if (!mbar_wait(&s_full[q], uint32_t(j) & 1u, &g_err_attn)) { ok = false; break; }
      tc_fence_after();
      // pass 1: row maximum of the scaled, masked scores
      float mx = -INFINITY;
      if (cls != 0) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld32(tS + c * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            float x = __uint_as_float(v[e]) * scale_log2;
            if (cls == 2 && !mask_allowed(i, key0 + c * 32 + e, n_meta, window, is_global))
              x = -INFINITY;
            mx = fmaxf(mx, x);
          }
        }
      }
      // lazy rescale decision
      float alpha = 1.f;
      bool resc = false;
      if (m_run == -INFINITY) {
        m_run = mx;
      } else if (mx > m_run + 8.f) {
        alpha = ex2(m_run - mx);
        m_run = mx;
        resc = true;
      }
      l_run *= alpha;
      if (j > 0) {
        if (!mbar_wait(&o_done[q], uint32_t(j - 1) & 1u, &g_err_attn)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, resc)) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t v[32];
            tmem_ld32(tO + c * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
            tmem_st32(tO + c * 32, v);
          }
          tmem_wait_st();
        }
      }
      // pass 2: P = exp2(x - m), bf16, into the swizzled K-major tile
      const float mref = (m_run == -INFINITY) ? 0.f : m_run;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
        if (cls != 0) {
          tmem_ld32(tS + c * 32, v);
          tmem_wait_ld();
        }
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float p0 = 0.f, p1 = 0.f;
          if (cls != 0) {
            float x0 = __uint_as_float(v[e]) * scale_log2;
            float x1 = __uint_as_float(v[e + 1]) * scale_log2;
            if (cls == 2) {
              if (!mask_allowed(i, key0 + c * 32 + e, n_meta, window, is_global)) x0 = -INFINITY;
              if (!mask_allowed(i, key0 + c * 32 + e + 1, n_meta, window, is_global)) x1 = -INFINITY;
            }
            p0 = ex2(x0 - mref);
            p1 = ex2(x1 - mref);
          }
          __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
          l_run += __low2float(pb) + __high2float(pb);
          pk[e >> 1] = *reinterpret_cast<uint32_t *>(&pb);
        }
        // keys c*32 .. c*32+31 -> atom c/2, 16-byte chunks (c%2)*4 .. +3
        const uint32_t atom = p_base + (c >> 1) * (P_BYTES / 2) + r * 128;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int chunk = (c & 1) * 4 + t;
          st_shared_v4(atom + ((chunk ^ (r & 7)) << 4), pk[4 * t], pk[4 * t + 1], pk[4 * t + 2],
                       pk[4 * t + 3]);
        }
      }
      fence_proxy_async();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[q]);
      ++j;
    }
    // epilogue: O / l -> bf16 rows of the output
    if (ok && nstream > 0 && mbar_wait(&o_done[q], uint32_t(nstream - 1) & 1u, &g_err_attn)) {
      tc_fence_after();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      const int E = H * 128;
      __nv_bfloat16 *dst = out + ((long long)b * L + i) * E + h * 128;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
        tmem_ld32(tO + c * 32, v);
        tmem_wait_ld();
        if (i < L) {
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            st_global_v4(dst + c * 32 + t * 8,
                         pack_bf16x2(__uint_as_float(v[8 * t]) * inv, __uint_as_float(v[8 * t + 1]) * inv),
                         pack_bf16x2(__uint_as_float(v[8 * t + 2]) * inv, __uint_as_float(v[8 * t + 3]) * inv),
                         pack_bf16x2(__uint_as_float(v[8 * t + 4]) * inv, __uint_as_float(v[8 * t + 5]) * inv),
                         pack_bf16x2(__uint_as_float(v[8 * t + 6]) * inv, __uint_as_float(v[8 * t + 7]) * inv));
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

static hymba_status attention_prefill_tc(const AttnArgs &a, cudaStream_t s) {
  using namespace fa;
  static unsigned attr_set = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(attr_set & (1u << (dev & 31)))) {
    if (cudaFuncSetAttribute(attn_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) !=
        cudaSuccess) {
      set_error("cudaFuncSetAttribute(attention smem) failed");
      return HYMBA_ERR_CUDA;
    }
    attr_set |= 1u << (dev & 31);
  }
  CUtensorMap tq, tk, tv;
  const uint64_t dq[3] = {(uint64_t)a.H * 64, (uint64_t)a.L, (uint64_t)a.B};
  const uint64_t sq[2] = {(uint64_t)a.H * 64 * 2, (uint64_t)a.L * a.H * 64 * 2};
  const uint64_t dk[3] = {(uint64_t)a.Hkv * 64, (uint64_t)a.L, (uint64_t)a.B};
  const uint64_t sk[2] = {(uint64_t)a.Hkv * 64 * 2, (uint64_t)a.L * a.Hkv * 64 * 2};
  const uint64_t dv[3] = {(uint64_t)a.Hkv * 128, (uint64_t)a.L, (uint64_t)a.B};
  const uint64_t sv[2] = {(uint64_t)a.Hkv * 128 * 2, (uint64_t)a.L * a.Hkv * 128 * 2};
  const uint32_t box[3] = {64, 128, 1};
  if (!make_tmap(&tq, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, dq, sq, box)) return HYMBA_ERR_CUDA;
  if (!make_tmap(&tk, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, dk, sk, box)) return HYMBA_ERR_CUDA;
  if (!make_tmap(&tv, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, dv, sv, box)) return HYMBA_ERR_CUDA;
  const int nqt = (a.L + QT - 1) / QT;
  const int npairs = (nqt + 1) / 2;
  const long long blocks = (long long)npairs * a.H * a.B;
  if (blocks > 0x7fffffffLL) {
    set_error("attention grid too large");
    return HYMBA_ERR_UNSUPPORTED;
  }
  attn_fwd_tc_kernel<<<(unsigned)blocks, THREADS, SMEM, s>>>(
      tq, tk, tv, reinterpret_cast<__nv_bfloat16 *>(a.o), a.L, a.H, a.Hkv, a.n_meta, a.window,
      a.is_global, a.scale * 1.4426950408889634f, npairs);
  note_launch(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("attention launch failed: %s", cudaGetErrorString(e));
    return HYMBA_ERR_CUDA;
  }
  return HYMBA_OK;
}

// ---------------------------------------------------------------------------
// CUDA-core prefill attention (fp32 storage): one warp per (query, head).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void attn_fwd_simt_kernel(const T *__restrict__ q, const T *__restrict__ k,
                                     const T *__restrict__ v, T *__restrict__ o, int B, int L, int H,
                                     int Hkv, int dqk, int dv, int n_meta, int window, int is_global,
                                     float scale) {
  const long long wid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= (long long)B * L * H) return;
  const int h = int(wid % H);
  const long long bi = wid / H;
  const int i = int(bi % L);
  const int b = int(bi / L);
  const int g = h / (H / Hkv);
  const T *qr = q + ((long long)b * L + i) * H * dqk + h * dqk;
  float mx = -INFINITY, l = 0.f;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};  // dv <= 256: lane owns columns lane + 32*t
  for (int j = 0; j <= i; ++j) {
    if (!mask_allowed(i, j, n_meta, window, is_global)) continue;
    const T *kr = k + ((long long)b * L + j) * Hkv * dqk + g * dqk;
    float part = 0.f;
    for (int d = lane; d < dqk; d += 32) part += Store<T>::to_f(qr[d]) * Store<T>::to_f(kr[d]);
#pragma unroll
    for (int off = 16; off; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    const float sc = part * scale;
    const float mn = fmaxf(mx, sc);
    const float alpha = expf(mx - mn);
    const float p = expf(sc - mn);
    l = l * alpha + p;
    const T *vr = v + ((long long)b * L + j) * Hkv * dv + g * dv;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const int d = lane + 32 * t;
      if (d < dv) acc[t] = acc[t] * alpha + p * Store<T>::to_f(vr[d]);
    }
    mx = mn;
  }
  T *orow = o + ((long long)b * L + i) * H * dv + h * dv;
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    const int d = lane + 32 * t;
    if (d < dv) orow[d] = Store<T>::from_f(acc[t] / l);
  }
}

hymba_status attention_prefill(const AttnArgs &a, hymba_dtype dt, cudaStream_t s) {
  if (dt == HYMBA_BF16) {
    if (a.dqk != 64 || a.dv != 128) {
      set_error("bf16 attention kernel supports head_dim_qk 64 and head_dim_v 128 only");
      return HYMBA_ERR_UNSUPPORTED;
    }
    return attention_prefill_tc(a, s);
  }
  if (a.dv > 256) {
    set_error("fp32 attention supports head_dim_v <= 256");
    return HYMBA_ERR_UNSUPPORTED;
  }
  const long long warps = (long long)a.B * a.L * a.H;
  const int tpb = 256;
  const long long blocks = (warps * 32 + tpb - 1) / tpb;
  attn_fwd_simt_kernel<float><<<(unsigned)blocks, tpb, 0, s>>>(
      (const float *)a.q, (const float *)a.k, (const float *)a.v, (float *)a.o, a.B, a.L, a.H,
      a.Hkv, a.dqk, a.dv, a.n_meta, a.window, a.is_global, a.scale);
  note_launch(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("attention launch failed: %s", cudaGetErrorString(e));
    return HYMBA_ERR_CUDA;
  }
  return HYMBA_OK;
}

// ---------------------------------------------------------------------------
// Decode attention: one query per sequence over the layer's K/V store.
// Split over key chunks (partial softmax per chunk), then a combine kernel.
// The query heads of one kv group share every K/V read.
// ---------------------------------------------------------------------------
constexpr int DEC_CHUNK = 256;
constexpr int DEC_MAXREP = 8;

__host__ __device__ __forceinline__ long long dec_visible(long long pos, int n_meta, int window,
                                                          int is_global, long long *win0) {
  // visible positions: [0, meta_end) and [win0, pos]
  if (is_global) {
    *win0 = 0;
    return pos + 1;
  }
  const long long meta_end = n_meta < pos + 1 ? n_meta : pos + 1;
  long long w0 = pos - window + 1;
  if (w0 < meta_end) w0 = meta_end;
  *win0 = w0;
  return meta_end + (pos - w0 + 1);
}
__host__ __device__ __forceinline__ long long dec_position(long long vi, int n_meta,
                                                           long long pos, long long win0,
                                                           int is_global) {
  if (is_global) return vi;
  const long long meta_end = n_meta < pos + 1 ? n_meta : pos + 1;
  return vi < meta_end ? vi : win0 + (vi - meta_end);
}
__host__ __device__ __forceinline__ long long kv_slot_of(long long p, int n_meta, int window,
                                                         int is_global) {
  if (is_global || p < n_meta) return p;
  return n_meta + (p - n_meta) % window;
}

size_t decode_attn_workspace_floats(int B, int H, int dv, long long pos, int n_meta, int window,
                                    int is_global) {
  long long w0;
  const long long nvis = dec_visible(pos, n_meta, window, is_global, &w0);
  const long long nsplit = (nvis + DEC_CHUNK - 1) / DEC_CHUNK;
  return (size_t)B * H * nsplit * (dv + 2);
}

template <typename T>
__global__ void __launch_bounds__(128)
    attn_decode_partial_kernel(const T *__restrict__ q, const T *__restrict__ kc,
                               const T *__restrict__ vc, float *__restrict__ part, int H, int Hkv,
                               int dqk, int dv, int cap, long long pos, int n_meta, int window,
                               int is_global, float scale_log2, int nsplit) {
  __shared__ float qs[DEC_MAXREP][128];
  __shared__ float sc[DEC_MAXREP][DEC_CHUNK];
  __shared__ float red[DEC_MAXREP][4];
  __shared__ float mxs[DEC_MAXREP], sums[DEC_MAXREP];
  const int split = blockIdx.y;
  const int bg = blockIdx.x;
  const int b = bg / Hkv, g = bg % Hkv;
  const int rep = H / Hkv;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  for (int idx = tid; idx < rep * dqk; idx += 128) {
    const int r = idx / dqk, d = idx % dqk;
    qs[r][d] = Store<T>::to_f(q[(long long)b * H * dqk + (g * rep + r) * dqk + d]) * scale_log2;
  }
  __syncthreads();
  long long w0;
  const long long nvis = dec_visible(pos, n_meta, window, is_global, &w0);
  const long long v0 = (long long)split * DEC_CHUNK;
  const int nk = (int)min((long long)DEC_CHUNK, nvis - v0);
  const T *kbase = kc + ((long long)b * Hkv + g) * cap * dqk;
  const T *vbase = vc + ((long long)b * Hkv + g) * cap * dv;
  for (int t = tid; t < DEC_CHUNK; t += 128) {
    if (t < nk) {
      const long long p = dec_position(v0 + t, n_meta, pos, w0, is_global);
      const T *kr = kbase + kv_slot_of(p, n_meta, window, is_global) * dqk;
      float acc[DEC_MAXREP];
#pragma unroll
      for (int r = 0; r < DEC_MAXREP; ++r) acc[r] = 0.f;
      for (int d = 0; d < dqk; ++d) {
        const float kv = Store<T>::to_f(kr[d]);
#pragma unroll
        for (int r = 0; r < DEC_MAXREP; ++r)
          if (r < rep) acc[r] = fmaf(qs[r][d], kv, acc[r]);
      }
      for (int r = 0; r < rep; ++r) sc[r][t] = acc[r];
    } else {
      for (int r = 0; r < rep; ++r) sc[r][t] = -INFINITY;
    }
  }
  __syncthreads();
  // per-head max and sum over the chunk
  for (int r = 0; r < rep; ++r) {
    float m = fmaxf(sc[r][tid], sc[r][tid + 128]);
#pragma unroll
    for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (lane == 0) red[r][wid] = m;
  }
  __syncthreads();
  if (tid < rep) mxs[tid] = fmaxf(fmaxf(red[tid][0], red[tid][1]), fmaxf(red[tid][2], red[tid][3]));
  __syncthreads();
  for (int r = 0; r < rep; ++r) {
    const float p0 = ex2(sc[r][tid] - mxs[r]);
    const float p1 = ex2(sc[r][tid + 128] - mxs[r]);
    sc[r][tid] = p0;
    sc[r][tid + 128] = p1;
    float s = p0 + p1;
#pragma unroll
    for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) red[r][wid] = s;
  }
  __syncthreads();
  if (tid < rep) sums[tid] = red[tid][0] + red[tid][1] + red[tid][2] + red[tid][3];
  __syncthreads();
  // o[r][d] = sum_t p[r][t] V[t][d]
  for (int d = tid; d < dv; d += 128) {
    float acc[DEC_MAXREP];
#pragma unroll
    for (int r = 0; r < DEC_MAXREP; ++r) acc[r] = 0.f;
    for (int t = 0; t < nk; ++t) {
      const long long p = dec_position(v0 + t, n_meta, pos, w0, is_global);
      const float vv = Store<T>::to_f(vbase[kv_slot_of(p, n_meta, window, is_global) * dv + d]);
#pragma unroll
      for (int r = 0; r < DEC_MAXREP; ++r)
        if (r < rep) acc[r] = fmaf(sc[r][t], vv, acc[r]);
    }
    for (int r = 0; r < rep; ++r) {
      float *dst = part + (((long long)b * H + g * rep + r) * nsplit + split) * (dv + 2);
      dst[2 + d] = acc[r];
    }
  }
  if (tid < rep) {
    float *dst = part + (((long long)b * H + g * rep + tid) * nsplit + split) * (dv + 2);
    dst[0] = mxs[tid];
    dst[1] = sums[tid];
  }
}

template <typename T>
__global__ void attn_decode_combine_kernel(const float *__restrict__ part, T *__restrict__ o, int H,
                                           int dv, int nsplit) {
  const int bh = blockIdx.x;
  const float *base = part + (long long)bh * nsplit * (dv + 2);
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, base[s * (dv + 2)]);
  float Lsum = 0.f;
  for (int s = 0; s < nsplit; ++s) Lsum += base[s * (dv + 2) + 1] * ex2(base[s * (dv + 2)] - M);
  for (int d = threadIdx.x; d < dv; d += blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < nsplit; ++s)
      acc += base[s * (dv + 2) + 2 + d] * ex2(base[s * (dv + 2)] - M);
    o[(long long)bh * dv + d] = Store<T>::from_f(acc / Lsum);
  }
}

hymba_status attention_decode(const DecodeAttnArgs &a, hymba_dtype dt, cudaStream_t s) {
  const int rep = a.H / a.Hkv;
  if (rep > DEC_MAXREP || a.dqk > 128) {
    set_error("decode attention supports H/Hkv <= 8 and head_dim_qk <= 128");
    return HYMBA_ERR_UNSUPPORTED;
  }
  long long w0;
  const long long nvis = dec_visible(a.pos, a.n_meta, a.window, a.is_global, &w0);
  const int nsplit = (int)((nvis + DEC_CHUNK - 1) / DEC_CHUNK);
  dim3 grid(a.B * a.Hkv, nsplit);
  const float sl2 = a.scale * 1.4426950408889634f;
  if (dt == HYMBA_BF16) {
    attn_decode_partial_kernel<__nv_bfloat16><<<grid, 128, 0, s>>>(
        (const __nv_bfloat16 *)a.q, (const __nv_bfloat16 *)a.k_cache, (const __nv_bfloat16 *)a.v_cache,
        a.partial, a.H, a.Hkv, a.dqk, a.dv, a.cap, a.pos, a.n_meta, a.window, a.is_global, sl2, nsplit);
    attn_decode_combine_kernel<__nv_bfloat16><<<a.B * a.H, 128, 0, s>>>(
        a.partial, (__nv_bfloat16 *)a.o, a.H, a.dv, nsplit);
  } else {
    attn_decode_partial_kernel<float><<<grid, 128, 0, s>>>(
        (const float *)a.q, (const float *)a.k_cache, (const float *)a.v_cache, a.partial, a.H,
        a.Hkv, a.dqk, a.dv, a.cap, a.pos, a.n_meta, a.window, a.is_global, sl2, nsplit);
    attn_decode_combine_kernel<float><<<a.B * a.H, 128, 0, s>>>(a.partial, (float *)a.o, a.H,
                                                                 a.dv, nsplit);
  }
  note_launch(2);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("decode attention launch failed: %s", cudaGetErrorString(e));
    return HYMBA_ERR_CUDA;
  }
  return HYMBA_OK;
}

// ---------------------------------------------------------------------------
// Decode K/V store emission after prefill: meta rows, and the last W rows of a
// sliding-window layer (every row of a global layer), at their slots.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void kv_emit_kernel(const T *__restrict__ kseq, const T *__restrict__ vseq,
                               T *__restrict__ kc, T *__restrict__ vc, int B, int L, int Hkv,
                               int dqk, int dv, int cap, int n_meta, int window, int is_global,
                               long long n_keep, int meta_keep, long long start) {
  const long long total = (long long)B * Hkv * n_keep;
  const long long idx = (long long)blockIdx.x * blockDim.y + threadIdx.y;
  if (idx >= total) return;
  const long long kk = idx % n_keep;
  const long long bg = idx / n_keep;
  const int g = int(bg % Hkv), b = int(bg / Hkv);
  const long long p = kk < meta_keep ? kk : start + (kk - meta_keep);
  const long long slot = kv_slot_of(p, n_meta, window, is_global);
  const T *ks = kseq + ((long long)b * L + p) * Hkv * dqk + g * dqk;
  const T *vs = vseq + ((long long)b * L + p) * Hkv * dv + g * dv;
  T *kd = kc + (((long long)b * Hkv + g) * cap + slot) * dqk;
  T *vd = vc + (((long long)b * Hkv + g) * cap + slot) * dv;
  for (int d = threadIdx.x; d < dqk; d += blockDim.x) kd[d] = ks[d];
  for (int d = threadIdx.x; d < dv; d += blockDim.x) vd[d] = vs[d];
}

hymba_status kv_cache_emit(const KvEmitArgs &a, hymba_dtype dt, cudaStream_t s) {
  int meta_keep;
  long long start, n_keep;
  if (a.is_global) {
    meta_keep = 0;
    start = 0;
    n_keep = a.L;
  } else {
    meta_keep = std::min(a.n_meta, a.L);
    start = std::max<long long>(meta_keep, (long long)a.L - a.window);
    n_keep = meta_keep + (a.L - start);
  }
  const long long total = (long long)a.B * a.Hkv * n_keep;
  if (total == 0) return HYMBA_OK;
  dim3 block(32, 8);
  const long long blocks = (total + 7) / 8;
  if (dt == HYMBA_BF16)
    kv_emit_kernel<__nv_bfloat16><<<(unsigned)blocks, block, 0, s>>>(
        (const __nv_bfloat16 *)a.k_seq, (const __nv_bfloat16 *)a.v_seq, (__nv_bfloat16 *)a.k_cache,
        (__nv_bfloat16 *)a.v_cache, a.B, a.L, a.Hkv, a.dqk, a.dv, a.cap, a.n_meta, a.window,
        a.is_global, n_keep, meta_keep, start);
  else
    kv_emit_kernel<float><<<(unsigned)blocks, block, 0, s>>>(
        (const float *)a.k_seq, (const float *)a.v_seq, (float *)a.k_cache, (float *)a.v_cache, a.B,
        a.L, a.Hkv, a.dqk, a.dv, a.cap, a.n_meta, a.window, a.is_global, n_keep, meta_keep, start);
  note_launch(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("kv emit launch failed: %s", cudaGetErrorString(e));
    return HYMBA_ERR_CUDA;
  }
  return HYMBA_OK;
}

// ---------------------------------------------------------------------------
// Mask bitmap dump (same predicate and tile classification as the kernels).
// ---------------------------------------------------------------------------
__global__ void mask_bits_kernel(int L, int n_meta, int window, int is_global, uint32_t *bits) {
  const int words = (L + 31) / 32;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)L * words) return;
  const int i = int(idx / words), w = int(idx % words);
  uint32_t v = 0;
  for (int t = 0; t < 32; ++t) {
    const int j = w * 32 + t;
    if (j < L && mask_allowed(i, j, n_meta, window, is_global)) v |= 1u << t;
  }
  bits[idx] = v;
}
__global__ void mask_tiles_kernel(int L, int n_meta, int window, int is_global, uint8_t *cls) {
  const int nt = (L + 127) / 128;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= nt * nt) return;
  const int qt = idx / nt, kt = idx % nt;
  cls[idx] = (uint8_t)seq_tile_class(qt, kt, L, n_meta, window, is_global);
}

hymba_status mask_bitmap(int L, int n_meta, int window, int is_global, uint32_t *bits,
                         uint8_t *tile_class, cudaStream_t s) {
  const long long n = (long long)L * ((L + 31) / 32);
  if (n > 0) mask_bits_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(L, n_meta, window, is_global, bits);
  if (tile_class) {
    const int nt = (L + 127) / 128;
    if (nt > 0)
      mask_tiles_kernel<<<(nt * nt + 255) / 256, 256, 0, s>>>(L, n_meta, window, is_global, tile_class);
  }
  note_launch((n > 0 ? 1 : 0) + (tile_class ? 1 : 0));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("mask bitmap launch failed: %s", cudaGetErrorString(e));
    return HYMBA_ERR_CUDA;
  }
  return HYMBA_OK;
}

unsigned take_error_attn() {
  unsigned v = 0, z = 0;
  cudaMemcpyFromSymbol(&v, g_err_attn, sizeof(v));
  if (v) cudaMemcpyToSymbol(g_err_attn, &z, sizeof(z));
  return v;
}

}  // namespace hymba
