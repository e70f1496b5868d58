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
//   warps 4-7, 8-11 : one softmax warpgroup per query tile, one thread per row:
//                row max over S (tcgen05.ld), lazy rescaling of O in TMEM only
//                when the max grows by more than 2^8, exp2, P (bf16) written back
//                into the first 64 columns of its own S (tcgen05.st), from where
//                the P V MMA reads it as its A operand.
// The two query tiles ping-pong: the MMA order per key tile is P V then the next
// S for one query tile, then the same for the other, so while one warpgroup
// computes its softmax the tensor core runs the other tile's MMAs.  Key tiles with no visible pair are
// never loaded; fully visible tiles skip the per-element mask.
//
// fp32 path and decode: CUDA-core kernels (small or bandwidth-bound work).
#include <algorithm>
#include <cstdlib>
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
constexpr int NQ = 2;            // query tiles per work item
constexpr int Q_BYTES = QT * 128;        // 64 bf16 per row
constexpr int K_BYTES = KT * 128;
constexpr int V_BYTES = KT * 256;        // two 64-column boxes
constexpr int P_BYTES = QT * 256;        // O staging of one query tile: two 64-column swizzle atoms
constexpr int OFF_Q = 0;                 // two buffers (this item's and the next one's)
constexpr int OFF_K = OFF_Q + 2 * NQ * Q_BYTES;
constexpr int OFF_V = OFF_K + 2 * K_BYTES;
constexpr int OFF_P = OFF_V + 2 * V_BYTES;  // O staging for the TMA stores
constexpr int OFF_BAR = OFF_P + NQ * P_BYTES;
constexpr int NBAR = 2 * 6 + 3 * NQ + 1 + 2 * NQ;
constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
static_assert(SMEM <= 232448, "attention shared memory");
constexpr int THREADS = 128 + NQ * 128;  // warpgroup 0: TMA + MMA; one softmax warpgroup per query tile
// Register split (setmaxnreg): launch 168 per thread = 64,512; warpgroup 0 drops to 72,
// the softmax warpgroups rise to 216: 128 * 72 + 256 * 216 = 64,512.
constexpr int REG_CTRL = 72;
constexpr int REG_SOFTMAX = 216;
constexpr uint32_t IDESC_S = make_idesc(128, 1, 0, 0);
constexpr uint32_t IDESC_PV = make_idesc(128, 1, 0, 1);
}  // namespace fa

// Class of the (query tile, key tile) pair as the prefill kernel sees it.
__device__ __forceinline__ int fa_tile_class(int qtile, int kt, int L, int q_off, int n_meta, int window,
                                             int is_global) {
  return seq_tile_class(qtile, kt, L, q_off, n_meta, window, is_global);
}
// Key tiles streamed for the query-tile pair (qa, qa+1) (query positions from
// q_off + 128 qa): every tile holding a pair visible from some row of the pair.  The keys visible from rows [i0, i1] are
// [0, min(m, i1+1)) and [i0 - W + 1, i1] (all of [0, i1] for a global layer), so
// the tiles are [0, a_end) followed by [lo, hi].  Same sequence in every role.
struct FaTiles {
  int a_end, lo, hi;
  __device__ __forceinline__ int first() const { return a_end > 0 ? 0 : lo; }
  __device__ __forceinline__ int next(int kt) const { return kt + 1 < a_end ? kt + 1 : max(kt + 1, lo); }
};
__device__ __forceinline__ FaTiles fa_tiles(int qa, int L, int q_off, int n_meta, int window, int is_global) {
  FaTiles t;
  const long long i0 = (long long)q_off + (long long)qa * fa::QT;
  const long long i1 = min((long long)q_off + (long long)(qa + 2) * fa::QT, (long long)L) - 1;
  t.hi = (int)(i1 / fa::KT);
  if (is_global) {
    t.a_end = 0;
    t.lo = 0;
    return t;
  }
  const long long me = min((long long)n_meta, i1 + 1);
  t.a_end = (int)((me + fa::KT - 1) / fa::KT);
  t.lo = (int)(max(0LL, i0 - window + 1) / fa::KT);
  if (t.lo < t.a_end) t.lo = t.a_end;
  return t;
}

// Work item of the persistent kernel: (sequence, head, query-tile pair), heads fastest,
// then pairs from the last (the most key tiles in a causal layer) to the first, then
// sequences: the items running at one time are neighbouring pairs of one sequence with
// all their heads, so a K/V tile is read from DRAM once and then shared through L2 by
// the query heads of its group and by the overlapping windows of neighbouring pairs.
struct FaItem {
  int b, h, qa;  // qa: first query tile of the pair
};
__device__ __forceinline__ FaItem fa_item(long long it, int H, int BH, int npairs) {
  (void)BH;
  const int h = (int)(it % H);
  const long long rest = it / H;
  const int pair = npairs - 1 - (int)(rest % npairs);
  return {(int)(rest / npairs), h, 2 * pair};
}
__device__ __forceinline__ int fa_count(const FaTiles &t) {
  int n = 0;
  for (int kt = t.first(); kt <= t.hi; kt = t.next(kt)) ++n;
  return n;
}

// Visible keys of query position i inside the 128-key tile that starts at key0, as column
// ranges of the tile: [0, hi1) (meta keys) and [lo2, hi2) (the window, up to the query
// itself).  A global layer has hi1 = lo2 = 0.
struct FaCols {
  int hi1, lo2, hi2;
};
__device__ __forceinline__ FaCols fa_cols(long long i, long long key0, int n_meta, int window,
                                          int is_global) {
  const long long meta_end = is_global ? 0 : min((long long)n_meta, i + 1);
  const long long win_lo = is_global ? 0 : max((long long)n_meta, i - window + 1);
  FaCols c;
  c.hi1 = (int)max(0LL, min(128LL, meta_end - key0));
  c.lo2 = (int)max(0LL, min(128LL, win_lo - key0));
  c.hi2 = (int)max(0LL, min(128LL, i + 1 - key0));
  return c;
}
__device__ __forceinline__ uint32_t low_bits(int n) {
  return n <= 0 ? 0u : (n >= 32 ? 0xffffffffu : (1u << n) - 1u);
}
// Keep-mask of the 32 columns col0..col0+31 of a partially visible tile.
__device__ __forceinline__ uint32_t fa_keep32(const FaCols &c, int col0) {
  return low_bits(c.hi1 - col0) | (low_bits(c.hi2 - col0) & ~low_bits(c.lo2 - col0));
}
__device__ __forceinline__ void mask_cols(uint32_t (&v)[32], uint32_t keep) {
#pragma unroll
  for (int e = 0; e < 32; ++e)
    if (!(keep & (1u << e))) v[e] = __float_as_uint(-INFINITY);
}
// Row max over the 128 scores of one row: eight chains of three-input maxima.
__device__ __forceinline__ float row_max128(const uint32_t (&s0)[32], const uint32_t (&s1)[32],
                                            const uint32_t (&s2)[32], const uint32_t (&s3)[32]) {
  float m[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) m[t] = fmaxf(__uint_as_float(s0[t]), __uint_as_float(s0[t + 8]));
#pragma unroll
  for (int t = 0; t < 8; ++t) m[t] = fmax3(m[t], __uint_as_float(s0[t + 16]), __uint_as_float(s0[t + 24]));
#pragma unroll
  for (int e = 0; e < 32; e += 16)
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      m[t] = fmax3(m[t], __uint_as_float(s1[e + t]), __uint_as_float(s1[e + t + 8]));
      m[t] = fmax3(m[t], __uint_as_float(s2[e + t]), __uint_as_float(s2[e + t + 8]));
      m[t] = fmax3(m[t], __uint_as_float(s3[e + t]), __uint_as_float(s3[e + t + 8]));
    }
  return fmaxf(fmax3(m[0], m[1], m[2]), fmax3(fmax3(m[3], m[4], m[5]), m[6], m[7]));
}
// P for 32 keys of a row: exp2(s * scale - m) packed to bf16 pairs; returns the fp32
// sum as a pair of partial sums.  Scale and shift run as packed fp32x2 FMAs; one key
// pair in eight takes its exponentials from the degree-3 polynomial on the FMA pipe
// (relative error 7.5e-5, well inside the bf16 rounding of P) and the others from
// the MUFU.  The kernel is bound by issue more than by the MUFU: on a batch-32 layer
// 0, 1, 2, 3 pairs of eight ran within 2 % of each other (1 fastest) and 4, 5, 6 pairs
// were 6-17 % slower.
constexpr int kPolyPairsOf8 = 1;  // key pairs of every eight on the polynomial
__device__ __forceinline__ float2 p_pack(const uint32_t (&v)[32], uint32_t (&pk)[16], float2 scale2,
                                         float2 nm2) {
  float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    const float2 x = ffma2(make_float2(__uint_as_float(v[e]), __uint_as_float(v[e + 1])), scale2, nm2);
    const float2 p = ((e >> 1) & 7) < kPolyPairsOf8 ? exp2_poly2<3>(x) : make_float2(ex2(x.x), ex2(x.y));
    ls[(e >> 1) & 1] = fadd2(ls[(e >> 1) & 1], p);
    pk[e >> 1] = pack_bf16x2(p.x, p.y);
  }
  return fadd2(ls[0], ls[1]);
}
// Keys c*32 .. c*32+31 of row r into the 128-byte swizzled K-major P tile
// (atom c/2, 16-byte chunks (c%2)*4 .. +3).
__device__ __forceinline__ void p_store(const uint32_t (&pk)[16], int c, int r, uint32_t p_base) {
  const uint32_t atom = p_base + (c >> 1) * (fa::P_BYTES / 2) + r * 128;
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const int chunk = (c & 1) * 4 + t;
    st_shared_v4(atom + ((chunk ^ (r & 7)) << 4), pk[4 * t], pk[4 * t + 1], pk[4 * t + 2],
                 pk[4 * t + 3]);
  }
}

// Persistent: one CTA per SM walks the work items blockIdx.x, + gridDim.x, ...; the
// K/V ring and every per-tile barrier count tiles across item boundaries, so the next
// item's Q and first K/V tiles stream in, and its first S = Q K^T is issued, while the
// current item's last tile is still in the softmax; the softmax warpgroups write the
// finished item's O between its last tile and the next item's first.
__global__ void __launch_bounds__(fa::THREADS, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                       int L, int q_off, int B, int H, int Hkv, int n_meta, int window, int is_global,
                       float scale_log2, int npairs, long long wlim) {
  pdl_wait();
  pdl_trigger();
  using namespace fa;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  uint64_t *q_full = bars + 0, *q_empty = bars + 2;    // [2]: Q buffers
  uint64_t *k_full = bars + 4, *k_empty = bars + 6;    // [2]: K stages
  uint64_t *v_full = bars + 8, *v_empty = bars + 10;   // [2]: V stages
  uint64_t *s_full = bars + 12, *p_full = bars + 14;   // [NQ]: S ready / P written over it
  uint64_t *o_done = bars + 16;                        // [NQ]: P V retired
  uint64_t *drain = bars + 18;
  uint64_t *o_staged = bars + 19, *o_stored = bars + 21;  // [NQ]: O rows staged / stored
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NBAR);

  const int warp = warp_id(), lane = lane_id();
  const int BH = B * H;
  const long long n_items = (long long)BH * npairs;

  if (warp == 0 && lane == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(&q_full[x], 1);
      mbar_init(&q_empty[x], 1);
      mbar_init(&k_full[x], 1);
      mbar_init(&k_empty[x], 1);
      mbar_init(&v_full[x], 1);
      mbar_init(&v_empty[x], 1);
    }
    for (int q = 0; q < NQ; ++q) {
      mbar_init(&s_full[q], 1);
      mbar_init(&p_full[q], 4);
      mbar_init(&o_done[q], 1);
    }
    mbar_init(drain, 1);
    for (int q = 0; q < NQ; ++q) {
      mbar_init(&o_staged[q], 128);
      mbar_init(&o_stored[q], 1);
    }
    fence_barrier_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmO);
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

  if (warp < 4) {
   asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REG_CTRL));
   if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      bool ok = true;
      long long g = 0;  // tiles issued so far (all items)
      uint32_t nq[2] = {0, 0}, nk[2] = {0, 0}, nv[2] = {0, 0};
      int itk = 0;
      for (long long it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++itk) {
        const FaItem w = fa_item(it, H, BH, npairs);
        const int gkv = w.h / (H / Hkv);
        const int qb = itk & 1;
        if (!mbar_wait(&q_empty[qb], ((uint32_t(itk) >> 1) & 1u) ^ 1u, &g_err_attn, wlim)) { ok = false; break; }
        mbar_arrive_expect_tx(&q_full[qb], NQ * Q_BYTES);
        for (int q = 0; q < NQ; ++q)
          tma_load_3d(smem + OFF_Q + (qb * NQ + q) * Q_BYTES, &tmQ, &q_full[qb], w.h * 64, (w.qa + q) * QT, w.b);
        ++nq[qb];
        const FaTiles t = fa_tiles(w.qa, L, q_off, n_meta, window, is_global);
        for (int kt = t.first(); kt <= t.hi; kt = t.next(kt), ++g) {
          const int st = int(g & 1);
          const uint32_t ph = uint32_t(g >> 1) & 1u;
          if (!mbar_wait(&k_empty[st], ph ^ 1u, &g_err_attn, wlim)) { ok = false; break; }
          mbar_arrive_expect_tx(&k_full[st], K_BYTES);
          tma_load_3d(smem + OFF_K + st * K_BYTES, &tmK, &k_full[st], gkv * 64, kt * KT, w.b);
          ++nk[st];
          if (!mbar_wait(&v_empty[st], ph ^ 1u, &g_err_attn, wlim)) { ok = false; break; }
          mbar_arrive_expect_tx(&v_full[st], V_BYTES);
          uint8_t *vdst = smem + OFF_V + st * V_BYTES;
          tma_load_3d(vdst, &tmV, &v_full[st], gkv * 128, kt * KT, w.b);
          tma_load_3d(vdst + V_BYTES / 2, &tmV, &v_full[st], gkv * 128 + 64, kt * KT, w.b);
          ++nv[st];
        }
      }
      if (!ok) {
        for (int x = 0; x < 2; ++x) {
          if (nq[x]) mbar_wait_drain(&q_full[x], (nq[x] - 1) & 1u, &g_err_attn, wlim);
          if (nk[x]) mbar_wait_drain(&k_full[x], (nk[x] - 1) & 1u, &g_err_attn, wlim);
          if (nv[x]) mbar_wait_drain(&v_full[x], (nv[x] - 1) & 1u, &g_err_attn, wlim);
        }
      }
    }
   } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer: one flat walk over the tiles of all items ----------------
      auto issue_S = [&](int q, int st, int qb) {
        const uint32_t qa_ = smem_u32(smem + OFF_Q) + (qb * NQ + q) * Q_BYTES;
        const uint32_t ka = smem_u32(smem + OFF_K + st * K_BYTES);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_bf16_ss(tmem + 256 * q, make_sdesc(qa_ + 32 * k, 16, 1024),
                      make_sdesc(ka + 32 * k, 16, 1024), IDESC_S, k > 0 ? 1u : 0u);
        mma_commit(&s_full[q]);
      };
      // O += P V with P (bf16 pairs) in the first 64 columns of the tile's S
      auto issue_PV = [&](int q, int st, bool acc_prev) {
        const uint32_t va = smem_u32(smem + OFF_V + st * V_BYTES);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bd = make_sdesc(va + kk * 2048, V_BYTES / 2, 1024);
          mma_bf16_ts(tmem + 256 * q + 128, tmem + 256 * q + 8 * kk, bd, IDESC_PV,
                      (acc_prev || kk > 0) ? 1u : 0u);
        }
        mma_commit(&o_done[q]);
      };
      bool ok = true;
      long long it = blockIdx.x;
      int itk = 0;
      if (it < n_items) {
        FaItem w = fa_item(it, H, BH, npairs);
        int n = fa_count(fa_tiles(w.qa, L, q_off, n_meta, window, is_global));
        // S of the first tile
        ok = mbar_wait(&q_full[0], 0, &g_err_attn, wlim) && mbar_wait(&k_full[0], 0, &g_err_attn, wlim);
        if (ok) {
          tc_fence_after();
          for (int q = 0; q < NQ; ++q) issue_S(q, 0, 0);
          mma_commit(&k_empty[0]);
          if (n == 1) mma_commit(&q_empty[0]);
        }
        long long g = 0;  // current tile (all items)
        int j = 0;        // its index within the item
        while (ok) {
          // the next tile: the same item's, or the first of the next item
          const bool same = j + 1 < n;
          const long long it_next = same ? it : it + gridDim.x;
          const bool has_next = it_next < n_items;
          const int qb_next = same ? (itk & 1) : ((itk + 1) & 1);
          int n_next = n;
          const long long g1 = g + 1;
          const int st = int(g & 1), st1 = int(g1 & 1);
          if (has_next) {
            if (!same) {
              const FaItem wn = fa_item(it_next, H, BH, npairs);
              n_next = fa_count(fa_tiles(wn.qa, L, q_off, n_meta, window, is_global));
              if (!mbar_wait(&q_full[qb_next], (uint32_t(itk + 1) >> 1) & 1u, &g_err_attn, wlim)) { ok = false; break; }
            }
            if (!mbar_wait(&k_full[st1], uint32_t(g1 >> 1) & 1u, &g_err_attn, wlim)) { ok = false; break; }
          }
          if (!mbar_wait(&v_full[st], uint32_t(g >> 1) & 1u, &g_err_attn, wlim)) { ok = false; break; }
          // per query tile: P V of this tile, then S of the next one into the same columns
          // (the tensor core runs them in order, so P is read before S overwrites it)
          for (int q = 0; q < NQ && ok; ++q) {
            if (!mbar_wait(&p_full[q], uint32_t(g) & 1u, &g_err_attn, wlim)) { ok = false; break; }
            tc_fence_after();
            issue_PV(q, st, j > 0);
            if (has_next) issue_S(q, st1, qb_next);
          }
          if (!ok) break;
          mma_commit(&v_empty[st]);
          if (!has_next) break;
          mma_commit(&k_empty[st1]);
          // the last S of an item releases its Q buffer once it has run
          if ((same ? j + 1 : 0) == (same ? n : n_next) - 1) mma_commit(&q_empty[qb_next]);
          g = g1;
          if (same) {
            ++j;
          } else {
            it = it_next;
            ++itk;
            n = n_next;
            j = 0;
          }
        }
      }
      if (!ok) {
        // Drain issued MMAs before tensor memory is released.
        mma_commit(drain);
        mbar_wait_drain(drain, 0, &g_err_attn, wlim);
      }
    }
   }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REG_SOFTMAX));
    // ---------------- softmax warpgroups ----------------
    const int q = (warp - 4) >> 2;        // query tile of this warpgroup
    const int quarter = warp & 3;         // TMEM lane quarter
    const int r = quarter * 32 + lane;    // row within the tile
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const uint32_t tS = tmem + 256 * q + lane_off;
    const uint32_t tO = tS + 128;
    const uint32_t p_base = smem_u32(smem + OFF_P + q * P_BYTES);
    bool ok = true;
    long long g = 0;  // tiles done (all items)
    int itk = 0;      // items done
    for (long long it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++itk) {
      const FaItem w = fa_item(it, H, BH, npairs);
      const int qtile = w.qa + q;
      const long long i = (long long)q_off + (long long)qtile * QT + r;  // query position
      const FaTiles tiles = fa_tiles(w.qa, L, q_off, n_meta, window, is_global);
      float m_run = -INFINITY, l_run = 0.f;
      int j = 0;
      for (int kt = tiles.first(); kt <= tiles.hi; kt = tiles.next(kt), ++g, ++j) {
        const int cls = fa_tile_class(qtile, kt, L, q_off, n_meta, window, is_global);  // uniform
        if (!mbar_wait(&s_full[q], uint32_t(g) & 1u, &g_err_attn, wlim)) { ok = false; break; }
        tc_fence_after();
        if (cls == 0) {
          // no visible pair in this tile (or the query tile lies past the sequence):
          // S is not read and P is zero; the running max and sum are unchanged
          uint32_t zero[16];
#pragma unroll
          for (int t = 0; t < 16; ++t) zero[t] = 0u;
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_st16(tS + 16 * c, zero);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_full[q]);
          continue;
        }
        // the whole S row in registers: four loads, one wait
        uint32_t s0[32], s1[32], s2[32], s3[32];
        tmem_ld32(tS, s0);
        tmem_ld32(tS + 32, s1);
        tmem_ld32(tS + 64, s2);
        tmem_ld32(tS + 96, s3);
        tmem_wait_ld();
        if (cls != 1) {
          // partial tile: keep the column ranges of this row
          const FaCols fc = fa_cols(i, (long long)kt * KT, n_meta, window, is_global);
          mask_cols(s0, fa_keep32(fc, 0));
          mask_cols(s1, fa_keep32(fc, 32));
          mask_cols(s2, fa_keep32(fc, 64));
          mask_cols(s3, fa_keep32(fc, 96));
        }
        // row max (scale > 0, so the max commutes with the scaling)
        const float mx = row_max128(s0, s1, s2, s3) * scale_log2;
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
        // P = exp2(s * scale - m) as packed bf16 pairs
        const float nm = (m_run == -INFINITY) ? 0.f : -m_run;
        const float2 nm2 = make_float2(nm, nm), scale2 = make_float2(scale_log2, scale_log2);
        uint32_t pk0[16], pk1[16], pk2[16], pk3[16];
        const float2 ps = fadd2(fadd2(p_pack(s0, pk0, scale2, nm2), p_pack(s1, pk1, scale2, nm2)),
                                fadd2(p_pack(s2, pk2, scale2, nm2), p_pack(s3, pk3, scale2, nm2)));
        l_run += ps.x + ps.y;
        if (__any_sync(0xffffffffu, resc)) {
          // O grows by the new max: rescale it once the previous tile's P V has retired
          if (!mbar_wait(&o_done[q], uint32_t(g - 1) & 1u, &g_err_attn, wlim)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t v[32];
            tmem_ld32(tO + c * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
            tmem_st32(tO + c * 32, v);
          }
        }
        // P over the first 64 columns of S (already in registers; the previous tile's
        // P V read its P before this tile's S was written)
        tmem_st16(tS, pk0);
        tmem_st16(tS + 16, pk1);
        tmem_st16(tS + 32, pk2);
        tmem_st16(tS + 48, pk3);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[q]);
      }
      if (!ok) break;
      // the item's output once its last P V has retired: O / l -> bf16 rows written into
      // this tile's P buffer (idle until the next item's first P) as two 128-byte-swizzled
      // 64-column boxes, then two TMA tile stores (rows past the sequence are not written)
      if (!mbar_wait(&o_done[q], uint32_t(g - 1) & 1u, &g_err_attn, wlim)) { ok = false; break; }
      tc_fence_after();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      {
        uint32_t v[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tO + c * 32, v[c]);
        tmem_wait_ld();
        tc_fence_before();  // O is in registers: the next item's first P V may overwrite it
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(v[c][2 * e]) * inv, __uint_as_float(v[c][2 * e + 1]) * inv);
          p_store(pk, c, r, p_base);
        }
      }
      fence_proxy_async();
      mbar_arrive(&o_staged[q]);
      if (quarter == 0 && lane == 0) {
        // every row of the tile staged -> two stores; the buffer is released once they
        // have read it (released on a failed wait too, so that no thread waits forever)
        if (mbar_wait(&o_staged[q], uint32_t(itk) & 1u, &g_err_attn, wlim)) {
          const uint8_t *stage = smem + OFF_P + q * P_BYTES;
          tma_store_3d(&tmO, stage, w.h * 128, qtile * QT, w.b);
          tma_store_3d(&tmO, stage + P_BYTES / 2, w.h * 128 + 64, qtile * QT, w.b);
          bulk_commit();
          bulk_wait_read();
        }
        mbar_arrive(&o_stored[q]);
      }
      if (!mbar_wait(&o_stored[q], uint32_t(itk) & 1u, &g_err_attn, wlim)) { ok = false; break; }
    }
    if (quarter == 0 && lane == 0) bulk_wait_all();
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
  static DeviceOnce attr_set;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr_set.done(dev)) {
    if (cudaFuncSetAttribute(attn_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) !=
        cudaSuccess) {
      set_error("cudaFuncSetAttribute(attention smem) failed");
      return HYMBA_ERR_CUDA;
    }
    attr_set.mark(dev);
  }
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (sms <= 0) sms = 148;
  CUtensorMap tq, tk, tv, to;
  const uint64_t dq[3] = {(uint64_t)a.H * 64, (uint64_t)a.Lq, (uint64_t)a.B};
  const uint64_t sq[2] = {(uint64_t)a.H * 64 * 2, (uint64_t)a.Lq * a.H * 64 * 2};
  const uint64_t dk[3] = {(uint64_t)a.Hkv * 64, (uint64_t)a.L, (uint64_t)a.B};
  const uint64_t sk[2] = {(uint64_t)a.Hkv * 64 * 2, (uint64_t)a.L * a.Hkv * 64 * 2};
  const uint64_t dv[3] = {(uint64_t)a.Hkv * 128, (uint64_t)a.L, (uint64_t)a.B};
  const uint64_t sv[2] = {(uint64_t)a.Hkv * 128 * 2, (uint64_t)a.L * a.Hkv * 128 * 2};
  const uint32_t box[3] = {64, 128, 1};
  if (!make_tmap(&tq, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, dq, sq, box)) return HYMBA_ERR_CUDA;
  if (!make_tmap(&tk, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, dk, sk, box)) return HYMBA_ERR_CUDA;
  if (!make_tmap(&tv, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, dv, sv, box)) return HYMBA_ERR_CUDA;
  const uint64_t dout[3] = {(uint64_t)a.H * 128, (uint64_t)a.Lq, (uint64_t)a.B};
  const uint64_t sout[2] = {(uint64_t)a.H * 128 * 2, (uint64_t)a.Lq * a.H * 128 * 2};
  if (!make_tmap(&to, a.o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, dout, sout, box)) return HYMBA_ERR_CUDA;
  const int nqt = (a.Lq + QT - 1) / QT;
  const int npairs = (nqt + 1) / 2;
  const long long items = (long long)npairs * a.H * a.B;
  if (items == 0) return HYMBA_OK;
  const unsigned grid = (unsigned)std::min<long long>(items, sms);
  launch_kernel(attn_fwd_tc_kernel, dim3(grid), dim3(THREADS), (size_t)SMEM, s, tq, tk, tv, to, a.L, a.q_off, a.B,
                a.H, a.Hkv, a.n_meta, a.window, a.is_global, a.scale * 1.4426950408889634f, npairs,
                wait_limit_cycles());
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
                                     const T *__restrict__ v, T *__restrict__ o, int B, int L, int q_off,
                                     int Lq, int H, int Hkv, int dqk, int dv, int n_meta, int window,
                                     int is_global, float scale) {
  pdl_wait();
  pdl_trigger();
  const long long wid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= (long long)B * Lq * H) return;
  const int h = int(wid % H);
  const long long bi = wid / H;
  const int row = int(bi % Lq);
  const int i = q_off + row;  // query position
  const int b = int(bi / Lq);
  const int g = h / (H / Hkv);
  const T *qr = q + ((long long)b * Lq + row) * H * dqk + h * dqk;
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
  T *orow = o + ((long long)b * Lq + row) * H * dv + h * dv;
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
  const long long warps = (long long)a.B * a.Lq * a.H;
  const int tpb = 256;
  const long long blocks = (warps * 32 + tpb - 1) / tpb;
  launch_kernel(attn_fwd_simt_kernel<float>, dim3((unsigned)blocks), dim3(tpb), 0, s, (const float *)a.q,
                (const float *)a.k, (const float *)a.v, (float *)a.o, a.B, a.L, a.q_off, a.Lq, a.H, a.Hkv,
                a.dqk, a.dv, a.n_meta, a.window, a.is_global, a.scale);
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
// A CTA takes 64 consecutive slots of one (sequence, kv head) and all the query
// heads of that group, so every K/V byte is read once: the slots' K and V rows are
// contiguous and arrive in shared memory by two bulk copies.  Softmax does not depend
// on key order, so the slots are streamed in memory order: a sliding-window
// store's slots are exactly the visible positions once the context fills the
// window; before that, slot validity masks the unwritten ones.  Partial
// (max, sum, unnormalised output) per chunk, merged by a combine kernel.
// ---------------------------------------------------------------------------
constexpr int DEC_CHUNK = 64;
constexpr int DEC_MAXREP = 8;

__host__ __device__ __forceinline__ long long kv_slot_of(long long p, int n_meta, int window,
                                                         int is_global) {
  if (is_global || p < n_meta) return p;
  return n_meta + (p - n_meta) % window;
}
// Slots a query at `pos` may read: every position of a global store, the meta
// rows and the ring of a sliding-window store.
__host__ __device__ __forceinline__ long long dec_slots(long long pos, int n_meta, int window,
                                                       int is_global) {
  return is_global ? pos + 1 : (long long)n_meta + window;
}
// Whether slot s holds a position visible from `pos`.
__device__ __forceinline__ bool dec_slot_valid(long long s, long long pos, int n_meta, int window,
                                               int is_global) {
  if (is_global) return s <= pos;
  if (s < n_meta) return s <= pos;
  // the most recent position p <= pos stored in ring slot s
  long long back = (pos - s) % window;
  if (back < 0) back += window;
  return pos - back >= n_meta;
}

// Whether key slot s takes part in the decode attention of the query at `pos`: inside the
// slots the query may read and holding a visible position.  Both decode kernels mask with
// this predicate.
__device__ __forceinline__ bool dec_key_valid(long long s, long long nslots, long long pos, int n_meta,
                                              int window, int is_global) {
  return s < nslots && dec_slot_valid(s, pos, n_meta, window, is_global);
}

size_t decode_attn_workspace_floats(int B, int H, int dv, long long pos, int n_meta, int window,
                                    int is_global) {
  const long long nslots = dec_slots(pos, n_meta, window, is_global);
  const long long nsplit = (nslots + DEC_CHUNK - 1) / DEC_CHUNK;
  return (size_t)B * H * nsplit * (dv + 2);
}

template <typename T>
__device__ __forceinline__ void ld_row16(const T *p, float (&v)[16 / sizeof(T)]) {
  uint4 raw = __ldg(reinterpret_cast<const uint4 *>(p));
  if constexpr (sizeof(T) == 2) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __low2float(h[i]);
      v[2 * i + 1] = __high2float(h[i]);
    }
  } else {
    const float *f = reinterpret_cast<const float *>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = f[i];
  }
}

// Bulk copy global -> shared (contiguous, 16-byte aligned, size % 16 == 0), completion
// counted on an mbarrier.  Plain (no multicast) form.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

template <typename T>
__global__ void __launch_bounds__(128)
    attn_decode_partial_kernel(const T *__restrict__ q, const T *__restrict__ kc,
                               const T *__restrict__ vc, float *__restrict__ part, int H, int Hkv,
                               int dqk, int dv, int cap, long long pos, int n_meta, int window,
                               int is_global, float scale_log2, int nsplit, long long wlim) {
  constexpr int V = 16 / sizeof(T);
  extern __shared__ __align__(128) uint8_t dsm[];
  T *sk = reinterpret_cast<T *>(dsm);                               // [DEC_CHUNK][dqk]
  T *sv = reinterpret_cast<T *>(dsm + DEC_CHUNK * dqk * sizeof(T));  // [DEC_CHUNK][dv]
  __shared__ float qs[DEC_MAXREP][128];
  __shared__ float sc[DEC_MAXREP][DEC_CHUNK];
  __shared__ float red[DEC_MAXREP][4];
  __shared__ float stat[DEC_MAXREP][2];
  __shared__ float opart[DEC_MAXREP][128];
  __shared__ uint64_t bar;
  const int split = blockIdx.y;
  const int bg = blockIdx.x;
  const int b = bg / Hkv, g = bg % Hkv;
  const int rep = H / Hkv;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const long long s0 = (long long)split * DEC_CHUNK;
  const long long nslots = dec_slots(pos, n_meta, window, is_global);
  const int ns = (int)min((long long)DEC_CHUNK, nslots - s0);
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0) {
    const uint32_t kb = (uint32_t)(ns * dqk * sizeof(T)), vb = (uint32_t)(ns * dv * sizeof(T));
    mbar_arrive_expect_tx(&bar, kb + vb);
    bulk_load(sk, kc + (((long long)b * Hkv + g) * cap + s0) * dqk, kb, &bar);
    bulk_load(sv, vc + (((long long)b * Hkv + g) * cap + s0) * dv, vb, &bar);
  }
  for (int idx = tid; idx < rep * dqk; idx += 128) {
    const int r = idx / dqk, d = idx % dqk;
    qs[r][d] = Store<T>::to_f(q[(long long)b * H * dqk + (g * rep + r) * dqk + d]) * scale_log2;
  }
  __syncthreads();
  bool ok = mbar_wait(&bar, 0, &g_err_attn, wlim);
  if (!ok && tid == 0) mbar_wait_drain(&bar, 0, &g_err_attn, wlim);  // no copy outlives the CTA
  __syncthreads();
  // scores: two threads per key, each half of the head dim (16-byte pieces read in a
  // rotated order, conflict-free), combined by a shuffle
  {
    const int key = tid >> 1, part_ = tid & 1;
    const bool valid = ok && dec_key_valid(s0 + key, nslots, pos, n_meta, window, is_global);
    float acc[DEC_MAXREP];
#pragma unroll
    for (int r = 0; r < DEC_MAXREP; ++r) acc[r] = 0.f;
    if (valid) {
      const int npc = dqk / V / 2;  // pieces in this thread's half
      const T *kr = sk + key * dqk + part_ * (dqk / 2);
      for (int pc0 = 0; pc0 < npc; ++pc0) {
        const int pc = (pc0 + key) % npc;
        const uint4 raw = *reinterpret_cast<const uint4 *>(kr + pc * V);
        float kv[V];
        if constexpr (sizeof(T) == 2) {
          const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            kv[2 * i] = bf16_lo(w[i]);
            kv[2 * i + 1] = bf16_hi(w[i]);
          }
        } else {
          const float *f = reinterpret_cast<const float *>(&raw);
#pragma unroll
          for (int i = 0; i < 4; ++i) kv[i] = f[i];
        }
        const int d0 = part_ * (dqk / 2) + pc * V;
#pragma unroll
        for (int i = 0; i < V; ++i)
#pragma unroll
          for (int r = 0; r < DEC_MAXREP; ++r)
            if (r < rep) acc[r] = fmaf(qs[r][d0 + i], kv[i], acc[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < DEC_MAXREP; ++r) acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], 1);
    if (part_ == 0) {
#pragma unroll
      for (int r = 0; r < DEC_MAXREP; ++r)
        if (r < rep) sc[r][key] = valid ? acc[r] : -INFINITY;
    }
  }
  __syncthreads();
  // per-head max and sum over the chunk
  for (int r = 0; r < rep; ++r) {
    float m = tid < DEC_CHUNK ? sc[r][tid] : -INFINITY;
#pragma unroll
    for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (lane == 0) red[r][wid] = m;
  }
  __syncthreads();
  if (tid < rep) stat[tid][0] = fmaxf(fmaxf(red[tid][0], red[tid][1]), fmaxf(red[tid][2], red[tid][3]));
  __syncthreads();
  for (int r = 0; r < rep; ++r) {
    const float mr = stat[r][0];
    float p = 0.f;
    if (tid < DEC_CHUNK) {
      p = mr == -INFINITY ? 0.f : ex2(sc[r][tid] - mr);
      sc[r][tid] = p;
    }
    float sum = p;
#pragma unroll
    for (int off = 16; off; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane == 0) red[r][wid] = sum;
  }
  __syncthreads();
  if (tid < rep) stat[tid][1] = (red[tid][0] + red[tid][1]) + (red[tid][2] + red[tid][3]);
  // o[r][d] = sum_t p[r][t] V[t][d]: thread = (column pair, half of the keys)
  const int npair = dv / 2;
  const int half = tid / 64, cp = tid % 64;
  for (int c0 = 0; c0 < npair; c0 += 64) {  // uniform trip count: barriers inside
    const int c = c0 + cp;
    const bool active = ok && c < npair;
    float acc0[DEC_MAXREP], acc1[DEC_MAXREP];
#pragma unroll
    for (int r = 0; r < DEC_MAXREP; ++r) acc0[r] = acc1[r] = 0.f;
    const int t0 = half * (DEC_CHUNK / 2), t1 = active ? min(ns, t0 + DEC_CHUNK / 2) : t0;
    for (int t = t0; t < t1; ++t) {
      float v0, v1;
      if constexpr (sizeof(T) == 2) {
        const __nv_bfloat162 v2 = *reinterpret_cast<const __nv_bfloat162 *>(sv + t * dv + 2 * c);
        v0 = __low2float(v2);
        v1 = __high2float(v2);
      } else {
        const float2 v2 = *reinterpret_cast<const float2 *>(sv + t * dv + 2 * c);
        v0 = v2.x;
        v1 = v2.y;
      }
#pragma unroll
      for (int r = 0; r < DEC_MAXREP; ++r)
        if (r < rep) {
          const float p = sc[r][t];
          acc0[r] = fmaf(p, v0, acc0[r]);
          acc1[r] = fmaf(p, v1, acc1[r]);
        }
    }
    if (half == 1) {
#pragma unroll
      for (int r = 0; r < DEC_MAXREP; ++r)
        if (r < rep) {
          opart[r][2 * cp] = acc0[r];
          opart[r][2 * cp + 1] = acc1[r];
        }
    }
    __syncthreads();
    if (half == 0 && active) {
#pragma unroll
      for (int r = 0; r < DEC_MAXREP; ++r)
        if (r < rep) {
          float *dst = part + (((long long)b * H + g * rep + r) * nsplit + split) * (dv + 2);
          dst[2 + 2 * c] = acc0[r] + opart[r][2 * cp];
          dst[2 + 2 * c + 1] = acc1[r] + opart[r][2 * cp + 1];
        }
    }
    __syncthreads();
  }
  if (tid < rep) {
    float *dst = part + (((long long)b * H + g * rep + tid) * nsplit + split) * (dv + 2);
    dst[0] = stat[tid][0];
    dst[1] = stat[tid][1];
  }
}

// First chunk of every run: a run starts at chunk 0 of a (sequence, kv head) or at the
// first item of a CTA's range.
__host__ __device__ __forceinline__ bool dec_run_start(long long item, int chunk, long long per) {
  return chunk == 0 || item % per == 0;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                          uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// byte offset of 16-byte chunk `ch` (0..7) of row `row` in a 128-byte-swizzled tile
__device__ __forceinline__ uint32_t sw128(int row, int ch) {
  return uint32_t(row * 128 + ((ch ^ (row & 7)) << 4));
}

// ---- bf16 decode attention on the tensor cores (mma.sync m16n8k16) ---------------
// Persistent: the work is the list of 128-slot chunks of every (sequence, kv head), item
// i = (b * Hkv + g) * nchunks + chunk, cut into equal contiguous ranges, one per CTA (two
// CTAs per SM).  A CTA streams its chunks through two shared-memory stages by 3-D TMA
// (128-byte swizzle, rows past the store's capacity read as zero), the next chunk's copy
// in flight while the current one is computed, across (sequence, kv head) boundaries too.
// Eight warps; warp w takes keys 16w..16w+15 of every chunk:
//   S = Q K^T with the query heads of the group in rows 0..rep-1 of a 16-row tile (two
//   8-key n-tiles), an online softmax in registers, then O^T += V^T P^T, in which the
//   value columns fill the 16 MMA rows (eight 16-column m-tiles) and the query heads the
//   8 columns, so no MMA row of the P V product is idle and O takes 32 registers.  The S
//   fragment of a head row (keys 2gc, 2gc+1 of an n-tile) is already the B fragment of
//   P^T, and V^T comes from ldmatrix.trans of the natural [slot][column] tile.
// Where a run of chunks of one (sequence, kv head) ends inside the CTA's range, the eight
// warps' states are merged in shared memory (warps 4..7 into 0..3, then the four) into one
// partial (max, sum, O) per query head, stored at the slot of the run's first chunk; the
// branch fuse kernel merges the run-start slots.
namespace dtc {
constexpr int SLOTS = 128;
constexpr int STAGES = 2;
constexpr int WARPS = 8;
constexpr int THREADS = WARPS * 32;
constexpr int KW = SLOTS / WARPS;  // 16 keys per warp: one k-step of P V
constexpr int K_BYTES = SLOTS * 128;
constexpr int V_BYTES = SLOTS * 256;
constexpr int STAGE = K_BYTES + V_BYTES;
// merge buffer [4][rep][130] floats: warps 4..7 merge into warps 0..3 first
__host__ __device__ constexpr int merge_bytes(int rep) { return 4 * rep * 130 * 4; }
__host__ __device__ constexpr int smem_bytes(int rep) { return STAGES * STAGE + merge_bytes(rep) + 8 * STAGES + 1024; }
constexpr int CTAS_PER_SM = 2;
static_assert(KW == 16, "one 16-key k-step per warp");
}  // namespace dtc

__global__ void __launch_bounds__(dtc::THREADS, 2)
    attn_decode_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                           const __nv_bfloat16 *__restrict__ q, float *__restrict__ part, int H,
                           int Hkv, long long pos, int n_meta, int window, int is_global,
                           float scale_log2, long long n_items, long long per, long long wlim) {
  using namespace dtc;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t *sm = dsm_raw + ((1024 - (smem_u32(dsm_raw) & 1023)) & 1023);
  const int rep = H / Hkv;
  float *mw = reinterpret_cast<float *>(sm + STAGES * STAGE);                             // [4][rep][130]
  uint64_t *full = reinterpret_cast<uint64_t *>(sm + STAGES * STAGE + merge_bytes(rep));  // [STAGES]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gr = lane >> 2, gc = lane & 3;  // mma group row / column pair
  const int h0 = 2 * gc, h1 = 2 * gc + 1;   // the query heads of this lane's O^T columns
  const long long nslots = dec_slots(pos, n_meta, window, is_global);
  const int nchunks = (int)((nslots + SLOTS - 1) / SLOTS);
  const long long i0 = (long long)blockIdx.x * per;
  const long long i1 = min(n_items, i0 + per);
  if (i0 >= i1) return;
  const int nloc = (int)(i1 - i0);
  auto issue = [&](int k) {  // item i0 + k into stage k % STAGES
    const long long it = i0 + k;
    const int bg = (int)(it / nchunks), s0 = (int)(it % nchunks) * SLOTS;
    const int st = k % STAGES;
    uint8_t *dst = sm + st * STAGE;
    mbar_arrive_expect_tx(&full[st], STAGE);
    tma_load_3d(dst, &tmK, &full[st], 0, s0, bg);
    tma_load_3d(dst + K_BYTES, &tmV, &full[st], 0, s0, bg);
    tma_load_3d(dst + K_BYTES + V_BYTES / 2, &tmV, &full[st], 64, s0, bg);
  };
  // The first chunks are requested before the wait for the preceding kernel, up to the
  // chunk that holds this step's slot (written by the step's input projection, which may
  // be the preceding kernel).  Every other slot was written by an earlier step, and when a
  // kernel starts, the kernel two launches before it in the stream has completed.
  const int new_chunk = (int)(kv_slot_of(pos, n_meta, window, is_global) / SLOTS);
  int issued = 0;
  if (tid == 0) {
    for (int st = 0; st < STAGES; ++st) mbar_init(&full[st], 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    for (; issued < min(STAGES, nloc) && (int)((i0 + issued) % nchunks) != new_chunk; ++issued) issue(issued);
  }
  pdl_wait();
  pdl_trigger();
  __syncthreads();
  if (tid == 0)
    for (; issued < min(STAGES, nloc); ++issued) issue(issued);
  float m_run = -INFINITY, l_run = 0.f;  // head gr, over this warp's keys of the run
  float oacc[8][4];  // m-tile mt: [0], [1] = (column 16mt+gr; heads h0, h1), [2], [3] = column +8
  uint32_t qa[4][2];  // Q fragments [k-step][a0a1 / a4a5]; rows 8..15 are zero
  // this warp's (max, sum, O) for the heads below rep into merge slot `slot`
  auto put = [&](int slot) {
    float *base = mw + slot * rep * 130;
    if (gr < rep && gc == 0) {
      base[gr * 130] = m_run;
      base[gr * 130 + 1] = l_run;
    }
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      if (h0 < rep) {
        base[h0 * 130 + 2 + 16 * mt + gr] = oacc[mt][0];
        base[h0 * 130 + 2 + 16 * mt + gr + 8] = oacc[mt][2];
      }
      if (h1 < rep) {
        base[h1 * 130 + 2 + 16 * mt + gr] = oacc[mt][1];
        base[h1 * 130 + 2 + 16 * mt + gr + 8] = oacc[mt][3];
      }
    }
  };
  bool ok = true;
  int k = 0;
  for (; k < nloc; ++k) {
    const long long it = i0 + k;
    const int bg = (int)(it / nchunks), chunk = (int)(it % nchunks);
    const int b = bg / Hkv, g = bg % Hkv;
    if (k == 0 || chunk == 0) {  // a run starts: fresh state, the group's queries
      m_run = -INFINITY;
      l_run = 0.f;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) oacc[mt][e] = 0.f;
      const bool live = gr < rep;
      const uint32_t *qr =
          reinterpret_cast<const uint32_t *>(q + ((long long)b * H + g * rep + (live ? gr : 0)) * 64);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        qa[ks][0] = live ? __ldg(qr + ks * 8 + gc) : 0u;
        qa[ks][1] = live ? __ldg(qr + ks * 8 + 4 + gc) : 0u;
      }
    }
    const int st = k % STAGES;
    ok = mbar_wait(&full[st], uint32_t(k / STAGES) & 1u, &g_err_attn, wlim);
    if (__syncthreads_or(!ok)) { ok = false; break; }
    const uint32_t kb = smem_u32(sm + st * STAGE), vb = kb + K_BYTES;
    const long long s0 = (long long)chunk * SLOTS;
    // ---- S = Q K^T for this warp's 16 keys (two n-tiles of 8) ----
    float sacc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[nt][e] = 0.f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int key = warp * KW + nt * 8 + (lane & 7);
#pragma unroll
      for (int kp = 0; kp < 2; ++kp) {  // two k-steps per ldmatrix.x4
        const int ch = kp * 4 + (lane >> 3);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kb + sw128(key, ch), b0, b1, b2, b3);
        mma16816(sacc[nt], qa[2 * kp][0], 0u, qa[2 * kp][1], 0u, b0, b1);
        mma16816(sacc[nt], qa[2 * kp + 1][0], 0u, qa[2 * kp + 1][1], 0u, b2, b3);
      }
    }
    // ---- online softmax, head gr (values sacc[nt][0..1], keys 8nt + 2gc + {0,1}) ----
    float mx = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int key = warp * KW + nt * 8 + 2 * gc + e;
        const bool valid = dec_key_valid(s0 + key, nslots, pos, n_meta, window, is_global);
        const float x = valid ? sacc[nt][e] * scale_log2 : -INFINITY;
        sacc[nt][e] = x;
        mx = fmaxf(mx, x);
      }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m_run, mx);
    const float mref = m_new == -INFINITY ? 0.f : m_new;
    const float alpha = m_run == -INFINITY ? 0.f : ex2(m_run - mref);
    m_run = m_new;
    const float p00 = ex2(sacc[0][0] - mref), p01 = ex2(sacc[0][1] - mref);
    const float p10 = ex2(sacc[1][0] - mref), p11 = ex2(sacc[1][1] - mref);
    // P^T as the B fragment: b0b1 = keys 2gc, 2gc+1 of head gr, b2b3 = keys 8 + 2gc, 9 + 2gc
    const uint32_t pb0 = pack_bf16x2(p00, p01), pb1 = pack_bf16x2(p10, p11);
    float lsum = (p00 + p01) + (p10 + p11);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
    l_run = fmaf(l_run, alpha, lsum);
    // rescale by the alphas of heads h0, h1 (held by the lanes of rows h0, h1)
    const float al0 = __shfl_sync(0xffffffffu, alpha, h0 * 4), al1 = __shfl_sync(0xffffffffu, alpha, h1 * 4);
    // ---- O^T += V^T P^T: eight m-tiles of 16 value columns, one 16-key k-step ----
    {
      const int j = lane >> 3;  // ldmatrix matrix: keys (j >> 1) * 8.., columns 8 (j & 1)..
      const int key = warp * KW + (j >> 1) * 8 + (lane & 7);
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const int chg = 2 * mt + (j & 1);  // 16-byte chunk of value columns (0..15)
        const uint32_t addr = vb + (chg >> 3) * (V_BYTES / 2) + sw128(key, chg & 7);
        uint32_t a0, a1, a2, a3;
        ldsm_x4_t(addr, a0, a1, a2, a3);
        oacc[mt][0] *= al0;
        oacc[mt][1] *= al1;
        oacc[mt][2] *= al0;
        oacc[mt][3] *= al1;
        mma16816(oacc[mt], a0, a1, a2, a3, pb0, pb1);
      }
    }
    __syncthreads();  // every warp is done with stage st
    if (tid == 0 && issued < nloc) issue(issued++);
    if (chunk == nchunks - 1 || k == nloc - 1) {
      // the run ends: warps 4..7 merge into warps 0..3, then the four into the run-start slot
      if (warp >= 4) put(warp - 4);
      __syncthreads();
      if (warp < 4) {
        const float *base = mw + warp * rep * 130;
        const float m2 = gr < rep ? base[gr * 130] : -INFINITY;
        const float l2 = gr < rep ? base[gr * 130 + 1] : 0.f;
        const float M = fmaxf(m_run, m2);
        const float s1 = m_run == -INFINITY ? 0.f : ex2(m_run - M);
        const float s2 = m2 == -INFINITY ? 0.f : ex2(m2 - M);
        l_run = l_run * s1 + l2 * s2;
        m_run = M;
        const float a10 = __shfl_sync(0xffffffffu, s1, h0 * 4), a11 = __shfl_sync(0xffffffffu, s1, h1 * 4);
        const float a20 = __shfl_sync(0xffffffffu, s2, h0 * 4), a21 = __shfl_sync(0xffffffffu, s2, h1 * 4);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          const float o00 = h0 < rep ? base[h0 * 130 + 2 + 16 * mt + gr] : 0.f;
          const float o02 = h0 < rep ? base[h0 * 130 + 2 + 16 * mt + gr + 8] : 0.f;
          const float o11 = h1 < rep ? base[h1 * 130 + 2 + 16 * mt + gr] : 0.f;
          const float o13 = h1 < rep ? base[h1 * 130 + 2 + 16 * mt + gr + 8] : 0.f;
          oacc[mt][0] = oacc[mt][0] * a10 + o00 * a20;
          oacc[mt][2] = oacc[mt][2] * a10 + o02 * a20;
          oacc[mt][1] = oacc[mt][1] * a11 + o11 * a21;
          oacc[mt][3] = oacc[mt][3] * a11 + o13 * a21;
        }
      }
      __syncthreads();  // warps 0..3 have read the slots they now overwrite
      if (warp < 4) put(warp);
      __syncthreads();
      const int run_chunk = (int)(max(i0, it - chunk) - (it - chunk));  // the run began at item max(i0, it - chunk)
      for (int idx = tid; idx < rep * 130; idx += THREADS) {
        const int r = idx / 130, col = idx % 130;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, mw[(w * rep + r) * 130]);
        float acc = 0.f;
        if (col == 0) {
          acc = M;
        } else {
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const float mw_ = mw[(w * rep + r) * 130];
            if (mw_ != -INFINITY) acc += mw[(w * rep + r) * 130 + col] * ex2(mw_ - M);
          }
        }
        part[(((long long)b * H + g * rep + r) * nchunks + run_chunk) * 130 + col] = acc;
      }
      __syncthreads();  // the merge buffer is reused by the next run
    }
  }
  if (!ok && tid == 0) {
    // copies issued past the failed wait must land before the CTA leaves
    for (int kk = k; kk < issued; ++kk)
      mbar_wait_drain(&full[kk % STAGES], uint32_t(kk / STAGES) & 1u, &g_err_attn, wlim);
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
  for (int s = 0; s < nsplit; ++s) {
    const float ms = base[s * (dv + 2)];
    if (ms != -INFINITY) Lsum += base[s * (dv + 2) + 1] * ex2(ms - M);
  }
  for (int d = threadIdx.x; d < dv; d += blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < nsplit; ++s) {
      const float ms = base[s * (dv + 2)];
      if (ms != -INFINITY) acc += base[s * (dv + 2) + 2 + d] * ex2(ms - M);
    }
    o[(long long)bh * dv + d] = Store<T>::from_f(acc / Lsum);
  }
}

// Merges the run partials of one (sequence, query head): the slots of the chunks that
// start a run of the persistent tensor-core kernel, i.e. chunk 0 and every chunk whose
// item index is a multiple of `per` (the first at per - item0 % per, then every per).
template <typename T>
__global__ void attn_decode_combine_runs_kernel(const float *__restrict__ part, T *__restrict__ o, int H,
                                                int Hkv, int dv, int nchunks, long long per) {
  const int bh = blockIdx.x;
  const int b = bh / H, h = bh % H, g = h / (H / Hkv);
  const long long item0 = ((long long)b * Hkv + g) * nchunks;
  const long long r0 = item0 % per;
  const long long cfirst = r0 == 0 ? per : per - r0;  // first run start after chunk 0
  const float *base = part + (long long)bh * nchunks * (dv + 2);
  auto slot = [&](long long k) { return k == 0 ? 0LL : cfirst + (k - 1) * per; };
  long long nruns = 1;
  if (cfirst < nchunks) nruns += 1 + (nchunks - 1 - cfirst) / per;
  float M = -INFINITY;
  for (long long k = 0; k < nruns; ++k) M = fmaxf(M, base[slot(k) * (dv + 2)]);
  float Lsum = 0.f;
  for (long long k = 0; k < nruns; ++k) {
    const float ms = base[slot(k) * (dv + 2)];
    if (ms != -INFINITY) Lsum += base[slot(k) * (dv + 2) + 1] * ex2(ms - M);
  }
  for (int d = threadIdx.x; d < dv; d += blockDim.x) {
    float acc = 0.f;
    for (long long k = 0; k < nruns; ++k) {
      const float ms = base[slot(k) * (dv + 2)];
      if (ms != -INFINITY) acc += base[slot(k) * (dv + 2) + 2 + d] * ex2(ms - M);
    }
    o[(long long)bh * dv + d] = Store<T>::from_f(acc / Lsum);
  }
}

hymba_status attention_decode(DecodeAttnArgs &a, hymba_dtype dt, cudaStream_t s) {
  a.nchunks_out = 0;
  const int rep = a.H / a.Hkv;
  const int V = dt == HYMBA_BF16 ? 8 : 4;
  if (rep > DEC_MAXREP || a.dqk > 128 || a.dqk % V || a.dv > 256 || a.dv % 2) {
    set_error("decode attention supports H/Hkv <= 8, head_dim_qk <= 128 (multiple of 16 bytes), "
              "even head_dim_v <= 256");
    return HYMBA_ERR_UNSUPPORTED;
  }
  const long long nslots = dec_slots(a.pos, a.n_meta, a.window, a.is_global);
  const int nsplit = (int)((nslots + DEC_CHUNK - 1) / DEC_CHUNK);
  dim3 grid(a.B * a.Hkv, nsplit);
  const float sl2 = a.scale * 1.4426950408889634f;
  const int esz = dt == HYMBA_BF16 ? 2 : 4;
  const int dsmem = DEC_CHUNK * (a.dqk + a.dv) * esz;
  {
    static DeviceOnce attr_set;
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr_set.done(dev)) {
      const int most = DEC_CHUNK * (128 + 256) * 4;
      if (cudaFuncSetAttribute(attn_decode_partial_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               most) != cudaSuccess ||
          cudaFuncSetAttribute(attn_decode_partial_kernel<__nv_bfloat16>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, most) != cudaSuccess) {
        set_error("cudaFuncSetAttribute(decode attention smem) failed");
        return HYMBA_ERR_CUDA;
      }
      attr_set.mark(dev);
    }
  }
  if (dt == HYMBA_BF16 && a.dqk == 64 && a.dv == 128) {
    static DeviceOnce attr_tc;
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr_tc.done(dev)) {
      if (cudaFuncSetAttribute(attn_decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               dtc::smem_bytes(DEC_MAXREP)) != cudaSuccess) {
        set_error("cudaFuncSetAttribute(decode attention smem) failed");
        return HYMBA_ERR_CUDA;
      }
      attr_tc.mark(dev);
    }
    CUtensorMap tk, tv;
    const uint64_t dk[3] = {64, (uint64_t)a.cap, (uint64_t)a.B * a.Hkv};
    const uint64_t sk[2] = {64 * 2, (uint64_t)a.cap * 64 * 2};
    const uint64_t dvv[3] = {128, (uint64_t)a.cap, (uint64_t)a.B * a.Hkv};
    const uint64_t svv[2] = {128 * 2, (uint64_t)a.cap * 128 * 2};
    const uint32_t box[3] = {64, (uint32_t)dtc::SLOTS, 1};
    if (!make_tmap(&tk, a.k_cache, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, dk, sk, box)) return HYMBA_ERR_CUDA;
    if (!make_tmap(&tv, a.v_cache, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, dvv, svv, box)) return HYMBA_ERR_CUDA;
    // equal contiguous ranges of the (sequence, kv head, chunk) items, two CTAs per SM
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
    const int nchunks = (int)((nslots + dtc::SLOTS - 1) / dtc::SLOTS);
    const long long n_items = (long long)a.B * a.Hkv * nchunks;
    const long long grid_tc = std::min<long long>(n_items, (long long)dtc::CTAS_PER_SM * sms);
    const long long per = (n_items + grid_tc - 1) / grid_tc;
    launch_kernel(attn_decode_tc_kernel, dim3((unsigned)((n_items + per - 1) / per)), dim3(dtc::THREADS),
                  (size_t)dtc::smem_bytes(rep), s, tk, tv, (const __nv_bfloat16 *)a.q, a.partial, a.H, a.Hkv,
                  (long long)a.pos, a.n_meta, a.window, a.is_global, sl2, n_items, per, wait_limit_cycles());
    if (a.fuse_later) {
      a.nchunks_out = nchunks;
      a.per_out = per;
      note_launch(1);
    } else {
      attn_decode_combine_runs_kernel<__nv_bfloat16><<<a.B * a.H, 128, 0, s>>>(
          a.partial, (__nv_bfloat16 *)a.o, a.H, a.Hkv, a.dv, nchunks, per);
      note_launch(2);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
      set_error("decode attention launch failed: %s", cudaGetErrorString(e));
      return HYMBA_ERR_CUDA;
    }
    return HYMBA_OK;
  } else if (dt == HYMBA_BF16) {
    attn_decode_partial_kernel<__nv_bfloat16><<<grid, 128, dsmem, s>>>(
        (const __nv_bfloat16 *)a.q, (const __nv_bfloat16 *)a.k_cache, (const __nv_bfloat16 *)a.v_cache,
        a.partial, a.H, a.Hkv, a.dqk, a.dv, a.cap, a.pos, a.n_meta, a.window, a.is_global, sl2, nsplit,
        wait_limit_cycles());
    attn_decode_combine_kernel<__nv_bfloat16><<<a.B * a.H, 128, 0, s>>>(
        a.partial, (__nv_bfloat16 *)a.o, a.H, a.dv, nsplit);
  } else {
    attn_decode_partial_kernel<float><<<grid, 128, dsmem, s>>>(
        (const float *)a.q, (const float *)a.k_cache, (const float *)a.v_cache, a.partial, a.H,
        a.Hkv, a.dqk, a.dv, a.cap, a.pos, a.n_meta, a.window, a.is_global, sl2, nsplit, wait_limit_cycles());
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
// Meta rows of K/V into every sequence (prefill from a precomputed meta cache)
// ---------------------------------------------------------------------------
__global__ void kv_broadcast_kernel(const uint4 *__restrict__ src, uint4 *__restrict__ dst, int B,
                                    long long seq_vecs, long long meta_vecs) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)B * meta_vecs) return;
  const long long b = i / meta_vecs, r = i - b * meta_vecs;
  dst[b * seq_vecs + r] = __ldg(src + r);
}

hymba_status kv_broadcast_meta(const KvBroadcastArgs &a, hymba_dtype dt, cudaStream_t s) {
  const int es = dt == HYMBA_BF16 ? 2 : 4;
  const void *src[2] = {a.k_meta, a.v_meta};
  void *dst[2] = {a.k_seq, a.v_seq};
  const int width[2] = {a.kw, a.vw};
  for (int t = 0; t < 2; ++t) {
    const long long row_bytes = (long long)width[t] * es;  // a multiple of 16 (validated by the caller)
    const long long meta_vecs = (long long)a.m * row_bytes / 16, seq_vecs = (long long)a.L * row_bytes / 16;
    const long long n = (long long)a.B * meta_vecs;
    if (n == 0) continue;
    kv_broadcast_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(
        reinterpret_cast<const uint4 *>(src[t]), reinterpret_cast<uint4 *>(dst[t]), a.B, seq_vecs, meta_vecs);
    note_launch(1);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("meta K/V broadcast launch failed: %s", cudaGetErrorString(e));
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
  pdl_wait();
  pdl_trigger();
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
    launch_kernel(kv_emit_kernel<__nv_bfloat16>, dim3((unsigned)blocks), block, 0, s,
                  (const __nv_bfloat16 *)a.k_seq, (const __nv_bfloat16 *)a.v_seq, (__nv_bfloat16 *)a.k_cache,
                  (__nv_bfloat16 *)a.v_cache, a.B, a.L, a.Hkv, a.dqk, a.dv, a.cap, a.n_meta, a.window,
                  a.is_global, n_keep, meta_keep, start);
  else
    launch_kernel(kv_emit_kernel<float>, dim3((unsigned)blocks), block, 0, s, (const float *)a.k_seq,
                  (const float *)a.v_seq, (float *)a.k_cache, (float *)a.v_cache, a.B, a.L, a.Hkv, a.dqk,
                  a.dv, a.cap, a.n_meta, a.window, a.is_global, n_keep, meta_keep, start);
  note_launch(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("kv emit launch failed: %s", cudaGetErrorString(e));
    return HYMBA_ERR_CUDA;
  }
  return HYMBA_OK;
}

// ---------------------------------------------------------------------------
// Mask dumps for bit-exact checks, produced by the kernels' own masking code.
// ---------------------------------------------------------------------------
// Tensor-core prefill kernel: a key of row i is visible iff its 128-key tile is among the
// tiles fa_tiles() streams for the row's query-tile pair, the tile is not skipped by its
// class, and, in a partially visible tile, its column is in the keep-mask the softmax
// applies.  One thread per (row, 32-key word).
__global__ void mask_bits_tc_kernel(int L, int n_meta, int window, int is_global, uint32_t *bits) {
  const int words = (L + 31) / 32;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)L * words) return;
  const int i = int(idx / words), w = int(idx % words);
  const int qtile = i / fa::QT, kt = (w * 32) / fa::KT;
  const FaTiles t = fa_tiles(qtile & ~1, L, 0, n_meta, window, is_global);
  bool streamed = false;
  for (int k = t.first(); k <= t.hi; k = t.next(k)) streamed |= (k == kt);
  uint32_t v = 0;
  if (streamed) {
    const int cls = fa_tile_class(qtile, kt, L, 0, n_meta, window, is_global);
    if (cls == 1) v = 0xffffffffu;
    else if (cls == 2) v = fa_keep32(fa_cols(i, (long long)kt * fa::KT, n_meta, window, is_global),
                                     (w * 32) % fa::KT);
  }
  bits[idx] = v;
}
// CUDA-core (fp32) prefill kernel: the per-pair predicate it evaluates.
__global__ void mask_bits_simt_kernel(int L, int n_meta, int window, int is_global, uint32_t *bits) {
  const int words = (L + 31) / 32;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)L * words) return;
  const int i = int(idx / words), w = int(idx % words);
  uint32_t v = 0;
  for (int t = 0; t < 32; ++t) {
    const int j = w * 32 + t;
    if (j < L && j <= i && mask_allowed(i, j, n_meta, window, is_global)) v |= 1u << t;
  }
  bits[idx] = v;
}
__global__ void mask_tiles_kernel(int L, int n_meta, int window, int is_global, uint8_t *cls) {
  const int nt = (L + 127) / 128;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= nt * nt) return;
  const int qt = idx / nt, kt = idx % nt;
  cls[idx] = (uint8_t)fa_tile_class(qt, kt, L, 0, n_meta, window, is_global);
}
// Decode kernels: bit s of the dump is set iff slot s takes part (dec_key_valid).
__global__ void decode_mask_kernel(long long pos, int n_meta, int window, int is_global, int capacity,
                                   uint32_t *bits) {
  const int words = (capacity + 31) / 32;
  const int w = blockIdx.x * blockDim.x + threadIdx.x;
  if (w >= words) return;
  const long long nslots = dec_slots(pos, n_meta, window, is_global);
  uint32_t v = 0;
  for (int e = 0; e < 32; ++e) {
    const long long s = (long long)w * 32 + e;
    if (s < capacity && dec_key_valid(s, nslots, pos, n_meta, window, is_global)) v |= 1u << e;
  }
  bits[w] = v;
}

hymba_status mask_bitmap(int L, int n_meta, int window, int is_global, int path, uint32_t *bits,
                         uint8_t *tile_class, cudaStream_t s) {
  const long long n = (long long)L * ((L + 31) / 32);
  if (n > 0) {
    if (path == 0)
      mask_bits_tc_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(L, n_meta, window, is_global, bits);
    else
      mask_bits_simt_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(L, n_meta, window, is_global, bits);
  }
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

hymba_status decode_mask(long long pos, int n_meta, int window, int is_global, int capacity,
                         uint32_t *bits, cudaStream_t s) {
  const int words = (capacity + 31) / 32;
  decode_mask_kernel<<<(words + 127) / 128, 128, 0, s>>>(pos, n_meta, window, is_global, capacity, bits);
  note_launch(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("decode mask launch failed: %s", cudaGetErrorString(e));
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
