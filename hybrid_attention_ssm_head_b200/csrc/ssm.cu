// SSM heads of the hybrid-head layer (Hymba §2.1 Eq. 2, "we adopt Mamba"):
//   u = SiLU(causal depthwise conv_K(x_ssm) + b)
//   h_t = exp(delta_t A) * h_{t-1} + delta_t B_t u_t,   y_t = C_t . h_t + D u_t
//   y_ssm = y * SiLU(z)
// [delta, B, C] come from the projection GEMMs; A = -exp(A_log).
//
// Scan layout: one thread per (sequence, channel) carrying the d_state = 16
// states in registers; B_t and C_t (shared by all channels of a sequence) are
// staged through shared memory 32 steps at a time.  When there are too few
// (sequence, channel) pairs to fill the GPU, time is split into chunks:
// pass 1 scans each chunk from zero and records its end state and sum of
// delta (the chunk's decay is exp(A * sum delta)); pass 2 chains the chunk
// start states; pass 3 rescans each chunk from its true start and writes y.
// The exponentials run on the MUFU (ex2.approx) with A pre-scaled by log2(e).
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace hymba {

constexpr int kStates = 16;
constexpr int kScanTB = 32;

__device__ __forceinline__ float ex2f_(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------------------
// causal conv + SiLU (prefill)
// ---------------------------------------------------------------------------
template <typename T>
struct Vec16 {
  static constexpr int N = 16 / sizeof(T);
};

template <typename T>
__device__ __forceinline__ void load_vec(const T *p, float (&v)[Vec16<T>::N]) {
  uint4 raw = *reinterpret_cast<const uint4 *>(p);
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
template <typename T>
__device__ __forceinline__ void store_vec(T *p, const float (&v)[Vec16<T>::N]) {
  uint4 raw;
  if constexpr (sizeof(T) == 2) {
    uint32_t *w = reinterpret_cast<uint32_t *>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
  } else {
    float *f = reinterpret_cast<float *>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) f[i] = v[i];
  }
  *reinterpret_cast<uint4 *>(p) = raw;
}

constexpr int kConvTB = 8;

// One thread: VEC channels x kConvTB rows.  The kConvTB + 3 input rows it needs are
// loaded up front (16-byte vectors, coalesced across the warp) so that all loads
// are in flight together.
template <typename T>
__global__ void __launch_bounds__(128) conv_silu_kernel(ConvArgs a) {
  constexpr int V = Vec16<T>::N;
  constexpr int NR = kConvTB + 3;
  const int nvec = a.E / V;
  const int tblocks = (a.L + kConvTB - 1) / kConvTB;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)a.B * tblocks * nvec) return;
  const int cv = int(idx % nvec);
  const long long rest = idx / nvec;
  const int tb = int(rest % tblocks);
  const int b = int(rest / tblocks);
  const int c0 = cv * V;
  const int K = a.K;
  const T *x = reinterpret_cast<const T *>(a.x);
  T *u = reinterpret_cast<T *>(a.u);
  const int t0 = tb * kConvTB;
  // raw[r] = x[t0 - 3 + r] (zero outside the sequence)
  uint4 raw[NR];
#pragma unroll
  for (int r = 0; r < NR; ++r) {
    const int t = t0 - 3 + r;
    if (t >= 0 && t < a.L)
      raw[r] = __ldg(reinterpret_cast<const uint4 *>(x + ((long long)b * a.L + t) * a.ld_x + c0));
    else
      raw[r] = make_uint4(0, 0, 0, 0);
  }
  float w[4][V], bias[V];
#pragma unroll
  for (int i = 0; i < V; ++i) {
    bias[i] = a.bias[c0 + i];
#pragma unroll
    for (int k = 0; k < 4; ++k) w[k][i] = k < K ? a.w[(c0 + i) * K + k] : 0.f;
  }
  auto val = [&](int r, int i) -> float {
    if constexpr (sizeof(T) == 2) {
      const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&raw[r]);
      return (i & 1) ? __high2float(h[i >> 1]) : __low2float(h[i >> 1]);
    } else {
      return reinterpret_cast<const float *>(&raw[r])[i];
    }
  };
#pragma unroll
  for (int tt = 0; tt < kConvTB; ++tt) {
    const int t = t0 + tt;
    if (t >= a.L) break;
    float o[V];
#pragma unroll
    for (int i = 0; i < V; ++i) {
      // tap k multiplies x[t - (K-1) + k] = raw[tt + 3 - (K-1) + k]
      float acc = bias[i];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (k < K) acc = fmaf(w[k][i], val(tt + 4 - K + k, i), acc);
      o[i] = silu_f(acc);
    }
    store_vec<T>(u + ((long long)b * a.L + t) * a.E + c0, o);
  }
  if (a.conv_state && t0 + kConvTB >= a.L) {
    // the last K-1 rows of x, oldest first: x[L-K+1 .. L-1] = raw[L-K+1 - t0 + 3 ..]
    T *cs = reinterpret_cast<T *>(a.conv_state);
    for (int r = 0; r < K - 1; ++r) {
      const int rr = a.L - (K - 1) + r - t0 + 3;
      float v[V];
#pragma unroll
      for (int i = 0; i < V; ++i) v[i] = (rr >= 0 && rr < NR) ? val(rr, i) : 0.f;
      store_vec<T>(cs + ((long long)b * (K - 1) + r) * a.E + c0, v);
    }
  }
}

hymba_status conv_silu(const ConvArgs &a, hymba_dtype dt, cudaStream_t s) {
  const int V = dt == HYMBA_BF16 ? 8 : 4;
  const long long n = (long long)a.B * ((a.L + kConvTB - 1) / kConvTB) * (a.E / V);
  if (n == 0) return HYMBA_OK;
  const unsigned blocks = (unsigned)((n + 127) / 128);
  if (dt == HYMBA_BF16)
    conv_silu_kernel<__nv_bfloat16><<<blocks, 128, 0, s>>>(a);
  else
    conv_silu_kernel<float><<<blocks, 128, 0, s>>>(a);
  note_launch(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("conv launch failed: %s", cudaGetErrorString(e));
    return HYMBA_ERR_CUDA;
  }
  return HYMBA_OK;
}

// ---------------------------------------------------------------------------
// decode conv: one new row per sequence, conv window kept in conv_state
// ---------------------------------------------------------------------------
template <typename T>
__global__ void decode_conv_kernel(DecodeConvArgs a) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)a.B * a.E) return;
  const int c = int(idx % a.E), b = int(idx / a.E);
  const int K = a.K;
  T *cs = reinterpret_cast<T *>(a.conv_state);
  float win[4];
  for (int r = 0; r < K - 1; ++r) win[r] = Store<T>::to_f(cs[((long long)b * (K - 1) + r) * a.E + c]);
  const float x = Store<T>::to_f(reinterpret_cast<const T *>(a.x)[(long long)b * a.ld_x + c]);
  win[K - 1] = x;
  float acc = a.bias[c];
  for (int k = 0; k < K; ++k) acc = fmaf(a.w[c * K + k], win[k], acc);
  reinterpret_cast<T *>(a.u)[(long long)b * a.E + c] = Store<T>::from_f(silu_f(acc));
  for (int r = 0; r < K - 1; ++r) cs[((long long)b * (K - 1) + r) * a.E + c] = Store<T>::from_f(win[r + 1]);
}

hymba_status decode_conv(const DecodeConvArgs &a, hymba_dtype dt, cudaStream_t s) {
  const long long n = (long long)a.B * a.E;
  const unsigned blocks = (unsigned)((n + 255) / 256);
  if (dt == HYMBA_BF16)
    decode_conv_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(a);
  else
    decode_conv_kernel<float><<<blocks, 256, 0, s>>>(a);
  note_launch(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("decode conv launch failed: %s", cudaGetErrorString(e));
    return HYMBA_ERR_CUDA;
  }
  return HYMBA_OK;
}

// ---------------------------------------------------------------------------
// selective scan
// ---------------------------------------------------------------------------
// mode 0: scan from the chunk's start state and write y (and the final state);
// mode 1: scan from zero, record the chunk's end state and sum of delta.
template <typename T>
__global__ void __launch_bounds__(128)
    scan_kernel(ScanArgs a, int chunks, int Tc, int mode, const float *__restrict__ hstart,
                float *__restrict__ hend, float *__restrict__ dsum_out) {
  __shared__ float sbc[kScanTB][2 * kStates];
  const int E = a.E;
  const int cblocks = E / blockDim.x;
  const int c = (blockIdx.x % cblocks) * blockDim.x + threadIdx.x;
  const int rest = blockIdx.x / cblocks;
  const int k = rest % chunks;
  const int b = rest / chunks;
  const int t0 = k * Tc, t1 = min(a.L, t0 + Tc);
  const T *u = reinterpret_cast<const T *>(a.u);
  const T *dl = reinterpret_cast<const T *>(a.delta);
  const T *z = reinterpret_cast<const T *>(a.z);
  T *y = reinterpret_cast<T *>(a.y);

  float A2[kStates], h[kStates];
#pragma unroll
  for (int n = 0; n < kStates; ++n) A2[n] = -__expf(a.a_log[c * kStates + n]) * 1.4426950408889634f;
  const long long sidx = (((long long)b * chunks + k) * E + c) * kStates;
  if (mode == 0 && chunks > 1) {
#pragma unroll
    for (int n = 0; n < kStates; ++n) h[n] = hstart[sidx + n];
  } else if (mode == 0 && a.h_in) {
#pragma unroll
    for (int n = 0; n < kStates; ++n) h[n] = a.h_in[((long long)b * E + c) * kStates + n];
  } else {
#pragma unroll
    for (int n = 0; n < kStates; ++n) h[n] = 0.f;
  }
  const float Dc = a.d_skip[c];
  float dsum = 0.f;
  for (int tb = t0; tb < t1; tb += kScanTB) {
    const int nt = min(kScanTB, t1 - tb);
    __syncthreads();
    for (int e = threadIdx.x; e < nt * 2 * kStates; e += blockDim.x) {
      const int tt = e / (2 * kStates), j = e % (2 * kStates);
      sbc[tt][j] = a.bc[((long long)b * a.L + tb + tt) * a.ld_bc + a.bc_col + j];
    }
    __syncthreads();
#pragma unroll 2
    for (int tt = 0; tt < nt; ++tt) {
      const long long row = (long long)b * a.L + tb + tt;
      const float d = Store<T>::to_f(dl[row * E + c]);
      const float uu = Store<T>::to_f(u[row * E + c]);
      const float du = d * uu;
      float acc = 0.f;
#pragma unroll
      for (int n = 0; n < kStates; ++n) {
        const float dA = ex2f_(d * A2[n]);
        h[n] = fmaf(dA, h[n], du * sbc[tt][n]);
        acc = fmaf(sbc[tt][kStates + n], h[n], acc);
      }
      if (mode == 0) {
        acc = fmaf(Dc, uu, acc);
        const float zz = Store<T>::to_f(z[row * a.ld_z + c]);
        y[row * E + c] = Store<T>::from_f(acc * silu_f(zz));
      } else {
        dsum += d;
      }
    }
  }
  if (mode == 1) {
#pragma unroll
    for (int n = 0; n < kStates; ++n) hend[sidx + n] = h[n];
    dsum_out[((long long)b * chunks + k) * E + c] = dsum;
  } else if (k == chunks - 1 && a.h_out) {
#pragma unroll
    for (int n = 0; n < kStates; ++n) a.h_out[((long long)b * E + c) * kStates + n] = h[n];
  }
}

// Chains chunk start states: H_0 = h_in (or 0); H_{k+1} = exp(A * dsum_k) H_k + hend_k.
__global__ void scan_combine_kernel(const float *__restrict__ a_log, const float *__restrict__ h_in,
                                    const float *__restrict__ hend, const float *__restrict__ dsum,
                                    float *__restrict__ hstart, int B, int E, int chunks) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)B * E) return;
  const int c = int(idx % E), b = int(idx / E);
  float A2[kStates], H[kStates];
#pragma unroll
  for (int n = 0; n < kStates; ++n) {
    A2[n] = -__expf(a_log[c * kStates + n]) * 1.4426950408889634f;
    H[n] = h_in ? h_in[((long long)b * E + c) * kStates + n] : 0.f;
  }
  for (int k = 0; k < chunks; ++k) {
    const long long sidx = (((long long)b * chunks + k) * E + c) * kStates;
    const float ds = dsum[((long long)b * chunks + k) * E + c];
#pragma unroll
    for (int n = 0; n < kStates; ++n) {
      hstart[sidx + n] = H[n];
      H[n] = fmaf(ex2f_(A2[n] * ds), H[n], hend[sidx + n]);
    }
  }
}

static int scan_chunks(int B, int L, int E) {
  // enough (sequence, channel, chunk) threads to fill the GPU a couple of times;
  // chunking costs a second pass of exponentials, so stay at 1 when possible.
  const long long target = 2LL * 148 * 512;
  const long long pairs = (long long)B * E;
  if (pairs >= target / 2) return 1;
  long long c = (target + pairs - 1) / pairs;
  const long long maxc = std::max(1, L / 64);
  return (int)std::max(1LL, std::min(c, maxc));
}

size_t scan_workspace_floats(int B, int L, int E, int N, int *chunks_out) {
  const int ch = scan_chunks(B, L, E);
  if (chunks_out) *chunks_out = ch;
  if (ch == 1) return 0;
  return (size_t)B * ch * E * (2 * N + 1);
}

static int scan_block(int E) {
  if (E % 128 == 0) return 128;
  if (E % 64 == 0) return 64;
  return 32;
}

hymba_status selective_scan(const ScanArgs &a, hymba_dtype dt, cudaStream_t s) {
  int chunks = 1;
  scan_workspace_floats(a.B, a.L, a.E, a.N, &chunks);
  const int Tc = (a.L + chunks - 1) / chunks;
  const int bs = scan_block(a.E);
  const unsigned blocks = (unsigned)((long long)a.B * chunks * (a.E / bs));
  float *hend = nullptr, *hstart = nullptr, *dsum = nullptr;
  if (chunks > 1) {
    const size_t st = (size_t)a.B * chunks * a.E * a.N;
    hend = a.chunk_ws;
    hstart = hend + st;
    dsum = hstart + st;
  }
  auto launch = [&](int mode) {
    if (dt == HYMBA_BF16)
      scan_kernel<__nv_bfloat16><<<blocks, bs, 0, s>>>(a, chunks, Tc, mode, hstart, hend, dsum);
    else
      scan_kernel<float><<<blocks, bs, 0, s>>>(a, chunks, Tc, mode, hstart, hend, dsum);
  };
  if (chunks > 1) {
    launch(1);
    const long long n = (long long)a.B * a.E;
    scan_combine_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(a.a_log, a.h_in, hend, dsum,
                                                                    hstart, a.B, a.E, chunks);
  }
  launch(0);
  note_launch(chunks > 1 ? 3 : 1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("scan launch failed: %s", cudaGetErrorString(e));
    return HYMBA_ERR_CUDA;
  }
  return HYMBA_OK;
}

}  // namespace hymba
