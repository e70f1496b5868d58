// Fusion of the two branches (Hymba §2.1 Eq. 3): each branch output is
// RMS-normalised over its d_inner channels, re-scaled per channel by beta and
// the two are averaged:  f = (beta_1 * o / rms(o) + beta_2 * y / rms(y)) / 2.
// One CTA per token row; 16-byte vector loads held (packed) in registers across
// the row reduction, so each input is read once.
#include "common.cuh"
#include "kernels.h"

namespace hymba {

template <typename T>
__device__ __forceinline__ void ld16(const T *p, float (&v)[16 / sizeof(T)]) {
  uint4 raw = __ldg(reinterpret_cast<const uint4 *>(p));
  if constexpr (sizeof(T) == 2) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = bf16_lo(w[i]);
      v[2 * i + 1] = bf16_hi(w[i]);
    }
  } else {
    const float *f = reinterpret_cast<const float *>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = f[i];
  }
}

template <typename T>
__device__ __forceinline__ void unpack16(const uint4 &raw, float (&v)[16 / sizeof(T)]) {
  if constexpr (sizeof(T) == 2) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = bf16_lo(w[i]);
      v[2 * i + 1] = bf16_hi(w[i]);
    }
  } else {
    v[0] = __uint_as_float(raw.x);
    v[1] = __uint_as_float(raw.y);
    v[2] = __uint_as_float(raw.z);
    v[3] = __uint_as_float(raw.w);
  }
}

// Single read: each of the 128 threads keeps up to NV 16-byte vectors of both
// branches in registers across the block reduction, as raw (packed) words, so that
// more rows fit on an SM; they are unpacked again for the output pass.
template <typename T, int NV>
__global__ void __launch_bounds__(128) fuse_kernel(FuseArgs a) {
  constexpr int V = 16 / sizeof(T);
  __shared__ float red[2][4];
  const long long row = blockIdx.x;
  const T *o = reinterpret_cast<const T *>(a.o) + row * a.E;
  const T *y = reinterpret_cast<const T *>(a.y) + row * a.E;
  T *f = reinterpret_cast<T *>(a.f) + row * a.E;
  uint4 ro_[NV], ry_[NV];
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int c = (threadIdx.x + j * 128) * V;
    if (c < a.E) {
      ro_[j] = __ldg(reinterpret_cast<const uint4 *>(o + c));
      ry_[j] = __ldg(reinterpret_cast<const uint4 *>(y + c));
    }
  }
  float so = 0.f, sy = 0.f;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int c = (threadIdx.x + j * 128) * V;
    if (c < a.E) {
      float vo[V], vy[V];
      unpack16<T>(ro_[j], vo);
      unpack16<T>(ry_[j], vy);
#pragma unroll
      for (int i = 0; i < V; ++i) {
        so = fmaf(vo[i], vo[i], so);
        sy = fmaf(vy[i], vy[i], sy);
      }
    }
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) {
    so += __shfl_xor_sync(0xffffffffu, so, off);
    sy += __shfl_xor_sync(0xffffffffu, sy, off);
  }
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    red[0][w] = so;
    red[1][w] = sy;
  }
  __syncthreads();
  so = red[0][0] + red[0][1] + red[0][2] + red[0][3];
  sy = red[1][0] + red[1][1] + red[1][2] + red[1][3];
  const float ro = 0.5f * rsqrtf(so / a.E + a.eps);
  const float ry = 0.5f * rsqrtf(sy / a.E + a.eps);
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int c = (threadIdx.x + j * 128) * V;
    if (c < a.E) {
      float vo[V], vy[V], ba[V], bs[V], out[V];
      unpack16<T>(ro_[j], vo);
      unpack16<T>(ry_[j], vy);
#pragma unroll
      for (int i = 0; i < V; i += 4) {  // per-channel beta as 16-byte loads
        const float4 a4 = __ldg(reinterpret_cast<const float4 *>(a.beta_attn + c + i));
        const float4 s4 = __ldg(reinterpret_cast<const float4 *>(a.beta_ssm + c + i));
        ba[i] = a4.x; ba[i + 1] = a4.y; ba[i + 2] = a4.z; ba[i + 3] = a4.w;
        bs[i] = s4.x; bs[i + 1] = s4.y; bs[i + 2] = s4.z; bs[i + 3] = s4.w;
      }
#pragma unroll
      for (int i = 0; i < V; ++i) out[i] = fmaf(ba[i] * ro, vo[i], bs[i] * ry * vy[i]);
      if constexpr (sizeof(T) == 2) {
        st_global_v4(f + c, pack_bf16x2(out[0], out[1]), pack_bf16x2(out[2], out[3]),
                     pack_bf16x2(out[4], out[5]), pack_bf16x2(out[6], out[7]));
      } else {
        st_global_v4(f + c, __float_as_uint(out[0]), __float_as_uint(out[1]),
                     __float_as_uint(out[2]), __float_as_uint(out[3]));
      }
    }
  }
}

// Rows wider than the register path: two passes, the second from L1/L2.
template <typename T>
__global__ void __launch_bounds__(256) fuse_wide_kernel(FuseArgs a) {
  constexpr int V = 16 / sizeof(T);
  __shared__ float red[2][8];
  const long long row = blockIdx.x;
  const T *o = reinterpret_cast<const T *>(a.o) + row * a.E;
  const T *y = reinterpret_cast<const T *>(a.y) + row * a.E;
  T *f = reinterpret_cast<T *>(a.f) + row * a.E;
  float so = 0.f, sy = 0.f;
  for (int c = threadIdx.x * V; c < a.E; c += blockDim.x * V) {
    float vo[V], vy[V];
    ld16<T>(o + c, vo);
    ld16<T>(y + c, vy);
#pragma unroll
    for (int i = 0; i < V; ++i) {
      so = fmaf(vo[i], vo[i], so);
      sy = fmaf(vy[i], vy[i], sy);
    }
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) {
    so += __shfl_xor_sync(0xffffffffu, so, off);
    sy += __shfl_xor_sync(0xffffffffu, sy, off);
  }
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    red[0][w] = so;
    red[1][w] = sy;
  }
  __syncthreads();
  so = 0.f;
  sy = 0.f;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) {
    so += red[0][i];
    sy += red[1][i];
  }
  const float ro = 0.5f * rsqrtf(so / a.E + a.eps);
  const float ry = 0.5f * rsqrtf(sy / a.E + a.eps);
  for (int c = threadIdx.x * V; c < a.E; c += blockDim.x * V) {
    float vo[V], vy[V], out[V];
    ld16<T>(o + c, vo);
    ld16<T>(y + c, vy);
#pragma unroll
    for (int i = 0; i < V; ++i)
      out[i] = fmaf(a.beta_attn[c + i] * ro, vo[i], a.beta_ssm[c + i] * ry * vy[i]);
    if constexpr (sizeof(T) == 2) {
      st_global_v4(f + c, pack_bf16x2(out[0], out[1]), pack_bf16x2(out[2], out[3]),
                   pack_bf16x2(out[4], out[5]), pack_bf16x2(out[6], out[7]));
    } else {
      st_global_v4(f + c, __float_as_uint(out[0]), __float_as_uint(out[1]),
                   __float_as_uint(out[2]), __float_as_uint(out[3]));
    }
  }
}

hymba_status fuse_branches(const FuseArgs &a, hymba_dtype dt, cudaStream_t s) {
  if (a.M == 0) return HYMBA_OK;
  const int V = dt == HYMBA_BF16 ? 8 : 4;
  const bool regs = a.E <= 128 * V * 4;
  if (dt == HYMBA_BF16) {
    if (regs)
      fuse_kernel<__nv_bfloat16, 4><<<a.M, 128, 0, s>>>(a);
    else
      fuse_wide_kernel<__nv_bfloat16><<<a.M, 256, 0, s>>>(a);
  } else {
    if (regs)
      fuse_kernel<float, 4><<<a.M, 128, 0, s>>>(a);
    else
      fuse_wide_kernel<float><<<a.M, 256, 0, s>>>(a);
  }
  note_launch(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("fuse launch failed: %s", cudaGetErrorString(e));
    return HYMBA_ERR_CUDA;
  }
  return HYMBA_OK;
}

template <typename T>
__global__ void convert_kernel(const float *__restrict__ src, T *__restrict__ dst, long long n) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) dst[i] = Store<T>::from_f(src[i]);
}

hymba_status convert_f32_to(const float *src, void *dst, long long n, hymba_dtype dt,
                            cudaStream_t s) {
  if (n == 0) return HYMBA_OK;
  const unsigned blocks = (unsigned)((n + 255) / 256);
  if (dt == HYMBA_BF16)
    convert_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(src, (__nv_bfloat16 *)dst, n);
  else
    convert_kernel<float><<<blocks, 256, 0, s>>>(src, (float *)dst, n);
  note_launch(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("convert launch failed: %s", cudaGetErrorString(e));
    return HYMBA_ERR_CUDA;
  }
  return HYMBA_OK;
}

// Decode fuse straight from the attention's run partials: CTA = one sequence, thread =
// one value column d of every head.  Per head the runs' (max, sum) pairs give the merge
// weights 2^(m_r - M) / L; the merged O stays in registers (fp32) for the two RMS norms
// (the SSM row is read twice, the second time from cache).
template <int MAXH>
__global__ void __launch_bounds__(128) fuse_decode_kernel(FuseDecodeArgs a) {
  __shared__ float red[2][4];
  const int b = blockIdx.x, d = threadIdx.x;  // blockDim == dv == 128
  const int rep = a.H / a.Hkv, E = a.H * a.dv;
  float o[MAXH];
  float so = 0.f;
#pragma unroll
  for (int h = 0; h < MAXH; ++h) {
    o[h] = 0.f;
    if (h >= a.H) continue;
    const int g = h / rep;
    const long long item0 = ((long long)b * a.Hkv + g) * a.nchunks;
    const long long r0 = item0 % a.per;
    const long long cfirst = r0 == 0 ? a.per : a.per - r0;
    long long nruns = 1;
    if (cfirst < a.nchunks) nruns += 1 + (a.nchunks - 1 - cfirst) / a.per;
    const float *base = a.part + ((long long)b * a.H + h) * a.nchunks * (a.dv + 2);
    float M = -INFINITY;
    for (long long k = 0; k < nruns; ++k) M = fmaxf(M, base[(k == 0 ? 0 : cfirst + (k - 1) * a.per) * (a.dv + 2)]);
    float Ls = 0.f, acc = 0.f;
    for (long long k = 0; k < nruns; ++k) {
      const float *r = base + (k == 0 ? 0 : cfirst + (k - 1) * a.per) * (a.dv + 2);
      if (r[0] != -INFINITY) {
        const float wgt = ex2_ftz(r[0] - M);
        Ls = fmaf(r[1], wgt, Ls);
        acc = fmaf(r[2 + d], wgt, acc);
      }
    }
    o[h] = acc / Ls;
    so = fmaf(o[h], o[h], so);
  }
  const __nv_bfloat16 *y = reinterpret_cast<const __nv_bfloat16 *>(a.y) + (long long)b * E;
  float sy = 0.f;
#pragma unroll
  for (int h = 0; h < MAXH; ++h) {
    const float yv = h < a.H ? __bfloat162float(y[h * a.dv + d]) : 0.f;
    sy = fmaf(yv, yv, sy);
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) {
    so += __shfl_xor_sync(0xffffffffu, so, off);
    sy += __shfl_xor_sync(0xffffffffu, sy, off);
  }
  if ((d & 31) == 0) {
    red[0][d >> 5] = so;
    red[1][d >> 5] = sy;
  }
  __syncthreads();
  so = red[0][0] + red[0][1] + red[0][2] + red[0][3];
  sy = red[1][0] + red[1][1] + red[1][2] + red[1][3];
  const float ro = 0.5f * rsqrtf(so / E + a.eps);
  const float ry = 0.5f * rsqrtf(sy / E + a.eps);
  __nv_bfloat16 *f = reinterpret_cast<__nv_bfloat16 *>(a.f) + (long long)b * E;
#pragma unroll
  for (int h = 0; h < MAXH; ++h) {
    if (h >= a.H) continue;
    const int c = h * a.dv + d;
    f[c] = __float2bfloat16_rn(fmaf(a.beta_attn[c] * ro, o[h], a.beta_ssm[c] * ry * __bfloat162float(y[c])));
  }
}

hymba_status fuse_decode(const FuseDecodeArgs &a, cudaStream_t s) {
  if (a.dv != 128 || a.H > 32) {
    set_error("fuse_decode needs d_v 128 and at most 32 heads");
    return HYMBA_ERR_UNSUPPORTED;
  }
  fuse_decode_kernel<32><<<a.B, 128, 0, s>>>(a);
  note_launch(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("decode fuse launch failed: %s", cudaGetErrorString(e));
    return HYMBA_ERR_CUDA;
  }
  return HYMBA_OK;
}

}  // namespace hymba
