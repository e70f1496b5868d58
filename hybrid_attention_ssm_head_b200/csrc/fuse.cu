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
  pdl_wait();
  pdl_trigger();
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
  pdl_wait();
  pdl_trigger();
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
      launch_kernel(fuse_kernel<__nv_bfloat16, 4>, dim3(a.M), dim3(128), 0, s, a);
    else
      launch_kernel(fuse_wide_kernel<__nv_bfloat16>, dim3(a.M), dim3(256), 0, s, a);
  } else {
    if (regs)
      launch_kernel(fuse_kernel<float, 4>, dim3(a.M), dim3(128), 0, s, a);
    else
      launch_kernel(fuse_wide_kernel<float>, dim3(a.M), dim3(256), 0, s, a);
  }
  note_launch(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("fuse launch failed: %s", cudaGetErrorString(e));
    return HYMBA_ERR_CUDA;
  }
  return HYMBA_OK;
}

// Decode fuse straight from the attention's run partials: CTA = one sequence, warp h =
// head h, lane = four value columns.  Per head the runs' (max, sum) pairs give the merge
// weights 2^(m_r - M) / L; the merged O (fp32, four values per lane) stays in registers
// for the two RMS norms.
__global__ void __launch_bounds__(1024) fuse_decode_kernel(FuseDecodeArgs a) {
  __shared__ float red[2][32];
  const int b = blockIdx.x, h = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rep = a.H / a.Hkv, E = a.H * a.dv;
  const bool live = h < a.H;
  const int c = h * a.dv + 4 * lane;
  // beta before the wait for the preceding kernels; the SSM branch's output row after it
  // (the scan step that writes it is a direct predecessor when it ran on a side stream
  // joined into this one, and may then still be running when this kernel starts)
  float4 ba = make_float4(0.f, 0.f, 0.f, 0.f), bs = ba, yv = ba;
  if (live) {
    ba = *reinterpret_cast<const float4 *>(a.beta_attn + c);
    bs = *reinterpret_cast<const float4 *>(a.beta_ssm + c);
  }
  pdl_wait();
  pdl_trigger();
  float4 ov = make_float4(0.f, 0.f, 0.f, 0.f);
  float so = 0.f, sy = 0.f;
  if (live) {
    const uint2 raw = *reinterpret_cast<const uint2 *>(reinterpret_cast<const __nv_bfloat16 *>(a.y) +
                                                       (long long)b * E + c);
    yv = make_float4(bf16_lo(raw.x), bf16_hi(raw.x), bf16_lo(raw.y), bf16_hi(raw.y));
    const int g = h / rep;
    const long long item0 = ((long long)b * a.Hkv + g) * a.nchunks;
    const long long r0 = item0 % a.per;
    const long long cfirst = r0 == 0 ? a.per : a.per - r0;
    int nruns = 1;
    if (cfirst < a.nchunks) nruns += 1 + (int)((a.nchunks - 1 - cfirst) / a.per);
    const float *base = a.part + ((long long)b * a.H + h) * a.nchunks * (a.dv + 2);
    auto run = [&](long long k) { return base + (k == 0 ? 0 : cfirst + (k - 1) * a.per) * (a.dv + 2); };
    constexpr int KR = 4;  // up to KR runs: every (max, sum) and O requested at once
    if (nruns <= KR) {
      float2 ml[KR];
      float4 o[KR];
#pragma unroll
      for (int k = 0; k < KR; ++k) {
        ml[k] = make_float2(-INFINITY, 0.f);
        o[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (k < nruns) {
          const float *r = run(k);
          ml[k] = *reinterpret_cast<const float2 *>(r);
          // O starts at offset 2 (8-byte aligned): two float2 loads per lane
          const float2 p0 = *reinterpret_cast<const float2 *>(r + 2 + 4 * lane);
          const float2 p1 = *reinterpret_cast<const float2 *>(r + 2 + 4 * lane + 2);
          o[k] = make_float4(p0.x, p0.y, p1.x, p1.y);
        }
      }
      float M = -INFINITY;
#pragma unroll
      for (int k = 0; k < KR; ++k) M = fmaxf(M, ml[k].x);
      float L = 0.f;
#pragma unroll
      for (int k = 0; k < KR; ++k)
        if (ml[k].x != -INFINITY) L = fmaf(ml[k].y, ex2_ftz(ml[k].x - M), L);
      const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
      for (int k = 0; k < KR; ++k) {
        if (ml[k].x == -INFINITY) continue;
        const float w = ex2_ftz(ml[k].x - M) * inv;
        ov.x = fmaf(o[k].x, w, ov.x);
        ov.y = fmaf(o[k].y, w, ov.y);
        ov.z = fmaf(o[k].z, w, ov.z);
        ov.w = fmaf(o[k].w, w, ov.w);
      }
    } else {
      // the runs' (max, sum) pairs, 32 runs per round across the lanes
      float M = -INFINITY;
      for (int k0 = 0; k0 < nruns; k0 += 32)
        if (k0 + lane < nruns) M = fmaxf(M, run(k0 + lane)[0]);
#pragma unroll
      for (int off = 16; off; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
      float L = 0.f;
      for (int k0 = 0; k0 < nruns; k0 += 32) {
        if (k0 + lane < nruns) {
          const float *r = run(k0 + lane);
          if (r[0] != -INFINITY) L = fmaf(r[1], ex2_ftz(r[0] - M), L);
        }
      }
#pragma unroll
      for (int off = 16; off; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
      const float inv = L > 0.f ? 1.f / L : 0.f;
      for (int k = 0; k < nruns; ++k) {
        const float *r = run(k);
        const float mk = r[0];
        if (mk == -INFINITY) continue;
        const float w = ex2_ftz(mk - M) * inv;
        const float2 p0 = *reinterpret_cast<const float2 *>(r + 2 + 4 * lane);
        const float2 p1 = *reinterpret_cast<const float2 *>(r + 2 + 4 * lane + 2);
        ov.x = fmaf(p0.x, w, ov.x);
        ov.y = fmaf(p0.y, w, ov.y);
        ov.z = fmaf(p1.x, w, ov.z);
        ov.w = fmaf(p1.y, w, ov.w);
      }
    }
    so = ov.x * ov.x + ov.y * ov.y + ov.z * ov.z + ov.w * ov.w;
    sy = yv.x * yv.x + yv.y * yv.y + yv.z * yv.z + yv.w * yv.w;
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) {
    so += __shfl_xor_sync(0xffffffffu, so, off);
    sy += __shfl_xor_sync(0xffffffffu, sy, off);
  }
  if (lane == 0) {
    red[0][h] = so;
    red[1][h] = sy;
  }
  __syncthreads();
  if (h == 0) {
    float a0 = lane < (int)(blockDim.x >> 5) ? red[0][lane] : 0.f;
    float a1 = lane < (int)(blockDim.x >> 5) ? red[1][lane] : 0.f;
#pragma unroll
    for (int off = 16; off; off >>= 1) {
      a0 += __shfl_xor_sync(0xffffffffu, a0, off);
      a1 += __shfl_xor_sync(0xffffffffu, a1, off);
    }
    if (lane == 0) {
      red[0][0] = a0;
      red[1][0] = a1;
    }
  }
  __syncthreads();
  if (!live) return;
  const float ro = 0.5f * rsqrtf(red[0][0] / E + a.eps);
  const float ry = 0.5f * rsqrtf(red[1][0] / E + a.eps);
  uint2 outw;
  outw.x = pack_bf16x2(fmaf(ba.x * ro, ov.x, bs.x * ry * yv.x), fmaf(ba.y * ro, ov.y, bs.y * ry * yv.y));
  outw.y = pack_bf16x2(fmaf(ba.z * ro, ov.z, bs.z * ry * yv.z), fmaf(ba.w * ro, ov.w, bs.w * ry * yv.w));
  *reinterpret_cast<uint2 *>(reinterpret_cast<__nv_bfloat16 *>(a.f) + (long long)b * E + c) = outw;
}

hymba_status fuse_decode(const FuseDecodeArgs &a, cudaStream_t s) {
  if (a.dv != 128 || a.H > 32) {
    set_error("fuse_decode needs d_v 128 and at most 32 heads");
    return HYMBA_ERR_UNSUPPORTED;
  }
  launch_kernel(fuse_decode_kernel, dim3(a.B), dim3(32 * a.H), 0, s, a);
  note_launch(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("decode fuse launch failed: %s", cudaGetErrorString(e));
    return HYMBA_ERR_CUDA;
  }
  return HYMBA_OK;
}


// ---------------------------------------------------------------------------
// RMS norm with a learnable weight (the Hymba block's pre-norms):
//   y[r, :] = x[r, :] / sqrt(mean(x[r, :]^2) + eps) * w
// One warp per row; the row stays in registers as packed 16-byte vectors between the
// reduction and the scaling, so it is read once.
// ---------------------------------------------------------------------------
template <typename T, int NV>
__global__ void __launch_bounds__(256) rmsnorm_kernel(const T *__restrict__ x, const float *__restrict__ w,
                                                      T *__restrict__ y, long long M, int d, float eps) {
  constexpr int V = 16 / sizeof(T);
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  const int nvec = d / V;
  const T *xr = x + row * d;
  uint4 raw[NV];
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int v = lane + 32 * j;
    if (v < nvec) {
      raw[j] = __ldg(reinterpret_cast<const uint4 *>(xr + v * V));
      float f[V];
      unpack16<T>(raw[j], f);
#pragma unroll
      for (int i = 0; i < V; ++i) ss = fmaf(f[i], f[i], ss);
    }
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  const float inv = rsqrtf(ss / d + eps);
  T *yr = y + row * d;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int v = lane + 32 * j;
    if (v < nvec) {
      float f[V];
      unpack16<T>(raw[j], f);
#pragma unroll
      for (int i = 0; i < V; i += 4) {
        const float4 w4 = __ldg(reinterpret_cast<const float4 *>(w + v * V + i));
        f[i] *= inv * w4.x;
        f[i + 1] *= inv * w4.y;
        f[i + 2] *= inv * w4.z;
        f[i + 3] *= inv * w4.w;
      }
      if constexpr (sizeof(T) == 2) {
        st_global_v4(yr + v * V, pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                     pack_bf16x2(f[6], f[7]));
      } else {
        st_global_v4(yr + v * V, __float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                     __float_as_uint(f[3]));
      }
    }
  }
}

hymba_status rms_norm_rows(const void *x, const float *w, void *y, long long M, int d, float eps, hymba_dtype dt,
                           cudaStream_t s) {
  const int V = dt == HYMBA_BF16 ? 8 : 4;
  if (d % V || d / V > 32 * 8) {
    set_error("rms norm rows of %d elements: need a multiple of %d, at most %d", d, V, 32 * 8 * V);
    return HYMBA_ERR_UNSUPPORTED;
  }
  if (M == 0) return HYMBA_OK;
  const unsigned blocks = (unsigned)((M * 32 + 255) / 256);
  if (dt == HYMBA_BF16)
    rmsnorm_kernel<__nv_bfloat16, 8><<<blocks, 256, 0, s>>>((const __nv_bfloat16 *)x, w, (__nv_bfloat16 *)y, M,
                                                              d, eps);
  else
    rmsnorm_kernel<float, 8><<<blocks, 256, 0, s>>>((const float *)x, w, (float *)y, M, d, eps);
  note_launch(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("rms norm launch failed: %s", cudaGetErrorString(e));
    return HYMBA_ERR_CUDA;
  }
  return HYMBA_OK;
}

}  // namespace hymba
