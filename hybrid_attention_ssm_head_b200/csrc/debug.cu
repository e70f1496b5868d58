// Small helper kernels: the rotary-embedding table of the input projection's epilogue, and
// device helpers evaluated on caller-given inputs so that tests can check them directly
// against their stated error bounds.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace hymba {

template <int DEG>
__global__ void exp2_poly_kernel(const float *__restrict__ x, float *__restrict__ y, long long n) {
  const long long i = 2 * ((long long)blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float2 in = make_float2(x[i], i + 1 < n ? x[i + 1] : 0.f);
  const float2 out = exp2_poly2<DEG>(in);
  y[i] = out.x;
  if (i + 1 < n) y[i + 1] = out.y;
}

hymba_status exp2_poly_eval(int degree, const float *x, float *y, long long n, cudaStream_t s) {
  if (n <= 0) return HYMBA_OK;
  const long long pairs = (n + 1) / 2;
  const unsigned blocks = (unsigned)((pairs + 255) / 256);
  if (degree == 3)
    exp2_poly_kernel<3><<<blocks, 256, 0, s>>>(x, y, n);
  else
    exp2_poly_kernel<5><<<blocks, 256, 0, s>>>(x, y, n);
  note_launch(1);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("exp2 polynomial launch failed: %s", cudaGetErrorString(e));
    return HYMBA_ERR_CUDA;
  }
  return HYMBA_OK;
}

// Rotary table in double precision (the angle of a late position is large), stored fp32.
__global__ void rope_table_kernel(float2 *tab, int npos, long long pos0, int hd, double log2_base) {
  pdl_wait();
  pdl_trigger();
  const int hp = hd >> 1;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)npos * hp) return;
  const int i = (int)(idx % hp);
  const long long p = pos0 + idx / hp;
  const double ang = (double)p * exp2(-2.0 * i / hd * log2_base);
  double sn, cn;
  sincos(ang, &sn, &cn);
  tab[idx] = make_float2((float)cn, (float)sn);
}

hymba_status rope_table(float2 *tab, int npos, long long pos0, int hd, float base, cudaStream_t s) {
  const long long n = (long long)npos * (hd / 2);
  if (n <= 0) return HYMBA_OK;
  launch_kernel(rope_table_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, tab, npos, pos0, hd,
                log2((double)base));
  note_launch(1);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("rotary table launch failed: %s", cudaGetErrorString(e));
    return HYMBA_ERR_CUDA;
  }
  return HYMBA_OK;
}

}  // namespace hymba
