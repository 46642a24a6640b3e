// moe_norm.cu -- the fixed normalisation between stacked layers: unit-gain RMSNorm of an
// FP32 row followed by the round-to-nearest-even cast to bf16,
//   x[t, i] = bf16(y[t, i] / sqrt(mean_i y[t, i]^2 + eps)).
// One CTA per row; the sum of squares is reduced in a fixed order (deterministic).
#include "moe_common.cuh"

namespace {

__global__ void __launch_bounds__(256) k_rmsnorm_bf16(const float *__restrict__ y, __nv_bfloat16 *__restrict__ x,
                                                      int d, float eps) {
  __shared__ float part[8];
  const int t = blockIdx.x;
  const float *yr = y + (size_t)t * d;
  float s = 0.f;
  for (int i = threadIdx.x; i < d; i += 256) s = fmaf(yr[i], yr[i], s);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) tot += part[w];
  const float inv = 1.0f / sqrtf(tot / (float)d + eps);
  __nv_bfloat16 *xr = x + (size_t)t * d;
  for (int i = threadIdx.x; i < d; i += 256) xr[i] = __float2bfloat16_rn(yr[i] * inv);
}

}  // namespace

int moe_launch_rmsnorm(cudaStream_t s, const float *y, void *x_out, int T, int d, float eps) {
  moe_prof_mark(s, MOE_K_NORM, true);
  k_rmsnorm_bf16<<<T, 256, 0, s>>>(y, static_cast<__nv_bfloat16 *>(x_out), d, eps);
  if (cudaGetLastError() != cudaSuccess) return -1;
  moe_prof_count(1);
  moe_prof_mark(s, MOE_K_NORM, false);
  return 0;
}
