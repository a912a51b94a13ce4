// Stack glue between decode layers: residual add + RMSNorm (unit weight) -> BF16.
#include "common.cuh"
#include "launch.h"

namespace msb {

constexpr int kGlueNT = 256;

// One CTA per token: h += y (FP32), x_next = BF16(h / sqrt(mean(h^2) + eps)).
__global__ void __launch_bounds__(kGlueNT) residual_rmsnorm_kernel(float* __restrict__ h,
                                                                   const uint16_t* __restrict__ y,
                                                                   uint16_t* __restrict__ xn, int d,
                                                                   float eps) {
  __shared__ float red[kGlueNT / 32];
  const int t = blockIdx.x;
  float* hr = h + (size_t)t * d;
  float ss = 0.f;
  for (int i = threadIdx.x; i < d; i += kGlueNT) {
    float v = hr[i];
    if (y) v += __uint_as_float((uint32_t)y[(size_t)t * d + i] << 16);
    hr[i] = v;
    ss = fmaf(v, v, ss);
  }
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < kGlueNT / 32; ++w) tot += red[w];
  const float inv = 1.0f / sqrtf(tot / (float)d + eps);
  for (int i = threadIdx.x; i < d; i += kGlueNT)
    xn[(size_t)t * d + i] = __bfloat16_as_ushort(__float2bfloat16_rn(hr[i] * inv));
}

int launch_residual_rmsnorm(float* h, const uint16_t* y, uint16_t* x_next, int B, int d, float eps,
                            cudaStream_t st) {
  residual_rmsnorm_kernel<<<B, kGlueNT, 0, st>>>(h, y, x_next, d, eps);
  return cudaGetLastError() == cudaSuccess ? MSB_OK : MSB_ECUDA;
}

}  // namespace msb
