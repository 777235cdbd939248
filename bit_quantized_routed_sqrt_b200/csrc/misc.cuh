// misc.cuh -- small stateless kernels: RMS renormalisation and the score diagnostic.
#pragma once
#include "common.cuh"

namespace ds4 {

// x[t,i] = bf16_rne(y[t,i] / sqrt(mean_i y[t,i]^2 + 1e-6)); one CTA of 256 threads per token.
__global__ void __launch_bounds__(256) rms_renorm_kernel(const float *__restrict__ y, int H, __nv_bfloat16 *__restrict__ x) {
    __shared__ float part[8];
    const int t = blockIdx.x;
    const float *yt = y + (size_t)t * H;
    float ss = 0.0f;
    for (int i = threadIdx.x; i < H; i += blockDim.x) ss = fmaf(yt[i], yt[i], ss);
    ss = warp_sum(ss);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) tot += part[w];
    const float inv = 1.0f / sqrtf(tot / (float)H + 1e-6f);
    for (int i = threadIdx.x; i < H; i += blockDim.x) x[(size_t)t * H + i] = __float2bfloat16_rn(yt[i] * inv);
}

__global__ void score_eval_kernel(const float *__restrict__ l, int n, float *__restrict__ s, int variant) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) s[i] = variant == 0 ? router_score(l[i]) : router_score_naive(l[i]);
}

}  // namespace ds4
