// fp8_weights.cu -- fp8 (E4M3) storage of the estimator's projection weights.
//
// News page ("Veda from ByteDance, HKU and USTC: an open method that speeds up
// video generation fivefold", "Why this matters for users"): the predictor is
// distributed in fp8, half the size of its bf16 file, with nearly the same
// tile recall.  Encoding: OCP FP8 E4M3 with one scale per head,
//   s[h] = max |W[h]| / 448  (1 if the head is all zeros),
//   W8[h] = e4m3(W[h] / s[h])  (round to nearest even, saturating at +-448),
//   dequantised weight = fp32(e4m3 value * s[h]),
// the fp32 weight the estimator then computes with.  The scale and W / s are
// fp32 operations; the conversions are CUDA's fp8 intrinsics.
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "internal.h"

namespace veda {

namespace {

constexpr int kQThreads = 256;

__global__ void __launch_bounds__(kQThreads) quantize_e4m3_kernel(const float* __restrict__ W,
                                                                  long long n,
                                                                  uint8_t* __restrict__ codes,
                                                                  float* __restrict__ scale) {
    const long long base = (long long)blockIdx.x * n;
    __shared__ float part[kQThreads];
    float amax = 0.f;
    for (long long i = threadIdx.x; i < n; i += kQThreads) amax = fmaxf(amax, fabsf(W[base + i]));
    part[threadIdx.x] = amax;
    __syncthreads();
    for (int w = kQThreads / 2; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w) part[threadIdx.x] = fmaxf(part[threadIdx.x], part[threadIdx.x + w]);
        __syncthreads();
    }
    const float m = part[0];
    const float s = m > 0.f ? __fdiv_rn(m, 448.0f) : 1.0f;
    if (threadIdx.x == 0) scale[blockIdx.x] = s;
    for (long long i = threadIdx.x; i < n; i += kQThreads)
        codes[base + i] = __nv_cvt_float_to_fp8(__fdiv_rn(W[base + i], s), __NV_SATFINITE, __NV_E4M3);
}

__global__ void __launch_bounds__(kQThreads) dequantize_e4m3_kernel(const uint8_t* __restrict__ codes,
                                                                    const float* __restrict__ scale,
                                                                    long long n,
                                                                    float* __restrict__ W) {
    const long long base = (long long)blockIdx.x * n;
    const float s = scale[blockIdx.x];
    for (long long i = threadIdx.x; i < n; i += kQThreads) {
        const __half h = __half(__nv_cvt_fp8_to_halfraw(codes[base + i], __NV_E4M3));
        W[base + i] = __fmul_rn(__half2float(h), s);
    }
}

}  // namespace

veda_status launch_quantize_e4m3(const float* W, int H, long long n, uint8_t* codes, float* scale,
                                 cudaStream_t s) {
    quantize_e4m3_kernel<<<H, kQThreads, 0, s>>>(W, n, codes, scale);
    return cuda_check(cudaGetLastError(), "fp8 quantize launch");
}

veda_status launch_dequantize_e4m3(const uint8_t* codes, const float* scale, int H, long long n,
                                   float* W, cudaStream_t s) {
    dequantize_e4m3_kernel<<<H, kQThreads, 0, s>>>(codes, scale, n, W);
    return cuda_check(cudaGetLastError(), "fp8 dequantize launch");
}

}  // namespace veda
