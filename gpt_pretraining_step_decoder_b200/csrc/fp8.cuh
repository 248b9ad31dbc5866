// fp8.cuh -- per-tensor e4m3 quantization for the FP8 GEMM path.
//
// Karpathy's llm.c post lists FP8 training as "imminent"; the decoder-rtx
// posts train without it.  The per-tensor form here: amax = max |x|, inv =
// 448 / amax (one fp32 division), code = e4m3(x * inv) rounded to nearest
// even with saturation to +-448 (the hardware conversion
// cvt.rn.satfinite.e4m3x2.f32), scale = amax / 448 for the product's
// epilogue.  amax is exact (a maximum), so every code depends only on x.
#pragma once
#include <cuda_fp8.h>
#include "common.cuh"

constexpr int FP8_AMAX_BLOCKS = 512;  // fixed grid of the max pass

template <typename T>
__global__ void __launch_bounds__(256) fp8_amax_kernel(const T* __restrict__ x, long long n, float* __restrict__ part) {
  __shared__ float wmax[8];
  float m = 0.f;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    m = fmaxf(m, fabsf(to_f(x[i])));
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < 8; ++w) t = fmaxf(t, wmax[w]);
    part[blockIdx.x] = t;
  }
}

// codes of x (pairs of elements per thread), scale = amax / 448 (block 0)
template <typename T>
__global__ void __launch_bounds__(256) fp8_quantize_kernel(const T* __restrict__ x, long long n,
                                                           const float* __restrict__ part, uint8_t* __restrict__ q,
                                                           float* __restrict__ scale) {
  __shared__ float s_amax;
  if (threadIdx.x < 32) {
    float m = 0.f;
    for (int i = threadIdx.x; i < FP8_AMAX_BLOCKS; i += 32) m = fmaxf(m, part[i]);
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (threadIdx.x == 0) s_amax = m;
  }
  __syncthreads();
  const float amax = s_amax;
  const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 1.f;
  if (blockIdx.x == 0 && threadIdx.x == 0) *scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  const long long n2 = n / 2;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n2; i += (long long)gridDim.x * blockDim.x) {
    const float2 v = make_float2(__fmul_rn(to_f(x[2 * i]), inv), __fmul_rn(to_f(x[2 * i + 1]), inv));
    const __nv_fp8x2_storage_t c = __nv_cvt_float2_to_fp8x2(v, __NV_SATFINITE, __NV_E4M3);
    reinterpret_cast<__nv_fp8x2_storage_t*>(q)[i] = c;
  }
}
