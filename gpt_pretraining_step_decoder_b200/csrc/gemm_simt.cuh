// gemm_simt.cuh -- fp32-accumulating SIMT GEMM (plain FFMA, no TF32).
//
// The contraction of the fp32 parity mode, where tensor cores would lose
// precision.  64 x 64 output tile per 256-thread block, 4 x 4 outputs per
// thread, K staged through shared memory 16 at a time.  Any layout and any
// size (ragged edges are predicated).
#pragma once
#include "gemm_common.cuh"

template <typename in_t>
__device__ __forceinline__ float op_load(const GemmOperand& o, long long r, long long k,
                                         long long rows, long long K) {
  if (r >= rows || k >= K) return 0.f;
  const in_t* p = reinterpret_cast<const in_t*>(o.ptr);
  return to_f(o.kmajor ? p[r * o.ld + k] : p[k * o.ld + r]);
}

template <typename in_t, typename act_t>
__global__ void __launch_bounds__(256) gemm_simt_kernel(int M, int N, int K, GemmOperand A,
                                                        GemmOperand B, GemmEpilogue e) {
  __shared__ float As[16][64 + 4];
  __shared__ float Bs[16][64 + 4];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const long long m0 = (long long)blockIdx.y * 64, n0 = (long long)blockIdx.x * 64;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 64 * 16; i += 256) {
      int r, k;
      // walk along the stored contiguous dimension for coalescing
      if (A.kmajor) { r = i / 16; k = i % 16; } else { k = i / 64; r = i % 64; }
      As[k][r] = op_load<in_t>(A, m0 + r, k0 + k, M, K);
      if (B.kmajor) { r = i / 16; k = i % 16; } else { k = i / 64; r = i % 64; }
      Bs[k][r] = op_load<in_t>(B, n0 + r, k0 + k, N, K);
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = As[kk][ty * 4 + i]; b[i] = Bs[kk][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      long long m = m0 + ty * 4 + i, n = n0 + tx * 4 + j;
      if (m < M && n < N) epi_apply_one<act_t>(e, m, n, acc[i][j]);
    }
}

template <typename in_t, typename act_t>
static void gemm_simt(int M, int N, int K, GemmOperand A, GemmOperand B, GemmEpilogue e,
                      cudaStream_t st) {
  dim3 grid(cdiv(N, 64), cdiv(M, 64));
  gemm_simt_kernel<in_t, act_t><<<grid, 256, 0, st>>>(M, N, K, A, B, e);
}
