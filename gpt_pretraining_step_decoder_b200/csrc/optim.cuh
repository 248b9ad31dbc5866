// optim.cuh -- dense-weight optimizer and initialisation kernels.
#pragma once
#include "common.cuh"

// AdamW over the flat fp32 parameter buffer ("$1000 tier nanochat run",
// `setup_optimizers`: torch.optim.AdamW, betas (0.8, 0.95), eps 1e-10,
// decoupled weight decay), with per-group learning rates: [0, e_end) the
// token embedding, [e_end, h_end) the untied LM head, the rest the matrices.
// The global-norm clip coefficient (or 1) is read from the device.  Writes
// the bf16 GEMM copy in the same pass when p_lp is not null.
struct AdamArgs {
  float* p; const float* g; float* m; float* v; bf16* p_lp;
  long long n, e_end, h_end;
  float lr_e, lr_h, lr_m, b1, b2, eps, wd, bc1, bc2;
  const float* clip;
};

__global__ void adamw_kernel(AdamArgs a) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  const float coef = a.clip ? *a.clip : 1.f;
  const long long n4 = a.n / 4;
  for (long long i4 = (long long)blockIdx.x * blockDim.x + threadIdx.x; i4 < n4;
       i4 += (long long)gridDim.x * blockDim.x) {
    const long long i = i4 * 4;
    const float lr = (i < a.e_end) ? a.lr_e : (i < a.h_end) ? a.lr_h : a.lr_m;
    float p[4], g[4], m[4], v[4];
    load4(a.p + i, p); load4(a.g + i, g); load4(a.m + i, m); load4(a.v + i, v);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float gk = g[k] * coef;
      m[k] = a.b1 * m[k] + (1.f - a.b1) * gk;
      v[k] = a.b2 * v[k] + (1.f - a.b2) * gk * gk;
      p[k] = p[k] * (1.f - lr * a.wd);
      p[k] = p[k] - lr * (m[k] / a.bc1) / (sqrtf(v[k] / a.bc2) + a.eps);
    }
    store4(a.p + i, p); store4(a.m + i, m); store4(a.v + i, v);
    if (a.p_lp) store4(a.p_lp + i, p);
  }
}

// Deterministic global L2 norm: fixed grid, per-block partials, then one
// block sums the partials in order and forms min(1, clip / (norm + 1e-6)).
constexpr int NORM_BLOCKS = 1024;
__global__ void sumsq_partial_kernel(const float* __restrict__ g, long long n, double* __restrict__ part) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  __shared__ double sh[32];
  double s = 0.0;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const double x = g[i];
    s += x * x;
  }
  s = warp_sum_d(s);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (lane == 0) sh[wid] = s;
  __syncthreads();
  if (wid == 0) {
    double r = (lane < (int)(blockDim.x >> 5)) ? sh[lane] : 0.0;
    r = warp_sum_d(r);
    if (lane == 0) part[blockIdx.x] = r;
  }
}
__global__ void clip_coef_kernel(const double* __restrict__ part, int nparts, float max_norm,
                                 float* __restrict__ coef, float* __restrict__ norm_out, unsigned* err) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  __shared__ double sh[32];
  double s = 0.0;
  for (int i = threadIdx.x; i < nparts; i += blockDim.x) s += part[i];
  s = warp_sum_d(s);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (lane == 0) sh[wid] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += sh[w];
    const double nrm = sqrt(t);
    if (norm_out) *norm_out = (float)nrm;
    if (!isfinite(nrm)) set_error(err, GPT_EBIT_NONFINITE);
    *coef = (float)fmin(1.0, (double)max_norm / (nrm + 1e-6));
  }
}

// *out = sum of the partials in order (one block)
__global__ void sum_partials_kernel(const double* __restrict__ part, int nparts, double* __restrict__ out) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  __shared__ double sh[32];
  double s = 0.0;
  for (int i = threadIdx.x; i < nparts; i += blockDim.x) s += part[i];
  s = warp_sum_d(s);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (lane == 0) sh[wid] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += sh[w];
    *out = t;
  }
}

// fp32 master -> bf16 copy (round to nearest even).
__global__ void to_bf16_kernel(const float* __restrict__ src, bf16* __restrict__ dst, long long n) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x)
    dst[i] = __float2bfloat16_rn(src[i]);
}

// out[i] = (beta ? out[i] : 0) + add[i]
__global__ void accumulate_kernel(float* __restrict__ out, const float* __restrict__ add, long long n,
                                  int beta) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x)
    out[i] = (beta ? out[i] : 0.f) + add[i];
}

// ---------------------------------------------------------------- init RNG
// Philox-4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As
// Easy as 1, 2, 3", SC'11): 10 rounds of the multiply-xor round function
// with the published multipliers and Weyl key increments.
__device__ __forceinline__ void philox4x32_10(uint32_t c[4], uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = (uint64_t)0xD2511F53u * c[0];
    const uint64_t p1 = (uint64_t)0xCD9E8D57u * c[2];
    const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    const uint32_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
    c[0] = n0; c[1] = lo1; c[2] = n2; c[3] = lo0;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
}

// dst[i] = std * N(0,1), i < n, from counters (i/4, stream); Box-Muller on
// pairs of 32-bit uniforms mapped to (0, 1].
template <typename T>
__global__ void init_normal_kernel(T* __restrict__ dst, long long n, float stdv,
                                   unsigned long long seed, uint32_t stream) {
  const long long n4 = (n + 3) / 4;
  for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < n4;
       q += (long long)gridDim.x * blockDim.x) {
    uint32_t c[4] = {(uint32_t)q, (uint32_t)(q >> 32), stream, 0u};
    philox4x32_10(c, (uint32_t)seed, (uint32_t)(seed >> 32));
    float z[4];
#pragma unroll
    for (int k = 0; k < 4; k += 2) {
      const float u1 = ((float)c[k] + 1.f) * 2.3283064365386963e-10f;  // (0, 1]
      const float u2 = (float)c[k + 1] * 2.3283064365386963e-10f;
      const float rad = sqrtf(-2.f * logf(u1));
      float s, co;
      sincospif(2.f * u2, &s, &co);
      z[k] = rad * co;
      z[k + 1] = rad * s;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const long long i = q * 4 + k;
      if (i < n) dst[i] = from_f<T>(stdv * z[k]);
    }
  }
}
