// muon.cuh -- Muon for a matrix parameter: Nesterov momentum, the update
// orthogonalised by a quintic Newton-Schulz iteration run in bf16 on the
// tcgen05 GEMM, then the scaled step (modded-nanogpt README, "Proposed
// optimizer"; nanochat discussion #8, `zeropower_via_newtonschulz5` and
// `Muon.step`).
//
// The host side (gpt.cu, muon_update) runs per Newton-Schulz step three GEMMs
// -- A = X X^T (X^T X for a tall matrix), A A, and B X (X B) -- with fp32
// outputs; the kernels here are the elementwise parts between them.  All
// element counts are multiples of 4 (the entry point asks for row and column
// counts that are multiples of 8), so every kernel moves float4 / 4 x bf16.
// Sums are formed in a fixed order (no atomics): results are reproducible.
#pragma once
#include "common.cuh"

constexpr int MUON_THREADS = 256;
constexpr int MUON_NORM_BLOCKS = 256;  // fixed grid of the sum-of-squares pass

// The update U = (1 - mu) g + mu * m' with Nesterov momentum, else m'.
__device__ __forceinline__ float muon_u(float g, float m_new, float mu, int nesterov) {
  return nesterov ? (1.f - mu) * g + mu * m_new : m_new;
}

// m <- mu m + (1 - mu) g in place; each block writes the sum of U^2 over its
// grid-stride share (fixed grid, fixed order) to partials[blockIdx.x].
__global__ void __launch_bounds__(MUON_THREADS) muon_momentum_kernel(const float* __restrict__ G,
                                                                     float* __restrict__ M, long long n4, float mu,
                                                                     int nesterov, float* __restrict__ partials) {
  __shared__ float wsum[MUON_THREADS / 32];
  float ss = 0.f;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    const float4 g = reinterpret_cast<const float4*>(G)[i];
    float4 m = reinterpret_cast<float4*>(M)[i];
    m.x = mu * m.x + (1.f - mu) * g.x;
    m.y = mu * m.y + (1.f - mu) * g.y;
    m.z = mu * m.z + (1.f - mu) * g.z;
    m.w = mu * m.w + (1.f - mu) * g.w;
    reinterpret_cast<float4*>(M)[i] = m;
    const float u0 = muon_u(g.x, m.x, mu, nesterov), u1 = muon_u(g.y, m.y, mu, nesterov);
    const float u2 = muon_u(g.z, m.z, mu, nesterov), u3 = muon_u(g.w, m.w, mu, nesterov);
    ss += (u0 * u0 + u1 * u1) + (u2 * u2 + u3 * u3);
  }
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < MUON_THREADS / 32; ++w) t += wsum[w];
    partials[blockIdx.x] = t;
  }
}

// X = bf16(U / (||U||_F + eps)), U recomputed from g and the updated m.
__global__ void __launch_bounds__(MUON_THREADS) muon_normalize_kernel(const float* __restrict__ G,
                                                                      const float* __restrict__ M, long long n4,
                                                                      float mu, int nesterov,
                                                                      const float* __restrict__ partials, int nparts,
                                                                      float eps, bf16* __restrict__ X) {
  __shared__ float inv_norm;
  if (threadIdx.x < 32) {
    float s = 0.f;
    for (int i = threadIdx.x; i < nparts; i += 32) s += partials[i];
    s = warp_sum(s);
    if (threadIdx.x == 0) inv_norm = 1.f / (sqrtf(s) + eps);
  }
  __syncthreads();
  const float inv = inv_norm;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    const float4 g = reinterpret_cast<const float4*>(G)[i];
    const float4 m = reinterpret_cast<const float4*>(M)[i];
    const float v[4] = {muon_u(g.x, m.x, mu, nesterov) * inv, muon_u(g.y, m.y, mu, nesterov) * inv,
                        muon_u(g.z, m.z, mu, nesterov) * inv, muon_u(g.w, m.w, mu, nesterov) * inv};
    store4(X + 4 * i, v);
  }
}

// out = bf16(a * x + c * y) over n4 float4 groups; x is bf16 (A or X), y fp32
// (a GEMM output).  Both linear steps of the iteration take this form:
// B = b A + c (A A), and X <- a X + 1 * (B X).
__global__ void __launch_bounds__(MUON_THREADS) muon_combine_kernel(const bf16* __restrict__ x,
                                                                    const float* __restrict__ y, long long n4, float a,
                                                                    float c, bf16* __restrict__ out) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    float xv[4];
    load4(x + 4 * i, xv);
    const float4 yv = reinterpret_cast<const float4*>(y)[i];
    const float v[4] = {a * xv[0] + c * yv.x, a * xv[1] + c * yv.y, a * xv[2] + c * yv.z, a * xv[3] + c * yv.w};
    store4(out + 4 * i, v);
  }
}

// out = bf16(y) (the A product, read as a bf16 GEMM operand by the next one)
__global__ void __launch_bounds__(MUON_THREADS) muon_to_bf16_kernel(const float* __restrict__ y, long long n4,
                                                                    bf16* __restrict__ out) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    const float4 yv = reinterpret_cast<const float4*>(y)[i];
    const float v[4] = {yv.x, yv.y, yv.z, yv.w};
    store4(out + 4 * i, v);
  }
}

// W -= step * X (fp32 master weight, bf16 orthogonalised update)
__global__ void __launch_bounds__(MUON_THREADS) muon_apply_kernel(float* __restrict__ W, const bf16* __restrict__ X,
                                                                  long long n4, float step) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    float xv[4];
    load4(X + 4 * i, xv);
    float4 w = reinterpret_cast<float4*>(W)[i];
    w.x -= step * xv[0];
    w.y -= step * xv[1];
    w.z -= step * xv[2];
    w.w -= step * xv[3];
    reinterpret_cast<float4*>(W)[i] = w;
  }
}

// ---------------------------------------------------------------- batched form
// The training step runs Muon on every block matrix at once, grouped by shape.
// A group's matrices sit in the flat parameter buffers at a regular pattern:
// matrix j starts at base + (j / per_layer) * layer_stride + (j % per_layer) *
// inner_stride (elements), e.g. the q, k, v blocks and the projection of every
// layer.  Each kernel runs a fixed number of blocks per matrix (grid.y = the
// matrix), so per-matrix sums come out in a fixed order.
struct MuonGroup {
  long long base, layer_stride, inner_stride;
  int per_layer, nmat, rows, cols;
};
constexpr int MUON_BATCH_BLOCKS = 64;  // blocks per matrix of the sum-of-squares pass

__device__ __forceinline__ long long muon_off(const MuonGroup& g, int j) {
  return g.base + (long long)(j / g.per_layer) * g.layer_stride + (long long)(j % g.per_layer) * g.inner_stride;
}

// m <- mu m + (1 - mu) c g for every matrix of the group (c: the global clip
// coefficient, 1 when `clip` is null); per block the sum of U^2 of its share
// of the matrix to partials[j * MUON_BATCH_BLOCKS + block].
__global__ void __launch_bounds__(MUON_THREADS) muon_batch_momentum_kernel(
    const float* __restrict__ Gall, float* __restrict__ Mall, MuonGroup grp, float mu, int nesterov,
    const float* __restrict__ clip, float* __restrict__ partials) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  __shared__ float wsum[MUON_THREADS / 32];
  const int j = blockIdx.y;
  const long long off = muon_off(grp, j);
  const float* G = Gall + off;
  float* M = Mall + off;
  const long long n4 = (long long)grp.rows * grp.cols / 4;
  const float c = clip ? *clip : 1.f;
  float ss = 0.f;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    float4 g = reinterpret_cast<const float4*>(G)[i];
    g.x *= c; g.y *= c; g.z *= c; g.w *= c;
    float4 m = reinterpret_cast<float4*>(M)[i];
    m.x = mu * m.x + (1.f - mu) * g.x;
    m.y = mu * m.y + (1.f - mu) * g.y;
    m.z = mu * m.z + (1.f - mu) * g.z;
    m.w = mu * m.w + (1.f - mu) * g.w;
    reinterpret_cast<float4*>(M)[i] = m;
    const float u0 = muon_u(g.x, m.x, mu, nesterov), u1 = muon_u(g.y, m.y, mu, nesterov);
    const float u2 = muon_u(g.z, m.z, mu, nesterov), u3 = muon_u(g.w, m.w, mu, nesterov);
    ss += (u0 * u0 + u1 * u1) + (u2 * u2 + u3 * u3);
  }
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < MUON_THREADS / 32; ++w) t += wsum[w];
    partials[j * MUON_BATCH_BLOCKS + blockIdx.x] = t;
  }
}

// X_j = bf16(U_j / (||U_j||_F + eps)) into the group's contiguous iterate
// [nmat, rows, cols], U recomputed from the clipped g and the updated m.
__global__ void __launch_bounds__(MUON_THREADS) muon_batch_normalize_kernel(
    const float* __restrict__ Gall, const float* __restrict__ Mall, MuonGroup grp, float mu, int nesterov,
    const float* __restrict__ clip, const float* __restrict__ partials, float eps, bf16* __restrict__ Xall) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  __shared__ float inv_norm;
  const int j = blockIdx.y;
  if (threadIdx.x < 32) {
    float s = 0.f;
    for (int i = threadIdx.x; i < MUON_BATCH_BLOCKS; i += 32) s += partials[j * MUON_BATCH_BLOCKS + i];
    s = warp_sum(s);
    if (threadIdx.x == 0) inv_norm = 1.f / (sqrtf(s) + eps);
  }
  __syncthreads();
  const float inv = inv_norm;
  const long long off = muon_off(grp, j);
  const float* G = Gall + off;
  const float* M = Mall + off;
  const long long n4 = (long long)grp.rows * grp.cols / 4;
  bf16* X = Xall + (long long)j * grp.rows * grp.cols;
  const float c = clip ? *clip : 1.f;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    float4 g = reinterpret_cast<const float4*>(G)[i];
    g.x *= c; g.y *= c; g.z *= c; g.w *= c;
    const float4 m = reinterpret_cast<const float4*>(M)[i];
    const float v[4] = {muon_u(g.x, m.x, mu, nesterov) * inv, muon_u(g.y, m.y, mu, nesterov) * inv,
                        muon_u(g.z, m.z, mu, nesterov) * inv, muon_u(g.w, m.w, mu, nesterov) * inv};
    store4(X + 4 * i, v);
  }
}

// W_j -= step * X_j in the fp32 master, and the bf16 copy the GEMMs read
__global__ void __launch_bounds__(MUON_THREADS) muon_batch_apply_kernel(float* __restrict__ Wall,
                                                                        bf16* __restrict__ Wlp_all,
                                                                        const bf16* __restrict__ Xall,
                                                                        MuonGroup grp, float step) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  const int j = blockIdx.y;
  const long long off = muon_off(grp, j);
  float* W = Wall + off;
  bf16* Wlp = Wlp_all ? Wlp_all + off : nullptr;
  const long long n4 = (long long)grp.rows * grp.cols / 4;
  const bf16* X = Xall + (long long)j * grp.rows * grp.cols;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    float xv[4];
    load4(X + 4 * i, xv);
    float4 w = reinterpret_cast<float4*>(W)[i];
    w.x -= step * xv[0];
    w.y -= step * xv[1];
    w.z -= step * xv[2];
    w.w -= step * xv[3];
    reinterpret_cast<float4*>(W)[i] = w;
    if (Wlp) {
      const float v[4] = {w.x, w.y, w.z, w.w};
      store4(Wlp + 4 * i, v);
    }
  }
}

