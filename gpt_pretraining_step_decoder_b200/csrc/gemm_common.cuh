// gemm_common.cuh -- operand and epilogue description shared by the GEMMs.
//
// Every dense contraction of the step is C[m, n] = sum_k A[m, k] * B[n, k]
// followed by an epilogue.  Operands are row-major buffers read either
// K-major (element [r, k] at ptr[r * ld + k]) or MN-major (element [r, k] at
// ptr[k * ld + r]); this covers forward (x W^T), data-gradient (dY W) and
// weight-gradient (dY^T X) products without any transposed copies.
#pragma once
#include "common.cuh"

struct GemmOperand {
  const void* ptr;
  long long ld;   // elements between consecutive rows of the stored buffer
  int kmajor;     // 1: [rows, K] storage; 0: [K, rows] storage
};

enum EpiMode {
  EPI_STORE = 0,      // C(act) = alpha * acc
  EPI_STORE_F32 = 1,  // C(f32) = alpha * acc
  EPI_ACCUM_F32 = 2,  // C(f32) = (beta ? C : 0) + alpha * acc
  EPI_RELU2 = 3,      // C(act) = relu(acc)^2                        (ReLU^2 forward)
  EPI_DRELU2 = 4,     // C(act) = 2 * sqrt(aux(act)) * acc, aux = relu(a)^2  (ReLU^2 backward:
                      // d relu(a)^2 / da = 2 relu(a) = 2 sqrt(relu(a)^2))
  EPI_LOGITS = 5,     // z = softcap(acc); per (row, column tile) m = max z and
                      // s = sum exp(z - m) into stats; C(bf16) = exp(z - m) (the tile-local
                      // softmax numerators); z at the row's target column into ztgt
                      // (tensor-core path only)
  EPI_QKV = 6,        // fused q|k|v projection output (tensor-core path, 128-wide heads):
                      // q, k heads rotated (RoPE) and RMS-normalised per head, v heads plus
                      // the value-table row; C(act) = result
  EPI_AXPBY = 7,      // C(act) = alpha * acc + aux_scale * aux(act), aux of C's shape and ld
                      // (the Newton-Schulz polynomial's combinations; tensor-core path)
};

struct GemmEpilogue {
  int mode;
  void* C;          // output [M, ldc]
  long long ldc;
  void* C2;         // unused second output
  const void* aux;  // EPI_DRELU2 input relu(a)^2, EPI_AXPBY input; same ld as C
  float alpha;
  int beta;
  float softcap;    // EPI_LOGITS: 0 = off, else z = softcap * tanh(acc / softcap)
  float2* stats;    // EPI_LOGITS: [M, n_tiles] (max, sum of exp(z - max))
  const int32_t* targets;  // EPI_LOGITS: target column per row (< 0: none), nullable
  float* ztgt;             // EPI_LOGITS: z at the target column per row
  // EPI_QKV: RoPE turns per position of the 64 frequencies ([64] float2, an
  // fp32 hi + lo pair each), per-(row, head) rstd outputs, optional value
  // table [rows, H*128] (bf16) and its row per position
  const float2* rope;
  float* rstd_q;
  float* rstd_k;
  const void* hv;
  const int32_t* rv;
  int T, H, qk_norm;
  float eps;
  // FP8 path: acc is further multiplied by *scale_a * *scale_b (device scalars; null = 1)
  const float* scale_a;
  const float* scale_b;
  float aux_scale;  // EPI_AXPBY
};

template <typename act_t>
__device__ __forceinline__ void epi_apply_one(const GemmEpilogue& e, long long m, long long n,
                                              float acc) {
  const long long off = m * e.ldc + n;
  acc *= e.alpha;
  switch (e.mode) {
    case EPI_STORE: reinterpret_cast<act_t*>(e.C)[off] = from_f<act_t>(acc); break;
    case EPI_STORE_F32: reinterpret_cast<float*>(e.C)[off] = acc; break;
    case EPI_ACCUM_F32: {
      float* c = reinterpret_cast<float*>(e.C);
      c[off] = (e.beta ? c[off] : 0.f) + acc;
      break;
    }
    case EPI_RELU2: {
      const float r = fmaxf(acc, 0.f);
      reinterpret_cast<act_t*>(e.C)[off] = from_f<act_t>(r * r);
      break;
    }
    case EPI_DRELU2: {
      const float g = to_f(reinterpret_cast<const act_t*>(e.aux)[off]);
      reinterpret_cast<act_t*>(e.C)[off] = from_f<act_t>(2.f * sqrtf(g) * acc);
      break;
    }
    case EPI_AXPBY: {
      const float g = to_f(reinterpret_cast<const act_t*>(e.aux)[off]);
      reinterpret_cast<act_t*>(e.C)[off] = from_f<act_t>(acc + e.aux_scale * g);
      break;
    }
    default:  // EPI_LOGITS and EPI_QKV exist only in the tensor-core kernel's epilogue
      break;
  }
}

// Sum split-K partials [S, M, N] (fp32, in split order) into the epilogue.
template <typename act_t>
__global__ void splitk_reduce_kernel(const float* __restrict__ part, int S, int M, int N,
                                     GemmEpilogue e) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  const long long total = (long long)M * N;
  const bool vec = (N % 4) == 0 && (e.ldc % 4) == 0 && (e.mode == EPI_ACCUM_F32 || e.mode == EPI_STORE_F32);
  if (vec) {
    // four consecutive columns of one row per thread (same sum order per element)
    const long long total4 = total / 4;
    for (long long i4 = (long long)blockIdx.x * blockDim.x + threadIdx.x; i4 < total4;
         i4 += (long long)gridDim.x * blockDim.x) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s = 0; s < S; ++s) {
        const float4 v = reinterpret_cast<const float4*>(part + (long long)s * total)[i4];
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
      }
      const long long i = i4 * 4, m = i / N, n = i % N;
      float4* c = reinterpret_cast<float4*>(reinterpret_cast<float*>(e.C) + m * e.ldc + n);
      if (e.mode == EPI_ACCUM_F32 && e.beta) {
        const float4 o = *c;
        acc.x = o.x + acc.x * e.alpha; acc.y = o.y + acc.y * e.alpha;
        acc.z = o.z + acc.z * e.alpha; acc.w = o.w + acc.w * e.alpha;
      } else {
        acc.x *= e.alpha; acc.y *= e.alpha; acc.z *= e.alpha; acc.w *= e.alpha;
      }
      *c = acc;
    }
    return;
  }
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < S; ++s) acc += part[(long long)s * total + i];
    epi_apply_one<act_t>(e, i / N, i % N, acc);
  }
}
