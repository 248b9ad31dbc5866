// attention_fa.cuh -- fused causal flash attention, forward and backward,
// bf16 operands, fp32 accumulation, head_dim 128, on the tensor cores
// (warp-level m16n8k16 MMA).
//
// Causal softmax attention as in the "$1000 tier nanochat run" module
// (`F.scaled_dot_product_attention(q, k, v, is_causal=True)`, scale
// 1/sqrt(hd)), computed tile by tile without materialising the T x T scores:
// the forward keeps a running row max and sum (online softmax) and stores the
// log-sum-exp per row; the backward recomputes the probabilities from it.
// The backward is split into a key-block kernel (dK, dV) and a query-block
// kernel (dQ) so that every output element has exactly one writer -- no
// atomics, bit-reproducible.
//
// q, k, v are read in place from the fused projection output qkv [B*T, 3*a]
// (head h of q at column h*128, of k at a + h*128, of v at 2a + h*128); o and
// the gradients use the same token-major layout.  Shared-memory rows of 128
// bf16 are XOR-swizzled in 16-byte chunks (chunk ^ row%8) so ldmatrix is
// bank-conflict free.  Tiles are fetched with cp.async, double-buffered;
// rows at or beyond T are zero-filled.
#pragma once
#include "common.cuh"

namespace fa {

constexpr int HD = 128;
constexpr int ROWB = HD * 2;  // bytes per smem row

__device__ __forceinline__ uint32_t saddr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return (uint32_t)(row * ROWB + ((chunk ^ (row & 7)) << 4));
}
__device__ __forceinline__ void cp16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Copy `rows` rows of 128 bf16 (row stride ld elements, starting at token
// row r0 of a sequence of length T) into a swizzled tile; rows >= T are zero.
__device__ __forceinline__ void load_tile(uint32_t sdst, const bf16* g, long long ld, int r0, int rows, int T,
                                          int tid, int nthreads) {
  for (int i = tid; i < rows * 16; i += nthreads) {
    const int r = i >> 4, c = i & 15;
    const bool valid = (r0 + r) < T;
    const bf16* src = g + (long long)(valid ? (r0 + r) : 0) * ld + c * 8;
    cp16(sdst + swz(r, c), src, valid);
  }
}

// A fragments (16 rows x 16 k) for k-step kk of the 16 rows starting at r0.
__device__ __forceinline__ void lda_frag(uint32_t base, int r0, int kk, int lane, uint32_t (&a)[4]) {
  const int row = r0 + (lane & 15), chunk = kk * 2 + (lane >> 4);
  ldsm_x4(base + swz(row, chunk), a[0], a[1], a[2], a[3]);
}
// B fragments for two n-tiles (rows n0..n0+15 of a [n][k] tile), k-step kk.
__device__ __forceinline__ void ldb_nk(uint32_t base, int n0, int kk, int lane, uint32_t& b0, uint32_t& b1,
                                       uint32_t& b2, uint32_t& b3) {
  const int row = n0 + (lane & 7) + ((lane >> 4) << 3), chunk = kk * 2 + ((lane >> 3) & 1);
  ldsm_x4(base + swz(row, chunk), b0, b1, b2, b3);
}
// B fragments for two n-tiles (columns n0..n0+15) of a [k][n] tile, k rows k0..k0+15.
__device__ __forceinline__ void ldb_kn(uint32_t base, int k0, int n0, int lane, uint32_t& b0, uint32_t& b1,
                                       uint32_t& b2, uint32_t& b3) {
  const int row = k0 + (lane & 7) + (((lane >> 3) & 1) << 3), chunk = (n0 >> 3) + (lane >> 4);
  ldsm_x4_t(base + swz(row, chunk), b0, b1, b2, b3);
}

constexpr float LOG2E = 1.4426950408889634f;

// ------------------------------------------------------------------ forward
// CTA: 128 query rows (8 warps x 16), key tiles of 64, double-buffered.
constexpr int F_BQ = 128, F_BK = 64, F_THREADS = 256;
constexpr int F_SMEM = (F_BQ + 4 * F_BK) * ROWB;

__global__ void __launch_bounds__(F_THREADS) fa_fwd_kernel(const bf16* __restrict__ qkv, bf16* __restrict__ out,
                                                          float* __restrict__ lse_out, int T, int H) {
  extern __shared__ __align__(128) uint8_t sm[];
  const int a = H * HD;
  const long long ld = 3LL * a;
  const int qb = gridDim.x - 1 - blockIdx.x;  // longest (latest) query blocks first
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int q0 = qb * F_BQ;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const bf16* qg = qkv + (long long)b * T * ld + h * HD;
  const bf16* kg = qg + a;
  const bf16* vg = qg + 2 * a;
  const uint32_t sQ = saddr(sm);
  const uint32_t sK0 = sQ + F_BQ * ROWB, sV0 = sK0 + 2 * F_BK * ROWB;
  const int n_kb = min(cdiv(q0 + F_BQ, F_BK), cdiv(T, F_BK));

  load_tile(sQ, qg, ld, q0, F_BQ, T, tid, F_THREADS);
  load_tile(sK0, kg, ld, 0, F_BK, T, tid, F_THREADS);
  load_tile(sV0, vg, ld, 0, F_BK, T, tid, F_THREADS);
  cp_commit();
  cp_wait_all();
  __syncthreads();

  uint32_t qf[8][4];
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) lda_frag(sQ, warp * 16, kk, lane, qf[kk]);

  const float c = rsqrtf((float)HD) * LOG2E;
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  const int row0 = q0 + warp * 16 + g;  // this thread's rows: row0 and row0 + 8

  for (int kb = 0; kb < n_kb; ++kb) {
    const int cur = kb & 1;
    if (kb + 1 < n_kb) {
      const int nxt = cur ^ 1;
      load_tile(sK0 + nxt * F_BK * ROWB, kg, ld, (kb + 1) * F_BK, F_BK, T, tid, F_THREADS);
      load_tile(sV0 + nxt * F_BK * ROWB, vg, ld, (kb + 1) * F_BK, F_BK, T, tid, F_THREADS);
    }
    cp_commit();
    const uint32_t sK = sK0 + cur * F_BK * ROWB, sV = sV0 + cur * F_BK * ROWB;
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        ldb_nk(sK, np * 16, kk, lane, b0, b1, b2, b3);
        mma16816(s[2 * np], qf[kk], b0, b1);
        mma16816(s[2 * np + 1], qf[kk], b2, b3);
      }
    }
    const int k0 = kb * F_BK;
    const bool need_mask = (k0 + F_BK - 1 > q0 + warp * 16) || (k0 + F_BK > T);
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v = s[i][e] * c;
        if (need_mask) {
          const int key = k0 + i * 8 + 2 * t4 + (e & 1);
          const int row = row0 + ((e >> 1) << 3);
          if (key > row || key >= T) v = -INFINITY;
        }
        s[i][e] = v;
      }
    float mx[2] = {m[0], m[1]};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      mx[0] = fmaxf(mx[0], fmaxf(s[i][0], s[i][1]));
      mx[1] = fmaxf(mx[1], fmaxf(s[i][2], s[i][3]));
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
    }
    float alpha[2], sum[2] = {0.f, 0.f}, base[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      base[r] = (mx[r] == -INFINITY) ? 0.f : mx[r];
      alpha[r] = exp2f(m[r] - base[r]);
      m[r] = mx[r];
    }
    uint32_t pa[4][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float p0 = exp2f(s[i][0] - base[0]), p1 = exp2f(s[i][1] - base[0]);
      const float p2 = exp2f(s[i][2] - base[1]), p3 = exp2f(s[i][3] - base[1]);
      sum[0] += p0 + p1;
      sum[1] += p2 + p3;
      // C fragment of n-tile i -> A fragment of k-step i/2
      pa[i >> 1][(i & 1) * 2 + 0] = pack_bf16(p0, p1);
      pa[i >> 1][(i & 1) * 2 + 1] = pack_bf16(p2, p3);
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) l[r] = l[r] * alpha[r] + sum[r];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      o[i][0] *= alpha[0]; o[i][1] *= alpha[0];
      o[i][2] *= alpha[1]; o[i][3] *= alpha[1];
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int np = 0; np < 8; ++np) {
        uint32_t b0, b1, b2, b3;
        ldb_kn(sV, kk * 16, np * 16, lane, b0, b1, b2, b3);
        mma16816(o[2 * np], pa[kk], b0, b1);
        mma16816(o[2 * np + 1], pa[kk], b2, b3);
      }
    }
    cp_wait_all();
    __syncthreads();
  }
  // row sums over the quad
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l[r] += __shfl_xor_sync(0xffffffffu, l[r], 1);
    l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = row0 + r * 8;
    if (row >= T) continue;
    const float inv = 1.f / l[r];
    bf16* orow = out + ((long long)b * T + row) * a + h * HD;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      *reinterpret_cast<uint32_t*>(orow + i * 8 + 2 * t4) = pack_bf16(o[i][2 * r] * inv, o[i][2 * r + 1] * inv);
    }
    if (t4 == 0) lse_out[(long long)bh * T + row] = (m[r] + log2f(l[r])) * 0.6931471805599453f;
  }
}

// ------------------------------------------------------------------ backward: dK, dV
// CTA: 64 keys (4 warps x 16); query tiles of 64 from the diagonal on.
constexpr int B_BK = 64, B_BQ = 64, B_THREADS = 128;
constexpr int B_SMEM = (2 * B_BK + 4 * B_BQ) * ROWB + 4 * B_BQ * 4;

__global__ void __launch_bounds__(B_THREADS) fa_bwd_dkdv_kernel(const bf16* __restrict__ qkv,
                                                               const bf16* __restrict__ dout,
                                                               const float* __restrict__ lse,
                                                               const float* __restrict__ Dv,
                                                               bf16* __restrict__ dqkv, int T, int H) {
  extern __shared__ __align__(128) uint8_t sm[];
  const int a = H * HD;
  const long long ld = 3LL * a;
  const int kb = gridDim.x - 1 - blockIdx.x;
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int k0 = kb * B_BK;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const bf16* qg = qkv + (long long)b * T * ld + h * HD;
  const bf16* kg = qg + a;
  const bf16* vg = qg + 2 * a;
  const bf16* og = dout + (long long)b * T * a + h * HD;
  const uint32_t sK = saddr(sm), sV = sK + B_BK * ROWB;
  const uint32_t sQ0 = sV + B_BK * ROWB, sO0 = sQ0 + 2 * B_BQ * ROWB;
  float* sL = reinterpret_cast<float*>(sm + (2 * B_BK + 4 * B_BQ) * ROWB);  // [2][64] lse*log2e
  float* sD = sL + 2 * B_BQ;                                               // [2][64] D
  const float* lse_bh = lse + (long long)bh * T;
  const float* D_bh = Dv + (long long)bh * T;

  const int qb_first = k0 / B_BQ, n_qb = cdiv(T, B_BQ);
  load_tile(sK, kg, ld, k0, B_BK, T, tid, B_THREADS);
  load_tile(sV, vg, ld, k0, B_BK, T, tid, B_THREADS);
  auto load_q = [&](int qb, int buf) {
    load_tile(sQ0 + buf * B_BQ * ROWB, qg, ld, qb * B_BQ, B_BQ, T, tid, B_THREADS);
    load_tile(sO0 + buf * B_BQ * ROWB, og, a, qb * B_BQ, B_BQ, T, tid, B_THREADS);
    for (int i = tid; i < B_BQ; i += B_THREADS) {
      const int q = qb * B_BQ + i;
      sL[buf * B_BQ + i] = (q < T) ? lse_bh[q] * LOG2E : INFINITY;
      sD[buf * B_BQ + i] = (q < T) ? D_bh[q] : 0.f;
    }
  };
  if (qb_first < n_qb) load_q(qb_first, 0);
  cp_commit();
  cp_wait_all();
  __syncthreads();

  const float c = rsqrtf((float)HD) * LOG2E;
  float dk[16][4], dv[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[i][e] = dv[i][e] = 0.f;
  const int key0 = k0 + warp * 16 + g;  // this thread's keys: key0 and key0 + 8

  for (int qb = qb_first; qb < n_qb; ++qb) {
    const int cur = (qb - qb_first) & 1;
    __syncthreads();  // the other buffer is free
    if (qb + 1 < n_qb) load_q(qb + 1, cur ^ 1);
    cp_commit();
    const uint32_t sQ = sQ0 + cur * B_BQ * ROWB, sO = sO0 + cur * B_BQ * ROWB;
    const float* L = sL + cur * B_BQ;
    const float* Dq = sD + cur * B_BQ;
    const int qs = qb * B_BQ;
    // S^T = K Q^T  (16 keys x 64 queries per warp)
    float st[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) st[i][0] = st[i][1] = st[i][2] = st[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t af[4];
      lda_frag(sK, warp * 16, kk, lane, af);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        ldb_nk(sQ, np * 16, kk, lane, b0, b1, b2, b3);
        mma16816(st[2 * np], af, b0, b1);
        mma16816(st[2 * np + 1], af, b2, b3);
      }
    }
    // P^T = exp2(S^T c - lse_q log2e), causal: key <= query
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int ql = i * 8 + 2 * t4 + (e & 1);
        const int key = key0 + ((e >> 1) << 3);
        const float p = exp2f(st[i][e] * c - L[ql]);
        st[i][e] = (key <= qs + ql) ? p : 0.f;
      }
    // dV += P^T dO
    {
      uint32_t pa[4][4];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        pa[i >> 1][(i & 1) * 2 + 0] = pack_bf16(st[i][0], st[i][1]);
        pa[i >> 1][(i & 1) * 2 + 1] = pack_bf16(st[i][2], st[i][3]);
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
#pragma unroll
        for (int np = 0; np < 8; ++np) {
          uint32_t b0, b1, b2, b3;
          ldb_kn(sO, kk * 16, np * 16, lane, b0, b1, b2, b3);
          mma16816(dv[2 * np], pa[kk], b0, b1);
          mma16816(dv[2 * np + 1], pa[kk], b2, b3);
        }
    }
    // dP^T = V dO^T, dS^T = P^T (dP^T - D_q)
    float dpt[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) dpt[i][0] = dpt[i][1] = dpt[i][2] = dpt[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t af[4];
      lda_frag(sV, warp * 16, kk, lane, af);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        ldb_nk(sO, np * 16, kk, lane, b0, b1, b2, b3);
        mma16816(dpt[2 * np], af, b0, b1);
        mma16816(dpt[2 * np + 1], af, b2, b3);
      }
    }
    uint32_t da[4][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float d[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) d[e] = st[i][e] * (dpt[i][e] - Dq[i * 8 + 2 * t4 + (e & 1)]);
      da[i >> 1][(i & 1) * 2 + 0] = pack_bf16(d[0], d[1]);
      da[i >> 1][(i & 1) * 2 + 1] = pack_bf16(d[2], d[3]);
    }
    // dK += dS^T Q
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
      for (int np = 0; np < 8; ++np) {
        uint32_t b0, b1, b2, b3;
        ldb_kn(sQ, kk * 16, np * 16, lane, b0, b1, b2, b3);
        mma16816(dk[2 * np], da[kk], b0, b1);
        mma16816(dk[2 * np + 1], da[kk], b2, b3);
      }
    cp_wait_all();
  }
  const float scale = rsqrtf((float)HD);
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int key = key0 + r * 8;
    if (key >= T) continue;
    bf16* krow = dqkv + ((long long)b * T + key) * ld + a + h * HD;
    bf16* vrow = krow + a;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      *reinterpret_cast<uint32_t*>(krow + i * 8 + 2 * t4) = pack_bf16(dk[i][2 * r] * scale, dk[i][2 * r + 1] * scale);
      *reinterpret_cast<uint32_t*>(vrow + i * 8 + 2 * t4) = pack_bf16(dv[i][2 * r], dv[i][2 * r + 1]);
    }
  }
}

// ------------------------------------------------------------------ backward: dQ
// CTA: 64 queries (4 warps x 16); key tiles of 64 up to the diagonal.
constexpr int Q_SMEM = (2 * B_BQ + 4 * B_BK) * ROWB;

__global__ void __launch_bounds__(B_THREADS) fa_bwd_dq_kernel(const bf16* __restrict__ qkv,
                                                             const bf16* __restrict__ dout,
                                                             const float* __restrict__ lse,
                                                             const float* __restrict__ Dv,
                                                             bf16* __restrict__ dqkv, int T, int H) {
  extern __shared__ __align__(128) uint8_t sm[];
  const int a = H * HD;
  const long long ld = 3LL * a;
  const int qb = gridDim.x - 1 - blockIdx.x;
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int q0 = qb * B_BQ;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const bf16* qg = qkv + (long long)b * T * ld + h * HD;
  const bf16* kg = qg + a;
  const bf16* vg = qg + 2 * a;
  const bf16* og = dout + (long long)b * T * a + h * HD;
  const uint32_t sQ = saddr(sm), sO = sQ + B_BQ * ROWB;
  const uint32_t sK0 = sO + B_BQ * ROWB, sV0 = sK0 + 2 * B_BK * ROWB;
  const int n_kb = min(cdiv(q0 + B_BQ, B_BK), cdiv(T, B_BK));

  load_tile(sQ, qg, ld, q0, B_BQ, T, tid, B_THREADS);
  load_tile(sO, og, a, q0, B_BQ, T, tid, B_THREADS);
  load_tile(sK0, kg, ld, 0, B_BK, T, tid, B_THREADS);
  load_tile(sV0, vg, ld, 0, B_BK, T, tid, B_THREADS);
  cp_commit();
  cp_wait_all();
  __syncthreads();

  uint32_t qf[8][4], of[8][4];
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    lda_frag(sQ, warp * 16, kk, lane, qf[kk]);
    lda_frag(sO, warp * 16, kk, lane, of[kk]);
  }
  const int row0 = q0 + warp * 16 + g;
  float Lr[2], Dr[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = row0 + r * 8;
    Lr[r] = (row < T) ? lse[(long long)bh * T + row] * LOG2E : INFINITY;
    Dr[r] = (row < T) ? Dv[(long long)bh * T + row] : 0.f;
  }
  const float c = rsqrtf((float)HD) * LOG2E;
  float dq[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) dq[i][0] = dq[i][1] = dq[i][2] = dq[i][3] = 0.f;

  for (int kb = 0; kb < n_kb; ++kb) {
    const int cur = kb & 1;
    if (kb + 1 < n_kb) {
      load_tile(sK0 + (cur ^ 1) * B_BK * ROWB, kg, ld, (kb + 1) * B_BK, B_BK, T, tid, B_THREADS);
      load_tile(sV0 + (cur ^ 1) * B_BK * ROWB, vg, ld, (kb + 1) * B_BK, B_BK, T, tid, B_THREADS);
    }
    cp_commit();
    const uint32_t sK = sK0 + cur * B_BK * ROWB, sV = sV0 + cur * B_BK * ROWB;
    const int k0 = kb * B_BK;
    float s[8][4], dp[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[i][e] = dp[i][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        ldb_nk(sK, np * 16, kk, lane, b0, b1, b2, b3);
        mma16816(s[2 * np], qf[kk], b0, b1);
        mma16816(s[2 * np + 1], qf[kk], b2, b3);
        ldb_nk(sV, np * 16, kk, lane, b0, b1, b2, b3);
        mma16816(dp[2 * np], of[kk], b0, b1);
        mma16816(dp[2 * np + 1], of[kk], b2, b3);
      }
    uint32_t da[4][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float d[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = k0 + i * 8 + 2 * t4 + (e & 1);
        const int r = e >> 1;
        const int row = row0 + r * 8;
        const float p = (key <= row && key < T) ? exp2f(s[i][e] * c - Lr[r]) : 0.f;
        d[e] = p * (dp[i][e] - Dr[r]);
      }
      da[i >> 1][(i & 1) * 2 + 0] = pack_bf16(d[0], d[1]);
      da[i >> 1][(i & 1) * 2 + 1] = pack_bf16(d[2], d[3]);
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
      for (int np = 0; np < 8; ++np) {
        uint32_t b0, b1, b2, b3;
        ldb_kn(sK, kk * 16, np * 16, lane, b0, b1, b2, b3);
        mma16816(dq[2 * np], da[kk], b0, b1);
        mma16816(dq[2 * np + 1], da[kk], b2, b3);
      }
    cp_wait_all();
    __syncthreads();
  }
  const float scale = rsqrtf((float)HD);
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = row0 + r * 8;
    if (row >= T) continue;
    bf16* qrow = dqkv + ((long long)b * T + row) * ld + h * HD;
#pragma unroll
    for (int i = 0; i < 16; ++i)
      *reinterpret_cast<uint32_t*>(qrow + i * 8 + 2 * t4) = pack_bf16(dq[i][2 * r] * scale, dq[i][2 * r + 1] * scale);
  }
}

}  // namespace fa
