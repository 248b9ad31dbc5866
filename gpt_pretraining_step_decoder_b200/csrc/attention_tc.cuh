// attention_tc.cuh -- causal flash attention forward on the 5th-generation
// tensor cores (tcgen05 + TMEM + TMA), bf16 in, fp32 accumulate, head_dim 128.
//
// Same operation as fa::fa_fwd_kernel (causal softmax attention with scale
// 1/sqrt(hd), "$1000 tier nanochat run", `F.scaled_dot_product_attention(...,
// is_causal=True)`): o = softmax(q k^T / sqrt(hd) + causal) v and the row
// log-sum-exp for the backward pass.
//
// One CTA per (128-query tile, sequence, head), heaviest tiles first:
//   warp 0      TMA: Q once, then K_j and V_j (128 keys) into 2-deep rings
//               with separate barriers, so K_{j+2} loads as soon as S_j
//               has read K_j;
//   warp 1      one thread issues S_j = Q K_j^T into TMEM (two S buffers, so
//               S_{j+1} is computed while row j's softmax runs) and
//               O += P_j V_j into a TMEM accumulator;
//   warps 2..5  softmax, one query row per thread: read S_j from TMEM, mask,
//               running max, exp2, row sum, write P_j as bf16 into a swizzled
//               shared-memory tile (the MMA's A operand, double-buffered).
//               O is rescaled in TMEM only when a row max grows by more than
//               2^8 (log2 units) over the max in use, so most tiles skip it;
//               the exponentials then stay below 2^8, safe in fp32 and bf16.
// Epilogue: O / l to bf16 o, lse = (m + log2 l) ln 2.  Every wait is bounded.
#pragma once
#include "gemm_tc.cuh"

namespace fatc {

constexpr int BQ = 128, BKV = 128, HD = 128;
constexpr int THREADS = 192;
constexpr int TILE_BYTES = 128 * 128 * 2;          // one 128 x 128 bf16 tile
constexpr int SMEM_BYTES = TILE_BYTES /*Q*/ + 2 * 2 * TILE_BYTES /*K,V x 2 stages*/ +
                           2 * TILE_BYTES /*P x 2*/ + 1024 /*align*/ + 256 /*barriers*/;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float RESCALE_THRESHOLD = 8.f;  // log2 units

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// K-major 128 x 128 operand tile = two 128 x 64 sub-tiles (128-byte swizzle);
// descriptor of MMA k-step k (16 elements along K).
__device__ __forceinline__ uint64_t kmaj_desc(uint32_t base, int k) {
  return tc::smem_desc(base + (k >> 2) * (TILE_BYTES / 2) + (k & 3) * 32, 16, 1024);
}
// MN-major 128 (N) x 128 (K) operand tile = two K-blocks of 64 rows, each two
// 64-wide N chunks of 8 KB; descriptor of MMA k-step k.
__device__ __forceinline__ uint64_t mnmaj_desc(uint32_t base, int k) {
  return tc::smem_desc(base + (k >> 2) * (TILE_BYTES / 2) + (k & 3) * 2048, 8192, 1024);
}

__global__ void __launch_bounds__(THREADS, 1)
    fa_tc_fwd_kernel(const __grid_constant__ CUtensorMap tmQK, const __grid_constant__ CUtensorMap tmV,
                     bf16* __restrict__ out, float* __restrict__ lse_out, int T, int H, unsigned* err) {
  using namespace tc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + TILE_BYTES;            // [2 stages]
  uint8_t* sV = sK + 2 * TILE_BYTES;        // [2 stages]
  uint8_t* sP = sV + 2 * TILE_BYTES;        // [2 buffers]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + 2 * TILE_BYTES);
  uint64_t* q_full = bars;                  // 1
  uint64_t* k_full = bars + 1;              // 2
  uint64_t* k_empty = bars + 3;             // 2 (S_j done with K_j)
  uint64_t* v_full = bars + 5;              // 2
  uint64_t* v_empty = bars + 7;             // 2 (PV_j done with V_j)
  uint64_t* s_full = bars + 9;              // 2
  uint64_t* s_empty = bars + 11;            // 2
  uint64_t* p_full = bars + 13;             // 2
  uint64_t* p_free = bars + 15;             // 2 (PV_j done: P buffer and O are free)
  uint64_t* o_full = bars + 17;             // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 18);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = gridDim.x - 1 - blockIdx.x;  // heaviest tiles first
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int a = H * HD;
  const int q0 = qt * BQ;
  const int n_kv = min(qt + 1, (T + BKV - 1) / BKV);
  const int row_base = b * T;  // token row of position 0 of this sequence

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], 128);
      mbar_init(&p_full[s], 128);
      mbar_init(&p_free[s], 1);
    }
    mbar_init(o_full, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;  // S0: cols 0..127, S1: 128..255, O: 256..383

  if (warp == 0) {
    if (lane < 2) {
      // ---------------------------------------------------------------- TMA
      // lane 0 streams Q and the K tiles, lane 1 the V tiles: a K buffer is
      // refilled as soon as S_j has read it, independently of PV_j.
      const bool is_k = lane == 0;
      uint64_t* full = is_k ? k_full : v_full;
      uint64_t* empty = is_k ? k_empty : v_empty;
      bool ok = true;
      if (is_k) {
        mbar_expect_tx(q_full, TILE_BYTES);
        tma_load_2d(sQ, &tmQK, q_full, h * HD, row_base + q0);
        tma_load_2d(sQ + TILE_BYTES / 2, &tmQK, q_full, h * HD + 64, row_base + q0);
      }
      int issued = 0;
      for (int j = 0; j < n_kv && ok; ++j) {
        const int s = j & 1;
        if (!mbar_wait(&empty[s], ((j >> 1) & 1) ^ 1, abort_flag, err)) { ok = false; break; }
        mbar_expect_tx(&full[s], TILE_BYTES);
        const int kr = row_base + j * BKV;
        if (is_k) {
          uint8_t* k = sK + s * TILE_BYTES;
          tma_load_2d(k, &tmQK, &full[s], a + h * HD, kr);
          tma_load_2d(k + TILE_BYTES / 2, &tmQK, &full[s], a + h * HD + 64, kr);
        } else {
          // V as an MN-major operand: K-block kb (keys 64kb..), N chunk nc (hd 64nc..)
          uint8_t* v = sV + s * TILE_BYTES;
          for (int kb = 0; kb < 2; ++kb)
            for (int nc = 0; nc < 2; ++nc)
              tma_load_2d(v + kb * (TILE_BYTES / 2) + nc * 8192, &tmV, &full[s], 2 * a + h * HD + 64 * nc,
                          kr + 64 * kb);
        }
        ++issued;
      }
      // let every copy land before the CTA can exit
      const uint64_t t0 = globaltimer_ns();
      if (is_k)
        while (!mbar_try_wait(q_full, 0)) if (globaltimer_ns() - t0 > GPT_WAIT_LIMIT_NS) break;
      for (int j = (issued > 2 ? issued - 2 : 0); j < issued; ++j) {
        const uint64_t t1 = globaltimer_ns();
        while (!mbar_try_wait(&full[j & 1], (j >> 1) & 1))
          if (globaltimer_ns() - t1 > GPT_WAIT_LIMIT_NS) break;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA
      // S = Q K^T: A = Q (K-major), B = K (K-major), N = 128
      const uint32_t idesc_s = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(128 >> 3) << 17) |
                               ((uint32_t)(128 >> 4) << 24);
      // O += P V: A = P (K-major), B = V (MN-major), N = 128
      const uint32_t idesc_o = idesc_s | (1u << 16);
      const uint32_t aQ = smem_u32(sQ);
      bool ok = mbar_wait(q_full, 0, abort_flag, err);
      for (int j = 0; j <= n_kv && ok; ++j) {
        if (j < n_kv) {
          const int s = j & 1;
          if (!mbar_wait(&k_full[s], (j >> 1) & 1, abort_flag, err)) { ok = false; break; }
          if (!mbar_wait(&s_empty[s], ((j >> 1) & 1) ^ 1, abort_flag, err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t aK = smem_u32(sK + s * TILE_BYTES);
#pragma unroll
          for (int k = 0; k < HD / 16; ++k)
            tc_mma(tmem + s * 128, kmaj_desc(aQ, k), kmaj_desc(aK, k), idesc_s, k > 0 ? 1u : 0u);
          tc_commit(&s_full[s]);
          tc_commit(&k_empty[s]);
        }
        if (j >= 1) {
          const int jp = j - 1, s = jp & 1;
          if (!mbar_wait(&p_full[s], (jp >> 1) & 1, abort_flag, err)) { ok = false; break; }
          if (!mbar_wait(&v_full[s], (jp >> 1) & 1, abort_flag, err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t aP = smem_u32(sP + s * TILE_BYTES);
          const uint32_t aV = smem_u32(sV + s * TILE_BYTES);
#pragma unroll
          for (int k = 0; k < BKV / 16; ++k)
            tc_mma(tmem + 256, kmaj_desc(aP, k), mnmaj_desc(aV, k), idesc_o, (jp > 0 || k > 0) ? 1u : 0u);
          tc_commit(&p_free[s]);
          tc_commit(&v_empty[s]);
          if (jp == n_kv - 1) tc_commit(o_full);
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax
    const int q = warp & 3;
    const int r = q * 32 + lane;               // row within the tile
    const int qpos = q0 + r;                   // query position in the sequence
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const float c = rsqrtf((float)HD) * LOG2E;
    float m_use = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int s = j & 1;
      if (!warp_wait(&s_full[s], (j >> 1) & 1, abort_flag, err)) { ok = false; break; }
      tc_fence_after();
      float sv[128];
      {
        uint32_t r0[32], r1[32], r2[32], r3[32];
        const uint32_t base = tmem + lane_off + s * 128;
        tmem_ld32_nowait(base, r0);
        tmem_ld32_nowait(base + 32, r1);
        tmem_ld32_nowait(base + 64, r2);
        tmem_ld32_nowait(base + 96, r3);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          sv[i] = __uint_as_float(r0[i]);
          sv[32 + i] = __uint_as_float(r1[i]);
          sv[64 + i] = __uint_as_float(r2[i]);
          sv[96 + i] = __uint_as_float(r3[i]);
        }
      }
      tc_fence_before();
      mbar_arrive(&s_empty[s]);  // the S buffer may be overwritten
      const int k0 = j * BKV;
      if (k0 + BKV - 1 > qpos) {  // causal mask on the diagonal tile
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (k0 + i > qpos) sv[i] = -INFINITY;
      }
      // row max of the raw scores (the scale c > 0 commutes with max), as 8
      // independent partial maxima so the reduction is not one long chain
      float pm[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) pm[u] = sv[u];
#pragma unroll
      for (int i = 8; i < 128; ++i) pm[i & 7] = fmaxf(pm[i & 7], sv[i]);
      const float mx = c * fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                                 fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
      if (j == 0) {
        m_use = mx;
      } else if (__any_sync(0xffffffffu, mx > m_use + RESCALE_THRESHOLD)) {
        // grow the max in use: O_{<j} and l scale by 2^(m_old - m_new); the
        // previous PV product must have landed in O first.  The decision is
        // warp-wide (the TMEM accesses below are warp-collective); rows whose
        // max did not grow rescale by exactly 1.
        const float m_new = fmaxf(m_use, mx);
        const float alpha = exp2f(m_use - m_new);
        if (!warp_wait(&p_free[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t ob = tmem + lane_off + 256;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t o[32];
          tmem_ld32_nowait(ob + cc * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(ob + cc * 32, o);
        }
        tmem_wait_st();
        l *= alpha;
        m_use = m_new;
      }
      // P_j = exp2(s - m_use) as bf16 into the P buffer of this parity, once
      // the PV product that read it two tiles ago is done
      if (j >= 2 && !warp_wait(&p_free[s], ((j - 2) >> 1) & 1, abort_flag, err)) { ok = false; break; }
      uint8_t* pb = sP + s * TILE_BYTES;
      float ps[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // 8 independent partial sums
      const float nm = -m_use;
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {  // 16 chunks of 8 keys
        float p[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) { p[e] = exp2f(fmaf(sv[ch * 8 + e], c, nm)); ps[e] += p[e]; }
        uint4 w;
        __nv_bfloat162 b0 = __floats2bfloat162_rn(p[0], p[1]), b1 = __floats2bfloat162_rn(p[2], p[3]);
        __nv_bfloat162 b2 = __floats2bfloat162_rn(p[4], p[5]), b3 = __floats2bfloat162_rn(p[6], p[7]);
        w.x = *reinterpret_cast<uint32_t*>(&b0); w.y = *reinterpret_cast<uint32_t*>(&b1);
        w.z = *reinterpret_cast<uint32_t*>(&b2); w.w = *reinterpret_cast<uint32_t*>(&b3);
        const int sub = ch >> 3, jj = ch & 7;
        *reinterpret_cast<uint4*>(pb + sub * (TILE_BYTES / 2) + r * 128 + ((jj ^ (r & 7)) << 4)) = w;
      }
      l += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
      mbar_arrive(&p_full[s]);
    }
    // ---------------------------------------------------------------- epilogue
    if (__all_sync(0xffffffffu, ok) && warp_wait(o_full, 0, abort_flag, err)) {
      tc_fence_after();
      const float inv = 1.f / l;
      const uint32_t ob = tmem + lane_off + 256;
      bf16* orow = out + ((long long)row_base + qpos) * a + h * HD;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t o[32];
        tmem_ld32_nowait(ob + cc * 32, o);
        tmem_wait_ld();
        if (qpos < T) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 w;
            __nv_bfloat162 b0 = __floats2bfloat162_rn(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv);
            __nv_bfloat162 b1 = __floats2bfloat162_rn(__uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
            __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(o[i + 4]) * inv, __uint_as_float(o[i + 5]) * inv);
            __nv_bfloat162 b3 = __floats2bfloat162_rn(__uint_as_float(o[i + 6]) * inv, __uint_as_float(o[i + 7]) * inv);
            w.x = *reinterpret_cast<uint32_t*>(&b0); w.y = *reinterpret_cast<uint32_t*>(&b1);
            w.z = *reinterpret_cast<uint32_t*>(&b2); w.w = *reinterpret_cast<uint32_t*>(&b3);
            *reinterpret_cast<uint4*>(orow + cc * 32 + i) = w;
          }
        }
      }
      if (qpos < T) lse_out[(long long)bh * T + qpos] = (m_use + log2f(l)) * 0.6931471805599453f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

}  // namespace fatc
