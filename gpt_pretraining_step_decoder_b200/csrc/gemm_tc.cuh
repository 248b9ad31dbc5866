// gemm_tc.cuh -- bf16 GEMM on the 5th-generation tensor cores (sm_100a).
//
// C[m, n] = sum_k A[m, k] B[n, k] with bf16 operands and fp32 accumulation in
// tensor memory, followed by one of the epilogues of gemm_common.cuh.
//
// Design (one CTA per SM, persistent over output tiles):
//   warp 0      one elected thread issues TMA tile loads (128-byte swizzle)
//               into a STAGES-deep shared-memory ring;
//   warp 1      allocates TMEM and one elected thread issues tcgen05.mma
//               (M = 128, N = BN, K = 16 per instruction) into one of two
//               TMEM accumulators, committing to mbarriers;
//   warps 2..5  the epilogue: tcgen05.ld of the finished accumulator (one
//               TMEM lane = one output row per thread), apply the epilogue,
//               store to global, release the accumulator.
// The two accumulators let the epilogue of tile i overlap the MMAs of tile
// i + 1.  K-major and MN-major operands are both read straight from their
// row-major buffers (the UMMA descriptor's major-ness bit), so forward,
// data-gradient and weight-gradient products need no transposed copies.
// Split-K writes fp32 partials that a second kernel sums in split order
// (deterministic; no atomics).  Every mbarrier wait is bounded: on timeout
// the CTA sets GPT_EBIT_TIMEOUT, stops issuing work, waits (bounded) for its
// own TMA copies in flight and frees its TMEM before returning.
#pragma once
#include <cuda.h>
#include "gemm_common.cuh"

namespace tc {

constexpr int BM = 128;
constexpr int BK = 64;  // bf16 elements per 128-byte swizzle row
constexpr int NUM_THREADS = 192;

template <int BN> struct Cfg {
  static constexpr int STAGES = (BN == 256) ? 4 : 6;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN;  // two accumulators (power of two >= 32)
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
};

struct Params {
  int M, N, K;
  int a_kmajor, b_kmajor;
  int m_tiles, n_tiles, splits, kb_per_split, kb_total;
  GemmEpilogue epi;
  float* partial;  // splits > 1: fp32 [splits, M, N]
  unsigned* err;
};

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait on `bar` reaching `parity`.  Returns false (and raises the
// CTA's abort flag and the device error word) when the budget runs out or
// another role of this CTA has already aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > GPT_WAIT_LIMIT_NS) {
        *abort_flag = 1;
        set_error(err, GPT_EBIT_TIMEOUT);
        return false;
      }
    }
  }
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor (sm_100 format): start address, leading
// and stride byte offsets (16-byte units), version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Load one operand tile (rows x BK) of the k-block `kb` into `dst`.
// K-major: one box {BK, rows}.  MN-major: rows/64 boxes {64, BK}, each 8 KB.
__device__ __forceinline__ void load_operand(uint8_t* dst, const CUtensorMap* map, uint64_t* bar,
                                             int kmajor, int rows, int r0, int kb) {
  if (kmajor) {
    tma_load_2d(dst, map, bar, kb * BK, r0);
  } else {
    for (int j = 0; j < rows / 64; ++j) tma_load_2d(dst + j * 64 * BK * 2, map, bar, r0 + 64 * j, kb * BK);
  }
}

// Descriptor of UMMA k-step `k` (16 elements of K) inside an operand tile.
__device__ __forceinline__ uint64_t operand_desc(uint32_t base, int kmajor, int k) {
  if (kmajor) return smem_desc(base + k * 32, 16, 1024);
  return smem_desc(base + k * 16 * 128, 64 * BK * 2, 1024);
}

template <typename act_t>
__device__ __forceinline__ void epilogue_row32(const Params& p, long long m, int n0,
                                               const uint32_t (&r)[32], int split) {
  const GemmEpilogue& e = p.epi;
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  if (m >= p.M) return;
  if (p.splits > 1) {
    float* dst = p.partial + ((long long)split * p.M + m) * p.N + n0;
    if (n0 + 32 <= p.N) {
#pragma unroll
      for (int i = 0; i < 32; i += 4) store4(dst + i, &v[i]);
    } else {
      for (int i = 0; i < 32 && n0 + i < p.N; ++i) dst[i] = v[i];
    }
    return;
  }
  if (n0 + 32 > p.N) {
    for (int i = 0; i < 32 && n0 + i < p.N; ++i) epi_apply_one<act_t>(e, m, n0 + i, v[i]);
    return;
  }
  const long long off = m * e.ldc + n0;
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] *= e.alpha;
  switch (e.mode) {
    case EPI_STORE: {
      act_t* c = reinterpret_cast<act_t*>(e.C) + off;
#pragma unroll
      for (int i = 0; i < 32; i += 4) store4(c + i, &v[i]);
      break;
    }
    case EPI_STORE_F32: {
      float* c = reinterpret_cast<float*>(e.C) + off;
#pragma unroll
      for (int i = 0; i < 32; i += 4) store4(c + i, &v[i]);
      break;
    }
    case EPI_ACCUM_F32: {
      float* c = reinterpret_cast<float*>(e.C) + off;
      if (e.beta) {
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          float o[4];
          load4(c + i, o);
          o[0] += v[i]; o[1] += v[i + 1]; o[2] += v[i + 2]; o[3] += v[i + 3];
          store4(c + i, o);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; i += 4) store4(c + i, &v[i]);
      }
      break;
    }
    case EPI_RELU2: {
      act_t* c = reinterpret_cast<act_t*>(e.C) + off;
      act_t* c2 = reinterpret_cast<act_t*>(e.C2) + off;
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        float rr[4], gg[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) { rr[j] = fmaxf(v[i + j], 0.f); gg[j] = rr[j] * rr[j]; }
        store4(c + i, rr);
        store4(c2 + i, gg);
      }
      break;
    }
    case EPI_DRELU2: {
      act_t* c = reinterpret_cast<act_t*>(e.C) + off;
      const act_t* a = reinterpret_cast<const act_t*>(e.aux) + off;
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        float rr[4], o[4];
        load4(a + i, rr);
#pragma unroll
        for (int j = 0; j < 4; ++j) o[j] = 2.f * rr[j] * v[i + j];
        store4(c + i, o);
      }
      break;
    }
  }
}

template <int BN, typename act_t>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const Params p) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles = p.m_tiles * p.n_tiles * p.splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(&tfull[s], 1); mbar_init(&tempty[s], 128); }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(C::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_phase[C::STAGES];
      bool issued[C::STAGES];
      for (int s = 0; s < C::STAGES; ++s) issued[s] = false;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        const int split = t % p.splits;
        const int mn = t / p.splits;
        const int m0 = (mn / p.n_tiles) * BM, n0 = (mn % p.n_tiles) * BN;
        const int kb0 = split * p.kb_per_split;
        const int kb1 = min(kb0 + p.kb_per_split, p.kb_total);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err)) { ok = false; break; }
          mbar_expect_tx(&full[stage], C::STAGE_BYTES);
          load_operand(sA + stage * C::A_BYTES, &tmA, &full[stage], p.a_kmajor, BM, m0, kb);
          load_operand(sB + stage * C::B_BYTES, &tmB, &full[stage], p.b_kmajor, BN, n0, kb);
          issued[stage] = true;
          issued_phase[stage] = phase;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // make sure no copy is still landing in this CTA's shared memory
      for (int s = 0; s < C::STAGES; ++s) {
        if (!issued[s]) continue;
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&full[s], issued_phase[s])) {
          if (globaltimer_ns() - t0 > GPT_WAIT_LIMIT_NS) { set_error(p.err, GPT_EBIT_TIMEOUT); break; }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(!p.a_kmajor) << 15) |
                             ((uint32_t)(!p.b_kmajor) << 16) | ((uint32_t)(BN >> 3) << 17) |
                             ((uint32_t)(BM >> 4) << 24);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        const int split = t % p.splits;
        const int kb0 = split * p.kb_per_split;
        const int kb1 = min(kb0 + p.kb_per_split, p.kb_total);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b_base = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            tc_mma(d_tmem, operand_desc(a_base, p.a_kmajor, k), operand_desc(b_base, p.b_kmajor, k),
                   idesc, (kb > kb0 || k > 0) ? 1u : 0u);
          }
          tc_commit(&empty[stage]);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        tc_commit(&tfull[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
      const int split = t % p.splits;
      const int mn = t / p.splits;
      const long long m0 = (long long)(mn / p.n_tiles) * BM;
      const int n0 = (mn % p.n_tiles) * BN;
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag, p.err)) break;
      tc_fence_after();
      const long long m = m0 + q * 32 + lane;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN + c * 32, r);
        if (n0 + c * 32 < p.N) epilogue_row32<act_t>(p, m, n0 + c * 32, r, split);
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(C::TMEM_COLS));
  }
}

}  // namespace tc
