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
//   warps 2..9  the epilogue: tcgen05.ld of the finished accumulator (one
//               TMEM lane = one output row per thread; two warps share each
//               32-lane quarter, one per half of the tile's columns), apply
//               the epilogue, stage 128-byte rows in shared memory and write
//               them with asynchronous TMA stores (TMA reduce-add for fp32
//               accumulation), then release the accumulator.
// The two accumulators let the epilogue of tile i overlap the MMAs of tile
// i + 1.
//
// CG = 2 runs the same roles on a cluster of two CTAs (a pair of SMs) that
// share 256 x BN output tiles through tcgen05.mma.cta_group::2: each CTA loads
// its own 128 rows of A and half of the tile's B rows (BN / 2), the MMA
// thread of the even CTA issues M = 256 products that read both CTAs' shared
// memory and write each CTA's 128 accumulator rows into its own TMEM, and
// each CTA drains its own rows.  Per SM the tensor core then reads 8 KB of
// operands per 128-cycle MMA instead of 12 KB, and TMA writes 32 KB instead
// of 48 KB per k-block, which is what bounds the one-SM form: a k-block's
// operand traffic through shared memory (TMA writes plus MMA reads) is about
// 1.5x what shared memory moves in the k-block's MMA time.  The loads of both
// CTAs complete on the even CTA's stage barrier; its MMA commits release the
// stage and publish the accumulator in both CTAs (tcgen05.commit multicast);
// the odd CTA's epilogue warps release the accumulator on the even CTA's
// barrier.  No TMA load is multicast.
//
// F8 = 1 takes e4m3 operands (tcgen05.mma kind::f8f6f4, K = 32 per
// instruction): a k-block is still one 128-byte swizzle row per operand row,
// now 128 elements, so the stage layout, the descriptors and the epilogues are
// those of the bf16 form; the epilogue multiplies by the two operands' scales
// (device scalars).  K-major operands only.  K-major and MN-major operands are both read straight from their
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
constexpr int EPI_WARPS = 8;
constexpr int NUM_THREADS = 64 + 32 * EPI_WARPS;

// Epilogue kind of one kernel instantiation (compile time, so each kernel
// carries only its own epilogue code).
enum KMode {
  K_STORE = 0,    // bf16 output
  K_STORE_F32,    // fp32 output (also accumulate with beta = 0)
  K_REDUCE_F32,   // fp32 C += acc by TMA reduce-add (accumulate with beta = 1)
  K_PARTIAL,      // split-K fp32 partials [splits, M, N]
  K_RELU2,        // bf16 relu(acc)^2
  K_DRELU2,       // bf16 2 sqrt(aux) acc
  K_LOGITS,       // bf16 exp(z - tile max), z = softcap(acc), + per-tile row statistics
  K_QKV,          // bf16 q|k|v with RoPE + QK-norm (+ value-table row) per 128-wide head
  K_AXPBY,        // bf16 acc + aux_scale * aux (aux streamed like the ReLU^2 backward's)
};

// The ReLU^2-backward epilogue streams activations through a ring of its
// own, which costs a pipeline stage; every other epilogue uses the light
// configuration.  Host and kernel both take the configuration from here.
template <int KM> struct KmHeavy {
  static constexpr int value = (KM == K_DRELU2 || KM == K_AXPBY) ? 1 : 0;
};

// HEAVY = 1 (ReLU^2 backward, the Newton-Schulz combinations) trades one
// pipeline stage for each epilogue warp's two input blocks (its whole half
// tile of the second input), which also serve as its
// output staging; the other epilogues stage through one block per warp.
// BN = 128, 192 or 256 (192 only with fp32 outputs: 96 columns per epilogue
// warp = three 32-column fp32 blocks); the ring takes what shared memory has
// left after the epilogue's buffers, at most 6 stages.
template <int BN, int HEAVY, int CG = 1> struct Cfg {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_ROWS = BN / CG;               // B rows this CTA loads per k-block
  static constexpr int B_BYTES = B_ROWS * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN <= 256 ? 256 : 512;  // two accumulators, power of two
  static constexpr int NSTG = HEAVY ? 0 : 1;           // staging blocks per epilogue warp
  static constexpr int NAUX = 2;                       // activation blocks per epilogue warp (ReLU^2 bwd)
  static constexpr int AUX = HEAVY ? NAUX * 32 * 128 : 0;  // activation bytes per epilogue warp
  static constexpr int FIXED = EPI_WARPS * (NSTG * 32 * 128 + AUX) + 1024 /*align*/ + 512 /*barriers*/ +
                               512 /*RoPE turns*/;
  static constexpr int STAGES = (232448 - FIXED) / STAGE_BYTES > 6 ? 6 : (232448 - FIXED) / STAGE_BYTES;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + FIXED;
};

struct Params {
  int M, N, K;   // m_tiles counts tiles of CG * BM rows
  int batch;     // > 1: `batch` independent products of this shape, the third
                 // coordinate of 3-D tensor maps (store epilogues only, no split-K)
  int a_kmajor, b_kmajor;
  int m_tiles, n_tiles, splits, kb_per_split, kb_total;
  int group_m;  // tile order: groups of group_m m-blocks, m fastest inside a group
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
// The same wait made warp-uniform: every lane waits, and the warp proceeds only
// if all lanes succeeded.  Used wherever the warp next executes .sync.aligned
// tcgen05 instructions, which must never be reached by a partial warp.
// A barrier that is already complete costs one try_wait and one vote (about
// 40 cycles measured on B200, against about 120 through the bounded loop's
// divergent early return).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned* err) {
  if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
  const bool ok = mbar_wait(bar, parity, abort_flag, err);
  return __all_sync(0xffffffffu, ok);
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
__device__ __forceinline__ void tc_mma_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                            int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// ---- CTA-pair (cta_group::2) forms
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the variable at shared::cta address `addr` in CTA `rank`
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// TMA load into this CTA's shared memory whose completion is counted on the
// barrier at shared::cluster address `bar` (this CTA's or the pair peer's)
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* map, uint32_t bar, int x, int y,
                                                 int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrive on the barrier at this offset in both CTAs of the pair once the
// issuing thread's earlier tcgen05 operations are complete
__device__ __forceinline__ void tc_mma_pair_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"((uint16_t)3)
      : "memory");
}
// ---- warp-issued forms: the whole (converged) warp executes the call and
// elect.sync picks the one lane that issues.  Measured on B200: issuing from a
// converged warp keeps the operand descriptors on the warp-uniform path, which
// takes about a fifth off the issue time of short products, and a commit
// between products then costs nothing (from a lone lane each commit stalled
// the issuing thread for about 100 cycles).  The election depends only on the
// active mask, so a full warp elects the same lane at every call, and that
// lane's commits track the products it issued.
#define TC_ELECT_ISSUE(instr) \
  "{\n\t.reg .pred p, e;\n\telect.sync _|e, 0xffffffff;\n\tsetp.ne.b32 p, %4, 0;\n\t@e " instr ";\n\t}"
__device__ __forceinline__ void tc_mma_w(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(TC_ELECT_ISSUE("tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p") ::"r"(d_tmem),
               "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
               : "memory");
}
__device__ __forceinline__ void tc_mma_f8_w(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(TC_ELECT_ISSUE("tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p") ::"r"(d_tmem),
               "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
               : "memory");
}
__device__ __forceinline__ void tc_mma_pair_w(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(TC_ELECT_ISSUE("tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p") ::"r"(d_tmem),
               "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
               : "memory");
}
__device__ __forceinline__ void tc_mma_pair_f8_w(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                 uint32_t accumulate) {
  asm volatile(TC_ELECT_ISSUE("tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p") ::"r"(d_tmem),
               "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
               : "memory");
}
// A from tensor memory (the `ts` form), warp-issued
__device__ __forceinline__ void tc_mma_ts_w(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(TC_ELECT_ISSUE("tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p") ::"r"(d_tmem),
               "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
               : "memory");
}
#undef TC_ELECT_ISSUE
__device__ __forceinline__ void tc_commit_w(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tc_commit_pair_w(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;\n\t}" ::"r"(
          smem_u32(bar)),
      "h"((uint16_t)3)
      : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
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
// k-block starting at element kx; B3: product z of a batch (3-D tensor map).
template <bool B3>
__device__ __forceinline__ void load_operand(uint8_t* dst, const CUtensorMap* map, uint64_t* bar,
                                             int kmajor, int rows, int r0, int kx, int z) {
  if (kmajor) {
    if constexpr (B3) tma_load_3d(dst, map, bar, kx, r0, z);
    else tma_load_2d(dst, map, bar, kx, r0);
  } else {
    for (int j = 0; j < rows / 64; ++j) {
      if constexpr (B3) tma_load_3d(dst + j * 64 * BK * 2, map, bar, r0 + 64 * j, kx, z);
      else tma_load_2d(dst + j * 64 * BK * 2, map, bar, r0 + 64 * j, kx);
    }
  }
}
// the same, counted on the pair's stage barrier at shared::cluster address `bar`
template <bool B3>
__device__ __forceinline__ void load_operand_pair(uint8_t* dst, const CUtensorMap* map, uint32_t bar,
                                                  int kmajor, int rows, int r0, int kx, int z) {
  if (kmajor) {
    if constexpr (B3) tma_load_3d_pair(dst, map, bar, kx, r0, z);
    else tma_load_2d_pair(dst, map, bar, kx, r0);
  } else {
    for (int j = 0; j < rows / 64; ++j) {
      if constexpr (B3) tma_load_3d_pair(dst + j * 64 * BK * 2, map, bar, r0 + 64 * j, kx, z);
      else tma_load_2d_pair(dst + j * 64 * BK * 2, map, bar, r0 + 64 * j, kx);
    }
  }
}

// Descriptor of UMMA k-step `k` (16 elements of K) inside an operand tile.
__device__ __forceinline__ uint64_t operand_desc(uint32_t base, int kmajor, int k) {
  if (kmajor) return smem_desc(base + k * 32, 16, 1024);
  return smem_desc(base + k * 16 * 128, 64 * BK * 2, 1024);
}

// ------------------------------------------------------------------ epilogue
// Each epilogue warp owns 32 output rows (its TMEM lane quarter) and walks the
// tile in column blocks of 32 fp32 (fp32 outputs) or 64 bf16 (bf16 outputs),
// i.e. 128-byte rows.  TMEM -> registers (one row per lane; row-local work such
// as the cross-entropy statistics happens here) -> a 32 x 128-byte staging
// block in shared memory written in the TMA 128-byte swizzle (conflict-free)
// -> one asynchronous TMA store, or a TMA reduce-add when the product is
// accumulated into an fp32 buffer (residual stream, weight gradients).  The
// ReLU^2 backward's second input is brought in by TMA one block ahead.
constexpr int STG_BYTES = 32 * 128;  // per epilogue warp
constexpr int AUX_BYTES = 32 * 128;

__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, uint32_t (&r)[32]) {
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
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
               : "memory");
}
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, const void* src, int x, int y) {
  asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// z = cap * tanh(acc / cap) (nanochat's logit softcap) for a block of
// values, with tanh(x) = 1 - 2 / (exp(2x) + 1).  Called only under a
// warp-uniform `cap > 0` test around the whole block, so the default
// (no softcap) path carries none of this arithmetic.
template <int NVAL>
__device__ __forceinline__ void softcap_block(float (&v)[NVAL], float cap) {
  const float two_over_cap = 2.f / cap;
#pragma unroll
  for (int i = 0; i < NVAL; ++i) v[i] = cap * (1.f - __fdividef(2.f, __expf(v[i] * two_over_cap) + 1.f));
}

// Output tile (m-block, n-block) of linear tile index mn.  Tiles come in
// groups of group_m m-blocks; inside a group the m-block varies fastest, so
// the CTAs running at one time cover about group_m x (SMs / group_m) tiles
// and read each A row-block and B column-block from HBM about once per group
// (the rest of the reuse comes from L2).
__device__ __forceinline__ void tile_coords(int mn, const Params& p, int& mt, int& nt) {
  const int per_group = p.group_m * p.n_tiles;
  const int g = mn / per_group;
  const int first_m = g * p.group_m;
  const int gsize = min(p.group_m, p.m_tiles - first_m);
  const int r = mn - g * per_group;
  mt = first_m + r % gsize;
  nt = r / gsize;
}

// byte offset of 16-byte chunk j of row r in a 128-byte-swizzled block
// two fp32 lanes per instruction (sm_100 packed f32x2 arithmetic):
// (y0, y1) = (x0, x1) * c + d
__device__ __forceinline__ void fma2(float& y0, float& y1, float x0, float x1, float c, float d) {
  asm("{\n\t.reg .b64 a, b, e, r;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %4};\n\tmov.b64 e, {%5, %5};\n\t"
      "fma.rn.f32x2 r, a, b, e;\n\tmov.b64 {%0, %1}, r;\n\t}"
      : "=f"(y0), "=f"(y1)
      : "f"(x0), "f"(x1), "f"(c), "f"(d));
}
// (y0, y1) += (x0, x1)
__device__ __forceinline__ void add2(float& y0, float& y1, float x0, float x1) {
  asm("{\n\t.reg .b64 a, b;\n\tmov.b64 a, {%0, %1};\n\tmov.b64 b, {%2, %3};\n\t"
      "add.rn.f32x2 a, a, b;\n\tmov.b64 {%0, %1}, a;\n\t}"
      : "+f"(y0), "+f"(y1)
      : "f"(x0), "f"(x1));
}
// (y0, y1) = (x0, x1) * c + (d0, d1)
__device__ __forceinline__ void fma2v(float& y0, float& y1, float x0, float x1, float c, float d0, float d1) {
  asm("{\n\t.reg .b64 a, b, e, r;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %4};\n\tmov.b64 e, {%5, %6};\n\t"
      "fma.rn.f32x2 r, a, b, e;\n\tmov.b64 {%0, %1}, r;\n\t}"
      : "=f"(y0), "=f"(y1)
      : "f"(x0), "f"(x1), "f"(c), "f"(d0), "f"(d1));
}
// (y0, y1) = (p0, p1) * ((x0, x1) - (d0, d1))
__device__ __forceinline__ void mulsub2(float& y0, float& y1, float p0, float p1, float x0, float x1, float d0,
                                        float d1) {
  asm("{\n\t.reg .b64 a, b, q;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\tmov.b64 q, {%6, %7};\n\t"
      "sub.rn.f32x2 a, a, b;\n\tmul.rn.f32x2 a, a, q;\n\tmov.b64 {%0, %1}, a;\n\t}"
      : "=f"(y0), "=f"(y1)
      : "f"(x0), "f"(x1), "f"(d0), "f"(d1), "f"(p0), "f"(p1));
}
__device__ __forceinline__ uint32_t swz128(int r, int j) { return (uint32_t)(r * 128 + ((j ^ (r & 7)) << 4)); }

// cos and sin of the RoPE angle t theta_f from the frequency's turns per
// position u = hi + lo (an fp32 pair): t hi = p + e exactly (e = fma(t, hi,
// -p)), the whole turns k = rint(p) drop out exactly, and the remaining
// fraction of a turn, in [-1/2, 1/2], goes to the special-function unit's
// sin / cos.  Absolute error ~1e-6 for positions below 2^16.
__device__ __forceinline__ void rope_cos_sin(float tf, float2 u, float& c, float& s) {
  const float p = tf * u.x;
  const float e = fmaf(tf, u.x, -p);
  const float k = rintf(p);
  const float fr = (p - k) + fmaf(tf, u.y, e);
  __sincosf(6.28318530717958648f * fr, &s, &c);
}

template <int BN, int KM, typename act_t, int CG, int F8 = 0, bool B3 = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmAux,
                   const Params p) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  using C = Cfg<BN, KmHeavy<KM>::value, CG>;
  static_assert(CG == 1 || CG == 2, "one CTA or a CTA pair per tile");
  constexpr int KE = F8 ? 128 : BK;  // operand elements per 128-byte k-block row
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint8_t* stg_all = smem + C::STAGES * C::STAGE_BYTES;
  uint8_t* aux_all = stg_all + EPI_WARPS * C::NSTG * STG_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(aux_all + EPI_WARPS * C::AUX);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* auxbar = tempty + 2;  // NAUX per epilogue warp
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(auxbar + EPI_WARPS * C::NAUX);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float2* sturns = reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(full) + 512);  // [64]
  static_assert((2 * C::STAGES + 4 + EPI_WARPS * C::NAUX) * 8 + 8 <= 512, "barrier area");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if constexpr (KM == K_QKV)
    if (threadIdx.x < 64 && p.epi.rope != nullptr) sturns[threadIdx.x] = p.epi.rope[threadIdx.x];
  const int per_product = p.m_tiles * p.n_tiles * p.splits;
  const int tiles = B3 ? per_product * p.batch : per_product;
  // CTA pair: rank 0 issues the MMAs; tile t goes to pair blockIdx.x / CG
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;
  const int unit = blockIdx.x / CG, n_units = gridDim.x / CG;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    // tempty: one arrival per epilogue warp (of both CTAs of a pair)
    for (int s = 0; s < 2; ++s) { mbar_init(&tfull[s], 1); mbar_init(&tempty[s], CG * EPI_WARPS); }
    for (int s = 0; s < EPI_WARPS * C::NAUX; ++s) mbar_init(&auxbar[s], 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    // a pair allocates together: the same columns in both CTAs' TMEM
    if constexpr (CG == 2) {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_slot)),
                   "r"(C::TMEM_COLS));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    } else {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_slot)),
                   "r"(C::TMEM_COLS));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
  }
  tc_fence_before();
  __syncthreads();
  // the pair's barriers are initialised and its TMEM allocated before either
  // CTA signals the other
  if constexpr (CG == 2) cluster_sync_all();
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
      for (int t = unit; t < tiles && ok; t += n_units) {
        const int z = B3 ? t / per_product : 0;
        const int tt = B3 ? t % per_product : t;
        const int split = tt % p.splits;
        const int mn = tt / p.splits;
        int mt, nt;
        tile_coords(mn, p, mt, nt);
        // this CTA's A rows and B rows of the tile
        const int m0 = (mt * CG + (int)rank) * BM, n0 = nt * BN + (int)rank * C::B_ROWS;
        const int kb0 = split * p.kb_per_split;
        const int kb1 = min(kb0 + p.kb_per_split, p.kb_total);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err)) { ok = false; break; }
          if constexpr (CG == 2) {
            // both CTAs' bytes complete on the even CTA's stage barrier, which
            // that CTA arms for the pair
            const uint32_t bar0 = mapa_shared(smem_u32(&full[stage]), 0);
            if (rank == 0) mbar_expect_tx(&full[stage], CG * C::STAGE_BYTES);
            load_operand_pair<B3>(sA + stage * C::A_BYTES, &tmA, bar0, p.a_kmajor, BM, m0, kb * KE, z);
            load_operand_pair<B3>(sB + stage * C::B_BYTES, &tmB, bar0, p.b_kmajor, C::B_ROWS, n0, kb * KE, z);
          } else {
            mbar_expect_tx(&full[stage], C::STAGE_BYTES);
            load_operand<B3>(sA + stage * C::A_BYTES, &tmA, &full[stage], p.a_kmajor, BM, m0, kb * KE, z);
            load_operand<B3>(sB + stage * C::B_BYTES, &tmB, &full[stage], p.b_kmajor, BN, n0, kb * KE, z);
          }
          issued[stage] = true;
          issued_phase[stage] = phase;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // make sure no copy is still landing in this CTA's shared memory (the
      // odd CTA of a pair cannot wait on the even CTA's barriers: every one
      // of its copies is consumed by an MMA before the pair finishes, and an
      // aborted pair waits out its copies before tearing down)
      for (int s = 0; s < C::STAGES; ++s) {
        if (!issued[s] || rank != 0) continue;
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&full[s], issued_phase[s])) {
          if (globaltimer_ns() - t0 > GPT_WAIT_LIMIT_NS) { set_error(p.err, GPT_EBIT_TIMEOUT); break; }
        }
      }
    }
  } else if (warp == 1) {
    if (rank == 0) {
      // ------------------------------------------------------------ MMA issuer
      // the whole warp runs the loop; one elected lane issues (tc_*_w)
      // D fp32; A, B bf16 (kind::f16) or e4m3 (kind::f8f6f4: format code 0)
      const uint32_t idesc = (1u << 4) | (F8 ? 0u : (1u << 7) | (1u << 10)) | ((uint32_t)(!p.a_kmajor) << 15) |
                             ((uint32_t)(!p.b_kmajor) << 16) | ((uint32_t)(BN >> 3) << 17) |
                             ((uint32_t)((CG * BM) >> 4) << 24);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = unit; t < tiles && ok; t += n_units) {
        const int split = (B3 ? t % per_product : t) % p.splits;
        const int kb0 = split * p.kb_per_split;
        const int kb1 = min(kb0 + p.kb_per_split, p.kb_total);
        if (!warp_wait(&tempty[acc], acc_phase ^ 1, abort_flag, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!warp_wait(&full[stage], phase, abort_flag, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b_base = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // 32 bytes of K per instruction: 16 bf16 or 32 e4m3
            const uint64_t ad = operand_desc(a_base, p.a_kmajor, k), bd = operand_desc(b_base, p.b_kmajor, k);
            const uint32_t acc_in = (kb > kb0 || k > 0) ? 1u : 0u;
            if constexpr (CG == 2 && F8) tc_mma_pair_f8_w(d_tmem, ad, bd, idesc, acc_in);
            else if constexpr (CG == 2) tc_mma_pair_w(d_tmem, ad, bd, idesc, acc_in);
            else if constexpr (F8) tc_mma_f8_w(d_tmem, ad, bd, idesc, acc_in);
            else tc_mma_w(d_tmem, ad, bd, idesc, acc_in);
          }
          if constexpr (CG == 2) tc_commit_pair_w(&empty[stage]);
          else tc_commit_w(&empty[stage]);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        if constexpr (CG == 2) tc_commit_pair_w(&tfull[acc]);
        else tc_commit_w(&tfull[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    constexpr int HALF = BN / 2;         // columns per epilogue warp
    const int ew = warp - 2;             // 0 .. EPI_WARPS-1
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    const int ccol = (ew >> 2) * HALF;   // first tile column of this warp's half
    uint8_t* stg_base = stg_all + ew * C::NSTG * STG_BYTES;
    uint8_t* auxs = aux_all + ew * C::AUX;
    uint64_t* abar = &auxbar[ew * C::NAUX];  // abar[b] guards activation block b
    uint32_t aux_phase = 0;                  // bit b: parity of the next wait on abar[b]
    uint32_t aux_pending = 0;                // bit b: a load into block b is in flight
    const GemmEpilogue& e = p.epi;
    // acc scale: alpha times the operands' device scales (the FP8 path), if any
    float ealpha = e.alpha;
    if constexpr (F8) ealpha *= (e.scale_a ? *e.scale_a : 1.f) * (e.scale_b ? *e.scale_b : 1.f);
    constexpr bool f32out = KM == K_STORE_F32 || KM == K_REDUCE_F32 || KM == K_PARTIAL;
    constexpr bool has_aux = KM == K_DRELU2 || KM == K_AXPBY;
    constexpr int CW = f32out ? 32 : 64;  // columns per 128-byte staging row
    static_assert(!has_aux || HALF / CW <= C::NAUX, "one activation block per column block");
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    // the accumulator-empty barrier lives in the even CTA of a pair
    const uint32_t tempty0 = CG == 2 ? mapa_shared(smem_u32(&tempty[0]), 0) : 0u;
    for (int t = unit; t < tiles && ok; t += n_units) {
      const int z = B3 ? t / per_product : 0;
      const int tt = B3 ? t % per_product : t;
      const int split = tt % p.splits;
      const int mn = tt / p.splits;
      int mt, nt;
      tile_coords(mn, p, mt, nt);
      const int m0 = (mt * CG + (int)rank) * BM;  // this CTA's 128 accumulator rows
      const int n0 = nt * BN + ccol;  // first output column of this warp
      const int mrow0 = m0 + q * 32;
      const long long m = (long long)mrow0 + lane;
      const int nblk = (p.N - n0 <= 0) ? 0 : min(HALF / CW, (p.N - n0 + CW - 1) / CW);
      if (has_aux) {
        // this half tile's ReLU^2 activations, ahead of the accumulator; the
        // blocks double as output staging, so the previous tile's stores
        // must have read them first
        if (lane == 0) bulk_wait_read0();
        __syncwarp();
        for (int b = 0; b < nblk; ++b) {
          if (lane == 0) {
            mbar_expect_tx(&abar[b], AUX_BYTES);
            if constexpr (B3) tma_load_3d(auxs + b * AUX_BYTES, &tmAux, &abar[b], n0 + b * 64, mrow0, z);
            else tma_load_2d(auxs + b * AUX_BYTES, &tmAux, &abar[b], n0 + b * 64, mrow0);
          }
          aux_pending |= 1u << b;
        }
      }
      if (!warp_wait(&tfull[acc], acc_phase, abort_flag, p.err)) { ok = false; break; }
      tc_fence_after();
      float rmax = -INFINITY, rsum = 0.f;
      const uint32_t trow = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN + ccol;
      int ytgt = -1;
      // The store, ReLU^2 and fp32 epilogues take the warp's whole half tile
      // from TMEM into registers at once and hand the accumulator back to the
      // MMA warp before any arithmetic or store, so the MMA of the tile after
      // next does not wait for this tile's stores (measured faster on B200).
      // The logits and ReLU^2-backward epilogues hold fewer registers: they
      // read a block at a time and release the accumulator at the tile's end
      // (holding the whole half tile spilled and measured slower there).
      constexpr bool PRE = KM != K_QKV && KM != K_LOGITS && KM != K_DRELU2 && KM != K_AXPBY;
      float accr[PRE ? HALF : 1];
      if constexpr (PRE) {
        uint32_t r[HALF / 32][32];
#pragma unroll
        for (int q2 = 0; q2 < HALF / 32; ++q2) tmem_ld32_nowait(trow + q2 * 32, r[q2]);
        tmem_wait_ld();
#pragma unroll
        for (int q2 = 0; q2 < HALF / 32; ++q2)
#pragma unroll
          for (int i = 0; i < 32; ++i) accr[q2 * 32 + i] = __uint_as_float(r[q2][i]) * ealpha;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (CG == 2) mbar_arrive_cluster(tempty0 + acc * 8);
          else mbar_arrive(&tempty[acc]);
        }
      }
      if constexpr (KM == K_LOGITS) {
        // first pass over the accumulator: the half tile's row maximum, so
        // that the stored numerators exp(z - max) lie in (0, 1]
        ytgt = (e.targets != nullptr && m < p.M) ? e.targets[m] : -1;
#pragma unroll 1
        for (int c = 0; c < HALF / 32; ++c) {
          const int nc = n0 + c * 32;
          if (nc >= p.N) break;  // warp-uniform
          uint32_t r[32];
          tmem_ld32_nowait(trow + c * 32, r);
          tmem_wait_ld();
          const int nv = min(32, p.N - nc);
          float z[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) z[i] = __uint_as_float(r[i]) * ealpha;
          if (e.softcap > 0.f) softcap_block<32>(z, e.softcap);
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i < nv) rmax = fmaxf(rmax, z[i]);
        }
      }
      if constexpr (KM == K_QKV && HALF == 128) {
        // one 128-wide head (this warp's half tile); this lane owns row m of it
        // (the host launches this epilogue with 256-column tiles only)
        const bool row_ok = m < p.M;
        const int tpos = row_ok ? (int)(m % e.T) : 0;
        if (n0 < p.N) {  // warp-uniform
          const int head = n0 / 128, sec = head / e.H, hi = head % e.H;
          float v[128];
          {
            uint32_t r0[32], r1[32], r2[32], r3[32];
            tmem_ld32_nowait(trow, r0);
            tmem_ld32_nowait(trow + 32, r1);
            tmem_ld32_nowait(trow + 64, r2);
            tmem_ld32_nowait(trow + 96, r3);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              v[i] = __uint_as_float(r0[i]);
              v[32 + i] = __uint_as_float(r1[i]);
              v[64 + i] = __uint_as_float(r2[i]);
              v[96 + i] = __uint_as_float(r3[i]);
            }
          }
          if (sec < 2) {
            // RoPE ("$1000 tier nanochat run", apply_rotary_emb): y1 = x1 cos + x2 sin,
            // y2 = -x1 sin + x2 cos over the two halves of the head, then QK-norm;
            // cos / sin of frequency i at this row's position from its turns table
            const float tf = (float)tpos;
            float ss = 0.f;
#pragma unroll
            for (int i = 0; i < 64; ++i) {
              float wc, ws;
              rope_cos_sin(tf, sturns[i], wc, ws);
              const float x1 = v[i], x2 = v[i + 64];
              v[i] = x1 * wc + x2 * ws;
              v[i + 64] = -x1 * ws + x2 * wc;
              ss += v[i] * v[i] + v[i + 64] * v[i + 64];
            }
            if (e.qk_norm) {
              const float rs = rsqrtf(ss / 128.f + e.eps);
#pragma unroll
              for (int i = 0; i < 128; ++i) v[i] *= rs;
              if (row_ok) (sec == 0 ? e.rstd_q : e.rstd_k)[m * e.H + hi] = rs;
            }
          } else if (e.hv && row_ok) {
            // the value-table row of this position (decoder-rtx posts: table "added to values")
            // row rv[m] of the value table, or (rv null) row m of a per-position bias
            const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const act_t*>(e.hv) +
                                                              (long long)(e.rv ? e.rv[m] : m) * (e.H * 128) +
                                                              hi * 128);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const uint4 raw = src[j];
              const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
              for (int hq = 0; hq < 4; ++hq) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[hq]));
                v[j * 8 + 2 * hq] += f.x;
                v[j * 8 + 2 * hq + 1] += f.y;
              }
            }
          }
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint8_t* stg = stg_base;
            if (lane == 0) bulk_wait_read0();
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float* x = &v[half * 64 + 8 * j];
              uint4 o;
              __nv_bfloat162 b0 = __floats2bfloat162_rn(x[0], x[1]), b1 = __floats2bfloat162_rn(x[2], x[3]);
              __nv_bfloat162 b2 = __floats2bfloat162_rn(x[4], x[5]), b3 = __floats2bfloat162_rn(x[6], x[7]);
              o.x = *reinterpret_cast<uint32_t*>(&b0); o.y = *reinterpret_cast<uint32_t*>(&b1);
              o.z = *reinterpret_cast<uint32_t*>(&b2); o.w = *reinterpret_cast<uint32_t*>(&b3);
              *reinterpret_cast<uint4*>(stg + swz128(lane, j)) = o;
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmC, stg, n0 + half * 64, mrow0);
              bulk_commit();
            }
          }
        }
      }
      // one output block: epilogue arithmetic on its values v, staging, TMA copy
      auto out_block = [&](int c, float (&v)[64]) -> bool {
        const int nc = n0 + c * CW;
        uint8_t* stg = stg_base;
        if constexpr (KM == K_LOGITS) {
          const int nv = min(64, p.N - nc);
          const int yo = ytgt - nc;  // target column within this block, if here
          if (yo >= 0 && yo < 64) {  // rare: this row's target logit
            float zt = 0.f;
#pragma unroll
            for (int i = 0; i < 64; ++i) zt = (i == yo) ? v[i] : zt;
            e.ztgt[m] = zt;
          }
          // numerators exp(z - max) = 2^(z log2 e - max log2 e), the arguments
          // and the row sum (8 independent partial sums) two lanes at a time
          constexpr float L2E = 1.4426950408889634f;
          const float nb = -rmax * L2E;
          float ps[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          if (nv == 64) {  // warp-uniform: all but the vocabulary's last block
#pragma unroll
            for (int i = 0; i < 64; i += 2) {
              float x0, x1;
              fma2(x0, x1, v[i], v[i + 1], L2E, nb);
              float p0, p1;
              asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(p0) : "f"(x0));
              asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(p1) : "f"(x1));
              add2(ps[(i >> 1) & 7], ps[((i >> 1) + 4) & 7], p0, p1);
              v[i] = p0;
              v[i + 1] = p1;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 64; ++i) {
              const float pr = (i < nv) ? __expf(v[i] - rmax) : 0.f;
              ps[i & 7] += pr;
              v[i] = pr;
            }
          }
          rsum += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
        } else if constexpr (KM == K_RELU2) {
#pragma unroll
          for (int i = 0; i < 64; ++i) { const float r = fmaxf(v[i], 0.f); v[i] = r * r; }
        } else if constexpr (KM == K_DRELU2) {
          if (!warp_wait(&abar[c], (aux_phase >> c) & 1u, abort_flag, p.err)) return false;
          aux_phase ^= 1u << c;
          aux_pending &= ~(1u << c);
          stg = auxs + c * AUX_BYTES;  // each lane rewrites only its own row below
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint4 raw = *reinterpret_cast<const uint4*>(stg + swz128(lane, j));
            const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              // d relu(a)^2 / da = 2 relu(a) = 2 g rsqrt(g) for g = relu(a)^2 > 0
              const float2 gg = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[h]));
              v[j * 8 + 2 * h] *= gg.x > 0.f ? 2.f * gg.x * rsqrtf(gg.x) : 0.f;
              v[j * 8 + 2 * h + 1] *= gg.y > 0.f ? 2.f * gg.y * rsqrtf(gg.y) : 0.f;
            }
          }
        } else if constexpr (KM == K_AXPBY) {
          if (!warp_wait(&abar[c], (aux_phase >> c) & 1u, abort_flag, p.err)) return false;
          aux_phase ^= 1u << c;
          aux_pending &= ~(1u << c);
          stg = auxs + c * AUX_BYTES;  // each lane rewrites only its own row below
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint4 raw = *reinterpret_cast<const uint4*>(stg + swz128(lane, j));
            const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const float2 gg = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[h]));
              v[j * 8 + 2 * h] = fmaf(e.aux_scale, gg.x, v[j * 8 + 2 * h]);
              v[j * 8 + 2 * h + 1] = fmaf(e.aux_scale, gg.y, v[j * 8 + 2 * h + 1]);
            }
          }
        }
        if constexpr (!has_aux) {
          // the TMA store that last used the staging block must have read it
          if (lane == 0) bulk_wait_read0();
          __syncwarp();
        }
        if constexpr (f32out) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<float4*>(stg + swz128(lane, j)) =
                make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            uint4 o;
            __nv_bfloat162 b0 = __floats2bfloat162_rn(v[8 * j], v[8 * j + 1]);
            __nv_bfloat162 b1 = __floats2bfloat162_rn(v[8 * j + 2], v[8 * j + 3]);
            __nv_bfloat162 b2 = __floats2bfloat162_rn(v[8 * j + 4], v[8 * j + 5]);
            __nv_bfloat162 b3 = __floats2bfloat162_rn(v[8 * j + 6], v[8 * j + 7]);
            o.x = *reinterpret_cast<uint32_t*>(&b0);
            o.y = *reinterpret_cast<uint32_t*>(&b1);
            o.z = *reinterpret_cast<uint32_t*>(&b2);
            o.w = *reinterpret_cast<uint32_t*>(&b3);
            *reinterpret_cast<uint4*>(stg + swz128(lane, j)) = o;
          }
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          if constexpr (KM == K_PARTIAL) tma_store_3d(&tmC, stg, nc, mrow0, split);
          else if constexpr (KM == K_REDUCE_F32) tma_reduce_add_2d(&tmC, stg, nc, mrow0);
          else if constexpr (B3) tma_store_3d(&tmC, stg, nc, mrow0, z);
          else tma_store_2d(&tmC, stg, nc, mrow0);
          bulk_commit();
        }
        return true;
      };
      if constexpr (PRE) {
#pragma unroll
        for (int c = 0; c < HALF / CW; ++c) {
          if (c >= nblk) break;  // warp-uniform
          float v[64];
#pragma unroll
          for (int i = 0; i < CW; ++i) v[i] = accr[c * CW + i];
          if (!out_block(c, v)) { ok = false; break; }
        }
      } else if constexpr (KM != K_QKV) {
#pragma unroll 1
        for (int c = 0; c < nblk; ++c) {
          float v[64];
          {
            uint32_t r0[32], r1[32];
            tmem_ld32_nowait(trow + c * CW, r0);
            if (CW == 64) tmem_ld32_nowait(trow + c * CW + 32, r1);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r0[i]) * ealpha;
            if (CW == 64) {
#pragma unroll
              for (int i = 0; i < 32; ++i) v[32 + i] = __uint_as_float(r1[i]) * ealpha;
            }
          }
          if (KM == K_LOGITS && e.softcap > 0.f) softcap_block<64>(v, e.softcap);
          if (!out_block(c, v)) { ok = false; break; }
        }
      }
      if (!ok) break;
      // per (row, half tile) statistics of the logits
      if (KM == K_LOGITS && nblk > 0 && m < p.M)
        e.stats[m * ((p.N + HALF - 1) / HALF) + nt * 2 + (ew >> 2)] = make_float2(rmax, rsum);
      if constexpr (!PRE) {  // these epilogues read TMEM up to their last block
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (CG == 2) mbar_arrive_cluster(tempty0 + acc * 8);
          else mbar_arrive(&tempty[acc]);
        }
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
    if (lane == 0) bulk_wait0();  // all of this warp's stores are complete
    if (has_aux && lane == 0) {
      // an aborted tile may leave activation loads in flight: let them land
      for (int b = 0; b < C::NAUX; ++b) {
        if (!((aux_pending >> b) & 1u)) continue;
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&abar[b], (aux_phase >> b) & 1u)) {
          if (globaltimer_ns() - t0 > GPT_WAIT_LIMIT_NS) break;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  // an aborted CTA (or pair) may still have copies landing: let them finish (bounded)
  if (*abort_flag) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 1000000ull) {}
  }
  if constexpr (CG == 2) {
    // neither CTA frees TMEM or leaves while its peer may still read its
    // shared memory, write its TMEM or arrive on its barriers
    cluster_sync_all();
  }
  if (warp == 1) {
    tc_fence_after();
    if constexpr (CG == 2)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::TMEM_COLS));
    else
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::TMEM_COLS));
  }
}

}  // namespace tc
