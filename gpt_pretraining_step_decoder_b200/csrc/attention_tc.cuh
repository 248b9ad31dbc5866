// attention_tc.cuh -- causal flash attention forward on the 5th-generation
// tensor cores (tcgen05 + TMEM + TMA), bf16 in, fp32 accumulate, head_dim 128.
//
// Causal softmax attention with scale 1/sqrt(hd) ("$1000 tier nanochat run",
// `F.scaled_dot_product_attention(..., is_causal=True)`): o = softmax(q k^T /
// sqrt(hd) + causal) v, and the row log-sum-exp for the backward pass, kept
// in log2 units (lse2 = lse / ln 2) since both backward kernels use exp2.
//
// Persistent: one CTA per SM walks the (128-query tile, sequence, head)
// items heaviest first (item i of CTA c is c + i * gridDim.x); the K/V rings,
// S buffers and P buffers run on across items, the next item's Q loads as
// soon as the previous item's last S has read Q, and O alternates between two
// TMEM accumulators so an item's epilogue overlaps the next item's MMAs
// (measured on B200: per-CTA set-up and epilogue took about as long as the
// work of a short causal tile).  Roles:
//   warp 0      TMA: Q once, then K_j and V_j (128 keys) into 2-deep rings
//               with separate barriers, so K_{j+2} loads as soon as S_j
//               has read K_j;
//   warp 1      one thread issues S_j = Q K_j^T into TMEM (two S buffers, so
//               S_{j+1} is computed while row j's softmax runs) and
//               O += P_j V_j into a TMEM accumulator;
//   warps 2..5  softmax, one query row per thread: read S_j from TMEM, mask,
//               running max, exp2, row sum, write P_j as bf16 pairs (packed on
//               the integer pipe) over the first half of S_j's own TMEM
//               columns: the PV product takes P as its A operand from TMEM,
//               so shared memory carries only Q, K and V.  S_{j+2} reuses the
//               buffer once PV_j has read it.
//               O is rescaled in TMEM only when a row max grows by more than
//               2^8 (log2 units) over the max in use, so most tiles skip it;
//               the exponentials then stay below 2^8, safe in fp32 and bf16.
// Epilogue: O / l to bf16 o, lse2 = m + log2 l.  Every wait is bounded.
#pragma once
#include "gemm_tc.cuh"

namespace fatc {

constexpr int BQ = 128, BKV = 128, HD = 128;
constexpr int PV_WARP = 6;        // warps 2..5 are the softmax warps
constexpr int THREADS = 224;
constexpr int TILE_BYTES = 128 * 128 * 2;          // one 128 x 128 bf16 tile
constexpr int SMEM_BYTES = TILE_BYTES /*Q*/ + 2 * 2 * TILE_BYTES /*K,V x 2 stages*/ + 1024 /*align*/ +
                           256 /*barriers*/;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float RESCALE_THRESHOLD = 8.f;  // log2 units

// 2^x with the SFU's approximate exponential (PTX ex2.approx.ftz.f32; the
// probabilities it feeds are rounded to bf16 right after)
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// max of three (one sm_100 instruction)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

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
// 16 consecutive 32-bit TMEM columns of the warp's 32 lanes from registers
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
// W (8, 16 or 32) consecutive 32-bit TMEM columns of the warp's 32 lanes
template <int W>
__device__ __forceinline__ void tmem_ldw(uint32_t taddr, uint32_t (&r)[W]) {
  static_assert(W == 8 || W == 16 || W == 32, "tcgen05.ld width");
  if constexpr (W == 32) {
    tc::tmem_ld32_nowait(taddr, r);
  } else if constexpr (W == 16) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
  } else {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
  }
}
template <int W>
__device__ __forceinline__ void tmem_stw(uint32_t taddr, const uint32_t (&r)[W]) {
  static_assert(W == 8 || W == 16, "tcgen05.st width");
  if constexpr (W == 16) {
    tmem_st16(taddr, r);
  } else {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
  }
}

// D (TMEM) += A (TMEM, bf16 packed two per column along K) x B (shared memory)
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// two floats as a bf16 pair (a in the low half), rounded half away from zero in
// magnitude on the integer pipe: add half a bf16 unit in the last place to the
// fp32 bit pattern, keep the upper 16 bits.  Equal to round-to-nearest-even
// except on exact ties; it leaves the transcendental unit to the exponentials.
__device__ __forceinline__ uint32_t pack_bf16x2_int(float a, float b) {
  return __byte_perm(__float_as_uint(a) + 0x8000u, __float_as_uint(b) + 0x8000u, 0x7632);
}
__device__ __forceinline__ uint32_t pack_bf16x2_rn(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}


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

// Work item i of the grid (heaviest first): query tile and (sequence, head).
__device__ __forceinline__ void fwd_item(int i, int n_qt, int BH, int& qt, int& bh) {
  qt = n_qt - 1 - i / BH;
  bh = i % BH;
}

// The forward on tcgen05, persistent: one CTA per SM over the (query tile,
// sequence, head) items heaviest first.  Warp 0: TMA (lane 0 Q and the K
// ring, lane 1 the V ring); warp 1: MMA, issued as a whole warp (one elected
// lane); warps 2..5: softmax, one per TMEM lane quarter (32 query rows x 128
// keys each).
// TMEM: S (fp32, one step at a time) in columns 0..127; the probabilities P
// as bf16 pairs in packed buffer b at 128 + 64 b (the A operand of the PV
// product); O in 256 + 128 ob, alternating per item.  Step g + 1's scores wait
// only until the softmax warps have loaded step g's, and the PV product of
// step g only for step g's probabilities, so the score product of one step
// and the PV product of the previous one keep the tensor pipe busy together.
// The item's O leaves through shared memory: each softmax warp writes its 32
// rows as bf16 (two 64-column blocks in the 128-byte swizzle) and stores them
// with TMA copies (rows past the sequence end clipped by the map's T extent).
constexpr int STG_BYTES_FWD = 4 * 2 * 32 * 128;   // 4 softmax warps x two 32 x 64 bf16 blocks
constexpr int SMEM_BYTES_TC = SMEM_BYTES + STG_BYTES_FWD;

__global__ void __launch_bounds__(THREADS, 1)
    fa_tc_fwd_kernel(const __grid_constant__ CUtensorMap tmQK, const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmO, float* __restrict__ lse_out, int T, int H, int BH,
                     unsigned* err) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  using namespace tc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + TILE_BYTES;            // [2 stages]
  uint8_t* sV = sK + 2 * TILE_BYTES;        // [2 stages]
  uint8_t* sStg = sV + 2 * TILE_BYTES;      // [4 softmax warps][2 blocks]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sStg + STG_BYTES_FWD);
  uint64_t* q_full = bars;                  // 1
  uint64_t* q_empty = bars + 1;             // 1 (the item's last S has read Q)
  uint64_t* k_full = bars + 2;              // 2
  uint64_t* k_empty = bars + 4;             // 2 (S done with K)
  uint64_t* v_full = bars + 6;              // 2
  uint64_t* v_empty = bars + 8;             // 2 (PV done with V)
  uint64_t* s_full = bars + 10;             // 1: S of the step computed
  uint64_t* s_read = bars + 11;             // 1: the softmax warps have loaded it
  uint64_t* p_full = bars + 12;             // 2 (per packed buffer: P written)
  uint64_t* p_free = bars + 14;             // 2 (per packed buffer: PV done with it, O updated)
  uint64_t* o_full = bars + 16;             // 2 (per O buffer: the item's last PV is done)
  uint64_t* o_empty = bars + 18;            // 2 (per O buffer: the softmax warps have read it)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 20);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int a = H * HD;
  const int n_qt = (T + BQ - 1) / BQ;
  const int total = n_qt * BH;
  // this CTA's items: blockIdx.x, blockIdx.x + gridDim.x, ...
  const int first = blockIdx.x, stride = gridDim.x;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(s_read, 4);      // one arrival per softmax warp
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&p_full[s], 4);
      mbar_init(&p_free[s], 1);
      mbar_init(&o_full[s], 1);
      mbar_init(&o_empty[s], 4);
    }
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
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane < 2) {
      // ---------------------------------------------------------------- TMA
      // lane 0 streams Q (once per item, after the previous item's last S
      // has read it) and the K tiles, lane 1 the V tiles; the rings run on
      // across items.
      const bool is_k = lane == 0;
      uint64_t* full = is_k ? k_full : v_full;
      uint64_t* empty = is_k ? k_empty : v_empty;
      bool ok = true;
      int g = 0, nq = 0;  // tiles issued, Q tiles issued
      for (int i = first, k = 0; i < total && ok; i += stride, ++k) {
        int qt, bh;
        fwd_item(i, n_qt, BH, qt, bh);
        const int b = bh / H, h = bh % H, row_base = b * T, n_kv = qt + 1;
        if (is_k) {
          if (k > 0 && !mbar_wait(q_empty, (k - 1) & 1, abort_flag, err)) { ok = false; break; }
          mbar_expect_tx(q_full, TILE_BYTES);
          tma_load_2d(sQ, &tmQK, q_full, h * HD, row_base + qt * BQ);
          tma_load_2d(sQ + TILE_BYTES / 2, &tmQK, q_full, h * HD + 64, row_base + qt * BQ);
          ++nq;
        }
        for (int j = 0; j < n_kv && ok; ++j, ++g) {
          const int s = g & 1;
          if (!mbar_wait(&empty[s], ((g >> 1) & 1) ^ 1, abort_flag, err)) { ok = false; break; }
          mbar_expect_tx(&full[s], TILE_BYTES);
          const int kr = row_base + j * BKV;
          if (is_k) {
            uint8_t* kt = sK + s * TILE_BYTES;
            tma_load_2d(kt, &tmQK, &full[s], a + h * HD, kr);
            tma_load_2d(kt + TILE_BYTES / 2, &tmQK, &full[s], a + h * HD + 64, kr);
          } else {
            // V as an MN-major operand: K-block kb (keys 64kb..), N chunk nc (hd 64nc..)
            uint8_t* v = sV + s * TILE_BYTES;
            for (int kb = 0; kb < 2; ++kb)
              for (int nc = 0; nc < 2; ++nc)
                tma_load_2d(v + kb * (TILE_BYTES / 2) + nc * 8192, &tmV, &full[s], 2 * a + h * HD + 64 * nc,
                            kr + 64 * kb);
          }
        }
      }
      // let every copy land before the CTA can exit
      if (is_k && nq > 0) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(q_full, (nq - 1) & 1)) if (globaltimer_ns() - t0 > GPT_WAIT_LIMIT_NS) break;
      }
      for (int j = (g > 2 ? g - 2 : 0); j < g; ++j) {
        const uint64_t t1 = globaltimer_ns();
        while (!mbar_try_wait(&full[j & 1], (j >> 1) & 1))
          if (globaltimer_ns() - t1 > GPT_WAIT_LIMIT_NS) break;
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA: scores
    // Two MMA warps, each running as a whole warp with one elected lane
    // issuing: this one issues S of every step of this CTA's items in order,
    // warp PV_WARP the PV products, so neither waits behind the other's
    // barriers.  S = Q K^T: A = Q (K-major), B = K (K-major), N = 128
    const uint32_t idesc_s = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(128 >> 3) << 17) |
                             ((uint32_t)(128 >> 4) << 24);
    const uint32_t aQ = smem_u32(sQ);
    bool ok = true;
    int g = 0;
    for (int i = first, k = 0; i < total && ok; i += stride, ++k) {
      int qt, bh;
      fwd_item(i, n_qt, BH, qt, bh);
      const int n_kv = qt + 1;
      if (!warp_wait(q_full, k & 1, abort_flag, err)) { ok = false; break; }
      for (int j = 0; j < n_kv; ++j, ++g) {
        const int s = g & 1;
        if (!warp_wait(&k_full[s], (g >> 1) & 1, abort_flag, err)) { ok = false; break; }
        // S of step g overwrites step g - 1's: the softmax warps have loaded it
        if (g >= 1 && !warp_wait(s_read, (g - 1) & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t aK = smem_u32(sK + s * TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk)
          tc_mma_w(tmem, kmaj_desc(aQ, kk), kmaj_desc(aK, kk), idesc_s, kk > 0 ? 1u : 0u);
        tc_commit_w(s_full);
        tc_commit_w(&k_empty[s]);
      }
      if (ok) tc_commit_w(q_empty);   // the item's last S: Q may be replaced
    }
  } else if (warp == PV_WARP) {
    // ---------------------------------------------------------------- MMA: PV
    // O += P V: A = P (TMEM), B = V (MN-major), N = 128
    const uint32_t idesc_o = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(128 >> 3) << 17) |
                             ((uint32_t)(128 >> 4) << 24);
    bool ok = true;
    int g = 0;
    for (int i = first, k = 0; i < total && ok; i += stride, ++k) {
      int qt, bh;
      fwd_item(i, n_qt, BH, qt, bh);
      const int n_kv = qt + 1, ob = k & 1;
      // the first PV of an item overwrites its O buffer: the softmax warps
      // must have read that buffer for the item two positions back
      if (k >= 2 && !warp_wait(&o_empty[ob], ((k - 2) >> 1) & 1, abort_flag, err)) { ok = false; break; }
      for (int j = 0; j < n_kv; ++j, ++g) {
        const int s = g & 1;
        if (!warp_wait(&p_full[s], (g >> 1) & 1, abort_flag, err)) { ok = false; break; }
        if (!warp_wait(&v_full[s], (g >> 1) & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t aV = smem_u32(sV + s * TILE_BYTES);
        // k-step kk covers keys 16kk..16kk+15: packed P columns 8kk..8kk+7
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk)
          tc_mma_ts_w(tmem + 256 + ob * 128, tmem + 128 + s * 64 + kk * 8, mnmaj_desc(aV, kk), idesc_o,
                      (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit_w(&p_free[s]);
        tc_commit_w(&v_empty[s]);
      }
      if (ok) tc_commit_w(&o_full[ob]);   // the item's last PV: O is complete
    }
  } else if (warp < PV_WARP) {
    // ------------------------------------------------------------------ softmax
    const int q = warp & 3;
    const int r = q * 32 + lane;               // row within the tile
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const float c = rsqrtf((float)HD) * LOG2E;
    uint8_t* stg = sStg + (warp - 2) * (2 * 32 * 128);
    bool ok = true;
    int g = 0;  // global step
    for (int i = first, k = 0; i < total && ok; i += stride, ++k) {
      int qt, bh;
      fwd_item(i, n_qt, BH, qt, bh);
      const int b = bh / H, h = bh % H, n_kv = qt + 1;
      const int qpos = qt * BQ + r;              // query position in the sequence
      const int ob = k & 1;
      float m_use = -INFINITY, l = 0.f;
      for (int j = 0; j < n_kv; ++j, ++g) {
        const int s = g & 1;
        if (!warp_wait(s_full, g & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        float sv[128];
        {
          uint32_t r0[32], r1[32], r2[32], r3[32];
          const uint32_t base = tmem + lane_off;
          tmem_ld32_nowait(base, r0);
          tmem_ld32_nowait(base + 32, r1);
          tmem_ld32_nowait(base + 64, r2);
          tmem_ld32_nowait(base + 96, r3);
          tmem_wait_ld();
#pragma unroll
          for (int ii = 0; ii < 32; ++ii) {
            sv[ii] = __uint_as_float(r0[ii]);
            sv[32 + ii] = __uint_as_float(r1[ii]);
            sv[64 + ii] = __uint_as_float(r2[ii]);
            sv[96 + ii] = __uint_as_float(r3[ii]);
          }
        }
        // loaded: the next step's S may overwrite these columns
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_read);
        const int k0 = j * BKV;
        if (k0 + BKV - 1 > qpos) {  // causal mask on the diagonal tile
#pragma unroll
          for (int ii = 0; ii < 128; ++ii)
            if (k0 + ii > qpos) sv[ii] = -INFINITY;
        }
        // row max of the raw scores (the scale c > 0 commutes with max), as 8
        // independent partial maxima so the reduction is not one long chain
        float pm[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) pm[u] = fmaxf(sv[u], sv[8 + u]);
#pragma unroll
        for (int ii = 16; ii < 128; ii += 16)
#pragma unroll
          for (int u = 0; u < 8; ++u) pm[u] = fmax3(pm[u], sv[ii + u], sv[ii + 8 + u]);
        const float mx = c * fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                                   fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
        if (j == 0) {
          m_use = mx;
        } else if (__any_sync(0xffffffffu, mx > m_use + RESCALE_THRESHOLD)) {
          // grow the max in use: O_{<j} and l scale by 2^(m_old - m_new); the
          // previous PV product must have landed in O first.  The decision is
          // warp-wide (the TMEM accesses below are warp-collective); rows
          // whose max did not grow rescale by exactly 1.
          const float m_new = fmaxf(m_use, mx);
          const float alpha = exp2f(m_use - m_new);
          if (!warp_wait(&p_free[(g - 1) & 1], ((g - 1) >> 1) & 1, abort_flag, err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t obase = tmem + lane_off + 256 + ob * 128;
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t o[32];
            tmem_ld32_nowait(obase + cc * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int ii = 0; ii < 32; ++ii) o[ii] = __float_as_uint(__uint_as_float(o[ii]) * alpha);
            tmem_st32(obase + cc * 32, o);
          }
          tmem_wait_st();
          l *= alpha;
          m_use = m_new;
        }
        // packed buffer s was last read by the PV product of step g - 2
        if (g >= 2 && !warp_wait(&p_free[s], ((g - 2) >> 1) & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        // P = exp2(s - m_use) as bf16 pairs in packed buffer s, the A operand
        // of the PV product (arguments and partial sums two lanes at a time)
        float ps[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // 8 independent partial sums
        const float nm = -m_use;
        const uint32_t pbase = tmem + lane_off + 128 + s * 64;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {  // 4 chunks of 32 keys = 16 packed columns
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float x0, x1;
            fma2(x0, x1, sv[ch * 32 + 2 * e], sv[ch * 32 + 2 * e + 1], c, nm);
            const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
            add2(ps[2 * (e & 3)], ps[2 * (e & 3) + 1], p0, p1);
            w[e] = pack_bf16x2_int(p0, p1);
          }
          tmem_st16(pbase + ch * 16, w);
        }
        l += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[s]);
      }
      if (!ok) break;
      // ------------------------------------------------------------ item epilogue
      if (!warp_wait(&o_full[ob], (k >> 1) & 1, abort_flag, err)) { ok = false; break; }
      tc_fence_after();
      if (qpos < T) lse_out[(long long)bh * T + qpos] = m_use + log2f(l);  // log2 units
      // the previous item's stores have read the staging blocks
      if (lane == 0) bulk_wait_read0();
      __syncwarp();
      const float inv = 1.f / l;
      const uint32_t obase = tmem + lane_off + 256 + ob * 128;
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {   // two 64-column halves, one staging block each
        uint32_t o0[32], o1[32];
        tmem_ld32_nowait(obase + hb * 64, o0);
        tmem_ld32_nowait(obase + hb * 64 + 32, o1);
        tmem_wait_ld();
        if (hb == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&o_empty[ob]);  // this O buffer may be overwritten
        }
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {   // 16-byte chunk jj of the block: columns 8jj..8jj+7
          const uint32_t* src = jj < 4 ? o0 + 8 * jj : o1 + 8 * (jj - 4);
          uint4 wv;
          wv.x = pack_bf16x2_rn(__uint_as_float(src[0]) * inv, __uint_as_float(src[1]) * inv);
          wv.y = pack_bf16x2_rn(__uint_as_float(src[2]) * inv, __uint_as_float(src[3]) * inv);
          wv.z = pack_bf16x2_rn(__uint_as_float(src[4]) * inv, __uint_as_float(src[5]) * inv);
          wv.w = pack_bf16x2_rn(__uint_as_float(src[6]) * inv, __uint_as_float(src[7]) * inv);
          *reinterpret_cast<uint4*>(stg + hb * 4096 + swz128(lane, jj)) = wv;
        }
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0 && qt * BQ + q * 32 < T) {  // rows past T are clipped; a block wholly past it is skipped
        tma_store_3d(&tmO, stg, h * HD, qt * BQ + q * 32, b);
        tma_store_3d(&tmO, stg + 4096, h * HD + 64, qt * BQ + q * 32, b);
        bulk_commit();
      }
    }
    if (lane == 0) bulk_wait0();  // this warp's stores are complete
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

}  // namespace fatc

// ============================================================================
// Backward on tcgen05: with P = exp(s/sqrt(hd) - lse) recomputed from the
// forward's log-sum-exp (kept in log2 units) and D_q = rowsum(dO_q * O_q),
//   dV = P^T dO,  dS = P (dP - D) with dP = dO V^T,  dK = dS^T Q / sqrt(hd),
//   dQ = dS K / sqrt(hd).
// Two kernels so every output element has one writer (no atomics): one CTA
// per 128-key tile computes dK, dV over the query tiles (64 queries) from the
// diagonal on; one CTA per 128-query tile computes dQ over the key tiles (64
// keys) up to the diagonal.
//
// A K-major 128-byte-swizzled tile [rows x 128 hd] (two 64-column halves) is
// also, byte for byte, the MN-major layout of the same matrix read as
// [N = hd, K = rows]: the halves are the two 64-wide N chunks (LBO = half
// size) and 8-row groups are 1 KB apart.  So Q, K and dO are loaded once and
// read through both descriptors.
namespace fatcb {

using fatc::LOG2E;
using fatc::fast_exp2;
using fatc::tmem_wait_st;
using fatc::tmem_st16;
using fatc::tc_mma_ts;
using fatc::pack_bf16x2_int;
using fatc::pack_bf16x2_rn;
using fatc::tmem_ldw;
using fatc::tmem_stw;

// K-major [rows x 128] tile, MMA k-step k over the 128 columns
__device__ __forceinline__ uint64_t kdesc128(uint32_t base, int half_bytes, int k) {
  return tc::smem_desc(base + (k >> 2) * half_bytes + (k & 3) * 32, 16, 1024);
}
// the same [rows x 128] tile read MN-major as [N = 128 (two halves), K = rows]
__device__ __forceinline__ uint64_t mndesc(uint32_t base, int half_bytes, int k) {
  return tc::smem_desc(base + k * 2048, half_bytes, 1024);
}
__device__ __forceinline__ uint32_t idesc(int n, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)b_mn << 16) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(128 >> 4) << 24);
}
// ---------------------------------------------------------------- dK, dV
// 2 + 4 * NCG warps: 0 TMA (lane 0 the Q/dO ring, lane 1 the K/V tiles), 1
// MMA, the rest compute.  Compute warp w owns TMEM lane quarter w % 4 (32 key
// rows) and column group (w - 2) / 4 of the 64 query columns, so NCG warps
// per scheduler share the elementwise work.
// Persistent: one CTA per SM over the (key tile, sequence, head) items,
// heaviest first.  smem: two K/V buffers [128 x 128] x 2 (64 KB each, item k
// in buffer k & 1, so the next item's keys load while this item runs) and
// the Q_i, dO_i [64 x 128] ring (16 KB each, DKDV_QS stages).  P^T and dS^T
// never touch shared memory: each compute warp writes them as bf16 over the
// fp32 S^T / dP^T columns it has just read (its own lanes and columns), and
// the dV / dK products take them as their A operand straight from TMEM.  The
// S^T / dP^T buffers alternate, so step i+1's S^T / dP^T products run while
// step i's elementwise work does.  lse and D come straight from global
// memory.
// The MMA warp issues as a whole warp (one elected lane), and the dV and dK
// products commit separately: step i + 2's S^T product waits only for step
// i's dV product (which read P^T from that buffer) and its dP^T product for
// step i's dK product, each of which the tensor pipe has finished or is
// finishing while the other runs, so the pipe never drains between steps.
// An item's dK and dV leave through shared memory: the item's K/V buffer is
// free once its last S^T / dP^T products are done, and each compute warp
// writes its 32 rows x 64 columns of dK and of dV there as bf16 in the
// 128-byte swizzle and stores them with TMA copies (rows past the sequence
// end clipped by the map's T extent).  The buffer returns to the K/V loader
// once those copies have read it.
constexpr int NCG = 2;
constexpr int CSP = 64 / NCG;
constexpr int MMA_G_WARP = 2 + 4 * NCG;          // the warp that issues the gradient products
constexpr int THREADS_B = 64 + 32 * 4 * NCG + 32;
constexpr int KV_T = 32768, QT64 = 16384;

constexpr int STG_WARP = 32 * 128;   // one compute warp's 32 x 64 bf16 block (128-byte rows)
constexpr int DKDV_QS = 3;
constexpr int KV_BUF = 2 * KV_T;   // K and V of one item
constexpr int DKDV_SMEM = 2 * KV_BUF + DKDV_QS * 2 * QT64 + 1024 + 256;

__global__ void __launch_bounds__(THREADS_B, 1)
    fa_tc_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm128, const __grid_constant__ CUtensorMap tm64,
                          const __grid_constant__ CUtensorMap tmDO, const __grid_constant__ CUtensorMap tmG,
                          const float* __restrict__ lse2, const float* __restrict__ Dv, int T, int H, int BH,
                          unsigned* err) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  using namespace tc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sKV = smem;                        // [2 buffers]: K then V
  uint8_t* sQ = sKV + 2 * KV_BUF;             // [DKDV_QS stages]
  uint8_t* sO = sQ + DKDV_QS * QT64;          // dO [DKDV_QS stages]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sO + DKDV_QS * QT64);
  uint64_t* kv_full = bars;                   // 2 (per K/V buffer)
  uint64_t* kv_free = kv_full + 2;            // 2 (per K/V buffer: the item's dK/dV copies have read it)
  uint64_t* q_full = kv_free + 2;             // DKDV_QS
  uint64_t* q_empty = q_full + DKDV_QS;       // DKDV_QS
  uint64_t* s_full = q_empty + DKDV_QS;       // 1: S^T, dP^T of the step computed
  uint64_t* s_read = s_full + 1;              // 1: the compute warps have loaded them
  uint64_t* p_full = s_read + 1;              // 2: P^T, dS^T of the packed buffer written
  uint64_t* g_done = p_full + 2;              // 2: the dV, dK products have read the packed buffer
  uint64_t* acc_full = g_done + 2;            // 1: the item's last dV/dK products are done
  uint64_t* acc_empty = acc_full + 1;         // 1: the compute warps have read dV/dK
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 1);
  static_assert((12 + 2 * DKDV_QS) * 8 + 8 <= 256, "barrier area");
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int a = H * 128;
  const int n_kt = (T + 127) / 128, nq = (T + 63) / 64;
  const int total = n_kt * BH;
  const int first = blockIdx.x, stride = gridDim.x;
  // item i (heaviest first): key tile kt, (sequence, head) bh, query steps of 64 from the diagonal on
  auto item = [&](int i, int& kt, int& bh, int& n_it) {
    kt = i / BH;
    bh = i % BH;
    n_it = nq - 2 * kt;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_free[s], 4 * NCG);
      mbar_init(&p_full[s], 4 * NCG);  // one arrival per compute warp
      mbar_init(&g_done[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_read, 4 * NCG);
    for (int s = 0; s < DKDV_QS; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 2);   // released by both MMA warps
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 4 * NCG);
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
  // S^T: cols 0..63, dP^T: 64..127 (fp32, one step at a time); packed buffer b
  // at 128 + 64 b: P^T in its first 32 columns, dS^T in the next 32 (bf16
  // pairs, column group grp at 16 grp); dV: 256; dK: 384.
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 1) {
      // ---------------------------------------------------------------- TMA: K, V
      bool ok = true;
      int nkv = 0;
      for (int i = first, k = 0; i < total && ok; i += stride, ++k) {
        int kt, bh, n_it;
        item(i, kt, bh, n_it);
        const int b = bh / H, h = bh % H, kr = b * T + kt * 128, kb = k & 1;
        // the dK/dV copies of item k - 2 have read this buffer
        if (k >= 2 && !mbar_wait(&kv_free[kb], ((k - 2) >> 1) & 1, abort_flag, err)) { ok = false; break; }
        uint8_t* kv = sKV + kb * KV_BUF;
        mbar_expect_tx(&kv_full[kb], KV_BUF);
        tma_load_2d(kv, &tm128, &kv_full[kb], a + h * 128, kr);
        tma_load_2d(kv + KV_T / 2, &tm128, &kv_full[kb], a + h * 128 + 64, kr);
        tma_load_2d(kv + KV_T, &tm128, &kv_full[kb], 2 * a + h * 128, kr);
        tma_load_2d(kv + KV_T + KV_T / 2, &tm128, &kv_full[kb], 2 * a + h * 128 + 64, kr);
        ++nkv;
      }
      for (int k = (nkv > 2 ? nkv - 2 : 0); k < nkv; ++k) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&kv_full[k & 1], (k >> 1) & 1)) if (globaltimer_ns() - t0 > GPT_WAIT_LIMIT_NS) break;
      }
    } else if (lane == 0) {
      // ---------------------------------------------------------------- TMA: Q, dO ring
      bool ok = true;
      int g = 0;
      for (int i = first; i < total && ok; i += stride) {
        int kt, bh, n_it;
        item(i, kt, bh, n_it);
        const int b = bh / H, h = bh % H, row_base = b * T;
        for (int j = 0; j < n_it && ok; ++j, ++g) {
          const int s = g % DKDV_QS;
          if (!mbar_wait(&q_empty[s], ((g / DKDV_QS) & 1) ^ 1, abort_flag, err)) { ok = false; break; }
          mbar_expect_tx(&q_full[s], 2 * QT64);
          const int qr = row_base + (2 * kt + j) * 64;
          uint8_t* q = sQ + s * QT64;
          uint8_t* o = sO + s * QT64;
          tma_load_2d(q, &tm64, &q_full[s], h * 128, qr);
          tma_load_2d(q + QT64 / 2, &tm64, &q_full[s], h * 128 + 64, qr);
          tma_load_2d(o, &tmDO, &q_full[s], h * 128, qr);
          tma_load_2d(o + QT64 / 2, &tmDO, &q_full[s], h * 128 + 64, qr);
        }
      }
      for (int j = (g > DKDV_QS ? g - DKDV_QS : 0); j < g; ++j) {
        const uint64_t t1 = globaltimer_ns();
        while (!mbar_try_wait(&q_full[j % DKDV_QS], (j / DKDV_QS) & 1))
          if (globaltimer_ns() - t1 > GPT_WAIT_LIMIT_NS) break;
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA: scores
    // Two MMA warps, each running as a whole warp with one elected lane
    // issuing: this one issues S^T, dP^T of every step of this CTA's items in
    // order, warp MMA_G_WARP the dV, dK products, so neither waits behind
    // the other's barriers; the tensor pipe interleaves the two streams.
    const uint32_t id_s = idesc(64, false);   // S^T = K Q^T, dP^T = V dO^T (N = 64 queries)
    bool ok = true;
    int g = 0;
    for (int i = first, k = 0; i < total && ok; i += stride, ++k) {
      int kt, bh, n_it;
      item(i, kt, bh, n_it);
      const int kb = k & 1;
      if (!warp_wait(&kv_full[kb], (k >> 1) & 1, abort_flag, err)) { ok = false; break; }
      for (int j = 0; j < n_it; ++j, ++g) {
        const int st = g % DKDV_QS;
        if (!warp_wait(&q_full[st], (g / DKDV_QS) & 1, abort_flag, err)) { ok = false; break; }
        // S^T, dP^T of step g overwrite step g - 1's: the compute warps have loaded those
        if (g >= 1 && !warp_wait(s_read, (g - 1) & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t aK = smem_u32(sKV + kb * KV_BUF), aV = aK + KV_T;
        const uint32_t aQ = smem_u32(sQ + st * QT64), aO = smem_u32(sO + st * QT64);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc_mma_w(tmem, kdesc128(aK, KV_T / 2, kk), kdesc128(aQ, QT64 / 2, kk), id_s, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc_mma_w(tmem + 64, kdesc128(aV, KV_T / 2, kk), kdesc128(aO, QT64 / 2, kk), id_s, kk > 0 ? 1u : 0u);
        tc_commit_w(s_full);
        tc_commit_w(&q_empty[st]);   // one of the stage's two releases
      }
    }
  } else if (warp == MMA_G_WARP) {
    // ---------------------------------------------------------------- MMA: gradients
    const uint32_t id_g = idesc(128, true);   // dV += P^T dO, dK += dS^T Q (N = 128, B MN-major)
    bool ok = true;
    int g = 0;
    for (int i = first, k = 0; i < total && ok; i += stride, ++k) {
      int kt, bh, n_it;
      item(i, kt, bh, n_it);
      // the item's first products overwrite dV, dK: the previous item's have been read
      if (k >= 1 && !warp_wait(acc_empty, (k - 1) & 1, abort_flag, err)) { ok = false; break; }
      for (int j = 0; j < n_it; ++j, ++g) {
        const int s = g & 1, st = g % DKDV_QS;
        if (!warp_wait(&p_full[s], (g >> 1) & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t aQ = smem_u32(sQ + st * QT64), aO = smem_u32(sO + st * QT64);
        // k-step kk covers queries 16kk..16kk+15: packed columns 8kk..8kk+7
        const uint32_t pb = tmem + 128 + s * 64;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma_ts_w(tmem + 256, pb + 8 * kk, mndesc(aO, QT64 / 2, kk), id_g, (j > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma_ts_w(tmem + 384, pb + 32 + 8 * kk, mndesc(aQ, QT64 / 2, kk), id_g, (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit_w(&g_done[s]);
        tc_commit_w(&q_empty[st]);   // the stage's other release
      }
      if (ok) tc_commit_w(acc_full);   // the item's dV, dK are complete
    }
  } else if (warp < MMA_G_WARP) {
    // ---------------------------------------------------------------- P^T, dS^T
    const int q4 = warp & 3, grp = (warp - 2) >> 2;
    const int r = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const float c = rsqrtf(128.f) * LOG2E;
    const int blk = (grp * 4 + q4) * STG_WARP;   // this warp's 32 x 64 block inside the K (dK) / V (dV) halves
    bool ok = true;
    bool store_pending = false;   // the previous item's dK/dV copies may still be reading its buffer
    int g = 0;
    for (int i = first, k = 0; i < total && ok; i += stride, ++k) {
      int kt, bh, n_it;
      item(i, kt, bh, n_it);
      const int b = bh / H, h = bh % H;
      const int k0 = kt * 128, qi0 = 2 * kt;
      const int key = k0 + r;
      const int warp_key_max = k0 + q4 * 32 + 31;
      const float* lse_bh = lse2 + (long long)bh * T;
      const float* D_bh = Dv + (long long)bh * T;
      for (int j = 0; j < n_it; ++j, ++g) {
        const int s = g & 1;
        const int qbase = (qi0 + j) * 64 + grp * CSP;
        // this group's CSP (lse2, D) pairs, fetched before the scores arrive
        const bool fullc = qbase + CSP <= T;  // warp-uniform
        float lv[CSP], dv[CSP];
        if (fullc) {
#pragma unroll
          for (int e4 = 0; e4 < CSP / 4; ++e4) {
            const float4 l4 = *reinterpret_cast<const float4*>(lse_bh + qbase + 4 * e4);
            const float4 d4 = *reinterpret_cast<const float4*>(D_bh + qbase + 4 * e4);
            lv[4 * e4] = l4.x; lv[4 * e4 + 1] = l4.y; lv[4 * e4 + 2] = l4.z; lv[4 * e4 + 3] = l4.w;
            dv[4 * e4] = d4.x; dv[4 * e4 + 1] = d4.y; dv[4 * e4 + 2] = d4.z; dv[4 * e4 + 3] = d4.w;
          }
        } else {
#pragma unroll
          for (int e = 0; e < CSP; ++e) {
            lv[e] = qbase + e < T ? lse_bh[qbase + e] : 0.f;
            dv[e] = qbase + e < T ? D_bh[qbase + e] : 0.f;
          }
        }
        if (!warp_wait(s_full, g & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t cs = tmem + lane_off + grp * CSP;   // this warp's S^T columns
        const uint32_t cd = cs + 64;                       // and dP^T columns
        float sv[CSP], dp[CSP];
        {
          uint32_t r0[CSP], r1[CSP];
          tmem_ldw<CSP>(cs, r0);
          tmem_ldw<CSP>(cd, r1);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < CSP; ++e) { sv[e] = __uint_as_float(r0[e]); dp[e] = __uint_as_float(r1[e]); }
        }
        // loaded: the next step's S^T, dP^T may overwrite these columns
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_read);
        // P^T[key, q] = exp2(s c - lse2_q) for key <= q < T; dS^T = P^T (dP^T - D_q).
        // Off the diagonal every key of the warp is <= every query of the group
        // (warp-uniform), so the causal test drops out.
        if (fullc && warp_key_max <= qbase) {
#pragma unroll
          for (int e = 0; e < CSP; e += 2) {   // two lanes of fp32 per instruction
            float x0, x1;
            fma2v(x0, x1, sv[e], sv[e + 1], c, -lv[e], -lv[e + 1]);
            const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
            sv[e] = p0;
            sv[e + 1] = p1;
            mulsub2(dp[e], dp[e + 1], p0, p1, dp[e], dp[e + 1], dv[e], dv[e + 1]);
          }
        } else {
#pragma unroll
          for (int e = 0; e < CSP; ++e) {
            const int qq = qbase + e;
            const float p = (key <= qq && qq < T) ? fast_exp2(fmaf(sv[e], c, -lv[e])) : 0.f;
            sv[e] = p;
            dp[e] = p * (dp[e] - dv[e]);
          }
        }
        // bf16 pairs into packed buffer s (this warp's own lanes and columns),
        // once the dV, dK products of step g - 2 have read it
        uint32_t pw[CSP / 2], dw[CSP / 2];
#pragma unroll
        for (int jj = 0; jj < CSP / 2; ++jj) {
          pw[jj] = pack_bf16x2_rn(sv[2 * jj], sv[2 * jj + 1]);
          dw[jj] = pack_bf16x2_int(dp[2 * jj], dp[2 * jj + 1]);
        }
        if (g >= 2 && !warp_wait(&g_done[s], ((g - 2) >> 1) & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t pbw = tmem + lane_off + 128 + s * 64 + grp * (CSP / 2);
        tmem_stw<CSP / 2>(pbw, pw);
        tmem_stw<CSP / 2>(pbw + 32, dw);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[s]);
        if (j == 0 && store_pending) {
          // the previous item's dK/dV copies have had a step to read its K/V
          // buffer: hand the buffer back to the K/V loader
          if (lane == 0) {
            bulk_wait_read0();
            mbar_arrive(&kv_free[(k - 1) & 1]);
          }
          store_pending = false;
        }
      }
      if (!ok) break;
      // ------------------------------------------------------------ item epilogue
      if (!warp_wait(acc_full, k & 1, abort_flag, err)) { ok = false; break; }
      tc_fence_after();
      static_assert(NCG == 2, "two 64-column groups of dK and dV");
      uint32_t v0[32], v1[32], k0r[32], k1r[32];
      tmem_ld32_nowait(tmem + lane_off + 256 + grp * 64, v0);
      tmem_ld32_nowait(tmem + lane_off + 256 + grp * 64 + 32, v1);
      tmem_ld32_nowait(tmem + lane_off + 384 + grp * 64, k0r);
      tmem_ld32_nowait(tmem + lane_off + 384 + grp * 64 + 32, k1r);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);  // the next item's products may overwrite dV, dK
      // staging: this item's K/V buffer (its last S^T / dP^T products are done)
      uint8_t* stK = sKV + (k & 1) * KV_BUF + blk;
      uint8_t* stV = stK + KV_T;
      const float sc = rsqrtf(128.f);
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const uint32_t* sv_ = jj < 4 ? v0 + 8 * jj : v1 + 8 * (jj - 4);
        const uint32_t* sk_ = jj < 4 ? k0r + 8 * jj : k1r + 8 * (jj - 4);
        uint4 wv, wk;
        wv.x = pack_bf16x2_rn(__uint_as_float(sv_[0]), __uint_as_float(sv_[1]));
        wv.y = pack_bf16x2_rn(__uint_as_float(sv_[2]), __uint_as_float(sv_[3]));
        wv.z = pack_bf16x2_rn(__uint_as_float(sv_[4]), __uint_as_float(sv_[5]));
        wv.w = pack_bf16x2_rn(__uint_as_float(sv_[6]), __uint_as_float(sv_[7]));
        wk.x = pack_bf16x2_rn(__uint_as_float(sk_[0]) * sc, __uint_as_float(sk_[1]) * sc);
        wk.y = pack_bf16x2_rn(__uint_as_float(sk_[2]) * sc, __uint_as_float(sk_[3]) * sc);
        wk.z = pack_bf16x2_rn(__uint_as_float(sk_[4]) * sc, __uint_as_float(sk_[5]) * sc);
        wk.w = pack_bf16x2_rn(__uint_as_float(sk_[6]) * sc, __uint_as_float(sk_[7]) * sc);
        *reinterpret_cast<uint4*>(stV + swz128(lane, jj)) = wv;
        *reinterpret_cast<uint4*>(stK + swz128(lane, jj)) = wk;
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (k0 + q4 * 32 < T) {  // rows past T are clipped; a block wholly past it is skipped
          tma_store_3d(&tmG, stK, a + h * 128 + grp * 64, k0 + q4 * 32, b);
          tma_store_3d(&tmG, stV, 2 * a + h * 128 + grp * 64, k0 + q4 * 32, b);
        }
        bulk_commit();
      }
      store_pending = true;
    }
    if (lane == 0) bulk_wait0();  // this warp's stores are complete
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

// ---------------------------------------------------------------- dQ
// Warps as above; the compute warps' column groups split the 64 key columns.
// Persistent like the forward: one CTA per SM over the (query tile,
// sequence, head) items heaviest first; the K/V ring and the S/dP buffers run
// on across items, Q/dO for the next item load once the item's last S/dP has
// read them, and dQ alternates between two TMEM accumulators.  dS is written
// as bf16 over the dP columns each compute warp has just read and feeds the
// dQ product from TMEM.
// The MMA warp issues as a whole warp (one elected lane).  Step g's score
// product needs only that the compute warps have read buffer g & 1 (they
// released step g - 2 before the dQ product of step g - 2 was issued); its dP
// product waits for that dQ product, which the score product separates from
// it in the tensor pipe, so the pipe never drains between steps.
// The item's dQ leaves through shared memory: each compute warp writes its 32
// rows x 64 columns as bf16 in the 128-byte swizzle and stores them with one
// TMA copy (rows past the sequence end are clipped by the map's T extent).
// smem: Q, dO [128 x 128] (32 KB each); per stage K_j, V_j [64 x 128] (16 KB
// each, DQ_STAGES stages); 8 staging blocks of 4 KB.
constexpr int DQ_STAGES = 4;
constexpr int DQ_SMEM = 2 * KV_T + DQ_STAGES * 2 * QT64 + 4 * NCG * STG_WARP + 1024 + 256;

__global__ void __launch_bounds__(THREADS_B, 1)
    fa_tc_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm128, const __grid_constant__ CUtensorMap tm64,
                        const __grid_constant__ CUtensorMap tmDO, const __grid_constant__ CUtensorMap tmG,
                        const float* __restrict__ lse2, const float* __restrict__ Dv, int T, int H, int BH,
                        unsigned* err) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  using namespace tc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sO = sQ + KV_T;
  uint8_t* sK = sO + KV_T;                   // [stages]
  uint8_t* sV = sK + DQ_STAGES * QT64;       // [stages]
  uint8_t* sStg = sV + DQ_STAGES * QT64;     // [compute warps]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sStg + 4 * NCG * STG_WARP);
  uint64_t* q_full = bars;                      // 1
  uint64_t* q_empty = q_full + 1;               // 1 (the item's last S/dP have read Q and dO)
  uint64_t* kv_full = q_empty + 1;              // DQ_STAGES
  uint64_t* kv_empty = kv_full + DQ_STAGES;     // DQ_STAGES
  uint64_t* s_full = kv_empty + DQ_STAGES;      // 1: S, dP of the step computed
  uint64_t* s_read = s_full + 1;                // 1: the compute warps have loaded them
  uint64_t* p_full = s_read + 1;                // 2: dS of the packed buffer written (all compute warps)
  uint64_t* g_done = p_full + 2;                // 2: the dQ product has read the packed buffer
  uint64_t* o_full = g_done + 2;                // 2 (per dQ buffer: the item's last product is done)
  uint64_t* o_empty = o_full + 2;               // 2 (per dQ buffer: the compute warps have read it)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_empty + 2);
  static_assert((2 + 2 * DQ_STAGES + 10) * 8 + 8 <= 256, "barrier area");
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int a = H * 128;
  const int n_qt = (T + 127) / 128;
  const int total = n_qt * BH;
  const int first = blockIdx.x, stride = gridDim.x;
  // item i (heaviest first): query tile qt, (sequence, head) bh, key tiles of 64 up to the diagonal
  auto item = [&](int i, int& qt, int& bh, int& n_it) {
    qt = n_qt - 1 - i / BH;
    bh = i % BH;
    n_it = min((qt * 128 + 128) / 64, (T + 63) / 64);
  };

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < DQ_STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 2);   // released by both MMA warps
    }
    mbar_init(s_full, 1);
    mbar_init(s_read, 4 * NCG);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&p_full[s], 4 * NCG);  // one arrival per compute warp
      mbar_init(&g_done[s], 1);
      mbar_init(&o_full[s], 1);
      mbar_init(&o_empty[s], 4 * NCG);
    }
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
  // S: cols 0..63, dP: 64..127 (fp32, one step at a time); packed dS buffer b
  // at 128 + 32 b (bf16 pairs, column group grp at 16 grp); dQ: 256 and 384
  // (alternating per item)
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- TMA
      bool ok = true;
      int g = 0, nq = 0;
      for (int i = first, k = 0; i < total && ok; i += stride, ++k) {
        int qt, bh, n_it;
        item(i, qt, bh, n_it);
        const int b = bh / H, h = bh % H, row_base = b * T, q0 = qt * 128;
        if (k > 0 && !mbar_wait(q_empty, (k - 1) & 1, abort_flag, err)) { ok = false; break; }
        mbar_expect_tx(q_full, 2 * KV_T);
        tma_load_2d(sQ, &tm128, q_full, h * 128, row_base + q0);
        tma_load_2d(sQ + KV_T / 2, &tm128, q_full, h * 128 + 64, row_base + q0);
        // dO [128 x 128] through the 64-row map: half hf (64 columns) x row block rb
        for (int hf = 0; hf < 2; ++hf)
          for (int rb = 0; rb < 2; ++rb)
            tma_load_2d(sO + hf * (KV_T / 2) + rb * 8192, &tmDO, q_full, h * 128 + 64 * hf, row_base + q0 + 64 * rb);
        ++nq;
        for (int j = 0; j < n_it && ok; ++j, ++g) {
          const int s = g % DQ_STAGES;
          if (!mbar_wait(&kv_empty[s], ((g / DQ_STAGES) & 1) ^ 1, abort_flag, err)) { ok = false; break; }
          mbar_expect_tx(&kv_full[s], 2 * QT64);
          const int kr = row_base + j * 64;
          uint8_t* kt = sK + s * QT64;
          uint8_t* v = sV + s * QT64;
          tma_load_2d(kt, &tm64, &kv_full[s], a + h * 128, kr);
          tma_load_2d(kt + QT64 / 2, &tm64, &kv_full[s], a + h * 128 + 64, kr);
          tma_load_2d(v, &tm64, &kv_full[s], 2 * a + h * 128, kr);
          tma_load_2d(v + QT64 / 2, &tm64, &kv_full[s], 2 * a + h * 128 + 64, kr);
        }
      }
      if (nq > 0) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(q_full, (nq - 1) & 1)) if (globaltimer_ns() - t0 > GPT_WAIT_LIMIT_NS) break;
      }
      for (int j = (g > DQ_STAGES ? g - DQ_STAGES : 0); j < g; ++j) {
        const uint64_t t1 = globaltimer_ns();
        while (!mbar_try_wait(&kv_full[j % DQ_STAGES], (j / DQ_STAGES) & 1))
          if (globaltimer_ns() - t1 > GPT_WAIT_LIMIT_NS) break;
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA: scores
    // Two MMA warps as in the dK/dV kernel: this one issues S and dP of every
    // step, warp MMA_G_WARP the dQ products.
    const uint32_t id_s = idesc(64, false);   // S = Q K^T, dP = dO V^T (N = 64 keys)
    const uint32_t aQ = smem_u32(sQ), aO = smem_u32(sO);
    bool ok = true;
    int g = 0;
    for (int i = first, k = 0; i < total && ok; i += stride, ++k) {
      int qt, bh, n_it;
      item(i, qt, bh, n_it);
      if (!warp_wait(q_full, k & 1, abort_flag, err)) { ok = false; break; }
      for (int j = 0; j < n_it; ++j, ++g) {
        const int st = g % DQ_STAGES;
        if (!warp_wait(&kv_full[st], (g / DQ_STAGES) & 1, abort_flag, err)) { ok = false; break; }
        // S, dP of step g overwrite step g - 1's: the compute warps have loaded those
        if (g >= 1 && !warp_wait(s_read, (g - 1) & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t aK = smem_u32(sK + st * QT64), aV = smem_u32(sV + st * QT64);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc_mma_w(tmem, kdesc128(aQ, KV_T / 2, kk), kdesc128(aK, QT64 / 2, kk), id_s, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc_mma_w(tmem + 64, kdesc128(aO, KV_T / 2, kk), kdesc128(aV, QT64 / 2, kk), id_s, kk > 0 ? 1u : 0u);
        tc_commit_w(s_full);
        tc_commit_w(&kv_empty[st]);   // one of the stage's two releases
      }
      if (ok) tc_commit_w(q_empty);   // the item's last S/dP: Q and dO may be replaced
    }
  } else if (warp == MMA_G_WARP) {
    // ---------------------------------------------------------------- MMA: dQ
    const uint32_t id_g = idesc(128, true);   // dQ += dS K (N = 128, B MN-major)
    bool ok = true;
    int g = 0;
    for (int i = first, k = 0; i < total && ok; i += stride, ++k) {
      int qt, bh, n_it;
      item(i, qt, bh, n_it);
      const int ob = k & 1;
      // the item's first product overwrites its dQ buffer: the compute warps
      // have read that buffer for the item two positions back
      if (k >= 2 && !warp_wait(&o_empty[ob], ((k - 2) >> 1) & 1, abort_flag, err)) { ok = false; break; }
      for (int j = 0; j < n_it; ++j, ++g) {
        const int s = g & 1, st = g % DQ_STAGES;
        if (!warp_wait(&p_full[s], (g >> 1) & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t aK = smem_u32(sK + st * QT64);
        // k-step kk covers keys 16kk..16kk+15: packed columns 8kk..8kk+7
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma_ts_w(tmem + 256 + ob * 128, tmem + 128 + s * 32 + 8 * kk, mndesc(aK, QT64 / 2, kk), id_g,
                      (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit_w(&g_done[s]);
        tc_commit_w(&kv_empty[st]);   // the stage's other release
      }
      if (ok) tc_commit_w(&o_full[ob]);   // the item's dQ is complete
    }
  } else if (warp < MMA_G_WARP) {
    // ---------------------------------------------------------------- dS
    const int q4 = warp & 3, grp = (warp - 2) >> 2;
    const int r = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const float c = rsqrtf(128.f) * LOG2E;
    uint8_t* stg = sStg + (warp - 2) * STG_WARP;
    bool ok = true;
    int g = 0;
    for (int i = first, k = 0; i < total && ok; i += stride, ++k) {
      int qt, bh, n_it;
      item(i, qt, bh, n_it);
      const int b = bh / H, h = bh % H;
      const int qpos = qt * 128 + r;
      const bool valid = qpos < T;
      const float L = valid ? lse2[(long long)bh * T + qpos] : 0.f;  // log2 units
      const float Dq = valid ? Dv[(long long)bh * T + qpos] : 0.f;
      const int ob = k & 1;
      for (int j = 0; j < n_it; ++j, ++g) {
        const int s = g & 1;
        if (!warp_wait(s_full, g & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        float sv[CSP], dp[CSP];
        {
          uint32_t r0[CSP], r1[CSP];
          tmem_ldw<CSP>(tmem + lane_off + grp * CSP, r0);        // this warp's S columns
          tmem_ldw<CSP>(tmem + lane_off + 64 + grp * CSP, r1);   // and dP columns
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < CSP; ++e) { sv[e] = __uint_as_float(r0[e]); dp[e] = __uint_as_float(r1[e]); }
        }
        // loaded: the next step's S, dP may overwrite these columns
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_read);
        const int kbase = j * 64 + grp * CSP;
#pragma unroll
        for (int e = 0; e < CSP; e += 2) {   // two lanes of fp32 per instruction
          float x0, x1;
          fma2(x0, x1, sv[e], sv[e + 1], c, -L);
          const float p0 = (valid && kbase + e <= qpos) ? fast_exp2(x0) : 0.f;
          const float p1 = (valid && kbase + e + 1 <= qpos) ? fast_exp2(x1) : 0.f;
          mulsub2(dp[e], dp[e + 1], p0, p1, dp[e], dp[e + 1], Dq, Dq);
        }
        // dS as bf16 pairs into packed buffer s (this warp's own lanes and
        // columns), once the dQ product of step g - 2 has read it
        uint32_t dw[CSP / 2];
#pragma unroll
        for (int jj = 0; jj < CSP / 2; ++jj) dw[jj] = pack_bf16x2_int(dp[2 * jj], dp[2 * jj + 1]);
        if (g >= 2 && !warp_wait(&g_done[s], ((g - 2) >> 1) & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        tmem_stw<CSP / 2>(tmem + lane_off + 128 + s * 32 + grp * (CSP / 2), dw);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[s]);
      }
      if (!ok) break;
      if (!warp_wait(&o_full[ob], (k >> 1) & 1, abort_flag, err)) { ok = false; break; }
      tc_fence_after();
      // this warp's 32 rows x 64 columns of dQ (column group grp)
      static_assert(NCG == 2, "two 64-column groups of dQ");
      uint32_t o0[32], o1[32];
      tmem_ld32_nowait(tmem + lane_off + 256 + ob * 128 + grp * 64, o0);
      tmem_ld32_nowait(tmem + lane_off + 256 + ob * 128 + grp * 64 + 32, o1);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_empty[ob]);  // this dQ buffer may be overwritten
      // the previous item's store has read the staging block
      if (lane == 0) bulk_wait_read0();
      __syncwarp();
      const float sc = rsqrtf(128.f);
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const uint32_t* src = jj < 4 ? o0 + 8 * jj : o1 + 8 * (jj - 4);
        uint4 w;
        w.x = pack_bf16x2_rn(__uint_as_float(src[0]) * sc, __uint_as_float(src[1]) * sc);
        w.y = pack_bf16x2_rn(__uint_as_float(src[2]) * sc, __uint_as_float(src[3]) * sc);
        w.z = pack_bf16x2_rn(__uint_as_float(src[4]) * sc, __uint_as_float(src[5]) * sc);
        w.w = pack_bf16x2_rn(__uint_as_float(src[6]) * sc, __uint_as_float(src[7]) * sc);
        *reinterpret_cast<uint4*>(stg + swz128(lane, jj)) = w;
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0 && qt * 128 + q4 * 32 < T) {  // rows past T are clipped; a block wholly past it is skipped
        tma_store_3d(&tmG, stg, h * 128 + grp * 64, qt * 128 + q4 * 32, b);
        bulk_commit();
      }
    }
    if (lane == 0) bulk_wait0();  // this warp's stores are complete
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

}  // namespace fatcb
