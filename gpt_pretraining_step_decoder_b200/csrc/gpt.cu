// gpt.cu -- C ABI of libgpt_b200.so and the host-side step orchestration.
//
// All device memory comes from the caller's arena; this file carves it,
// enqueues every kernel of a forward / backward / optimizer step on one CUDA
// stream, and maps the device error word to status codes.  The meaning of
// each entry point is documented in include/gpt.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdarg>
#include <cstdlib>
#include <cstring>
#include <type_traits>
#include <atomic>
#include <map>
#include <string>
#include <vector>

#include "../../include/gpt.h"
#include "common.cuh"
#include "gemm_common.cuh"
#include "gemm_simt.cuh"
#include "gemm_tc.cuh"
#include "attention_tc.cuh"
#include "layers.cuh"
#include "ngram.cuh"
#include "optim.cuh"
#include "muon.cuh"
#include "fp8.cuh"

// Run the statements with NV = d / 128 (vec4 chunks per lane of a row kernel)
// as a compile-time constant; rows that are not a multiple of 128 use MAXV.
#define WITH_NV(d, ...);                                      \
  do {                                                       \
    switch (((d) % 128 == 0) ? (d) / 128 : 0) {              \
      case 1: { constexpr int NV = 1; __VA_ARGS__; } break;  \
      case 2: { constexpr int NV = 2; __VA_ARGS__; } break;  \
      case 4: { constexpr int NV = 4; __VA_ARGS__; } break;  \
      case 6: { constexpr int NV = 6; __VA_ARGS__; } break;  \
      case 8: { constexpr int NV = 8; __VA_ARGS__; } break;  \
      case 16: { constexpr int NV = 16; __VA_ARGS__; } break; \
      default: { constexpr int NV = MAXV; __VA_ARGS__; } break; \
    }                                                        \
  } while (0)

// ======================================================================== errors
static thread_local std::string g_last_error;

static int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

#define CUDA_TRY(expr)                                                                    \
  do {                                                                                    \
    cudaError_t e_ = (expr);                                                              \
    if (e_ != cudaSuccess)                                                                \
      return fail(GPT_ERR_CUDA, "%s failed: %s (%s:%d)", #expr, cudaGetErrorString(e_),   \
                  __FILE__, __LINE__);                                                    \
  } while (0)

#define LAUNCH_CHECK() CUDA_TRY(cudaGetLastError())

#define TRY(expr)            \
  do {                       \
    int s_ = (expr);         \
    if (s_ != GPT_OK) return s_; \
  } while (0)

extern "C" const char* gpt_last_error(void) { return g_last_error.c_str(); }

// Kernels this library has launched in this process (read by gpt_launch_count).
static std::atomic<long long> g_launches{0};

// ======================================================================== device props
static int device_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

// standalone operations' error word (one per device that loads the library)
__device__ unsigned g_ngram_err;

// ======================================================================== TMA maps
static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

static int get_encode() {
  if (g_encode) return GPT_OK;
  cudaDriverEntryPointQueryResult q;
  void* fn = nullptr;
  CUDA_TRY(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q));
  if (!fn || q != cudaDriverEntryPointSuccess) return fail(GPT_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return GPT_OK;
}

// Tensor map of `rank` dims (innermost first) with byte strides for dims 1..,
// 128-byte swizzle, zero fill outside the tensor.
static int make_tmap_gen(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* ptr,
                         const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                         CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  TRY(get_encode());
  if (reinterpret_cast<uintptr_t>(ptr) & 15) return fail(GPT_ERR_ARG, "TMA operand %p not 16-byte aligned", ptr);
  for (int i = 0; i + 1 < rank; ++i)
    if (strides_bytes[i] & 15) return fail(GPT_ERR_ARG, "TMA row pitch %llu not a multiple of 16 bytes",
                                           (unsigned long long)strides_bytes[i]);
  cuuint64_t d[3], s[2];
  cuuint32_t b[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) { d[i] = dims[i]; b[i] = box[i]; }
  for (int i = 0; i + 1 < rank; ++i) s[i] = strides_bytes[i];
  CUresult r = g_encode(m, dt, rank, const_cast<void*>(ptr), d, s, b, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(GPT_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return GPT_OK;
}

// 2-D bf16 map over a row-major [outer, inner] buffer with row pitch `ld` elements.
static int make_tmap(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint64_t ld,
                     uint32_t box_inner, uint32_t box_outer) {
  const uint64_t dims[2] = {inner, outer}, str[1] = {ld * 2};
  const uint32_t box[2] = {box_inner, box_outer};
  return make_tmap_gen(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, dims, str, box);
}

// ======================================================================== GEMM dispatch
// CTA pairs (tcgen05 cta_group::2) for every GEMM with 256-column tiles,
// unless GPT_GEMM_CTA_PAIR=0 in the environment or gptx_set_gemm_cta_pairs(0)
// selects one-CTA tiles.
static std::atomic<int> g_gemm_pairs{-1};
static bool gemm_pairs_enabled() {
  int v = g_gemm_pairs.load();
  if (v < 0) {
    const char* e = getenv("GPT_GEMM_CTA_PAIR");
    v = (e && e[0] == '0') ? 0 : 1;
    g_gemm_pairs.store(v);
  }
  return v == 1;
}

extern "C" int gptx_set_gemm_cta_pairs(int on) {
  g_gemm_pairs.store(on ? 1 : 0);
  return GPT_OK;
}

// Programmatic dependent launch for the step's frequent kernels (GEMM,
// split-K reduce, attention, norms, RoPE backward, cross-entropy, AdamW):
// each is set up while the kernel before it in the stream finishes, and calls
// pdl_wait() before touching global memory.  Measured on B200: 33.97 -> 33.25
// ms per GPT-2-small step, about the time the step spent between kernels.
// GPT_PDL=0 in the environment launches them plainly.
static bool pdl_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("GPT_PDL");
    v = (e && e[0] == '0') ? 0 : 1;
  }
  return v == 1;
}
static void pdl_attr(cudaLaunchAttribute& a) {
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = 1;
}
template <typename... KArgs, typename... Args>
static void launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  pdl_attr(at[0]);
  cfg.attrs = at;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Pairs of SMs that can hold one pair-mode GEMM cluster each at a time (the
// persistent grid's size in units of tiles); computed once per kernel.
template <typename K>
static int resident_clusters(K* kernel, int smem, int cg) {
  if (cg == 1) return device_sms();
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = cg; at[0].val.clusterDim.y = 1; at[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(cg * (device_sms() / cg));
  cfg.blockDim = dim3(tc::NUM_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n < 1) {
    cudaGetLastError();
    n = device_sms() / cg;
  }
  return n;
}

template <int BN, int KM, int CG, int F8 = 0, bool B3 = false>
static int gemm_tc_launch_k(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tcm,
                            const CUtensorMap& taux, const tc::Params& p, cudaStream_t st) {
  using C = tc::Cfg<BN, tc::KmHeavy<KM>::value, CG>;
  static_assert(C::SMEM_BYTES <= 232448, "shared memory budget");
  auto kernel = tc::gemm_tc_kernel<BN, KM, bf16, CG, F8, B3>;
  static int units = 0;
  if (!units) {
    CUDA_TRY(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES));
    units = resident_clusters(kernel, C::SMEM_BYTES, CG);
  }
  const int tiles = p.m_tiles * p.n_tiles * p.splits * p.batch;
  const int grid = CG * (tiles < units ? tiles : units);
  ++g_launches;
  {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[2];
    int na = 0;
    if constexpr (CG == 2) {
      at[na].id = cudaLaunchAttributeClusterDimension;
      at[na].val.clusterDim.x = CG; at[na].val.clusterDim.y = 1; at[na].val.clusterDim.z = 1;
      ++na;
    }
    if (pdl_enabled()) pdl_attr(at[na++]);
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(tc::NUM_THREADS);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = st;
    cfg.attrs = at;
    cfg.numAttrs = na;
    CUDA_TRY(cudaLaunchKernelEx(&cfg, kernel, ta, tb, tcm, taux, p));
  }
  LAUNCH_CHECK();
  return GPT_OK;
}

// `n` independent products of one shape whose operands and outputs lie at
// fixed element strides (n = 1: a single product).
struct GemmBatch {
  int n = 1;
  long long sa = 0, sb = 0, sc = 0;
};

// 3-D bf16 map over `batch` row-major [outer, inner] matrices `stride` elements apart
static int make_tmap3(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint64_t ld, int batch,
                      long long stride, uint32_t box_inner, uint32_t box_outer) {
  const uint64_t dims[3] = {inner, outer, (uint64_t)batch}, str[2] = {ld * 2, (uint64_t)stride * 2};
  const uint32_t box[3] = {box_inner, box_outer, 1};
  return make_tmap_gen(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, ptr, dims, str, box);
}

template <int BN, int CG = 1>
static int gemm_tc_launch(int M, int N, int K, GemmOperand A, GemmOperand B, GemmEpilogue e,
                          int splits, float* partial, unsigned* err, cudaStream_t st,
                          const GemmBatch& bt = GemmBatch()) {
  static_assert(CG == 1 || BN == 256, "CTA pairs take 256-column tiles");
  const bool b3 = bt.n > 1;
  if (b3 && (splits > 1 || (e.mode != EPI_STORE && e.mode != EPI_STORE_F32 && e.mode != EPI_AXPBY)))
    return fail(GPT_ERR_ARG, "batched GEMMs take store or AXPBY epilogues without split-K");
  CUtensorMap ta, tb, tcm, taux;
  if (b3) {
    if (A.kmajor) TRY(make_tmap3(&ta, A.ptr, K, M, A.ld, bt.n, bt.sa, tc::BK, tc::BM));
    else TRY(make_tmap3(&ta, A.ptr, M, K, A.ld, bt.n, bt.sa, 64, tc::BK));
    if (B.kmajor) TRY(make_tmap3(&tb, B.ptr, K, N, B.ld, bt.n, bt.sb, tc::BK, BN / CG));
    else TRY(make_tmap3(&tb, B.ptr, N, K, B.ld, bt.n, bt.sb, 64, tc::BK));
  } else {
    if (A.kmajor) TRY(make_tmap(&ta, A.ptr, K, M, A.ld, tc::BK, tc::BM));
    else TRY(make_tmap(&ta, A.ptr, M, K, A.ld, 64, tc::BK));
    // a CTA of a pair loads half of the tile's B rows
    if (B.kmajor) TRY(make_tmap(&tb, B.ptr, K, N, B.ld, tc::BK, BN / CG));
    else TRY(make_tmap(&tb, B.ptr, N, K, B.ld, 64, tc::BK));
  }
  tc::Params p;
  p.M = M; p.N = N; p.K = K;
  p.batch = bt.n;
  p.a_kmajor = A.kmajor; p.b_kmajor = B.kmajor;
  p.m_tiles = cdiv(M, CG * tc::BM);
  p.n_tiles = cdiv(N, BN);
  // n-fastest order while the whole B operand stays in L2; grouped m-blocks
  // when B is large (the LM head's vocab-sized operand): all of them when A
  // itself fits in L2 (the logits of a row chunk: each vocab tile is read
  // from HBM once, A from L2), else groups of 16
  const bool big_b = (double)N * K * 2 > 32.0 * (1 << 20), small_a = (double)M * K * 2 <= 32.0 * (1 << 20);
  p.group_m = big_b ? (small_a || p.m_tiles < 16 ? p.m_tiles : 16) : 1;
  p.kb_total = cdiv(K, tc::BK);
  if (splits < 1) splits = 1;
  if (splits > p.kb_total) splits = p.kb_total;
  p.kb_per_split = cdiv(p.kb_total, splits);
  p.splits = cdiv(p.kb_total, p.kb_per_split);
  p.epi = e;
  p.partial = partial;
  p.err = err;
  // output map: split-K partials [splits, M, N] fp32 (3-D so each split clips at M),
  // fp32 outputs in 32-column boxes, bf16 outputs in 64-column boxes (128-byte rows)
  if (b3) {
    const bool f32 = e.mode == EPI_STORE_F32;
    const uint64_t dims[3] = {(uint64_t)N, (uint64_t)M, (uint64_t)bt.n};
    const uint64_t str[2] = {(uint64_t)e.ldc * (f32 ? 4 : 2), (uint64_t)bt.sc * (f32 ? 4 : 2)};
    const uint32_t box[3] = {f32 ? 32u : 64u, 32, 1};
    TRY(make_tmap_gen(&tcm, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, e.C, dims,
                      str, box));
  } else if (p.splits > 1) {
    const uint64_t dims[3] = {(uint64_t)N, (uint64_t)M, (uint64_t)p.splits};
    const uint64_t str[2] = {(uint64_t)N * 4, (uint64_t)M * N * 4};
    const uint32_t box[3] = {32, 32, 1};
    TRY(make_tmap_gen(&tcm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, partial, dims, str, box));
  } else if (e.mode == EPI_STORE_F32 || e.mode == EPI_ACCUM_F32) {
    const uint64_t dims[2] = {(uint64_t)N, (uint64_t)M}, str[1] = {(uint64_t)e.ldc * 4};
    const uint32_t box[2] = {32, 32};
    TRY(make_tmap_gen(&tcm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, e.C, dims, str, box));
  } else {
    TRY(make_tmap(&tcm, e.C, N, M, e.ldc, 64, 32));
  }
  if (p.splits == 1 && (e.mode == EPI_DRELU2 || e.mode == EPI_AXPBY)) {
    if (!e.aux) return fail(GPT_ERR_ARG, "this epilogue needs its second input");
    if (b3) TRY(make_tmap3(&taux, e.aux, N, M, e.ldc, bt.n, bt.sc, 64, 32));
    else TRY(make_tmap(&taux, e.aux, N, M, e.ldc, 64, 32));
  } else {
    taux = tcm;
  }
  int km;
  if (p.splits > 1) km = tc::K_PARTIAL;
  else if (e.mode == EPI_STORE) km = tc::K_STORE;
  else if (e.mode == EPI_STORE_F32 || (e.mode == EPI_ACCUM_F32 && !e.beta)) km = tc::K_STORE_F32;
  else if (e.mode == EPI_ACCUM_F32) km = tc::K_REDUCE_F32;
  else if (e.mode == EPI_RELU2) km = tc::K_RELU2;
  else if (e.mode == EPI_DRELU2) km = tc::K_DRELU2;
  else if (e.mode == EPI_QKV) km = tc::K_QKV;
  else if (e.mode == EPI_AXPBY) km = tc::K_AXPBY;
  else km = tc::K_LOGITS;
  if (km == tc::K_QKV && BN != 256) return fail(GPT_ERR_ARG, "QKV epilogue needs 256-column tiles (N >= 256)");
  if (b3) {
    // batched products: their own kernel instances (the third tensor-map coordinate)
    if (km == tc::K_STORE_F32) TRY((gemm_tc_launch_k<BN, tc::K_STORE_F32, CG, 0, true>(ta, tb, tcm, taux, p, st)));
    else if (km == tc::K_AXPBY) TRY((gemm_tc_launch_k<BN, tc::K_AXPBY, CG, 0, true>(ta, tb, tcm, taux, p, st)));
    else TRY((gemm_tc_launch_k<BN, tc::K_STORE, CG, 0, true>(ta, tb, tcm, taux, p, st)));
    return GPT_OK;
  }
  if constexpr (BN == 192) {  // fp32 outputs only
    switch (km) {
      case tc::K_STORE_F32: TRY((gemm_tc_launch_k<BN, tc::K_STORE_F32, CG>(ta, tb, tcm, taux, p, st))); break;
      case tc::K_REDUCE_F32: TRY((gemm_tc_launch_k<BN, tc::K_REDUCE_F32, CG>(ta, tb, tcm, taux, p, st))); break;
      case tc::K_PARTIAL: TRY((gemm_tc_launch_k<BN, tc::K_PARTIAL, CG>(ta, tb, tcm, taux, p, st))); break;
      default: return fail(GPT_ERR_ARG, "192-column tiles take fp32-output epilogues only");
    }
  } else {
  switch (km) {
    case tc::K_STORE: TRY((gemm_tc_launch_k<BN, tc::K_STORE, CG>(ta, tb, tcm, taux, p, st))); break;
    case tc::K_STORE_F32: TRY((gemm_tc_launch_k<BN, tc::K_STORE_F32, CG>(ta, tb, tcm, taux, p, st))); break;
    case tc::K_REDUCE_F32: TRY((gemm_tc_launch_k<BN, tc::K_REDUCE_F32, CG>(ta, tb, tcm, taux, p, st))); break;
    case tc::K_PARTIAL: TRY((gemm_tc_launch_k<BN, tc::K_PARTIAL, CG>(ta, tb, tcm, taux, p, st))); break;
    case tc::K_RELU2: TRY((gemm_tc_launch_k<BN, tc::K_RELU2, CG>(ta, tb, tcm, taux, p, st))); break;
    case tc::K_DRELU2: TRY((gemm_tc_launch_k<BN, tc::K_DRELU2, CG>(ta, tb, tcm, taux, p, st))); break;
    case tc::K_QKV: TRY((gemm_tc_launch_k<BN, tc::K_QKV, CG>(ta, tb, tcm, taux, p, st))); break;
    case tc::K_AXPBY: TRY((gemm_tc_launch_k<BN, tc::K_AXPBY, CG>(ta, tb, tcm, taux, p, st))); break;
    default: TRY((gemm_tc_launch_k<BN, tc::K_LOGITS, CG>(ta, tb, tcm, taux, p, st))); break;
  }
  }
  if (p.splits > 1) {
    const long long total = (long long)M * N;
    int blocks = (int)((total + 255) / 256);
    if (blocks > 4 * device_sms()) blocks = 4 * device_sms();
    ++g_launches; launch_pdl(splitk_reduce_kernel<bf16>, blocks, 256, 0, st, partial, p.splits, M, N, e);
    LAUNCH_CHECK();
  }
  return GPT_OK;
}

// FP8 product: C = (*sa * *sb) * A_q B_q^T with e4m3 operands A_q [M, K] and
// B_q [N, K] (K-major, row pitches lda / ldb bytes), 256-column tiles, fp32 or
// bf16 output; CTA pairs when enabled.
template <int CG>
static int gemm_f8_launch(int M, int N, int K, const uint8_t* A, long long lda, const uint8_t* B, long long ldb,
                          GemmEpilogue e, unsigned* err, cudaStream_t st) {
  CUtensorMap ta, tb, tcm;
  {
    const uint64_t da[2] = {(uint64_t)K, (uint64_t)M}, sa[1] = {(uint64_t)lda};
    const uint32_t ba[2] = {128, tc::BM};
    TRY(make_tmap_gen(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, A, da, sa, ba));
    const uint64_t db[2] = {(uint64_t)K, (uint64_t)N}, sb[1] = {(uint64_t)ldb};
    const uint32_t bb[2] = {128, (uint32_t)(256 / CG)};
    TRY(make_tmap_gen(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, B, db, sb, bb));
  }
  tc::Params p;
  p.M = M; p.N = N; p.K = K; p.batch = 1;
  p.a_kmajor = 1; p.b_kmajor = 1;
  p.m_tiles = cdiv(M, CG * tc::BM);
  p.n_tiles = cdiv(N, 256);
  p.group_m = 1;
  p.kb_total = cdiv(K, 128);
  p.splits = 1; p.kb_per_split = p.kb_total;
  p.epi = e; p.partial = nullptr; p.err = err;
  if (e.mode == EPI_STORE_F32) {
    const uint64_t dims[2] = {(uint64_t)N, (uint64_t)M}, str[1] = {(uint64_t)e.ldc * 4};
    const uint32_t box[2] = {32, 32};
    TRY(make_tmap_gen(&tcm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, e.C, dims, str, box));
    return gemm_tc_launch_k<256, tc::K_STORE_F32, CG, 1>(ta, tb, tcm, tcm, p, st);
  }
  TRY(make_tmap(&tcm, e.C, N, M, e.ldc, 64, 32));
  return gemm_tc_launch_k<256, tc::K_STORE, CG, 1>(ta, tb, tcm, tcm, p, st);
}

// Choose split-K so a small-output, long-K product still fills the GPU.
// Share of the SMs' tile slots doing useful columns: tiles over whole waves,
// times the used fraction of the last column tile.  A tile of a CTA pair
// covers 256 rows and takes two SMs.
static double tile_efficiency(int M, int N, int BN, int splits, int cg = 1) {
  const long long tiles = (long long)cdiv(M, 128 * cg) * cdiv(N, BN) * splits;
  const long long units = device_sms() / cg;
  const double waves = (double)((tiles + units - 1) / units);
  return ((double)tiles / (waves * units)) * ((double)N / ((double)cdiv(N, BN) * BN));
}

// Split-K factor for a product with few output tiles (under 1.5 waves of SMs;
// larger products pay more for the fp32 partials than a fuller last wave
// returns): the one that fills whole waves best (tile_efficiency), keeping at
// least 8 k-blocks per split; on a tie the smaller factor.
static int pick_splits(int M, int N, int K, int BN, int cg = 1) {
  const int kb = cdiv(K, 64);
  const long long tiles = (long long)cdiv(M, 128 * cg) * cdiv(N, BN);
  const long long units = device_sms() / cg;
  if (tiles >= units + units / 2) return 1;
  int best = 1;
  double best_eff = tile_efficiency(M, N, BN, 1, cg);
  for (int s = 2; s <= 16 && kb / s >= 8; ++s) {
    const double e = tile_efficiency(M, N, BN, s, cg);
    if (e > best_eff + 1e-9) { best = s; best_eff = e; }
  }
  return best;
}

// ======================================================================== live timing
// Optional per-kernel-class timing with CUDA events recorded on the model's
// stream around each kernel (or small group of kernels) while enabled.
struct ProfRec {
  const char* cls;
  cudaEvent_t a, b;
  double flops, bytes;
  long long launches;
};
struct Prof {
  bool on = false;
  std::vector<ProfRec> recs;
  std::vector<cudaEvent_t> pool;
  size_t used = 0;
  cudaEvent_t get() {
    if (used == pool.size()) {
      cudaEvent_t e = nullptr;
      cudaEventCreate(&e);
      pool.push_back(e);
    }
    return pool[used++];
  }
};
struct ProfScope {
  Prof* p = nullptr;
  cudaStream_t st = nullptr;
  long idx = -1;
  long long l0 = 0;
  ProfScope(Prof* prof, cudaStream_t s, const char* cls, double flops, double bytes) : p(prof), st(s) {
    if (!p || !p->on) return;
    ProfRec r;
    r.cls = cls; r.a = p->get(); r.b = p->get(); r.flops = flops; r.bytes = bytes; r.launches = 0;
    l0 = g_launches.load();
    cudaEventRecord(r.a, st);
    p->recs.push_back(r);
    idx = (long)p->recs.size() - 1;
  }
  ~ProfScope() {
    if (idx < 0) return;
    ProfRec& r = p->recs[idx];
    r.launches = g_launches.load() - l0;
    cudaEventRecord(r.b, st);
  }
};

struct GemmCtx {
  bool bf16;
  float* splitk;          // fp32 scratch for split-K partials
  long long splitk_elems;
  unsigned* err;
  cudaStream_t st;
  Prof* prof;
};

static int gemm(const GemmCtx& g, int M, int N, int K, GemmOperand A, GemmOperand B, GemmEpilogue e,
                bool allow_split = false, const char* label = "gemm") {
  if (M <= 0 || N <= 0 || K <= 0) return GPT_OK;
  ProfScope ps(g.prof, g.st, label, 2.0 * M * N * K, 0.0);
  if (!g.bf16) {
    gemm_simt<float, float>(M, N, K, A, B, e, g.st);
    LAUNCH_CHECK();
    return GPT_OK;
  }
  const bool f32out = e.mode == EPI_ACCUM_F32 || e.mode == EPI_STORE_F32;
  const bool split_ok = allow_split && f32out;
  auto splits_for = [&](int bn, int cg = 1) {
    if (!split_ok) return 1;
    int s = pick_splits(M, N, K, bn, cg);
    while (s > 1 && (long long)s * M * N > g.splitk_elems) --s;
    return s;
  };
  // 256-column tiles on CTA pairs (256 x 256 output tiles) whenever N >= 256,
  // except for the two epilogues that bound their kernels (the logits'
  // statistics and the ReLU^2 backward's activation stream), which measured
  // faster on one-SM tiles (B200: LM-head logits 2.55 vs 2.79 ms, ReLU^2
  // backward 2.04 vs 2.17 ms per GPT-2-small step)
  if (N >= 256 && gemm_pairs_enabled() && e.mode != EPI_LOGITS && e.mode != EPI_DRELU2)
    return gemm_tc_launch<256, 2>(M, N, K, A, B, e, splits_for(256, 2), g.splitk, g.err, g.st);
  // one-CTA tiles: 256 wide (128 below 256 columns); fp32 outputs may take 192
  // when that fills the last wave of SMs better (N = 768: 4 x 192 instead of 3 x 256)
  int BN = (N >= 256) ? 256 : 128;
  int splits = splits_for(BN);
  if (f32out && N >= 256 && tile_efficiency(M, N, 192, splits_for(192)) > tile_efficiency(M, N, 256, splits) + 0.03) {
    BN = 192;
    splits = splits_for(192);
  }
  if (BN == 256) return gemm_tc_launch<256>(M, N, K, A, B, e, splits, g.splitk, g.err, g.st);
  if (BN == 192) return gemm_tc_launch<192>(M, N, K, A, B, e, splits, g.splitk, g.err, g.st);
  return gemm_tc_launch<128>(M, N, K, A, B, e, splits, g.splitk, g.err, g.st);
}

static GemmOperand op_k(const void* p, long long ld) { return GemmOperand{p, ld, 1}; }
static GemmOperand op_mn(const void* p, long long ld) { return GemmOperand{p, ld, 0}; }
static GemmEpilogue epi(int mode, void* C, long long ldc, int beta = 0, void* C2 = nullptr,
                        const void* aux = nullptr, float alpha = 1.f) {
  GemmEpilogue e;
  e.mode = mode; e.C = C; e.ldc = ldc; e.C2 = C2; e.aux = aux; e.alpha = alpha; e.beta = beta;
  e.softcap = 0.f; e.stats = nullptr; e.targets = nullptr; e.ztgt = nullptr;
  e.rope = nullptr; e.rstd_q = e.rstd_k = nullptr; e.hv = nullptr; e.rv = nullptr;
  e.scale_a = e.scale_b = nullptr;
  e.aux_scale = 0.f;
  e.T = e.H = e.qk_norm = 0; e.eps = 0.f;
  return e;
}

// ======================================================================== arena plan
struct Carver {
  size_t off = 0;
  size_t take(size_t bytes) {
    off = (off + 255) & ~size_t(255);
    size_t r = off;
    off += bytes;
    return r;
  }
};

struct DenseTensor {
  std::string name;
  long long off;  // element offset in the flat dense buffers
  long long rows, cols;
};

struct LayerActs {
  size_t u, rstd1, qkv, rstd_q, rstd_k, o, lse, u2, rstd2, g;
};

struct Plan {
  // dense flat buffers
  std::vector<DenseTensor> dense;
  long long dense_n = 0, e_end = 0, h_end = 0;
  size_t P, G, M, V, Plp;
  size_t hx = 0, hv = 0, hx_state = 0, hv_state = 0;
  size_t h3 = 0, rows_3 = 0, s3g = 0, p3 = 0, vb = 0, gv16 = 0;  // frozen trigram statistics
  long long blocks_begin = 0;  // element offset of h0.wqkv: the block matrices start here
  size_t x, emb_rstd, xf, rstd_f, tok_copy, rows_x, rows_v;
  std::vector<LayerActs> layers;
  size_t dx, dx_lp, du, dqkv, da, dout, Dattn, gv, dxf, pending;
  size_t logits, dz, ce_stats, ce_ztgt, tok_loss, ce_scale, ce_count, loss_scratch;
  size_t sort_keys_a, sort_keys_b, sort_vals_a, sort_vals_b, sort_counts, part_head, part_tail;
  size_t splitk; long long splitk_elems;
  size_t norm_part, clip_coef, grad_norm, rope_cs, rope_turns, err;
  // Muon (matrix_optimizer == GPT_MATRIX_MUON): the block matrices in three
  // same-shape groups and one scratch sized for the largest group
  MuonGroup muon_groups[3];
  int n_muon_groups = 0;
  size_t mu_x, mu_xn, mu_abf, mu_bm, mu_part;
  int chunk;
  size_t total;
};

static bool cfg_bf16(const gpt_config& c) { return c.dtype == GPT_DTYPE_BF16; }

static int validate(const gpt_config* c) {
  if (!c) return fail(GPT_ERR_ARG, "null config");
  if (c->n_layer < 1 || c->d_model < 1 || c->n_head < 1 || c->head_dim < 2 || c->d_ff < 1 ||
      c->vocab < 2 || c->seq_len < 1 || c->micro_batch < 1 || c->grad_accum < 1)
    return fail(GPT_ERR_CONFIG, "non-positive dimension in config");
  if (c->dtype != GPT_DTYPE_F32 && c->dtype != GPT_DTYPE_BF16)
    return fail(GPT_ERR_CONFIG, "dtype must be GPT_DTYPE_F32 or GPT_DTYPE_BF16");
  if (c->d_model != c->n_head * c->head_dim)
    return fail(GPT_ERR_CONFIG, "d_model (%d) != n_head * head_dim (%d)", c->d_model, c->n_head * c->head_dim);
  if (c->n_kv_head != 0 && c->n_kv_head != c->n_head)
    return fail(GPT_ERR_CONFIG, "grouped KV heads are not supported (n_kv_head must equal n_head)");
  if (c->head_dim % 2 || c->head_dim > 128) return fail(GPT_ERR_CONFIG, "head_dim must be even and <= 128");
  if (c->d_model % 4 || c->d_model > 2048 || c->d_ff % 4)
    return fail(GPT_ERR_CONFIG, "d_model must be a multiple of 4 and <= 2048; d_ff a multiple of 4");
  if (cfg_bf16(*c)) {
    if (c->head_dim != 128) return fail(GPT_ERR_CONFIG, "bf16 mode needs head_dim == 128");
    if (c->d_model % 64 || c->d_ff % 64 || c->vocab % 64)
      return fail(GPT_ERR_CONFIG, "bf16 mode needs d_model, d_ff, vocab multiples of 64");
    if (c->seq_len % 4) return fail(GPT_ERR_CONFIG, "bf16 mode needs seq_len a multiple of 4");
  }
  if (c->x0_rows < 0 || c->v_rows < 0 || c->x0_rows > 0x7fffffffLL || c->v_rows > 0x7fffffffLL)
    return fail(GPT_ERR_CONFIG, "table rows out of range");
  const long long N = (long long)c->micro_batch * c->seq_len;
  if (N > (1LL << 24)) return fail(GPT_ERR_CONFIG, "too many tokens per micro-batch");
  if (c->norm_eps <= 0.f || c->rope_base <= 1.f) return fail(GPT_ERR_CONFIG, "bad norm_eps or rope_base");
  if (c->tri_rows < 0 || c->tri_rows > 0x7fffffffLL) return fail(GPT_ERR_CONFIG, "tri_rows out of range");
  if (c->tri_rows && (c->tri_width < 4 || c->tri_width > 1024 || c->tri_width % (cfg_bf16(*c) ? 64 : 4)))
    return fail(GPT_ERR_CONFIG, "tri_width must be in [4, 1024], a multiple of 64 in bf16 mode (4 in fp32 mode)");
  if (c->matrix_optimizer != GPT_MATRIX_ADAMW && c->matrix_optimizer != GPT_MATRIX_MUON)
    return fail(GPT_ERR_CONFIG, "matrix_optimizer must be GPT_MATRIX_ADAMW or GPT_MATRIX_MUON");
  if (c->matrix_optimizer == GPT_MATRIX_MUON) {
    if (!cfg_bf16(*c)) return fail(GPT_ERR_CONFIG, "Muon runs in bf16 mode only");
    if (!(c->muon_momentum >= 0.f && c->muon_momentum < 1.f) || c->muon_ns_steps < 0 || c->muon_ns_steps > 64)
      return fail(GPT_ERR_CONFIG, "Muon needs 0 <= muon_momentum < 1 and 0 <= muon_ns_steps <= 64");
  }
  return GPT_OK;
}

static void make_plan(const gpt_config& c, Plan& p) {
  const bool b16 = cfg_bf16(c);
  const size_t es = b16 ? 2 : 4;  // activation element size
  const long long N = (long long)c.micro_batch * c.seq_len;
  const long long d = c.d_model, a = (long long)c.n_head * c.head_dim, F = c.d_ff, V = c.vocab;
  const long long BH = (long long)c.micro_batch * c.n_head;
  // ---- dense flat layout: [wte][lm_head][layers...], each padded to 64 elements
  long long off = 0;
  auto add = [&](const std::string& nm, long long r, long long k) {
    p.dense.push_back({nm, off, r, k});
    off += ((r * k + 63) / 64) * 64;
  };
  add("wte", V, d);
  p.e_end = off;
  if (!c.tie_embeddings) add("lm_head", V, d);
  p.h_end = off;
  if (c.tri_rows) add("vproj", a, c.tri_width);   // matrix learning rate (past h_end)
  p.blocks_begin = off;
  for (int l = 0; l < c.n_layer; ++l) {
    add("h" + std::to_string(l) + ".wqkv", 3 * a, d);
    add("h" + std::to_string(l) + ".wo", d, a);
    add("h" + std::to_string(l) + ".w1", F, d);
    add("h" + std::to_string(l) + ".w2", d, F);
  }
  p.dense_n = off;
  Carver cv;
  p.P = cv.take(off * 4);
  p.G = cv.take(off * 4);
  p.M = cv.take(off * 4);
  p.V = cv.take(off * 4);
  p.Plp = b16 ? cv.take(off * 2) : 0;
  const size_t tes = b16 ? 2 : 4;
  if (c.x0_rows) { p.hx = cv.take(c.x0_rows * d * tes); p.hx_state = cv.take(c.x0_rows * 4); }
  if (c.v_rows) { p.hv = cv.take(c.v_rows * a * tes); p.hv_state = cv.take(c.v_rows * 4); }
  if (c.tri_rows) {
    p.h3 = cv.take(c.tri_rows * c.tri_width * tes);
    p.rows_3 = cv.take(N * 4);
    p.s3g = cv.take(N * c.tri_width * es);
    p.p3 = cv.take(N * a * 4);
    p.vb = cv.take(N * a * es);
    p.gv16 = b16 ? cv.take(N * a * 2) : 0;
  }
  // ---- activations
  p.x = cv.take(N * d * 4);
  p.emb_rstd = cv.take(N * 4);
  p.tok_copy = cv.take(N * 4);
  p.rows_x = cv.take(N * 4);
  p.rows_v = cv.take(N * 4);
  p.layers.resize(c.n_layer);
  for (int l = 0; l < c.n_layer; ++l) {
    LayerActs& L = p.layers[l];
    L.u = cv.take(N * d * es);
    L.rstd1 = cv.take(N * 4);
    L.qkv = cv.take(N * 3 * a * es);
    L.rstd_q = cv.take(N * c.n_head * 4);
    L.rstd_k = cv.take(N * c.n_head * 4);
    L.o = cv.take(N * a * es);
    L.lse = cv.take(BH * c.seq_len * 4);
    L.u2 = cv.take(N * d * es);
    L.rstd2 = cv.take(N * 4);
    L.g = cv.take(N * F * es);
  }
  p.xf = cv.take(N * d * es);
  p.rstd_f = cv.take(N * 4);
  // ---- backward work
  p.dx = cv.take(N * d * 4);
  p.dx_lp = cv.take(N * d * es);
  p.du = cv.take(N * d * 4);
  p.dqkv = cv.take(N * 3 * a * es);
  p.da = cv.take(N * F * es);
  p.dout = cv.take(N * a * es);
  p.Dattn = cv.take(BH * c.seq_len * 4);
  p.gv = (c.v_rows || c.tri_rows) ? cv.take(N * a * 4) : 0;
  p.dxf = cv.take(N * d * 4);
  p.pending = cv.take(V * d * 4);
  // ---- LM head chunk
  long long chunk = c.lm_chunk_rows > 0 ? c.lm_chunk_rows : 8192;
  if (chunk > N) chunk = N;
  p.chunk = (int)chunk;
  // fp32 mode materialises fp32 logits; bf16 mode writes the tile-local
  // softmax numerators straight into dz and rescales them in place
  p.logits = b16 ? 0 : cv.take(chunk * V * 4);
  p.dz = cv.take(chunk * V * es);
  p.ce_stats = cv.take(chunk * ((V + 63) / 64) * 8);  // (max, sum) per half tile
  p.ce_ztgt = cv.take(chunk * 4);
  p.tok_loss = cv.take(N * 4);
  p.ce_scale = cv.take(4);
  p.ce_count = cv.take(4);
  p.loss_scratch = cv.take(4);
  // ---- bucketing workspace (positions by row / by token)
  const long long nchunks = (N + CHUNK - 1) / CHUNK;
  p.sort_keys_a = cv.take(N * 4);
  p.sort_keys_b = cv.take(N * 4);
  p.sort_vals_a = cv.take(N * 4);
  p.sort_vals_b = cv.take(N * 4);
  p.sort_counts = cv.take(256 * radix_blocks(N) * 4);
  p.part_head = cv.take(nchunks * (d > a ? d : a) * 4);
  p.part_tail = cv.take(nchunks * (d > a ? d : a) * 4);
  // ---- split-K partials: the largest weight gradient x 8 splits
  long long mx = 3 * a * d;
  if (F * d > mx) mx = F * d;
  p.splitk_elems = b16 ? 8 * mx : 0;
  p.splitk = b16 ? cv.take(p.splitk_elems * 4) : 0;
  p.norm_part = cv.take(NORM_BLOCKS * 8);
  p.clip_coef = cv.take(4);
  p.grad_norm = cv.take(4);
  p.rope_cs = cv.take((long long)c.seq_len * c.head_dim * 4);
  p.rope_turns = cv.take((long long)c.head_dim / 2 * 8);
  p.err = cv.take(16);
  if (c.matrix_optimizer == GPT_MATRIX_MUON) {
    // groups: [q, k, v, proj] x layers ([a, d] each; a == d), w1 [F, d] x layers, w2 [d, F] x layers
    int i0 = 0;
    while (p.dense[i0].name != "h0.wqkv") ++i0;
    const long long o0 = p.dense[i0].off;
    const long long lstride = c.n_layer > 1 ? p.dense[i0 + 4].off - o0 : 0;
    p.muon_groups[0] = MuonGroup{o0, lstride, a * d, 4, 4 * c.n_layer, (int)a, (int)d};
    p.muon_groups[1] = MuonGroup{o0 + 4 * a * d, lstride, 0, 1, c.n_layer, (int)F, (int)d};
    p.muon_groups[2] = MuonGroup{o0 + 4 * a * d + F * d, lstride, 0, 1, c.n_layer, (int)d, (int)F};
    p.n_muon_groups = 3;
    long long xn = 0, rr = 0, nm = 0;
    for (int gi = 0; gi < 3; ++gi) {
      const MuonGroup& g = p.muon_groups[gi];
      const long long R = g.rows < g.cols ? g.rows : g.cols;
      xn = std::max(xn, (long long)g.nmat * g.rows * g.cols);
      rr = std::max(rr, (long long)g.nmat * R * R);
      nm = std::max(nm, (long long)g.nmat);
    }
    p.mu_x = cv.take(xn * 2); p.mu_xn = cv.take(xn * 2);
    p.mu_abf = cv.take(rr * 2); p.mu_bm = cv.take(rr * 2);
    p.mu_part = cv.take(nm * MUON_BATCH_BLOCKS * 4);
  }
  p.total = cv.take(0) + 256;
}

// ======================================================================== model
struct gpt_model {
  gpt_config cfg;
  Plan plan;
  uint8_t* base;
  size_t bytes;
  cudaStream_t st;
  int micro = 0;
  long long step_t = 0;
  bool have_fwd = false;
  bool defer_tables = false;  // gpt_set_table_exchange: backward leaves the table gradients for the caller
  Prof prof;
  template <typename T> T* at(size_t off) const { return reinterpret_cast<T*>(base + off); }
  unsigned* err() const { return at<unsigned>(plan.err); }
};

static const DenseTensor* find_dense(const gpt_model* m, const std::string& name) {
  for (const auto& t : m->plan.dense)
    if (t.name == name) return &t;
  return nullptr;
}

extern "C" int gpt_default_config(gpt_config* c) {
  if (!c) return fail(GPT_ERR_ARG, "null config");
  memset(c, 0, sizeof(*c));
  c->n_layer = 2; c->d_model = 128; c->n_head = 4; c->head_dim = 32; c->n_kv_head = 4;
  c->d_ff = 512; c->vocab = 512; c->seq_len = 64; c->micro_batch = 4; c->grad_accum = 1;
  c->dtype = GPT_DTYPE_F32; c->tie_embeddings = 1; c->qk_norm = 1;
  c->rope_base = 10000.f; c->norm_eps = 1.1920929e-07f; c->softcap = 0.f; c->init_std = 0.02f;
  c->adam_b1 = 0.8f; c->adam_b2 = 0.95f; c->adam_eps = 1e-10f; c->weight_decay = 0.f;
  c->grad_clip = 0.f;
  c->lr_mult_embed = c->lr_mult_head = c->lr_mult_matrix = c->lr_mult_table = 1.f;
  c->x0_rows = 0; c->v_rows = 0; c->table_beta = 0.95f; c->table_eps = 1e-10f;
  c->hash_p1 = 2654435761ull; c->hash_p2 = 2246822519ull;
  c->lm_chunk_rows = 0;
  c->matrix_optimizer = GPT_MATRIX_ADAMW; c->muon_momentum = 0.95f; c->muon_ns_steps = 5; c->muon_nesterov = 1;
  c->tri_rows = 0; c->tri_width = 64; c->hash_p3 = 3266489917ull;
  return GPT_OK;
}

extern "C" int gpt_workspace_bytes(const gpt_config* cfg, size_t* bytes) {
  if (!bytes) return fail(GPT_ERR_ARG, "null bytes");
  TRY(validate(cfg));
  Plan p;
  make_plan(*cfg, p);
  *bytes = p.total;
  return GPT_OK;
}

extern "C" int gpt_flops_per_token(const gpt_config* c, long long* flops, long long* flops_causal) {
  TRY(validate(c));
  const long long d = c->d_model, a = (long long)c->n_head * c->head_dim, F = c->d_ff, V = c->vocab;
  const long long mat = (long long)c->n_layer * (3 * a * d + d * a + F * d + d * F) + V * d;
  const long long attn = 12LL * c->n_layer * c->n_head * c->head_dim * c->seq_len;
  if (flops) *flops = 6 * mat + attn;
  if (flops_causal) *flops_causal = 6 * mat + attn / 2;
  return GPT_OK;
}

static int grid_for(long long n, int per_block) {
  long long b = (n + per_block - 1) / per_block;
  return (int)(b < 1 ? 1 : b);
}

static int refresh_lp(gpt_model* m) {
  if (!cfg_bf16(m->cfg)) return GPT_OK;
  const Plan& p = m->plan;
  ++g_launches; launch_pdl(to_bf16_kernel, 4 * device_sms(), 256, 0, m->st, m->at<float>(p.P), m->at<bf16>(p.Plp), p.dense_n);
  LAUNCH_CHECK();
  return GPT_OK;
}

extern "C" int gpt_create(const gpt_config* cfg, unsigned long long seed, void* arena, size_t arena_bytes,
                          void* cuda_stream, gpt_model** out) {
  if (!out || !arena) return fail(GPT_ERR_ARG, "null arena or out");
  *out = nullptr;
  TRY(validate(cfg));
  if (reinterpret_cast<uintptr_t>(arena) & 255) return fail(GPT_ERR_ARG, "arena not 256-byte aligned");
  gpt_model* m = new gpt_model();
  m->cfg = *cfg;
  make_plan(m->cfg, m->plan);
  if (arena_bytes < m->plan.total) {
    size_t need = m->plan.total;
    delete m;
    return fail(GPT_ERR_WORKSPACE, "arena too small: %zu < %zu bytes", arena_bytes, need);
  }
  if (m->plan.n_muon_groups) {
    // the block matrices must sit at the regular offsets the Muon groups assume
    const Plan& pl = m->plan;
    for (int l = 0; l < cfg->n_layer; ++l) {
      const long long L = l * pl.muon_groups[0].layer_stride;
      const std::string pre = "h" + std::to_string(l) + ".";
      if (find_dense(m, pre + "wqkv")->off != pl.muon_groups[0].base + L ||
          find_dense(m, pre + "wo")->off != pl.muon_groups[0].base + L + 3 * pl.muon_groups[0].inner_stride ||
          find_dense(m, pre + "w1")->off != pl.muon_groups[1].base + L ||
          find_dense(m, pre + "w2")->off != pl.muon_groups[2].base + L) {
        delete m;
        return fail(GPT_ERR_CONFIG, "Muon groups: unexpected parameter layout");
      }
    }
  }
  m->base = static_cast<uint8_t*>(arena);
  m->bytes = arena_bytes;
  m->st = static_cast<cudaStream_t>(cuda_stream);
  const Plan& p = m->plan;
  const gpt_config& c = m->cfg;
  cudaError_t e = cudaMemsetAsync(arena, 0, p.total, m->st);
  if (e != cudaSuccess) { delete m; return fail(GPT_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e)); }
  const int blocks = 8 * device_sms();
  uint32_t stream_id = 1;
  for (const auto& t : p.dense) {
    ++g_launches; init_normal_kernel<float><<<blocks, 256, 0, m->st>>>(m->at<float>(p.P) + t.off, t.rows * t.cols,
                                                        c.init_std, seed, stream_id++);
  }
  const long long a = (long long)c.n_head * c.head_dim;
  if (c.x0_rows) {
    if (cfg_bf16(c)) {
      ++g_launches; init_normal_kernel<bf16><<<blocks, 256, 0, m->st>>>(m->at<bf16>(p.hx), c.x0_rows * c.d_model, c.init_std, seed, 0x10000u);
    } else {
      ++g_launches; init_normal_kernel<float><<<blocks, 256, 0, m->st>>>(m->at<float>(p.hx), c.x0_rows * c.d_model, c.init_std, seed, 0x10000u);
    }
  }
  if (c.v_rows) {
    if (cfg_bf16(c)) {
      ++g_launches; init_normal_kernel<bf16><<<blocks, 256, 0, m->st>>>(m->at<bf16>(p.hv), c.v_rows * a, c.init_std, seed, 0x10001u);
    } else {
      ++g_launches; init_normal_kernel<float><<<blocks, 256, 0, m->st>>>(m->at<float>(p.hv), c.v_rows * a, c.init_std, seed, 0x10001u);
    }
  }
  ++g_launches; rope_table_kernel<<<grid_for((long long)c.seq_len * c.head_dim / 2, 256), 256, 0, m->st>>>(
      m->at<float>(p.rope_cs), m->at<float2>(p.rope_turns), c.seq_len, c.head_dim, (double)c.rope_base);
  e = cudaGetLastError();
  if (e != cudaSuccess) { delete m; return fail(GPT_ERR_CUDA, "init launch: %s", cudaGetErrorString(e)); }
  int s = refresh_lp(m);
  if (s != GPT_OK) { delete m; return s; }
  *out = m;
  return GPT_OK;
}

extern "C" int gpt_destroy(gpt_model* m) {
  if (!m) return fail(GPT_ERR_ARG, "null model");
  cudaStreamSynchronize(m->st);
  for (cudaEvent_t e : m->prof.pool) cudaEventDestroy(e);
  delete m;
  return GPT_OK;
}

extern "C" int gpt_set_stream(gpt_model* m, void* s) {
  if (!m) return fail(GPT_ERR_ARG, "null model");
  m->st = static_cast<cudaStream_t>(s);
  return GPT_OK;
}

extern "C" int gpt_num_params(const gpt_model* m, long long* dense, long long* table) {
  if (!m) return fail(GPT_ERR_ARG, "null model");
  long long dn = 0;
  for (const auto& t : m->plan.dense) dn += t.rows * t.cols;
  if (dense) *dense = dn;
  if (table) *table = m->cfg.x0_rows * m->cfg.d_model + m->cfg.v_rows * (long long)m->cfg.n_head * m->cfg.head_dim;
  return GPT_OK;
}

extern "C" int gpt_params_changed(gpt_model* m) {
  if (!m) return fail(GPT_ERR_ARG, "null model");
  return refresh_lp(m);
}

extern "C" int gpt_sync_status(gpt_model* m) {
  if (!m) return fail(GPT_ERR_ARG, "null model");
  CUDA_TRY(cudaStreamSynchronize(m->st));
  unsigned w = 0;
  CUDA_TRY(cudaMemcpy(&w, m->err(), 4, cudaMemcpyDeviceToHost));
  if (w) CUDA_TRY(cudaMemset(m->err(), 0, 4));
  if (w & GPT_EBIT_TIMEOUT) return fail(GPT_ERR_TIMEOUT, "a kernel's bounded wait gave up");
  if (w & GPT_EBIT_INPUT) return fail(GPT_ERR_INPUT, "token, target or row id out of range");
  if (w & GPT_EBIT_NONFINITE) return fail(GPT_ERR_NONFINITE, "non-finite loss or gradient norm");
  return GPT_OK;
}

extern "C" int gpt_tensor(gpt_model* m, const char* name, int kind, void** ptr, int* dtype,
                          long long shape[4]) {
  if (!m || !name || !ptr) return fail(GPT_ERR_ARG, "null argument");
  const Plan& p = m->plan;
  const gpt_config& c = m->cfg;
  const bool b16 = cfg_bf16(c);
  long long sh[4] = {1, 1, 1, 1};
  int dt = GPT_DTYPE_F32;
  void* ptr_out = nullptr;
  const std::string nm(name);
  const long long N = (long long)c.micro_batch * c.seq_len;
  const long long a = (long long)c.n_head * c.head_dim;
  if (kind == GPT_KIND_ACT) {
    if (nm == "per_token_loss") { ptr_out = m->at<float>(p.tok_loss); sh[0] = c.micro_batch; sh[1] = c.seq_len; }
    else if (nm == "rows_x" && c.x0_rows) { ptr_out = m->at<int32_t>(p.rows_x); dt = GPT_DTYPE_I32; sh[0] = c.micro_batch; sh[1] = c.seq_len; }
    else if (nm == "rows_v" && c.v_rows) { ptr_out = m->at<int32_t>(p.rows_v); dt = GPT_DTYPE_I32; sh[0] = c.micro_batch; sh[1] = c.seq_len; }
    else if (nm == "rows_3" && c.tri_rows) { ptr_out = m->at<int32_t>(p.rows_3); dt = GPT_DTYPE_I32; sh[0] = c.micro_batch; sh[1] = c.seq_len; }
    else if (nm == "grad_norm") { ptr_out = m->at<float>(p.grad_norm); }
    else if (nm == "table_grad_x" && c.x0_rows) { ptr_out = m->at<float>(p.dx); sh[0] = N; sh[1] = c.d_model; }
    else if (nm == "table_grad_v" && c.v_rows) { ptr_out = m->at<float>(p.gv); sh[0] = N; sh[1] = a; }
    else return fail(GPT_ERR_ARG, "unknown activation '%s'", name);
  } else if (nm == "*") {
    // the whole flat dense buffer of this kind (tensors padded to 64 elements)
    sh[0] = p.dense_n;
    switch (kind) {
      case GPT_KIND_PARAM: ptr_out = m->at<float>(p.P); break;
      case GPT_KIND_GRAD: ptr_out = m->at<float>(p.G); break;
      case GPT_KIND_ADAM_M: ptr_out = m->at<float>(p.M); break;
      case GPT_KIND_ADAM_V: ptr_out = m->at<float>(p.V); break;
      default: return fail(GPT_ERR_ARG, "flat buffer '*' has kinds PARAM, GRAD, ADAM_M, ADAM_V");
    }
  } else if (nm == "h3") {
    if (!c.tri_rows) return fail(GPT_ERR_ARG, "trigram table absent");
    if (kind != GPT_KIND_PARAM) return fail(GPT_ERR_ARG, "the trigram table has kind PARAM only");
    ptr_out = m->base + p.h3; dt = b16 ? GPT_DTYPE_BF16 : GPT_DTYPE_F32;
    sh[0] = c.tri_rows; sh[1] = c.tri_width;
  } else if (nm == "hx" || nm == "hv") {
    const bool isx = nm == "hx";
    const long long rows = isx ? c.x0_rows : c.v_rows;
    if (!rows) return fail(GPT_ERR_ARG, "table '%s' absent", name);
    sh[0] = rows; sh[1] = isx ? c.d_model : a;
    if (kind == GPT_KIND_PARAM) { ptr_out = m->base + (isx ? p.hx : p.hv); dt = b16 ? GPT_DTYPE_BF16 : GPT_DTYPE_F32; }
    else if (kind == GPT_KIND_ROW_STATE) { ptr_out = m->base + (isx ? p.hx_state : p.hv_state); sh[1] = 1; }
    else return fail(GPT_ERR_ARG, "tables have kinds PARAM and ROW_STATE only");
  } else {
    const DenseTensor* t = find_dense(m, nm);
    if (!t) return fail(GPT_ERR_ARG, "unknown tensor '%s'", name);
    sh[0] = t->rows; sh[1] = t->cols;
    switch (kind) {
      case GPT_KIND_PARAM: ptr_out = m->at<float>(p.P) + t->off; break;
      case GPT_KIND_GRAD: ptr_out = m->at<float>(p.G) + t->off; break;
      case GPT_KIND_ADAM_M: ptr_out = m->at<float>(p.M) + t->off; break;
      case GPT_KIND_ADAM_V: ptr_out = m->at<float>(p.V) + t->off; break;
      case GPT_KIND_PARAM_LP:
        if (!b16) return fail(GPT_ERR_ARG, "no bf16 copy in fp32 mode");
        ptr_out = m->at<bf16>(p.Plp) + t->off; dt = GPT_DTYPE_BF16; break;
      default: return fail(GPT_ERR_ARG, "bad kind %d for '%s'", kind, name);
    }
  }
  *ptr = ptr_out;
  if (dtype) *dtype = dt;
  if (shape) for (int i = 0; i < 4; ++i) shape[i] = sh[i];
  return GPT_OK;
}

// ======================================================================== bucketing
struct SortWs {
  uint32_t *ka, *kb, *counts;
  int32_t *va, *vb;
  float *part_head, *part_tail;  // [n / CHUNK, d] partial sums of runs that cross chunk edges
};

static SortWs sort_ws(const gpt_model* m) {
  const Plan& p = m->plan;
  SortWs w;
  w.ka = m->at<uint32_t>(p.sort_keys_a); w.kb = m->at<uint32_t>(p.sort_keys_b);
  w.va = m->at<int32_t>(p.sort_vals_a); w.vb = m->at<int32_t>(p.sort_vals_b);
  w.counts = m->at<uint32_t>(p.sort_counts);
  w.part_head = m->at<float>(p.part_head); w.part_tail = m->at<float>(p.part_tail);
  return w;
}

// Stable sort of the positions 0..n-1 by key (row id in [0, key_range); an
// invalid id sorts as key_range with position -1).  Leaves the sorted keys in
// *keys_out and the positions in *perm_out; with uniq_out / n_uniq_out given,
// also the distinct valid keys in ascending order and their number.
static int bucket_by_key(const SortWs& w, const int32_t* keys, int n, long long key_range,
                         const uint32_t** keys_out, const int32_t** perm_out, int32_t* uniq_out,
                         int* n_uniq_out, unsigned* err, cudaStream_t st) {
  int bits = 1;
  while (bits < 32 && (1LL << bits) <= key_range) ++bits;  // the value key_range must fit
  const int passes = (bits + 7) / 8;
  const int items = radix_items(n);
  const long long nblk = radix_blocks(n);
  const int scanned = nblk > RADIX_FUSED_MAX_BLOCKS;
  const uint32_t* kin = nullptr;
  const int32_t* vin = nullptr;
  uint32_t* kout = w.ka;
  int32_t* vout = w.va;
  for (int ps = 0; ps < passes; ++ps) {
    const int32_t* raw = ps == 0 ? keys : nullptr;
    ++g_launches; launch_pdl(radix_hist_kernel, (unsigned)nblk, RADIX_THREADS, 0, st, kin, raw, n, key_range, items, 8 * ps, w.counts);
    if (scanned) { ++g_launches; launch_pdl(radix_offsets_kernel, 1, 1024, 0, st, w.counts, (int)nblk); }
    ++g_launches; launch_pdl(radix_scatter_kernel, (unsigned)nblk, RADIX_THREADS, 0, st, kin, vin, raw, n, key_range, items, 8 * ps,
                                                                  w.counts, scanned, kout, vout, err);
    LAUNCH_CHECK();
    kin = kout;
    vin = vout;
    kout = (kout == w.ka) ? w.kb : w.ka;
    vout = (vout == w.va) ? w.vb : w.va;
  }
  if (uniq_out || n_uniq_out) {
    ++g_launches; launch_pdl(unique_keys_kernel, 1, 1024, 0, st, kin, n, key_range, uniq_out, n_uniq_out);
    LAUNCH_CHECK();
  }
  *keys_out = kin;
  *perm_out = vin;
  return GPT_OK;
}

// Dynamic shared memory above the default 48 KB needs the kernel's opt-in.
template <typename K>
static int allow_smem(K* kernel, size_t bytes) {
  if (bytes > 48 * 1024)
    CUDA_TRY(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes));
  return GPT_OK;
}

template <typename tab_t, int MAXT, bool STAGE>
static int launch_table_chunk(tab_t* table, float* state, int d, const float* grad, const uint32_t* skeys,
                              const int32_t* perm, int n, long long n_rows, const SortWs& w, float lr, float beta,
                              float eps, int nt, long long nchunks, cudaStream_t st) {
  static bool attr = false;
  if (!attr) {
    CUDA_TRY(cudaFuncSetAttribute(table_chunk_kernel<tab_t, MAXT, STAGE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)table_chunk_smem<tab_t>(MAXT, STAGE)));
    // all of the unified L1 / shared storage as shared memory: occupancy is set by it
    CUDA_TRY(cudaFuncSetAttribute(table_chunk_kernel<tab_t, MAXT, STAGE>,
                                  cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared));
    attr = true;
  }
  ++g_launches;
  launch_pdl(table_chunk_kernel<tab_t, MAXT, STAGE>, (unsigned)nchunks, nt, table_chunk_smem<tab_t>(nt, STAGE), st,
      table, state, d, grad, skeys, perm, n, n_rows, w.part_head, w.part_tail, lr, beta, eps);
  return GPT_OK;
}

template <typename tab_t>
static int table_update(const SortWs& w, tab_t* table, float* state, long long n_rows, int d,
                        const int32_t* rows, const float* grad, int n, float lr, float beta, float eps,
                        int32_t* uniq_out, int* n_uniq_out, unsigned* err, cudaStream_t st) {
  const uint32_t* skeys;
  const int32_t* perm;
  TRY(bucket_by_key(w, rows, n, n_rows, &skeys, &perm, uniq_out, n_uniq_out, err, st));
  const long long nchunks = (n + CHUNK - 1) / CHUNK;
  const int chunk_threads = (d / 4 + 31) / 32 * 32;  // one float4 column group a thread (d <= 2048)
  if (chunk_threads <= 256) {
    TRY((launch_table_chunk<tab_t, 256, true>(table, state, d, grad, skeys, perm, n, n_rows, w, lr, beta, eps,
                                              chunk_threads, nchunks, st)));
  } else {
    // rows wider than 1024: fp32 table values no longer fit beside the gradients
    constexpr bool stage = sizeof(tab_t) == 2;
    TRY((launch_table_chunk<tab_t, 512, stage>(table, state, d, grad, skeys, perm, n, n_rows, w, lr, beta, eps,
                                               chunk_threads, nchunks, st)));
  }
  const size_t chain_smem = (size_t)(CHAIN_WARPS - 1) * d * 4;  // <= 56 KB (d <= 2048)
  const unsigned chain_grid = (unsigned)((nchunks + CHAIN_WARPS - 1) / CHAIN_WARPS);
  WITH_NV(d, TRY(allow_smem(table_chain_kernel<NV, tab_t>, chain_smem)); ++g_launches;
          launch_pdl(table_chain_kernel<NV, tab_t>, chain_grid, CHAIN_WARPS * 32, chain_smem, st,
              table, state, d, skeys, n, n_rows, w.part_head, w.part_tail, lr, beta, eps););
  LAUNCH_CHECK();
  return GPT_OK;
}

// ======================================================================== forward
template <typename act_t>
static int attention_fwd(gpt_model* m, const act_t* qkv, act_t* o, float* lse) {
  const gpt_config& c = m->cfg;
  ProfScope ps(&m->prof, m->st, "attention_fwd",
               2.0 * c.micro_batch * c.n_head * (double)c.seq_len * c.seq_len * c.head_dim, 0.0);
  if (std::is_same<act_t, bf16>::value) {
    static bool attr = false;
    if (!attr) {
      CUDA_TRY(cudaFuncSetAttribute(fatc::fa_tc_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    fatc::SMEM_BYTES_TC));
      attr = true;
    }
    const long long a = (long long)c.n_head * c.head_dim, ntok = (long long)c.micro_batch * c.seq_len;
    CUtensorMap tqk, tv;
    TRY(make_tmap(&tqk, qkv, 3 * a, ntok, 3 * a, 64, 128));
    TRY(make_tmap(&tv, qkv, 3 * a, ntok, 3 * a, 64, 64));
    // persistent: one CTA per SM (or per item when there are fewer)
    const long long items = (long long)cdiv(c.seq_len, fatc::BQ) * c.micro_batch * c.n_head;
    const int grid = items < device_sms() ? (int)items : device_sms();
    // the output as [B][T][a] for the TMA stores of O: 32-row x 64-column
    // blocks, rows past a sequence's end clipped
    CUtensorMap to;
    TRY(make_tmap3(&to, o, a, c.seq_len, a, c.micro_batch, (long long)c.seq_len * a, 64, 32));
    ++g_launches; launch_pdl(fatc::fa_tc_fwd_kernel, grid, fatc::THREADS, fatc::SMEM_BYTES_TC, m->st,
        tqk, tv, to, lse, c.seq_len, c.n_head, c.micro_batch * c.n_head, m->err());
    LAUNCH_CHECK();
    return GPT_OK;
  }
  dim3 grid(cdiv(c.seq_len, 4), c.micro_batch * c.n_head);
  ++g_launches; attn_fwd_simt_kernel<act_t><<<grid, 128, 4 * c.head_dim * 4, m->st>>>(qkv, o, lse, c.micro_batch, c.seq_len,
                                                                        c.n_head, c.head_dim);
  LAUNCH_CHECK();
  return GPT_OK;
}

template <typename act_t>
static int attention_bwd(gpt_model* m, const act_t* qkv, const act_t* o, const act_t* dout,
                         const float* lse, float* Dv, act_t* dqkv) {
  const gpt_config& c = m->cfg;
  const long long N = (long long)c.micro_batch * c.seq_len;
  ProfScope ps(&m->prof, m->st, "attention_bwd",
               5.0 * c.micro_batch * c.n_head * (double)c.seq_len * c.seq_len * c.head_dim, 0.0);
  if (std::is_same<act_t, bf16>::value && c.head_dim == 128) {
    const long long warps = cdiv_ll(N * c.n_head, ATTN_PRE_ROWS);
    ++g_launches; launch_pdl(attn_bwd_pre_hd128_kernel, grid_for(warps * 32, 256), 256, 0, m->st,
        reinterpret_cast<const bf16*>(o), reinterpret_cast<const bf16*>(dout), Dv, c.micro_batch, c.seq_len,
        c.n_head);
  } else {
    ++g_launches; launch_pdl(attn_bwd_pre_kernel<act_t>, grid_for(N * c.n_head * 32, 256), 256, 0, m->st,
        o, dout, Dv, c.micro_batch, c.seq_len, c.n_head, c.head_dim);
  }
  LAUNCH_CHECK();
  if (std::is_same<act_t, bf16>::value) {
    static bool attr = false;
    if (!attr) {
      CUDA_TRY(cudaFuncSetAttribute(fatcb::fa_tc_bwd_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    fatcb::DKDV_SMEM));
      CUDA_TRY(cudaFuncSetAttribute(fatcb::fa_tc_bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    fatcb::DQ_SMEM));
      attr = true;
    }
    const long long a = (long long)c.n_head * c.head_dim;
    CUtensorMap t128, t64, tdo;
    TRY(make_tmap(&t128, qkv, 3 * a, N, 3 * a, 64, 128));
    TRY(make_tmap(&t64, qkv, 3 * a, N, 3 * a, 64, 64));
    TRY(make_tmap(&tdo, dout, a, N, a, 64, 64));
    // dqkv as [B][T][3a] for the TMA stores of dQ, dK, dV: 32-row x 64-column
    // blocks, rows past a sequence's end clipped
    CUtensorMap tg;
    TRY(make_tmap3(&tg, dqkv, 3 * a, c.seq_len, 3 * a, c.micro_batch, (long long)c.seq_len * 3 * a, 64, 32));
    const int BH = c.micro_batch * c.n_head;
    const long long items = (long long)cdiv(c.seq_len, 128) * BH;  // key tiles (dK, dV) = query tiles (dQ)
    const int grid = items < device_sms() ? (int)items : device_sms();  // persistent
    ++g_launches; launch_pdl(fatcb::fa_tc_bwd_dkdv_kernel, grid, fatcb::THREADS_B, fatcb::DKDV_SMEM, m->st,
        t128, t64, tdo, tg, lse, Dv, c.seq_len, c.n_head, BH, m->err());
    ++g_launches; launch_pdl(fatcb::fa_tc_bwd_dq_kernel, grid, fatcb::THREADS_B, fatcb::DQ_SMEM, m->st,
        t128, t64, tdo, tg, lse, Dv, c.seq_len, c.n_head, BH, m->err());
    LAUNCH_CHECK();
    return GPT_OK;
  }
  dim3 grid(cdiv(c.seq_len, 4), c.micro_batch * c.n_head);
  ++g_launches; attn_bwd_dq_simt_kernel<act_t><<<grid, 128, 4 * 2 * c.head_dim * 4, m->st>>>(
      qkv, dout, lse, Dv, dqkv, c.micro_batch, c.seq_len, c.n_head, c.head_dim);
  ++g_launches; attn_bwd_dkdv_simt_kernel<act_t><<<grid, 128, 4 * 2 * c.head_dim * 4, m->st>>>(
      qkv, dout, lse, Dv, dqkv, c.micro_batch, c.seq_len, c.n_head, c.head_dim);
  LAUNCH_CHECK();
  return GPT_OK;
}

template <typename act_t>
static int forward_impl(gpt_model* m, const int32_t* tokens, const int32_t* targets, float* loss_dev) {
  const gpt_config& c = m->cfg;
  const Plan& p = m->plan;
  const bool b16 = cfg_bf16(c);
  cudaStream_t st = m->st;
  const int N = c.micro_batch * c.seq_len;
  const int d = c.d_model, H = c.n_head, hd = c.head_dim, a = H * hd, F = c.d_ff, V = c.vocab;
  unsigned* err = m->err();
  GemmCtx g{b16, m->at<float>(p.splitk), p.splitk_elems, err, st, &m->prof};
  // weights read by the GEMMs: the bf16 copy in bf16 mode, the master in fp32 mode
  auto W = [&](const std::string& nm) -> const act_t* {
    const DenseTensor* t = find_dense(m, nm);
    return b16 ? reinterpret_cast<const act_t*>(m->at<bf16>(p.Plp) + t->off)
               : reinterpret_cast<const act_t*>(m->at<float>(p.P) + t->off);
  };
  const size_t es = sizeof(act_t);
  Prof* pf = &m->prof;
  CUDA_TRY(cudaMemcpyAsync(m->at<int32_t>(p.tok_copy), tokens, (size_t)N * 4, cudaMemcpyDeviceToDevice, st));
  if (c.x0_rows || c.v_rows) {
    ProfScope ps(pf, st, "ngram_hash", 0.0, (double)N * 12);
    ++g_launches; launch_pdl(ngram_hash_kernel, grid_for(N, 256), 256, 0, st,
        tokens, c.micro_batch, c.seq_len, V, c.hash_p1, c.hash_p2, c.x0_rows ? c.x0_rows : 1,
        c.x0_rows ? m->at<int32_t>(p.rows_x) : nullptr, c.v_rows ? c.v_rows : 1,
        c.v_rows ? m->at<int32_t>(p.rows_v) : nullptr, err);
    LAUNCH_CHECK();
  }
  // per-position value bias of the frozen trigram statistics: vb = S3[r3] vproj^T
  // (+ the value-table row), added to v by every layer
  const act_t* vbias = c.v_rows ? reinterpret_cast<const act_t*>(m->base + p.hv) : nullptr;
  const int32_t* vrows = m->at<int32_t>(p.rows_v);
  if (c.tri_rows) {
    const int w3 = c.tri_width;
    {
      ProfScope ps(pf, st, "trigram_gather", 0.0, (double)N * (12 + 2.0 * w3 * es));
      ++g_launches; launch_pdl(trigram_hash_kernel, grid_for(N, 256), 256, 0, st,
          tokens, c.micro_batch, c.seq_len, V, c.hash_p1, c.hash_p2, c.hash_p3, c.tri_rows,
          m->at<int32_t>(p.rows_3), err);
      const act_t* h3 = reinterpret_cast<const act_t*>(m->base + p.h3);
      act_t* s3g = m->at<act_t>(p.s3g);
      if (b16) {
        ++g_launches; launch_pdl(ngram_gather_bf16x8_kernel, grid_for((long long)(N + 1) / 2 * 32, 256), 256, 0, st,
            m->at<int32_t>(p.rows_3), N, reinterpret_cast<const bf16*>(h3), c.tri_rows, w3,
            reinterpret_cast<bf16*>(s3g), 0, err);
      } else {
        ++g_launches; launch_pdl(ngram_gather_kernel<act_t>, grid_for((long long)N * 32, 256), 256, 0, st,
            m->at<int32_t>(p.rows_3), N, h3, c.tri_rows, w3, s3g, 0, err);
      }
      LAUNCH_CHECK();
    }
    TRY(gemm(g, N, a, w3, op_k(m->at<act_t>(p.s3g), w3), op_k(W("vproj"), w3),
             epi(EPI_STORE_F32, m->at<float>(p.p3), a), false, "gemm.vproj_fwd"));
    {
      ProfScope ps(pf, st, "value_bias", 0.0, (double)N * a * (4 + es + (c.v_rows ? es : 0)));
      ++g_launches; launch_pdl(value_bias_kernel<act_t>, 4 * device_sms(), 256, 0, st,
          m->at<float>(p.p3), vbias, vrows, N, a, m->at<act_t>(p.vb));
      LAUNCH_CHECK();
    }
    vbias = m->at<act_t>(p.vb);
    vrows = nullptr;  // row n of the bias for position n
  }
  float* x = m->at<float>(p.x);
  {
  ProfScope ps(pf, st, "embed", 0.0, (double)N * d * (es + 4 + (c.x0_rows ? es : 0)));
  WITH_NV(d, ++g_launches; launch_pdl(embed_fwd_kernel<NV, act_t, act_t>, grid_for((long long)N * 32, 256), 256, 0, st,
      tokens, W("wte"), c.x0_rows ? reinterpret_cast<const act_t*>(m->base + p.hx) : nullptr,
      m->at<int32_t>(p.rows_x), x, m->at<float>(p.emb_rstd), N, d, V, c.norm_eps, err););
  LAUNCH_CHECK();
  }
  const double norm_bytes = (double)N * d * (4 + es) + 4.0 * N;
  const int rows_blocks = grid_for((long long)N * 32, 256);
  for (int l = 0; l < c.n_layer; ++l) {
    const LayerActs& L = p.layers[l];
    const std::string pre = "h" + std::to_string(l) + ".";
    act_t* u = m->at<act_t>(L.u);
    act_t* qkv = m->at<act_t>(L.qkv);
    act_t* o = m->at<act_t>(L.o);
    act_t* u2 = m->at<act_t>(L.u2);
    {
      ProfScope ps(pf, st, "rmsnorm_fwd", 0.0, norm_bytes);
      WITH_NV(d, ++g_launches; launch_pdl(rmsnorm_fwd_kernel<NV, act_t>, rows_blocks, 256, 0, st, x, u, m->at<float>(L.rstd1), N, d, c.norm_eps););
      LAUNCH_CHECK();
    }
    if (b16) {
      // QKV projection with RoPE + QK-norm (+ value-table row) in its epilogue
      GemmEpilogue eq = epi(EPI_QKV, qkv, 3 * a);
      eq.rope = m->at<float2>(p.rope_turns);
      eq.rstd_q = m->at<float>(L.rstd_q);
      eq.rstd_k = m->at<float>(L.rstd_k);
      eq.hv = vbias;
      eq.rv = vrows;
      eq.T = c.seq_len; eq.H = H; eq.qk_norm = c.qk_norm; eq.eps = c.norm_eps;
      TRY(gemm(g, N, 3 * a, d, op_k(u, d), op_k(W(pre + "wqkv"), d), eq, false, "gemm.qkv_fwd"));
    } else {
      TRY(gemm(g, N, 3 * a, d, op_k(u, d), op_k(W(pre + "wqkv"), d), epi(EPI_STORE, qkv, 3 * a), false, "gemm.qkv_fwd"));
      ProfScope ps(pf, st, "rope_qknorm_fwd", 0.0, (double)N * a * es * (4 + (c.v_rows ? 3 : 0)));
      ++g_launches; rope_qknorm_fwd_kernel<act_t, act_t><<<grid_for((long long)N * H * 32, 256), 256, 0, st>>>(
          qkv, m->at<float>(p.rope_cs), m->at<float>(L.rstd_q), m->at<float>(L.rstd_k), vbias, vrows, N,
          c.seq_len, H, hd, c.qk_norm, c.norm_eps);
      LAUNCH_CHECK();
    }
    TRY(attention_fwd<act_t>(m, qkv, o, m->at<float>(L.lse)));
    TRY(gemm(g, N, d, a, op_k(o, a), op_k(W(pre + "wo"), a), epi(EPI_ACCUM_F32, x, d, 1), false, "gemm.o_fwd"));
    {
      ProfScope ps(pf, st, "rmsnorm_fwd", 0.0, norm_bytes);
      WITH_NV(d, ++g_launches; launch_pdl(rmsnorm_fwd_kernel<NV, act_t>, rows_blocks, 256, 0, st, x, u2, m->at<float>(L.rstd2), N, d, c.norm_eps););
      LAUNCH_CHECK();
    }
    TRY(gemm(g, N, F, d, op_k(u2, d), op_k(W(pre + "w1"), d),
             epi(EPI_RELU2, m->at<act_t>(L.g), F), false, "gemm.up_fwd"));
    TRY(gemm(g, N, d, F, op_k(m->at<act_t>(L.g), F), op_k(W(pre + "w2"), F), epi(EPI_ACCUM_F32, x, d, 1), false, "gemm.down_fwd"));
  }
  act_t* xf = m->at<act_t>(p.xf);
  {
    ProfScope ps(pf, st, "rmsnorm_fwd", 0.0, norm_bytes);
    WITH_NV(d, ++g_launches; launch_pdl(rmsnorm_fwd_kernel<NV, act_t>, rows_blocks, 256, 0, st, x, xf, m->at<float>(p.rstd_f), N, d, c.norm_eps););
  }
  ++g_launches; launch_pdl(ce_prepare_kernel, 1, 1024, 0, st, targets, N, c.grad_accum, m->at<float>(p.ce_scale), m->at<int>(p.ce_count));
  LAUNCH_CHECK();
  // chunked LM head + cross-entropy; the head's gradient pieces are formed
  // here while each logits chunk is live: dxf (fp32) and the pending head
  // weight gradient, which backward adds into the dense gradient.
  const act_t* Wlm = W(c.tie_embeddings ? "wte" : "lm_head");
  float* logits = b16 ? nullptr : m->at<float>(p.logits);
  act_t* dz = m->at<act_t>(p.dz);
  for (int r0 = 0, ci = 0; r0 < N; r0 += p.chunk, ++ci) {
    const int rows = (N - r0 < p.chunk) ? (N - r0) : p.chunk;
    if (b16) {
      GemmEpilogue el = epi(EPI_LOGITS, dz, V);
      el.softcap = c.softcap;
      el.stats = m->at<float2>(p.ce_stats);
      el.targets = targets + r0;
      el.ztgt = m->at<float>(p.ce_ztgt);
      TRY(gemm(g, rows, V, d, op_k(xf + (long long)r0 * d, d), op_k(Wlm, d), el, false, "gemm.lm_fwd"));
      ProfScope ps(pf, st, "cross_entropy", 0.0, (double)rows * V * 4);
      const int tcols = V >= 256 ? 128 : 64, ntl = cdiv(V, tcols);  // half-tile statistics
      ++g_launches; launch_pdl(ce_prob_kernel, rows, 256, ntl * 4, st,
          reinterpret_cast<bf16*>(dz), m->at<float2>(p.ce_stats), ntl, tcols, targets + r0, m->at<float>(p.ce_ztgt),
          m->at<float>(p.tok_loss) + r0, V, c.softcap, m->at<float>(p.ce_scale), err);
      LAUNCH_CHECK();
    } else {
      TRY(gemm(g, rows, V, d, op_k(xf + (long long)r0 * d, d), op_k(Wlm, d), epi(EPI_STORE_F32, logits, V), false,
               "gemm.lm_fwd"));
      ProfScope ps(pf, st, "cross_entropy", 0.0, (double)rows * V * (4 + es));
      ++g_launches; ce_chunk_kernel<act_t><<<rows, 512, 0, st>>>(logits, dz, targets + r0, m->at<float>(p.tok_loss) + r0, V,
                                                   c.softcap, m->at<float>(p.ce_scale), err);
      LAUNCH_CHECK();
    }
    TRY(gemm(g, rows, d, V, op_k(dz, V), op_mn(Wlm, d), epi(EPI_STORE_F32, m->at<float>(p.dxf) + (long long)r0 * d, d), true,
             "gemm.lm_dgrad"));
    TRY(gemm(g, V, d, rows, op_mn(dz, V), op_mn(xf + (long long)r0 * d, d),
             epi(EPI_ACCUM_F32, m->at<float>(p.pending), d, ci > 0), true, "gemm.lm_wgrad"));
  }
  ++g_launches; launch_pdl(loss_reduce_kernel, 1, 1024, 0, st, m->at<float>(p.tok_loss), N, m->at<int>(p.ce_count), loss_dev, err);
  LAUNCH_CHECK();
  m->have_fwd = true;
  return GPT_OK;
}

// ======================================================================== backward
static int optimizer_step_impl(gpt_model* m, float lr);

template <typename act_t>
static int backward_impl(gpt_model* m, float lr, bool do_step) {
  const gpt_config& c = m->cfg;
  const Plan& p = m->plan;
  const bool b16 = cfg_bf16(c);
  cudaStream_t st = m->st;
  const int N = c.micro_batch * c.seq_len;
  const int d = c.d_model, H = c.n_head, hd = c.head_dim, a = H * hd, F = c.d_ff, V = c.vocab;
  unsigned* err = m->err();
  GemmCtx g{b16, m->at<float>(p.splitk), p.splitk_elems, err, st, &m->prof};
  auto W = [&](const std::string& nm) -> const act_t* {
    const DenseTensor* t = find_dense(m, nm);
    return b16 ? reinterpret_cast<const act_t*>(m->at<bf16>(p.Plp) + t->off)
               : reinterpret_cast<const act_t*>(m->at<float>(p.P) + t->off);
  };
  auto Gp = [&](const std::string& nm) -> float* { return m->at<float>(p.G) + find_dense(m, nm)->off; };
  const int beta = m->micro > 0;
  const int rows_blocks = grid_for((long long)N * 32, 256);
  const size_t es = sizeof(act_t);
  Prof* pf = &m->prof;
  const double nb_bytes = (double)N * d * (4 + es + 4 + es) + 4.0 * N + (double)N * d * 4;
  // LM-head weight gradient staged by the forward pass
  float* g_head = Gp(c.tie_embeddings ? "wte" : "lm_head");
  {
    ProfScope ps(pf, st, "head_grad_accumulate", 0.0, (double)V * d * 12);
    ++g_launches; launch_pdl(accumulate_kernel, 4 * device_sms(), 256, 0, st, g_head, m->at<float>(p.pending), (long long)V * d, beta);
    if (!c.tie_embeddings && !beta) CUDA_TRY(cudaMemsetAsync(Gp("wte"), 0, (size_t)V * d * 4, st));
  }
  float* dx = m->at<float>(p.dx);
  act_t* dx_lp = m->at<act_t>(p.dx_lp);
  float* du = m->at<float>(p.du);
  act_t* dqkv = m->at<act_t>(p.dqkv);
  act_t* da = m->at<act_t>(p.da);
  act_t* dout = m->at<act_t>(p.dout);
  { ProfScope psn(pf, st, "rmsnorm_bwd", 0.0, nb_bytes); WITH_NV(d, ++g_launches; launch_pdl(rmsnorm_bwd_kernel<NV, act_t>, rows_blocks, 256, 0, st, m->at<float>(p.dxf), m->at<act_t>(p.xf),
                                                        m->at<float>(p.rstd_f), dx, dx_lp, N, d, 0););
  LAUNCH_CHECK(); }
  for (int l = c.n_layer - 1; l >= 0; --l) {
    const LayerActs& L = p.layers[l];
    const std::string pre = "h" + std::to_string(l) + ".";
    // ---- MLP: x += relu(u2 W1^T)^2 W2^T
    TRY(gemm(g, d, F, N, op_mn(dx_lp, d), op_mn(m->at<act_t>(L.g), F), epi(EPI_ACCUM_F32, Gp(pre + "w2"), F, beta), true, "gemm.down_wgrad"));
    TRY(gemm(g, N, F, d, op_k(dx_lp, d), op_mn(W(pre + "w2"), F), epi(EPI_DRELU2, da, F, 0, nullptr, m->at<act_t>(L.g)), false, "gemm.down_dgrad"));
    TRY(gemm(g, F, d, N, op_mn(da, F), op_mn(m->at<act_t>(L.u2), d), epi(EPI_ACCUM_F32, Gp(pre + "w1"), d, beta), true, "gemm.up_wgrad"));
    TRY(gemm(g, N, d, F, op_k(da, F), op_mn(W(pre + "w1"), d), epi(EPI_STORE_F32, du, d), false, "gemm.up_dgrad"));
    { ProfScope psn(pf, st, "rmsnorm_bwd", 0.0, nb_bytes); WITH_NV(d, ++g_launches; launch_pdl(rmsnorm_bwd_kernel<NV, act_t>, rows_blocks, 256, 0, st, du, m->at<act_t>(L.u2), m->at<float>(L.rstd2), dx, dx_lp, N, d, 1););
    LAUNCH_CHECK(); }
    // ---- attention: x += o Wo^T
    TRY(gemm(g, d, a, N, op_mn(dx_lp, d), op_mn(m->at<act_t>(L.o), a), epi(EPI_ACCUM_F32, Gp(pre + "wo"), a, beta), true, "gemm.o_wgrad"));
    TRY(gemm(g, N, a, d, op_k(dx_lp, d), op_mn(W(pre + "wo"), a), epi(EPI_STORE, dout, a), false, "gemm.o_dgrad"));
    TRY(attention_bwd<act_t>(m, m->at<act_t>(L.qkv), m->at<act_t>(L.o), dout, m->at<float>(L.lse),
                             m->at<float>(p.Dattn), dqkv));
    {
      ProfScope ps(pf, st, "rope_qknorm_bwd", 0.0, (double)N * a * es * 6 + (c.v_rows ? (double)N * a * (es + 8) : 0.0));
      if (b16)  // hd == 128 in bf16 mode
        ++g_launches, launch_pdl(rope_qknorm_bwd_hd128_kernel, grid_for((long long)N * H * 32, 256), 256, 0, st,
            reinterpret_cast<bf16*>(dqkv), reinterpret_cast<const bf16*>(m->at<act_t>(L.qkv)), m->at<float>(p.rope_cs),
            m->at<float>(L.rstd_q), m->at<float>(L.rstd_k), p.gv ? m->at<float>(p.gv) : nullptr,
            l != c.n_layer - 1, N, c.seq_len, H, c.qk_norm);
      else
        ++g_launches, rope_qknorm_bwd_kernel<act_t><<<grid_for((long long)N * H * 32, 256), 256, 0, st>>>(
            dqkv, m->at<act_t>(L.qkv), m->at<float>(p.rope_cs), m->at<float>(L.rstd_q), m->at<float>(L.rstd_k),
            p.gv ? m->at<float>(p.gv) : nullptr, l != c.n_layer - 1, N, c.seq_len, H, hd, c.qk_norm);
      LAUNCH_CHECK();
    }
    TRY(gemm(g, 3 * a, d, N, op_mn(dqkv, 3 * a), op_mn(m->at<act_t>(L.u), d), epi(EPI_ACCUM_F32, Gp(pre + "wqkv"), d, beta), true, "gemm.qkv_wgrad"));
    TRY(gemm(g, N, d, 3 * a, op_k(dqkv, 3 * a), op_mn(W(pre + "wqkv"), d), epi(EPI_STORE_F32, du, d), false, "gemm.qkv_dgrad"));
    { ProfScope psn(pf, st, "rmsnorm_bwd", 0.0, nb_bytes); WITH_NV(d, ++g_launches; launch_pdl(rmsnorm_bwd_kernel<NV, act_t>, rows_blocks, 256, 0, st, du, m->at<act_t>(L.u), m->at<float>(L.rstd1), dx, dx_lp, N, d, 1););
    LAUNCH_CHECK(); }
  }
  // dx now holds dL/dx0 per position.
  if (c.tri_rows) {
    // projection of the frozen trigram statistics: d vproj += gv^T S3[r3], gv the
    // value gradient summed over layers (no gradient reaches the table)
    const int w3 = c.tri_width;
    const act_t* gva;
    if (b16) {
      ProfScope ps(pf, st, "value_grad_bf16", 0.0, (double)N * a * 6);
      ++g_launches; launch_pdl(to_bf16_kernel, 4 * device_sms(), 256, 0, st, m->at<float>(p.gv), m->at<bf16>(p.gv16),
                                                                     (long long)N * a);
      LAUNCH_CHECK();
      gva = reinterpret_cast<const act_t*>(m->at<bf16>(p.gv16));
    } else {
      gva = reinterpret_cast<const act_t*>(m->at<float>(p.gv));
    }
    TRY(gemm(g, a, w3, N, op_mn(gva, a), op_mn(m->at<act_t>(p.s3g), w3),
             epi(EPI_ACCUM_F32, Gp("vproj"), w3, beta), true, "gemm.vproj_wgrad"));
  }
  const SortWs w = sort_ws(m);
  {
    // token embedding gradient, bucketed by token id
    ProfScope ps(pf, st, "embedding_grad", 0.0, (double)N * d * 4);
    const uint32_t* skeys;
    const int32_t* perm;
    TRY(bucket_by_key(w, m->at<int32_t>(p.tok_copy), N, V, &skeys, &perm, nullptr, nullptr, err, st));
    const long long nchunks = (N + CHUNK - 1) / CHUNK;
    WITH_NV(d, ++g_launches; launch_pdl(emb_chunk_kernel<NV, act_t>, grid_for(nchunks * 32, 128), 128, 0, st,
        Gp("wte"), W("wte"), d, dx, m->at<float>(p.emb_rstd), skeys, perm, N, V, w.part_head, w.part_tail););
    const size_t chain_smem = (size_t)(CHAIN_WARPS - 1) * d * 4;
    const unsigned chain_grid = (unsigned)((nchunks + CHAIN_WARPS - 1) / CHAIN_WARPS);
    WITH_NV(d, TRY(allow_smem(emb_chain_kernel<NV>, chain_smem)); ++g_launches;
            launch_pdl(emb_chain_kernel<NV>, chain_grid, CHAIN_WARPS * 32, chain_smem, st,
                Gp("wte"), d, skeys, N, V, w.part_head, w.part_tail););
    LAUNCH_CHECK();
  }
  const float lr_t = lr * c.lr_mult_table;
  if (c.v_rows && !m->defer_tables) {
    ProfScope ps(pf, st, "table_update", 0.0, (double)N * a * 4);
    TRY(table_update<act_t>(w, reinterpret_cast<act_t*>(m->base + p.hv), m->at<float>(p.hv_state), c.v_rows, a,
                            m->at<int32_t>(p.rows_v), m->at<float>(p.gv), N, lr_t, c.table_beta, c.table_eps,
                            nullptr, nullptr, err, st));
  }
  if (c.x0_rows && !m->defer_tables) {
    ProfScope ps(pf, st, "table_update", 0.0, (double)N * d * 4);
    TRY(table_update<act_t>(w, reinterpret_cast<act_t*>(m->base + p.hx), m->at<float>(p.hx_state), c.x0_rows, d,
                            m->at<int32_t>(p.rows_x), dx, N, lr_t, c.table_beta, c.table_eps, nullptr, nullptr, err, st));
  }
  m->micro += 1;
  m->have_fwd = false;
  if (do_step && m->micro == c.grad_accum) return optimizer_step_impl(m, lr);
  return GPT_OK;
}

// `bt.n` same-shape products in one launch (store epilogues, no split-K)
static int gemm_batched(const GemmCtx& g, const GemmBatch& bt, int M, int N, int K, GemmOperand A, GemmOperand B,
                        GemmEpilogue e, const char* label) {
  ProfScope ps(g.prof, g.st, label, 2.0 * M * N * K * bt.n, 0.0);
  if (N >= 256 && gemm_pairs_enabled())
    return gemm_tc_launch<256, 2>(M, N, K, A, B, e, 1, g.splitk, g.err, g.st, bt);
  return gemm_tc_launch<128, 1>(M, N, K, A, B, e, 1, g.splitk, g.err, g.st, bt);
}

// Muon on every block matrix, one group of same-shape matrices at a time:
// momentum (on the clipped gradient) with a per-matrix sum of squares, the
// normalised bf16 iterate, muon_ns_steps Newton-Schulz steps as batched GEMMs
// over the group (X X^T or X^T X, A A, then B X or X B), and the scaled step
// into the fp32 master and its bf16 copy.  Every product leaves its GEMM
// rounded to bf16, as in the pages' bf16 iteration (A, A A, B X each a bf16
// matmul output; B = b A + c A A and X <- a X + B X formed from bf16 values,
// rounded once), which halves the iteration's elementwise traffic.
static int muon_step_impl(gpt_model* m, float lr, const float* clip) {
  const gpt_config& c = m->cfg;
  const Plan& p = m->plan;
  cudaStream_t st = m->st;
  float* P = m->at<float>(p.P);
  float* G = m->at<float>(p.G);
  float* M = m->at<float>(p.M);
  bf16* Plp = m->at<bf16>(p.Plp);
  bf16* x = m->at<bf16>(p.mu_x);
  bf16* xn = m->at<bf16>(p.mu_xn);
  bf16* abf = m->at<bf16>(p.mu_abf);
  bf16* bm = m->at<bf16>(p.mu_bm);
  float* part = m->at<float>(p.mu_part);
  const GemmCtx g{true, m->at<float>(p.splitk), p.splitk_elems, m->err(), st, &m->prof};
  const float ca = 3.4445f, cb = -4.7750f, cc = 2.0315f;  // a x + b x^3 + c x^5
  for (int gi = 0; gi < p.n_muon_groups; ++gi) {
    const MuonGroup& grp = p.muon_groups[gi];
    const int rows = grp.rows, cols = grp.cols, nmat = grp.nmat;
    const int R = rows < cols ? rows : cols;
    const bool tall = rows > cols;
    const long long n = (long long)rows * cols, rr = (long long)R * R;
    const unsigned per_mat = (unsigned)std::min<long long>((n / 4 + MUON_THREADS - 1) / MUON_THREADS, MUON_BATCH_BLOCKS);
    {
      // bytes: g, m read + m written; g, m read + bf16 iterate written
      ProfScope ps(&m->prof, st, "muon_elementwise", 0.0, (double)nmat * n * (12 + 10));
      ++g_launches;
      launch_pdl(muon_batch_momentum_kernel, dim3(MUON_BATCH_BLOCKS, nmat), MUON_THREADS, 0, st,
          G, M, grp, c.muon_momentum, c.muon_nesterov, clip, part);
      ++g_launches;
      launch_pdl(muon_batch_normalize_kernel, dim3(per_mat, nmat), MUON_THREADS, 0, st,
          G, M, grp, c.muon_momentum, c.muon_nesterov, clip, part, 1e-7f, x);
      LAUNCH_CHECK();
    }
    for (int it = 0; it < c.muon_ns_steps; ++it) {
      if (!tall)
        TRY(gemm_batched(g, GemmBatch{nmat, n, n, rr}, R, R, cols, op_k(x, cols), op_k(x, cols),
                         epi(EPI_STORE, abf, R), "muon.gram"));
      else
        TRY(gemm_batched(g, GemmBatch{nmat, n, n, rr}, R, R, rows, op_mn(x, cols), op_mn(x, cols),
                         epi(EPI_STORE, abf, R), "muon.gram"));
      // B = b A + c A A, the combination taken in the square product's epilogue
      GemmEpilogue esq = epi(EPI_AXPBY, bm, R, 0, nullptr, abf, cc);
      esq.aux_scale = cb;
      TRY(gemm_batched(g, GemmBatch{nmat, rr, rr, rr}, R, R, R, op_k(abf, R), op_mn(abf, R), esq, "muon.square"));
      // X' = a X + B X (X B when tall), the combination in the product's epilogue
      GemmEpilogue epo = epi(EPI_AXPBY, xn, cols, 0, nullptr, x, 1.f);
      epo.aux_scale = ca;
      if (!tall)
        TRY(gemm_batched(g, GemmBatch{nmat, rr, n, n}, rows, cols, R, op_k(bm, R), op_mn(x, cols), epo,
                         "muon.poly"));
      else
        TRY(gemm_batched(g, GemmBatch{nmat, n, rr, n}, rows, cols, R, op_k(x, cols), op_mn(bm, R), epo,
                         "muon.poly"));
      LAUNCH_CHECK();
      std::swap(x, xn);
    }
    // weights are [out, in] = [rows, cols]
    const float step = (float)(lr * c.lr_mult_matrix * std::sqrt(std::max(1.0, (double)rows / cols)));
    {
      ProfScope ps(&m->prof, st, "muon_elementwise", 0.0, (double)nmat * n * 12);
      ++g_launches;
      launch_pdl(muon_batch_apply_kernel, dim3(per_mat, nmat), MUON_THREADS, 0, st, P, Plp, x, grp, step);
    }
    LAUNCH_CHECK();
    // the next group starts from the scratch's first iterate buffer again
    if (x != m->at<bf16>(p.mu_x)) std::swap(x, xn);
  }
  return GPT_OK;
}

// Global-norm clip (optional) and AdamW over the accumulated dense gradient
// (with Muon: AdamW over the embedding and head, Muon over the block matrices).
static int optimizer_step_impl(gpt_model* m, float lr) {
  const gpt_config& c = m->cfg;
  const Plan& p = m->plan;
  const bool b16 = cfg_bf16(c);
  const bool muon = c.matrix_optimizer == GPT_MATRIX_MUON;
  cudaStream_t st = m->st;
  unsigned* err = m->err();
  float* coef = nullptr;
  {
    ProfScope ps(&m->prof, st, "adamw", 0.0, (double)(muon ? p.blocks_begin : p.dense_n) * (b16 ? 30 : 28));
    m->micro = 0;
    m->step_t += 1;
    if (c.grad_clip > 0.f) {
      ++g_launches; launch_pdl(sumsq_partial_kernel, NORM_BLOCKS, 256, 0, st, m->at<float>(p.G), p.dense_n, m->at<double>(p.norm_part));
      ++g_launches; launch_pdl(clip_coef_kernel, 1, 256, 0, st, m->at<double>(p.norm_part), NORM_BLOCKS, c.grad_clip,
                                         m->at<float>(p.clip_coef), m->at<float>(p.grad_norm), err);
      LAUNCH_CHECK();
      coef = m->at<float>(p.clip_coef);
    }
    AdamArgs aa;
    aa.p = m->at<float>(p.P); aa.g = m->at<float>(p.G); aa.m = m->at<float>(p.M); aa.v = m->at<float>(p.V);
    aa.p_lp = b16 ? m->at<bf16>(p.Plp) : nullptr;
    aa.n = muon ? p.blocks_begin : p.dense_n; aa.e_end = p.e_end; aa.h_end = p.h_end;
    aa.lr_e = lr * c.lr_mult_embed; aa.lr_h = lr * c.lr_mult_head; aa.lr_m = lr * c.lr_mult_matrix;
    aa.b1 = c.adam_b1; aa.b2 = c.adam_b2; aa.eps = c.adam_eps; aa.wd = c.weight_decay;
    aa.bc1 = (float)(1.0 - pow((double)c.adam_b1, (double)m->step_t));
    aa.bc2 = (float)(1.0 - pow((double)c.adam_b2, (double)m->step_t));
    aa.clip = coef;
    ++g_launches; launch_pdl(adamw_kernel, 8 * device_sms(), 256, 0, st, aa);
    LAUNCH_CHECK();
  }
  if (muon) TRY(muon_step_impl(m, lr, coef));
  return GPT_OK;
}

extern "C" int gpt_forward_loss(gpt_model* m, const int32_t* tokens, const int32_t* targets, float* loss_dev) {
  if (!m || !tokens || !targets || !loss_dev) return fail(GPT_ERR_ARG, "null argument");
  if (cfg_bf16(m->cfg)) return forward_impl<bf16>(m, tokens, targets, loss_dev);
  return forward_impl<float>(m, tokens, targets, loss_dev);
}

extern "C" int gpt_backward_step(gpt_model* m, float lr) {
  if (!m) return fail(GPT_ERR_ARG, "null model");
  if (!m->have_fwd) return fail(GPT_ERR_STATE, "gpt_backward_step needs a preceding gpt_forward_loss");
  if (!std::isfinite(lr)) return fail(GPT_ERR_ARG, "learning rate not finite");
  if (cfg_bf16(m->cfg)) return backward_impl<bf16>(m, lr, true);
  return backward_impl<float>(m, lr, true);
}

extern "C" int gpt_backward(gpt_model* m, float lr) {
  if (!m) return fail(GPT_ERR_ARG, "null model");
  if (!m->have_fwd) return fail(GPT_ERR_STATE, "gpt_backward needs a preceding gpt_forward_loss");
  if (!std::isfinite(lr)) return fail(GPT_ERR_ARG, "learning rate not finite");
  if (cfg_bf16(m->cfg)) return backward_impl<bf16>(m, lr, false);
  return backward_impl<float>(m, lr, false);
}

extern "C" int gpt_set_table_exchange(gpt_model* m, int on) {
  if (!m) return fail(GPT_ERR_ARG, "null model");
  m->defer_tables = on != 0;
  return GPT_OK;
}

extern "C" int gpt_optimizer_step(gpt_model* m, float lr) {
  if (!m) return fail(GPT_ERR_ARG, "null model");
  if (m->micro == 0) return fail(GPT_ERR_STATE, "gpt_optimizer_step needs at least one gpt_backward");
  if (!std::isfinite(lr)) return fail(GPT_ERR_ARG, "learning rate not finite");
  return optimizer_step_impl(m, lr);
}

// ---- sharded optimizer step (data parallelism with a reduce-scattered gradient)
extern "C" int gpt_grad_sumsq(gpt_model* m, long long lo, long long hi, double* out_dev) {
  if (!m || !out_dev || lo < 0 || hi < lo || hi > m->plan.dense_n)
    return fail(GPT_ERR_ARG, "gpt_grad_sumsq: bad range");
  const Plan& p = m->plan;
  ++g_launches; launch_pdl(sumsq_partial_kernel, NORM_BLOCKS, 256, 0, m->st, m->at<float>(p.G) + lo, hi - lo,
                                                                      m->at<double>(p.norm_part));
  ++g_launches; launch_pdl(sum_partials_kernel, 1, 256, 0, m->st, m->at<double>(p.norm_part), NORM_BLOCKS, out_dev);
  LAUNCH_CHECK();
  return GPT_OK;
}

extern "C" int gpt_optimizer_step_range(gpt_model* m, float lr, long long lo, long long hi,
                                        const double* grad_sumsq_dev) {
  if (!m) return fail(GPT_ERR_ARG, "null model");
  const gpt_config& c = m->cfg;
  const Plan& p = m->plan;
  if (m->micro == 0) return fail(GPT_ERR_STATE, "gpt_optimizer_step_range needs at least one gpt_backward");
  if (!std::isfinite(lr)) return fail(GPT_ERR_ARG, "learning rate not finite");
  if (lo < 0 || hi < lo || hi > p.dense_n || (lo & 3) || (hi & 3))
    return fail(GPT_ERR_ARG, "gpt_optimizer_step_range: range must lie in the flat buffer, ends multiples of 4");
  if (c.matrix_optimizer == GPT_MATRIX_MUON)
    return fail(GPT_ERR_CONFIG, "a sharded optimizer step needs whole matrices for Muon: use gpt_optimizer_step");
  if (c.grad_clip > 0.f && !grad_sumsq_dev)
    return fail(GPT_ERR_ARG, "grad_clip > 0 needs the global gradient sum of squares");
  const bool b16 = cfg_bf16(c);
  cudaStream_t st = m->st;
  ProfScope ps(&m->prof, st, "adamw", 0.0, (double)(hi - lo) * (b16 ? 30 : 28));
  m->micro = 0;
  m->step_t += 1;
  float* coef = nullptr;
  if (c.grad_clip > 0.f) {
    ++g_launches; launch_pdl(clip_coef_kernel, 1, 256, 0, st, grad_sumsq_dev, 1, c.grad_clip, m->at<float>(p.clip_coef),
                                                       m->at<float>(p.grad_norm), m->err());
    coef = m->at<float>(p.clip_coef);
  }
  AdamArgs aa;
  aa.p = m->at<float>(p.P) + lo; aa.g = m->at<float>(p.G) + lo; aa.m = m->at<float>(p.M) + lo;
  aa.v = m->at<float>(p.V) + lo;
  aa.p_lp = b16 ? m->at<bf16>(p.Plp) + lo : nullptr;
  aa.n = hi - lo; aa.e_end = std::max(0LL, p.e_end - lo); aa.h_end = std::max(0LL, p.h_end - lo);
  aa.lr_e = lr * c.lr_mult_embed; aa.lr_h = lr * c.lr_mult_head; aa.lr_m = lr * c.lr_mult_matrix;
  aa.b1 = c.adam_b1; aa.b2 = c.adam_b2; aa.eps = c.adam_eps; aa.wd = c.weight_decay;
  aa.bc1 = (float)(1.0 - pow((double)c.adam_b1, (double)m->step_t));
  aa.bc2 = (float)(1.0 - pow((double)c.adam_b2, (double)m->step_t));
  aa.clip = coef;
  ++g_launches; launch_pdl(adamw_kernel, 8 * device_sms(), 256, 0, st, aa);
  LAUNCH_CHECK();
  return GPT_OK;
}

extern "C" int gpt_launch_count(long long* n) {
  if (!n) return fail(GPT_ERR_ARG, "null pointer");
  *n = g_launches.load();
  return GPT_OK;
}

extern "C" int gpt_profile_enable(gpt_model* m, int on) {
  if (!m) return fail(GPT_ERR_ARG, "null model");
  if (on) {
    m->prof.recs.clear();
    m->prof.used = 0;
  }
  m->prof.on = on != 0;
  return GPT_OK;
}

extern "C" int gpt_profile_read(gpt_model* m, gpt_prof_entry* out, int cap, int* n) {
  if (!m || !n || (cap > 0 && !out)) return fail(GPT_ERR_ARG, "null argument");
  CUDA_TRY(cudaStreamSynchronize(m->st));
  std::vector<gpt_prof_entry> agg;
  for (const ProfRec& r : m->prof.recs) {
    float ms = 0.f;
    CUDA_TRY(cudaEventElapsedTime(&ms, r.a, r.b));
    gpt_prof_entry* e = nullptr;
    for (auto& x : agg)
      if (strncmp(x.name, r.cls, sizeof(x.name)) == 0) e = &x;
    if (!e) {
      gpt_prof_entry z;
      memset(&z, 0, sizeof(z));
      strncpy(z.name, r.cls, sizeof(z.name) - 1);
      agg.push_back(z);
      e = &agg.back();
    }
    e->scopes += 1;
    e->launches += r.launches;
    e->ms += ms;
    e->flops += r.flops;
    e->bytes += r.bytes;
  }
  *n = (int)agg.size();
  for (int i = 0; i < (int)agg.size() && i < cap; ++i) out[i] = agg[i];
  m->prof.recs.clear();
  m->prof.used = 0;
  return GPT_OK;
}

// ======================================================================== standalone ngram
extern "C" int ngram_hash(const int32_t* tokens, int B, int T, int vocab, unsigned long long p1,
                          unsigned long long p2, long long rows, int32_t* rows_out, void* stream) {
  if (!tokens || !rows_out || B < 0 || T < 0 || vocab < 1 || rows < 1 || rows > 0x7fffffffLL)
    return fail(GPT_ERR_ARG, "ngram_hash: bad argument");
  if ((long long)B * T == 0) return GPT_OK;
  unsigned* err = nullptr;
  CUDA_TRY(cudaGetSymbolAddress((void**)&err, g_ngram_err));
  ++g_launches; launch_pdl(ngram_hash_kernel, grid_for((long long)B * T, 256), 256, 0, (cudaStream_t)stream,
      tokens, B, T, vocab, p1, p2, rows, rows_out, 1, nullptr, err);
  LAUNCH_CHECK();
  return GPT_OK;
}

extern "C" int ngram_gather(const int32_t* rows, int n, const void* table, long long n_rows, int d, int dtype,
                            void* out, int accumulate, void* stream) {
  if (!rows || !table || !out || n < 0 || n_rows < 1 || d < 4 || d % 4 || d > 2048)
    return fail(GPT_ERR_ARG, "ngram_gather: bad argument (d must be a multiple of 4, <= 2048)");
  if (n == 0) return GPT_OK;
  unsigned* err = nullptr;
  CUDA_TRY(cudaGetSymbolAddress((void**)&err, g_ngram_err));
  const int grid = grid_for((long long)n * 32, 256);
  const bool vec16 = d % 8 == 0 && (reinterpret_cast<uintptr_t>(table) & 15) == 0 &&
                     (reinterpret_cast<uintptr_t>(out) & 15) == 0;
  if (dtype == GPT_DTYPE_BF16 && vec16) {
    // two rows a warp
    ++g_launches; launch_pdl(ngram_gather_bf16x8_kernel, grid_for((long long)(n + 1) / 2 * 32, 256), 256, 0, (cudaStream_t)stream, rows, n, (const bf16*)table, n_rows,
                                                                      d, (bf16*)out, accumulate, err);
  } else if (dtype == GPT_DTYPE_BF16) {
    ++g_launches; launch_pdl(ngram_gather_kernel<bf16>, grid, 256, 0, (cudaStream_t)stream, rows, n, (const bf16*)table, n_rows, d,
                                                                      (bf16*)out, accumulate, err);
  } else if (dtype == GPT_DTYPE_F32) {
    ++g_launches; launch_pdl(ngram_gather_kernel<float>, grid, 256, 0, (cudaStream_t)stream, rows, n, (const float*)table, n_rows, d,
                                                                       (float*)out, accumulate, err);
  } else {
    return fail(GPT_ERR_ARG, "ngram_gather: dtype must be F32 or BF16");
  }
  LAUNCH_CHECK();
  return GPT_OK;
}

struct NgramWsPlan {
  size_t ka, kb, va, vb, counts, part_head, part_tail, total;
};

static NgramWsPlan ngram_ws_plan(int n, int d) {
  NgramWsPlan w;
  Carver cv;
  const long long nchunks = ((long long)n + CHUNK - 1) / CHUNK;
  w.ka = cv.take((size_t)n * 4); w.kb = cv.take((size_t)n * 4);
  w.va = cv.take((size_t)n * 4); w.vb = cv.take((size_t)n * 4);
  w.counts = cv.take(256 * radix_blocks(n) * 4);
  w.part_head = cv.take(nchunks * (size_t)d * 4);
  w.part_tail = cv.take(nchunks * (size_t)d * 4);
  w.total = cv.take(0);
  return w;
}

extern "C" int ngram_sparse_update_workspace_bytes(int n, int d, size_t* bytes) {
  if (!bytes || n < 0 || d < 4) return fail(GPT_ERR_ARG, "ngram_sparse_update_workspace_bytes: bad argument");
  *bytes = ngram_ws_plan(n, d).total;
  return GPT_OK;
}

extern "C" int ngram_sparse_update(void* table, float* row_state, long long n_rows, int d, int dtype,
                                   const int32_t* rows, const float* grad, int n, float lr, float beta, float eps,
                                   int32_t* updated_rows_out, int* n_updated_out_dev, void* workspace,
                                   size_t ws_bytes, void* stream) {
  if (!table || !row_state || !rows || !grad || n < 0 || n_rows < 1 || n_rows > 0x7fffffffLL || d < 4 ||
      d % 4 || d > 2048)
    return fail(GPT_ERR_ARG, "ngram_sparse_update: bad argument (d must be a multiple of 4, <= 2048)");
  if (dtype != GPT_DTYPE_F32 && dtype != GPT_DTYPE_BF16) return fail(GPT_ERR_ARG, "ngram_sparse_update: bad dtype");
  if (n == 0) {
    if (n_updated_out_dev) CUDA_TRY(cudaMemsetAsync(n_updated_out_dev, 0, 4, (cudaStream_t)stream));
    return GPT_OK;
  }
  const NgramWsPlan pl = ngram_ws_plan(n, d);
  if (!workspace || ws_bytes < pl.total)
    return fail(GPT_ERR_WORKSPACE, "ngram_sparse_update: workspace %zu < %zu bytes", ws_bytes, pl.total);
  if (reinterpret_cast<uintptr_t>(workspace) & 255) return fail(GPT_ERR_ARG, "workspace not 256-byte aligned");
  uint8_t* b = static_cast<uint8_t*>(workspace);
  SortWs w;
  w.ka = (uint32_t*)(b + pl.ka); w.kb = (uint32_t*)(b + pl.kb);
  w.va = (int32_t*)(b + pl.va); w.vb = (int32_t*)(b + pl.vb);
  w.counts = (uint32_t*)(b + pl.counts);
  w.part_head = (float*)(b + pl.part_head); w.part_tail = (float*)(b + pl.part_tail);
  cudaStream_t st = (cudaStream_t)stream;
  // rows outside the table are rejected on the device before bucketing
  unsigned* err = nullptr;
  CUDA_TRY(cudaGetSymbolAddress((void**)&err, g_ngram_err));
  if (dtype == GPT_DTYPE_BF16)
    return table_update<bf16>(w, (bf16*)table, row_state, n_rows, d, rows, grad, n, lr, beta, eps,
                              updated_rows_out, n_updated_out_dev, err, st);
  return table_update<float>(w, (float*)table, row_state, n_rows, d, rows, grad, n, lr, beta, eps,
                             updated_rows_out, n_updated_out_dev, err, st);
}

extern "C" int ngram_sync_status(void* stream) {
  CUDA_TRY(cudaStreamSynchronize((cudaStream_t)stream));
  unsigned w = 0;
  CUDA_TRY(cudaMemcpyFromSymbol(&w, g_ngram_err, 4));
  if (w) {
    unsigned z = 0;
    CUDA_TRY(cudaMemcpyToSymbol(g_ngram_err, &z, 4));
  }
  if (w & GPT_EBIT_INPUT) return fail(GPT_ERR_INPUT, "row or token id out of range");
  if (w & GPT_EBIT_TIMEOUT) return fail(GPT_ERR_TIMEOUT, "a kernel's bounded wait gave up");
  return GPT_OK;
}

// ======================================================================== kernel-level test entry
// One thread waits, with the kernels' bounded-wait loop, on an mbarrier that
// nothing arrives on; when the limit passes it records a timeout and returns.
__global__ void wait_probe_kernel(unsigned long long limit_ns, unsigned* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  const uint64_t t0 = globaltimer_ns();
  while (!tc::mbar_try_wait(&bar, 0)) {
    if (globaltimer_ns() - t0 > limit_ns) {
      set_error(err, GPT_EBIT_TIMEOUT);
      return;
    }
  }
}

extern "C" int gptx_wait_probe(int limit_us, void* stream) {
  const long long us = limit_us < 1 ? 1 : (limit_us > 2000000 ? 2000000 : limit_us);
  unsigned* err = nullptr;
  CUDA_TRY(cudaGetSymbolAddress(reinterpret_cast<void**>(&err), g_ngram_err));
  ++g_launches;
  wait_probe_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((unsigned long long)us * 1000ull, err);
  LAUNCH_CHECK();
  return GPT_OK;
}

extern "C" int gptx_gemm_bf16(int M, int N, int K, const void* A, long long lda, int a_kmajor, const void* B,
                              long long ldb, int b_kmajor, int mode, void* C, long long ldc, const void* aux,
                              int beta, int splits, void* workspace, size_t ws_bytes, void* stream) {
  if (M < 1 || N < 1 || K < 1 || !A || !B || !C || ldc < N || mode < EPI_STORE || mode > EPI_LOGITS)
    return fail(GPT_ERR_ARG, "gptx_gemm_bf16: bad argument");
  if (mode == EPI_DRELU2 && !aux) return fail(GPT_ERR_ARG, "gptx_gemm_bf16: ReLU^2 backward needs aux");
  if (splits < 1) splits = 1;
  if (splits > 1 && (mode != EPI_ACCUM_F32 && mode != EPI_STORE_F32))
    return fail(GPT_ERR_ARG, "gptx_gemm_bf16: split-K only for fp32 outputs");
  if (splits > 1 && (!workspace || ws_bytes < (size_t)splits * M * N * 4))
    return fail(GPT_ERR_WORKSPACE, "gptx_gemm_bf16: split-K needs splits*M*N*4 bytes of workspace");
  const size_t stats_bytes = (size_t)M * cdiv(N, N >= 256 ? 128 : 64) * 8;
  if (mode == EPI_LOGITS && (!workspace || ws_bytes < stats_bytes + (aux ? (size_t)M * 4 : 0)))
    return fail(GPT_ERR_WORKSPACE,
                "gptx_gemm_bf16: logits need M*n_blocks*8 bytes of workspace for statistics (+ M*4 with targets)");
  unsigned* err = nullptr;
  CUDA_TRY(cudaGetSymbolAddress((void**)&err, g_ngram_err));
  GemmEpilogue e = epi(mode, C, ldc, beta, nullptr, mode == EPI_LOGITS ? nullptr : aux);
  if (mode == EPI_LOGITS) {
    e.stats = (float2*)workspace;
    e.targets = (const int32_t*)aux;
    e.ztgt = aux ? (float*)((uint8_t*)workspace + stats_bytes) : nullptr;
  }
  GemmOperand a{A, lda, a_kmajor ? 1 : 0}, b{B, ldb, b_kmajor ? 1 : 0};
  GemmCtx g{true, (float*)workspace, (long long)(ws_bytes / 4), err, (cudaStream_t)stream, nullptr};
  // the same tile shape the step would take for this shape
  const bool f32out = mode == EPI_ACCUM_F32 || mode == EPI_STORE_F32;
  if (N >= 256 && gemm_pairs_enabled())
    return gemm_tc_launch<256, 2>(M, N, K, a, b, e, splits, (float*)workspace, err, g.st);
  if (f32out && N >= 256 && tile_efficiency(M, N, 192, splits) > tile_efficiency(M, N, 256, splits) + 0.03)
    return gemm_tc_launch<192>(M, N, K, a, b, e, splits, (float*)workspace, err, g.st);
  if (N >= 256) return gemm_tc_launch<256>(M, N, K, a, b, e, splits, (float*)workspace, err, g.st);
  return gemm_tc_launch<128>(M, N, K, a, b, e, splits, (float*)workspace, err, g.st);
}

// ======================================================================== trigram statistics
extern "C" int trigram_tally_workspace_bytes(long long rows, int width, size_t* bytes) {
  if (!bytes || rows < 1 || width < 1) return fail(GPT_ERR_ARG, "trigram_tally_workspace_bytes: bad argument");
  *bytes = (size_t)rows * width * 4;
  return GPT_OK;
}

extern "C" int trigram_tally(const int32_t* streams, int S, int L, int vocab, unsigned long long p1,
                             unsigned long long p2, unsigned long long p3, long long rows, int width, int dtype,
                             void* table, void* workspace, size_t ws_bytes, void* stream) {
  if (!table || S < 0 || L < 0 || vocab < 1 || rows < 1 || rows > 0x7fffffffLL || width < 1 || width > 1024 ||
      (S > 0 && L > 0 && !streams))
    return fail(GPT_ERR_ARG, "trigram_tally: bad argument");
  if (dtype != GPT_DTYPE_F32 && dtype != GPT_DTYPE_BF16) return fail(GPT_ERR_ARG, "trigram_tally: bad dtype");
  const size_t need = (size_t)rows * width * 4;
  if (!workspace || ws_bytes < need) return fail(GPT_ERR_WORKSPACE, "trigram_tally: needs %zu bytes of workspace", need);
  if (reinterpret_cast<uintptr_t>(workspace) & 255) return fail(GPT_ERR_ARG, "workspace not 256-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  unsigned* err = nullptr;
  CUDA_TRY(cudaGetSymbolAddress((void**)&err, g_ngram_err));
  unsigned* counts = static_cast<unsigned*>(workspace);
  CUDA_TRY(cudaMemsetAsync(counts, 0, need, st));
  const long long npos = L > 1 ? (long long)S * (L - 1) : 0;
  if (npos > 0) {
    ++g_launches; trigram_count_kernel<<<grid_for(npos, 256), 256, 0, st>>>(streams, S, L, vocab, p1, p2, p3, rows,
                                                                           width, counts, err);
  }
  if (dtype == GPT_DTYPE_BF16) {
    ++g_launches; trigram_normalize_kernel<bf16><<<grid_for(rows * 32, 256), 256, 0, st>>>(counts, rows, width,
                                                                                           (bf16*)table);
  } else {
    ++g_launches; trigram_normalize_kernel<float><<<grid_for(rows * 32, 256), 256, 0, st>>>(counts, rows, width,
                                                                                            (float*)table);
  }
  LAUNCH_CHECK();
  return GPT_OK;
}

// ======================================================================== FP8 (e4m3) GEMM path
extern "C" int fp8_quantize_workspace_bytes(size_t* bytes) {
  if (!bytes) return fail(GPT_ERR_ARG, "fp8_quantize_workspace_bytes: null pointer");
  *bytes = FP8_AMAX_BLOCKS * 4;
  return GPT_OK;
}

extern "C" int fp8_quantize(const void* x, int dtype, long long n, uint8_t* q, float* scale, void* workspace,
                            size_t ws_bytes, void* stream) {
  if (!x || !q || !scale || n < 0 || (n & 1)) return fail(GPT_ERR_ARG, "fp8_quantize: bad argument (n even)");
  if (dtype != GPT_DTYPE_F32 && dtype != GPT_DTYPE_BF16) return fail(GPT_ERR_ARG, "fp8_quantize: bad dtype");
  if (!workspace || ws_bytes < (size_t)FP8_AMAX_BLOCKS * 4)
    return fail(GPT_ERR_WORKSPACE, "fp8_quantize: needs %d bytes of workspace", FP8_AMAX_BLOCKS * 4);
  cudaStream_t st = (cudaStream_t)stream;
  float* part = static_cast<float*>(workspace);
  const unsigned qgrid = (unsigned)std::max<long long>(1, std::min<long long>((n / 2 + 255) / 256, 8LL * device_sms()));
  if (dtype == GPT_DTYPE_BF16) {
    ++g_launches; fp8_amax_kernel<bf16><<<FP8_AMAX_BLOCKS, 256, 0, st>>>((const bf16*)x, n, part);
    ++g_launches; fp8_quantize_kernel<bf16><<<qgrid, 256, 0, st>>>((const bf16*)x, n, part, q, scale);
  } else {
    ++g_launches; fp8_amax_kernel<float><<<FP8_AMAX_BLOCKS, 256, 0, st>>>((const float*)x, n, part);
    ++g_launches; fp8_quantize_kernel<float><<<qgrid, 256, 0, st>>>((const float*)x, n, part, q, scale);
  }
  LAUNCH_CHECK();
  return GPT_OK;
}

extern "C" int gptx_gemm_fp8(int M, int N, int K, const uint8_t* A, long long lda, const uint8_t* B, long long ldb,
                             const float* scale_a, const float* scale_b, int out_dtype, void* C, long long ldc,
                             void* stream) {
  if (M < 1 || N < 1 || K < 1 || !A || !B || !C || !scale_a || !scale_b || ldc < N || lda < K || ldb < K)
    return fail(GPT_ERR_ARG, "gptx_gemm_fp8: bad argument");
  if ((lda | ldb) & 15) return fail(GPT_ERR_ARG, "gptx_gemm_fp8: row pitches must be multiples of 16 bytes");
  if (out_dtype != GPT_DTYPE_F32 && out_dtype != GPT_DTYPE_BF16) return fail(GPT_ERR_ARG, "gptx_gemm_fp8: bad out_dtype");
  unsigned* err = nullptr;
  CUDA_TRY(cudaGetSymbolAddress((void**)&err, g_ngram_err));
  GemmEpilogue e = epi(out_dtype == GPT_DTYPE_F32 ? EPI_STORE_F32 : EPI_STORE, C, ldc);
  e.scale_a = scale_a;
  e.scale_b = scale_b;
  if (gemm_pairs_enabled()) return gemm_f8_launch<2>(M, N, K, A, lda, B, ldb, e, err, (cudaStream_t)stream);
  return gemm_f8_launch<1>(M, N, K, A, lda, B, ldb, e, err, (cudaStream_t)stream);
}

// ======================================================================== Muon
// Byte offsets of muon_update's scratch inside the caller's workspace.
struct MuonWs {
  size_t x, xn, abf, bm, a, aa, p, partials, splitk, total;
  long long splitk_elems;
};

static MuonWs muon_ws_plan(int rows, int cols) {
  const long long n = (long long)rows * cols, R = rows < cols ? rows : cols;
  Carver cv;
  MuonWs w;
  w.x = cv.take(n * 2);        // X (bf16), the iterate
  w.xn = cv.take(n * 2);       // its successor
  w.abf = cv.take(R * R * 2);  // A = X X^T (or X^T X) as the bf16 operand of A A
  w.bm = cv.take(R * R * 2);   // B = b A + c A A (bf16)
  w.a = cv.take(R * R * 4);    // A (fp32 GEMM output)
  w.aa = cv.take(R * R * 4);   // A A (fp32)
  w.p = cv.take(n * 4);        // B X (or X B) (fp32)
  w.partials = cv.take((size_t)MUON_NORM_BLOCKS * 4);
  w.splitk_elems = 4 * R * R;  // split-K partials of the two R x R products
  w.splitk = cv.take((size_t)w.splitk_elems * 4);
  w.total = cv.off + 256;      // + slack to align the caller's base to 256 bytes
  return w;
}

extern "C" int muon_update_workspace_bytes(int rows, int cols, size_t* bytes) {
  if (!bytes || rows < 8 || cols < 8 || rows % 8 || cols % 8)
    return fail(GPT_ERR_ARG, "muon_update_workspace_bytes: rows and cols must be positive multiples of 8");
  *bytes = muon_ws_plan(rows, cols).total;
  return GPT_OK;
}

extern "C" int muon_update(float* W, float* M, const float* G, int rows, int cols, int out_rows, float lr,
                           float momentum, int nesterov, int ns_steps, void* workspace, size_t ws_bytes,
                           void* stream) {
  if (!W || !M || !G || rows < 8 || cols < 8 || rows % 8 || cols % 8 || ns_steps < 0 || ns_steps > 64 ||
      !(momentum >= 0.f && momentum < 1.f))
    return fail(GPT_ERR_ARG, "muon_update: bad argument (rows, cols multiples of 8; 0 <= momentum < 1; "
                             "0 <= ns_steps <= 64)");
  if ((reinterpret_cast<uintptr_t>(W) | reinterpret_cast<uintptr_t>(M) | reinterpret_cast<uintptr_t>(G)) & 15)
    return fail(GPT_ERR_ARG, "muon_update: W, M and G must be 16-byte aligned");
  const MuonWs p = muon_ws_plan(rows, cols);
  if (!workspace || ws_bytes < p.total)
    return fail(GPT_ERR_WORKSPACE, "muon_update: needs %zu bytes of workspace", p.total);
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(workspace) + 255) & ~uintptr_t(255));
  bf16* x = reinterpret_cast<bf16*>(base + p.x);
  bf16* xn = reinterpret_cast<bf16*>(base + p.xn);
  bf16* abf = reinterpret_cast<bf16*>(base + p.abf);
  bf16* bm = reinterpret_cast<bf16*>(base + p.bm);
  float* A = reinterpret_cast<float*>(base + p.a);
  float* AA = reinterpret_cast<float*>(base + p.aa);
  float* P = reinterpret_cast<float*>(base + p.p);
  float* partials = reinterpret_cast<float*>(base + p.partials);
  float* splitk = reinterpret_cast<float*>(base + p.splitk);
  unsigned* err = nullptr;
  CUDA_TRY(cudaGetSymbolAddress((void**)&err, g_ngram_err));
  cudaStream_t st = (cudaStream_t)stream;
  const long long n4 = (long long)rows * cols / 4;
  const int R = rows < cols ? rows : cols;
  const long long r4 = (long long)R * R / 4;
  const bool tall = rows > cols;  // iterate as X^T X and X B: the small R x R products either way
  auto grid = [](long long n) { const long long b = (n + MUON_THREADS - 1) / MUON_THREADS, cap = 4LL * device_sms();
                                return (unsigned)(b < 1 ? 1 : (b > cap ? cap : b)); };
  ++g_launches;
  muon_momentum_kernel<<<MUON_NORM_BLOCKS, MUON_THREADS, 0, st>>>(G, M, n4, momentum, nesterov, partials);
  ++g_launches;
  muon_normalize_kernel<<<grid(n4), MUON_THREADS, 0, st>>>(G, M, n4, momentum, nesterov, partials,
                                                            MUON_NORM_BLOCKS, 1e-7f, x);
  LAUNCH_CHECK();
  const GemmCtx g{true, splitk, p.splitk_elems, err, st, nullptr};
  const float ca = 3.4445f, cb = -4.7750f, cc = 2.0315f;  // a x + b x^3 + c x^5
  for (int it = 0; it < ns_steps; ++it) {
    if (!tall) TRY(gemm(g, R, R, cols, op_k(x, cols), op_k(x, cols), epi(EPI_STORE_F32, A, R), true, "muon.gram"));
    else TRY(gemm(g, R, R, rows, op_mn(x, cols), op_mn(x, cols), epi(EPI_STORE_F32, A, R), true, "muon.gram"));
    ++g_launches;
    muon_to_bf16_kernel<<<grid(r4), MUON_THREADS, 0, st>>>(A, r4, abf);
    TRY(gemm(g, R, R, R, op_k(abf, R), op_mn(abf, R), epi(EPI_STORE_F32, AA, R), true, "muon.square"));
    ++g_launches;
    muon_combine_kernel<<<grid(r4), MUON_THREADS, 0, st>>>(abf, AA, r4, cb, cc, bm);
    if (!tall) TRY(gemm(g, rows, cols, R, op_k(bm, R), op_mn(x, cols), epi(EPI_STORE_F32, P, cols), false, "muon.poly"));
    else TRY(gemm(g, rows, cols, R, op_k(x, cols), op_mn(bm, R), epi(EPI_STORE_F32, P, cols), false, "muon.poly"));
    ++g_launches;
    muon_combine_kernel<<<grid(n4), MUON_THREADS, 0, st>>>(x, P, n4, ca, 1.f, xn);
    LAUNCH_CHECK();
    bf16* t = x; x = xn; xn = t;
  }
  const double out_dim = out_rows ? rows : cols, in_dim = out_rows ? cols : rows;
  const float step = (float)(lr * std::sqrt(std::max(1.0, out_dim / in_dim)));
  ++g_launches;
  muon_apply_kernel<<<grid(n4), MUON_THREADS, 0, st>>>(W, x, n4, step);
  LAUNCH_CHECK();
  return GPT_OK;
}

// ======================================================================== allocation-free table update
// Scratch for ngram_sparse_update_noalloc: a fixed array in the library's own
// device image, so the entry point never asks for device memory.  Every GPU
// that loads the library holds these bytes until the process exits.  All
// calls share it; each call writes every scratch byte it later reads, so
// nothing has to start at zero.
#define GPT_NOALLOC_SCRATCH_BYTES (16u << 20)
static __device__ __align__(256) unsigned char g_noalloc_scratch[GPT_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch per device.  In host code the symbol
// itself is only a host-side stand-in, so the address is looked up with the
// device current, once, the first time the device is used.
static std::atomic<void*> g_noalloc_addr[128];

extern "C" int ngram_sparse_update_noalloc(void* table, float* row_state, long long n_rows, int d, int dtype,
                                           const int32_t* rows, const float* grad, int n, float lr, float beta,
                                           float eps, int32_t* updated_rows_out, int* n_updated_out_dev,
                                           void* stream) {
  if (n < 0 || d < 4) return fail(GPT_ERR_ARG, "ngram_sparse_update_noalloc: bad argument");
  const size_t need = ngram_ws_plan(n, d).total;
  if (need > GPT_NOALLOC_SCRATCH_BYTES)
    return fail(GPT_ERR_WORKSPACE,
                "ngram_sparse_update_noalloc: n = %d positions of width d = %d need %zu bytes of scratch, "
                "more than the %u-byte built-in buffer; use ngram_sparse_update with a workspace",
                n, d, need, (unsigned)GPT_NOALLOC_SCRATCH_BYTES);
  // the scratch address and the launches belong to the device that owns the stream
  int cur = 0, dev = 0;
  CUDA_TRY(cudaGetDevice(&cur));
  CUDA_TRY(cudaStreamGetDevice((cudaStream_t)stream, &dev));
  if (dev < 0 || dev >= 128) return fail(GPT_ERR_ARG, "ngram_sparse_update_noalloc: device index %d out of range", dev);
  if (dev != cur) CUDA_TRY(cudaSetDevice(dev));
  void* scratch = g_noalloc_addr[dev].load();
  cudaError_t e = cudaSuccess;
  if (!scratch) {
    e = cudaGetSymbolAddress(&scratch, g_noalloc_scratch);
    if (e == cudaSuccess) g_noalloc_addr[dev].store(scratch);
  }
  const int s = e != cudaSuccess
                    ? fail(GPT_ERR_CUDA, "cudaGetSymbolAddress(g_noalloc_scratch): %s", cudaGetErrorString(e))
                    : ngram_sparse_update(table, row_state, n_rows, d, dtype, rows, grad, n, lr, beta, eps,
                                          updated_rows_out, n_updated_out_dev, scratch, GPT_NOALLOC_SCRATCH_BYTES,
                                          stream);
  if (dev != cur) CUDA_TRY(cudaSetDevice(cur));
  return s;
}
