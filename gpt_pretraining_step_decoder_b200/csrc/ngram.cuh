// ngram.cuh -- hashed bigram tables: hash, row gather, atomics-free bucketing
// of positions by row, and the sparse per-row-magnitude update fused with the
// gradient segment-sum (decoder-rtx posts: "Two huge bi-gram hash tables",
// "inlined the optimizer in their backward math", "sparse, no first moment,
// and only per-row magnitude").
//
// Bucketing: positions are sorted by row with a stable LSD radix sort (8-bit
// digits, two launches a digit: per-tile histograms, then a stable scatter
// whose blocks derive their own global offsets from the histograms and rank
// equal digits with warp match masks).  The first pass reads the caller's
// int32 rows directly.  No atomics anywhere, so sums are formed in position
// order and results are bit-reproducible.
//
// Update: the sorted positions are cut into fixed chunks of 16; one block owns
// a chunk (each thread four columns of every row), its warps find the runs of
// equal rows in it with ballots.  A run that lies inside the chunk is finished
// by that block (sum -> mean square -> row state -> row update).  A run that
// crosses chunk boundaries leaves one partial sum per chunk it touches; a
// second launch adds those partials in a grouping fixed by the run's length
// (chunk order for short runs, contiguous shares for long ones) and finishes
// the row.  Every row has exactly one writer.  (The token-embedding gradient
// uses the same bucketing with one warp per chunk.)
#pragma once
#include "common.cuh"
#include "layers.cuh"

constexpr int RADIX_THREADS = 256;
constexpr int RADIX_MAX_ITEMS = 8;   // keys per thread per block, at most
constexpr int RADIX_FUSED_MAX_BLOCKS = 256;  // above this, offsets come from a scan launch
constexpr int CHUNK = 16;            // sorted positions per warp in the update (<= 32)

// keys per thread so that a sort of n keys runs on about 96 blocks (or on
// as many 2048-key tiles as it needs beyond that; measured on B200, 192
// blocks of fewer keys are no faster)
static inline int radix_items(long long n) {
  int it = 1;
  while (it < RADIX_MAX_ITEMS && (n + (long long)RADIX_THREADS * it - 1) / ((long long)RADIX_THREADS * it) > 96) it <<= 1;
  return it;
}
static inline long long radix_blocks(long long n) {
  const long long tile = (long long)RADIX_THREADS * radix_items(n);
  return (n + tile - 1) / tile;
}

// ---------------------------------------------------------------- hash
// key = (a*p1 mod 2^64) XOR (c*p2 mod 2^64), a = tokens[t-1] (vocab at t = 0)
__global__ void ngram_hash_kernel(const int32_t* __restrict__ tok, int B, int T, int V,
                                  unsigned long long p1, unsigned long long p2, long long rows_a,
                                  int32_t* __restrict__ out_a, long long rows_b,
                                  int32_t* __restrict__ out_b, unsigned* err) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  const long long n = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= (long long)B * T) return;
  const int t = (int)(n % T);
  int c = tok[n];
  int a = (t > 0) ? tok[n - 1] : V;
  if (c < 0 || c >= V || a < 0 || a > V) {
    set_error(err, GPT_EBIT_INPUT);
    if (out_a) out_a[n] = 0;
    if (out_b) out_b[n] = 0;
    return;
  }
  const unsigned long long key = ((unsigned long long)a * p1) ^ ((unsigned long long)c * p2);
  if (out_a) out_a[n] = (int32_t)(key % (unsigned long long)rows_a);
  if (out_b) out_b[n] = (int32_t)(key % (unsigned long long)rows_b);
}

// ---------------------------------------------------------------- gather
template <typename tab_t>
__global__ void ngram_gather_kernel(const int32_t* __restrict__ rows, int n,
                                    const tab_t* __restrict__ table, long long n_rows, int d,
                                    tab_t* __restrict__ out, int accumulate, unsigned* err) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= n) return;
  const long long r = rows[warp];
  if (r < 0 || r >= n_rows) {
    if (lane == 0) set_error(err, GPT_EBIT_INPUT);
    return;
  }
  for (int c = lane * 4; c < d; c += 128) {
    float v[4], o[4];
    load4(table + r * d + c, v);
    if (accumulate) {
      load4(out + (long long)warp * d + c, o);
      v[0] += o[0]; v[1] += o[1]; v[2] += o[2]; v[3] += o[3];
    }
    store4(out + (long long)warp * d + c, v);
  }
}


// bf16 rows with d % 8 == 0 and 16-byte aligned buffers: 16-byte accesses
// (8 values per lane), the row copied as raw bits unless accumulating.
__global__ void ngram_gather_bf16x8_kernel(const int32_t* __restrict__ rows, int n,
                                           const bf16* __restrict__ table, long long n_rows, int d,
                                           bf16* __restrict__ out, int accumulate, unsigned* err) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  // two rows a warp, both rows' loads in flight before any store (a short
  // call is bound by how much a warp has in flight, not by its instructions)
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int i0 = 2 * warp;
  if (i0 >= n) return;
  const int nr = min(2, n - i0);
  long long r[2] = {0, 0};
  bool ok[2] = {false, false};
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    if (u < nr) {
      r[u] = rows[i0 + u];
      ok[u] = r[u] >= 0 && r[u] < n_rows;
      if (!ok[u] && lane == 0) set_error(err, GPT_EBIT_INPUT);
    }
  }
  const int nc = d / 8;
  for (int c0 = 0; c0 < nc; c0 += 32 * 4) {
    uint4 v[2][4];
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int c = c0 + lane + 32 * k;
        if (ok[u] && c < nc) v[u][k] = __ldg(reinterpret_cast<const uint4*>(table + r[u] * d) + c);
      }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (!ok[u]) continue;
      uint4* dst = reinterpret_cast<uint4*>(out + (long long)(i0 + u) * d);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int c = c0 + lane + 32 * k;
        if (c >= nc) continue;
        uint4 x = v[u][k];
        if (accumulate) {
          const uint4 o = dst[c];
          const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&x);
          const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&o);
          uint4 sum;
          __nv_bfloat162* s2 = reinterpret_cast<__nv_bfloat162*>(&sum);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 xa = __bfloat1622float2(a2[i]), ya = __bfloat1622float2(o2[i]);
            s2[i] = __floats2bfloat162_rn(xa.x + ya.x, xa.y + ya.y);
          }
          x = sum;
        }
        dst[c] = x;
      }
    }
  }
}

// ---------------------------------------------------------------- radix sort
// Keys are row ids in [0, key_range).  The first pass reads the caller's
// int32 rows; an id outside the range sets the error word and is sorted as
// key_range itself with position -1.  Those form one run past every real
// row, which every consumer skips, so no out-of-range row is ever read or
// written.  (The digit passes therefore cover the value key_range.)
__device__ __forceinline__ uint32_t radix_key(const uint32_t* __restrict__ keys, const int32_t* __restrict__ raw,
                                              long long idx, long long key_range, bool& ok) {
  if (raw == nullptr) { ok = true; return keys[idx]; }
  const int32_t k = raw[idx];
  ok = k >= 0 && (long long)k < key_range;
  return ok ? (uint32_t)k : (uint32_t)key_range;
}

// counts layout: block-major [nblocks][256]
__global__ void __launch_bounds__(RADIX_THREADS) radix_hist_kernel(const uint32_t* __restrict__ keys,
                                                                  const int32_t* __restrict__ raw, int n,
                                                                  long long key_range, int items, int shift,
                                                                  uint32_t* __restrict__ counts) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  constexpr int NW = RADIX_THREADS / 32;
  __shared__ uint32_t wh[NW][256];  // per-warp digit counts
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < NW * 256; i += RADIX_THREADS) (&wh[0][0])[i] = 0;
  __syncthreads();
  const long long base = (long long)blockIdx.x * RADIX_THREADS * items;
  const uint32_t lt = (1u << lane) - 1u;
  // all of the tile's keys are requested before any is counted
  uint32_t dg[RADIX_MAX_ITEMS];
#pragma unroll
  for (int round = 0; round < RADIX_MAX_ITEMS; ++round) {
    const long long idx = base + (long long)round * RADIX_THREADS + threadIdx.x;
    dg[round] = 256u;
    if (round < items && idx < n) {
      bool ok;
      dg[round] = (radix_key(keys, raw, idx, key_range, ok) >> shift) & 255u;
    }
  }
#pragma unroll
  for (int round = 0; round < RADIX_MAX_ITEMS; ++round) {
    if (round >= items) break;
    const uint32_t dgt = dg[round];
    const uint32_t peers = __match_any_sync(0xffffffffu, dgt);
    // the lowest lane of each digit group adds the group's size: one writer
    // per (warp, digit), so no atomics are needed
    if (dgt < 256u && (peers & lt) == 0) wh[w][dgt] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  uint32_t s = 0;
  for (int ww = 0; ww < NW; ++ww) s += wh[ww][threadIdx.x];
  counts[(long long)blockIdx.x * 256 + threadIdx.x] = s;
}

// For many blocks: replace every count by its stable global offset (the
// exclusive scan of the counts taken digit-major: all blocks of digit 0, then
// digit 1, ...).  One block; each thread scans a contiguous stretch.
__global__ void __launch_bounds__(1024) radix_offsets_kernel(uint32_t* __restrict__ counts, int nblk) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  __shared__ uint32_t sh[1024];
  const long long n = 256LL * nblk;
  const long long per = (n + 1023) / 1024;
  const long long beg = threadIdx.x * per, end = beg + per < n ? beg + per : n;
  uint32_t local = 0;
  for (long long i = beg; i < end; ++i) local += counts[(i % nblk) * 256 + i / nblk];
  sh[threadIdx.x] = local;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    const uint32_t v = (threadIdx.x >= off) ? sh[threadIdx.x - off] : 0;
    __syncthreads();
    sh[threadIdx.x] += v;
    __syncthreads();
  }
  uint32_t run = sh[threadIdx.x] - local;
  for (long long i = beg; i < end; ++i) {
    uint32_t& c = counts[(i % nblk) * 256 + i / nblk];
    const uint32_t v = c;
    c = run;
    run += v;
  }
}

// Stable scatter.  Element order within a tile is idx = base + round*256 +
// tid; ranks among equal digits follow that order (warp match masks inside a
// warp, per-warp digit counts across warps, running totals across rounds).
// With `scanned` == 0 each block first derives its global offsets from the
// histograms: offset(digit, b) = sum of all blocks' counts of smaller digits
// + sum of counts of this digit in blocks before b.
__global__ void __launch_bounds__(RADIX_THREADS) radix_scatter_kernel(
    const uint32_t* __restrict__ keys_in, const int32_t* __restrict__ vals_in, const int32_t* __restrict__ raw,
    int n, long long key_range, int items, int shift, const uint32_t* __restrict__ counts, int scanned,
    uint32_t* __restrict__ keys_out, int32_t* __restrict__ vals_out, unsigned* err) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  constexpr int NW = RADIX_THREADS / 32;
  __shared__ uint32_t wcount[NW][256];
  __shared__ uint32_t running[256];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  if (scanned) {
    running[threadIdx.x] = counts[(long long)blockIdx.x * 256 + threadIdx.x];
  } else {
    uint32_t total = 0, before = 0;
    for (int b = 0; b < (int)gridDim.x; ++b) {
      const uint32_t c = counts[(long long)b * 256 + threadIdx.x];
      total += c;
      if (b < (int)blockIdx.x) before += c;
    }
    // exclusive scan of the per-digit totals over the 256 threads
    uint32_t incl = total;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    if (lane == 31) wcount[0][w] = incl;
    __syncthreads();
    uint32_t wbase = 0;
    for (int ww = 0; ww < w; ++ww) wbase += wcount[0][ww];
    running[threadIdx.x] = wbase + incl - total + before;
  }
  const long long base = (long long)blockIdx.x * RADIX_THREADS * items;
  // all of the tile's keys and values are requested before any is ranked
  uint32_t kk[RADIX_MAX_ITEMS];
  int32_t vv[RADIX_MAX_ITEMS];
#pragma unroll
  for (int round = 0; round < RADIX_MAX_ITEMS; ++round) {
    const long long idx = base + (long long)round * RADIX_THREADS + threadIdx.x;
    kk[round] = 0;
    vv[round] = 0;
    if (round < items && idx < n) {
      bool ok;
      kk[round] = radix_key(keys_in, raw, idx, key_range, ok);
      if (raw != nullptr) {
        vv[round] = ok ? (int32_t)idx : -1;
        if (!ok) set_error(err, GPT_EBIT_INPUT);
      } else {
        vv[round] = vals_in[idx];
      }
    }
  }
#pragma unroll
  for (int round = 0; round < RADIX_MAX_ITEMS; ++round) {
    if (round >= items) break;
    __syncthreads();
    for (int i = threadIdx.x; i < NW * 256; i += RADIX_THREADS) (&wcount[0][0])[i] = 0;
    __syncthreads();
    const long long idx = base + (long long)round * RADIX_THREADS + threadIdx.x;
    const bool valid = idx < n;
    const uint32_t key = kk[round];
    const int32_t val = vv[round];
    const uint32_t dgt = valid ? (key >> shift) & 255u : 256u;  // 256 = no digit (invalid lane)
    const uint32_t peers = __match_any_sync(0xffffffffu, dgt);
    const uint32_t lt = (1u << lane) - 1u;
    const uint32_t rank_in_warp = __popc(peers & lt);
    if (valid && rank_in_warp == 0) wcount[w][dgt] = __popc(peers);
    __syncthreads();
    if (valid) {
      uint32_t before = 0;
      for (int ww = 0; ww < w; ++ww) before += wcount[ww][dgt];
      const uint32_t pos = running[dgt] + before + rank_in_warp;
      keys_out[pos] = key;
      vals_out[pos] = val;
    }
    __syncthreads();
    {
      uint32_t tot = 0;
      for (int ww = 0; ww < NW; ++ww) tot += wcount[ww][threadIdx.x];
      running[threadIdx.x] += tot;
    }
  }
}

// Distinct sorted keys in ascending order and their number (one block; only
// for callers that ask for the updated-row list).
__global__ void __launch_bounds__(1024) unique_keys_kernel(const uint32_t* __restrict__ skeys, int n,
                                                           long long key_range, int32_t* __restrict__ uniq_out,
                                                           int* __restrict__ n_uniq_out) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  __shared__ int sh[1024];
  const int per = (n + 1023) / 1024;
  const int beg = threadIdx.x * per, end = min(beg + per, n);
  int heads = 0;
  for (int i = beg; i < end; ++i) heads += ((i == 0 || skeys[i] != skeys[i - 1]) && skeys[i] < key_range);
  sh[threadIdx.x] = heads;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    const int v = (threadIdx.x >= off) ? sh[threadIdx.x - off] : 0;
    __syncthreads();
    sh[threadIdx.x] += v;
    __syncthreads();
  }
  int sid = sh[threadIdx.x] - heads;
  if (uniq_out)
    for (int i = beg; i < end; ++i)
      if ((i == 0 || skeys[i] != skeys[i - 1]) && skeys[i] < key_range) uniq_out[sid++] = (int32_t)skeys[i];
  if (threadIdx.x == 1023 && n_uniq_out) *n_uniq_out = sh[1023];
}

// ---------------------------------------------------------------- runs in a chunk
// One warp, chunk c = sorted positions [CHUNK*c, CHUNK*c + len).  Lane l holds the
// l-th key and position.  start_mask / end_mask mark the lanes where a run of
// equal keys starts / ends inside the chunk (lane 0 always starts one, lane
// len-1 always ends one); cont_in: the chunk's first run began in an earlier
// chunk; cont_out: its last run goes on into the next chunk.
struct ChunkRuns {
  uint32_t key;
  int32_t pos;
  unsigned start_mask, end_mask;
  int len;
  bool cont_in, cont_out;
};

__device__ __forceinline__ ChunkRuns chunk_runs(const uint32_t* __restrict__ skeys, const int32_t* __restrict__ perm,
                                                int n, int c) {
  const int lane = threadIdx.x & 31;
  const long long base = (long long)c * CHUNK;
  ChunkRuns r;
  r.len = (int)min((long long)CHUNK, n - base);
  const bool valid = lane < r.len;
  r.key = valid ? skeys[base + lane] : 0xffffffffu;
  r.pos = valid ? perm[base + lane] : -1;
  const uint32_t up = __shfl_up_sync(0xffffffffu, r.key, 1);
  const uint32_t dn = __shfl_down_sync(0xffffffffu, r.key, 1);
  r.start_mask = __ballot_sync(0xffffffffu, valid && (lane == 0 || up != r.key));
  r.end_mask = __ballot_sync(0xffffffffu, valid && (lane == r.len - 1 || dn != r.key));
  const uint32_t first = __shfl_sync(0xffffffffu, r.key, 0);
  const uint32_t last = __shfl_sync(0xffffffffu, r.key, r.len - 1);
  r.cont_in = c > 0 && skeys[base - 1] == first;
  r.cont_out = base + CHUNK < n && skeys[base + CHUNK] == last;
  return r;
}

// What the warp does with the run that ends at lane q.
enum RunKind { RUN_WHOLE = 0, RUN_TAIL = 1, RUN_HEAD = 2 };
__device__ __forceinline__ int run_kind(const ChunkRuns& r, int q) {
  const unsigned upto = (q == 31) ? 0xffffffffu : ((2u << q) - 1u);
  const int s = 31 - __clz(r.start_mask & upto);
  if (s == 0 && r.cont_in) return RUN_TAIL;             // continues a run from before
  if (q == r.len - 1 && r.cont_out) return RUN_HEAD;    // starts a run that goes on
  return RUN_WHOLE;
}

// Chunk c starts a run that goes on into later chunks: returns its key and
// the last chunk it reaches, else false.  Called by whole warps: the end of
// the run is found by a 32-way search over the sorted keys (a few rounds of
// one load per lane instead of one dependent load per chunk of a long run).
__device__ __forceinline__ bool chained_run(const uint32_t* __restrict__ skeys, int n, int c, uint32_t& key,
                                            int& last_chunk) {
  const long long base = (long long)c * CHUNK;
  if (base + CHUNK >= n) return false;
  key = skeys[base + CHUNK - 1];
  if (skeys[base + CHUNK] != key) return false;
  if (c > 0 && skeys[base - 1] == key) return false;
  // first index with a different key lies in (lo, hi]; skeys[lo] == key
  const int lane = threadIdx.x & 31;
  long long lo = base + CHUNK, hi = n;
  while (hi - lo > 1) {
    const long long step = (hi - lo + 31) / 32;
    const long long probe = lo + (long long)(lane + 1) * step;
    const bool same = probe < hi && skeys[probe] == key;
    const int cnt = __popc(__ballot_sync(0xffffffffu, same));  // keys sorted: a prefix of the lanes
    const long long nlo = lo + (long long)cnt * step;
    const long long nhi = lo + (long long)(cnt + 1) * step;
    lo = nlo;
    if (nhi < hi) hi = nhi;
  }
  last_chunk = (int)((hi - 1) / CHUNK);
  return true;
}

// Four table values per lane in their storage type (8 bytes for bf16), so a
// prefetched row costs half the registers of its fp32 copy.
template <typename T> struct Raw4;
template <> struct Raw4<float> {
  using type = float4;
  static __device__ __forceinline__ void unpack(const type& r, float v[4]) { v[0] = r.x; v[1] = r.y; v[2] = r.z; v[3] = r.w; }
  static __device__ __forceinline__ type pack(const float v[4]) { return make_float4(v[0], v[1], v[2], v[3]); }
};
template <> struct Raw4<bf16> {
  using type = uint2;
  static __device__ __forceinline__ void unpack(const type& r, float v[4]) {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.y));
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
  }
  static __device__ __forceinline__ type pack(const float v[4]) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
    return make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
  }
};

template <int NV, typename T>
__device__ __forceinline__ void load_raw_row(const T* __restrict__ src, int d, typename Raw4<T>::type (&v)[NV]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int c = (j * 32 + lane) * 4;
    if (c < d) v[j] = *reinterpret_cast<const typename Raw4<T>::type*>(src + c);
  }
}

// ---------------------------------------------------------------- row update
// Apply the per-row-magnitude step to one row with its summed gradient G
// (held by the warp, 4 values per lane per 128 columns): m = mean(G^2),
// s <- beta*s + (1-beta)*m, W <- W - lr*G/(sqrt(s) + eps).  w holds the old
// row, s_old the old state.
template <int NV, typename tab_t>
__device__ __forceinline__ void table_row_apply(tab_t* __restrict__ table, float* __restrict__ state,
                                                long long r, int d, const float (&G)[NV][4],
                                                const typename Raw4<tab_t>::type (&w)[NV], float s_old,
                                                float lr, float beta, float eps) {
  const int lane = threadIdx.x & 31;
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int c = (j * 32 + lane) * 4;
    if (c < d) ss += G[j][0] * G[j][0] + G[j][1] * G[j][1] + G[j][2] * G[j][2] + G[j][3] * G[j][3];
  }
  ss = warp_sum(ss);
  const float s_new = beta * s_old + (1.f - beta) * (ss / d);
  const float step = lr / (sqrtf(s_new) + eps);
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int c = (j * 32 + lane) * 4;
    if (c < d) {
      float x[4];
      Raw4<tab_t>::unpack(w[j], x);
#pragma unroll
      for (int i = 0; i < 4; ++i) x[i] -= step * G[j][i];
      *reinterpret_cast<typename Raw4<tab_t>::type*>(table + r * d + c) = Raw4<tab_t>::pack(x);
    }
  }
  if (lane == 0) state[r] = s_new;
}

template <int NV, typename T>
__device__ __forceinline__ void load_row(const T* __restrict__ src, int d, float (&v)[NV][4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int c = (j * 32 + lane) * 4;
    if (c < d) load4(src + c, v[j]);
    else v[j][0] = v[j][1] = v[j][2] = v[j][3] = 0.f;
  }
}

template <int NV>
__device__ __forceinline__ void store_row(float* __restrict__ dst, int d, const float (&v)[NV][4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int c = (j * 32 + lane) * 4;
    if (c < d) store4(dst + c, v[j]);
  }
}

template <int NV>
__device__ __forceinline__ void zero_row(float (&v)[NV][4]) {
#pragma unroll
  for (int j = 0; j < NV; ++j) v[j][0] = v[j][1] = v[j][2] = v[j][3] = 0.f;
}

template <int NV>
__device__ __forceinline__ void add_row(float (&a)[NV][4], const float (&b)[NV][4]) {
#pragma unroll
  for (int j = 0; j < NV; ++j)
#pragma unroll
    for (int i = 0; i < 4; ++i) a[j][i] += b[j][i];
}

// Sum of each of 16 values over the 32 lanes of a warp in 16 shuffles (a
// butterfly that halves the list at every step instead of 16 separate
// reductions).  On return lane l holds the total of value (l >> 1) & 15; the
// grouping is fixed, so the result is reproducible.
__device__ __forceinline__ float warp_sum16(float (&v)[16]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int h = 8; h >= 1; h >>= 1) {
    const bool hi = (lane >> 1) & h;  // bit of the lane that picks the kept half
#pragma unroll
    for (int i = 0; i < h; ++i) {
      const float keep = hi ? v[i + h] : v[i], give = hi ? v[i] : v[i + h];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, give, 2 * h);
    }
  }
  return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
}

// Asynchronous global -> shared copies of one thread's own values (Ampere-style
// cp.async): the data lands in shared memory without holding registers while
// in flight, and after the wait the issuing thread reads it back itself.
template <int BYTES>
__device__ __forceinline__ void cp_async_own(void* dst, const void* src) {
  static_assert(BYTES == 8 || BYTES == 16, "cp.async size");
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  if constexpr (BYTES == 16)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_own() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Dynamic shared memory of table_chunk_kernel for a block of nt threads.
template <typename tab_t>
static inline size_t table_chunk_smem(int nt, bool stage_rows) {
  return (size_t)CHUNK * nt * (sizeof(float4) + (stage_rows ? sizeof(typename Raw4<tab_t>::type) : 0));
}

// One block per chunk of CHUNK sorted positions; thread t owns columns
// [4t, 4t + 4) of every row, so a block has d / 4 threads rounded up to whole
// warps (at most MAXT).  Every gradient value of the chunk and (STAGE_ROWS)
// the table values of the rows whose runs end inside it are requested into
// shared memory before any is used: a chunk costs one memory round trip after
// its keys, instead of one per position, and holds no registers meanwhile, so
// the shared memory a block takes sets how many chunks an SM has in flight.
// Runs inside the chunk are summed in position order and applied (their sums
// of squares reduced across the block at once); a run's part that touches a
// chunk boundary goes to part_tail[c] (the chunk's first run, begun earlier)
// or part_head[c] (its last run, going on).  Without STAGE_ROWS (rows too
// wide for the staging buffer) the table values are read when applied.
template <typename tab_t, int MAXT, bool STAGE_ROWS>
__global__ void __launch_bounds__(MAXT) table_chunk_kernel(
    tab_t* __restrict__ table, float* __restrict__ state, int d, const float* __restrict__ grad,
    const uint32_t* __restrict__ skeys, const int32_t* __restrict__ perm, int n, long long n_rows,
    float* __restrict__ part_head, float* __restrict__ part_tail, float lr, float beta, float eps) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  static_assert(CHUNK == 16, "warp_sum16 reduces one value per position of a chunk");
  static_assert(MAXT <= 512, "ss_sh holds 16 warps");
  using raw_t = typename Raw4<tab_t>::type;
  extern __shared__ __align__(16) unsigned char chunk_sh[];
  __shared__ float ss_sh[16][CHUNK];  // [warp][run-end position]: the warp's share of sum G^2
  const int c = blockIdx.x, nt = blockDim.x, t = threadIdx.x;
  const int lane = t & 31, warp = t >> 5, nwarps = nt >> 5;
  float4* gs = reinterpret_cast<float4*>(chunk_sh);           // [CHUNK][nt]: gradients, then run sums
  raw_t* ws = reinterpret_cast<raw_t*>(gs + (size_t)CHUNK * nt);  // [CHUNK][nt]: table values
  const int col = 4 * t;
  const bool own = col < d;
  const ChunkRuns r = chunk_runs(skeys, perm, n, c);  // every warp finds the same runs
  // positions with a gradient row (not past the chunk's end, not invalid ids)
  const unsigned has = __ballot_sync(0xffffffffu, r.pos >= 0) & ((1u << CHUNK) - 1u);
  // run ends whose row this block finishes (not the run of invalid ids)
  unsigned whole = 0;
#pragma unroll
  for (int q = 0; q < CHUNK; ++q) {
    const uint32_t kq = __shfl_sync(0xffffffffu, r.key, q);
    if (((r.end_mask >> q) & 1u) && run_kind(r, q) == RUN_WHOLE && kq < n_rows) whole |= 1u << q;
  }
#pragma unroll
  for (int q = 0; q < CHUNK; ++q) {
    const int p = __shfl_sync(0xffffffffu, r.pos, q);
    const uint32_t kq = __shfl_sync(0xffffffffu, r.key, q);
    if (own && ((has >> q) & 1u)) cp_async_own<16>(gs + q * nt + t, grad + (long long)p * d + col);
    if constexpr (STAGE_ROWS)
      if (own && ((whole >> q) & 1u)) cp_async_own<sizeof(raw_t)>(ws + q * nt + t, table + (long long)kq * d + col);
  }
  const float s_old = ((whole >> lane) & 1u) ? state[r.key] : 0.f;  // lane q: state of run end q
  cp_async_wait_own();
  // run sums in position order; gs[q] becomes the sum of the run ending at q
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float ss[CHUNK];
#pragma unroll
  for (int q = 0; q < CHUNK; ++q) {
    if (own && ((has >> q) & 1u)) {
      const float4 v = gs[q * nt + t];
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    ss[q] = 0.f;
    if ((r.end_mask >> q) & 1u) {
      ss[q] = ((acc.x * acc.x + acc.y * acc.y) + acc.z * acc.z) + acc.w * acc.w;
      if (own) gs[q * nt + t] = acc;
      acc = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  const float wss = warp_sum16(ss);
  if ((lane & 1) == 0) ss_sh[warp][lane >> 1] = wss;
  // boundary runs: partial sums for the chain launch
#pragma unroll
  for (int q = 0; q < CHUNK; ++q) {
    if (!own || !((r.end_mask >> q) & 1u) || ((whole >> q) & 1u)) continue;
    const int kind = run_kind(r, q);
    if (kind == RUN_WHOLE) continue;  // the run of invalid ids
    *reinterpret_cast<float4*>((kind == RUN_TAIL ? part_tail : part_head) + (long long)c * d + col) = gs[q * nt + t];
  }
  __syncthreads();
  // lane q: the block's sum G^2 of run end q in warp order, then its new state and step
  float tot = 0.f;
  if (lane < CHUNK)
    for (int ww = 0; ww < nwarps; ++ww) tot += ss_sh[ww][lane];
  const float s_new = beta * s_old + (1.f - beta) * (tot / d);
  const float step = lr / (sqrtf(s_new) + eps);
  if (warp == 0 && ((whole >> lane) & 1u)) state[r.key] = s_new;
#pragma unroll
  for (int q = 0; q < CHUNK; ++q) {
    const float st = __shfl_sync(0xffffffffu, step, q);
    const uint32_t kq = __shfl_sync(0xffffffffu, r.key, q);
    if (!own || !((whole >> q) & 1u)) continue;
    raw_t* dst = reinterpret_cast<raw_t*>(table + (long long)kq * d + col);
    const raw_t wv = STAGE_ROWS ? ws[q * nt + t] : *dst;
    const float4 G = gs[q * nt + t];
    float x[4];
    Raw4<tab_t>::unpack(wv, x);
    x[0] -= st * G.x; x[1] -= st * G.y; x[2] -= st * G.z; x[3] -= st * G.w;
    *dst = Raw4<tab_t>::pack(x);
  }
}

// G += part_tail[first..last] in chunk order; several rows are loaded before
// any is added, so a long run's partials stream instead of queueing one by one.
template <int NV>
__device__ __forceinline__ void chain_sum(const float* __restrict__ part_tail, int d, int first, int last,
                                          float (&G)[NV][4]) {
  constexpr int CHAIN_U = NV <= 8 ? 2 : 1;  // rows in flight per warp within 128 registers
  for (int cc = first; cc <= last; cc += CHAIN_U) {
    float t[CHAIN_U][NV][4];
#pragma unroll
    for (int u = 0; u < CHAIN_U; ++u) {
      if (cc + u <= last) load_row<NV>(part_tail + (long long)(cc + u) * d, d, t[u]);
      else zero_row<NV>(t[u]);
    }
#pragma unroll
    for (int u = 0; u < CHAIN_U; ++u)
      if (cc + u <= last) add_row<NV>(G, t[u]);
  }
}

// Sum of a chained run's partials: part_head[c] and part_tail[c+1..last].  The
// block's CHAIN_WARPS warps each add a contiguous share of the tail partials in
// chunk order; warp 0 then adds head + shares in warp order.  The grouping is
// fixed by (c, last), so the result is reproducible.  Returns true in warp 0,
// which then holds the sum in G.  sh: (CHAIN_WARPS - 1) * d floats; the caller
// synchronises the block before sh is used again.
constexpr int CHAIN_WARPS = 8;  // warps of a chain block, and chunks it scans for chain starts
template <int NV>
__device__ __forceinline__ bool chain_block_sum(const float* __restrict__ part_head,
                                                const float* __restrict__ part_tail, int d, int c, int last,
                                                float* __restrict__ sh, float (&G)[NV][4]) {
  const int w = threadIdx.x >> 5;
  const int nparts = last - c;
  const int per = (nparts + CHAIN_WARPS - 1) / CHAIN_WARPS;
  const int b = c + 1 + w * per, e = min(last, b + per - 1);
  float S[NV][4];
  zero_row<NV>(S);
  if (b <= e) chain_sum<NV>(part_tail, d, b, e, S);
  if (w > 0) store_row<NV>(sh + (w - 1) * d, d, S);
  __syncthreads();
  if (w != 0) return false;
  load_row<NV>(part_head + (long long)c * d, d, G);
  add_row<NV>(G, S);
  for (int ww = 1; ww < CHAIN_WARPS; ++ww) {
    float t[NV][4];
    load_row<NV>(sh + (ww - 1) * d, d, t);
    add_row<NV>(G, t);
  }
  return true;
}

// Chains are finished in two ways.  Warp w of a block checks chunk
// blockIdx.x * CHAIN_WARPS + w; if it starts a run that goes on into at most
// CHAIN_SHORT later chunks (nearly all of them), the warp alone adds
// part_head[c] + part_tail[c+1] + ... + part_tail[last] in chunk order and
// finishes the row, so a block's short chains proceed in parallel.  Longer
// chains are listed in shared memory and summed by all warps of the block
// (chain_block_sum) after a block barrier.  Which way a chain takes depends
// only on its length, so every row's sum has one fixed grouping.
constexpr int CHAIN_SHORT = 4;

template <int NV>
__device__ __forceinline__ void chain_warp_sum(const float* __restrict__ part_head,
                                               const float* __restrict__ part_tail, int d, int c, int last,
                                               float (&G)[NV][4]) {
  load_row<NV>(part_head + (long long)c * d, d, G);
  chain_sum<NV>(part_tail, d, c + 1, last, G);
}

// The scan of the block's chunks: returns true in a warp whose chunk starts a
// short chain (key, last filled in); long chains go to the block's lists.
// Ends with a block barrier.
__device__ __forceinline__ bool chain_scan(const uint32_t* __restrict__ skeys, int n, long long key_limit,
                                           uint32_t& key, int& last, int* flag, int* lastc, uint32_t* keyc) {
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x * CHAIN_WARPS + w;
  key = 0;
  last = 0;
  const bool ok = chained_run(skeys, n, c, key, last) && key < key_limit;  // warp-uniform
  const bool longc = ok && last - c > CHAIN_SHORT;
  if (lane == 0) { flag[w] = longc; lastc[w] = last; keyc[w] = key; }
  __syncthreads();
  return ok && !longc;
}

template <int NV, typename tab_t>
__global__ void __launch_bounds__(CHAIN_WARPS * 32, NV <= 6 ? 2 : 1) table_chain_kernel(
    tab_t* __restrict__ table, float* __restrict__ state, int d, const uint32_t* __restrict__ skeys, int n,
    long long n_rows, const float* __restrict__ part_head, const float* __restrict__ part_tail, float lr,
    float beta, float eps) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  extern __shared__ float chain_sh[];
  __shared__ int flag[CHAIN_WARPS], lastc[CHAIN_WARPS];
  __shared__ uint32_t keyc[CHAIN_WARPS];
  uint32_t key;
  int last;
  if (chain_scan(skeys, n, n_rows, key, last, flag, lastc, keyc)) {
    const int c = blockIdx.x * CHAIN_WARPS + (threadIdx.x >> 5);
    typename Raw4<tab_t>::type w[NV];
    load_raw_row<NV>(table + (long long)key * d, d, w);
    const float s_old = state[key];
    float G[NV][4];
    chain_warp_sum<NV>(part_head, part_tail, d, c, last, G);
    table_row_apply<NV>(table, state, key, d, G, w, s_old, lr, beta, eps);
  }
  for (int i = 0; i < CHAIN_WARPS; ++i) {
    if (!flag[i]) continue;  // block-uniform
    const uint32_t k = keyc[i];
    float G[NV][4];
    if (chain_block_sum<NV>(part_head, part_tail, d, blockIdx.x * CHAIN_WARPS + i, lastc[i], chain_sh, G)) {
      typename Raw4<tab_t>::type w[NV];
      load_raw_row<NV>(table + (long long)k * d, d, w);
      table_row_apply<NV>(table, state, k, d, G, w, state[k], lr, beta, eps);
    }
    __syncthreads();  // chain_sh is refilled for the next chain
  }
}

// ---------------------------------------------------------------- embedding grad
// Token-embedding backward through h = norm(wte[tok]): de_t = rstd_t *
// (dx0_t - h_t * mean(dx0_t * h_t)) with h_t = wte[tok_t] * rstd_t, summed per
// token id over its positions (same bucketing as the tables) and added to
// the fp32 gradient dwte.
template <int NV, typename w_t>
__global__ void __launch_bounds__(128, NV <= 6 ? 5 : (NV <= 8 ? 4 : 2)) emb_chunk_kernel(
    float* __restrict__ dwte, const w_t* __restrict__ wte, int d, const float* __restrict__ dx0,
    const float* __restrict__ rstd, const uint32_t* __restrict__ skeys, const int32_t* __restrict__ perm, int n,
    long long vocab, float* __restrict__ part_head, float* __restrict__ part_tail) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  const int c = (int)(((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  if ((long long)c * CHUNK >= n) return;
  constexpr int TAB_U = 1;  // positions a step: one keeps the kernel near 80 registers, 20 warps an SM
  const ChunkRuns r = chunk_runs(skeys, perm, n, c);
  float G[NV][4];
  zero_row<NV>(G);
  for (int q0 = 0; q0 < r.len; q0 += TAB_U) {
    float g[TAB_U][NV][4], e[TAB_U][NV][4], rs[TAB_U];
    int kind[TAB_U];
    bool ends[TAB_U];
    uint32_t key[TAB_U];
#pragma unroll
    for (int u = 0; u < TAB_U; ++u) {
      const int q = q0 + u;
      const bool in = q < r.len;
      const int qs = in ? q : r.len - 1;
      const int p = __shfl_sync(0xffffffffu, r.pos, qs);
      key[u] = __shfl_sync(0xffffffffu, r.key, qs);
      ends[u] = in && ((r.end_mask >> q) & 1u);
      kind[u] = ends[u] ? run_kind(r, q) : RUN_WHOLE;
      rs[u] = 0.f;
      if (in && p >= 0) {
        load_row<NV>(dx0 + (long long)p * d, d, g[u]);
        load_row<NV>(wte + (long long)key[u] * d, d, e[u]);
        rs[u] = rstd[p];
      } else {
        zero_row<NV>(g[u]);
        zero_row<NV>(e[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < TAB_U; ++u) {
      float dot = 0.f;
#pragma unroll
      for (int j = 0; j < NV; ++j)
        dot += g[u][j][0] * e[u][j][0] + g[u][j][1] * e[u][j][1] + g[u][j][2] * e[u][j][2] + g[u][j][3] * e[u][j][3];
      dot = warp_sum(dot) * rs[u] / d;  // mean(dx0 * h)
#pragma unroll
      for (int j = 0; j < NV; ++j)
#pragma unroll
        for (int i = 0; i < 4; ++i) G[j][i] += rs[u] * (g[u][j][i] - e[u][j][i] * rs[u] * dot);
      if (!ends[u]) continue;
      if (kind[u] == RUN_WHOLE) {
        if (key[u] < vocab) {  // the run's sum added into dwte
          float* dst = dwte + (long long)key[u] * d;
          const int lane = threadIdx.x & 31;
#pragma unroll
          for (int j = 0; j < NV; ++j) {
            const int col = (j * 32 + lane) * 4;
            if (col < d) {
              float t[4];
              load4(dst + col, t);
              for (int i = 0; i < 4; ++i) t[i] += G[j][i];
              store4(dst + col, t);
            }
          }
        }
      } else {
        store_row<NV>((kind[u] == RUN_TAIL ? part_tail : part_head) + (long long)c * d, d, G);
      }
      zero_row<NV>(G);
    }
  }
}

template <int NV>
__global__ void __launch_bounds__(CHAIN_WARPS * 32, NV <= 6 ? 2 : 1) emb_chain_kernel(float* __restrict__ dwte, int d,
                                                                       const uint32_t* __restrict__ skeys, int n,
                                                                       long long vocab,
                                                                       const float* __restrict__ part_head,
                                                                       const float* __restrict__ part_tail) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  extern __shared__ float chain_sh[];
  __shared__ int flag[CHAIN_WARPS], lastc[CHAIN_WARPS];
  __shared__ uint32_t keyc[CHAIN_WARPS];
  uint32_t key;
  int last;
  if (chain_scan(skeys, n, vocab, key, last, flag, lastc, keyc)) {
    const int c = blockIdx.x * CHAIN_WARPS + (threadIdx.x >> 5);
    float o[NV][4], G[NV][4];
    load_row<NV>(dwte + (long long)key * d, d, o);
    chain_warp_sum<NV>(part_head, part_tail, d, c, last, G);
    add_row<NV>(o, G);
    store_row<NV>(dwte + (long long)key * d, d, o);
  }
  for (int i = 0; i < CHAIN_WARPS; ++i) {
    if (!flag[i]) continue;  // block-uniform
    const uint32_t k = keyc[i];
    float G[NV][4];
    if (chain_block_sum<NV>(part_head, part_tail, d, blockIdx.x * CHAIN_WARPS + i, lastc[i], chain_sh, G)) {
      float o[NV][4];
      load_row<NV>(dwte + (long long)k * d, d, o);
      add_row<NV>(o, G);
      store_row<NV>(dwte + (long long)k * d, d, o);
    }
    __syncthreads();  // chain_sh is refilled for the next chain
  }
}

// ============================================================================
// Frozen trigram statistics table (decoder-rtx posts: "a 2M row tri-gram stats
// table (tallied from dataset, frozen), projected and added to values").  The
// row of position t hashes the token triple (x_{t-2}, x_{t-1}, x_t) in the form
// of the bigram key, key = a2*p1 XOR a1*p2 XOR c*p3 over uint64, the vocabulary
// size standing for tokens before the start; row = key mod rows.  A row holds
// the next-token statistics tallied over a token stream: the share of its
// occurrences whose next token falls in bucket (next mod width).

__device__ __forceinline__ unsigned long long trigram_key(int a2, int a1, int c, unsigned long long p1,
                                                          unsigned long long p2, unsigned long long p3) {
  return ((unsigned long long)a2 * p1) ^ ((unsigned long long)a1 * p2) ^ ((unsigned long long)c * p3);
}

// rows of every position of tokens [B, T]; out-of-range ids set the error word and give row 0
__global__ void trigram_hash_kernel(const int32_t* __restrict__ tok, int B, int T, int V, unsigned long long p1,
                                    unsigned long long p2, unsigned long long p3, long long rows,
                                    int32_t* __restrict__ out, unsigned* err) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  const long long n = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= (long long)B * T) return;
  const int t = (int)(n % T);
  const int c = tok[n];
  const int a1 = t > 0 ? tok[n - 1] : V;
  const int a2 = t > 1 ? tok[n - 2] : V;
  if (c < 0 || c >= V || a1 < 0 || a1 > V || a2 < 0 || a2 > V) {
    set_error(err, GPT_EBIT_INPUT);
    out[n] = 0;
    return;
  }
  out[n] = (int32_t)(trigram_key(a2, a1, c, p1, p2, p3) % (unsigned long long)rows);
}

// counts[row, next mod width] += 1 for every position t < L - 1 of streams [S, L]
// (integer adds: the counts do not depend on their order)
__global__ void trigram_count_kernel(const int32_t* __restrict__ streams, int S, int L, int V,
                                     unsigned long long p1, unsigned long long p2, unsigned long long p3,
                                     long long rows, int width, unsigned* __restrict__ counts, unsigned* err) {
  const long long n = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= (long long)S * (L - 1)) return;
  const long long s = n / (L - 1);
  const int t = (int)(n % (L - 1));
  const int32_t* x = streams + s * L;
  const int c = x[t], nx = x[t + 1];
  const int a1 = t > 0 ? x[t - 1] : V;
  const int a2 = t > 1 ? x[t - 2] : V;
  if (c < 0 || c >= V || nx < 0 || nx >= V || a1 < 0 || a1 > V || a2 < 0 || a2 > V) {
    set_error(err, GPT_EBIT_INPUT);
    return;
  }
  const long long r = (long long)(trigram_key(a2, a1, c, p1, p2, p3) % (unsigned long long)rows);
  atomicAdd(&counts[r * width + nx % width], 1u);
}

// table[row, :] = counts[row, :] / (sum of the row's counts); rows never seen stay 0.
// One warp per row; the sum is exact (integers) and each entry one fp32 division.
template <typename tab_t>
__global__ void trigram_normalize_kernel(const unsigned* __restrict__ counts, long long rows, int width,
                                         tab_t* __restrict__ table) {
  const long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const unsigned* c = counts + r * width;
  unsigned long long tot = 0;
  for (int b = lane; b < width; b += 32) tot += c[b];
  for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
  const float ft = (float)tot;
  for (int b = lane; b < width; b += 32) table[r * width + b] = from_f<tab_t>(tot ? (float)c[b] / ft : 0.f);
}

// vb[t] = p3[t] (+ the value-table row hv[rv[t]]) in the activation type:
// the per-position value bias every layer adds to v
template <typename act_t>
__global__ void value_bias_kernel(const float* __restrict__ p3, const act_t* __restrict__ hv,
                                  const int32_t* __restrict__ rv, long long N, int a, act_t* __restrict__ vb) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  const long long total4 = N * a / 4;
  for (long long i4 = (long long)blockIdx.x * blockDim.x + threadIdx.x; i4 < total4;
       i4 += (long long)gridDim.x * blockDim.x) {
    const long long i = i4 * 4, n = i / a, j = i % a;
    float v[4];
    load4(p3 + i, v);
    if (hv) {
      float h[4];
      load4(hv + (long long)rv[n] * a + j, h);
      v[0] += h[0]; v[1] += h[1]; v[2] += h[2]; v[3] += h[3];
    }
    store4(vb + i, v);
  }
}
