// ngram.cuh -- hashed bigram tables: hash, row gather, atomics-free bucketing
// of positions by row, and the sparse per-row-magnitude update fused with the
// gradient segment-sum (decoder-rtx posts: "Two huge bi-gram hash tables",
// "inlined the optimizer in their backward math", "sparse, no first moment,
// and only per-row magnitude").
//
// Bucketing: positions are sorted by row with a stable LSD radix sort (8-bit
// digits; per-tile histograms, one exclusive scan, stable scatter ranked with
// warp match masks) -- no atomics anywhere, so sums are formed in position
// order and results are bit-reproducible.  Runs of equal rows (segments) are
// cut into pieces of at most PIECE positions; one warp sums one piece.  A
// segment that fits in one piece is finished by that warp (sum -> mean square
// -> row state -> row update); longer segments write per-piece partial sums
// that a second pass adds in piece order before updating the row.
#pragma once
#include "common.cuh"
#include "layers.cuh"

constexpr int RADIX_THREADS = 256;
constexpr int RADIX_ITEMS = 8;
constexpr int RADIX_TILE = RADIX_THREADS * RADIX_ITEMS;  // 2048 keys per block
constexpr int PIECE = 32;                                // positions per warp task

// ---------------------------------------------------------------- hash
// key = (a*p1 mod 2^64) XOR (c*p2 mod 2^64), a = tokens[t-1] (vocab at t = 0)
__global__ void ngram_hash_kernel(const int32_t* __restrict__ tok, int B, int T, int V,
                                  unsigned long long p1, unsigned long long p2, long long rows_a,
                                  int32_t* __restrict__ out_a, long long rows_b,
                                  int32_t* __restrict__ out_b, unsigned* err) {
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

// ---------------------------------------------------------------- radix sort
// counts layout: digit-major [256][nblocks] so one exclusive scan gives every
// (digit, block) its stable global offset.
__global__ void __launch_bounds__(RADIX_THREADS) radix_hist_kernel(const uint32_t* __restrict__ keys,
                                                                  int n, int shift,
                                                                  uint32_t* __restrict__ counts) {
  constexpr int NW = RADIX_THREADS / 32;
  __shared__ uint32_t wh[NW][256];  // per-warp digit counts
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < NW * 256; i += RADIX_THREADS) (&wh[0][0])[i] = 0;
  __syncthreads();
  const int base = blockIdx.x * RADIX_TILE;
  const uint32_t lt = (1u << lane) - 1u;
  for (int round = 0; round < RADIX_ITEMS; ++round) {
    const int idx = base + round * RADIX_THREADS + threadIdx.x;
    const uint32_t dgt = (idx < n) ? ((keys[idx] >> shift) & 255u) : 256u;
    const uint32_t peers = __match_any_sync(0xffffffffu, dgt);
    // the lowest lane of each digit group adds the group's size: one writer
    // per (warp, digit), so no atomics are needed
    if (dgt < 256u && (peers & lt) == 0) wh[w][dgt] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  uint32_t s = 0;
  for (int ww = 0; ww < NW; ++ww) s += wh[ww][threadIdx.x];
  counts[(long long)threadIdx.x * gridDim.x + blockIdx.x] = s;
}

// Exclusive scan of `n` counters in one block (sequential chunks + block scan).
__global__ void __launch_bounds__(1024) exclusive_scan_kernel(uint32_t* __restrict__ data, int n) {
  __shared__ uint32_t sh[1024];
  const int per = (n + 1023) / 1024;
  const int beg = threadIdx.x * per, end = min(beg + per, n);
  uint32_t local = 0;
  for (int i = beg; i < end; ++i) local += data[i];
  sh[threadIdx.x] = local;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    uint32_t v = (threadIdx.x >= off) ? sh[threadIdx.x - off] : 0;
    __syncthreads();
    sh[threadIdx.x] += v;
    __syncthreads();
  }
  uint32_t run = sh[threadIdx.x] - local;
  for (int i = beg; i < end; ++i) {
    const uint32_t v = data[i];
    data[i] = run;
    run += v;
  }
}

// Stable scatter: element order within a tile is idx = base + round*256 + tid;
// ranks among equal digits follow that order (warp match masks inside a warp,
// per-warp digit counts across warps, running totals across rounds).
__global__ void __launch_bounds__(RADIX_THREADS) radix_scatter_kernel(
    const uint32_t* __restrict__ keys_in, const int32_t* __restrict__ vals_in, int n, int shift,
    const uint32_t* __restrict__ offsets, uint32_t* __restrict__ keys_out,
    int32_t* __restrict__ vals_out) {
  constexpr int NW = RADIX_THREADS / 32;
  __shared__ uint32_t wcount[NW][256];
  __shared__ uint32_t running[256];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  running[threadIdx.x] = offsets[(long long)threadIdx.x * gridDim.x + blockIdx.x];
  const int base = blockIdx.x * RADIX_TILE;
  for (int round = 0; round < RADIX_ITEMS; ++round) {
    for (int i = threadIdx.x; i < NW * 256; i += RADIX_THREADS) (&wcount[0][0])[i] = 0;
    __syncthreads();
    const int idx = base + round * RADIX_THREADS + threadIdx.x;
    const bool valid = idx < n;
    uint32_t key = 0, dgt = 256;  // 256 = no digit (invalid lane)
    int32_t val = 0;
    if (valid) { key = keys_in[idx]; val = vals_in[idx]; dgt = (key >> shift) & 255u; }
    const uint32_t peers = __match_any_sync(0xffffffffu, dgt);
    const uint32_t lt = (1u << lane) - 1u;
    const uint32_t rank_in_warp = __popc(peers & lt);
    if (valid && rank_in_warp == 0) wcount[w][dgt] = __popc(peers);
    __syncthreads();
    uint32_t before = 0;
    if (valid) {
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
    __syncthreads();
  }
}

// Sort input: (key, position).  Keys outside [0, key_range) set the error
// word; they are sorted as key_range - 1 with position -1, which every
// consumer skips, so no out-of-range row is ever read or written.
__global__ void iota_kernel(const int32_t* __restrict__ keys_in, uint32_t* __restrict__ keys,
                            int32_t* __restrict__ vals, int n, long long key_range, unsigned* err) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int32_t k = keys_in[i];
  if (k < 0 || (long long)k >= key_range) {
    set_error(err, GPT_EBIT_INPUT);
    keys[i] = (uint32_t)(key_range - 1);
    vals[i] = -1;
  } else {
    keys[i] = (uint32_t)k;
    vals[i] = i;
  }
}

// ---------------------------------------------------------------- segments
// From sorted keys, build (single block):
//   pieces: pstart[p], plen[p], pseg[p], pslot[p] (-1: the piece is a whole
//           segment; else its partial-sum slot)
//   long segments: lseg_first_slot[s], lseg_nslots[s], lseg_key[s]
//   counters[0] = #pieces, counters[1] = #long segments, counters[2] = #segments
// and (optionally) the distinct keys in ascending order.
__global__ void __launch_bounds__(1024) segments_kernel(
    const uint32_t* __restrict__ skeys, int n, int32_t* __restrict__ seg_start /* [n+1] */,
    int32_t* __restrict__ pstart, int32_t* __restrict__ plen, int32_t* __restrict__ pseg,
    int32_t* __restrict__ pslot, int32_t* __restrict__ lseg_first_slot,
    int32_t* __restrict__ lseg_nslots, int32_t* __restrict__ lseg_seg, int32_t* __restrict__ counters,
    int32_t* __restrict__ uniq_out, int* __restrict__ n_uniq_out) {
  __shared__ int sh[1024];
  const int per = (n + 1023) / 1024;
  const int beg = threadIdx.x * per, end = min(beg + per, n);
  // pass 1: segment heads
  int heads = 0;
  for (int i = beg; i < end; ++i) heads += (i == 0 || skeys[i] != skeys[i - 1]);
  sh[threadIdx.x] = heads;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    int v = (threadIdx.x >= off) ? sh[threadIdx.x - off] : 0;
    __syncthreads();
    sh[threadIdx.x] += v;
    __syncthreads();
  }
  int sid = sh[threadIdx.x] - heads;
  const int U = sh[1023];
  for (int i = beg; i < end; ++i) {
    if (i == 0 || skeys[i] != skeys[i - 1]) {
      seg_start[sid] = i;
      if (uniq_out) uniq_out[sid] = (int32_t)skeys[i];
      ++sid;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) seg_start[U] = n;
  __syncthreads();
  // pass 2: pieces per segment, partial slots for long segments
  const int sper = (U + 1023) / 1024;
  const int sbeg = threadIdx.x * sper, send = min(sbeg + sper, U);
  int np = 0, nslot = 0, nlong = 0;
  for (int s = sbeg; s < send; ++s) {
    const int len = seg_start[s + 1] - seg_start[s];
    const int k = (len + PIECE - 1) / PIECE;
    np += k;
    if (k > 1) { nslot += k; ++nlong; }
  }
  __syncthreads();
  sh[threadIdx.x] = np;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    int v = (threadIdx.x >= off) ? sh[threadIdx.x - off] : 0;
    __syncthreads();
    sh[threadIdx.x] += v;
    __syncthreads();
  }
  int p = sh[threadIdx.x] - np;
  const int NP = sh[1023];
  __syncthreads();
  sh[threadIdx.x] = (nslot << 0);
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    int v = (threadIdx.x >= off) ? sh[threadIdx.x - off] : 0;
    __syncthreads();
    sh[threadIdx.x] += v;
    __syncthreads();
  }
  int slot = sh[threadIdx.x] - nslot;
  __syncthreads();
  sh[threadIdx.x] = nlong;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    int v = (threadIdx.x >= off) ? sh[threadIdx.x - off] : 0;
    __syncthreads();
    sh[threadIdx.x] += v;
    __syncthreads();
  }
  int ls = sh[threadIdx.x] - nlong;
  const int NL = sh[1023];
  for (int s = sbeg; s < send; ++s) {
    const int st = seg_start[s], len = seg_start[s + 1] - st;
    const int k = (len + PIECE - 1) / PIECE;
    if (k > 1) {
      lseg_first_slot[ls] = slot;
      lseg_nslots[ls] = k;
      lseg_seg[ls] = s;
      ++ls;
    }
    for (int j = 0; j < k; ++j) {
      pstart[p] = st + j * PIECE;
      plen[p] = min(PIECE, len - j * PIECE);
      pseg[p] = s;
      pslot[p] = (k > 1) ? slot + j : -1;
      ++p;
    }
    if (k > 1) slot += k;
  }
  if (threadIdx.x == 0) {
    counters[0] = NP;
    counters[1] = NL;
    counters[2] = U;
    if (n_uniq_out) *n_uniq_out = U;
  }
}

// ---------------------------------------------------------------- row update
// Apply the per-row-magnitude step to one row with its summed gradient G
// (held by the warp, 4 values per lane per chunk).
template <int NV, typename tab_t>
__device__ __forceinline__ void table_row_update(tab_t* __restrict__ table, float* __restrict__ state,
                                                 long long r, int d, const float (&G)[NV][4],
                                                 float lr, float beta, float eps) {
  const int lane = threadIdx.x & 31;
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int c = (j * 32 + lane) * 4;
    if (c < d) ss += G[j][0] * G[j][0] + G[j][1] * G[j][1] + G[j][2] * G[j][2] + G[j][3] * G[j][3];
  }
  ss = warp_sum(ss);
  const float s_new = beta * state[r] + (1.f - beta) * (ss / d);
  const float step = lr / (sqrtf(s_new) + eps);
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int c = (j * 32 + lane) * 4;
    if (c < d) {
      float w[4];
      load4(table + r * d + c, w);
#pragma unroll
      for (int i = 0; i < 4; ++i) w[i] -= step * G[j][i];
      store4(table + r * d + c, w);
    }
  }
  __syncwarp();
  if (lane == 0) state[r] = s_new;
}

// Sum the gradient rows of one piece (in sorted = position order).
template <int NV>
__device__ __forceinline__ void piece_sum(const float* __restrict__ grad, const int32_t* __restrict__ perm,
                                          int st, int len, int d, float (&G)[NV][4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < NV; ++j) G[j][0] = G[j][1] = G[j][2] = G[j][3] = 0.f;
  for (int q = 0; q < len; ++q) {
    const long long pos = perm[st + q];
    if (pos < 0) continue;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int c = (j * 32 + lane) * 4;
      if (c < d) {
        float g[4];
        load4(grad + pos * d + c, g);
        G[j][0] += g[0]; G[j][1] += g[1]; G[j][2] += g[2]; G[j][3] += g[3];
      }
    }
  }
}

// One warp per piece: whole segments are updated directly; pieces of long
// segments store their partial sums.
template <int NV, typename tab_t>
__global__ void table_piece_kernel(tab_t* __restrict__ table, float* __restrict__ state, int d,
                                   const float* __restrict__ grad, const uint32_t* __restrict__ skeys,
                                   const int32_t* __restrict__ perm, const int32_t* __restrict__ pstart,
                                   const int32_t* __restrict__ plen, const int32_t* __restrict__ pslot,
                                   const int32_t* __restrict__ counters, float* __restrict__ partial,
                                   float lr, float beta, float eps) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= counters[0]) return;
  const int st = pstart[warp], len = plen[warp], slot = pslot[warp];
  float G[NV][4];
  piece_sum<NV>(grad, perm, st, len, d, G);
  if (slot < 0) {
    table_row_update<NV>(table, state, (long long)skeys[st], d, G, lr, beta, eps);
  } else {
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int c = (j * 32 + lane) * 4;
      if (c < d) store4(partial + (long long)slot * d + c, G[j]);
    }
  }
}

// One warp per long segment: add its partial sums in piece order, update.
template <int NV, typename tab_t>
__global__ void table_long_kernel(tab_t* __restrict__ table, float* __restrict__ state, int d,
                                  const uint32_t* __restrict__ skeys, const int32_t* __restrict__ seg_start,
                                  const int32_t* __restrict__ lseg_first_slot,
                                  const int32_t* __restrict__ lseg_nslots, const int32_t* __restrict__ lseg_seg,
                                  const int32_t* __restrict__ counters, const float* __restrict__ partial,
                                  float lr, float beta, float eps) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= counters[1]) return;
  const int first = lseg_first_slot[warp], k = lseg_nslots[warp];
  const long long r = skeys[seg_start[lseg_seg[warp]]];
  float G[NV][4];
#pragma unroll
  for (int j = 0; j < NV; ++j) G[j][0] = G[j][1] = G[j][2] = G[j][3] = 0.f;
  for (int q = 0; q < k; ++q) {
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int c = (j * 32 + lane) * 4;
      if (c < d) {
        float g[4];
        load4(partial + (long long)(first + q) * d + c, g);
        G[j][0] += g[0]; G[j][1] += g[1]; G[j][2] += g[2]; G[j][3] += g[3];
      }
    }
  }
  table_row_update<NV>(table, state, r, d, G, lr, beta, eps);
}

// ---------------------------------------------------------------- embedding grad
// Token-embedding backward through h = norm(wte[tok]): de_t = rstd_t *
// (dx0_t - h_t * mean(dx0_t * h_t)) with h_t = wte[tok_t] * rstd_t, summed per
// token id over its positions (same bucketing as the tables) and added to
// the fp32 gradient dwte.
template <int NV, typename w_t>
__device__ __forceinline__ void emb_piece_sum(const float* __restrict__ dx0, const w_t* __restrict__ wte,
                                              const float* __restrict__ rstd, const int32_t* __restrict__ perm,
                                              long long row, int st, int len, int d, float (&G)[NV][4]) {
  const int lane = threadIdx.x & 31;
  float e[NV][4];
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    G[j][0] = G[j][1] = G[j][2] = G[j][3] = 0.f;
    const int c = (j * 32 + lane) * 4;
    if (c < d) load4(wte + row * d + c, e[j]);
  }
  for (int q = 0; q < len; ++q) {
    const long long pos = perm[st + q];
    if (pos < 0) continue;
    const float r = rstd[pos];
    float g[NV][4];
    float dot = 0.f;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int c = (j * 32 + lane) * 4;
      if (c < d) {
        load4(dx0 + pos * d + c, g[j]);
        dot += g[j][0] * e[j][0] + g[j][1] * e[j][1] + g[j][2] * e[j][2] + g[j][3] * e[j][3];
      }
    }
    dot = warp_sum(dot) * r / d;  // mean(dx0 * h)
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int c = (j * 32 + lane) * 4;
      if (c < d)
#pragma unroll
        for (int i = 0; i < 4; ++i) G[j][i] += r * (g[j][i] - e[j][i] * r * dot);
    }
  }
}

template <int NV, typename w_t>
__global__ void emb_piece_kernel(float* __restrict__ dwte, const w_t* __restrict__ wte, int d,
                                 const float* __restrict__ dx0, const float* __restrict__ rstd,
                                 const uint32_t* __restrict__ skeys, const int32_t* __restrict__ perm,
                                 const int32_t* __restrict__ pstart, const int32_t* __restrict__ plen,
                                 const int32_t* __restrict__ pslot, const int32_t* __restrict__ counters,
                                 float* __restrict__ partial) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= counters[0]) return;
  const int st = pstart[warp], len = plen[warp], slot = pslot[warp];
  const long long row = skeys[st];
  float G[NV][4];
  emb_piece_sum<NV>(dx0, wte, rstd, perm, row, st, len, d, G);
  float* dst = (slot < 0) ? dwte + row * d : partial + (long long)slot * d;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int c = (j * 32 + lane) * 4;
    if (c < d) {
      float o[4];
      if (slot < 0) {
        load4(dst + c, o);
        o[0] += G[j][0]; o[1] += G[j][1]; o[2] += G[j][2]; o[3] += G[j][3];
      } else {
        o[0] = G[j][0]; o[1] = G[j][1]; o[2] = G[j][2]; o[3] = G[j][3];
      }
      store4(dst + c, o);
    }
  }
}

__global__ void emb_long_kernel(float* __restrict__ dwte, int d, const uint32_t* __restrict__ skeys,
                                const int32_t* __restrict__ seg_start,
                                const int32_t* __restrict__ lseg_first_slot,
                                const int32_t* __restrict__ lseg_nslots, const int32_t* __restrict__ lseg_seg,
                                const int32_t* __restrict__ counters, const float* __restrict__ partial) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= counters[1]) return;
  const int first = lseg_first_slot[warp], k = lseg_nslots[warp];
  const long long row = skeys[seg_start[lseg_seg[warp]]];
  for (int c = lane * 4; c < d; c += 128) {
    float o[4];
    load4(dwte + row * d + c, o);
    for (int q = 0; q < k; ++q) {
      float g[4];
      load4(partial + (long long)(first + q) * d + c, g);
      o[0] += g[0]; o[1] += g[1]; o[2] += g[2]; o[3] += g[3];
    }
    store4(dwte + row * d + c, o);
  }
}
