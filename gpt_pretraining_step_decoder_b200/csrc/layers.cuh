// layers.cuh -- memory-bound layer kernels of the decoder step.
//
// One warp per row (token) for the row-wise normalisations; 128-bit (fp32) or
// 64-bit (bf16) vector accesses along the row; reductions with warp shuffles.
// act_t is the activation type (float in the fp32 mode, bf16 otherwise); the
// residual stream and its gradient stay fp32 in both modes.
#pragma once
#include "common.cuh"

constexpr int MAXV = 16;  // vec4 chunks per lane: rows up to 32 * 4 * 16 = 2048 wide
// Row kernels take NV = vec4 chunks per lane as a template parameter so their
// per-row register arrays are exactly as large as the row (d = 128 * NV when
// d is a multiple of 128, else NV = MAXV with predication).

// --------------------------------------------------------------------------
// Token embedding + parameter-free RMSNorm + optional x0 bigram row
// ("$1000 tier nanochat run", `GPT.forward`: x = norm(wte(idx)); decoder-rtx
// posts: a 2M-row bigram table "added to x0").
//   x[t] = wte[tok_t] * rstd_t + Hx[rx_t],   rstd_t = 1/sqrt(mean(wte[tok_t]^2) + eps)
template <int NV, typename w_t, typename tab_t>
__global__ void embed_fwd_kernel(const int32_t* __restrict__ tok, const w_t* __restrict__ wte,
                                 const tab_t* __restrict__ hx, const int32_t* __restrict__ rx,
                                 float* __restrict__ x, float* __restrict__ rstd_out, int N, int d,
                                 int V, float eps, unsigned* err) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= N) return;
  int id = tok[warp];
  if (id < 0 || id >= V) {
    if (lane == 0) set_error(err, GPT_EBIT_INPUT);
    id = 0;
  }
  float v[NV][4];
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int c = (j * 32 + lane) * 4;
    if (c < d) {
      load4(wte + (long long)id * d + c, v[j]);
      ss += v[j][0] * v[j][0] + v[j][1] * v[j][1] + v[j][2] * v[j][2] + v[j][3] * v[j][3];
    }
  }
  ss = warp_sum(ss);
  const float rstd = rsqrtf(ss / d + eps);
  if (lane == 0) rstd_out[warp] = rstd;
  const long long row = hx ? (long long)rx[warp] : 0;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int c = (j * 32 + lane) * 4;
    if (c < d) {
      float o[4] = {v[j][0] * rstd, v[j][1] * rstd, v[j][2] * rstd, v[j][3] * rstd};
      if (hx) {
        float h[4];
        load4(hx + row * d + c, h);
        o[0] += h[0]; o[1] += h[1]; o[2] += h[2]; o[3] += h[3];
      }
      store4(x + (long long)warp * d + c, o);
    }
  }
}

// --------------------------------------------------------------------------
// RMSNorm forward ("$1000 tier nanochat run", `norm`: F.rms_norm without
// affine parameters): u = x * rstd, rstd = 1/sqrt(mean(x^2) + eps).
template <int NV, typename act_t>
__global__ void rmsnorm_fwd_kernel(const float* __restrict__ x, act_t* __restrict__ u,
                                   float* __restrict__ rstd_out, int N, int d, float eps) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= N) return;
  const float* xr = x + (long long)warp * d;
  float v[NV][4];
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int c = (j * 32 + lane) * 4;
    if (c < d) {
      load4(xr + c, v[j]);
      ss += v[j][0] * v[j][0] + v[j][1] * v[j][1] + v[j][2] * v[j][2] + v[j][3] * v[j][3];
    }
  }
  ss = warp_sum(ss);
  const float rstd = rsqrtf(ss / d + eps);
  if (lane == 0) rstd_out[warp] = rstd;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int c = (j * 32 + lane) * 4;
    if (c < d) {
      float o[4] = {v[j][0] * rstd, v[j][1] * rstd, v[j][2] * rstd, v[j][3] * rstd};
      store4(u + (long long)warp * d + c, o);
    }
  }
}

// RMSNorm backward: dx (+)= rstd * (du - u * mean(du * u)); also writes the
// activation-typed copy of dx that the next GEMMs read.  One warp per row; the
// row's du, u, rstd and (accumulating) old dx are all requested before the
// reduction, so a row costs one memory round trip.
template <int NV, typename act_t>
__global__ void rmsnorm_bwd_kernel(const float* __restrict__ du, const act_t* __restrict__ u,
                                   const float* __restrict__ rstd, float* __restrict__ dx,
                                   act_t* __restrict__ dx_lp, int N, int d, int accumulate) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= N) return;
  const long long base = (long long)warp * d;
  float g[NV][4], y[NV][4], o[NV][4];
  const float r = rstd[warp];
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int c = (j * 32 + lane) * 4;
    if (c < d) {
      load4(du + base + c, g[j]);
      load4(u + base + c, y[j]);
      if (accumulate) load4(dx + base + c, o[j]);
      else o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    }
  }
  float dot = 0.f;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int c = (j * 32 + lane) * 4;
    if (c < d) dot += g[j][0] * y[j][0] + g[j][1] * y[j][1] + g[j][2] * y[j][2] + g[j][3] * y[j][3];
  }
  dot = warp_sum(dot) / d;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int c = (j * 32 + lane) * 4;
    if (c < d) {
#pragma unroll
      for (int i = 0; i < 4; ++i) o[j][i] += r * (g[j][i] - y[j][i] * dot);
      store4(dx + base + c, o[j]);
      store4(dx_lp + base + c, o[j]);
    }
  }
}

// --------------------------------------------------------------------------
// RoPE cos/sin table: theta[t, i] = t * base^(-2i/hd) for i < hd/2
// ("$1000 tier nanochat run", `_precompute_rotary_embeddings`), evaluated in
// double precision and stored fp32 (the pages keep a bf16 table).
// (cos, sin) of t * base^(-2j/hd) for every position t and frequency j < hd/2,
// position-major cs[t][j] (one warp per position reads a contiguous row), and
// for the QKV GEMM epilogue, which computes each row's cos / sin itself, the
// frequencies' turns per position base^(-2j/hd) / (2 pi) as fp32 hi + lo.
__global__ void rope_table_kernel(float* __restrict__ cs, float2* __restrict__ turns, int T, int hd, double base) {
  const int h = hd / 2;
  const long long total = (long long)T * h;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(i / h), j = (int)(i % h);
    const double inv_freq = 1.0 / pow(base, (2.0 * j) / hd);
    if (t == 0) {
      // turns per position of frequency j, as an unevaluated fp32 sum hi + lo
      const double u = inv_freq / 6.283185307179586476925287;
      const float hi = (float)u;
      turns[j] = make_float2(hi, (float)(u - (double)hi));
    }
    const double th = t * inv_freq;
    cs[2 * i] = (float)cos(th);
    cs[2 * i + 1] = (float)sin(th);
  }
}

// Per (position, head): rotate q and k ("$1000 tier nanochat run",
// `apply_rotary_emb`: y1 = x1 cos + x2 sin, y2 = -x1 sin + x2 cos), then
// RMSNorm each head (QK-norm, `q, k = norm(q), norm(k)` after RoPE), and add
// the value-table row to v (decoder-rtx posts: 1M-row table "added to
// values").  In place on qkv [N, 3a]; rstd_q/rstd_k [N, H].
template <typename act_t, typename tab_t>
__global__ void rope_qknorm_fwd_kernel(act_t* __restrict__ qkv, const float* __restrict__ cs,
                                       float* __restrict__ rstd_q, float* __restrict__ rstd_k,
                                       const tab_t* __restrict__ hv, const int32_t* __restrict__ rv,
                                       int N, int T, int H, int hd, int qk_norm, float eps) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= N * H) return;
  const int n = warp / H, h = warp % H, t = n % T;
  const int a = H * hd, half = hd / 2;
  act_t* row = qkv + (long long)n * 3 * a;
  for (int which = 0; which < 2; ++which) {
    act_t* x = row + which * a + h * hd;
    float y1[2], y2[2];
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int i = lane + 32 * k;
      y1[k] = y2[k] = 0.f;
      if (i < half) {
        const float c = cs[2 * ((long long)t * half + i)], s = cs[2 * ((long long)t * half + i) + 1];
        const float x1 = to_f(x[i]), x2 = to_f(x[i + half]);
        y1[k] = x1 * c + x2 * s;
        y2[k] = -x1 * s + x2 * c;
        ss += y1[k] * y1[k] + y2[k] * y2[k];
      }
    }
    float r = 1.f;
    if (qk_norm) {
      ss = warp_sum(ss);
      r = rsqrtf(ss / hd + eps);
      if (lane == 0) (which == 0 ? rstd_q : rstd_k)[(long long)n * H + h] = r;
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int i = lane + 32 * k;
      if (i < half) {
        x[i] = from_f<act_t>(y1[k] * r);
        x[i + half] = from_f<act_t>(y2[k] * r);
      }
    }
  }
  if (hv) {
    // the value-table row of this position, or (rv null) row n of a per-position bias
    act_t* v = row + 2 * a + h * hd;
    const tab_t* src = hv + (long long)(rv ? rv[n] : n) * a + h * hd;
    for (int i = lane; i < hd; i += 32) v[i] = from_f<act_t>(to_f(v[i]) + to_f(src[i]));
  }
}

// Backward of the above, in place on dqkv: QK-norm backward with the saved
// normalised q/k and rstd, then the inverse rotation (rotation by -theta).
// The v part is summed over layers into gv (fp32 [N, a]) for the value table.
template <typename act_t>
__global__ void rope_qknorm_bwd_kernel(act_t* __restrict__ dqkv, const act_t* __restrict__ qkv,
                                       const float* __restrict__ cs, const float* __restrict__ rstd_q,
                                       const float* __restrict__ rstd_k, float* __restrict__ gv,
                                       int gv_accumulate, int N, int T, int H, int hd, int qk_norm) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= N * H) return;
  const int n = warp / H, h = warp % H, t = n % T;
  const int a = H * hd, half = hd / 2;
  for (int which = 0; which < 2; ++which) {
    act_t* g = dqkv + (long long)n * 3 * a + which * a + h * hd;
    const act_t* y = qkv + (long long)n * 3 * a + which * a + h * hd;
    float g1[2], g2[2], y1[2], y2[2];
    float dot = 0.f;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int i = lane + 32 * k;
      g1[k] = g2[k] = y1[k] = y2[k] = 0.f;
      if (i < half) {
        g1[k] = to_f(g[i]); g2[k] = to_f(g[i + half]);
        y1[k] = to_f(y[i]); y2[k] = to_f(y[i + half]);
        dot += g1[k] * y1[k] + g2[k] * y2[k];
      }
    }
    float r = 1.f;
    if (qk_norm) {
      dot = warp_sum(dot) / hd;
      r = (which == 0 ? rstd_q : rstd_k)[(long long)n * H + h];
    } else {
      dot = 0.f;
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int i = lane + 32 * k;
      if (i < half) {
        const float d1 = r * (g1[k] - y1[k] * dot), d2 = r * (g2[k] - y2[k] * dot);
        const float c = cs[2 * ((long long)t * half + i)], s = cs[2 * ((long long)t * half + i) + 1];
        g[i] = from_f<act_t>(d1 * c - d2 * s);
        g[i + half] = from_f<act_t>(d1 * s + d2 * c);
      }
    }
  }
  if (gv) {
    const act_t* dv = dqkv + (long long)n * 3 * a + 2 * a + h * hd;
    float* dst = gv + (long long)n * a + h * hd;
    for (int i = lane; i < hd; i += 32) dst[i] = (gv_accumulate ? dst[i] : 0.f) + to_f(dv[i]);
  }
}

// The same backward for bf16 activations and hd = 128, vectorised: lane l
// owns elements 4j..4j+3 (j = l & 15) of half l >> 4 of the head, so each lane
// moves 8-byte pieces of dq, dk, q and k at once; the rotation partner of
// element i (i + 64 or i - 64) sits in lane l ^ 16.
__global__ void __launch_bounds__(256) rope_qknorm_bwd_hd128_kernel(
    bf16* __restrict__ dqkv, const bf16* __restrict__ qkv, const float* __restrict__ cs,
    const float* __restrict__ rstd_q, const float* __restrict__ rstd_k, float* __restrict__ gv, int gv_accumulate,
    int N, int T, int H, int qk_norm) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= N * H) return;  // whole warp
  const int n = warp / H, h = warp % H, t = n % T;
  const int a = H * 128;
  const int j = lane & 15, hf = lane >> 4, i0 = hf * 64 + 4 * j;
  const long long base = (long long)n * 3 * a + h * 128 + i0;
  float g[2][4], y[2][4];
#pragma unroll
  for (int w = 0; w < 2; ++w) {
    const uint2 rg = *reinterpret_cast<const uint2*>(dqkv + base + w * a);
    const uint2 ry = *reinterpret_cast<const uint2*>(qkv + base + w * a);
    const float2 g01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&rg.x));
    const float2 g23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&rg.y));
    const float2 y01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ry.x));
    const float2 y23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ry.y));
    g[w][0] = g01.x; g[w][1] = g01.y; g[w][2] = g23.x; g[w][3] = g23.y;
    y[w][0] = y01.x; y[w][1] = y01.y; y[w][2] = y23.x; y[w][3] = y23.y;
  }
  // QK-norm backward: d = r (g - y mean(g y)) per head
  float d[2][4];
#pragma unroll
  for (int w = 0; w < 2; ++w) {
    float dot = 0.f, r = 1.f;
    if (qk_norm) {
      dot = g[w][0] * y[w][0] + g[w][1] * y[w][1] + g[w][2] * y[w][2] + g[w][3] * y[w][3];
      dot = warp_sum(dot) * (1.f / 128.f);
      r = (w == 0 ? rstd_q : rstd_k)[(long long)n * H + h];
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) d[w][e] = r * (g[w][e] - y[w][e] * dot);
  }
  // RoPE backward: dx1 = dy1 c - dy2 s, dx2 = dy1 s + dy2 c, frequencies 4j..4j+3
  const float4* c4 = reinterpret_cast<const float4*>(cs + 2 * ((long long)t * 64 + 4 * j));
  const float4 ca = c4[0], cb = c4[1];
  const float cc[4] = {ca.x, ca.z, cb.x, cb.z}, ss[4] = {ca.y, ca.w, cb.y, cb.w};
#pragma unroll
  for (int w = 0; w < 2; ++w) {
    float o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float other = __shfl_xor_sync(0xffffffffu, d[w][e], 16);
      const float d1 = hf == 0 ? d[w][e] : other, d2 = hf == 0 ? other : d[w][e];
      o[e] = hf == 0 ? d1 * cc[e] - d2 * ss[e] : d1 * ss[e] + d2 * cc[e];
    }
    uint2 out;
    __nv_bfloat162 b01 = __floats2bfloat162_rn(o[0], o[1]), b23 = __floats2bfloat162_rn(o[2], o[3]);
    out.x = *reinterpret_cast<uint32_t*>(&b01);
    out.y = *reinterpret_cast<uint32_t*>(&b23);
    *reinterpret_cast<uint2*>(dqkv + base + w * a) = out;
  }
  if (gv) {  // value-table gradient: sum of dv over the layers, per position
    const uint2 rv = *reinterpret_cast<const uint2*>(dqkv + base + 2 * a);
    const float2 v01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&rv.x));
    const float2 v23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&rv.y));
    float4* dst = reinterpret_cast<float4*>(gv + (long long)n * a + h * 128 + i0);
    float4 acc = gv_accumulate ? *dst : make_float4(0.f, 0.f, 0.f, 0.f);
    acc.x += v01.x; acc.y += v01.y; acc.z += v23.x; acc.w += v23.y;
    *dst = acc;
  }
}

// --------------------------------------------------------------------------
// Cross-entropy over one chunk of rows of fp32 logits [rows, V], fused
// forward and backward ("$1000 tier nanochat run", `GPT.forward`: optional
// softcap c*tanh(z/c), logits in fp32, F.cross_entropy(ignore_index=-1)).
//   loss_t = logsumexp(z_t) - z_t[y_t]           (0 for ignored targets)
//   dlogits = (softmax(z_t) - onehot(y_t)) * scale * dz/dlogit
// scale = 1 / (n_valid * grad_accum) is read from the device.
template <typename act_t>
__global__ void __launch_bounds__(512) ce_chunk_kernel(float* __restrict__ logits,
                                                       act_t* __restrict__ dz,
                                                       const int32_t* __restrict__ targets,
                                                       float* __restrict__ tok_loss, int V,
                                                       float softcap, const float* __restrict__ scale_dev,
                                                       unsigned* err) {
  __shared__ float sh[32];
  const long long row = blockIdx.x;
  float* z = logits + row * V;
  act_t* g = dz + row * V;
  int y = targets[row];
  if (y < -1 || y >= V) {
    if (threadIdx.x == 0) set_error(err, GPT_EBIT_INPUT);
    y = -1;
  }
  float mx = -INFINITY;
  for (int i = threadIdx.x; i < V; i += blockDim.x) {
    float v = z[i];
    if (softcap > 0.f) { v = softcap * tanhf(v / softcap); z[i] = v; }
    mx = fmaxf(mx, v);
  }
  mx = block_max(mx, sh);
  float se = 0.f;
  for (int i = threadIdx.x; i < V; i += blockDim.x) se += expf(z[i] - mx);
  se = block_sum(se, sh);
  const float lse = mx + logf(se);
  if (threadIdx.x == 0) {
    const float l = (y >= 0) ? (lse - z[y]) : 0.f;
    tok_loss[row] = l;
    if (y >= 0 && !isfinite(l)) set_error(err, GPT_EBIT_NONFINITE);
  }
  const float sc = (y >= 0) ? *scale_dev : 0.f;
  for (int i = threadIdx.x; i < V; i += blockDim.x) {
    const float zi = z[i];
    float gi = (expf(zi - lse) - (i == y ? 1.f : 0.f)) * sc;
    if (softcap > 0.f) { const float tt = zi / softcap; gi *= (1.f - tt * tt); }
    g[i] = from_f<act_t>(gi);
  }
}

// Cross-entropy from the logits GEMM's block-local numerators (bf16 mode),
// one block per row: lse = M + log sum_j s_j exp(m_j - M) over the row's
// column blocks j (m_j block max, s_j = sum exp(z - m_j), M = max m_j); loss =
// lse - z[y]; and in place over the numerators e_c = exp(z_c - m_j):
// dz_c = (e_c exp(m_j - lse) - [c == y]) * scale (* (1 - (z_c/cap)^2) with a
// softcap, z_c recovered as m_j + log e_c).  ("$1000 tier nanochat run":
// cross-entropy over softcapped logits; the chunking keeps logits bounded.)
__global__ void __launch_bounds__(256) ce_prob_kernel(bf16* __restrict__ ez, const float2* __restrict__ stats,
                                                      int n_tiles, int tile_cols,
                                                      const int32_t* __restrict__ targets,
                                                      const float* __restrict__ ztgt,
                                                      float* __restrict__ tok_loss, int V, float softcap,
                                                      const float* __restrict__ scale_dev, unsigned* err) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  extern __shared__ float fac[];  // exp(m_j - lse) per column block
  __shared__ float sh[32];
  const long long row = blockIdx.x;
  bf16* g = ez + row * V;
  int y = targets[row];
  if (y < -1 || y >= V) {
    if (threadIdx.x == 0) set_error(err, GPT_EBIT_INPUT);
    y = -1;
  }
  const float2* st = stats + row * n_tiles;
  float mx = -INFINITY;
  for (int j = threadIdx.x; j < n_tiles; j += blockDim.x) mx = fmaxf(mx, st[j].x);
  mx = block_max(mx, sh);
  float se = 0.f;
  for (int j = threadIdx.x; j < n_tiles; j += blockDim.x) se += st[j].y * __expf(st[j].x - mx);
  se = block_sum(se, sh);
  const float lse = mx + logf(se);
  for (int j = threadIdx.x; j < n_tiles; j += blockDim.x) fac[j] = __expf(st[j].x - lse);
  if (threadIdx.x == 0) {
    const float l = (y >= 0) ? (lse - ztgt[row]) : 0.f;
    tok_loss[row] = l;
    if (y >= 0 && !isfinite(l)) set_error(err, GPT_EBIT_NONFINITE);
  }
  __syncthreads();
  const float sc = (y >= 0) ? *scale_dev : 0.f;
  const int stride = blockDim.x * 8;
  int i0 = threadIdx.x * 8;
  if (softcap <= 0.f && (V & 7) == 0) {
    // four 16-byte pieces per thread in flight: every load of the group is
    // requested before any of its stores (the buffer is rewritten in place)
    for (; i0 + 3 * stride + 8 <= V; i0 += 4 * stride) {
      uint4 raw[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) raw[u] = *reinterpret_cast<const uint4*>(g + i0 + u * stride);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * stride;
        const float f = fac[i / tile_cols];
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw[u]);
        uint4 out;
        __nv_bfloat162* ho = reinterpret_cast<__nv_bfloat162*>(&out);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 t = __bfloat1622float2(h[k]);
          const float o0 = (t.x * f - (i + 2 * k == y ? 1.f : 0.f)) * sc;
          const float o1 = (t.y * f - (i + 2 * k + 1 == y ? 1.f : 0.f)) * sc;
          ho[k] = __floats2bfloat162_rn(o0, o1);
        }
        *reinterpret_cast<uint4*>(g + i) = out;
      }
    }
  }
  for (int i = i0; i < V; i += stride) {
    // 8 columns never straddle a block (tile_cols is a multiple of 8)
    const int j = i / tile_cols;
    const float f = fac[j];
    const int nv = min(8, V - i);
    float e8[8];
    if (nv == 8 && (V & 7) == 0) {
      const uint4 raw = *reinterpret_cast<const uint4*>(g + i);
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 t = __bfloat1622float2(h[k]);
        e8[2 * k] = t.x;
        e8[2 * k + 1] = t.y;
      }
    } else {
      for (int k = 0; k < 8; ++k) e8[k] = k < nv ? __bfloat162float(g[i + k]) : 0.f;
    }
    float o[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) o[k] = (e8[k] * f - (i + k == y ? 1.f : 0.f)) * sc;
    if (softcap > 0.f) {  // block-uniform: the default path skips all of this
      const float inv = 1.f / softcap;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        // z = m_j + log e (e = 0: p = 0 and dz = 0 off the target anyway)
        const float tt = (i + k == y) ? ztgt[row] * inv : (e8[k] > 0.f ? (st[j].x + __logf(e8[k])) * inv : 1.f);
        o[k] *= (1.f - tt * tt);
      }
    }
    if (nv == 8 && (V & 7) == 0) {
      uint4 raw;
      __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
      for (int k = 0; k < 4; ++k) h[k] = __floats2bfloat162_rn(o[2 * k], o[2 * k + 1]);
      *reinterpret_cast<uint4*>(g + i) = raw;
    } else {
      for (int k = 0; k < nv; ++k) g[i + k] = __float2bfloat16_rn(o[k]);
    }
  }
}

// Counts non-ignored targets and sets scale = 1/(count * A) (single block).
__global__ void ce_prepare_kernel(const int32_t* __restrict__ targets, int N, int A,
                                  float* __restrict__ scale_out, int* __restrict__ count_out) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  __shared__ float sh[32];
  float c = 0.f;
  for (int i = threadIdx.x; i < N; i += blockDim.x) c += (targets[i] >= 0) ? 1.f : 0.f;
  c = block_sum(c, sh);
  if (threadIdx.x == 0) {
    const int n = (int)(c + 0.5f);
    *count_out = n;
    *scale_out = n > 0 ? 1.f / ((float)n * (float)A) : 0.f;
  }
}

// loss = sum(tok_loss) / count, summed in a fixed order (single block, fp64).
__global__ void loss_reduce_kernel(const float* __restrict__ tok_loss, int N,
                                   const int* __restrict__ count, float* __restrict__ loss_out,
                                   unsigned* err) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  __shared__ double sh[32];
  double s = 0.0;
  for (int i = threadIdx.x; i < N; i += blockDim.x) s += tok_loss[i];
  s = warp_sum_d(s);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (lane == 0) sh[wid] = s;
  __syncthreads();
  if (wid == 0) {
    double r = (lane < (int)(blockDim.x >> 5)) ? sh[lane] : 0.0;
    r = warp_sum_d(r);
    if (lane == 0) {
      const float l = *count > 0 ? (float)(r / *count) : 0.f;
      *loss_out = l;
      if (!isfinite(l)) set_error(err, GPT_EBIT_NONFINITE);
    }
  }
}

// --------------------------------------------------------------------------
// Causal softmax attention, SIMT reference kernels (any head_dim <= 128, any
// T; fp32 accumulation).  The fp32 mode's attention.  q, k, v are read from
// qkv [N, 3a]; o is [N, a]; lse [B*H, T] is the log-sum-exp of the scaled
// scores.  One warp per query row (forward, dq) or key row (dk, dv).
template <typename act_t>
__global__ void attn_fwd_simt_kernel(const act_t* __restrict__ qkv, act_t* __restrict__ o,
                                     float* __restrict__ lse_out, int B, int T, int H, int hd) {
  extern __shared__ float qs[];  // [warps][hd]
  const int wib = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * (blockDim.x >> 5) + wib;
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  if (i >= T) return;
  const int a = H * hd;
  const float scale = rsqrtf((float)hd);
  float* q = qs + wib * hd;
  const act_t* qrow = qkv + ((long long)b * T + i) * 3 * a + h * hd;
  for (int c = lane; c < hd; c += 32) q[c] = to_f(qrow[c]);
  __syncwarp();
  float m = -INFINITY, l = 0.f;
  for (int j = lane; j <= i; j += 32) {
    const act_t* krow = qkv + ((long long)b * T + j) * 3 * a + a + h * hd;
    float s = 0.f;
    for (int c = 0; c < hd; ++c) s = fmaf(q[c], to_f(krow[c]), s);
    s *= scale;
    const float mn = fmaxf(m, s);
    l = l * expf(m - mn) + expf(s - mn);
    m = mn;
  }
  const float M = warp_max(m);
  l = (m == -INFINITY) ? 0.f : l * expf(m - M);
  l = warp_sum(l);
  const float lse = M + logf(l);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int j0 = 0; j0 <= i; j0 += 32) {
    const int j = j0 + lane;
    float p = 0.f;
    if (j <= i) {
      const act_t* krow = qkv + ((long long)b * T + j) * 3 * a + a + h * hd;
      float s = 0.f;
      for (int c = 0; c < hd; ++c) s = fmaf(q[c], to_f(krow[c]), s);
      p = expf(s * scale - lse);
    }
    const int cnt = min(32, i - j0 + 1);
    for (int jj = 0; jj < cnt; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, p, jj);
      const act_t* vrow = qkv + ((long long)b * T + j0 + jj) * 3 * a + 2 * a + h * hd;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int c = lane + 32 * k;
        if (c < hd) acc[k] = fmaf(pj, to_f(vrow[c]), acc[k]);
      }
    }
  }
  act_t* orow = o + ((long long)b * T + i) * a + h * hd;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int c = lane + 32 * k;
    if (c < hd) orow[c] = from_f<act_t>(acc[k]);
  }
  if (lane == 0) lse_out[(long long)bh * T + i] = lse;
}

// D[bh, i] = sum_c dO[i, c] * O[i, c] for bf16 heads of 128: a warp takes
// ROWS (position, head) rows, two at a time (16 lanes a row, 16 bytes of each
// operand a lane), with all of its loads requested before any is used.
constexpr int ATTN_PRE_ROWS = 8;
__global__ void __launch_bounds__(256) attn_bwd_pre_hd128_kernel(const bf16* __restrict__ o,
                                                                 const bf16* __restrict__ dout,
                                                                 float* __restrict__ Dout, int B, int T, int H) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31, half = lane >> 4, ch = lane & 15;
  const long long rows = (long long)B * T * H, r0 = warp * ATTN_PRE_ROWS;
  if (r0 >= rows) return;  // whole warp
  uint4 ro[ATTN_PRE_ROWS / 2], rd[ATTN_PRE_ROWS / 2];
#pragma unroll
  for (int k = 0; k < ATTN_PRE_ROWS / 2; ++k) {
    const long long r = r0 + 2 * k + half;   // row = n * H + h, 128 contiguous values
    ro[k] = make_uint4(0u, 0u, 0u, 0u);
    rd[k] = ro[k];
    if (r < rows) {
      ro[k] = *reinterpret_cast<const uint4*>(o + r * 128 + 8 * ch);
      rd[k] = *reinterpret_cast<const uint4*>(dout + r * 128 + 8 * ch);
    }
  }
#pragma unroll
  for (int k = 0; k < ATTN_PRE_ROWS / 2; ++k) {
    const uint32_t wo[4] = {ro[k].x, ro[k].y, ro[k].z, ro[k].w}, wd[4] = {rd[k].x, rd[k].y, rd[k].z, rd[k].w};
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wo[q]));
      const float2 d = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wd[q]));
      s = fmaf(a.x, d.x, fmaf(a.y, d.y, s));
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    const long long r = r0 + 2 * k + half;
    if (ch == 0 && r < rows) {
      const long long n = r / H;
      const int h = (int)(r % H), b = (int)(n / T), t = (int)(n % T);
      Dout[((long long)b * H + h) * T + t] = s;
    }
  }
}

// D[bh, i] = sum_c dO[i, c] * O[i, c]  (softmax-backward row term)
template <typename act_t>
__global__ void attn_bwd_pre_kernel(const act_t* __restrict__ o, const act_t* __restrict__ dout,
                                    float* __restrict__ Dout, int B, int T, int H, int hd) {
  pdl_wait();     // the previous kernel in the stream has completed (programmatic launch)
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= B * T * H) return;
  const int n = warp / H, h = warp % H, b = n / T, t = n % T;
  const int a = H * hd;
  float s = 0.f;
  if (sizeof(act_t) == 2 && hd == 128) {
    // bf16 head of 128: 8 bytes (4 values) of each operand per lane
    const uint2 ro = *reinterpret_cast<const uint2*>(o + (long long)n * a + h * 128 + 4 * lane);
    const uint2 rd = *reinterpret_cast<const uint2*>(dout + (long long)n * a + h * 128 + 4 * lane);
    const float2 o01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ro.x));
    const float2 o23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ro.y));
    const float2 d01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&rd.x));
    const float2 d23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&rd.y));
    s = o01.x * d01.x + o01.y * d01.y + o23.x * d23.x + o23.y * d23.y;
  } else {
    for (int c = lane; c < hd; c += 32)
      s += to_f(o[(long long)n * a + h * hd + c]) * to_f(dout[(long long)n * a + h * hd + c]);
  }
  s = warp_sum(s);
  if (lane == 0) Dout[((long long)b * H + h) * T + t] = s;
}

// dq for one query row per warp: dq = scale * sum_j P_ij (dP_ij - D_i) k_j
template <typename act_t>
__global__ void attn_bwd_dq_simt_kernel(const act_t* __restrict__ qkv, const act_t* __restrict__ dout,
                                        const float* __restrict__ lse, const float* __restrict__ Dv,
                                        act_t* __restrict__ dqkv, int B, int T, int H, int hd) {
  extern __shared__ float sm[];  // [warps][2*hd]
  const int wib = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * (blockDim.x >> 5) + wib;
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  if (i >= T) return;
  const int a = H * hd;
  const float scale = rsqrtf((float)hd);
  float* q = sm + wib * 2 * hd;
  float* go = q + hd;
  const long long n = (long long)b * T + i;
  for (int c = lane; c < hd; c += 32) {
    q[c] = to_f(qkv[n * 3 * a + h * hd + c]);
    go[c] = to_f(dout[n * a + h * hd + c]);
  }
  __syncwarp();
  const float L = lse[(long long)bh * T + i], Di = Dv[(long long)bh * T + i];
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int j0 = 0; j0 <= i; j0 += 32) {
    const int j = j0 + lane;
    float ds = 0.f;
    if (j <= i) {
      const act_t* krow = qkv + ((long long)b * T + j) * 3 * a + a + h * hd;
      const act_t* vrow = krow + a;
      float s = 0.f, dp = 0.f;
      for (int c = 0; c < hd; ++c) {
        s = fmaf(q[c], to_f(krow[c]), s);
        dp = fmaf(go[c], to_f(vrow[c]), dp);
      }
      const float p = expf(s * scale - L);
      ds = p * (dp - Di);
    }
    const int cnt = min(32, i - j0 + 1);
    for (int jj = 0; jj < cnt; ++jj) {
      const float d = __shfl_sync(0xffffffffu, ds, jj);
      const act_t* krow = qkv + ((long long)b * T + j0 + jj) * 3 * a + a + h * hd;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int c = lane + 32 * k;
        if (c < hd) acc[k] = fmaf(d, to_f(krow[c]), acc[k]);
      }
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int c = lane + 32 * k;
    if (c < hd) dqkv[n * 3 * a + h * hd + c] = from_f<act_t>(acc[k] * scale);
  }
}

// dk, dv for one key row per warp: dv = sum_i P_ij dO_i, dk = scale * sum_i dS_ij q_i
template <typename act_t>
__global__ void attn_bwd_dkdv_simt_kernel(const act_t* __restrict__ qkv, const act_t* __restrict__ dout,
                                          const float* __restrict__ lse, const float* __restrict__ Dv,
                                          act_t* __restrict__ dqkv, int B, int T, int H, int hd) {
  extern __shared__ float sm[];  // [warps][2*hd]
  const int wib = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x * (blockDim.x >> 5) + wib;
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  if (j >= T) return;
  const int a = H * hd;
  const float scale = rsqrtf((float)hd);
  float* kk = sm + wib * 2 * hd;
  float* vv = kk + hd;
  const long long nj = (long long)b * T + j;
  for (int c = lane; c < hd; c += 32) {
    kk[c] = to_f(qkv[nj * 3 * a + a + h * hd + c]);
    vv[c] = to_f(qkv[nj * 3 * a + 2 * a + h * hd + c]);
  }
  __syncwarp();
  float dk[4] = {0.f, 0.f, 0.f, 0.f}, dv[4] = {0.f, 0.f, 0.f, 0.f};
  for (int i0 = j; i0 < T; i0 += 32) {
    const int i = i0 + lane;
    float p = 0.f, ds = 0.f;
    if (i < T) {
      const long long ni = (long long)b * T + i;
      const act_t* qrow = qkv + ni * 3 * a + h * hd;
      const act_t* grow = dout + ni * a + h * hd;
      float s = 0.f, dp = 0.f;
      for (int c = 0; c < hd; ++c) {
        s = fmaf(to_f(qrow[c]), kk[c], s);
        dp = fmaf(to_f(grow[c]), vv[c], dp);
      }
      p = expf(s * scale - lse[(long long)bh * T + i]);
      ds = p * (dp - Dv[(long long)bh * T + i]);
    }
    const int cnt = min(32, T - i0);
    for (int ii = 0; ii < cnt; ++ii) {
      const float pi = __shfl_sync(0xffffffffu, p, ii);
      const float di = __shfl_sync(0xffffffffu, ds, ii);
      const long long ni = (long long)b * T + i0 + ii;
      const act_t* qrow = qkv + ni * 3 * a + h * hd;
      const act_t* grow = dout + ni * a + h * hd;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int c = lane + 32 * k;
        if (c < hd) {
          dv[k] = fmaf(pi, to_f(grow[c]), dv[k]);
          dk[k] = fmaf(di, to_f(qrow[c]), dk[k]);
        }
      }
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int c = lane + 32 * k;
    if (c < hd) {
      dqkv[nj * 3 * a + a + h * hd + c] = from_f<act_t>(dk[k] * scale);
      dqkv[nj * 3 * a + 2 * a + h * hd + c] = from_f<act_t>(dv[k]);
    }
  }
}
