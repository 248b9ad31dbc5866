"""FP8 (e4m3) GEMM path (fp64 oracle; test infrastructure only, see
oracle/__init__.py).

Karpathy's llm.c post lists FP8 training as "imminent"; the decoder-rtx posts
train without FP8.  The pages give no recipe, so the readings here are the
plainest per-tensor form:

  * format e4m3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; no
    infinities, the all-ones exponent and mantissa is NaN, largest finite
    value 448, subnormals m/8 * 2^-6);
  * per-tensor scaling: amax = max |x|, inv = 448 / amax (1 when amax is 0),
    code = e4m3(x * inv) rounded to nearest, ties to the even code, values
    beyond 448 saturated to +-448; the tensor's scale is s = amax / 448;
  * product: C = (s_a s_b) * sum_k A_q[m, k] B_q[n, k] with the codes decoded.

Where floating point decides a code, the scaled value x * inv is formed in
fp32 exactly as the kernel forms it (inv an fp32 division, then one fp32
multiply), so the decision is taken in the same precision on both sides.
"""

import numpy as np

E4M3_MAX = 448.0


def e4m3_decode(codes):
    """Values of e4m3 codes (uint8 array) as float64; NaN codes give nan."""
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * 2.0 ** (e - 7))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return sign * val


def _positive_grid():
    codes = np.arange(0, 0x7F)          # 0x00 .. 0x7E: every non-negative finite value, increasing
    return codes, e4m3_decode(codes)


def e4m3_encode(x):
    """Nearest e4m3 code of every value of x (ties to the code with an even
    mantissa), saturating beyond +-448; NaN gives 0x7F."""
    x = np.asarray(x, dtype=np.float64)
    codes, grid = _positive_grid()
    a = np.abs(x)
    idx = np.searchsorted(grid, np.minimum(a, E4M3_MAX))       # grid[idx-1] < a <= grid[idx]
    idx = np.clip(idx, 1, len(grid) - 1)
    lo, hi = grid[idx - 1], grid[idx]
    take_hi = (hi - a < a - lo) | ((hi - a == a - lo) & (codes[idx] % 2 == 0))
    out = np.where(take_hi, codes[idx], codes[idx - 1])
    out = np.where(a == 0, 0, out)
    out = np.where(a >= E4M3_MAX, 0x7E, out)
    out = out | np.where(np.signbit(x), 0x80, 0)                # the sign survives rounding to zero
    out = np.where(np.isnan(x), 0x7F, out)
    return out.astype(np.uint8)


def quantize(x):
    """Per-tensor e4m3 quantization: (codes uint8, scale s as fp32)."""
    x32 = np.asarray(x, dtype=np.float32)
    amax = np.float32(np.max(np.abs(x32))) if x32.size else np.float32(0)
    inv = np.float32(E4M3_MAX) / amax if amax > 0 else np.float32(1.0)
    scale = amax / np.float32(E4M3_MAX) if amax > 0 else np.float32(1.0)
    v = (x32 * np.float32(inv)).astype(np.float32)            # one fp32 multiply, as the kernel
    return e4m3_encode(v.astype(np.float64)), np.float32(scale)


def gemm(qa, sa, qb, sb):
    """C [M, N] = (sa * sb) * decode(qa) [M, K] @ decode(qb) [N, K]^T in fp64."""
    return (float(sa) * float(sb)) * (e4m3_decode(qa) @ e4m3_decode(qb).T)
