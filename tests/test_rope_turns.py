"""The RoPE angle reduction the QKV GEMM epilogue uses, replayed on the host.

The epilogue gets cos / sin of t * theta_f (theta_f = base^(-2f/hd), the
rotary frequencies of "$1000 tier nanochat run", apply_rotary_emb) from the
frequency's turns per position u = theta_f / (2 pi), stored as an fp32 pair
hi + lo: t hi = p + e exactly (p the fp32 product, e = fma(t, hi, -p) its
rounding error), the whole turns rint(p) drop out exactly, and the fraction
(p - k) + fma(t, lo, e) in [-1/2, 1/2] goes to sin / cos.  Each fp32 step is
replayed here exactly (float64 holds the products and the fused sums before
their single rounding to float32), and the result is checked against the
float64 cos / sin of t * theta_f for every position below 2^16.
"""

import numpy as np

F32 = np.float32


def turns_table(hd=128, base=10000.0):
    f = np.arange(hd // 2)
    inv_freq = 1.0 / np.power(base, (2.0 * f) / hd)
    u = inv_freq / (2.0 * np.pi)
    hi = u.astype(F32)
    lo = (u - hi.astype(np.float64)).astype(F32)
    return inv_freq, hi, lo


def reduced_angle(t, hi, lo):
    """The epilogue's fp32 steps, each rounded once as the GPU rounds it."""
    t64 = t.astype(np.float64)
    prod = t64 * hi.astype(np.float64)            # exact: <= 17 + 24 significant bits
    p = prod.astype(F32)                           # t * hi rounded
    e = (prod - p.astype(np.float64)).astype(F32)  # fma(t, hi, -p): exact in fp32
    k = np.rint(p).astype(F32)
    d = (p.astype(np.float64) - k.astype(np.float64)).astype(F32)          # exact (Sterbenz)
    tl = (t64 * lo.astype(np.float64) + e.astype(np.float64)).astype(F32)  # fma(t, lo, e)
    fr = (d.astype(np.float64) + tl.astype(np.float64)).astype(F32)
    return (F32(2.0 * np.pi) * fr).astype(np.float64)   # the argument handed to sin / cos


def test_turns_split_is_exact_fp32_pair():
    inv_freq, hi, lo = turns_table()
    u = inv_freq / (2.0 * np.pi)
    # hi + lo carries u to ~2^-48 relative, far below fp32 resolution
    assert np.all(np.abs(hi.astype(np.float64) + lo.astype(np.float64) - u) <= 4e-15 * u)
    assert hi[0] == F32(1.0 / (2.0 * np.pi))


def test_reduced_angle_matches_fp64_rotation_below_2_16():
    inv_freq, hi, lo = turns_table()
    t = np.arange(1 << 16)
    worst = 0.0
    for f in range(len(hi)):
        x = reduced_angle(t, hi[f], lo[f])
        assert np.all(np.abs(x) <= np.pi + 0.01)          # half a turn, up to the small low-word term
        th = t * inv_freq[f]
        err = max(np.max(np.abs(np.cos(x) - np.cos(th))), np.max(np.abs(np.sin(x) - np.sin(th))))
        worst = max(worst, err)
    # the reduction itself is good to ~1e-6 absolute (the special-function
    # unit then adds its own error on [-pi, pi]); bf16 outputs round at ~4e-3
    assert worst < 1e-6, worst


def test_reduced_angle_catches_a_dropped_low_word():
    """Without the lo word (u rounded to fp32 alone) the angle drifts by
    t * |u - hi| * 2 pi, which is far above the bound at long positions:
    the test above would fail on that mistake."""
    inv_freq, hi, lo = turns_table()
    t = np.arange(1 << 16)
    x = reduced_angle(t, hi[0], np.zeros_like(lo[0]))
    th = t * inv_freq[0]
    assert np.max(np.abs(np.cos(x) - np.cos(th))) > 1e-5
