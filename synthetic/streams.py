"""Seeded token streams and initial weights.

Token streams stand in for the FineWeb token shards the pages train on (the
modded-nanogpt README and the nanochat $1000-tier run both train on FineWeb);
no dataset is available, so tokens are drawn i.i.d. from a Zipf(s) law over
the vocabulary: p_k proportional to (k+1)^-s, token id = rank, so id 0 is the
most frequent.  Sampling is by inverse CDF on uniforms from numpy's PCG64.

Initial weights are N(0, init_std) from the same generator family.  In the
bf16 workloads every weight and table value is rounded to the nearest bf16 so
that the fp32 master copy and the bf16 copy used by the kernels start equal.
"""

import numpy as np


def _zipf_cdf(vocab, s):
    k = np.arange(1, vocab + 1, dtype=np.float64)
    p = k ** (-s)
    c = np.cumsum(p)
    return c / c[-1]


def zipf_stream(n, vocab, seed, s=1.1):
    """n i.i.d. Zipf(s) token ids in [0, vocab) as int64."""
    rng = np.random.Generator(np.random.PCG64(seed))
    u = rng.random(n)
    ids = np.searchsorted(_zipf_cdf(vocab, s), u, side="right")
    return np.minimum(ids, vocab - 1).astype(np.int64)


def repeated_spans(seqs, seed, frac=0.10, span=256):
    """Overwrite ~frac of each sequence with copies of earlier spans.

    Per sequence, non-overlapping span-aligned destination slots with start
    >= span are picked uniformly to cover ``frac`` of the positions; each is
    overwritten by a copy of an earlier span whose source start is uniform in
    [0, dst - span].  ``seqs`` is [B, T+1] and is modified in place.
    """
    rng = np.random.Generator(np.random.PCG64(seed + 7919))
    B, L = seqs.shape
    slots = np.arange(span, L - span + 1, span)
    n_dst = int(round(frac * L / span))
    for b in range(B):
        if n_dst == 0 or len(slots) == 0:
            continue
        dst = np.sort(rng.choice(slots, size=min(n_dst, len(slots)), replace=False))
        for d in dst:
            src = int(rng.integers(0, d - span + 1))
            seqs[b, d:d + span] = seqs[b, src:src + span].copy()
    return seqs


def tokens_and_targets(B, T, vocab, seed, s=1.1, repeat_frac=0.0, span=256,
                       ignore_frac=0.0, micro=0):
    """Tokens [B, T] and next-token targets [B, T] as int32.

    Each sequence draws T+1 ids; tokens = s[:T], targets = s[1:].  ``micro``
    selects an independent micro-batch of the same stream family.  With
    ``ignore_frac`` > 0 that fraction of targets is set to -1 (ignored).
    """
    sub = seed * 1000003 + micro
    seqs = zipf_stream(B * (T + 1), vocab, sub, s).reshape(B, T + 1)
    if repeat_frac > 0:
        repeated_spans(seqs, sub, repeat_frac, span)
    tok = np.ascontiguousarray(seqs[:, :T]).astype(np.int32)
    tgt = np.ascontiguousarray(seqs[:, 1:]).astype(np.int32)
    if ignore_frac > 0:
        rng = np.random.Generator(np.random.PCG64(sub + 17))
        tgt[rng.random(tgt.shape) < ignore_frac] = -1
    return tok, tgt


def round_to_bf16(a):
    """Round float values to the nearest bf16 (ties to even); returns float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    bits = a.view(np.uint32).astype(np.uint64)
    bias = 0x7FFF + ((bits >> 16) & 1)
    out = ((bits + bias) >> 16) << 16
    return out.astype(np.uint32).view(np.float32).reshape(a.shape)


def param_shapes(cfg):
    """Ordered {name: shape} of every trainable tensor in the exported layout.

    Linear weights follow the (out, in) convention: y = x @ W.T.  The fused
    attention input projection stacks q, k and v heads along its rows.
    """
    d, H, hd, F, V = (cfg["d_model"], cfg["n_head"], cfg["head_dim"],
                      cfg["d_ff"], cfg["vocab"])
    a = H * hd
    out = {"wte": (V, d)}
    if not cfg["tie_embeddings"]:
        out["lm_head"] = (V, d)
    if cfg.get("tri_rows", 0):
        out["vproj"] = (a, cfg["tri_width"])   # projection of the frozen trigram statistics
    for layer in range(cfg["n_layer"]):
        out[f"h{layer}.wqkv"] = (3 * a, d)
        out[f"h{layer}.wo"] = (d, a)
        out[f"h{layer}.w1"] = (F, d)
        out[f"h{layer}.w2"] = (d, F)
    if cfg["x0_rows"]:
        out["hx"] = (cfg["x0_rows"], d)
    if cfg["v_rows"]:
        out["hv"] = (cfg["v_rows"], a)
    return out


def init_params(cfg, seed=None, std=None, skip_tables=False):
    """Seeded N(0, std) initial values for every tensor of ``param_shapes``.

    Returned as float64 arrays (rounded through bf16 first in bf16 mode).
    Tables can be skipped for workloads whose tables are too large to build
    on the host; their rows are then handled by row-sampled checks.
    """
    seed = cfg["seed"] if seed is None else seed
    std = cfg["init_std"] if std is None else std
    rng = np.random.Generator(np.random.PCG64(seed * 7 + 3))
    out = {}
    for name, shape in param_shapes(cfg).items():
        if skip_tables and name in ("hx", "hv"):
            continue
        w = (rng.standard_normal(shape, dtype=np.float32) * np.float32(std))
        if cfg["dtype"] == "bf16":
            w = round_to_bf16(w)
        out[name] = w.astype(np.float64)
    return out
