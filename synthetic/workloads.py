"""Workload shapes of the five decoder configurations and the small parity cases.

Each workload is a plain dict whose keys mirror the fields of the C struct
``gpt_config`` (include/gpt.h).  Values not fixed by the pages are the readings
recorded in the design notes (hash constants, eps, table optimizer constants).

Sources of the shapes:
  * tiny fp32 decoder with a 1024-row x0 table;
  * GPT-2-small-style decoder (12 x 768, 6 heads of 128, MLP 3072, tied vocab
    50304, seq 1024, micro-batch 32) -- the shape of the modded-nanogpt 124M
    record ("Modded-NanoGPT" README, "architectural modernizations");
  * the same decoder at seq 2048 with 192K tokens per step via gradient
    accumulation plus the two hashed bigram tables of the decoder-rtx run
    (Chris McCormick's posts: "Two huge bi-gram hash tables: 2M rows, added to
    x0; 1M rows, added to values", "Batch size of 192K");
  * nanochat d32 shape (nanochat discussion #8, run1000.sh notes: 32 layers,
    model_dim 2048, 16 heads, vocab 65,536, 8 x 2048 tokens per micro-batch);
  * a long-context sweep at a fixed 64K tokens per step.
"""

import copy

_BASE = dict(
    n_layer=2, d_model=128, n_head=4, head_dim=32, d_ff=512, vocab=512,
    seq_len=64, micro_batch=4, grad_accum=1,
    dtype="f32", tie_embeddings=1, qk_norm=1,
    rope_base=10000.0, norm_eps=1.1920929e-07, softcap=0.0, init_std=0.02,
    adam_b1=0.8, adam_b2=0.95, adam_eps=1e-10, weight_decay=0.0, grad_clip=0.0,
    lr_mult_embed=1.0, lr_mult_head=1.0, lr_mult_matrix=1.0, lr_mult_table=1.0,
    x0_rows=0, v_rows=0, table_beta=0.95, table_eps=1e-10,
    hash_p1=2654435761, hash_p2=2246822519,
    tri_rows=0, tri_width=64, hash_p3=3266489917,
    seed=0, zipf_s=1.1, repeat_frac=0.0, repeat_span=256,
)


def _mk(**kw):
    w = copy.deepcopy(_BASE)
    w.update(kw)
    return w


WORKLOADS = {
    # tiny decoder, fp32 (oracle-tight mode)
    "tiny_fp32": _mk(name="tiny_fp32", x0_rows=1024, seed=0),
    # GPT-2-small-style decoder, bf16, 32K tokens per step
    "gpt2s_bf16": _mk(name="gpt2s_bf16", dtype="bf16", n_layer=12, d_model=768,
                      n_head=6, head_dim=128, d_ff=3072, vocab=50304,
                      seq_len=1024, micro_batch=32, seed=1),
    # same decoder, seq 2048, 6 x 32K = 192K tokens per step, both bigram tables
    "gpt2s_tables_bf16": _mk(name="gpt2s_tables_bf16", dtype="bf16", n_layer=12,
                             d_model=768, n_head=6, head_dim=128, d_ff=3072,
                             vocab=50304, seq_len=2048, micro_batch=16,
                             grad_accum=6, x0_rows=2097152, v_rows=1048576,
                             seed=2),
    # nanochat-d32-shaped decoder, untied head, ~1.88B parameters
    "d32_bf16": _mk(name="d32_bf16", dtype="bf16", n_layer=32, d_model=2048,
                    n_head=16, head_dim=128, d_ff=8192, vocab=65536,
                    seq_len=2048, micro_batch=8, tie_embeddings=0, seed=3),
}
for _T, _B in ((2048, 32), (4096, 16), (8192, 8), (16384, 4)):
    WORKLOADS[f"long{_T}_bf16"] = _mk(
        name=f"long{_T}_bf16", dtype="bf16", n_layer=16, d_model=1024, n_head=8,
        head_dim=128, d_ff=4096, vocab=50304, seq_len=_T, micro_batch=_B,
        seed=4, repeat_frac=0.10)


def workload(name, **overrides):
    """Return a copy of a named workload with optional field overrides."""
    w = copy.deepcopy(WORKLOADS[name])
    w.update(overrides)
    return w


def small_case(name, **overrides):
    """A reduced copy of a workload that the fp64 oracle finishes in seconds.

    Widths (d_model, heads, head_dim, d_ff) are kept so the kernels run the
    same tile shapes; depth, batch, sequence and vocab shrink.  The sequence
    length is chosen so that it is not a multiple of the 128-row tiles.
    """
    w = workload(name)
    if w["dtype"] == "bf16":
        w.update(n_layer=2, seq_len=200, micro_batch=2, vocab=4096 + 64,
                 grad_accum=1)
        if w["x0_rows"]:
            w.update(x0_rows=4096, v_rows=2048)
    w.update(overrides)
    return w
