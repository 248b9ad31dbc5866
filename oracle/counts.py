"""Parameter and FLOP counts (oracle; test infrastructure only).

nanochat discussion #8, pasted ``GPT.estimate_flops`` (PaLM appendix B form):
flops/token = 6 * (matmul parameters) + 12 * l * h * q * t with l layers, h
heads, q head dim, t sequence length.  The pasted code subtracts the input
embedding from all parameters, which counts the untied LM head once; the same
reading is applied to tied models by counting the shared matrix once as the LM
head.  Table parameters are lookups and carry no matmul FLOPs.
"""


def num_params(cfg):
    """(dense, table) parameter counts."""
    d, H, hd, F, V = (cfg["d_model"], cfg["n_head"], cfg["head_dim"],
                      cfg["d_ff"], cfg["vocab"])
    a = H * hd
    per_layer = 3 * a * d + d * a + F * d + d * F
    dense = V * d + cfg["n_layer"] * per_layer
    if not cfg["tie_embeddings"]:
        dense += V * d
    table = cfg["x0_rows"] * d + cfg["v_rows"] * a
    return dense, table


def flops_per_token(cfg, causal=False):
    """Training FLOPs per token; ``causal`` halves the attention term."""
    d, H, hd, F, V, L, T = (cfg["d_model"], cfg["n_head"], cfg["head_dim"],
                            cfg["d_ff"], cfg["vocab"], cfg["n_layer"],
                            cfg["seq_len"])
    a = H * hd
    mat = L * (3 * a * d + d * a + F * d + d * F) + V * d
    attn = 12 * L * H * hd * T
    if causal:
        attn //= 2
    return 6 * mat + attn
