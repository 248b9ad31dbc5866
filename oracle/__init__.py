"""fp64 CPU oracle of the decoder training step -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously correct NumPy float64 code for what the CUDA library
computes: the forward pass, a hand-derived backward pass, the hashed bigram
tables with their sparse per-row-magnitude update, and AdamW.  It shares no
code with the CUDA path; only the seeded input generators in ``synthetic``
feed both.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import it -- the product path never does.

Sources (each function names the passage it follows):
  * nanochat discussion #8 "$1000 tier nanochat run" -- the user-pasted GPT
    module: ``norm``, ``apply_rotary_emb``, ``_precompute_rotary_embeddings``,
    ``CausalSelfAttention.forward``, ``Block.forward``, ``GPT.forward``,
    ``GPT.estimate_flops``, ``setup_optimizers`` (AdamW betas/eps) and the
    training loop (gradient accumulation, clipping);
  * modded-nanogpt README, "Other general differences": rotary embeddings,
    ReLU^2 activation, RMSNorm without affine parameters;
  * Chris McCormick's decoder-rtx posts: hand-written backward, bigram hash
    tables added to x0 and to the attention values, "sparse, no first moment,
    and only per-row magnitude" optimizer inlined into their backward;
  * modded-nanogpt README "Proposed optimizer" and the nanochat page's
    ``zeropower_via_newtonschulz5`` / ``Muon.step``: Muon for the matrix
    parameters (``muon``; no CUDA path yet).

Parity status per function is listed in ``PINS`` below; every entry is pinned
by a ``-m "not gpu"`` test in tests/test_oracle_*.py.
"""

PINS = {
    "hashing.bigram_keys": "hand-worked golden example + pure-int brute force",
    "model.rmsnorm": "torch.nn.functional.rms_norm; unit-RMS invariant",
    "model.rope": "complex-multiplication identity; norm preservation; t=0 identity",
    "model.causal_attention": "torch scaled_dot_product_attention(is_causal); rows sum to 1",
    "model.forward": "torch fp64 module built from library ops; ln V closed form; causality",
    "model.backward": "central finite differences; torch autograd of the library-op module",
    "optim.adamw": "closed-form first step -lr*sign(g); torch.optim.AdamW",
    "optim.table_update": "closed-form first step; two-step recurrence by hand",
    "counts.num_params / flops_per_token": "nanochat d32 printed values",
    "muon.newton_schulz": "singular values through the scalar quintic (known SVD); cubic coefficients "
                          "converge to numpy's polar factor; the pages' (0.5, 1.5) spread",
    "muon.muon_update": "closed-form Nesterov / plain momentum directions; sqrt(out/in) step scale "
                        "through the step's singular values",
}
