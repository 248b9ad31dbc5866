"""Training-step semantics of the library, restated in fp64 (test infrastructure).

Mirrors the two calls of the C library: ``forward_loss`` then
``backward_step(lr)``.  Gradient accumulation follows the nanochat training
loop (nanochat discussion #8, pasted loop: loss / gradient_accumulation_steps,
backward every micro-batch, clip + optimizer step + zero_grad every
``grad_accum`` micro-batches).  The bigram tables are updated inside every
backward call from that micro-batch's gradient (the decoder-rtx posts inline
the table optimizer into backward, so no table gradient survives the call).

With ``matrix_optimizer == "muon"`` the block matrices take Muon and only the
embedding and the head take AdamW, as in the nanochat setup
(``setup_optimizers``: Muon for the transformer matrices, AdamW for the rest;
the pasted training loop clips the gradient norm of all parameters before
either optimizer steps).  The fused q|k|v weight is three matrices to Muon
(nanochat's separate ``c_q``, ``c_k``, ``c_v``), each orthogonalised on its
own; the attention projection and the two MLP weights are one matrix each.
"""

import numpy as np

from . import model, muon, optim
from .hashing import bigram_rows
from .trigram import P3, trigram_rows


def muon_blocks(cfg, name, shape):
    """Row ranges of a dense parameter that Muon treats as separate matrices
    ([] for parameters that AdamW steps)."""
    if not name.startswith("h"):
        return []
    if name.endswith(".wqkv"):
        a = cfg["n_head"] * cfg["head_dim"]
        return [(0, a), (a, 2 * a), (2 * a, 3 * a)]
    return [(0, shape[0])]


class OracleTrainer:
    def __init__(self, cfg, params, table_state=None):
        self.cfg = cfg
        self.P = {k: np.array(v, dtype=np.float64) for k, v in params.items()}
        self.dense = [k for k in self.P if k not in ("hx", "hv", "h3")]
        self.m = {k: np.zeros_like(self.P[k]) for k in self.dense}
        self.v = {k: np.zeros_like(self.P[k]) for k in self.dense}
        self.acc = {k: np.zeros_like(self.P[k]) for k in self.dense}
        self.S = {}
        for t in ("hx", "hv"):
            if t in self.P:
                rows = self.P[t].shape[0]
                self.S[t] = (np.zeros(rows) if table_state is None
                             else np.array(table_state[t], dtype=np.float64))
        self.micro = 0
        self.t = 0
        self.cache = None
        self.last_grads = None
        self.last_updated_rows = {}

    def rows(self, tokens):
        cfg = self.cfg
        rx = rv = None
        if cfg["x0_rows"]:
            rx = bigram_rows(tokens, cfg["vocab"], cfg["hash_p1"], cfg["hash_p2"],
                             cfg["x0_rows"])
        if cfg["v_rows"]:
            rv = bigram_rows(tokens, cfg["vocab"], cfg["hash_p1"], cfg["hash_p2"],
                             cfg["v_rows"])
        return rx, rv

    def rows3(self, tokens):
        cfg = self.cfg
        if not cfg.get("tri_rows", 0):
            return None
        return trigram_rows(tokens, cfg["vocab"], cfg["hash_p1"], cfg["hash_p2"], cfg["tri_rows"],
                            cfg.get("hash_p3", P3))

    def forward_loss(self, tokens, targets):
        rx, rv = self.rows(tokens)
        loss, per_tok, c = model.forward(self.cfg, self.P, tokens, targets, rx, rv, self.rows3(tokens))
        c["rx"], c["rv"] = rx, rv
        self.cache = c
        return loss, per_tok

    def backward_step(self, lr):
        cfg = self.cfg
        A = cfg["grad_accum"]
        G, gx0, gv = model.backward(cfg, self.P, self.cache, scale=1.0 / A)
        self.last_grads = G
        self.last_gx0, self.last_gv = gx0, gv
        for k in self.dense:
            self.acc[k] += G[k]
        lr_t = lr * cfg["lr_mult_table"]
        if "hv" in self.P:
            self.P["hv"], self.S["hv"], self.last_updated_rows["hv"] = optim.table_update(
                self.P["hv"], self.S["hv"], self.cache["rv"], gv, lr_t,
                cfg["table_beta"], cfg["table_eps"])
        if "hx" in self.P:
            self.P["hx"], self.S["hx"], self.last_updated_rows["hx"] = optim.table_update(
                self.P["hx"], self.S["hx"], self.cache["rx"], gx0, lr_t,
                cfg["table_beta"], cfg["table_eps"])
        self.micro += 1
        stepped = False
        if self.micro == A:
            self.optimizer_step(lr)
            stepped = True
        self.cache = None
        return stepped

    def optimizer_step(self, lr):
        """Clip, then AdamW (and Muon on the block matrices when configured)
        over the accumulated gradient ``self.acc``; zeroes it."""
        cfg = self.cfg
        self.accum_grads = {k: self.acc[k].copy() for k in self.dense}
        coef = optim.clip_coef([self.acc[k] for k in self.dense], cfg["grad_clip"])
        self.t += 1
        use_muon = cfg.get("matrix_optimizer", "adamw") == "muon"
        for k in self.dense:
            mult = (cfg["lr_mult_embed"] if k == "wte" else
                    cfg["lr_mult_head"] if k == "lm_head" else
                    cfg["lr_mult_matrix"])
            blocks = muon_blocks(cfg, k, self.P[k].shape) if use_muon else []
            if blocks:
                # Muon on each block; the AdamW first moment buffer holds its momentum
                g = self.acc[k] * coef
                for r0, r1 in blocks:
                    self.P[k][r0:r1], self.m[k][r0:r1] = muon.muon_update(
                        self.P[k][r0:r1], g[r0:r1], self.m[k][r0:r1], lr * mult,
                        cfg.get("muon_momentum", 0.95), nesterov=bool(cfg.get("muon_nesterov", 1)),
                        steps=cfg.get("muon_ns_steps", 5))
                self.acc[k][...] = 0.0
                continue
            self.P[k], self.m[k], self.v[k] = optim.adamw(
                self.P[k], self.acc[k] * coef, self.m[k], self.v[k], self.t,
                lr * mult, cfg["adam_b1"], cfg["adam_b2"], cfg["adam_eps"],
                cfg["weight_decay"])
            self.acc[k][...] = 0.0
        self.micro = 0
