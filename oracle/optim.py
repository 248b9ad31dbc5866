"""Optimizers of the training step (fp64 oracle; test infrastructure only).

* AdamW for the dense weights -- nanochat discussion #8, pasted
  ``setup_optimizers``: ``torch.optim.AdamW`` with betas (0.8, 0.95), eps 1e-10,
  weight decay 0 (the report lists weight_decay 0.0000); optional global-norm
  clipping as in the training loop's ``clip_grad_norm_(..., max_norm=1.0)``.
* The bigram-table optimizer of Chris McCormick's decoder-rtx posts: "sparse,
  no first moment, and only per-row magnitude", inlined into the tables'
  backward so that no table gradient buffer exists.  Reading taken: a lazy
  RMSprop with one scalar second moment per row, s_r <- beta*s_r + (1-beta) *
  mean(G_r^2), W_r <- W_r - lr * G_r / (sqrt(s_r) + eps), applied to touched
  rows only, no bias correction.
"""

import numpy as np


def clip_coef(grads, max_norm):
    """Global-L2 clip coefficient min(1, max_norm / (||g|| + 1e-6)) as in
    ``torch.nn.utils.clip_grad_norm_``; 1.0 when max_norm <= 0."""
    if max_norm <= 0:
        return 1.0
    total = np.sqrt(sum(float(np.sum(g * g)) for g in grads))
    return min(1.0, max_norm / (total + 1e-6))


def adamw(p, g, m, v, t, lr, b1, b2, eps, wd):
    """One AdamW step (torch semantics, decoupled decay) at step number t >= 1.

    Returns the new (p, m, v).
    """
    m = b1 * m + (1.0 - b1) * g
    v = b2 * v + (1.0 - b2) * g * g
    p = p * (1.0 - lr * wd)
    mhat = m / (1.0 - b1 ** t)
    vhat = v / (1.0 - b2 ** t)
    p = p - lr * mhat / (np.sqrt(vhat) + eps)
    return p, m, v


def table_update(W, s, rows, g, lr, beta, eps):
    """Sparse per-row-magnitude update of a bigram table.

    W [R, d] table, s [R] per-row second moments, rows [N] row of each
    position, g [N, d] gradient of each position.  For each touched row r:
    G = sum of g over its positions; m = mean(G^2); s_r = beta*s_r + (1-beta)*m;
    W_r -= lr * G / (sqrt(s_r) + eps).  Returns (W, s, sorted unique rows).
    """
    W = W.copy()
    s = s.copy()
    rows = np.asarray(rows).reshape(-1)
    uniq = np.unique(rows)
    for r in uniq:
        Gr = g[rows == r].sum(axis=0)
        m = float(np.mean(Gr * Gr))
        s[r] = beta * s[r] + (1.0 - beta) * m
        W[r] = W[r] - lr * Gr / (np.sqrt(s[r]) + eps)
    return W, s, uniq
