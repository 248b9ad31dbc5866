"""Muon for the matrix parameters (fp64 oracle; test infrastructure only).

What it computes, from two of the pages:
  * modded-nanogpt README, "Proposed optimizer": SGD with Nesterov momentum
    whose update is orthogonalised by a quintic Newton-Schulz iteration
    (coefficients chosen for the largest slope at zero, five steps, the
    matrix first scaled by its Frobenius norm plus 1e-7, a tall matrix
    handled through its transpose);
  * nanochat discussion #8 "$1000 tier nanochat run", the pasted
    ``zeropower_via_newtonschulz5`` and ``Muon.step``: the same iteration
    written as A = X X^T, B = b A + c A^2, X <- a X + B X; the momentum buffer
    moved toward the gradient by (1 - momentum); the Nesterov direction
    (1 - momentum) g + momentum * buffer; the step scaled by
    sqrt(max(1, rows / cols)) of the weight in its [out, in] layout; and the
    momentum schedule 0.85 -> 0.95 over the first 300 steps.

Both pages run the iteration in bf16 on the GPU; here it is float64, so it
gives the exact polynomial of the normalised input that the bf16 iteration
approximates.  Readings where the pages leave a step open:
  * the two pages order "scale by the norm" and "transpose" differently; the
    Frobenius norm does not change under transposition, so they agree;
  * the step scale uses the weight's [out, in] (nn.Linear) orientation: a
    caller that stores a weight as [in, out] passes its transpose;
  * ``nesterov=False`` uses the buffer itself as the direction.
"""

import numpy as np

NS5_COEFFS = (3.4445, -4.7750, 2.0315)  # (a, b, c) of a x + b x^3 + c x^5
NS_EPS = 1e-7


def newton_schulz(G, steps=5, coeffs=NS5_COEFFS, eps=NS_EPS):
    """Zeroth-power (orthogonalisation) iteration of a 2-D matrix G.

    X = G / (||G||_F + eps), taken as its transpose when G has more rows
    than columns so X is wide; then ``steps`` times
    X <- a X + (b A + c A A) X with A = X X^T; the result has G's shape.
    On G = U diag(s) V^T this maps every singular value s_i to
    f(s_i / (||s|| + eps)) with f the scalar polynomial a x + b x^3 + c x^5
    applied ``steps`` times, and keeps U and V.
    """
    G = np.asarray(G, dtype=np.float64)
    if G.ndim != 2:
        raise ValueError("newton_schulz expects a 2-D matrix")
    a, b, c = coeffs
    tall = G.shape[0] > G.shape[1]
    X = G.T if tall else G
    X = X / (np.linalg.norm(X) + eps)  # Frobenius norm
    for _ in range(steps):
        A = X @ X.T
        B = b * A + c * (A @ A)
        X = a * X + B @ X
    return X.T if tall else X


def muon_momentum(step):
    """Momentum at optimizer step ``step`` (0-based): linear from 0.85 to
    0.95 over the first 300 steps, then 0.95."""
    frac = min(step / 300.0, 1.0)
    return (1.0 - frac) * 0.85 + frac * 0.95


def muon_update(W, G, M, lr, momentum, nesterov=True, steps=5):
    """One Muon step of a weight W [out, in] with gradient G and momentum
    buffer M (same shape).  Returns (new W, new M):

      M <- momentum * M + (1 - momentum) * G
      U  = (1 - momentum) * G + momentum * M     (nesterov; else U = M)
      W <- W - lr * sqrt(max(1, out / in)) * newton_schulz(U, steps)
    """
    W = np.asarray(W, dtype=np.float64)
    G = np.asarray(G, dtype=np.float64)
    M = np.asarray(M, dtype=np.float64)
    M = momentum * M + (1.0 - momentum) * G
    U = (1.0 - momentum) * G + momentum * M if nesterov else M
    scale = np.sqrt(max(1.0, W.shape[0] / W.shape[1]))
    return W - lr * scale * newton_schulz(U, steps), M
