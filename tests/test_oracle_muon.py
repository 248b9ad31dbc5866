"""Pins of the Muon oracle (CPU only).

Every check here reaches the oracle's result by another route than its own
matrix iteration: the singular-value form of the Newton-Schulz polynomial
(scalar arithmetic on a matrix built from a known SVD), the textbook cubic
iteration converging to the polar factor from numpy's SVD, the pages' stated
spread of the resulting singular values, and closed forms of the momentum
recurrences.
"""

import numpy as np

from oracle import muon


def _scalar_ns(x, steps, coeffs=muon.NS5_COEFFS):
    a, b, c = coeffs
    for _ in range(steps):
        x = a * x + b * x ** 3 + c * x ** 5
    return x


def _orthonormal(rng, n, k):
    q, r = np.linalg.qr(rng.standard_normal((n, k)))
    return q * np.sign(np.diag(r))  # a fixed sign per column


def _with_spectrum(rng, rows, cols, s):
    k = min(rows, cols)
    U, V = _orthonormal(rng, rows, k), _orthonormal(rng, cols, k)
    return U, V, U @ np.diag(s) @ V.T


def test_ns5_maps_singular_values_through_the_scalar_polynomial():
    """On G = U diag(s) V^T the iteration keeps U and V and sends s_i to the
    quintic a x + b x^3 + c x^5, iterated five times, of s_i / (||s|| + eps)."""
    rng = np.random.default_rng(0)
    for rows, cols in ((6, 17), (17, 6), (9, 9)):
        k = min(rows, cols)
        s = 3.7 * np.geomspace(1.0, 0.05, k)
        U, V, G = _with_spectrum(rng, rows, cols, s)
        x = s / (np.sqrt(np.sum(s * s)) + muon.NS_EPS)
        want = U @ np.diag([_scalar_ns(float(v), 5) for v in x]) @ V.T
        got = muon.newton_schulz(G, steps=5)
        assert got.shape == G.shape
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_cubic_coefficients_converge_to_the_polar_factor():
    """With the classical cubic coefficients (1.5, -0.5, 0) the same
    iteration is the textbook Newton-Schulz polar iteration: it converges to
    U V^T, the orthogonal polar factor that numpy's SVD gives."""
    rng = np.random.default_rng(1)
    for rows, cols in ((5, 12), (12, 5), (7, 7)):
        G = rng.standard_normal((rows, cols)) + 0.5 * np.eye(rows, cols)
        u, s, vt = np.linalg.svd(G, full_matrices=False)
        assert s.min() / s.max() > 1e-2  # well conditioned: converges in 60 steps
        got = muon.newton_schulz(G, steps=60, coeffs=(1.5, -0.5, 0.0))
        np.testing.assert_allclose(got, u @ vt, rtol=0, atol=1e-10)


def test_ns5_singular_values_lie_between_half_and_three_halves():
    """The pages: five steps of the quintic do not give U V^T but U S' V^T
    with the diagonal of S' roughly in (0.5, 1.5)."""
    rng = np.random.default_rng(2)
    for rows, cols in ((64, 256), (256, 64), (96, 384)):
        G = rng.standard_normal((rows, cols))
        sv = np.linalg.svd(muon.newton_schulz(G), compute_uv=False)
        assert sv.min() > 0.5 and sv.max() < 1.5, (sv.min(), sv.max())


def test_transposed_input_gives_transposed_output():
    rng = np.random.default_rng(3)
    G = rng.standard_normal((11, 30))
    np.testing.assert_allclose(muon.newton_schulz(G.T), muon.newton_schulz(G).T, rtol=0, atol=1e-13)


def test_nesterov_and_plain_momentum_directions_closed_form():
    """A 1 x 2 weight with gradients e1 then e2: after two steps the plain
    buffer is (1-mu) [mu, 1] and the Nesterov direction (1-mu) [mu^2, 1+mu].
    The iteration keeps a row vector's direction and sends its length
    l / (l + eps) through the scalar polynomial, so the second step moves W
    by lr * f * direction / |direction|."""
    mu, lr = 0.95, 0.02
    e1, e2 = np.array([[1.0, 0.0]]), np.array([[0.0, 1.0]])
    for nesterov, direction in ((True, np.array([mu * mu, 1.0 + mu])), (False, np.array([mu, 1.0]))):
        W0, M0 = np.zeros((1, 2)), np.zeros((1, 2))
        W1, M1 = muon.muon_update(W0, e1, M0, lr, mu, nesterov=nesterov)
        W2, M2 = muon.muon_update(W1, e2, M1, lr, mu, nesterov=nesterov)
        np.testing.assert_allclose(M2[0], (1 - mu) * np.array([mu, 1.0]), rtol=1e-15)
        u = (1 - mu) * direction
        length = float(np.linalg.norm(u))
        f = _scalar_ns(length / (length + muon.NS_EPS), 5)
        np.testing.assert_allclose((W1 - W2)[0], lr * f * u / length, rtol=1e-12)


def test_step_scale_is_sqrt_of_out_over_in_for_tall_weights():
    """W [out, in]: the step is lr * sqrt(max(1, out/in)) times the
    orthogonalised update; checked through the step's singular values."""
    rng = np.random.default_rng(4)
    lr = 0.05
    for rows, cols, scale in ((12, 3, 2.0), (3, 12, 1.0), (8, 8, 1.0)):
        k = min(rows, cols)
        s = np.geomspace(2.0, 0.3, k)
        _, _, G = _with_spectrum(rng, rows, cols, s)
        W = rng.standard_normal((rows, cols))
        Wn, _ = muon.muon_update(W, G, np.zeros_like(G), lr, momentum=0.0)
        step_sv = np.linalg.svd((W - Wn) / lr, compute_uv=False)
        x = s / (np.sqrt(np.sum(s * s)) + muon.NS_EPS)
        want = np.sort([scale * _scalar_ns(float(v), 5) for v in x])[::-1]
        np.testing.assert_allclose(step_sv, want, rtol=1e-10)


def test_momentum_schedule_endpoints():
    """0.85 at the first step, 0.95 from step 300 on, linear in between."""
    assert muon.muon_momentum(0) == 0.85
    assert abs(muon.muon_momentum(150) - 0.90) < 1e-15
    assert abs(muon.muon_momentum(300) - 0.95) < 1e-15
    assert muon.muon_momentum(5000) == 0.95


# --------------------------------------------------------------------------- Muon in the training step
def _muon_step_case(**kw):
    from synthetic import init_params, tokens_and_targets, workload
    w = workload("tiny_fp32", x0_rows=0, n_layer=1, seq_len=16, micro_batch=2, vocab=96, **kw)
    params = init_params(w)
    tok, tgt = tokens_and_targets(2, 16, 96, 5)
    return w, params, tok, tgt


def _one_step(w, params, tok, tgt, lr=0.02):
    from oracle.step import OracleTrainer
    orc = OracleTrainer(w, params)
    orc.forward_loss(tok, tgt)
    orc.backward_step(lr)
    return orc


def test_muon_step_leaves_embedding_and_head_to_adamw():
    """matrix_optimizer = "muon": the token embedding and the untied head take
    exactly the AdamW step they take with AdamW everywhere (same gradient,
    same clip), while every block matrix moves differently."""
    w_a, params, tok, tgt = _muon_step_case(tie_embeddings=0)
    w_m = dict(w_a, matrix_optimizer="muon", muon_momentum=0.9)
    oa, om_ = _one_step(w_a, params, tok, tgt), _one_step(w_m, params, tok, tgt)
    for k in ("wte", "lm_head"):
        np.testing.assert_array_equal(om_.P[k], oa.P[k])
    for k in ("h0.wqkv", "h0.wo", "h0.w1", "h0.w2"):
        assert np.abs(om_.P[k] - oa.P[k]).max() > 1e-4


def test_muon_step_orthogonalises_q_k_v_separately():
    """The fused q|k|v weight is three matrices to Muon: each block's step has
    its non-zero singular values in (0.5, 1.5) (five quintic steps; the
    gradient of 32 tokens has rank <= 32, and the iteration keeps zero
    singular values at zero), and the q block's step is not the q rows of the
    whole fused matrix's orthogonalised update."""
    from oracle.step import muon_blocks
    lr, mu = 0.02, 0.9
    w, params, tok, tgt = _muon_step_case(matrix_optimizer="muon", muon_momentum=mu)
    orc = _one_step(w, params, tok, tgt, lr)
    W0 = np.asarray(params["h0.wqkv"], dtype=np.float64)
    step = (W0 - orc.P["h0.wqkv"]) / lr
    blocks = muon_blocks(w, "h0.wqkv", W0.shape)
    assert len(blocks) == 3
    for r0, r1 in blocks:
        sv = np.linalg.svd(step[r0:r1], compute_uv=False)   # [a, d]: wide or square, scale 1
        nz = sv[sv > 1e-8]
        assert 0 < len(nz) <= 32
        assert nz.min() > 0.5 and nz.max() < 1.5, (nz.min(), nz.max())
    g = orc.accum_grads["h0.wqkv"]
    u = (1 - mu) * g + mu * (1 - mu) * g      # Nesterov direction from a zero buffer
    whole = np.sqrt(max(1.0, W0.shape[0] / W0.shape[1])) * muon.newton_schulz(u)
    r0, r1 = blocks[0]
    assert np.linalg.norm(step[r0:r1] - whole[r0:r1]) > 0.1 * np.linalg.norm(step[r0:r1])


def test_muon_step_clips_before_the_momentum():
    """The global-norm clip is taken over all dense gradients before Muon: the
    momentum buffer after the first step is (1 - mu) * coef * g, with coef =
    max_norm / (||g|| + 1e-6) when the norm is above max_norm."""
    mu = 0.9
    w, params, tok, tgt = _muon_step_case(matrix_optimizer="muon", muon_momentum=mu, grad_clip=1e-3)
    orc = _one_step(w, params, tok, tgt)
    norm = np.sqrt(sum(float(np.sum(orc.accum_grads[k] ** 2)) for k in orc.dense))
    assert norm > 1e-3
    coef = 1e-3 / (norm + 1e-6)
    for k in ("h0.wo", "h0.w1"):
        np.testing.assert_allclose(orc.m[k], (1 - mu) * coef * orc.accum_grads[k], rtol=1e-12)
