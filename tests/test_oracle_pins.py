"""Pins of the fp64 oracle against facts fixed outside the oracle itself.

Each test ties one oracle function to a library routine, a closed form, an
invariant, a hand-worked example or the pages' printed numbers, so that a
dropped term, a wrong sign or index, or a transposed operand fails here.
"""

import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import counts, hashing, model, optim
from oracle.step import OracleTrainer
from synthetic import workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


# ----------------------------------------------------------------------- hashing
def test_hash_hand_worked_example():
    rows = []
    with open(os.path.join(GOLDEN, "bigram_hash_example.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append([int(x) for x in line.split()])
    rows = np.array(rows)
    tok = np.array([[5, 7, 5, 0]])
    keys = hashing.bigram_keys(tok, 512, 2654435761, 2246822519)
    assert [int(k) for k in keys[0]] == list(rows[:, 1])
    assert list(hashing.bigram_rows(tok, 512, 2654435761, 2246822519, 1024)[0]) == list(rows[:, 2])
    assert list(hashing.bigram_rows(tok, 512, 2654435761, 2246822519, 2048)[0]) == list(rows[:, 3])


def test_hash_buckets_spread_and_depend_on_previous_token():
    tok = RNG.integers(0, 50304, size=(8, 512))
    r = hashing.bigram_rows(tok, 50304, 2654435761, 2246822519, 256)
    hist = np.bincount(r.reshape(-1), minlength=256)
    exp = r.size / 256
    chi2 = float(((hist - exp) ** 2 / exp).sum())
    assert chi2 < 400  # 255 dof; far below for a well-spread hash
    # same current token, different previous token -> different key
    k = hashing.bigram_keys(np.array([[1, 9, 2, 9]]), 100, 2654435761, 2246822519)
    assert k[0, 1] != k[0, 3]


# ----------------------------------------------------------------------- norms
def test_rmsnorm_matches_torch_and_has_unit_rms():
    x = RNG.standard_normal((5, 7, 48)) * 3.0
    eps = 1.1920929e-07
    y, rstd = model.rmsnorm(x, eps)
    ref = F.rms_norm(torch.from_numpy(x), (48,), eps=eps).numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-6)


# ----------------------------------------------------------------------- RoPE
def test_rope_hand_values_at_t1():
    cos, sin = model.rope_tables(2, 4, 10000.0)
    # theta[1] = (1, 1 * 10000^(-2/4)) = (1, 0.01)
    np.testing.assert_allclose(cos[1], [math.cos(1.0), math.cos(0.01)], rtol=1e-15)
    x = np.array([[1.0, 0.0, 0.0, 0.0], [1.0, 0.0, 0.0, 0.0]])
    y = model.rope(x, cos, sin)
    np.testing.assert_allclose(y[0], [1, 0, 0, 0], atol=1e-15)   # t = 0: identity
    np.testing.assert_allclose(y[1], [math.cos(1.0), 0, -math.sin(1.0), 0], atol=1e-15)


def test_rope_is_complex_rotation_and_preserves_norms():
    T, hd = 11, 16
    cos, sin = model.rope_tables(T, hd, 10000.0)
    x = RNG.standard_normal((3, T, hd))
    y = model.rope(x, cos, sin)
    h = hd // 2
    # (y1 + i y2) = (x1 + i x2) * exp(-i theta)
    t = np.arange(T)[:, None]
    theta = t * 10000.0 ** (-np.arange(0, hd, 2) / hd)[None, :]
    zc = (x[..., :h] + 1j * x[..., h:]) * np.exp(-1j * theta)
    np.testing.assert_allclose(y[..., :h], zc.real, atol=1e-12)
    np.testing.assert_allclose(y[..., h:], zc.imag, atol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-12)
    # relative-position invariance of q.k
    q, k = RNG.standard_normal(hd), RNG.standard_normal(hd)
    Q = model.rope(np.tile(q, (T, 1)), cos, sin)
    K = model.rope(np.tile(k, (T, 1)), cos, sin)
    np.testing.assert_allclose(Q[7] @ K[4], Q[3] @ K[0], rtol=1e-10)
    # backward is the transpose
    dy = RNG.standard_normal((3, T, hd))
    lhs = np.sum(model.rope(x, cos, sin) * dy)
    rhs = np.sum(x * model.rope_bwd(dy, cos, sin))
    assert abs(lhs - rhs) < 1e-10


# ----------------------------------------------------------------------- attention
def test_attention_matches_torch_sdpa_and_rows_sum_to_one():
    q, k, v = (RNG.standard_normal((2, 3, 9, 8)) for _ in range(3))
    o, p = model.causal_attention(q, k, v)
    ref = F.scaled_dot_product_attention(*(torch.from_numpy(a) for a in (q, k, v)),
                                         is_causal=True).numpy()
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=1e-14)
    assert np.all(np.triu(p[0, 0], k=1) == 0)
    o1, _ = model.causal_attention(q[..., :1, :], k[..., :1, :], v[..., :1, :])
    np.testing.assert_allclose(o1, v[..., :1, :], rtol=1e-15)   # T = 1: o = v


# ----------------------------------------------------------------------- full model
def tiny_cfg(**kw):
    c = workload("tiny_fp32", n_layer=2, d_model=16, n_head=2, head_dim=8,
                 d_ff=64, vocab=37, seq_len=7, micro_batch=2, x0_rows=13, v_rows=11)
    c.update(kw)
    return c


def tiny_params(cfg, std=0.3):
    from synthetic import param_shapes
    return {k: RNG.standard_normal(s) * std for k, s in param_shapes(cfg).items()}


def tiny_batch(cfg):
    tok = RNG.integers(0, cfg["vocab"], size=(cfg["micro_batch"], cfg["seq_len"]))
    tgt = RNG.integers(0, cfg["vocab"], size=tok.shape)
    tgt[0, 2] = -1
    return tok, tgt


def torch_reference_loss(cfg, P, tok, tgt, rx, rv):
    """The same decoder written with torch library ops, for autograd.

    F.embedding, F.rms_norm, F.scaled_dot_product_attention, F.relu and
    F.cross_entropy(ignore_index=-1); RoPE as multiplication by exp(-i theta).
    """
    B, T = tok.shape
    d, H, hd = cfg["d_model"], cfg["n_head"], cfg["head_dim"]
    eps = cfg["norm_eps"]
    a = H * hd
    x = F.rms_norm(F.embedding(torch.from_numpy(tok), P["wte"]), (d,), eps=eps)
    if "hx" in P:
        x = x + F.embedding(torch.from_numpy(rx), P["hx"])
    theta = torch.arange(T, dtype=torch.float64)[:, None] * \
        cfg["rope_base"] ** (-torch.arange(0, hd, 2, dtype=torch.float64) / hd)[None, :]
    rot = torch.exp(-1j * theta)

    def rotate(z):  # z [B, T, H, hd]
        zc = torch.complex(z[..., :hd // 2], z[..., hd // 2:]) * rot[None, :, None, :]
        return torch.cat([zc.real, zc.imag], dim=-1)

    for layer in range(cfg["n_layer"]):
        u = F.rms_norm(x, (d,), eps=eps)
        qkv = u @ P[f"h{layer}.wqkv"].T
        q, k, v = qkv.split(a, dim=-1)
        if "hv" in P:
            v = v + F.embedding(torch.from_numpy(rv), P["hv"])
        q, k, v = (z.reshape(B, T, H, hd) for z in (q, k, v))
        q, k = rotate(q), rotate(k)
        if cfg["qk_norm"]:
            q, k = F.rms_norm(q, (hd,), eps=eps), F.rms_norm(k, (hd,), eps=eps)
        o = F.scaled_dot_product_attention(q.transpose(1, 2), k.transpose(1, 2),
                                           v.transpose(1, 2), is_causal=True)
        x = x + o.transpose(1, 2).reshape(B, T, a) @ P[f"h{layer}.wo"].T
        u2 = F.rms_norm(x, (d,), eps=eps)
        x = x + F.relu(u2 @ P[f"h{layer}.w1"].T).square() @ P[f"h{layer}.w2"].T
    w_lm = P["wte"] if cfg["tie_embeddings"] else P["lm_head"]
    z = F.rms_norm(x, (d,), eps=eps) @ w_lm.T
    if cfg["softcap"] > 0:
        z = cfg["softcap"] * torch.tanh(z / cfg["softcap"])
    return F.cross_entropy(z.reshape(B * T, -1), torch.from_numpy(tgt).reshape(-1).long(),
                           ignore_index=-1)


@pytest.mark.parametrize("variant", [
    dict(),
    dict(tie_embeddings=0, softcap=15.0),
    dict(qk_norm=0, x0_rows=0, v_rows=0),
])
def test_model_forward_backward_matches_torch_autograd(variant):
    cfg = tiny_cfg(**variant)
    P = tiny_params(cfg)
    tok, tgt = tiny_batch(cfg)
    tr = OracleTrainer(cfg, P)
    rx, rv = tr.rows(tok)
    loss, _, cache = model.forward(cfg, tr.P, tok, tgt, rx, rv)
    G, gx0, gv = model.backward(cfg, tr.P, cache, scale=0.5)

    TP = {k: torch.tensor(v, requires_grad=True) for k, v in P.items()}
    ref = torch_reference_loss(cfg, TP, tok, tgt, rx, rv)
    (0.5 * ref).backward()
    assert abs(loss - ref.item()) < 1e-12 * max(1.0, abs(loss))
    for k, g in G.items():
        np.testing.assert_allclose(g, TP[k].grad.numpy(), rtol=1e-9, atol=1e-12, err_msg=k)
    N = tok.size
    if "hx" in P:
        dhx = np.zeros_like(P["hx"])
        np.add.at(dhx, rx.reshape(N), gx0)
        np.testing.assert_allclose(dhx, TP["hx"].grad.numpy(), rtol=1e-9, atol=1e-12)
    if "hv" in P:
        dhv = np.zeros_like(P["hv"])
        np.add.at(dhv, rv.reshape(N), gv)
        np.testing.assert_allclose(dhv, TP["hv"].grad.numpy(), rtol=1e-9, atol=1e-12)


def test_backward_matches_central_finite_differences():
    cfg = tiny_cfg(tie_embeddings=0, softcap=15.0)
    P = tiny_params(cfg)
    tok, tgt = tiny_batch(cfg)
    tr = OracleTrainer(cfg, P)
    rx, rv = tr.rows(tok)

    def f(Pd):
        return model.forward(cfg, Pd, tok, tgt, rx, rv)[0]

    _, _, cache = model.forward(cfg, tr.P, tok, tgt, rx, rv)
    G, gx0, gv = model.backward(cfg, tr.P, cache)
    N = tok.size
    dt = {"hx": np.zeros_like(P["hx"]), "hv": np.zeros_like(P["hv"])}
    np.add.at(dt["hx"], rx.reshape(N), gx0)
    np.add.at(dt["hv"], rv.reshape(N), gv)
    h = 1e-6
    for name in P:
        grad = G[name] if name in G else dt[name]
        flat = np.argsort(-np.abs(grad).reshape(-1))[:3].tolist() + \
            RNG.integers(0, grad.size, 3).tolist()
        for i in flat:
            idx = np.unravel_index(i, grad.shape)
            Pp = {k: v.copy() for k, v in tr.P.items()}
            Pm = {k: v.copy() for k, v in tr.P.items()}
            Pp[name][idx] += h
            Pm[name][idx] -= h
            fd = (f(Pp) - f(Pm)) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-7 + 1e-6 * abs(grad[idx]), (name, idx, fd, grad[idx])


def test_loss_is_ln_vocab_when_head_is_zero():
    for tie in (0, 1):
        cfg = tiny_cfg(tie_embeddings=tie)
        P = tiny_params(cfg)
        P["wte" if tie else "lm_head"][:] = 0.0
        tok, tgt = tiny_batch(cfg)
        tr = OracleTrainer(cfg, P)
        loss, per_tok = tr.forward_loss(tok, tgt)
        assert abs(loss - math.log(cfg["vocab"])) < 1e-12


def test_causality():
    cfg = tiny_cfg()
    P = tiny_params(cfg)
    tok, tgt = tiny_batch(cfg)
    tr = OracleTrainer(cfg, P)
    _, a = tr.forward_loss(tok, tgt)
    tok2 = tok.copy()
    tok2[:, 4:] = (tok2[:, 4:] + 5) % cfg["vocab"]
    _, b = tr.forward_loss(tok2, tgt)
    np.testing.assert_array_equal(a[:, :4], b[:, :4])
    assert np.any(a[:, 4:] != b[:, 4:])


# ----------------------------------------------------------------------- optimizers
def test_adamw_first_step_is_minus_lr_sign_and_matches_torch():
    g = RNG.standard_normal((4, 5))
    p0 = RNG.standard_normal((4, 5))
    p1, m, v = optim.adamw(p0, g, 0 * g, 0 * g, 1, 1e-3, 0.8, 0.95, 1e-10, 0.0)
    np.testing.assert_allclose(p1 - p0, -1e-3 * np.sign(g), rtol=1e-6)
    # three steps with weight decay vs torch.optim.AdamW
    tp = torch.tensor(p0, requires_grad=True)
    opt = torch.optim.AdamW([tp], lr=2e-3, betas=(0.8, 0.95), eps=1e-10, weight_decay=0.1)
    p, m, v = p0.copy(), 0 * p0, 0 * p0
    for t in range(1, 4):
        gt = RNG.standard_normal(p0.shape)
        tp.grad = torch.tensor(gt)
        opt.step()
        p, m, v = optim.adamw(p, gt, m, v, t, 2e-3, 0.8, 0.95, 1e-10, 0.1)
    np.testing.assert_allclose(p, tp.detach().numpy(), rtol=1e-12, atol=1e-15)


def test_clip_coef_matches_torch():
    gs = [RNG.standard_normal((3, 4)) * 2, RNG.standard_normal(7)]
    ts = [torch.zeros_like(torch.tensor(g), requires_grad=True) for g in gs]
    for t, g in zip(ts, gs):
        t.grad = torch.tensor(g)
    torch.nn.utils.clip_grad_norm_(ts, max_norm=1.0)
    c = optim.clip_coef(gs, 1.0)
    for t, g in zip(ts, gs):
        np.testing.assert_allclose(g * c, t.grad.numpy(), rtol=1e-12)


def test_clip_coef_leaves_small_gradients_alone():
    """Below max_norm torch's clip_grad_norm_ does not scale gradients up."""
    gs = [RNG.standard_normal((3, 4)) * 1e-3, RNG.standard_normal(7) * 1e-3]
    ts = [torch.zeros_like(torch.tensor(g), requires_grad=True) for g in gs]
    for t, g in zip(ts, gs):
        t.grad = torch.tensor(g)
    torch.nn.utils.clip_grad_norm_(ts, max_norm=1.0)
    c = optim.clip_coef(gs, 1.0)
    assert c == 1.0
    for t, g in zip(ts, gs):
        np.testing.assert_array_equal(g * c, t.grad.numpy())


def test_table_update_closed_form_and_two_step_recurrence():
    W = np.zeros((5, 4))
    s = np.zeros(5)
    rows = np.array([3, 1, 3])
    g = np.array([[1.0, 2.0, 0.0, -1.0], [0.5, 0.5, 0.5, 0.5], [1.0, 0.0, 2.0, 1.0]])
    W1, s1, u = optim.table_update(W, s, rows, g, lr=0.1, beta=0.95, eps=0.0)
    assert list(u) == [1, 3]
    # row 3: G = (2, 2, 2, 0), mean G^2 = 3, s = 0.05*3 = 0.15
    assert abs(s1[3] - 0.15) < 1e-15
    np.testing.assert_allclose(W1[3], -0.1 * np.array([2, 2, 2, 0]) / math.sqrt(0.15), rtol=1e-14)
    # first step closed form: -lr * G / sqrt((1-beta) mean G^2)
    np.testing.assert_allclose(W1[1], -0.1 * 0.5 / math.sqrt(0.05 * 0.25) * np.ones(4), rtol=1e-14)
    assert np.all(W1[[0, 2, 4]] == 0) and np.all(s1[[0, 2, 4]] == 0)
    # second step on row 3 with G = (1, 1, 1, 1): s = 0.95*0.15 + 0.05*1 = 0.1925
    W2, s2, _ = optim.table_update(W1, s1, np.array([3]), np.ones((1, 4)), 0.1, 0.95, 0.0)
    assert abs(s2[3] - 0.1925) < 1e-15
    np.testing.assert_allclose(W2[3], W1[3] - 0.1 / math.sqrt(0.1925), rtol=1e-14)
    assert s2[1] == s1[1]


def test_accumulation_sums_scaled_micro_grads():
    cfg = tiny_cfg(grad_accum=2, x0_rows=0, v_rows=0)
    P = tiny_params(cfg)
    tok, tgt = tiny_batch(cfg)
    tr = OracleTrainer(cfg, P)
    tr.forward_loss(tok, tgt)
    assert tr.backward_step(1e-3) is False
    assert all(np.all(tr.P[k] == P[k]) for k in tr.dense)   # no dense step yet
    tr.forward_loss(tok, tgt)
    assert tr.backward_step(1e-3) is True
    one = OracleTrainer(tiny_cfg(x0_rows=0, v_rows=0), P)
    one.forward_loss(tok, tgt)
    one.backward_step(1e-3)
    for k in tr.dense:
        np.testing.assert_allclose(tr.accum_grads[k], one.accum_grads[k], rtol=1e-12, atol=1e-15)


def _one_step(cfg, P, lr, batch):
    tr = OracleTrainer(cfg, P)
    tok, tgt = batch
    tr.forward_loss(tok, tgt)
    tr.backward_step(lr)
    return tr


def test_learning_rate_multipliers_scale_their_own_groups():
    """A group's step uses lr * its multiplier: a zero multiplier leaves
    exactly that group untouched, and (lr 1, multipliers 2) equals (lr 2,
    multipliers 1) everywhere, tables included."""
    base = tiny_cfg(grad_accum=1)
    P = tiny_params(base)
    batch = tiny_batch(base)
    dense = [k for k in P if k not in ("hx", "hv")]
    mats = [k for k in dense if k.startswith("h")]
    for group, keys in (("lr_mult_matrix", mats), ("lr_mult_embed", ["wte"]), ("lr_mult_table", ["hx", "hv"])):
        tr = _one_step(dict(base, **{group: 0.0}), P, 1e-2, batch)
        for k in P:
            if k in keys:
                np.testing.assert_array_equal(tr.P[k], P[k])
            else:
                assert not np.array_equal(tr.P[k], P[k]), (group, k)
    mults = {m: 2.0 for m in ("lr_mult_matrix", "lr_mult_embed", "lr_mult_head", "lr_mult_table")}
    a = _one_step(dict(base, **mults), P, 1e-2, batch)
    b = _one_step(base, P, 2e-2, batch)
    for k in P:
        np.testing.assert_allclose(a.P[k], b.P[k], rtol=1e-14, atol=1e-17)


# ----------------------------------------------------------------------- counts
def test_counts_reproduce_nanochat_d32_printed_values():
    cfg = workload("d32_bf16")
    dense, table = counts.num_params(cfg)
    assert dense == 1_879_048_192 and table == 0       # "Number of parameters: 1,879,048,192"
    f = counts.flops_per_token(cfg)
    assert f == 12_079_595_520 and f"{f:e}" == "1.207960e+10"   # "1.207960e+10"


def test_counts_gpt2_small_and_tiny():
    assert counts.flops_per_token(workload("gpt2s_bf16")) == 854_654_976
    assert counts.flops_per_token(workload("gpt2s_bf16"), causal=True) == 798_031_872
    assert counts.flops_per_token(workload("tiny_fp32")) == 2_949_120
    assert counts.flops_per_token(workload("gpt2s_tables_bf16")) == 967_901_184
