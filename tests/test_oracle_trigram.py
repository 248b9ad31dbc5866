"""Pins of the frozen trigram statistics table's oracle (oracle/trigram.py and
the projection into the values in oracle/model.py)."""

import collections
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import hashing, model, trigram
from oracle.step import OracleTrainer
from synthetic import init_params, tokens_and_targets, workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
P1, P2 = 2654435761, 2246822519


def test_trigram_hash_hand_worked_example():
    rows = []
    with open(os.path.join(GOLDEN, "trigram_hash_example.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append([int(x) for x in line.split()])
    rows = np.array(rows)
    tok = np.array([[5, 7, 5, 0]])
    keys = trigram.trigram_keys(tok, 512, P1, P2)
    assert [int(k) for k in keys[0]] == list(rows[:, 1])
    assert list(trigram.trigram_rows(tok, 512, P1, P2, 1024)[0]) == list(rows[:, 2])
    assert list(trigram.trigram_rows(tok, 512, P1, P2, 2048)[0]) == list(rows[:, 3])


def test_trigram_key_without_the_oldest_token_is_the_bigram_key():
    """With p1 = 0 the x[t-2] term vanishes and the key is the (pinned) bigram
    key of (x[t-1], x[t]) with constants (p2, p3)."""
    tok = np.random.default_rng(1).integers(0, 300, size=(3, 40))
    np.testing.assert_array_equal(trigram.trigram_keys(tok, 300, 0, P2, trigram.P3),
                                  hashing.bigram_keys(tok, 300, P2, trigram.P3))


def test_tally_brute_force_and_normalisation():
    """Counts against an explicit count of (row, next-token bucket) pairs; every
    occurring row's statistics sum to 1; one count per position with a next token."""
    rng = np.random.default_rng(7)
    streams = rng.integers(0, 40, size=(3, 25))
    n_rows, width = 37, 8
    want = collections.Counter()
    for s in streams:
        for t in range(len(s) - 1):
            a2 = int(s[t - 2]) if t > 1 else 40
            a1 = int(s[t - 1]) if t > 0 else 40
            key = ((a2 * P1) % 2 ** 64) ^ ((a1 * P2) % 2 ** 64) ^ ((int(s[t]) * trigram.P3) % 2 ** 64)
            want[(key % n_rows, int(s[t + 1]) % width)] += 1
    uniq, counts = trigram.tally_counts(streams, 40, P1, P2, n_rows, width)
    got = {(int(r), b): int(counts[i, b]) for i, r in enumerate(uniq) for b in range(width) if counts[i, b]}
    assert got == dict(want)
    assert counts.sum() == 3 * 24
    _, stats = trigram.tally_stats(streams, 40, P1, P2, n_rows, width)
    np.testing.assert_allclose(stats.sum(axis=1), 1.0, rtol=1e-15)
    table = trigram.dense_stats(streams, 40, P1, P2, n_rows, width)
    assert not table[np.setdiff1d(np.arange(n_rows), uniq)].any()


def _tri_case(**kw):
    w = workload("tiny_fp32", x0_rows=0, n_layer=2, seq_len=16, micro_batch=2, vocab=96,
                 tri_rows=64, tri_width=8, **kw)
    P = init_params(w)
    streams = np.random.default_rng(3).integers(0, 96, size=(6, 33))
    P["h3"] = trigram.dense_stats(streams, 96, P1, P2, 64, 8)
    tok, tgt = tokens_and_targets(2, 16, 96, 5)
    tgt[0, 3] = -1
    return w, P, tok, tgt


def test_projection_matches_torch_autograd():
    """The decoder with v += vproj S3[row] in every layer, written with torch
    library ops (F.embedding of the frozen table, a matmul, autograd): loss
    and every dense gradient, vproj's included, and nothing reaches S3."""
    w, P, tok, tgt = _tri_case(v_rows=0)
    tr = OracleTrainer(w, P)
    r3 = tr.rows3(tok)
    loss, _, cache = model.forward(w, tr.P, tok, tgt, None, None, r3)
    G, _, _ = model.backward(w, tr.P, cache)
    assert set(G) == set(tr.dense) and "h3" not in G
    B, T = tok.shape
    d, H, hd = w["d_model"], w["n_head"], w["head_dim"]
    a, eps = H * hd, w["norm_eps"]
    TP = {k: torch.tensor(v, requires_grad=(k != "h3")) for k, v in P.items()}
    x = F.rms_norm(F.embedding(torch.from_numpy(tok), TP["wte"]), (d,), eps=eps)
    vb = F.embedding(torch.from_numpy(r3), TP["h3"]) @ TP["vproj"].T
    theta = torch.arange(T, dtype=torch.float64)[:, None] * \
        w["rope_base"] ** (-torch.arange(0, hd, 2, dtype=torch.float64) / hd)[None, :]
    rot = torch.exp(-1j * theta)

    def rotate(z):
        zc = torch.complex(z[..., :hd // 2], z[..., hd // 2:]) * rot[None, :, None, :]
        return torch.cat([zc.real, zc.imag], dim=-1)

    for layer in range(w["n_layer"]):
        u = F.rms_norm(x, (d,), eps=eps)
        q, k, v = (u @ TP[f"h{layer}.wqkv"].T).split(a, dim=-1)
        v = v + vb
        q, k, v = (z.reshape(B, T, H, hd) for z in (q, k, v))
        q, k = F.rms_norm(rotate(q), (hd,), eps=eps), F.rms_norm(rotate(k), (hd,), eps=eps)
        o = F.scaled_dot_product_attention(q.transpose(1, 2), k.transpose(1, 2), v.transpose(1, 2), is_causal=True)
        x = x + o.transpose(1, 2).reshape(B, T, a) @ TP[f"h{layer}.wo"].T
        x = x + F.relu(F.rms_norm(x, (d,), eps=eps) @ TP[f"h{layer}.w1"].T).square() @ TP[f"h{layer}.w2"].T
    z = F.rms_norm(x, (d,), eps=eps) @ TP["wte"].T
    ref = F.cross_entropy(z.reshape(B * T, -1), torch.from_numpy(tgt).reshape(-1).long(), ignore_index=-1)
    ref.backward()
    assert abs(loss - ref.item()) < 1e-12 * max(1.0, abs(loss))
    for k, g in G.items():
        np.testing.assert_allclose(g, TP[k].grad.numpy(), rtol=1e-9, atol=1e-12, err_msg=k)


def test_projection_gradient_matches_central_finite_differences():
    w, P, tok, tgt = _tri_case(v_rows=32)
    tr = OracleTrainer(w, P)
    rx, rv = tr.rows(tok)
    r3 = tr.rows3(tok)
    _, _, cache = model.forward(w, tr.P, tok, tgt, rx, rv, r3)
    G, _, _ = model.backward(w, tr.P, cache)
    g = G["vproj"]
    rng = np.random.default_rng(11)
    h = 1e-6
    for i in np.argsort(-np.abs(g).reshape(-1))[:4].tolist() + rng.integers(0, g.size, 4).tolist():
        idx = np.unravel_index(i, g.shape)
        Pp = {k: v.copy() for k, v in tr.P.items()}
        Pm = {k: v.copy() for k, v in tr.P.items()}
        Pp["vproj"][idx] += h
        Pm["vproj"][idx] -= h
        fd = (model.forward(w, Pp, tok, tgt, rx, rv, r3)[0] - model.forward(w, Pm, tok, tgt, rx, rv, r3)[0]) / (2 * h)
        assert abs(fd - g[idx]) <= 1e-7 + 1e-6 * abs(g[idx]), (idx, fd, g[idx])


def test_zero_projection_is_the_model_without_the_table():
    w, P, tok, tgt = _tri_case(v_rows=0)
    P["vproj"][...] = 0.0
    tr = OracleTrainer(w, P)
    loss3 = model.forward(w, tr.P, tok, tgt, None, None, tr.rows3(tok))[0]
    w0 = dict(w, tri_rows=0)
    P0 = {k: v for k, v in P.items() if k not in ("vproj", "h3")}
    assert loss3 == model.forward(w0, P0, tok, tgt)[0]


def test_table_is_frozen_in_the_trainer():
    w, P, tok, tgt = _tri_case(v_rows=0)
    tr = OracleTrainer(w, P)
    tr.forward_loss(tok, tgt)
    tr.backward_step(1e-2)
    np.testing.assert_array_equal(tr.P["h3"], P["h3"])
    assert np.abs(tr.P["vproj"] - P["vproj"]).max() > 0
