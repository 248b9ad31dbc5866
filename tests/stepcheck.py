"""Whole-step parity helpers: run the same micro-batches through the CUDA
library and the fp64 oracle and compare gradients, updated weights (as
changes from the starting weights), AdamW moments and table row states.

AdamW's second moment is seeded on both sides before the step, with values of
the size of the step's own squared gradient (from an oracle pre-pass).  With
zero moments the first AdamW step is -lr*sign(g) element by element, so a
bf16 rounding that flips the sign of a near-zero gradient element moves that
weight by 2*lr; seeded moments make the update smooth in g, and the change of
every weight is then compared at the same bar as the gradient.  Seeded
moments are also what the optimizer sees in the middle of a run.
"""

import numpy as np

from oracle import model as omodel
from oracle.step import OracleTrainer
from synthetic import init_params, tokens_and_targets
from tests.helpers import device_ints, export, import_params, rel_l2, to_cfg


def micro_batches(w, steps, ignore_frac=0.05):
    B, T, V = w["micro_batch"], w["seq_len"], w["vocab"]
    return [tokens_and_targets(B, T, V, w["seed"], w["zipf_s"], w["repeat_frac"], ignore_frac=ignore_frac, micro=s)
            for s in range(steps)]


def seed_second_moments(g, model, orc, w, batches):
    """v0 = mean(G^2) of each tensor's gradient on the first micro-batch (oracle,
    loss scaled 1/grad_accum) times a seeded factor in [0.5, 2], rounded to
    fp32 and written to both sides."""
    import torch
    tok, tgt = batches[0]
    rx, rv = orc.rows(tok)
    _, _, cache = omodel.forward(w, orc.P, tok, tgt, rx, rv, orc.rows3(tok))
    G, _, _ = omodel.backward(w, orc.P, cache, scale=1.0 / w["grad_accum"])
    rng = np.random.default_rng(777)
    for k in orc.dense:
        ms = float(np.mean(G[k] ** 2)) or 1e-20
        v0 = (ms * rng.uniform(0.5, 2.0, size=G[k].shape)).astype(np.float32)
        orc.v[k] = v0.astype(np.float64)
        model.tensor(k, g.KIND_ADAM_V).copy_(torch.from_numpy(v0))


def run_pair(g, w, steps, lr=1e-3, ignore_frac=0.05, seed_moments=True, prepare=None):
    """Run `steps` micro-batches through gpt_forward_loss + gpt_backward_step on
    the GPU and through the oracle trainer; returns (model, oracle, losses,
    last tokens, starting parameters).  `prepare(model, params)`, if given,
    fills further model state before the run and adds the oracle's copy of it
    to `params` (the frozen trigram statistics)."""
    cfg = to_cfg(w)
    params = init_params(w)
    model = g.Model(cfg, seed=w["seed"])
    import_params(model, params)
    if prepare is not None:
        prepare(model, params)
    orc = OracleTrainer(w, params)
    batches = micro_batches(w, steps, ignore_frac)
    if seed_moments:
        seed_second_moments(g, model, orc, w, batches)
    losses = []
    for tok, tgt in batches:
        loss = model.forward_loss(device_ints(tok), device_ints(tgt))
        model.backward_step(lr)
        status = model.sync_status()
        assert status == g.GPT_OK, g.gpt_last_error()
        lo, _ = orc.forward_loss(tok, tgt)
        orc.backward_step(lr)
        losses.append((float(loss.item()), lo))
    return model, orc, losses, batches[-1][0], params


def check(g, w, model, orc, losses, params, tol_loss, tol, stepped=True, no_change=()):
    """Loss, accumulated gradient, and (after an AdamW step) the change of every
    dense weight and both AdamW moments; table row states and updated-row sets.
    Weights named in `no_change` skip the weight-change comparison (their
    update is compared elsewhere)."""
    for lg, lo in losses:
        assert abs(lg - lo) / abs(lo) < tol_loss, (lg, lo)
    worst = []
    grads = orc.accum_grads if stepped else orc.acc
    for name in orc.dense:
        eg = rel_l2(export(model, name, g.KIND_GRAD), grads[name])
        assert eg < tol, (name, "grad", eg)
        row = [name, eg]
        if stepped:
            p0 = np.asarray(params[name], dtype=np.float64)
            ed = rel_l2(export(model, name, g.KIND_PARAM) - p0, orc.P[name] - p0)
            em = rel_l2(export(model, name, g.KIND_ADAM_M), orc.m[name])
            ev = rel_l2(export(model, name, g.KIND_ADAM_V), orc.v[name])
            assert name in no_change or ed < tol, (name, "weight change", ed)
            assert em < tol, (name, "adam m", em)
            assert ev < tol, (name, "adam v", ev)
            row += [ed, em, ev]
        worst.append(tuple(row))
    for t in ("hx", "hv"):
        if t not in orc.P:
            continue
        s_gpu = export(model, t, g.KIND_ROW_STATE)[:, 0]
        # updated-row set: every row with a non-zero state was touched
        np.testing.assert_array_equal(np.nonzero(s_gpu)[0], np.nonzero(orc.S[t])[0])
        assert rel_l2(s_gpu, orc.S[t]) < tol
        p0 = np.asarray(params[t], dtype=np.float64)
        assert rel_l2(export(model, t) - p0, orc.P[t] - p0) < tol
    return worst
