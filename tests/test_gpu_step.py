"""Full training-step parity on the GPU against the fp64 oracle, through the C ABI.

Same seeded weights (imported into the model) and the same seeded Zipf token
streams feed both sides.  Bars: fp32 mode 1e-4; bf16 mode loss 1e-2 relative
and per-tensor gradient / updated-weight relative L2 2e-2; hash rows and
updated-row sets bit-exact.
"""

import numpy as np
import pytest

from oracle.step import OracleTrainer
from synthetic import init_params, small_case, tokens_and_targets, workload
from tests.helpers import device_ints, export, import_params, rel_l2, to_cfg

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    import torch
    import gpt_pretraining_step_decoder_b200 as g
    assert torch.cuda.is_available()
    return g


def run_pair(g, w, steps, lr=1e-3, ignore_frac=0.05):
    """Run `steps` micro-batches on the GPU and the oracle; return both sides."""
    cfg = to_cfg(w)
    params = init_params(w)
    model = g.Model(cfg, seed=w["seed"])
    import_params(model, params)
    orc = OracleTrainer(w, params)
    B, T, V = w["micro_batch"], w["seq_len"], w["vocab"]
    losses = []
    for s in range(steps):
        tok, tgt = tokens_and_targets(B, T, V, w["seed"], w["zipf_s"], w["repeat_frac"],
                                      ignore_frac=ignore_frac, micro=s)
        loss = model.forward_loss(device_ints(tok), device_ints(tgt))
        model.backward_step(lr)
        status = model.sync_status()
        assert status == g.GPT_OK, g.gpt_last_error()
        lo, _ = orc.forward_loss(tok, tgt)
        orc.backward_step(lr)
        losses.append((float(loss.item()), lo))
    return model, orc, losses, tok


def check(g, w, model, orc, losses, tol_loss, tol):
    for lg, lo in losses:
        assert abs(lg - lo) / abs(lo) < tol_loss, (lg, lo)
    worst = []
    for name in orc.dense:
        eg = rel_l2(export(model, name, g.KIND_GRAD), orc.accum_grads[name])
        ep = rel_l2(export(model, name, g.KIND_PARAM), orc.P[name])
        worst.append((eg, ep, name))
        assert eg < tol, (name, "grad", eg)
        assert ep < tol, (name, "param", ep)
    for t in ("hx", "hv"):
        if t not in orc.P:
            continue
        s_gpu = export(model, t, g.KIND_ROW_STATE)[:, 0]
        # updated-row set: every row with a non-zero state was touched
        np.testing.assert_array_equal(np.nonzero(s_gpu)[0], np.nonzero(orc.S[t])[0])
        assert rel_l2(s_gpu, orc.S[t]) < tol
    return worst


def test_fp32_tiny_two_steps(g):
    w = workload("tiny_fp32")
    model, orc, losses, tok = run_pair(g, w, steps=2)
    # hash rows bit-exact
    rx = model.tensor("rows_x", g.KIND_ACT).cpu().numpy()
    np.testing.assert_array_equal(rx, orc.rows(tok)[0])
    check(g, w, model, orc, losses, 1e-4, 1e-4)
    # x0 table: delta of every touched row
    W0 = init_params(w)["hx"]
    assert rel_l2(export(model, "hx") - W0, orc.P["hx"] - W0) < 1e-4


@pytest.mark.parametrize("variant", [dict(), dict(tie_embeddings=0, softcap=15.0, grad_clip=1.0)])
def test_fp32_variants(g, variant):
    w = workload("tiny_fp32", **variant)
    model, orc, losses, _ = run_pair(g, w, steps=1)
    check(g, w, model, orc, losses, 1e-4, 1e-4)


def test_bf16_gpt2_small_shape(g):
    w = small_case("gpt2s_bf16", grad_accum=2)
    model, orc, losses, _ = run_pair(g, w, steps=2)
    check(g, w, model, orc, losses, 1e-2, 2e-2)


def test_bf16_softcap_untied_clip(g):
    """The tensor-core path with nanochat's logit softcap (z = 15 tanh(acc/15)),
    an untied head and global-norm clipping."""
    w = small_case("gpt2s_bf16", grad_accum=2, softcap=15.0, tie_embeddings=0, grad_clip=1.0)
    model, orc, losses, _ = run_pair(g, w, steps=2)
    check(g, w, model, orc, losses, 1e-2, 2e-2)


def test_bf16_with_tables(g):
    # two micro-batches per AdamW step: both table updates happen (one per
    # backward call) and the accumulated dense gradient is compared before the
    # first AdamW step, whose -lr*sign(g) update would otherwise amplify bf16
    # noise on near-zero gradient elements into the next step
    w = small_case("gpt2s_tables_bf16", grad_accum=2)
    model, orc, losses, tok = run_pair(g, w, steps=2)
    check(g, w, model, orc, losses, 1e-2, 2e-2)
    rx = model.tensor("rows_x", g.KIND_ACT).cpu().numpy()
    rv = model.tensor("rows_v", g.KIND_ACT).cpu().numpy()
    ox, ov = orc.rows(tok)
    np.testing.assert_array_equal(rx, ox)
    np.testing.assert_array_equal(rv, ov)
    P0 = init_params(w)
    for t in ("hx", "hv"):
        assert rel_l2(export(model, t) - P0[t], orc.P[t] - P0[t]) < 2e-2


def test_backward_without_forward_is_a_state_error(g):
    model = g.Model(to_cfg(workload("tiny_fp32")))
    with pytest.raises(g.GptError) as e:
        model.backward_step(1e-3)
    assert e.value.code == g.GPT_ERR_STATE


def test_out_of_range_token_reports_input_error(g):
    w = workload("tiny_fp32")
    model = g.Model(to_cfg(w))
    tok, tgt = tokens_and_targets(w["micro_batch"], w["seq_len"], w["vocab"], 0)
    tok[1, 5] = w["vocab"] + 3
    model.forward_loss(device_ints(tok), device_ints(tgt))
    assert model.sync_status() == g.GPT_ERR_INPUT
    assert model.sync_status() == g.GPT_OK


def test_bf16_long_ragged_sequence(g):
    # T = 520: several 128-row query tiles and 64-key tiles with a ragged tail
    w = small_case("gpt2s_bf16", n_layer=1, seq_len=520, micro_batch=1, vocab=1024, grad_accum=2)
    model, orc, losses, _ = run_pair(g, w, steps=2)
    check(g, w, model, orc, losses, 1e-2, 2e-2)
