"""Data-parallel table exchange on one GPU, through the C ABI.

In table exchange mode the backward leaves each position's table gradient to
the caller; dp.exchange_tables then applies the sparse update through
ngram_sparse_update.  With one rank nothing is gathered, so the tables, row
states and dense gradients must equal, bit for bit, those of a twin model
that applied the update inline (same kernels, same inputs, same order).
"""

import numpy as np
import pytest

from synthetic import small_case, tokens_and_targets, workload
from tests.helpers import device_ints, to_cfg

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    import torch
    import gpt_pretraining_step_decoder_b200 as g
    assert torch.cuda.is_available()
    return g


@pytest.mark.parametrize("w", [
    small_case("gpt2s_tables_bf16", grad_accum=2),
    workload("tiny_fp32", v_rows=512, grad_accum=2),
], ids=["bf16_tables", "fp32_tables"])
def test_table_exchange_mode_equals_inline_update(g, w):
    import torch
    from gpt_pretraining_step_decoder_b200 import dp
    cfg = to_cfg(w)
    inline, deferred = g.Model(cfg, seed=w["seed"]), g.Model(cfg, seed=w["seed"])
    deferred.set_table_exchange(True)
    B, T, V, lr = w["micro_batch"], w["seq_len"], w["vocab"], 1e-3
    for s in range(w["grad_accum"]):
        tok, tgt = tokens_and_targets(B, T, V, w["seed"], w["zipf_s"], w["repeat_frac"], micro=s)
        for m in (inline, deferred):
            m.forward_loss(device_ints(tok), device_ints(tgt))
            m.backward(lr)
        dp.exchange_tables(deferred, lr)
    torch.cuda.synchronize()
    for m in (inline, deferred):
        assert m.sync_status() == g.GPT_OK, g.gpt_last_error()
    for t in ("hx", "hv"):
        for kind in (g.KIND_PARAM, g.KIND_ROW_STATE):
            a = inline.tensor(t, kind).float().cpu().numpy()
            b = deferred.tensor(t, kind).float().cpu().numpy()
            np.testing.assert_array_equal(a, b)
    assert torch.equal(inline.flat_grad(), deferred.flat_grad())
    # the tables did move
    fresh = g.Model(cfg, seed=w["seed"])
    assert not torch.equal(fresh.tensor("hx").float(), deferred.tensor("hx").float())


@pytest.mark.parametrize("tables,dense", [("sharded", "sharded"), ("inline", "sharded"), ("sharded", "replicated")])
def test_sharded_forms_on_one_gpu_equal_the_plain_step(g, tables, dense):
    """With one rank the row-sharded table exchange owns every row and the
    sharded dense step's slice is the whole buffer: dp.train_step must give,
    bit for bit, the tables, row states and weights of gpt_backward_step
    (same kernels, same sums; the clip norm's partial sums are added in the
    same order).  Global clipping on."""
    import torch
    from gpt_pretraining_step_decoder_b200 import dp
    w = small_case("gpt2s_tables_bf16", grad_accum=2, grad_clip=0.5)
    cfg = to_cfg(w)
    plain, sharded = g.Model(cfg, seed=w["seed"]), g.Model(cfg, seed=w["seed"])
    B, T, V, lr = w["micro_batch"], w["seq_len"], w["vocab"], 1e-3
    batches = [tuple(device_ints(x) for x in tokens_and_targets(B, T, V, w["seed"], w["zipf_s"], w["repeat_frac"],
                                                                micro=s)) for s in range(w["grad_accum"])]
    for tok, tgt in batches:
        plain.forward_loss(tok, tgt)
        plain.backward_step(lr)
    dp.train_step(sharded, batches, lr, tables=tables, dense=dense)
    torch.cuda.synchronize()
    for m in (plain, sharded):
        assert m.sync_status() == g.GPT_OK, g.gpt_last_error()
    assert not sharded.table_exchange
    for t in ("hx", "hv"):
        for kind in (g.KIND_PARAM, g.KIND_ROW_STATE):
            np.testing.assert_array_equal(plain.tensor(t, kind).float().cpu().numpy(),
                                          sharded.tensor(t, kind).float().cpu().numpy())
    assert torch.equal(plain.flat_param(), sharded.flat_param())
    np.testing.assert_array_equal(plain.tensor("h0.w1", g.KIND_PARAM_LP).float().cpu().numpy(),
                                  sharded.tensor("h0.w1", g.KIND_PARAM_LP).float().cpu().numpy())


def test_deferred_tables_on_one_gpu_match_the_oracle(g):
    """tables="deferred" through the CUDA library on one GPU: both micro-batches'
    forwards see the initial tables, each table takes one sparse update over
    both micro-batches' (row, gradient) pairs at the optimizer step, and the
    dense weights take AdamW on the accumulated gradient -- against the oracle
    doing the same with its own forward/backward, table update and AdamW."""
    import torch
    from gpt_pretraining_step_decoder_b200 import dp
    from oracle import model as omodel, optim
    from oracle.step import OracleTrainer
    from synthetic import init_params
    from tests.helpers import export, import_params, rel_l2
    w = small_case("gpt2s_tables_bf16", grad_accum=2)
    params = init_params(w)
    m = g.Model(to_cfg(w), seed=w["seed"])
    import_params(m, params)
    B, T, V, lr = w["micro_batch"], w["seq_len"], w["vocab"], 1e-2
    host = [tokens_and_targets(B, T, V, w["seed"], w["zipf_s"], w["repeat_frac"], ignore_frac=0.05, micro=s)
            for s in range(2)]
    dp.train_step(m, [tuple(device_ints(x) for x in b) for b in host], lr, tables="deferred")
    assert m.sync_status() == g.GPT_OK, g.gpt_last_error()
    orc = OracleTrainer(w, params)
    pairs = {"hx": ([], []), "hv": ([], [])}
    for tok, tgt in host:
        rx, rv = orc.rows(tok)
        _, _, cache = omodel.forward(w, orc.P, tok, tgt, rx, rv)
        G, gx0, gv = omodel.backward(w, orc.P, cache, scale=0.5)
        for k in orc.dense:
            orc.acc[k] += G[k]
        for t, rows, gr in (("hx", rx, gx0), ("hv", rv, gv)):
            pairs[t][0].append(rows.reshape(-1))
            pairs[t][1].append(gr)
    for t in ("hv", "hx"):
        W0 = np.asarray(params[t], dtype=np.float64)
        Wn, Sn, uniq = optim.table_update(W0, np.zeros(W0.shape[0]), np.concatenate(pairs[t][0]),
                                          np.concatenate(pairs[t][1]), lr * w["lr_mult_table"], w["table_beta"],
                                          w["table_eps"])
        s_gpu = export(m, t, g.KIND_ROW_STATE)[:, 0]
        np.testing.assert_array_equal(np.nonzero(s_gpu)[0], uniq)
        assert rel_l2(s_gpu, Sn) < 2e-2
        assert rel_l2(export(m, t) - W0, Wn - W0) < 2e-2
    grads = {k: orc.acc[k].copy() for k in orc.dense}
    orc.optimizer_step(lr)
    for k in orc.dense:
        assert rel_l2(export(m, k, g.KIND_GRAD), grads[k]) < 2e-2, k
        assert rel_l2(export(m, k, g.KIND_ADAM_M), orc.m[k]) < 2e-2, k
