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
