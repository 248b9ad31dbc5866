"""Host-made faults on the GPU, reported through the device error word."""

import pytest

from synthetic import tokens_and_targets, workload
from tests.helpers import device_ints, to_cfg

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    import torch
    import gpt_pretraining_step_decoder_b200 as g
    assert torch.cuda.is_available()
    return g


def test_nan_weight_reports_nonfinite_loss(g):
    """A NaN written into the embedding row of a token makes the loss
    non-finite; the next sync reports GPT_ERR_NONFINITE (no trap)."""
    import torch
    w = workload("tiny_fp32")
    model = g.Model(to_cfg(w), seed=w["seed"])
    tok, tgt = tokens_and_targets(w["micro_batch"], w["seq_len"], w["vocab"], w["seed"], w["zipf_s"],
                                  w["repeat_frac"])
    model.forward_loss(device_ints(tok), device_ints(tgt))
    assert model.sync_status() == g.GPT_OK
    model.tensor("wte")[int(tok[0, 0])] = float("nan")
    g.gpt_params_changed(model.h)
    loss = model.forward_loss(device_ints(tok), device_ints(tgt))
    torch.cuda.synchronize()
    assert model.sync_status() == g.GPT_ERR_NONFINITE
    assert not torch.isfinite(loss).all()
