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


def test_bounded_wait_gives_up_and_context_stays_usable(g):
    """A bounded wait on a barrier nothing arrives on gives up after its limit
    (50 ms here), the standalone status reports GPT_ERR_TIMEOUT once and is
    then clear, and the same stream runs a table gather correctly after it."""
    import time
    import numpy as np
    import torch
    s = torch.cuda.current_stream()
    assert g.ngram_sync_status(s) == g.GPT_OK
    t0 = time.perf_counter()
    g.gptx_wait_probe(50_000, s)
    assert g.ngram_sync_status(s) == g.GPT_ERR_TIMEOUT
    assert time.perf_counter() - t0 >= 0.04
    assert g.ngram_sync_status(s) == g.GPT_OK   # read and cleared
    # the context still runs kernels: a gather of known rows
    table = torch.arange(64 * 16, dtype=torch.float32, device="cuda").reshape(64, 16).to(torch.bfloat16)
    rows = torch.tensor([3, 0, 63, 3], dtype=torch.int32, device="cuda")
    out = torch.zeros(4, 16, dtype=torch.bfloat16, device="cuda")
    g.ngram_gather(rows, 4, table, 64, 16, g.DTYPE_BF16, out, 0, s)
    torch.cuda.synchronize()
    assert g.ngram_sync_status(s) == g.GPT_OK
    np.testing.assert_array_equal(out.float().cpu().numpy(), table.float().cpu().numpy()[[3, 0, 63, 3]])
