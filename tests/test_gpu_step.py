"""Full training-step parity on the GPU against the fp64 oracle, through the C ABI.

Same seeded weights (imported into the model) and the same seeded Zipf token
streams feed both sides.  Bars: fp32 mode 1e-4; bf16 mode loss 1e-2 relative
and per-tensor gradient / weight-change / AdamW-moment relative L2 2e-2; hash
rows and updated-row sets bit-exact.  Updated weights are compared as their
change from the starting weights (W - W0), never as W itself.
"""

import numpy as np
import pytest

from synthetic import init_params, small_case, tokens_and_targets, workload
from tests.helpers import device_ints, export, rel_l2, to_cfg
from tests.stepcheck import check, run_pair

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    import torch
    import gpt_pretraining_step_decoder_b200 as g
    assert torch.cuda.is_available()
    return g


def test_fp32_tiny_two_steps(g):
    w = workload("tiny_fp32")
    model, orc, losses, tok, params = run_pair(g, w, steps=2)
    # hash rows bit-exact
    rx = model.tensor("rows_x", g.KIND_ACT).cpu().numpy()
    np.testing.assert_array_equal(rx, orc.rows(tok)[0])
    check(g, w, model, orc, losses, params, 1e-4, 1e-4)


def test_fp32_adamw_from_zero_moments(g):
    """The first AdamW step from zero moments (-lr*sign(g) up to eps) in fp32,
    where no gradient element is near enough to zero for its sign to flip."""
    w = workload("tiny_fp32")
    model, orc, losses, _, params = run_pair(g, w, steps=1, seed_moments=False)
    check(g, w, model, orc, losses, params, 1e-4, 1e-4)


@pytest.mark.parametrize("variant", [dict(), dict(tie_embeddings=0, softcap=15.0, grad_clip=1.0)])
def test_fp32_variants(g, variant):
    w = workload("tiny_fp32", **variant)
    model, orc, losses, _, params = run_pair(g, w, steps=1)
    check(g, w, model, orc, losses, params, 1e-4, 1e-4)


def test_bf16_gpt2_small_shape(g):
    w = small_case("gpt2s_bf16", grad_accum=2)
    model, orc, losses, _, params = run_pair(g, w, steps=2)
    check(g, w, model, orc, losses, params, 1e-2, 2e-2)


def test_bf16_softcap_untied_clip(g):
    """The tensor-core path with nanochat's logit softcap (z = 15 tanh(acc/15)),
    an untied head and global-norm clipping."""
    w = small_case("gpt2s_bf16", grad_accum=2, softcap=15.0, tie_embeddings=0, grad_clip=1.0)
    model, orc, losses, _, params = run_pair(g, w, steps=2)
    check(g, w, model, orc, losses, params, 1e-2, 2e-2)


def test_bf16_with_tables(g):
    # two micro-batches per AdamW step: both table updates happen (one per
    # backward call) and the accumulated dense gradient is compared before the
    # first AdamW step, whose -lr*sign(g) update would otherwise amplify bf16
    # noise on near-zero gradient elements into the next step
    w = small_case("gpt2s_tables_bf16", grad_accum=2)
    model, orc, losses, tok, params = run_pair(g, w, steps=2)
    check(g, w, model, orc, losses, params, 1e-2, 2e-2)
    rx = model.tensor("rows_x", g.KIND_ACT).cpu().numpy()
    rv = model.tensor("rows_v", g.KIND_ACT).cpu().numpy()
    ox, ov = orc.rows(tok)
    np.testing.assert_array_equal(rx, ox)
    np.testing.assert_array_equal(rv, ov)


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
    model, orc, losses, _, params = run_pair(g, w, steps=2)
    check(g, w, model, orc, losses, params, 1e-2, 2e-2)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_lm_head_several_ragged_chunks(g, dtype):
    """The LM head + cross-entropy in chunks of 136 rows (N = 400: 136, 136,
    128), so the head's weight gradient is accumulated over several chunks
    and the last chunk is ragged; the whole step is compared."""
    if dtype == "bf16":
        w = small_case("gpt2s_bf16", grad_accum=2, lm_chunk_rows=136)
        model, orc, losses, _, params = run_pair(g, w, steps=2)
        check(g, w, model, orc, losses, params, 1e-2, 2e-2)
    else:
        w = workload("tiny_fp32", lm_chunk_rows=136, tie_embeddings=0)   # N = 256: 136 + 120
        model, orc, losses, _, params = run_pair(g, w, steps=2)
        check(g, w, model, orc, losses, params, 1e-4, 1e-4)
