"""The frozen trigram statistics table on the GPU against the oracle.

The table is tallied on the GPU (trigram_tally) and by the oracle from the
same seeded token streams; the row set is bit-exact, the statistics agree to
fp32 rounding (fp32 tables) or to bf16 rounding (bf16 tables).  Whole steps
with the table projected into the values are compared like every other step
(fp32 mode 1e-4; bf16 mode 2e-2), the projection's gradient included.
"""

import numpy as np
import pytest

from oracle import trigram
from synthetic import small_case, workload, zipf_stream
from tests.helpers import device_ints, export, rel_l2
from tests.stepcheck import check, run_pair

pytestmark = pytest.mark.gpu
P1, P2 = 2654435761, 2246822519


@pytest.fixture(scope="module")
def g():
    import torch
    import gpt_pretraining_step_decoder_b200 as g
    assert torch.cuda.is_available()
    return g


def tally_streams(vocab, S, L, seed):
    return zipf_stream(S * L, vocab, seed).reshape(S, L)


def gpu_tally(g, streams, vocab, rows, width, dtype, table):
    import torch
    S, L = streams.shape
    ws_bytes = g.trigram_tally_workspace_bytes(rows, width)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    g.trigram_tally(device_ints(streams), S, L, vocab, P1, P2, trigram.P3, rows, width, dtype, table, ws, ws_bytes)
    torch.cuda.synchronize()
    assert g.ngram_sync_status() == g.GPT_OK


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("rows,width,S,L", [(4096, 64, 16, 513), (1000, 8, 3, 77), (2097152, 64, 64, 2049)])
def test_tally_matches_oracle(g, dtype, rows, width, S, L):
    import torch
    vocab = 50304
    streams = tally_streams(vocab, S, L, 11 + rows % 97)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    table = torch.full((rows, width), 5.0, dtype=tdt, device="cuda")   # overwritten everywhere
    gpu_tally(g, streams, vocab, rows, width, g.DTYPE_F32 if dtype == "f32" else g.DTYPE_BF16, table)
    uniq, stats = trigram.tally_stats(streams, vocab, P1, P2, rows, width)
    got = table.float().cpu().numpy().astype(np.float64)
    nz = np.nonzero(got.any(axis=1))[0]
    np.testing.assert_array_equal(nz, uniq)                            # the rows that occur, bit-exact
    rtol = 1e-6 if dtype == "f32" else 2 ** -8
    np.testing.assert_allclose(got[uniq], stats, rtol=rtol, atol=0)


def test_tally_counts_out_of_range_tokens_as_errors(g):
    import torch
    streams = tally_streams(512, 2, 40, 3)
    streams[1, 7] = 600
    table = torch.zeros((256, 8), dtype=torch.float32, device="cuda")
    ws_bytes = g.trigram_tally_workspace_bytes(256, 8)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    g.trigram_tally(device_ints(streams), 2, 40, 512, P1, P2, trigram.P3, 256, 8, g.DTYPE_F32, table, ws, ws_bytes)
    assert g.ngram_sync_status() == g.GPT_ERR_INPUT
    assert g.ngram_sync_status() == g.GPT_OK


def _prepare(g, w, seed):
    """Tally the model's table on the GPU, the oracle's copy on the host, from the same streams."""
    def prepare(model, params):
        streams = tally_streams(w["vocab"], 8, 257, seed)
        dt = g.DTYPE_BF16 if w["dtype"] == "bf16" else g.DTYPE_F32
        gpu_tally(g, streams, w["vocab"], w["tri_rows"], w["tri_width"], dt, model.tensor("h3"))
        params["h3"] = trigram.dense_stats(streams, w["vocab"], P1, P2, w["tri_rows"], w["tri_width"])
        # the same statistics on both sides (the GPU table holds them rounded to its dtype)
        tol = 1e-6 if w["dtype"] != "bf16" else 2 ** -8
        np.testing.assert_allclose(export(model, "h3"), params["h3"], rtol=tol, atol=0)
    return prepare


def test_fp32_step_with_trigram_table(g):
    w = workload("tiny_fp32", tri_rows=1024, tri_width=8)
    model, orc, losses, tok, params = run_pair(g, w, steps=2, prepare=_prepare(g, w, 21))
    np.testing.assert_array_equal(model.tensor("rows_3", g.KIND_ACT).cpu().numpy(), orc.rows3(tok))
    check(g, w, model, orc, losses, params, 1e-4, 1e-4)
    assert rel_l2(export(model, "h3"), params["h3"]) < 1e-6   # frozen: unchanged by the steps


def test_bf16_step_with_trigram_and_bigram_tables(g):
    """Both bigram tables and the trigram statistics: the value bias adds the
    value-table row and the projected statistics; two micro-batches, AdamW."""
    w = small_case("gpt2s_tables_bf16", grad_accum=2, tri_rows=4096, tri_width=64)
    model, orc, losses, tok, params = run_pair(g, w, steps=2, prepare=_prepare(g, w, 22))
    np.testing.assert_array_equal(model.tensor("rows_3", g.KIND_ACT).cpu().numpy(), orc.rows3(tok))
    check(g, w, model, orc, losses, params, 1e-2, 2e-2)
