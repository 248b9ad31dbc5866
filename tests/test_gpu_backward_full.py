"""Backward parity in the launch configurations the benchmark times.

A full-size micro-batch is too large for the fp64 oracle, but the loss of a
sequence depends only on that sequence (attention is causal inside each
sequence) and an ignored target (-1) contributes nothing to the loss.  So the
GPU runs the whole micro-batch -- every attention work item, every LM-head
chunk, the split-K weight gradients over all N rows -- with the targets of
all but two sequences set to -1, and its gradients must equal the oracle's
gradients of the loss over those two sequences alone.  That covers, at full
size: the persistent attention kernels' multi-item loops (more items than
SMs), the multi-chunk LM-head gradient accumulation, and split-K over
K = N = 32768.

Bars (bf16): loss 1e-2 relative; every dense gradient, the per-position
table gradients and the updated table rows 2e-2 relative L2; hash rows and
updated-row sets bit-exact.

The nanochat-d32 widths (d 2048, 16 heads of 128, MLP 8192, untied vocab
65536) and the long-context widths (d 1024, 8 heads, MLP 4096, T 2048) take a
whole training step, compared with the oracle step.
"""

import numpy as np
import pytest

from oracle import hashing, model as omodel, optim
from synthetic import init_params, round_to_bf16, tokens_and_targets, workload
from tests.helpers import device_ints, export, import_params, rel_l2, to_cfg
from tests.stepcheck import check, run_pair

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    import torch
    import gpt_pretraining_step_decoder_b200 as g
    assert torch.cuda.is_available()
    return g


def masked_batch(w, keep, ignore_frac=0.02):
    """Full-size tokens/targets with every target outside the sequences `keep` set to -1."""
    tok, tgt = tokens_and_targets(w["micro_batch"], w["seq_len"], w["vocab"], w["seed"], w["zipf_s"],
                                  w["repeat_frac"], ignore_frac=ignore_frac)
    mask = np.ones(w["micro_batch"], dtype=bool)
    mask[list(keep)] = False
    tgt = tgt.copy()
    tgt[mask] = -1
    return tok, tgt


def oracle_two(w, params, tok, tgt, keep, rows=None, rows3=None):
    """Oracle loss and gradients of the loss over the sequences `keep` alone."""
    wk = dict(w, micro_batch=len(keep))
    rx = rv = None
    if rows is not None:
        rx, rv = rows
    loss, _, cache = omodel.forward(wk, params, tok[list(keep)], tgt[list(keep)], rx, rv, rows3)
    G, gx0, gv = omodel.backward(wk, params, cache, scale=1.0)
    return loss, G, gx0, gv


def compare_dense(g, gm, G, tol=2e-2):
    worst = 0.0
    for name, ref in G.items():
        e = rel_l2(export(gm, name, g.KIND_GRAD), ref)
        assert e < tol, (name, e)
        worst = max(worst, e)
    return worst


def test_gpt2_small_full_launch_backward(g):
    """12 x 768 widths, 32 x 1024 tokens, tied vocab 50304, two layers: 1536
    attention items per kernel over 148 SMs, four 8192-row LM-head chunks
    (the kept sequences sit in the first and the last), split-K weight
    gradients over K = 32768."""
    w = workload("gpt2s_bf16", n_layer=2)
    keep = (0, 29)
    params = init_params(w)
    gm = g.Model(to_cfg(w), seed=w["seed"])
    import_params(gm, params)
    tok, tgt = masked_batch(w, keep)
    loss = gm.forward_loss(device_ints(tok), device_ints(tgt))
    gm.backward(1e-3)                     # gradients only: no optimizer step
    assert gm.sync_status() == g.GPT_OK, g.gpt_last_error()
    lo, G, _, _ = oracle_two(w, params, tok, tgt, keep)
    assert abs(float(loss.item()) - lo) / lo < 1e-2
    compare_dense(g, gm, G)


def test_tables_full_launch_backward_and_update(g):
    """Both bigram tables at full size (2,097,152 and 1,048,576 rows x 768),
    16 x 2048 tokens, two layers.  The table gradients per position (x0 and
    value table, the latter summed over layers) are read in exchange mode and
    compared with the oracle's; then the sparse update over all 32768
    positions is applied and the changed rows compared with the oracle's
    update over the two kept sequences (every other position's gradient is
    exactly zero)."""
    import torch
    from gpt_pretraining_step_decoder_b200 import dp
    w = workload("gpt2s_tables_bf16", n_layer=2, grad_accum=1)
    keep = (1, 14)
    T, d = w["seq_len"], w["d_model"]
    params = init_params(w, skip_tables=True)
    tok, tgt = masked_batch(w, keep)
    rx = hashing.bigram_rows(tok[list(keep)], w["vocab"], w["hash_p1"], w["hash_p2"], w["x0_rows"])
    rv = hashing.bigram_rows(tok[list(keep)], w["vocab"], w["hash_p1"], w["hash_p2"], w["v_rows"])
    ux, uv = np.unique(rx), np.unique(rv)
    rng = np.random.default_rng(4343)
    vx = round_to_bf16((rng.standard_normal((len(ux), d)) * 0.02).astype(np.float32))
    vv = round_to_bf16((rng.standard_normal((len(uv), d)) * 0.02).astype(np.float32))

    gm = g.Model(to_cfg(w), seed=w["seed"])
    import_params(gm, params)
    for name, u, vals in (("hx", ux, vx), ("hv", uv, vv)):
        t = gm.tensor(name)
        t.zero_()
        t[torch.from_numpy(u).cuda()] = torch.from_numpy(vals).to(t.dtype).cuda()
    gm.set_table_exchange(True)
    loss = gm.forward_loss(device_ints(tok), device_ints(tgt))
    gm.backward(1e-3)
    assert gm.sync_status() == g.GPT_OK, g.gpt_last_error()
    np.testing.assert_array_equal(gm.tensor("rows_x", g.KIND_ACT).cpu().numpy()[list(keep)], rx)
    np.testing.assert_array_equal(gm.tensor("rows_v", g.KIND_ACT).cpu().numpy()[list(keep)], rv)

    pc = dict(params)
    pc["hx"], pc["hv"] = vx.astype(np.float64), vv.astype(np.float64)
    crx, crv = np.searchsorted(ux, rx), np.searchsorted(uv, rv)
    wc = dict(w, x0_rows=len(ux), v_rows=len(uv))
    lo, G, gx0, gv = oracle_two(wc, pc, tok, tgt, keep, rows=(crx, crv))
    assert abs(float(loss.item()) - lo) / lo < 1e-2
    compare_dense(g, gm, G)
    pos = np.concatenate([np.arange(b * T, (b + 1) * T) for b in keep])
    ggx = gm.tensor("table_grad_x", g.KIND_ACT).cpu().numpy()
    ggv = gm.tensor("table_grad_v", g.KIND_ACT).cpu().numpy()
    assert rel_l2(ggx[pos], gx0) < 2e-2
    assert rel_l2(ggv[pos], gv) < 2e-2
    rest = np.setdiff1d(np.arange(ggx.shape[0]), pos)
    assert not ggx[rest].any() and not ggv[rest].any()   # ignored sequences: exactly zero

    # the sparse update over all positions, as the inline path would apply it
    lr = 1e-2
    dp.exchange_tables(gm, lr)
    gm.set_table_exchange(False)
    assert g.ngram_sync_status() == g.GPT_OK
    for name, u, vals, rows_c, grad in (("hx", ux, vx, crx, gx0), ("hv", uv, vv, crv, gv)):
        W, S, _ = optim.table_update(vals.astype(np.float64), np.zeros(len(u)), rows_c.reshape(-1), grad,
                                     lr * w["lr_mult_table"], w["table_beta"], w["table_eps"])
        st = gm.tensor(name, g.KIND_ROW_STATE)[:, 0].cpu().numpy()
        np.testing.assert_array_equal(np.nonzero(st)[0], u)          # updated-row set
        assert rel_l2(st[u], S) < 2e-2
        Wg = gm.tensor(name)[torch.from_numpy(u).cuda()].float().cpu().numpy().astype(np.float64)
        assert rel_l2(Wg - vals, W - vals) < 2e-2


def test_d32_widths_full_step(g):
    """nanochat-d32 widths: d 2048, 16 heads of 128, MLP 8192, untied vocab
    65536; one layer, T 256; one whole training step with AdamW."""
    w = workload("d32_bf16", n_layer=1, seq_len=256, micro_batch=1)
    model, orc, losses, _, params = run_pair(g, w, steps=1)
    check(g, w, model, orc, losses, params, 1e-2, 2e-2)


def test_long_context_widths_full_step(g):
    """Long-context widths: d 1024, 8 heads of 128, MLP 4096, vocab 50304,
    T 2048 with the repeated-span token stream; one layer; a whole step."""
    w = workload("long2048_bf16", n_layer=1, micro_batch=1)
    model, orc, losses, _, params = run_pair(g, w, steps=1)
    check(g, w, model, orc, losses, params, 1e-2, 2e-2)


def test_trigram_table_full_launch_backward(g):
    """The frozen trigram statistics at full size (2,097,152 rows x 64, tallied
    on the GPU from 64 x 2049 tokens) with both bigram tables, 16 x 2048
    tokens, two layers: every dense gradient, the projection's included,
    over the two kept sequences.  The oracle tallies the same streams and
    keeps only the rows the kept sequences touch."""
    import torch
    from oracle import trigram
    from synthetic import zipf_stream
    w = workload("gpt2s_tables_bf16", n_layer=2, grad_accum=1, tri_rows=2097152, tri_width=64)
    keep = (2, 13)
    params = init_params(w, skip_tables=True)
    tok, tgt = masked_batch(w, keep)
    kt = tok[list(keep)]
    gm = g.Model(to_cfg(w), seed=w["seed"])
    import_params(gm, params)
    for name in ("hx", "hv"):
        gm.tensor(name).zero_()
    streams = zipf_stream(64 * 2049, w["vocab"], 777).reshape(64, 2049)
    ws_bytes = g.trigram_tally_workspace_bytes(w["tri_rows"], 64)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    g.trigram_tally(device_ints(streams), 64, 2049, w["vocab"], w["hash_p1"], w["hash_p2"], w["hash_p3"],
                    w["tri_rows"], 64, g.DTYPE_BF16, gm.tensor("h3"), ws, ws_bytes)
    loss = gm.forward_loss(device_ints(tok), device_ints(tgt))
    gm.backward(1e-3)
    assert gm.sync_status() == g.GPT_OK, g.gpt_last_error()
    r3 = trigram.trigram_rows(kt, w["vocab"], w["hash_p1"], w["hash_p2"], w["tri_rows"], w["hash_p3"])
    np.testing.assert_array_equal(gm.tensor("rows_3", g.KIND_ACT).cpu().numpy()[list(keep)], r3)
    uniq, stats = trigram.tally_stats(streams, w["vocab"], w["hash_p1"], w["hash_p2"], w["tri_rows"], 64,
                                      w["hash_p3"])
    u3 = np.unique(r3)
    s3 = np.zeros((len(u3), 64))
    hit = np.isin(u3, uniq)
    s3[hit] = stats[np.searchsorted(uniq, u3[hit])]
    assert hit.sum() > 0
    pc = dict(params)
    pc["h3"] = s3
    # the tables are zero here, so the oracle carries them as zero rows
    rx = hashing.bigram_rows(kt, w["vocab"], w["hash_p1"], w["hash_p2"], w["x0_rows"])
    rv = hashing.bigram_rows(kt, w["vocab"], w["hash_p1"], w["hash_p2"], w["v_rows"])
    pc["hx"] = np.zeros((1, w["d_model"]))
    pc["hv"] = np.zeros((1, w["d_model"]))
    wc = dict(w, x0_rows=1, v_rows=1, tri_rows=len(u3))
    lo, G, _, _ = oracle_two(wc, pc, tok, tgt, keep, rows=(0 * rx, 0 * rv), rows3=np.searchsorted(u3, r3))
    assert abs(float(loss.item()) - lo) / lo < 1e-2
    compare_dense(g, gm, G)
