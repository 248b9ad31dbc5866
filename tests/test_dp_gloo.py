"""Data-parallel host logic with two gloo ranks on the CPU.

Each rank takes its own slice of the token stream (dp.rank_stream_seed),
computes its gradient with the fp64 oracle, and averages it with
dp.average_gradients -- the same call the GPU path makes on the flat fp32
gradient.  The average must equal the gradient of the loss over both ranks'
sequences taken together (every target valid, equal counts per rank), and the
AdamW step that follows must leave bit-identical replicas.
"""

import os
import socket

import numpy as np
import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cfg():
    from synthetic import workload
    return workload("tiny_fp32", x0_rows=0, n_layer=1, seq_len=16, micro_batch=2, vocab=96)


def _batch(cfg, seed):
    from synthetic import tokens_and_targets
    return tokens_and_targets(cfg["micro_batch"], cfg["seq_len"], cfg["vocab"], seed, cfg["zipf_s"], 0.0)


def _flat(G, keys):
    return np.concatenate([np.asarray(G[k], dtype=np.float64).reshape(-1) for k in keys])


def _rank_main(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist
    from gpt_pretraining_step_decoder_b200 import dp
    from oracle import model, optim
    from synthetic import init_params

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        cfg = _cfg()
        params = init_params(cfg, seed=3)
        keys = sorted(params)
        tok, tgt = _batch(cfg, dp.rank_stream_seed(cfg["seed"], rank))
        _, _, cache = model.forward(cfg, params, tok, tgt, None, None)
        G, _, _ = model.backward(cfg, params, cache, scale=1.0)
        flat = torch.from_numpy(_flat(G, keys))
        dp.average_gradients(flat)
        avg = flat.numpy()

        # the same step taken by every rank from the averaged gradient
        new, off = {}, 0
        for k in keys:
            n = np.asarray(params[k]).size
            g = avg[off:off + n].reshape(np.shape(params[k]))
            off += n
            z = np.zeros_like(g)
            new[k], _, _ = optim.adamw(np.asarray(params[k], dtype=np.float64), g, z, z.copy(), 1, 1e-3,
                                       cfg["adam_b1"], cfg["adam_b2"], cfg["adam_eps"], cfg["weight_decay"])
        mine = torch.from_numpy(_flat(new, keys))
        all_params = [torch.empty_like(mine) for _ in range(world)]
        dist.all_gather(all_params, mine)
        if rank == 0:
            np.save(os.path.join(out_dir, "avg.npy"), avg)
            np.save(os.path.join(out_dir, "params.npy"), torch.stack(all_params).numpy())
    finally:
        dist.destroy_process_group()


def test_two_rank_gradient_average_equals_joint_batch(tmp_path):
    import torch.multiprocessing as mp
    from gpt_pretraining_step_decoder_b200 import dp
    from oracle import model, optim
    from synthetic import init_params

    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    avg = np.load(tmp_path / "avg.npy")
    reps = np.load(tmp_path / "params.npy")

    cfg = _cfg()
    params = init_params(cfg, seed=3)
    keys = sorted(params)
    toks, tgts = zip(*[_batch(cfg, dp.rank_stream_seed(cfg["seed"], r)) for r in range(world)])
    joint = dict(cfg, micro_batch=cfg["micro_batch"] * world)
    _, _, cache = model.forward(joint, params, np.concatenate(toks), np.concatenate(tgts), None, None)
    G, _, _ = model.backward(joint, params, cache, scale=1.0)
    ref = _flat(G, keys)
    assert np.abs(avg - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())

    # replicas identical bit for bit, and equal to one joint-batch AdamW step
    np.testing.assert_array_equal(reps[0], reps[1])
    new = {}
    for k in keys:
        g = np.asarray(G[k], dtype=np.float64)
        z = np.zeros_like(g)
        new[k], _, _ = optim.adamw(np.asarray(params[k], dtype=np.float64), g, z, z.copy(), 1, 1e-3,
                                   cfg["adam_b1"], cfg["adam_b2"], cfg["adam_eps"], cfg["weight_decay"])
    np.testing.assert_allclose(reps[0], _flat(new, keys), rtol=0, atol=1e-9)


def test_rank_streams_differ():
    from gpt_pretraining_step_decoder_b200 import dp
    cfg = _cfg()
    a, _ = _batch(cfg, dp.rank_stream_seed(cfg["seed"], 0))
    b, _ = _batch(cfg, dp.rank_stream_seed(cfg["seed"], 1))
    assert a.shape == b.shape and not np.array_equal(a, b)


def _table_cfg():
    from synthetic import workload
    # few rows, so the two ranks' positions share rows and the exchange matters
    return workload("tiny_fp32", n_layer=1, seq_len=16, micro_batch=2, vocab=96, x0_rows=64, v_rows=32)


def _table_grads(cfg, params, tok, tgt, scale=1.0):
    from oracle import hashing, model
    rx = hashing.bigram_rows(tok, cfg["vocab"], cfg["hash_p1"], cfg["hash_p2"], cfg["x0_rows"])
    rv = hashing.bigram_rows(tok, cfg["vocab"], cfg["hash_p1"], cfg["hash_p2"], cfg["v_rows"])
    _, _, cache = model.forward(cfg, params, tok, tgt, rx, rv)
    _, gx0, gv = model.backward(cfg, params, cache, scale=scale)
    return rx.reshape(-1), gx0, rv.reshape(-1), gv


def _apply_tables(cfg, params, rows_v, gv, rows_x, gx0, lr):
    from oracle import optim
    out = {}
    for t, rows, g in (("hv", rows_v, gv), ("hx", rows_x, gx0)):
        W = np.asarray(params[t], dtype=np.float64)
        out[t], out[t + "_state"], _ = optim.table_update(W, np.zeros(W.shape[0]), rows, g, lr,
                                                          cfg["table_beta"], cfg["table_eps"])
    return out


def _table_rank_main(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist
    from gpt_pretraining_step_decoder_b200 import dp
    from synthetic import init_params

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        cfg = _table_cfg()
        params = init_params(cfg, seed=3)
        tok, tgt = _batch(cfg, dp.rank_stream_seed(cfg["seed"], rank))
        rx, gx0, rv, gv = _table_grads(cfg, params, tok, tgt)
        ex = {}
        for name, rows, g in (("x", rx, gx0), ("v", rv, gv)):
            r_all, g_all = dp.gather_table_grads(torch.from_numpy(rows.astype(np.int32)), torch.from_numpy(g))
            ex[name] = (r_all.numpy(), g_all.numpy())
        new = _apply_tables(cfg, params, ex["v"][0], ex["v"][1], ex["x"][0], ex["x"][1], 1e-2)
        flat = torch.from_numpy(np.concatenate([new[k].reshape(-1) for k in ("hv", "hv_state", "hx", "hx_state")]))
        reps = [torch.empty_like(flat) for _ in range(world)]
        dist.all_gather(reps, flat)
        if rank == 0:
            np.save(os.path.join(out_dir, "tables.npy"), torch.stack(reps).numpy())
    finally:
        dist.destroy_process_group()


def test_two_rank_table_exchange_equals_joint_batch_update(tmp_path):
    """Replicated bigram tables: each rank's per-position table gradients are
    gathered in rank order (scaled by 1/world) and every rank applies the same
    sparse update.  The replicas must be bit-identical and equal the update a
    single process makes from the joint batch's gradients."""
    import torch.multiprocessing as mp
    from gpt_pretraining_step_decoder_b200 import dp
    from synthetic import init_params

    world = 2
    mp.spawn(_table_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    reps = np.load(tmp_path / "tables.npy")
    np.testing.assert_array_equal(reps[0], reps[1])

    cfg = _table_cfg()
    params = init_params(cfg, seed=3)
    toks, tgts = zip(*[_batch(cfg, dp.rank_stream_seed(cfg["seed"], r)) for r in range(world)])
    joint = dict(cfg, micro_batch=cfg["micro_batch"] * world)
    rx, gx0, rv, gv = _table_grads(joint, params, np.concatenate(toks), np.concatenate(tgts))
    ref = _apply_tables(cfg, params, rv, gv, rx, gx0, 1e-2)
    flat = np.concatenate([ref[k].reshape(-1) for k in ("hv", "hv_state", "hx", "hx_state")])
    np.testing.assert_allclose(reps[0], flat, rtol=1e-12, atol=1e-15)
    # the exchange mattered: the ranks' positions share rows
    rows0 = set(_table_grads(cfg, params, toks[0], tgts[0])[0])
    rows1 = set(_table_grads(cfg, params, toks[1], tgts[1])[0])
    assert rows0 & rows1


class _OracleModel:
    """The slice of `Model` that dp.train_step uses, backed by the fp64 oracle
    on CPU tensors (table updates inline unless the exchange mode is on)."""

    def __init__(self, cfg, params):
        import types
        import torch
        self.torch, self.stream, self.w = torch, None, cfg
        self.cfg = types.SimpleNamespace(x0_rows=cfg["x0_rows"], v_rows=cfg["v_rows"], dtype=0,
                                         lr_mult_table=cfg["lr_mult_table"], table_beta=cfg["table_beta"],
                                         table_eps=cfg["table_eps"])
        self.P = {k: np.array(v, dtype=np.float64) for k, v in params.items()}
        self.keys = sorted(k for k in self.P if k not in ("hx", "hv"))
        self.S = {t: np.zeros(self.P[t].shape[0]) for t in ("hx", "hv")}
        self.grad = torch.zeros(sum(self.P[k].size for k in self.keys), dtype=torch.float64)
        self.table_exchange, self.calls = False, []

    def set_table_exchange(self, on):
        self.table_exchange = bool(on)
        self.calls.append("exchange_on" if on else "exchange_off")

    def forward_loss(self, tok, tgt):
        from oracle import hashing, model
        w = self.w
        self.rx = hashing.bigram_rows(tok, w["vocab"], w["hash_p1"], w["hash_p2"], w["x0_rows"])
        self.rv = hashing.bigram_rows(tok, w["vocab"], w["hash_p1"], w["hash_p2"], w["v_rows"])
        self.loss, _, self.cache = model.forward(w, self.P, tok, tgt, self.rx, self.rv)
        self.calls.append("forward")

    def backward(self, lr):
        from oracle import model, optim
        G, self.gx0, self.gv = model.backward(self.w, self.P, self.cache, scale=1.0)
        self.grad += self.torch.from_numpy(_flat(G, self.keys))
        if not self.table_exchange:
            lr_t = lr * self.cfg.lr_mult_table
            for t, rows, g in (("hv", self.rv, self.gv), ("hx", self.rx, self.gx0)):
                self.P[t], self.S[t], _ = optim.table_update(self.P[t], self.S[t], rows.reshape(-1), g, lr_t,
                                                             self.cfg.table_beta, self.cfg.table_eps)
        self.calls.append("backward")

    def tensor(self, name, kind=0):
        import gpt_pretraining_step_decoder_b200 as g
        t = self.torch
        if kind == g.KIND_ACT:
            return {"rows_x": t.from_numpy(self.rx.astype(np.int32)), "rows_v": t.from_numpy(self.rv.astype(np.int32)),
                    "table_grad_x": t.from_numpy(self.gx0), "table_grad_v": t.from_numpy(self.gv)}[name]
        if kind == g.KIND_PARAM:
            return t.from_numpy(self.P[name])  # shares memory: updated in place
        if kind == g.KIND_ROW_STATE:
            return t.from_numpy(self.S[name])
        raise KeyError(name)

    def flat_grad(self):
        return self.grad

    def optimizer_step(self, lr):
        self.calls.append("optimizer")


def _oracle_sparse_update(W, state, n_rows, d, dtype, rows, grad, n, lr, beta, eps, upd, nupd, ws, ws_bytes,
                          stream=None):
    """Stands in for the CUDA ngram_sparse_update inside the CPU ranks."""
    from oracle import optim
    assert rows.numel() == n and tuple(grad.shape) == (n, d) and W.shape == (n_rows, d) and dtype == 0
    newW, newS, uniq = optim.table_update(W.numpy(), state.numpy(), rows.numpy(), grad.numpy(), lr, beta, eps)
    W.copy_(W.new_tensor(newW))
    state.copy_(state.new_tensor(newS))
    if upd is not None:
        upd[:len(uniq)] = upd.new_tensor(uniq)
    if nupd is not None:
        nupd[0] = len(uniq)


def _train_rank_main(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist
    import gpt_pretraining_step_decoder_b200 as g
    from gpt_pretraining_step_decoder_b200 import dp
    from synthetic import init_params

    g.ngram_sparse_update = _oracle_sparse_update
    g.ngram_sparse_update_workspace_bytes = lambda n, d: 1
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        cfg = dict(_table_cfg(), lr_mult_table=0.5)
        m = _OracleModel(cfg, init_params(cfg, seed=3))
        batches = [_batch(cfg, dp.rank_stream_seed(cfg["seed"], rank) + 7 * s) for s in range(2)]
        dp.train_step(m, batches, 2e-2)
        flat = torch.from_numpy(np.concatenate([m.P[t].reshape(-1) for t in ("hv", "hx")] +
                                               [m.S[t] for t in ("hv", "hx")]))
        reps = [torch.empty_like(flat) for _ in range(world)]
        dist.all_gather(reps, flat)
        if rank == 0:
            np.save(os.path.join(out_dir, "tables.npy"), torch.stack(reps).numpy())
            np.save(os.path.join(out_dir, "calls.npy"), np.array(m.calls))
    finally:
        dist.destroy_process_group()


def test_train_step_exchanges_tables_after_every_backward(tmp_path):
    """dp.train_step with two ranks and tables: exchange mode on, the tables
    exchanged after each micro-batch's backward (value table, then x0; the
    table lr multiplier applied; gradients scaled 1/world), replicas equal,
    and equal to one process updating per micro-batch over the joint batch."""
    import torch.multiprocessing as mp
    from gpt_pretraining_step_decoder_b200 import dp
    from oracle import model, optim
    from synthetic import init_params

    world = 2
    mp.spawn(_train_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    reps = np.load(tmp_path / "tables.npy")
    calls = list(np.load(tmp_path / "calls.npy"))
    assert calls == ["exchange_on", "forward", "backward", "forward", "backward", "optimizer", "exchange_off"]
    np.testing.assert_array_equal(reps[0], reps[1])

    cfg = dict(_table_cfg(), lr_mult_table=0.5)
    P = {k: np.array(v, dtype=np.float64) for k, v in init_params(cfg, seed=3).items()}
    S = {t: np.zeros(P[t].shape[0]) for t in ("hx", "hv")}
    joint = dict(cfg, micro_batch=cfg["micro_batch"] * world)
    for s in range(2):
        parts = [_batch(cfg, dp.rank_stream_seed(cfg["seed"], r) + 7 * s) for r in range(world)]
        tok = np.concatenate([p[0] for p in parts])
        tgt = np.concatenate([p[1] for p in parts])
        rx, gx0, rv, gv = _table_grads(joint, P, tok, tgt)
        for t, rows, g in (("hv", rv, gv), ("hx", rx, gx0)):
            P[t], S[t], _ = optim.table_update(P[t], S[t], rows, g, 2e-2 * 0.5, cfg["table_beta"], cfg["table_eps"])
    ref = np.concatenate([P[t].reshape(-1) for t in ("hv", "hx")] + [S[t] for t in ("hv", "hx")])
    np.testing.assert_allclose(reps[0], ref, rtol=1e-11, atol=1e-14)


def _deferred_rank_main(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist
    import gpt_pretraining_step_decoder_b200 as g
    from gpt_pretraining_step_decoder_b200 import dp
    from synthetic import init_params

    g.ngram_sparse_update = _oracle_sparse_update
    g.ngram_sparse_update_workspace_bytes = lambda n, d: 1
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        cfg = dict(_table_cfg(), lr_mult_table=0.5)
        m = _OracleModel(cfg, init_params(cfg, seed=3))
        batches = [_batch(cfg, dp.rank_stream_seed(cfg["seed"], rank) + 7 * s) for s in range(2)]
        dp.train_step(m, batches, 2e-2, tables="deferred")
        flat = torch.from_numpy(np.concatenate([m.P[t].reshape(-1) for t in ("hv", "hx")] +
                                               [m.S[t] for t in ("hv", "hx")]))
        reps = [torch.empty_like(flat) for _ in range(world)]
        dist.all_gather(reps, flat)
        if rank == 0:
            np.save(os.path.join(out_dir, "tables.npy"), torch.stack(reps).numpy())
    finally:
        dist.destroy_process_group()


def test_train_step_deferred_tables_take_one_update_per_step(tmp_path):
    """tables="deferred": both micro-batches' (row, gradient) pairs of both
    ranks are collected and each table takes one sparse update at the
    optimizer step; the forwards of the step all see the initial tables."""
    import torch.multiprocessing as mp
    from gpt_pretraining_step_decoder_b200 import dp
    from oracle import optim
    from synthetic import init_params

    world = 2
    mp.spawn(_deferred_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    reps = np.load(tmp_path / "tables.npy")
    np.testing.assert_array_equal(reps[0], reps[1])

    cfg = dict(_table_cfg(), lr_mult_table=0.5)
    P = {k: np.array(v, dtype=np.float64) for k, v in init_params(cfg, seed=3).items()}
    joint = dict(cfg, micro_batch=cfg["micro_batch"] * world)
    acc = {"hv": ([], []), "hx": ([], [])}
    for s in range(2):
        parts = [_batch(cfg, dp.rank_stream_seed(cfg["seed"], r) + 7 * s) for r in range(world)]
        rx, gx0, rv, gv = _table_grads(joint, P, np.concatenate([p[0] for p in parts]),
                                       np.concatenate([p[1] for p in parts]))
        for t, rows, g in (("hv", rv, gv), ("hx", rx, gx0)):
            acc[t][0].append(rows)
            acc[t][1].append(g)
    out = []
    for t in ("hv", "hx"):
        W, S, _ = optim.table_update(P[t], np.zeros(P[t].shape[0]), np.concatenate(acc[t][0]),
                                     np.concatenate(acc[t][1]), 2e-2 * 0.5, cfg["table_beta"], cfg["table_eps"])
        out.append((W, S))
    ref = np.concatenate([out[0][0].reshape(-1), out[1][0].reshape(-1), out[0][1], out[1][1]])
    np.testing.assert_allclose(reps[0], ref, rtol=1e-11, atol=1e-14)
    # and it is not the inline schedule, whose second micro-batch sees updated tables
    Pi = {k: np.array(v, dtype=np.float64) for k, v in init_params(cfg, seed=3).items()}
    Si = {t: np.zeros(Pi[t].shape[0]) for t in ("hx", "hv")}
    for s in range(2):
        parts = [_batch(cfg, dp.rank_stream_seed(cfg["seed"], r) + 7 * s) for r in range(world)]
        rx, gx0, rv, gv = _table_grads(joint, Pi, np.concatenate([p[0] for p in parts]),
                                       np.concatenate([p[1] for p in parts]))
        for t, rows, g in (("hv", rv, gv), ("hx", rx, gx0)):
            Pi[t], Si[t], _ = optim.table_update(Pi[t], Si[t], rows, g, 2e-2 * 0.5, cfg["table_beta"],
                                                 cfg["table_eps"])
    inline = np.concatenate([Pi["hv"].reshape(-1), Pi["hx"].reshape(-1), Si["hv"], Si["hx"]])
    assert np.abs(inline - ref).max() > 1e-6


def test_train_step_restores_inline_table_updates(monkeypatch):
    """After a deferred train_step (one process, no process group) the model is
    back in inline mode: a plain backward updates the tables again."""
    import gpt_pretraining_step_decoder_b200 as g
    from gpt_pretraining_step_decoder_b200 import dp
    from synthetic import init_params

    monkeypatch.setattr(g, "ngram_sparse_update", _oracle_sparse_update)
    monkeypatch.setattr(g, "ngram_sparse_update_workspace_bytes", lambda n, d: 1)

    cfg = _table_cfg()
    m = _OracleModel(cfg, init_params(cfg, seed=3))
    dp.train_step(m, [_batch(cfg, 11)], 2e-2, tables="deferred")
    assert m.calls[0] == "exchange_on" and m.calls[-1] == "exchange_off"
    assert not m.table_exchange
    hx0 = m.P["hx"].copy()
    m.forward_loss(*_batch(cfg, 12))
    m.backward(2e-2)
    assert np.abs(m.P["hx"] - hx0).max() > 0


def test_train_step_restores_exchange_mode_when_a_call_fails():
    """An exception inside the step (here: a failing backward) still turns
    the exchange mode back off."""
    from gpt_pretraining_step_decoder_b200 import dp
    from synthetic import init_params

    cfg = _table_cfg()
    m = _OracleModel(cfg, init_params(cfg, seed=3))

    def broken(lr):
        raise RuntimeError("backward failed")
    m.backward = broken
    with pytest.raises(RuntimeError):
        dp.train_step(m, [_batch(cfg, 11)], 2e-2, tables="deferred")
    assert not m.table_exchange


def test_train_step_rejects_unknown_modes():
    from gpt_pretraining_step_decoder_b200 import dp
    with pytest.raises(ValueError):
        dp.train_step(None, [], 1e-3, tables="striped")
    with pytest.raises(ValueError):
        dp.train_step(None, [], 1e-3, dense="zero3")


# --------------------------------------------------------------------------- row-sharded table exchange
def _sharded_rank_main(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist
    import gpt_pretraining_step_decoder_b200 as g
    from gpt_pretraining_step_decoder_b200 import dp
    from synthetic import init_params

    g.ngram_sparse_update = _oracle_sparse_update
    g.ngram_sparse_update_workspace_bytes = lambda n, d: 1
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        cfg = dict(_table_cfg(), lr_mult_table=0.5)
        m = _OracleModel(cfg, init_params(cfg, seed=3))
        batches = [_batch(cfg, dp.rank_stream_seed(cfg["seed"], rank) + 7 * s) for s in range(2)]
        dp.train_step(m, batches, 2e-2, tables="sharded")
        flat = torch.from_numpy(np.concatenate([m.P[t].reshape(-1) for t in ("hv", "hx")] +
                                               [m.S[t] for t in ("hv", "hx")]))
        reps = [torch.empty_like(flat) for _ in range(world)]
        dist.all_gather(reps, flat)
        if rank == 0:
            np.save(os.path.join(out_dir, "tables.npy"), torch.stack(reps).numpy())
            np.save(os.path.join(out_dir, "calls.npy"), np.array(m.calls))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_row_sharded_table_exchange_equals_joint_batch_update(tmp_path, world):
    """tables="sharded": every row's gradient goes to its owner (row mod
    world), the owner updates its rows over the pairs in rank order, the
    updated rows are gathered back: replicas bit-identical and equal, bit
    for bit, to one process updating per micro-batch over the joint batch."""
    import torch.multiprocessing as mp
    from gpt_pretraining_step_decoder_b200 import dp
    from oracle import optim
    from synthetic import init_params

    mp.spawn(_sharded_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    reps = np.load(tmp_path / "tables.npy")
    for r in range(1, world):
        np.testing.assert_array_equal(reps[0], reps[r])
    cfg = dict(_table_cfg(), lr_mult_table=0.5)
    P = {k: np.array(v, dtype=np.float64) for k, v in init_params(cfg, seed=3).items()}
    S = {t: np.zeros(P[t].shape[0]) for t in ("hx", "hv")}
    joint = dict(cfg, micro_batch=cfg["micro_batch"] * world)
    for s in range(2):
        parts = [_batch(cfg, dp.rank_stream_seed(cfg["seed"], r) + 7 * s) for r in range(world)]
        rx, gx0, rv, gv = _table_grads(joint, P, np.concatenate([p[0] for p in parts]),
                                       np.concatenate([p[1] for p in parts]))
        for t, rows, g in (("hv", rv, gv), ("hx", rx, gx0)):
            P[t], S[t], _ = optim.table_update(P[t], S[t], rows, g, 2e-2 * 0.5, cfg["table_beta"],
                                               cfg["table_eps"])
    ref = np.concatenate([P[t].reshape(-1) for t in ("hv", "hx")] + [S[t] for t in ("hv", "hx")])
    np.testing.assert_allclose(reps[0], ref, rtol=1e-12, atol=1e-15)


# --------------------------------------------------------------------------- sharded dense optimizer step
class _FlatOracleModel:
    """The slice of `Model` the dense paths of dp.train_step use, over flat
    fp64 buffers with the oracle's forward/backward and AdamW (group learning
    rates by position: embedding, then head, then matrices)."""

    def __init__(self, cfg, params):
        import types
        import torch
        from synthetic import param_shapes
        self.torch, self.w, self.stream = torch, cfg, None
        self.cfg = types.SimpleNamespace(x0_rows=0, v_rows=0)
        self.table_exchange = False
        self.names = [k for k in param_shapes(cfg) if k not in ("hx", "hv")]
        self.shapes = {k: np.asarray(params[k]).shape for k in self.names}
        sizes = [int(np.prod(self.shapes[k])) for k in self.names]
        self.offs = np.concatenate([[0], np.cumsum(sizes)])
        self.P = torch.from_numpy(np.concatenate([np.asarray(params[k], np.float64).reshape(-1) for k in self.names]))
        self.G, self.M, self.V = (torch.zeros_like(self.P) for _ in range(3))
        self.e_end = int(self.offs[1])
        self.h_end = int(self.offs[2]) if "lm_head" in self.names else self.e_end
        self.t = 0

    def _dict(self):
        return {k: self.P[self.offs[i]:self.offs[i + 1]].numpy().reshape(self.shapes[k])
                for i, k in enumerate(self.names)}

    def forward_loss(self, tok, tgt):
        from oracle import model
        self.cache = model.forward(self.w, self._dict(), tok, tgt)[2]

    def backward(self, lr):
        from oracle import model
        G, _, _ = model.backward(self.w, self._dict(), self.cache)
        self.G += self.torch.from_numpy(np.concatenate([G[k].reshape(-1) for k in self.names]))

    def flat_grad(self):
        return self.G

    def flat_param(self):
        return self.P

    def params_changed(self):
        pass

    def grad_sumsq(self, lo, hi, out):
        out[0] = float((self.G[lo:hi] ** 2).sum())

    def _adamw(self, lr, lo, hi, coef):
        from oracle import optim
        w = self.w
        bounds = sorted({lo, hi, min(max(self.e_end, lo), hi), min(max(self.h_end, lo), hi)})
        for a, b in zip(bounds[:-1], bounds[1:]):
            mult = w["lr_mult_embed"] if a < self.e_end else (w["lr_mult_head"] if a < self.h_end
                                                               else w["lr_mult_matrix"])
            p, m, v = optim.adamw(self.P[a:b].numpy(), self.G[a:b].numpy() * coef, self.M[a:b].numpy(),
                                  self.V[a:b].numpy(), self.t, lr * mult, w["adam_b1"], w["adam_b2"],
                                  w["adam_eps"], w["weight_decay"])
            self.P[a:b], self.M[a:b], self.V[a:b] = (self.torch.from_numpy(np.asarray(z)) for z in (p, m, v))

    def optimizer_step(self, lr):
        from oracle import optim
        self.t += 1
        self._adamw(lr, 0, self.P.numel(), optim.clip_coef([self.G.numpy()], self.w["grad_clip"]))
        self.G.zero_()

    def optimizer_step_range(self, lr, lo, hi, sumsq):
        self.t += 1
        coef = 1.0
        if self.w["grad_clip"] > 0:
            coef = min(1.0, self.w["grad_clip"] / (float(np.sqrt(float(sumsq[0]))) + 1e-6))
        self._adamw(lr, lo, hi, coef)
        self.G.zero_()


def _dense_cfg():
    from synthetic import workload
    return workload("tiny_fp32", x0_rows=0, n_layer=1, seq_len=16, micro_batch=2, vocab=96, tie_embeddings=0,
                    grad_clip=0.05, lr_mult_head=0.5, lr_mult_embed=2.0)


def _dense_rank_main(rank, world, port, out_dir, dense):
    import torch
    import torch.distributed as dist
    from gpt_pretraining_step_decoder_b200 import dp
    from synthetic import init_params
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        cfg = _dense_cfg()
        m = _FlatOracleModel(cfg, init_params(cfg, seed=5))
        for step in range(2):
            batches = [_batch(cfg, dp.rank_stream_seed(cfg["seed"], rank) + 11 * step + s) for s in range(2)]
            dp.train_step(m, batches, 1e-2, dense=dense)
        reps = [torch.empty_like(m.P) for _ in range(world)]
        dist.all_gather(reps, m.P)
        if rank == 0:
            np.save(os.path.join(out_dir, f"params_{dense}.npy"), torch.stack(reps).numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_dense_step_equals_replicated_step(tmp_path, world):
    """dense="sharded" (reduce-scatter, AdamW on each rank's slice with the
    all-reduced clip norm, all-gather) gives the replicated all-reduce +
    AdamW result on every rank: two optimizer steps with clipping active and
    three learning-rate groups, a slice boundary inside a tensor."""
    import torch.multiprocessing as mp
    for dense in ("replicated", "sharded"):
        mp.spawn(_dense_rank_main, args=(world, _free_port(), str(tmp_path), dense), nprocs=world, join=True)
    rep = np.load(tmp_path / "params_replicated.npy")
    sh = np.load(tmp_path / "params_sharded.npy")
    for r in range(world):
        np.testing.assert_array_equal(sh[r], sh[0])
    np.testing.assert_allclose(sh[0], rep[0], rtol=1e-10, atol=1e-13)
