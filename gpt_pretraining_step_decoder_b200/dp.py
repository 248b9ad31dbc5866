"""Data parallelism: one process per GPU, a full replica of the dense weights
on every rank.

Each rank runs forward and backward on its own micro-batches (its own slice
of the token stream), the fp32 dense gradient is averaged across ranks with
one all-reduce (NCCL over NVLink / NVSwitch on GPUs, gloo on CPU), and every
rank then takes the identical AdamW step, so the replicas stay equal.  The
loss of a rank is the mean over its own valid targets; the average of the
rank gradients equals the gradient of the global mean when every rank has the
same number of valid targets (the synthetic streams have none ignored).

The bigram tables are replicas too.  With more than one rank the model's
backward leaves each position's table gradient in place (table exchange
mode); every rank gathers the (row, gradient) pairs of all ranks in rank order
and applies one identical sparse update to its replica, so the tables stay
equal and each update is the one a single process would make over all ranks'
positions together (the gradients scaled by 1/world like the dense ones).

Two sharded forms cut the traffic and the per-rank optimizer work:
  * dense="sharded": the flat gradient is reduce-scattered (each rank gets
    the rank average of its 1/world slice), each rank takes the AdamW step of
    its slice only (the global clip norm from an all-reduced sum of squares),
    and the updated fp32 slices are all-gathered (ZeRO-1 style sharding of
    the optimizer state's work; every rank still holds the whole state);
  * tables="sharded": row r of a table belongs to rank r mod world.  Every
    rank sends each position's (row, gradient) pair to the row's owner
    (all-to-all), each owner applies the sparse update to its own rows over
    the pairs it received (in rank order, so each row's sum runs over the
    same positions in the same order as a single process over the joint
    batch), and the owners' updated rows and row states are all-gathered
    into every replica.  Per rank this moves about N*d*4 bytes of gradient
    instead of world*N*d*4.
"""

import torch
import torch.distributed as dist


def rank_stream_seed(seed, rank):
    """Seed of the token stream that rank `rank` trains on."""
    return seed + 1000 * rank


def average_gradients(flat_grad, group=None):
    """In-place mean of a flat gradient tensor over the ranks of `group` (a
    no-op in a process without a process group)."""
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    if world > 1:
        dist.all_reduce(flat_grad, op=dist.ReduceOp.SUM, group=group)
        flat_grad.mul_(1.0 / world)
    return flat_grad


def gather_table_grads(rows, grad, group=None):
    """All ranks' (row, gradient) pairs of one table, concatenated in rank
    order: rows [world * n] int32 and grad [world * n, d] scaled by 1/world
    (each rank's loss is the mean over its own positions).  Every rank holds
    the same n positions."""
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rows = rows.reshape(-1)
    grad = grad.reshape(rows.numel(), -1)
    if world == 1:
        return rows, grad
    all_rows = [torch.empty_like(rows) for _ in range(world)]
    all_grad = [torch.empty_like(grad) for _ in range(world)]
    dist.all_gather(all_rows, rows, group=group)
    dist.all_gather(all_grad, grad, group=group)
    return torch.cat(all_rows), torch.cat(all_grad).mul_(1.0 / world)


# (table, rows buffer, per-position gradient buffer, row-count field), in the
# order the inline update takes them: value table, then x0 table
_TABLES = (("hv", "rows_v", "table_grad_v", "v_rows"), ("hx", "rows_x", "table_grad_x", "x0_rows"))


def _apply_table_update(model, table, n_rows, rows, grad, lr):
    """One ngram_sparse_update of the model's replica of `table` over the
    (row, gradient) pairs given, with the table learning-rate multiplier."""
    import gpt_pretraining_step_decoder_b200 as g
    cfg = model.cfg
    W = model.tensor(table, g.KIND_PARAM)
    state = model.tensor(table, g.KIND_ROW_STATE)
    n, d = grad.shape
    ws_bytes = g.ngram_sparse_update_workspace_bytes(n, d)
    ws = getattr(model, "_table_ws", None)
    if ws is None or ws.numel() < ws_bytes:
        ws = model.torch.empty(ws_bytes, dtype=model.torch.uint8, device=grad.device)
        model._table_ws = ws
    g.ngram_sparse_update(W, state, n_rows, d, cfg.dtype, rows, grad, n, lr * cfg.lr_mult_table, cfg.table_beta,
                          cfg.table_eps, None, None, ws, ws.numel(), model.stream)


def _table_grads(model, group):
    """[(table, n_rows, rows, grad)] of every present table after a backward in
    exchange mode, gathered over the ranks of `group`."""
    import gpt_pretraining_step_decoder_b200 as g
    out = []
    for table, rows_name, grad_name, rows_field in _TABLES:
        n_rows = getattr(model.cfg, rows_field)
        if n_rows:
            rows, grad = gather_table_grads(model.tensor(rows_name, g.KIND_ACT),
                                            model.tensor(grad_name, g.KIND_ACT), group)
            out.append((table, n_rows, rows, grad))
    return out


def exchange_tables(model, lr, group=None):
    """After a backward in table exchange mode: gather every rank's table
    gradients and apply the identical sparse update to this rank's replicas
    (value table, then x0 table, the order of the inline update)."""
    for table, n_rows, rows, grad in _table_grads(model, group):
        _apply_table_update(model, table, n_rows, rows, grad, lr)


def _shard(n, world, rank):
    """[lo, hi) of rank's slice of n elements: equal slices, multiples of 4."""
    per = -(-n // world)
    per = -(-per // 4) * 4
    lo = min(n, rank * per)
    return lo, min(n, lo + per), per


def sharded_optimizer_step(model, lr, group=None):
    """Reduce-scatter of the flat dense gradient (rank average), AdamW on this
    rank's slice, all-gather of the updated fp32 slices, bf16 copies refreshed."""
    torch = model.torch
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    flat = model.flat_grad()
    n = flat.numel()
    lo, hi, per = _shard(n, world, rank)
    if world > 1:
        buf = torch.zeros(world * per, dtype=flat.dtype, device=flat.device)
        buf[:n].copy_(flat)
        mine = torch.empty(per, dtype=flat.dtype, device=flat.device)
        dist.reduce_scatter_tensor(mine, buf, op=dist.ReduceOp.SUM, group=group)
        flat[lo:hi].copy_(mine[:hi - lo].mul_(1.0 / world))
    sumsq = torch.zeros(1, dtype=torch.float64, device=flat.device)
    model.grad_sumsq(lo, hi, sumsq)
    if world > 1:
        dist.all_reduce(sumsq, op=dist.ReduceOp.SUM, group=group)
    model.optimizer_step_range(lr, lo, hi, sumsq)
    if world > 1:
        params = model.flat_param()
        mine = torch.zeros(per, dtype=params.dtype, device=params.device)
        mine[:hi - lo].copy_(params[lo:hi])
        full = torch.empty(world * per, dtype=params.dtype, device=params.device)
        dist.all_gather_into_tensor(full, mine, group=group)
        params.copy_(full[:n])
        model.params_changed()


def _all_to_all_uneven(x, send_counts, group):
    """Rows of x grouped by destination (send_counts[r] rows to rank r); returns
    the rows received, grouped by source rank in rank order."""
    import torch as _t
    counts = _t.tensor(send_counts, dtype=_t.int64, device=x.device)
    recv = _t.empty_like(counts)
    dist.all_to_all_single(recv, counts, group=group)
    recv_counts = recv.tolist()
    out = x.new_empty((sum(recv_counts),) + tuple(x.shape[1:]))
    dist.all_to_all_single(out, x.contiguous(), output_split_sizes=recv_counts, input_split_sizes=list(send_counts),
                           group=group)
    return out


def _all_gather_uneven(x, group):
    """All ranks' rows of x concatenated in rank order (row counts may differ)."""
    import torch as _t
    world = dist.get_world_size(group)
    k = _t.tensor([x.shape[0]], dtype=_t.int64, device=x.device)
    ks = [_t.empty_like(k) for _ in range(world)]
    dist.all_gather(ks, k, group=group)
    ks = [int(v.item()) for v in ks]
    mx = max(ks)
    pad = x.new_zeros((mx,) + tuple(x.shape[1:]))
    pad[:x.shape[0]] = x
    parts = [x.new_empty((mx,) + tuple(x.shape[1:])) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return _t.cat([p[:c] for p, c in zip(parts, ks)])


def exchange_tables_sharded(model, lr, group=None):
    """After a backward in table exchange mode: the row-sharded exchange (row
    r owned by rank r mod world), see the module notes.  Value table, then x0
    table, like the inline update."""
    import gpt_pretraining_step_decoder_b200 as g
    torch = model.torch
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    for table, rows_name, grad_name, rows_field in _TABLES:
        n_rows = getattr(model.cfg, rows_field)
        if not n_rows:
            continue
        rows = model.tensor(rows_name, g.KIND_ACT).reshape(-1)
        grad = model.tensor(grad_name, g.KIND_ACT)
        grad = grad.reshape(rows.numel(), -1)
        owner = rows.long() % world
        order = torch.sort(owner, stable=True).indices
        send = torch.bincount(owner, minlength=world).tolist()
        r_rows = rows[order]
        r_grad = grad[order]
        if world > 1:
            r_rows = _all_to_all_uneven(r_rows, send, group)
            r_grad = _all_to_all_uneven(r_grad, send, group).mul_(1.0 / world)
        W = model.tensor(table, g.KIND_PARAM)
        state = model.tensor(table, g.KIND_ROW_STATE).reshape(-1)
        n, d = r_grad.shape
        upd = torch.empty(max(n, 1), dtype=torch.int32, device=rows.device)
        n_upd = torch.zeros(1, dtype=torch.int32, device=rows.device)
        if n:
            ws_bytes = g.ngram_sparse_update_workspace_bytes(n, d)
            ws = getattr(model, "_table_ws", None)
            if ws is None or ws.numel() < ws_bytes:
                ws = torch.empty(ws_bytes, dtype=torch.uint8, device=rows.device)
                model._table_ws = ws
            g.ngram_sparse_update(W, state, n_rows, d, model.cfg.dtype, r_rows, r_grad, n,
                                  lr * model.cfg.lr_mult_table, model.cfg.table_beta, model.cfg.table_eps,
                                  upd, n_upd, ws, ws.numel(), model.stream)
        if world > 1:
            k = int(n_upd.item())
            mine = upd[:k].long()
            all_rows = _all_gather_uneven(mine, group)
            all_vals = _all_gather_uneven(W[mine], group)
            all_state = _all_gather_uneven(state[mine], group)
            W[all_rows] = all_vals
            state[all_rows] = all_state


def train_step(model, micro_batches, lr, group=None, loss_host=None, tables="inline", dense="replicated"):
    """One data-parallel optimizer step of a `Model`: forward + backward of
    every (tokens, targets) pair on this rank, gradient average, AdamW.

    tables="inline": the bigram tables are updated after every micro-batch
    (inside backward on one rank; exchanged after each backward when there
    are several).  tables="deferred": every micro-batch's (row, gradient)
    pairs are collected (gathered over the ranks) and each table takes one
    sparse update over all of them at the optimizer step, so every forward of
    the step sees the same tables.  tables="sharded": after every backward,
    the row-sharded exchange (each row's gradient to its owner, the owners'
    updated rows gathered back).  dense="sharded": reduce-scatter, AdamW on
    this rank's slice, all-gather (sharded_optimizer_step)."""
    if tables not in ("inline", "deferred", "sharded"):
        raise ValueError(f"tables must be 'inline', 'deferred' or 'sharded', not {tables!r}")
    if dense not in ("replicated", "sharded"):
        raise ValueError(f"dense must be 'replicated' or 'sharded', not {dense!r}")
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    has_tables = bool(model.cfg.x0_rows or model.cfg.v_rows)
    deferred = has_tables and tables == "deferred"
    sharded_tables = has_tables and tables == "sharded"
    exchange = has_tables and (world > 1 or deferred or sharded_tables)
    was_exchange = model.table_exchange
    if exchange:
        model.set_table_exchange(True)
    try:
        pending = {}
        for tok, tgt in micro_batches:
            model.forward_loss(tok, tgt)
            model.backward(lr)
            if deferred:
                for table, n_rows, rows, grad in _table_grads(model, group):
                    # copies: the buffers are rewritten by the next forward
                    pending.setdefault(table, (n_rows, [], []))[1].append(rows.clone())
                    pending[table][2].append(grad.clone())
            elif sharded_tables:
                exchange_tables_sharded(model, lr, group)
            elif exchange:
                exchange_tables(model, lr, group)
            if loss_host is not None:
                loss_host.copy_(model.loss, non_blocking=True)
        for table, *_ in _TABLES:
            if table in pending:
                n_rows, rows, grads = pending[table]
                _apply_table_update(model, table, n_rows, model.torch.cat(rows), model.torch.cat(grads), lr)
        if dense == "sharded":
            sharded_optimizer_step(model, lr, group)
        else:
            average_gradients(model.flat_grad(), group)
            model.optimizer_step(lr)
    finally:
        # a later plain backward_step must update the tables inline again
        if exchange and not was_exchange:
            model.set_table_exchange(False)
