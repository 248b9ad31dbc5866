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


def train_step(model, micro_batches, lr, group=None, loss_host=None, tables="inline"):
    """One data-parallel optimizer step of a `Model`: forward + backward of
    every (tokens, targets) pair on this rank, gradient average, AdamW.

    tables="inline": the bigram tables are updated after every micro-batch
    (inside backward on one rank; exchanged after each backward when there
    are several).  tables="deferred": every micro-batch's (row, gradient)
    pairs are collected (gathered over the ranks) and each table takes one
    sparse update over all of them at the optimizer step, so every forward of
    the step sees the same tables."""
    if tables not in ("inline", "deferred"):
        raise ValueError(f"tables must be 'inline' or 'deferred', not {tables!r}")
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    has_tables = bool(model.cfg.x0_rows or model.cfg.v_rows)
    deferred = has_tables and tables == "deferred"
    exchange = has_tables and (world > 1 or deferred)
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
            elif exchange:
                exchange_tables(model, lr, group)
            if loss_host is not None:
                loss_host.copy_(model.loss, non_blocking=True)
        for table, *_ in _TABLES:
            if table in pending:
                n_rows, rows, grads = pending[table]
                _apply_table_update(model, table, n_rows, model.torch.cat(rows), model.torch.cat(grads), lr)
        average_gradients(model.flat_grad(), group)
        model.optimizer_step(lr)
    finally:
        # a later plain backward_step must update the tables inline again
        if exchange and not was_exchange:
            model.set_table_exchange(False)
