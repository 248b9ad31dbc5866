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
    """In-place mean of a flat gradient tensor over the ranks of `group`."""
    world = dist.get_world_size(group)
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


def exchange_tables(model, lr, group=None):
    """After a backward in table exchange mode: gather every rank's table
    gradients and apply the identical sparse update to this rank's replicas
    (value table, then x0 table, the order of the inline update)."""
    import gpt_pretraining_step_decoder_b200 as g
    cfg = model.cfg
    lr_t = lr * cfg.lr_mult_table
    for table, rows_name, grad_name, n_rows in (("hv", "rows_v", "table_grad_v", cfg.v_rows),
                                                ("hx", "rows_x", "table_grad_x", cfg.x0_rows)):
        if not n_rows:
            continue
        rows, grad = gather_table_grads(model.tensor(rows_name, g.KIND_ACT), model.tensor(grad_name, g.KIND_ACT),
                                        group)
        W = model.tensor(table, g.KIND_PARAM)
        state = model.tensor(table, g.KIND_ROW_STATE)
        n, d = grad.shape
        ws_bytes = g.ngram_sparse_update_workspace_bytes(n, d)
        ws = getattr(model, "_table_ws", None)
        if ws is None or ws.numel() < ws_bytes:
            ws = model.torch.empty(ws_bytes, dtype=model.torch.uint8, device=grad.device)
            model._table_ws = ws
        g.ngram_sparse_update(W, state, n_rows, d, cfg.dtype, rows, grad, n, lr_t, cfg.table_beta, cfg.table_eps,
                              None, None, ws, ws.numel(), model.stream)


def train_step(model, micro_batches, lr, group=None, loss_host=None):
    """One data-parallel optimizer step of a `Model`: forward + backward of
    every (tokens, targets) pair on this rank (with the tables exchanged
    after each backward when there are several ranks), gradient average,
    AdamW."""
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    exchange = world > 1 and (model.cfg.x0_rows or model.cfg.v_rows)
    if exchange:
        model.set_table_exchange(True)
    for tok, tgt in micro_batches:
        model.forward_loss(tok, tgt)
        model.backward(lr)
        if exchange:
            exchange_tables(model, lr, group)
        if loss_host is not None:
            loss_host.copy_(model.loss, non_blocking=True)
    average_gradients(model.flat_grad(), group)
    model.optimizer_step(lr)
