"""Data parallelism: one process per GPU, a full replica of the dense weights
on every rank.

Each rank runs forward and backward on its own micro-batches (its own slice
of the token stream), the fp32 dense gradient is averaged across ranks with
one all-reduce (NCCL over NVLink / NVSwitch on GPUs, gloo on CPU), and every
rank then takes the identical AdamW step, so the replicas stay equal.  The
loss of a rank is the mean over its own valid targets; the average of the
rank gradients equals the gradient of the global mean when every rank has the
same number of valid targets (the synthetic streams have none ignored).

The bigram-table updates run inline in each rank's backward on that rank's
positions only: the tables are rank-local here, not an exchanged replica.
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


def train_step(model, micro_batches, lr, group=None, loss_host=None):
    """One data-parallel optimizer step of a `Model`: forward + backward of
    every (tokens, targets) pair on this rank, gradient average, AdamW."""
    for tok, tgt in micro_batches:
        model.forward_loss(tok, tgt)
        model.backward(lr)
        if loss_host is not None:
            loss_host.copy_(model.loss, non_blocking=True)
    average_gradients(model.flat_grad(), group)
    model.optimizer_step(lr)
