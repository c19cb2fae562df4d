"""Host-side plumbing of the multi-GPU run: one process per GPU, each with its own batch.

Every (b, h) scan is independent, so a run over N GPUs gives each rank B rows of the global batch
of N*B rows (weak scaling) and exchanges nothing on the data path. The one exchange is dW0: the
persistent weight W0 is shared over the batch, so its gradient sums over all N*B rows and the
per-rank sums are all-reduced. Time is measured on each rank's device and the job time is the
maximum over ranks.

These helpers only move tensors through ``torch.distributed``; they work with any backend (NCCL
on GPUs, gloo on the CPU in the tests).
"""

from . import inputs

RANK_SEED_STRIDE = 1000


def rank_seed(config_index: int, rank: int) -> int:
    """Seed of the generator for this rank's shard of a workload's global batch."""
    return inputs.SEED_BASE + config_index + RANK_SEED_STRIDE * rank


def global_batch(batch_per_rank: int, world: int) -> int:
    return batch_per_rank * world


def allreduce_dW0(dW0, dist, group=None):
    """Sum the per-rank dW0 [H, d_out, d_in] over ranks, in place."""
    if dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(dW0, op=dist.ReduceOp.SUM, group=group)
    return dW0


def max_over_ranks(ms: float, dist, device="cpu", group=None) -> float:
    """The slowest rank's time: the job is done when the last rank is."""
    if not (dist.is_initialized() and dist.get_world_size(group) > 1):
        return float(ms)
    import torch
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def weak_scaling_value(tokens_per_rank: int, world: int, steps: int, ms: float) -> float:
    """Whole-job throughput: tokens all ranks processed over the slowest rank's time."""
    return tokens_per_rank * world * steps / (ms * 1e-3)
