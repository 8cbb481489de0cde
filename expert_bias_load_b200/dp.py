"""Data-parallel router step: each rank routes its own tokens, the per-expert
loads are summed over all ranks, and every rank applies the same bias update.

"SMEBU Load Balancing" defines n_i as the tokens routed to expert i in the
optimizer step; with the batch split over ranks that is the sum of the ranks'
local loads, so the one exchange the step needs is an all-reduce (sum) of the
int32 load vector (N_r values, 1 KiB at N_r = 256) between the router pass and
the bias update.  Because the update is deterministic, bias and momentum stay
bit-identical on every rank without any broadcast.

The compute callables default to the CUDA library; the collective goes through
torch.distributed (NCCL on GPUs).  Tests swap the callables for CPU ones to
check the exchange logic on `gloo` ranks.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def global_loads(counts: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the per-expert loads over the ranks of `group`, in place."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(counts, op=dist.ReduceOp.SUM, group=group)
    return counts


class DataParallelRouterStep:
    """One optimizer step of the router with the bias update on global loads.

    route(hidden, bias, counts) -> anything      accumulates local loads into counts
    update(counts, bias, momentum, maxvio)       bias update from global loads; resets counts

    stream: the CUDA stream route and update run on, if not torch's current
    one; the all-reduce is then issued on it too, so the three stay ordered.
    """

    def __init__(self, route, update, group=None, stream=None):
        self.route = route
        self.update = update
        self.group = group
        self.stream = stream

    def __call__(self, hidden, bias, momentum, counts, maxvio=None):
        out = self.route(hidden, bias, counts)
        if self.stream is not None:
            with torch.cuda.stream(self.stream):
                global_loads(counts, self.group)
        else:
            global_loads(counts, self.group)
        self.update(counts, bias, momentum, maxvio)
        return out


def cuda_step(W_router, K, lam=5e-4, beta=0.5, kappa=2.0, group=None, stream=None):
    """The step on the CUDA library: router_forward (GEMM mode) on this rank's
    hidden states, an all-reduce of the loads, smebu_step with reset_counts so
    the next step starts at 0."""
    import expert_bias_load_b200 as ebl

    def route(hidden, bias, counts):
        return ebl.router_forward(hidden, W_router, bias, K, counts, stream=stream)

    def update(counts, bias, momentum, maxvio):
        ebl.smebu_step(counts, bias, momentum, lam, beta, kappa, reset_counts=True, maxvio=maxvio, stream=stream)

    return DataParallelRouterStep(route, update, group, stream)


def cuda_logits_step(K, lam=5e-4, beta=0.5, kappa=2.0, group=None, stream=None):
    """The same step fed with this rank's precomputed fp32 router logits
    (router_forward_logits, the bit-exact mode): the global loads, and with
    them bias and momentum, equal those of one process that routes the
    concatenated batch."""
    import expert_bias_load_b200 as ebl

    def route(logits, bias, counts):
        return ebl.router_forward_logits(logits, bias, K, counts, stream=stream)

    def update(counts, bias, momentum, maxvio):
        ebl.smebu_step(counts, bias, momentum, lam, beta, kappa, reset_counts=True, maxvio=maxvio, stream=stream)

    return DataParallelRouterStep(route, update, group, stream)
