"""One MoE batch sharded by tokens over the ranks of a process group.

Each rank holds a consecutive slice of the batch's tokens (rank 0 first) and a
full copy of the weights. Tokens are independent given the routing except for
two steps, which need one small collective each (NCCL over NVLink on GPUs):

* the capacity drop (youngju.dev (zh) "SwitchRouter") ranks each expert's pairs in
  token order over the whole batch: the ranks all-gather their pre-drop counts
  per expert [E] int32, and each rank keeps for expert e at most the capacity
  left by the ranks before it;
* the load-balancing statistics are means over the whole batch: the ranks add
  their fp64 sums [1 + 2E] with a sum all-reduce.

Every arithmetic step runs in the library's kernels (``moe_route_shard``,
``moe_forward_shard``, ``moe_aux_finalize``); this module only orders the calls and
the two collectives. ``forward_sharded`` takes the per-rank steps as an object, so
the same exchange logic drives the CUDA layer and any other implementation of the
three steps.
"""
from __future__ import annotations

from typing import Optional

import torch
import torch.distributed as dist

from . import binding as B
from . import synth


def shard_bounds(n_tokens_total: int, n_shards: int):
    """Consecutive token slices [(start, stop)] of a batch over n_shards ranks, the
    first n_tokens_total % n_shards slices one token longer."""
    base, extra = divmod(n_tokens_total, n_shards)
    out, a = [], 0
    for r in range(n_shards):
        b = a + base + (1 if r < extra else 0)
        out.append((a, b))
        a = b
    return out


def check_placement(shard: int, n_shards: int, group=None, caller_exchanges: bool = False):
    """A shard's place must be its rank in the process group. Without a group only
    the one-shard layout is valid: the other shards' counts would never arrive, and
    the capacity left to this shard could not be computed. A caller that gathers
    the counts itself (caller_exchanges) may place shards freely: it then passes
    every shard's counts to forward_shard, whose check guards the library's read."""
    if not 0 <= shard < n_shards:
        raise ValueError(f"shard {shard} is not one of {n_shards} shards")
    if caller_exchanges:
        return
    if not dist.is_initialized():
        if n_shards != 1:
            raise ValueError(f"{n_shards} shards need a process group of {n_shards} ranks; "
                             "none is initialised")
        return
    if dist.get_world_size(group) != n_shards or dist.get_rank(group) != shard:
        raise ValueError("shard / n_shards must be this rank's place in the process group")


def check_counts_all(counts_all: torch.Tensor, n_shards: int, n_experts: int, device):
    """counts_all must be every shard's pre-drop counts, [n_shards, E] int32 on the
    layer's device: the library reads n_shards * E of them through a raw pointer."""
    if tuple(counts_all.shape) != (n_shards, n_experts):
        raise ValueError(f"counts_all has shape {tuple(counts_all.shape)}, "
                         f"expected ({n_shards}, {n_experts})")
    if counts_all.dtype != torch.int32:
        raise ValueError(f"counts_all must be int32, not {counts_all.dtype}")
    if not _same_device(counts_all.device, device):
        raise ValueError(f"counts_all is on {counts_all.device}, the layer on {device}")


def _same_device(a, b) -> bool:
    a, b = torch.device(a), torch.device(b)
    if a.type != b.type:
        return False
    if a.type != "cuda":
        return True
    cur = torch.cuda.current_device()
    return (cur if a.index is None else a.index) == (cur if b.index is None else b.index)


def forward_sharded(steps, x, n_experts: int, group=None, want_aux: bool = False, y=None):
    """One rank's part of the layer over a token-sharded batch.

    ``steps`` provides ``route_shard(x, want_aux) -> (counts [E] int32, part or None,
    routed)``, ``forward_shard(x, routed, counts_all [W, E], y) -> y`` and
    ``aux_finalize(part) -> aux``. Every rank takes the same collectives in the same
    order: the all-gather of the counts, then (with ``want_aux``) the all-reduce of
    the sums. Returns (y, aux or None)."""
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    counts, part, routed = steps.route_shard(x, want_aux)
    if world == 1:
        counts_all = counts.reshape(1, n_experts)
    else:
        counts_all = counts.new_empty((world, n_experts))
        dist.all_gather(list(counts_all.unbind(0)), counts, group=group)
        if want_aux:
            dist.all_reduce(part, op=dist.ReduceOp.SUM, group=group)
    y = steps.forward_shard(x, routed, counts_all, y)
    aux = steps.aux_finalize(part) if want_aux else None
    return y, aux


class ShardedMoELayer:
    """This rank's shard of a token-sharded MoE layer on the GPU.

    ``workload`` describes the whole batch (its T is the batch's token count);
    this rank runs ``shard_bounds(T, n_shards)[shard]`` of it."""

    def __init__(self, workload: synth.Workload, params: dict, shard: int, n_shards: int,
                 device="cuda", group=None, caller_exchanges: bool = False):
        """caller_exchanges: the caller gathers every shard's counts itself and calls
        route_shard / forward_shard / aux_finalize directly (forward, which runs the
        collectives over the process group, is then unavailable)."""
        check_placement(shard, n_shards, group, caller_exchanges)
        self.caller_exchanges = caller_exchanges
        self.n_tokens_total = workload.T
        self.shard, self.n_shards, self.group = shard, n_shards, group
        a, b = shard_bounds(workload.T, n_shards)[shard]
        self.rows = (a, b)
        self.local = workload.replace(T=b - a)
        self.layer = B.MoELayer(self.local, params, device)

    # the three per-rank steps of forward_sharded
    def route_shard(self, x, want_aux):
        L, E, k = self.layer, self.local.n_experts, self.local.top_k
        T, dev = self.local.T, L.device
        routed = {"topk_idx": torch.empty((T, k), dtype=torch.int32, device=dev),
                  "topk_gate": torch.empty((T, k), dtype=torch.float32, device=dev)}
        counts = torch.empty(E, dtype=torch.int32, device=dev)
        part = torch.empty(1 + 2 * E, dtype=torch.float64, device=dev) if want_aux else None
        L.route_shard(x, None, routed["topk_idx"], routed["topk_gate"], counts, part)
        return counts, part, routed

    def forward_shard(self, x, routed, counts_all, y=None):
        check_counts_all(counts_all, self.n_shards, self.local.n_experts, self.layer.device)
        counts_all = counts_all.contiguous()
        desc = B.MoeShard(n_tokens_total=self.n_tokens_total, n_shards=self.n_shards,
                          shard=self.shard, counts_all=counts_all.data_ptr())
        return self.layer.forward_shard(desc, x, routed, y)

    def aux_finalize(self, part):
        return self.layer.aux_finalize(self.n_tokens_total, part)

    def forward(self, x: torch.Tensor, y: Optional[torch.Tensor] = None, want_aux: bool = False):
        """x: this rank's tokens [T_shard, d] on the device. Returns (y, aux or None)."""
        if self.caller_exchanges:
            raise RuntimeError("a layer built with caller_exchanges=True has no process "
                               "group to exchange over; call its three steps directly")
        return forward_sharded(self, x, self.local.n_experts, self.group, want_aux, y)
