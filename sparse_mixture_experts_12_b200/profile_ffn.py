"""One workload's routed expert-FFN call, repeated: the launch that profilers capture.

Draws the workload's seeded inputs (seed 0, as the benchmark does), routes and
permutes them through the library, then calls ``moe_expert_ffn`` ``--reps``
times on the permuted rows. Under a profiler, skip the first call's launches
(cold caches, first-use setup) and capture the second call's.

    python -m sparse_mixture_experts_12_b200.profile_ffn --workload mixtral_prefill --reps 2
"""
from __future__ import annotations

import argparse
import json

import torch

from . import binding as B
from . import synth


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--workload", default="mixtral_prefill", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--reps", type=int, default=2)
    args = ap.parse_args(argv)
    wl = synth.WORKLOADS[args.workload]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    inp = synth.generate(wl, seed=0)
    layer = B.MoELayer(wl, inp, dev)
    x = inp["x"].to(dev)
    T, E, k, d = wl.T, wl.n_experts, wl.top_k, wl.d_model
    if wl.routing == synth.ROUTING_EXPERT_CHOICE:  # each expert's C picked rows
        C = int(wl.capacity_factor * T // E)
        logits = torch.empty((T, E), dtype=torch.float32, device=dev)
        idx = torch.empty((E, C), dtype=torch.int32, device=dev)
        score = torch.empty((E, C), dtype=torch.float32, device=dev)
        layer.route_expert_choice(x, logits, idx, score)
        xp = x[idx.reshape(-1).long()].contiguous()
        off = (torch.arange(E + 1, dtype=torch.int32, device=dev) * C).contiguous()
    else:
        taps = layer.new_taps()
        layer.route(x, taps["logits"], taps["topk_idx"], taps["topk_gate"])
        xp = torch.empty((T * k, d), dtype=wl.torch_dtype, device=dev)
        off = torch.empty(E + 1, dtype=torch.int32, device=dev)
        layer.permute(x, taps["topk_idx"], taps["counts"], off, taps["perm"], taps["inv"], xp)
    yp = torch.empty_like(xp)
    torch.cuda.synchronize()
    for _ in range(args.reps):
        layer.expert_ffn(xp, off, yp)
    torch.cuda.synchronize()
    code, info = layer.last_device_error()
    print(json.dumps({"workload": wl.name, "rows": int(off[-1]), "reps": args.reps,
                      "device_error": [code, info]}))
    return 0 if code == 0 else 1


if __name__ == "__main__":
    raise SystemExit(main())
