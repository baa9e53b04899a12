"""One workload's routing step, repeated: the launch that profilers capture.

Builds a layer with the workload's seeded router weights (seed 0, as the
benchmark draws them) and calls ``moe_route`` on its seeded tokens ``--reps``
times. Under a profiler, skip the first call's launch and capture a later one.

    python -m sparse_mixture_experts_12_b200.profile_route --workload switch --reps 3
"""
from __future__ import annotations

import argparse
import json

import torch

from . import binding as B
from . import synth


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--workload", default="switch", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--reps", type=int, default=3)
    args = ap.parse_args(argv)
    wl = synth.WORKLOADS[args.workload]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    inp = synth.generate(wl, seed=0, with_weights=False)
    params = {k: None for k in ("w1", "w3", "w2", "b1", "b2", "ws_gate", "ws_up", "ws_down")}
    params.update(w_router=inp["w_router"], b_router=inp["b_router"],
                  logit_bias=inp["logit_bias"])
    layer = B.MoELayer(wl, params, dev)
    x = inp["x"].to(dev)
    T, E, k = wl.T, wl.n_experts, wl.top_k
    logits = torch.empty((T, E), dtype=torch.float32, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    gate = torch.empty((T, k), dtype=torch.float32, device=dev)
    for _ in range(args.reps):
        layer.route(x, logits, idx, gate)
    torch.cuda.synchronize()
    code, info = layer.last_device_error()
    print(json.dumps({"workload": wl.name, "reps": args.reps, "device_error": [code, info]}))
    return 0 if code == 0 else 1


if __name__ == "__main__":
    raise SystemExit(main())
