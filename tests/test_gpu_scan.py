"""The permute step's scan over several CTAs.

A warp scans each expert's per-tile counts, eight experts per CTA; the CTA that
draws the last ticket (an atomicInc on the third word of the workspace header,
wrapping at the grid size) lays out the experts. Checked here, through the whole
layer on the GPU: the counts, offsets and the drop rule against a plain histogram
of the layer's own routing indices (the capacity rule of youngju.dev (zh)
"SwitchRouter": the first cap pairs of each expert in token order are kept), for
expert counts that give one, two and many scan CTAs; the ticket word is zero again
after every call; a second call on the same workspace lays out the same way.
"""
import numpy as np
import pytest
import torch

from sparse_mixture_experts_12_b200 import binding as B
from sparse_mixture_experts_12_b200 import build as BUILD
from sparse_mixture_experts_12_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("the GPU tests need a CUDA device")
    BUILD.build()
    B.load()


def _ticket(layer) -> int:
    return int(layer.ws[:16].view(torch.int32)[2].item())


@pytest.mark.parametrize("E,k,T,cf", [
    (8, 2, 700, 0.0),      # one scan CTA
    (13, 2, 700, 1.0),     # two CTAs, capacity
    (130, 1, 3000, 1.25),  # 17 CTAs, capacity, skewed loads
    (256, 8, 257, 2.0),    # 32 CTAs, k = 8
], ids=["E8", "E13_cap", "E130_cap", "E256_k8"])
def test_scan_layout_and_ticket(E, k, T, cf):
    wl = synth.Workload(f"scan_E{E}", T=T, d_model=64, n_experts=E, top_k=k, d_ff=128,
                        act=synth.ACT_RELU, gate_mode=0, dtype=synth.DT_BF16,
                        capacity_factor=cf, logit_bias_std=1.5 if E == 130 else 0.0)
    inp = synth.generate(wl, seed=E + k)
    layer = B.MoELayer(wl, inp, DEV)
    x = inp["x"].to(DEV)
    assert _ticket(layer) == 0
    layouts = []
    for _ in range(2):
        taps = layer.new_taps()
        layer.forward(x, taps=taps)
        torch.cuda.synchronize()
        assert layer.last_device_error() == (0, 0)
        assert _ticket(layer) == 0
        layouts.append({n: taps[n].cpu().numpy() for n in ("topk_idx", "counts", "offsets",
                                                            "inv")})
    a, b = layouts
    for n in ("counts", "offsets", "inv"):
        assert np.array_equal(a[n], b[n]), n
    idx = a["topk_idx"].reshape(-1)
    counts = np.bincount(idx, minlength=E)
    assert np.array_equal(a["counts"], counts)
    cap = int(np.floor(cf * T * k / E)) if cf > 0 else None
    kept = counts if cap is None else np.minimum(counts, cap)
    assert np.array_equal(a["offsets"], np.concatenate([[0], np.cumsum(kept)]))
    # each expert keeps its first `cap` pairs in token order, laid out in that order
    seen = np.zeros(E, dtype=np.int64)
    for p, e in enumerate(idx):
        want = a["offsets"][e] + seen[e] if (cap is None or seen[e] < cap) else -1
        assert a["inv"][p] == want, (p, e)
        seen[e] += 1
