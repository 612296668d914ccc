"""Seeded synthetic inputs for the MoE layer forward pass.

This module is shared by the CUDA-path tests, the benchmark and the oracle tests.  It draws
random numbers and converts tensors to host arrays; it holds none of the layer's arithmetic.

Recipe (the pages' workloads use trained gpt-oss weights and real text, neither of which is
here; these draws stand in for them with the same shapes):

* every tensor has its own ``torch.Generator`` on the target device, seeded with
  ``seed * 1000 + slot`` where slot is 0 x, 1 W_router, 2 b_router, 3 W_gate_up, 4 W_down,
  5 Zipf ranks (always a CPU generator), 6 token sample (CPU generator).  Weights therefore do
  not depend on T, so one layer serves a sweep over token counts;
* values are drawn as float32 normals, scaled, then rounded to bf16 (round to nearest even):
  x ~ N(0, 1); W_router [H,E] and W_gate_up [E,H,2I] ~ N(0, 1/H); W_down [E,I,H] ~ N(0, 1/I);
  b_router ~ N(0, 0.1) kept in float32.  N(m, v) names the variance v;
* W_gate_up and W_down are drawn one expert at a time (``[H,2I]`` then the next expert);
* MXFP4 experts (``weights="mxfp4"``): ``gu_codes [E, 2I, H/2]``, ``gu_scales [E, H/32, 2I]``,
  ``dn_codes [E, H, I/2]``, ``dn_scales [E, I/32, H]`` (uint8; the layout the oracle's
  ``dequant_mxfp4`` reads).  Every block byte is uniform on 0..255 (two uniform 4-bit codes);
  every scale byte is s0 + {-1, 0, +1} uniformly, with s0 = 127 + round(log2(1 / (4 *
  sqrt(fan_in)))), which puts the dequantized weights' spread near 1/sqrt(fan_in) like the bf16
  draws (0.8/sqrt(fan_in) at fan_in = 2880).  Slots 7 (gate/up) and 8 (down), drawn one expert
  at a time (codes, then scales);
* skewed routing adds ``-c * s * ln(rank_e)`` to b_router, rank a seeded permutation of
  1..E and s = 1.1, so expert popularity falls off like a Zipf law.  c is the scale that gives
  a max/mean expert load of 4.0 on a 4096-token sample; it is computed by
  ``tests/golden/make_zipf_scale.py`` from the oracle's routing and stored in
  ``tests/golden/zipf_scale.json``.
"""

from __future__ import annotations

import json
import math
import os
from dataclasses import dataclass, field

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
ZIPF_SCALE_FILE = os.path.join(os.path.dirname(_HERE), "tests", "golden", "zipf_scale.json")
ZIPF_S = 1.1


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    E: int
    k: int
    I: int
    seed: int
    zipf: bool = False
    oracle_sample: int = 0          # 0: the oracle checks every token
    sweep: tuple = field(default=())  # token counts of a sweep (T is the largest)
    weights: str = "bf16"             # expert weight format: "bf16" or "mxfp4"


# The five workloads: a tiny layer; the 20b layer (H = I = 2880, 32 experts, top-4) in decode
# (16 tokens) and prefill (8192 tokens); a packed 131,072-token sequence with skewed routing;
# the 120b layer (128 experts) over 1..32 decode tokens.
WORKLOADS = {
    "tiny": Workload("tiny", T=64, H=256, E=8, k=2, I=256, seed=0),
    "20b_decode": Workload("20b_decode", T=16, H=2880, E=32, k=4, I=2880, seed=1),
    "20b_prefill": Workload("20b_prefill", T=8192, H=2880, E=32, k=4, I=2880, seed=2),
    "131k_skewed": Workload("131k_skewed", T=131072, H=2880, E=32, k=4, I=2880, seed=3,
                            zipf=True, oracle_sample=4096),
    "120b_sweep": Workload("120b_sweep", T=32, H=2880, E=128, k=4, I=2880, seed=4,
                           sweep=(1, 8, 12, 16, 32)),
    # the 20b decode layer with its experts in their native MXFP4 format (W4A16)
    "20b_decode_mxfp4": Workload("20b_decode_mxfp4", T=16, H=2880, E=32, k=4, I=2880, seed=5,
                                 weights="mxfp4"),
}


def _gen(seed: int, slot: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000 + slot)
    return g


def zipf_scale() -> float:
    with open(ZIPF_SCALE_FILE) as f:
        return float(json.load(f)["c"])


def zipf_bias(E: int, seed: int, c: float) -> torch.Tensor:
    """-c * s * ln(rank_e) with rank a seeded permutation of 1..E (float32, CPU)."""
    rank = torch.randperm(E, generator=_gen(seed, 5, "cpu")) + 1
    return (-c * ZIPF_S * torch.log(rank.to(torch.float64))).to(torch.float32)


def draw_x(T: int, H: int, seed: int, device="cpu") -> torch.Tensor:
    return torch.randn((T, H), generator=_gen(seed, 0, device), device=device,
                       dtype=torch.float32).to(torch.bfloat16)


def draw_router(H: int, E: int, seed: int, device="cpu", zipf: bool = False,
                c: float | None = None):
    W_router = (torch.randn((H, E), generator=_gen(seed, 1, device), device=device,
                            dtype=torch.float32) * (1.0 / math.sqrt(H))).to(torch.bfloat16)
    b_router = torch.randn((E,), generator=_gen(seed, 2, device), device=device,
                           dtype=torch.float32) * math.sqrt(0.1)
    if zipf:
        b_router = b_router + zipf_bias(E, seed, zipf_scale() if c is None else c).to(device)
    return W_router, b_router


def _mx_scale_center(fan_in: int) -> int:
    return 127 + int(round(math.log2(1.0 / (4.0 * math.sqrt(fan_in)))))


def _draw_mx(E: int, N: int, K: int, seed: int, slot: int, device):
    g = _gen(seed, slot, device)
    codes = torch.empty((E, N, K // 2), dtype=torch.uint8, device=device)
    scales = torch.empty((E, K // 32, N), dtype=torch.uint8, device=device)
    s0 = _mx_scale_center(K)
    for e in range(E):
        codes[e] = torch.randint(0, 256, (N, K // 2), generator=g, device=device,
                                 dtype=torch.int32).to(torch.uint8)
        scales[e] = (torch.randint(-1, 2, (K // 32, N), generator=g, device=device,
                                   dtype=torch.int32) + s0).to(torch.uint8)
    return codes, scales


def draw_experts_mxfp4(E: int, H: int, I: int, seed: int, device="cpu"):
    """MXFP4 experts: (gu_codes, gu_scales, dn_codes, dn_scales), see the module recipe."""
    gu_codes, gu_scales = _draw_mx(E, 2 * I, H, seed, 7, device)
    dn_codes, dn_scales = _draw_mx(E, H, I, seed, 8, device)
    return gu_codes, gu_scales, dn_codes, dn_scales


def draw_experts(E: int, H: int, I: int, seed: int, device="cpu"):
    W_gate_up = torch.empty((E, H, 2 * I), dtype=torch.bfloat16, device=device)
    g = _gen(seed, 3, device)
    for e in range(E):
        W_gate_up[e] = (torch.randn((H, 2 * I), generator=g, device=device, dtype=torch.float32)
                        * (1.0 / math.sqrt(H))).to(torch.bfloat16)
    W_down = torch.empty((E, I, H), dtype=torch.bfloat16, device=device)
    g = _gen(seed, 4, device)
    for e in range(E):
        W_down[e] = (torch.randn((I, H), generator=g, device=device, dtype=torch.float32)
                     * (1.0 / math.sqrt(I))).to(torch.bfloat16)
    return W_gate_up, W_down


def make_inputs(T: int, H: int, E: int, k: int, I: int, seed: int, device="cpu",
                zipf: bool = False, experts: bool = True, weights: str = "bf16") -> dict:
    """All inputs of one layer call as torch tensors on ``device`` (see the module recipe).

    weights="bf16" gives W_gate_up / W_down; "mxfp4" gives gu_codes, gu_scales, dn_codes,
    dn_scales instead."""
    x = draw_x(T, H, seed, device)
    W_router, b_router = draw_router(H, E, seed, device, zipf)
    d = dict(x=x, W_router=W_router, b_router=b_router, T=T, H=H, E=E, k=k, I=I)
    if experts and weights == "mxfp4":
        (d["gu_codes"], d["gu_scales"], d["dn_codes"],
         d["dn_scales"]) = draw_experts_mxfp4(E, H, I, seed, device)
    elif experts:
        d["W_gate_up"], d["W_down"] = draw_experts(E, H, I, seed, device)
    return d


def workload_inputs(name: str, device="cpu", T: int | None = None, experts: bool = True) -> dict:
    w = WORKLOADS[name]
    return make_inputs(w.T if T is None else T, w.H, w.E, w.k, w.I, w.seed, device, w.zipf,
                       experts, w.weights)


def sample_tokens(T: int, n: int, seed: int) -> np.ndarray:
    """A seeded, sorted sample of n distinct token indices out of T."""
    if n >= T:
        return np.arange(T)
    p = torch.randperm(T, generator=_gen(seed, 6, "cpu"))[:n]
    return np.sort(p.numpy()).astype(np.int64)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 array of its bit patterns (on the host)."""
    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def host_inputs(d: dict) -> dict:
    """Host arrays of a ``make_inputs`` dict: bf16 tensors as uint16 bits, fp32 as float32."""
    out = {}
    for key, v in d.items():
        if isinstance(v, torch.Tensor):
            out[key] = bf16_bits(v) if v.dtype == torch.bfloat16 else v.detach().cpu().numpy()
        else:
            out[key] = v
    return out
