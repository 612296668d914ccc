"""GPU parity: the CUDA library against the fp64 oracle on the five seeded workloads.

Routing (expert indices, histogram, offsets, permutation) must be bit-exact apart from
reported near ties; outputs must satisfy |gpu - oracle| <= 1e-2 + 2e-2 |oracle| per element.
"""
import json

import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
from parity_util import check_outputs, compare_routing, gpu_route, host_route, inputs_on_gpu

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import mixture_experts_layer_48_b200 as moe


def _run(name, T=None, path=None, sample=None):
    w = mi.WORKLOADS[name]
    T = w.T if T is None else T
    d, h = inputs_on_gpu(T, w.H, w.E, w.k, w.I, w.seed, zipf=w.zipf)
    layer = moe.Moe(w.E, w.H, w.I, w.k)
    if path is not None:
        layer.set_path(path)
    ref_route = host_route(h, w.k)
    g = gpu_route(layer, d)
    rep = compare_routing(g, ref_route, w.k, w.E)
    out = layer.forward(d["x"], d["W_router"], d["b_router"], d["W_gate_up"], d["W_down"])
    assert layer.sync_status() == moe.MOE_OK
    tokens = np.arange(T) if not sample else mi.sample_tokens(T, sample, w.seed)
    out_gpu = out[torch.from_numpy(tokens).cuda()].double().cpu().numpy()
    ref_out = oracle.moe_forward_ref(h["x"], h["W_router"], h["b_router"], h["W_gate_up"],
                                     h["W_down"], w.k, tokens=tokens, route=ref_route)
    orep = check_outputs(out_gpu, tokens, h, ref_route, g, ref_out)
    rep.update(orep)
    print(name, T, json.dumps({k: v for k, v in rep.items() if k != "set_changed"}))
    return rep, g


def test_tiny():
    _run("tiny")


def test_20b_decode():
    _run("20b_decode")


@pytest.mark.parametrize("T", mi.WORKLOADS["120b_sweep"].sweep)
def test_120b_sweep(T):
    _run("120b_sweep", T=T)


def test_20b_prefill():
    _run("20b_prefill", sample=1024)


def test_131k_skewed():
    w = mi.WORKLOADS["131k_skewed"]
    rep, g = _run("131k_skewed", sample=w.oracle_sample)
    cnt = np.diff(g["expert_offsets"])
    ratio = cnt.max() / cnt.mean()
    print("131k max/mean expert load", ratio)
    assert 3.5 <= ratio <= 4.5


@pytest.fixture(scope="module")
def layer_120b():
    """The 120b-shaped layer (128 experts, top-4: hearth-lean-loomed-v1 card, intro) with 512
    seeded tokens, drawn once on the GPU and copied to the host for the oracle."""
    w = mi.WORKLOADS["120b_sweep"]
    d, h = inputs_on_gpu(512, w.H, w.E, w.k, w.I, w.seed)
    return w, d, h


@pytest.mark.parametrize("T", [65, 97, 512])
@pytest.mark.parametrize("path", ["gemm", "auto"])
def test_120b_above_the_crossover(layer_120b, T, path):
    """E = 128 at token counts where AUTO leaves the streaming path: the tcgen05 grouped GEMM
    (forced, and as AUTO picks it), every token's routing and output against the oracle."""
    w, d0, h0 = layer_120b
    d = dict(d0, x=d0["x"][:T].contiguous())
    h = dict(h0, x=h0["x"][:T])
    layer = moe.Moe(w.E, w.H, w.I, w.k)
    if path == "gemm":
        layer.set_path(moe.MOE_PATH_GEMM)
    ref_route = host_route(h, w.k)
    g = gpu_route(layer, d)
    rep = compare_routing(g, ref_route, w.k, w.E)
    out = layer.forward(d["x"], d["W_router"], d["b_router"], d["W_gate_up"], d["W_down"])
    assert layer.sync_status() == moe.MOE_OK
    tokens = np.arange(T)
    ref_out = oracle.moe_forward_ref(h["x"], h["W_router"], h["b_router"], h["W_gate_up"],
                                     h["W_down"], w.k, route=ref_route)
    rep.update(check_outputs(out.double().cpu().numpy(), tokens, h, ref_route, g, ref_out))
    print("120b", path, T, json.dumps({k: v for k, v in rep.items() if k != "set_changed"}))


@pytest.mark.parametrize("T", [1, 2, 3, 5, 8])
def test_120b_streaming_finishes_its_routing(layer_120b, T):
    """Calls of at most 8 tokens on the streaming family alone: the gate/up kernel finishes the
    routing from the router's partial logits in every CTA (no finalize kernel).  Outputs against
    the oracle, and the work list it left in the workspace has one entry per touched expert."""
    w, d0, h0 = layer_120b
    d = dict(d0, x=d0["x"][:T].contiguous())
    h = dict(h0, x=h0["x"][:T])
    layer = moe.Moe(w.E, w.H, w.I, w.k)
    layer.set_path(moe.MOE_PATH_STREAM)
    ref_route = host_route(h, w.k)
    g = gpu_route(layer, d)
    rep = compare_routing(g, ref_route, w.k, w.E)
    ws = torch.empty(layer.workspace_bytes(T), dtype=torch.uint8, device="cuda")
    out = layer.forward(d["x"], d["W_router"], d["b_router"], d["W_gate_up"], d["W_down"],
                        workspace=ws)
    assert layer.sync_status() == moe.MOE_OK
    touched = int((np.diff(g["expert_offsets"]) > 0).sum())
    assert layer.last_dispatch(T, workspace=ws)[0] == touched
    ref_out = oracle.moe_forward_ref(h["x"], h["W_router"], h["b_router"], h["W_gate_up"],
                                     h["W_down"], w.k, route=ref_route)
    rep.update(check_outputs(out.double().cpu().numpy(), np.arange(T), h, ref_route, g, ref_out))
    print("120b stream", T, json.dumps({k: v for k, v in rep.items() if k != "set_changed"}))
