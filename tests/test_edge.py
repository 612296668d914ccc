"""GPU edge cases: ragged and tiny token counts around every tile boundary, degenerate
expert counts, ties, one hot expert, the status codes of bad calls, the timeout path."""
import ctypes

import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
from parity_util import check_outputs, compare_routing, gpu_route, host_route, inputs_on_gpu

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import mixture_experts_layer_48_b200 as moe


def _check_layer(d, h, E, H, I, k, layer=None, path=None):
    layer = layer or moe.Moe(E, H, I, k)
    if path is not None:
        layer.set_path(path)
    T = d["x"].shape[0]
    ref_route = host_route(h, k)
    g = gpu_route(layer, d)
    compare_routing(g, ref_route, k, E)
    out = layer.forward(d["x"], d["W_router"], d["b_router"], d["W_gate_up"], d["W_down"])
    assert layer.sync_status() == moe.MOE_OK
    ref = oracle.moe_forward_ref(h["x"], h["W_router"], h["b_router"], h["W_gate_up"],
                                 h["W_down"], k, route=ref_route)
    check_outputs(out.double().cpu().numpy(), np.arange(T), h, ref_route, g, ref)
    return layer, g


_PATHS = {"stream": "MOE_PATH_STREAM", "gemm": "MOE_PATH_GEMM", "tile": "MOE_PATH_TILE"}


def _path(name):
    return getattr(moe, _PATHS[name])


@pytest.mark.parametrize("T", [1, 2, 3, 15, 16, 17, 31, 33, 63, 64, 65, 96, 127, 129, 300])
def test_ragged_token_counts(T):
    d, h = inputs_on_gpu(T, 256, 8, 2, 320, seed=100 + T)
    _check_layer(d, h, 8, 256, 320, 2)


@pytest.mark.parametrize("E,k", [(1, 1), (2, 1), (2, 2), (8, 1), (8, 8), (5, 3)])
def test_degenerate_expert_counts(E, k):
    d, h = inputs_on_gpu(40, 128, E, k, 192, seed=200 + E * 10 + k)
    _check_layer(d, h, E, 128, 192, k)


@pytest.mark.parametrize("T", [7, 100])
def test_k_equals_E_256(T):
    d, h = inputs_on_gpu(T, 64, 256, 256, 64, seed=300 + T, experts=False)
    layer = moe.Moe(256, 64, 64, 256)
    compare_routing(gpu_route(layer, d), host_route(h, 256), 256, 256)


@pytest.mark.parametrize("T", [5, 70])
def test_all_equal_logits(T):
    d, h = inputs_on_gpu(T, 128, 8, 3, 128, seed=400 + T)
    d["W_router"].zero_()
    d["b_router"].zero_()
    h = mi.host_inputs(d)
    layer, g = _check_layer(d, h, 8, 128, 128, 3)
    assert np.all(g["topk_idx"] == np.array([0, 1, 2]))
    np.testing.assert_allclose(g["topk_w"], 1 / 3, atol=1e-7)


@pytest.mark.parametrize("T", [40, 200])
def test_one_hot_expert(T):
    d, h = inputs_on_gpu(T, 128, 16, 2, 128, seed=500 + T)
    d["b_router"].zero_()
    d["b_router"][11] = 1000.0       # every token picks expert 11 first
    h = mi.host_inputs(d)
    layer, g = _check_layer(d, h, 16, 128, 128, 2)
    assert np.all(g["topk_idx"][:, 0] == 11)
    assert np.diff(g["expert_offsets"])[11] == T


def test_gpt_oss_shape_with_ragged_T():
    d, h = inputs_on_gpu(37, 2880, 32, 4, 2880, seed=600)
    _check_layer(d, h, 32, 2880, 2880, 4)


def test_forward_twice_agrees_and_overwrites_out():
    # fp32 atomics make the summation order vary between calls, so the bf16 SwiGLU output can
    # move by one bf16 step (2^-8 relative): runs agree to that noise, not bit for bit.
    d, h = inputs_on_gpu(24, 256, 8, 2, 256, seed=700)
    layer = moe.Moe(8, 256, 256, 2)
    out = torch.full((24, 256), 12345.0, device="cuda")
    a = layer.forward(d["x"], d["W_router"], d["b_router"], d["W_gate_up"], d["W_down"], out=out).clone()
    b = layer.forward(d["x"], d["W_router"], d["b_router"], d["W_gate_up"], d["W_down"])
    torch.cuda.synchronize()
    assert torch.isfinite(a).all()
    torch.testing.assert_close(a, b, atol=5e-4, rtol=1e-3)


def test_zero_tokens():
    layer = moe.Moe(8, 256, 256, 2)
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    Wr = torch.zeros((256, 8), dtype=torch.bfloat16, device="cuda")
    b = torch.zeros(8, device="cuda")
    Wgu = torch.zeros((8, 256, 512), dtype=torch.bfloat16, device="cuda")
    Wd = torch.zeros((8, 256, 256), dtype=torch.bfloat16, device="cuda")
    out = layer.forward(x, Wr, b, Wgu, Wd)
    assert out.shape == (0, 256)
    r = layer.route(x, Wr, b)
    assert r["expert_offsets"].cpu().tolist() == [0] * 9
    assert layer.sync_status() == moe.MOE_OK


def test_bad_calls_return_status_codes():
    d, _ = inputs_on_gpu(8, 256, 8, 2, 256, seed=800)
    layer = moe.Moe(8, 256, 256, 2)
    ws = torch.empty(layer.workspace_bytes(8), dtype=torch.uint8, device="cuda")
    out = torch.empty((8, 256), device="cuda")
    p = [d[k].data_ptr() for k in ("x", "W_router", "b_router", "W_gate_up", "W_down")]
    st = torch.cuda.current_stream().cuda_stream
    f = moe.moe_forward
    assert f(layer.handle, 8, *p, out.data_ptr(), ws.data_ptr(), ws.numel(), st) == moe.MOE_OK
    assert f(layer.handle, 8, *p, out.data_ptr(), ws.data_ptr(), ws.numel() - 1, st) == moe.MOE_ERR_WORKSPACE
    assert f(layer.handle, 8, *p, out.data_ptr(), 0, ws.numel(), st) == moe.MOE_ERR_WORKSPACE
    bad = list(p)
    bad[0] += 2  # misaligned x
    assert f(layer.handle, 8, *bad, out.data_ptr(), ws.data_ptr(), ws.numel(), st) == moe.MOE_ERR_ARG
    assert f(layer.handle, -1, *p, out.data_ptr(), ws.data_ptr(), ws.numel(), st) == moe.MOE_ERR_ARG
    assert f(layer.handle, 8, *p, 0, ws.data_ptr(), ws.numel(), st) == moe.MOE_ERR_ARG
    assert layer.sync_status() == moe.MOE_OK


def test_timeout_is_reported_not_hung():
    layer = moe.Moe(8, 256, 256, 2)
    layer.selftest_timeout(2000)   # 2 ms bounded wait on a barrier nothing completes
    assert layer.sync_status() == moe.MOE_ERR_TIMEOUT
    assert layer.sync_status() == moe.MOE_OK   # the word is cleared by the read
    d, h = inputs_on_gpu(16, 256, 8, 2, 256, seed=900)
    _check_layer(d, h, 8, 256, 256, 2, layer=layer)   # the context is still usable


def test_profile_counts_kernels():
    d, _ = inputs_on_gpu(16, 256, 8, 2, 256, seed=901)
    layer = moe.Moe(8, 256, 256, 2)
    layer.profile_begin(3)
    n0 = layer.launch_count()
    for _ in range(3):
        layer.forward(d["x"], d["W_router"], d["b_router"], d["W_gate_up"], d["W_down"])
    prof = layer.profile_end()
    assert layer.launch_count() - n0 == sum(v[1] for v in prof.values())
    assert prof["gate_up_stream"][1] == 3 and prof["down_stream"][1] == 3
    assert all(v[0] >= 0 for v in prof.values())


@pytest.mark.parametrize("T", [1, 5, 16, 64, 65, 200, 520])
@pytest.mark.parametrize("path", ["stream", "gemm", "tile"])
def test_every_path_matches_the_oracle(T, path):
    """Each kernel family for every expert at any T: the streaming kernels, the 2-SM row-tile
    grouped GEMM and the expert-tile kernels."""
    d, h = inputs_on_gpu(T, 256, 8, 2, 320, seed=1000 + T)
    _check_layer(d, h, 8, 256, 320, 2, path=_path(path))


@pytest.mark.parametrize("path", ["stream", "gemm", "tile"])
def test_every_path_gpt_oss_shape(path):
    d, h = inputs_on_gpu(300, 2880, 32, 4, 2880, seed=1100)
    _check_layer(d, h, 32, 2880, 2880, 4, path=_path(path))


def test_tune_measures_the_dispatch_thresholds_and_auto_follows_them():
    E, H, I, k = 32, 2880, 2880, 4
    d, h = inputs_on_gpu(1024, H, E, k, I, seed=1200)
    layer = moe.Moe(E, H, I, k)
    c = layer.tune(d["x"], d["W_router"], d["b_router"], d["W_gate_up"], d["W_down"])
    path, crossover = layer.get_path()
    s, t, _ = layer.get_dispatch()
    assert path == moe.MOE_PATH_AUTO and crossover == c
    assert 0 <= c <= 1024 and t >= 1
    print("measured: streaming in calls of <=", c, "tokens; tile_rows", t)
    assert layer.sync_status() == moe.MOE_OK
    # the layer with the measured thresholds still matches the oracle
    d2 = dict(d, x=d["x"][:300].contiguous())
    h2 = dict(h, x=h["x"][:300])
    _check_layer(d2, h2, E, H, I, k, layer=layer)


@pytest.mark.parametrize("T,path", [(10, "stream"), (100, "gemm"), (100, "tile"), (300, "auto")])
def test_forward_with_k_equal_E_256(T, path):
    """Every token uses all 256 experts (the widest routing the ABI accepts)."""
    p = moe.MOE_PATH_AUTO if path == "auto" else _path(path)
    d, h = inputs_on_gpu(T, 64, 256, 256, 64, seed=1300 + T)
    _check_layer(d, h, 256, 64, 64, 256, path=p)


def test_largest_token_count():
    """T = 2^20 (the largest T the ABI accepts) on a narrow layer; routing is checked on every
    token, outputs on a seeded sample."""
    T, H, E, k, I = 1 << 20, 64, 8, 2, 64
    d, h = inputs_on_gpu(T, H, E, k, I, seed=1400)
    layer = moe.Moe(E, H, I, k)
    ref_route = host_route(h, k)
    g = gpu_route(layer, d)
    compare_routing(g, ref_route, k, E)
    out = layer.forward(d["x"], d["W_router"], d["b_router"], d["W_gate_up"], d["W_down"])
    assert layer.sync_status() == moe.MOE_OK
    tokens = mi.sample_tokens(T, 2048, 1400)
    got = out[torch.from_numpy(tokens).cuda()].double().cpu().numpy()
    ref = oracle.moe_forward_ref(h["x"], h["W_router"], h["b_router"], h["W_gate_up"], h["W_down"],
                                 k, tokens=tokens, route=ref_route)
    check_outputs(got, tokens, h, ref_route, g, ref)


@pytest.mark.parametrize("path", ["stream", "gemm", "tile"])
def test_wide_hidden_and_intermediate(path):
    """H = I = 8192: long K loops and many column tiles in every path."""
    d, h = inputs_on_gpu(24, 8192, 2, 1, 8192, seed=1500)
    _check_layer(d, h, 2, 8192, 8192, 1, path=_path(path))


@pytest.mark.parametrize("T,per_expert", [(3, 0), (40, 0), (300, 0), (300, 1)])
def test_forward_replays_in_a_cuda_graph(T, per_expert):
    """One call captured in a CUDA graph, replayed on new tokens written into the captured
    input: the replay reads them and matches the oracle (streaming at 3 tokens, expert tiles at
    40, row tiles at 300; the per-expert dispatch at 300 may fork the row tiles onto the handle's
    second stream inside the capture)."""
    E, H, I, k = 8, 256, 320, 2
    d, _ = inputs_on_gpu(T, H, E, k, I, seed=2800 + T)
    layer = moe.Moe(E, H, I, k)
    layer.set_path(moe.MOE_PATH_AUTO, T)
    layer.set_dispatch(-1, 64, per_expert)
    x = d["x"].clone()
    out = torch.empty((T, H), dtype=torch.float32, device="cuda")
    ws = torch.empty(layer.workspace_bytes(T), dtype=torch.uint8, device="cuda")
    fwd = lambda: layer.forward(x, d["W_router"], d["b_router"], d["W_gate_up"], d["W_down"],
                                out=out, workspace=ws)
    fwd()  # tensor maps built outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fwd()
    x.copy_(mi.draw_x(T, H, 2900 + T, "cuda"))
    out.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    assert layer.sync_status() == moe.MOE_OK
    d2 = dict(d, x=x.clone())
    h2 = mi.host_inputs(d2)
    ref_route = host_route(h2, k)
    gr = gpu_route(layer, d2)
    compare_routing(gr, ref_route, k, E)
    ref = oracle.moe_forward_ref(h2["x"], h2["W_router"], h2["b_router"], h2["W_gate_up"],
                                 h2["W_down"], k, route=ref_route)
    check_outputs(out.double().cpu().numpy(), np.arange(T), h2, ref_route, gr, ref)
    del g
