"""Per-expert dispatch: in one call, each expert's rows go to the weight-streaming kernels, the
expert-tile kernels or the row-tile grouped GEMM according to its row count (decided on the
device).  The mid-token regime with skewed routing is where this matters: a few experts see
hundreds of rows, many see tens, some a handful (hearth-lean-loomed-v1 card, "Why 12-16
streams can be slow on Vulkan").  Every case is checked against the fp64 oracle on all tokens.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
from parity_util import check_outputs, compare_routing, gpu_route, host_route, inputs_on_gpu

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import mixture_experts_layer_48_b200 as moe


FAMILY_ROWS = (16, 128, 256)   # rows per work-list entry: streaming, expert tiles, row tiles


def _entry_rows(layer, T):
    """Rows per work-list entry of each family in a T-token call: expert tiles take 256 rows
    once the mean load reaches 128 rows per expert (handles created without MOE_TILE_ROWS)."""
    wide = T * layer.k >= 128 * layer.E
    return (FAMILY_ROWS[0], 256 if wide else 128, FAMILY_ROWS[2])


def _families(layer, T, counts):
    """Experts per family as the dispatch rule assigns them (the bench's mirror of the rule)."""
    import bench
    _, stream_T = layer.get_path()
    s, t, per_expert = layer.get_dispatch()
    f = bench.split_families(counts, "auto", T, stream_T, s, t, per_expert=per_expert)
    return tuple(len(f[k]) for k in ("stream", "tile", "gemm")), f


def _check_device_dispatch(layer, T, counts):
    """The work lists the last forward call built on the device agree with the rule."""
    _, f = _families(layer, T, counts)
    entries = layer.last_dispatch(T)
    rows = _entry_rows(layer, T)
    for i, k in enumerate(("stream", "tile", "gemm")):
        want = sum(-(-c // rows[i]) for c in f[k])
        assert entries[i] == want or (entries[i] == -1 and want == 0), (k, entries, want)
    return entries


def _run(T, E, H, I, k, seed, zipf=False, path=None, dispatch=None, crossover=-1):
    d, h = inputs_on_gpu(T, H, E, k, I, seed, zipf=zipf)
    layer = moe.Moe(E, H, I, k)
    if path is not None or crossover >= 0:
        layer.set_path(moe.MOE_PATH_AUTO if path is None else path, crossover)
    if dispatch is not None:
        layer.set_dispatch(*dispatch)
    ref_route = host_route(h, k)
    g = gpu_route(layer, d)
    rep = compare_routing(g, ref_route, k, E)
    out = layer.forward(d["x"], d["W_router"], d["b_router"], d["W_gate_up"], d["W_down"])
    assert layer.sync_status() == moe.MOE_OK
    ref = oracle.moe_forward_ref(h["x"], h["W_router"], h["b_router"], h["W_gate_up"],
                                 h["W_down"], k, route=ref_route)
    rep.update(check_outputs(out.double().cpu().numpy(), np.arange(T), h, ref_route, g, ref))
    return layer, g, rep


@pytest.mark.parametrize("T,dispatch,expect", [(256, (8, 40, 1), (True, True, True)),
                                               (512, (16, 100, 1), (True, True, True)),
                                               (1024, (16, 128, 1), (False, True, True)),
                                               (256, (8, 40, 0), (True, None, None)),
                                               (1024, (16, 128, 0), (False, False, True)),
                                               (1024, (16, 1000, 0), (False, True, False))])
def test_skewed_mid_T_mixes_the_families(T, dispatch, expect):
    """20b-shaped layer, Zipf-skewed routing, streaming allowed at this T.  With per-expert
    dispatch, streaming, expert tiles and row tiles take experts in the same call, and the work
    lists built on the device are the ones the rule gives for the call's histogram.  At 1024
    tokens the few experts under 16 rows are too few, with too many rows, to stream on their
    own: they join the expert tiles (the snap rule), while the skew across the tile boundary
    keeps row tiles for the largest experts.  Without it, the non-streamed experts take one
    tcgen05 family by their mean count (row tiles here, expert tiles once tile_rows is above
    that mean)."""
    layer, g, rep = _run(T, 32, 2880, 2880, 4, seed=3, zipf=True, dispatch=dispatch, crossover=T)
    counts = np.diff(g["expert_offsets"]).tolist()
    fam, _ = _families(layer, T, counts)
    entries = _check_device_dispatch(layer, T, counts)
    print("hybrid T=%d dispatch=%s experts per family %s entries %s %s" % (
        T, dispatch, fam, entries, json.dumps({k: v for k, v in rep.items() if k != "set_changed"})))
    assert all(want is None or (n > 0) == want for n, want in zip(fam, expect)), (fam, sorted(counts))
    if not dispatch[2]:
        assert fam[1] == 0 or fam[2] == 0, fam


@pytest.mark.parametrize("T", [1024, 1500])
def test_tight_loads_do_not_split_across_the_tile_boundary(T):
    """With no router bias the experts' loads sit close to T*k/E (128 and 188 rows here), the
    second call just below tile_rows = 192: the call's counts keep them all in one family (one
    launch per projection); the layer stays exact."""
    E, H, I, k = 32, 2880, 2880, 4
    d, h = inputs_on_gpu(T, H, E, k, I, seed=2700 + T)
    d["b_router"].zero_()
    h = mi.host_inputs(d)
    layer = moe.Moe(E, H, I, k)
    ref_route = host_route(h, k)
    g = gpu_route(layer, d)
    compare_routing(g, ref_route, k, E)
    counts = np.diff(g["expert_offsets"]).tolist()
    fam, _ = _families(layer, T, counts)
    print("tight loads T=%d counts %d..%d experts per family %s" % (T, min(counts), max(counts), fam))
    assert sum(1 for n in fam if n) == 1, (fam, counts)
    out = layer.forward(d["x"], d["W_router"], d["b_router"], d["W_gate_up"], d["W_down"])
    assert layer.sync_status() == moe.MOE_OK
    _check_device_dispatch(layer, T, counts)
    tokens = mi.sample_tokens(T, 256, 2700 + T)
    got = out[torch.from_numpy(tokens).cuda()].double().cpu().numpy()
    ref = oracle.moe_forward_ref(h["x"], h["W_router"], h["b_router"], h["W_gate_up"],
                                 h["W_down"], k, tokens=tokens, route=ref_route)
    check_outputs(got, tokens, h, ref_route, g, ref)


@pytest.mark.parametrize("T", [17, 40, 129, 300, 777])
def test_expert_tile_path_ragged(T):
    """Every expert through the expert-tile kernels: rows 1..16 per box, 1 or 2 row chunks of
    128, a half-filled last column block (I = 320: 128 + 128 + 64 gate/up columns)."""
    _run(T, 8, 256, 320, 2, seed=2000 + T, path=moe.MOE_PATH_TILE)


@pytest.mark.parametrize("T", [16, 96, 512])
def test_expert_tile_path_gpt_oss_shape(T):
    """H = I = 2880: 45 K stages, 23 gate/up column blocks (the last 64 wide), 12 down blocks
    (the last 64 wide)."""
    _run(T, 32, 2880, 2880, 4, seed=2100 + T, path=moe.MOE_PATH_TILE)


def test_expert_tile_path_120b_shape():
    _run(200, 128, 2880, 2880, 4, seed=2200, path=moe.MOE_PATH_TILE)


@pytest.mark.parametrize("T", [96, 192, 512, 2048])
def test_auto_20b_mid_T(T):
    """The default per-expert thresholds across the mid-token band of the 20b layer."""
    _run(T, 32, 2880, 2880, 4, seed=2300 + T)


def test_thresholds_round_trip():
    layer = moe.Moe(32, 2880, 2880, 4)
    # streaming by default while the expected touched experts' tiles fill < 2 waves of the SMs
    # or leave their last wave < 85 % full: 5 tokens for this layer on a 148-SM B200
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    T0 = layer.get_path()[1]

    def waves(T):
        return 32 * (1 - (1 - 4 / 32) ** T) * 23 / sms

    def streams(T):
        return waves(T) < 2 or waves(T) / math.ceil(waves(T)) < 0.85

    assert all(streams(T) for T in range(1, T0 + 1)) and not streams(T0 + 1)
    if sms == 148:
        assert T0 == 5
    assert layer.get_dispatch() == (16, 192, False)
    layer.set_dispatch(4, 100, 1)
    assert layer.get_dispatch() == (4, 100, True)
    layer.set_dispatch(-1, 50)
    assert layer.get_dispatch() == (4, 50, True)
    layer.set_dispatch(-1, -1, 0)
    assert layer.get_dispatch() == (4, 50, False)
    layer.set_path(moe.MOE_PATH_AUTO, 9)
    assert layer.get_path() == (moe.MOE_PATH_AUTO, 9) and layer.get_dispatch() == (4, 50, False)


def _wide_layer(E, H, I, k):
    """A handle whose row-tile GEMM uses 256 x 512 tiles (two MMAs per K step)."""
    old = os.environ.get("MOE_ROW_TILE")
    os.environ["MOE_ROW_TILE"] = "512"
    try:
        return moe.Moe(E, H, I, k)
    finally:
        if old is None:
            del os.environ["MOE_ROW_TILE"]
        else:
            os.environ["MOE_ROW_TILE"] = old


@pytest.mark.parametrize("T", [1, 65, 300, 520])
def test_wide_row_tiles_ragged(T):
    """The 256 x 512 row tiles: one or several 256-row chunks, a half-filled last column block
    (I = 320: 256 + 64 gate/up columns; H = 256: one down tile of which only the first half has
    columns), the next tile's first-half MMAs running while the second half drains."""
    E, H, I, k = 8, 256, 320, 2
    d, h = inputs_on_gpu(T, H, E, k, I, seed=2500 + T)
    layer = _wide_layer(E, H, I, k)
    layer.set_path(moe.MOE_PATH_GEMM)
    ref_route = host_route(h, k)
    g = gpu_route(layer, d)
    compare_routing(g, ref_route, k, E)
    out = layer.forward(d["x"], d["W_router"], d["b_router"], d["W_gate_up"], d["W_down"])
    assert layer.sync_status() == moe.MOE_OK
    ref = oracle.moe_forward_ref(h["x"], h["W_router"], h["b_router"], h["W_gate_up"],
                                 h["W_down"], k, route=ref_route)
    check_outputs(out.double().cpu().numpy(), np.arange(T), h, ref_route, g, ref)


@pytest.mark.parametrize("T,path", [(300, "gemm"), (2048, "auto")])
def test_wide_row_tiles_gpt_oss_shape(T, path):
    """H = I = 2880: 12 gate/up tiles per chunk (the last with 64 columns, no second half) and
    6 down tiles (the last with 320 columns)."""
    E, H, I, k = 32, 2880, 2880, 4
    d, h = inputs_on_gpu(T, H, E, k, I, seed=2600 + T)
    layer = _wide_layer(E, H, I, k)
    if path == "gemm":
        layer.set_path(moe.MOE_PATH_GEMM)
    ref_route = host_route(h, k)
    g = gpu_route(layer, d)
    compare_routing(g, ref_route, k, E)
    out = layer.forward(d["x"], d["W_router"], d["b_router"], d["W_gate_up"], d["W_down"])
    assert layer.sync_status() == moe.MOE_OK
    tokens = np.arange(T) if T <= 300 else mi.sample_tokens(T, 512, 2600)
    got = out[torch.from_numpy(tokens).cuda()].double().cpu().numpy()
    ref = oracle.moe_forward_ref(h["x"], h["W_router"], h["b_router"], h["W_gate_up"],
                                 h["W_down"], k, tokens=tokens, route=ref_route)
    check_outputs(got, tokens, h, ref_route, g, ref)


def _tile_rows_layer(E, H, I, k, rows):
    """A handle whose expert tiles take `rows` rows per tile (MOE_TILE_ROWS at creation)."""
    old = os.environ.get("MOE_TILE_ROWS")
    os.environ["MOE_TILE_ROWS"] = str(rows)
    try:
        return moe.Moe(E, H, I, k)
    finally:
        if old is None:
            del os.environ["MOE_TILE_ROWS"]
        else:
            os.environ["MOE_TILE_ROWS"] = old


def _check_tile_layer(layer, d, h, k, tokens):
    ref_route = host_route(h, k)
    g = gpu_route(layer, d)
    compare_routing(g, ref_route, k, layer.E)
    out = layer.forward(d["x"], d["W_router"], d["b_router"], d["W_gate_up"], d["W_down"])
    assert layer.sync_status() == moe.MOE_OK
    got = out[torch.from_numpy(tokens).cuda()].double().cpu().numpy()
    ref = oracle.moe_forward_ref(h["x"], h["W_router"], h["b_router"], h["W_gate_up"],
                                 h["W_down"], k, tokens=tokens, route=ref_route)
    check_outputs(got, tokens, h, ref_route, g, ref)
    return g


@pytest.mark.parametrize("T", [3, 40, 300, 1200])
def test_expert_tiles_of_256_rows_ragged(T):
    """256-row expert tiles (one accumulator buffer of 2 x 256 TMEM columns, 3 stages): rows 1..16
    per box, up to 16 boxes, experts of more than 256 rows split over two or three entries, a
    half-filled last column block (I = 320)."""
    E, H, I, k = 8, 256, 320, 2
    d, h = inputs_on_gpu(T, H, E, k, I, seed=3000 + T)
    layer = _tile_rows_layer(E, H, I, k, 256)
    layer.set_path(moe.MOE_PATH_TILE)
    g = _check_tile_layer(layer, d, h, k, np.arange(T))
    counts = np.diff(g["expert_offsets"])
    want = int(sum(-(-c // 256) for c in counts if c > 0))
    assert layer.last_dispatch(T)[1] == want


@pytest.mark.parametrize("T", [512, 2048])
def test_expert_tiles_of_256_rows_gpt_oss_shape(T):
    """H = I = 2880 with 256-row expert tiles: 45 K stages, 23 gate/up and 12 down column blocks
    (the last ones 64 wide)."""
    E, H, I, k = 32, 2880, 2880, 4
    d, h = inputs_on_gpu(T, H, E, k, I, seed=3100 + T)
    layer = _tile_rows_layer(E, H, I, k, 256)
    layer.set_path(moe.MOE_PATH_TILE)
    _check_tile_layer(layer, d, h, k, mi.sample_tokens(T, 384, 3100 + T))
