"""The device half of expert parallelism on one GPU: moe_permute, moe_experts on rows that arrive
as (source, expert) segments from several sources, moe_combine, and the whole ExpertParallelMoe
over a one-rank NCCL group.  Against the fp64 oracle (multi-GPU exchanges are covered by the
two-rank gloo test on CPU)."""
import os
import socket

import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
from parity_util import ATOL, RTOL, check_outputs, compare_routing, gpu_route, host_route, inputs_on_gpu

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import mixture_experts_layer_48_b200 as moe
    from mixture_experts_layer_48_b200 import ep


def _oracle_expert_rows(x_bits, row_w, seg_counts, h, first=0):
    """y[r] = row_w[r] * expert_mlp(x[r]) with the expert of r's (source, expert) segment."""
    S, El = seg_counts.shape
    y = np.zeros((x_bits.shape[0], h["H"]))
    r0 = 0
    for s in range(S):
        for e in range(El):
            n = int(seg_counts[s, e])
            if n:
                y[r0:r0 + n] = row_w[r0:r0 + n, None] * oracle.expert_mlp(
                    oracle.decode_bf16(x_bits[r0:r0 + n]),
                    oracle.decode_bf16(h["W_gate_up"][first + e]),
                    oracle.decode_bf16(h["W_down"][first + e]))
            r0 += n
    return y


@pytest.mark.parametrize("path", ["auto", "stream", "tile", "gemm"])
@pytest.mark.parametrize("S", [1, 3])
def test_experts_on_segments(path, S):
    """Rows of 8 experts from S sources (source-major segments, some empty), every family."""
    E, H, I, k = 8, 256, 320, 2
    d, h = inputs_on_gpu(1, H, E, k, I, seed=3000 + S)
    rng = np.random.default_rng(S)
    seg = rng.integers(0, 90, size=(S, E)).astype(np.int32)
    seg[0, 2] = 0
    seg[:, 6] = 3                        # a small expert: streamed under AUTO
    seg[-1, 5] = 300                     # a large expert: row tiles under AUTO
    R = int(seg.sum())
    x = mi.draw_x(R, H, 3100 + S, "cuda")
    row_w = torch.rand(R, generator=torch.Generator().manual_seed(S)).cuda()
    layer = moe.Moe(E, H, I, k)
    if path != "auto":
        layer.set_path({"stream": moe.MOE_PATH_STREAM, "tile": moe.MOE_PATH_TILE,
                        "gemm": moe.MOE_PATH_GEMM}[path])
    y = layer.experts(x, row_w, torch.from_numpy(seg).cuda(), d["W_gate_up"], d["W_down"])
    assert layer.sync_status() == moe.MOE_OK
    ref = _oracle_expert_rows(mi.bf16_bits(x), row_w.double().cpu().numpy(), seg, h)
    got = y.double().cpu().numpy()
    assert np.all(np.abs(got - ref) <= ATOL + RTOL * np.abs(ref))


def test_experts_reports_counts_that_do_not_add_up():
    E, H, I, k = 4, 128, 128, 2
    d, _ = inputs_on_gpu(1, H, E, k, I, seed=3200)
    layer = moe.Moe(E, H, I, k)
    x = mi.draw_x(40, H, 3201, "cuda")
    w = torch.ones(40, device="cuda")
    seg = torch.tensor([[10, 10, 10, 30]], dtype=torch.int32, device="cuda")   # 60 > 40 rows
    layer.experts(x, w, seg, d["W_gate_up"], d["W_down"])
    assert layer.sync_status() == moe.MOE_ERR_ARG
    assert layer.sync_status() == moe.MOE_OK


@pytest.mark.parametrize("T", [16, 300])
def test_route_permute_experts_combine_equals_the_layer(T):
    """The layer assembled from the expert-parallel building blocks with one source."""
    E, H, I, k = 32, 2880, 2880, 4
    d, h = inputs_on_gpu(T, H, E, k, I, seed=3300 + T)
    layer = moe.Moe(E, H, I, k)
    r = layer.route(d["x"], d["W_router"], d["b_router"])
    x_perm, row_w = layer.permute(d["x"], r)
    counts = torch.diff(r["expert_offsets"]).to(torch.int32).reshape(1, E)
    y = layer.experts(x_perm, row_w, counts, d["W_gate_up"], d["W_down"])
    out = layer.combine(r["inv_perm"], y)
    assert layer.sync_status() == moe.MOE_OK
    ref_route = host_route(h, k)
    g = {key: v.cpu().numpy().astype(np.int64 if v.dtype == torch.int32 else np.float64)
         for key, v in r.items()}
    compare_routing(g, ref_route, k, E)
    assert np.array_equal(mi.bf16_bits(x_perm), h["x"][g["perm"]])
    ref = oracle.moe_forward_ref(h["x"], h["W_router"], h["b_router"], h["W_gate_up"],
                                 h["W_down"], k, route=ref_route)
    check_outputs(out.double().cpu().numpy(), np.arange(T), h, ref_route, g, ref)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_expert_parallel_layer_on_one_rank_nccl():
    """ExpertParallelMoe over a one-rank NCCL group: the exchange is the identity, every kernel
    of the path runs on this GPU."""
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()), RANK="0",
                      WORLD_SIZE="1")
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=60))
    try:
        E, H, I, k, T = 32, 2880, 2880, 4, 64
        d, h = inputs_on_gpu(T, H, E, k, I, seed=3400)
        layer = ep.ExpertParallelMoe(E, H, I, k)
        out = layer(d["x"], d["W_router"], d["b_router"], d["W_gate_up"], d["W_down"])
        torch.cuda.synchronize()
        assert layer.ops.full.sync_status() == moe.MOE_OK
        assert layer.ops.local.sync_status() == moe.MOE_OK
        ref_route = host_route(h, k)
        g = gpu_route(layer.ops.full, d)
        compare_routing(g, ref_route, k, E)
        ref = oracle.moe_forward_ref(h["x"], h["W_router"], h["b_router"], h["W_gate_up"],
                                     h["W_down"], k, route=ref_route)
        check_outputs(out.double().cpu().numpy(), np.arange(T), h, ref_route, g, ref)
        assert layer.last_exchange["recv_rows"] == [T * k]
    finally:
        dist.destroy_process_group()
