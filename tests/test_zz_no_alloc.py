"""moe_route_static: routing for callers that cannot allocate device memory.

Such callers (a process whose device memory all belongs to another allocator, a serving loop
that forbids allocation after start-up, a C caller without an allocator) cannot pass the
workspace moe_route needs.  moe_route_static uses a fixed scratch array built into the
library instead.  This test calls it through the C ABI twice in a row and checks each result
against moe_route with a caller workspace, to the routing tolerances the parity tests use:
above 64 tokens the static call's router sums the logits in another order, so a token may
select differently only where the fp64 oracle's k-th / (k+1)-th logit gap is a near tie, and
the permutation must then be the one of the static call's own selection.
"""
import ctypes

import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
from parity_util import NEAR_TIE, W_TOL, host_route

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import mixture_experts_layer_48_b200 as moe


def _outputs(T, k, E):
    dev = "cuda"
    return dict(topk_idx=torch.empty((T, k), dtype=torch.int32, device=dev),
                topk_w=torch.empty((T, k), dtype=torch.float32, device=dev),
                expert_offsets=torch.empty((E + 1,), dtype=torch.int32, device=dev),
                perm=torch.empty((T * k,), dtype=torch.int32, device=dev),
                inv_perm=torch.empty((T, k), dtype=torch.int32, device=dev))


def _call_static(layer, d, o):
    st = torch.cuda.current_stream().cuda_stream
    return moe.moe_route_static(layer.handle, d["x"].shape[0], d["x"].data_ptr(),
                                d["W_router"].data_ptr(), d["b_router"].data_ptr(),
                                o["topk_idx"].data_ptr(), o["topk_w"].data_ptr(),
                                o["expert_offsets"].data_ptr(), o["perm"].data_ptr(),
                                o["inv_perm"].data_ptr(), st)


def _check_against_workspace_route(got, ref, gaps, E):
    """Routing of the static call against moe_route's, to the parity tests' tolerances."""
    diff = np.nonzero(np.any(got["topk_idx"] != ref["topk_idx"], axis=1))[0]
    for t in diff:                            # only near ties may select differently
        assert min(gaps["gap_k"][t], gaps["gap_in"][t]) < NEAR_TIE, f"token {t}"
    same = np.setdiff1d(np.arange(got["topk_idx"].shape[0]), diff)
    assert np.abs(got["topk_w"][same] - ref["topk_w"][same]).max() <= W_TOL
    # the permutation is unique given the selection: the static call's own, bit for bit
    idx = got["topk_idx"].astype(np.int64)
    perm, inv = oracle.permutation(idx, E)
    assert np.array_equal(got["expert_offsets"], oracle.expert_offsets(oracle.expert_histogram(idx, E)))
    assert np.array_equal(got["perm"], perm) and np.array_equal(got["inv_perm"], inv)
    if diff.size == 0:
        for key in ("expert_offsets", "perm", "inv_perm"):
            assert np.array_equal(got[key], ref[key]), key
    return int(diff.size)


@pytest.mark.parametrize("T", [16, 300])   # the single-block and the multi-block routing chain
def test_static_scratch_route_matches_workspace_route(T):
    E, H, k = 32, 2880, 4
    d = mi.make_inputs(T, H, E, k, 64, seed=1234 + T, device="cuda", experts=False)
    gaps = host_route(mi.host_inputs(d), k)
    layer = moe.Moe(E, H, 64, k)
    ref = {key: v.cpu().numpy() for key, v in layer.route(d["x"], d["W_router"], d["b_router"]).items()}
    for _ in range(2):                       # two calls in a row share the one scratch array
        o = _outputs(T, k, E)
        for v in o.values():
            v.fill_(-7)
        assert _call_static(layer, d, o) == moe.MOE_OK
        torch.cuda.synchronize()
        got = {key: v.cpu().numpy() for key, v in o.items()}
        n_diff = _check_against_workspace_route(got, ref, gaps, E)
        if T <= 64:                          # same kernels, same order: identical
            assert n_diff == 0
            assert np.array_equal(got["topk_w"], ref["topk_w"])
    assert layer.sync_status() == moe.MOE_OK


def test_static_scratch_rejects_sizes_beyond_its_array():
    # Refused before anything is launched: 64 tokens with H = 16384 and 256 experts need
    # 64 x 64 x 256 x 4 B of partial logits (4 MiB), and 131,008 tokens need 2047 blocks x 1 KB of
    # per-block expert counts, both more than the 2 MiB array; 64 tokens with H = 2880 and
    # 256 experts (12 slices: 768 KiB) and 130,944 tokens with 256 experts (2046 KiB) fit.
    assert moe.moe_route_static_max_bytes() == 2 << 20
    for E, T, H, ok in ((256, 64, 2880, True), (256, 64, 16384, False),
                        (256, 130944, 64, True), (256, 131008, 64, False)):
        layer = moe.Moe(E, H, 64, 4)
        d = mi.make_inputs(T, H, E, 4, 64, seed=7, device="cuda", experts=False)
        o = _outputs(T, 4, E)
        st = _call_static(layer, d, o)
        assert st == (moe.MOE_OK if ok else moe.MOE_ERR_WORKSPACE), (E, T)
    torch.cuda.synchronize()
