"""Expert parallelism on CPU: two gloo ranks run the layer with the experts split between them
(ExpertParallelMoe: per-expert count exchange, row dispatch, local experts, results back,
combine), with the device work done by the fp64 oracle.  Each rank's routing must equal the
oracle's bit for bit, every rank must receive exactly the rows its experts own, and each rank's
output must equal the single-rank oracle layer on its tokens (to fp64 rounding: the combine adds
the k results in slot order, the oracle in expert order)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import moe_inputs as mi
import oracle


class OracleOps:
    """Device work of an expert-parallel layer, in float64 on the host (test only)."""

    def __init__(self, E, H, I, k, first):
        self.E, self.H, self.I, self.k, self.first = E, H, I, k, first

    def route(self, x, W_router, b_router):
        r = oracle.moe_route_ref(x.view(torch.int16).numpy().view(np.uint16),
                                 W_router.view(torch.int16).numpy().view(np.uint16),
                                 b_router.numpy(), self.k)
        return dict(topk_idx=torch.from_numpy(r["idx"]).to(torch.int32),
                    topk_w=torch.from_numpy(r["w"]),
                    expert_offsets=torch.from_numpy(r["offsets"]).to(torch.int32),
                    perm=torch.from_numpy(r["perm"]).to(torch.int32),
                    inv_perm=torch.from_numpy(r["inv_perm"]).to(torch.int32))

    def permute(self, x, r):
        perm = r["perm"].long()
        x_perm = x[perm].contiguous()
        row_w = torch.empty(perm.numel(), dtype=torch.float64)
        inv = r["inv_perm"].long()
        row_w[inv.reshape(-1)] = r["topk_w"].reshape(-1)
        return x_perm, row_w

    def experts(self, x_rows, row_w, seg_counts, Wgu_local, Wdn_local):
        bits = x_rows.view(torch.int16).numpy().view(np.uint16)
        y = np.zeros((x_rows.shape[0], self.H))
        S, El = seg_counts.shape
        r0 = 0
        for s in range(S):
            for e in range(El):
                n = int(seg_counts[s, e])
                if n:
                    xs = oracle.decode_bf16(bits[r0:r0 + n])
                    gu = oracle.decode_bf16(Wgu_local[e].view(torch.int16).numpy().view(np.uint16))
                    dn = oracle.decode_bf16(Wdn_local[e].view(torch.int16).numpy().view(np.uint16))
                    y[r0:r0 + n] = row_w[r0:r0 + n].numpy()[:, None] * oracle.expert_mlp(xs, gu, dn)
                r0 += n
        assert r0 == x_rows.shape[0]
        return torch.from_numpy(y)

    def combine(self, inv_perm, y_rows):
        inv = inv_perm.long()
        out = torch.zeros((inv.shape[0], self.H), dtype=torch.float64)
        for j in range(inv.shape[1]):
            out += y_rows[inv[:, j]]
        return out


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, shape, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from mixture_experts_layer_48_b200 import ep
        T, H, E, k, I = shape
        d = mi.make_inputs(T * world, H, E, k, I, seed=77, device="cpu")
        x_all = d["x"]
        x = x_all[rank * T:(rank + 1) * T].contiguous()          # this rank's tokens
        first, last = ep.expert_range(E, world, rank)
        layer = ep.ExpertParallelMoe(E, H, I, k, ops=OracleOps(E, H, I, k, first))
        out = layer(x, d["W_router"], d["b_router"], d["W_gate_up"][first:last],
                    d["W_down"][first:last])
        h = mi.host_inputs(d)
        xb = h["x"][rank * T:(rank + 1) * T]
        route = oracle.moe_route_ref(xb, h["W_router"], h["b_router"], k)
        ref = oracle.moe_forward_ref(xb, h["W_router"], h["b_router"], h["W_gate_up"], h["W_down"],
                                     k, route=route)
        err = float(np.abs(out.numpy() - ref).max() / max(1e-300, np.abs(ref).max()))
        # rows this rank's experts own, summed over every rank's tokens
        full = oracle.moe_route_ref(h["x"], h["W_router"], h["b_router"], k)
        owned = int(full["count"][first:last].sum())
        q.put((rank, err, layer.last_exchange["recv_rows"], owned,
               layer.last_exchange["recv_counts"].numpy().tolist(),
               route["count"].tolist(), None))
    except Exception as e:  # report, do not hang the other rank's queue read
        q.put((rank, None, None, None, None, None, repr(e)))
        raise
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("shape", [(24, 64, 8, 2, 32), (40, 128, 6, 3, 64)])
def test_two_rank_expert_parallel_layer_matches_the_oracle(shape):
    T, H, E, k, I = shape
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, shape, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=120)
    for rank, err, recv_rows, owned, recv_counts, counts, exc in res:
        assert exc is None, exc
        assert err <= 1e-12, (rank, err)
        assert sum(recv_rows) == owned, (rank, recv_rows, owned)
    assert all(p.exitcode == 0 for p in procs)
    # the count exchange: what rank s sent to rank g is rank s's histogram over g's experts
    El = E // 2
    for g, _, _, _, recv_counts, _, _ in res:
        for s in range(2):
            assert recv_counts[s] == res[s][5][g * El:(g + 1) * El]


def test_expert_ranges_and_split_sizes():
    from mixture_experts_layer_48_b200 import ep
    assert [ep.expert_range(32, 4, g) for g in range(4)] == [(0, 8), (8, 16), (16, 24), (24, 32)]
    with pytest.raises(ValueError):
        ep.expert_range(30, 4, 0)
    c = torch.tensor([3, 0, 2, 5, 1, 1, 0, 4])
    assert ep.split_sizes(c, 2) == [10, 6] and ep.split_sizes(c, 4) == [3, 7, 2, 4]
