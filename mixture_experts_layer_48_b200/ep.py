"""Expert parallelism: the MoE layer with its E experts split over the G GPUs of a process group.

One process per GPU (torch.distributed, NCCL over NVLink / NVSwitch).  GPU g owns experts
[g*E/G, (g+1)*E/G) and holds only their weights; every GPU keeps the router and its own tokens.
A forward pass on GPU g:

  1. route its tokens over all E experts                       moe_route    (full handle)
  2. put the routed rows in expert order, with their weights   moe_permute  (full handle)
  3. dispatch: the rows of the experts GPU p owns are the contiguous run
     x_perm[offsets[p*E/G] : offsets[(p+1)*E/G]]; one all-to-all exchanges the per-expert row
     counts (E/G ints per peer), one all-to-all the rows (sizes from the counts), one their
     routing weights
  4. its experts on the rows it received, grouped as (source GPU, expert) segments
                                                                moe_experts  (local handle)
  5. combine: one all-to-all sends every weighted result back to the row's home GPU, in the
     order the rows left, then each token adds its k results  moe_combine  (full handle)

The exchange sizes come from the histogram, so the host reads 2*G integers per call (NCCL's
all-to-all takes its split sizes on the host).  The row exchange carries bf16 bit patterns in
pairs as int32, so any backend moves them unchanged.  No multicast loads are involved: each rank's
kernels read only their own GPU's memory; the transfers are NCCL's.

The pages ran every expert on every GPU (Persona Kappa forum post, "The Config":
expert-parallel degree 1).  Splitting them divides the expert weight bytes each GPU streams in
decode by G, at the cost of the two exchanges.

The device work is done by an ``ops`` object (default: :class:`CudaOps`, the library's
kernels); the exchange logic here does not depend on it.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


class CudaOps:
    """The device work of an expert-parallel layer, on the library's kernels."""

    def __init__(self, E: int, H: int, I: int, k: int, E_local: int):
        from . import Moe
        self.full = Moe(E, H, I, k)          # router over all experts, permute, combine
        self.local = Moe(E_local, H, I, k)   # this GPU's experts

    def route(self, x, W_router, b_router) -> dict:
        return self.full.route(x, W_router, b_router)

    def permute(self, x, r):
        return self.full.permute(x, r)

    def experts(self, x_rows, row_w, seg_counts, W_gate_up_local, W_down_local):
        return self.local.experts(x_rows, row_w, seg_counts, W_gate_up_local, W_down_local)

    def combine(self, inv_perm, y_rows):
        return self.full.combine(inv_perm, y_rows)


def expert_range(E: int, G: int, g: int) -> tuple[int, int]:
    """Experts [first, last) owned by rank g of G (contiguous blocks of E/G)."""
    if E % G:
        raise ValueError(f"{E} experts do not split evenly over {G} ranks")
    n = E // G
    return g * n, (g + 1) * n


def split_sizes(counts: torch.Tensor, G: int) -> list[int]:
    """Rows per owner rank from per-expert row counts [E] (contiguous expert blocks)."""
    return [int(v) for v in counts.reshape(G, -1).sum(dim=1).tolist()]


def _a2a(out: torch.Tensor, inp: torch.Tensor, out_splits, in_splits, group) -> torch.Tensor:
    """all_to_all_single on raw elements: bf16 rows (an even number of elements, H % 64 == 0)
    travel as pairs of bit patterns in int32, which every backend moves unchanged."""
    src = inp.contiguous().view(torch.int32) if inp.dtype == torch.bfloat16 else inp
    dst = out.view(torch.int32) if out.dtype == torch.bfloat16 else out
    dist.all_to_all_single(dst, src.contiguous(), output_split_sizes=out_splits,
                           input_split_sizes=in_splits, group=group)
    return out


class ExpertParallelMoe:
    """One expert-parallel MoE layer.  Weights passed to :meth:`forward` are this rank's experts
    only: W_gate_up_local [E/G, H, 2I], W_down_local [E/G, I, H]."""

    def __init__(self, E: int, H: int, I: int, k: int, group=None, ops=None):
        self.E, self.H, self.I, self.k = E, H, I, k
        self.group = group
        self.G = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.first, self.last = expert_range(E, self.G, self.rank)
        self.E_local = self.last - self.first
        self.ops = ops if ops is not None else CudaOps(E, H, I, k, self.E_local)
        self.last_exchange: dict = {}

    def forward(self, x, W_router, b_router, W_gate_up_local, W_down_local) -> torch.Tensor:
        G, El, grp = self.G, self.E_local, self.group
        r = self.ops.route(x, W_router, b_router)
        x_perm, row_w = self.ops.permute(x, r)
        counts = torch.diff(r["expert_offsets"].to(torch.int64)).to(torch.int32)      # [E]
        # per-expert counts to their owners: recv[s, e] = rows of local expert e from rank s
        recv_counts = torch.empty((G, El), dtype=torch.int32, device=counts.device)
        dist.all_to_all_single(recv_counts, counts.reshape(G, El).contiguous(), group=grp)
        send_rows = split_sizes(counts, G)
        recv_rows = [int(v) for v in recv_counts.sum(dim=1).tolist()]
        dev = x_perm.device
        x_recv = torch.empty((sum(recv_rows), self.H), dtype=x_perm.dtype, device=dev)
        w_recv = torch.empty((sum(recv_rows),), dtype=row_w.dtype, device=dev)
        _a2a(x_recv, x_perm, recv_rows, send_rows, grp)
        _a2a(w_recv, row_w, recv_rows, send_rows, grp)
        y_recv = self.ops.experts(x_recv, w_recv, recv_counts, W_gate_up_local, W_down_local)
        y_back = torch.empty((x_perm.shape[0], self.H), dtype=y_recv.dtype, device=dev)
        _a2a(y_back, y_recv, send_rows, recv_rows, grp)
        self.last_exchange = dict(send_rows=send_rows, recv_rows=recv_rows,
                                  recv_counts=recv_counts.cpu())
        return self.ops.combine(r["inv_perm"], y_back)

    __call__ = forward
