"""Oracle for the top-k routed SwiGLU Mixture-of-Experts layer forward pass.

TEST INFRASTRUCTURE ONLY.  This module is the slow, plain CPU definition that the CUDA
library is checked against.  Only the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import it.  It shares no code with the CUDA path and
imports nothing from it.

What it computes (all arithmetic in numpy float64, from the bf16 bit patterns the GPU reads,
each bf16 value widened exactly):

* router logits      l[t,e] = sum_h x[t,h] * W_router[h,e] + b_router[e].  The layer is a
    mixture of SwiGLU experts that routes each token to 4 of 32 experts (Persona Kappa forum
    post, "Architecture Summary" table and "Notable Details"; kappa-20b-131k model card,
    "Model Details" table), 4 of 128 for the 120b body (hearth-lean-loomed-v1 card, intro).
* top-k selection     the k largest logits of each token, largest first; equal logits are
    ordered by the lower expert index.  The pages name top-4 routing only; the tie rule is
    this library's stated reading.
* routing weights     softmax over the k selected logits only.
* histogram / offsets / permutation   count of rows per expert, its exclusive prefix sum,
    and the stable token-to-row map: inside an expert's segment rows are in ascending token
    order.  Per-expert dispatch of a few tokens each is the regime the hearth-lean-loomed-v1
    card discusses ("Why 12-16 streams can be slow on Vulkan").
* expert MLP          g = x W_gate_up[e][:, :I],  u = x W_gate_up[e][:, I:],
    h = silu(g) * u with silu(z) = z / (1 + exp(-z)),  y = h W_down[e].  The pages name the
    SwiGLU expert but print no formula; this is its plain form.
* combine             out[t] = sum_j w[t,j] * y_(t, S_j)   in float64.

MXFP4 expert weights (W4A16).  The checkpoints' experts are natively MXFP4 with bf16
activations (Persona Kappa forum post, "Quantization-Aware Training"; kappa-20b-131k card,
"Architecture"); the pages name the format only.  This oracle reads it as the OCP Microscaling
(MX) v1.0 FP4 format: E2M1 elements (sign, 2 exponent bits with bias 1, 1 mantissa bit;
exponent 0 is subnormal) in blocks of 32 consecutive elements along the reduction dimension,
each block sharing one E8M0 scale 2^(s-127) (s = 255 encodes NaN).  Storage of one expert's
[K, N] matrix: ``codes [N, K/2]`` uint8 (byte j of row n holds element k = 2j in bits 0-3 and
k = 2j + 1 in bits 4-7) and ``scales [K/32, N]`` uint8.  The dequantized weights then enter the
same float64 layer as the bf16 ones.

Nothing is rounded between steps: the GPU rounds the SwiGLU output h to bf16 before the down
projection and accumulates in fp32; those differences are what the tests' tolerance covers.

Each function is pinned by the CPU tests against brute force on tiny inputs, closed forms, a
hand-computed example, invariants and library special cases.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "decode_bf16",
    "router_logits",
    "topk_select",
    "routing_weights",
    "selection_gaps",
    "expert_histogram",
    "expert_offsets",
    "permutation",
    "silu",
    "swiglu",
    "expert_mlp",
    "moe_route_ref",
    "moe_forward_ref",
    "moe_token_output_ref",
    "decode_e2m1",
    "decode_e8m0",
    "dequant_mxfp4",
    "moe_forward_mxfp4_ref",
]


def decode_bf16(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16 / int16 array) exactly to float64.

    A bfloat16 is the upper 16 bits of an IEEE binary32, so placing the pattern in the top
    half of a 32-bit word gives the same number as a float32, which float64 holds exactly.
    """
    b = np.asarray(bits)
    if b.dtype not in (np.uint16, np.int16):
        raise TypeError(f"bf16 bit patterns must be uint16/int16, got {b.dtype}")
    u32 = b.view(np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):  # NaN patterns stay NaN
        return u32.view(np.float32).astype(np.float64)


def router_logits(x: np.ndarray, W_router: np.ndarray, b_router: np.ndarray) -> np.ndarray:
    """l[t,e] = sum_h x[t,h] W_router[h,e] + b_router[e]; x [T,H], W_router [H,E], b [E] (float64)."""
    return x @ W_router + b_router[None, :]


def topk_select(logits: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest logits per row, largest first, equal values by lower index.

    A stable sort of the negated logits keeps equal values in ascending index order.
    """
    order = np.argsort(-logits, axis=1, kind="stable")
    return order[:, :k].astype(np.int64)


def routing_weights(logits: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """Softmax over the selected logits only: w[t,j] = exp(l_j - l_0) / sum_j' exp(l_j' - l_0).

    l_0 is the largest selected logit (slot 0), which keeps every exponent <= 0.
    """
    sel = np.take_along_axis(logits, idx, axis=1)
    z = np.exp(sel - sel[:, :1])
    return z / z.sum(axis=1, keepdims=True)


def selection_gaps(logits: np.ndarray, k: int) -> tuple[np.ndarray, np.ndarray]:
    """Per token: (gap between the k-th and (k+1)-th largest logit, smallest gap inside the top k).

    The first decides whether the selected set is well separated from the rest (inf when k = E);
    the second whether the order of the selected slots is (inf when k = 1).
    """
    T, E = logits.shape
    s = -np.sort(-logits, axis=1)
    gap_k = np.full(T, np.inf) if k >= E else s[:, k - 1] - s[:, k]
    gap_in = np.full(T, np.inf) if k == 1 else np.min(s[:, : k - 1] - s[:, 1:k], axis=1)
    return gap_k, gap_in


def expert_histogram(idx: np.ndarray, E: int) -> np.ndarray:
    """count[e] = number of (token, slot) pairs routed to expert e."""
    return np.bincount(idx.ravel(), minlength=E).astype(np.int64)


def expert_offsets(count: np.ndarray) -> np.ndarray:
    """Exclusive prefix sum with the total appended: offsets[0] = 0, offsets[e+1] = offsets[e] + count[e]."""
    return np.concatenate([[0], np.cumsum(count)]).astype(np.int64)


def permutation(idx: np.ndarray, E: int) -> tuple[np.ndarray, np.ndarray]:
    """Stable token-to-row map.

    Rows are grouped by expert (expert 0's segment first).  Inside a segment the tokens routed
    to that expert appear in ascending token order.  perm[r] = token of row r;
    inv_perm[t, j] = row that holds token t's slot-j expert.
    """
    T, k = idx.shape
    perm = np.empty(T * k, dtype=np.int64)
    inv_perm = np.empty((T, k), dtype=np.int64)
    r = 0
    for e in range(E):
        tok, slot = np.nonzero(idx == e)  # row-major scan: ascending t
        n = tok.size
        perm[r : r + n] = tok
        inv_perm[tok, slot] = np.arange(r, r + n)
        r += n
    assert r == T * k
    return perm, inv_perm


def silu(z: np.ndarray) -> np.ndarray:
    """silu(z) = z / (1 + exp(-z)); exp overflow for very negative z correctly gives -0."""
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def swiglu(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    """SwiGLU gating: silu(gate) * up."""
    return silu(g) * u


def expert_mlp(xrows: np.ndarray, W_gate_up_e: np.ndarray, W_down_e: np.ndarray) -> np.ndarray:
    """One expert on a block of rows: y = swiglu(x Wg, x Wu) W_down.

    W_gate_up_e is [H, 2I] with the gate in columns [0, I) and the up projection in [I, 2I);
    W_down_e is [I, H].  All float64.
    """
    I = W_down_e.shape[0]
    gu = xrows @ W_gate_up_e
    return swiglu(gu[:, :I], gu[:, I:]) @ W_down_e


def _logits_chunked(x_bits, W_router_bits, b_router, chunk=8192):
    Wr = decode_bf16(W_router_bits)
    b = np.asarray(b_router, dtype=np.float32).astype(np.float64)
    T = x_bits.shape[0]
    out = np.empty((T, Wr.shape[1]), dtype=np.float64)
    for t0 in range(0, T, chunk):
        out[t0 : t0 + chunk] = router_logits(decode_bf16(x_bits[t0 : t0 + chunk]), Wr, b)
    return out


def moe_route_ref(x_bits, W_router_bits, b_router, k: int) -> dict:
    """Routing half of the layer for every token.

    x_bits [T,H] and W_router_bits [H,E] are bf16 bit patterns, b_router [E] float32.
    Returns a dict with logits, idx [T,k], w [T,k], count [E], offsets [E+1], perm [T*k],
    inv_perm [T,k], gap_k [T] and gap_in [T] (see selection_gaps).
    """
    E = W_router_bits.shape[1]
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    logits = _logits_chunked(x_bits, W_router_bits, b_router)
    idx = topk_select(logits, k)
    w = routing_weights(logits, idx)
    count = expert_histogram(idx, E)
    offsets = expert_offsets(count)
    perm, inv_perm = permutation(idx, E)
    gap_k, gap_in = selection_gaps(logits, k)
    return dict(logits=logits, idx=idx, w=w, count=count, offsets=offsets, perm=perm,
                inv_perm=inv_perm, gap_k=gap_k, gap_in=gap_in)


def _layer_out(x_bits, route, tokens, gate_up_of, down_of) -> np.ndarray:
    """out[t] = sum_j w[t,j] * expert_mlp(x[t], e = idx[t,j]); experts come from the getters."""
    T, H = x_bits.shape
    toks = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    idx, w = route["idx"][toks], route["w"][toks]
    xs = decode_bf16(x_bits[toks])
    out = np.zeros((toks.size, H), dtype=np.float64)
    for e in np.unique(idx):
        rows, slots = np.nonzero(idx == e)
        y = expert_mlp(xs[rows], gate_up_of(e), down_of(e))
        out[rows] += w[rows, slots][:, None] * y
    return out


def moe_forward_ref(x_bits, W_router_bits, b_router, W_gate_up_bits, W_down_bits, k: int,
                    tokens=None, route: dict | None = None) -> np.ndarray:
    """Whole layer: out[t] = sum_j w[t,j] * expert_mlp(x[t], e = idx[t,j]) in float64.

    W_gate_up_bits [E,H,2I], W_down_bits [E,I,H] are bf16 bit patterns.  ``tokens`` restricts
    the output to those token indices (routing is still that of the whole batch, which does not
    change a token's result: the layer is token-wise).  Experts are widened to float64 one at a
    time so the largest layers fit in host memory.  Returns out [len(tokens) or T, H].
    """
    if route is None:
        route = moe_route_ref(x_bits, W_router_bits, b_router, k)
    return _layer_out(x_bits, route, tokens, lambda e: decode_bf16(W_gate_up_bits[e]),
                      lambda e: decode_bf16(W_down_bits[e]))


def decode_e2m1(codes) -> np.ndarray:
    """FP4 E2M1 element codes (low 4 bits) to float64.

    Bit 3 is the sign, bits 2-1 the exponent field e (bias 1), bit 0 the mantissa m:
    e = 0 gives the subnormal m * 2^(1-1) * 0.5 = m / 2, otherwise 2^(e-1) * (1 + m / 2).
    """
    c = np.asarray(codes).astype(np.int64) & 0xF
    sign, e, m = c >> 3, (c >> 1) & 3, c & 1
    mag = np.where(e == 0, 0.5 * m, np.ldexp(1.0 + 0.5 * m, e - 1))
    return np.where(sign == 1, -mag, mag)


def decode_e8m0(s) -> np.ndarray:
    """E8M0 shared scale codes to float64: 2^(s - 127), and NaN for s = 255."""
    s = np.asarray(s).astype(np.int64)
    return np.where(s == 255, np.nan, np.ldexp(1.0, np.minimum(s, 254) - 127))


def dequant_mxfp4(codes, scales) -> np.ndarray:
    """MXFP4 matrices to float64: codes [..., N, K/2] uint8, scales [..., K/32, N] uint8 ->
    W [..., K, N] with W[k, n] = e2m1(element k of row n) * 2^(scales[k // 32, n] - 127)."""
    b = np.asarray(codes, dtype=np.uint8)
    elems = np.stack([b & 0xF, b >> 4], axis=-1).reshape(*b.shape[:-1], 2 * b.shape[-1])
    vals = np.swapaxes(decode_e2m1(elems), -1, -2)            # [..., K, N]
    return vals * np.repeat(decode_e8m0(scales), 32, axis=-2)  # scale rows repeat per block


def moe_forward_mxfp4_ref(x_bits, W_router_bits, b_router, gu_codes, gu_scales, dn_codes,
                          dn_scales, k: int, tokens=None, route: dict | None = None) -> np.ndarray:
    """Whole layer with MXFP4 experts: the bf16 layer above on the dequantized weights.

    gu_codes [E, 2I, H/2], gu_scales [E, H/32, 2I] hold W_gate_up [E, H, 2I] (gate columns
    [0, I), up columns [I, 2I)); dn_codes [E, H, I/2], dn_scales [E, I/32, H] hold W_down
    [E, I, H].  Activations and the router stay bf16.
    """
    if route is None:
        route = moe_route_ref(x_bits, W_router_bits, b_router, k)
    return _layer_out(x_bits, route, tokens, lambda e: dequant_mxfp4(gu_codes[e], gu_scales[e]),
                      lambda e: dequant_mxfp4(dn_codes[e], dn_scales[e]))


def moe_token_output_ref(x_bits_t, logits_t, experts, W_gate_up_bits, W_down_bits) -> np.ndarray:
    """One token's output on a GIVEN ordered expert set (used to re-check near-tie tokens).

    The weights are the softmax of this token's float64 logits over ``experts``.
    """
    experts = np.asarray(experts, dtype=np.int64)
    sel = logits_t[experts]
    z = np.exp(sel - sel.max())
    w = z / z.sum()
    xt = decode_bf16(x_bits_t)[None, :]
    out = np.zeros(x_bits_t.shape[-1], dtype=np.float64)
    for j, e in enumerate(experts):
        out += w[j] * expert_mlp(xt, decode_bf16(W_gate_up_bits[e]), decode_bf16(W_down_bits[e]))[0]
    return out
