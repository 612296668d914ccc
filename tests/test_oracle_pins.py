"""Pins the fp64 oracle to things other than itself (CPU only).

* brute force: pure-Python loops (no numpy) on tiny inputs, with their own bf16 decoding,
  their own top-k (repeated arg-max) and their own exp-based SwiGLU;
* a hand-computed 2-token, 4-expert layer whose expected values are closed forms in the
  logistic function (it has a three-way tie and two empty experts);
* library special cases: k = E gives the full softmax (scipy), E = 1 / k = 1 gives a dense
  SwiGLU MLP (numpy matmul + scipy expit), torch's own bf16 -> float conversion;
* invariants: weights sum to 1, each token appears k times, histogram sums to T*k,
  perm[inv_perm] is the identity, segments ascend;
* planted mistakes: each plausible error planted in the oracle makes one of these fail.
"""
import math
import struct

import numpy as np
import pytest
import scipy.special
import torch

import moe_inputs as mi
import oracle
from oracle import moe_ref


# ----------------------------------------------------------------------------------------
# pure-Python brute force
# ----------------------------------------------------------------------------------------
def py_bf16(bits: int) -> float:
    return struct.unpack(">f", struct.pack(">I", (int(bits) & 0xFFFF) << 16))[0]


def py_layer(x, Wr, br, Wgu, Wd, k):
    """Lists of Python floats in, routing and output out. No numpy anywhere."""
    T, H, E, I = len(x), len(x[0]), len(Wr[0]), len(Wd[0])
    res = dict(idx=[], w=[], out=[])
    for t in range(T):
        logit = [sum(x[t][h] * Wr[h][e] for h in range(H)) + br[e] for e in range(E)]
        chosen = []
        for _ in range(k):  # repeated arg-max; strict '>' keeps the lower index on ties
            best = None
            for e in range(E):
                if e in chosen:
                    continue
                if best is None or logit[e] > logit[best]:
                    best = e
            chosen.append(best)
        m = logit[chosen[0]]
        z = [math.exp(logit[e] - m) for e in chosen]
        w = [v / sum(z) for v in z]
        out = [0.0] * H
        for j, e in enumerate(chosen):
            hvec = []
            for i in range(I):
                g = sum(x[t][h] * Wgu[e][h][i] for h in range(H))
                u = sum(x[t][h] * Wgu[e][h][I + i] for h in range(H))
                hvec.append(g / (1.0 + math.exp(-g)) * u)
            for c in range(H):
                out[c] += w[j] * sum(hvec[i] * Wd[e][i][c] for i in range(I))
        res["idx"].append(chosen)
        res["w"].append(w)
        res["out"].append(out)
    count = [0] * E
    for t in range(T):
        for e in res["idx"][t]:
            count[e] += 1
    offsets = [0]
    for e in range(E):
        offsets.append(offsets[-1] + count[e])
    perm, inv = [None] * (T * k), [[None] * k for _ in range(T)]
    fill = offsets[:-1][:]
    for t in range(T):          # ascending t: a stable counting sort
        for j, e in enumerate(res["idx"][t]):
            perm[fill[e]] = t
            inv[t][j] = fill[e]
            fill[e] += 1
    res.update(count=count, offsets=offsets, perm=perm, inv_perm=inv)
    return res


def tiny_case(T, H, E, k, I, seed):
    d = mi.make_inputs(T, H, E, k, I, seed, "cpu")
    return mi.host_inputs(d)


def to_py(bits2d):
    return [[py_bf16(v) for v in row] for row in bits2d]


def check_against_brute(h, orc=oracle):
    x, Wr, br = h["x"], h["W_router"], h["b_router"]
    Wgu, Wd, k = h["W_gate_up"], h["W_down"], h["k"]
    ref = py_layer(to_py(x), to_py(Wr), [float(v) for v in br],
                   [to_py(Wgu[e]) for e in range(Wgu.shape[0])],
                   [to_py(Wd[e]) for e in range(Wd.shape[0])], k)
    r = orc.moe_route_ref(x, Wr, br, k)
    out = orc.moe_forward_ref(x, Wr, br, Wgu, Wd, k)
    assert r["idx"].tolist() == ref["idx"]
    np.testing.assert_allclose(r["w"], np.array(ref["w"]), rtol=1e-12, atol=1e-15)
    assert r["count"].tolist() == ref["count"]
    assert r["offsets"].tolist() == ref["offsets"]
    assert r["perm"].tolist() == ref["perm"]
    assert r["inv_perm"].tolist() == ref["inv_perm"]
    np.testing.assert_allclose(out, np.array(ref["out"]), rtol=1e-10, atol=1e-12)


BRUTE_CASES = [
    # T, H, E, k, I, seed
    (5, 8, 4, 2, 8, 11),
    (7, 6, 5, 3, 4, 12),
    (3, 4, 3, 3, 2, 13),
    (6, 8, 6, 1, 3, 14),
    (1, 5, 2, 2, 5, 15),
]


@pytest.mark.parametrize("case", BRUTE_CASES)
def test_oracle_matches_brute_force(case):
    check_against_brute(tiny_case(*case))


def test_bf16_decoding_matches_torch_everywhere():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    mine = oracle.decode_bf16(bits)
    lib = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], lib[~nan])
    # also against the pure-Python decoding on a few patterns
    for b in (0x0000, 0x8000, 0x3F80, 0xBF80, 0x4049, 0x0001, 0x7F7F, 0xFF7F):
        assert oracle.decode_bf16(np.array([b], np.uint16))[0] == py_bf16(b)


# ----------------------------------------------------------------------------------------
# hand-computed example (closed forms in the logistic function)
# ----------------------------------------------------------------------------------------
def bf16_from_values(a):
    t = torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)
    assert torch.equal(t.to(torch.float32), torch.tensor(np.asarray(a, dtype=np.float32)))
    return mi.bf16_bits(t)


def hand_example():
    x = bf16_from_values([[1, 0], [0, 1]])
    Wr = bf16_from_values([[1, 2, 3, 0], [0, 2, 2, 2]])
    br = np.zeros(4, np.float32)
    # W_gate_up[e] = [[gate_h0, up_h0], [gate_h1, up_h1]]  (H = 2, I = 1)
    Wgu = bf16_from_values([[[-1, 1], [1, -1]], [[1, 1], [0, 0]], [[2, 1], [1, 1]], [[0, 0], [2, 1]]])
    Wd = bf16_from_values([[[3, 3]], [[1, 1]], [[1, -1]], [[0, 1]]])
    return x, Wr, br, Wgu, Wd, 2


def sig(z):
    return 1.0 / (1.0 + math.exp(-z))


def check_hand_example(orc=oracle):
    x, Wr, br, Wgu, Wd, k = hand_example()
    r = orc.moe_route_ref(x, Wr, br, k)
    out = orc.moe_forward_ref(x, Wr, br, Wgu, Wd, k)
    # token 0: logits [1,2,3,0] -> experts (2,1), weights (sig(1), 1-sig(1))
    # token 1: logits [0,2,2,2] -> three-way tie -> experts (1,2), weights (1/2, 1/2)
    assert r["idx"].tolist() == [[2, 1], [1, 2]]
    np.testing.assert_allclose(r["w"], [[sig(1), 1 - sig(1)], [0.5, 0.5]], rtol=0, atol=1e-15)
    assert r["count"].tolist() == [0, 2, 2, 0]
    assert r["offsets"].tolist() == [0, 0, 2, 4, 4]
    assert r["perm"].tolist() == [0, 1, 0, 1]
    assert r["inv_perm"].tolist() == [[2, 0], [1, 3]]
    # token 0: expert 2 has g=2,u=1 -> h=2 sig(2), y=h*[1,-1]; expert 1 has g=u=1 -> h=sig(1), y=h*[1,1]
    h2, h1 = 2 * sig(2), sig(1)
    o0 = [sig(1) * h2 + (1 - sig(1)) * h1, -sig(1) * h2 + (1 - sig(1)) * h1]
    # token 1: expert 1 has g=u=0 -> 0; expert 2 has g=u=1 -> h=sig(1), y=h*[1,-1]
    o1 = [0.5 * sig(1), -0.5 * sig(1)]
    np.testing.assert_allclose(out, [o0, o1], rtol=0, atol=1e-14)
    # the printed decimals of the worked example
    np.testing.assert_allclose(out, [[1.484440453, -1.091216587], [0.365529289, -0.365529289]],
                               atol=5e-9)


def test_hand_example():
    check_hand_example()


# ----------------------------------------------------------------------------------------
# library special cases
# ----------------------------------------------------------------------------------------
def test_k_equals_E_is_full_softmax():
    h = tiny_case(9, 16, 6, 6, 4, 21)
    r = oracle.moe_route_ref(h["x"], h["W_router"], h["b_router"], 6)
    full = scipy.special.softmax(r["logits"], axis=1)
    np.testing.assert_allclose(r["w"], np.take_along_axis(full, r["idx"], 1), rtol=1e-12)
    assert sorted(r["idx"][0].tolist()) == list(range(6))
    assert np.all(np.diff(np.take_along_axis(r["logits"], r["idx"], 1), axis=1) <= 0)


def test_single_expert_is_dense_swiglu_mlp():
    h = tiny_case(10, 16, 1, 1, 12, 22)
    out = oracle.moe_forward_ref(h["x"], h["W_router"], h["b_router"], h["W_gate_up"], h["W_down"], 1)
    x = torch.from_numpy(h["x"].view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    W = torch.from_numpy(h["W_gate_up"][0].view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    Wd = torch.from_numpy(h["W_down"][0].view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    g, u = x @ W[:, :12], x @ W[:, 12:]
    dense = (g * scipy.special.expit(g) * u) @ Wd
    np.testing.assert_allclose(out, dense, rtol=1e-12, atol=1e-14)


def test_all_equal_logits_pick_lowest_indices_with_equal_weights():
    T, H, E, k = 4, 8, 7, 3
    x = mi.bf16_bits(torch.randn(T, H).to(torch.bfloat16))
    Wr = np.zeros((H, E), np.uint16)  # bf16 zero
    r = oracle.moe_route_ref(x, Wr, np.zeros(E, np.float32), k)
    assert r["idx"].tolist() == [[0, 1, 2]] * T
    np.testing.assert_allclose(r["w"], 1.0 / k, rtol=0, atol=1e-15)
    assert r["count"].tolist() == [T, T, T, 0, 0, 0, 0]
    assert r["perm"].tolist() == list(range(T)) * 3


def test_selection_gaps_against_brute():
    rng = np.random.default_rng(5)
    l = rng.standard_normal((20, 9))
    for k in (1, 3, 9):
        gk, gi = oracle.selection_gaps(l, k)
        for t in range(20):
            s = sorted(l[t].tolist(), reverse=True)
            assert gk[t] == (math.inf if k == 9 else s[k - 1] - s[k])
            assert gi[t] == (math.inf if k == 1 else min(s[j] - s[j + 1] for j in range(k - 1)))


# ----------------------------------------------------------------------------------------
# invariants at a moderate size
# ----------------------------------------------------------------------------------------
@pytest.mark.parametrize("T,E,k", [(300, 8, 2), (257, 32, 4), (64, 128, 4), (33, 5, 5)])
def test_routing_invariants(T, E, k):
    h = tiny_case(T, 64, E, k, 8, 30 + E)
    r = oracle.moe_route_ref(h["x"], h["W_router"], h["b_router"], k)
    idx, perm, inv = r["idx"], r["perm"], r["inv_perm"]
    np.testing.assert_allclose(r["w"].sum(1), 1.0, rtol=0, atol=1e-12)
    assert np.all(r["w"][:, :-1] >= r["w"][:, 1:])
    assert r["count"].sum() == T * k
    assert np.array_equal(np.bincount(perm, minlength=T), np.full(T, k))
    assert np.array_equal(perm[inv], np.repeat(np.arange(T)[:, None], k, 1))
    assert np.array_equal(np.sort(inv.ravel()), np.arange(T * k))
    for t in range(T):
        assert len(set(idx[t].tolist())) == k
        rest = np.setdiff1d(np.arange(E), idx[t])
        if rest.size:
            assert r["logits"][t, idx[t]].min() >= r["logits"][t, rest].max()
    for e in range(E):
        seg = perm[r["offsets"][e]: r["offsets"][e + 1]]
        assert np.all(np.diff(seg) > 0)
        assert np.all(np.any(idx[seg] == e, axis=1))


def _brute_logits(h, rows):
    """Pure-Python logits of the given token rows (own bf16 decoding, plain loops)."""
    x, Wr, br = h["x"], h["W_router"], h["b_router"]
    H, E = Wr.shape
    return [[sum(py_bf16(x[t][c]) * py_bf16(Wr[c][e]) for c in range(H)) + float(br[e])
             for e in range(E)] for t in rows]


def check_chunked_logits(orc=moe_ref):
    """The oracle computes the router logits in token chunks; every chunk size, including ones
    that leave a ragged last chunk, gives the brute-force logits for every row."""
    h = tiny_case(17, 6, 4, 2, 4, 51)
    brute = np.array(_brute_logits(h, range(17)))
    for chunk in (1, 4, 5, 16, 17, 64):
        got = orc._logits_chunked(h["x"], h["W_router"], h["b_router"], chunk=chunk)
        np.testing.assert_allclose(got, brute, rtol=1e-13, atol=1e-14)
    # the default chunk (8192 tokens): routing of the rows on both sides of the first boundary
    # and of the one-row tail
    T = 8192 + 1
    h = mi.host_inputs(mi.make_inputs(T, 4, 3, 2, 4, 52, "cpu", experts=False))
    r = orc.moe_route_ref(h["x"], h["W_router"], h["b_router"], 2)
    rows = [0, 8190, 8191, 8192]
    np.testing.assert_allclose(r["logits"][rows], np.array(_brute_logits(h, rows)),
                               rtol=1e-13, atol=1e-14)
    for i, t in enumerate(rows):
        lg = r["logits"][t]
        best = sorted(range(3), key=lambda e: (-lg[e], e))[:2]
        assert r["idx"][t].tolist() == best


def test_chunked_router_logits_across_chunk_boundaries():
    check_chunked_logits()


def test_token_subset_equals_full_rows():
    h = tiny_case(40, 32, 6, 2, 16, 41)
    args = (h["x"], h["W_router"], h["b_router"], h["W_gate_up"], h["W_down"], 2)
    full = oracle.moe_forward_ref(*args)
    toks = np.array([0, 7, 8, 39])
    np.testing.assert_allclose(oracle.moe_forward_ref(*args, tokens=toks), full[toks],
                               rtol=1e-13, atol=1e-15)
    r = oracle.moe_route_ref(*args[:3], 2)
    for t in toks:
        one = oracle.moe_token_output_ref(h["x"][t], r["logits"][t], r["idx"][t],
                                          h["W_gate_up"], h["W_down"])
        np.testing.assert_allclose(one, full[t], rtol=1e-12, atol=1e-14)


def test_zipf_scale_gives_fourfold_max_over_mean_load():
    w = mi.WORKLOADS["131k_skewed"]
    x = mi.draw_x(4096, w.H, w.seed, "cpu")
    Wr, b = mi.draw_router(w.H, w.E, w.seed, "cpu", zipf=True)
    r = oracle.moe_route_ref(mi.bf16_bits(x), mi.bf16_bits(Wr), b.numpy(), w.k)
    ratio = r["count"].max() / r["count"].mean()
    assert abs(ratio - 4.0) <= 0.1, ratio


# ----------------------------------------------------------------------------------------
# planted mistakes: each must be caught by the pins above
# ----------------------------------------------------------------------------------------
def _gate_up_swapped(xrows, Wgu, Wd):
    I = Wd.shape[0]
    gu = xrows @ Wgu
    return moe_ref.swiglu(gu[:, I:], gu[:, :I]) @ Wd


def _softmax_over_all(logits, idx):
    z = np.exp(logits - logits.max(1, keepdims=True))
    z = z / z.sum(1, keepdims=True)
    return np.take_along_axis(z, idx, 1)


def _ties_to_higher(logits, k):
    E = logits.shape[1]
    order = np.argsort(-logits[:, ::-1], axis=1, kind="stable")
    return (E - 1 - order)[:, :k]


def _unstable_perm(idx, E):
    perm, inv = _ORIG_PERM(idx, E)
    off = moe_ref.expert_offsets(moe_ref.expert_histogram(idx, E))
    perm2, inv2 = perm.copy(), inv.copy()
    for e in range(E):
        a, b = off[e], off[e + 1]
        perm2[a:b] = perm[a:b][::-1]
        for r in range(a, b):
            t = perm[r]
            inv2[t][idx[t] == e] = a + b - 1 - r
    return perm2, inv2


def _silu_sign(z):
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(z))


def _no_bias(x, W, b):
    return x @ W


def _weights_unnormalised(logits, idx):
    sel = np.take_along_axis(logits, idx, axis=1)
    return np.exp(sel - sel[:, :1])


def _down_transposed(xrows, Wgu, Wd):
    I = Wd.shape[0]
    gu = xrows @ Wgu
    hh = moe_ref.swiglu(gu[:, :I], gu[:, I:])
    return hh @ Wd[::-1, :]   # rows of W_down taken in the wrong order


_ORIG_PERM = moe_ref.permutation


def _chunk_tail_dropped(x_bits, W_router_bits, b_router, chunk=8192):
    Wr = moe_ref.decode_bf16(W_router_bits)
    b = np.asarray(b_router, dtype=np.float32).astype(np.float64)
    T = x_bits.shape[0]
    out = np.zeros((T, Wr.shape[1]))
    for t0 in range(0, T - T % chunk, chunk):        # the ragged last chunk is skipped
        out[t0:t0 + chunk] = moe_ref.router_logits(moe_ref.decode_bf16(x_bits[t0:t0 + chunk]), Wr, b)
    return out


def _chunk_bias_once(x_bits, W_router_bits, b_router, chunk=8192):
    Wr = moe_ref.decode_bf16(W_router_bits)
    b = np.asarray(b_router, dtype=np.float32).astype(np.float64)
    T = x_bits.shape[0]
    out = np.empty((T, Wr.shape[1]))
    for t0 in range(0, T, chunk):                     # bias added to the first chunk only
        out[t0:t0 + chunk] = moe_ref.router_logits(moe_ref.decode_bf16(x_bits[t0:t0 + chunk]), Wr,
                                                   b if t0 == 0 else 0 * b)
    return out


CHUNK_MUTANTS = {"chunk_tail_dropped": _chunk_tail_dropped, "chunk_bias_once": _chunk_bias_once}


@pytest.mark.parametrize("name", sorted(CHUNK_MUTANTS))
def test_planted_chunking_mistake_is_caught(name, monkeypatch):
    monkeypatch.setattr(moe_ref, "_logits_chunked", CHUNK_MUTANTS[name])
    with pytest.raises(AssertionError):
        check_chunked_logits(moe_ref)

MUTANTS = {
    "gate_up_swapped": ("expert_mlp", _gate_up_swapped),
    "softmax_over_all_experts": ("routing_weights", _softmax_over_all),
    "ties_to_higher_index": ("topk_select", _ties_to_higher),
    "unstable_permutation": ("permutation", _unstable_perm),
    "silu_sign": ("silu", _silu_sign),
    "dropped_bias": ("router_logits", _no_bias),
    "weights_unnormalised": ("routing_weights", _weights_unnormalised),
    "down_rows_misindexed": ("expert_mlp", _down_transposed),
}


def _pins_pass() -> bool:
    try:
        check_hand_example(moe_ref)
        for case in BRUTE_CASES[:2]:
            check_against_brute(tiny_case(*case), moe_ref)
    except AssertionError:
        return False
    return True


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, monkeypatch):
    fn_name, mutant = MUTANTS[name]
    monkeypatch.setattr(moe_ref, fn_name, mutant)
    assert not _pins_pass(), f"planted mistake {name} went unnoticed"


def test_unplanted_oracle_passes_the_same_checks():
    assert _pins_pass()
