"""Pins the oracle's MXFP4 weight decoding (CPU only).

The pages name the experts' native format, MXFP4 with bf16 activations (Persona Kappa forum
post, "Quantization-Aware Training"), without defining it; the oracle reads it as the OCP
Microscaling v1.0 FP4 format.  Pinned here against things other than the oracle itself:

* a generic pure-Python minifloat decoder (exact rationals) for E2M1 (2 exponent bits,
  bias 1, 1 mantissa bit, subnormals) and the format's known value set {0, 0.5, ..., 6};
* E8M0 special cases (2^0, the extremes, NaN at 255) and pure-Python powers of two;
* pure-Python element-by-element dequantization (nibble order, block of 32, scale layout);
* the MXFP4 layer equals the already-pinned bf16 layer run on the dequantized weights;
* planted mistakes in the decoding are caught by these checks.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import moe_inputs as mi
from oracle import moe_ref


def py_minifloat(code: int, ebits: int, mbits: int, bias: int) -> Fraction:
    """Sign / exponent / mantissa fields of a (1 + ebits + mbits)-bit float, exactly."""
    sign = (code >> (ebits + mbits)) & 1
    e = (code >> mbits) & ((1 << ebits) - 1)
    m = code & ((1 << mbits) - 1)
    frac = Fraction(m, 1 << mbits)
    if e == 0:
        mag = frac * Fraction(2) ** (1 - bias)
    else:
        mag = (1 + frac) * Fraction(2) ** (e - bias)
    return -mag if sign else mag


def py_dequant(blocks, scales):
    """blocks [N][K/2], scales [K/32][N] (nested lists of ints) -> W [K][N] as floats."""
    N, K = len(blocks), 2 * len(blocks[0])
    W = [[0.0] * N for _ in range(K)]
    for n in range(N):
        for k in range(K):
            byte = blocks[n][k // 2]
            code = (byte >> (4 * (k % 2))) & 0xF
            s = scales[k // 32][n]
            W[k][n] = float(py_minifloat(code, 2, 1, 1)) * math.ldexp(1.0, s - 127)
    return W


def check_e2m1(ref):
    got = ref.decode_e2m1(np.arange(16))
    for c in range(16):
        want = py_minifloat(c, 2, 1, 1)
        assert got[c] == float(want), (c, got[c], want)
        assert math.copysign(1.0, got[c]) == (-1.0 if c >= 8 else 1.0)
    assert sorted(set(np.abs(got).tolist())) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def check_dequant(ref, seed=0):
    rng = np.random.default_rng(seed)
    for E, N, K in ((1, 5, 64), (3, 2, 96)):
        blocks = rng.integers(0, 256, size=(E, N, K // 2)).astype(np.uint8)
        scales = rng.integers(100, 150, size=(E, K // 32, N)).astype(np.uint8)
        got = ref.dequant_mxfp4(blocks, scales)
        assert got.shape == (E, K, N)
        for e in range(E):
            want = np.array(py_dequant(blocks[e].tolist(), scales[e].tolist()))
            np.testing.assert_array_equal(got[e], want)


def test_e2m1_matches_generic_minifloat_and_value_set():
    check_e2m1(moe_ref)


def test_e8m0_special_values():
    s = np.array([0, 1, 126, 127, 128, 200, 254, 255])
    got = moe_ref.decode_e8m0(s)
    for si, g in zip(s[:-1].tolist(), got[:-1].tolist()):
        assert g == math.ldexp(1.0, si - 127)
    assert got[3] == 1.0 and got[-2] == 2.0 ** 127 and got[0] == 2.0 ** -127
    assert np.isnan(got[-1])


def test_dequant_matches_elementwise_python():
    check_dequant(moe_ref)


def test_dequantized_values_are_exact_in_bf16():
    d = mi.make_inputs(3, 64, 4, 2, 64, 11, weights="mxfp4")
    W = moe_ref.dequant_mxfp4(d["gu_codes"].numpy(), d["gu_scales"].numpy())
    back = torch.from_numpy(W).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(back, W)


@pytest.mark.parametrize("T,E,k", [(5, 4, 2), (9, 8, 3)])
def test_mxfp4_layer_equals_bf16_layer_on_dequantized_weights(T, E, k):
    H, I = 64, 64
    d = mi.make_inputs(T, H, E, k, I, 12 + T, weights="mxfp4")
    h = mi.host_inputs(d)
    out_mx = moe_ref.moe_forward_mxfp4_ref(h["x"], h["W_router"], h["b_router"], h["gu_codes"],
                                           h["gu_scales"], h["dn_codes"], h["dn_scales"], k)
    Wgu = moe_ref.dequant_mxfp4(h["gu_codes"], h["gu_scales"])
    Wd = moe_ref.dequant_mxfp4(h["dn_codes"], h["dn_scales"])
    bits = lambda W: mi.bf16_bits(torch.from_numpy(W).to(torch.bfloat16))
    out_bf = moe_ref.moe_forward_ref(h["x"], h["W_router"], h["b_router"], bits(Wgu), bits(Wd), k)
    np.testing.assert_array_equal(out_mx, out_bf)
    assert Wgu.shape == (E, H, 2 * I) and Wd.shape == (E, I, H)


def test_generated_weights_have_the_bf16_draws_spread():
    d = mi.make_inputs(1, 2880, 2, 1, 2880, 5, weights="mxfp4")
    W = moe_ref.dequant_mxfp4(d["gu_codes"][0].numpy(), d["gu_scales"][0].numpy())
    assert 0.5 < W.std() * math.sqrt(2880) < 1.5


# ---- planted mistakes -------------------------------------------------------------------
_ORIG_E2M1 = moe_ref.decode_e2m1
_ORIG_E8M0 = moe_ref.decode_e8m0
_ORIG_DEQ = moe_ref.dequant_mxfp4


def _e2m1_bias0(codes):
    c = np.asarray(codes).astype(np.int64) & 0xF
    sign, e, m = c >> 3, (c >> 1) & 3, c & 1
    mag = np.where(e == 0, 0.5 * m, np.ldexp(1.0 + 0.5 * m, e))
    return np.where(sign == 1, -mag, mag)


def _e2m1_no_subnormal(codes):
    c = np.asarray(codes).astype(np.int64) & 0xF
    sign, e, m = c >> 3, (c >> 1) & 3, c & 1
    mag = np.ldexp(1.0 + 0.5 * m, e - 1)
    return np.where(sign == 1, -mag, mag)


def _e8m0_bias128(s):
    return _ORIG_E8M0(np.asarray(s).astype(np.int64) - 1)


def _deq_nibbles_swapped(blocks, scales):
    b = np.asarray(blocks, dtype=np.uint8)
    return _ORIG_DEQ(((b & 0xF) << 4) | (b >> 4), scales)


def _deq_blocks_of_16(blocks, scales):
    b = np.asarray(blocks, dtype=np.uint8)
    codes = np.stack([b & 0xF, b >> 4], axis=-1).reshape(*b.shape[:-1], 2 * b.shape[-1])
    vals = np.swapaxes(moe_ref.decode_e2m1(codes), -1, -2)
    sc = np.repeat(moe_ref.decode_e8m0(scales), 16, axis=-2)
    sc = np.concatenate([sc, sc], axis=-2)[..., : vals.shape[-2], :]
    return vals * sc


MX_MUTANTS = {
    "e2m1_exponent_bias_0": ("decode_e2m1", _e2m1_bias0),
    "e2m1_without_subnormals": ("decode_e2m1", _e2m1_no_subnormal),
    "e8m0_bias_128": ("decode_e8m0", _e8m0_bias128),
    "nibble_order_swapped": ("dequant_mxfp4", _deq_nibbles_swapped),
    "scale_blocks_of_16": ("dequant_mxfp4", _deq_blocks_of_16),
}


def _mx_pins_pass() -> bool:
    try:
        check_e2m1(moe_ref)
        check_dequant(moe_ref)
    except AssertionError:
        return False
    return True


@pytest.mark.parametrize("name", sorted(MX_MUTANTS))
def test_planted_mxfp4_mistake_is_caught(name, monkeypatch):
    fn_name, mutant = MX_MUTANTS[name]
    monkeypatch.setattr(moe_ref, fn_name, mutant)
    assert not _mx_pins_pass(), f"planted mistake {name} went unnoticed"


def test_unplanted_mxfp4_decoding_passes_the_same_checks():
    assert _mx_pins_pass()
