"""Pins of the oracle's MX codecs (E2M1, E4M3, E8M0, OCP block rule, packing).

Independent sources: the OCP MX v1.0 element tables (written out below), the
float8 decoders that PyTorch ships (``torch.float8_e4m3fn``,
``torch.float8_e8m0fnu``) and PyTorch's round-to-nearest-even float8 encoder,
plus the per-expert MXFP4 size printed on the Strata DEEPSEEK41.md page.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import moe as om
from oracle import mx

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_e2m1_table():
    # OCP MX v1.0 FP4 E2M1: magnitudes for codes 0..7, sign in bit 3
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    got = mx.decode_e2m1(np.arange(16))
    assert list(got[:8]) == mags
    assert list(-got[8:]) == mags
    assert np.all(np.signbit(got[8:]))


def test_e4m3_decode_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    got = mx.decode_e4m3(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan) and nan.sum() == 2
    assert np.array_equal(got[~nan], ref[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9


def test_e8m0_decode_matches_torch():
    codes = np.arange(255, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e8m0fnu).double().numpy()
    assert np.array_equal(mx.decode_e8m0(codes), ref)
    assert np.isnan(mx.decode_e8m0(255))


def test_e4m3_encode_roundtrip_and_rne():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF, 0x80)], dtype=np.uint8)
    assert np.array_equal(mx.encode_e4m3(mx.decode_e4m3(codes)), codes)
    # torch's float -> float8_e4m3fn cast rounds to nearest even for in-range values
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.standard_normal(20000) * 40, rng.standard_normal(20000) * 1e-2,
                        np.linspace(-447.9, 447.9, 5001)])
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = mx.encode_e4m3(v)
    assert np.array_equal(mx.decode_e4m3(got), mx.decode_e4m3(ref))
    # saturation instead of NaN
    assert mx.decode_e4m3(mx.encode_e4m3(np.array([1e6, -500.0, 470.0])))[0] == 448.0
    assert list(mx.decode_e4m3(mx.encode_e4m3(np.array([-500.0, 470.0])))) == [-448.0, 448.0]


def test_e2m1_encode_ties_and_saturation():
    # midpoints round to the neighbour with a zero mantissa bit
    v = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, 100.0, -0.74, -5.1])
    expect = [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 6.0, 6.0, -0.5, -6.0]
    assert list(mx.decode_e2m1(mx.encode_e2m1(v))) == expect
    assert np.array_equal(mx.encode_e2m1(mx.decode_e2m1(np.arange(16))),
                          np.array([c if c != 8 else 8 for c in range(16)], dtype=np.uint8))


def test_mx_block_rule():
    # amax = 448 -> floor(log2) = 8 -> shared exponent 0 (code 127) for E4M3
    blk = np.zeros(32); blk[5] = 448.0; blk[6] = -1.0
    q, s = mx.quantize_mx(blk, "e4m3")
    assert s.tolist() == [127] and mx.decode_e4m3(q)[5] == 448.0
    # amax = 1 -> X = 2^-8, the element becomes 256 exactly
    blk = np.full(32, 0.5); blk[0] = 1.0
    q, s = mx.quantize_mx(blk, "e4m3")
    assert s.tolist() == [127 - 8] and mx.decode_e4m3(q)[0] == 256.0
    # E2M1: amax 3 -> X = 0.5 -> 6; amax 7 -> X = 1 and 7 saturates to 6 (OCP clipping)
    q, s = mx.quantize_mx(np.full(32, 3.0), "e2m1")
    assert s.tolist() == [126] and np.all(mx.decode_e2m1(q) == 6.0)
    q, s = mx.quantize_mx(np.full(32, 7.0), "e2m1")
    assert s.tolist() == [127] and np.all(mx.decode_e2m1(q) == 6.0)
    # all-zero block: code 0, zero elements
    q, s = mx.quantize_mx(np.zeros(64), "e4m3")
    assert s.tolist() == [0, 0] and np.all(q == 0)
    # blocks are independent, along the last axis, 32 wide
    v = np.concatenate([np.full(32, 1.0), np.full(32, 1024.0)])
    _, s = mx.quantize_mx(v[None, :], "e4m3")
    assert s.tolist() == [[119, 129]]


def test_mx_exact_values_roundtrip():
    rng = np.random.default_rng(1)
    # values exactly representable: E2M1 codes times a power of two per block
    codes = rng.integers(0, 16, size=(6, 64)).astype(np.uint8)
    codes[:, ::32] = 7                                   # make amax = 6 in every block
    scales = rng.integers(100, 140, size=(6, 2)).astype(np.uint8)
    v = mx.dequantize_mx(codes, scales, "e2m1")
    q, s = mx.quantize_mx(v, "e2m1")
    assert np.array_equal(s, scales)
    assert np.array_equal(mx.decode_e2m1(q), mx.decode_e2m1(codes))
    # quant(dequant(q)) == q for E4M3 with the largest code in each block
    c8 = rng.integers(0, 0x7E, size=(4, 64)).astype(np.uint8)
    c8[:, ::32] = 0x7E
    s8 = rng.integers(110, 130, size=(4, 2)).astype(np.uint8)
    q8, r8 = mx.quantize_mx(mx.dequantize_mx(c8, s8, "e4m3"), "e4m3")
    assert np.array_equal(r8, s8)
    assert np.array_equal(mx.decode_e4m3(q8), mx.decode_e4m3(c8))


def test_mx_error_bound():
    # E4M3 keeps 3 mantissa bits: relative error <= 2^-4 for values in the normal range
    rng = np.random.default_rng(4)
    v = rng.standard_normal((64, 256))
    rt = mx.mx_roundtrip(v, "e4m3")
    _, s = mx.quantize_mx(v, "e4m3")
    X = np.repeat(mx.decode_e8m0(s), 32, axis=-1)
    r = np.abs(v) / X
    normal = (r >= 2.0 ** -6) & (r <= 448.0)
    assert np.all(np.abs(rt - v)[normal] <= 2.0 ** -4 * np.abs(v)[normal])
    sub = r < 2.0 ** -6
    assert np.all(np.abs(rt - v)[sub] <= 2.0 ** -10 * X[sub])
    # above 448 * X the OCP rule clips to +-448 * X (amax / X lies in [256, 512))
    sat = r > 448.0
    assert sat.any() and np.all(np.abs(rt[sat]) == 448.0 * X[sat])
    assert np.all(r < 512.0)


def test_e2m1_packing_nibble_order():
    assert mx.pack_e2m1(np.array([1, 2, 0xF, 0x3], dtype=np.uint8)).tolist() == [0x21, 0x3F]
    c = np.random.default_rng(5).integers(0, 16, size=(3, 64)).astype(np.uint8)
    assert np.array_equal(mx.unpack_e2m1(mx.pack_e2m1(c)), c)


def test_flash_expert_mxfp4_size_matches_page():
    """Strata DEEPSEEK41.md, "Where it goes": 15,360 routed experts of 18.8 MB, 288.8 GB."""
    with open(os.path.join(GOLDEN, "page_constants.json")) as f:
        pc = json.load(f)
    H, I = pc["dim"]["value"], pc["moe_inter_dim"]["value"]
    per_expert = 2 * mx.mxfp4_bytes(I, H) + mx.mxfp4_bytes(H, I)
    assert per_expert == 18_800_640
    assert round(per_expert / 1e6, 1) == pc["routed_expert_mb_mxfp4"]["value"]
    total = per_expert * pc["n_layers"]["value"] * pc["n_routed_experts"]["value"]
    assert pc["n_layers"]["value"] * pc["n_routed_experts"]["value"] == pc["routed_experts_total"]["value"]
    assert round(total / 1e9, 1) == pc["routed_experts_gb_mxfp4"]["value"]


def test_mx_mirror_mode_is_exact_on_representable_inputs():
    # inputs already on the MXFP8 grid: mirror mode changes nothing for x;
    # the layer differs only through h's quantisation
    rng = np.random.default_rng(8)
    T, H, I, E = 4, 64, 32, 3
    x = mx.mx_roundtrip(rng.standard_normal((T, H)), "e4m3")
    w1 = rng.standard_normal((E, I, H)) / 8; w3 = rng.standard_normal((E, I, H)) / 8
    w2 = rng.standard_normal((E, H, I)) / 6
    o_a, h_a = om.expert_forward(x, w1[0], w3[0], w2[0], 10.0, mx_act=False)
    o_b, h_b = om.expert_forward(x, w1[0], w3[0], w2[0], 10.0, mx_act=True)
    assert np.array_equal(h_a, h_b)
    assert np.allclose(o_b, mx.mx_roundtrip(h_a, "e4m3") @ w2[0].T, rtol=1e-14)
    assert not np.allclose(o_a, o_b, rtol=1e-6)


def test_mxfp8_expert_values_match_torch_decoders():
    """MXFP8 weights (E4M3 codes + E8M0 scales per 32) served by from_mxfp8 equal
    PyTorch's float8_e4m3fn and float8_e8m0fnu decodings of the same bytes, and
    the routed experts are marked for the MX mirror."""
    rng = np.random.default_rng(12)
    E, I_, H_, S = 2, 32, 64, 1
    w = [rng.standard_normal((E, I_, H_)) / 8, rng.standard_normal((E, I_, H_)) / 8,
         rng.standard_normal((E, H_, I_)) / 6]
    q = [mx.quantize_mxfp8(a) for a in w]
    sh = [np.zeros((S, I_, H_)), np.zeros((S, I_, H_)), np.zeros((S, H_, I_))]
    src = om.ExpertSource.from_mxfp8(q[0][0], q[0][1], q[1][0], q[1][1], q[2][0], q[2][1], *sh)
    assert src.routed_is_mx
    for e in range(E):
        for got, (codes, scales) in zip(src.routed(e), q):
            v = torch.from_numpy(codes[e].copy()).view(torch.float8_e4m3fn).to(torch.float64)
            sc = torch.from_numpy(scales[e].copy()).view(torch.float8_e8m0fnu).to(torch.float64)
            ref = (v.reshape(v.shape[0], -1, 32) * sc[..., None]).reshape(v.shape).numpy()
            assert np.array_equal(got, ref)
    # the stored values are the round trip of the weights they were quantised from
    assert np.array_equal(src.routed(1)[2], mx.mx_roundtrip(w[2][1], "e4m3"))


def test_flash_expert_mxfp8_size():
    """One byte per value plus one E8M0 byte per 32: 3 H I (1 + 1/32) for a Flash expert."""
    H_, I_ = 5120, 2304
    per_expert = 2 * mx.mxfp8_bytes(I_, H_) + mx.mxfp8_bytes(H_, I_)
    assert per_expert == 3 * H_ * I_ * 33 // 32 == 36_495_360
