"""OCP microscaling (MX) codecs for the oracle: E2M1 and E4M3 elements, E8M0 scales.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this module; only
tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference arm do.

What the pages fix (DeepSeek-V4.1-Flash checkpoint config and the MAX
DeepseekV41Config encodings):
  * routed experts are stored as FP4 ("expert_dtype": "fp4", inference/config.json),
    with the packed-pair encoding ``float4_e2m1fnx2`` (MAX DeepseekV41Config,
    SUPPORTED_ENCODINGS);
  * the family's block scales are ``float8_e8m0`` with one scale per 32 values
    (inference-research "DeepSeek-V4-Pro" page, FlashMLA KV layout paragraph);
  * a routed expert of the Flash shape occupies 18.8 MB (Strata DEEPSEEK41.md,
    "Where it goes" table), i.e. 4.25 bits per parameter;
  * the checkpoint's other weights are FP8 ("dtype": "fp8", inference/config.json)
    and MAX's default encoding is float8_e4m3fn (DeepseekV41Config
    DEFAULT_ENCODING / SUPPORTED_ENCODINGS).

Readings adopted where the pages are silent:
  * block rule = OCP MX v1.0: shared exponent floor(log2(amax)) - emax_elem,
    clamped to the E8M0 range, elements rounded to nearest-even and saturated
    to the element format's largest finite magnitude (E4M3: 448, E2M1: 6);
  * an all-zero block gets scale code 0 and zero elements;
  * E2M1 packing: element 2j in the low nibble, element 2j+1 in the high nibble;
  * FP8 expert weights are MXFP8: E4M3 values with one E8M0 scale per 32 along
    the input dimension, by the same block rule (the pages give no FP8 scale
    granularity; this is the family's per-32 E8M0 convention).

Everything here is exact float64 arithmetic: every E2M1, E4M3 and E8M0 value is
a dyadic rational that float64 represents exactly, and scaling by a power of two
is exact inside float64's range.
"""
from __future__ import annotations

import numpy as np

MX_BLOCK = 32          # elements sharing one E8M0 scale
E8M0_BIAS = 127
E8M0_NAN = 0xFF

# Largest power-of-two exponent of each element format (OCP MX v1.0, emax_elem).
EMAX_E4M3 = 8          # 448 = 1.75 * 2**8
EMAX_E2M1 = 2          # 6   = 1.5  * 2**2
MAXABS_E4M3 = 448.0
MAXABS_E2M1 = 6.0


# ----------------------------------------------------------------------------
# decoders (bit fields -> exact float64)
# ----------------------------------------------------------------------------
def decode_e2m1(code):
    """E2M1: 1 sign bit (bit 3), 2 exponent bits (bits 2-1, bias 1), 1 mantissa bit.

    Exponent field 0 is subnormal (0 or 0.5); there is no Inf and no NaN.
    """
    c = np.asarray(code, dtype=np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = (c & 0x1).astype(np.float64)
    mag = np.where(e == 0, m * 0.5, (1.0 + m * 0.5) * np.exp2(e.astype(np.float64) - 1.0))
    return sign * mag


def decode_e4m3(code):
    """E4M3 ("fn" variant): sign bit 7, exponent bits 6-3 (bias 7), mantissa bits 2-0.

    Exponent 0 is subnormal (m/8 * 2**-6); S.1111.111 is NaN; there is no Inf.
    """
    c = np.asarray(code, dtype=np.int64) & 0xFF
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6,
                   (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 15) & ((c & 0x7) == 7), np.nan, mag)
    return sign * mag


def decode_e8m0(code):
    """E8M0 scale: 2**(code - 127); code 0xFF is NaN."""
    c = np.asarray(code, dtype=np.int64) & 0xFF
    v = np.exp2(c.astype(np.float64) - E8M0_BIAS)
    return np.where(c == E8M0_NAN, np.nan, v)


# ----------------------------------------------------------------------------
# element encoders: round to nearest, ties to even, saturating
# ----------------------------------------------------------------------------
def _rne(v):
    """Round half to even (numpy's rint does exactly this)."""
    return np.rint(v)


def encode_e4m3(v):
    """Nearest-even E4M3 code of float64 values, saturating at +-448. No NaN input."""
    v = np.asarray(v, dtype=np.float64)
    sign = np.signbit(v)
    a = np.abs(v)
    # Exponent of the binade holding a (a = f * 2**ex, f in [0.5, 1)).
    _, ex = np.frexp(a)
    e_unb = ex.astype(np.int64) - 1                       # a in [2**e_unb, 2**(e_unb+1))
    normal = a >= 2.0 ** -6
    # Normal binade: 8 steps of 2**(e_unb-3) per binade.
    e_cl = np.maximum(e_unb, -6)
    q = _rne(a / np.exp2(e_cl.astype(np.float64) - 3.0))   # in [8, 16] for normals
    # Subnormal range: steps of 2**-9.
    q_sub = _rne(a / 2.0 ** -9)                            # in [0, 8]
    code = np.where(
        normal,
        # q == 16 rolls into the next binade with mantissa 0
        np.where(q >= 16, ((e_cl + 1 + 7) << 3), ((e_cl + 7) << 3) | (q.astype(np.int64) - 8)),
        np.where(q_sub >= 8, (1 << 3), q_sub.astype(np.int64)),
    )
    # Saturation: anything at or above 448 after rounding maps to 0x7E (448).
    over = (code > 0x7E) | (a >= MAXABS_E4M3)
    code = np.where(over, 0x7E, code)
    return (code | np.where(sign, 0x80, 0)).astype(np.uint8)


_E2M1_MAGS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def encode_e2m1(v):
    """Nearest-even E2M1 code of float64 values, saturating at +-6.

    The representable magnitudes are not evenly spaced, so rounding is done by
    comparing against the midpoints; on an exact midpoint the neighbour whose
    mantissa bit is 0 (the even one) wins.
    """
    v = np.asarray(v, dtype=np.float64)
    sign = np.signbit(v)
    a = np.minimum(np.abs(v), MAXABS_E2M1)
    idx = np.searchsorted(_E2M1_MAGS, a, side="left")     # first mag >= a
    idx = np.clip(idx, 0, 7)
    lo = np.clip(idx - 1, 0, 7)
    hi = idx
    d_lo = a - _E2M1_MAGS[lo]
    d_hi = _E2M1_MAGS[hi] - a
    choose_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ((hi & 1) == 0))
    code = np.where(choose_hi, hi, lo).astype(np.int64)
    return (code | np.where(sign, 0x8, 0)).astype(np.uint8)


# ----------------------------------------------------------------------------
# block quantisation (OCP MX v1.0 rule)
# ----------------------------------------------------------------------------
def mx_scale_codes(v, emax_elem):
    """E8M0 code per block of MX_BLOCK along the last axis.

    shared_exp = floor(log2(amax)) - emax_elem, clamped to [-127, 127];
    code = shared_exp + 127; an all-zero block gets code 0.
    """
    v = np.asarray(v, dtype=np.float64)
    assert v.shape[-1] % MX_BLOCK == 0
    blocks = v.reshape(*v.shape[:-1], v.shape[-1] // MX_BLOCK, MX_BLOCK)
    amax = np.abs(blocks).max(axis=-1)
    _, ex = np.frexp(amax)                  # amax = f * 2**ex, f in [0.5,1)
    fl = ex.astype(np.int64) - 1            # floor(log2(amax)) for amax > 0
    shared = np.clip(fl - emax_elem, -127, 127)
    code = np.where(amax > 0, shared + E8M0_BIAS, 0)
    return code.astype(np.uint8)


def quantize_mx(v, elem):
    """Quantise along the last axis in blocks of 32. Returns (element codes, scale codes).

    elem is 'e4m3' (MXFP8) or 'e2m1' (MXFP4). Element codes are one per byte.
    """
    if elem == "e4m3":
        emax, enc = EMAX_E4M3, encode_e4m3
    elif elem == "e2m1":
        emax, enc = EMAX_E2M1, encode_e2m1
    else:
        raise ValueError(elem)
    v = np.asarray(v, dtype=np.float64)
    sc = mx_scale_codes(v, emax)
    scale = decode_e8m0(sc)
    blocks = v.reshape(*v.shape[:-1], v.shape[-1] // MX_BLOCK, MX_BLOCK)
    q = enc(blocks / scale[..., None])
    return q.reshape(v.shape), sc


def dequantize_mx(codes, scales, elem):
    """Exact float64 values of MX-encoded data (codes one per byte, scales per 32)."""
    dec = decode_e4m3 if elem == "e4m3" else decode_e2m1
    vals = dec(codes)
    sh = vals.shape
    blocks = vals.reshape(*sh[:-1], sh[-1] // MX_BLOCK, MX_BLOCK)
    return (blocks * decode_e8m0(scales)[..., None]).reshape(sh)


def mx_roundtrip(v, elem):
    """Quantise then dequantise: the value an MX consumer sees."""
    q, s = quantize_mx(v, elem)
    return dequantize_mx(q, s, elem)


# ----------------------------------------------------------------------------
# float4_e2m1fnx2 packing
# ----------------------------------------------------------------------------
def pack_e2m1(codes):
    """Pack E2M1 codes (one per byte) two per byte: even element -> low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    assert c.shape[-1] % 2 == 0
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


def unpack_e2m1(packed):
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def quantize_mxfp4_packed(w):
    """Weights [..., K] -> (packed E2M1 [..., K/2] uint8, E8M0 [..., K/32] uint8)."""
    q, s = quantize_mx(w, "e2m1")
    return pack_e2m1(q), s


def dequantize_mxfp4_packed(packed, scales):
    return dequantize_mx(unpack_e2m1(packed), scales, "e2m1")


def quantize_mxfp8(w):
    """Weights [..., K] -> (E4M3 codes [..., K] uint8, E8M0 [..., K/32] uint8): MXFP8."""
    return quantize_mx(w, "e4m3")


def dequantize_mxfp8(codes, scales):
    return dequantize_mx(codes, scales, "e4m3")


def mxfp8_bytes(rows, cols):
    """Storage of an MXFP8 [rows, cols] matrix: 1 byte per value + 1 byte per 32."""
    assert cols % MX_BLOCK == 0
    return rows * cols + rows * cols // MX_BLOCK


def mxfp4_bytes(rows, cols):
    """Storage of an MXFP4 [rows, cols] matrix: 4 bits per value + 1 byte per 32."""
    assert cols % MX_BLOCK == 0
    return rows * cols // 2 + rows * cols // MX_BLOCK
