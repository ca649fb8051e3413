"""Element formats used by the routed MoE FFN, decoded and encoded in numpy.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Formats (their names come from the pages; their bit layouts are the public
OCP 8-bit floating point / OCP microscaling definitions, which the pages
reference by name only):

* E4M3 ``float8_e4m3fn`` -- flashinfer.megamoe.MegaMoESymmBuffer, staging
  view ``x`` (E4M3 [capacity, hidden]); flashinfer.fused_moe.
  MoEActivationPack, NVFP4 block scales ``float8_e4m3fn [M, H/16]``.
  1 sign, 4 exponent (bias 7), 3 mantissa bits; no infinities; S.1111.111
  is NaN; largest finite magnitude 448; smallest subnormal 2**-9.
* E2M1 (FP4) -- flashinfer.fused_moe.MoEActivationPack, "packed uint8
  [M, H/2] values".  1 sign, 2 exponent (bias 1), 1 mantissa bit; the eight
  magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6; no NaN, no infinity.  Two codes
  per byte, element 2i in the low nibble (reading: the pages do not state
  the nibble order).
* BF16 -- flashinfer.fused_moe.MoEActivationPack, "BF16: raw bfloat16".
* UE8M0 -- flashinfer.fused_moe.MoEActivationPack, MXFP8 "token-major uint8
  [M, H/32] UE8M0 scales"; Struct_mega_ffn_ep_combine_send names the E8M0
  sibling.  An unsigned power of two: code c is 2**(c - 127), code 255 is
  NaN (the OCP microscaling scale format).

Encoders round to nearest, ties to even, and saturate to the largest finite
magnitude ("satfinite"), the reading taken where the pages are silent.
"""

import numpy as np

E4M3_MAX = 448.0
E2M1_MAX = 6.0


# ----------------------------------------------------------------------------
# E4M3 (float8_e4m3fn)
# ----------------------------------------------------------------------------

def e4m3_decode(codes):
    """Decode uint8 E4M3 codes to float64 (NaN for the two NaN codes)."""
    c = np.asarray(codes, dtype=np.uint8)
    if c.size > 256:
        return _E4M3_TABLE[c]
    return _e4m3_decode_fields(c)


def _e4m3_decode_fields(codes):
    """The field-by-field E4M3 definition (also builds the 256-entry table)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    exp = (c >> 3) & 0xF
    man = c & 0x7
    normal = (1.0 + man / 8.0) * np.ldexp(1.0, exp - 7)
    subnormal = (man / 8.0) * np.ldexp(1.0, -6)
    mag = np.where(exp == 0, subnormal, normal)
    mag = np.where((exp == 15) & (man == 7), np.nan, mag)
    return sign * mag


def e4m3_encode(values):
    """Encode float values (float32 or float64) to E4M3, RNE, saturating.

    Magnitudes at or above 448 saturate to 448 (code 0x7E); NaN maps to 0x7F
    with the sign of the input.
    """
    v = np.asarray(values, dtype=np.float64)
    neg = np.signbit(v)
    a = np.abs(v)
    nan = np.isnan(a)
    a = np.where(nan, 0.0, a)
    code = np.zeros(a.shape, dtype=np.int64)

    # Subnormal range: a < 2**-6.  Quantum 2**-9; a mantissa of 8 rolls over
    # into the smallest normal (code 0x08), which is exactly code value 8.
    sub = a < 2.0 ** -6
    q_sub = np.rint(a / 2.0 ** -9).astype(np.int64)          # half-to-even
    code = np.where(sub, q_sub, code)

    # Normal range.
    _, ex = np.frexp(np.where(sub, 1.0, a))                   # a = f * 2**ex, f in [0.5, 1)
    e_unb = ex - 1
    q = np.rint(np.ldexp(np.where(sub, 1.0, a), -e_unb) * 8.0 - 8.0).astype(np.int64)
    carry = q == 8
    e_unb = np.where(carry, e_unb + 1, e_unb)
    q = np.where(carry, 0, q)
    biased = e_unb + 7
    norm_code = (biased << 3) | q
    code = np.where(sub, code, norm_code)

    sat = (a >= E4M3_MAX) | (~sub & ((biased > 15) | ((biased == 15) & (q == 7))))
    code = np.where(sat, 0x7E, code)
    code = np.where(nan, 0x7F, code)
    code = code | np.where(neg, 0x80, 0)
    return code.astype(np.uint8)


# ----------------------------------------------------------------------------
# E2M1 (FP4)
# ----------------------------------------------------------------------------

def e2m1_decode(nibbles):
    """Decode 4-bit E2M1 codes (values 0..15, any integer dtype) to float64."""
    c = np.asarray(nibbles)
    if c.size > 16:
        return _E2M1_TABLE[c.astype(np.int64) & 0xF]
    return _e2m1_decode_fields(c)


def _e2m1_decode_fields(nibbles):
    """The field-by-field E2M1 definition (also builds the 16-entry table)."""
    c = np.asarray(nibbles).astype(np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    exp = (c >> 1) & 0x3
    man = c & 0x1
    mag = np.where(exp == 0, man * 0.5, (1.0 + man / 2.0) * np.ldexp(1.0, exp - 1))
    return sign * mag


def e2m1_encode(values):
    """Encode float values to 4-bit E2M1 codes, RNE, saturating at 6.

    Returns int codes 0..15 (uint8).  A negative value that rounds to zero
    keeps its sign bit (code 0x8), as the IEEE-style rounding does.
    """
    v = np.asarray(values, dtype=np.float64)
    neg = np.signbit(v)
    a = np.abs(v)
    a = np.where(np.isnan(a), 0.0, a)

    small = a < 1.0
    # Below 1.0 the quantum is 0.5; a rounded mantissa of 2 is the code of 1.0.
    q_small = np.rint(a * 2.0).astype(np.int64)

    _, ex = np.frexp(np.where(small, 1.0, a))
    e_unb = ex - 1
    q = np.rint(np.ldexp(np.where(small, 1.0, a), -e_unb) * 2.0 - 2.0).astype(np.int64)
    carry = q == 2
    e_unb = np.where(carry, e_unb + 1, e_unb)
    q = np.where(carry, 0, q)
    biased = e_unb + 1
    norm_code = (biased << 1) | q
    norm_code = np.where(biased > 3, 0x7, norm_code)

    code = np.where(small, q_small, norm_code)
    code = np.where(a >= E2M1_MAX, 0x7, code)
    code = code | np.where(neg, 0x8, 0)
    return code.astype(np.uint8)


_E4M3_TABLE = _e4m3_decode_fields(np.arange(256, dtype=np.uint8))
_E2M1_TABLE = _e2m1_decode_fields(np.arange(16))


def fp4_unpack(packed, n):
    """Unpack uint8 [..., n/2] into nibble codes [..., n]; element 2i is the low nibble."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (n,), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def fp4_pack(codes):
    """Pack nibble codes [..., n] (n even) into uint8 [..., n/2]; element 2i -> low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


# ----------------------------------------------------------------------------
# UE8M0 (MX block scale)
# ----------------------------------------------------------------------------

def ue8m0_decode(codes):
    """uint8 UE8M0 codes -> float64: 2**(code - 127); code 255 is NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    v = np.ldexp(1.0, c - 127)
    return np.where(c == 255, np.nan, v)


# ----------------------------------------------------------------------------
# BF16
# ----------------------------------------------------------------------------

def bf16_decode(bits):
    """uint16 BF16 bit patterns -> float64 (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def bf16_encode(values):
    """float32 values -> uint16 BF16, round to nearest even (NaN stays NaN).

    The input is first rounded to float32 (numpy's RNE cast) when it is
    float64: the kernels keep these values in FP32 registers before the BF16
    rounding, so the oracle rounds at the same two points.
    """
    f = np.asarray(values, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint32)
    nan = np.isnan(f)
    r = np.where(nan, ((u >> 16) | 0x40).astype(np.uint32), r)
    return r.astype(np.uint16)
