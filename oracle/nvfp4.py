"""NVFP4 encode/decode in plain numpy (oracle; test infrastructure only).

Source: the Basalt project page ("Basalt", section "All the numbers", list "Engines: commit,
and what is not NVIDIA's weights") names the expert format NVFP4 and says the engine keeps
NVIDIA's NVFP4 experts bit-exact, including the llama.cpp row's ``input_scale`` (a static
activation scale). The pages do not define the format; readings R1-R3 in the package
docstring fill the gap.
"""
from __future__ import annotations

import numpy as np

F32 = np.float32
E2M1_MAX = 6.0
E4M3_MAX = 448.0
NVFP4_BLOCK = 16


# --------------------------------------------------------------------------- decode tables

def _e2m1_value(code: int) -> float:
    """Value of a 4-bit E2M1 code: bit 3 sign, bits 2-1 exponent (bias 1), bit 0 mantissa."""
    s = -1.0 if code & 0x8 else 1.0
    e = (code >> 1) & 0x3
    m = code & 0x1
    if e == 0:
        return s * 0.5 * m                      # subnormal: 0 or 0.5
    return s * (2.0 ** (e - 1)) * (1.0 + 0.5 * m)


def _e4m3_value(byte: int) -> float:
    """Value of an E4M3 ("fn") byte: bit 7 sign, bits 6-3 exponent (bias 7), bits 2-0
    mantissa; S.1111.111 is NaN, there is no infinity."""
    s = -1.0 if byte & 0x80 else 1.0
    e = (byte >> 3) & 0xF
    m = byte & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (2.0 ** -6) * (m / 8.0)
    return s * (2.0 ** (e - 7)) * (1.0 + m / 8.0)


E2M1_TABLE = np.array([_e2m1_value(c) for c in range(16)], dtype=np.float64)
E4M3_TABLE = np.array([_e4m3_value(b) for b in range(256)], dtype=np.float64)

# positive finite E4M3 bytes 0x00..0x7E, increasing in value
_E4M3_POS = E4M3_TABLE[:0x7F]


# --------------------------------------------------------------------------- rounding

def e4m3_encode_rne_sat(v) -> np.ndarray:
    """Round non-negative float32 values to E4M3 (nearest, ties to even mantissa),
    saturating at 448. Returns bytes (sign bit always 0).

    Works on the binary exponent: for v >= 2**-6 the spacing of E4M3 values in
    [2**e, 2**(e+1)) is 2**(e-3); below 2**-6 (subnormals) it is 2**-9. v / spacing is an
    exact float64 operation, and np.rint rounds half to even, which is the even mantissa."""
    v = np.asarray(v, dtype=np.float64)
    if np.any(v < 0) or np.any(~np.isfinite(v)):
        raise ValueError("e4m3_encode_rne_sat expects finite non-negative values")
    _, ex = np.frexp(v)                      # v = f * 2**ex, f in [0.5, 1)
    e = np.maximum(ex - 1, -6)               # v in [2**e, 2**(e+1)) for normals
    spacing = np.ldexp(1.0, e - 3)
    r = np.rint(v / spacing) * spacing       # nearest multiple, ties to even multiple
    r = np.minimum(r, E4M3_MAX)
    # value -> byte (r is now exactly an E4M3 value)
    idx = np.searchsorted(_E4M3_POS, r)
    assert np.all(_E4M3_POS[idx] == r)
    return idx.astype(np.uint8)


# thresholds on |v| between consecutive E2M1 magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6};
# at an exact midpoint the magnitude with even mantissa bit (even code) wins.
_E2M1_MID = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
_E2M1_TIE_UP = np.array([False, True, False, True, False, True, False])  # tie goes to upper?


def e2m1_encode_rne_sat(v) -> np.ndarray:
    """Round float32 values to E2M1 codes (nearest, ties to even, saturate at 6).
    A negative value (or -0.0) keeps sign bit 0x8 even when it rounds to zero."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    mag = np.zeros(a.shape, dtype=np.uint8)
    for i, (mid, up) in enumerate(zip(_E2M1_MID, _E2M1_TIE_UP)):
        above = (a >= mid) if up else (a > mid)
        mag += above.astype(np.uint8)
    sign = np.signbit(v).astype(np.uint8) << 3
    return (mag | sign).astype(np.uint8)


# --------------------------------------------------------------------------- quantise

def tensor_scale(x_f32: np.ndarray) -> np.float32:
    """Dynamic tensor scale (reading R2): amax / (6 * 448) in float32, 1.0 for all-zero."""
    amax = F32(np.max(np.abs(x_f32))) if x_f32.size else F32(0.0)
    return F32(amax / F32(E2M1_MAX * E4M3_MAX)) if amax > 0 else F32(1.0)


def quantize(x, ts=None):
    """Quantise a float32 matrix [rows][cols] to NVFP4 (readings R1-R3).

    Per 16-element block b of a row, in float32 with IEEE round-to-nearest:
        sb    = (amax_b / 6) / ts
        s     = E4M3_rne_sat(sb)                     (scale byte)
        denom = E4M3(s) * ts
        q_i   = E2M1_rne_sat(x_i / denom)            (all +0 when E4M3(s) == 0)
    ts is the given static scale, or the dynamic tensor scale when ts is None.
    Returns (codes uint8 [rows][cols/2], element 2i in the low nibble; scales uint8
    [rows][cols/16]; ts float32)."""
    x = np.asarray(x, dtype=F32)
    if x.ndim != 2 or x.shape[1] % NVFP4_BLOCK:
        raise ValueError("quantize expects [rows][cols] with cols % 16 == 0")
    rows, cols = x.shape
    ts = tensor_scale(x) if ts is None else F32(ts)
    xb = x.reshape(rows, cols // NVFP4_BLOCK, NVFP4_BLOCK)
    amax_b = np.max(np.abs(xb), axis=2)                         # float32, exact
    sb = (amax_b / F32(E2M1_MAX)) / ts                          # two float32 divisions
    s = e4m3_encode_rne_sat(sb)
    sval = E4M3_TABLE[s].astype(F32)                            # exact in float32
    denom = (sval * ts).astype(F32)                             # float32 multiply
    zero_blk = sval == 0
    safe = np.where(zero_blk, F32(1.0), denom)[:, :, None]
    q = e2m1_encode_rne_sat((xb / safe).astype(F32))            # float32 division
    q = np.where(zero_blk[:, :, None], np.uint8(0), q)
    q = q.reshape(rows, cols)
    codes = (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)
    return codes, s.astype(np.uint8), F32(ts)


def unpack_codes(codes: np.ndarray) -> np.ndarray:
    """[rows][cols/2] packed bytes -> [rows][cols] 4-bit codes (element 2i = low nibble)."""
    codes = np.asarray(codes, dtype=np.uint8)
    out = np.empty((codes.shape[0], codes.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = codes & 0xF
    out[:, 1::2] = codes >> 4
    return out


def dequantize(codes, scales, ts) -> np.ndarray:
    """Exact float64 value of an NVFP4 matrix: e2m1(q) * e4m3(s) * ts (reading R1).
    The product of a 2-bit and a 4-bit significand with a float32 fits a float64 exactly."""
    q = unpack_codes(codes)
    s = np.asarray(scales, dtype=np.uint8)
    rows, cols = q.shape
    sv = np.repeat(E4M3_TABLE[s], NVFP4_BLOCK, axis=1)
    return E2M1_TABLE[q] * sv * np.float64(F32(ts))
