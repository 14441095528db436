"""Pins for the oracle's NVFP4 encode/decode (CPU only).

Each test checks the oracle against something other than itself: the E2M1 value list of
the OCP microscaling format, torch's float8_e4m3fn cast (a library routine), brute-force
nearest-value search, hand-worked examples in tests/golden/, and invariants.
"""
import os

import numpy as np
import pytest
import torch

from oracle import nvfp4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "nvfp4_blocks.txt")


def test_e2m1_table_matches_format_value_list():
    # OCP MX v1.0 FP4 (E2M1): positive codes 0..7 encode these magnitudes, code | 8 negates
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for c in range(8):
        assert nvfp4.E2M1_TABLE[c] == mags[c]
        assert nvfp4.E2M1_TABLE[c | 8] == -mags[c]
    assert np.signbit(nvfp4.E2M1_TABLE[8])  # code 0x8 is -0


def test_e4m3_table_matches_torch_float8():
    b = torch.arange(256, dtype=torch.uint8)
    ref = b.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = nvfp4.E4M3_TABLE
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(ours))
    assert nan.sum() == 2  # 0x7F and 0xFF
    assert np.array_equal(ref[~nan], ours[~nan])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x08] == 2.0 ** -6


def test_dequant_products_exact_for_all_codes_and_scales():
    # every (E2M1 code, finite E4M3 byte) product is exact in float32 (and float64)
    finite = [s for s in range(256) if not np.isnan(nvfp4.E4M3_TABLE[s])]
    assert len(finite) == 254
    codes = np.arange(16, dtype=np.uint8)
    packed = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)[None, :]  # one row, 16 codes
    for s in finite:
        v = nvfp4.dequantize(packed, np.array([[s]], np.uint8), np.float32(1.0))[0]
        exact = torch.tensor(nvfp4.E2M1_TABLE).double() * float(
            torch.tensor([s], dtype=torch.uint8).view(torch.float8_e4m3fn).double())
        assert np.array_equal(v, exact.numpy())
        assert np.array_equal(v.astype(np.float32).astype(np.float64), v)


def _dense_grid():
    vals = set()
    pos = nvfp4.E4M3_TABLE[:0x7F]
    for a, b in zip(pos[:-1], pos[1:]):
        mid = (a + b) / 2
        for v in (a, b, mid):
            vals.add(float(np.float32(v)))
        # neighbours of the midpoint
        vals.add(float(np.nextafter(np.float32(mid), np.float32(0))))
        vals.add(float(np.nextafter(np.float32(mid), np.float32(1e9))))
    rng = np.random.default_rng(0)
    vals.update(rng.uniform(0, 448, 4000).astype(np.float32).tolist())
    vals.update(np.exp2(rng.uniform(-12, 8.8, 4000)).astype(np.float32).tolist())
    return np.array(sorted(vals), dtype=np.float32)


def test_e4m3_rounding_matches_torch_cast_in_range():
    g = _dense_grid()
    g = g[g <= 448]
    ref = torch.from_numpy(g).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = nvfp4.e4m3_encode_rne_sat(g)
    assert np.array_equal(ref, ours)


def test_e4m3_rounding_brute_force_nearest_even_and_saturation():
    g = np.concatenate([_dense_grid(), np.float32([448, 460, 464, 479, 480, 1e4, 3e38])])
    pos = nvfp4.E4M3_TABLE[:0x7F]
    ours = nvfp4.e4m3_encode_rne_sat(g)
    for v, byte in zip(g.astype(np.float64), ours):
        if v >= 448:
            assert byte == 0x7E
            continue
        dist = np.abs(pos - v)
        best = np.flatnonzero(dist == dist.min())
        want = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        assert byte == want, (v, byte, want)


def test_e2m1_rounding_brute_force_nearest_even():
    mags = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    grid = set()
    for a, b in zip(mags[:-1], mags[1:]):
        m = (a + b) / 2
        for v in (a, b, m, np.nextafter(m, 0), np.nextafter(m, 10)):
            grid.add(float(np.float32(v)))
    grid.update(np.random.default_rng(1).uniform(0, 8, 3000).astype(np.float32).tolist())
    grid.update([6.0, 7.0, 1e30])
    g = np.array(sorted(grid), dtype=np.float32)
    g = np.concatenate([g, -g])
    codes = nvfp4.e2m1_encode_rne_sat(g)
    for v, c in zip(g.astype(np.float64), codes):
        a = abs(v)
        if a >= 6:
            want = 7
        else:
            dist = np.abs(mags - a)
            best = np.flatnonzero(dist == dist.min())
            want = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        assert (c & 7) == want, (v, c, want)
        assert (c >> 3) == (1 if np.signbit(v) else 0)


def test_e2m1_midpoint_table():
    # the tie cases spelled out: 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for v, want in ties.items():
        c = nvfp4.e2m1_encode_rne_sat(np.float32([v, -v]))
        assert nvfp4.E2M1_TABLE[c[0]] == want
        assert nvfp4.E2M1_TABLE[c[1]] == -want
    c = nvfp4.e2m1_encode_rne_sat(np.float32([-0.0, 0.0, -0.1]))
    assert list(c) == [8, 0, 8]


def _load_golden():
    cases = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, ts, xs, sc, cb = [p.strip() for p in line.split("|")]
        x = np.array([float(v) for v in xs.split()], dtype=np.float32)
        cases.append((name, np.float32(float(ts)), x, int(sc, 16),
                      bytes.fromhex(cb.replace(" ", ""))))
    return cases


@pytest.mark.parametrize("case", _load_golden(), ids=lambda c: c[0])
def test_golden_blocks(case):
    name, ts, x, scale, code_bytes = case
    codes, scales, ts_out = nvfp4.quantize(x[None, :], ts=ts)
    assert ts_out == ts
    assert scales[0, 0] == scale, name
    assert bytes(codes[0]) == code_bytes, (name, bytes(codes[0]).hex())


def test_dynamic_tensor_scale_and_zero_tensor():
    x = np.zeros((2, 32), np.float32)
    c, s, ts = nvfp4.quantize(x)
    assert ts == np.float32(1.0) and not c.any() and not s.any()
    x[1, 5] = -2688.0
    c, s, ts = nvfp4.quantize(x)
    assert ts == np.float32(1.0)
    # block amax 2688 -> (2688/6)/1 = 448 -> 0x7E; element -> -2688/448 = -6 -> 0xF
    assert s[1, 0] == 0x7E and (c[1, 2] >> 4) == 0xF
    x[1, 5] = 1.0
    _, _, ts = nvfp4.quantize(x)
    assert ts == np.float32(1.0) / np.float32(2688.0)


def test_quantize_error_within_half_step_unless_saturated():
    rng = np.random.default_rng(7)
    x = (rng.standard_normal((64, 256)) * rng.uniform(0.01, 10, (64, 1))).astype(np.float32)
    c, s, ts = nvfp4.quantize(x)
    xq = nvfp4.dequantize(c, s, ts)
    q = nvfp4.unpack_codes(c)
    scale = np.repeat(nvfp4.E4M3_TABLE[s], 16, axis=1) * np.float64(ts)
    # spacing of E2M1 around each chosen value, in units of the block scale
    mags = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    up = np.array([.5, .5, .5, .5, 1, 1, 2, np.inf])
    dn = np.array([.5, .5, .5, .5, .5, 1, 1, 2])
    m = q & 7
    a = np.abs(x.astype(np.float64)) / scale
    sat = (m == 7) & (a > 6)
    err = np.abs(a - mags[m])
    half = np.where(a >= mags[m], up[m], dn[m]) / 2
    assert np.all((err <= half * (1 + 1e-6)) | sat)
    # the block maximum maps to code 6 or saturates unless its scale was rounded down a lot
    bmax = np.abs(x.reshape(64, 16, 16)).max(axis=2)
    assert np.all(bmax > 0)
    rel = np.abs(xq - x) / np.repeat(bmax, 16, axis=1)
    assert rel.max() < 0.25


def test_quantize_layout_low_nibble_first_and_scale_rows():
    x = np.zeros((3, 32), np.float32)
    x[2, 0] = 6.0      # element 0 of row 2 -> low nibble of byte 0
    x[2, 1] = -3.0     # element 1 -> high nibble of byte 0
    x[2, 17] = 1.0     # second block of row 2
    c, s, ts = nvfp4.quantize(x, ts=np.float32(1.0))
    assert c.shape == (3, 16) and s.shape == (3, 2)
    # block amax 6 -> scale 1.0 (0x38): 6 -> code 7 (low nibble), -3 -> code 0xD (high)
    assert c[2, 0] == (0x7 | (0xD << 4))
    assert s[2, 0] == 0x38 and s[2, 1] != 0 and not c[:2].any()
