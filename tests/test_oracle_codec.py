"""Pins for the oracle's NVFP4 codec (E2M1 codes, E4M3 scales, fp32 tensor scale).

Pinned against: hand-worked values (tests/golden, OCP MX v1.0 formats), torch's
own float8_e4m3fn conversion (a library routine), exact round trips and the
per-token byte count printed on the pages.
"""
import numpy as np
import pytest
import torch

import oracle
from tests._common import golden_dict, golden_lines


def test_e2m1_values_match_handworked_table():
    for code, val in golden_lines("e2m1_codes.txt"):
        c = int(code, 16)
        got = oracle.e2m1_value(c)
        assert got == float(val), (code, got, val)
        assert np.signbit(got) == (c >= 8)


def test_e4m3_values_match_torch_float8_e4m3fn():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        got = oracle.e4m3_value(c)
        if np.isnan(ref[c]):
            assert np.isnan(got), c
        else:
            assert got == ref[c], (hex(c), got, ref[c])
    # landmarks of the FN variant
    assert oracle.e4m3_value(0x7E) == 448.0
    assert oracle.e4m3_value(0x01) == 2.0 ** -9
    assert oracle.e4m3_value(0x08) == 2.0 ** -6
    assert oracle.e4m3_value(0x38) == 1.0


def test_e2m1_rounding_handworked():
    for x, code in golden_lines("e2m1_rounding.txt"):
        assert oracle.e2m1_encode(np.float32(float(x))) == int(code, 16), (x, code)


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(0)
    # random magnitudes across the whole range + every representable value + every midpoint
    vals = list(np.float32(np.exp(rng.uniform(np.log(2.0 ** -12), np.log(440.0), 20000))))
    rep = sorted({oracle.e4m3_value(c) for c in range(0x7F)})
    vals += [np.float32(v) for v in rep]
    vals += [np.float32((a + b) / 2) for a, b in zip(rep[:-1], rep[1:])]
    vals += [np.float32(v) * np.float32(1 + 2 ** -20) for v in rep[1:]]
    x = torch.tensor(np.array(vals, dtype=np.float32))
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(v) for v in vals], dtype=np.uint8)
    bad = np.nonzero(ref != got)[0]
    assert bad.size == 0, [(vals[i], hex(got[i]), hex(ref[i])) for i in bad[:5]]


def test_e4m3_encode_saturates_and_ties():
    assert oracle.e4m3_encode(448.0) == 0x7E
    assert oracle.e4m3_encode(460.0) == 0x7E
    assert oracle.e4m3_encode(1e9) == 0x7E
    assert oracle.e4m3_encode(0.0) == 0x00
    # subnormal tie 1.5 * 2^-9 between codes 0x01 and 0x02 -> even mantissa (0x02)
    assert oracle.e4m3_encode(np.float32(1.5 * 2 ** -9)) == 0x02
    # 2.5 * 2^-9 between 0x02 and 0x03 -> 0x02
    assert oracle.e4m3_encode(np.float32(2.5 * 2 ** -9)) == 0x02
    # below half the smallest subnormal -> 0
    assert oracle.e4m3_encode(np.float32(0.5 * 2 ** -9)) == 0x00
    # 1.0625 is the tie between 1.0 (0x38) and 1.125 (0x39) -> 0x38
    assert oracle.e4m3_encode(1.0625) == 0x38
    assert oracle.e4m3_encode(1.1875) == 0x3A  # tie between 1.125 and 1.25 -> even (1.25)


def test_nvfp4_group_handworked():
    g = golden_dict("nvfp4_group.txt")
    st = float(g["tensor_scale"][0])
    x = np.array([float(v) for v in g["x"]], dtype=np.float32).reshape(1, 16)
    c = oracle.nvfp4_encode(x, st)
    assert list(c.data.reshape(-1)) == [int(b, 16) for b in g["bytes"]]
    assert list(c.scale.reshape(-1)) == [int(g["scale"][0], 16)]
    dec = oracle.nvfp4_decode(c).reshape(-1)
    assert list(dec) == [float(v) for v in g["decoded"]]


def test_nvfp4_zero_group_and_layout():
    x = np.zeros((3, 32), dtype=np.float32)
    x[1, 16:] = 1.0  # only the second group of vector 1 is nonzero
    c = oracle.nvfp4_encode(x, 1.0 / (6 * 448))
    assert c.data.shape == (3, 16) and c.scale.shape == (3, 2)
    assert not c.data[0].any() and not c.scale[0].any()
    assert c.scale[1, 0] == 0 and c.scale[1, 1] != 0
    assert not c.data[1, :8].any() and c.data[1, 8:].all()
    assert (oracle.nvfp4_decode(c) == x).all()


def test_nvfp4_round_trip_exact_on_grid():
    """Groups whose values lie on the grid and whose amax = 6*s*s_t decode back exactly."""
    rng = np.random.default_rng(1)
    st = np.float32(0.0123)
    scales = [oracle.e4m3_value(c) for c in range(0x10, 0x7E)]
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)
    xs = []
    for i in range(500):
        s = scales[rng.integers(len(scales))]
        m = rng.choice(grid, 16) * rng.choice([-1, 1], 16)
        m[rng.integers(16)] = 6.0 * rng.choice([-1, 1])
        denom = np.float32(np.float32(s) * st)
        xs.append((m * np.float64(denom)).astype(np.float32))
    x = np.stack(xs)
    c = oracle.nvfp4_encode(x, st)
    assert (oracle.nvfp4_decode(c) == x).all()


def test_nvfp4_error_bound_random():
    """|decode(encode(x)) - x| <= half an E2M1 step of the group's scale (+ E4M3 rounding slack)."""
    rng = np.random.default_rng(2)
    x = rng.standard_normal((256, 128)).astype(np.float32)
    st = oracle.tensor_scale(x)
    assert st == np.float32(np.abs(x).max()) / np.float32(2688.0)
    c = oracle.nvfp4_encode(x, st)
    y = oracle.nvfp4_decode(c)
    g = x.reshape(256, 8, 16)
    amax = np.abs(g).max(-1, keepdims=True)
    err = np.abs(y.reshape(256, 8, 16) - g)
    # E2M1 spacing is at most 2 * denom with denom ~ amax/6 (E4M3 rounding < 1/16 relative)
    assert (err <= amax / 6 * (1 + 1 / 16) + 1e-7).all()
    rel = np.linalg.norm(y - x) / np.linalg.norm(x)
    assert 0.05 < rel < 0.15  # 4-bit data with per-16 scales


def test_nvfp4_bytes_per_token_matches_pages():
    """9/16 byte per element = 34,560 / 61,440 (NVFP4 vs FP8 bytes per token on the pages)."""
    g = golden_dict("page_figures.txt")
    nv, f8 = int(g["nvfp4_bytes_per_token"][0]), int(g["fp8_bytes_per_token"][0])
    for dim in (64, 128):
        c = oracle.nvfp4_encode(np.ones((1, dim), dtype=np.float32), 1.0)
        per_elem = (c.data.nbytes + c.scale.nbytes) / dim
        assert per_elem == nv / f8 == 9 / 16
    assert 1 - nv / f8 == float(g["saving_fraction"][0])
