"""Pins of the oracle's number formats against things other than itself:
the page's E2M1 table, library casts (ml_dtypes), and the exhaustive C sweep
(all 2^32 fp32 inputs, brute force vs arithmetic restatement)."""
import os
import subprocess

import ml_dtypes
import numpy as np
import pytest

from oracle import formats as F

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _golden_table():
    rows = []
    with open(os.path.join(ROOT, "tests", "golden", "e2m1_table.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            c, v = line.split()
            rows.append((int(c), float(v)))
    return rows


def test_e2m1_decode_matches_page_table():
    rows = _golden_table()
    assert len(rows) == 16
    for c, v in rows:
        got = F.e2m1_decode(np.array([c], dtype=np.uint8))[0]
        assert got == v and np.signbit(got) == np.signbit(v), (c, v, got)


def test_e2m1_round_trip_all_codes():
    codes = np.arange(16, dtype=np.uint8)
    vals = F.e2m1_decode(codes).astype(np.float32)
    assert np.array_equal(F.e2m1_encode(vals), codes)


def _boundary_windows(points, width):
    """All fp32 within +-width ulps of each point (both signs)."""
    out = []
    for p in points:
        b = np.array([p], dtype=np.float32).view(np.uint32)[0].astype(np.int64)
        lo = max(b - width, 0)
        bits = np.arange(lo, b + width + 1, dtype=np.int64).astype(np.uint32)
        v = bits.view(np.float32)
        out.append(v)
        out.append(-v)
    return np.concatenate(out)


def _all_bf16_patterns():
    bits = (np.arange(1 << 16, dtype=np.uint32) << 16).view(np.float32)
    return bits[np.isfinite(bits)]


def test_e2m1_encode_matches_ml_dtypes_cast():
    mids = [0.0, 0.25, 0.5, 0.75, 1.0, 1.25, 1.5, 1.75, 2.0, 2.5, 3.0, 3.5, 4.0, 5.0, 6.0, 7.0, 8.0]
    rng = np.random.default_rng(0)
    rnd = rng.integers(0, 2**32, size=1 << 20, dtype=np.uint64).astype(np.uint32).view(np.float32)
    rnd = rnd[np.isfinite(rnd)]
    x = np.concatenate([_boundary_windows(mids, 4096), _all_bf16_patterns(), rnd]).astype(np.float32)
    ours = F.e2m1_encode(x)
    lib = x.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    bad = np.nonzero(ours != lib)[0]
    assert bad.size == 0, f"{bad.size} mismatches, e.g. x={x[bad[:5]]} ours={ours[bad[:5]]} lib={lib[bad[:5]]}"


def test_e2m1_ties_listed_in_reading():
    # the reading's tie list: 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4, >=6 -> 6
    x = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 100.0, -0.1, -0.0], dtype=np.float32)
    want = np.array([0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 6.0, 6.0, -0.0, -0.0])
    got = F.e2m1_decode(F.e2m1_encode(x))
    assert np.array_equal(got, want)
    assert np.array_equal(np.signbit(got), np.signbit(want))


def test_e4m3_values_closed_form():
    v = F.E4M3_VALUES
    assert v[0] == 0 and v[1] == 2.0**-9 and v[0x08] == 2.0**-6 and v[0x38] == 1.0 and v[0x7E] == 448.0
    assert np.all(np.diff(v) > 0)


def test_e4m3_encode_matches_ml_dtypes_cast_in_range():
    mids = list(F.E4M3_VALUES[:-1] + np.diff(F.E4M3_VALUES) / 2) + list(F.E4M3_VALUES)
    x = np.abs(np.concatenate([_boundary_windows(mids, 64), _all_bf16_patterns()])).astype(np.float32)
    x = x[x <= 448.0]
    ours = F.e4m3_encode_pos(x)
    lib = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    bad = np.nonzero(ours != lib)[0]
    assert bad.size == 0, f"{bad.size} mismatches, e.g. x={x[bad[:5]]}"


def test_e4m3_saturates_at_448():
    x = np.array([448.0, 449.0, 464.0, 500.0, 3.0e38], dtype=np.float32)
    assert np.all(F.e4m3_encode_pos(x) == 0x7E)


def test_ue8m0_decode():
    assert F.ue8m0_decode(np.array([127]))[0] == 1.0
    assert F.ue8m0_decode(np.array([0]))[0] == 2.0**-127
    assert F.ue8m0_decode(np.array([254]))[0] == 2.0**127
    assert np.isnan(F.ue8m0_decode(np.array([255]))[0])


def test_floor_log2_exact_including_subnormals():
    e = np.arange(-149, 128)
    x = np.ldexp(1.0, e).astype(np.float32)
    assert np.array_equal(F.floor_log2_f32(x), e)
    # just below each power of two (normal range) the floor drops by one
    xb = np.nextafter(x[30:], np.float32(0), dtype=np.float32)
    assert np.array_equal(F.floor_log2_f32(xb), e[30:] - 1)


def test_nibble_packing_order():
    codes = np.array([[1, 2, 3, 4]], dtype=np.uint8)
    packed = F.pack_nibbles(codes)
    assert packed.tolist() == [[0x21, 0x43]]
    assert np.array_equal(F.unpack_nibbles(packed), codes)
    # the same convention as the library's packed-pair cast
    lib = np.array([0.5, 1.0], dtype=np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8)
    assert F.pack_nibbles(lib[None, :])[0, 0] == (lib[0] | (lib[1] << 4))


def test_bf16_rounding_matches_library_on_fp32_inputs():
    import torch

    rng = np.random.default_rng(1)
    x = rng.standard_normal(1 << 16).astype(np.float32) * np.float32(3.0)
    x = np.concatenate([x, _boundary_windows([1.0, 1.00390625, 3.0], 256)]).astype(np.float32)
    ours = F.f64_to_bf16_rne(x.astype(np.float64))
    lib = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, lib)


def test_bf16_rounding_is_single_step_from_fp64():
    # 1 + 2^-8 + 2^-30 lies just above the bf16 midpoint between 1 and 1+2^-7:
    # one rounding from fp64 goes up; rounding to fp32 first would land exactly
    # on the midpoint (1 + 2^-8 + 2^-30 -> 1 + 2^-8 in fp32) and tie to 1.0.
    x = np.array([1.0 + 2.0**-8 + 2.0**-30])
    up = F.bf16_bits_to_f32(F.f64_to_bf16_rne(x))[0]
    assert up == np.float32(1.0 + 2.0**-7)


def _sweep_binary():
    exe = os.path.join(ROOT, "oracle", "_build", "sweep")
    src = os.path.join(ROOT, "oracle", "sweep.c")
    if not os.path.exists(exe) or os.path.getmtime(exe) < os.path.getmtime(src):
        os.makedirs(os.path.dirname(exe), exist_ok=True)
        subprocess.check_call(["gcc", "-O2", "-o", exe, src, "-lm", "-lpthread"])
    return exe


@pytest.mark.parametrize("fmt", ["e2m1", "e4m3"])
def test_exhaustive_sweep_brute_force_vs_arithmetic(fmt):
    exe = _sweep_binary()
    n = str(min(32, max(1, len(os.sched_getaffinity(0)))))
    out = subprocess.run([exe, fmt, n], capture_output=True, text=True, timeout=900)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "mismatches=0" in out.stdout
