"""Pins for the oracle's float32 -> fp16 / bf16 conversion and 16-bit decode.

The conversion is the operation of float32ToFloat16Bits / float32ToBFloat16Bits
in makarna/pkg/kvcache/paged_cache.go: nearest value, ties to the even
fraction, overflow to infinity; NaN inputs are quieted with the payload's top
bits kept (the reading of the NaN case). It is pinned three ways: hand-derived
cases (tests/golden/convert_cases.txt), GCC's own IEEE casts over ALL 2^32
float32 patterns, and numpy's float16 cast on a random sample.
"""

import ctypes as C
import os
import subprocess

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def _golden():
    rows = []
    with open(os.path.join(HERE, "golden", "convert_cases.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                a, b, c = (int(x, 16) for x in line.split())
                rows.append((a, b, c))
    return rows


@pytest.fixture(scope="module")
def pin_lib(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("pins") / "gcc_casts.so")
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", out,
                           os.path.join(HERE, "pins", "gcc_casts.c")])
    L = C.CDLL(out)
    L.pin_compare_range.restype = C.c_int64
    L.pin_compare_range.argtypes = [C.c_uint64, C.c_uint64, C.c_int, C.c_void_p, C.POINTER(C.c_int64)]
    L.pin_cast.restype = C.c_uint16
    L.pin_cast.argtypes = [C.c_uint32, C.c_int]
    return L


def test_golden_hand_cases(orc):
    rows = _golden()
    assert len(rows) >= 20
    bits = np.array([r[0] for r in rows], dtype=np.uint32)
    f = bits.view(np.float32)
    assert np.array_equal(orc.convert(f, "f16"), np.array([r[1] for r in rows], dtype=np.uint16))
    assert np.array_equal(orc.convert(f, "bf16"), np.array([r[2] for r in rows], dtype=np.uint16))


def test_golden_cases_agree_with_gcc(pin_lib):
    # the hand derivations themselves are checked against the compiler's casts
    for a, b, c in _golden():
        assert pin_lib.pin_cast(a, 1) == b, hex(a)
        assert pin_lib.pin_cast(a, 2) == c, hex(a)


@pytest.mark.parametrize("kv_dtype,code", [("f16", 1), ("bf16", 2)])
def test_exhaustive_all_float32_patterns(orc, pin_lib, kv_dtype, code):
    chunk = 1 << 28
    for start in range(0, 1 << 32, chunk):
        got = orc.convert_range(start, chunk, kv_dtype)
        first = C.c_int64(-1)
        bad = pin_lib.pin_compare_range(start, chunk, code, got.ctypes.data_as(C.c_void_p), C.byref(first))
        assert bad == 0, f"{kv_dtype}: {bad} mismatches, first at pattern {start + first.value:#010x}"


def test_f16_matches_numpy_on_sample(orc):
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 1 << 32, size=1 << 20, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    finite = ~np.isnan(x)
    want = x[finite].astype(np.float16).view(np.uint16)
    assert np.array_equal(orc.convert(x[finite], "f16"), want)


def test_decode_f16_all_patterns(orc):
    b = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = orc.value16(b, "f16")
    want = b.view(np.float16).astype(np.float64)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])
    # signed zeros keep their sign
    assert np.signbit(got[0x8000]) and not np.signbit(got[0])


def test_decode_bf16_all_patterns(orc):
    b = np.arange(1 << 16, dtype=np.uint32)
    got = orc.value16(b.astype(np.uint16), "bf16")
    want = (b << 16).astype(np.uint32).view(np.float32).astype(np.float64)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])


def test_round_trip_is_identity_on_16bit_values(orc):
    # every finite 16-bit value converts back to itself (value -> float32 is exact)
    for kv in ("f16", "bf16"):
        b = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
        vals = orc.value16(b, kv)
        fin = np.isfinite(vals)
        back = orc.convert(vals[fin].astype(np.float32), kv)
        assert np.array_equal(back, b[fin]), kv
