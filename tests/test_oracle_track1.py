"""Pins of the oracle's Track-1 block-scaled formats (oracle.qmv_block_scaled,
oracle.dequant_block_scaled_f32, and the E5M2 / signed-integer / block-scale
decoders) against things other than the oracle itself:

  * the format table typed from the wh-iron audit's Track 1 table
    (tests/golden/track1_formats.txt);
  * hand-worked E5M2 values and every E5M2 byte against torch's float8_e5m2
    cast and against numpy's binary16 (E5M2 is the top byte of a half);
  * hand-worked two's-complement fields, and every field of every width
    against numpy's int8 arithmetic shift;
  * FP16 / FP32 / E8M0 / E4M3 block scales against numpy / torch casts;
  * exact rational brute force of the dot product for all 30 formats, with
    codes read by a test-side bit reader and elements decoded by library
    casts (torch float8 types, numpy shifts) and the hand E2M1 table;
  * the exact fp32 rounding of every dequantized weight;
  * closed forms: all-zero codes give 0, a unit x selects a dequantized column;
  * the generic function reproduces the three original FP formats.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
FORMATS = sorted(oracle.TRACK1)


def _rows(name):
    out = []
    for line in open(os.path.join(GOLD, name)):
        line = line.strip()
        if line and not line.startswith("#"):
            out.append(line.split())
    return out


def _same(a, b):
    if math.isnan(b):
        return math.isnan(a)
    return a == b and math.copysign(1.0, a) == math.copysign(1.0, b)


# ------------------------------------------------------------- the table ----
def test_format_table_matches_the_pages():
    gold = _rows("track1_formats.txt")
    assert len(gold) == 30 and len(oracle.TRACK1) == 30
    for name, elem, block, scale, glob in gold:
        e, bits, blk, sk, ug = oracle.TRACK1[name]
        if elem.startswith("int"):
            assert (e, bits) == ("int", int(elem[3:])), name
        else:
            assert (e, bits) == (elem, 4 if elem == "e2m1" else 8), name
        assert blk == int(block) and sk == scale and ug == (glob == "fp32"), name


# ---------------------------------------------------------------- E5M2 -----
def test_e5m2_hand_values():
    for code, val in _rows("e5m2_spot.txt"):
        assert _same(oracle.e5m2(int(code, 0)), float(val)), code


def test_e5m2_every_byte_vs_torch_and_half():
    b = torch.arange(256, dtype=torch.uint8)
    ref = b.view(torch.float8_e5m2).to(torch.float64).numpy()
    half = (np.arange(256, dtype=np.uint16) << 8).view(np.float16).astype(np.float64)
    for c in range(256):
        got = oracle.e5m2(c)
        assert _same(got, float(ref[c])), hex(c)
        assert _same(got, float(half[c])), hex(c)


# ------------------------------------------------------- signed integers ----
def test_sint_hand_values():
    for bits, field, val in _rows("sint_values.txt"):
        assert oracle.sint(int(field), int(bits)) == float(val), (bits, field)


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 8])
def test_sint_every_field_vs_numpy_shift(bits):
    f = np.arange(1 << bits, dtype=np.uint16)
    # place the field at the top of an int8 and shift it back down arithmetically
    ref = ((f << (8 - bits)).astype(np.uint8).view(np.int8) >> (8 - bits)).astype(np.int64)
    got = [oracle.sint(int(v), bits) for v in f]
    assert got == [float(r) for r in ref]


# -------------------------------------------------------- block scales -----
def test_block_scales_vs_library_casts():
    g = np.random.default_rng(3)
    f32 = g.standard_normal(64).astype(np.float32)
    assert np.array_equal(oracle.block_scales(f32, 64, "f32"), f32.astype(np.float64))
    h = np.arange(0, 65536, 97, dtype=np.uint16)
    h = h[(h & 0x7C00) != 0x7C00]                 # finite halves, subnormals included
    ref = h.view(np.float16).astype(np.float64)
    assert np.array_equal(oracle.block_scales(h, len(h), "f16"), ref)
    e = np.arange(0, 255, dtype=np.uint8)
    assert list(oracle.block_scales(e, len(e), "e8m0")) == [math.ldexp(1.0, int(v) - 127) for v in e]
    b = np.arange(256, dtype=np.uint8)
    ref4 = torch.from_numpy(b).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got4 = oracle.block_scales(b, 256, "e4m3")
    assert all(_same(float(x), float(y)) for x, y in zip(got4, ref4))


# ---------------------------------------------- test-side exact decoding ----
_E2M1 = {int(c): float(v) for c, v in _rows("e2m1_values.txt")}
_E4M3 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
_E5M2 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e5m2).to(torch.float64).numpy()


def _fields(row, K, bits):
    """Test-side reader: K b-bit fields of the row's little-endian bit stream
    (numpy unpackbits in little bit order, then weights 2^i)."""
    bitsarr = np.unpackbits(np.asarray(row, dtype=np.uint8), bitorder="little")[: K * bits]
    return (bitsarr.reshape(K, bits).astype(np.int64) << np.arange(bits)).sum(axis=1)


def _elem_exact(field, elem, bits):
    if elem == "e2m1":
        return Fraction(_E2M1[int(field)])
    if elem == "e4m3":
        return Fraction(float(_E4M3[int(field)]))
    if elem == "e5m2":
        return Fraction(float(_E5M2[int(field)]))
    v = np.array([field << (8 - bits)], dtype=np.uint16).astype(np.uint8).view(np.int8)[0] >> (8 - bits)
    return Fraction(int(v))


def _scale_exact(raw, kind):
    if kind == "e8m0":
        return Fraction(2) ** (int(raw) - 127)
    if kind == "e4m3":
        return Fraction(float(_E4M3[int(raw)]))
    if kind == "f32":
        return Fraction(float(np.float32(raw)))
    return Fraction(float(np.uint16(raw).view(np.float16)))


def _w_exact(c, n, k):
    K, bits, blk = c["K"], c["bits"], c["block"]
    f = _fields(c["w"][0][n], K, bits)[k]
    v = _elem_exact(f, c["elem"], bits) * _scale_exact(c["scales"][0][n, k // blk], c["scale"])
    if c["use_global"]:
        v *= Fraction(float(c["global"]))
    return v


def _case(fmt, M, N, K, dtype, seed, **kw):
    return synth.bs_case(M, N, K, *oracle.TRACK1[fmt], dtype, seed=seed, **kw)


def _f32_round(fr: Fraction) -> float:
    f = np.float32(float(fr))
    best = None
    for cand in (f, np.nextafter(f, np.float32(np.inf)), np.nextafter(f, np.float32(-np.inf))):
        if not np.isfinite(cand):
            continue
        key = (abs(Fraction(float(cand)) - fr), int(np.float32(cand).view(np.uint32)) & 1)
        if best is None or key < best[0]:
            best = (key, cand)
    return float(best[1])


# ------------------------------------------------------- the dot product ----
@pytest.mark.parametrize("fmt", FORMATS)
def test_block_scaled_dot_exact_bruteforce(fmt):
    blk = oracle.TRACK1[fmt][2]
    M, N, K, dtype = 2, 3, 2 * max(blk, 32), "bf16"
    c = _case(fmt, M, N, K, dtype, seed=len(fmt) * 7 + 1)
    y, absdot = oracle.qmv_block_scaled(c["x"][0], c["w"][0], c["scales"][0], c["global"], M, N, K, fmt, dtype)
    xv = synth.storage_to_float(c["x"][0], dtype).astype(np.float64)
    for n in range(N):
        ws = [_w_exact(c, n, k) for k in range(K)]
        for m in range(M):
            acc = sum((Fraction(float(xv[m, k])) * ws[k] for k in range(K)), Fraction(0))
            tot = sum((abs(Fraction(float(xv[m, k])) * ws[k]) for k in range(K)), Fraction(0))
            assert abs(Fraction(y[m, n]) - acc) <= tot * Fraction(2) ** -45, (fmt, m, n)
            assert abs(Fraction(absdot[m, n]) - tot) <= tot * Fraction(2) ** -45


@pytest.mark.parametrize("fmt", FORMATS)
def test_block_scaled_dequant_rounds_the_exact_weight(fmt):
    blk = oracle.TRACK1[fmt][2]
    N, K = 3, 2 * max(blk, 32)
    c = _case(fmt, 1, N, K, "f32", seed=len(fmt) * 11 + 2)
    d = oracle.dequant_block_scaled_f32(c["w"][0], c["scales"][0], c["global"], N, K, fmt)
    for n in range(N):
        for k in range(K):
            assert d[n, k] == _f32_round(_w_exact(c, n, k)), (fmt, n, k)


@pytest.mark.parametrize("fmt", ["nvfp8", "fp8_e4m3", "fp8_e5m2_f16", "int8", "mxint3", "fp4_f16"])
def test_block_scaled_dequant_f16_subnormal_and_wide_scales(fmt):
    """Scales far from 1: f16 subnormal twins (where wide-range elements push
    them, per the audit) and large f32 scales, still one rounding."""
    blk = oracle.TRACK1[fmt][2]
    N, K = 2, 2 * max(blk, 32)
    lo = (1e-7, 5e-6) if oracle.TRACK1[fmt][3] == "f16" else (1e3, 1e5)
    c = _case(fmt, 1, N, K, "f32", seed=17, scale_range=lo)
    d = oracle.dequant_block_scaled_f32(c["w"][0], c["scales"][0], c["global"], N, K, fmt)
    for n in range(N):
        for k in range(K):
            assert d[n, k] == _f32_round(_w_exact(c, n, k))


@pytest.mark.parametrize("fmt", ["int2", "int5_f16", "mxint8", "fp4", "nvfp8_f16", "mxfp8_e5m2"])
def test_block_scaled_all_zero_codes_give_zero(fmt):
    blk = oracle.TRACK1[fmt][2]
    M, N, K = 2, 4, 2 * max(blk, 32)
    c = _case(fmt, M, N, K, "f16", seed=5)
    w = np.zeros_like(c["w"][0])
    y, a = oracle.qmv_block_scaled(c["x"][0], w, c["scales"][0], c["global"], M, N, K, fmt, "f16")
    assert np.all(y == 0.0) and np.all(a == 0.0)


@pytest.mark.parametrize("fmt", ["int3", "mxint6", "fp8_e5m2", "nvfp8", "fp4_f16", "nvfp4"])
def test_block_scaled_unit_x_selects_a_column(fmt):
    blk = oracle.TRACK1[fmt][2]
    M, N, K = 1, 5, 4 * max(blk, 32)
    c = _case(fmt, M, N, K, "f32", seed=9)
    d = oracle.dequant_block_scaled_f32(c["w"][0], c["scales"][0], c["global"], N, K, fmt)
    for k in (0, 1, K // 2 + 3, K - 1):
        x = np.zeros((1, K), np.float32)
        x[0, k] = 1.0
        y, _ = oracle.qmv_block_scaled(x, c["w"][0], c["scales"][0], c["global"], M, N, K, fmt, "f32")
        # y is the exact weight (every product fits fp64); the fp32 dequant is
        # its one rounding
        ref = [float(_w_exact(c, n, k)) for n in range(N)]
        assert np.array_equal(y[0], np.array(ref)), (fmt, k)
        assert np.array_equal(d[:, k], y[0].astype(np.float32)), (fmt, k)


@pytest.mark.parametrize("fmt,mode", [("nvfp4", "nvfp4"), ("mxfp4", "mxfp4"), ("mxfp8_e4m3", "mxfp8")])
def test_block_scaled_reproduces_the_original_fp_formats(fmt, mode):
    M, N, K, dtype = 3, 7, 256, "bf16"
    c = synth.fp_case(M, N, K, mode, dtype, seed=23)
    a = oracle.qmv_block_scaled(c["x"][0], c["w"][0], c["scales"][0], c["global"], M, N, K, fmt, dtype)
    b = oracle.qmv_fp(c["x"][0], c["w"][0], c["scales"][0], c["global"], M, N, K, mode, dtype)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_nvfp4_with_a_16_code_tail_block():
    """K % 32 == 16 is a valid NVFP4 shape (blocks of 16): brute force."""
    M, N, K = 2, 3, 48
    c = _case("nvfp4", M, N, K, "f32", seed=31)
    y, _ = oracle.qmv_block_scaled(c["x"][0], c["w"][0], c["scales"][0], c["global"], M, N, K, "nvfp4", "f32")
    xv = c["x"][0].astype(np.float64)
    for n in range(N):
        for m in range(M):
            acc = sum((Fraction(float(xv[m, k])) * _w_exact(c, n, k) for k in range(K)), Fraction(0))
            assert abs(Fraction(y[m, n]) - acc) <= abs(acc) * Fraction(2) ** -40 + Fraction(2) ** -60
