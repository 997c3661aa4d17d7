"""Pins of the fp64 oracle to things other than itself (CPU only).

Each test ties one oracle function to a value printed on the pages, a hand-worked
example, a library routine, a closed form, an invariant or exact rational brute
force, so that a dropped term, wrong sign, wrong index or transposed operand in
the oracle fails at least one of them:

  codecs           E2M1 hand table (all 16 codes), E4M3 all 256 bytes vs torch's
                   float8_e4m3fn + spot values, E8M0 spot values, binary16 /
                   bfloat16 decoders vs numpy / torch for every bit pattern;
  affine unpack    pack geometry, hand-packed rows for every width, and the
                   single-bit bijection invariant of the LSB-first reading;
  dequantization   min/max quantize -> pack -> dequantize round trip; fp32
                   rounding vs exact rationals (round-to-odd sum);
  product          exact Fraction brute force on tiny shapes (affine and FP),
                   the all-zero-code closed form, x = e_k selects a column;
  sum(x)           the emulated low-precision sum(x) mutant fails the test
                   tolerance on the precision case, the widened sum passes;
  quantizer        fp32 -> binary16 / bfloat16 rounding vs numpy / torch; codes
                   of weights on an exact grid recovered bit for bit for every
                   width (through the pinned unpack); a constant group; brute
                   force nearest code in exact rationals.
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
from qmv_tol import check

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _read_pairs(name):
    rows = []
    for line in open(os.path.join(GOLD, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        a, b = line.split()
        rows.append((int(a, 0), float(b)))
    return rows


def _same(a, b):
    if math.isnan(b):
        return math.isnan(a)
    return a == b and math.copysign(1.0, a) == math.copysign(1.0, b)


# ---------------------------------------------------------------- codecs ----
def test_e2m1_hand_table():
    rows = _read_pairs("e2m1_values.txt")
    assert len(rows) == 16
    for c, v in rows:
        assert _same(oracle.e2m1(c), v), (c, oracle.e2m1(c), v)


def test_e4m3_all_bytes_vs_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        assert _same(oracle.e4m3(c), float(ref[c])), (hex(c), oracle.e4m3(c), ref[c])


def test_e4m3_spot_values():
    for c, v in _read_pairs("e4m3_spot.txt"):
        assert _same(oracle.e4m3(c), v), (hex(c), oracle.e4m3(c), v)


def test_e8m0_spot_values():
    for e, v in _read_pairs("e8m0_spot.txt"):
        assert _same(oracle.e8m0(e), v), (e, oracle.e8m0(e), v)


def test_e8m0_vs_torch_if_available():
    if not hasattr(torch, "float8_e8m0fnu"):
        pytest.skip("torch has no float8_e8m0fnu")
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    for e in range(256):
        assert _same(oracle.e8m0(e), float(ref[e])), (e, oracle.e8m0(e), ref[e])


def test_f16_decoder_every_pattern():
    pats = np.arange(65536, dtype=np.uint32)
    ref = pats.astype(np.uint16).view(np.float16).astype(np.float64)
    got = np.array([oracle.f16_value(int(p)) for p in pats])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    m = ~np.isnan(ref)
    assert np.array_equal(got[m], ref[m])
    assert np.array_equal(np.signbit(got[m]), np.signbit(ref[m]))


def test_bf16_decoder_every_pattern():
    pats = torch.arange(65536, dtype=torch.int32).to(torch.int16)
    ref = pats.view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.bf16_value(p & 0xFFFF) for p in range(65536)])
    got = got[np.arange(65536).astype(np.int16).astype(np.int64) & 0xFFFF]
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    m = ~np.isnan(ref)
    assert np.array_equal(got[m], ref[m])


# --------------------------------------------------------- affine unpack ----
def test_pack_geometry():
    # get_pack_factor / get_bytes_per_pack with an 8-bit word (MLX quantized_nax.h)
    expect = {2: (4, 1), 3: (8, 3), 4: (2, 1), 5: (8, 5), 6: (4, 3), 8: (1, 1)}
    for bits, (pf, bpp) in expect.items():
        assert oracle.pack_factor(bits) == pf
        assert oracle.bytes_per_pack(bits) == bpp
        for K in (32, 64, 128, 512, 2560, 4096):
            assert oracle.row_bytes(K, bits) * 8 == K * bits


def _golden_packs():
    out = []
    for line in open(os.path.join(GOLD, "affine_packs.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        b, codes, by = (s.strip() for s in line.split("|"))
        out.append((int(b), [int(c) for c in codes.split()], bytes.fromhex(by.replace(" ", ""))))
    return out


@pytest.mark.parametrize("bits,codes,packed", _golden_packs())
def test_affine_hand_packed_rows(bits, codes, packed):
    row = np.frombuffer(packed, dtype=np.uint8)
    assert len(codes) * bits == 8 * len(packed)
    got = oracle.affine_codes(row, len(codes), bits)
    assert list(got) == codes


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 8])
def test_affine_single_bit_bijection(bits):
    """Setting bit t of an all-zero row (bits counted LSB-first through the
    bytes) must set exactly code t // bits to 2^(t % bits)."""
    nbytes = 15 if bits in (3, 5) else 6           # whole packs
    K = nbytes * 8 // bits
    for t in range(nbytes * 8):
        row = np.zeros(nbytes, dtype=np.uint8)
        row[t // 8] = 1 << (t % 8)
        got = oracle.affine_codes(row, K, bits)
        want = np.zeros(K, dtype=np.uint32)
        want[t // bits] = 1 << (t % bits)
        assert np.array_equal(got, want), (bits, t, got, want)


# ------------------------------------------------------------ helpers -------
def _py_pack(codes, bits):
    """Test-side packer: a plain LSB-first bit stream writer."""
    v = 0
    for i, c in enumerate(codes):
        assert 0 <= c < (1 << bits)
        v |= int(c) << (bits * i)
    n = len(codes) * bits // 8
    return np.frombuffer(v.to_bytes(n, "little"), dtype=np.uint8).copy()


def _py_codes(row, K, bits):
    v = int.from_bytes(bytes(row), "little")
    return [(v >> (bits * i)) & ((1 << bits) - 1) for i in range(K)]


def _val(raw, dtype):
    """Exact values of raw storage via library casts (numpy / torch)."""
    return synth.storage_to_float(np.asarray(raw), dtype).astype(np.float64)


def _f32_round(fr: Fraction) -> float:
    """Correctly rounded (nearest, ties to even) float32 of an exact rational."""
    f = np.float32(float(fr))
    cands = [f, np.nextafter(f, np.float32(np.inf)), np.nextafter(f, np.float32(-np.inf))]
    best = None
    for c in cands:
        if not np.isfinite(c):
            continue
        d = abs(Fraction(float(c)) - fr)
        key = (d, int(np.float32(c).view(np.uint32)) & 1)
        if best is None or key < best[0]:
            best = (key, c)
    return float(best[1])


# ---------------------------------------------------------- dequant pins ----
@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 8])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_minmax_roundtrip(bits, dtype):
    """Host min/max quantizer (scale = (max - min) / (2^b - 1), bias = min,
    q = round((w - bias) / scale)), test-side packer, then the oracle's
    dequantization: |w - w_hat| <= scale / 2 (+ dtype rounding of scale/bias)
    and the codes come back exactly from w_hat."""
    g = np.random.default_rng(bits)
    N, K, group = 3, 128, 32
    w = g.standard_normal((N, K))
    qmax = (1 << bits) - 1
    codes = np.zeros((N, K), dtype=np.int64)
    s_vals = np.zeros((N, K // group)); b_vals = np.zeros((N, K // group))
    for n in range(N):
        for j in range(K // group):
            blk = w[n, j * group:(j + 1) * group]
            lo, hi = blk.min(), blk.max()
            s_vals[n, j], b_vals[n, j] = (hi - lo) / qmax, lo
    s_raw = synth.to_storage(s_vals, dtype); b_raw = synth.to_storage(b_vals, dtype)
    s_q, b_q = _val(s_raw, dtype), _val(b_raw, dtype)
    for n in range(N):
        for k in range(K):
            j = k // group
            codes[n, k] = min(qmax, max(0, round((w[n, k] - b_q[n, j]) / s_q[n, j])))
    packed = np.stack([_py_pack(codes[n], bits) for n in range(N)])
    w_hat = oracle.dequant_affine_f32(packed, s_raw, b_raw, N, K, bits, group, dtype)
    for n in range(N):
        for k in range(K):
            j = k // group
            # exact dequant of the stored code, rounded once to fp32
            assert w_hat[n, k] == _f32_round(Fraction(s_q[n, j]) * int(codes[n, k]) + Fraction(b_q[n, j]))
            back = round((float(w_hat[n, k]) - b_q[n, j]) / s_q[n, j])
            assert back == codes[n, k]
    err = np.abs(w - w_hat.astype(np.float64))
    tol = np.repeat(s_q, group, axis=1) * 0.5 + np.abs(w) * 2.0 ** -7 + 1e-6
    # bf16 rounding of the min/max moves the grid a little; clamped ends may add one step
    tol += np.repeat(s_q, group, axis=1) * (1.0 if dtype == "bf16" else 1e-6)
    assert (err <= tol).all()


def test_round_f32_sum_exact():
    g = np.random.default_rng(7)
    cases = []
    for _ in range(2000):
        a = float(np.float32(g.standard_normal()) * np.float32(g.integers(0, 256)))
        b = float(np.float32(g.standard_normal() * 10.0 ** g.integers(-30, 4)))
        cases.append((a, b))
    # adversarial: the fp64 sum rounds to an exact fp32 tie
    one = 1.0
    cases += [(one + 2.0 ** -24, 2.0 ** -80), (one + 2.0 ** -24, -2.0 ** -80),
              (one + 3 * 2.0 ** -24, 2.0 ** -79), (-(one + 2.0 ** -24), -2.0 ** -80)]
    for a, b in cases:
        want = _f32_round(Fraction(a) + Fraction(b))
        got = oracle.round_f32_sum(a, b)
        assert got == want, (a, b, got, want)


@pytest.mark.parametrize("mode", ["mxfp4", "nvfp4", "mxfp8"])
def test_fp_dequant_exact(mode):
    c = synth.fp_case(1, 4, 64, mode, "bf16", seed=11)
    w, sc = c["w"][0], c["scales"][0]
    glob = c["global"]
    out = oracle.dequant_fp_f32(w, sc, glob, 4, 64, mode)
    e2m1 = {cc: v for cc, v in _read_pairs("e2m1_values.txt")}
    e4 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    blk = synth.FP_BLOCK[mode]
    for n in range(4):
        for k in range(64):
            if mode == "mxfp8":
                e = Fraction(float(e4[w[n, k]]))
            else:
                e = Fraction(e2m1[(int(w[n, k // 2]) >> (4 * (k % 2))) & 0xF])
            s = int(sc[n, k // blk])
            if mode == "nvfp4":
                want = _f32_round(e * Fraction(float(e4[s])) * Fraction(float(glob)))
            else:
                want = _f32_round(e * Fraction(2) ** (s - 127))
            assert out[n, k] == want, (mode, n, k, out[n, k], want)


# ---------------------------------------------------------- product pins ----
@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 8])
@pytest.mark.parametrize("group", [32, 64])
@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
def test_affine_dot_exact_bruteforce(bits, group, dtype):
    M, N, K = 2, 3, 2 * group
    c = synth.affine_case(M, N, K, bits, group, dtype, seed=bits * 100 + group)
    x, w, s, b = c["x"][0], c["w"][0], c["scales"][0], c["biases"][0]
    y, absdot = oracle.qmv_affine(x, w, s, b, M, N, K, bits, group, dtype)
    xv, sv, bv = _val(x, dtype), _val(s, dtype), _val(b, dtype)
    for n in range(N):
        codes = _py_codes(w[n], K, bits)
        for m in range(M):
            acc = Fraction(0); aacc = Fraction(0)
            for k in range(K):
                j = k // group
                t = Fraction(xv[m, k]) * (Fraction(sv[n, j]) * codes[k] + Fraction(bv[n, j]))
                acc += t; aacc += abs(t)
            assert abs(Fraction(y[m, n]) - acc) <= aacc * Fraction(2) ** -40
            assert abs(Fraction(absdot[m, n]) - aacc) <= aacc * Fraction(2) ** -40


@pytest.mark.parametrize("mode", ["mxfp4", "nvfp4", "mxfp8"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_fp_dot_exact_bruteforce(mode, dtype):
    M, N, K = 2, 3, 64
    c = synth.fp_case(M, N, K, mode, dtype, seed=5)
    x, w, sc, glob = c["x"][0], c["w"][0], c["scales"][0], c["global"]
    y, absdot = oracle.qmv_fp(x, w, sc, glob, M, N, K, mode, dtype)
    xv = _val(x, dtype)
    e2m1 = {cc: v for cc, v in _read_pairs("e2m1_values.txt")}
    e4 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    blk = synth.FP_BLOCK[mode]
    for n in range(N):
        for m in range(M):
            acc = Fraction(0)
            for k in range(K):
                if mode == "mxfp8":
                    e = Fraction(float(e4[w[n, k]]))
                else:
                    e = Fraction(e2m1[(int(w[n, k // 2]) >> (4 * (k % 2))) & 0xF])
                s = int(sc[n, k // blk])
                scale = (Fraction(float(e4[s])) * Fraction(float(glob))) if mode == "nvfp4" \
                    else Fraction(2) ** (s - 127)
                acc += Fraction(xv[m, k]) * e * scale
            assert abs(Fraction(y[m, n]) - acc) <= Fraction(absdot[m, n]) * Fraction(2) ** -40


@pytest.mark.parametrize("bits", [3, 4, 6])
def test_all_zero_codes_closed_form(bits):
    """q = 0 everywhere: y[m, n] = sum_groups bias[n, g] * sum_{k in g} x[m, k]."""
    M, N, K, group = 2, 4, 256, 64
    c = synth.affine_case(M, N, K, bits, group, "bf16", seed=3)
    w = np.zeros_like(c["w"][0])
    y, _ = oracle.qmv_affine(c["x"][0], w, c["scales"][0], c["biases"][0], M, N, K, bits, group, "bf16")
    xv, bv = _val(c["x"][0], "bf16"), _val(c["biases"][0], "bf16")
    for m in range(M):
        for n in range(N):
            want = sum(Fraction(bv[n, j]) * sum(Fraction(v) for v in xv[m, j * group:(j + 1) * group])
                       for j in range(K // group))
            assert abs(Fraction(y[m, n]) - want) <= abs(want) * Fraction(2) ** -48 + Fraction(2) ** -200


@pytest.mark.parametrize("bits", [2, 5, 8])
def test_unit_x_selects_column(bits):
    """x = e_k: y[0, n] = scale[n, k/g] * q[n, k] + bias[n, k/g] (codes from the
    test-side reader, values from library casts)."""
    N, K, group = 5, 128, 32
    c = synth.affine_case(1, N, K, bits, group, "f32", seed=9)
    for k in (0, 1, 37, 127):
        x = np.zeros((1, K), dtype=np.float32); x[0, k] = 1.0
        y, _ = oracle.qmv_affine(x, c["w"][0], c["scales"][0], c["biases"][0], 1, N, K, bits, group, "f32")
        for n in range(N):
            q = _py_codes(c["w"][0][n], K, bits)[k]
            want = float(c["scales"][0][n, k // group]) * q + float(c["biases"][0][n, k // group])
            assert y[0, n] == want


# ------------------------------------------------------------- qvm pins ----
@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 8])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_qvm_equals_qmv_of_the_transpose(bits, dtype):
    """qvm over W stored [K, N] equals qmv over W^T stored [N, K].  The test
    transposes the codes with its own bit-stream reader and writer.  qvm's
    scales and biases are drawn constant over blocks of 32 rows, so W^T's
    parameters fit qmv's [N, K/32] layout: p^T[n, kb] = p[32 kb, n / group].
    Both sums run over k in order on the same fp64 terms: equal bit for bit."""
    M, N, K, group = 2, 128, 96, 64
    c = synth.qvm_case(M, N, K, bits, group, dtype, seed=bits)
    sc = np.repeat(c["scales"][::32], 32, axis=0).copy()
    bi = np.repeat(c["biases"][::32], 32, axis=0).copy()
    y, a = oracle.qvm_affine(c["x"], c["w"], sc, bi, M, N, K, bits, group, dtype)
    codes = np.array([_py_codes(c["w"][k], N, bits) for k in range(K)])      # [K, N]
    wt = np.stack([_py_pack(codes[:, n], bits) for n in range(N)])          # [N, K*bits/8]
    cols = np.arange(N) // group
    sct = np.ascontiguousarray(sc[::32][:, cols].T)                          # [N, K/32]
    bit = np.ascontiguousarray(bi[::32][:, cols].T)
    yt, at = oracle.qmv_affine(c["x"], wt, sct, bit, M, N, K, bits, 32, dtype)
    assert np.array_equal(y, yt) and np.array_equal(a, at)


@pytest.mark.parametrize("bits", [2, 3, 5, 8])
def test_qvm_unit_x_selects_row(bits):
    """x = e_k: y[0, n] = scale[k, n/g] * q[k, n] + bias[k, n/g] (codes from the
    test-side reader, values from library casts)."""
    N, K, group = 96, 40, 32
    c = synth.qvm_case(1, N, K, bits, group, "f32", seed=11)
    for k in (0, 1, 17, 39):
        x = np.zeros((1, K), dtype=np.float32); x[0, k] = 1.0
        y, _ = oracle.qvm_affine(x, c["w"], c["scales"], c["biases"], 1, N, K, bits, group, "f32")
        q = _py_codes(c["w"][k], N, bits)
        for n in range(N):
            want = float(c["scales"][k, n // group]) * q[n] + float(c["biases"][k, n // group])
            assert y[0, n] == want, (k, n)


@pytest.mark.parametrize("bits", [3, 4, 6])
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_qvm_exact_bruteforce(bits, dtype):
    """Random per-(k, group) scales and biases: y against exact rationals."""
    M, N, K, group = 2, 64, 24, 32
    c = synth.qvm_case(M, N, K, bits, group, dtype, seed=bits + 50)
    y, absdot = oracle.qvm_affine(c["x"], c["w"], c["scales"], c["biases"], M, N, K, bits, group, dtype)
    xv, sv, bv = _val(c["x"], dtype), _val(c["scales"], dtype), _val(c["biases"], dtype)
    codes = [_py_codes(c["w"][k], N, bits) for k in range(K)]
    for m in range(M):
        for n in range(0, N, 7):
            acc = Fraction(0); aacc = Fraction(0)
            for k in range(K):
                t = Fraction(xv[m, k]) * (Fraction(sv[k, n // group]) * codes[k][n] + Fraction(bv[k, n // group]))
                acc += t; aacc += abs(t)
            assert abs(Fraction(y[m, n]) - acc) <= aacc * Fraction(2) ** -40
            assert abs(Fraction(absdot[m, n]) - aacc) <= aacc * Fraction(2) ** -40


# ---------------------------------------------------------- gather pins ----
def _expert_stack(E, N, K, bits, group, seed):
    cs = [synth.affine_case(1, N, K, bits, group, "f32", seed=seed + e) for e in range(E)]
    return (np.stack([c["w"][0] for c in cs]), np.stack([c["scales"][0] for c in cs]),
            np.stack([c["biases"][0] for c in cs]))


def test_gather_unit_x_selects_the_routed_expert():
    """x[t] = e_k: y[t, 0, n] is element (n, k) of expert ids[t]'s weights
    (codes from the test-side reader, values from library casts)."""
    E, N, K, bits, group = 4, 6, 64, 4, 32
    w, sc, bi = _expert_stack(E, N, K, bits, group, seed=40)
    ids = np.array([2, 0, 2, 3], dtype=np.int32)
    ks = [5, 17, 40, 63]
    x = np.zeros((len(ids), 1, K), dtype=np.float32)
    for t, k in enumerate(ks):
        x[t, 0, k] = 1.0
    y, _ = oracle.qmv_affine_gather(x, w, sc, bi, ids, 1, N, K, bits, group, "f32", E)
    for t, (e, k) in enumerate(zip(ids, ks)):
        for n in range(N):
            q = _py_codes(w[e, n], K, bits)[k]
            assert y[t, 0, n] == float(sc[e, n, k // group]) * q + float(bi[e, n, k // group])


def test_gather_token_permutation_and_bad_id():
    """Permuting the tokens (x rows with their ids) permutes the outputs; an
    id outside the stack gives a NaN token and leaves the others unchanged."""
    E, N, K, bits, group = 3, 5, 64, 3, 32
    w, sc, bi = _expert_stack(E, N, K, bits, group, seed=60)
    x = synth.affine_case(2, 1, K, bits, group, "f32", seed=61, batch=4)["x"]         # [4, 2, K]
    ids = np.array([1, 2, 0, 1], dtype=np.int32)
    y, _ = oracle.qmv_affine_gather(x, w, sc, bi, ids, 2, N, K, bits, group, "f32", E)
    perm = np.array([3, 1, 0, 2])
    yp, _ = oracle.qmv_affine_gather(np.ascontiguousarray(x[perm]), w, sc, bi, ids[perm], 2, N, K, bits, group,
                                     "f32", E)
    assert np.array_equal(yp, y[perm])
    bad = ids.copy(); bad[2] = E
    yb, _ = oracle.qmv_affine_gather(x, w, sc, bi, bad, 2, N, K, bits, group, "f32", E)
    assert np.isnan(yb[2]).all() and np.array_equal(np.delete(yb, 2, 0), np.delete(y, 2, 0))


# ------------------------------------------------------------ sum(x) pin ----
def _emulate_kernel_bf16(case, widened):
    """fp32 emulation of a qmv whose bias term uses sum(x) per group, either
    widened per element (correct) or formed as bf16 sums of 4 consecutive x
    before widening (the low-precision variant MLX's fix removed)."""
    K, g = case["K"], case["group"]
    x = _val(case["x"][0], "bf16").astype(np.float32)[0]
    w = case["w"][0]
    N = w.shape[0]
    bits = case["bits"]
    s = _val(case["scales"][0], "bf16").astype(np.float32)
    b = _val(case["biases"][0], "bf16").astype(np.float32)
    codes = np.array([_py_codes(w[n], K, bits) for n in range(N)], dtype=np.float32)
    ng = K // g
    xq = (codes * x[None, :]).reshape(N, ng, g).astype(np.float64).sum(-1).astype(np.float32)
    if widened:
        sx = x.reshape(ng, g).astype(np.float32).sum(-1, dtype=np.float32)
    else:
        xt = torch.from_numpy(x.reshape(ng, g // 4, 4)).to(torch.bfloat16)
        four = ((xt[..., 0] + xt[..., 1]) + xt[..., 2]) + xt[..., 3]      # rounded in bf16
        sx = four.to(torch.float32).sum(-1).numpy()
    y = (s * xq + b * sx[None, :]).sum(-1, dtype=np.float32)
    return torch.from_numpy(y).to(torch.bfloat16).to(torch.float64).numpy()


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6])
def test_low_precision_sum_x_fails_tolerance(bits):
    """The precision case at every width it names: sum(x) widened per element
    passes every output without the floor clause; the bf16-pairwise sum(x)
    mutant fails a majority of the outputs."""
    case = synth.affine_case(1, 512, 2560, bits, 64, "bf16", seed=2, precision=True)
    y_ref, absdot = oracle.qmv_affine(case["x"][0], case["w"][0], case["scales"][0], case["biases"][0],
                                      1, 512, 2560, bits, 64, "bf16", threads=8)
    ok_good, needed = check(_emulate_kernel_bf16(case, True)[None, :], y_ref, absdot, "bf16")
    ok_bad, _ = check(_emulate_kernel_bf16(case, False)[None, :], y_ref, absdot, "bf16")
    assert ok_good.all() and needed == 0
    assert (~ok_bad).sum() > 256, int((~ok_bad).sum())


# ------------------------------------------------------------- quantizer ----
def _f32_specials():
    rng = np.random.default_rng(77)
    v = np.concatenate([
        rng.standard_normal(4000).astype(np.float32) * np.float32(3.0),
        (rng.standard_normal(2000) * 1e-5).astype(np.float32),           # binary16 subnormal range
        np.array([0.0, -0.0, 1.0, -1.0, 65504.0, 65519.0, 65520.0, 6e-8, 2.0 ** -24, 2.0 ** -25,
                  1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8], dtype=np.float32),
    ])
    # exact ties of the binary16 / bfloat16 grids
    base = rng.integers(0, 1 << 10, 500).astype(np.uint32)
    ties16 = np.array([(1.0 + (b + 0.5) / 1024.0) for b in base], dtype=np.float32)
    tiesbf = ((rng.integers(0x3F80, 0x4080, 500).astype(np.uint32) << 16) | 0x8000).view(np.float32)
    return np.concatenate([v, ties16, tiesbf])


def test_f32_to_f16_matches_numpy():
    with np.errstate(over="ignore"):                 # values past the f16 range round to infinity
        for v in _f32_specials():
            assert oracle.f32_to_f16(v) == int(np.float32(v).astype(np.float16).view(np.uint16)), v


def test_f32_to_bf16_matches_torch():
    v = _f32_specials()
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    got = np.array([oracle.f32_to_bf16(x) for x in v], dtype=np.uint16)
    assert np.array_equal(got, ref)


def _bits_of(a, dtype):
    if dtype == "f32":
        return np.asarray(a, dtype=np.float32)
    if dtype == "f16":
        return np.asarray(a, dtype=np.float32).astype(np.float16).view(np.uint16)
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 8])
@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_quantize_exact_grid_recovers_codes(bits, dtype):
    """Weights bias + q * scale with scale a power of two, every code present in
    each group: min = bias, max = bias + (2^b - 1) scale, so the quantizer must
    return exactly that scale, that bias and the codes q (read back through the
    pinned unpack)."""
    rng = np.random.default_rng(bits * 10 + len(dtype))
    qmax = (1 << bits) - 1
    group, N = 64, 3
    K = 4 * group
    q = rng.integers(0, qmax + 1, (N, K))
    q[:, ::group] = 0
    q[:, 1::group] = qmax
    scale, bias = 2.0 ** -3, -1.5
    w = (bias + q * scale).astype(np.float32)
    wq, sc, bi = oracle.quantize_affine(_bits_of(w, dtype), N, K, bits, group, dtype)
    assert np.array_equal(sc, np.full_like(sc, _bits_of([scale], dtype)[0]))
    assert np.array_equal(bi, np.full_like(bi, _bits_of([bias], dtype)[0]))
    for n in range(N):
        assert np.array_equal(oracle.affine_codes(wq[n], K, bits), q[n].astype(np.uint32))


def test_quantize_signed_zero_extremes_keep_the_first_met():
    """min / max by strict comparisons in element order: of +0 and -0 the first
    one met is the bias (or the maximum), whatever follows."""
    w = np.zeros((2, 32), dtype=np.float32)
    w[0, :] = np.arange(32) * 0.5
    w[0, 3] = -0.0                       # +0 at 0 comes first: bias +0
    w[1, :] = np.arange(32) * 0.5
    w[1, 0] = -0.0                       # -0 first: bias -0
    _, _, bi = oracle.quantize_affine(w, 2, 32, 4, 32, "f32")
    assert np.signbit(bi[1, 0]) and not np.signbit(bi[0, 0])


def test_quantize_subnormal_range_takes_the_nearest_code():
    """A range in the fp32 subnormals: scale below 2^-128 (its reciprocal would
    overflow), yet the quotient (w - bias) / scale is an ordinary number and
    every code is the nearest grid point (exact rationals)."""
    w = (np.arange(32, dtype=np.float32) * np.float32(1e-41)).reshape(1, 32)
    wq, sc, bi = oracle.quantize_affine(w, 1, 32, 4, 32, "f32")
    assert 0 < sc[0, 0] < 2.0 ** -128 and bi[0, 0] == 0.0
    codes = oracle.affine_codes(wq[0], 32, 4)
    s = Fraction(float(sc[0, 0]))
    for k in range(32):
        d = [abs(Fraction(float(w[0, k])) - s * c) for c in range(16)]
        assert d[int(codes[k])] == min(d), (k, codes[k])
    assert codes[0] == 0 and codes[31] == 15


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_quantize_exact_half_quotients_round_to_even(dtype):
    """Group min 0 and max 45 at 4 bits: scale 45 / 15 = 3 exactly.  The
    weights 7.5 and 13.5 sit exactly halfway between grid points (quotients 2.5
    and 4.5): the nearest-integer rule with ties to even gives codes 2 and 4.
    (A reciprocal-times-difference reading would give 3 and 5 here: 1 / 3
    rounds up in fp32, pushing both products just past the half.)"""
    w = np.zeros((1, 32), dtype=np.float32)
    w[0, 1] = 45.0
    w[0, 2] = 7.5
    w[0, 3] = 13.5
    w[0, 4] = 10.5                      # quotient 3.5: ties to 4
    wq, sc, bi = oracle.quantize_affine(_bits_of(w, dtype), 1, 32, 4, 32, dtype)
    assert np.array_equal(sc, _bits_of([3.0], dtype).reshape(1, 1))
    codes = oracle.affine_codes(wq[0], 32, 4)
    assert list(codes[:5]) == [0, 15, 2, 4, 4]


def test_quantize_constant_group():
    w = np.full((1, 32), 0.7, dtype=np.float32)
    wq, sc, bi = oracle.quantize_affine(w, 1, 32, 4, 32, "f32")
    assert sc[0, 0] == 0.0 and bi[0, 0] == np.float32(0.7) and not wq.any()


@pytest.mark.parametrize("bits", [3, 4, 8])
def test_quantize_nearest_code_brute_force(bits):
    """Each code is the nearest of the 2^b grid points bias_T + q scale_T to w
    (exact rationals), except where the distance to two grid points is equal
    within the fp32 rounding of the difference and the quotient."""
    rng = np.random.default_rng(bits)
    group, N, K = 32, 4, 64
    w = (rng.standard_normal((N, K)) * 0.3).astype(np.float32)
    wq, sc, bi = oracle.quantize_affine(w, N, K, bits, group, "f32")
    qmax = (1 << bits) - 1
    for n in range(N):
        codes = oracle.affine_codes(wq[n], K, bits)
        for k in range(K):
            s = Fraction(float(sc[n, k // group])); b = Fraction(float(bi[n, k // group]))
            x = Fraction(float(w[n, k]))
            d = [abs(x - (b + s * c)) for c in range(qmax + 1)]
            best = min(d)
            got = d[int(codes[k])]
            if got != best:
                assert float(got - best) <= 1e-6 * float(s), (n, k, codes[k])
            assert float(got) <= float(s) / 2 * (1 + 1e-6) or codes[k] in (0, qmax)


# ------------------------------------------------------ FP quantizer pins ----
@pytest.mark.parametrize("a,code", [(0.0, 0), (0.24, 0), (0.25, 0), (0.26, 1), (0.75, 2), (1.25, 2), (1.75, 4),
                                    (2.5, 4), (3.5, 6), (4.9, 6), (5.0, 6), (5.1, 7), (6.0, 7), (7.0, 7), (1e9, 7),
                                    (6.7e35, 7), (1e300, 7)])
def test_nearest_e2m1_hand_cases(a, code):
    """E2M1 magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}: the midpoints go to the even
    code, anything past 6 saturates to 6 (code 7)."""
    assert oracle.nearest_e2m1(a) == code


def test_nearest_e4m3_vs_torch_in_range():
    """Inside the finite range torch's float8_e4m3fn conversion rounds to
    nearest even exactly as the definition does; past 448 the quantizer
    saturates (code 0x7E)."""
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.uniform(0, 448, 4000), np.exp2(rng.uniform(-12, 8.8, 4000)),
                        np.arange(0, 2 ** -6, 2 ** -10)]).astype(np.float32)
    a = a[a <= 448]
    want = torch.from_numpy(a).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.nearest_e4m3(float(v)) for v in a], dtype=np.uint8)
    assert np.array_equal(got, want)
    assert oracle.nearest_e4m3(449.0) == 0x7E and oracle.nearest_e4m3(1e30) == 0x7E
    assert oracle.nearest_e4m3(3e38 / 7) == 0x7E and oracle.nearest_e4m3(1e300) == 0x7E


def _fp_grid_weights(mode, N, K, rng):
    """Weights that lie exactly on a block's element grid, with the block
    maximum at the largest element, so the quantizer must return their codes."""
    fp8 = mode == "mxfp8"
    blk = 16 if mode == "nvfp4" else 32
    vals = np.array([oracle.e4m3(c) for c in range(127)]) if fp8 else np.array([oracle.e2m1(c) for c in range(8)])
    top = len(vals) - 1
    codes = rng.integers(0, top + 1, size=(N, K))
    codes[:, ::blk] = top                                   # every block reaches the top element
    sign = rng.integers(0, 2, size=(N, K))
    if mode == "nvfp4":
        s_codes = rng.integers(8, 100, size=(N, K // blk))  # normal E4M3 scales
        scale = np.array([[oracle.e4m3(c) for c in r] for r in s_codes])
    else:
        s_codes = rng.integers(120, 135, size=(N, K // blk))
        scale = np.exp2(s_codes.astype(np.float64) - 127)
    g = 0.5 if mode == "nvfp4" else 1.0                      # NVFP4: a non-unit global scale
    w = vals[codes] * np.repeat(scale, blk, axis=1) * g * np.where(sign == 1, -1.0, 1.0)
    return w.astype(np.float32), codes, sign, s_codes, g


@pytest.mark.parametrize("mode", ["mxfp4", "mxfp8", "nvfp4"])
def test_quantize_fp_recovers_grid_weights(mode):
    """On-grid weights come back exactly (codes with their signs, scale
    bytes): MX scale byte = floor(log2(amax)) - emax + 127; NVFP4 scale =
    amax / (6 * global) with global 0.5."""
    rng = np.random.default_rng(7)
    N, K = 4, 128
    w, codes, sign, s_codes, g = _fp_grid_weights(mode, N, K, rng)
    wq, sc = oracle.quantize_fp(w, N, K, mode, "f32", global_scale=g)
    assert np.array_equal(sc, s_codes.astype(np.uint8))
    fp8 = mode == "mxfp8"
    got = wq.astype(np.int64) if fp8 else np.stack([wq & 0xF, wq >> 4], axis=-1).reshape(N, K).astype(np.int64)
    sbit = 0x80 if fp8 else 0x8
    want = codes + sign * sbit
    want[codes == 0] = 0                                    # +0 and -0 (not < 0) take code 0
    assert np.array_equal(got, want)


@pytest.mark.parametrize("mode", ["mxfp4", "mxfp8", "nvfp4"])
def test_quantize_fp_dequant_error_bound(mode):
    """Random weights: quantize, dequantize with the oracle's decoder; each
    weight is within half an element step (times the block scale) of its
    dequantized value, the step taken at the element's own magnitude, except
    past the largest element, where it saturates."""
    rng = np.random.default_rng(11)
    N, K = 3, 256
    w = (rng.standard_normal((N, K)) * 0.3).astype(np.float32)
    g = 0.7
    wq, sc = oracle.quantize_fp(w, N, K, mode, "f32", global_scale=g)
    deq = oracle.dequant_fp_f32(wq, sc, g if mode == "nvfp4" else None, N, K, mode)
    blk = 16 if mode == "nvfp4" else 32
    if mode == "nvfp4":
        bscale = np.array([[oracle.e4m3(int(c)) for c in r] for r in sc]) * np.float32(g)
    else:
        bscale = np.exp2(sc.astype(np.float64) - 127)
    bs = np.repeat(bscale, blk, axis=1)
    d = np.abs(w.astype(np.float64)) / bs
    if mode == "mxfp8":
        step = np.where(d < 2 ** -6, 2 ** -9, np.exp2(np.floor(np.log2(np.maximum(d, 2 ** -6))) - 3))
    else:
        step = np.where(d < 2, 0.5, np.where(d < 4, 1.0, 2.0))
    err = np.abs(w.astype(np.float64) - deq.astype(np.float64))
    top = 448.0 if mode == "mxfp8" else 6.0
    # past the largest element (MX scales put the block maximum in [4, 8) or
    # [256, 512) elements) the code saturates: the error is the excess
    bound = np.where(d > top, (d - top) * bs, 0.5 * step * bs)
    ulp = np.abs(deq.astype(np.float64)) * 2.0 ** -23      # the dequantized value is one fp32 rounding
    assert (err <= bound * (1 + 1e-6) + ulp + 1e-30).all()
    sat = d > top
    assert (np.abs(np.abs(deq[sat]) - (top * bs)[sat]) <= ulp[sat]).all()


# ------------------------------------------------------------ SwiGLU pins ----
def _swiglu_case(M, N, K, bits, group, seed):
    cg = synth.affine_case(M, N, K, bits, group, "f32", seed=seed)
    cu = synth.affine_case(M, N, K, bits, group, "f32", seed=seed + 1)
    return cg["x"][0], (cg["w"][0], cg["scales"][0], cg["biases"][0]), (cu["w"][0], cu["scales"][0], cu["biases"][0])


def test_swiglu_unit_x_closed_form():
    """x = e_k: gate and up are single dequantized weights (test-side reader,
    library casts), and mid = g * u / (1 + e^-g) by the math library."""
    N, K, bits, group = 6, 64, 4, 32
    _, (wg, sg, bg), (wu, su, bu) = _swiglu_case(1, N, K, bits, group, seed=70)
    for k in (0, 33, 63):
        x = np.zeros((1, K), dtype=np.float32); x[0, k] = 1.0
        mid, g, u, _, _ = oracle.qmv_affine_swiglu(x, wg, sg, bg, wu, su, bu, 1, N, K, bits, group, "f32")
        for n in range(N):
            gv = float(sg[n, k // group]) * _py_codes(wg[n], K, bits)[k] + float(bg[n, k // group])
            uv = float(su[n, k // group]) * _py_codes(wu[n], K, bits)[k] + float(bu[n, k // group])
            assert g[0, n] == gv and u[0, n] == uv
            assert math.isclose(mid[0, n], gv * uv / (1.0 + math.exp(-gv)), rel_tol=1e-15, abs_tol=1e-300)


def test_swiglu_clamp_route_weight_and_limits():
    """The clamp limits gate from above and up on both sides only when it is
    above 1e-6; the route weight scales mid exactly; silu(g) -> g for large g
    and -> 0 for very negative g."""
    M, N, K, bits, group = 2, 8, 128, 4, 64
    x, (wg, sg, bg), (wu, su, bu) = _swiglu_case(M, N, K, bits, group, seed=80)
    args = (x, wg, sg, bg, wu, su, bu, M, N, K, bits, group, "f32")
    m0, g, u, _, _ = oracle.qmv_affine_swiglu(*args)
    m2, _, _, _, _ = oracle.qmv_affine_swiglu(*args, route_weight=2.0)
    assert np.array_equal(m2, 2.0 * m0)
    rows, _, _, _, _ = oracle.qmv_affine_swiglu(*args, route_weight=np.array([0.5, 4.0]))   # one per x row
    assert np.array_equal(rows[0], 0.5 * m0[0]) and np.array_equal(rows[1], 4.0 * m0[1])
    tiny, _, _, _, _ = oracle.qmv_affine_swiglu(*args, clamp=1e-7)          # at or below 1e-6: no clamp
    assert np.array_equal(tiny, m0)
    c = float(np.median(np.abs(np.concatenate([g.ravel(), u.ravel()]))))
    mc, _, _, _, _ = oracle.qmv_affine_swiglu(*args, clamp=c)
    gc, uc = np.minimum(g, c), np.clip(u, -c, c)
    assert np.allclose(mc, gc * uc / (1.0 + np.exp(-gc)), rtol=1e-15, atol=0)
    assert (np.abs(uc) <= c).all() and (gc <= c).all() and not np.array_equal(mc, m0)
    # limits of silu on planted rows: scale every bias of the gate to +-40
    big = np.full_like(bg, 40.0); neg = np.full_like(bg, -40.0)
    zero_w = np.zeros_like(wg); ones = np.ones((M, K), dtype=np.float32) / K
    mp, gp, up, _, _ = oracle.qmv_affine_swiglu(ones, zero_w, sg, big, wu, su, bu, M, N, K, bits, group, "f32")
    assert np.allclose(mp, gp * up, rtol=1e-15)                               # silu(40) = 40 (1 - 4e-18)
    mn, _, _, _, _ = oracle.qmv_affine_swiglu(ones, zero_w, sg, neg, wu, su, bu, M, N, K, bits, group, "f32")
    assert (np.abs(mn) < 1e-15 * np.abs(up) + 1e-300).all()                   # silu(-40) = -40 e^-40


# ------------------------------------------------ fp64 dequant, QKV, RMSNorm ----
@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 8])
@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_dequant_f64_rounds_to_the_f32_check(bits, dtype):
    """The fp64 weights round (once) to exactly the pinned fp32 check values."""
    c = synth.affine_case(1, 5, 128, bits, 32, dtype, seed=bits)
    w64 = oracle.dequant_affine_f64(c["w"][0], c["scales"][0], c["biases"][0], 5, 128, bits, 32, dtype)
    w32 = oracle.dequant_affine_f32(c["w"][0], c["scales"][0], c["biases"][0], 5, 128, bits, 32, dtype)
    assert np.array_equal(w64.astype(np.float32), w32)


def test_dequant_f64_is_the_column_of_a_unit_x():
    """x = e_k through the qmv oracle returns column k of the fp64 weights."""
    N, K, bits, g = 7, 64, 5, 32
    c = synth.affine_case(1, N, K, bits, g, "f32", seed=4)
    W = oracle.dequant_affine_f64(c["w"][0], c["scales"][0], c["biases"][0], N, K, bits, g, "f32")
    for k in (0, 31, 63):
        x = np.zeros((1, K), dtype=np.float32); x[0, k] = 1.0
        y, _ = oracle.qmv_affine(x, c["w"][0], c["scales"][0], c["biases"][0], 1, N, K, bits, g, "f32")
        assert np.array_equal(y[0], W[:, k])


def test_qkv_is_qmv_of_the_stacked_matrix():
    """[Q | K | V] equals one qmv over the three matrices stacked along N, bit
    for bit (the same fp64 sums)."""
    M, Nq, Nkv, K, bits, g = 2, 24, 8, 128, 4, 64
    cs = [synth.affine_case(M, n, K, bits, g, "bf16", seed=50 + i) for i, n in enumerate((Nq, Nkv, Nkv))]
    x = cs[0]["x"][0]
    t = [(c["w"][0], c["scales"][0], c["biases"][0]) for c in cs]
    y, a = oracle.qmv_affine_qkv(x, *t, M, Nq, Nkv, K, bits, g, "bf16")
    ws = np.concatenate([c["w"][0] for c in cs]); ss = np.concatenate([c["scales"][0] for c in cs])
    bs = np.concatenate([c["biases"][0] for c in cs])
    y2, a2 = oracle.qmv_affine(x, ws, ss, bs, M, Nq + 2 * Nkv, K, bits, g, "bf16")
    assert np.array_equal(y, y2) and np.array_equal(a, a2)
    rows = [0, Nq - 1, Nq, Nq + Nkv, Nq + 2 * Nkv - 1]
    yr, _ = oracle.qmv_affine_qkv(x, *t, M, Nq, Nkv, K, bits, g, "bf16", rows=rows)
    assert np.array_equal(yr[:, rows], y2[:, rows])


def test_rms_norm_closed_forms():
    """Constant rows: x = c gives gamma * c / sqrt(c^2 + eps); with eps = 0 and
    gamma = 1 every row has unit RMS; scaling x leaves it unchanged (eps = 0)."""
    K = 64
    g = np.linspace(0.5, 2.0, K)
    x = np.full((1, K), 3.0)
    assert np.allclose(oracle.rms_norm(x, g, 1e-2), g * 3.0 / math.sqrt(9.0 + 1e-2), rtol=1e-15, atol=0)
    rng = np.random.default_rng(0)
    x = rng.standard_normal((3, K))
    xh = oracle.rms_norm(x, np.ones(K), 0.0)
    assert np.allclose(np.sqrt(np.mean(xh * xh, axis=1)), 1.0, rtol=1e-14)
    assert np.allclose(oracle.rms_norm(7.5 * x, g, 0.0), oracle.rms_norm(x, g, 0.0), rtol=1e-14)


def test_rms_norm_qmv_unit_x_and_scaling():
    """x = 2 e_k (eps 0): xh = gamma_k sqrt(K) e_k, so y = gamma_k sqrt(K)
    times column k of the weights; and y of alpha x equals y of x (eps 0)."""
    N, K, bits, grp = 6, 64, 4, 32
    c = synth.affine_case(1, N, K, bits, grp, "f32", seed=12)
    gam = synth.to_storage(np.linspace(0.5, 1.5, K), "f32")
    W = oracle.dequant_affine_f64(c["w"][0], c["scales"][0], c["biases"][0], N, K, bits, grp, "f32")
    k = 17
    x = np.zeros((1, K), dtype=np.float32); x[0, k] = 2.0
    y, _ = oracle.qmv_affine_rms_norm(x, gam, 0.0, c["w"][0], c["scales"][0], c["biases"][0], 1, N, K, bits, grp, "f32")
    assert np.allclose(y[0], float(gam[k]) * math.sqrt(K) * W[:, k], rtol=1e-14, atol=0)
    xs = synth.to_storage(np.random.default_rng(1).standard_normal((1, K)), "f32")
    y1, _ = oracle.qmv_affine_rms_norm(xs, gam, 0.0, c["w"][0], c["scales"][0], c["biases"][0], 1, N, K, bits, grp, "f32")
    y2, _ = oracle.qmv_affine_rms_norm(xs * np.float32(4.0), gam, 0.0, c["w"][0], c["scales"][0], c["biases"][0], 1, N,
                                       K, bits, grp, "f32")
    assert np.allclose(y1, y2, rtol=1e-13, atol=1e-300)
