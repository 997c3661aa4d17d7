"""GPU parity of the affine quantizer (qmv_quantize_affine) against the oracle.

The packed codes, scales and biases are integers and bit patterns defined by
fp32 operations (min / max, subtract, divide, round to nearest even, round to
the element type).  The kernel reaches the same codes through a reciprocal per
group with an exact-division fallback near every rounding edge, so every byte
must match exactly.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from gpu_util import THREADS, dev, require_cuda

pytestmark = pytest.mark.gpu

BITS = [2, 3, 4, 5, 6, 8]
GROUPS = [32, 64, 128]
DTYPES = ["f32", "f16", "bf16"]
STORAGE = {"f32": np.float32, "f16": np.uint16, "bf16": np.uint16}
ESIZE = {"f32": 4, "f16": 2, "bf16": 2}


@pytest.fixture(scope="module")
def q():
    return require_cuda()


def _weights(N, K, dtype, seed):
    """Normal weights with a few large outliers, stored as dtype bit patterns."""
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((N, K)) * 0.05).astype(np.float32)
    idx = rng.integers(0, N * K, max(1, N * K // 500))
    w.reshape(-1)[idx] *= 40.0
    t = torch.from_numpy(w).to({"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[dtype])
    return t.view(torch.int32 if dtype == "f32" else torch.int16).numpy().view(STORAGE[dtype]).copy()


def _run(q, w, N, K, bits, group, dtype, w_offset=0):
    rb = K * bits // 8
    wq = torch.full((N * rb,), 0xA5, dtype=torch.uint8, device="cuda")
    es = ESIZE[dtype]
    sc = torch.full((N * (K // group) * es,), 0xA5, dtype=torch.uint8, device="cuda")
    bi = torch.full_like(sc, 0xA5)
    q.qmv_quantize_affine(dev(w, w_offset), wq, sc, bi, N, K, bits, group, dtype)
    torch.cuda.synchronize()
    st = STORAGE[dtype]
    return (wq.cpu().numpy().reshape(N, rb), sc.cpu().numpy().view(st).reshape(N, K // group),
            bi.cpu().numpy().view(st).reshape(N, K // group))


def _check(got, ref, what):
    for name, g, r in zip(("codes", "scales", "biases"), got, ref):
        if not np.array_equal(g.view(np.uint8), r.view(np.uint8)):
            bad = np.argwhere(g.view(np.uint8) != r.view(np.uint8))
            raise AssertionError(f"{what}: {name} differ at {len(bad)} bytes, first {bad[:4].tolist()}")


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("group", GROUPS)
@pytest.mark.parametrize("dtype", DTYPES)
def test_quantize_bitexact_grid(q, bits, group, dtype):
    N, K = 37, 3 * max(group, 128)
    w = _weights(N, K, dtype, seed=bits * 1000 + group + len(dtype))
    got = _run(q, w, N, K, bits, group, dtype)
    ref = oracle.quantize_affine(w, N, K, bits, group, dtype, threads=THREADS)
    _check(got, ref, f"b{bits} g{group} {dtype}")


@pytest.mark.parametrize("dtype", DTYPES)
def test_quantize_unaligned_rows_take_the_scalar_path(q, dtype):
    """w starting one element past a 16-byte boundary (scalar loads): same bytes."""
    N, K, bits, group = 9, 640, 5, 64
    w = _weights(N, K, dtype, seed=11)
    got = _run(q, w, N, K, bits, group, dtype, w_offset=ESIZE[dtype])
    ref = oracle.quantize_affine(w, N, K, bits, group, dtype)
    _check(got, ref, f"unaligned {dtype}")


@pytest.mark.parametrize("dtype", DTYPES)
def test_quantize_special_groups(q, dtype):
    """Constant groups (scale 0, codes 0), groups of +0 / -0 in both orders
    and with a zero minimum or maximum, a tiny range, exact ties of the code
    grid, a subnormal range whose scale has an infinite reciprocal, exact
    half quotients (ties to even by the division), and (f32) a range past the
    fp32 maximum (infinite scale: every code 0)."""
    N, K, group, bits = 5, 256, 64, 4
    w = np.zeros((N, K), dtype=np.float32)
    w[0, :64] = 0.75                                   # constant
    w[0, 64:128] = np.where(np.arange(64) % 2 == 0, 0.0, -0.0)
    w[0, 128:192] = np.where(np.arange(64) % 2 == 0, -0.0, 0.0)
    w[0, 192:256] = -np.arange(64, dtype=np.float32) * 0.25     # max 0 first ...
    w[0, 200] = -0.0                                          # ... then -0
    w[1, :64] = 1.0 + np.arange(64, dtype=np.float32) * np.float32(2.0 ** -20)    # tiny range
    w[1, 64:128] = np.arange(64, dtype=np.float32) * 0.125     # min 0 first
    w[1, 70] = -0.0
    w[1, 128:192] = np.arange(64, dtype=np.float32) * 0.125
    w[1, 128] = -0.0                                          # min -0 first, +0 later
    w[1, 150] = 0.0
    w[2, :64] = np.arange(64, dtype=np.float32) % 31 * 0.5                       # ties: (w - 0) / 1.0
    rng = np.random.default_rng(5)
    w[3] = rng.standard_normal(K).astype(np.float32)
    w[4, :64] = np.arange(64, dtype=np.float32) * np.float32(1e-41)              # subnormal range
    w[4, 64:128] = 0.0
    w[4, 65], w[4, 66], w[4, 67], w[4, 68] = 45.0, 7.5, 13.5, 10.5               # scale 3: quotients 2.5, 4.5, 3.5
    if dtype == "f32":
        w[4, 128:192] = np.linspace(-3e38, 3e38, 64, dtype=np.float32)          # max - min overflows
    t = torch.from_numpy(w).to({"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[dtype])
    wb = t.view(torch.int32 if dtype == "f32" else torch.int16).numpy().view(STORAGE[dtype]).copy()
    got = _run(q, wb, N, K, bits, group, dtype)
    ref = oracle.quantize_affine(wb, N, K, bits, group, dtype)
    _check(got, ref, f"special {dtype}")


def test_quantize_then_qmv_matches_oracle(q):
    """The quantizer's output is a valid qmv_affine input: quantize on the GPU,
    multiply on the GPU, compare with the oracle product of the same bytes."""
    from qmv_tol import assert_close
    N, K, bits, group, M = 300, 2048, 4, 64, 2
    w = _weights(N, K, "bf16", seed=21)
    wq, sc, bi = _run(q, w, N, K, bits, group, "bf16")
    rng = np.random.default_rng(22)
    x = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)).to(torch.bfloat16)
    xb = x.view(torch.int16).numpy().view(np.uint16).copy()
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    q.qmv_affine(dev(xb), dev(wq), dev(sc), dev(bi), y, M, N, K, bits, group, "bf16")
    torch.cuda.synchronize()
    ref, ad = oracle.qmv_affine(xb, wq, sc, bi, M, N, K, bits, group, "bf16", threads=THREADS)
    assert_close(y.float().cpu().numpy().astype(np.float64), ref, ad, "bf16", what="quantize -> qmv")


def test_quantize_large_matrix_sampled(q):
    """16384 x 16384 bf16 at 4-bit g64 (the bandwidth-probe matrix): rows
    sampled across the whole matrix match the oracle bit for bit."""
    N = K = 16384
    bits, group = 4, 64
    torch.manual_seed(0)
    wt = (torch.randn((N, K), device="cuda") * 0.05).to(torch.bfloat16)
    rb = K * bits // 8
    wq = torch.empty((N, rb), dtype=torch.uint8, device="cuda")
    sc = torch.empty((N, K // group), dtype=torch.bfloat16, device="cuda")
    bi = torch.empty_like(sc)
    q.qmv_quantize_affine(wt, wq, sc, bi, N, K, bits, group, "bf16")
    torch.cuda.synchronize()
    rows = sorted({0, 1, 4095, 8191, 16383} | set(np.random.default_rng(3).integers(0, N, 27).tolist()))
    wr = wt[rows].view(torch.int16).cpu().numpy().view(np.uint16).copy()
    ref = oracle.quantize_affine(wr, len(rows), K, bits, group, "bf16", threads=THREADS)
    got = (wq[rows].cpu().numpy(), sc[rows].view(torch.int16).cpu().numpy().view(np.uint16),
           bi[rows].view(torch.int16).cpu().numpy().view(np.uint16))
    _check(got, ref, "16384^2 sampled rows")
