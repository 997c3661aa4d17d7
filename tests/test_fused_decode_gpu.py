"""GPU parity of the fused decode variants against the oracle: Q / K / V in
one launch (qmv_affine_qkv) and RMSNorm fused into the qmv
(qmv_affine_rms_norm).  Same tolerance as every qmv test (qmv_tol.py); the
RMSNorm keeps the normalized x in fp32, so its outputs meet the same bars
against the fp64 composition."""
from __future__ import annotations

import zlib

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import THREADS, TORCH_DT, compare, dev, require_cuda, sample_rows, to_f64

pytestmark = pytest.mark.gpu

BITS = [2, 3, 4, 5, 6, 8]
DTYPES = ["f32", "f16", "bf16"]


@pytest.fixture(scope="module")
def q():
    return require_cuda()


@pytest.fixture(autouse=True)
def _auto_config(q):
    q.qmv_force_config()
    yield
    q.qmv_force_config()


def _seed(*parts):
    return zlib.crc32("/".join(str(p) for p in parts).encode()) & 0x7FFFFFFF


# ------------------------------------------------------------------ QKV ----
def _qkv(q, M, Nq, Nkv, K, bits, group, dtype, seed, w_offset=0):
    cs = [synth.affine_case(M, n, K, bits, group, dtype, seed=seed + i) for i, n in enumerate((Nq, Nkv, Nkv))]
    x = cs[0]["x"][0]
    t = [(c["w"][0], c["scales"][0], c["biases"][0]) for c in cs]
    y = torch.full((M, Nq + 2 * Nkv), float("nan"), dtype=TORCH_DT[dtype], device="cuda")
    dt = [tuple(dev(a, w_offset if j == 0 else 0) for j, a in enumerate(tt)) for tt in t]
    q.qmv_affine_qkv(dev(x), *dt, y, M, Nq, Nkv, K, bits, group, dtype)
    torch.cuda.synchronize()
    return to_f64(y), x, t


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("M", [1, 3, 8])
def test_qkv_grid(q, bits, dtype, M):
    Nq, Nkv, K, group = 320, 72, 1024, 64
    y, x, t = _qkv(q, M, Nq, Nkv, K, bits, group, dtype, _seed("qkv", bits, dtype, M))
    ref, ad = oracle.qmv_affine_qkv(x, *t, M, Nq, Nkv, K, bits, group, dtype, threads=THREADS)
    compare(y, ref, ad, dtype, what=f"qkv b{bits} {dtype} M{M}")


@pytest.mark.parametrize("bits", [3, 4])
def test_qkv_misaligned_and_no_kv(q, bits):
    """Weights off a 16-byte boundary take the 4-byte path; Nkv = 0 is Q only."""
    M, Nq, Nkv, K, group = 2, 130, 34, 512, 32
    y, x, t = _qkv(q, M, Nq, Nkv, K, bits, group, "f16", _seed("qkvm", bits), w_offset=4)
    ref, ad = oracle.qmv_affine_qkv(x, *t, M, Nq, Nkv, K, bits, group, "f16", threads=THREADS)
    compare(y, ref, ad, "f16", what=f"qkv misaligned b{bits}")
    y, x, t = _qkv(q, M, Nq, 0, K, bits, group, "f16", _seed("qkv0", bits))
    ref, ad = oracle.qmv_affine_qkv(x, *t, M, Nq, 0, K, bits, group, "f16", threads=THREADS)
    compare(y, ref, ad, "f16", what=f"qkv q only b{bits}")


@pytest.mark.parametrize("M", [1, 8])
def test_qkv_7b_shape(q, M):
    """7B-class attention with grouped K / V: Nq = 4096, Nkv = 1024, K = 4096,
    4-bit g64 bf16 (sampled rows across the three parts and their seams)."""
    Nq, Nkv, K = 4096, 1024, 4096
    y, x, t = _qkv(q, M, Nq, Nkv, K, 4, 64, "bf16", _seed("qkv7b", M))
    rows = sorted(set(sample_rows(Nq + 2 * Nkv, 40) + [Nq - 1, Nq, Nq + Nkv - 1, Nq + Nkv]))
    ref, ad = oracle.qmv_affine_qkv(x, *t, M, Nq, Nkv, K, 4, 64, "bf16", rows=rows, threads=THREADS)
    compare(y, ref, ad, "bf16", rows=rows, what=f"qkv 7b M{M}")


# -------------------------------------------------------------- RMSNorm ----
def _norm_case(M, N, K, bits, group, dtype, seed, scale=30.0):
    c = synth.affine_case(M, N, K, bits, group, dtype, seed=seed)
    g = synth.rng(seed + 7)
    c["x"] = synth.to_storage(synth.storage_to_float(c["x"], dtype) * scale, dtype)
    gamma = synth.to_storage(g.uniform(0.5, 1.5, size=K), dtype)
    return c, gamma


def _run_norm(q, c, gamma, eps):
    M, N, K = c["M"], c["N"], c["K"]
    y = torch.full((M, N), float("nan"), dtype=TORCH_DT[c["dtype"]], device="cuda")
    q.qmv_affine_rms_norm(dev(c["x"][0]), dev(gamma), eps, dev(c["w"][0]), dev(c["scales"][0]), dev(c["biases"][0]),
                          y, M, N, K, c["bits"], c["group"], c["dtype"])
    torch.cuda.synchronize()
    return to_f64(y)


def _ref_norm(c, gamma, eps, rows=None):
    return oracle.qmv_affine_rms_norm(c["x"][0], gamma, eps, c["w"][0], c["scales"][0], c["biases"][0], c["M"],
                                      c["N"], c["K"], c["bits"], c["group"], c["dtype"], rows=rows, threads=THREADS)


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("M", [1, 3, 8])
def test_rms_norm_grid(q, bits, dtype, M):
    N, K, group = 300, 2048, 64
    c, gamma = _norm_case(M, N, K, bits, group, dtype, _seed("rms", bits, dtype, M))
    y = _run_norm(q, c, gamma, 1e-5)
    ref, ad = _ref_norm(c, gamma, 1e-5)
    compare(y, ref, ad, dtype, what=f"rms b{bits} {dtype} M{M}")


@pytest.mark.parametrize("eps", [0.0, 1e-2, 50.0])
@pytest.mark.parametrize("path", [0, 1])
def test_rms_norm_eps_and_paths(q, eps, path):
    """eps from 0 to larger than mean(x^2) of some rows; 4-byte and 16-byte
    chunk paths; narrow N spreads K over several warps."""
    q.qmv_force_config(path, -1, -1, -1)
    c, gamma = _norm_case(4, 40, 4096, 4, 128, "bf16", _seed("rmse", eps, path), scale=3.0)
    y = _run_norm(q, c, gamma, eps)
    ref, ad = _ref_norm(c, gamma, eps)
    compare(y, ref, ad, "bf16", what=f"rms eps{eps} path{path}")


def test_rms_norm_layer_shape(q):
    """The 7B down projection's input width (K = 14336), gate+up-sized N,
    sampled rows."""
    M, N, K = 2, 8192, 14336
    c, gamma = _norm_case(M, N, K, 4, 64, "bf16", 99)
    y = _run_norm(q, c, gamma, 1e-6)
    rows = sample_rows(N, 40)
    ref, ad = _ref_norm(c, gamma, 1e-6, rows=rows)
    compare(y, ref, ad, "bf16", rows=rows, what="rms layer")


def test_rms_norm_scale_invariance(q):
    """eps = 0: scaling x by a power of two leaves every output bit unchanged
    (the normalization divides it out exactly)."""
    c, gamma = _norm_case(2, 256, 1024, 4, 64, "f32", 5)
    y1 = _run_norm(q, c, gamma, 0.0)
    c2 = dict(c, x=(c["x"] * np.float32(8.0)).astype(np.float32))
    y2 = _run_norm(q, c2, gamma, 0.0)
    assert np.array_equal(y1, y2)
