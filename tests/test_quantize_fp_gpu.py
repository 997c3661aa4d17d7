"""GPU parity of the block-scaled FP quantizer (qmv_quantize_fp) against the
oracle.  Codes and scale bytes are decided by the same fp32 values on both
sides (the oracle by searching every element value, the kernel by compares
and bit rounding), so every byte must match exactly."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from gpu_util import THREADS, dev, require_cuda

pytestmark = pytest.mark.gpu

MODES = ["mxfp4", "nvfp4", "mxfp8"]
DTYPES = ["f32", "f16", "bf16"]
TORCH = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@pytest.fixture(scope="module")
def q():
    return require_cuda()


def _storage(w, dtype):
    t = torch.from_numpy(np.ascontiguousarray(w, dtype=np.float32)).to(TORCH[dtype])
    return t.view(torch.int32 if dtype == "f32" else torch.int16).numpy().view(
        np.float32 if dtype == "f32" else np.uint16).copy()


def _run(q, wb, N, K, mode, dtype, g=None, w_offset=0, q_offset=0):
    fp8 = mode == "mxfp8"
    blk = 16 if mode == "nvfp4" else 32
    rb = K if fp8 else K // 2
    wqb = torch.full((N * rb + 32,), 0xA5, dtype=torch.uint8, device="cuda")
    wq = wqb[q_offset:q_offset + N * rb]
    sc = torch.full((N * (K // blk),), 0xA5, dtype=torch.uint8, device="cuda")
    gs = torch.tensor([g], dtype=torch.float32, device="cuda") if mode == "nvfp4" else None
    q.qmv_quantize_fp(dev(wb, w_offset), wq, sc, gs, N, K, mode, dtype)
    torch.cuda.synchronize()
    return wq.cpu().numpy().reshape(N, rb), sc.cpu().numpy().reshape(N, K // blk)


def _check(got, ref, what):
    for name, a, b in zip(("codes", "scales"), got, ref):
        if not np.array_equal(a, b):
            bad = np.argwhere(a != b)
            raise AssertionError(f"{what}: {name} differ at {len(bad)} bytes, first {bad[:4].tolist()}")


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("dtype", DTYPES)
def test_quantize_fp_bitexact(q, mode, dtype):
    rng = np.random.default_rng(len(mode) * 10 + len(dtype))
    N, K = 37, 512
    w = rng.standard_normal((N, K)) * np.exp2(rng.integers(-6, 6, size=(N, 1)))
    w.reshape(-1)[rng.integers(0, N * K, N * K // 300)] *= 50.0           # outliers saturate
    wb = _storage(w, dtype)
    g = 0.37
    got = _run(q, wb, N, K, mode, dtype, g=g)
    ref = oracle.quantize_fp(wb, N, K, mode, dtype, global_scale=np.float32(g), threads=THREADS)
    _check(got, ref, f"{mode} {dtype}")


@pytest.mark.parametrize("mode", MODES)
def test_quantize_fp_unaligned_takes_the_scalar_path(q, mode):
    N, K = 5, 256
    wb = _storage(np.random.default_rng(3).standard_normal((N, K)), "bf16")
    got = _run(q, wb, N, K, mode, "bf16", g=1.5, w_offset=2, q_offset=4)
    ref = oracle.quantize_fp(wb, N, K, mode, "bf16", global_scale=np.float32(1.5))
    _check(got, ref, f"unaligned {mode}")


@pytest.mark.parametrize("mode", MODES)
def test_quantize_fp_special_blocks(q, mode):
    """All-zero and -0 blocks, exact ties of the element grid, tiny (subnormal
    fp32) values, values near the E4M3 subnormal boundary, huge values."""
    N, K = 6, 64
    w = np.zeros((N, K), dtype=np.float32)
    w[0, 32:64] = -0.0
    w[1] = np.tile(np.array([6, 5, 3.5, 2.5, 1.75, 1.25, 0.75, 0.25], dtype=np.float32), 8)    # ties at scale 1
    w[2] = np.linspace(-1e-39, 1e-39, K, dtype=np.float32)
    w[3] = np.exp2(np.linspace(-14, -4, K)).astype(np.float32) * np.where(np.arange(K) % 2, -1, 1)
    w[4] = np.float32(3e38) * np.where(np.arange(K) % 3 == 0, 1, -0.5)
    w[5] = np.random.default_rng(9).standard_normal(K).astype(np.float32) * 1e-3
    got = _run(q, w, N, K, mode, "f32", g=1.0)
    ref = oracle.quantize_fp(w, N, K, mode, "f32", global_scale=1.0)
    _check(got, ref, f"special {mode}")


@pytest.mark.parametrize("mode", MODES)
def test_quantize_fp_then_qmv_fp(q, mode):
    """The quantizer's output is a valid qmv_fp input: quantize and multiply on
    the GPU, compare with the oracle product of the same bytes."""
    from qmv_tol import assert_close
    N, K, M = 300, 2048, 2
    rng = np.random.default_rng(21)
    wb = _storage(rng.standard_normal((N, K)) * 0.05, "bf16")
    g = 0.02
    wq, sc = _run(q, wb, N, K, mode, "bf16", g=g)
    x = _storage(rng.standard_normal((M, K)), "bf16")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    gs = torch.tensor([g], dtype=torch.float32, device="cuda") if mode == "nvfp4" else None
    q.qmv_fp(dev(x), dev(wq), dev(sc), gs, y, M, N, K, mode, "bf16")
    torch.cuda.synchronize()
    ref, ad = oracle.qmv_fp(x, wq, sc, np.float32(g) if mode == "nvfp4" else None, M, N, K, mode, "bf16",
                            threads=THREADS)
    assert_close(y.float().cpu().numpy().astype(np.float64), ref, ad, "bf16", what=f"quantize_fp -> qmv_fp {mode}")


def test_quantize_fp_large_matrix_sampled(q):
    """16384 x 16384 bf16 -> NVFP4: sampled rows match the oracle bit for bit."""
    N = K = 16384
    torch.manual_seed(0)
    wt = (torch.randn((N, K), device="cuda") * 0.05).to(torch.bfloat16)
    wq = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
    sc = torch.empty((N, K // 16), dtype=torch.uint8, device="cuda")
    g = torch.tensor([0.01], dtype=torch.float32, device="cuda")
    q.qmv_quantize_fp(wt, wq, sc, g, N, K, "nvfp4", "bf16")
    torch.cuda.synchronize()
    rows = sorted({0, 1, 8191, 16383} | set(np.random.default_rng(4).integers(0, N, 20).tolist()))
    wr = wt[rows].view(torch.int16).cpu().numpy().view(np.uint16).copy()
    ref = oracle.quantize_fp(wr, len(rows), K, "nvfp4", "bf16", global_scale=np.float32(0.01), threads=THREADS)
    _check((wq[rows].cpu().numpy(), sc[rows].cpu().numpy()), ref, "16384^2 nvfp4 sampled")
