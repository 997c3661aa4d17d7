"""The sum(x) precision case on every kernel family, at a weight-ring size.

The MLX pull request "affine_qmv_fast_rows / fp_qmv_fast_rows" fixes a
low-precision sum(x) in the bias term: with x ~ U(1e-4, 1e-3) and the symmetric
zero point bias = -scale * (2^b - 1) / 2, the bias term cancels most of
scale * sum(x * q) and a sum(x) formed in bf16 fails the 1-ulp bar (the mutant
pin in test_oracle_pins.py).  Each kernel family forms its bias term its own
way (the tensor-core kernels add 128 to every code and take 128 * sum(x~) back
out in the fp32 epilogue), so each is forced onto the case here, at
N = 16384, K = 2560 (10-26 MB of packed weights: ring sized), with M = 1 and
M = 8, in every x dtype.  The block-scaled FP formats have no bias term; they
get the same all-positive x, where their signed elements cancel.  Every output
row is compared with the oracle; the floor clause may decide at most a quarter
of them (the session summary prints how many it did).
"""
from __future__ import annotations

import zlib

import pytest

import synth
from gpu_util import compare, oracle_affine, oracle_fp, require_cuda, run_affine, run_fp

pytestmark = pytest.mark.gpu

N, K = 16384, 2560
PATHS = {0: "narrow", 1: "wide", 3: "tc", 4: "tcb", 5: "direct", 6: "tcf", 8: "tcg"}
PREC_FLOOR_FRAC = 0.25


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


def _cases():
    out = []
    for path in (0, 1, 3, 4, 5):
        for M in (1, 8):
            for bits in (2, 3, 4, 5, 6):
                out.append((path, M, bits, "bf16"))
            for dtype in ("f16", "f32"):
                for bits in (2, 4, 5):
                    out.append((path, M, bits, dtype))
    for bits in (2, 3, 4, 5, 6):
        out.append((6, 1, bits, "bf16"))       # the CUDA-core ring: one bf16 x row
    for M in (1, 8):
        for dtype in ("bf16", "f16"):
            out.append((8, M, 4, dtype))       # the per-group tensor-core ring: 4-bit, 16-bit x
    return out


@pytest.mark.parametrize("path,M,bits,dtype", _cases())
def test_precision_case_every_kernel(q, path, M, bits, dtype):
    q.qmv_force_config(path, -1, -1, -1)
    plan = q.qmv_describe_plan("affine", M, N, K, bits, 64, dtype)
    assert f"path={PATHS[path]} " in plan, plan
    c = synth.affine_case(M, N, K, bits, 64, dtype, seed=_seed("precall", path, M, bits, dtype), precision=True)
    y = run_affine(q, c)[0]
    ref, ad = oracle_affine(c)
    compare(y, ref, ad, dtype, what=f"precision path={PATHS[path]} b{bits} {dtype} M{M}",
            max_floor_frac=PREC_FLOOR_FRAC)
    torch_sync_fault_free(q)


@pytest.mark.parametrize("mode", ["mxfp4", "nvfp4", "mxfp8"])
@pytest.mark.parametrize("path", [0, 1, 5])
@pytest.mark.parametrize("M", [1, 8])
def test_precision_case_fp_formats(q, mode, path, M):
    q.qmv_force_config(path, -1, -1, -1)
    fam = {"mxfp4": "mxfp4", "nvfp4": "nvfp4", "mxfp8": "mxfp8"}[mode]
    plan = q.qmv_describe_plan(fam, M, N, K, 0, 0, "bf16")
    assert f"path={PATHS[path]} " in plan, plan
    c = synth.fp_case(M, N, K, mode, "bf16", seed=_seed("precfp", mode, path, M), precision=True)
    y = run_fp(q, c)[0]
    ref, ad = oracle_fp(c)
    compare(y, ref, ad, "bf16", what=f"precision {mode} path={PATHS[path]} M{M}", max_floor_frac=PREC_FLOOR_FRAC)


def torch_sync_fault_free(q):
    """No bounded ring wait expired during the call."""
    import torch
    torch.cuda.synchronize()
    assert q.qmv_device_fault(clear=True) == 0
