"""GPU parity of the tensor-memory (tcgen05) affine qmv kernel (qmv_umma.cuh),
forced with qmv_force_config(7), against the fp64 oracle.

Covers every width x group it supports (2-bit needs groups of 64+), M = 1..8,
ragged N (a partial last 128-row tile), K split over clusters of 1..8 CTAs
(forced through the warps_k field), more row tiles than clusters (the
persistent loop), the sum(x) precision case, and checks that no bounded wait
expired.  Same tolerance as every qmv test (qmv_tol.py).
"""
from __future__ import annotations

import zlib

import numpy as np
import pytest
import torch

import synth
from gpu_util import compare, oracle_affine, require_cuda, run_affine, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    return require_cuda()


@pytest.fixture(autouse=True)
def _forced(q):
    q.qmv_device_fault(clear=True)
    q.qmv_force_config(7, -1, -1, -1)
    yield
    q.qmv_force_config()
    torch.cuda.synchronize()
    assert q.qmv_device_fault(clear=True) == 0


def _seed(*parts):
    return zlib.crc32("/".join(str(p) for p in parts).encode()) & 0x7FFFFFFF


def _plan(q, M, N, K, bits, group):
    return q.qmv_describe_plan("affine", M, N, K, bits, group, "bf16")


def test_umma_small_first(q):
    """One tile, one CTA: the smallest case of the kernel."""
    M, N, K, bits, group = 1, 128, 1024, 4, 64
    q.qmv_force_config(7, -1, 1, -1)
    assert "path=umma" in _plan(q, M, N, K, bits, group)
    c = synth.affine_case(M, N, K, bits, group, "bf16", seed=11)
    y = run_affine(q, c)[0]
    ref, ad = oracle_affine(c)
    compare(y, ref, ad, "bf16", what="umma first")


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 8])
@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("M", [1, 3, 8])
def test_umma_path_grid(q, bits, group, M):
    N, K = 333, 2048
    plan = _plan(q, M, N, K, bits, group)
    if bits == 2 and group == 32:
        assert "path=umma" not in plan
        pytest.skip("2-bit units span two groups of 32")
    if bits == 5 and "path=umma" not in plan:
        pytest.skip("5-bit ring stages (80 KB) leave no room for this x range: " + plan.split()[0])
    assert "path=umma" in plan, plan
    c = synth.affine_case(M, N, K, bits, group, "bf16", seed=_seed("umma", bits, group, M))
    y = run_affine(q, c)[0]
    ref, ad = oracle_affine(c)
    compare(y, ref, ad, "bf16", what=f"umma b{bits} g{group} M{M}")


@pytest.mark.parametrize("S", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("bits", [4, 3])
def test_umma_k_split(q, S, bits):
    """K over S CTAs of a cluster (distributed shared memory reduction)."""
    M, N, K, group = 2, 300, 8192, 64
    q.qmv_force_config(7, -1, S, -1)
    plan = _plan(q, M, N, K, bits, group)
    assert "path=umma" in plan and f"warps_k={S} " in plan, plan
    c = synth.affine_case(M, N, K, bits, group, "bf16", seed=_seed("ummaS", S, bits))
    y = run_affine(q, c)[0]
    ref, ad = oracle_affine(c)
    compare(y, ref, ad, "bf16", what=f"umma S{S} b{bits}")


@pytest.mark.parametrize("M", [1, 8])
def test_umma_persistent_tiles(q, M):
    """More 128-row tiles than clusters fit at once, ragged last tile."""
    N, K, bits, group = 148 * 128 * 2 + 77, 1024, 4, 64
    q.qmv_force_config(7, -1, 1, -1)
    assert "path=umma" in _plan(q, M, N, K, bits, group)
    c = synth.affine_case(M, N, K, bits, group, "bf16", seed=_seed("ummaP", M))
    y = run_affine(q, c)[0]
    rows = sample_rows(N, 64) + list(range(N - 130, N))
    rows = sorted(set(rows))
    ref, ad = oracle_affine(c, rows=rows)
    compare(y, ref, ad, "bf16", rows=rows, what=f"umma persistent M{M}")


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6])
@pytest.mark.parametrize("M", [1, 8])
def test_umma_precision_case(q, bits, M):
    N, K = 4096, 2560
    plan = _plan(q, M, N, K, bits, 64)
    if "path=umma" not in plan:
        pytest.skip("shape outside the kernel's shared-memory budget: " + plan.split()[0])
    c = synth.affine_case(M, N, K, bits, 64, "bf16", seed=_seed("ummaprec", bits, M), precision=True)
    y = run_affine(q, c)[0]
    ref, ad = oracle_affine(c)
    compare(y, ref, ad, "bf16", what=f"umma precision b{bits} M{M}", max_floor_frac=0.25)


@pytest.mark.parametrize("M", [1, 8])
def test_umma_probe_and_layer_shapes(q, M):
    """The bandwidth probe and the 7B layer's projections, sampled rows."""
    for (N, K) in [(16384, 16384), (6144, 4096), (4096, 4096), (28672, 4096), (4096, 14336)]:
        assert "path=umma" in _plan(q, M, N, K, 4, 64)
        c = synth.affine_case(M, N, K, 4, 64, "bf16", seed=_seed("ummaL", N, K, M))
        y = run_affine(q, c)[0]
        rows = sample_rows(N, 32)
        ref, ad = oracle_affine(c, rows=rows)
        compare(y, ref, ad, "bf16", rows=rows, what=f"umma {N}x{K} M{M}")
