"""GPU parity of the per-group tensor-core ring kernel (path 8, "tcg": 4-bit
affine codes, bf16 / f16 x, one fp32 epilogue per scale group) against the
fp64 oracle, element by element, within the qmv output tolerance.

Covered: every group size x dtype x M in 1..8 at a ragged N; the qmm row
counts 9..64 (up to 32 rows a launch); block shapes of 8 to 16 consumer
warps; x tiled along K with several row blocks per persistent block (x staged
again for each); batches with shared and per-entry x; the bitwise-prefix
property of the tail rows; the size rules that send a call elsewhere; and the
decode layer's four projections at full size on sampled rows.
"""
from __future__ import annotations

import zlib

import pytest
import torch

import oracle
import synth
from gpu_util import THREADS, TORCH_DT, compare, dev, oracle_affine, require_cuda, run_affine, to_f64

pytestmark = pytest.mark.gpu

SHAPES = [(8, 1), (4, 2), (2, 4), (1, 8), (8, 2), (4, 4), (2, 8), (1, 16), (1, 13), (4, 3), (2, 7), (1, 9)]  # (warps_k, warps_rows)


@pytest.fixture(scope="module")
def q():
    return require_cuda()


@pytest.fixture(autouse=True)
def _config(q):
    q.qmv_force_config(8, -1, -1, -1)
    q.qmv_device_fault(clear=True)
    yield
    q.qmv_force_config()
    torch.cuda.synchronize()
    assert q.qmv_device_fault(clear=True) == 0     # no bounded ring wait expired


def _seed(*parts):
    return zlib.crc32("/".join(str(p) for p in parts).encode()) & 0x7FFFFFFF


@pytest.mark.parametrize("M", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("group", [32, 64, 128])
def test_tcg_path_grid(q, group, dtype, M):
    N, K = 100, 2048
    assert "path=tcg " in q.qmv_describe_plan("affine", M, N, K, 4, group, dtype)
    c = synth.affine_case(M, N, K, 4, group, dtype, seed=_seed("tcg", group, dtype, M))
    y = run_affine(q, c)[0]
    ref, ad = oracle_affine(c)
    compare(y, ref, ad, dtype, what=f"tcg g{group} {dtype} M{M}")


def _qmm(q, c, M, N, K):
    y = torch.full((M, N), float("nan"), dtype=TORCH_DT[c["dtype"]], device="cuda")
    q.qmv_qmm_affine(dev(c["x"][0]), dev(c["w"][0]), dev(c["scales"][0]), dev(c["biases"][0]), y, M, N, K,
                     c["bits"], c["group"], c["dtype"])
    torch.cuda.synchronize()
    return to_f64(y)


@pytest.mark.parametrize("M", [9, 16, 17, 32, 33, 64])
@pytest.mark.parametrize("group,dtype", [(64, "bf16"), (32, "f16"), (128, "bf16")])
def test_tcg_qmm_rows(q, M, group, dtype):
    N, K = 300, 2048
    c = synth.affine_case(M, N, K, 4, group, dtype, seed=_seed("tcgqmm", M, group, dtype))
    plan = q.qmv_describe_plan("affine", M, N, K, 4, group, dtype)
    assert "path=tcg " in plan and (M <= 32 or "chunked32" in plan), plan
    y = _qmm(q, c, M, N, K)
    ref, ad = oracle.qmv_affine(c["x"][0], c["w"][0], c["scales"][0], c["biases"][0], M, N, K, 4, group, dtype,
                                threads=THREADS)
    compare(y, ref, ad, dtype, what=f"tcg qmm M={M} g{group} {dtype}")


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("M", [4, 8])
def test_tcg_block_shapes(q, shape, M):
    wk, wr = shape
    q.qmv_force_config(8, -1, wk, wr)
    N, K = 333, 2048
    plan = q.qmv_describe_plan("affine", M, N, K, 4, 64, "bf16")
    assert "path=tcg " in plan and f"warps_k={wk} warps_rows={wr} " in plan, plan
    c = synth.affine_case(M, N, K, 4, 64, "bf16", seed=_seed("tcgshape", shape, M), batch=2)
    y = run_affine(q, c)
    for b in range(2):
        ref, ad = oracle_affine(c, b=b)
        compare(y[b], ref, ad, "bf16", what=f"tcg shape {shape} M{M} batch{b}")


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_tcg_x_tiles_and_row_blocks(q, dtype):
    """K = 14336 at M = 8 does not fit shared memory whole: x is staged in two
    tiles, again for each of a block's row blocks (16-row blocks, N = 2500:
    157 row blocks over at most 148 blocks)."""
    q.qmv_force_config(8, -1, 8, 1)
    M, N, K = 8, 2500, 14336
    plan = q.qmv_describe_plan("affine", M, N, K, 4, 64, dtype)
    assert "path=tcg " in plan and "tile_iters=28 " not in plan, plan
    c = synth.affine_case(M, N, K, 4, 64, dtype, seed=_seed("tcgxt", dtype))
    y = run_affine(q, c)[0]
    rows = sorted(set(list(range(0, N, 7)) + list(range(2368, N)) + [N - 1]))
    ref, ad = oracle_affine(c, rows=rows)
    compare(y, ref, ad, dtype, rows=rows, what=f"tcg x tiles {dtype}")


@pytest.mark.parametrize("x_batched", [True, False])
def test_tcg_batched(q, x_batched):
    c = synth.affine_case(4, 200, 1024, 4, 64, "bf16", seed=_seed("tcgbatch", x_batched), batch=3)
    y = run_affine(q, c, x_batched=x_batched)
    for b in range(3):
        ref, ad = oracle_affine(c, b=b, x_batched=x_batched)
        compare(y[b], ref, ad, "bf16", what=f"tcg batch {b} x_batched={x_batched}")


def test_tcg_tail_rows_bitwise_prefix(q):
    """With the launch shape pinned, row n's result does not depend on N."""
    q.qmv_force_config(8, -1, 8, 2)
    K = 2048
    big = synth.affine_case(3, 48, K, 4, 64, "bf16", seed=_seed("tcgtail"))
    yb = run_affine(q, big)[0]
    for n in (1, 5, 17, 33):
        small = dict(big)
        small["N"] = n
        small["w"] = big["w"][:, :n].copy()
        small["scales"] = big["scales"][:, :n].copy()
        small["biases"] = big["biases"][:, :n].copy()
        ys = run_affine(q, small)[0]
        assert (ys == yb[:, :n]).all(), n


@pytest.mark.parametrize("case", ["3bit", "f32", "k_not_8_groups", "w_misaligned"])
def test_tcg_size_rules_send_elsewhere(q, case):
    """Calls outside the kernel's rules run on another kernel, correctly."""
    bits, dtype, K, w_off = 4, "bf16", 2048, 0
    if case == "3bit":
        bits = 3
    elif case == "f32":
        dtype = "f32"
    elif case == "k_not_8_groups":
        K = 1088                                   # 17 groups of 64
    else:
        w_off = 4
    M, N = 4, 150
    if case != "w_misaligned":
        assert "path=tcg " not in q.qmv_describe_plan("affine", M, N, K, bits, 64, dtype)
    c = synth.affine_case(M, N, K, bits, 64, dtype, seed=_seed("tcgrule", case))
    y = run_affine(q, c, w_offset=w_off)[0]
    ref, ad = oracle_affine(c)
    compare(y, ref, ad, dtype, what=f"tcg rule {case}")


@pytest.mark.parametrize("shape", [("qkv", 6144, 4096), ("o", 4096, 4096), ("gate_up", 28672, 4096),
                                   ("down", 4096, 14336)])
def test_tcg_layer_shapes(q, shape):
    """The 7B decode layer's projections at M = 8, 4-bit g64 bf16, sampled rows."""
    name, N, K = shape
    M = 8
    assert "path=tcg " in q.qmv_describe_plan("affine", M, N, K, 4, 64, "bf16")
    c = synth.affine_case(M, N, K, 4, 64, "bf16", seed=_seed("tcglayer", name))
    y = run_affine(q, c)[0]
    rows = list(range(0, N, 61)) + [N - 1]
    ref, ad = oracle_affine(c, rows=rows)
    compare(y, ref, ad, "bf16", rows=rows, what=f"tcg layer {name}")
