"""GPU parity of the small-M qmm (qmv_qmm_affine: up to 64 x rows, as chunks of
32, 16 or 8 rows through the qmv kernels -- the per-group tensor-core ring for
4-bit codes; forced or for few row tiles, one launch of the tensor-memory
kernel) against the oracle, element by element, within the qmv
output tolerance.  Row counts cover one chunk plus a ragged remainder, several
full chunks and the maximum of 64."""
from __future__ import annotations

import pytest
import torch

import oracle
import synth
from gpu_util import THREADS, TORCH_DT, dev, require_cuda, to_f64
from qmv_tol import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    return require_cuda()


def _run(q, c, M, N, K):
    y = torch.full((M, N), float("nan"), dtype=TORCH_DT[c["dtype"]], device="cuda")
    q.qmv_qmm_affine(dev(c["x"][0]), dev(c["w"][0]), dev(c["scales"][0]), dev(c["biases"][0]), y, M, N, K,
                     c["bits"], c["group"], c["dtype"])
    torch.cuda.synchronize()
    return to_f64(y)


@pytest.mark.parametrize("M", [9, 16, 23, 33, 64])
@pytest.mark.parametrize("bits,group,dtype", [(4, 64, "bf16"), (3, 32, "f16"), (8, 128, "f32"), (6, 64, "bf16")])
def test_qmm_rows(q, M, bits, group, dtype):
    N, K = 1000, 1024
    c = synth.affine_case(M, N, K, bits, group, dtype, seed=M * 10 + bits)
    y = _run(q, c, M, N, K)
    ref, ad = oracle.qmv_affine(c["x"][0], c["w"][0], c["scales"][0], c["biases"][0], M, N, K, bits, group, dtype,
                                threads=THREADS)
    assert_close(y, ref, ad, dtype, what=f"qmm M={M} b{bits} g{group} {dtype}")


def test_qmm_layer_shape(q):
    """The 7B down projection (4096 x 14336, 4-bit g64 bf16) at M = 32, sampled rows."""
    M, N, K = 32, 4096, 14336
    c = synth.affine_case(M, N, K, 4, 64, "bf16", seed=77)
    y = _run(q, c, M, N, K)
    rows = list(range(0, N, 97)) + [N - 1]
    ref, ad = oracle.qmv_affine(c["x"][0], c["w"][0], c["scales"][0], c["biases"][0], M, N, K, 4, 64, "bf16",
                                rows=rows, threads=THREADS)
    assert_close(y[:, rows], ref[:, rows], ad[:, rows], "bf16", what="qmm 4096x14336 M=32")


@pytest.mark.parametrize("M", [9, 16, 33, 64])
@pytest.mark.parametrize("shape", [(28672, 4096), (4096, 14336)])
@pytest.mark.parametrize("forced", [-1, 7])
def test_qmm_layer_shapes(q, M, shape, forced):
    """qmm beyond 8 rows on the 7B gate+up and down shapes (4-bit g64 bf16),
    sampled rows: by default chunks of up to 32 rows through the per-group
    tensor-core ring kernel; forced (path 7), one launch of the tensor-memory
    kernel where x fits its shared memory."""
    N, K = shape
    q.qmv_force_config(forced, -1, -1, -1)
    try:
        plan = q.qmv_describe_plan("affine", M, N, K, 4, 64, "bf16")
        fits = M * K <= 33 * 14336          # 64 x rows over K = 14336: x needs more than 16 CTAs
        if forced == 7:
            assert plan.startswith("path=umma") == fits, plan
        else:
            assert plan.startswith(f"path=chunked{16 if M <= 16 else 32} ") and "path=tcg" in plan, plan
        c = synth.affine_case(M, N, K, 4, 64, "bf16", seed=M * 100 + K)
        y = _run(q, c, M, N, K)
    finally:
        q.qmv_force_config()
    rows = list(range(0, N, N // 40)) + [N - 1]
    ref, ad = oracle.qmv_affine(c["x"][0], c["w"][0], c["scales"][0], c["biases"][0], M, N, K, 4, 64, "bf16",
                                rows=rows, threads=THREADS)
    assert_close(y[:, rows], ref[:, rows], ad[:, rows], "bf16", what=f"qmm {plan.split()[0]} {N}x{K} M={M}")


def test_qmm_plans(q):
    """4-bit codes with bf16 / f16 x: 16 or 32 rows a launch through the
    per-group tensor-core ring.  Other widths, tall matrices: 32 rows a chunk
    through the tensor-core ring where a super-block holds one group (g128),
    16 where it holds two (g64).  Few row tiles, bf16: one tensor-memory
    launch."""
    plan = lambda M, N, K, b, g, dt: q.qmv_describe_plan("affine", M, N, K, b, g, dt)
    for args, want in [((64, 8000, 1024, 4, 128, "bf16"), "path=chunked32 chunks=2 path=tcg "),
                       ((33, 8000, 1024, 4, 64, "bf16"), "path=chunked32 chunks=2 path=tcg "),
                       ((12, 8000, 1024, 4, 64, "f16"), "path=chunked16 chunks=1 path=tcg "),
                       ((33, 1000, 1024, 4, 64, "bf16"), "path=chunked32 chunks=2 path=tcg "),
                       ((64, 8000, 1024, 3, 128, "bf16"), "path=chunked32 chunks=2 path=tcb "),
                       ((33, 8000, 1024, 3, 64, "bf16"), "path=chunked16 chunks=3 path=tcb "),
                       ((33, 1000, 1024, 8, 64, "bf16"), "path=umma ")]:
        assert plan(*args).startswith(want), (args, plan(*args))


def test_qmm_rejects_more_than_64_rows(q):
    e = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(Exception):
        q.qmv_qmm_affine(e, e, e, e, e, 65, 64, 64, 4, 64, "bf16")
