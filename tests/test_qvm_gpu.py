"""GPU parity of qvm (qmv_qvm_affine: x times an affine W stored [K, N]) against
the oracle, element by element, within the output tolerance of the qmv tests
(1 ulp of the element type, or the fp32-accumulation floor of sum|x.w|).

Shapes span several 1024-column tiles with a ragged last tile, row counts
that are not multiples of the 8 warps x 4 rows in flight, the K split over
blocks (workspace) and the single-block form (no workspace), every width,
group and element type, M from 1 to 8 (row chunks of 2), K = 0 and a sampled
16384 x 16384 matrix."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import THREADS, TORCH_DT, dev, require_cuda, to_f64
from qmv_tol import assert_close

pytestmark = pytest.mark.gpu

BITS = [2, 3, 4, 5, 6, 8]
GROUPS = [32, 64, 128]
DTYPES = ["f32", "f16", "bf16"]


@pytest.fixture(scope="module")
def q():
    return require_cuda()


def _workspace(q, M, N):
    return torch.zeros(q.qmv_qvm_workspace_bytes(M, N), dtype=torch.uint8, device="cuda")


def _run(q, c, ws):
    M, N, K = c["M"], c["N"], c["K"]
    y = torch.full((M, N), float("nan"), dtype=TORCH_DT[c["dtype"]], device="cuda")
    q.qmv_qvm_affine(dev(c["x"]), dev(c["w"]), dev(c["scales"]), dev(c["biases"]), y, M, N, K, c["bits"],
                     c["group"], c["dtype"], workspace=ws)
    torch.cuda.synchronize()
    return to_f64(y)


def _oracle(c, cols=None):
    return oracle.qvm_affine(c["x"], c["w"], c["scales"], c["biases"], c["M"], c["N"], c["K"], c["bits"],
                             c["group"], c["dtype"], cols=cols, threads=THREADS)


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("group", GROUPS)
@pytest.mark.parametrize("dtype", DTYPES)
def test_qvm_grid_split(q, bits, group, dtype):
    """K split over blocks through the workspace; 1408 columns = one full
    1024-column tile and a ragged one; 777 rows."""
    M, N, K = 2, 1408, 777
    c = synth.qvm_case(M, N, K, bits, group, dtype, seed=bits * 1000 + group + len(dtype))
    ws = _workspace(q, M, N)
    y = _run(q, c, ws)
    ref, ad = _oracle(c)
    assert_close(y, ref, ad, dtype, what=f"qvm b{bits} g{group} {dtype}")
    assert not ws.any(), "the workspace must come back all zero"


@pytest.mark.parametrize("bits", [3, 4, 8])
@pytest.mark.parametrize("dtype", DTYPES)
def test_qvm_single_block_without_workspace(q, bits, dtype):
    M, N, K, group = 1, 2048, 300, 64
    c = synth.qvm_case(M, N, K, bits, group, dtype, seed=7 + bits)
    y = _run(q, c, None)
    ref, ad = _oracle(c)
    assert_close(y, ref, ad, dtype, what=f"qvm no workspace b{bits} {dtype}")


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8])
def test_qvm_x_rows(q, M):
    """x rows in chunks of two (the last one half full for odd M)."""
    N, K, bits, group = 1024, 1000, 4, 64
    c = synth.qvm_case(M, N, K, bits, group, "bf16", seed=M)
    y = _run(q, c, _workspace(q, M, N))
    ref, ad = _oracle(c)
    assert_close(y, ref, ad, "bf16", what=f"qvm M={M}")


@pytest.mark.parametrize("N,K", [(32, 1), (64, 5), (96, 33), (256, 64), (4096, 17), (3200, 4099)])
def test_qvm_shapes(q, N, K):
    """Narrow N (a single partly used warp), tiny and ragged K."""
    M, bits, group = 2, 5, 32
    c = synth.qvm_case(M, N, K, bits, group, "f16", seed=N + K)
    for ws in (None, _workspace(q, M, N)):
        y = _run(q, c, ws)
        ref, ad = _oracle(c)
        assert_close(y, ref, ad, "f16", what=f"qvm N={N} K={K} ws={ws is not None}")


def test_qvm_k_zero_writes_zero(q):
    M, N = 3, 512
    y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    e = torch.empty(16, dtype=torch.uint8, device="cuda")
    q.qmv_qvm_affine(e, e, e, e, y, M, N, 0, 4, 64, "bf16", workspace=_workspace(q, M, N))
    torch.cuda.synchronize()
    assert (y == 0).all()


def test_qvm_precision_case(q):
    """x ~ U(1e-4, 1e-3) with symmetric zero points: the bias term cancels most
    of the scale term, exposing low-precision partial sums."""
    for bits in (2, 3, 4, 5, 6):
        c = synth.qvm_case(1, 2048, 2560, bits, 64, "bf16", seed=bits, precision=True)
        y = _run(q, c, _workspace(q, 1, 2048))
        ref, ad = _oracle(c)
        assert_close(y, ref, ad, "bf16", what=f"qvm precision b{bits}")


def test_qvm_repeated_calls_share_the_workspace(q):
    """Two calls in a row on one workspace (and a third of another shape):
    each result matches, and the workspace is zero after each."""
    ws = _workspace(q, 4, 3072)
    for i, (M, N, K) in enumerate([(4, 3072, 2048), (4, 3072, 2048), (1, 1024, 4096)]):
        c = synth.qvm_case(M, N, K, 4, 128, "bf16", seed=100 + i)
        y = _run(q, c, ws)
        ref, ad = _oracle(c)
        assert_close(y, ref, ad, "bf16", what=f"qvm call {i}")
        assert not ws.any()


def test_qvm_large_matrix_sampled(q):
    """16384 x 16384 at 4-bit g64, bf16, M = 1 with the workspace (the launch
    the benchmark times): sampled columns across every tile match the oracle."""
    M, N, K, bits, group = 1, 16384, 16384, 4, 64
    c = synth.qvm_case(M, N, K, bits, group, "bf16", seed=42)
    y = _run(q, c, _workspace(q, M, N))
    cols = sorted({0, 1, 1023, 1024, 8191, 16383} | set(np.random.default_rng(1).integers(0, N, 42).tolist()))
    ref, ad = _oracle(c, cols=cols)
    assert_close(y[:, cols], ref[:, cols], ad[:, cols], "bf16", what="qvm 16384^2 sampled")
