"""GPU parity of the expert-indexed qmv (qmv_affine_gather) against the oracle:
each token multiplies its x rows by the weight matrix its device-side expert
id selects.  Covers repeated and unused experts, shared and per-token x, the
few-rows kernel (small N) and the row-tiled kernel, every width, and an
out-of-range id (NaN token, the others unchanged)."""
from __future__ import annotations

import numpy as np
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


def _stack(E, N, K, bits, group, dtype, seed):
    cs = [synth.affine_case(1, N, K, bits, group, dtype, seed=seed + e) for e in range(E)]
    return (np.stack([c["w"][0] for c in cs]), np.stack([c["scales"][0] for c in cs]),
            np.stack([c["biases"][0] for c in cs]))


def _run(q, x, w, sc, bi, ids, M, N, K, bits, group, dtype, E, x_batched=True):
    T = len(ids)
    y = torch.full((T, M, N), float("nan"), dtype=TORCH_DT[dtype], device="cuda")
    idt = torch.from_numpy(np.asarray(ids, dtype=np.int32)).cuda()
    q.qmv_affine_gather(dev(x), dev(w), dev(sc), dev(bi), idt, y, M, N, K, bits, group, dtype, T, E,
                        x_batched=x_batched)
    torch.cuda.synchronize()
    return to_f64(y)


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 8])
@pytest.mark.parametrize("N", [40, 1000])
@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
def test_gather_matches_oracle(q, bits, N, dtype):
    E, T, M, K, group = 6, 7, 2, 1024, 64
    w, sc, bi = _stack(E, N, K, bits, group, dtype, seed=bits * 31 + N)
    x = synth.affine_case(M, 1, K, bits, group, dtype, seed=5, batch=T)["x"]
    ids = np.array([3, 0, 3, 5, 1, 3, 0], dtype=np.int32)           # repeats; expert 2, 4 unused
    y = _run(q, x, w, sc, bi, ids, M, N, K, bits, group, dtype, E)
    ref, ad = oracle.qmv_affine_gather(x, w, sc, bi, ids, M, N, K, bits, group, dtype, E, threads=THREADS)
    assert_close(y, ref, ad, dtype, what=f"gather b{bits} N={N} {dtype}")


@pytest.mark.parametrize("N", [24, 1536])
def test_gather_shared_x_and_bad_id(q, N):
    E, T, M, K, bits, group = 4, 5, 1, 2048, 4, 128
    w, sc, bi = _stack(E, N, K, bits, group, "bf16", seed=N)
    x = synth.affine_case(M, 1, K, bits, group, "bf16", seed=8)["x"][0]      # one [M, K] for every token
    ids = np.array([1, 7, 0, -1, 3], dtype=np.int32)                          # 7 and -1: no such expert
    y = _run(q, x, w, sc, bi, ids, M, N, K, bits, group, "bf16", E, x_batched=False)
    ref, ad = oracle.qmv_affine_gather(x, w, sc, bi, ids, M, N, K, bits, group, "bf16", E, x_batched=False,
                                       threads=THREADS)
    assert np.isnan(y[1]).all() and np.isnan(y[3]).all()
    good = [0, 2, 4]
    assert_close(y[good], ref[good], ad[good], "bf16", what=f"gather shared x N={N}")
