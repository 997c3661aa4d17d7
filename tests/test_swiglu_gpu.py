"""GPU parity of the fused gate + up projection with SwiGLU
(qmv_affine_swiglu) against the oracle (oracle.qmv_affine_swiglu).

Tolerance, derived from the qmv bars: the kernel forms gate and up as fp32
accumulators held to the f32 bar (REL_FLOOR * sum|x*w| of each), applies the
activation in fp32 and rounds mid once.  With f(g) = silu(clamp(g)) and
|f'| <= 1.1, an accumulator error e_g, e_u moves mid by at most
rw * (1.1 |e_g| |u| + |f(g)| |e_u|); the activation's own fp32 operations (exp,
one division, three products) add a few fp32 ulps, bounded by 2^-20 |mid|.  An
output passes when it is within 1 ulp of its dtype at mid_ref (the workload's
bar), or within that propagated bound.
"""
from __future__ import annotations

import zlib

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import THREADS, TORCH_DT, dev, require_cuda, sample_rows, to_f64
from qmv_tol import REL_FLOOR, ulp

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


def _case(M, N, K, bits, group, dtype, seed):
    cg = synth.affine_case(M, N, K, bits, group, dtype, seed=seed)
    cu = synth.affine_case(M, N, K, bits, group, dtype, seed=seed + 1)
    return cg, cu


def _run(q, cg, cu, M, N, K, bits, group, dtype, clamp=0.0, rw=None, w_offset=0, x=None):
    mid = torch.full((M, N), float("nan"), dtype=TORCH_DT[dtype], device="cuda")
    rwd = torch.tensor(np.asarray(rw, dtype=np.float32), device="cuda") if rw is not None else None
    xx = cg["x"][0] if x is None else x
    q.qmv_affine_swiglu(dev(xx), dev(cg["w"][0], w_offset), dev(cg["scales"][0]), dev(cg["biases"][0]),
                        dev(cu["w"][0], w_offset), dev(cu["scales"][0]), dev(cu["biases"][0]), rwd, mid,
                        M, N, K, bits, group, dtype, clamp)
    torch.cuda.synchronize()
    return to_f64(mid)


def _check(got, cg, cu, M, N, K, bits, group, dtype, clamp=0.0, rw=None, rows=None, what="", x=None):
    xx = cg["x"][0] if x is None else x
    r = list(range(N)) if rows is None else rows
    mid, g, u, ag, au = oracle.qmv_affine_swiglu(
        np.ascontiguousarray(xx), cg["w"][0], cg["scales"][0], cg["biases"][0], cu["w"][0], cu["scales"][0],
        cu["biases"][0], M, N, K, bits, group, dtype, clamp=clamp,
        route_weight=1.0 if rw is None else np.asarray(rw, np.float64), threads=THREADS)
    mid, g, u, ag, au = (a[:, r] for a in (mid, g, u, ag, au))
    got = got[:, r]
    gc, uc = (np.minimum(g, clamp), np.clip(u, -clamp, clamp)) if clamp > 1e-6 else (g, u)
    with np.errstate(over="ignore"):
        silu = gc / (1.0 + np.exp(-gc))
    w = np.ones((M, 1)) if rw is None else np.abs(np.asarray(rw, np.float64)).reshape(M, 1)
    bound = REL_FLOOR * w * (1.1 * ag * np.abs(uc) + np.abs(silu) * au) + 2.0 ** -20 * np.abs(mid)
    err = np.abs(got - mid)
    ok = err <= bound
    if dtype != "f32":
        ok |= err <= ulp(mid, dtype)
    # past the dtype's largest finite value mid rounds to an infinity
    top = {"f16": 65520.0, "bf16": 3.3961514e38, "f32": 3.4028236e38}[dtype]
    over = np.abs(mid) >= top
    ok = np.where(over, got == np.sign(mid) * np.inf, ok)
    if not ok.all():
        i = tuple(np.argwhere(~ok)[0])
        raise AssertionError(f"{what}: {int((~ok).sum())} / {ok.size} out of tolerance; first at {i}: "
                             f"got={got[i]!r} ref={mid[i]!r} bound={bound[i]!r}")


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("M", [1, 3, 8])
def test_swiglu_grid(q, bits, dtype, M):
    N, K, group = 300, 1024, 64
    cg, cu = _case(M, N, K, bits, group, dtype, _seed("sw", bits, dtype, M))
    got = _run(q, cg, cu, M, N, K, bits, group, dtype)
    _check(got, cg, cu, M, N, K, bits, group, dtype, what=f"swiglu b{bits} {dtype} M{M}")


@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("path", [0, 1])
def test_swiglu_clamp_and_route_weights(q, group, path):
    """Clamp at the median |gate|, |up| (so both sides clamp) and one route
    weight per x row; narrow (4-byte) and wide (16-byte) loads."""
    q.qmv_force_config(path, -1, -1, -1)
    M, N, K, bits, dtype = 4, 257, 2048, 4, "bf16"
    cg, cu = _case(M, N, K, bits, group, dtype, _seed("swc", group, path))
    _, g, u, _, _ = oracle.qmv_affine_swiglu(cg["x"][0], cg["w"][0], cg["scales"][0], cg["biases"][0],
                                             cu["w"][0], cu["scales"][0], cu["biases"][0], M, N, K, bits, group,
                                             dtype, threads=THREADS)
    clamp = float(np.median(np.abs(np.concatenate([g.ravel(), u.ravel()]))))
    rw = [0.5, 2.0, 1.0, 3.25]
    got = _run(q, cg, cu, M, N, K, bits, group, dtype, clamp=clamp, rw=rw)
    _check(got, cg, cu, M, N, K, bits, group, dtype, clamp=clamp, rw=rw, what=f"clamp g{group} path{path}")
    # at or below 1e-6 the clamp is off: the same as no clamp, bit for bit
    a = _run(q, cg, cu, M, N, K, bits, group, dtype, clamp=1e-7)
    b = _run(q, cg, cu, M, N, K, bits, group, dtype, clamp=0.0)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("bits", [3, 4, 8])
def test_swiglu_misaligned_weights_and_split_k(q, bits):
    """Weights 4 bytes off a 16-byte boundary take the 4-byte path; narrow N
    spreads K over several warps (the cross-warp pair epilogue)."""
    M, N, K, group, dtype = 2, 20, 4096, 64, "f16"
    cg, cu = _case(M, N, K, bits, group, dtype, _seed("swm", bits))
    got = _run(q, cg, cu, M, N, K, bits, group, dtype, w_offset=4)
    _check(got, cg, cu, M, N, K, bits, group, dtype, what=f"misaligned b{bits}")
    q.qmv_force_config(1, 2, 4, 1)                  # 2 rows per warp, K over 4 warps
    got = _run(q, cg, cu, M, N, K, bits, group, dtype)
    _check(got, cg, cu, M, N, K, bits, group, dtype, what=f"split-K b{bits}")


def test_swiglu_large_gate_limits(q):
    """Gate biases of +-40: silu(40) = 40, silu(-40) -> 0 (exp overflows to
    inf only below about -88; here e^40 is finite)."""
    M, N, K, bits, group, dtype = 1, 64, 256, 4, 64, "f32"
    cg, cu = _case(M, N, K, bits, group, dtype, 91)
    cg = dict(cg)
    cg["w"] = np.zeros_like(cg["w"])
    b = np.where(np.arange(N)[:, None] % 2 == 0, 40.0, -40.0) * np.ones((1, K // group))
    cg["biases"] = synth.to_storage(b[None], dtype)
    x = synth.to_storage(np.full((1, K), 1.0 / K), dtype)
    got = _run(q, cg, cu, M, N, K, bits, group, dtype, x=x)
    _check(got, cg, cu, M, N, K, bits, group, dtype, x=x, what="limits")


@pytest.mark.parametrize("M", [1, 8])
def test_swiglu_7b_gate_up(q, M):
    """The 7B-class layer's gate + up pair (two 14336 x 4096 matrices, 4-bit
    g64 bf16), sampled rows."""
    N, K, bits, group, dtype = 14336, 4096, 4, 64, "bf16"
    cg, cu = _case(M, N, K, bits, group, dtype, _seed("sw7b", M))
    got = _run(q, cg, cu, M, N, K, bits, group, dtype, clamp=10.0)
    _check(got, cg, cu, M, N, K, bits, group, dtype, clamp=10.0, rows=sample_rows(N, 40), what=f"7b M{M}")


def test_swiglu_empty_and_k0(q):
    M, N, K, bits, group, dtype = 2, 16, 0, 4, 64, "bf16"
    mid = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    x = torch.zeros(1, dtype=torch.bfloat16, device="cuda")
    q.qmv_affine_swiglu(x, None, None, None, None, None, None, None, mid, M, N, K, bits, group, dtype)
    torch.cuda.synchronize()
    assert (mid.float() == 0).all()
    q.qmv_affine_swiglu(None, None, None, None, None, None, None, None, mid, 0, N, 64, bits, group, dtype)
    with pytest.raises(q.QmvError):
        q.qmv_affine_swiglu(x, x, x, x, x, x, x, None, mid, M, N, 64, bits, group, dtype, -1.0)
