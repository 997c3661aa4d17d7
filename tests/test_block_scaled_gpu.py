"""GPU parity of the Track-1 block-scaled formats (qmv_block_scaled and its
check kernel qmv_dequant_block_scaled_f32) against the fp64 oracle
(oracle.qmv_block_scaled / oracle.dequant_block_scaled_f32).

Covers all 30 formats of the wh-iron audit's Track 1 table: every format x
dtype x M in {1, 3, 8} on a ragged N; the 16-code tail block (K % 32 == 16)
of NVFP4 / NVFP8; every code byte of every element type through the check
kernel (bit-exact, NaN and infinity included); the CUDA-core row-tiled kernel
on both load widths and the few-rows kernel, forced; the sum(x) precision case
for the signed integers (read as offset binary with a -2^(b-1) * scale bias);
layer-sized matrices on sampled rows; the row-tail prefix rule; batches.
Same tolerance as every qmv test (qmv_tol.py).
"""
from __future__ import annotations

import zlib

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import THREADS, compare, dev, require_cuda, sample_rows, to_f64, y_buffer

pytestmark = pytest.mark.gpu

FORMATS = sorted(oracle.TRACK1)
SIXTEEN = [f for f in FORMATS if oracle.TRACK1[f][2] == 16]


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


def _case(fmt, M, N, K, dtype, seed, **kw):
    return synth.bs_case(M, N, K, *oracle.TRACK1[fmt], dtype, seed=seed, **kw)


def _glob(c):
    if c["global"] is None:
        return None
    return torch.tensor(np.full(c["batch"], c["global"], dtype=np.float32), device="cuda")


def _run(q, c, fmt, w_offset=0, x_batched=True):
    B, M, N, K = c["batch"], c["M"], c["N"], c["K"]
    x = c["x"] if x_batched else c["x"][:1]
    y = y_buffer(B, M, N, c["dtype"])
    args = (dev(x), dev(c["w"], w_offset), dev(c["scales"]), _glob(c), y, M, N, K, fmt, c["dtype"])
    if B == 1 and x_batched:
        q.qmv_block_scaled(*args)
    else:
        q.qmv_block_scaled_batched(*args, B, x_batched)
    torch.cuda.synchronize()
    return to_f64(y)


def _oracle(c, fmt, rows=None, b=0, x_batched=True):
    xb = b if x_batched else 0
    return oracle.qmv_block_scaled(np.ascontiguousarray(c["x"][xb]), np.ascontiguousarray(c["w"][b]),
                                   np.ascontiguousarray(c["scales"][b]), c["global"], c["M"], c["N"], c["K"],
                                   fmt, c["dtype"], rows=rows, threads=THREADS)


def _same_bits(a, b):
    """Bit-equal fp32 arrays, any NaN matching any NaN."""
    a = np.asarray(a, np.float32)
    b = np.asarray(b, np.float32)
    na, nb = np.isnan(a), np.isnan(b)
    return np.array_equal(na, nb) and np.array_equal(a[~na].view(np.uint32), b[~nb].view(np.uint32))


# ------------------------------------------------------------ the layout ----
def test_format_info_matches_the_oracle_table(q):
    assert sorted(q.FORMATS) == FORMATS
    for f in FORMATS:
        e, bits, blk, sk, ug = oracle.TRACK1[f]
        info = q.qmv_format_info(f)
        assert info == {"element_bits": bits, "block": blk, "scale_bytes": synth.bs_case(
            1, 1, blk * 2, e, bits, blk, sk, ug, "f32", 0)["scale_bytes"], "has_global": ug}, f


# ------------------------------------------------------ the check kernel ----
@pytest.mark.parametrize("fmt", FORMATS)
def test_bs_dequant_bit_exact(q, fmt):
    blk = oracle.TRACK1[fmt][2]
    N = 37
    for K in ([512, 528] if blk == 16 else [512]):
        c = _case(fmt, 1, N, K, "f32", _seed("dq", fmt, K))
        out = torch.empty((N, K), dtype=torch.float32, device="cuda")
        q.qmv_dequant_block_scaled_f32(dev(c["w"][0]), dev(c["scales"][0]), _glob(c), out, N, K, fmt)
        torch.cuda.synchronize()
        ref = oracle.dequant_block_scaled_f32(c["w"][0], c["scales"][0], c["global"], N, K, fmt)
        assert _same_bits(out.cpu().numpy(), ref), (fmt, K)


@pytest.mark.parametrize("fmt", ["mxfp8_e5m2", "fp8_e5m2", "fp8_e5m2_f16", "nvfp8", "fp8_e4m3_f16", "fp4",
                                 "int8", "mxint5", "int3_f16", "int2"])
def test_bs_dequant_every_code(q, fmt):
    """Every code byte (E5M2 infinities and NaNs, E4M3 NaNs, every int field)
    under several scales, bit for bit (NaN as NaN)."""
    e, bits, blk, sk, ug = oracle.TRACK1[fmt]
    K = 2048                             # K * bits / 8 = 256 * bits bytes: every byte value
    N = 4
    c = _case(fmt, 1, N, K, "f32", _seed("every", fmt))
    row = np.tile(np.arange(256, dtype=np.uint8), bits)
    c["w"] = np.ascontiguousarray(np.broadcast_to(row, (1, N, row.size)))
    out = torch.empty((N, K), dtype=torch.float32, device="cuda")
    q.qmv_dequant_block_scaled_f32(dev(c["w"][0]), dev(c["scales"][0]), _glob(c), out, N, K, fmt)
    torch.cuda.synchronize()
    ref = oracle.dequant_block_scaled_f32(c["w"][0], c["scales"][0], c["global"], N, K, fmt)
    assert _same_bits(out.cpu().numpy(), ref), fmt


def test_bs_dequant_f16_subnormal_scales(q):
    for fmt in ("fp8_e5m2_f16", "int4_f16", "nvfp8_f16"):
        blk = oracle.TRACK1[fmt][2]
        N, K = 8, 8 * blk
        c = _case(fmt, 1, N, K, "f32", _seed("sub", fmt), scale_range=(1e-7, 5e-6))
        out = torch.empty((N, K), dtype=torch.float32, device="cuda")
        q.qmv_dequant_block_scaled_f32(dev(c["w"][0]), dev(c["scales"][0]), None, out, N, K, fmt)
        torch.cuda.synchronize()
        ref = oracle.dequant_block_scaled_f32(c["w"][0], c["scales"][0], None, N, K, fmt)
        assert _same_bits(out.cpu().numpy(), ref), fmt


# ----------------------------------------------------------- the product ----
@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("M", [1, 3, 8])
def test_bs_qmv_grid(q, fmt, dtype, M):
    N, K = 300, 1024
    c = _case(fmt, M, N, K, dtype, _seed("grid", fmt, dtype, M))
    y = _run(q, c, fmt)[0]
    ref, ad = _oracle(c, fmt)
    compare(y, ref, ad, dtype, what=f"{fmt} {dtype} M{M}")


@pytest.mark.parametrize("fmt", SIXTEEN)
@pytest.mark.parametrize("M", [1, 4])
@pytest.mark.parametrize("N", [5, 300])
def test_bs_sixteen_code_tail_block(q, fmt, M, N):
    """K % 32 == 16: the last block of each row lies outside the 32-code units
    (both the few-rows and the row-tiled kernel)."""
    for K in (48, 1040, 4112):
        c = _case(fmt, M, N, K, "bf16", _seed("tail16", fmt, M, N, K))
        y = _run(q, c, fmt)[0]
        ref, ad = _oracle(c, fmt)
        compare(y, ref, ad, "bf16", what=f"{fmt} K{K} M{M} N{N}")


def test_nvfp4_tail_block_through_qmv_fp(q):
    M, N, K = 2, 77, 2064
    c = _case("nvfp4", M, N, K, "f16", _seed("fp16tail"))
    y = y_buffer(1, M, N, "f16")
    q.qmv_fp(dev(c["x"]), dev(c["w"]), dev(c["scales"]), _glob(c), y, M, N, K, "nvfp4", "f16")
    torch.cuda.synchronize()
    ref, ad = _oracle(c, "nvfp4")
    compare(to_f64(y)[0], ref, ad, "f16", what="qmv_fp nvfp4 K%32==16")


@pytest.mark.parametrize("fmt", ["int3", "mxint6", "int8_f16", "fp8_e5m2", "nvfp8_f16", "fp4_f16", "mxfp8_e5m2"])
@pytest.mark.parametrize("path", [0, 1, 5])
def test_bs_forced_paths(q, fmt, path):
    """Row-tiled kernel on 4-byte loads (0) and 16-byte loads (1), and the
    few-rows kernel (5), forced."""
    q.qmv_force_config(path, -1, -1, -1)
    for M in (1, 5):
        c = _case(fmt, M, 129, 2048, "bf16", _seed("paths", fmt, path, M))
        plan = q.qmv_describe_plan(fmt, M, 129, 2048, dtype="bf16")
        want = {0: "path=narrow", 1: "path=wide", 5: "path=direct"}[path]
        if path == 1 and "path=wide" not in plan:
            pytest.skip("no 16-byte chunk for this width: " + plan.split()[0])
        assert want in plan, plan
        y = _run(q, c, fmt)[0]
        ref, ad = _oracle(c, fmt)
        compare(y, ref, ad, "bf16", what=f"{fmt} path{path} M{M}")


RING_FORMATS = [f for f in FORMATS if not f.startswith(("int", "mxint"))]


@pytest.mark.parametrize("fmt", RING_FORMATS)
def test_bs_weight_ring_path(q, fmt):
    """One bf16 x row through the weight ring (forced path 6): ragged row
    blocks, several stages per row block, more row blocks than the grid."""
    q.qmv_force_config(6, -1, -1, -1)
    for (N, K) in [(333, 4096), (148 * 128 * 2 + 45, 1024)]:
        plan = q.qmv_describe_plan(fmt, 1, N, K, dtype="bf16")
        assert "path=tcf" in plan, plan
        c = _case(fmt, 1, N, K, "bf16", _seed("ring", fmt, N, K))
        y = _run(q, c, fmt)[0]
        rows = sample_rows(N, 64) + list(range(N - 70, N))
        rows = sorted(set(rows))
        ref, ad = _oracle(c, fmt, rows=rows)
        compare(y, ref, ad, "bf16", rows=rows, what=f"ring {fmt} {N}x{K}")
    assert q.qmv_device_fault(clear=True) == 0


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "mxfp8_e4m3", "fp8_e5m2_f16", "nvfp8"])
def test_bs_weight_ring_precision_and_batch(q, fmt):
    """The precision case and a batch of 2 (NVFP4: one global per entry)
    through the weight ring (forced)."""
    N, K = 2048, 6144
    q.qmv_force_config(6, -1, -1, -1)
    assert "path=tcf" in q.qmv_describe_plan(fmt, 1, N, K, dtype="bf16")
    c = _case(fmt, 1, N, K, "bf16", _seed("ringprec", fmt), precision=True)
    y = _run(q, c, fmt)[0]
    ref, ad = _oracle(c, fmt)
    compare(y, ref, ad, "bf16", what=f"ring precision {fmt}", max_floor_frac=0.25)
    c = _case(fmt, 1, 300, 2048, "bf16", _seed("ringbatch", fmt), batch=2)
    if c["global"] is not None:
        c["global"] = np.float32(1.5)
    y = _run(q, c, fmt)
    for b in range(2):
        ref, ad = _oracle(c, fmt, b=b)
        compare(y[b], ref, ad, "bf16", what=f"ring batch {fmt} {b}")
    assert q.qmv_device_fault(clear=True) == 0


@pytest.mark.parametrize("fmt", ["int2", "int3", "int4", "int5", "int6", "int8", "mxint4", "int4_f16"])
@pytest.mark.parametrize("M", [1, 8])
def test_bs_signed_int_precision_case(q, fmt, M):
    """x ~ U(1e-4, 1e-3): the offset-binary partial and the -2^(b-1) * scale *
    sum(x) bias term cancel to a small residue, as in the affine precision
    case; sum(x) is widened per element."""
    c = _case(fmt, M, 4096, 2560, "bf16", _seed("prec", fmt, M), precision=True)
    y = _run(q, c, fmt)[0]
    ref, ad = _oracle(c, fmt)
    compare(y, ref, ad, "bf16", what=f"precision {fmt} M{M}", max_floor_frac=0.25)


@pytest.mark.parametrize("fmt", ["nvfp8", "fp8_e5m2", "mxfp8_e5m2", "fp4"])
def test_bs_fp_precision_case(q, fmt):
    c = _case(fmt, 2, 2048, 2048, "f16", _seed("fprec", fmt), precision=True)
    y = _run(q, c, fmt)[0]
    ref, ad = _oracle(c, fmt)
    compare(y, ref, ad, "f16", what=f"precision {fmt}", max_floor_frac=0.25)


@pytest.mark.parametrize("fmt", ["int4", "mxint4", "int8", "mxfp8_e5m2", "nvfp8", "fp4_f16"])
@pytest.mark.parametrize("M", [1, 8])
def test_bs_layer_shapes(q, fmt, M):
    """7B-layer projections (6144x4096, 28672x4096, 4096x14336), sampled rows."""
    for (N, K) in [(6144, 4096), (28672, 4096), (4096, 14336)]:
        c = _case(fmt, M, N, K, "bf16", _seed("layer", fmt, M, N, K))
        y = _run(q, c, fmt)[0]
        rows = sample_rows(N, 32)
        ref, ad = _oracle(c, fmt, rows=rows)
        compare(y, ref, ad, "bf16", rows=rows, what=f"{fmt} {N}x{K} M{M}")


@pytest.mark.parametrize("fmt", ["int5", "mxint2", "fp8_e5m2_f16", "nvfp8"])
def test_bs_tail_rows_bitwise_prefix(q, fmt):
    q.qmv_force_config(1 if oracle.TRACK1[fmt][1] % 4 == 0 else 0, 2, 1, 4)     # row tile = 8
    big = _case(fmt, 1, 24, 2048, "bf16", _seed("rowtail", fmt))
    yb = _run(q, big, fmt)[0]
    for n in (1, 5, 9, 17):
        small = dict(big, N=n, w=big["w"][:, :n].copy(), scales=big["scales"][:, :n].copy())
        assert np.array_equal(_run(q, small, fmt)[0], yb[:, :n]), (fmt, n)


@pytest.mark.parametrize("fmt", ["nvfp4", "int6_f16", "mxfp8_e5m2"])
@pytest.mark.parametrize("x_batched", [True, False])
def test_bs_batched(q, fmt, x_batched):
    B, M, N, K = 3, 2, 65, 1024
    c = _case(fmt, M, N, K, "bf16", _seed("batch", fmt, x_batched), batch=B)
    y = _run(q, c, fmt, x_batched=x_batched)       # NVFP4: the same global for every entry
    for b in range(B):
        ref, ad = _oracle(c, fmt, b=b, x_batched=x_batched)
        compare(y[b], ref, ad, "bf16", what=f"{fmt} batch {b}")


def test_bs_misaligned_weights_take_the_narrow_path(q):
    for fmt in ("int4", "mxfp8_e5m2", "fp4_f16"):
        c = _case(fmt, 2, 200, 1024, "f16", _seed("mis", fmt))
        y = _run(q, c, fmt, w_offset=4)[0]
        ref, ad = _oracle(c, fmt)
        compare(y, ref, ad, "f16", what=f"{fmt} w+4")


def test_bs_argument_errors(q):
    c = _case("nvfp8", 1, 4, 64, "bf16", 1)
    x, w, s = dev(c["x"]), dev(c["w"]), dev(c["scales"])
    y = y_buffer(1, 1, 4, "bf16")
    with pytest.raises(q.QmvError):                       # format out of range
        q.qmv_block_scaled(x, w, s, None, y, 1, 4, 64, 30, "bf16")
    with pytest.raises(q.QmvError):                       # K not a multiple of the block
        q.qmv_block_scaled(x, w, s, None, y, 1, 4, 40, "nvfp8", "bf16")
    g = torch.ones(1, device="cuda")
    with pytest.raises(q.QmvError):                       # a global for a format without one
        q.qmv_block_scaled(x, w, s, g, y, 1, 4, 64, "nvfp8", "bf16")
    with pytest.raises(q.QmvError):                       # NVFP4 without its global
        q.qmv_block_scaled(x, w, s, None, y, 1, 4, 64, "nvfp4", "bf16")
    with pytest.raises(q.QmvError):                       # FP32 scales off a 4-byte boundary
        q.qmv_block_scaled(x, w, dev(c["scales"], 2), None, y, 1, 4, 64, "nvfp8", "bf16")
