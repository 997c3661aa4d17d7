"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, on the
same seeded host bytes.  Every test here needs a B200 and is marked ``gpu``.

Bars (see qmv_tol.py): dequantized weights bit-exact; f16 / bf16 outputs within
1 ulp of the fp64 oracle (or 1e-5 * sum|x*w| where the sum cancels); f32 outputs
within 1e-5 * sum|x*w|.  Workloads: every shape the workload list names, at
full size (oracle on sampled rows) and at small sizes (oracle on every row),
plus ragged N and K, batches, M = 1..8, empty and degenerate cases.
"""
from __future__ import annotations

import zlib

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import (THREADS, compare, dev, oracle_affine, oracle_fp, require_cuda, run_affine, run_fp,
                      sample_rows, to_f64, y_buffer)

pytestmark = pytest.mark.gpu

BITS = [2, 3, 4, 5, 6, 8]
GROUPS = [32, 64, 128]
DTYPES = ["f32", "f16", "bf16"]
MODES = ["mxfp4", "nvfp4", "mxfp8"]


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


# ------------------------------------------------------------- native code --
def test_native_library_is_what_runs(q):
    c = synth.affine_case(1, 8, 64, 4, 64, "bf16", seed=1)
    run_affine(q, c)
    maps = open("/proc/self/maps").read()
    assert q.LIB_PATH in maps


# ------------------------------------------------------- dequant bit-exact --
def _bits_equal(a, b):
    a = np.asarray(a, np.float32); b = np.asarray(b, np.float32)
    nan = np.isnan(a) & np.isnan(b)
    return bool(np.all(nan | (a.view(np.uint32) == b.view(np.uint32))))


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("group", GROUPS)
@pytest.mark.parametrize("dtype", DTYPES)
def test_dequant_affine_bit_exact(q, bits, group, dtype):
    N, K = 37, 384
    c = synth.affine_case(1, N, K, bits, group, dtype, seed=_seed("dqa", bits, group, dtype))
    out = torch.empty((N, K), dtype=torch.float32, device="cuda")
    q.qmv_dequant_affine_f32(dev(c["w"]), dev(c["scales"]), dev(c["biases"]), out, N, K, bits, group, dtype)
    torch.cuda.synchronize()
    ref = oracle.dequant_affine_f32(c["w"][0], c["scales"][0], c["biases"][0], N, K, bits, group, dtype)
    assert _bits_equal(out.cpu().numpy(), ref)


@pytest.mark.parametrize("mode", MODES)
def test_dequant_fp_bit_exact_all_codes(q, mode):
    """Every code byte and every scale byte (NaN encodings included)."""
    bits, blk = synth.FP_BITS[mode], synth.FP_BLOCK[mode]
    N, K = 256, 512
    w = np.tile(np.arange(256, dtype=np.uint8), N * K * bits // 8 // 256 + 1)[: N * K * bits // 8]
    w = np.ascontiguousarray(np.random.default_rng(3).permutation(w).reshape(N, K * bits // 8))
    sc = (np.arange(N * (K // blk)) % 256).astype(np.uint8).reshape(N, K // blk)
    g = np.float32(1.3) if mode == "nvfp4" else None
    out = torch.empty((N, K), dtype=torch.float32, device="cuda")
    gd = torch.tensor([g], device="cuda") if g is not None else None
    q.qmv_dequant_fp_f32(dev(w), dev(sc), gd, out, N, K, mode)
    torch.cuda.synchronize()
    ref = oracle.dequant_fp_f32(w, sc, g, N, K, mode)
    assert _bits_equal(out.cpu().numpy(), ref)


# ---------------------------------------------------- the small workload ----
def test_small_config_4bit(q):
    """M=1, N=256, K=512, 4-bit g64 bf16, seed 0 (every row checked)."""
    c = synth.affine_case(1, 256, 512, 4, 64, "bf16", seed=0)
    y = run_affine(q, c)[0]
    ref, ad = oracle_affine(c)
    compare(y, ref, ad, "bf16", what="small 4-bit")


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("group", GROUPS)
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("M", [1, 3, 8])
def test_affine_grid(q, bits, group, dtype, M):
    N, K = 67, 512
    c = synth.affine_case(M, N, K, bits, group, dtype, seed=_seed("grid", bits, group, dtype, M))
    y = run_affine(q, c)[0]
    ref, ad = oracle_affine(c)
    compare(y, ref, ad, dtype, what=f"b{bits} g{group} {dtype} M{M}")


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("M", [1, 2, 5])
def test_affine_narrow_path_ragged_k(q, bits, M):
    """K a multiple of the group but not of the wide chunk -> 4-byte chunks."""
    N, K, group = 45, 480, 32
    c = synth.affine_case(M, N, K, bits, group, "bf16", seed=_seed("narrow", bits, M))
    y = run_affine(q, c)[0]
    ref, ad = oracle_affine(c)
    compare(y, ref, ad, "bf16", what=f"narrow b{bits}")


@pytest.mark.parametrize("bits", BITS)
def test_affine_misaligned_w_uses_narrow_path(q, bits):
    N, K, group = 33, 1024, 64
    c = synth.affine_case(2, N, K, bits, group, "f16", seed=_seed("mis", bits))
    y = run_affine(q, c, w_offset=4)[0]
    ref, ad = oracle_affine(c)
    compare(y, ref, ad, "f16", what=f"misaligned b{bits}")


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("N", [1, 3, 5, 12, 17])
def test_fast_rows_output_sizes(q, bits, N):
    """The MLX fast_rows test sizes: K=2560, group 64, with batched weights."""
    c = synth.affine_case(1, N, 2560, bits, 64, "bf16", seed=_seed("rows", bits, N), batch=2)
    y = run_affine(q, c)
    for b in range(2):
        ref, ad = oracle_affine(c, b=b)
        compare(y[b], ref, ad, "bf16", what=f"rows b{bits} N{N} batch{b}")


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("N", [1, 3, 5, 7, 8, 9, 12, 17])
def test_fp_output_sizes(q, mode, dtype, N):
    """The MLX fp fast_rows test sizes, all three modes and dtypes, batched."""
    c = synth.fp_case(1, N, 1024, mode, dtype, seed=_seed("fprows", mode, dtype, N), batch=2)
    y = run_fp(q, c)
    for b in range(2):
        ref, ad = oracle_fp(c, b=b)
        compare(y[b], ref, ad, dtype, what=f"{mode} {dtype} N{N} b{b}")


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("shape", [(5, 1024, 2), (12, 4096, 1)])
@pytest.mark.parametrize("x_batched", [True, False])
def test_fp_workload_shapes(q, mode, shape, x_batched):
    """Block-scaled FP workload shapes: (N=5, K=1024, batch=2 weights) and
    (N=12, K=4096), bf16 x; x either batched or shared."""
    N, K, B = shape
    c = synth.fp_case(1, N, K, mode, "bf16", seed=_seed("fpw", mode, N), batch=B)
    y = run_fp(q, c, x_batched=x_batched)
    for b in range(B):
        ref, ad = oracle_fp(c, b=b, x_batched=x_batched)
        compare(y[b], ref, ad, "bf16", what=f"{mode} N{N} K{K} b{b}")


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("M", [2, 4, 8])
def test_fp_multi_m(q, mode, M):
    c = synth.fp_case(M, 77, 2048, mode, "bf16", seed=_seed("fpm", mode, M))
    y = run_fp(q, c)[0]
    ref, ad = oracle_fp(c)
    compare(y, ref, ad, "bf16", what=f"{mode} M{M}")


def test_fp_nan_codes_propagate(q):
    c = synth.fp_case(1, 4, 64, "mxfp8", "bf16", seed=4)
    c["w"][0, 2, 5] = 0x7F           # NaN element in row 2
    c["scales"][0, 3, 1] = 0xFF      # NaN block scale in row 3
    y = run_fp(q, c)[0]
    ref, ad = oracle_fp(c)
    assert np.isnan(y[0, 2]) and np.isnan(y[0, 3])
    compare(y, ref, ad, "bf16", what="nan")


# ------------------------------------------------------- tail invariant ----
@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("n", [1, 3, 5, 12, 17])
def test_tail_rows_bitwise_prefix(q, bits, n):
    """N = n equals, bit for bit, the first n rows of the same weights padded
    to a whole row tile (same launch shape), as the MLX fast_rows tests check."""
    q.qmv_force_config(1, 4, 1, 4)            # row tile = 16
    K, group = 2560, 64
    pad = 16 * ((n + 15) // 16)
    big = synth.affine_case(1, pad, K, bits, group, "bf16", seed=_seed("tail", bits, n))
    small = dict(big, N=n, w=big["w"][:, :n].copy(), scales=big["scales"][:, :n].copy(),
                 biases=big["biases"][:, :n].copy())
    yb = run_affine(q, big)[0]
    ys = run_affine(q, small)[0]
    assert np.array_equal(ys, yb[:, :n])


@pytest.mark.parametrize("mode", MODES)
def test_fp_tail_rows_bitwise_prefix(q, mode):
    q.qmv_force_config(1, 2, 1, 4)            # row tile = 8
    big = synth.fp_case(1, 24, 4096, mode, "bf16", seed=_seed("fptail", mode))
    for n in (1, 5, 9, 17):
        small = dict(big, N=n, w=big["w"][:, :n].copy(), scales=big["scales"][:, :n].copy())
        assert np.array_equal(run_fp(q, small)[0], run_fp(q, big)[0][:, :n])


# --------------------------------------------------------- precision case ---
@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6])
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_precision_case_sum_x(q, bits, dtype):
    """x ~ U(1e-4, 1e-3), symmetric zero point: the bias term dominates and a
    low-precision sum(x) would fail (see the mutant pin); every row checked."""
    c = synth.affine_case(1, 4096, 2560, bits, 64, dtype, seed=_seed("prec", bits, dtype), precision=True)
    y = run_affine(q, c)[0]
    ref, ad = oracle_affine(c)
    compare(y, ref, ad, dtype, what=f"precision b{bits} {dtype}")


# -------------------------------------------------- full-size workloads ----
@pytest.mark.parametrize("bits", [2, 3, 5, 6])
@pytest.mark.parametrize("group", GROUPS)
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("M", [1, 4])
def test_sweep_full_size(q, bits, group, dtype, M):
    """Affine sweep at N = K = 4096 (oracle on sampled rows)."""
    c = synth.affine_case(M, 4096, 4096, bits, group, dtype, seed=_seed("sweep", bits, group, dtype, M))
    y = run_affine(q, c)[0]
    rows = sample_rows(4096)
    ref, ad = oracle_affine(c, rows=rows)
    compare(y, ref, ad, dtype, rows=rows, what=f"sweep b{bits} g{group} {dtype} M{M}")


LAYER = [("qkv", 6144, 4096), ("o", 4096, 4096), ("gate_up", 28672, 4096), ("down", 4096, 14336)]


@pytest.mark.parametrize("M", [1, 8])
def test_decode_layer_chain(q, M):
    """7B-class decode layer, 4-bit g64 bf16, the four projections chained:
    each input is the previous output truncated to the next K (oracle fed the
    GPU's actual input, sampled rows)."""
    x = synth.affine_case(M, 1, 4096, 4, 64, "bf16", seed=_seed("layer_x", M))["x"]
    for i, (name, N, K) in enumerate(LAYER):
        c = synth.affine_case(M, N, K, 4, 64, "bf16", seed=_seed("layer", name, M))
        c["x"] = np.ascontiguousarray(x[:, :, :K])
        y = run_affine(q, c)[0]
        rows = sample_rows(N, 32)
        ref, ad = oracle_affine(c, rows=rows)
        compare(y, ref, ad, "bf16", rows=rows, what=f"layer {name} M{M}")
        # next input: this output (bf16 storage), truncated; rescaled to unit
        # RMS on the host so the chain stays in range (parity-only variant)
        yv = y.astype(np.float32)
        yv = yv / np.sqrt(np.mean(yv ** 2, axis=-1, keepdims=True) + 1e-30)
        x = synth.to_storage(yv[None], "bf16")


@pytest.mark.parametrize("M", [1, 8])
def test_bandwidth_probe_16384(q, M):
    c = synth.affine_case(M, 16384, 16384, 4, 64, "bf16", seed=_seed("probe", M))
    y = run_affine(q, c)[0]
    rows = sample_rows(16384, 24)
    ref, ad = oracle_affine(c, rows=rows)
    compare(y, ref, ad, "bf16", rows=rows, what=f"probe M{M}")


# ------------------------------------------------------------ the chain ----
@pytest.mark.parametrize("N", [1, 3, 4, 5, 12, 17, 4096])
def test_chained_calls_8bit(q, N):
    """64 dependent calls, 8-bit g64 bf16, K=2560: call t reads the previous
    output zero-padded (N < K) or truncated (N >= K) to K.  Each call is checked
    against the oracle fed the GPU's actual input, while that input is finite."""
    K, T = 2560, 64
    c = synth.affine_case(1, N, K, 8, 64, "bf16", seed=_seed("chain", N))
    L = max(N, K)
    w, s, b = dev(c["w"]), dev(c["scales"]), dev(c["biases"])
    x0 = torch.zeros(L, dtype=torch.bfloat16, device="cuda")
    x0[:K] = torch.from_numpy(c["x"][0, 0].view(np.int16)).view(torch.bfloat16).cuda()
    bufs = [torch.zeros(L, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    rows = sample_rows(N, 24)
    checked = 0
    for t in range(T):
        xin = x0 if t == 0 else bufs[(t - 1) % 2]
        yout = bufs[t % 2]
        q.qmv_affine(xin, w, s, b, yout, 1, N, K, 8, 64, "bf16")
        torch.cuda.synchronize()
        xh = xin[:K].cpu().view(torch.int16).numpy().view(np.uint16).reshape(1, K)
        xf = xin[:K].float().cpu().numpy()
        # fp32 partial sums of x*q over a 32-code unit overflow once |x| nears
        # fp32_max / (32 * 255) ~ 4e34 (the same range as the scale*sum(xq) +
        # bias*sum(x) formulation on the pages); stop checking before that
        if not np.isfinite(xf).all() or np.abs(xf).max() > 1e30:
            break
        if t % 8 == 0 or N < 4096:
            cc = dict(c, x=xh[None])
            ref, ad = oracle_affine(cc, rows=rows)
            compare(to_f64(yout[:N]).reshape(1, N), ref, ad, "bf16", rows=rows, what=f"chain N{N} t{t}")
            checked += 1
    assert checked >= 2


# ------------------------------------------------------- batches & edges ----
@pytest.mark.parametrize("x_batched", [True, False])
@pytest.mark.parametrize("bits", [3, 4])
def test_affine_batched(q, x_batched, bits):
    c = synth.affine_case(2, 300, 1024, bits, 64, "bf16", seed=_seed("batch", bits, x_batched), batch=3)
    y = run_affine(q, c, x_batched=x_batched)
    for b in range(3):
        ref, ad = oracle_affine(c, b=b, x_batched=x_batched)
        compare(y[b], ref, ad, "bf16", what=f"batch {b}")


def test_k_zero_writes_zeros(q):
    y = torch.full((2, 5), 7.0, dtype=torch.bfloat16, device="cuda")
    dummy = torch.zeros(64, dtype=torch.uint8, device="cuda")
    q.qmv_affine(dummy, dummy, dummy, dummy, y, 2, 5, 0, 4, 64, "bf16")
    torch.cuda.synchronize()
    assert (y.float() == 0).all()


def test_empty_m_or_n_leaves_y(q):
    y = torch.full((4,), 7.0, dtype=torch.bfloat16, device="cuda")
    q.qmv_affine(None, None, None, None, y, 0, 4, 64, 4, 64, "bf16")
    q.qmv_affine(None, None, None, None, y, 1, 0, 64, 4, 64, "bf16")
    torch.cuda.synchronize()
    assert (y.float() == 7).all()


@pytest.mark.parametrize("cfg", [(1, 1, 1, 1), (1, 2, 1, 4), (1, 4, 1, 2), (1, 1, 8, 1), (1, 1, 3, 2),
                                 (0, 1, 1, 4), (0, 1, 4, 2), (1, 2, 2, 4)])
@pytest.mark.parametrize("bits", [3, 4, 8])
def test_forced_launch_shapes(q, cfg, bits):
    """Every launch shape the picker can choose gives the same (tolerance) answer."""
    q.qmv_force_config(*cfg)
    c = synth.affine_case(2, 131, 2048, bits, 64, "bf16", seed=_seed("forced", cfg, bits))
    y = run_affine(q, c)[0]
    ref, ad = oracle_affine(c)
    compare(y, ref, ad, "bf16", what=f"forced {cfg} b{bits}")


@pytest.mark.parametrize("M", [5, 8])
def test_x_tiles_when_x_exceeds_shared_memory(q, M):
    """M * K large enough that x is staged in several K tiles."""
    c = synth.affine_case(M, 96, 16384, 4, 128, "f32", seed=_seed("tiles", M))
    y = run_affine(q, c)[0]
    ref, ad = oracle_affine(c)
    compare(y, ref, ad, "f32", what=f"tiles M{M}")


def test_non_default_stream(q):
    c = synth.affine_case(1, 100, 1024, 5, 32, "bf16", seed=77)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        y = run_affine(q, c, stream=s)[0]
    ref, ad = oracle_affine(c)
    compare(y, ref, ad, "bf16", what="stream")


# ----------------------------------------------------- tensor-core path ----
@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("group", GROUPS)
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("M", [1, 3, 8])
def test_tensor_core_path_grid(q, bits, group, dtype, M):
    """The tensor-core kernel forced on every width / group / dtype (it falls
    back to the CUDA-core kernel only for 2-bit with group 32)."""
    q.qmv_force_config(3, -1, -1, -1)
    N, K = 100, 1024
    plan = q.qmv_describe_plan("affine", M, N, K, bits, group, dtype)
    assert ("path=tc" in plan) == (not (bits == 2 and group == 32)), plan
    c = synth.affine_case(M, N, K, bits, group, dtype, seed=_seed("tc", bits, group, dtype, M))
    y = run_affine(q, c)[0]
    ref, ad = oracle_affine(c)
    compare(y, ref, ad, dtype, what=f"tc b{bits} g{group} {dtype} M{M}")


@pytest.mark.parametrize("cfg", [(3, -1, 1, 1), (3, -1, 8, 1), (3, -1, 1, 8), (3, -1, 3, 2), (3, -1, 2, 4)])
@pytest.mark.parametrize("bits", [2, 5, 8])
def test_tensor_core_block_shapes(q, cfg, bits):
    q.qmv_force_config(*cfg)
    c = synth.affine_case(2, 333, 2048, bits, 64, "bf16", seed=_seed("tcshape", cfg, bits), batch=2)
    y = run_affine(q, c)
    for b in range(2):
        ref, ad = oracle_affine(c, b=b)
        compare(y[b], ref, ad, "bf16", what=f"tc shape {cfg} b{bits} batch{b}")


@pytest.mark.parametrize("bits", BITS)
def test_tensor_core_tail_rows_bitwise_prefix(q, bits):
    q.qmv_force_config(3, -1, 2, 1)            # 16-row tiles, K over 2 warps
    K = 2560
    big = synth.affine_case(1, 48, K, bits, 64, "bf16", seed=_seed("tctail", bits))
    yb = run_affine(q, big)[0]
    for n in (1, 5, 17, 33):
        small = dict(big, N=n, w=big["w"][:, :n].copy(), scales=big["scales"][:, :n].copy(),
                     biases=big["biases"][:, :n].copy())
        assert np.array_equal(run_affine(q, small)[0], yb[:, :n])


def test_tensor_core_x_tiles(q):
    """M=8, f32 x, K large enough that x is staged in several K tiles."""
    q.qmv_force_config(3, -1, -1, -1)
    c = synth.affine_case(8, 80, 16384, 4, 32, "f32", seed=_seed("tctile"))
    assert "path=tc" in q.qmv_describe_plan("affine", 8, 80, 16384, 4, 32, "f32")
    y = run_affine(q, c)[0]
    ref, ad = oracle_affine(c)
    compare(y, ref, ad, "f32", what="tc tiles")


# ------------------------------------------ tensor cores + bulk-copy ring ----
@pytest.fixture
def ring(q):
    """Force the bulk-ring kernel; afterwards no bounded wait may have expired."""
    q.qmv_device_fault(clear=True)
    yield
    torch.cuda.synchronize()
    assert q.qmv_device_fault(clear=True) == 0


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("group", GROUPS)
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("M", [1, 3, 8])
def test_bulk_ring_path_grid(q, ring, bits, group, dtype, M):
    """The bulk-ring kernel on every width / group / dtype (2-bit with group
    32 falls back: a 64-code unit would span two groups)."""
    q.qmv_force_config(4, -1, -1, -1)
    N, K = 100, 1024
    plan = q.qmv_describe_plan("affine", M, N, K, bits, group, dtype)
    assert ("path=tcb" in plan) == (not (bits == 2 and group == 32)), plan
    c = synth.affine_case(M, N, K, bits, group, dtype, seed=_seed("tcb", bits, group, dtype, M))
    y = run_affine(q, c)[0]
    ref, ad = oracle_affine(c)
    compare(y, ref, ad, dtype, what=f"tcb b{bits} g{group} {dtype} M{M}")


@pytest.mark.parametrize("cfg", [(4, -1, 1, 1), (4, -1, 8, 1), (4, -1, 1, 8), (4, -1, 2, 4), (4, -1, 4, 2),
                                 (4, -1, 3, 2), (4, -1, 6, 2), (4, -1, 4, 3), (4, -1, 12, 1), (4, -1, 3, 4)])
@pytest.mark.parametrize("bits", [2, 3, 5, 8])
def test_bulk_ring_block_shapes(q, ring, cfg, bits):
    q.qmv_force_config(*cfg)
    c = synth.affine_case(2, 333, 2048, bits, 64, "bf16", seed=_seed("tcbshape", cfg, bits), batch=2)
    assert "path=tcb" in q.qmv_describe_plan("affine", 2, 333, 2048, bits, 64, "bf16")
    y = run_affine(q, c)
    for b in range(2):
        ref, ad = oracle_affine(c, b=b)
        compare(y[b], ref, ad, "bf16", what=f"tcb shape {cfg} b{bits} batch{b}")


@pytest.mark.parametrize("bits", [3, 4])
@pytest.mark.parametrize("M", [1, 3])
def test_bulk_ring_persistent_row_blocks(q, ring, bits, M):
    """More row blocks than SMs: each block walks several row blocks and the
    ring runs across their boundaries; K = 5760 leaves a ragged last stage."""
    q.qmv_force_config(4, -1, 8, 1)
    N, K = 16 * 148 * 2 + 37, 5760
    c = synth.affine_case(M, N, K, bits, 64, "bf16", seed=_seed("tcbpers", bits, M))
    plan = q.qmv_describe_plan("affine", M, N, K, bits, 64, "bf16")
    assert "path=tcb" in plan and "grid=148 " in plan, plan
    y = run_affine(q, c)[0]
    rows = sorted(set(sample_rows(N, 96)) | {0, 15, 16, N - 38, N - 37, N - 1})
    ref, ad = oracle_affine(c, rows=rows)
    compare(y[:, rows], ref[:, rows], ad[:, rows], "bf16", what=f"tcb persistent b{bits} M{M}")


@pytest.mark.parametrize("bits", BITS)
def test_bulk_ring_tail_rows_bitwise_prefix(q, ring, bits):
    q.qmv_force_config(4, -1, 2, 1)            # 16-row tiles, K over 2 warps
    K = 2560
    big = synth.affine_case(1, 48, K, bits, 64, "bf16", seed=_seed("tcbtail", bits))
    yb = run_affine(q, big)[0]
    for n in (1, 5, 17, 33):
        small = dict(big, N=n, w=big["w"][:, :n].copy(), scales=big["scales"][:, :n].copy(),
                     biases=big["biases"][:, :n].copy())
        assert np.array_equal(run_affine(q, small)[0], yb[:, :n])


@pytest.mark.parametrize("bits,group,M", [(4, 64, 1), (4, 32, 8), (3, 128, 2), (8, 128, 1), (5, 64, 3)])
def test_bulk_ring_scales_in_or_out_of_ring(q, ring, bits, group, M):
    """Scales and biases ride in the ring when 16-byte aligned and read from
    global memory otherwise: the two give bitwise equal outputs."""
    q.qmv_force_config(4, -1, 4, 2)
    N, K = 300, 4096
    plan = q.qmv_describe_plan("affine", M, N, K, bits, group, "bf16")
    assert "path=tcb" in plan and "scale_ring=1" in plan, plan
    c = synth.affine_case(M, N, K, bits, group, "bf16", seed=_seed("tcbscale", bits, group, M), batch=2)
    y_in = run_affine(q, c)
    y_out = run_affine(q, c, s_offset=2)
    assert np.array_equal(y_in, y_out)
    for b in range(2):
        ref, ad = oracle_affine(c, b=b)
        compare(y_in[b], ref, ad, "bf16", what=f"tcb scales b{bits} g{group} M{M} batch{b}")


@pytest.mark.parametrize("N", [80, 16 * 148 + 5])
def test_bulk_ring_x_tiles(q, ring, N):
    """M=8, f32 x, K large enough that x is staged in several K tiles (and,
    with more row blocks than SMs, staged again for every row block)."""
    q.qmv_force_config(4, -1, 8, 1)
    K = 16384
    plan = q.qmv_describe_plan("affine", 8, N, K, 4, 32, "f32")
    assert "path=tcb" in plan and "tile_iters=128" not in plan, plan
    c = synth.affine_case(8, N, K, 4, 32, "f32", seed=_seed("tcbtile", N))
    y = run_affine(q, c)[0]
    rows = list(range(N)) if N <= 80 else sorted(set(sample_rows(N, 48)) | {N - 1})
    ref, ad = oracle_affine(c, rows=rows)
    compare(y[:, rows], ref[:, rows], ad[:, rows], "f32", what="tcb tiles")


# ------------------------------- CUDA cores + weight ring, one bf16 x row ----
@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("group", GROUPS)
@pytest.mark.parametrize("K", [1024, 5760])
def test_fma_ring_path_grid(q, ring, bits, group, K):
    """The CUDA-core ring kernel on every width and group (2-bit with group 32
    falls back: a 64-code unit would span two groups); K = 5760 leaves an odd
    number of super-blocks for most widths (a half-empty last step)."""
    q.qmv_force_config(6, -1, -1, -1)
    N = 100
    sb = 512 // bits if bits in (2, 4, 8) else 128       # codes per super-block
    if K % sb != 0:
        pytest.skip("K not a whole number of super-blocks")
    plan = q.qmv_describe_plan("affine", 1, N, K, bits, group, "bf16")
    assert ("path=tcf" in plan) == (not (bits == 2 and group == 32)), plan
    c = synth.affine_case(1, N, K, bits, group, "bf16", seed=_seed("tcf", bits, group, K))
    y = run_affine(q, c)[0]
    ref, ad = oracle_affine(c)
    compare(y, ref, ad, "bf16", what=f"tcf b{bits} g{group} K{K}")


@pytest.mark.parametrize("cfg", [(6, -1, 1, 8), (6, -1, 2, 4), (6, -1, 4, 2), (6, -1, 8, 1), (6, -1, 1, 12),
                                 (6, -1, 3, 4), (6, -1, 6, 2), (6, -1, 12, 1), (6, -1, 2, 6), (6, -1, 4, 3)])
@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 8])
def test_fma_ring_block_shapes(q, ring, cfg, bits):
    unit_bytes = 16 if bits in (2, 4, 8) else 4 * bits
    if 2 * cfg[2] * 4 * unit_bytes > 2048:
        pytest.skip("a stage of 2 * wk super-blocks exceeds one tensor-copy box (256 x 8 bytes)")
    q.qmv_force_config(*cfg)
    c = synth.affine_case(1, 333, 2048, bits, 64, "bf16", seed=_seed("tcfshape", cfg, bits), batch=2)
    assert "path=tcf" in q.qmv_describe_plan("affine", 1, 333, 2048, bits, 64, "bf16")
    y = run_affine(q, c)
    for b in range(2):
        ref, ad = oracle_affine(c, b=b)
        compare(y[b], ref, ad, "bf16", what=f"tcf shape {cfg} b{bits} batch{b}")


@pytest.mark.parametrize("bits", [3, 4])
def test_fma_ring_persistent_row_blocks(q, ring, bits):
    """More row blocks than SMs, a ragged last stage and a ragged last row block."""
    q.qmv_force_config(6, -1, 8, 1)
    N, K = 16 * 148 * 2 + 37, 5760
    c = synth.affine_case(1, N, K, bits, 64, "bf16", seed=_seed("tcfpers", bits))
    plan = q.qmv_describe_plan("affine", 1, N, K, bits, 64, "bf16")
    assert "path=tcf" in plan and "grid=148 " in plan, plan
    y = run_affine(q, c)[0]
    rows = sorted(set(sample_rows(N, 96)) | {0, 15, 16, N - 38, N - 37, N - 1})
    ref, ad = oracle_affine(c, rows=rows)
    compare(y[:, rows], ref[:, rows], ad[:, rows], "bf16", what=f"tcf persistent b{bits}")


@pytest.mark.parametrize("bits", BITS)
def test_fma_ring_tail_rows_bitwise_prefix(q, ring, bits):
    q.qmv_force_config(6, -1, 4, 2)
    K = 2560
    big = synth.affine_case(1, 48, K, bits, 64, "bf16", seed=_seed("tcftail", bits))
    yb = run_affine(q, big)[0]
    for n in (1, 5, 17, 33):
        small = dict(big, N=n, w=big["w"][:, :n].copy(), scales=big["scales"][:, :n].copy(),
                     biases=big["biases"][:, :n].copy())
        assert np.array_equal(run_affine(q, small)[0], yb[:, :n])


@pytest.mark.parametrize("bits,group", [(4, 64), (4, 32), (3, 128), (8, 128), (5, 64), (2, 128)])
def test_fma_ring_scales_in_or_out_of_ring(q, ring, bits, group):
    q.qmv_force_config(6, -1, 4, 2)
    N, K = 300, 4096
    plan = q.qmv_describe_plan("affine", 1, N, K, bits, group, "bf16")
    assert "path=tcf" in plan and "scale_ring=1" in plan, plan
    c = synth.affine_case(1, N, K, bits, group, "bf16", seed=_seed("tcfscale", bits, group), batch=2)
    y_in = run_affine(q, c)
    y_out = run_affine(q, c, s_offset=2)
    assert np.array_equal(y_in, y_out)
    for b in range(2):
        ref, ad = oracle_affine(c, b=b)
        compare(y_in[b], ref, ad, "bf16", what=f"tcf scales b{bits} g{group} batch{b}")


@pytest.mark.parametrize("N", [80, 16 * 148 + 5])
def test_fma_ring_x_tiles(q, ring, N):
    """K large enough that x is staged in several K tiles (and again for every
    row block when there are more row blocks than SMs)."""
    q.qmv_force_config(6, -1, 8, 1)
    K = 65536
    plan = q.qmv_describe_plan("affine", 1, N, K, 4, 64, "bf16")
    assert "path=tcf" in plan and "tile_iters=512" not in plan, plan
    c = synth.affine_case(1, N, K, 4, 64, "bf16", seed=_seed("tcftile", N))
    y = run_affine(q, c)[0]
    rows = list(range(N)) if N <= 80 else sorted(set(sample_rows(N, 48)) | {N - 1})
    ref, ad = oracle_affine(c, rows=rows)
    compare(y[:, rows], ref[:, rows], ad[:, rows], "bf16", what="tcf tiles")


# ----------------------------------------- few rows: the latency kernel ----
@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("M", [1, 3, 8])
@pytest.mark.parametrize("K", [480, 2560, 19200])
def test_direct_path_grid(q, bits, dtype, M, K):
    """N <= 64 rows: every width and dtype, one to two units per lane and
    (K = 19200, 600 units) units dequantized after the wait."""
    group = 32 if K == 480 else 64
    N = 17
    plan = q.qmv_describe_plan("affine", M, N, K, bits, group, dtype)
    assert "path=direct" in plan, plan
    c = synth.affine_case(M, N, K, bits, group, dtype, seed=_seed("direct", bits, dtype, M, K))
    y = run_affine(q, c)[0]
    ref, ad = oracle_affine(c)
    compare(y, ref, ad, dtype, what=f"direct b{bits} {dtype} M{M} K{K}")


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("M", [1, 4])
def test_direct_path_fp(q, mode, dtype, M):
    q.qmv_force_config(5, -1, -1, -1)
    c = synth.fp_case(M, 9, 2048, mode, dtype, seed=_seed("directfp", mode, dtype, M), batch=2)
    y = run_fp(q, c)
    for b in range(2):
        ref, ad = oracle_fp(c, b=b)
        compare(y[b], ref, ad, dtype, what=f"direct {mode} {dtype} M{M} batch{b}")


@pytest.mark.parametrize("bits", [3, 8])
def test_direct_path_misaligned_and_batched(q, bits):
    """4-byte aligned weights (no 16-byte loads) and batch 2 with a shared x."""
    c = synth.affine_case(2, 40, 2560, bits, 64, "bf16", seed=_seed("directmis", bits), batch=2)
    y = run_affine(q, c, w_offset=4, x_batched=False)
    for b in range(2):
        ref, ad = oracle_affine(c, b=b, x_batched=False)
        compare(y[b], ref, ad, "bf16", what=f"direct misaligned b{bits} batch{b}")


@pytest.mark.parametrize("bits", [3, 4, 8])
def test_cuda_core_path_grid(q, bits):
    """The CUDA-core kernel (wide and narrow chunks) stays covered."""
    for path in (1, 0):
        q.qmv_force_config(path, -1, -1, -1)
        c = synth.affine_case(3, 300, 1024, bits, 64, "f16", seed=_seed("cc", bits, path))
        y = run_affine(q, c)[0]
        ref, ad = oracle_affine(c)
        compare(y, ref, ad, "f16", what=f"cuda-core path{path} b{bits}")
