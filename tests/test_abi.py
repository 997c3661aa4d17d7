"""C ABI checks that need no GPU: the library loads, exports every function
include/qmv.h declares, and rejects bad arguments on the host with the status
the header documents (no kernel is launched for any of these calls)."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

import weight_quantized_matrix_b200 as q

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
EINVAL, EUNSUP, EALIGN = -1, -2, -3


def _declared():
    names = set()
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(qmv_\w+)\s*\(", src, flags=re.M))
    return sorted(names)


def test_header_declares_entry_points():
    names = _declared()
    for must in ("qmv_affine", "qmv_fp", "qmv_affine_batched", "qmv_fp_batched",
                 "qmv_dequant_affine_f32", "qmv_dequant_fp_f32", "qmv_status_string"):
        assert must in names


@pytest.mark.parametrize("name", _declared())
def test_library_exports(name):
    lib = ctypes.CDLL(q.LIB_PATH)
    assert hasattr(lib, name), name


L = q.lib()
FAKE = 1 << 20          # an aligned fake address: validation rejects before any use


def aff(**kw):
    a = dict(x=FAKE, w=FAKE, s=FAKE, b=FAKE, y=FAKE, M=1, N=8, K=128, bits=4, g=64, dt=2, st=None)
    a.update(kw)
    return L.qmv_affine(a["x"], a["w"], a["s"], a["b"], a["y"], a["M"], a["N"], a["K"], a["bits"], a["g"],
                        a["dt"], a["st"])


def fp(**kw):
    a = dict(x=FAKE, w=FAKE, s=FAKE, gs=None, y=FAKE, M=1, N=8, K=128, mode=0, dt=2, st=None)
    a.update(kw)
    return L.qmv_fp(a["x"], a["w"], a["s"], a["gs"], a["y"], a["M"], a["N"], a["K"], a["mode"], a["dt"], a["st"])


@pytest.mark.parametrize("bits", [0, 1, 7, 9, 16])
def test_bad_bits(bits):
    assert aff(bits=bits) == EUNSUP


@pytest.mark.parametrize("g", [0, 16, 48, 256])
def test_bad_group(g):
    assert aff(g=g) == EUNSUP


def test_k_not_multiple_of_group():
    assert aff(K=96, g=64) == EINVAL


def test_negative_sizes():
    assert aff(M=-1) == EINVAL
    assert aff(N=-1) == EINVAL
    assert aff(K=-64) == EINVAL


def test_m_above_max():
    assert aff(M=9) == EUNSUP


def test_bad_dtype():
    assert aff(dt=3) == EUNSUP
    assert fp(dt=-1) == EUNSUP


def test_null_pointers():
    for k in ("x", "w", "s", "b", "y"):
        assert aff(**{k: None}) == EINVAL, k


def test_misaligned_pointers():
    assert aff(w=FAKE + 2) == EALIGN          # w_packed needs 4 bytes
    assert aff(x=FAKE + 1) == EALIGN          # bf16 elements
    assert aff(s=FAKE + 1) == EALIGN
    assert aff(y=FAKE + 1, dt=0) == EALIGN


def test_empty_is_noop_without_launch():
    assert aff(M=0) == 0
    assert aff(N=0) == 0
    assert aff(M=0, x=None, w=None, s=None, b=None) == 0


def test_fp_validation():
    assert fp(mode=3) == EUNSUP
    assert fp(mode=1, gs=None) == EINVAL           # NVFP4 needs the global scale
    assert fp(mode=0, gs=FAKE) == EINVAL           # MX modes take none
    assert fp(mode=0, K=48) == EINVAL
    assert fp(mode=2, K=40) == EINVAL
    assert fp(mode=1, gs=FAKE, K=40) == EINVAL     # not a multiple of the 16 block
    assert fp(mode=1, gs=FAKE + 2) == EALIGN
    # (K = 48 is a valid NVFP4 shape, with a 16-code tail block: the GPU tests run it)


def bs(**kw):
    a = dict(x=FAKE, w=FAKE, s=FAKE, gs=None, y=FAKE, M=1, N=8, K=128, fmt=4, dt=2, st=None)
    a.update(kw)
    return L.qmv_block_scaled(a["x"], a["w"], a["s"], a["gs"], a["y"], a["M"], a["N"], a["K"], a["fmt"], a["dt"],
                              a["st"])


def test_block_scaled_validation_before_any_launch():
    F = q.FORMATS
    assert bs(fmt=-1) == EUNSUP and bs(fmt=30) == EUNSUP
    assert bs(fmt=F["nvfp4"]) == EINVAL                  # NVFP4 needs its global
    assert bs(fmt=F["nvfp4"], gs=FAKE + 2) == EALIGN
    assert bs(fmt=F["nvfp8"], gs=FAKE) == EINVAL         # no global for the rest
    assert bs(fmt=F["nvfp8"], K=40) == EINVAL            # not a multiple of the 16 block
    assert bs(fmt=F["fp4"], K=48) == EINVAL              # blocks of 32
    assert bs(fmt=F["int4"], K=96) == EINVAL             # groups of 64
    assert bs(fmt=F["nvfp8"], s=FAKE + 2) == EALIGN      # FP32 scales
    assert bs(fmt=F["int4_f16"], s=FAKE + 1) == EALIGN   # FP16 scales
    assert bs(fmt=F["int8"], w=FAKE + 2) == EALIGN
    assert bs(fmt=F["int3"], M=9) == EUNSUP
    assert bs(fmt=F["mxint5"], x=None) == EINVAL
    assert bs(fmt=F["fp8_e5m2"], M=0) == 0 and bs(fmt=F["fp8_e5m2"], N=0) == 0
    assert L.qmv_block_scaled_batched(FAKE, FAKE, FAKE, None, FAKE, 1, 8, 128, 4, 2, 0, 1, None) == EINVAL
    out = FAKE
    assert L.qmv_dequant_block_scaled_f32(FAKE, FAKE, None, out + 4, 8, 128, 4, None) == EALIGN
    assert L.qmv_dequant_block_scaled_f32(FAKE, FAKE, None, out, 8, 128, 31, None) == EUNSUP
    assert L.qmv_dequant_block_scaled_f32(FAKE, FAKE, None, out, 0, 128, 4, None) == 0


def test_format_info_of_every_format():
    """The C table against the pages' Track-1 layout: bits per code, block,
    scale bytes, global."""
    want = {"nvfp4": (4, 16, 1, True), "mxfp4": (4, 32, 1, False), "mxfp8_e4m3": (8, 32, 1, False),
            "mxfp8_e5m2": (8, 32, 1, False), "nvfp8": (8, 16, 4, False), "fp4": (4, 32, 4, False),
            "fp8_e4m3": (8, 32, 4, False), "fp8_e5m2": (8, 32, 4, False), "nvfp8_f16": (8, 16, 2, False),
            "fp4_f16": (4, 32, 2, False), "fp8_e4m3_f16": (8, 32, 2, False), "fp8_e5m2_f16": (8, 32, 2, False)}
    for b in (2, 3, 4, 5, 6, 8):
        want[f"int{b}"] = (b, 64, 4, False)
        want[f"mxint{b}"] = (b, 32, 1, False)
        want[f"int{b}_f16"] = (b, 64, 2, False)
    assert set(want) == set(q.FORMATS) and len(want) == 30
    for name, (bits, blk, sb, g) in want.items():
        assert q.qmv_format_info(name) == {"element_bits": bits, "block": blk, "scale_bytes": sb,
                                          "has_global": g}, name
    with pytest.raises(q.QmvError):
        q.qmv_format_info(30)


def test_block_scaled_plans():
    """Every format plans on the few-rows or the row-tiled kernel, never on
    the affine-only kernels; the FP formats with FP32 / FP16 block scales also
    on the weight ring for one large bf16 x row (scales in the ring), the
    others reach it only when forced (path 6)."""
    for name in q.FORMATS:
        fp = not name.startswith(("int", "mxint"))
        wide_scales = q.qmv_format_info(name)["scale_bytes"] >= 2
        for (M, N, K) in [(1, 4, 1024), (1, 4096, 4096), (8, 14336, 4096), (1, 14336, 4096)]:
            plan = q.qmv_describe_plan(name, M, N, K, dtype="bf16")
            bits = q.qmv_format_info(name)["element_bits"]
            ring_ok = fp and wide_scales and M == 1 and N * K * bits / 8 >= 10 * 1024 * 1024
            assert plan.split()[0] in ("path=direct", "path=wide", "path=narrow") + (("path=tcf",) if ring_ok else ()), \
                (name, plan)
            if ring_ok:
                assert "path=tcf" in plan and "scale_ring=1" in plan, (name, plan)
        q.qmv_force_config(6, -1, -1, -1)
        try:
            ring = q.qmv_describe_plan(name, 1, 14336, 4096, dtype="bf16")
            assert ("path=tcf" in ring) == fp, (name, ring)
            assert "path=tcf" not in q.qmv_describe_plan(name, 1, 14336, 4096, dtype="f16"), name
        finally:
            q.qmv_force_config()


def _tcg_fields(plan):
    """The per-group ring's launch fields from a plan (after any qmm chunk prefix)."""
    tail = plan[plan.index("path=tcg "):]
    return {k: v for k, v in (kv.split("=", 1) for kv in tail.split() if "=" in kv)}


def test_per_group_ring_plans():
    """4-bit affine with bf16 / f16 x takes the per-group tensor-core ring from
    8 x rows (from 4 at N >= 20000), and qmm in chunks of 16 / 32 rows; other
    widths, f32 x, K not a multiple of 8 groups and unaligned weights go
    elsewhere.  Its shapes: wk in {1, 2, 4, 8}, 8..16 consumer warps plus the
    producer, one persistent block per row block up to one per SM, shared
    memory within the limit."""
    plan = lambda M, N, K, **kw: q.qmv_describe_plan("affine", M, N, K, bits=kw.pop("bits", 4),
                                                     group_size=kw.pop("g", 64), **kw)
    for dt in ("bf16", "f16"):
        for g in (32, 64, 128):
            assert "path=tcg " in plan(8, 4096, 4096, g=g, dtype=dt)
    assert "path=tcg " in plan(4, 28672, 4096)
    assert "path=tcg " not in plan(4, 4096, 4096)
    assert "path=tcg " not in plan(2, 28672, 4096)
    for bits in (2, 3, 5, 6, 8):
        assert "path=tcg " not in plan(8, 4096, 4096, bits=bits)
    assert "path=tcg " not in plan(8, 4096, 4096, dtype="f32")
    assert "path=tcg " not in plan(8, 4096, 1088)                  # 17 groups
    assert "path=tcg " not in plan(8, 4096, 4096, w_align16=False)
    assert plan(16, 4096, 4096).startswith("path=chunked16 chunks=1 path=tcg ")
    assert plan(33, 4096, 4096).startswith("path=chunked32 chunks=2 path=tcg ")
    assert plan(64, 28672, 4096).startswith("path=chunked32 chunks=2 path=tcg ")
    sms = 148
    for N, K in [(6144, 4096), (4096, 4096), (28672, 4096), (4096, 14336), (16384, 16384), (100, 1024), (2500, 14336)]:
        for M in (8, 16, 32):
            f = _tcg_fields(plan(M, N, K))
            wk, wr = int(f["warps_k"]), int(f["warps_rows"])
            assert wk in (1, 2, 4, 8) and 8 <= wk * wr <= 16, (N, K, M, f)
            assert int(f["block"]) == 32 * (wk * wr + 1), (N, K, M, f)
            assert int(f["grid"]) == min(-(-N // (16 * wr)), sms), (N, K, M, f)
            assert int(f["smem"]) <= 227 * 1024, (N, K, M, f)
            assert int(f["maxm"]) == (8 if M <= 8 else 16 if M <= 16 else 32), (N, K, M, f)
    # the tall layer shape: one row block per SM, 13 row tiles of 16 on 138 SMs
    f = _tcg_fields(plan(8, 28672, 4096))
    assert (f["warps_k"], f["warps_rows"], f["grid"]) == ("1", "13", "138"), f


def test_batched_validation():
    assert L.qmv_affine_batched(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 8, 128, 4, 64, 2, 0, 1, None) == EINVAL
    assert L.qmv_affine_batched(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 8, 128, 4, 64, 2, 70000, 1, None) == EINVAL
    assert L.qmv_affine_batched(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 8, 128, 4, 64, 2, 2, 3, None) == EINVAL
    assert L.qmv_fp_batched(FAKE, FAKE, FAKE, None, FAKE, 1, 8, 128, 0, 2, 0, 1, None) == EINVAL


def test_dequant_validation():
    assert L.qmv_dequant_affine_f32(FAKE, FAKE, FAKE, FAKE, 8, 128, 7, 64, 2, None) == EUNSUP
    assert L.qmv_dequant_affine_f32(FAKE, FAKE, FAKE, FAKE, 8, 100, 4, 64, 2, None) == EINVAL
    assert L.qmv_dequant_affine_f32(FAKE, FAKE, FAKE, FAKE + 4, 8, 128, 4, 64, 2, None) == EALIGN
    assert L.qmv_dequant_affine_f32(FAKE, FAKE, FAKE, FAKE, 0, 128, 4, 64, 2, None) == 0
    assert L.qmv_dequant_fp_f32(FAKE, FAKE, None, FAKE, 8, 128, 1, None) == EINVAL


def test_status_strings():
    for st in (0, -1, -2, -3, -4):
        assert q.qmv_status_string(st)
    assert q.qmv_status_string(-99) == "unknown status"


def test_python_binding_raises():
    with pytest.raises(q.QmvError) as e:
        q.qmv_affine(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 8, 128, 7, 64, "bf16", stream=0)
    assert e.value.status == EUNSUP


def test_plan_no_n_cliff():
    """Any N gets a plan (no N % 8 generic fallback): N <= 64 the latency
    kernel, larger N the row-tiled kernels, whatever N % 8 is."""
    for n in (1, 3, 5, 7, 8, 9, 12, 17, 64, 65, 512):
        s = q.qmv_describe_plan("affine", 1, n, 2560, bits=8, group_size=64)
        assert "path=direct" in s, (n, s)
    for n in (513, 4095, 4096, 4097):
        s = q.qmv_describe_plan("affine", 1, n, 2560, bits=8, group_size=64)
        assert "path=wide" in s, (n, s)
    # few output rows: the latency kernel, for every format
    assert "path=direct" in q.qmv_describe_plan("affine", 1, 64, 96, bits=3, group_size=32)
    assert "path=direct" in q.qmv_describe_plan("affine", 1, 64, 4096, bits=4, group_size=32, w_align16=False)
    assert "path=direct" in q.qmv_describe_plan("mxfp4", 2, 12, 4096)
    assert "path=direct" not in q.qmv_describe_plan("affine", 1, 513, 4096, bits=4, group_size=64)
    assert "path=direct" not in q.qmv_describe_plan("affine", 3, 65, 4096, bits=4, group_size=64)
    # 3-bit tensor-core units are 12 bytes: 4-byte alignment is enough
    assert "path=tc" in q.qmv_describe_plan("affine", 4, 100, 4096, bits=3, group_size=32, w_align16=False)


def test_fast_extension_forwards_status():
    """The CPython entry points are the in-tree extension over the same
    library and return the C ABI's status unchanged."""
    assert os.path.dirname(q._fast.__file__) == os.path.dirname(q.LIB_PATH.rsplit("/lib/", 1)[0] + "/")
    assert q._fast.affine(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 8, 128, 7, 64, 2, 1, 1, 0) == EUNSUP
    assert q._fast.affine(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 8, 96, 4, 64, 2, 1, 1, 0) == EINVAL
    assert q._fast.fp(FAKE, FAKE, FAKE, None, FAKE, 1, 8, 128, 1, 2, 1, 1, 0) == EINVAL
    assert q._fast.affine(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 8, 128, 4, 64, 2, 1, 1, 0) == 0
    with pytest.raises(TypeError):
        q._fast.affine(FAKE)
    # sizes beyond a C int raise instead of being narrowed (2^32 + 8 would wrap to 8)
    with pytest.raises(OverflowError):
        q._fast.affine(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2 ** 32 + 8, 128, 4, 64, 2, 1, 1, 0)
    with pytest.raises(OverflowError):
        q._fast.fp(FAKE, FAKE, FAKE, None, FAKE, 1, 8, -(2 ** 31) - 1, 1, 2, 1, 1, 0)


def test_build_module_loads_without_the_library(tmp_path):
    """The build script runs on a fresh checkout, where libqmv.so does not
    exist yet: loading it by path must not import the package (whose import
    needs the library)."""
    import subprocess
    import sys
    code = (
        "import importlib.util, sys\n"
        f"spec = importlib.util.spec_from_file_location('b', {str(ROOT)!r} + '/weight_quantized_matrix_b200/build_lib.py')\n"
        "m = importlib.util.module_from_spec(spec); spec.loader.exec_module(m)\n"
        "assert callable(m.build) and callable(m.build_ext)\n"
        "assert 'weight_quantized_matrix_b200' not in sys.modules\n"
    )
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=str(tmp_path))
    assert r.returncode == 0, r.stderr


def test_quantize_validation_before_any_launch():
    """Argument errors of the quantizer come back as statuses before any CUDA
    call (host-side checks; fake device pointers are never dereferenced)."""
    F = FAKE
    assert L.qmv_quantize_affine(F, F, F, F, 8, 128, 7, 64, 2, None) == EUNSUP       # bits
    assert L.qmv_quantize_affine(F, F, F, F, 8, 128, 4, 48, 2, None) == EUNSUP       # group
    assert L.qmv_quantize_affine(F, F, F, F, 8, 128, 4, 64, 5, None) == EUNSUP       # dtype
    assert L.qmv_quantize_affine(F, F, F, F, 8, 100, 4, 64, 2, None) == EINVAL       # K % group
    assert L.qmv_quantize_affine(F, F, F, F, -1, 128, 4, 64, 2, None) == EINVAL      # N < 0
    assert L.qmv_quantize_affine(None, F, F, F, 8, 128, 4, 64, 2, None) == EINVAL    # null
    assert L.qmv_quantize_affine(F + 1, F, F, F, 8, 128, 4, 64, 2, None) == EALIGN   # w alignment
    assert L.qmv_quantize_affine(F, F + 2, F, F, 8, 128, 4, 64, 2, None) == EALIGN   # packed alignment
    assert L.qmv_quantize_affine(F, F, F, F, 0, 128, 4, 64, 2, None) == 0            # empty: nothing to do


def test_qvm_validation_before_any_launch():
    """qvm argument errors come back as statuses before any CUDA call."""
    F = FAKE

    def qvm(x=F, w=F, s=F, b=F, y=F, M=1, N=128, K=64, bits=4, g=64, dt=2, ws=None):
        return L.qmv_qvm_affine(x, w, s, b, y, M, N, K, bits, g, dt, ws, None)

    assert qvm(bits=7) == EUNSUP
    assert qvm(g=48) == EUNSUP
    assert qvm(dt=5) == EUNSUP
    assert qvm(N=96) == EINVAL                  # N % group
    assert qvm(M=9) == EINVAL                   # M > 8
    assert qvm(K=-1) == EINVAL
    assert qvm(w=None) == EINVAL
    assert qvm(y=None) == EINVAL
    assert qvm(w=F + 4) == EALIGN               # w_packed needs 16 bytes
    assert qvm(x=F + 1) == EALIGN
    assert qvm(ws=F + 8) == EALIGN
    assert qvm(M=0) == 0 and qvm(N=0) == 0      # empty: nothing to do


def test_qvm_workspace_size():
    """fp32 [M, N] partial sums (rounded to 256 bytes) plus one counter per
    (1024-column tile, x row), also rounded to 256 bytes."""
    assert q.qmv_qvm_workspace_bytes(1, 16384) == 65536 + 256
    assert q.qmv_qvm_workspace_bytes(8, 4096) == 131072 + 256
    assert q.qmv_qvm_workspace_bytes(3, 32) == 512 + 256
    assert q.qmv_qvm_workspace_bytes(-1, 32) == 0


def test_qmm_validation_before_any_launch():
    F = FAKE

    def qmm(x=F, w=F, s=F, b=F, y=F, M=16, N=128, K=128, bits=4, g=64, dt=2):
        return L.qmv_qmm_affine(x, w, s, b, y, M, N, K, bits, g, dt, None)

    assert qmm(M=65) == EINVAL
    assert qmm(M=-1) == EINVAL
    assert qmm(bits=7) == EUNSUP
    assert qmm(K=100) == EINVAL
    assert qmm(b=None) == EINVAL
    assert qmm(x=F + 1) == EALIGN
    assert qmm(M=0) == 0 and qmm(N=0) == 0


def test_gather_validation_before_any_launch():
    F = FAKE

    def g(x=F, w=F, s=F, b=F, ids=F, y=F, M=1, N=64, K=128, bits=4, gs=64, dt=2, T=4, E=8, xb=1):
        return L.qmv_affine_gather(x, w, s, b, ids, y, M, N, K, bits, gs, dt, T, E, xb, None)

    assert g(ids=None) == EINVAL
    assert g(ids=F + 2) == EALIGN
    assert g(T=0) == EINVAL and g(T=65536) == EINVAL
    assert g(E=0) == EINVAL
    assert g(xb=2) == EINVAL
    assert g(bits=7) == EUNSUP
    assert g(M=0) == 0


def test_quantize_fp_validation_before_any_launch():
    F = FAKE

    def qf(w=F, wq=F, s=F, g=None, N=8, K=128, mode=0, dt=2):
        return L.qmv_quantize_fp(w, wq, s, g, N, K, mode, dt, None)

    assert qf(mode=5) == EUNSUP
    assert qf(dt=7) == EUNSUP
    assert qf(K=48) == EINVAL                   # MX blocks of 32
    assert qf(mode=1, K=40, g=F) == EINVAL      # NVFP4 blocks of 16
    assert qf(mode=1) == EINVAL                 # NVFP4 needs the global scale
    assert qf(g=F) == EINVAL                    # MX takes none
    assert qf(w=None) == EINVAL
    assert qf(w=F + 1) == EALIGN
    assert qf(N=0) == 0


def test_swiglu_validation_before_any_launch():
    F = FAKE

    def sw(x=F, wg=F, sg=F, bg=F, wu=F, su=F, bu=F, rw=None, y=F, M=1, N=64, K=128, bits=4, gs=64, dt=2,
           clamp=0.0):
        return L.qmv_affine_swiglu(x, wg, sg, bg, wu, su, bu, rw, y, M, N, K, bits, gs, dt, ctypes.c_float(clamp),
                                   None)

    assert sw(bits=7) == EUNSUP and sw(gs=16) == EUNSUP
    assert sw(K=100) == EINVAL
    assert sw(clamp=-1.0) == EINVAL and sw(clamp=float("nan")) == EINVAL
    assert sw(wu=None) == EINVAL and sw(bu=None) == EINVAL and sw(bg=None) == EINVAL
    assert sw(wu=F + 2) == EALIGN and sw(su=F + 1) == EALIGN and sw(rw=F + 2) == EALIGN
    assert sw(M=9) == EUNSUP
    assert sw(M=-1) == EINVAL
    assert sw(M=0) == 0 and sw(N=0) == 0


def test_qkv_and_rms_norm_validation_before_any_launch():
    F = FAKE

    def qkv(x=F, wq=F, wk=F, wv=F, y=F, M=1, Nq=64, Nkv=16, K=128, bits=4, gs=64, dt=2):
        return L.qmv_affine_qkv(x, wq, F, F, wk, F, F, wv, F, F, y, M, Nq, Nkv, K, bits, gs, dt, None)

    assert qkv(bits=7) == EUNSUP and qkv(K=100) == EINVAL and qkv(Nkv=-1) == EINVAL
    assert qkv(wk=None) == EINVAL and qkv(wv=F + 2) == EALIGN
    assert qkv(M=9) == EUNSUP and qkv(M=0) == 0 and qkv(Nq=0, Nkv=0) == 0

    def rms(x=F, g=F, eps=1e-6, w=F, s=F, b=F, y=F, M=1, N=64, K=128, bits=4, gs=64, dt=2):
        return L.qmv_affine_rms_norm(x, g, ctypes.c_float(eps), w, s, b, y, M, N, K, bits, gs, dt, None)

    assert rms(eps=-1.0) == EINVAL and rms(eps=float("nan")) == EINVAL and rms(eps=float("inf")) == EINVAL
    assert rms(g=None) == EINVAL and rms(g=F + 1) == EALIGN and rms(bits=1) == EUNSUP
    assert rms(M=0) == 0


@pytest.mark.parametrize("name", _declared())
def test_python_binding_has_every_entry_point(name):
    """The binding exposes each C-ABI entry point under the same name."""
    assert callable(getattr(q, name, None)), name
