"""fp64 CPU oracle for the weight-quantized matrix-vector product (qmv).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` leg of ``bench.py`` may import this
package.  The CUDA library never loads it and shares no code with it.

The arithmetic lives in ``qmv_oracle.c`` (plain C, fp64); this module only
compiles it with gcc and marshals numpy arrays through ctypes.  Calls release
the GIL, so a thread pool over row ranges runs them in parallel
(``threads`` argument).

Page citations for each function are in the C file: the MLX
``quantized_nax.h`` source page (pack geometry, LSB-first codes,
``w = scale * q + bias``), the wh-iron kernel-op coverage audit (the 30 Track 1
formats: E2M1 / E4M3 / E5M2 / signed-int elements with E8M0, E4M3, FP32 or
FP16 block scales) and the MLX pull request adding
``affine_qmv_fast_rows`` (fp32-widened sum(x)).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qmv_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F32, F16, BF16 = 0, 1, 2
MXFP4, NVFP4, MXFP8 = 0, 1, 2
DTYPE_CODES = {"f32": F32, "f16": F16, "bf16": BF16}
FP_MODES = {"mxfp4": MXFP4, "nvfp4": NVFP4, "mxfp8": MXFP8}

# Track-1 symmetric block-scaled formats (wh-iron kernel-op coverage audit,
# "Quantization precision coverage", Track 1 table): name -> (element, element
# bits, block along K, block-scale type, FP32 global).  The integer rows: int2..8
# with an FP32 scale per group of 64, mxint2..8 with an E8M0 scale per 32; every
# FP32-scaled format has an FP16-scale twin "<name>_f16" (same element and
# block).  30 formats.
_ELEM_CODES = {"e2m1": 0, "e4m3": 1, "e5m2": 2, "int": 3}
_SCALE_CODES = {"e8m0": 0, "e4m3": 1, "f32": 2, "f16": 3}
TRACK1 = {
    "nvfp4": ("e2m1", 4, 16, "e4m3", True),
    "mxfp4": ("e2m1", 4, 32, "e8m0", False),
    "mxfp8_e4m3": ("e4m3", 8, 32, "e8m0", False),
    "mxfp8_e5m2": ("e5m2", 8, 32, "e8m0", False),
    "nvfp8": ("e4m3", 8, 16, "f32", False),
    "fp4": ("e2m1", 4, 32, "f32", False),
    "fp8_e4m3": ("e4m3", 8, 32, "f32", False),
    "fp8_e5m2": ("e5m2", 8, 32, "f32", False),
}
for _b in (2, 3, 4, 5, 6, 8):
    TRACK1[f"int{_b}"] = ("int", _b, 64, "f32", False)
for _b in (2, 3, 4, 5, 6, 8):
    TRACK1[f"mxint{_b}"] = ("int", _b, 32, "e8m0", False)
for _name in [n for n, v in TRACK1.items() if v[3] == "f32"]:
    _e, _bb, _blk, _, _g = TRACK1[_name]
    TRACK1[_name + "_f16"] = (_e, _bb, _blk, "f16", _g)


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` next to its source with gcc (no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
             "-ffp-contract=off", _SRC, "-o", _LIB, "-lm"])
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        ll, i, p, d, f, u = (ctypes.c_longlong, ctypes.c_int, ctypes.c_void_p,
                             ctypes.c_double, ctypes.c_float, ctypes.c_uint32)
        L.oracle_f16_value.argtypes = [u]; L.oracle_f16_value.restype = d
        L.oracle_bf16_value.argtypes = [u]; L.oracle_bf16_value.restype = d
        L.oracle_pack_factor.argtypes = [i]; L.oracle_pack_factor.restype = i
        L.oracle_bytes_per_pack.argtypes = [i]; L.oracle_bytes_per_pack.restype = i
        L.oracle_row_bytes.argtypes = [ll, i]; L.oracle_row_bytes.restype = ll
        L.oracle_affine_code.argtypes = [p, ll, i]; L.oracle_affine_code.restype = u
        L.oracle_e2m1.argtypes = [u]; L.oracle_e2m1.restype = d
        L.oracle_e4m3.argtypes = [u]; L.oracle_e4m3.restype = d
        L.oracle_e8m0.argtypes = [u]; L.oracle_e8m0.restype = d
        L.oracle_round_f32_sum.argtypes = [d, d]; L.oracle_round_f32_sum.restype = f
        L.oracle_dequant_affine_f32.argtypes = [p, p, p, p, ll, ll, i, i, i, ll, ll]
        L.oracle_dequant_affine_f32.restype = None
        L.oracle_dequant_fp_f32.argtypes = [p, p, f, p, ll, ll, i, ll, ll]
        L.oracle_dequant_fp_f32.restype = None
        L.oracle_qmv_affine.argtypes = [p, p, p, p, p, p, ll, ll, ll, i, i, i, ll, ll]
        L.oracle_qmv_affine.restype = None
        L.oracle_qmv_fp.argtypes = [p, p, p, f, p, p, ll, ll, ll, i, i, ll, ll]
        L.oracle_qvm_affine.argtypes = [p, p, p, p, p, p, ll, ll, ll, i, i, i, ll, ll]
        L.oracle_qvm_affine.restype = None
        L.oracle_qmv_fp.restype = None
        L.oracle_f32_to_bf16.argtypes = [f]; L.oracle_f32_to_bf16.restype = u
        L.oracle_f32_to_f16.argtypes = [f]; L.oracle_f32_to_f16.restype = u
        L.oracle_quantize_affine.argtypes = [p, p, p, p, ll, ll, i, i, i, ll, ll]
        L.oracle_quantize_fp.argtypes = [p, p, p, f, ll, ll, i, i, ll, ll]
        L.oracle_quantize_fp.restype = None
        L.oracle_nearest_e2m1.argtypes = [d]; L.oracle_nearest_e2m1.restype = u
        L.oracle_nearest_e4m3.argtypes = [d]; L.oracle_nearest_e4m3.restype = u
        L.oracle_quantize_affine.restype = None
        L.oracle_dequant_affine_f64.argtypes = [p, p, p, p, ll, ll, i, i, i, ll, ll]
        L.oracle_dequant_affine_f64.restype = None
        L.oracle_e5m2.argtypes = [u]; L.oracle_e5m2.restype = d
        L.oracle_sint.argtypes = [u, i]; L.oracle_sint.restype = d
        L.oracle_block_scale.argtypes = [p, ll, i]; L.oracle_block_scale.restype = d
        L.oracle_dequant_block_scaled_f32.argtypes = [p, p, i, f, p, ll, ll, i, i, i, i, ll, ll]
        L.oracle_dequant_block_scaled_f32.restype = None
        L.oracle_qmv_block_scaled.argtypes = [p, p, p, i, f, p, p, ll, ll, ll, i, i, i, i, i, ll, ll]
        L.oracle_qmv_block_scaled.restype = None
        _lib = L
    return _lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


def _ranges(rows, threads):
    """Split a row list/range into contiguous (n0, n1) runs, then into chunks."""
    rows = list(rows)
    runs, start = [], None
    for i, r in enumerate(rows):
        if start is None:
            start, prev = r, r
        elif r == prev + 1:
            prev = r
        else:
            runs.append((start, prev + 1)); start, prev = r, r
    if start is not None:
        runs.append((start, prev + 1))
    out = []
    for a, b in runs:
        step = max(1, (b - a + threads - 1) // threads)
        out += [(s, min(b, s + step)) for s in range(a, b, step)]
    return out


def _run(fn, ranges, threads):
    if threads <= 1 or len(ranges) <= 1:
        for a, b in ranges:
            fn(a, b)
        return
    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(lambda r: fn(*r), ranges))


# ---- scalar codecs (pinned in tests/test_oracle_pins.py) -------------------
def f16_value(h): return lib().oracle_f16_value(int(h))
def bf16_value(h): return lib().oracle_bf16_value(int(h))
def pack_factor(bits): return lib().oracle_pack_factor(bits)
def bytes_per_pack(bits): return lib().oracle_bytes_per_pack(bits)
def row_bytes(K, bits): return lib().oracle_row_bytes(K, bits)
def e2m1(c): return lib().oracle_e2m1(int(c))
def e4m3(c): return lib().oracle_e4m3(int(c))
def e8m0(e): return lib().oracle_e8m0(int(e))
def e5m2(c): return lib().oracle_e5m2(int(c))
def sint(q, bits): return lib().oracle_sint(int(q), int(bits))
def round_f32_sum(a, b): return lib().oracle_round_f32_sum(float(a), float(b))
def f32_to_bf16(v): return lib().oracle_f32_to_bf16(float(v))
def f32_to_f16(v): return lib().oracle_f32_to_f16(float(v))


def affine_codes(row: np.ndarray, K: int, bits: int) -> np.ndarray:
    """All K codes of one packed row (uint8 array)."""
    row = np.ascontiguousarray(row, dtype=np.uint8)
    L = lib()
    return np.array([L.oracle_affine_code(_ptr(row), k, bits) for k in range(K)], dtype=np.uint32)


# ---- dequantization (fp32 out) ----------------------------------------------
def dequant_affine_f32(w, scales, biases, N, K, bits, group, dtype, rows=None, threads=1):
    out = np.zeros((N, K), dtype=np.float32)
    L = lib()
    fn = lambda a, b: L.oracle_dequant_affine_f32(_ptr(w), _ptr(scales), _ptr(biases), _ptr(out),
                                                  N, K, bits, group, DTYPE_CODES[dtype], a, b)
    _run(fn, _ranges(range(N) if rows is None else rows, threads), threads)
    return out


def dequant_fp_f32(w, scales, global_scale, N, K, mode, rows=None, threads=1):
    out = np.zeros((N, K), dtype=np.float32)
    L = lib()
    g = float(global_scale) if global_scale is not None else 1.0
    fn = lambda a, b: L.oracle_dequant_fp_f32(_ptr(w), _ptr(scales), g, _ptr(out), N, K,
                                              FP_MODES[mode], a, b)
    _run(fn, _ranges(range(N) if rows is None else rows, threads), threads)
    return out


def block_scales(scales, count, kind):
    """The first ``count`` block scales of a raw scale array, widened exactly
    (kind: "e8m0", "e4m3", "f32" or "f16")."""
    a = np.ascontiguousarray(scales)
    L = lib()
    return np.array([L.oracle_block_scale(_ptr(a), i, _SCALE_CODES[kind]) for i in range(count)])


def _track1(fmt):
    e, b, blk, sk, g = TRACK1[fmt]
    return _ELEM_CODES[e], b, blk, _SCALE_CODES[sk], g


def dequant_block_scaled_f32(w, scales, global_scale, N, K, fmt, rows=None, threads=1):
    """fp32 dequantized weights of a Track-1 format (the exact value rounded
    once); ``global_scale`` only for NVFP4."""
    out = np.zeros((N, K), dtype=np.float32)
    el, b, blk, sk, ug = _track1(fmt)
    g = float(global_scale) if ug else 1.0
    L = lib()
    fn = lambda a, c: L.oracle_dequant_block_scaled_f32(_ptr(w), _ptr(scales), int(ug), g, _ptr(out), N, K,
                                                        el, b, blk, sk, a, c)
    _run(fn, _ranges(range(N) if rows is None else rows, threads), threads)
    return out


def qmv_block_scaled(x, w, scales, global_scale, M, N, K, fmt, dtype, rows=None, threads=1):
    """y = x . w_hat^T for a Track-1 format, fp64: returns (y, absdot), both
    float64 [M, N]; rows not requested stay NaN."""
    y = np.full((M, N), np.nan); a = np.full((M, N), np.nan)
    el, b, blk, sk, ug = _track1(fmt)
    g = float(global_scale) if ug else 1.0
    L = lib()
    fn = lambda r0, r1: L.oracle_qmv_block_scaled(_ptr(x), _ptr(w), _ptr(scales), int(ug), g, _ptr(y), _ptr(a),
                                                  M, N, K, el, b, blk, sk, DTYPE_CODES[dtype], r0, r1)
    _run(fn, _ranges(range(N) if rows is None else rows, threads), threads)
    return y, a


# ---- the product --------------------------------------------------------------
def qmv_affine(x, w, scales, biases, M, N, K, bits, group, dtype, rows=None, threads=1):
    """Return (y, absdot), both float64 [M, N]; rows not requested stay NaN."""
    y = np.full((M, N), np.nan); a = np.full((M, N), np.nan)
    L = lib()
    fn = lambda r0, r1: L.oracle_qmv_affine(_ptr(x), _ptr(w), _ptr(scales), _ptr(biases), _ptr(y),
                                            _ptr(a), M, N, K, bits, group, DTYPE_CODES[dtype], r0, r1)
    _run(fn, _ranges(range(N) if rows is None else rows, threads), threads)
    return y, a


def qmv_affine_gather(x, w, scales, biases, ids, M, N, K, bits, group, dtype, n_experts, x_batched=True,
                      threads=1):
    """Expert-indexed qmv (wh-iron kernel-op coverage audit, "gather_qmv /
    gather_qmm" row; DS4 moe.metal, kernel_mul_mv_id: the ids tensor selects
    the routed expert of each slot).  Token t multiplies x[t] (or the shared
    x) by matrix ids[t] of the stacks w [E, N, row bytes], scales / biases
    [E, N, K/group], each product being qmv_affine above.  An id outside
    [0, n_experts) has no matrix: that token's outputs are NaN.  Returns (y,
    absdot), float64 [T, M, N]."""
    T = len(ids)
    y = np.full((T, M, N), np.nan); a = np.full((T, M, N), np.nan)
    for t in range(T):
        e = int(ids[t])
        if not 0 <= e < n_experts:
            continue
        xt = np.ascontiguousarray(x[t] if x_batched else x)
        y[t], a[t] = qmv_affine(xt, np.ascontiguousarray(w[e]), np.ascontiguousarray(scales[e]),
                                np.ascontiguousarray(biases[e]), M, N, K, bits, group, dtype, threads=threads)
    return y, a


def qvm_affine(x, w, scales, biases, M, N, K, bits, group, dtype, cols=None, threads=1):
    """x [M, K] times W stored [K, N] (packed rows of N codes, scales and
    biases [K, N / group]).  Return (y, absdot), both float64 [M, N]; columns
    not requested stay NaN."""
    y = np.full((M, N), np.nan); a = np.full((M, N), np.nan)
    L = lib()
    fn = lambda c0, c1: L.oracle_qvm_affine(_ptr(x), _ptr(w), _ptr(scales), _ptr(biases), _ptr(y),
                                            _ptr(a), M, N, K, bits, group, DTYPE_CODES[dtype], c0, c1)
    _run(fn, _ranges(range(N) if cols is None else cols, threads), threads)
    return y, a


def qmv_fp(x, w, scales, global_scale, M, N, K, mode, dtype, rows=None, threads=1):
    y = np.full((M, N), np.nan); a = np.full((M, N), np.nan)
    L = lib()
    g = float(global_scale) if global_scale is not None else 1.0
    fn = lambda r0, r1: L.oracle_qmv_fp(_ptr(x), _ptr(w), _ptr(scales), g, _ptr(y), _ptr(a),
                                        M, N, K, FP_MODES[mode], DTYPE_CODES[dtype], r0, r1)
    _run(fn, _ranges(range(N) if rows is None else rows, threads), threads)
    return y, a


# ---- affine quantizer -------------------------------------------------------
def quantize_affine(w, N, K, bits, group, dtype, rows=None, threads=1):
    """Quantize w ([N, K] elements of `dtype`, given as a numpy array of that
    element's storage: float32, or uint16 bit patterns for f16 / bf16) into
    (packed codes uint8 [N, row_bytes], scales, biases) with the storage of
    `dtype`.  Rows outside `rows` stay zero."""
    w = np.ascontiguousarray(w)
    st = np.float32 if dtype == "f32" else np.uint16
    wq = np.zeros((N, row_bytes(K, bits)), dtype=np.uint8)
    sc = np.zeros((N, K // group), dtype=st)
    bi = np.zeros((N, K // group), dtype=st)
    L = lib()
    fn = lambda a, b: L.oracle_quantize_affine(_ptr(w), _ptr(wq), _ptr(sc), _ptr(bi), N, K, bits, group,
                                               DTYPE_CODES[dtype], a, b)
    _run(fn, _ranges(range(N) if rows is None else rows, threads), threads)
    return wq, sc, bi


# ---- FP quantizer -----------------------------------------------------------
def nearest_e2m1(a): return lib().oracle_nearest_e2m1(float(a))
def nearest_e4m3(a): return lib().oracle_nearest_e4m3(float(a))


def quantize_fp(w, N, K, mode, dtype, global_scale=1.0, rows=None, threads=1):
    """Quantize w ([N, K] storage of `dtype`) to (codes uint8 [N, K/2] (FP4,
    low nibble = even k) or [N, K] (FP8), scale bytes uint8 [N, K/block])."""
    w = np.ascontiguousarray(w)
    fp8 = mode == "mxfp8"
    blk = 16 if mode == "nvfp4" else 32
    wq = np.zeros((N, K if fp8 else K // 2), dtype=np.uint8)
    sc = np.zeros((N, K // blk), dtype=np.uint8)
    L = lib()
    fn = lambda a, b: L.oracle_quantize_fp(_ptr(w), _ptr(wq), _ptr(sc), float(global_scale), N, K, FP_MODES[mode],
                                           DTYPE_CODES[dtype], a, b)
    _run(fn, _ranges(range(N) if rows is None else rows, threads), threads)
    return wq, sc


def dequant_affine_f64(w, scales, biases, N, K, bits, group, dtype, rows=None, threads=1):
    """Dequantized affine weights [N, K] in fp64 (rows outside `rows` stay 0)."""
    out = np.zeros((N, K), dtype=np.float64)
    L = lib()
    w = np.ascontiguousarray(w); scales = np.ascontiguousarray(scales); biases = np.ascontiguousarray(biases)
    fn = lambda a, b: L.oracle_dequant_affine_f64(_ptr(w), _ptr(scales), _ptr(biases), _ptr(out),
                                                  N, K, bits, group, DTYPE_CODES[dtype], a, b)
    _run(fn, _ranges(range(N) if rows is None else rows, threads), threads)
    return out


def _widen(a, dtype):
    """Stored elements of `dtype` (float32, or uint16 bit patterns) as exact fp64."""
    a = np.asarray(a)
    if dtype == "f32":
        return a.astype(np.float64)
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(
        torch.float16 if dtype == "f16" else torch.bfloat16)
    return t.to(torch.float64).numpy()


# ---- batched Q / K / V projection --------------------------------------------
def qmv_affine_qkv(x, q3, k3, v3, M, Nq, Nkv, K, bits, group, dtype, rows=None, threads=1):
    """The three decode projections of one x in one call (wh-iron kernel-op
    coverage audit, "batched_qkv_qgemv" row: Q / K / V qGEMV in one dispatch,
    output concatenated [Q | K | V], K and V of the same size for grouped-query
    attention).  q3, k3, v3 are (w_packed, scales, biases) triples with Nq,
    Nkv, Nkv rows.  Returns (y, absdot), float64 [M, Nq + 2 Nkv]: each part is
    qmv_affine of its matrix."""
    parts = []
    for (w, sc, bi), n, off in ((q3, Nq, 0), (k3, Nkv, Nq), (v3, Nkv, Nq + Nkv)):
        r = None if rows is None else [t - off for t in rows if off <= t < off + n]
        parts.append(qmv_affine(x, w, sc, bi, M, n, K, bits, group, dtype, rows=r, threads=threads))
    y = np.concatenate([p_[0] for p_ in parts], axis=1)
    a = np.concatenate([p_[1] for p_ in parts], axis=1)
    return y, a


# ---- RMSNorm fused into the qmv -----------------------------------------------
def rms_norm(x, gamma, eps):
    """x * gamma / sqrt(mean(x^2) + eps) per row, fp64 (x, gamma float64)."""
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return x * r * gamma


def qmv_affine_rms_norm(x, gamma, eps, w, scales, biases, M, N, K, bits, group, dtype, rows=None, threads=1):
    """RMSNorm of x fused into the affine qmv (wh-iron kernel-op coverage
    audit, "rms_norm_qgemv" row): y[m, n] = sum_k xh[m, k] * w_hat[n, k] with
    xh = rms_norm(x, gamma, eps) kept in full precision (it is not rounded to
    the element type between the two steps), x and gamma stored in `dtype`.
    fp64 throughout.  Returns (y, absdot) float64 [M, N]."""
    xh = rms_norm(_widen(x, dtype).reshape(M, K), _widen(gamma, dtype).reshape(1, K), float(eps))
    W = dequant_affine_f64(w, scales, biases, N, K, bits, group, dtype, rows=rows, threads=threads)
    return xh @ W.T, np.abs(xh) @ np.abs(W).T


# ---- fused gate + up with SwiGLU ---------------------------------------------
def qmv_affine_swiglu(x, w_gate, s_gate, b_gate, w_up, s_up, b_up, M, N, K, bits, group, dtype, clamp=0.0,
                      route_weight=1.0, threads=1):
    """Decode gate/up projection fused with the SwiGLU activation (DS4
    moe.metal, kernel_dsv4_moe_swiglu_weight and the paired swiglu matvec:
    mid = silu(clamp(gate)) * clamp(up) * route_weight; wh-iron audit, swiglu
    row).  gate = x W_gate^T and up = x W_up^T are qmv_affine products (fp64);
    when clamp > 1e-6 the gate is limited to <= clamp and up to [-clamp,
    clamp]; silu(g) = g / (1 + exp(-g)).  All in fp64.  route_weight is one
    number, or one per x row (the page's kernel reads one weight per routed
    token).  Returns (mid, gate, up, absdot_gate, absdot_up), each float64
    [M, N]."""
    g, ag = qmv_affine(x, w_gate, s_gate, b_gate, M, N, K, bits, group, dtype, threads=threads)
    u, au = qmv_affine(x, w_up, s_up, b_up, M, N, K, bits, group, dtype, threads=threads)
    gc, uc = g, u
    if clamp > 1e-6:
        gc = np.minimum(g, clamp)
        uc = np.clip(u, -clamp, clamp)
    with np.errstate(over="ignore"):             # exp(-g) -> inf for very negative g: silu -> -0
        silu = gc / (1.0 + np.exp(-gc))
    rw = np.asarray(route_weight, dtype=np.float64)
    rw = rw.reshape(M, 1) if rw.ndim == 1 else rw
    return silu * uc * rw, g, u, ag, au
