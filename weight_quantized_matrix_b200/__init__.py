"""Python binding of libqmv.so (include/qmv.h): the weight-quantized
matrix-vector product on B200.

Argument marshalling only.  Every function takes device buffers as torch
tensors (or raw integer device addresses), passes their pointers and sizes to
the C ABI of the same name, and raises :class:`QmvError` on a non-zero status.
The per-call entry points go through the CPython extension ``_qmv_fast``
(csrc/qmv_py.c), the rest through ctypes.
All compute happens in the CUDA kernels of libqmv.so; there is no fallback: if
the library has not been built, importing this package raises ImportError.

The stream defaults to torch's current CUDA stream.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "QmvError", "qmv_affine", "qmv_affine_batched", "qmv_fp", "qmv_fp_batched",
    "qmv_dequant_affine_f32", "qmv_dequant_fp_f32", "qmv_quantize_affine", "qmv_quantize_fp", "qmv_affine_gather", "qmv_affine_swiglu", "qmv_affine_qkv", "qmv_affine_rms_norm", "qmv_qmm_affine", "qmv_qvm_affine",
    "qmv_qvm_workspace_bytes", "qmv_qvm_affine_noalloc", "qmv_status_string",
    "qmv_last_cuda_error",
    "qmv_describe_plan", "qmv_force_config", "DTYPES", "FP_MODES", "LIB_PATH", "lib",
    "qmv_block_scaled", "qmv_block_scaled_batched", "qmv_dequant_block_scaled_f32", "qmv_format_info",
    "FORMATS", "qmv_test_skip_last_copy",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libqmv.so")

DTYPES = {"f32": 0, "f16": 1, "bf16": 2}
FP_MODES = {"mxfp4": 0, "nvfp4": 1, "mxfp8": 2}
# qmv_format of include/qmv.h: the Track-1 formats by the names of the wh-iron
# audit's table ("Quantization precision coverage")
FORMATS = {name: i for i, name in enumerate(
    ["nvfp4", "mxfp4", "mxfp8_e4m3", "mxfp8_e5m2", "nvfp8", "fp4", "fp8_e4m3", "fp8_e5m2"]
    + [f"int{b}" for b in (2, 3, 4, 5, 6, 8)] + [f"mxint{b}" for b in (2, 3, 4, 5, 6, 8)]
    + ["nvfp8_f16", "fp4_f16", "fp8_e4m3_f16", "fp8_e5m2_f16"] + [f"int{b}_f16" for b in (2, 3, 4, 5, 6, 8)])}
STATUS = {0: "QMV_OK", -1: "QMV_EINVAL", -2: "QMV_EUNSUPPORTED", -3: "QMV_EALIGN", -4: "QMV_ECUDA"}

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libqmv.so not found at {LIB_PATH}; build it with "
        "`python weight_quantized_matrix_b200/build_lib.py` (needs nvcc)")

try:
    _lib = ctypes.CDLL(LIB_PATH)
except OSError as _e:
    raise ImportError(
        f"libqmv.so at {LIB_PATH} does not load ({_e}); rebuild it with "
        "`python weight_quantized_matrix_b200/build_lib.py --force`") from _e
try:
    from . import _qmv_fast as _fast      # per-call entry points (CPython extension over libqmv.so)
except ImportError as _e:
    raise ImportError(
        "the _qmv_fast extension is missing; build it with "
        "`python weight_quantized_matrix_b200/build_lib.py` (needs gcc)") from _e
_p, _i, _ll = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong
_lib.qmv_affine.argtypes = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _p]
_lib.qmv_affine_batched.argtypes = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _p]
_lib.qmv_fp.argtypes = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _p]
_lib.qmv_fp_batched.argtypes = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _p]
_lib.qmv_dequant_affine_f32.argtypes = [_p, _p, _p, _p, _i, _i, _i, _i, _i, _p]
_lib.qmv_dequant_fp_f32.argtypes = [_p, _p, _p, _p, _i, _i, _i, _p]
_lib.qmv_quantize_affine.argtypes = [_p, _p, _p, _p, _i, _i, _i, _i, _i, _p]
_lib.qmv_qvm_affine.argtypes = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _p, _p]
_lib.qmv_qmm_affine.argtypes = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _p]
_lib.qmv_affine_gather.argtypes = [_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _i, _p]
_lib.qmv_quantize_fp.argtypes = [_p, _p, _p, _p, _i, _i, _i, _i, _p]
_lib.qmv_quantize_fp.restype = _i
_lib.qmv_affine_swiglu.argtypes = [_p, _p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, ctypes.c_float, _p]
_lib.qmv_affine_swiglu.restype = _i
_lib.qmv_affine_qkv.argtypes = [_p] * 11 + [_i] * 7 + [_p]
_lib.qmv_affine_qkv.restype = _i
_lib.qmv_affine_rms_norm.argtypes = [_p, _p, ctypes.c_float, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _p]
_lib.qmv_affine_rms_norm.restype = _i
_lib.qmv_affine_gather.restype = _i
_lib.qmv_qmm_affine.restype = _i
_lib.qmv_qvm_workspace_bytes.argtypes = [_i, _i]
_lib.qmv_qvm_workspace_bytes.restype = ctypes.c_size_t
_lib.qmv_status_string.argtypes = [_i]
_lib.qmv_status_string.restype = ctypes.c_char_p
_lib.qmv_last_cuda_error.argtypes = []
_lib.qmv_describe_plan.argtypes = [_i, _i, _i, _i, _i, _i, _i, _i, ctypes.c_char_p, _i]
_lib.qmv_block_scaled.argtypes = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _p]
_lib.qmv_block_scaled_batched.argtypes = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _p]
_lib.qmv_dequant_block_scaled_f32.argtypes = [_p, _p, _p, _p, _i, _i, _i, _p]
_lib.qmv_format_info.argtypes = [_i] + [ctypes.POINTER(ctypes.c_int)] * 4
_lib.qmv_device_fault.argtypes = [ctypes.POINTER(ctypes.c_uint), _i]
_lib.qmv_force_config.argtypes = [_i, _i, _i, _i]
_lib.qmv_test_skip_last_copy.argtypes = [_i]
_lib.qmv_force_config.restype = None
for _f in ("qmv_affine", "qmv_affine_batched", "qmv_fp", "qmv_fp_batched",
           "qmv_dequant_affine_f32", "qmv_dequant_fp_f32", "qmv_quantize_affine", "qmv_qvm_affine",
           "qmv_last_cuda_error",
           "qmv_describe_plan", "qmv_device_fault"):
    getattr(_lib, _f).restype = _i


def lib() -> ctypes.CDLL:
    return _lib


class QmvError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        name = STATUS.get(status, str(status))
        msg = f"{what}: {name} ({_lib.qmv_status_string(status).decode()})"
        if status == -4:
            msg += f", cudaError {_lib.qmv_last_cuda_error()}"
        super().__init__(msg)


def _ptr(a):
    if a is None:
        return None
    if isinstance(a, int):
        return a
    return a.data_ptr()


def _dtype(d):
    if isinstance(d, int):
        return d
    if isinstance(d, str):
        return DTYPES[d]
    import torch
    return {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}[d]


def _mode(m):
    return m if isinstance(m, int) else FP_MODES[m]


def _format(f):
    return f if isinstance(f, int) else FORMATS[f]


_raw_stream = None


def _stream(s):
    global _raw_stream
    if s is None:
        if _raw_stream is None:
            import torch
            c = torch._C
            if hasattr(c, "_cuda_getCurrentRawStream") and hasattr(c, "_cuda_getDevice"):
                _raw_stream = lambda: c._cuda_getCurrentRawStream(c._cuda_getDevice())  # noqa: E731
            else:
                _raw_stream = lambda: torch.cuda.current_stream().cuda_stream  # noqa: E731
        return _raw_stream()
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(st, what):
    if st != 0:
        raise QmvError(st, what)


def qmv_affine(x, w_packed, scales, biases, y, M, N, K, bits, group_size, dtype, stream=None):
    st = _fast.affine(_ptr(x), _ptr(w_packed), _ptr(scales), _ptr(biases), _ptr(y), M, N, K, bits, group_size,
                      _dtype(dtype), 1, 1, _stream(stream))
    if st:
        raise QmvError(st, "qmv_affine")


def qmv_affine_batched(x, w_packed, scales, biases, y, M, N, K, bits, group_size, dtype, batch,
                       x_batched=True, stream=None):
    _check(_fast.affine(_ptr(x), _ptr(w_packed), _ptr(scales), _ptr(biases), _ptr(y), M, N, K, bits,
                        group_size, _dtype(dtype), batch, int(bool(x_batched)), _stream(stream)),
           "qmv_affine_batched")


def qmv_fp(x, w_packed, scales, global_scale, y, M, N, K, mode, dtype, stream=None):
    st = _fast.fp(_ptr(x), _ptr(w_packed), _ptr(scales), _ptr(global_scale), _ptr(y), M, N, K, _mode(mode),
                  _dtype(dtype), 1, 1, _stream(stream))
    if st:
        raise QmvError(st, "qmv_fp")


def qmv_fp_batched(x, w_packed, scales, global_scale, y, M, N, K, mode, dtype, batch, x_batched=True,
                   stream=None):
    _check(_fast.fp(_ptr(x), _ptr(w_packed), _ptr(scales), _ptr(global_scale), _ptr(y), M, N, K, _mode(mode),
                    _dtype(dtype), batch, int(bool(x_batched)), _stream(stream)), "qmv_fp_batched")


def qmv_block_scaled(x, w_packed, scales, global_scale, y, M, N, K, fmt, dtype, stream=None):
    """qmv for a Track-1 block-scaled format (name in FORMATS or a qmv_format
    value); global_scale: a device float tensor for NVFP4, else None."""
    st = _fast.block_scaled(_ptr(x), _ptr(w_packed), _ptr(scales), _ptr(global_scale), _ptr(y), M, N, K,
                            _format(fmt), _dtype(dtype), 1, 1, _stream(stream))
    if st:
        raise QmvError(st, "qmv_block_scaled")


def qmv_block_scaled_batched(x, w_packed, scales, global_scale, y, M, N, K, fmt, dtype, batch, x_batched=True,
                             stream=None):
    _check(_fast.block_scaled(_ptr(x), _ptr(w_packed), _ptr(scales), _ptr(global_scale), _ptr(y), M, N, K,
                              _format(fmt), _dtype(dtype), batch, int(bool(x_batched)), _stream(stream)),
           "qmv_block_scaled_batched")


def qmv_dequant_block_scaled_f32(w_packed, scales, global_scale, w_out, N, K, fmt, stream=None):
    _check(_lib.qmv_dequant_block_scaled_f32(_ptr(w_packed), _ptr(scales), _ptr(global_scale), _ptr(w_out), N, K,
                                             _format(fmt), _stream(stream)), "qmv_dequant_block_scaled_f32")


def qmv_format_info(fmt) -> dict:
    """Layout of a Track-1 format: bits per code, block, bytes per scale, and
    whether it takes a global scale."""
    v = [ctypes.c_int(0) for _ in range(4)]
    _check(_lib.qmv_format_info(_format(fmt), *[ctypes.byref(a) for a in v]), "qmv_format_info")
    return {"element_bits": v[0].value, "block": v[1].value, "scale_bytes": v[2].value,
            "has_global": bool(v[3].value)}


def qmv_dequant_affine_f32(w_packed, scales, biases, w_out, N, K, bits, group_size, dtype, stream=None):
    _check(_lib.qmv_dequant_affine_f32(_ptr(w_packed), _ptr(scales), _ptr(biases), _ptr(w_out), N, K,
                                       bits, group_size, _dtype(dtype), _stream(stream)),
           "qmv_dequant_affine_f32")


def qmv_dequant_fp_f32(w_packed, scales, global_scale, w_out, N, K, mode, stream=None):
    _check(_lib.qmv_dequant_fp_f32(_ptr(w_packed), _ptr(scales), _ptr(global_scale), _ptr(w_out), N, K,
                                   _mode(mode), _stream(stream)), "qmv_dequant_fp_f32")


def qmv_quantize_affine(w, w_packed, scales, biases, N, K, bits, group_size, dtype, stream=None):
    """Affine quantizer (C ABI qmv_quantize_affine): w [N, K] in dtype ->
    packed codes [N, K*bits/8] bytes, scales and biases [N, K/group_size] in
    dtype, all caller-owned device buffers."""
    _check(_lib.qmv_quantize_affine(_ptr(w), _ptr(w_packed), _ptr(scales), _ptr(biases), N, K, bits,
                                    group_size, _dtype(dtype), _stream(stream)), "qmv_quantize_affine")


def qmv_quantize_fp(w, w_packed, scales, global_scale, N, K, mode, dtype, stream=None):
    """Block-scaled FP quantizer (C ABI qmv_quantize_fp): w [N, K] in dtype ->
    codes and scale bytes in the layout qmv_fp reads; global_scale is a device
    float tensor for NVFP4, None for the MX modes."""
    _check(_lib.qmv_quantize_fp(_ptr(w), _ptr(w_packed), _ptr(scales), _ptr(global_scale), N, K, FP_MODES[mode],
                                _dtype(dtype), _stream(stream)), "qmv_quantize_fp")


def qmv_affine_gather(x, w_packed, scales, biases, expert_ids, y, M, N, K, bits, group_size, dtype, n_tokens,
                      n_experts, x_batched=True, stream=None):
    """Expert-indexed qmv (C ABI qmv_affine_gather): y[t] = x[t] times the
    dequantized matrix expert_ids[t] of the stack; expert_ids is a device
    int32 tensor."""
    _check(_lib.qmv_affine_gather(_ptr(x), _ptr(w_packed), _ptr(scales), _ptr(biases), _ptr(expert_ids), _ptr(y),
                                  M, N, K, bits, group_size, _dtype(dtype), n_tokens, n_experts,
                                  1 if x_batched else 0, _stream(stream)), "qmv_affine_gather")


def qmv_qmm_affine(x, w_packed, scales, biases, y, M, N, K, bits, group_size, dtype, stream=None):
    """Small-M qmm (C ABI qmv_qmm_affine): qmv_affine's layouts with up to 64
    x rows, run as chunks of 8 rows back to back on the stream."""
    _check(_lib.qmv_qmm_affine(_ptr(x), _ptr(w_packed), _ptr(scales), _ptr(biases), _ptr(y), M, N, K, bits,
                               group_size, _dtype(dtype), _stream(stream)), "qmv_qmm_affine")


def qmv_qvm_affine(x, w_packed, scales, biases, y, M, N, K, bits, group_size, dtype, workspace=None,
                   stream=None):
    """qvm (C ABI qmv_qvm_affine): x [M, K] times W stored [K, N] (w_packed
    [K, N*bits/8] bytes, scales / biases [K, N/group_size]) -> y [M, N].
    workspace: None, or a zero-filled device buffer of
    qmv_qvm_workspace_bytes(M, N) bytes that every call leaves zero."""
    _check(_lib.qmv_qvm_affine(_ptr(x), _ptr(w_packed), _ptr(scales), _ptr(biases), _ptr(y), M, N, K, bits,
                               group_size, _dtype(dtype), _ptr(workspace), _stream(stream)), "qmv_qvm_affine")


_lib.qmv_qvm_affine_noalloc.argtypes = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _p]
_lib.qmv_qvm_affine_noalloc.restype = _i


def qmv_qvm_affine_noalloc(x, w_packed, scales, biases, y, M, N, K, bits, group_size, dtype, stream=None):
    """qvm for callers that cannot allocate device memory (C ABI
    qmv_qvm_affine_noalloc): as qmv_qvm_affine, with the K-split scratch in a
    fixed 1 MiB array the library holds; calls that overlap on the GPU race."""
    _check(_lib.qmv_qvm_affine_noalloc(_ptr(x), _ptr(w_packed), _ptr(scales), _ptr(biases), _ptr(y), M, N, K,
                                       bits, group_size, _dtype(dtype), _stream(stream)),
           "qmv_qvm_affine_noalloc")


def qmv_qvm_workspace_bytes(M, N) -> int:
    return int(_lib.qmv_qvm_workspace_bytes(M, N))


def qmv_status_string(status: int) -> str:
    return _lib.qmv_status_string(status).decode()


def qmv_last_cuda_error() -> int:
    return _lib.qmv_last_cuda_error()


def qmv_affine_swiglu(x, w_gate, s_gate, b_gate, w_up, s_up, b_up, route_weight, mid, M, N, K, bits, group_size,
                      dtype, clamp=0.0, stream=None):
    """Fused gate + up projection with SwiGLU: mid = silu(clamp(x W_gate^T)) *
    clamp(x W_up^T) * route_weight (route_weight: device float32 [M] or None)."""
    _check(_lib.qmv_affine_swiglu(_ptr(x), _ptr(w_gate), _ptr(s_gate), _ptr(b_gate), _ptr(w_up), _ptr(s_up),
                                  _ptr(b_up), _ptr(route_weight), _ptr(mid), M, N, K, bits, group_size,
                                  _dtype(dtype), ctypes.c_float(clamp), _stream(stream)), "qmv_affine_swiglu")


def qmv_affine_qkv(x, q3, k3, v3, y, M, Nq, Nkv, K, bits, group_size, dtype, stream=None):
    """Q, K and V projections in one launch; q3, k3, v3 are (w_packed, scales,
    biases) and y is [M, Nq + 2 Nkv] = [Q | K | V]."""
    _check(_lib.qmv_affine_qkv(_ptr(x), *(_ptr(t) for t in q3), *(_ptr(t) for t in k3), *(_ptr(t) for t in v3),
                               _ptr(y), M, Nq, Nkv, K, bits, group_size, _dtype(dtype), _stream(stream)),
           "qmv_affine_qkv")


def qmv_affine_rms_norm(x, gamma, eps, w_packed, scales, biases, y, M, N, K, bits, group_size, dtype, stream=None):
    """RMSNorm of x (gamma [K], eps) fused into the affine qmv."""
    _check(_lib.qmv_affine_rms_norm(_ptr(x), _ptr(gamma), ctypes.c_float(eps), _ptr(w_packed), _ptr(scales),
                                    _ptr(biases), _ptr(y), M, N, K, bits, group_size, _dtype(dtype), _stream(stream)),
           "qmv_affine_rms_norm")


def qmv_describe_plan(family, M, N, K, bits=4, group_size=64, dtype="bf16", w_align16=True) -> str:
    """Text of the launch the picker chooses; family 'affine', an FP mode name
    (qmv_fp) or a Track-1 format name (qmv_block_scaled)."""
    if family == "affine":
        fam = 0
    elif family in FP_MODES:
        fam = 1 + FP_MODES[family]
    else:
        fam = 100 + _format(family)
    buf = ctypes.create_string_buffer(256)
    _check(_lib.qmv_describe_plan(fam, M, N, K, bits, group_size, _dtype(dtype), int(w_align16), buf, 256),
           "qmv_describe_plan")
    return buf.value.decode()


def qmv_device_fault(clear=False) -> int:
    """Fault word of the current device (nonzero: a bounded wait in a kernel
    expired and that call's output is undefined); synchronous."""
    code = ctypes.c_uint(0)
    _check(_lib.qmv_device_fault(ctypes.byref(code), int(bool(clear))), "qmv_device_fault")
    return code.value


def qmv_test_skip_last_copy(enable=True):
    """NOT FOR PRODUCTION USE: make the weight-ring kernels' block (0, 0) skip
    its final stage so the bounded waits run out (see include/qmv.h)."""
    _lib.qmv_test_skip_last_copy(int(bool(enable)))


def qmv_force_config(path=-1, rows_per_warp=-1, warps_k=-1, warps_rows=-1):
    """Test / benchmark knob (process-wide, not for production): pin the
    picker's path (8 per-group tensor-core ring, 7 tcgen05, 6 CUDA-core ring,
    5 few-rows, 4 tensor-core ring, 3 tensor cores, 1 / 0 CUDA-core wide /
    4-byte, -1 automatic) and launch-shape fields; no arguments restores
    automatic plans."""
    _lib.qmv_force_config(path, rows_per_warp, warps_k, warps_rows)
