"""Helpers for the GPU parity tests: move synthetic cases to the device, call
the C ABI through the Python binding, read results back, and run the oracle
on the same host bytes."""
from __future__ import annotations

import os

import numpy as np
import pytest
import torch

import oracle
from qmv_tol import FLOOR_FRAC, assert_close

THREADS = max(1, min(16, os.cpu_count() or 1))
TORCH_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def require_cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests (no silent skip)")
    import weight_quantized_matrix_b200 as q  # raises ImportError if libqmv.so is missing
    return q


def dev(a: np.ndarray, offset_bytes: int = 0) -> torch.Tensor:
    """Copy raw storage to the device as bytes; `offset_bytes` shifts the start
    inside a larger allocation (to test alignment paths)."""
    b = np.ascontiguousarray(a).view(np.uint8).reshape(-1)
    t = torch.empty(b.size + offset_bytes + 16, dtype=torch.uint8, device="cuda")
    t[offset_bytes:offset_bytes + b.size].copy_(torch.from_numpy(b))
    return t[offset_bytes:offset_bytes + b.size]


def y_buffer(batch, M, N, dtype):
    return torch.full((batch, M, N), float("nan"), dtype=TORCH_DT[dtype], device="cuda")


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def run_affine(q, c, w_offset=0, x_batched=True, stream=None, s_offset=0):
    B, M, N, K = c["batch"], c["M"], c["N"], c["K"]
    x = c["x"] if x_batched else c["x"][:1]
    y = y_buffer(B, M, N, c["dtype"])
    args = (dev(x), dev(c["w"], w_offset), dev(c["scales"], s_offset), dev(c["biases"], s_offset), y, M, N, K,
            c["bits"], c["group"], c["dtype"])
    if B == 1 and x_batched:
        q.qmv_affine(*args, stream=stream)
    else:
        q.qmv_affine_batched(*args, B, x_batched, stream=stream)
    torch.cuda.synchronize()
    return to_f64(y)


def run_fp(q, c, x_batched=True):
    B, M, N, K = c["batch"], c["M"], c["N"], c["K"]
    x = c["x"] if x_batched else c["x"][:1]
    y = y_buffer(B, M, N, c["dtype"])
    g = None
    if c["mode"] == "nvfp4":
        g = torch.tensor(np.full(B, c["global"], dtype=np.float32), device="cuda")
    args = (dev(x), dev(c["w"]), dev(c["scales"]), g, y, M, N, K, c["mode"], c["dtype"])
    if B == 1 and x_batched:
        q.qmv_fp(*args)
    else:
        q.qmv_fp_batched(*args, B, x_batched)
    torch.cuda.synchronize()
    return to_f64(y)


def oracle_affine(c, rows=None, b=0, x_batched=True):
    xb = b if x_batched else 0
    return oracle.qmv_affine(np.ascontiguousarray(c["x"][xb]), np.ascontiguousarray(c["w"][b]),
                             np.ascontiguousarray(c["scales"][b]), np.ascontiguousarray(c["biases"][b]),
                             c["M"], c["N"], c["K"], c["bits"], c["group"], c["dtype"], rows=rows,
                             threads=THREADS)


def oracle_fp(c, rows=None, b=0, x_batched=True):
    xb = b if x_batched else 0
    return oracle.qmv_fp(np.ascontiguousarray(c["x"][xb]), np.ascontiguousarray(c["w"][b]),
                         np.ascontiguousarray(c["scales"][b]), c["global"], c["M"], c["N"], c["K"],
                         c["mode"], c["dtype"], rows=rows, threads=THREADS)


def sample_rows(N, n=48):
    """Evenly spaced rows plus the first and last few (covers every tile edge
    class at full size without running the oracle on all N rows)."""
    if N <= n:
        return list(range(N))
    s = set(np.linspace(0, N - 1, n).astype(int).tolist()) | {0, 1, 2, N - 3, N - 2, N - 1}
    return sorted(s)


def compare(y, ref, absdot, dtype, rows=None, what="", max_floor_frac=FLOOR_FRAC):
    """assert_close on the given rows; returns how many outputs the fp32 floor
    clause decided (bounded by max_floor_frac of them)."""
    if rows is not None:
        y, ref, absdot = y[:, rows], ref[:, rows], absdot[:, rows]
    return assert_close(y, ref, absdot, dtype, what, max_floor_frac=max_floor_frac)
