"""Seeded synthetic inputs for the qmv tests and benchmark.

This module is shared by the oracle side and the CUDA side, so it holds none
of the method's arithmetic: it draws random numbers, rounds them to the storage
dtype with a plain cast, and returns raw bytes.  Packed weights are uniform
random BYTES, which makes every code of every width uniform over its full range
(2/3/4/5/6/8-bit affine codes and the 16 E2M1 codes alike); E4M3 codes are
drawn from the 254 non-NaN byte values.  Nothing here unpacks, decodes or
multiplies anything.

Distributions (from the workload descriptions the tests and bench cover):
  affine:  x ~ N(0, 1), scales ~ U(0.005, 0.02), biases ~ N(0, 0.01), all
           rounded to the dtype; the precision case draws x ~ U(1e-4, 1e-3) and
           uses the symmetric zero point bias = -scale * (2^bits - 1) / 2 that a
           min/max quantizer gives for zero-mean weights.
  FP:      E8M0 block exponents ~ U{118..130}; NVFP4 block scales are positive,
           non-zero, non-NaN E4M3 bytes (0x01..0x7E); NVFP4 global ~ U(0.5, 2).
  Track-1 block-scaled (bs_case): codes are uniform random bytes for E2M1 and
           the signed integers, uniform over the 254 non-NaN bytes for E4M3
           and over the 248 finite bytes for E5M2 (exponent field not all
           ones); E8M0 and E4M3 scales as above (E8M0 ~ U{111..123} for E5M2
           elements, whose range is 2^7 wider); FP32 / FP16 scales ~
           U(0.005, 0.02) (rounded to f16 for the FP16 twins), or a caller's
           range.
"""
from __future__ import annotations

import numpy as np
import torch

_TORCH = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
ELEM_BYTES = {"f32": 4, "f16": 2, "bf16": 2}


def rng(seed: int) -> np.random.Generator:
    """Counter-based generator (Philox) so any seed is reproducible anywhere."""
    return np.random.Generator(np.random.Philox(seed))


def to_storage(values: np.ndarray, dtype: str) -> np.ndarray:
    """Round float values to ``dtype`` (a plain cast) and return the raw storage:
    float32 for f32, uint16 bit patterns for f16 / bf16."""
    t = torch.from_numpy(np.ascontiguousarray(values, dtype=np.float32)).to(_TORCH[dtype])
    if dtype == "f32":
        return t.numpy().copy()
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def storage_to_float(raw: np.ndarray, dtype: str) -> np.ndarray:
    """Raw storage back to float32 values (a plain widening cast)."""
    if dtype == "f32":
        return raw.astype(np.float32)
    t = torch.from_numpy(raw.view(np.int16).copy()).view(_TORCH[dtype])
    return t.to(torch.float32).numpy()


def random_bytes(g: np.random.Generator, shape) -> np.ndarray:
    return g.integers(0, 256, size=shape, dtype=np.uint8)


def affine_case(M, N, K, bits, group, dtype, seed, batch=1, precision=False):
    """One affine problem.  Shapes: x [batch, M, K], w [batch, N, K*bits/8] u8,
    scales / biases [batch, N, K/group]; x, scales and biases are raw storage
    of ``dtype``."""
    g = rng(seed)
    if precision:
        x = g.uniform(1e-4, 1e-3, size=(batch, M, K))
    else:
        x = g.standard_normal(size=(batch, M, K))
    w = random_bytes(g, (batch, N, K * bits // 8))
    s = g.uniform(0.005, 0.02, size=(batch, N, K // group))
    s_raw = to_storage(s, dtype)
    if precision:
        b = -storage_to_float(s_raw, dtype).astype(np.float64) * ((2 ** bits - 1) / 2.0)
    else:
        b = g.normal(0.0, 0.01, size=(batch, N, K // group))
    return {
        "x": to_storage(x, dtype), "w": w, "scales": s_raw, "biases": to_storage(b, dtype),
        "M": M, "N": N, "K": K, "bits": bits, "group": group, "dtype": dtype, "batch": batch,
    }


def qvm_case(M, N, K, bits, group, dtype, seed, precision=False):
    """One qvm problem (W stored [K, N], grouped along N).  x [M, K], w
    [K, N*bits/8] u8, scales / biases [K, N/group]; x, scales and biases are
    raw storage of ``dtype``.  Same value distributions as affine_case."""
    g = rng(seed)
    if precision:
        x = g.uniform(1e-4, 1e-3, size=(M, K))
    else:
        x = g.standard_normal(size=(M, K))
    w = random_bytes(g, (K, N * bits // 8))
    s = g.uniform(0.005, 0.02, size=(K, N // group))
    s_raw = to_storage(s, dtype)
    if precision:
        b = -storage_to_float(s_raw, dtype).astype(np.float64) * ((2 ** bits - 1) / 2.0)
    else:
        b = g.normal(0.0, 0.01, size=(K, N // group))
    return {"x": to_storage(x, dtype), "w": w, "scales": s_raw, "biases": to_storage(b, dtype),
            "M": M, "N": N, "K": K, "bits": bits, "group": group, "dtype": dtype}


FP_BLOCK = {"mxfp4": 32, "nvfp4": 16, "mxfp8": 32}
FP_BITS = {"mxfp4": 4, "nvfp4": 4, "mxfp8": 8}
_E4M3_NON_NAN = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)


def fp_case(M, N, K, mode, dtype, seed, batch=1, precision=False):
    """One block-scaled FP problem.  w [batch, N, K*bits/8] u8 codes, scales
    [batch, N, K/block] u8, global (NVFP4 only) a float32 scalar.  The
    precision case draws x ~ U(1e-4, 1e-3) (all positive, as the affine one)."""
    g = rng(seed)
    x = g.uniform(1e-4, 1e-3, size=(batch, M, K)) if precision else g.standard_normal(size=(batch, M, K))
    bits, blk = FP_BITS[mode], FP_BLOCK[mode]
    if bits == 4:
        w = random_bytes(g, (batch, N, K // 2))
    else:
        w = _E4M3_NON_NAN[g.integers(0, len(_E4M3_NON_NAN), size=(batch, N, K))]
    if mode == "nvfp4":
        sc = g.integers(0x01, 0x7F, size=(batch, N, K // blk), dtype=np.uint8)
        glob = np.float32(g.uniform(0.5, 2.0))
    else:
        sc = g.integers(118, 131, size=(batch, N, K // blk), dtype=np.uint8)
        glob = None
    return {
        "x": to_storage(x, dtype), "w": np.ascontiguousarray(w, dtype=np.uint8), "scales": sc,
        "global": glob, "M": M, "N": N, "K": K, "mode": mode, "dtype": dtype, "batch": batch,
    }


# E5M2 bytes whose exponent field (bits 2..6) is not all ones: the finite codes
_E5M2_FINITE = np.array([c for c in range(256) if (c & 0x7C) != 0x7C], dtype=np.uint8)
_SCALE_BYTES = {"e8m0": 1, "e4m3": 1, "f32": 4, "f16": 2}


def bs_case(M, N, K, elem, bits, block, scale, use_global, dtype, seed, batch=1, precision=False,
            scale_range=(0.005, 0.02)):
    """One Track-1 block-scaled problem, described by its layout: ``elem`` in
    {"e2m1", "e4m3", "e5m2", "int"}, ``bits`` per code, ``block`` codes per
    scale along K, ``scale`` in {"e8m0", "e4m3", "f32", "f16"}.  Returns w
    [batch, N, K*bits/8] u8, scales [batch, N, K/block] as raw storage (u8,
    float32 or uint16 f16 patterns), x raw storage of ``dtype``, and the
    global (a float32 scalar when ``use_global``)."""
    g = rng(seed)
    x = g.uniform(1e-4, 1e-3, size=(batch, M, K)) if precision else g.standard_normal(size=(batch, M, K))
    rb = K * bits // 8
    if elem == "e4m3":
        w = _E4M3_NON_NAN[g.integers(0, len(_E4M3_NON_NAN), size=(batch, N, rb))]
    elif elem == "e5m2":
        w = _E5M2_FINITE[g.integers(0, len(_E5M2_FINITE), size=(batch, N, rb))]
    else:
        w = random_bytes(g, (batch, N, rb))
    shape = (batch, N, K // block)
    if scale == "e8m0":
        # E5M2 reaches 2^7 further than E4M3 (57344 vs 448): its exponents sit
        # 7 lower so the weights span the same magnitudes as MXFP8-E4M3's
        lo = 111 if elem == "e5m2" else 118
        sc = g.integers(lo, lo + 13, size=shape, dtype=np.uint8)
    elif scale == "e4m3":
        sc = g.integers(0x01, 0x7F, size=shape, dtype=np.uint8)
    elif scale == "f32":
        sc = g.uniform(*scale_range, size=shape).astype(np.float32)
    else:
        sc = to_storage(g.uniform(*scale_range, size=shape), "f16")
    glob = np.float32(g.uniform(0.5, 2.0)) if use_global else None
    return {
        "x": to_storage(x, dtype), "w": np.ascontiguousarray(w, dtype=np.uint8), "scales": np.ascontiguousarray(sc),
        "global": glob, "M": M, "N": N, "K": K, "dtype": dtype, "batch": batch,
        "elem": elem, "bits": bits, "block": block, "scale": scale, "use_global": use_global,
        "scale_bytes": _SCALE_BYTES[scale],
    }
