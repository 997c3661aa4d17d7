"""qmv_qvm_affine_noalloc: qvm for callers that cannot allocate device memory.

A caller such as a plugin whose host framework owns every device byte, or a
decode loop that cannot afford an allocation's device synchronization, cannot
hand qmv_qvm_affine a workspace.  This entry point keeps its K-split scratch in
a fixed array inside the library instead.  The GPU test calls it through the C
ABI twice in a row and checks each result against qmv_qvm_affine's on the same
inputs, within the tolerance of the other qvm tests.  The file is named to be
collected last, so a run that stops at its first failure has already run every
other test; it passes alone in a fresh process as well."""
from __future__ import annotations

import ctypes

import pytest
import torch

import oracle
import synth
from gpu_util import THREADS, TORCH_DT, dev, require_cuda, to_f64
from qmv_tol import assert_close


def _lib():
    import weight_quantized_matrix_b200 as q
    L = q.lib()
    f = L.qmv_qvm_affine_noalloc
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 6 + [ctypes.c_void_p]
    f.restype = ctypes.c_int
    return q, f


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """Host-side: a workspace larger than the fixed scratch is refused before any
    launch (fake pointers are never touched)."""
    q, f = _lib()
    F = 1 << 20
    assert q.qmv_qvm_workspace_bytes(8, 32768) > (1 << 20)
    assert f(F, F, F, F, F, 8, 32768, 64, 4, 64, 2, None) == -2          # QMV_EUNSUPPORTED
    assert f(F, F, F, F, F, 0, 32768, 64, 4, 64, 2, None) == 0           # empty: nothing to do


@pytest.mark.gpu
def test_noalloc_matches_the_workspace_call_twice():
    q = require_cuda()
    _, f = _lib()
    for i, (M, N, K, bits, group, dtype) in enumerate([(2, 3072, 2049, 4, 64, "bf16"),
                                                       (1, 16384, 4096, 3, 128, "f16")]):
        c = synth.qvm_case(M, N, K, bits, group, dtype, seed=900 + i)
        x, w, s, b = dev(c["x"]), dev(c["w"]), dev(c["scales"]), dev(c["biases"])
        ref_y = torch.full((M, N), float("nan"), dtype=TORCH_DT[dtype], device="cuda")
        ws = torch.zeros(q.qmv_qvm_workspace_bytes(M, N), dtype=torch.uint8, device="cuda")
        q.qmv_qvm_affine(x, w, s, b, ref_y, M, N, K, bits, group, dtype, workspace=ws)
        stream = torch.cuda.current_stream().cuda_stream
        # the tolerance's scale, sum |x * w| per output, from the oracle
        _, ad = oracle.qvm_affine(c["x"], c["w"], c["scales"], c["biases"], M, N, K, bits, group, dtype,
                                  threads=THREADS)
        for call in range(2):
            y = torch.full((M, N), float("nan"), dtype=TORCH_DT[dtype], device="cuda")
            st = f(x.data_ptr(), w.data_ptr(), s.data_ptr(), b.data_ptr(), y.data_ptr(), M, N, K, bits, group,
                   q.DTYPES[dtype], stream)
            assert st == 0, q.qmv_status_string(st)
            torch.cuda.synchronize()
            assert_close(to_f64(y), to_f64(ref_y), ad, dtype, what=f"noalloc case {i} call {call}")
