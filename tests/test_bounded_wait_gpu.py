"""The bounded ring waits run out and report, without a fault or a hang.

qmv_test_skip_last_copy makes the producer warp of block (0, 0) of a
weight-ring kernel skip its final stage (no expected-bytes arrival, no tensor
copy).  Nothing ever completes that stage's barrier, so the block's consumer
warps give up their bounded wait (about one second) and OR code 1 into the
device fault word, and the producer gives up waiting for its own copies on that
stage and ORs code 4.  The kernel returns normally, nothing is left in flight,
and the next call on the same context is correct again.  Covered for the
three weight-ring kernels: the CUDA-core ring (one bf16 x row), the
tensor-core ring and the per-group tensor-core ring (several x rows).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from gpu_util import compare, oracle_affine, require_cuda, run_affine

pytestmark = pytest.mark.gpu

CONSUMER, FREE_STAGE, OWN_COPIES = 1, 2, 4


@pytest.fixture(scope="module")
def q():
    return require_cuda()


@pytest.fixture(autouse=True)
def _clean(q):
    q.qmv_test_skip_last_copy(False)
    q.qmv_force_config()
    q.qmv_device_fault(clear=True)
    yield
    q.qmv_test_skip_last_copy(False)
    q.qmv_force_config()
    q.qmv_device_fault(clear=True)


@pytest.mark.parametrize("path,M,want", [(6, 1, "path=tcf"), (4, 4, "path=tcb"), (8, 4, "path=tcg")])
def test_ring_wait_runs_out_and_reports(q, path, M, want):
    N, K, bits, group = 333, 4096, 4, 64
    q.qmv_force_config(path, -1, -1, -1)
    assert want in q.qmv_describe_plan("affine", M, N, K, bits, group, "bf16")
    c = synth.affine_case(M, N, K, bits, group, "bf16", seed=404 + M)

    q.qmv_test_skip_last_copy(True)
    try:
        run_affine(q, c)                       # returns; its output is undefined
    finally:
        q.qmv_test_skip_last_copy(False)
    torch.cuda.synchronize()                    # the context is still usable
    code = q.qmv_device_fault(clear=True)
    assert code == CONSUMER | OWN_COPIES, code
    assert q.qmv_device_fault() == 0

    # the same call, hook off: correct, and no wait expires
    y = run_affine(q, c)
    ref, ad = oracle_affine(c)
    compare(y[0], ref, ad, "bf16", what=f"after the expired wait ({want})")
    assert q.qmv_device_fault() == 0
