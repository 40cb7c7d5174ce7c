"""Failure detection on the GPU without a fault: a bounded wait that nothing
satisfies must expire, report RET_ERR_TIMEOUT through the device error word,
and leave the context usable for the next call.

The self-test kernel waits on a shared-memory barrier that nothing arrives
on, through the same bounded wait the tensor-core kernels use (about two
seconds of SM clock); it never traps and holds nothing when it gives up.
"""

import time

import pytest
import torch

import oracle
from linear_recurrent_sequence_retention_b200 import ops, workloads as W
from tests._util import assert_close

pytestmark = pytest.mark.gpu


def test_bounded_wait_expires_and_is_reported():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    ops.check_device_error()                          # start from a clear error word
    t0 = time.perf_counter()
    ops.selftest_wait_timeout()
    with pytest.raises(ops.RetentionError) as info:
        ops.check_device_error()
    waited = time.perf_counter() - t0
    assert info.value.status == ops.RET_ERR_TIMEOUT
    assert 0.2 < waited < 30.0, f"the bounded wait took {waited:.2f} s"
    # the word was cleared by the read
    ops.check_device_error()


def test_context_usable_after_timeout():
    ops.selftest_wait_timeout()
    with pytest.raises(ops.RetentionError):
        ops.check_device_error()
    B, T, H, dk, dv, chunk = 1, 300, 2, 128, 128, 128
    q, k, v, _ = W.make_qkvg(B, T, H, dk, dv, "bf16", seed=21, gate=False)
    gam = W.head_gammas(H)
    o = ops.chunkwise_fwd(q.cuda(), k.cuda(), v.cuda(), gam, chunk, out_dtype=torch.float32)
    ops.check_device_error()
    ref = oracle.msr_parallel(W.to_f64(q), W.to_f64(k), W.to_f64(v), gam)
    assert_close(W.to_f64(o), ref, "bf16", 2, "o after a reported time-out")
