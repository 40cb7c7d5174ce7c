"""The tensor-core chunkwise path computes its MMA operands (decayed scores,
decayed query rows, the carried state, zeta * K and the value rows) in fp16.
A value outside fp16's range must not pass silently: the kernels flag it and
retention_check_device_error() returns RET_ERR_RANGE.  In-range inputs, the
workloads' N(0,1)/sqrt(d_k) scale among them, must not raise it.
"""

import pytest
import torch

from linear_recurrent_sequence_retention_b200 import ops, workloads as W

pytestmark = pytest.mark.gpu


def _run(q, k, v, chunk=128, **kw):
    gam = W.head_gammas(q.shape[2])
    return ops.chunkwise_fwd(q.cuda(), k.cuda(), v.cuda(), gam, chunk, **kw)


def _expect_range_error():
    with pytest.raises(ops.RetentionError) as ei:
        ops.check_device_error()
    assert ei.value.status == ops.RET_ERR_RANGE, ei.value
    ops.check_device_error()           # the read cleared the word


def test_in_range_inputs_raise_nothing():
    q, k, v, g = W.make_qkvg(2, 600, 2, 128, 256, "bf16", seed=3)
    _run(q, k, v, g=g.cuda(), return_state=True)
    ops.check_device_error()


def test_value_beyond_f16_is_reported():
    q, k, v, _ = W.make_qkvg(1, 300, 2, 64, 128, "bf16", seed=4, gate=False)
    v[0, 17, 1, 5] = 1.0e5             # a bf16 value fp16 cannot hold
    _run(q, k, v)
    _expect_range_error()


def test_scores_beyond_f16_are_reported():
    q, k, v, _ = W.make_qkvg(1, 200, 1, 128, 128, "bf16", seed=5, gate=False)
    q[0, 50] = 40.0
    k[0, 50] = 40.0                    # q.k = 128 * 1600 > 65504
    _run(q, k, v)
    _expect_range_error()


def test_state_beyond_f16_is_reported():
    q, k, v, _ = W.make_qkvg(1, 300, 1, 64, 64, "bf16", seed=6, gate=False)
    S0 = torch.zeros(1, 1, 64, 64)
    S0[0, 0, 3, 7] = 1.0e6             # the carried state leaves fp16's range
    _run(q, k, v, state_in=S0.cuda())
    _expect_range_error()
