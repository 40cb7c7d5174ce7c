"""GPU parity of retention_recurrent_steps (Tn decode steps in one pass over
the state) against the fp64 oracle's recurrence applied token by token.

float32 inputs (and shapes outside the tensor-core kernel) are computed in
float32 on CUDA cores from exact inputs, so the Tn outputs and the updated
state are held to the float32 bound (relative L2 <= 1e-5) per head and
overall.  bf16 inputs with 12 or more tokens, d_k in {128, 256} and d_v a
multiple of 128 run on the tensor cores (tf32 products on the float32 state)
and are held to the bf16-input bound, plus relative L2 <= 2e-3 as a precision
check.  The tests span one to sixteen
tokens, d_v not a multiple of the 128-column block, gamma = 0 and gamma = 1
heads, agreement with Tn single-step calls, several 512-column blocks with a
ragged last one over hundreds of blocks, and the largest supported d_k.
"""

import numpy as np
import pytest
import torch

import oracle
from linear_recurrent_sequence_retention_b200 import ops, workloads as W
from tests._util import assert_close, rel_l2

pytestmark = pytest.mark.gpu


def _tensor_core(dtype, dk, dv, Tn):
    return dtype == "bf16" and dk in (128, 256) and dv % 128 == 0 and Tn >= 12


def _check(got, ref, dtype, dk, dv, axis, what, Tn=16, **kw):
    if _tensor_core(dtype, dk, dv, Tn):
        assert_close(f64(got), ref, "bf16", axis, what, **kw)
        assert rel_l2(f64(got), ref) <= 2e-3, (what, rel_l2(f64(got), ref))
    else:
        assert_close(f64(got), ref, "f32", axis, what, **kw)

f64 = W.to_f64


def _inputs(N, Tn, H, dk, dv, dtype, seed):
    q, k, v, _ = W.make_qkvg(N, Tn, H, dk, dv, dtype, seed=seed, gate=False)
    S0 = W.make_state(N, H, dk, dv, seed=seed + 1, scale=0.1)
    return q, k, v, S0


def _oracle(q, k, v, S0, gam):
    N, Tn, H, dk = q.shape
    dv = v.shape[3]
    o = np.zeros((N, Tn, H, dv))
    S = f64(S0).copy()
    for n in range(N):
        for h in range(H):
            Snh = S[n, h]
            for t in range(Tn):
                o[n, t, h], Snh = oracle.recurrent_step(f64(q[n, t, h]), f64(k[n, t, h]),
                                                        f64(v[n, t, h]), gam[h], Snh)
            S[n, h] = Snh
    return o, S


@pytest.mark.parametrize("Tn", [1, 3, 8, 16])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_steps_match_oracle(Tn, dtype):
    N, H, dk, dv = 3, 4, 256, 512
    q, k, v, S0 = _inputs(N, Tn, H, dk, dv, dtype, seed=Tn)
    gam = W.head_gammas(H)
    S = S0.clone().cuda()
    o = ops.recurrent_steps(q.cuda(), k.cuda(), v.cuda(), gam, S)
    ops.check_device_error()
    o_ref, S_ref = _oracle(q, k, v, S0, gam)
    _check(o, o_ref, dtype, dk, dv, 2, f"o Tn={Tn}", Tn=Tn)
    _check(S, S_ref, dtype, dk, dv, 1, f"state Tn={Tn}", Tn=Tn)


def test_ragged_columns_and_extreme_gammas():
    N, Tn, H, dk, dv = 2, 5, 3, 64, 100          # d_v not a multiple of 128
    q, k, v, S0 = _inputs(N, Tn, H, dk, dv, "bf16", seed=9)
    gam = np.array([0.0, 1.0, 0.9])
    S = S0.clone().cuda()
    o = ops.recurrent_steps(q.cuda(), k.cuda(), v.cuda(), gam, S, out_dtype=torch.float32)
    ops.check_device_error()
    o_ref, S_ref = _oracle(q, k, v, S0, gam)
    assert_close(f64(o), o_ref, "f32", 2, "o")
    assert_close(f64(S), S_ref, "f32", 1, "state")


def test_equals_repeated_single_steps():
    N, Tn, H, dk, dv = 4, 16, 2, 256, 512
    q, k, v, S0 = _inputs(N, Tn, H, dk, dv, "bf16", seed=31)
    gam = W.head_gammas(H)
    Sm, Ss = S0.clone().cuda(), S0.clone().cuda()
    om = ops.recurrent_steps(q.cuda(), k.cuda(), v.cuda(), gam, Sm)
    os_ = [ops.recurrent_step(q[:, t].contiguous().cuda(), k[:, t].contiguous().cuda(),
                              v[:, t].contiguous().cuda(), gam, Ss) for t in range(Tn)]
    ops.check_device_error()
    _check(om, np.stack([f64(x) for x in os_], axis=1), "bf16", dk, dv, 2, "o vs single steps")
    _check(Sm, f64(Ss), "bf16", dk, dv, 1, "state vs single steps")


def test_bf16_output_and_rejects():
    N, Tn, H, dk, dv = 2, 4, 2, 128, 256
    q, k, v, S0 = _inputs(N, Tn, H, dk, dv, "bf16", seed=5)
    gam = W.head_gammas(H)
    S = S0.clone().cuda()
    o = ops.recurrent_steps(q.cuda(), k.cuda(), v.cuda(), gam, S, out_dtype=torch.bfloat16)
    ops.check_device_error()
    o_ref, _ = _oracle(q, k, v, S0, gam)
    assert_close(f64(o), o_ref, "bf16", 2, "o bf16", stored_bf16=True)     # tensor cores, bf16 stores
    # 17 tokens per call is beyond the kernel's range: refused, nothing enqueued
    q17, k17, v17, _ = _inputs(1, 17, H, dk, dv, "bf16", seed=6)
    with pytest.raises(ops.RetentionError) as info:
        ops.recurrent_steps(q17.cuda(), k17.cuda(), v17.cuda(), gam, S[:1].clone())
    assert info.value.status == ops.RET_ERR_UNSUPPORTED


def test_many_items_ragged_blocks_and_rows():
    """592 blocks (37 sequences x 8 heads x 2 column blocks); d_v = 644 (a
    132-column last block), d_k = 68 (17 groups of 4 rows)."""
    N, Tn, H, dk, dv = 37, 7, 8, 68, 644
    q, k, v, S0 = _inputs(N, Tn, H, dk, dv, "bf16", seed=41)
    gam = W.head_gammas(H)
    S = S0.clone().cuda()
    o = ops.recurrent_steps(q.cuda(), k.cuda(), v.cuda(), gam, S)
    ops.check_device_error()
    o_ref, S_ref = _oracle(q, k, v, S0, gam)
    assert_close(f64(o), o_ref, "f32", 2, "o")
    assert_close(f64(S), S_ref, "f32", 1, "state")


def test_largest_dk():
    """d_k = 512, the largest the call accepts, float32 inputs."""
    N, Tn, H, dk, dv = 2, 16, 2, 512, 256
    q, k, v, S0 = _inputs(N, Tn, H, dk, dv, "f32", seed=43)
    gam = W.head_gammas(H)
    S = S0.clone().cuda()
    o = ops.recurrent_steps(q.cuda(), k.cuda(), v.cuda(), gam, S)
    ops.check_device_error()
    o_ref, S_ref = _oracle(q, k, v, S0, gam)
    assert_close(f64(o), o_ref, "f32", 2, "o")
    assert_close(f64(S), S_ref, "f32", 1, "state")


@pytest.mark.parametrize("Tn", [12, 16])
def test_tensor_core_many_states_and_blocks(Tn):
    """The tensor-core kernel (12 or more tokens) over more (sequence, head) states
    than SMs, d_k = 128 and four 128-column blocks, gamma = 0 and gamma = 1 heads
    among them."""
    N, H, dk, dv = 75, 4, 128, 512
    q, k, v, S0 = _inputs(N, Tn, H, dk, dv, "bf16", seed=50 + Tn)
    gam = np.array([0.0, 1.0, 0.9, 0.999])
    S = S0.clone().cuda()
    o = ops.recurrent_steps(q.cuda(), k.cuda(), v.cuda(), gam, S)
    ops.check_device_error()
    o_ref, S_ref = _oracle(q, k, v, S0, gam)
    _check(o, o_ref, "bf16", dk, dv, 2, "o", Tn=Tn)
    _check(S, S_ref, "bf16", dk, dv, 1, "state", Tn=Tn)


def test_tensor_core_bf16_output():
    """16 tokens on the tensor cores with bfloat16 outputs (d_k = 256, d_v = 256)."""
    N, Tn, H, dk, dv = 3, 16, 2, 256, 256
    q, k, v, S0 = _inputs(N, Tn, H, dk, dv, "bf16", seed=61)
    gam = W.head_gammas(H)
    S = S0.clone().cuda()
    o = ops.recurrent_steps(q.cuda(), k.cuda(), v.cuda(), gam, S, out_dtype=torch.bfloat16)
    ops.check_device_error()
    o_ref, S_ref = _oracle(q, k, v, S0, gam)
    assert_close(f64(o), o_ref, "bf16", 2, "o bf16", stored_bf16=True)
    _check(S, S_ref, "bf16", dk, dv, 1, "state", Tn=Tn)


def test_tensor_core_widest_value_head():
    """d_k = 128 with d_v = 768 (six 128-column blocks, the widest whose operand
    tiles fit), 13 tokens."""
    N, Tn, H, dk, dv = 4, 13, 3, 128, 768
    q, k, v, S0 = _inputs(N, Tn, H, dk, dv, "bf16", seed=71)
    gam = W.head_gammas(H)
    S = S0.clone().cuda()
    o = ops.recurrent_steps(q.cuda(), k.cuda(), v.cuda(), gam, S)
    ops.check_device_error()
    o_ref, S_ref = _oracle(q, k, v, S0, gam)
    _check(o, o_ref, "bf16", dk, dv, 2, "o", Tn=Tn)
    _check(S, S_ref, "bf16", dk, dv, 1, "state", Tn=Tn)
