"""GPU parity of the tensor-core parallel form (retention_parallel_fwd, bf16
inputs) against the fp64 oracle's parallel form (Q K^T * D) V, through the C
ABI.

Tolerance as for the tensor-core chunkwise path: relative L2 <= 1e-2 and
max-abs <= 3e-2 * RMS, over the whole output and per head, on float32
outputs; bf16-stored outputs add the store's own rounding.  Cases span one
and many 128-row tiles with a ragged tail, T = 1, every supported (d_k, d_v)
pair, the head shapes of the two bench workloads (128/256 at T = 2048 in
full; 256/512 at T = 8192 on sampled (b, h) pairs, checked one pair at a time
against the oracle), and the gamma = 0 and gamma = 1 extremes.
"""

import numpy as np
import pytest
import torch

import oracle
from linear_recurrent_sequence_retention_b200 import ops, workloads as W
from tests._util import assert_close

pytestmark = pytest.mark.gpu

f64 = W.to_f64


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    ops.check_device_error()


def _run(B, T, H, dk, dv, out_dtype, seed, gam=None):
    q, k, v, _ = W.make_qkvg(B, T, H, dk, dv, "bf16", seed=seed, gate=False)
    gam = W.head_gammas(H) if gam is None else np.asarray(gam, dtype=np.float64)
    ref = oracle.msr_parallel(f64(q), f64(k), f64(v), gam)
    assert ops.parallel_workspace_size(torch.bfloat16, B, T, H, dk, dv) > 0
    o = ops.parallel_fwd(q.cuda(), k.cuda(), v.cuda(), gam, out_dtype=out_dtype)
    ops.check_device_error()
    return o, ref


@pytest.mark.parametrize("dk,dv", [
    (64, 64), (64, 512), (128, 128), (128, 256), (128, 512), (256, 64), (256, 256), (256, 512),
])
def test_head_dims_f32_out(dk, dv):
    T = 3 * 128 + 45                          # several row blocks and a ragged tail
    o, ref = _run(2, T, 2, dk, dv, torch.float32, seed=dk + dv)
    assert_close(f64(o), ref, "bf16", 2, "o")


@pytest.mark.parametrize("T", [1, 5, 127, 128, 129, 1000])
def test_lengths(T):
    o, ref = _run(2, T, 3, 128, 256, torch.float32, seed=T)
    assert_close(f64(o), ref, "bf16", 2, "o")


def test_bf16_out():
    o, ref = _run(2, 700, 2, 256, 512, torch.bfloat16, seed=9)
    assert_close(f64(o), ref, "bf16", 2, "o", stored_bf16=True)


def test_gamma_extremes():
    """gamma = 0 keeps only the diagonal term; gamma = 1 is plain causal linear attention."""
    o, ref = _run(1, 600, 3, 128, 128, torch.float32, seed=2, gam=[0.0, 1.0, 0.5])
    assert_close(f64(o), ref, "bf16", 2, "o")


def test_long_sequence():
    """Positions up to 6000: decays over the whole range, 47 row blocks."""
    o, ref = _run(1, 6000, 2, 128, 128, torch.float32, seed=4, gam=[1 - 2.0 ** -5, 1 - 2.0 ** -12])
    assert_close(f64(o), ref, "bf16", 2, "o")


def test_cfg2_heads_full():
    """The B=4, T=2048, H=8, d_k=128, d_v=256 workload in full."""
    wl = W.WORKLOADS["msr_b4_h8_t2048_dk128_dv256_c128"]
    o, ref = _run(wl.B, wl.T, wl.H, wl.dk, wl.dv, torch.float32, seed=0)
    assert_close(f64(o), ref, "bf16", 2, "o")


def test_6p7b_heads_t8192_sampled():
    """The 6.7B head shape at T = 8192, B=2, H=16: the whole output on the GPU,
    the oracle on sampled (b, h) pairs (each an independent sequence)."""
    wl = W.WORKLOADS["msr_6p7b_b2_h16_t8192_dk256_dv512_c512"]
    B, T, H, dk, dv = wl.B, wl.T, wl.H, wl.dk, wl.dv
    q, k, v, _ = W.make_qkvg(B, T, H, dk, dv, "bf16", seed=0, gate=False)
    gam = W.head_gammas(H)
    o = ops.parallel_fwd(q.cuda(), k.cuda(), v.cuda(), gam, out_dtype=torch.float32).cpu()
    ops.check_device_error()
    for b, h in ((0, 0), (1, 15), (1, 6)):
        ref = oracle.msr_parallel(f64(q[b:b + 1, :, h:h + 1]), f64(k[b:b + 1, :, h:h + 1]),
                                  f64(v[b:b + 1, :, h:h + 1]), gam[h:h + 1])
        assert_close(f64(o[b:b + 1, :, h:h + 1]), ref, "bf16", None, f"b={b} h={h}")


def test_matches_chunkwise_form():
    """The parallel and chunkwise tensor-core forms agree (the pages state the
    forms give the same values) to within the bf16 bound of each other."""
    B, T, H, dk, dv = 2, 1500, 2, 128, 256
    q, k, v, _ = W.make_qkvg(B, T, H, dk, dv, "bf16", seed=6, gate=False)
    gam = W.head_gammas(H)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o_par = ops.parallel_fwd(qd, kd, vd, gam, out_dtype=torch.float32)
    o_chk = ops.chunkwise_fwd(qd, kd, vd, gam, 256, out_dtype=torch.float32)
    ref = oracle.msr_parallel(f64(q), f64(k), f64(v), gam)
    assert_close(f64(o_par), ref, "bf16", 2, "parallel")
    assert_close(f64(o_chk), ref, "bf16", 2, "chunkwise")
    assert_close(f64(o_par), f64(o_chk), "bf16", 2, "parallel vs chunkwise")


def test_range_error_reported():
    B, T, H, dk, dv = 1, 300, 1, 128, 128
    q, k, v, _ = W.make_qkvg(B, T, H, dk, dv, "bf16", seed=1, gate=False)
    v[0, 17, 0, 5] = 1e5                       # no fp16 image
    ops.parallel_fwd(q.cuda(), k.cuda(), v.cuda(), [0.9])
    with pytest.raises(ops.RetentionError) as e:
        ops.check_device_error()
    assert e.value.status == ops.RET_ERR_RANGE


def test_repeat_calls_identical_and_workspace_contents_ignored():
    B, T, H, dk, dv = 1, 900, 2, 256, 512
    q, k, v, _ = W.make_qkvg(B, T, H, dk, dv, "bf16", seed=8, gate=False)
    gam = W.head_gammas(H)
    args = (q.cuda(), k.cuda(), v.cuda(), gam)
    ws = torch.full((ops.parallel_workspace_size(torch.bfloat16, B, T, H, dk, dv),), 255,
                    dtype=torch.uint8, device="cuda")
    o1 = ops.parallel_fwd(*args, workspace=ws)
    ws.fill_(7)
    o2 = ops.parallel_fwd(*args, workspace=ws)
    assert torch.equal(o1, o2)
