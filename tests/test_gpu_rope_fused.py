"""GPU parity of the chunkwise forward with the rotary position encoding in
the same call (retention_chunkwise_fwd_rope), through the C ABI.

Two checks per case:
- bit for bit against the two-call route, retention_rope followed by
  retention_chunkwise_fwd on the caller's buffers (the one-call entry keeps
  its rotated copies in the workspace);
- against the fp64 oracle, rope of q and k (the standard rotary form applied
  after the projections, abeam.tech summary of the RetNet paper) rounded to
  bf16, followed by the chunkwise form and, when gated, the GroupNorm + swish
  gate, at the bf16 tolerance with float32 outputs.  The rotated operands are
  bf16 on both routes (the input precision), and that rounding is part of the
  computation: without it the reference differs from itself by up to
  5.5e-2 * RMS on the gated output of the 6.7B head shape, where the plain
  bound is 3e-2.  The rotation itself is pinned separately (the rotary
  parity test: the kernel's bf16 values equal the rounded oracle's but for
  rare one-unit differences at rounding boundaries).
Cases: the 6.7B head shape (d_k 256, d_v 512, chunk 512) with a ragged tail,
an incoming state with bf16 output, positions up to 9000 (large angles), and
packed sequences whose positions restart at each sequence.
"""

import numpy as np
import pytest
import torch

import oracle
from linear_recurrent_sequence_retention_b200 import ops, workloads as W
from tests._util import assert_close

pytestmark = pytest.mark.gpu

f64 = W.to_f64
BASE = 10000.0


def _rot(x, cu=None):
    """Oracle rotation of a bf16 tensor, rounded to bf16 like the stored operands."""
    r = oracle.rope(f64(x), BASE, cu_seqlens=cu)
    return torch.from_numpy(r).to(torch.float32).to(torch.bfloat16).double().numpy()


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    ops.check_device_error()


def _both_routes(q, k, v, gam, chunk, cu=None, s0=None, g=None, out_dtype=torch.float32):
    kw = dict(cu_seqlens=cu, state_in=s0, g=g, return_state=True, out_dtype=out_dtype)
    y_fused, S_fused = ops.chunkwise_fwd(q, k, v, gam, chunk, rope_base=BASE, **kw)
    q_rot, k_rot = ops.rope(q, k, base=BASE, cu_seqlens=cu)
    y_sep, S_sep = ops.chunkwise_fwd(q_rot, k_rot, v, gam, chunk, **kw)
    ops.check_device_error()
    return y_fused, S_fused, y_sep, S_sep


@pytest.mark.parametrize("B,T,H,dk,dv,chunk,gated", [
    (2, 2 * 512 + 77, 2, 256, 512, 512, True),
    (2, 2 * 128 + 77, 3, 128, 256, 128, False),
    (1, 9000, 1, 128, 128, 256, True),
    (1, 300, 2, 64, 128, 128, True),
])
def test_fused_rope_matches_oracle(B, T, H, dk, dv, chunk, gated):
    q, k, v, g = W.make_qkvg(B, T, H, dk, dv, "bf16", seed=dk + dv + T)
    gam = W.head_gammas(H)
    o_ref, S_ref = oracle.msr_chunkwise(_rot(q), _rot(k), f64(v), gam, chunk)
    ref = oracle.norm_gate(o_ref, f64(g).reshape(B, T, H, dv)) if gated else o_ref
    y, S, y_sep, S_sep = _both_routes(q.cuda(), k.cuda(), v.cuda(), gam, chunk,
                                      g=g.cuda() if gated else None)
    assert torch.equal(y, y_sep), "fused and unfused rotary routes differ"
    assert torch.equal(S, S_sep), "fused and unfused rotary routes differ (state)"
    assert_close(f64(y), ref, "bf16", 2, "out")
    assert_close(f64(S), S_ref, "bf16", 1, "state_out")


def test_fused_rope_state_in_bf16_out():
    B, T, H, dk, dv, chunk = 2, 700, 3, 128, 256, 256
    q, k, v, g = W.make_qkvg(B, T, H, dk, dv, "bf16", seed=5)
    gam = W.head_gammas(H)
    s0 = W.make_state(B, H, dk, dv, seed=12, scale=0.05)
    o_ref, S_ref = oracle.msr_chunkwise(_rot(q), _rot(k), f64(v), gam, chunk, f64(s0))
    ref = oracle.norm_gate(o_ref, f64(g).reshape(B, T, H, dv))
    y, S, y_sep, S_sep = _both_routes(q.cuda(), k.cuda(), v.cuda(), gam, chunk, s0=s0.cuda(),
                                      g=g.cuda(), out_dtype=torch.bfloat16)
    assert torch.equal(y, y_sep) and torch.equal(S, S_sep)
    assert_close(f64(y), ref, "bf16", 2, "y", stored_bf16=True)
    assert_close(f64(S), S_ref, "bf16", 1, "state_out")


def test_fused_rope_packed_positions_restart():
    lens = [700, 0, 1, 300, 129, 33]
    cu = W.cu_seqlens_of(lens)
    Tt = int(cu[-1])
    H, dk, dv, chunk = 2, 128, 128, 128
    q, k, v, g = W.make_qkvg(1, Tt, H, dk, dv, "bf16", seed=21)
    gam = W.head_gammas(H)
    s0 = W.make_state(len(lens), H, dk, dv, seed=8, scale=0.05)
    o_ref, S_ref = oracle.msr_chunkwise_varlen(_rot(q, cu), _rot(k, cu), f64(v), gam, chunk, cu,
                                               f64(s0))
    ref = oracle.norm_gate(o_ref, f64(g).reshape(1, Tt, H, dv))
    y, S, y_sep, S_sep = _both_routes(q.cuda(), k.cuda(), v.cuda(), gam, chunk,
                                      cu=torch.from_numpy(cu).cuda(), s0=s0.cuda(), g=g.cuda())
    assert torch.equal(y, y_sep) and torch.equal(S, S_sep)
    assert_close(f64(y), ref, "bf16", 2, "y")
    assert_close(f64(S), S_ref, "bf16", 1, "state_out")


def test_fused_rope_leaves_inputs_and_rejects_bad_arguments():
    q, k, v, _ = W.make_qkvg(1, 200, 2, 128, 128, "bf16", seed=1, gate=False)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    ops.chunkwise_fwd(qd, kd, vd, W.head_gammas(2), 128, rope_base=BASE)
    assert torch.equal(qd.cpu(), q) and torch.equal(kd.cpu(), k)
    with pytest.raises(ops.RetentionError):
        ops.chunkwise_fwd(qd, kd, vd, W.head_gammas(2), 128, rope_base=1.0)
    with pytest.raises(ops.RetentionError):
        ops.chunkwise_fwd(qd.float(), kd.float(), vd.float(), W.head_gammas(2), 128,
                          rope_base=BASE)
    need = ops.chunkwise_fwd_rope_workspace_size(128, 1, 200, 2, 128, 128)
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(ops.RetentionError):
        ops.chunkwise_fwd(qd, kd, vd, W.head_gammas(2), 128, rope_base=BASE, workspace=small)
