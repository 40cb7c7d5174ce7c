"""GPU parity of the tensor-core chunkwise forward (bf16 in, f32 accumulate)
against the fp64 oracle, through the C ABI.

Tolerance (bf16 inputs): relative L2 <= 1e-2 and max-abs <= 3e-2 * RMS, over
the whole output and per head; float32 outputs are checked against exactly
that bound, bf16-stored outputs additionally allow the store's own rounding
(see tests/_util.py).  Sizes span several 128-row tiles, several chunks and a
ragged tail; the packed cases include empty, one-token and sub-tile
sequences.
"""

import numpy as np
import pytest
import torch

import oracle
from linear_recurrent_sequence_retention_b200 import ops, workloads as W
from tests._util import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    ops.check_device_error()


f64 = W.to_f64


def _run(B, T, H, dk, dv, chunk, gated, out_dtype, state_in=False, seed=0, gam=None):
    q, k, v, g = W.make_qkvg(B, T, H, dk, dv, "bf16", seed=seed)
    gam = W.head_gammas(H) if gam is None else np.asarray(gam)
    s0 = W.make_state(B, H, dk, dv, seed=seed + 7, scale=0.05) if state_in else None
    o_ref, S_ref = oracle.msr_chunkwise(f64(q), f64(k), f64(v), gam, chunk,
                                        None if s0 is None else f64(s0))
    ref = oracle.norm_gate(o_ref, f64(g).reshape(B, T, H, dv)) if gated else o_ref
    out, S = ops.chunkwise_fwd(q.cuda(), k.cuda(), v.cuda(), gam, chunk,
                               state_in=None if s0 is None else s0.cuda(),
                               g=g.cuda() if gated else None, return_state=True,
                               out_dtype=out_dtype)
    ops.check_device_error()
    return out, S, ref, S_ref


@pytest.mark.parametrize("dk,dv,chunk", [
    (128, 64, 128), (128, 128, 128), (128, 256, 128), (128, 256, 256),
    (256, 256, 512), (256, 512, 512), (256, 512, 128), (128, 512, 256), (256, 64, 256),
    (64, 128, 128), (64, 512, 256), (64, 64, 512),
])
@pytest.mark.parametrize("gated", [False, True])
def test_shapes_f32_out(dk, dv, chunk, gated):
    B, H = 2, 2
    T = 2 * chunk + 77                     # several chunks and a ragged tail
    out, S, ref, S_ref = _run(B, T, H, dk, dv, chunk, gated, torch.float32, seed=dk + dv + chunk)
    assert_close(f64(out), ref, "bf16", 2, "out")
    assert_close(f64(S), S_ref, "bf16", 1, "state_out")


@pytest.mark.parametrize("gated", [False, True])
def test_bf16_out_and_state_in(gated):
    B, T, H, dk, dv, chunk = 2, 700, 3, 128, 256, 256
    out, S, ref, S_ref = _run(B, T, H, dk, dv, chunk, gated, torch.bfloat16, state_in=True, seed=3)
    assert_close(f64(out), ref, "bf16", 2, "out", stored_bf16=True)
    assert_close(f64(S), S_ref, "bf16", 1, "state_out")


@pytest.mark.parametrize("T", [1, 5, 127, 128, 129])
def test_short_sequences(T):
    out, S, ref, S_ref = _run(1, T, 2, 128, 128, 128, False, torch.float32, seed=T)
    assert_close(f64(out), ref, "bf16", 2, "out")
    assert_close(f64(S), S_ref, "bf16", 1, "state_out")


def test_chunk_64_equals_oracle_chunk_64():
    """chunk = 64 is accepted (evaluated with 128-token tiles; same result)."""
    out, S, ref, S_ref = _run(1, 333, 2, 128, 128, 64, True, torch.float32, seed=11)
    assert_close(f64(out), ref, "bf16", 2, "out")
    assert_close(f64(S), S_ref, "bf16", 1, "state_out")


def test_gamma_extremes():
    """gamma = 0 (diagonal only) and gamma = 1 (no decay) heads."""
    out, S, ref, S_ref = _run(1, 600, 2, 128, 128, 256, False, torch.float32, seed=5,
                              gam=[0.0, 1.0])
    assert_close(f64(out), ref, "bf16", 2, "out")
    assert_close(f64(S), S_ref, "bf16", 1, "state_out")


def test_chunk_length_invariance_bf16():
    B, T, H, dk, dv = 1, 1024, 2, 128, 128
    q, k, v, _ = W.make_qkvg(B, T, H, dk, dv, "bf16", seed=8, gate=False)
    gam = W.head_gammas(H)
    ref = oracle.msr_parallel(f64(q), f64(k), f64(v), gam)
    for chunk in (64, 128, 256, 512):
        o = ops.chunkwise_fwd(q.cuda(), k.cuda(), v.cuda(), gam, chunk, out_dtype=torch.float32)
        assert_close(f64(o), ref, "bf16", 2, f"chunk={chunk}")


@pytest.mark.parametrize("dk", [128, 64])
def test_varlen_packed(dk):
    lens = [300, 0, 1, 77, 128, 129, 513, 64]
    cu = W.cu_seqlens_of(lens)
    H, dv, chunk = 2, 128, 128
    Tt = int(cu[-1])
    q, k, v, g = W.make_qkvg(1, Tt, H, dk, dv, "bf16", seed=13)
    gam = W.head_gammas(H)
    s0 = W.make_state(len(lens), H, dk, dv, seed=2, scale=0.05)
    o_ref, S_ref = oracle.msr_chunkwise_varlen(f64(q), f64(k), f64(v), gam, chunk, cu, f64(s0))
    y_ref = oracle.norm_gate(o_ref, f64(g).reshape(1, Tt, H, dv))
    y, S = ops.chunkwise_fwd(q.cuda(), k.cuda(), v.cuda(), gam, chunk,
                             cu_seqlens=torch.from_numpy(cu).cuda(), state_in=s0.cuda(),
                             g=g.cuda(), return_state=True, out_dtype=torch.float32)
    ops.check_device_error()
    assert_close(f64(y), y_ref, "bf16", 2, "y")
    assert_close(f64(S), S_ref, "bf16", 1, "state_out")
    np.testing.assert_array_equal(f64(S)[1], f64(s0)[1])     # empty sequence


def test_repeat_calls_identical():
    """Two calls on the same inputs give bit-identical outputs (no stale workspace use)."""
    B, T, H, dk, dv, chunk = 1, 900, 2, 128, 256, 256
    q, k, v, g = W.make_qkvg(B, T, H, dk, dv, "bf16", seed=4)
    gam = W.head_gammas(H)
    args = (q.cuda(), k.cuda(), v.cuda(), gam, chunk)
    ws = torch.full((ops.chunkwise_workspace_size(torch.bfloat16, chunk, B, T, H, dk, dv),),
                    255, dtype=torch.uint8, device="cuda")
    y1 = ops.chunkwise_fwd(*args, g=g.cuda(), workspace=ws)
    ws.fill_(7)
    y2 = ops.chunkwise_fwd(*args, g=g.cuda(), workspace=ws)
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("varlen", [False, True])
def test_phase_calls_equal_fused_call(varlen):
    """retention_chunkwise_states + retention_chunkwise_outputs == retention_chunkwise_fwd."""
    H, dk, dv, chunk = 2, 128, 256, 128
    if varlen:
        cu = torch.from_numpy(W.cu_seqlens_of([200, 0, 333])).cuda()
        B, T = 1, 533
    else:
        cu, B, T = None, 2, 400
    q, k, v, g = W.make_qkvg(B, T, H, dk, dv, "bf16", seed=17)
    q, k, v, g = q.cuda(), k.cuda(), v.cuda(), g.cuda()
    nst = 3 if varlen else B
    s0 = W.make_state(nst, H, dk, dv, seed=1, scale=0.05).cuda()
    gam = W.head_gammas(H)
    y1, S1 = ops.chunkwise_fwd(q, k, v, gam, chunk, cu_seqlens=cu, state_in=s0, g=g,
                               return_state=True)
    S2 = torch.empty_like(S1)
    ws = ops.chunkwise_states(k, v, gam, chunk, cu_seqlens=cu, state_in=s0, state_out=S2)
    y2 = ops.chunkwise_outputs(q, k, v, gam, chunk, ws, cu_seqlens=cu, has_state_in=True, g=g)
    ops.check_device_error()
    assert torch.equal(y1, y2)
    assert torch.equal(S1, S2)

