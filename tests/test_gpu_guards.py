"""Poisoned padding: every output is a view into a larger buffer whose guard
bytes before and after it hold a sentinel pattern; after the call the guard
bytes must be untouched (no kernel writes outside its output, including the
ragged last tile, packed sequence ends and TMA-stored tiles).
"""

import pytest
import torch

from linear_recurrent_sequence_retention_b200 import ops, workloads as W

pytestmark = pytest.mark.gpu

GUARD = 4096                      # bytes of sentinel on each side
SENTINEL = 0xA5


def guarded(shape, dtype):
    """(view, backing buffer) with GUARD sentinel bytes on both sides of the view."""
    n = 1
    for d in shape:
        n *= d
    esz = torch.empty(0, dtype=dtype).element_size()
    buf = torch.full((GUARD * 2 + n * esz,), SENTINEL, dtype=torch.uint8, device="cuda")
    view = buf[GUARD:GUARD + n * esz].view(dtype).view(*shape)
    return view, buf


def assert_guards(buf, what):
    head, tail = buf[:GUARD], buf[-GUARD:]
    assert bool((head == SENTINEL).all()), f"{what}: bytes written before the output"
    assert bool((tail == SENTINEL).all()), f"{what}: bytes written after the output"


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("gated", [False, True])
@pytest.mark.parametrize("dk,dv,chunk,T", [(128, 128, 128, 333), (256, 512, 512, 700),
                                           (128, 256, 256, 129), (64, 256, 128, 200)])
def test_chunkwise_tc_writes_only_its_outputs(out_dtype, gated, dk, dv, chunk, T):
    B, H = 2, 2
    q, k, v, g = W.make_qkvg(B, T, H, dk, dv, "bf16", seed=dk + T, gate=gated, device="cuda")
    out, ob = guarded((B, T, H, dv), out_dtype)
    S, sb = guarded((B, H, dk, dv), torch.float32)
    ops.chunkwise_fwd(q, k, v, W.head_gammas(H), chunk, g=g, out=out, state_out=S)
    ops.check_device_error()
    assert_guards(ob, "out")
    assert_guards(sb, "state_out")
    assert bool(torch.isfinite(out.float()).all())


def test_chunkwise_tc_varlen_writes_only_its_outputs():
    lens = [200, 0, 1, 129, 511]
    cu = torch.from_numpy(W.cu_seqlens_of(lens)).cuda()
    Tt = sum(lens)
    H, dk, dv, chunk = 2, 128, 256, 128
    q, k, v, g = W.make_qkvg(1, Tt, H, dk, dv, "bf16", seed=3, device="cuda")
    out, ob = guarded((1, Tt, H, dv), torch.bfloat16)
    S, sb = guarded((len(lens), H, dk, dv), torch.float32)
    ops.chunkwise_fwd(q, k, v, W.head_gammas(H), chunk, cu_seqlens=cu, g=g, out=out, state_out=S)
    ops.check_device_error()
    assert_guards(ob, "out")
    assert_guards(sb, "state_out")


def test_fp32_chunkwise_writes_only_its_outputs():
    B, T, H, dk, dv, chunk = 1, 77, 2, 32, 48, 16
    q, k, v, _ = W.make_qkvg(B, T, H, dk, dv, "f32", seed=5, gate=False, device="cuda")
    out, ob = guarded((B, T, H, dv), torch.float32)
    ops.chunkwise_fwd(q, k, v, W.head_gammas(H), chunk, out=out)
    ops.check_device_error()
    assert_guards(ob, "out")


def test_decode_writes_only_its_outputs():
    N, H, dk, dv = 3, 2, 256, 512
    q, k, v = W.make_step_inputs(N, H, dk, dv, "bf16", seed=2, device="cuda")
    S, sb = guarded((N, H, dk, dv), torch.float32)
    S.copy_(W.make_state(N, H, dk, dv, seed=4, scale=0.05).cuda())
    o, obuf = guarded((N, H, dv), torch.float32)
    ops.recurrent_step(q, k, v, W.head_gammas(H), S, out=o)
    ops.check_device_error()
    assert_guards(sb, "state")
    assert_guards(obuf, "o")


def test_norm_gate_writes_only_its_outputs():
    ntok, H, dv = 37, 3, 256
    o = torch.randn(ntok, H, dv, device="cuda")
    g = torch.randn(ntok, H * dv, device="cuda").to(torch.bfloat16)
    y, yb = guarded((ntok, H, dv), torch.bfloat16)
    ops.norm_gate(o, g, out=y)
    ops.check_device_error()
    assert_guards(yb, "y")
