"""The chunkwise forward that allocates nothing (retention_chunkwise_fwd_static_ws).

Some callers cannot call cudaMalloc (they run inside an allocator, under a
fixed device-memory budget, or must not grow their footprint after start-up);
this entry point serves them from scratch compiled into the library.  The
tests call it through the C ABI and compare it with the regular entry point,
which takes a caller-allocated workspace, on the same inputs, within the
tolerance of the other parity tests, on two calls in a row (the second call
finds the first call's leftovers in the shared scratch).  This file is named
to be collected last, and it also passes when run alone in a fresh process.
"""

import ctypes

import numpy as np
import pytest
import torch

from linear_recurrent_sequence_retention_b200 import ops, workloads as W
from tests._util import assert_close

pytestmark = pytest.mark.gpu


def _static_call(q, k, v, gam, chunk, g, out, state_out):
    B, T, H, dk = q.shape
    dv = v.shape[3]
    ng = ops.NormGate(g.data_ptr(), ops._dt(g), None, None, 1e-5) if g is not None else None
    return ops.lib().retention_chunkwise_fwd_static_ws(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
        ops._dt(q), (ctypes.c_double * H)(*[float(x) for x in gam]), chunk, None, 0, None,
        ctypes.c_void_p(state_out.data_ptr()), ctypes.c_void_p(out.data_ptr()), ops._dt(out),
        ctypes.byref(ng) if ng is not None else None, B, T, H, dk, dv,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("dtype,B,T,H,dk,dv,chunk,gated", [
    ("bf16", 1, 700, 2, 128, 256, 256, True),    # tensor-core kernels
    ("f32", 2, 77, 2, 16, 24, 16, False),         # CUDA-core kernels
])
def test_static_workspace_matches_caller_workspace(dtype, B, T, H, dk, dv, chunk, gated):
    assert torch.cuda.is_available()
    need = ops.chunkwise_workspace_size(W.torch_dtype(dtype), chunk, B, T, H, dk, dv)
    assert 0 < need <= ops.STATIC_WORKSPACE_BYTES
    gam = W.head_gammas(H)
    kind = "f32" if dtype == "f32" else "bf16"
    for call in range(2):
        q, k, v, g = W.make_qkvg(B, T, H, dk, dv, dtype, seed=100 + call, gate=gated)
        q, k, v = q.cuda(), k.cuda(), v.cuda()
        g = g.cuda() if gated else None
        ref, S_ref = ops.chunkwise_fwd(q, k, v, gam, chunk, g=g, return_state=True)
        out = torch.empty_like(ref)
        S = torch.empty_like(S_ref)
        st = _static_call(q, k, v, gam, chunk, g, out, S)
        assert st == ops.RET_OK, ops.status_string(st)
        ops.check_device_error()
        assert_close(W.to_f64(out), W.to_f64(ref), kind, 2, f"out call {call}",
                     stored_bf16=out.dtype == torch.bfloat16)
        assert_close(W.to_f64(S), W.to_f64(S_ref), kind, 1, f"state call {call}")


def test_static_workspace_rejects_requests_beyond_capacity():
    assert torch.cuda.is_available()
    B, T, H, dk, dv, chunk = 2, 8192, 16, 256, 512, 512
    assert ops.chunkwise_workspace_size(torch.bfloat16, chunk, B, T, H, dk, dv) > ops.STATIC_WORKSPACE_BYTES
    fake = ctypes.c_void_p(0x10000)      # never dereferenced: the call is rejected up front
    st = ops.lib().retention_chunkwise_fwd_static_ws(
        fake, fake, fake, ops.RET_BF16, (ctypes.c_double * H)(*W.head_gammas(H)), chunk, None, 0,
        None, None, fake, ops.RET_BF16, None, B, T, H, dk, dv, None)
    assert st == ops.RET_ERR_WORKSPACE
