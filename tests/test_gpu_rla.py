"""GPU parity of the residual linear attention (retention_rla_fwd) against the
fp64 oracle, through the C ABI.

float32 inputs run on the CUDA-core retention and are held to relative L2 <=
1e-5.  bf16 inputs run on the tensor-core kernels and are held to the
bf16-input tolerance (rel-L2 <= 1e-2, max-abs <= 3e-2 RMS, plus the bf16 store
where the output is stored as bf16) against the oracle's float64 feature map:
the library's bf16 storage of phi(q) and phi(k) is part of the error measured,
not of the reference.
Cases: windows 0, small and the page's 512, the window past a sequence,
packed sequences with empty and one-token ones.
"""

import numpy as np
import pytest
import torch

import oracle
from linear_recurrent_sequence_retention_b200 import ops, workloads as W
from tests._util import assert_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,B,T,H,dk,dv,window", [
    ("f32", 2, 200, 2, 32, 48, 0),
    ("f32", 1, 300, 1, 64, 64, 37),
    ("bf16", 1, 1100, 2, 128, 128, 512),
    ("bf16", 2, 600, 2, 64, 256, 5),
    ("bf16", 1, 300, 1, 256, 512, 299),   # the window covers the whole sequence: zeros
])
def test_rla_matches_oracle(dtype, B, T, H, dk, dv, window):
    q, k, v, _ = W.make_qkvg(B, T, H, dk, dv, dtype, seed=T + window, gate=False)
    ref = oracle.rla(W.to_f64(q), W.to_f64(k), W.to_f64(v), window)
    out = ops.rla_fwd(q.cuda(), k.cuda(), v.cuda(), window, out_dtype=torch.float32)
    if window >= T - 1:
        assert torch.all(out == 0)
        return
    assert_close(W.to_f64(out), ref, dtype, 2, f"rla {dtype} w{window}")


def test_rla_packed_sequences():
    lens = [400, 0, 1, 700, 90]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    Tt = int(cu[-1])
    q, k, v, _ = W.make_qkvg(1, Tt, 2, 64, 128, "bf16", seed=5, gate=False)
    ref = oracle.rla(W.to_f64(q), W.to_f64(k), W.to_f64(v), 64, cu_seqlens=cu)
    out = ops.rla_fwd(q.cuda(), k.cuda(), v.cuda(), 64, cu_seqlens=torch.from_numpy(cu).cuda(),
                      out_dtype=torch.bfloat16)
    assert_close(W.to_f64(out), ref, "bf16", 2, "rla packed", stored_bf16=True)


def test_rla_rejects_negative_window():
    q = torch.zeros(1, 8, 1, 64, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(ops.RetentionError):
        ops.rla_fwd(q, q, q, -1)


def test_rla_bench_workload_sampled():
    """RLA at the size bench.py times (B=4, T=2048, H=8, d_k=128, d_v=256, bf16,
    window 512), checked on two sampled (sequence, head) pairs."""
    B, T, H, dk, dv, w = 4, 2048, 8, 128, 256, 512
    q, k, v, _ = W.make_qkvg(B, T, H, dk, dv, "bf16", seed=0, gate=False)
    out = ops.rla_fwd(q.cuda(), k.cuda(), v.cuda(), w, out_dtype=torch.float32)
    for b, h in ((0, 0), (3, 7)):
        sl = (slice(b, b + 1), slice(None), slice(h, h + 1))
        ref = oracle.rla(W.to_f64(q[sl]), W.to_f64(k[sl]), W.to_f64(v[sl]), w)
        assert_close(W.to_f64(out[sl]), ref, "bf16", None, f"rla bench b{b} h{h}")
