"""GPU parity of the rotary position encoding (retention_rope) against the
fp64 oracle, through the C ABI.

float32: relative error per element <= 1e-6 of the row's largest entry (the
angle is reduced modulo 2 pi in double precision, the rotation is float32).
bfloat16: the kernel rounds its float32 rotation to nearest once, the oracle
rounds its float64 rotation the same way; the two may only differ where the
exact value lies within float32 error of a rounding boundary, by one bf16 unit
in the last place (or, where x0 cos - x1 sin cancels to nearly zero, by the
float32 error itself, 1e-6 of the row's scale), so every element is checked
against that and the number of differing elements must be tiny.  Cases: long sequences (large
angles), packed sequences (positions restart), in-place rotation, odd head
counts.
"""

import numpy as np
import pytest
import torch

import oracle
from linear_recurrent_sequence_retention_b200 import ops, workloads as W

pytestmark = pytest.mark.gpu


def _bf16_round(x64):
    return torch.from_numpy(x64).to(torch.float32).to(torch.bfloat16).double().numpy()


def _check(got, ref64, dtype, what):
    g = W.to_f64(got)
    if dtype == "f32":
        scale = np.abs(ref64).max(axis=-1, keepdims=True) + 1e-30
        err = np.abs(g - ref64) / scale
        assert err.max() <= 1e-6, f"{what}: max err {err.max():.3e}"
    else:
        r = _bf16_round(ref64)
        # one bf16 unit of the rounded value, plus the float32 rotation's own error
        # (relative to the row's scale: it shows where x0 c - x1 s cancels)
        row = np.abs(ref64).max(axis=-1, keepdims=True)
        ulp = np.abs(r) * 2.0 ** -7 + 1e-6 * row
        diff = np.abs(g - r)
        assert np.all(diff <= ulp), f"{what}: {np.sum(diff > ulp)} elements off by more than one ulp"
        frac = float(np.mean(diff > 0))
        assert frac <= 1e-3, f"{what}: {frac:.2e} of the elements differ from the rounded oracle"


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("B,T,H,d,base", [
    (2, 9000, 3, 64, 10000.0),     # positions up to 8999: large angles
    (1, 300, 16, 256, 10000.0),
    (3, 17, 1, 2, 500.0),          # one pair per head
])
def test_rope_matches_oracle(dtype, B, T, H, d, base):
    q, k, _, _ = W.make_qkvg(B, T, H, d, 8, dtype, seed=T + d, gate=False)
    rq, rk = ops.rope(q.cuda(), k.cuda(), base=base)
    _check(rq, oracle.rope(W.to_f64(q), base), dtype, "q")
    _check(rk, oracle.rope(W.to_f64(k), base), dtype, "k")


def test_rope_packed_and_in_place():
    lens = [700, 0, 1, 4000, 33]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    Tt = int(cu[-1])
    q, k, _, _ = W.make_qkvg(1, Tt, 2, 128, 8, "bf16", seed=3, gate=False)
    qd, kd = q.cuda(), k.cuda()
    ops.rope(qd, kd, cu_seqlens=torch.from_numpy(cu).cuda(), q_out=qd, k_out=kd)
    _check(qd, oracle.rope(W.to_f64(q), cu_seqlens=cu), "bf16", "q packed in place")
    _check(kd, oracle.rope(W.to_f64(k), cu_seqlens=cu), "bf16", "k packed in place")


def test_rope_rejects_bad_arguments():
    q = torch.zeros(1, 4, 1, 7, device="cuda")       # odd head dimension
    with pytest.raises(ops.RetentionError):
        ops.rope(q, q.clone())
    q = torch.zeros(1, 4, 1, 8, device="cuda")
    with pytest.raises(ops.RetentionError):
        ops.rope(q, q.clone(), base=1.0)


def test_rope_bench_workload():
    """The rotary encoding at the size bench.py times: q, k [2, 8192, 16, 256] bf16."""
    q, k, _, _ = W.make_qkvg(2, 8192, 16, 256, 8, "bf16", seed=0, gate=False)
    rq, rk = ops.rope(q.cuda(), k.cuda())
    _check(rq, oracle.rope(W.to_f64(q)), "bf16", "q full size")
    _check(rk, oracle.rope(W.to_f64(k)), "bf16", "k full size")
