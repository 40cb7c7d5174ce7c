"""GPU parity of the chunkwise backward (retention_chunkwise_bwd) against the
fp64 oracle's gradients, through the C ABI.

On the CUDA-core path the kernels compute every product and sum in float32
from inputs that are exact (float32, or bfloat16 widened exactly), so both
input dtypes are held to the float32 tolerance: relative L2 <= 1e-5 over each
gradient, whole and per head.  bf16 inputs with d_k in 64/128/256 and d_v in
64/128/256/512 run on the tensor-core kernels instead (the causal and
anti-causal forward retentions) and are held to the bf16-input tolerance (plus rel-L2 <= 1e-3
as a precision check: their computed MMA operands are fp16, unit roundoff
2^-11, which gives ~3e-4; operands rounded to bf16 alone would give ~2e-3).  Cases
span several chunks with ragged tails, chunk lengths of one token and longer
than the sequence, the largest supported heads, gamma = 0 and gamma = 1, an
initial state and an upstream state gradient, and packed sequences including
empty ones.  d_v = 512 (the 6.7B head shape) runs on the tensor cores only,
with the two retentions that contract over d_v split into halves; it is
checked at small sizes and on a sampled (sequence, head) pair at T = 8192.
"""

import numpy as np
import pytest
import torch

import oracle
from linear_recurrent_sequence_retention_b200 import ops, workloads as W
from tests._util import assert_close, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.init()
    yield
    ops.check_device_error()


def _inputs(B, T, H, dk, dv, dtype, seed, with_state):
    q, k, v, _ = W.make_qkvg(B, T, H, dk, dv, dtype, seed=seed, gate=False)
    g = torch.Generator().manual_seed(seed + 7)
    do = torch.randn(B, T, H, dv, generator=g).to(W.torch_dtype(dtype))
    S0 = torch.randn(B, H, dk, dv, generator=g) if with_state else None
    dS = torch.randn(B, H, dk, dv, generator=g) if with_state else None
    return q, k, v, do, S0, dS


def _tensor_core(dtype, dk, dv, gammas, with_dS):
    """Whether the call runs on the tensor-core path (the rule of the C ABI)."""
    heads = (64, 128, 256)
    return dtype == "bf16" and dk in heads and dv in heads + (512,)


def _check(got, ref, H, what, tc=False):
    names = ("dq", "dk", "dv", "d_state_in")
    for x, y, n in zip(got, ref, names):
        if x is None:
            continue
        axis = 2 if n != "d_state_in" else 1
        if tc:
            assert_close(W.to_f64(x), y, "bf16", axis, f"{what} {n}")
            assert rel_l2(W.to_f64(x), y) <= 1e-3, (what, n, rel_l2(W.to_f64(x), y))
        else:
            assert_close(W.to_f64(x), y, "f32", axis, f"{what} {n}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("B,T,H,dk,dv,chunk,with_state", [
    (2, 77, 2, 16, 24, 16, True),      # several chunks, ragged tail, dk != dv
    (1, 37, 2, 8, 8, 1, False),        # one-token chunks
    (1, 9, 1, 16, 16, 64, True),       # chunk longer than the sequence
    (1, 300, 3, 64, 128, 64, True),    # wider heads, several tiles
    (1, 130, 1, 256, 256, 128, True),  # largest supported heads
])
def test_backward_matches_oracle(dtype, B, T, H, dk, dv, chunk, with_state):
    q, k, v, do, S0, dS = _inputs(B, T, H, dk, dv, dtype, seed=T + dk, with_state=with_state)
    gam = W.head_gammas(H)
    ref = oracle.msr_backward(W.to_f64(q), W.to_f64(k), W.to_f64(v), gam, W.to_f64(do),
                              None if S0 is None else S0.double().numpy(),
                              None if dS is None else dS.double().numpy())
    got = ops.chunkwise_bwd(q.cuda(), k.cuda(), v.cuda(), do.cuda(), gam, chunk,
                            state_in=None if S0 is None else S0.cuda(),
                            d_state_out=None if dS is None else dS.cuda(), return_d_state=True)
    _check(got, ref, H, f"{dtype} B{B} T{T} dk{dk} dv{dv} C{chunk}",
           _tensor_core(dtype, dk, dv, gam, dS is not None))


@pytest.mark.parametrize("B,T,H,dk,dv,chunk,with_state", [
    (2, 300, 2, 64, 128, 128, True),     # several chunks and tiles, initial state
    (1, 700, 1, 128, 256, 64, False),    # 64-token chunks executed as 256
    (1, 200, 2, 256, 64, 256, True),     # d_k > d_v
    (1, 1030, 2, 128, 128, 512, False),  # 512-token chunks, ragged last chunk
])
@pytest.mark.parametrize("use_dS", [False, True])
def test_backward_tensor_core_path(B, T, H, dk, dv, chunk, with_state, use_dS):
    """bf16 inputs with heads of 64/128/256 run on the tensor-core forward kernels
    (three retentions: dQ causal, dV and dK anti-causal, a final-state gradient
    entering those two as the state after the last chunk); held to the
    bf16-input tolerance and, as a precision check, rel-L2 <= 1e-3."""
    q, k, v, do, S0, dS = _inputs(B, T, H, dk, dv, "bf16", seed=T + 3 * dk, with_state=True)
    S0 = S0 if with_state else None
    dS = dS if use_dS else None
    gam = W.head_gammas(H)
    assert _tensor_core("bf16", dk, dv, gam, use_dS)
    ref = oracle.msr_backward(W.to_f64(q), W.to_f64(k), W.to_f64(v), gam, W.to_f64(do),
                              None if S0 is None else S0.double().numpy(),
                              None if dS is None else dS.double().numpy())
    got = ops.chunkwise_bwd(q.cuda(), k.cuda(), v.cuda(), do.cuda(), gam, chunk,
                            state_in=None if S0 is None else S0.cuda(),
                            d_state_out=None if dS is None else dS.cuda(), return_d_state=True)
    _check(got, ref, H, f"tc T{T} dk{dk} dv{dv} dS={use_dS}", tc=True)


@pytest.mark.parametrize("use_dS", [False, True])
def test_backward_tensor_core_packed(use_dS):
    """The tensor-core path on packed sequences (the anti-causal walk runs inside
    each sequence; an empty sequence passes dS_T straight to its initial-state
    gradient)."""
    lens = [300, 0, 1, 129, 64]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    Tt = int(cu[-1])
    H, dk, dv, chunk = 2, 64, 64, 64
    q, k, v, do, _, _ = _inputs(1, Tt, H, dk, dv, "bf16", seed=21, with_state=False)
    g = torch.Generator().manual_seed(22)
    S0 = torch.randn(len(lens), H, dk, dv, generator=g)
    dS = torch.randn(len(lens), H, dk, dv, generator=g) if use_dS else None
    gam = W.head_gammas(H)
    ref = oracle.msr_backward_varlen(W.to_f64(q), W.to_f64(k), W.to_f64(v), gam, W.to_f64(do),
                                     cu, S0.double().numpy(),
                                     None if dS is None else dS.double().numpy())
    got = ops.chunkwise_bwd(q.cuda(), k.cuda(), v.cuda(), do.cuda(), gam, chunk,
                            cu_seqlens=torch.from_numpy(cu).cuda(), state_in=S0.cuda(),
                            d_state_out=None if dS is None else dS.cuda(), return_d_state=True)
    _check(got, ref, H, f"tc packed dS={use_dS}", tc=True)


@pytest.mark.parametrize("gammas", [[0.0, 0.96875], [1.0, 0.0]])
def test_backward_tensor_core_zero_and_unit_decay(gammas):
    """gamma = 0 heads on the tensor-core path with a final-state gradient: the
    state gradient reaches only the last token of each sequence (and, for an
    empty sequence, the initial-state gradient); gamma = 1 carries it to every
    token undecayed."""
    lens = [130, 0, 1, 65]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    Tt = int(cu[-1])
    H, dk, dv, chunk = 2, 64, 128, 64
    q, k, v, do, _, _ = _inputs(1, Tt, H, dk, dv, "bf16", seed=31, with_state=False)
    g = torch.Generator().manual_seed(32)
    S0 = torch.randn(len(lens), H, dk, dv, generator=g)
    dS = torch.randn(len(lens), H, dk, dv, generator=g)
    ref = oracle.msr_backward_varlen(W.to_f64(q), W.to_f64(k), W.to_f64(v), gammas, W.to_f64(do),
                                     cu, S0.double().numpy(), dS.double().numpy())
    got = ops.chunkwise_bwd(q.cuda(), k.cuda(), v.cuda(), do.cuda(), gammas, chunk,
                            cu_seqlens=torch.from_numpy(cu).cuda(), state_in=S0.cuda(),
                            d_state_out=dS.cuda(), return_d_state=True)
    _check(got, ref, H, f"tc gammas {gammas}", tc=True)


@pytest.mark.parametrize("dv", [64, 512])
def test_backward_tiny_decay_with_state_gradient(dv):
    """A gamma far below any that decays over one chunk, with a final-state
    gradient: the anti-causal passes start from dS_T itself, so nothing is
    divided by gamma (the state gradient reaches the last tokens only)."""
    B, T, H, dk, chunk = 1, 150, 2, 64, 64
    q, k, v, do, S0, dS = _inputs(B, T, H, dk, dv, "bf16", seed=41, with_state=True)
    gam = [1e-7, 0.9]
    assert _tensor_core("bf16", dk, dv, gam, True)
    ref = oracle.msr_backward(W.to_f64(q), W.to_f64(k), W.to_f64(v), gam, W.to_f64(do),
                              S0.double().numpy(), dS.double().numpy())
    got = ops.chunkwise_bwd(q.cuda(), k.cuda(), v.cuda(), do.cuda(), gam, chunk,
                            state_in=S0.cuda(), d_state_out=dS.cuda(), return_d_state=True)
    _check(got, ref, H, f"tiny gamma dv{dv}", tc=True)


@pytest.mark.parametrize("gammas", [[0.0, 1.0], [1.0, 0.5]])
def test_backward_extreme_decays(gammas):
    """gamma = 0 (diagonal only) and gamma = 1 (no decay) through several chunks."""
    B, T, H, dk, dv, chunk = 1, 70, 2, 16, 32, 16
    q, k, v, do, S0, dS = _inputs(B, T, H, dk, dv, "f32", seed=5, with_state=True)
    ref = oracle.msr_backward(W.to_f64(q), W.to_f64(k), W.to_f64(v), gammas, W.to_f64(do),
                              S0.double().numpy(), dS.double().numpy())
    got = ops.chunkwise_bwd(q.cuda(), k.cuda(), v.cuda(), do.cuda(), gammas, chunk,
                            state_in=S0.cuda(), d_state_out=dS.cuda(), return_d_state=True)
    _check(got, ref, H, f"gammas {gammas}")  # float32 inputs: CUDA cores


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_backward_packed_sequences(dtype):
    """Packed batch with an empty sequence, one-token and ragged sequences."""
    lens = [40, 0, 1, 77, 33]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    Tt = int(cu[-1])
    H, dk, dv, chunk = 2, 32, 16, 16
    q, k, v, do, _, _ = _inputs(1, Tt, H, dk, dv, dtype, seed=11, with_state=False)
    g = torch.Generator().manual_seed(12)
    S0 = torch.randn(len(lens), H, dk, dv, generator=g)
    dS = torch.randn(len(lens), H, dk, dv, generator=g)
    gam = W.head_gammas(H)
    ref = oracle.msr_backward_varlen(W.to_f64(q), W.to_f64(k), W.to_f64(v), gam, W.to_f64(do),
                                     cu, S0.double().numpy(), dS.double().numpy())
    got = ops.chunkwise_bwd(q.cuda(), k.cuda(), v.cuda(), do.cuda(), gam, chunk,
                            cu_seqlens=torch.from_numpy(cu).cuda(), state_in=S0.cuda(),
                            d_state_out=dS.cuda(), return_d_state=True)
    _check(got, ref, H, f"packed {dtype}")  # heads of 32/16: CUDA cores


def test_backward_chunk_length_does_not_matter():
    """Every chunk length evaluates the same gradients (to float32 rounding)."""
    B, T, H, dk, dv = 1, 100, 1, 32, 32
    q, k, v, do, S0, dS = _inputs(B, T, H, dk, dv, "f32", seed=9, with_state=True)
    args = [t.cuda() for t in (q, k, v, do)]
    base = ops.chunkwise_bwd(*args, W.head_gammas(H), 100, state_in=S0.cuda(),
                             d_state_out=dS.cuda(), return_d_state=True)
    for chunk in (1, 7, 32):
        got = ops.chunkwise_bwd(*args, W.head_gammas(H), chunk, state_in=S0.cuda(),
                                d_state_out=dS.cuda(), return_d_state=True)
        for x, y in zip(got, base):
            assert_close(W.to_f64(x), W.to_f64(y), "f32", None, f"chunk {chunk}")


@pytest.mark.parametrize("B,T,H,dk,chunk,with_state,use_dS", [
    (2, 300, 2, 128, 256, True, True),     # several chunks and tiles, both state terms
    (1, 700, 1, 256, 512, True, False),    # the 6.7B heads, 512-token chunks, ragged tail
    (1, 1030, 2, 64, 128, False, True),    # 128-token chunks executed as 256
])
def test_backward_tensor_core_dv512(B, T, H, dk, chunk, with_state, use_dS):
    """d_v = 512: dQ and dK run as two passes over the halves of d_v (the score
    contracts over d_v), the second adding to the first; dV in one pass."""
    dv = 512
    q, k, v, do, S0, dS = _inputs(B, T, H, dk, dv, "bf16", seed=T + dk, with_state=True)
    S0 = S0 if with_state else None
    dS = dS if use_dS else None
    gam = W.head_gammas(H)
    assert _tensor_core("bf16", dk, dv, gam, use_dS)
    ref = oracle.msr_backward(W.to_f64(q), W.to_f64(k), W.to_f64(v), gam, W.to_f64(do),
                              None if S0 is None else S0.double().numpy(),
                              None if dS is None else dS.double().numpy())
    got = ops.chunkwise_bwd(q.cuda(), k.cuda(), v.cuda(), do.cuda(), gam, chunk,
                            state_in=None if S0 is None else S0.cuda(),
                            d_state_out=None if dS is None else dS.cuda(), return_d_state=True)
    _check(got, ref, H, f"tc dv512 T{T} dk{dk} C{chunk} dS={use_dS}", tc=True)


def test_backward_tensor_core_dv512_packed():
    lens = [300, 0, 1, 257, 64]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    Tt = int(cu[-1])
    H, dk, dv, chunk = 2, 128, 512, 256
    q, k, v, do, _, _ = _inputs(1, Tt, H, dk, dv, "bf16", seed=23, with_state=False)
    g = torch.Generator().manual_seed(24)
    S0 = torch.randn(len(lens), H, dk, dv, generator=g)
    dS = torch.randn(len(lens), H, dk, dv, generator=g)
    gam = W.head_gammas(H)
    ref = oracle.msr_backward_varlen(W.to_f64(q), W.to_f64(k), W.to_f64(v), gam, W.to_f64(do),
                                     cu, S0.double().numpy(), dS.double().numpy())
    got = ops.chunkwise_bwd(q.cuda(), k.cuda(), v.cuda(), do.cuda(), gam, chunk,
                            cu_seqlens=torch.from_numpy(cu).cuda(), state_in=S0.cuda(),
                            d_state_out=dS.cuda(), return_d_state=True)
    _check(got, ref, H, "tc dv512 packed", tc=True)


def test_backward_6p7b_heads_t8192_sampled():
    """The 6.7B-shaped backward (B=2, T=8192, H=16, d_k=256, d_v=512, chunk 512)
    in full on the GPU, against the oracle on one sampled (sequence, head)."""
    B, T, H, dk, dv, C = 2, 8192, 16, 256, 512, 512
    q, k, v, do, _, dS = _inputs(B, T, H, dk, dv, "bf16", seed=88, with_state=True)
    gam = W.head_gammas(H)
    got = ops.chunkwise_bwd(q.cuda(), k.cuda(), v.cuda(), do.cuda(), gam, C,
                            d_state_out=dS.cuda(), return_d_state=True)
    b, h = 1, 15
    ref = oracle.retention_backward(W.to_f64(q[b, :, h]), W.to_f64(k[b, :, h]),
                                    W.to_f64(v[b, :, h]), gam[h], W.to_f64(do[b, :, h]),
                                    None, dS[b, h].double().numpy())
    for x, y, n in zip((got[0][b, :, h], got[1][b, :, h], got[2][b, :, h], got[3][b, h]), ref,
                       ("dq", "dk", "dv", "d_state_in")):
        assert_close(W.to_f64(x), y, "bf16", None, f"6.7B b{b} h{h} {n}")


def test_backward_rejects_unsupported_and_bad_arguments():
    q = torch.zeros(1, 8, 1, 512, device="cuda")
    v = torch.zeros(1, 8, 1, 16, device="cuda")
    with pytest.raises(ops.RetentionError):
        ops.chunkwise_bwd(q, q, v, v, [0.9], 4)
    assert ops.chunkwise_bwd_workspace_size(torch.float32, 4, 1, 8, 1, 512, 16) == 0
    assert ops.chunkwise_bwd_workspace_size(torch.float32, 0, 1, 8, 1, 16, 16) == 0
    assert ops.chunkwise_bwd_workspace_size(torch.float32, 4, 1, 8, 1, 16, 16) > 0
    # d_v = 512: bf16 on the tensor cores only
    assert ops.chunkwise_bwd_workspace_size(torch.bfloat16, 256, 1, 8, 1, 128, 512) > 0
    assert ops.chunkwise_bwd_workspace_size(torch.float32, 256, 1, 8, 1, 128, 512) == 0
    assert ops.chunkwise_bwd_workspace_size(torch.bfloat16, 256, 1, 8, 1, 16, 512) == 0


@pytest.mark.parametrize("path", ["tensor_core", "tensor_core_dS", "cuda_core"])
def test_backward_bench_workload_sampled(path):
    """The backward at the size bench.py times (B=4, T=2048, H=8, d_k=128, d_v=256,
    chunk 128), checked on two sampled (sequence, head) pairs: bf16 inputs on
    the tensor-core path without and with a final-state gradient, and the same
    values as float32 inputs (with one) on the CUDA-core path."""
    B, T, H, dk, dv, C = 4, 2048, 8, 128, 256, 128
    q, k, v, do, _, dS = _inputs(B, T, H, dk, dv, "bf16", seed=77, with_state=True)
    gam = W.head_gammas(H)
    use_dS = path != "tensor_core"
    x = [t.cuda() for t in (q, k, v, do)]
    if path == "cuda_core":
        x = [t.float() for t in x]
    got = ops.chunkwise_bwd(*x, gam, C, d_state_out=dS.cuda() if use_dS else None,
                            return_d_state=True)
    for b, h in ((0, 0), (3, 7)):
        ref = oracle.retention_backward(W.to_f64(q[b, :, h]), W.to_f64(k[b, :, h]),
                                        W.to_f64(v[b, :, h]), gam[h], W.to_f64(do[b, :, h]),
                                        None, dS[b, h].double().numpy() if use_dS else None)
        for x, y, n in zip((got[0][b, :, h], got[1][b, :, h], got[2][b, :, h], got[3][b, h]),
                           ref, ("dq", "dk", "dv", "d_state_in")):
            kind = "f32" if path == "cuda_core" else "bf16"
            assert_close(W.to_f64(x), y, kind, None, f"{path} b{b} h{h} {n}")
