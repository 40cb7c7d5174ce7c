"""Seeded synthetic workloads shared by the tests, the bench and the smoke check.

This module only draws random inputs and states the workload shapes; it holds
none of the retention arithmetic, so the CPU oracle and the CUDA library can
both be fed from it without sharing any of the method's code.

Recipe (the same for every workload):

* one ``torch.Generator`` seeded with ``seed`` (default 0), drawing float32
  ``randn`` in the order q, k, v, g;
* q, k and v are divided by sqrt(d_k), so the scores q.k have unit scale;
  the gate g is left at N(0, 1);
* the tensors are then cast to the workload's input dtype; consumers that
  need float64 upcast the *cast* values, so every side sees the same numbers;
* one fixed decay per head, gamma_h = 1 - 2^(-5-h) for h = 0..H-1 (the
  multi-scale decay of Multi-Scale Retention: every head forgets at its own
  fixed rate, from 1/32 per token for head 0 down to 2^-20 for head 15);
* variable-length batches draw their lengths with
  ``numpy.random.default_rng(seed).integers(lo, hi + 1, n)``.

The shapes mirror the pages' workloads: a 6.7B-class RetNet has 16 heads with
d_k = 256 and d_v = 512 and was trained and decoded at 8192 tokens; the
chunked form uses chunks of a few hundred tokens.
"""

from dataclasses import dataclass, field
import math

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    chunk: int
    dtype: str                      # input dtype: "f32" or "bf16"
    norm_gate: bool = False         # fused per-head GroupNorm + swish gate
    state_out: bool = False         # emit the final fp32 state
    varlen: tuple = None            # (n_seq, min_len, max_len) for packed batches
    decode_steps: int = 0           # single-token steps after the prefill
    description: str = ""


WORKLOADS = {
    "tiny_fp32_b1_h2_t64_d16_c16": Workload(
        "tiny_fp32_b1_h2_t64_d16_c16", B=1, T=64, H=2, dk=16, dv=16, chunk=16,
        dtype="f32",
        description="tiny fp32 case: parallel, recurrent and chunkwise forms"),
    "msr_b4_h8_t2048_dk128_dv256_c128": Workload(
        "msr_b4_h8_t2048_dk128_dv256_c128", B=4, T=2048, H=8, dk=128, dv=256,
        chunk=128, dtype="bf16", norm_gate=True,
        description="chunkwise MSR forward, bf16 in / fp32 accumulate, + GroupNorm + swish gate"),
    "msr_6p7b_b2_h16_t8192_dk256_dv512_c512": Workload(
        "msr_6p7b_b2_h16_t8192_dk256_dv512_c512", B=2, T=8192, H=16, dk=256, dv=512,
        chunk=512, dtype="bf16", norm_gate=True, state_out=True,
        description="6.7B-shaped long sequence, chunkwise, fused GroupNorm + gate, final fp32 state"),
    "decode_6p7b_n128_h16_dk256_dv512": Workload(
        "decode_6p7b_n128_h16_dk256_dv512", B=128, T=8192, H=16, dk=256, dv=512,
        chunk=512, dtype="bf16", decode_steps=1024,
        description="recurrent decode: 128 sequences, fp32 state from a chunkwise prefill "
                    "of 8192 bf16 tokens, then 1024 single-token steps"),
    "varlen_64seq_h8_d128_c64": Workload(
        "varlen_64seq_h8_d128_c64", B=1, T=0, H=8, dk=128, dv=128, chunk=64,
        dtype="bf16", varlen=(64, 512, 16384),
        description="packed variable-length batch, 64 sequences of U[512,16384] tokens, "
                    "state reset at every sequence start"),
}


def head_gammas(H):
    """Per-head fixed decays gamma_h = 1 - 2^(-5-h), as float64 (host)."""
    return np.array([1.0 - 2.0 ** (-5 - h) for h in range(H)], dtype=np.float64)


def varlen_lengths(n, lo, hi, seed=0):
    """Sequence lengths uniform in [lo, hi] (inclusive)."""
    return np.random.default_rng(seed).integers(lo, hi + 1, n).astype(np.int64)


def cu_seqlens_of(lengths):
    """Offsets [0, l0, l0+l1, ...] as int32."""
    out = np.zeros(len(lengths) + 1, dtype=np.int64)
    out[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    if out[-1] >= 2 ** 31:
        raise ValueError("total length does not fit int32 offsets")
    return out.astype(np.int32)


def torch_dtype(name):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def make_qkvg(B, T, H, dk, dv, dtype="bf16", seed=0, gate=True, device="cpu"):
    """Draw q, k: [B,T,H,dk], v: [B,T,H,dv] and g: [B,T,H*dv] (or None).

    q/k/v ~ N(0,1)/sqrt(dk), g ~ N(0,1), drawn in that order from one
    generator seeded with ``seed`` on ``device`` (CPU by default; a CUDA
    generator gives different numbers from the same seed), then cast.
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    s = 1.0 / math.sqrt(dk)
    td = torch_dtype(dtype)
    q = (torch.randn(B, T, H, dk, generator=gen, device=device) * s).to(td)
    k = (torch.randn(B, T, H, dk, generator=gen, device=device) * s).to(td)
    v = (torch.randn(B, T, H, dv, generator=gen, device=device) * s).to(td)
    g = None
    if gate:
        g = torch.randn(B, T, H * dv, generator=gen, device=device).to(td)
    return q, k, v, g


def make_step_inputs(N, H, dk, dv, dtype="bf16", seed=0, device="cpu"):
    """One decode step's q, k: [N,H,dk] and v: [N,H,dv], same recipe."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    s = 1.0 / math.sqrt(dk)
    td = torch_dtype(dtype)
    q = (torch.randn(N, H, dk, generator=gen, device=device) * s).to(td)
    k = (torch.randn(N, H, dk, generator=gen, device=device) * s).to(td)
    v = (torch.randn(N, H, dv, generator=gen, device=device) * s).to(td)
    return q, k, v


def make_state(N, H, dk, dv, seed=0, scale=1.0, device="cpu"):
    """A random fp32 state [N,H,dk,dv] (for tests that start from a given state)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return torch.randn(N, H, dk, dv, generator=gen, device=device) * scale


def to_f64(t):
    """Upcast a torch tensor (any dtype, any device) to a float64 numpy array."""
    return t.detach().to("cpu", torch.float64).numpy()
