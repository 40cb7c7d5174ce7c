"""Host-only checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments before touching the GPU."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "retention.h")


def _lib():
    from linear_recurrent_sequence_retention_b200 import ops
    if not os.path.exists(ops.LIBRARY_PATH):
        from linear_recurrent_sequence_retention_b200 import build
        build.build()
    return ops, ops.lib()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^RET_API\s+[\w\s\*]*?\b(\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("retention_parallel_fwd", "retention_chunkwise_fwd", "retention_recurrent_step",
                 "msr_norm_gate", "retention_chunkwise_workspace_size",
                 "retention_check_device_error", "retention_status_string",
                 "retention_abi_version"):
        assert name in syms


def test_library_exports_every_declared_symbol():
    ops, L = _lib()
    for name in declared_symbols():
        assert hasattr(L, name), f"libretention.so does not export {name}"
    assert set(ops.EXPORTED) <= set(declared_symbols())


def test_library_is_built_from_this_tree(monkeypatch):
    """The library embeds the hash of its sources; the binding refuses another tree's build."""
    ops, L = _lib()
    from linear_recurrent_sequence_retention_b200 import build
    sha = L.retention_source_sha().decode()
    assert re.fullmatch(r"[0-9a-f]{64}", sha) and sha == build.source_sha()
    monkeypatch.setattr(build, "source_sha", lambda: "0" * 64)
    with pytest.raises(RuntimeError, match="built from other sources"):
        ops._check_sources(L)


def test_abi_version_and_status_strings():
    ops, L = _lib()
    assert L.retention_abi_version() == 3
    for code in range(8):
        s = ops.status_string(code)
        assert s and "unknown" not in s
    assert "unknown" in ops.status_string(99)


FAKE = ctypes.c_void_p(0x10000)          # aligned, never dereferenced on these paths
MISALIGNED = ctypes.c_void_p(0x10004)
FAKE_WS = 0x100000                           # 256-byte aligned, never dereferenced


def _g(*vals):
    return (ctypes.c_double * len(vals))(*vals)


def test_parallel_rejects_bad_arguments():
    ops, L = _lib()
    f = L.retention_parallel_fwd
    ok = dict(B=1, T=8, H=2, dk=16, dv=16)
    args = lambda q=FAKE, gamma=_g(0.5, 0.9), dk=16, dv=16, T=8, H=2, o_dt=0, dt=0, ws=None, nb=0: (
        q, FAKE, FAKE, dt, gamma, FAKE, o_dt, ws, nb, 1, T, H, dk, dv, None)
    assert f(*args(q=None)) == ops.RET_ERR_INVALID_ARG
    assert f(*args(q=MISALIGNED)) == ops.RET_ERR_INVALID_ARG
    assert f(*args(gamma=_g(0.5, 1.5))) == ops.RET_ERR_INVALID_ARG
    assert f(*args(gamma=_g(-0.1, 0.5))) == ops.RET_ERR_INVALID_ARG
    assert f(*args(gamma=_g(float("nan"), 0.5))) == ops.RET_ERR_INVALID_ARG
    assert f(*args(T=0)) == ops.RET_ERR_INVALID_ARG
    assert f(*args(o_dt=7)) == ops.RET_ERR_INVALID_ARG
    assert f(*args(dk=300)) == ops.RET_ERR_UNSUPPORTED
    # bf16 at tensor-core head dims needs the workspace: missing, short or misaligned
    need = L.retention_parallel_workspace_size(ops.RET_BF16, 1, 8, 2, 128, 256)
    # fp16 copy of v, max(T, d_k) rows per sequence, then 256 bytes for the tile counter
    assert need == 1 * 128 * 2 * 256 * 2 + 256
    bf = dict(dt=ops.RET_BF16, dk=128, dv=256)
    assert f(*args(**bf)) == ops.RET_ERR_WORKSPACE
    assert f(*args(**bf, ws=FAKE_WS, nb=need - 256)) == ops.RET_ERR_WORKSPACE
    assert f(*args(**bf, ws=FAKE_WS + 16, nb=need)) == ops.RET_ERR_WORKSPACE
    assert f(*args(dt=ops.RET_BF16, dk=128, dv=300)) == ops.RET_ERR_UNSUPPORTED
    # float32 and non-tensor-core bf16 shapes need none
    assert L.retention_parallel_workspace_size(ops.RET_F32, 1, 8, 2, 128, 256) == 0
    assert L.retention_parallel_workspace_size(ops.RET_BF16, 1, 8, 2, 16, 16) == 0
    assert L.retention_parallel_workspace_size(ops.RET_BF16, 2, 1000, 3, 64, 512) == 2 * 1000 * 3 * 512 * 2 + 256


def test_workspace_size_query():
    ops, L = _lib()
    ws = L.retention_chunkwise_workspace_size
    # float32: meta (256 B) + one fp32 state per chunk
    assert ws(0, 16, 1, 64, 2, 16, 16, 0) == 256 + 4 * 2 * 16 * 16 * 4
    # ragged tail: ceil(70/16) = 5 chunks per sequence
    assert ws(0, 16, 3, 70, 2, 16, 16, 0) == 256 + 15 * 2 * 16 * 16 * 4
    # packed: ceil(Ttot/C) + nseq slots
    assert ws(0, 16, 1, 100, 2, 8, 8, 5) == 256 + (7 + 5) * 2 * 8 * 8 * 4
    assert ws(0, 0, 1, 64, 2, 16, 16, 0) == 0            # chunk < 1
    assert ws(0, 16, 1, 64, 65, 16, 16, 0) == 0          # H > 64
    assert ws(0, 16, 2, 64, 2, 16, 16, 3) == 0           # packed needs B == 1
    assert ws(0, 16, 1, 64, 2, 300, 16, 0) == 0          # fp32 path: dk <= 256


def test_tensor_core_workspace_layout():
    """bf16: meta words | fp16 state per executed chunk | fp16 copy of v, each rounded to 256 B;
    the executed chunk is 128 tokens, or 256 when dv >= 256, whatever chunk was asked for."""
    ops, L = _lib()
    ws = L.retention_chunkwise_workspace_size
    r256 = lambda b: (b + 255) // 256 * 256

    def expect(B, T, H, dk, dv, nseq=0):
        ce = 256 if dv >= 256 else 128
        ttot = T if nseq else B * T
        slots = (ttot + ce - 1) // ce + nseq if nseq else B * ((T + ce - 1) // ce)
        nmeta = nseq if nseq else B
        return (r256(4 * (2 * nmeta + 1)) + r256(slots * H * dk * dv * 2)
                + r256(ttot * H * dv * 2))
    for chunk in (64, 128, 256, 512):
        assert ws(1, chunk, 2, 8192, 16, 256, 512, 0) == expect(2, 8192, 16, 256, 512)
        assert ws(1, chunk, 4, 2048, 8, 128, 256, 0) == expect(4, 2048, 8, 128, 256)
        assert ws(1, chunk, 3, 1000, 2, 64, 128, 0) == expect(3, 1000, 2, 64, 128)
    assert ws(1, 64, 1, 550655, 8, 128, 128, 64) == expect(1, 550655, 8, 128, 128, nseq=64)


def test_chunkwise_rejects_bad_arguments():
    ops, L = _lib()
    f = L.retention_chunkwise_fwd
    NG = ops.NormGate

    def call(ws_bytes=1 << 20, ws=FAKE, gamma=None, cu=None, nseq=0, ng=None, q=FAKE):
        gamma = gamma or _g(0.5, 0.9)
        return f(q, FAKE, FAKE, 0, gamma, 16, cu, nseq, None, None, FAKE, 0,
                 ng, ws, ws_bytes, 1, 64, 2, 16, 16, None)
    assert call(ws_bytes=10) == ops.RET_ERR_WORKSPACE
    assert call(ws=None) == ops.RET_ERR_WORKSPACE
    assert call(ws=ctypes.c_void_p(0x10010)) == ops.RET_ERR_WORKSPACE   # not 256-B aligned
    assert call(gamma=_g(0.5, 2.0)) == ops.RET_ERR_INVALID_ARG
    assert call(cu=FAKE, nseq=0) == ops.RET_ERR_INVALID_ARG              # cu without nseq
    assert call(q=None) == ops.RET_ERR_INVALID_ARG
    bad = NG(None, 0, None, None, 1e-5)
    assert call(ng=ctypes.byref(bad)) == ops.RET_ERR_INVALID_ARG         # gate missing
    bad_eps = NG(0x10000, 0, None, None, -1.0)
    assert call(ng=ctypes.byref(bad_eps)) == ops.RET_ERR_INVALID_ARG


def test_decode_and_norm_gate_reject_bad_arguments():
    ops, L = _lib()
    st = L.retention_recurrent_step(FAKE, FAKE, FAKE, 1, _g(0.5), None, FAKE, 0, 1, 1, 8, 8, None)
    assert st == ops.RET_ERR_INVALID_ARG
    st = L.retention_recurrent_step(FAKE, FAKE, FAKE, 1, _g(0.5), FAKE, FAKE, 0, 1, 1, 2048, 8, None)
    assert st == ops.RET_ERR_UNSUPPORTED
    ng = ops.NormGate(0x10000, 1, None, None, 1e-5)
    assert L.msr_norm_gate(FAKE, 1, None, FAKE, 1, 4, 2, 8, None) == ops.RET_ERR_INVALID_ARG
    assert L.msr_norm_gate(FAKE, 1, ctypes.byref(ng), FAKE, 1, 4, 2, 2048, None) == ops.RET_ERR_UNSUPPORTED
    assert L.msr_norm_gate(FAKE, 1, ctypes.byref(ng), FAKE, 1, 0, 2, 8, None) == ops.RET_ERR_INVALID_ARG


def test_recurrent_steps_reject_bad_arguments():
    ops, L = _lib()
    f = L.retention_recurrent_steps
    # (q, k, v, in_dtype, gamma, state, o, o_dtype, N, Tn, H, dk, dv, stream)
    assert f(FAKE, FAKE, FAKE, 1, _g(0.5), None, FAKE, 0, 1, 4, 1, 8, 8, None) == ops.RET_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 1, _g(0.5), FAKE, FAKE, 0, 1, 0, 1, 8, 8, None) == ops.RET_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 1, _g(1.5), FAKE, FAKE, 0, 1, 4, 1, 8, 8, None) == ops.RET_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 1, _g(0.5), FAKE, FAKE, 0, 1, 17, 1, 8, 8, None) == ops.RET_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, 1, _g(0.5), FAKE, FAKE, 0, 1, 4, 1, 6, 8, None) == ops.RET_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, 1, _g(0.5), FAKE, FAKE, 0, 1, 4, 1, 1024, 8, None) == ops.RET_ERR_UNSUPPORTED


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    from linear_recurrent_sequence_retention_b200 import ops
    monkeypatch.setattr(ops, "_lib", None)
    monkeypatch.setattr(ops, "LIBRARY_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        ops.lib()


def test_backward_workspace_size_and_bad_arguments():
    ops, L = _lib()
    ws = L.retention_chunkwise_bwd_workspace_size
    # CUDA-core path: meta (256 B) + two fp32 states per chunk
    assert ws(0, 16, 1, 64, 2, 16, 16, 0) == 256 + 2 * 4 * 2 * 16 * 16 * 4
    # bf16 with heads 64/128/256 may take the tensor-core path: at least as large
    assert ws(1, 128, 1, 256, 2, 64, 64, 0) >= 256 + 2 * 2 * 2 * 64 * 64 * 4
    assert ws(0, 0, 1, 64, 2, 16, 16, 0) == 0            # chunk < 1
    assert ws(0, 16, 1, 64, 2, 300, 16, 0) == 0          # heads beyond 256
    assert ws(0, 16, 1, 64, 65, 16, 16, 0) == 0          # H > 64
    f = L.retention_chunkwise_bwd

    def call(q=FAKE, gamma=None, ws_ptr=FAKE, ws_bytes=1 << 24, cu=None, nseq=0, dq=FAKE):
        gamma = gamma or _g(0.5, 0.9)
        return f(q, FAKE, FAKE, FAKE, 0, gamma, 16, cu, nseq, None, None, dq, FAKE, FAKE, None,
                 ws_ptr, ws_bytes, 1, 64, 2, 16, 16, None)
    assert call(q=None) == ops.RET_ERR_INVALID_ARG
    assert call(dq=None) == ops.RET_ERR_INVALID_ARG
    assert call(q=MISALIGNED) == ops.RET_ERR_INVALID_ARG
    assert call(gamma=_g(0.5, 1.01)) == ops.RET_ERR_INVALID_ARG
    assert call(cu=FAKE, nseq=0) == ops.RET_ERR_INVALID_ARG
    assert call(ws_bytes=100) == ops.RET_ERR_WORKSPACE
    assert call(ws_ptr=ctypes.c_void_p(0x10010)) == ops.RET_ERR_WORKSPACE


def test_rope_rejects_bad_arguments():
    ops, L = _lib()
    f = L.retention_rope

    def call(q=FAKE, d=16, base=10000.0, cu=None, nseq=0, dtype=1):
        return f(q, FAKE, dtype, FAKE, FAKE, base, cu, nseq, 1, 8, 2, d, None)
    assert call(d=7) == ops.RET_ERR_INVALID_ARG          # odd head dimension
    assert call(base=1.0) == ops.RET_ERR_INVALID_ARG
    assert call(base=float("inf")) == ops.RET_ERR_INVALID_ARG
    assert call(q=None) == ops.RET_ERR_INVALID_ARG
    assert call(q=MISALIGNED) == ops.RET_ERR_INVALID_ARG
    assert call(cu=None, nseq=2) == ops.RET_ERR_INVALID_ARG
    assert call(dtype=5) == ops.RET_ERR_INVALID_ARG


def test_rla_workspace_size_and_bad_arguments():
    ops, L = _lib()
    ws = L.retention_rla_workspace_size
    assert ws(0, 1, 64, 2, 16, 16, 0) > 0
    assert ws(0, 1, 64, 2, 300, 16, 0) == 0              # f32 path: heads up to 256
    assert ws(1, 1, 64, 2, 100, 128, 0) == 0             # bf16 path: d_k in {64, 128, 256}
    f = L.retention_rla_fwd

    def call(window=4, ws_ptr=FAKE, ws_bytes=1 << 24, q=FAKE):
        return f(q, FAKE, FAKE, 0, window, None, 0, FAKE, 0, ws_ptr, ws_bytes, 1, 64, 2, 16, 16,
                 None)
    assert call(window=-1) == ops.RET_ERR_INVALID_ARG
    assert call(q=None) == ops.RET_ERR_INVALID_ARG
    assert call(ws_bytes=100) == ops.RET_ERR_WORKSPACE
    assert call(ws_ptr=None) == ops.RET_ERR_WORKSPACE


def test_chunkwise_executed_chunk():
    """The chunk the kernels evaluate: the caller's for float32 inputs; for bf16
    at least 128 tokens, and at least 256 when d_v >= 256; 0 if unsupported."""
    ops, L = _lib()
    assert L.retention_chunkwise_executed_chunk(ops.RET_F32, 16, 16, 16) == 16
    assert L.retention_chunkwise_executed_chunk(ops.RET_F32, 1, 256, 256) == 1
    assert L.retention_chunkwise_executed_chunk(ops.RET_BF16, 64, 128, 128) == 128
    assert L.retention_chunkwise_executed_chunk(ops.RET_BF16, 128, 128, 256) == 256
    assert L.retention_chunkwise_executed_chunk(ops.RET_BF16, 512, 256, 512) == 256
    assert L.retention_chunkwise_executed_chunk(ops.RET_BF16, 512, 128, 128) == 128
    assert L.retention_chunkwise_executed_chunk(ops.RET_BF16, 256, 64, 128) == 128
    assert L.retention_chunkwise_executed_chunk(ops.RET_BF16, 96, 128, 128) == 0     # unsupported chunk
    assert L.retention_chunkwise_executed_chunk(ops.RET_F32, 0, 16, 16) == 0        # invalid chunk
