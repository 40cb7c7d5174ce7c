"""Thin ctypes binding of libretention.so (C ABI in include/retention.h).

Argument marshalling only: every function checks the torch tensors it is
given, passes their device pointers, sizes and the current CUDA stream to the
C entry point of the same name, and raises :class:`RetentionError` on a
non-OK status.  All arithmetic happens in the library's CUDA kernels; there
is no CPU or PyTorch fallback, and calling any function without the built
library raises immediately.
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIBRARY_PATH = os.path.join(_HERE, "libretention.so")
_IN_TREE_LIBRARY = LIBRARY_PATH

RET_OK = 0
RET_ERR_INVALID_ARG = 1
RET_ERR_UNSUPPORTED = 2
RET_ERR_CUDA = 3
RET_ERR_TIMEOUT = 4
RET_ERR_WORKSPACE = 5
RET_ERR_DEVICE_DATA = 6
RET_ERR_RANGE = 7

RET_F32 = 0
RET_BF16 = 1

# Capacity of the library's built-in scratch (RETENTION_STATIC_WORKSPACE_BYTES).
STATIC_WORKSPACE_BYTES = 32 << 20

EXPORTED = (
    "retention_abi_version",
    "retention_source_sha",
    "retention_status_string",
    "retention_parallel_workspace_size",
    "retention_parallel_fwd",
    "retention_chunkwise_workspace_size",
    "retention_chunkwise_executed_chunk",
    "retention_chunkwise_fwd",
    "retention_chunkwise_states",
    "retention_chunkwise_outputs",
    "retention_chunkwise_fwd_static_ws",
    "retention_chunkwise_fwd_rope_workspace_size",
    "retention_chunkwise_fwd_rope",
    "retention_chunkwise_bwd_workspace_size",
    "retention_chunkwise_bwd",
    "retention_rope",
    "retention_rla_workspace_size",
    "retention_rla_fwd",
    "retention_recurrent_step",
    "retention_recurrent_steps",
    "msr_norm_gate",
    "retention_check_device_error",
    "retention_selftest_wait_timeout",
)


class RetentionError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


class NormGate(ctypes.Structure):
    _fields_ = [("g", ctypes.c_void_p), ("g_dtype", ctypes.c_int),
                ("weight", ctypes.c_void_p), ("bias", ctypes.c_void_p),
                ("eps", ctypes.c_float)]


_lib = None


def _check_sources(L):
    """Refuse the in-tree library if it was built from sources other than the tree's."""
    if (os.path.abspath(LIBRARY_PATH) != _IN_TREE_LIBRARY
            or not os.path.isdir(os.path.join(_HERE, "csrc"))):
        return
    from . import build
    want, got = build.source_sha(), L.retention_source_sha().decode()
    if got != want:
        raise RuntimeError(
            f"{LIBRARY_PATH} was built from other sources (library {got[:12]}, tree "
            f"{want[:12]}): rebuild it with `python -m linear_recurrent_sequence_retention_b200.build`")


def lib():
    """The loaded library (loads it on first use; raises if it is not built or is stale)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIBRARY_PATH):
        raise RuntimeError(
            f"{LIBRARY_PATH} is missing: build it with "
            "`python -m linear_recurrent_sequence_retention_b200.build` (needs nvcc)")
    L = ctypes.CDLL(LIBRARY_PATH)
    vp, ci, cd = ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(ctypes.c_double)
    L.retention_abi_version.restype = ci
    L.retention_abi_version.argtypes = []
    L.retention_source_sha.restype = ctypes.c_char_p
    L.retention_source_sha.argtypes = []
    _check_sources(L)
    L.retention_status_string.restype = ctypes.c_char_p
    L.retention_status_string.argtypes = [ci]
    L.retention_parallel_workspace_size.restype = ctypes.c_size_t
    L.retention_parallel_workspace_size.argtypes = [ci, ci, ci, ci, ci, ci]
    L.retention_parallel_fwd.restype = ci
    L.retention_parallel_fwd.argtypes = [vp, vp, vp, ci, cd, vp, ci, vp, ctypes.c_size_t,
                                         ci, ci, ci, ci, ci, vp]
    L.retention_chunkwise_workspace_size.restype = ctypes.c_size_t
    L.retention_chunkwise_workspace_size.argtypes = [ci, ci, ci, ci, ci, ci, ci, ci]
    L.retention_chunkwise_executed_chunk.restype = ci
    L.retention_chunkwise_executed_chunk.argtypes = [ci, ci, ci, ci]
    L.retention_chunkwise_fwd.restype = ci
    L.retention_chunkwise_fwd.argtypes = [vp, vp, vp, ci, cd, ci, vp, ci, vp, vp, vp, ci,
                                          ctypes.POINTER(NormGate), vp, ctypes.c_size_t,
                                          ci, ci, ci, ci, ci, vp]
    L.retention_chunkwise_states.restype = ci
    L.retention_chunkwise_states.argtypes = [vp, vp, ci, cd, ci, vp, ci, vp, vp, vp,
                                             ctypes.c_size_t, ci, ci, ci, ci, ci, vp]
    L.retention_chunkwise_outputs.restype = ci
    L.retention_chunkwise_outputs.argtypes = [vp, vp, vp, ci, cd, ci, vp, ci, ci, vp, ci,
                                              ctypes.POINTER(NormGate), vp, ctypes.c_size_t,
                                              ci, ci, ci, ci, ci, vp]
    L.retention_chunkwise_fwd_static_ws.restype = ci
    L.retention_chunkwise_fwd_static_ws.argtypes = [vp, vp, vp, ci, cd, ci, vp, ci, vp, vp, vp,
                                                    ci, ctypes.POINTER(NormGate),
                                                    ci, ci, ci, ci, ci, vp]
    L.retention_chunkwise_fwd_rope_workspace_size.restype = ctypes.c_size_t
    L.retention_chunkwise_fwd_rope_workspace_size.argtypes = [ci, ci, ci, ci, ci, ci, ci]
    L.retention_chunkwise_fwd_rope.restype = ci
    L.retention_chunkwise_fwd_rope.argtypes = [vp, vp, vp, ci, cd, ci, vp, ci, vp, vp, vp, ci,
                                               ctypes.POINTER(NormGate), ctypes.c_double, vp,
                                               ctypes.c_size_t, ci, ci, ci, ci, ci, vp]
    L.retention_chunkwise_bwd_workspace_size.restype = ctypes.c_size_t
    L.retention_chunkwise_bwd_workspace_size.argtypes = [ci, ci, ci, ci, ci, ci, ci, ci]
    L.retention_chunkwise_bwd.restype = ci
    L.retention_chunkwise_bwd.argtypes = [vp, vp, vp, vp, ci, cd, ci, vp, ci, vp, vp,
                                          vp, vp, vp, vp, vp, ctypes.c_size_t,
                                          ci, ci, ci, ci, ci, vp]
    L.retention_rope.restype = ci
    L.retention_rope.argtypes = [vp, vp, ci, vp, vp, ctypes.c_double, vp, ci, ci, ci, ci, ci, vp]
    L.retention_rla_workspace_size.restype = ctypes.c_size_t
    L.retention_rla_workspace_size.argtypes = [ci, ci, ci, ci, ci, ci, ci]
    L.retention_rla_fwd.restype = ci
    L.retention_rla_fwd.argtypes = [vp, vp, vp, ci, ci, vp, ci, vp, ci, vp, ctypes.c_size_t,
                                    ci, ci, ci, ci, ci, vp]
    L.retention_recurrent_step.restype = ci
    L.retention_recurrent_step.argtypes = [vp, vp, vp, ci, cd, vp, vp, ci, ci, ci, ci, ci, vp]
    L.retention_recurrent_steps.restype = ci
    L.retention_recurrent_steps.argtypes = [vp, vp, vp, ci, cd, vp, vp, ci, ci, ci, ci, ci, ci, vp]
    L.msr_norm_gate.restype = ci
    L.msr_norm_gate.argtypes = [vp, ci, ctypes.POINTER(NormGate), vp, ci, ci, ci, ci, vp]
    L.retention_check_device_error.restype = ci
    L.retention_check_device_error.argtypes = [vp]
    L.retention_selftest_wait_timeout.restype = ci
    L.retention_selftest_wait_timeout.argtypes = [vp]
    _lib = L
    return L


def status_string(status):
    return lib().retention_status_string(int(status)).decode()


def _check(status, where):
    if status != RET_OK:
        raise RetentionError(status, where)


def _dt(t):
    if t.dtype == torch.float32:
        return RET_F32
    if t.dtype == torch.bfloat16:
        return RET_BF16
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dev(t, name):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _gammas(gamma, H):
    vals = [float(x) for x in (gamma.tolist() if hasattr(gamma, "tolist") else gamma)]
    if len(vals) != H:
        raise ValueError(f"gamma needs {H} entries, got {len(vals)}")
    return (ctypes.c_double * H)(*vals)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def abi_version():
    return lib().retention_abi_version()


def parallel_workspace_size(dtype, B, T, H, dk, dv):
    """Bytes of workspace the parallel form needs (0: none, the CUDA-core kernel)."""
    code = RET_F32 if dtype == torch.float32 else RET_BF16
    return int(lib().retention_parallel_workspace_size(code, B, T, H, dk, dv))


def parallel_fwd(q, k, v, gamma, out_dtype=None, out=None, workspace=None, stream=None):
    """Parallel form; q,k: [B,T,H,dk], v: [B,T,H,dv] -> o [B,T,H,dv].  bf16
    inputs of the tensor-core head dims use a workspace (allocated here when
    not given)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, n)
    B, T, H, dk = q.shape
    dv = v.shape[3]
    if k.shape != q.shape or v.shape[:3] != q.shape[:3] or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v shapes/dtypes disagree")
    if out is None:
        out = torch.empty(B, T, H, dv, device=q.device, dtype=out_dtype or q.dtype)
    else:
        _dev(out, "out")
        if tuple(out.shape) != (B, T, H, dv):
            raise ValueError("out has the wrong shape")
    need = lib().retention_parallel_workspace_size(_dt(q), B, T, H, dk, dv)
    if need and workspace is None:
        workspace = alloc_workspace(need, q.device)
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib().retention_parallel_fwd(_ptr(q), _ptr(k), _ptr(v), _dt(q), _gammas(gamma, H),
                                      _ptr(out), _dt(out), _ptr(workspace), nbytes,
                                      B, T, H, dk, dv, _stream(stream))
    _check(st, "retention_parallel_fwd")
    return out


def chunkwise_workspace_size(dtype, chunk, B, T, H, dk, dv, nseq=0):
    code = RET_F32 if dtype == torch.float32 else RET_BF16
    return int(lib().retention_chunkwise_workspace_size(code, chunk, B, T, H, dk, dv, nseq))


def chunkwise_executed_chunk(dtype, chunk, dk, dv):
    """The chunk length the chunkwise kernels evaluate for ``chunk`` (0 if
    unsupported); every chunk length gives the same result."""
    code = RET_F32 if dtype == torch.float32 else RET_BF16
    return int(lib().retention_chunkwise_executed_chunk(code, chunk, dk, dv))


def alloc_workspace(nbytes, device):
    """A caller-owned workspace buffer (uint8, 256-byte aligned by the allocator)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def chunkwise_fwd_rope_workspace_size(chunk, B, T, H, dk, dv, nseq=0):
    return lib().retention_chunkwise_fwd_rope_workspace_size(chunk, B, T, H, dk, dv, nseq)


def chunkwise_fwd(q, k, v, gamma, chunk, cu_seqlens=None, state_in=None, return_state=False,
                  g=None, gn_weight=None, gn_bias=None, eps=1e-5, out_dtype=None, out=None,
                  state_out=None, workspace=None, stream=None, rope_base=None):
    """Chunkwise form (+ optional fused GroupNorm and swish gate when ``g`` is given).

    q,k: [B,T,H,dk]; v: [B,T,H,dv]; packed sequences: B = 1 and ``cu_seqlens``
    an int32 CUDA tensor [nseq+1].  Returns ``out`` ([B,T,H,dv]: o, or y when
    gated) and, with ``return_state``, the final fp32 states.  With
    ``rope_base`` (bf16 inputs only) q and k are first given the rotary
    position encoding of :func:`rope` inside the same call
    (``retention_chunkwise_fwd_rope``); q and k themselves are not modified.
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, n)
    B, T, H, dk = q.shape
    dv = v.shape[3]
    if k.shape != q.shape or v.shape[:3] != q.shape[:3] or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v shapes/dtypes disagree")
    nseq = 0
    if cu_seqlens is not None:
        _dev(cu_seqlens, "cu_seqlens")
        if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1:
            raise ValueError("cu_seqlens must be a 1-D int32 tensor")
        nseq = cu_seqlens.numel() - 1
        if nseq < 1:
            raise ValueError("cu_seqlens needs at least two entries")
    nstate = nseq if nseq else B
    if state_in is not None:
        _dev(state_in, "state_in")
        if state_in.dtype != torch.float32 or tuple(state_in.shape) != (nstate, H, dk, dv):
            raise ValueError(f"state_in must be float32 [{nstate},{H},{dk},{dv}]")
    if return_state and state_out is None:
        state_out = torch.empty(nstate, H, dk, dv, device=q.device, dtype=torch.float32)
    if state_out is not None:
        _dev(state_out, "state_out")
        if state_out.dtype != torch.float32 or tuple(state_out.shape) != (nstate, H, dk, dv):
            raise ValueError(f"state_out must be float32 [{nstate},{H},{dk},{dv}]")
    if out is None:
        out = torch.empty(B, T, H, dv, device=q.device, dtype=out_dtype or q.dtype)
    else:
        _dev(out, "out")
        if tuple(out.shape) != (B, T, H, dv):
            raise ValueError("out has the wrong shape")
    ng = None
    keep = []
    if g is not None:
        _dev(g, "g")
        if g.numel() != B * T * H * dv:
            raise ValueError("g must hold B*T*H*dv elements")
        for t, n in ((gn_weight, "gn_weight"), (gn_bias, "gn_bias")):
            if t is not None:
                _dev(t, n)
                if t.dtype != torch.float32 or t.numel() != H * dv:
                    raise ValueError(f"{n} must be float32 with H*dv elements")
        ng = NormGate(g.data_ptr(), _dt(g), gn_weight.data_ptr() if gn_weight is not None else None,
                      gn_bias.data_ptr() if gn_bias is not None else None, float(eps))
        keep.append(ng)
    if rope_base is not None:
        if _dt(q) != RET_BF16:
            raise RetentionError(RET_ERR_UNSUPPORTED, "retention_chunkwise_fwd_rope")
        need = lib().retention_chunkwise_fwd_rope_workspace_size(chunk, B, T, H, dk, dv, nseq)
        where = "retention_chunkwise_fwd_rope_workspace_size"
    else:
        need = lib().retention_chunkwise_workspace_size(_dt(q), chunk, B, T, H, dk, dv, nseq)
        where = "retention_chunkwise_workspace_size"
    if need == 0:
        st = RET_ERR_UNSUPPORTED if _dt(q) == RET_BF16 else RET_ERR_INVALID_ARG
        raise RetentionError(st, where)
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    head = (_ptr(q), _ptr(k), _ptr(v), _dt(q), _gammas(gamma, H), int(chunk),
            _ptr(cu_seqlens), nseq, _ptr(state_in), _ptr(state_out), _ptr(out), _dt(out),
            ctypes.byref(ng) if ng is not None else None)
    tail = (_ptr(workspace), workspace.numel() * workspace.element_size(), B, T, H, dk, dv,
            _stream(stream))
    if rope_base is not None:
        st = lib().retention_chunkwise_fwd_rope(*head, float(rope_base), *tail)
        _check(st, "retention_chunkwise_fwd_rope")
    else:
        st = lib().retention_chunkwise_fwd(*head, *tail)
        _check(st, "retention_chunkwise_fwd")
    return (out, state_out) if return_state else out


def chunkwise_states(k, v, gamma, chunk, cu_seqlens=None, state_in=None, state_out=None,
                     workspace=None, stream=None):
    """State phase only: per-chunk states into ``workspace`` (returned) and the
    final states into ``state_out`` (optional, float32 [nseq|B,H,dk,dv])."""
    for t, n in ((k, "k"), (v, "v")):
        _dev(t, n)
    B, T, H, dk = k.shape
    dv = v.shape[3]
    nseq = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    if cu_seqlens is not None:
        _dev(cu_seqlens, "cu_seqlens")
    need = lib().retention_chunkwise_workspace_size(_dt(k), chunk, B, T, H, dk, dv, nseq)
    if need == 0:
        raise RetentionError(RET_ERR_UNSUPPORTED if _dt(k) == RET_BF16 else RET_ERR_INVALID_ARG,
                             "retention_chunkwise_workspace_size")
    if workspace is None:
        workspace = alloc_workspace(need, k.device)
    for t, n in ((state_in, "state_in"), (state_out, "state_out")):
        if t is not None:
            _dev(t, n)
    st = lib().retention_chunkwise_states(
        _ptr(k), _ptr(v), _dt(k), _gammas(gamma, H), int(chunk), _ptr(cu_seqlens), nseq,
        _ptr(state_in), _ptr(state_out), _ptr(workspace),
        workspace.numel() * workspace.element_size(), B, T, H, dk, dv, _stream(stream))
    _check(st, "retention_chunkwise_states")
    return workspace


def chunkwise_outputs(q, k, v, gamma, chunk, workspace, cu_seqlens=None, has_state_in=False,
                      g=None, gn_weight=None, gn_bias=None, eps=1e-5, out_dtype=None, out=None,
                      stream=None):
    """Output phase only: reads the workspace of a preceding chunkwise_states call."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (workspace, "workspace")):
        _dev(t, n)
    B, T, H, dk = q.shape
    dv = v.shape[3]
    nseq = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty(B, T, H, dv, device=q.device, dtype=out_dtype or q.dtype)
    ng = None
    if g is not None:
        _dev(g, "g")
        ng = NormGate(g.data_ptr(), _dt(g), gn_weight.data_ptr() if gn_weight is not None else None,
                      gn_bias.data_ptr() if gn_bias is not None else None, float(eps))
    st = lib().retention_chunkwise_outputs(
        _ptr(q), _ptr(k), _ptr(v), _dt(q), _gammas(gamma, H), int(chunk), _ptr(cu_seqlens), nseq,
        1 if has_state_in else 0, _ptr(out), _dt(out),
        ctypes.byref(ng) if ng is not None else None, _ptr(workspace),
        workspace.numel() * workspace.element_size(), B, T, H, dk, dv, _stream(stream))
    _check(st, "retention_chunkwise_outputs")
    return out


def chunkwise_fwd_static_ws(q, k, v, gamma, chunk, cu_seqlens=None, state_in=None,
                            state_out=None, g=None, gn_weight=None, gn_bias=None, eps=1e-5,
                            out=None, out_dtype=None, stream=None):
    """chunkwise_fwd without a workspace argument: the library uses its built-in
    device scratch (STATIC_WORKSPACE_BYTES) and allocates nothing itself.
    Outputs (and ``state_out``, if given) must be preallocated by the caller
    only if they are passed; here they are created with torch for convenience."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, n)
    B, T, H, dk = q.shape
    dv = v.shape[3]
    nseq = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty(B, T, H, dv, device=q.device, dtype=out_dtype or q.dtype)
    ng = None
    if g is not None:
        _dev(g, "g")
        ng = NormGate(g.data_ptr(), _dt(g), gn_weight.data_ptr() if gn_weight is not None else None,
                      gn_bias.data_ptr() if gn_bias is not None else None, float(eps))
    st = lib().retention_chunkwise_fwd_static_ws(
        _ptr(q), _ptr(k), _ptr(v), _dt(q), _gammas(gamma, H), int(chunk), _ptr(cu_seqlens), nseq,
        _ptr(state_in), _ptr(state_out), _ptr(out), _dt(out),
        ctypes.byref(ng) if ng is not None else None, B, T, H, dk, dv, _stream(stream))
    _check(st, "retention_chunkwise_fwd_static_ws")
    return out


def chunkwise_bwd_workspace_size(dtype, chunk, B, T, H, dk, dv, nseq=0):
    code = RET_F32 if dtype == torch.float32 else RET_BF16
    return int(lib().retention_chunkwise_bwd_workspace_size(code, chunk, B, T, H, dk, dv, nseq))


def chunkwise_bwd(q, k, v, d_out, gamma, chunk, cu_seqlens=None, state_in=None,
                  d_state_out=None, return_d_state=False, workspace=None, stream=None):
    """Gradients of the chunkwise form (retention_chunkwise_bwd).

    q, k: [B,T,H,dk]; v, d_out: [B,T,H,dv], one dtype; packed sequences as in
    :func:`chunkwise_fwd`.  ``state_in`` is the forward's initial state and
    ``d_state_out`` the gradient of its final state (float32 [nseq|B,H,dk,dv],
    optional).  Returns float32 ``(dq, dk, dv)`` and, with ``return_d_state``,
    the gradient of the initial state.
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (d_out, "d_out")):
        _dev(t, n)
    B, T, H, dk = q.shape
    dv = v.shape[3]
    if (k.shape != q.shape or v.shape[:3] != q.shape[:3] or d_out.shape != v.shape
            or len({q.dtype, k.dtype, v.dtype, d_out.dtype}) != 1):
        raise ValueError("q, k, v, d_out shapes/dtypes disagree")
    nseq = 0
    if cu_seqlens is not None:
        _dev(cu_seqlens, "cu_seqlens")
        if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
            raise ValueError("cu_seqlens must be a 1-D int32 tensor with at least two entries")
        nseq = cu_seqlens.numel() - 1
    nstate = nseq if nseq else B
    for t, n in ((state_in, "state_in"), (d_state_out, "d_state_out")):
        if t is not None:
            _dev(t, n)
            if t.dtype != torch.float32 or tuple(t.shape) != (nstate, H, dk, dv):
                raise ValueError(f"{n} must be float32 [{nstate},{H},{dk},{dv}]")
    dq = torch.empty(B, T, H, dk, device=q.device, dtype=torch.float32)
    dkk = torch.empty(B, T, H, dk, device=q.device, dtype=torch.float32)
    dvv = torch.empty(B, T, H, dv, device=q.device, dtype=torch.float32)
    dS0 = (torch.empty(nstate, H, dk, dv, device=q.device, dtype=torch.float32)
           if return_d_state else None)
    need = lib().retention_chunkwise_bwd_workspace_size(_dt(q), chunk, B, T, H, dk, dv, nseq)
    if need == 0:
        raise RetentionError(RET_ERR_UNSUPPORTED if max(dk, dv) > 256 else RET_ERR_INVALID_ARG,
                             "retention_chunkwise_bwd_workspace_size")
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    st = lib().retention_chunkwise_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(d_out), _dt(q), _gammas(gamma, H), int(chunk),
        _ptr(cu_seqlens), nseq, _ptr(state_in), _ptr(d_state_out), _ptr(dq), _ptr(dkk),
        _ptr(dvv), _ptr(dS0), _ptr(workspace), workspace.numel() * workspace.element_size(),
        B, T, H, dk, dv, _stream(stream))
    _check(st, "retention_chunkwise_bwd")
    return (dq, dkk, dvv, dS0) if return_d_state else (dq, dkk, dvv)


def rope(q, k, base=10000.0, cu_seqlens=None, q_out=None, k_out=None, stream=None):
    """Rotary position encoding of q and k ([B,T,H,d], one dtype; packed
    sequences as in :func:`chunkwise_fwd`).  Returns ``(q_out, k_out)``; pass
    ``q_out=q, k_out=k`` to rotate in place."""
    _dev(q, "q")
    _dev(k, "k")
    if k.shape != q.shape or k.dtype != q.dtype or q.dim() != 4:
        raise ValueError("q and k must have one [B,T,H,d] shape and one dtype")
    B, T, H, d = q.shape
    nseq = 0
    if cu_seqlens is not None:
        _dev(cu_seqlens, "cu_seqlens")
        if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
            raise ValueError("cu_seqlens must be a 1-D int32 tensor with at least two entries")
        nseq = cu_seqlens.numel() - 1
    q_out = torch.empty_like(q) if q_out is None else q_out
    k_out = torch.empty_like(k) if k_out is None else k_out
    for t, n in ((q_out, "q_out"), (k_out, "k_out")):
        _dev(t, n)
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError(f"{n} must match q")
    st = lib().retention_rope(_ptr(q), _ptr(k), _dt(q), _ptr(q_out), _ptr(k_out), float(base),
                              _ptr(cu_seqlens), nseq, B, T, H, d, _stream(stream))
    _check(st, "retention_rope")
    return q_out, k_out


def rla_fwd(q, k, v, window, cu_seqlens=None, out_dtype=None, out=None, workspace=None,
            stream=None):
    """Residual linear attention (retention_rla_fwd): o_t = softmax(q_t) S_(t-w-1)
    with S_t = S_(t-1) + softmax(k_t)^T v_t.  q, k: [B,T,H,dk]; v: [B,T,H,dv];
    packed sequences as in :func:`chunkwise_fwd`.  Returns o [B,T,H,dv]."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, n)
    B, T, H, dk = q.shape
    dv = v.shape[3]
    if k.shape != q.shape or v.shape[:3] != q.shape[:3] or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v shapes/dtypes disagree")
    nseq = 0
    if cu_seqlens is not None:
        _dev(cu_seqlens, "cu_seqlens")
        if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
            raise ValueError("cu_seqlens must be a 1-D int32 tensor with at least two entries")
        nseq = cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty(B, T, H, dv, device=q.device, dtype=out_dtype or q.dtype)
    _dev(out, "out")
    need = lib().retention_rla_workspace_size(_dt(q), B, T, H, dk, dv, nseq)
    if need == 0:
        raise RetentionError(RET_ERR_UNSUPPORTED, "retention_rla_workspace_size")
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    st = lib().retention_rla_fwd(_ptr(q), _ptr(k), _ptr(v), _dt(q), int(window), _ptr(cu_seqlens),
                                 nseq, _ptr(out), _dt(out), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), B, T, H, dk, dv,
                                 _stream(stream))
    _check(st, "retention_rla_fwd")
    return out


def recurrent_step(q, k, v, gamma, state, out_dtype=torch.float32, out=None, stream=None):
    """One decode step; updates ``state`` [N,H,dk,dv] in place and returns o [N,H,dv]."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (state, "state")):
        _dev(t, n)
    N, H, dk = q.shape
    dv = v.shape[2]
    if state.dtype != torch.float32 or tuple(state.shape) != (N, H, dk, dv):
        raise ValueError(f"state must be float32 [{N},{H},{dk},{dv}]")
    if out is None:
        out = torch.empty(N, H, dv, device=q.device, dtype=out_dtype)
    st = lib().retention_recurrent_step(_ptr(q), _ptr(k), _ptr(v), _dt(q), _gammas(gamma, H),
                                        _ptr(state), _ptr(out), _dt(out), N, H, dk, dv,
                                        _stream(stream))
    _check(st, "retention_recurrent_step")
    return out


def recurrent_steps(q, k, v, gamma, state, out_dtype=torch.float32, out=None, stream=None):
    """Tn (<= 16) decode steps in one pass over the state; q,k: [N,Tn,H,dk], v: [N,Tn,H,dv];
    updates ``state`` [N,H,dk,dv] in place and returns o [N,Tn,H,dv].  bf16 inputs with
    Tn >= 12, dk in {128, 256} and dv a multiple of 128 run on the tensor cores (tf32
    products on the float32 state, within the bf16-input tolerance); everything else runs
    in float32 on CUDA cores."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (state, "state")):
        _dev(t, n)
    N, Tn, H, dk = q.shape
    dv = v.shape[3]
    if state.dtype != torch.float32 or tuple(state.shape) != (N, H, dk, dv):
        raise ValueError(f"state must be float32 [{N},{H},{dk},{dv}]")
    if out is None:
        out = torch.empty(N, Tn, H, dv, device=q.device, dtype=out_dtype)
    else:
        _dev(out, "out")
    g = _gammas(gamma, H)
    st = lib().retention_recurrent_steps(_ptr(q), _ptr(k), _ptr(v), _dt(q), g, _ptr(state),
                                         _ptr(out), _dt(out), N, Tn, H, dk, dv, _stream(stream))
    _check(st, "retention_recurrent_steps")
    return out


def norm_gate(o, g, weight=None, bias=None, eps=1e-5, out_dtype=None, out=None, stream=None):
    """Per-head GroupNorm + swish gate; o: [ntok,H,dv] (any leading dims), g same size.
    ``out`` (optional) is a preallocated contiguous output of o's size."""
    _dev(o, "o")
    _dev(g, "g")
    H, dv = o.shape[-2], o.shape[-1]
    ntok = o.numel() // (H * dv)
    if g.numel() != o.numel():
        raise ValueError("g must have as many elements as o")
    if out is None:
        y = torch.empty(o.shape, device=o.device, dtype=out_dtype or o.dtype)
    else:
        _dev(out, "out")
        if out.numel() != o.numel():
            raise ValueError("out must have as many elements as o")
        y = out
    ng = NormGate(g.data_ptr(), _dt(g), weight.data_ptr() if weight is not None else None,
                  bias.data_ptr() if bias is not None else None, float(eps))
    st = lib().msr_norm_gate(_ptr(o), _dt(o), ctypes.byref(ng), _ptr(y), _dt(y), ntok, H, dv,
                             _stream(stream))
    _check(st, "msr_norm_gate")
    return y


def check_device_error(stream=None):
    """Synchronise the stream and raise if a kernel reported a device-side error."""
    _check(lib().retention_check_device_error(_stream(stream)), "retention_check_device_error")


def selftest_wait_timeout(stream=None):
    """Enqueue the failure-detection self-test: one bounded wait that is never
    satisfied.  A following check_device_error() raises RET_ERR_TIMEOUT."""
    _check(lib().retention_selftest_wait_timeout(_stream(stream)), "retention_selftest_wait_timeout")
