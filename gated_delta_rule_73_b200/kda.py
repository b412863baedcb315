"""Thin ctypes binding of ``libkda_b200.so`` (argument marshalling only).

Every function here has the name of the C entry point it calls and does no
arithmetic of its own: it checks tensor dtypes/devices/contiguity, reads the
sizes off the shapes, passes raw device pointers and the current CUDA stream,
and turns a negative status into ``KdaError``.  PyTorch only provides device
memory, streams and events.  If the shared library is missing the import
fails loudly -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkda_b200.so")

KDA_BF16, KDA_F32 = 0, 1
KDA_QK_L2NORM, KDA_COMPLEX, KDA_FUSED, KDA_SPLIT = 1, 2, 4, 8
KDA_UNBOUNDED_DECAY, KDA_GATE_SOFTPLUS = 16, 32
STATUS = {0: "KDA_OK", -1: "KDA_ERR_ARG", -2: "KDA_ERR_SHAPE", -3: "KDA_ERR_ALIGN",
          -4: "KDA_ERR_UNSUPPORTED", -5: "KDA_ERR_CUDA", -6: "KDA_ERR_TIMEOUT",
          -7: "KDA_ERR_WORKSPACE"}


class KdaError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS.get(status, status)} ({status_string(status)})")


class kda_opts(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("flags", ctypes.c_uint), ("scale", ctypes.c_float),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
                ("events", ctypes.POINTER(ctypes.c_void_p)), ("n_events", ctypes.c_int)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m gated_delta_rule_73_b200.build` (no CPU fallback exists)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, ip, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    op = ctypes.POINTER(kda_opts)
    lib.kda_chunk_fwd.argtypes = [vp] * 8 + [ip] * 5 + [op, vp]
    lib.kda_chunk_fwd.restype = ip
    lib.kda_recurrent_step.argtypes = [vp] * 7 + [ip] * 4 + [op, vp]
    lib.kda_recurrent_step.restype = ip
    lib.kda_chunk_fwd_prologue.argtypes = [vp] * 10 + [ip] * 5 + [op, vp]
    lib.kda_chunk_fwd_prologue.restype = ip
    lib.kda_chunk_fwd_gated.argtypes = [vp] * 10 + [ctypes.c_float] + [ip] * 5 + [op, vp]
    lib.kda_chunk_fwd_gated.restype = ip
    lib.kda_recurrent_step_prologue.argtypes = [vp] * 10 + [ip] * 4 + [op, vp]
    lib.kda_recurrent_step_prologue.restype = ip
    lib.kda_conv_state_from_prefill.argtypes = [vp] * 4 + [ip] * 4 + [op, vp]
    lib.kda_conv_state_from_prefill.restype = ip
    lib.kda_chunk_fwd_noalloc.argtypes = [vp] * 8 + [ip] * 5 + [op, vp]
    lib.kda_chunk_fwd_noalloc.restype = ip
    lib.kda_chunk_bwd.argtypes = [vp] * 14 + [ip] * 5 + [op, vp]
    lib.kda_chunk_bwd.restype = ip
    lib.kda_chunk_bwd_workspace_bytes.argtypes = [ip] * 5 + [op]
    lib.kda_chunk_bwd_workspace_bytes.restype = sz
    lib.kda_segment_pair.argtypes = [vp] * 7 + [ip] * 5 + [op, vp]
    lib.kda_segment_pair.restype = ip
    lib.kda_segment_pair_workspace_bytes.argtypes = [ip] * 5 + [op]
    lib.kda_segment_pair_workspace_bytes.restype = sz
    lib.kda_segment_forward.argtypes = [vp] * 8 + [ip] * 5 + [op, vp]
    lib.kda_segment_forward.restype = ip
    lib.kda_affine_combine.argtypes = [vp, vp, ip, vp, vp, ip, ip, ip, vp]
    lib.kda_affine_combine.restype = ip
    lib.kda_selftest_bounded_wait.argtypes = [ctypes.c_uint, vp]
    lib.kda_selftest_bounded_wait.restype = ip
    lib.kda_device_status.argtypes = [vp]
    lib.kda_device_status.restype = ip
    lib.kda_set_wait_limit.argtypes = [ctypes.c_uint]
    lib.kda_set_wait_limit.restype = ctypes.c_uint
    lib.kda_chunk_workspace_bytes.argtypes = [ip] * 5 + [op]
    lib.kda_chunk_workspace_bytes.restype = sz
    lib.kda_prologue_workspace_bytes.argtypes = [ip] * 5 + [op]
    lib.kda_prologue_workspace_bytes.restype = sz
    lib.kda_status_string.argtypes = [ip]
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_abi_version.argtypes = []
    lib.kda_abi_version.restype = ip
    return lib


_lib = _load()


def status_string(status: int) -> str:
    return _lib.kda_status_string(int(status)).decode()


def kda_abi_version() -> int:
    return _lib.kda_abi_version()


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return KDA_BF16
    if t == torch.float32:
        return KDA_F32
    raise TypeError(f"unsupported activation dtype {t}; use bfloat16 or float32")


def make_opts(dtype: torch.dtype = torch.bfloat16, *, l2norm: bool = True, complex_gate: bool = False,
              scale: float = 1.0, workspace: torch.Tensor | None = None, events=None,
              fused: bool | None = None, unbounded: bool = False,
              gate_softplus: bool = False) -> kda_opts:
    o = kda_opts()
    o.dtype = _dtype_code(dtype)
    o.flags = ((KDA_QK_L2NORM if l2norm else 0) | (KDA_COMPLEX if complex_gate else 0)
               | (0 if fused is None else KDA_FUSED if fused else KDA_SPLIT)
               | (KDA_UNBOUNDED_DECAY if unbounded else 0)
               | (KDA_GATE_SOFTPLUS if gate_softplus else 0))
    o.scale = float(scale)
    if workspace is not None:
        o.workspace = workspace.data_ptr()
        o.workspace_bytes = workspace.numel() * workspace.element_size()
    if events:
        arr = (ctypes.c_void_p * len(events))()
        for i, ev in enumerate(events):
            if not ev.cuda_event:
                ev.record()          # torch creates the CUDA event lazily
            arr[i] = ev.cuda_event
        o.events = ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))
        o.n_events = len(events)
        o._keep = arr                # keep the array alive with the struct
    return o


def _ptr(t, name, dtype=None, device_required=True):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if device_required and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    return t.data_ptr()


def _shapes(**named):
    """Check every tensor against the shape the C call will assume (None = optional, absent).
    The library receives raw pointers and sizes only, so a mismatch here would otherwise
    become an out-of-bounds device access."""
    for name, (t, shape) in named.items():
        if t is None:
            continue
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def kda_chunk_workspace_bytes(B, T, H, dk, dv, opts: kda_opts | None = None) -> int:
    return int(_lib.kda_chunk_workspace_bytes(B, T, H, dk, dv, ctypes.byref(opts) if opts else None))


def kda_prologue_workspace_bytes(B, T, H, dk, dv, opts: kda_opts | None = None) -> int:
    return int(_lib.kda_prologue_workspace_bytes(B, T, H, dk, dv, ctypes.byref(opts) if opts else None))


def kda_chunk_fwd(q, k, v, g, beta, S0, out, S_T, opts: kda_opts, stream=None) -> None:
    """Call ``kda_chunk_fwd``; q,k,g [B,T,H,dk], v,out [B,T,H,dv], beta [B,T,H]."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    _shapes(k=(k, q.shape), g=(g, q.shape), v=(v, (B, T, H, dv)), beta=(beta, (B, T, H)),
            S0=(S0, (B, H, dk, dv)), out=(out, (B, T, H, dv)), S_T=(S_T, (B, H, dk, dv)))
    args = [_ptr(q, "q", dt), _ptr(k, "k", dt), _ptr(v, "v", dt), _ptr(g, "g", dt),
            _ptr(beta, "beta", dt), _ptr(S0, "S0", torch.float32), _ptr(out, "out", dt),
            _ptr(S_T, "S_T", torch.float32)]
    st = _lib.kda_chunk_fwd(*args, B, T, H, dk, dv, ctypes.byref(opts), _stream(stream))
    if st != 0:
        raise KdaError("kda_chunk_fwd", st)


def kda_chunk_bwd_workspace_bytes(B, T, H, dk, dv, opts: kda_opts | None = None) -> int:
    return int(_lib.kda_chunk_bwd_workspace_bytes(B, T, H, dk, dv, ctypes.byref(opts) if opts else None))


def kda_chunk_bwd(q, k, v, g, beta, S0, dout, dS_T, grad_q, grad_k, grad_v, grad_g, grad_beta,
                  grad_S0, opts: kda_opts, stream=None) -> None:
    """Call ``kda_chunk_bwd``: FP32 gradients of <dout, O> + <dS_T, S_T> of kda_chunk_fwd."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    f = torch.float32
    sq, sv, sS = (B, T, H, dk), (B, T, H, dv), (B, H, dk, dv)
    _shapes(k=(k, sq), g=(g, sq), v=(v, sv), beta=(beta, (B, T, H)), S0=(S0, sS), dout=(dout, sv),
            dS_T=(dS_T, sS), grad_q=(grad_q, sq), grad_k=(grad_k, sq), grad_v=(grad_v, sv),
            grad_g=(grad_g, sq), grad_beta=(grad_beta, (B, T, H)), grad_S0=(grad_S0, sS))
    args = [_ptr(q, "q", dt), _ptr(k, "k", dt), _ptr(v, "v", dt), _ptr(g, "g", dt),
            _ptr(beta, "beta", dt), _ptr(S0, "S0", f), _ptr(dout, "dout", dt), _ptr(dS_T, "dS_T", f),
            _ptr(grad_q, "grad_q", f), _ptr(grad_k, "grad_k", f), _ptr(grad_v, "grad_v", f),
            _ptr(grad_g, "grad_g", f), _ptr(grad_beta, "grad_beta", f), _ptr(grad_S0, "grad_S0", f)]
    st = _lib.kda_chunk_bwd(*args, B, T, H, dk, dv, ctypes.byref(opts), _stream(stream))
    if st != 0:
        raise KdaError("kda_chunk_bwd", st)


def kda_segment_pair_workspace_bytes(B, T, H, dk, dv, opts: kda_opts | None = None) -> int:
    return int(_lib.kda_segment_pair_workspace_bytes(B, T, H, dk, dv,
                                                     ctypes.byref(opts) if opts else None))


def kda_segment_pair(q, k, v, g, beta, M_out, B_out, opts: kda_opts, stream=None) -> None:
    """Call ``kda_segment_pair``: the segment's affine pair (M [B,H,dk,dk], B [B,H,dk,dv])."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    f = torch.float32
    _shapes(k=(k, q.shape), g=(g, q.shape), v=(v, (B, T, H, dv)), beta=(beta, (B, T, H)),
            M_out=(M_out, (B, H, dk, dk)), B_out=(B_out, (B, H, dk, dv)))
    args = [_ptr(q, "q", dt), _ptr(k, "k", dt), _ptr(v, "v", dt), _ptr(g, "g", dt),
            _ptr(beta, "beta", dt), _ptr(M_out, "M_out", f), _ptr(B_out, "B_out", f)]
    st = _lib.kda_segment_pair(*args, B, T, H, dk, dv, ctypes.byref(opts), _stream(stream))
    if st != 0:
        raise KdaError("kda_segment_pair", st)


def kda_segment_forward(q, k, v, g, beta, S0, out, S_T, opts: kda_opts, stream=None) -> None:
    """Call ``kda_segment_forward``: the segment's forward from S0 over the records a preceding
    ``kda_segment_pair`` left in ``opts.workspace`` (same inputs and workspace)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    _shapes(k=(k, q.shape), g=(g, q.shape), v=(v, (B, T, H, dv)), beta=(beta, (B, T, H)),
            S0=(S0, (B, H, dk, dv)), out=(out, (B, T, H, dv)), S_T=(S_T, (B, H, dk, dv)))
    args = [_ptr(q, "q", dt), _ptr(k, "k", dt), _ptr(v, "v", dt), _ptr(g, "g", dt),
            _ptr(beta, "beta", dt), _ptr(S0, "S0", torch.float32), _ptr(out, "out", dt),
            _ptr(S_T, "S_T", torch.float32)]
    st = _lib.kda_segment_forward(*args, B, T, H, dk, dv, ctypes.byref(opts), _stream(stream))
    if st != 0:
        raise KdaError("kda_segment_forward", st)


def kda_affine_combine(M, Bp, n, S0, S_out, stream=None) -> None:
    """Call ``kda_affine_combine``: S_out = fold of pairs 0..n-1 of M [R,BH,dk,dk], Bp
    [R,BH,dk,dv] onto S0 [BH,dk,dv] (None = zero)."""
    dk, dv = S_out.shape[-2], S_out.shape[-1]
    BH = S_out.numel() // (dk * dv)
    f = torch.float32
    R = M.shape[0]
    if Bp.shape[0] != R or not 0 <= n <= R:
        raise ValueError("M and Bp must stack the same number of pairs R, and 0 <= n <= R")
    if M.numel() != R * BH * dk * dk or Bp.numel() != R * BH * dk * dv:
        raise ValueError(f"M must hold [R, {BH}, {dk}, {dk}] and Bp [R, {BH}, {dk}, {dv}] values")
    if S0 is not None and S0.numel() != BH * dk * dv:
        raise ValueError("S0 must have the shape of S_out")
    st = _lib.kda_affine_combine(_ptr(M, "M", f), _ptr(Bp, "Bp", f), int(n), _ptr(S0, "S0", f),
                                 _ptr(S_out, "S_out", f), BH, dk, dv, _stream(stream))
    if st != 0:
        raise KdaError("kda_affine_combine", st)


KDA_WAIT_LIMIT_DEFAULT = 1 << 22


def kda_device_status(stream=None) -> int:
    """Call ``kda_device_status``: synchronise the stream, read and clear the device error
    words; returns the status (0, or KDA_ERR_TIMEOUT = -6 when a bounded wait gave up)."""
    return int(_lib.kda_device_status(_stream(stream)))


def kda_set_wait_limit(polls: int) -> int:
    """Call ``kda_set_wait_limit``; returns the previous limit."""
    return int(_lib.kda_set_wait_limit(int(polls)))


def kda_selftest_bounded_wait(limit: int, stream=None) -> int:
    """Call ``kda_selftest_bounded_wait``; returns its status (KDA_ERR_TIMEOUT = -6 expected)."""
    return int(_lib.kda_selftest_bounded_wait(int(limit), _stream(stream)))


def kda_chunk_fwd_noalloc(q, k, v, g, beta, S0, out, S_T, opts: kda_opts, stream=None) -> None:
    """Call ``kda_chunk_fwd_noalloc``: kda_chunk_fwd with the library's fixed
    device scratch instead of a workspace, for callers that cannot allocate."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    _shapes(k=(k, q.shape), g=(g, q.shape), v=(v, (B, T, H, dv)), beta=(beta, (B, T, H)),
            S0=(S0, (B, H, dk, dv)), out=(out, (B, T, H, dv)), S_T=(S_T, (B, H, dk, dv)))
    args = [_ptr(q, "q", dt), _ptr(k, "k", dt), _ptr(v, "v", dt), _ptr(g, "g", dt),
            _ptr(beta, "beta", dt), _ptr(S0, "S0", torch.float32), _ptr(out, "out", dt),
            _ptr(S_T, "S_T", torch.float32)]
    st = _lib.kda_chunk_fwd_noalloc(*args, B, T, H, dk, dv, ctypes.byref(opts), _stream(stream))
    if st != 0:
        raise KdaError("kda_chunk_fwd_noalloc", st)


def kda_recurrent_step(q, k, v, g, beta, S, out, opts: kda_opts, stream=None) -> None:
    """Call ``kda_recurrent_step``; q,k,g [N,H,dk], v,out [N,H,dv], beta [N,H], S [N,H,dk,dv]."""
    N, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    _shapes(k=(k, q.shape), g=(g, q.shape), v=(v, (N, H, dv)), beta=(beta, (N, H)),
            S=(S, (N, H, dk, dv)), out=(out, (N, H, dv)))
    args = [_ptr(q, "q", dt), _ptr(k, "k", dt), _ptr(v, "v", dt), _ptr(g, "g", dt),
            _ptr(beta, "beta", dt), _ptr(S, "S", torch.float32), _ptr(out, "out", dt)]
    st = _lib.kda_recurrent_step(*args, N, H, dk, dv, ctypes.byref(opts), _stream(stream))
    if st != 0:
        raise KdaError("kda_recurrent_step", st)


def kda_chunk_fwd_prologue(q_pre, k_pre, v_pre, conv_w, z, A, beta_logit, S0, out, S_T,
                           opts: kda_opts, stream=None) -> None:
    """Call ``kda_chunk_fwd_prologue`` (raw branch inputs; see include/kda.h)."""
    B, T, H, dk = q_pre.shape
    dv = v_pre.shape[-1]
    dt = q_pre.dtype
    _shapes(k_pre=(k_pre, q_pre.shape), z=(z, q_pre.shape), v_pre=(v_pre, (B, T, H, dv)),
            conv_w=(conv_w, (3, H * dk, 4)), A=(A, (H,)), beta_logit=(beta_logit, (B, T, H)),
            S0=(S0, (B, H, dk, dv)), out=(out, (B, T, H, dv)), S_T=(S_T, (B, H, dk, dv)))
    args = [_ptr(q_pre, "q_pre", dt), _ptr(k_pre, "k_pre", dt), _ptr(v_pre, "v_pre", dt),
            _ptr(conv_w, "conv_w", dt), _ptr(z, "z", dt), _ptr(A, "A", torch.float32),
            _ptr(beta_logit, "beta_logit", torch.float32), _ptr(S0, "S0", torch.float32),
            _ptr(out, "out", dt), _ptr(S_T, "S_T", torch.float32)]
    st = _lib.kda_chunk_fwd_prologue(*args, B, T, H, dk, dv, ctypes.byref(opts), _stream(stream))
    if st != 0:
        raise KdaError("kda_chunk_fwd_prologue", st)


def kda_chunk_fwd_gated(q, k, v, g, beta, S0, out, S_T, out_gate, norm_weight, norm_eps: float,
                        opts: kda_opts, stream=None) -> None:
    """Call ``kda_chunk_fwd_gated``: kda_chunk_fwd + out = RMSNorm(o) * w * sigmoid(out_gate)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    _shapes(k=(k, q.shape), g=(g, q.shape), v=(v, (B, T, H, dv)), beta=(beta, (B, T, H)),
            S0=(S0, (B, H, dk, dv)), out=(out, (B, T, H, dv)), S_T=(S_T, (B, H, dk, dv)),
            out_gate=(out_gate, (B, T, H, dv)), norm_weight=(norm_weight, (dv,)))
    args = [_ptr(q, "q", dt), _ptr(k, "k", dt), _ptr(v, "v", dt), _ptr(g, "g", dt),
            _ptr(beta, "beta", dt), _ptr(S0, "S0", torch.float32), _ptr(out, "out", dt),
            _ptr(S_T, "S_T", torch.float32), _ptr(out_gate, "out_gate", dt),
            _ptr(norm_weight, "norm_weight", torch.float32)]
    st = _lib.kda_chunk_fwd_gated(*args, float(norm_eps), B, T, H, dk, dv, ctypes.byref(opts),
                                  _stream(stream))
    if st != 0:
        raise KdaError("kda_chunk_fwd_gated", st)


def kda_recurrent_step_prologue(q_pre, k_pre, v_pre, conv_w, conv_state, z, A, beta_logit, S, out,
                                opts: kda_opts, stream=None) -> None:
    """Call ``kda_recurrent_step_prologue``; q_pre,k_pre,z [N,H,dk], v_pre,out [N,H,dv],
    conv_w [3,H*dk,4], conv_state [N,3,3,H*dk] (updated), A [H], beta_logit [N,H], S updated."""
    N, H, dk = q_pre.shape
    dv = v_pre.shape[-1]
    dt = q_pre.dtype
    _shapes(k_pre=(k_pre, q_pre.shape), z=(z, q_pre.shape), v_pre=(v_pre, (N, H, dv)),
            conv_w=(conv_w, (3, H * dk, 4)), conv_state=(conv_state, (N, 3, 3, H * dk)),
            A=(A, (H,)), beta_logit=(beta_logit, (N, H)), S=(S, (N, H, dk, dv)),
            out=(out, (N, H, dv)))
    args = [_ptr(q_pre, "q_pre", dt), _ptr(k_pre, "k_pre", dt), _ptr(v_pre, "v_pre", dt),
            _ptr(conv_w, "conv_w", dt), _ptr(conv_state, "conv_state", dt), _ptr(z, "z", dt),
            _ptr(A, "A", torch.float32), _ptr(beta_logit, "beta_logit", torch.float32),
            _ptr(S, "S", torch.float32), _ptr(out, "out", dt)]
    st = _lib.kda_recurrent_step_prologue(*args, N, H, dk, dv, ctypes.byref(opts), _stream(stream))
    if st != 0:
        raise KdaError("kda_recurrent_step_prologue", st)


def kda_conv_state_from_prefill(q_pre, k_pre, v_pre, conv_state, opts: kda_opts, stream=None) -> None:
    """Call ``kda_conv_state_from_prefill``: raw inputs [B,T,H,d] -> conv_state [B,3,3,H*d]."""
    B, T, H, d = q_pre.shape
    dt = q_pre.dtype
    _shapes(k_pre=(k_pre, q_pre.shape), v_pre=(v_pre, q_pre.shape),
            conv_state=(conv_state, (B, 3, 3, H * d)))
    args = [_ptr(q_pre, "q_pre", dt), _ptr(k_pre, "k_pre", dt), _ptr(v_pre, "v_pre", dt),
            _ptr(conv_state, "conv_state", dt)]
    st = _lib.kda_conv_state_from_prefill(*args, B, T, H, d, ctypes.byref(opts), _stream(stream))
    if st != 0:
        raise KdaError("kda_conv_state_from_prefill", st)


# ------------------------------------------------------------------ conveniences
def chunk_fwd(q, k, v, g, beta, S0=None, *, l2norm=True, complex_gate=False, scale=1.0,
              fused=None, unbounded=False, workspace=None, out=None, S_T=None, stream=None):
    """Allocate out / S_T / workspace with torch and run ``kda_chunk_fwd``."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    opts = make_opts(q.dtype, l2norm=l2norm, complex_gate=complex_gate, scale=scale, fused=fused,
                     unbounded=unbounded)
    if workspace is None:
        nbytes = kda_chunk_workspace_bytes(B, T, H, dk, dv, opts)
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    opts = make_opts(q.dtype, l2norm=l2norm, complex_gate=complex_gate, scale=scale,
                     workspace=workspace, fused=fused, unbounded=unbounded)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if S_T is None:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    kda_chunk_fwd(q, k, v, g, beta, S0, out, S_T, opts, stream)
    return out, S_T


def chunk_bwd(q, k, v, g, beta, S0, dout, dS_T=None, *, l2norm=True, complex_gate=False,
              scale=1.0, workspace=None, want_dS0=True, stream=None):
    """Allocate the FP32 gradients and the workspace with torch and run ``kda_chunk_bwd``;
    returns (dq, dk, dv, dg, dbeta, dS0 or None)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    opts = make_opts(q.dtype, l2norm=l2norm, complex_gate=complex_gate, scale=scale)
    if workspace is None:
        nbytes = kda_chunk_bwd_workspace_bytes(B, T, H, dk, dv, opts)
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    opts = make_opts(q.dtype, l2norm=l2norm, complex_gate=complex_gate, scale=scale,
                     workspace=workspace)
    e = lambda *shape: torch.empty(shape, dtype=torch.float32, device=q.device)
    grads = (e(B, T, H, dk), e(B, T, H, dk), e(B, T, H, dv), e(B, T, H, dk), e(B, T, H),
             e(B, H, dk, dv) if want_dS0 else None)
    kda_chunk_bwd(q, k, v, g, beta, S0, dout, dS_T, *grads, opts, stream)
    return grads


def segment_pair(q, k, v, g, beta, *, l2norm=True, complex_gate=False, fused=None,
                 unbounded=False, workspace=None, stream=None):
    """Run ``kda_segment_pair`` (workspace allocated unless given; pass the same one to
    ``segment_forward`` afterwards); returns (M, B)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    kw = dict(l2norm=l2norm, complex_gate=complex_gate, fused=fused, unbounded=unbounded)
    ws = workspace
    if ws is None:
        nbytes = kda_segment_pair_workspace_bytes(B, T, H, dk, dv, make_opts(q.dtype, **kw))
        ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    M = torch.empty((B, H, dk, dk), dtype=torch.float32, device=q.device)
    Bm = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    kda_segment_pair(q, k, v, g, beta, M, Bm, make_opts(q.dtype, workspace=ws, **kw), stream)
    return M, Bm


def segment_forward(q, k, v, g, beta, S0, workspace, *, l2norm=True, complex_gate=False, scale=1.0,
                    fused=None, unbounded=False, out=None, S_T=None, stream=None):
    """Run ``kda_segment_forward`` with the workspace a ``segment_pair`` call on the same inputs
    filled; returns (out, S_T)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    opts = make_opts(q.dtype, l2norm=l2norm, complex_gate=complex_gate, scale=scale, fused=fused,
                     unbounded=unbounded, workspace=workspace)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if S_T is None:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    kda_segment_forward(q, k, v, g, beta, S0, out, S_T, opts, stream)
    return out, S_T


def affine_combine(Ms, Bs, n, S0=None, *, out=None, stream=None):
    """Run ``kda_affine_combine`` over stacked pairs Ms [R,B,H,dk,dk], Bs [R,B,H,dk,dv]."""
    if out is None:
        out = torch.empty(Bs.shape[1:], dtype=torch.float32, device=Bs.device)
    kda_affine_combine(Ms, Bs, n, S0, out, stream)
    return out


def recurrent_step(q, k, v, g, beta, S, *, l2norm=True, complex_gate=False, scale=1.0,
                   out=None, stream=None):
    """Run ``kda_recurrent_step`` (S updated in place); returns out."""
    if out is None:
        out = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    opts = make_opts(q.dtype, l2norm=l2norm, complex_gate=complex_gate, scale=scale)
    kda_recurrent_step(q, k, v, g, beta, S, out, opts, stream)
    return out


def chunk_fwd_gated(q, k, v, g, beta, S0, out_gate, norm_weight=None, *, norm_eps=1e-5,
                    l2norm=True, complex_gate=False, scale=1.0, fused=None, unbounded=False,
                    stream=None):
    """Allocate and run ``kda_chunk_fwd_gated``; returns (out, S_T)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    kw = dict(l2norm=l2norm, complex_gate=complex_gate, scale=scale, fused=fused, unbounded=unbounded)
    opts = make_opts(q.dtype, **kw)
    nbytes = kda_chunk_workspace_bytes(B, T, H, dk, dv, opts)
    workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    opts = make_opts(q.dtype, workspace=workspace, **kw)
    out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    kda_chunk_fwd_gated(q, k, v, g, beta, S0, out, S_T, out_gate, norm_weight, norm_eps, opts, stream)
    return out, S_T


def recurrent_step_prologue(q_pre, k_pre, v_pre, conv_w, conv_state, z, A, beta_logit, S, *,
                            scale=1.0, gate_softplus=False, out=None, stream=None):
    """Run ``kda_recurrent_step_prologue`` (S and conv_state updated in place); returns out."""
    if out is None:
        out = torch.empty(v_pre.shape, dtype=q_pre.dtype, device=q_pre.device)
    opts = make_opts(q_pre.dtype, scale=scale, gate_softplus=gate_softplus)
    kda_recurrent_step_prologue(q_pre, k_pre, v_pre, conv_w, conv_state, z, A, beta_logit, S, out,
                                opts, stream)
    return out


def conv_state_from_prefill(q_pre, k_pre, v_pre, *, out=None, stream=None):
    """Return the decode conv state [B,3,3,H*d] continuing a prefill over q_pre, k_pre, v_pre."""
    B, T, H, d = q_pre.shape
    if out is None:
        out = torch.empty((B, 3, 3, H * d), dtype=q_pre.dtype, device=q_pre.device)
    kda_conv_state_from_prefill(q_pre, k_pre, v_pre, out, make_opts(q_pre.dtype), stream)
    return out


def chunk_fwd_prologue(q_pre, k_pre, v_pre, conv_w, z, A, beta_logit, S0=None, *, scale=1.0,
                       fused=None, gate_softplus=False, workspace=None, out=None, S_T=None,
                       stream=None):
    """Allocate and run ``kda_chunk_fwd_prologue``."""
    B, T, H, dk = q_pre.shape
    dv = v_pre.shape[-1]
    opts = make_opts(q_pre.dtype, scale=scale, fused=fused, gate_softplus=gate_softplus)
    if workspace is None:
        nbytes = kda_prologue_workspace_bytes(B, T, H, dk, dv, opts)
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q_pre.device)
    opts = make_opts(q_pre.dtype, scale=scale, workspace=workspace, fused=fused,
                     gate_softplus=gate_softplus)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q_pre.dtype, device=q_pre.device)
    if S_T is None:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q_pre.device)
    kda_chunk_fwd_prologue(q_pre, k_pre, v_pre, conv_w, z, A, beta_logit, S0, out, S_T, opts, stream)
    return out, S_T
