"""Thin torch binding of libmdn.  Argument marshalling only: every step of the
forward pass and of the decode step runs in the library's CUDA kernels.

Device tensors in -> device tensors out, on the current CUDA stream.  Host
(CPU) tensors are copied to the current device first and the results copied
back (pinned host memory makes those copies asynchronous).
"""
from __future__ import annotations

import threading
from typing import Optional

import torch

from . import _lib

_lock = threading.Lock()
_handle = None


def library():
    """The loaded libmdn (ctypes.CDLL)."""
    global _handle
    with _lock:
        if _handle is None:
            _handle = _lib.load()
        return _handle


class MDNError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {status_string(status)}"
        if status == _lib.MDN_ERR_CUDA:
            msg += f" [{library().mdn_last_cuda_error().decode()}]"
        super().__init__(msg)


def status_string(status: int) -> str:
    return library().mdn_status_string(int(status)).decode()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return _lib.MDN_F32
    if t.dtype == torch.bfloat16:
        return _lib.MDN_BF16
    raise TypeError(f"q, k, v must be float32 or bfloat16, got {t.dtype}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _check(status: int, where: str):
    if status != _lib.MDN_OK:
        raise MDNError(status, where)


def _stream_handle(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _need(t: Optional[torch.Tensor], dtype, shape, name):
    if t is None:
        return
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous {dtype} {tuple(shape)}, "
                         f"got {t.dtype} {tuple(t.shape)} contiguous={t.is_contiguous()}")


def chunk_fwd_workspace_size(B: int, T: int, H: int, d: int, C: int = 64,
                             dtype: torch.dtype = torch.bfloat16, flags: int = 0) -> int:
    """Scratch bytes of :func:`chunk_fwd` for these sizes and flags (the path they select)."""
    code = _lib.MDN_BF16 if dtype == torch.bfloat16 else _lib.MDN_F32
    return int(library().mdn_chunk_fwd_workspace_size_flags(B, T, H, d, d, C, code, int(flags)))


def chunk_fwd_status(workspace: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> int:
    """Synchronises ``stream`` and returns the status code that the kernels of the
    last chunk pass on ``workspace`` recorded (0 = MDN_OK; MDN_ERR_TIMEOUT means a
    bounded device wait ran out and the outputs are undefined)."""
    return int(library().mdn_chunk_fwd_status(_ptr(workspace), _stream_handle(stream)))


def chunk_fwd(q, k, v, alpha_log, mu_log, beta, eta, d: float = 0.5, S0=None, M0=None,
              C: int = 64, *, out=None, workspace: Optional[torch.Tensor] = None,
              flags: int = 0, stream: Optional[torch.cuda.Stream] = None):
    """Chunkwise MDN forward pass.  Returns (o, vtilde, S_T, M_T).

    q, k, v: [B,T,H,d] float32 or bfloat16; gates [B,T,H] float32; S0, M0
    [B,H,d,d] float32 or None.  ``out`` may hold preallocated (o, vtilde, S_T,
    M_T).  Host inputs are copied to the current device and results back.
    """
    if not q.is_cuda:
        dev = torch.device("cuda", torch.cuda.current_device())
        mv = lambda t: None if t is None else t.to(dev, non_blocking=True)
        res = chunk_fwd(mv(q), mv(k), mv(v), mv(alpha_log), mv(mu_log), mv(beta), mv(eta),
                        d, mv(S0), mv(M0), C, workspace=workspace, flags=flags,
                        stream=stream)
        if out is not None:
            for dst, src in zip(out, res):
                dst.copy_(src, non_blocking=True)
            return out
        return tuple(t.to("cpu") for t in res)
    B, T, H, D = q.shape
    code = _dtype_code(q)
    for name, t in (("k", k), ("v", v)):
        _need(t, q.dtype, q.shape, name)
    _need(q, q.dtype, q.shape, "q")
    for name, t in (("alpha_log", alpha_log), ("mu_log", mu_log), ("beta", beta), ("eta", eta)):
        _need(t, torch.float32, (B, T, H), name)
    _need(S0, torch.float32, (B, H, D, D), "S0")
    _need(M0, torch.float32, (B, H, D, D), "M0")
    if out is None:
        o = torch.empty_like(q)
        vt = torch.empty_like(q)
        S_T = torch.empty((B, H, D, D), dtype=torch.float32, device=q.device)
        M_T = torch.empty((B, H, D, D), dtype=torch.float32, device=q.device)
    else:
        o, vt, S_T, M_T = out
        _need(o, q.dtype, q.shape, "o")
        _need(vt, q.dtype, q.shape, "vtilde")
        _need(S_T, torch.float32, (B, H, D, D), "S_T")
        _need(M_T, torch.float32, (B, H, D, D), "M_T")
    lib = library()
    ws_bytes = int(lib.mdn_chunk_fwd_workspace_size_flags(B, T, H, D, D, C, code, int(flags)))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    status = lib.mdn_chunk_fwd(
        _ptr(q), _ptr(k), _ptr(v), code, _ptr(alpha_log), _ptr(mu_log), _ptr(beta), _ptr(eta),
        float(d), _ptr(S0), _ptr(M0), B, T, H, D, D, C, _ptr(o), _ptr(vt), _ptr(S_T), _ptr(M_T),
        _ptr(workspace), workspace.numel(), int(flags), _stream_handle(stream))
    _check(status, "mdn_chunk_fwd")
    return o, vt, S_T, M_T


def chunk_fwd_preact(q, k, v, x_eta, a, b, c, s: float = 1.0, mu_log_min: float = -2.0,
                     eta_act: str = "tanh", d: float = 0.5, S0=None, M0=None, C: int = 64, *,
                     out=None, workspace: Optional[torch.Tensor] = None, flags: int = 0,
                     stream: Optional[torch.cuda.Stream] = None):
    """:func:`chunk_fwd` with the gates computed inside the pass from their
    pre-activations x_eta, a, b, c ([B,T,H] float32; see :func:`gate_params`).
    Returns (o, vtilde, S_T, M_T)."""
    if eta_act not in _ETA_ACT:
        raise ValueError(f"eta_act must be one of {sorted(_ETA_ACT)}, got {eta_act!r}")
    B, T, H, D = q.shape
    code = _dtype_code(q)
    for name, t in (("k", k), ("v", v)):
        _need(t, q.dtype, q.shape, name)
    for name, t in (("x_eta", x_eta), ("a", a), ("b", b), ("c", c)):
        _need(t, torch.float32, (B, T, H), name)
    _need(S0, torch.float32, (B, H, D, D), "S0")
    _need(M0, torch.float32, (B, H, D, D), "M0")
    if out is None:
        out = (torch.empty_like(q), torch.empty_like(q),
               torch.empty((B, H, D, D), dtype=torch.float32, device=q.device),
               torch.empty((B, H, D, D), dtype=torch.float32, device=q.device))
    o, vt, S_T, M_T = out
    lib = library()
    ws_bytes = int(lib.mdn_chunk_fwd_workspace_size_flags(B, T, H, D, D, C, code, int(flags)))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    status = lib.mdn_chunk_fwd_preact(
        _ptr(q), _ptr(k), _ptr(v), code, _ptr(x_eta), _ptr(a), _ptr(b), _ptr(c), float(s),
        float(mu_log_min), _ETA_ACT[eta_act], float(d), _ptr(S0), _ptr(M0), B, T, H, D, D, C,
        _ptr(o), _ptr(vt), _ptr(S_T), _ptr(M_T), _ptr(workspace), workspace.numel(), int(flags),
        _stream_handle(stream))
    _check(status, "mdn_chunk_fwd_preact")
    return o, vt, S_T, M_T


def chunk_bwd(q, k, v, alpha_log, mu_log, beta, eta, d: float, vtilde, d_o, S0=None, M0=None,
              dS_T=None, dM_T=None, C: int = 64, *, workspace: Optional[torch.Tensor] = None,
              flags: int = 0, stream: Optional[torch.cuda.Stream] = None) -> dict:
    """Backward pass of :func:`chunk_fwd` from its saved ``vtilde``.  Returns a
    dict of fp32 tensors: dq, dk, dv, dalpha_log, dmu_log, dbeta, deta, dS0, dM0."""
    B, T, H, D = q.shape
    code = _dtype_code(q)
    for name, t in (("q", q), ("k", k), ("v", v), ("vtilde", vtilde), ("d_o", d_o)):
        _need(t, q.dtype, q.shape, name)
    for name, t in (("alpha_log", alpha_log), ("mu_log", mu_log), ("beta", beta), ("eta", eta)):
        _need(t, torch.float32, (B, T, H), name)
    for name, t in (("S0", S0), ("M0", M0), ("dS_T", dS_T), ("dM_T", dM_T)):
        _need(t, torch.float32, (B, H, D, D), name)
    f32 = lambda *s_: torch.empty(s_, dtype=torch.float32, device=q.device)
    g = dict(dq=f32(B, T, H, D), dk=f32(B, T, H, D), dv=f32(B, T, H, D),
             dalpha_log=f32(B, T, H), dmu_log=f32(B, T, H), dbeta=f32(B, T, H),
             deta=f32(B, T, H), dS0=f32(B, H, D, D), dM0=f32(B, H, D, D))
    lib = library()
    ws_bytes = int(lib.mdn_chunk_bwd_workspace_size(B, T, H, D, D, C, code))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    status = lib.mdn_chunk_bwd(
        _ptr(q), _ptr(k), _ptr(v), code, _ptr(alpha_log), _ptr(mu_log), _ptr(beta), _ptr(eta),
        float(d), _ptr(S0), _ptr(M0), _ptr(vtilde), _ptr(d_o), _ptr(dS_T), _ptr(dM_T),
        B, T, H, D, D, C, *(_ptr(g[n]) for n in ("dq", "dk", "dv", "dalpha_log", "dmu_log",
                                                  "dbeta", "deta", "dS0", "dM0")),
        _ptr(workspace), workspace.numel(), int(flags), _stream_handle(stream))
    _check(status, "mdn_chunk_bwd")
    return g


def chunk_fwd_varlen(q, k, v, alpha_log, mu_log, beta, eta, cu_seqlens: torch.Tensor,
                     d: float = 0.5, S0=None, M0=None, C: int = 64, *, out=None,
                     workspace: Optional[torch.Tensor] = None, flags: int = 0,
                     stream: Optional[torch.cuda.Stream] = None):
    """Chunkwise pass over N sequences packed along the token axis.

    q, k, v: [total_T,H,d]; gates [total_T,H] float32; cu_seqlens: int32
    [N+1] on the device (sequence s is tokens cu_seqlens[s]:cu_seqlens[s+1]);
    S0, M0: [N,H,d,d] float32 or None.  Returns (o, vtilde, S_T, M_T)."""
    total_T, H, D = q.shape
    N = cu_seqlens.numel() - 1
    if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_contiguous() or N < 0:
        raise ValueError("cu_seqlens: expected a contiguous int32 tensor of N+1 offsets")
    if cu_seqlens.device != q.device:
        raise ValueError("cu_seqlens must be on the same device as q")
    code = _dtype_code(q)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, q.dtype, q.shape, name)
    for name, t in (("alpha_log", alpha_log), ("mu_log", mu_log), ("beta", beta), ("eta", eta)):
        _need(t, torch.float32, (total_T, H), name)
    _need(S0, torch.float32, (N, H, D, D), "S0")
    _need(M0, torch.float32, (N, H, D, D), "M0")
    if out is None:
        o = torch.empty_like(q)
        vt = torch.empty_like(q)
        S_T = torch.empty((N, H, D, D), dtype=torch.float32, device=q.device)
        M_T = torch.empty((N, H, D, D), dtype=torch.float32, device=q.device)
    else:
        o, vt, S_T, M_T = out
        _need(o, q.dtype, q.shape, "o")
        _need(vt, q.dtype, q.shape, "vtilde")
        _need(S_T, torch.float32, (N, H, D, D), "S_T")
        _need(M_T, torch.float32, (N, H, D, D), "M_T")
    lib = library()
    ws_bytes = int(lib.mdn_chunk_fwd_varlen_workspace_size_flags(N, total_T, H, D, D, C, code,
                                                                 int(flags)))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    status = lib.mdn_chunk_fwd_varlen(
        _ptr(q), _ptr(k), _ptr(v), code, _ptr(alpha_log), _ptr(mu_log), _ptr(beta), _ptr(eta),
        float(d), _ptr(cu_seqlens), N, total_T, _ptr(S0), _ptr(M0), H, D, D, C, _ptr(o),
        _ptr(vt), _ptr(S_T), _ptr(M_T), _ptr(workspace), workspace.numel(), int(flags),
        _stream_handle(stream))
    _check(status, "mdn_chunk_fwd_varlen")
    return o, vt, S_T, M_T


def step(q, k, v, alpha_log, mu_log, beta, eta, d: float, S: torch.Tensor, M: torch.Tensor,
         *, o: Optional[torch.Tensor] = None, vtilde: Optional[torch.Tensor] = None,
         want_vtilde: bool = True, stream: Optional[torch.cuda.Stream] = None):
    """One decode token: S, M [B,H,d,d] float32 are updated in place.
    q, k, v: [B,H,d]; gates [B,H].  Returns (o, vtilde or None)."""
    B, H, D = q.shape
    code = _dtype_code(q)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, q.dtype, (B, H, D), name)
    for name, t in (("alpha_log", alpha_log), ("mu_log", mu_log), ("beta", beta), ("eta", eta)):
        _need(t, torch.float32, (B, H), name)
    _need(S, torch.float32, (B, H, D, D), "S")
    _need(M, torch.float32, (B, H, D, D), "M")
    if o is None:
        o = torch.empty_like(q)
    if vtilde is None and want_vtilde:
        vtilde = torch.empty_like(q)
    status = library().mdn_step(
        _ptr(q), _ptr(k), _ptr(v), code, _ptr(alpha_log), _ptr(mu_log), _ptr(beta), _ptr(eta),
        float(d), _ptr(S), _ptr(M), B, H, D, D, _ptr(o), _ptr(vtilde), 0, _stream_handle(stream))
    _check(status, "mdn_step")
    return o, vtilde


def step_with_delta_norm(q, k, v, alpha_log, mu_log, beta, eta, d: float, S: torch.Tensor,
                         M: torch.Tensor, *, o: Optional[torch.Tensor] = None,
                         vtilde: Optional[torch.Tensor] = None, ds_norm: Optional[torch.Tensor] = None,
                         want_vtilde: bool = True, stream: Optional[torch.cuda.Stream] = None):
    """As :func:`step`, and also returns ds_norm [B,H] = ||S_t - S_{t-1}||_F per head."""
    B, H, D = q.shape
    code = _dtype_code(q)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, q.dtype, (B, H, D), name)
    for name, t in (("alpha_log", alpha_log), ("mu_log", mu_log), ("beta", beta), ("eta", eta)):
        _need(t, torch.float32, (B, H), name)
    _need(S, torch.float32, (B, H, D, D), "S")
    _need(M, torch.float32, (B, H, D, D), "M")
    if o is None:
        o = torch.empty_like(q)
    if vtilde is None and want_vtilde:
        vtilde = torch.empty_like(q)
    if ds_norm is None:
        ds_norm = torch.empty((B, H), dtype=torch.float32, device=q.device)
    _need(ds_norm, torch.float32, (B, H), "ds_norm")
    status = library().mdn_step_delta_norm(
        _ptr(q), _ptr(k), _ptr(v), code, _ptr(alpha_log), _ptr(mu_log), _ptr(beta), _ptr(eta),
        float(d), _ptr(S), _ptr(M), B, H, D, D, _ptr(o), _ptr(vtilde), _ptr(ds_norm), 0,
        _stream_handle(stream))
    _check(status, "mdn_step_delta_norm")
    return o, vtilde, ds_norm


_ETA_ACT = {"tanh": 0, "2sigmoid": 1}


def gate_params(x_eta, a, b, c, s: float = 1.0, mu_log_min: float = -2.0,
                eta_act: str = "tanh", *, out=None, stream: Optional[torch.cuda.Stream] = None):
    """The four gates from pre-activations of any common shape (fp32, contiguous).
    Returns (alpha_log, mu_log, beta, eta) of that shape."""
    if eta_act not in _ETA_ACT:
        raise ValueError(f"eta_act must be one of {sorted(_ETA_ACT)}, got {eta_act!r}")
    shape = tuple(x_eta.shape)
    for name, t in (("x_eta", x_eta), ("a", a), ("b", b), ("c", c)):
        _need(t, torch.float32, shape, name)
    if out is None:
        out = tuple(torch.empty_like(x_eta) for _ in range(4))
    for name, t in zip(("alpha_log", "mu_log", "beta", "eta"), out):
        _need(t, torch.float32, shape, name)
    status = library().mdn_gate_params(
        _ptr(x_eta), _ptr(a), _ptr(b), _ptr(c), x_eta.numel(), float(s), float(mu_log_min),
        _ETA_ACT[eta_act], *(_ptr(t) for t in out), _stream_handle(stream))
    _check(status, "mdn_gate_params")
    return tuple(out)


def chunk_gate_prep(alpha_log, mu_log, beta, eta, C: int = 64, with_gamma: bool = True,
                    stream: Optional[torch.cuda.Stream] = None):
    """Chunk coefficients: (la, lm, lc, b) [B,H,NT*C] and gamma [B,H,NT,C,C] (or None)."""
    B, T, H = alpha_log.shape
    for name, t in (("alpha_log", alpha_log), ("mu_log", mu_log), ("beta", beta), ("eta", eta)):
        _need(t, torch.float32, (B, T, H), name)
    NT = (T + C - 1) // C
    mk = lambda *s: torch.empty(s, dtype=torch.float32, device=alpha_log.device)
    la, lm, lc, bco = (mk(B, H, NT * C) for _ in range(4))
    gamma = mk(B, H, NT, C, C) if with_gamma else None
    status = library().mdn_chunk_gate_prep(
        _ptr(alpha_log), _ptr(mu_log), _ptr(beta), _ptr(eta), B, T, H, C, _ptr(la), _ptr(lm),
        _ptr(lc), _ptr(bco), _ptr(gamma), _stream_handle(stream))
    _check(status, "mdn_chunk_gate_prep")
    return la, lm, lc, bco, gamma


def profile_enable(on: bool = True) -> bool:
    """Start/stop per-kernel event timing inside the library (see mdn.h)."""
    prev = library().mdn_profile_enable(1 if on else 0)
    if prev < 0:
        raise RuntimeError("mdn_profile_enable: could not create CUDA events")
    return bool(prev)


def profile_read(reset: bool = True) -> dict:
    """{kernel name: (total device ms, launches)} since the last reset."""
    import ctypes
    cap = 32
    names = (ctypes.c_char_p * cap)()
    ms = (ctypes.c_double * cap)()
    cnt = (ctypes.c_longlong * cap)()
    n = library().mdn_profile_read(1 if reset else 0, names, ms, cnt, cap)
    if n < 0:
        raise RuntimeError("mdn_profile_read failed")
    return {names[i].decode(): (ms[i], int(cnt[i])) for i in range(n)}
