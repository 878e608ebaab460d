"""Python binding of libosdn (the C ABI in include/osdn.h): argument marshalling only.

Every function here takes CUDA tensors, checks their dtype/shape/contiguity, allocates the
outputs the caller did not pass (``torch.empty`` on the inputs' device), and calls the
C entry point of the same name on the current CUDA stream.  All arithmetic runs in the
library's kernels.  There is no fallback: if ``libosdn.so`` is missing, importing this module
raises, and a non-OK status raises :class:`OsdnError`.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# OSDN_LIBRARY selects another build of the library (the debug-bounds build, libosdn_debug.so)
LIB_PATH = os.environ.get("OSDN_LIBRARY") or os.path.join(_PKG, "libosdn.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "osdn.h")

OSDN_OK = 0
OSDN_ERR_INVALID_ARG = 1
OSDN_ERR_UNSUPPORTED = 2
OSDN_ERR_ALIGNMENT = 3
OSDN_ERR_CUDA = 4
OSDN_ERR_DEVICE_TIMEOUT = 5
OSDN_ERR_DEVICE_BOUNDS = 6
OSDN_BF16 = 0
OSDN_F32 = 1

_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_f32 = ctypes.c_float


class OsdnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m delta_rule_recurrent_osdn_b200.build`"
            " (there is no non-CUDA implementation)")
    lib = ctypes.CDLL(LIB_PATH)
    lib.osdn_abi_version.argtypes = []
    lib.osdn_abi_version.restype = _i32
    lib.osdn_status_string.argtypes = [ctypes.c_int]
    lib.osdn_status_string.restype = ctypes.c_char_p
    lib.osdn_precond_scan.argtypes = [_vp, _vp, _vp, _f32, _vp, _vp, _vp, _vp, _vp, _i32, _i32,
                                      _i32, _i32, _i32, ctypes.c_int, _vp]
    lib.osdn_precond_scan.restype = ctypes.c_int
    lib.osdn_chunk_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _f32, _vp, _vp, _vp, _vp,
                                   _i32, _i32, _i32, _i32, _i32, _i32, _i32, ctypes.c_int, _vp]
    lib.osdn_chunk_fwd.restype = ctypes.c_int
    lib.osdn_fwd_workspace_bytes.argtypes = [_i32, _i32, _i32, _i32, ctypes.c_int]
    lib.osdn_fwd_workspace_bytes.restype = ctypes.c_size_t
    lib.osdn_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _f32, _vp, _vp, _f32, _vp, _vp,
                             _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32,
                             ctypes.c_int, _vp, ctypes.c_size_t, _vp]
    lib.osdn_fwd.restype = ctypes.c_int
    lib.osdn_step.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _f32, _f32, _vp, _vp, _vp, _vp,
                              _vp, _i32, _i32, _i32, _i32, ctypes.c_int, _vp]
    lib.osdn_step.restype = ctypes.c_int
    lib.osdn_bwd_workspace_bytes.argtypes = [_i32, _i32, _i32, _i32, _i32, _i32, ctypes.c_int]
    lib.osdn_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.osdn_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _f32, _vp, _vp, _f32, _vp, _vp, _vp, _vp,
                             _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32,
                             _i32, ctypes.c_int, _vp, ctypes.c_size_t, _vp]
    lib.osdn_bwd.restype = ctypes.c_int
    lib.osdn_rho_geomean.argtypes = [_vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp]
    lib.osdn_rho_geomean.restype = ctypes.c_int
    lib.osdn_get_device_status.argtypes = [_vp]
    lib.osdn_get_device_status.restype = ctypes.c_int
    lib.osdn_debug_watchdog_selftest.argtypes = [ctypes.c_int64, _vp]
    lib.osdn_debug_watchdog_selftest.restype = ctypes.c_int
    return lib


LIB = _load()


def header_symbols() -> list:
    """Names of the functions include/osdn.h declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^OSDN_API\s+[\w\s\*]*?(osdn_\w+)\s*\(", text, re.M)))


def status_string(status: int) -> str:
    return LIB.osdn_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != OSDN_OK:
        raise OsdnError(status, where)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _io(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return OSDN_BF16
    if t.dtype == torch.float32:
        return OSDN_F32
    raise TypeError(f"io tensors must be bfloat16 or float32, got {t.dtype}")


def _req(t, name, dtype=None, shape=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _seqs(cu_seqlens, B):
    if cu_seqlens is None:
        return 0, B
    _req(cu_seqlens, "cu_seqlens", torch.int32)
    n = cu_seqlens.numel() - 1
    return n, n


def osdn_precond_scan(k, beta, r=None, eta: float = 0.0, d0=None, cu_seqlens=None,
                      k_tilde=None, dT=None, return_dT: bool = True, rho=None, stream=None):
    """Phase 1: returns ``(k_tilde, dT)`` (``dT`` is None when ``return_dT`` is False).  Given a
    float32 tensor ``rho`` of shape [B, T, H], also writes the per-token residual-contraction
    ratio (1 - beta_t <d_t, k_t^2>)^2 there."""
    B, T, H, Dk = k.shape
    io = _io(k)
    num_seqs, N = _seqs(cu_seqlens, B)
    _req(k, "k")
    _req(beta, "beta", torch.float32, (B, T, H))
    _req(r, "r", torch.float32, (B, T, H))
    _req(d0, "d0", torch.float32, (N, H, Dk))
    if k_tilde is None:
        k_tilde = torch.empty_like(k)
    _req(k_tilde, "k_tilde", k.dtype, k.shape)
    if dT is None and return_dT:
        dT = torch.empty((N, H, Dk), dtype=torch.float32, device=k.device)
    _req(dT, "dT", torch.float32, (N, H, Dk))
    _req(rho, "rho", torch.float32, (B, T, H))
    _check(LIB.osdn_precond_scan(_p(k), _p(beta), _p(r), float(eta), _p(d0), _p(k_tilde), _p(dT),
                                 _p(rho), _p(cu_seqlens), num_seqs, B, T, H, Dk, io,
                                 _stream(stream)),
           "osdn_precond_scan")
    return k_tilde, dT


def _alpha(alpha, B, T, H, Dk):
    """(pointer, per_channel flag) of a gated backbone's decay: [B, T, H] or [B, T, H, Dk]."""
    if alpha is None:
        return None, 0
    per_channel = alpha.dim() == 4
    _req(alpha, "alpha", torch.float32, (B, T, H, Dk) if per_channel else (B, T, H))
    return _p(alpha), int(per_channel)


def osdn_chunk_fwd(q, k, k_tilde, v, beta, scale: float = 1.0, S0=None, chunk: int = 64,
                   cu_seqlens=None, o=None, ST=None, return_ST: bool = True, stream=None,
                   alpha=None):
    """Phase 2: returns ``(o, ST)`` (``ST`` is None when ``return_ST`` is False).  ``alpha``: the
    decay of a gated backbone, [B, T, H] (Gated DeltaNet) or [B, T, H, Dk] (Kimi Delta Attention)
    float32, or None."""
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    io = _io(q)
    num_seqs, N = _seqs(cu_seqlens, B)
    for name, t in (("q", q), ("k", k), ("k_tilde", k_tilde)):
        _req(t, name, q.dtype, (B, T, H, Dk))
    _req(v, "v", q.dtype, (B, T, H, Dv))
    _req(beta, "beta", torch.float32, (B, T, H))
    _req(S0, "S0", torch.float32, (N, H, Dv, Dk))
    if o is None:
        o = torch.empty_like(v)
    _req(o, "o", q.dtype, (B, T, H, Dv))
    if ST is None and return_ST:
        ST = torch.empty((N, H, Dv, Dk), dtype=torch.float32, device=q.device)
    _req(ST, "ST", torch.float32, (N, H, Dv, Dk))
    a_ptr, apc = _alpha(alpha, B, T, H, Dk)
    _check(LIB.osdn_chunk_fwd(_p(q), _p(k), _p(k_tilde), _p(v), _p(beta), a_ptr, apc,
                              float(scale), _p(S0),
                              _p(o), _p(ST), _p(cu_seqlens), num_seqs, B, T, H, Dk, Dv,
                              int(chunk), io, _stream(stream)),
           "osdn_chunk_fwd")
    return o, ST


def osdn_fwd_workspace_bytes(B: int, T: int, H: int, Dk: int, dtype=torch.bfloat16) -> int:
    io = OSDN_BF16 if dtype == torch.bfloat16 else OSDN_F32
    return int(LIB.osdn_fwd_workspace_bytes(B, T, H, Dk, io))


def osdn_fwd(q, k, v, beta, r=None, eta: float = 0.0, d0=None, S0=None, scale: float = 1.0,
             chunk: int = 64, cu_seqlens=None, o=None, ST=None, dT=None, k_tilde=None,
             workspace=None, return_states: bool = True, rho=None, stream=None, alpha=None):
    """Both phases: returns ``(o, ST, dT)`` (states None when ``return_states`` is False).
    ``alpha``: the decay of a gated backbone, as for :func:`osdn_chunk_fwd`.

    The call needs a device workspace of ``osdn_fwd_workspace_bytes`` bytes (for bf16 it holds
    the residual of k~'s rounding, and k~ itself when ``k_tilde`` is not given); when
    ``workspace`` is None it is allocated with torch (device memory plumbing).
    """
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    io = _io(q)
    num_seqs, N = _seqs(cu_seqlens, B)
    for name, t in (("q", q), ("k", k)):
        _req(t, name, q.dtype, (B, T, H, Dk))
    _req(v, "v", q.dtype, (B, T, H, Dv))
    _req(beta, "beta", torch.float32, (B, T, H))
    _req(r, "r", torch.float32, (B, T, H))
    _req(d0, "d0", torch.float32, (N, H, Dk))
    _req(S0, "S0", torch.float32, (N, H, Dv, Dk))
    _req(k_tilde, "k_tilde", q.dtype, (B, T, H, Dk))
    if o is None:
        o = torch.empty_like(v)
    _req(o, "o", q.dtype, (B, T, H, Dv))
    if return_states:
        if ST is None:
            ST = torch.empty((N, H, Dv, Dk), dtype=torch.float32, device=q.device)
        if dT is None:
            dT = torch.empty((N, H, Dk), dtype=torch.float32, device=q.device)
    _req(ST, "ST", torch.float32, (N, H, Dv, Dk))
    _req(dT, "dT", torch.float32, (N, H, Dk))
    _req(rho, "rho", torch.float32, (B, T, H))
    ws_bytes = 0
    need = int(LIB.osdn_fwd_workspace_bytes(B, T, H, Dk, io))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if workspace is not None:
        _req(workspace, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    a_ptr, apc = _alpha(alpha, B, T, H, Dk)
    _check(LIB.osdn_fwd(_p(q), _p(k), _p(v), _p(beta), _p(r), a_ptr, apc, float(eta), _p(d0),
                        _p(S0),
                        float(scale), _p(o), _p(ST), _p(dT), _p(rho), _p(k_tilde), _p(cu_seqlens),
                        num_seqs, B, T, H, Dk, Dv, int(chunk), io, _p(workspace), ws_bytes,
                        _stream(stream)),
           "osdn_fwd")
    return o, ST, dT


def osdn_step(q, k, v, beta, S, d, r=None, eta: float = 0.0, scale: float = 1.0, o=None,
              k_tilde=None, rho=None, stream=None, alpha=None):
    """One recurrent step per (sequence, head) (the decode path).  q, k: [N, H, Dk]; v: [N, H, Dv];
    beta, r: [N, H] float32; S: [N, H, Dv, Dk] and d: [N, H, Dk] float32, updated in place;
    alpha: the decay of a gated backbone, [N, H] (Gated DeltaNet) or [N, H, Dk] (Kimi Delta
    Attention) float32, or None.  Returns o [N, H, Dv] (and writes k_tilde [N, H, Dk] when given)."""
    N, H, Dk = q.shape
    Dv = v.shape[-1]
    io = _io(q)
    _req(q, "q")
    _req(k, "k", q.dtype, (N, H, Dk))
    _req(v, "v", q.dtype, (N, H, Dv))
    _req(beta, "beta", torch.float32, (N, H))
    _req(r, "r", torch.float32, (N, H))
    _req(S, "S", torch.float32, (N, H, Dv, Dk))
    _req(d, "d", torch.float32, (N, H, Dk))
    if o is None:
        o = torch.empty_like(v)
    _req(o, "o", q.dtype, (N, H, Dv))
    _req(k_tilde, "k_tilde", q.dtype, (N, H, Dk))
    _req(rho, "rho", torch.float32, (N, H))
    per_channel = alpha is not None and alpha.dim() == 3
    _req(alpha, "alpha", torch.float32, (N, H, Dk) if per_channel else (N, H))
    _check(LIB.osdn_step(_p(q), _p(k), _p(v), _p(beta), _p(r), _p(alpha), int(per_channel),
                         float(eta), float(scale), _p(S), _p(d), _p(o), _p(k_tilde), _p(rho), N, H,
                         Dk, Dv, io, _stream(stream)),
           "osdn_step")
    return o


def osdn_bwd(q, k, v, beta, dO, r=None, eta: float = 0.0, d0=None, S0=None, scale: float = 1.0,
             dST=None, ddT=None, cu_seqlens=None, workspace=None, stream=None):
    """Gradients of L (given dL/do = dO, and optionally dL/dS_T, dL/dd_T) with respect to every
    input of :func:`osdn_fwd`.  Returns a dict of float32 tensors dq, dk, dv, dbeta, dr (None
    without r), deta (one element), dS0, dd0.  A workspace of ``osdn_bwd_workspace_bytes``
    bytes is allocated with torch when none is given (device memory plumbing)."""
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    io = _io(q)
    num_seqs, N = _seqs(cu_seqlens, B)
    for name, t in (("q", q), ("k", k)):
        _req(t, name, q.dtype, (B, T, H, Dk))
    _req(v, "v", q.dtype, (B, T, H, Dv))
    _req(dO, "dO", q.dtype, (B, T, H, Dv))
    _req(beta, "beta", torch.float32, (B, T, H))
    _req(r, "r", torch.float32, (B, T, H))
    _req(d0, "d0", torch.float32, (N, H, Dk))
    _req(S0, "S0", torch.float32, (N, H, Dv, Dk))
    _req(dST, "dST", torch.float32, (N, H, Dv, Dk))
    _req(ddT, "ddT", torch.float32, (N, H, Dk))
    f32 = dict(dtype=torch.float32, device=q.device)
    g = {"dq": torch.empty((B, T, H, Dk), **f32), "dk": torch.empty((B, T, H, Dk), **f32),
         "dv": torch.empty((B, T, H, Dv), **f32), "dbeta": torch.empty((B, T, H), **f32),
         "dr": None if r is None else torch.empty((B, T, H), **f32),
         "deta": torch.empty((1,), **f32), "dS0": torch.empty((N, H, Dv, Dk), **f32),
         "dd0": torch.empty((N, H, Dk), **f32)}
    need = int(LIB.osdn_bwd_workspace_bytes(num_seqs, B, T, H, Dk, Dv, io))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _req(workspace, "workspace")
    _check(LIB.osdn_bwd(_p(q), _p(k), _p(v), _p(beta), _p(r), float(eta), _p(d0), _p(S0),
                        float(scale), _p(dO), _p(dST), _p(ddT), _p(g["dq"]), _p(g["dk"]),
                        _p(g["dv"]), _p(g["dbeta"]), _p(g["dr"]), _p(g["deta"]), _p(g["dS0"]),
                        _p(g["dd0"]), _p(cu_seqlens), num_seqs, B, T, H, Dk, Dv, io,
                        _p(workspace), workspace.numel(), _stream(stream)),
           "osdn_bwd")
    return g


def osdn_rho_geomean(rho, cu_seqlens=None, q_geo=None, stream=None):
    """q_geo [N, H] float32: exp(mean_t log rho_t) per (sequence, head), from a residual-ratio
    tensor rho [B, T, H] (the ``rho`` output of the scan or the forward pass)."""
    B, T, H = rho.shape
    _req(rho, "rho", torch.float32)
    num_seqs, N = _seqs(cu_seqlens, B)
    if q_geo is None:
        q_geo = torch.empty((N, H), dtype=torch.float32, device=rho.device)
    _req(q_geo, "q_geo", torch.float32, (N, H))
    _check(LIB.osdn_rho_geomean(_p(rho), _p(cu_seqlens), num_seqs, B, T, H, _p(q_geo),
                                _stream(stream)), "osdn_rho_geomean")
    return q_geo


def osdn_get_device_status(stream=None) -> int:
    """Synchronize the stream and return (and clear) the device status word."""
    return int(LIB.osdn_get_device_status(_stream(stream)))


def osdn_debug_watchdog_selftest(spin_limit: int, stream=None):
    _check(LIB.osdn_debug_watchdog_selftest(int(spin_limit), _stream(stream)),
           "osdn_debug_watchdog_selftest")
