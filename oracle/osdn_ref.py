"""fp64 CPU oracle for the OSDN forward pass and its gradient -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this module.  The product path (the CUDA library and its Python binding) never
imports, links or executes anything under ``oracle/``, and this module imports nothing
from the product package.

The arithmetic lives in ``osdn_ref.c`` (plain C, fp64, token by token, OpenMP over
(sequence, head)); this file only marshals numpy arrays into it.  The method follows the
technical summary pages of "OSDN: Improving Delta Rule with Provable Online
Preconditioning in Linear Attention": section 1 (loss and delta rule), section 2.1
(write-key scaling k~ = d (.) k), section 2.2 (closed-form surrogate and its gradient,
two-phase split) and section 2.3 (APF retention gate on d).  The readings taken where the
pages are silent are listed at the top of ``osdn_ref.c``.

Every function takes and returns float64 numpy arrays in the library's layouts:
``q, k, k_tilde: [B, T, H, Dk]``, ``v, o: [B, T, H, Dv]``, ``beta, r: [B, T, H]``,
``S: [N, H, Dv, Dk]``, ``d: [N, H, Dk]``; packed variable-length input uses ``B == 1`` and
a host ``cu_seqlens`` array of N+1 int32 offsets.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "osdn_ref.c")
_LIB_PATH = os.path.join(_HERE, "libosdn_ref.so")

_D = ctypes.POINTER(ctypes.c_double)
_I = ctypes.POINTER(ctypes.c_int32)
_i32 = ctypes.c_int32


def compile_source(src: str, out: str) -> str:
    """gcc -O2 -fopenmp, no fast-math and no FMA contraction."""
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(
        ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-fno-fast-math",
         "-ffp-contract=off", "-o", tmp, src, "-lm"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile ``osdn_ref.c`` into ``libosdn_ref.so`` when missing or stale."""
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(SOURCE):
        compile_source(SOURCE, _LIB_PATH)
    return _LIB_PATH


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_D)


def _cu(cu_seqlens):
    if cu_seqlens is None:
        return None, None
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    return cu, cu.ctypes.data_as(_I)


def _dims(k, cu):
    B, T, H, Dk = k.shape
    if cu is not None:
        assert B == 1, "packed input needs B == 1"
        assert cu[0] == 0 and cu[-1] == T and np.all(np.diff(cu) >= 0), "bad cu_seqlens"
        N = len(cu) - 1
    else:
        N = B
    return B, T, H, Dk, N


class Oracle:
    """The oracle's entry points bound to one compiled library."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        lib.osdn_ref_set_threads.argtypes = [ctypes.c_int]
        lib.osdn_ref_set_threads.restype = ctypes.c_int
        lib.osdn_ref_precond_scan.argtypes = [
            _D, _D, _D, ctypes.c_double, _D, _D, _D, _D, _I, _i32, _i32, _i32, _i32, _i32]
        lib.osdn_ref_precond_scan.restype = None
        lib.osdn_ref_delta_fwd.argtypes = [
            _D, _D, _D, _D, _D, ctypes.c_double, _D, _D, _D, _I, _i32, _i32, _i32, _i32, _i32,
            _i32]
        lib.osdn_ref_delta_fwd.restype = None
        lib.osdn_ref_fwd.argtypes = [
            _D, _D, _D, _D, _D, ctypes.c_double, _D, _D, ctypes.c_double, _D, _D, _D, _D, _I,
            _i32, _i32, _i32, _i32, _i32, _i32]
        lib.osdn_ref_fwd.restype = None
        lib.osdn_ref_fwd_gated.argtypes = [
            _D, _D, _D, _D, _D, ctypes.c_double, _D, _D, ctypes.c_double, _D, _i32, _D, _D, _D, _D,
            _I, _i32, _i32, _i32, _i32, _i32, _i32]
        lib.osdn_ref_fwd_gated.restype = None
        lib.osdn_ref_bwd.argtypes = [
            _D, _D, _D, _D, _D, ctypes.c_double, _D, _D, ctypes.c_double, _D, _D, _D, _D, _D, _D,
            _D, _D, _D, _D, _D, _I, _i32, _i32, _i32, _i32, _i32, _i32]
        lib.osdn_ref_bwd.restype = None
        lib.osdn_ref_bwd_gated.argtypes = [
            _D, _D, _D, _D, _D, ctypes.c_double, _D, _D, ctypes.c_double, _D, _i32, _D, _D, _D, _D,
            _D, _D, _D, _D, _D, _D, _D, _D, _I, _i32, _i32, _i32, _i32, _i32, _i32]
        lib.osdn_ref_bwd_gated.restype = None
        lib.osdn_ref_rho_geomean.argtypes = [_D, _D, _I, _i32, _i32, _i32, _i32]
        lib.osdn_ref_rho_geomean.restype = None
        self.lib = lib

    def set_threads(self, n: int = 0) -> int:
        """Set the OpenMP thread count (n <= 0 keeps it); returns the count in effect."""
        return int(self.lib.osdn_ref_set_threads(int(n)))

    def precond_scan(self, k, beta, r=None, eta=0.0, d0=None, cu_seqlens=None, with_rho=False):
        """Phase 1 (section 2.2, step 1 of the two-phase split): returns (k_tilde, dT), or
        (k_tilde, dT, rho) with the per-token residual-contraction ratio
        rho_t = (1 - beta_t <d_t, k_t^2>)^2 of section 3 when with_rho is set."""
        k, beta, r, d0 = _f64(k), _f64(beta), _f64(r), _f64(d0)
        cu, cup = _cu(cu_seqlens)
        B, T, H, Dk, N = _dims(k, cu)
        assert beta.shape == (B, T, H) and (r is None or r.shape == (B, T, H))
        assert d0 is None or d0.shape == (N, H, Dk)
        k_tilde = np.zeros_like(k)
        dT = np.zeros((N, H, Dk))
        rho = np.zeros((B, T, H)) if with_rho else None
        self.lib.osdn_ref_precond_scan(_ptr(k), _ptr(beta), _ptr(r), float(eta), _ptr(d0),
                                       _ptr(k_tilde), _ptr(dT), _ptr(rho), cup, N, B, T, H, Dk)
        return (k_tilde, dT, rho) if with_rho else (k_tilde, dT)

    def rho_geomean(self, rho, cu_seqlens=None, N=None):
        """q_geo [N, H]: the geometric mean over each sequence's tokens of the residual ratios
        rho [B, T, H] (section 3; the experiments' q_geo); 0 if a ratio is 0, 1 for a sequence
        without tokens."""
        rho = _f64(rho)
        cu, cup = _cu(cu_seqlens)
        B, T, H = rho.shape
        if cu is not None:
            assert B == 1 and cu[0] == 0 and cu[-1] == T and np.all(np.diff(cu) >= 0)
            N = len(cu) - 1
        else:
            N = B
        q_geo = np.zeros((N, H))
        self.lib.osdn_ref_rho_geomean(_ptr(rho), _ptr(q_geo), cup, N, B, T, H)
        return q_geo

    def delta_fwd(self, q, k, k_tilde, v, beta, scale=1.0, S0=None, cu_seqlens=None):
        """Phase 2 (section 2.1): delta rule with write key k_tilde. Returns (o, ST)."""
        q, k, k_tilde, v, beta, S0 = map(_f64, (q, k, k_tilde, v, beta, S0))
        cu, cup = _cu(cu_seqlens)
        B, T, H, Dk, N = _dims(k, cu)
        Dv = v.shape[-1]
        assert q.shape == k.shape == k_tilde.shape and v.shape == (B, T, H, Dv)
        assert S0 is None or S0.shape == (N, H, Dv, Dk)
        o = np.zeros((B, T, H, Dv))
        ST = np.zeros((N, H, Dv, Dk))
        self.lib.osdn_ref_delta_fwd(_ptr(q), _ptr(k), _ptr(k_tilde), _ptr(v), _ptr(beta),
                                    float(scale), _ptr(S0), _ptr(o), _ptr(ST), cup, N, B, T, H,
                                    Dk, Dv)
        return o, ST

    def fwd(self, q, k, v, beta, r=None, eta=0.0, d0=None, S0=None, scale=1.0, cu_seqlens=None):
        """Both phases in one token loop. Returns (o, k_tilde, ST, dT)."""
        q, k, v, beta, r, d0, S0 = map(_f64, (q, k, v, beta, r, d0, S0))
        cu, cup = _cu(cu_seqlens)
        B, T, H, Dk, N = _dims(k, cu)
        Dv = v.shape[-1]
        assert q.shape == k.shape and v.shape == (B, T, H, Dv) and beta.shape == (B, T, H)
        assert r is None or r.shape == (B, T, H)
        assert d0 is None or d0.shape == (N, H, Dk)
        assert S0 is None or S0.shape == (N, H, Dv, Dk)
        o = np.zeros((B, T, H, Dv))
        k_tilde = np.zeros_like(k)
        ST = np.zeros((N, H, Dv, Dk))
        dT = np.zeros((N, H, Dk))
        self.lib.osdn_ref_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(r), float(eta),
                              _ptr(d0), _ptr(S0), float(scale), _ptr(o), _ptr(k_tilde), _ptr(ST),
                              _ptr(dT), cup, N, B, T, H, Dk, Dv)
        return o, k_tilde, ST, dT


    def fwd_gated(self, q, k, v, beta, alpha, r=None, eta=0.0, d0=None, S0=None, scale=1.0,
                  cu_seqlens=None):
        """Both phases on a gated backbone: the state's key channels decay by alpha before each
        token's write (alpha [B,T,H]: Gated DeltaNet; [B,T,H,Dk]: Kimi Delta Attention).
        Returns (o, k_tilde, ST, dT) like ``fwd``."""
        q, k, v, beta, alpha, r, d0, S0 = map(_f64, (q, k, v, beta, alpha, r, d0, S0))
        cu, cup = _cu(cu_seqlens)
        B, T, H, Dk, N = _dims(k, cu)
        Dv = v.shape[-1]
        assert alpha.shape in ((B, T, H), (B, T, H, Dk))
        per_channel = 1 if alpha.shape == (B, T, H, Dk) else 0
        o = np.zeros((B, T, H, Dv))
        k_tilde = np.zeros_like(k)
        ST = np.zeros((N, H, Dv, Dk))
        dT = np.zeros((N, H, Dk))
        self.lib.osdn_ref_fwd_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(r), float(eta),
                                    _ptr(d0), _ptr(S0), float(scale), _ptr(alpha), per_channel,
                                    _ptr(o), _ptr(k_tilde), _ptr(ST), _ptr(dT), cup, N, B, T, H, Dk,
                                    Dv)
        return o, k_tilde, ST, dT

    def bwd(self, q, k, v, beta, dO, r=None, eta=0.0, d0=None, S0=None, scale=1.0, dST=None,
            ddT=None, cu_seqlens=None, alpha=None):
        """Gradient of L = <dO, o> + <dST, S_T> + <ddT, d_T> for the forward pass ``fwd`` (or
        ``fwd_gated`` when alpha is given) with the same arguments, by reverse-mode
        differentiation of its token loop.  Returns a dict with dq, dk, dv, dbeta, dr (None
        without r), deta (float), dS0, dd0, and dalpha (alpha's shape) when alpha is given."""
        q, k, v, beta, r, d0, S0, dO, dST, ddT, alpha = map(
            _f64, (q, k, v, beta, r, d0, S0, dO, dST, ddT, alpha))
        cu, cup = _cu(cu_seqlens)
        B, T, H, Dk, N = _dims(k, cu)
        Dv = v.shape[-1]
        assert q.shape == k.shape and v.shape == (B, T, H, Dv) and beta.shape == (B, T, H)
        assert dO.shape == v.shape and (r is None or r.shape == (B, T, H))
        assert d0 is None or d0.shape == (N, H, Dk)
        assert S0 is None or S0.shape == (N, H, Dv, Dk)
        assert dST is None or dST.shape == (N, H, Dv, Dk)
        assert ddT is None or ddT.shape == (N, H, Dk)
        g = {"dq": np.zeros_like(q), "dk": np.zeros_like(k), "dv": np.zeros_like(v),
             "dbeta": np.zeros_like(beta), "dr": None if r is None else np.zeros_like(r),
             "dS0": np.zeros((N, H, Dv, Dk)), "dd0": np.zeros((N, H, Dk))}
        deta = np.zeros(1)
        if alpha is None:
            self.lib.osdn_ref_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(r), float(eta),
                                  _ptr(d0), _ptr(S0), float(scale), _ptr(dO), _ptr(dST), _ptr(ddT),
                                  _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["dbeta"]),
                                  _ptr(g["dr"]), _ptr(deta), _ptr(g["dS0"]), _ptr(g["dd0"]), cup, N,
                                  B, T, H, Dk, Dv)
        else:
            assert alpha.shape in ((B, T, H), (B, T, H, Dk))
            g["dalpha"] = np.zeros_like(alpha)
            self.lib.osdn_ref_bwd_gated(
                _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(r), float(eta), _ptr(d0), _ptr(S0),
                float(scale), _ptr(alpha), 1 if alpha.ndim == 4 else 0, _ptr(dO), _ptr(dST),
                _ptr(ddT), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["dbeta"]),
                _ptr(g["dr"]), _ptr(deta), _ptr(g["dalpha"]), _ptr(g["dS0"]), _ptr(g["dd0"]), cup,
                N, B, T, H, Dk, Dv)
        g["deta"] = float(deta[0])
        return g


_default = None


def _oracle() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def set_threads(n: int = 0) -> int:
    return _oracle().set_threads(n)


def precond_scan(*args, **kwargs):
    return _oracle().precond_scan(*args, **kwargs)


def delta_fwd(*args, **kwargs):
    return _oracle().delta_fwd(*args, **kwargs)


def fwd(*args, **kwargs):
    return _oracle().fwd(*args, **kwargs)


def bwd(*args, **kwargs):
    return _oracle().bwd(*args, **kwargs)


def fwd_gated(*args, **kwargs):
    return _oracle().fwd_gated(*args, **kwargs)


def rho_geomean(*args, **kwargs):
    return _oracle().rho_geomean(*args, **kwargs)
