"""The C ABI without a GPU: the library loads, exports every symbol include/osdn.h declares,
and rejects bad arguments before anything reaches CUDA (no compute call is made here)."""
import ctypes

import pytest

osdn = pytest.importorskip("delta_rule_recurrent_osdn_b200.osdn")
L = osdn.LIB
A = 0x10000000  # a 16-byte aligned fake address; validation failures never dereference it


def fake(i):
    return ctypes.c_void_p(A + i * 0x1000000)


def chunk_call(**kw):
    args = dict(q=fake(1), k=fake(2), kt=fake(3), v=fake(4), beta=fake(5), alpha=None, apc=0,
                scale=1.0, S0=None, o=fake(6), ST=None, cu=None, num_seqs=0, B=1, T=8, H=1, Dk=128,
                Dv=128, chunk=64, io=osdn.OSDN_BF16)
    args.update(kw)
    return L.osdn_chunk_fwd(args["q"], args["k"], args["kt"], args["v"], args["beta"],
                            args["alpha"], args["apc"],
                            args["scale"], args["S0"], args["o"], args["ST"], args["cu"],
                            args["num_seqs"], args["B"], args["T"], args["H"], args["Dk"],
                            args["Dv"], args["chunk"], args["io"], None)


def scan_call(**kw):
    args = dict(k=fake(1), beta=fake(2), r=None, eta=0.1, d0=None, kt=fake(3), dT=None, rho=None,
                cu=None,
                num_seqs=0, B=1, T=8, H=1, Dk=128, io=osdn.OSDN_BF16)
    args.update(kw)
    return L.osdn_precond_scan(args["k"], args["beta"], args["r"], args["eta"], args["d0"],
                               args["kt"], args["dT"], args["rho"], args["cu"], args["num_seqs"],
                               args["B"],
                               args["T"], args["H"], args["Dk"], args["io"], None)


def test_exports_every_declared_symbol():
    names = osdn.header_symbols()
    assert {"osdn_precond_scan", "osdn_chunk_fwd", "osdn_fwd", "osdn_fwd_workspace_bytes",
            "osdn_status_string", "osdn_get_device_status"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_version_and_status_strings():
    assert L.osdn_abi_version() == 6
    for s in range(7):
        assert osdn.status_string(s)
    assert osdn.status_string(99) == "unknown status"


def test_workspace_size():
    # bf16: k~ and the residual of its rounding, each part rounded up to 256 bytes
    assert L.osdn_fwd_workspace_bytes(4, 4096, 16, 128, osdn.OSDN_BF16) == 2 * 4 * 4096 * 16 * 128 * 2
    assert L.osdn_fwd_workspace_bytes(1, 3, 1, 64, osdn.OSDN_BF16) == 2 * 512
    assert L.osdn_fwd_workspace_bytes(1, 3, 1, 64, osdn.OSDN_F32) == 768
    assert L.osdn_fwd_workspace_bytes(1, 1, 1, 96, osdn.OSDN_BF16) == 0


@pytest.mark.parametrize("kw,status", [
    (dict(Dk=96), osdn.OSDN_ERR_UNSUPPORTED),
    (dict(Dv=32), osdn.OSDN_ERR_UNSUPPORTED),
    (dict(chunk=32), osdn.OSDN_ERR_UNSUPPORTED),          # bf16 path runs 64-token chunks
    (dict(chunk=48, io=osdn.OSDN_F32), osdn.OSDN_ERR_UNSUPPORTED),
    (dict(q=None), osdn.OSDN_ERR_INVALID_ARG),
    (dict(o=None), osdn.OSDN_ERR_INVALID_ARG),
    (dict(B=-1), osdn.OSDN_ERR_INVALID_ARG),
    (dict(H=0), osdn.OSDN_ERR_INVALID_ARG),
    (dict(T=-5), osdn.OSDN_ERR_INVALID_ARG),
    (dict(io=7), osdn.OSDN_ERR_INVALID_ARG),
    (dict(cu=fake(9), num_seqs=2, B=2), osdn.OSDN_ERR_INVALID_ARG),  # packed needs B == 1
    (dict(v=ctypes.c_void_p(A + 8)), osdn.OSDN_ERR_ALIGNMENT),
    (dict(S0=ctypes.c_void_p(A + 4)), osdn.OSDN_ERR_ALIGNMENT),
    (dict(o=fake(1)), osdn.OSDN_ERR_INVALID_ARG),          # output aliases q
    (dict(beta=ctypes.c_void_p(A + 6 * 0x1000000 + 256)), osdn.OSDN_ERR_INVALID_ARG),  # in o
    (dict(S0=ctypes.c_void_p(A + 6 * 0x1000000)), osdn.OSDN_ERR_INVALID_ARG),
    (dict(ST=ctypes.c_void_p(A + 6 * 0x1000000 + 1024)), osdn.OSDN_ERR_INVALID_ARG),
    (dict(alpha=fake(8), apc=2), osdn.OSDN_ERR_INVALID_ARG),                    # flag not 0 / 1
    (dict(alpha=ctypes.c_void_p(A + 8 * 0x1000000 + 4)), osdn.OSDN_ERR_ALIGNMENT),
    (dict(alpha=ctypes.c_void_p(A + 6 * 0x1000000 + 32)), osdn.OSDN_ERR_INVALID_ARG),  # in o
])
def test_chunk_fwd_rejects(kw, status):
    assert chunk_call(**kw) == status


@pytest.mark.parametrize("kw,status", [
    (dict(Dk=32), osdn.OSDN_ERR_UNSUPPORTED),
    (dict(k=None), osdn.OSDN_ERR_INVALID_ARG),
    (dict(kt=None), osdn.OSDN_ERR_INVALID_ARG),
    (dict(kt=fake(1)), osdn.OSDN_ERR_INVALID_ARG),          # in place k~ == k
    (dict(kt=ctypes.c_void_p(A + 0x1000000 + 256)), osdn.OSDN_ERR_INVALID_ARG),  # overlap
    (dict(beta=ctypes.c_void_p(A + 3 * 0x1000000 + 64)), osdn.OSDN_ERR_INVALID_ARG),  # in k~
    (dict(r=ctypes.c_void_p(A + 3 * 0x1000000 + 512)), osdn.OSDN_ERR_INVALID_ARG),
    (dict(d0=ctypes.c_void_p(A + 3 * 0x1000000)), osdn.OSDN_ERR_INVALID_ARG),
    (dict(dT=ctypes.c_void_p(A + 3 * 0x1000000 + 1024)), osdn.OSDN_ERR_INVALID_ARG),
    (dict(rho=ctypes.c_void_p(A + 3 * 0x1000000 + 1536)), osdn.OSDN_ERR_INVALID_ARG),  # rho in k~
    (dict(rho=ctypes.c_void_p(A + 2 * 0x1000000)), osdn.OSDN_ERR_INVALID_ARG),        # rho = beta
    (dict(rho=ctypes.c_void_p(A + 9 * 0x1000000 + 4)), osdn.OSDN_ERR_ALIGNMENT),
    (dict(r=ctypes.c_void_p(A + 2)), osdn.OSDN_ERR_ALIGNMENT),
    (dict(cu=ctypes.c_void_p(A + 4), num_seqs=1), osdn.OSDN_ERR_ALIGNMENT),
    (dict(num_seqs=-1), osdn.OSDN_ERR_INVALID_ARG),
])
def test_precond_scan_rejects(kw, status):
    assert scan_call(**kw) == status


def test_fwd_needs_workspace_even_with_k_tilde_out():
    """In bf16 mode the workspace holds the lo term of k~ even when k~ goes to k_tilde_out."""
    st = L.osdn_fwd(fake(1), fake(2), fake(4), fake(5), None, None, 0, 0.1, None, None, 1.0,
                    fake(6), None, None, None, fake(8), None, 0, 1, 64, 1, 128, 128, 64,
                    osdn.OSDN_BF16, None, 0, None)
    assert st == osdn.OSDN_ERR_INVALID_ARG


@pytest.mark.parametrize("kw,status", [
    (dict(B=-1), osdn.OSDN_ERR_INVALID_ARG),
    (dict(H=0), osdn.OSDN_ERR_INVALID_ARG),
    (dict(cu=fake(9), num_seqs=2, B=2), osdn.OSDN_ERR_INVALID_ARG),
    (dict(rho=None), osdn.OSDN_ERR_INVALID_ARG),
    (dict(out=None), osdn.OSDN_ERR_INVALID_ARG),
    (dict(out=ctypes.c_void_p(A + 2 * 0x1000000 + 4)), osdn.OSDN_ERR_ALIGNMENT),
    (dict(out=ctypes.c_void_p(A + 1 * 0x1000000 + 16)), osdn.OSDN_ERR_INVALID_ARG),  # in rho
    (dict(B=0), osdn.OSDN_OK),  # no sequences: nothing to do
])
def test_rho_geomean_rejects(kw, status):
    args = dict(rho=fake(1), cu=None, num_seqs=0, B=2, T=64, H=4, out=fake(2))
    args.update(kw)
    assert L.osdn_rho_geomean(args["rho"], args["cu"], args["num_seqs"], args["B"], args["T"],
                              args["H"], args["out"], None) == status


def test_fwd_rejects_small_workspace():
    st = L.osdn_fwd(fake(1), fake(2), fake(4), fake(5), None, None, 0, 0.1, None, None, 1.0,
                    fake(6), None, None, None, None, None, 0, 1, 64, 1, 128, 128, 64,
                    osdn.OSDN_BF16, fake(7), 100, None)
    assert st == osdn.OSDN_ERR_INVALID_ARG
    st = L.osdn_fwd(fake(1), fake(2), fake(4), fake(5), None, None, 0, 0.1, None, None, 1.0,
                    fake(6), None, None, None, None, None, 0, 1, 64, 1, 128, 128, 64,
                    osdn.OSDN_BF16, ctypes.c_void_p(A + 0x7000010), 1 << 20, None)
    assert st == osdn.OSDN_ERR_ALIGNMENT  # workspace must be 256-byte aligned


def test_parity_metric_allows_exactly_the_output_rounding():
    """The GPU tests' metric: storing the exact value in bf16 costs nothing; anything beyond
    half an ulp counts."""
    import numpy as np
    from delta_rule_recurrent_osdn_b200.inputs import bf16_round
    from tests.gpu_util import rel_err
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(100000) * 3).astype(np.float32).astype(np.float64)
    xb = bf16_round(x.astype(np.float32)).astype(np.float64)
    assert rel_err(xb, x) > 1e-3           # raw rounding error is visible
    assert rel_err(xb, x, "bf16") == 0.0   # and is exactly what the allowance removes
    y = xb.copy()
    y[7] += 0.05
    assert 0.04 / 3 < rel_err(y, x, "bf16") < 0.06 / 2.9


def step_call(**kw):
    args = dict(q=fake(1), k=fake(2), v=fake(3), beta=fake(4), r=None, alpha=None, apc=0, eta=0.1,
                scale=1.0, S=fake(5), d=fake(6), o=fake(7), kt=None, rho=None, N=4, H=2, Dk=128,
                Dv=128, io=osdn.OSDN_BF16)
    args.update(kw)
    return L.osdn_step(args["q"], args["k"], args["v"], args["beta"], args["r"], args["alpha"],
                       args["apc"], args["eta"], args["scale"], args["S"], args["d"], args["o"],
                       args["kt"], args["rho"], args["N"], args["H"], args["Dk"], args["Dv"],
                       args["io"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(Dk=96), osdn.OSDN_ERR_UNSUPPORTED),
    (dict(Dv=32), osdn.OSDN_ERR_UNSUPPORTED),
    (dict(io=5), osdn.OSDN_ERR_INVALID_ARG),
    (dict(H=0), osdn.OSDN_ERR_INVALID_ARG),
    (dict(N=-1), osdn.OSDN_ERR_INVALID_ARG),
    (dict(S=None), osdn.OSDN_ERR_INVALID_ARG),
    (dict(o=None), osdn.OSDN_ERR_INVALID_ARG),
    (dict(S=ctypes.c_void_p(A + 5 * 0x1000000 + 8)), osdn.OSDN_ERR_ALIGNMENT),
    (dict(o=fake(1)), osdn.OSDN_ERR_INVALID_ARG),                                 # o aliases q
    (dict(d=ctypes.c_void_p(A + 5 * 0x1000000 + 4096)), osdn.OSDN_ERR_INVALID_ARG),  # d in S
    (dict(kt=fake(2)), osdn.OSDN_ERR_INVALID_ARG),                                # k~ aliases k
    (dict(rho=fake(4)), osdn.OSDN_ERR_INVALID_ARG),                               # rho = beta
    (dict(alpha=fake(8), apc=2), osdn.OSDN_ERR_INVALID_ARG),                     # flag not 0 / 1
    (dict(alpha=ctypes.c_void_p(A + 8 * 0x1000000 + 4)), osdn.OSDN_ERR_ALIGNMENT),
    (dict(alpha=ctypes.c_void_p(A + 5 * 0x1000000 + 64), apc=1), osdn.OSDN_ERR_INVALID_ARG),  # in S
    (dict(N=0), osdn.OSDN_OK),                                                    # nothing to do
])
def test_step_rejects(kw, status):
    assert step_call(**kw) == status


def bwd_call(**kw):
    args = dict(q=fake(1), k=fake(2), v=fake(3), beta=fake(4), r=None, eta=0.1, d0=None, S0=None,
                scale=1.0, dO=fake(5), dST=None, ddT=None, dq=fake(6), dk=fake(7), dv=fake(8),
                dbeta=fake(9), dr=None, deta=None, dS0=None, dd0=None, cu=None, num_seqs=0, B=1,
                T=64, H=2, Dk=128, Dv=128, io=osdn.OSDN_BF16, ws=fake(10), wsb=1 << 30)
    args.update(kw)
    a = args
    return L.osdn_bwd(a["q"], a["k"], a["v"], a["beta"], a["r"], a["eta"], a["d0"], a["S0"],
                      a["scale"], a["dO"], a["dST"], a["ddT"], a["dq"], a["dk"], a["dv"], a["dbeta"],
                      a["dr"], a["deta"], a["dS0"], a["dd0"], a["cu"], a["num_seqs"], a["B"], a["T"],
                      a["H"], a["Dk"], a["Dv"], a["io"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(Dk=96), osdn.OSDN_ERR_UNSUPPORTED),
    (dict(Dv=32), osdn.OSDN_ERR_UNSUPPORTED),
    (dict(dq=None), osdn.OSDN_ERR_INVALID_ARG),
    (dict(dO=None), osdn.OSDN_ERR_INVALID_ARG),
    (dict(wsb=1000), osdn.OSDN_ERR_INVALID_ARG),                     # workspace too small
    (dict(ws=ctypes.c_void_p(A + 10 * 0x1000000 + 16)), osdn.OSDN_ERR_ALIGNMENT),
    (dict(dk=fake(6)), osdn.OSDN_ERR_INVALID_ARG),                   # dk aliases dq
    (dict(dv=fake(3)), osdn.OSDN_ERR_INVALID_ARG),                   # dv aliases v
    (dict(dbeta=ctypes.c_void_p(A + 10 * 0x1000000 + 4096)), osdn.OSDN_ERR_INVALID_ARG),  # in ws
    (dict(deta=ctypes.c_void_p(A + 9 * 0x1000000 + 4)), osdn.OSDN_ERR_ALIGNMENT),
    (dict(B=-1), osdn.OSDN_ERR_INVALID_ARG),
])
def test_bwd_rejects(kw, status):
    assert bwd_call(**kw) == status


def test_bwd_workspace_size_grows_with_the_batch():
    small = L.osdn_bwd_workspace_bytes(0, 1, 64, 2, 128, 128, osdn.OSDN_BF16)
    big = L.osdn_bwd_workspace_bytes(0, 4, 4096, 16, 128, 128, osdn.OSDN_BF16)
    assert 0 < small < big
    assert big % 256 == 0
    assert L.osdn_bwd_workspace_bytes(0, 1, 64, 2, 96, 128, osdn.OSDN_BF16) == 0


def test_debug_bounds_build_exports_the_same_symbols_and_validates_alike():
    """libosdn_debug.so (-DOSDN_DEBUG_BOUNDS) is the same ABI: it loads, exports every declared
    symbol and rejects bad arguments on the host with the same status as the release build."""
    from delta_rule_recurrent_osdn_b200 import build as B
    lib = ctypes.CDLL(B.build(debug_bounds=True))
    for n in osdn.header_symbols():
        assert hasattr(lib, n), n
    lib.osdn_abi_version.restype = ctypes.c_int
    assert lib.osdn_abi_version() == L.osdn_abi_version()
    lib.osdn_fwd_workspace_bytes.restype = ctypes.c_int64
    lib.osdn_fwd_workspace_bytes.argtypes = L.osdn_fwd_workspace_bytes.argtypes
    assert lib.osdn_fwd_workspace_bytes(4, 4096, 16, 128, osdn.OSDN_BF16) == \
        L.osdn_fwd_workspace_bytes(4, 4096, 16, 128, osdn.OSDN_BF16)
    f = lib.osdn_chunk_fwd
    f.restype, f.argtypes = L.osdn_chunk_fwd.restype, L.osdn_chunk_fwd.argtypes
    bad = f(fake(1), fake(2), fake(3), fake(4), fake(5), None, 0, 1.0, None, fake(6), None, None,
            0, 1, 8, 1, 96, 128, 64, osdn.OSDN_BF16, None)
    assert bad == osdn.OSDN_ERR_UNSUPPORTED == chunk_call(Dk=96)
