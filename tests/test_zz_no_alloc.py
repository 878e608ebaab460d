"""osdn_fwd_noalloc: the forward pass for callers that cannot allocate device memory.

Some callers may not call cudaMalloc at all, for example a plugin inside a host framework that
owns every device allocation, or a latency-critical service that forbids allocation after
start-up.  For them the library keeps what phase 1 hands to phase 2 (the preconditioned keys,
as bf16 hi and lo terms in bf16 mode) in a fixed device array of its own (32 MiB), so the caller
passes only inputs and outputs.  These tests call that entry point through the C ABI, twice in a
row (the array keeps the previous call's contents), and require every output to be bit-identical
to the workspace-based osdn_fwd: both run the same kernels on the same inputs, so any difference
would be stale or misplaced scratch data.
"""
import ctypes

import numpy as np
import pytest
import torch

from delta_rule_recurrent_osdn_b200 import inputs as W
from tests.gpu_util import host

pytestmark = pytest.mark.gpu

_vp, _i32, _f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float


def _lib():
    from delta_rule_recurrent_osdn_b200 import osdn
    lib = osdn.LIB
    f = lib.osdn_fwd_noalloc
    f.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _f32, _vp, _vp, _f32, _vp, _vp, _vp, _vp, _vp,
                  _i32, _i32, _i32, _i32, _i32, _i32, _i32, ctypes.c_int, _vp]
    f.restype = ctypes.c_int
    return osdn, f


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(f, d, inp, o, ST, dT, io):
    B, T, H, Dk = d["q"].shape
    Dv = d["v"].shape[-1]
    cu = d["cu_seqlens"]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return f(_p(d["q"]), _p(d["k"]), _p(d["v"]), _p(d["beta"]), _p(d["r"]), None, 0, d["eta"],
             _p(d["d0"]),
             _p(d["S0"]), d["scale"], _p(o), _p(ST), _p(dT), None, _p(cu),
             0 if cu is None else cu.numel() - 1, B, T, H, Dk, Dv, d["chunk"], io, stream)


@pytest.mark.parametrize("cfg", [
    dict(B=2, T=2048, H=16, Dk=128, Dv=128, io="bf16", apf=True, eta=0.05, seed=21),
    dict(lengths=[300, 1, 0, 4100, 777], H=8, Dk=128, Dv=128, io="bf16", apf=True, eta=0.05,
         seed=22, init_state=True),
    dict(B=1, T=333, H=2, Dk=64, Dv=64, io="f32", apf=True, eta=0.1, seed=23),
])
def test_noalloc_matches_workspace_entry_point(cfg):
    torch.cuda.set_device(0)
    osdn, f = _lib()
    inp = W.make_inputs(cfg)
    d = W.to_torch(inp)
    io = osdn.OSDN_BF16 if inp.io == "bf16" else osdn.OSDN_F32
    want = osdn.osdn_fwd(d["q"], d["k"], d["v"], d["beta"], d["r"], d["eta"], d["d0"], d["S0"],
                         d["scale"], d["chunk"], d["cu_seqlens"])
    torch.cuda.synchronize()
    want = [host(t) for t in want]
    N, H, Dk, Dv = inp.N, inp.H, inp.Dk, inp.Dv
    for call in range(2):  # two calls in a row share (and reuse) the library's array
        o = torch.empty_like(d["v"])
        ST = torch.empty((N, H, Dv, Dk), dtype=torch.float32, device="cuda")
        dT = torch.empty((N, H, Dk), dtype=torch.float32, device="cuda")
        assert _noalloc(f, d, inp, o, ST, dT, io) == osdn.OSDN_OK
        torch.cuda.synchronize()
        assert osdn.osdn_get_device_status() == osdn.OSDN_OK
        got = [host(o), host(ST), host(dT)]
        for g, w in zip(got, want):
            np.testing.assert_array_equal(g, w, err_msg=f"call {call}")


def test_noalloc_rejects_keys_larger_than_its_array():
    """4 x 4096 tokens x 16 heads x 128 bf16 keys (64 MiB, twice that with the lo terms) exceed
    the 32 MiB array: the call is refused before anything is enqueued."""
    osdn, f = _lib()
    fake = ctypes.c_void_p(0x10000000)
    st = f(fake, fake, fake, fake, None, None, 0, 0.05, None, None, 1.0, fake, None, None, None,
           None, 0, 4, 4096, 16, 128, 128, 64, osdn.OSDN_BF16, None)
    assert st == osdn.OSDN_ERR_UNSUPPORTED
