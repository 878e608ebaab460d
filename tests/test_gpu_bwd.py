"""The backward pass on the GPU (osdn_bwd) against the oracle's gradient (oracle bwd: reverse-mode
differentiation of the fp64 token loop, pinned by finite differences in test_oracle_bwd.py), every
gradient element by element: max|gpu - oracle| / rms(oracle) <= 1e-2 (bf16 I/O) or 1e-4 (fp32
I/O); deta (a scalar) by its relative error.  Gradients are stored in fp32, so nothing is taken
off for output rounding.  Sizes span several 32-token chunks and end ragged; both io dtypes; every
(Dk, Dv) pair; packed sequences with empty and one-token members; a zero key; the 1.3B-layer shape
and the packed varlen workload (sampled sequences).
"""
import numpy as np
import pytest
import torch

from delta_rule_recurrent_osdn_b200 import inputs as W
from tests.gpu_util import TOL, host, rel_err, round_io

pytestmark = pytest.mark.gpu

NAMES = ("dq", "dk", "dv", "dbeta", "dr", "dS0", "dd0")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(0)


def cotangents(inp, seed, states=True):
    """dL/do in the io dtype's values, dL/dS_T and dL/dd_T in fp32 (or None)."""
    rng = np.random.default_rng(seed)
    dO = round_io(rng.standard_normal(inp.v.shape).astype(np.float32), inp.io)
    dST = ddT = None
    if states:
        dST = (0.3 * rng.standard_normal((inp.N, inp.H, inp.Dv, inp.Dk))).astype(np.float32)
        ddT = rng.standard_normal((inp.N, inp.H, inp.Dk)).astype(np.float32)
    return dO, dST, ddT


def gpu_bwd(inp, dO, dST, ddT):
    from delta_rule_recurrent_osdn_b200 import osdn
    d = W.to_torch(inp)
    dt = torch.bfloat16 if inp.io == "bf16" else torch.float32
    f = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()
    g = osdn.osdn_bwd(d["q"], d["k"], d["v"], d["beta"], torch.from_numpy(
        dO.astype(np.float32)).to("cuda", dt), d["r"], d["eta"], d["d0"], d["S0"], d["scale"],
        f(dST), f(ddT), d["cu_seqlens"])
    torch.cuda.synchronize()
    assert osdn.osdn_get_device_status() == osdn.OSDN_OK
    return {k_: host(v_) for k_, v_ in g.items()}


def oracle_bwd(ref, inp, dO, dST, ddT):
    return ref.bwd(inp.q, inp.k, inp.v, inp.beta, dO, inp.r, inp.eta, inp.d0, inp.S0, inp.scale,
                   dST, ddT, inp.cu_seqlens)


def check(got, want, io, report=None):
    errs = {}
    for n in NAMES:
        if want.get(n) is None:
            assert got.get(n) is None
            continue
        errs[n] = rel_err(got[n], want[n])
    errs["deta"] = abs(float(got["deta"][0]) - want["deta"]) / max(abs(want["deta"]), 1e-30)
    if report:
        print("BWD", report, {k_: f"{v_:.2e}" for k_, v_ in errs.items()})
    bad = {n: e for n, e in errs.items() if not e <= TOL[io]}
    assert not bad, f"gradient parity failed ({io}, tol {TOL[io]}): {errs}"
    return errs


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("T", [1, 31, 33, 100])
def test_bwd_ragged_lengths(ref, io, T):
    inp = W.make_inputs(dict(B=2, T=T, H=2, Dk=128, Dv=128, io=io, apf=True, eta=0.1, chunk=64,
                             seed=80 + T, init_state=True))
    dO, dST, ddT = cotangents(inp, 81 + T)
    check(gpu_bwd(inp, dO, dST, ddT), oracle_bwd(ref, inp, dO, dST, ddT), io)


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("Dk,Dv", [(64, 64), (64, 128), (128, 64), (128, 128)])
def test_bwd_head_dims(ref, io, Dk, Dv):
    inp = W.make_inputs(dict(B=1, T=90, H=3, Dk=Dk, Dv=Dv, io=io, apf=True, eta=0.1, chunk=64,
                             seed=82, init_state=True))
    dO, dST, ddT = cotangents(inp, 83)
    check(gpu_bwd(inp, dO, dST, ddT), oracle_bwd(ref, inp, dO, dST, ddT), io)


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_bwd_no_apf_no_state_cotangents_and_a_zero_key(ref, io):
    inp = W.make_inputs(dict(B=2, T=70, H=2, Dk=128, Dv=128, io=io, apf=False, eta=0.05,
                             chunk=64, seed=84))
    inp.k[:, [3, 40]] = 0.0
    dO, _, _ = cotangents(inp, 85, states=False)
    got = gpu_bwd(inp, dO, None, None)
    assert got["dr"] is None
    check(got, oracle_bwd(ref, inp, dO, None, None), io)


def test_bwd_packed_with_empty_and_tiny_sequences(ref):
    inp = W.make_inputs(dict(lengths=[1, 33, 0, 64, 100, 7], H=2, Dk=128, Dv=128, io="bf16",
                             apf=True, eta=0.1, chunk=64, seed=86, init_state=True))
    dO, dST, ddT = cotangents(inp, 87)
    got = gpu_bwd(inp, dO, dST, ddT)
    check(got, oracle_bwd(ref, inp, dO, dST, ddT), "bf16")
    # an empty sequence passes its cotangents through to its initial state
    np.testing.assert_array_equal(got["dS0"][2], dST[2])
    np.testing.assert_array_equal(got["dd0"][2], ddT[2])


def test_bwd_1p3b_shape(ref):
    """The 1.3B-layer workload (B=4, T=4096, H=16, d=128, bf16, APF): every gradient of every
    (sequence, head) against the oracle."""
    inp = W.make_inputs("1p3b_apf")
    dO, dST, ddT = cotangents(inp, 88)
    check(gpu_bwd(inp, dO, dST, ddT), oracle_bwd(ref, inp, dO, dST, ddT), "bf16",
          report="1p3b_apf")


def test_bwd_varlen_sampled_sequences(ref):
    """The packed varlen workload (32 sequences, U[128, 8192] tokens): the full GPU run, checked
    on the shortest, the longest and two other sequences, every head."""
    inp = W.make_inputs("varlen")
    dO, dST, ddT = cotangents(inp, 89)
    got = gpu_bwd(inp, dO, dST, ddT)
    lens = np.diff(inp.cu_seqlens)
    seqs = sorted({int(np.argmin(lens)), int(np.argmax(lens)), 3, 17})
    sub = W.select(inp, seqs=seqs)
    cu = inp.cu_seqlens
    rows = np.concatenate([np.arange(cu[n], cu[n + 1]) for n in seqs])
    want = oracle_bwd(ref, sub, dO[:, rows], dST[seqs], ddT[seqs])
    sel = {n: (got[n][:, rows] if n in ("dq", "dk", "dv", "dbeta", "dr") else got[n][seqs])
           for n in NAMES}
    errs = {n: rel_err(sel[n], want[n]) for n in NAMES}
    print("BWD varlen", {k_: f"{v_:.2e}" for k_, v_ in errs.items()})
    assert all(e <= TOL["bf16"] for e in errs.values()), errs


def test_bwd_is_deterministic():
    inp = W.make_inputs(dict(B=2, T=200, H=2, Dk=128, Dv=128, io="bf16", apf=True, eta=0.05,
                             chunk=64, seed=90, init_state=True))
    dO, dST, ddT = cotangents(inp, 91)
    a = gpu_bwd(inp, dO, dST, ddT)
    b = gpu_bwd(inp, dO, dST, ddT)
    for n in NAMES + ("deta",):
        np.testing.assert_array_equal(a[n], b[n])
