"""The residual-contraction ratio rho_t = (1 - beta_t <d_t, k_t^2>)^2 (technical summary,
section 3) emitted by phase 1 and by the decode step, against the oracle's."""
import numpy as np
import pytest
import torch

from delta_rule_recurrent_osdn_b200 import inputs as W
from tests.gpu_util import TOL, host, rel_err

pytestmark = pytest.mark.gpu


def _scan_rho(inp):
    from delta_rule_recurrent_osdn_b200 import osdn
    d = W.to_torch(inp)
    rho = torch.empty(d["beta"].shape, dtype=torch.float32, device="cuda")
    osdn.osdn_precond_scan(d["k"], d["beta"], d["r"], d["eta"], d["d0"], d["cu_seqlens"], rho=rho)
    torch.cuda.synchronize()
    assert osdn.osdn_get_device_status() == osdn.OSDN_OK
    return host(rho)


@pytest.mark.parametrize("case", [
    dict(B=2, T=300, H=4, Dk=128, Dv=128, io="bf16", apf=True, eta=0.05, seed=31),   # chunk path
    dict(B=2, T=300, H=4, Dk=128, Dv=128, io="bf16", apf=False, eta=0.05, seed=32),
    dict(B=1, T=200, H=3, Dk=128, Dv=128, io="bf16", apf=True, eta=0.0, seed=33),    # eta = 0
    dict(B=2, T=150, H=2, Dk=64, Dv=64, io="f32", apf=True, eta=0.1, seed=34),       # warp scan
    dict(lengths=[70, 1, 0, 200], H=2, Dk=128, Dv=128, io="bf16", apf=True, eta=0.05, seed=35,
         init_state=True),
])
def test_scan_rho_matches_oracle(ref, case):
    inp = W.make_inputs(dict(chunk=64, **case))
    got = _scan_rho(inp)
    _, _, want = ref.precond_scan(inp.k, inp.beta, inp.r, inp.eta, inp.d0, inp.cu_seqlens,
                                  with_rho=True)
    assert rel_err(got, want) <= TOL["f32"]
    assert np.all(got >= 0.0)


def test_fwd_rho_equals_scan_rho():
    from delta_rule_recurrent_osdn_b200 import osdn
    inp = W.make_inputs(dict(B=1, T=130, H=2, Dk=128, Dv=128, io="bf16", apf=True, eta=0.05,
                             chunk=64, seed=36))
    d = W.to_torch(inp)
    rho = torch.empty(d["beta"].shape, dtype=torch.float32, device="cuda")
    osdn.osdn_fwd(d["q"], d["k"], d["v"], d["beta"], d["r"], d["eta"], d["d0"], d["S0"],
                  d["scale"], 64, None, rho=rho)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host(rho), _scan_rho(inp))


def test_step_rho_matches_oracle(ref):
    from delta_rule_recurrent_osdn_b200 import osdn
    inp = W.make_inputs(dict(B=8, T=1, H=4, Dk=128, Dv=128, io="bf16", apf=True, eta=0.1,
                             chunk=64, seed=37, init_state=True))
    t = W.to_torch(inp)
    S, dd = t["S0"].clone(), t["d0"].clone()
    rho = torch.empty((8, 4), dtype=torch.float32, device="cuda")
    osdn.osdn_step(t["q"][:, 0].contiguous(), t["k"][:, 0].contiguous(), t["v"][:, 0].contiguous(),
                   t["beta"][:, 0].contiguous(), S, dd, t["r"][:, 0].contiguous(), t["eta"],
                   t["scale"], rho=rho)
    torch.cuda.synchronize()
    _, _, want = ref.precond_scan(inp.k, inp.beta, inp.r, inp.eta, inp.d0, with_rho=True)
    assert rel_err(host(rho), want[:, 0]) <= 1e-5


@pytest.mark.parametrize("case", [
    dict(lengths=[300, 0, 1, 700, 64], H=3, Dk=128, Dv=128, io="bf16", apf=True, eta=0.05,
         seed=38, init_state=True),
    dict(B=2, T=500, H=2, Dk=128, Dv=128, io="bf16", apf=False, eta=0.05, seed=39),
    dict(B=2, T=150, H=2, Dk=64, Dv=64, io="f32", apf=True, eta=0.1, seed=40),
])
def test_q_geo_of_the_forward_pass(ref, case):
    """q_geo = exp(mean_t log rho_t) per (sequence, head) from the forward pass's rho output,
    against the oracle's q_geo of the oracle's rho; and against the fp64 host reduction of the
    GPU's own rho (which isolates the reduction kernel)."""
    from delta_rule_recurrent_osdn_b200 import osdn
    inp = W.make_inputs(dict(chunk=64, **case))
    d = W.to_torch(inp)
    rho = torch.empty(d["beta"].shape, dtype=torch.float32, device="cuda")
    osdn.osdn_fwd(d["q"], d["k"], d["v"], d["beta"], d["r"], d["eta"], d["d0"], d["S0"],
                  d["scale"], 64, d["cu_seqlens"], rho=rho)
    q_geo = osdn.osdn_rho_geomean(rho, d["cu_seqlens"])
    torch.cuda.synchronize()
    assert osdn.osdn_get_device_status() == osdn.OSDN_OK
    got = host(q_geo)
    own = ref.rho_geomean(host(rho), inp.cu_seqlens)
    np.testing.assert_allclose(got, own, rtol=1e-5, atol=0)
    _, _, rho_ref = ref.precond_scan(inp.k, inp.beta, inp.r, inp.eta, inp.d0, inp.cu_seqlens,
                                     with_rho=True)
    want = ref.rho_geomean(rho_ref, inp.cu_seqlens)
    np.testing.assert_allclose(got, want, rtol=1e-3, atol=0)
    print("q_geo", got.ravel()[:8], "oracle", want.ravel()[:8])


def test_q_geo_zero_ratio_and_empty_sequence(ref):
    """A sequence holding a ratio of exactly 0 has q_geo 0; a sequence without tokens has 1."""
    from delta_rule_recurrent_osdn_b200 import osdn
    rng = np.random.default_rng(41)
    lengths = [5, 0, 1000, 1, 33]
    T = sum(lengths)
    rho = rng.uniform(0.05, 1.0, (1, T, 4)).astype(np.float32)
    rho[0, 7, 2] = 0.0       # sequence 2 (rows 5..1004), head 2
    rho[0, 1005, 0] = 0.0    # sequence 3 (its only row), head 0
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    out = host(osdn.osdn_rho_geomean(torch.from_numpy(rho).cuda(),
                                     torch.from_numpy(cu).cuda()))
    want = ref.rho_geomean(rho.astype(np.float64), cu)
    assert out[2, 2] == 0.0 and out[3, 0] == 0.0
    assert np.all(out[1] == 1.0)
    np.testing.assert_allclose(out, want, rtol=1e-5, atol=0)
