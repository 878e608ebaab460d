"""The decode step (osdn_step) against the oracle's token loop, and against the chunked forward
pass of the library itself."""
import numpy as np
import pytest
import torch

from delta_rule_recurrent_osdn_b200 import inputs as W
from tests.gpu_util import TOL, host, rel_err

pytestmark = pytest.mark.gpu


def _batch(io, N, T, H, Dk, Dv, seed, apf=True):
    return W.make_inputs(dict(B=N, T=T, H=H, Dk=Dk, Dv=Dv, io=io, apf=apf, eta=0.1, chunk=64,
                              seed=seed, init_state=True))


def _steps(inp, ts, alpha=None):
    """Run osdn_step over tokens ts of every sequence (alpha: optional decay, numpy [N, T, H] or
    [N, T, H, Dk]); returns numpy (o[N, len(ts), H, Dv], k_tilde[N, len(ts), H, Dk], S, d)."""
    from delta_rule_recurrent_osdn_b200 import osdn
    t = W.to_torch(inp)
    S = t["S0"].clone()
    d = t["d0"].clone()
    a = None if alpha is None else torch.from_numpy(alpha.astype(np.float32)).cuda()
    os_, kts = [], []
    for i in ts:
        kt = torch.empty_like(t["k"][:, i])
        o = osdn.osdn_step(t["q"][:, i].contiguous(), t["k"][:, i].contiguous(),
                           t["v"][:, i].contiguous(), t["beta"][:, i].contiguous(), S, d,
                           None if t["r"] is None else t["r"][:, i].contiguous(), t["eta"],
                           t["scale"], k_tilde=kt,
                           alpha=None if a is None else a[:, i].contiguous())
        os_.append(o)
        kts.append(kt)
    torch.cuda.synchronize()
    assert osdn.osdn_get_device_status() == osdn.OSDN_OK
    return (host(torch.stack(os_, 1)), host(torch.stack(kts, 1)), host(S), host(d))


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("Dk,Dv", [(128, 128), (64, 64), (128, 64), (64, 128)])
def test_single_step_matches_oracle(ref, io, Dk, Dv):
    inp = _batch(io, N=6, T=1, H=3, Dk=Dk, Dv=Dv, seed=21)
    o, kt, S, d = _steps(inp, [0])
    wo, wkt, wS, wd = ref.fwd(inp.q, inp.k, inp.v, inp.beta, inp.r, inp.eta, inp.d0, inp.S0,
                              inp.scale)
    assert rel_err(o, wo, io) <= TOL[io]
    assert rel_err(kt, wkt, io) <= TOL[io]
    assert rel_err(S, wS) <= 1e-5
    assert rel_err(d, wd) <= 1e-5


@pytest.mark.parametrize("apf", [True, False])
def test_step_sequence_matches_oracle(ref, apf):
    """24 consecutive steps equal the oracle's loop over the same 24 tokens."""
    inp = _batch("bf16", N=4, T=24, H=4, Dk=128, Dv=128, seed=22, apf=apf)
    o, kt, S, d = _steps(inp, range(24))
    wo, wkt, wS, wd = ref.fwd(inp.q, inp.k, inp.v, inp.beta, inp.r, inp.eta, inp.d0, inp.S0,
                              inp.scale)
    assert rel_err(o, wo, "bf16") <= TOL["bf16"]
    assert rel_err(kt, wkt, "bf16") <= TOL["bf16"]
    assert rel_err(S, wS) <= 1e-4
    assert rel_err(d, wd) <= 1e-4


def test_steps_equal_chunked_forward():
    """Decoding token by token gives the chunked forward pass's final states and outputs."""
    from delta_rule_recurrent_osdn_b200 import osdn
    inp = _batch("f32", N=2, T=200, H=2, Dk=128, Dv=128, seed=23)
    o, kt, S, d = _steps(inp, range(200))
    t = W.to_torch(inp)
    fo, fST, fdT = osdn.osdn_fwd(t["q"], t["k"], t["v"], t["beta"], t["r"], t["eta"], t["d0"],
                                 t["S0"], t["scale"], 64, None)
    torch.cuda.synchronize()
    assert rel_err(o, host(fo)) <= TOL["f32"]
    assert rel_err(S, host(fST)) <= TOL["f32"]
    assert rel_err(d, host(fdT)) <= TOL["f32"]


def test_zero_key_only_decays_d(ref):
    inp = _batch("f32", N=2, T=1, H=2, Dk=128, Dv=128, seed=24)
    inp.k[:] = 0.0
    o, kt, S, d = _steps(inp, [0])
    np.testing.assert_array_equal(S, inp.S0)  # u k~^T with k~ = 0
    np.testing.assert_allclose(d, inp.r[:, 0, :, None] * inp.d0, rtol=1e-6)


def test_many_heads():
    """A decode batch of 256 sequences x 16 heads (4096 CTAs) against the oracle on a sample."""
    from oracle import osdn_ref as R
    inp = _batch("bf16", N=256, T=1, H=16, Dk=128, Dv=128, seed=25)
    o, kt, S, d = _steps(inp, [0])
    pick = [0, 17, 255]
    sub = W.select(inp, pick, list(range(16)))
    wo, wkt, wS, wd = R.fwd(sub.q, sub.k, sub.v, sub.beta, sub.r, sub.eta, sub.d0, sub.S0,
                            sub.scale)
    assert rel_err(o[pick], wo, "bf16") <= TOL["bf16"]
    assert rel_err(S[pick], wS) <= 1e-5
    assert rel_err(d[pick], wd) <= 1e-5


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("per_channel", [False, True])
def test_gated_steps_match_oracle(ref, io, per_channel):
    """Decay of a gated backbone (Gated DeltaNet: per token and head; Kimi Delta Attention: per
    key channel) before each write: 24 steps equal the oracle's gated token loop."""
    inp = _batch(io, N=3, T=24, H=2, Dk=128, Dv=128, seed=26)
    rng = np.random.default_rng(27)
    shape = (3, 24, 2, 128) if per_channel else (3, 24, 2)
    alpha = (1 / (1 + np.exp(-(2 + rng.standard_normal(shape))))).astype(np.float32)
    o, kt, S, d = _steps(inp, range(24), alpha)
    wo, wkt, wS, wd = ref.fwd_gated(inp.q, inp.k, inp.v, inp.beta, alpha.astype(np.float64),
                                    r=inp.r, eta=inp.eta, d0=inp.d0, S0=inp.S0, scale=inp.scale)
    assert rel_err(o, wo, io) <= TOL[io]
    assert rel_err(kt, wkt, io) <= TOL[io]
    assert rel_err(S, wS) <= 1e-4
    assert rel_err(d, wd) <= 1e-4


def test_unit_decay_equals_ungated_step():
    """alpha == 1 gives the ungated step bit for bit."""
    inp = _batch("f32", N=2, T=6, H=2, Dk=128, Dv=128, seed=28)
    plain = _steps(inp, range(6))
    ones = _steps(inp, range(6), np.ones((2, 6, 2), dtype=np.float32))
    for a, b in zip(plain, ones):
        np.testing.assert_array_equal(a, b)
