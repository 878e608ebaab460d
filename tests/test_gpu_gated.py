"""OSDN on gated backbones through the chunked forward pass (osdn_fwd / osdn_chunk_fwd with
alpha), element by element against the oracle's gated form (oracle fwd_gated: the state's key
channels decay before each write, the gated delta rule of the Gated DeltaNet-2 page, section 1,
with OSDN's write key; phase 1 unchanged).  Gated DeltaNet decay (one factor per token and head)
and Kimi Delta Attention decay (one per key channel), bf16 and fp32 I/O, packed sequences, the
1.3B-layer shape, unit decay, and decay strong enough that the Gram ratios leave the fp32 range of
the reference-scaled factors.  Tolerances of tests/gpu_util.py.
"""
import numpy as np
import pytest
import torch

from delta_rule_recurrent_osdn_b200 import inputs as W
from tests.gpu_util import check_all, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(0)


def decay(inp, per_channel, seed, mean=2.0):
    """alpha = sigmoid(mean + N(0, 1)) per token and head (or per key channel)."""
    rng = np.random.default_rng(seed)
    shape = inp.beta.shape + ((inp.Dk,) if per_channel else ())
    return (1.0 / (1.0 + np.exp(-(mean + rng.standard_normal(shape))))).astype(np.float32)


def gated_gpu(inp, alpha, split=False):
    from delta_rule_recurrent_osdn_b200 import osdn
    d = W.to_torch(inp)
    a = torch.from_numpy(alpha).cuda()
    kt = torch.empty_like(d["k"])
    if split:
        kt, dT = osdn.osdn_precond_scan(d["k"], d["beta"], d["r"], d["eta"], d["d0"],
                                        d["cu_seqlens"], k_tilde=kt)
        o, ST = osdn.osdn_chunk_fwd(d["q"], d["k"], kt, d["v"], d["beta"], d["scale"], d["S0"],
                                    d["chunk"], d["cu_seqlens"], alpha=a)
    else:
        o, ST, dT = osdn.osdn_fwd(d["q"], d["k"], d["v"], d["beta"], d["r"], d["eta"], d["d0"],
                                  d["S0"], d["scale"], d["chunk"], d["cu_seqlens"], k_tilde=kt,
                                  alpha=a)
    torch.cuda.synchronize()
    assert osdn.osdn_get_device_status() == osdn.OSDN_OK
    return host(o), host(kt), host(ST), host(dT)


def gated_oracle(ref, inp, alpha):
    return ref.fwd_gated(inp.q, inp.k, inp.v, inp.beta, alpha.astype(np.float64), inp.r, inp.eta,
                         inp.d0, inp.S0, inp.scale, inp.cu_seqlens)


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("per_channel", [False, True])
@pytest.mark.parametrize("T", [63, 200])
def test_gated_small(ref, io, per_channel, T):
    inp = W.make_inputs(dict(B=2, T=T, H=2, Dk=128, Dv=128, io=io, apf=True, eta=0.05, chunk=64,
                             seed=61 + T, init_state=True))
    alpha = decay(inp, per_channel, 62 + T)
    check_all(gated_gpu(inp, alpha), gated_oracle(ref, inp, alpha), io)


@pytest.mark.parametrize("per_channel", [False, True])
def test_gated_packed_and_64_channel_heads(ref, per_channel):
    inp = W.make_inputs(dict(lengths=[70, 1, 0, 130, 64], H=3, Dk=64, Dv=64, io="f32", apf=True,
                             eta=0.1, chunk=32, seed=63, init_state=True))
    alpha = decay(inp, per_channel, 64)
    check_all(gated_gpu(inp, alpha), gated_oracle(ref, inp, alpha), "f32")


@pytest.mark.parametrize("per_channel", [False, True])
def test_gated_1p3b_shape(ref, per_channel):
    """The 1.3B-layer workload (B=4, T=4096, H=16, d=128, bf16, APF) on a gated backbone: every
    output of every (sequence, head) against the oracle."""
    inp = W.make_inputs("1p3b_apf")
    alpha = decay(inp, per_channel, 65)
    check_all(gated_gpu(inp, alpha), gated_oracle(ref, inp, alpha), "bf16")


def test_strong_decay_takes_the_per_term_path(ref):
    """alpha = 0.02 on a stretch of tokens: over half a chunk the log decay passes 80, so the
    Gram ratios are evaluated one exponential per term; still equal to the oracle."""
    inp = W.make_inputs(dict(B=1, T=192, H=2, Dk=128, Dv=128, io="f32", apf=False, eta=0.05,
                             chunk=64, seed=66, init_state=True))
    alpha = decay(inp, True, 67)
    alpha[:, 70:120] = 0.02
    check_all(gated_gpu(inp, alpha), gated_oracle(ref, inp, alpha), "f32")


@pytest.mark.parametrize("per_channel", [False, True])
def test_unit_decay_is_the_ungated_pass(per_channel):
    """alpha == 1 gives the ungated forward pass bit for bit (fp32 I/O: both run the same
    kernels); and the two-call path with alpha == 1 equals the one-call path's phase 2 input."""
    from tests.gpu_util import gpu_fwd
    inp = W.make_inputs(dict(B=2, T=150, H=2, Dk=128, Dv=128, io="f32", apf=True, eta=0.05,
                             chunk=64, seed=68, init_state=True))
    ones = np.ones(inp.beta.shape + ((inp.Dk,) if per_channel else ()), dtype=np.float32)
    for x, y in zip(gated_gpu(inp, ones), gpu_fwd(inp)):
        np.testing.assert_array_equal(x, y)


def test_gated_two_call_path_equals_one_call_in_fp32(ref):
    """osdn_precond_scan then osdn_chunk_fwd(alpha) equals osdn_fwd(alpha) bit for bit in fp32
    I/O (k~ crosses the calls unrounded there), and both equal the oracle."""
    inp = W.make_inputs(dict(B=2, T=200, H=2, Dk=128, Dv=128, io="f32", apf=True, eta=0.05,
                             chunk=64, seed=69, init_state=True))
    alpha = decay(inp, True, 70)
    got = gated_gpu(inp, alpha, split=True)
    one = gated_gpu(inp, alpha, split=False)
    for x, y in zip(got, one):
        np.testing.assert_array_equal(x, y)
    check_all(got, gated_oracle(ref, inp, alpha), "f32")
