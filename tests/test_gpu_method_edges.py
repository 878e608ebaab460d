"""The method's own special cases on the GPU forward pass (osdn_fwd), element by element against
the plain fp64 oracle, in bf16 and fp32 I/O (tolerances of tests/gpu_util.py).

  * a zero key (||k_t|| = 0) inside a chunk: the surrogate's gradient is taken as 0 there, so
    k~_t = 0, the state is not written and d only decays (technical summary, section 2.2: the
    closed form divides by ||k_t||^2);
  * an output scale != 1 (o_t = scale * S_t q_t);
  * eta = 0 with no APF gate: d stays 1, so k~ equals k bit for bit and the pass is the plain
    delta rule (section 1), which the oracle pins against an independent DeltaNet loop;
  * beta_t close to 1 (near-exact writes);
  * keys that are not unit-norm (norm 0.1, and norm 10 with beta scaled by 1/||k||^2 so that
    beta ||k||^2 stays in (0, 1): the plain delta rule diverges when beta ||k||^2 > 2), with and
    without APF.
Sizes span several chunks and end in a ragged one.
"""
import numpy as np
import pytest
import torch

from delta_rule_recurrent_osdn_b200 import inputs as W
from tests.gpu_util import check_all, gpu_fwd, oracle_fwd

pytestmark = pytest.mark.gpu

IOS = ["bf16", "f32"]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(0)


def base(io, apf=True, eta=0.05, seed=51, T=300, init=True):
    return W.make_inputs(dict(B=2, T=T, H=2, Dk=128, Dv=128, io=io, apf=apf, eta=eta, chunk=64,
                              seed=seed, init_state=init))


@pytest.mark.parametrize("io", IOS)
def test_zero_keys_inside_chunks(ref, io):
    inp = base(io, seed=52)
    zero = [0, 5, 63, 64, 100, 299]
    inp.k[:, zero] = 0.0
    got = gpu_fwd(inp)
    check_all(got, oracle_fwd(ref, inp), io)
    assert np.all(got[1][:, zero] == 0.0)  # k~ of a zero key is exactly zero


@pytest.mark.parametrize("io", IOS)
@pytest.mark.parametrize("scale", [0.37, 3.0])
def test_output_scale(ref, io, scale):
    inp = base(io, seed=53)
    check_all(gpu_fwd(inp, scale=scale), oracle_fwd(ref, inp, scale=scale), io)


@pytest.mark.parametrize("io", IOS)
def test_eta_zero_no_apf_is_the_delta_rule(ref, io):
    inp = base(io, apf=False, eta=0.0, seed=54, init=False)
    got = gpu_fwd(inp)
    np.testing.assert_array_equal(got[1], inp.k.astype(np.float64))  # k~ == k, bit for bit
    assert np.all(got[3] == 1.0)                                    # d stays 1
    check_all(got, oracle_fwd(ref, inp), io)


@pytest.mark.parametrize("io", IOS)
@pytest.mark.parametrize("apf", [True, False])
def test_beta_near_one(ref, io, apf):
    inp = base(io, apf=apf, seed=55)
    inp.beta = np.full_like(inp.beta, 0.999)
    check_all(gpu_fwd(inp), oracle_fwd(ref, inp), io)


@pytest.mark.parametrize("io", IOS)
@pytest.mark.parametrize("apf", [True, False])
@pytest.mark.parametrize("norm", [0.1, 10.0])
def test_keys_not_unit_norm(ref, io, apf, norm):
    inp = base(io, apf=apf, seed=56)
    k = inp.k.astype(np.float64) * norm
    inp.k = W.bf16_round(k.astype(np.float32)) if io == "bf16" else k.astype(np.float32)
    if norm > 1.0:
        inp.beta = (inp.beta / norm ** 2).astype(np.float32)
    check_all(gpu_fwd(inp), oracle_fwd(ref, inp), io)
