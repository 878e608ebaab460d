"""GPU edge cases and structural invariants, each checked against the oracle or exactly.

Sizes span several chunks and ragged tails; both io dtypes; every (Dk, Dv) pair; packed
sequences with empty and one-token members; zero-size calls; chunk-size invariance in fp32;
state chaining; device-side checks of cu_seqlens; the bounded-wait watchdog.
"""
import numpy as np
import pytest
import torch

from delta_rule_recurrent_osdn_b200 import inputs as W
from tests.gpu_util import TOL, check_all, gpu_fwd, host, oracle_fwd, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(0)


def small(io, T, H=2, Dk=128, Dv=128, B=2, apf=True, init=True, seed=5, **kw):
    cfg = dict(B=B, T=T, H=H, Dk=Dk, Dv=Dv, io=io, apf=apf, eta=0.1, chunk=64, seed=seed,
               init_state=init)
    cfg.update(kw)
    return W.make_inputs(cfg)


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200, 513])
def test_ragged_lengths(ref, io, T):
    inp = small(io, T)
    check_all(gpu_fwd(inp), oracle_fwd(ref, inp), io)


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("Dk,Dv", [(64, 64), (64, 128), (128, 64), (128, 128)])
def test_head_dims(ref, io, Dk, Dv):
    inp = small(io, 150, H=3, Dk=Dk, Dv=Dv, B=1)
    check_all(gpu_fwd(inp), oracle_fwd(ref, inp), io)


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_packed_with_empty_and_tiny_sequences(ref, io):
    inp = W.make_inputs(dict(lengths=[1, 64, 0, 65, 130, 7, 0, 200], H=2, Dk=128, Dv=128, io=io,
                             apf=True, eta=0.1, seed=6, init_state=True))
    got = gpu_fwd(inp)
    want = oracle_fwd(ref, inp)
    check_all(got, want, io)
    # empty sequences return their initial state unchanged
    for n in (2, 6):
        np.testing.assert_array_equal(got[2][n], inp.S0[n])
        np.testing.assert_array_equal(got[3][n], inp.d0[n])


def test_packed_many_short_sequences(ref):
    """Dozens of sequences shorter than a chunk: one 64-row window of the packed batch holds the
    starts of many chunks, which the persistent per-chunk kernels must all visit."""
    rng = np.random.default_rng(11)
    lengths = [int(x) for x in rng.integers(0, 9, size=40)] + [3, 70, 1]
    inp = W.make_inputs(dict(lengths=lengths, H=3, Dk=128, Dv=128, io="bf16", apf=True, eta=0.1,
                             seed=12, init_state=True))
    check_all(gpu_fwd(inp), oracle_fwd(ref, inp), "bf16")


def test_packed_equals_separate_calls(ref):
    """Packing is bookkeeping only: bit-identical to one call per sequence."""
    lengths = [70, 1, 129, 64]
    inp = W.make_inputs(dict(lengths=lengths, H=2, Dk=128, Dv=128, io="bf16", apf=True, eta=0.1,
                             seed=7, init_state=True))
    got = gpu_fwd(inp)
    cu = inp.cu_seqlens
    for n in range(len(lengths)):
        one = W.select(inp, seqs=[n])
        one.cu_seqlens = None  # the same sequence as a fixed-length batch of one
        g1 = gpu_fwd(one)
        np.testing.assert_array_equal(g1[0][0], got[0][0, cu[n]:cu[n + 1]])
        np.testing.assert_array_equal(g1[2][0], got[2][n])
        np.testing.assert_array_equal(g1[3][0], got[3][n])


def test_zero_sizes():
    from delta_rule_recurrent_osdn_b200 import osdn
    for B, T in [(0, 64), (2, 0)]:
        inp = small("bf16", max(T, 1), B=max(B, 1))
        d = W.to_torch(inp)
        q = d["q"][:B, :T].contiguous()
        k = d["k"][:B, :T].contiguous()
        v = d["v"][:B, :T].contiguous()
        beta = d["beta"][:B, :T].contiguous()
        r = d["r"][:B, :T].contiguous()
        S0 = d["S0"][:B].contiguous()
        d0 = d["d0"][:B].contiguous()
        o, ST, dT = osdn.osdn_fwd(q, k, v, beta, r, 0.1, d0, S0)
        torch.cuda.synchronize()
        assert o.numel() == 0
        if B > 0:  # no tokens: states pass through
            assert torch.equal(ST, S0) and torch.equal(dT, d0)


def test_chunk_size_invariance_fp32(ref):
    inp = small("f32", 300, H=2)
    outs = [gpu_fwd(inp, chunk=c) for c in (16, 32, 64)]
    want = oracle_fwd(ref, inp)
    for got in outs:
        check_all(got, want, "f32")
    for a, b in zip(outs[0], outs[2]):
        assert rel_err(a, b) <= 1e-5


def _bf16_step(x):
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    ax = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_state_chaining(io):
    """Two calls over the halves, the second starting from the first's S_T and d_T, equal one
    call over the whole sequence.

    The fp32 path restarts bit-for-bit up to summation order.  The tensor-core path forms a
    chunk's K S^T from the previous chunk's state and W when it continues a sequence, and
    directly from S_0 when it starts one: the two agree to the split operands' precision (about
    2^-16 of the state, bound 1e-4 of rms here), and each bf16 output may then round one step
    apart."""
    inp = small(io, 256, B=1)
    full = gpu_fwd(inp)
    first = W.select(inp)
    first.q, first.k, first.v = inp.q[:, :128], inp.k[:, :128], inp.v[:, :128]
    first.beta, first.r = inp.beta[:, :128], inp.r[:, :128]
    a = gpu_fwd(first)
    second = W.select(inp)
    second.q, second.k, second.v = inp.q[:, 128:], inp.k[:, 128:], inp.v[:, 128:]
    second.beta, second.r = inp.beta[:, 128:], inp.r[:, 128:]
    second.S0, second.d0 = a[2].astype(np.float32), a[3].astype(np.float32)
    b = gpu_fwd(second)
    o2 = np.concatenate([a[0], b[0]], axis=1).astype(np.float64)
    o1 = np.asarray(full[0], dtype=np.float64)
    if io == "f32":
        assert rel_err(o2, o1) <= 2e-6
        assert rel_err(b[2], full[2]) <= 2e-6
    else:
        rms = np.sqrt(np.mean(o1 ** 2))
        excess = np.abs(o2 - o1) - _bf16_step(np.maximum(np.abs(o1), np.abs(o2)))
        assert excess.max() / rms <= 1e-4
        assert rel_err(b[2], full[2]) <= 1e-4
    assert rel_err(b[3], full[3]) <= 2e-6  # phase 1 restarts exactly up to summation order


def test_no_apf_equals_unit_retention():
    inp = small("bf16", 200, apf=True)
    ones = W.select(inp)
    ones.r = np.ones_like(inp.r)
    none = W.select(inp)
    none.r = None
    for x, y in zip(gpu_fwd(ones), gpu_fwd(none)):
        np.testing.assert_array_equal(x, y)


def test_split_phases_equal_fused_entry(ref):
    inp = W.make_inputs("tiny_fp32")
    a = gpu_fwd(inp, split=True)
    b = gpu_fwd(inp, split=False)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_bad_cu_seqlens_reported_on_device():
    """Out-of-order offsets: the kernels skip the sequence and record OSDN_ERR_DEVICE_BOUNDS;
    the context stays usable."""
    from delta_rule_recurrent_osdn_b200 import osdn
    inp = W.make_inputs(dict(lengths=[64, 64, 64], H=2, Dk=128, Dv=128, io="bf16", apf=True,
                             eta=0.1, seed=8))
    d = W.to_torch(inp)
    bad = torch.tensor([0, 100, 50, 192], dtype=torch.int32, device="cuda")
    assert osdn.osdn_get_device_status() == osdn.OSDN_OK
    osdn.osdn_fwd(d["q"], d["k"], d["v"], d["beta"], d["r"], d["eta"], cu_seqlens=bad)
    assert osdn.osdn_get_device_status() == osdn.OSDN_ERR_DEVICE_BOUNDS
    assert osdn.osdn_get_device_status() == osdn.OSDN_OK  # read clears it
    gpu_fwd(inp)  # still works


def test_watchdog_times_out_cleanly():
    from delta_rule_recurrent_osdn_b200 import osdn
    assert osdn.osdn_get_device_status() == osdn.OSDN_OK
    osdn.osdn_debug_watchdog_selftest(1000)
    assert osdn.osdn_get_device_status() == osdn.OSDN_ERR_DEVICE_TIMEOUT
    x = torch.ones(4, device="cuda") * 2
    assert float(x.sum()) == 8.0


def test_misaligned_tensor_rejected():
    from delta_rule_recurrent_osdn_b200 import osdn
    inp = small("bf16", 64)
    d = W.to_torch(inp)
    flat = torch.empty(d["q"].numel() + 8, dtype=torch.bfloat16, device="cuda")
    q_mis = flat[1:1 + d["q"].numel()].view(d["q"].shape)
    with pytest.raises(osdn.OsdnError) as e:
        osdn.osdn_fwd(q_mis, d["k"], d["v"], d["beta"], d["r"], d["eta"])
    assert e.value.status == osdn.OSDN_ERR_ALIGNMENT
