"""GPU parity: the CUDA path against the fp64 oracle on the same seeded inputs.

Tolerance (written here, not derived from the GPU): max|gpu - oracle| / rms(oracle) <= 1e-2
for bf16 I/O and <= 1e-4 for fp32 I/O, for o, k~ (phase 1 output), S_T and d_T, where each
element's error first loses half an ulp of the exact value in the dtype the output is stored
in (bf16 for o and k~ in bf16 mode): rounding the exact fp64 o of the 340M and 1.3B workloads
to bf16 already gives 1.2% and 1.6% of rms(o).

osdn_fwd, the one-call forward pass, is compared with the plain fp64 oracle: nothing is rounded
between its phases (phase 1 hands k~ to phase 2 as two bf16 terms).  The two-call path
(osdn_precond_scan, then osdn_chunk_fwd) hands k~ over as one io-dtype tensor; it is compared
with the oracle's phase 2 fed that rounded k~.  Each test prints a "PARITY" line with the error
of every output against both references.
"""
import json

import numpy as np
import pytest
import torch

from delta_rule_recurrent_osdn_b200 import inputs as W
from tests.gpu_util import (TOL, check_all, gpu_fwd, oracle_fwd, oracle_fwd_split, rel_err)

pytestmark = pytest.mark.gpu

NAMES = ("o", "k_tilde", "ST", "dT")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(0)


def _report(case, path, got, want, want_split, io):
    """Asserts parity against `want`; prints both references' errors on one line."""
    res = check_all(got, want, io)
    other = {n: rel_err(g, w, None) for n, g, w in zip(NAMES, got, want_split)}
    print("PARITY " + json.dumps({"case": case, "path": path, "io": io, "vs_oracle": res["err"],
                                  "vs_oracle_raw": res["raw"],
                                  "vs_oracle_kt_rounded_raw": other}))
    return res


@pytest.mark.parametrize("name", ["tiny_fp32", "340m", "1p3b_apf"])
def test_workload_full_parity(ref, name):
    """Every output of every (sequence, head) against the plain fp64 oracle."""
    inp = W.make_inputs(name)
    got = gpu_fwd(inp)
    _report(name, "osdn_fwd", got, oracle_fwd(ref, inp), oracle_fwd_split(ref, inp), inp.io)


def test_long_context_sampled_heads(ref):
    """T = 65536 with S_0, d_0 passed in: the full GPU run, checked on three whole heads."""
    inp = W.make_inputs("long_ctx")
    got = gpu_fwd(inp)
    heads = [0, 7, 15]
    sub = W.select(inp, heads=heads)
    sel = (got[0][:, :, heads], got[1][:, :, heads], got[2][:, heads], got[3][:, heads])
    _report("long_ctx[heads 0,7,15]", "osdn_fwd", sel, oracle_fwd(ref, sub),
            oracle_fwd_split(ref, sub), inp.io)


def test_varlen_sampled_sequences(ref):
    """32 packed sequences: the full GPU run, checked on the shortest, the longest and two
    others, for three heads."""
    inp = W.make_inputs("varlen")
    got = gpu_fwd(inp)
    lens = np.diff(inp.cu_seqlens)
    seqs = sorted({int(np.argmin(lens)), int(np.argmax(lens)), 3, 17})
    heads = [0, 5, 11]
    sub = W.select(inp, seqs=seqs, heads=heads)
    cu = inp.cu_seqlens
    rows = np.concatenate([np.arange(cu[n], cu[n + 1]) for n in seqs])
    sel = (got[0][:, rows][:, :, heads], got[1][:, rows][:, :, heads],
           got[2][seqs][:, heads], got[3][seqs][:, heads])
    _report(f"varlen[seqs {seqs}, heads {heads}]", "osdn_fwd", sel, oracle_fwd(ref, sub),
            oracle_fwd_split(ref, sub), inp.io)


@pytest.mark.parametrize("name", ["340m", "1p3b_apf"])
def test_two_call_path_parity(ref, name):
    """osdn_precond_scan then osdn_chunk_fwd: k~ crosses as a bf16 tensor, so phase 2's
    reference is the oracle's phase 2 on that rounded k~."""
    inp = W.make_inputs(name)
    got = gpu_fwd(inp, split=True)
    _report(name, "osdn_precond_scan+osdn_chunk_fwd", got, oracle_fwd_split(ref, inp),
            oracle_fwd(ref, inp), inp.io)


@pytest.mark.parametrize("name", ["tiny_fp32", "1p3b_apf"])
def test_phases_separately(ref, name):
    """osdn_precond_scan against the oracle's phase 1; osdn_chunk_fwd fed the ORACLE's k~
    (rounded to the io dtype) against the oracle's phase 2 on that same k~."""
    from delta_rule_recurrent_osdn_b200 import osdn
    from tests.gpu_util import host
    inp = W.make_inputs(name)
    d = W.to_torch(inp)
    kt, dT = osdn.osdn_precond_scan(d["k"], d["beta"], d["r"], d["eta"], d["d0"])
    kt_ref, dT_ref = ref.precond_scan(inp.k, inp.beta, inp.r, inp.eta, inp.d0)
    assert rel_err(host(kt), kt_ref, inp.io) <= TOL[inp.io]
    assert rel_err(host(dT), dT_ref, "f32") <= TOL[inp.io]
    kt_in = kt_ref.astype(np.float32)
    if inp.io == "bf16":
        kt_in = W.bf16_round(kt_in)
    dt = torch.bfloat16 if inp.io == "bf16" else torch.float32
    kt_dev = torch.from_numpy(kt_in).to("cuda", dt)
    o, ST = osdn.osdn_chunk_fwd(d["q"], d["k"], kt_dev, d["v"], d["beta"], inp.scale, d["S0"],
                                inp.chunk)
    o_ref, ST_ref = ref.delta_fwd(inp.q, inp.k, kt_in, inp.v, inp.beta, inp.scale, inp.S0)
    assert rel_err(host(o), o_ref, inp.io) <= TOL[inp.io]
    assert rel_err(host(ST), ST_ref, "f32") <= TOL[inp.io]
