"""Runs every entry point of whichever library build OSDN_LIBRARY selects (the release build by
default) on fixed seeded workloads and writes, per output tensor, the SHA-256 of its bytes and,
per call, the device status word, as JSON.  tests/test_gpu_debug_bounds.py runs it once per build
and compares: the debug-bounds build must give the release build's outputs bit for bit and leave
the status word OK.

Usage: ``python -m tests.debug_bounds_run OUT.json``
"""
import hashlib
import json
import sys

import numpy as np
import torch

from delta_rule_recurrent_osdn_b200 import inputs as W
from delta_rule_recurrent_osdn_b200 import osdn


def digest(t):
    if t is None:
        return None
    return hashlib.sha256(t.detach().contiguous().cpu().view(torch.uint8).numpy().tobytes()
                          ).hexdigest()


def decay(inp, per_channel, seed):
    rng = np.random.default_rng(seed)
    shape = inp.beta.shape + ((inp.Dk,) if per_channel else ())
    a = 1.0 / (1.0 + np.exp(-(2.0 + rng.standard_normal(shape))))
    return torch.from_numpy(a.astype(np.float32)).cuda()


def fwd_case(cfg, chunk=None, alpha=None, rho=True):
    inp = W.make_inputs(cfg)
    d = W.to_torch(inp)
    kt = torch.empty_like(d["k"])
    rh = torch.empty(d["beta"].shape, device="cuda", dtype=torch.float32) if rho else None
    a = decay(inp, alpha, 7) if alpha is not None else None
    o, ST, dT = osdn.osdn_fwd(d["q"], d["k"], d["v"], d["beta"], d["r"], d["eta"], d["d0"],
                              d["S0"], d["scale"], chunk or d["chunk"], d["cu_seqlens"],
                              k_tilde=kt, rho=rh, alpha=a)
    out = dict(o=o, ST=ST, dT=dT, k_tilde=kt, rho=rh)
    if rho:
        out["q_geo"] = osdn.osdn_rho_geomean(rh, d["cu_seqlens"])
    return out


def two_call_case(cfg):
    inp = W.make_inputs(cfg)
    d = W.to_torch(inp)
    kt, dT = osdn.osdn_precond_scan(d["k"], d["beta"], d["r"], d["eta"], d["d0"],
                                    d["cu_seqlens"])
    o, ST = osdn.osdn_chunk_fwd(d["q"], d["k"], kt, d["v"], d["beta"], d["scale"], d["S0"],
                                d["chunk"], d["cu_seqlens"])
    return dict(o=o, ST=ST, dT=dT, k_tilde=kt)


def bwd_case(cfg):
    inp = W.make_inputs(cfg)
    d = W.to_torch(inp)
    rng = np.random.default_rng(5)
    dt = d["q"].dtype
    dO = torch.from_numpy(rng.standard_normal(inp.v.shape).astype(np.float32)).to("cuda", dt)
    dST = torch.from_numpy((0.3 * rng.standard_normal((inp.N, inp.H, inp.Dv, inp.Dk))
                            ).astype(np.float32)).cuda()
    ddT = torch.from_numpy(rng.standard_normal((inp.N, inp.H, inp.Dk)).astype(np.float32)).cuda()
    return osdn.osdn_bwd(d["q"], d["k"], d["v"], d["beta"], dO, d["r"], d["eta"], d["d0"],
                         d["S0"], d["scale"], dST, ddT, d["cu_seqlens"])


def step_case(N, H, Dk, Dv, dtype, seed, steps=5):
    g = torch.Generator().manual_seed(seed)
    S = (0.1 * torch.randn(N, H, Dv, Dk, generator=g)).cuda()
    dd = (1.0 + 0.1 * torch.rand(N, H, Dk, generator=g)).cuda()
    out = {}
    for i in range(steps):
        q = torch.randn(N, H, Dk, generator=g).to("cuda", dtype)
        k = torch.randn(N, H, Dk, generator=g).to("cuda", dtype)
        v = torch.randn(N, H, Dv, generator=g).to("cuda", dtype)
        beta = torch.rand(N, H, generator=g).cuda()
        r = (0.9 + 0.1 * torch.rand(N, H, generator=g)).cuda()
        out[f"o{i}"] = osdn.osdn_step(q, k, v, beta, S, dd, r, 0.05, Dk ** -0.5)
    out["S"], out["d"] = S, dd
    return out


CASES = {
    "fwd_bf16_packed": lambda: fwd_case(dict(lengths=[1, 33, 0, 64, 100, 7, 130], H=2, Dk=128,
                                             Dv=128, io="bf16", apf=True, eta=0.1, chunk=64,
                                             seed=11, init_state=True)),
    "fwd_bf16_1p3b": lambda: fwd_case("1p3b_apf"),
    "fwd_bf16_gated_channel": lambda: fwd_case(dict(B=2, T=200, H=2, Dk=128, Dv=128, io="bf16",
                                                    apf=True, eta=0.05, chunk=64, seed=12,
                                                    init_state=True), alpha=True),
    "fwd_f32_chunk32_d64": lambda: fwd_case(dict(lengths=[70, 1, 0, 130, 64], H=3, Dk=64, Dv=128,
                                                 io="f32", apf=True, eta=0.1, chunk=32, seed=13,
                                                 init_state=True), alpha=False),
    "fwd_f32_chunk16": lambda: fwd_case(dict(B=2, T=77, H=2, Dk=128, Dv=64, io="f32", apf=False,
                                             eta=0.05, chunk=16, seed=14), rho=False),
    "two_call_bf16_d64": lambda: two_call_case(dict(B=2, T=150, H=2, Dk=64, Dv=64, io="bf16",
                                                    apf=True, eta=0.05, chunk=64, seed=15,
                                                    init_state=True)),
    "bwd_bf16_packed": lambda: bwd_case(dict(lengths=[1, 33, 0, 64, 100, 7], H=2, Dk=128, Dv=128,
                                             io="bf16", apf=True, eta=0.1, chunk=64, seed=16,
                                             init_state=True)),
    "bwd_f32_d64": lambda: bwd_case(dict(B=1, T=90, H=3, Dk=64, Dv=128, io="f32", apf=True,
                                         eta=0.1, chunk=64, seed=17, init_state=True)),
    "step_bf16": lambda: step_case(8, 4, 128, 128, torch.bfloat16, 18),
    "step_f32_d64": lambda: step_case(3, 2, 64, 64, torch.float32, 19),
}


def main(path):
    torch.cuda.set_device(0)
    res = {"library": osdn.LIB_PATH}
    for name, fn in CASES.items():
        out = fn()
        torch.cuda.synchronize()
        res[name] = {"status": osdn.osdn_get_device_status(),
                     "outputs": {k: digest(v) for k, v in out.items()}}
    with open(path, "w") as f:
        json.dump(res, f, indent=1)


if __name__ == "__main__":
    main(sys.argv[1])
