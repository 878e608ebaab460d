"""The seeded input recipe of the named workloads, as the design describes it: shapes, the
distributions of every tensor, bf16 rounding of the token data in bf16 workloads, and the
varlen draw.  The big workloads are checked on copies with fewer tokens or heads, which draw from
the same recipe (the varlen lengths are drawn first, so they do not depend on H or d)."""
import numpy as np
import pytest

from delta_rule_recurrent_osdn_b200 import inputs as W


def small(name, **kw):
    cfg = dict(W.CONFIGS[name])
    cfg.update(kw)
    return W.make_inputs(cfg)


def is_bf16(a):
    return np.all(np.asarray(a, np.float32).view(np.uint32) & 0xFFFF == 0)


@pytest.mark.parametrize("name,kw", [("tiny_fp32", {}), ("340m", dict(B=2, T=512)),
                                     ("1p3b_apf", dict(B=1, T=512, H=4)),
                                     ("long_ctx", dict(T=2048, H=4)),
                                     ("varlen", dict(num_seqs=4, H=2))])
def test_recipe_of_every_workload(name, kw):
    cfg = dict(W.CONFIGS[name])
    cfg.update(kw)
    inp = W.make_inputs(cfg)
    B, T, H = inp.beta.shape
    assert inp.q.shape == inp.k.shape == (B, T, H, cfg["Dk"]) and inp.v.shape[-1] == cfg["Dv"]
    # q, k unit-norm per (token, head) before the io rounding
    tol = 1e-2 if cfg["io"] == "bf16" else 1e-5
    for a in (inp.q, inp.k):
        assert np.allclose(np.linalg.norm(a.astype(np.float64), axis=-1), 1.0, atol=tol)
    if cfg["io"] == "bf16":
        assert is_bf16(inp.q) and is_bf16(inp.k) and is_bf16(inp.v)
    # gates: beta = sigmoid(N(0, 1)), r = sigmoid(N(3, 1)) with APF, none without
    assert inp.beta.dtype == np.float32 and np.all((inp.beta > 0) & (inp.beta < 1))
    assert abs(float(np.median(inp.beta)) - 0.5) < 0.05
    if cfg["apf"]:
        assert np.all((inp.r > 0) & (inp.r < 1))
        assert abs(float(np.median(inp.r)) - 1 / (1 + np.exp(-3.0))) < 0.02
    else:
        assert inp.r is None
    assert inp.eta == cfg["eta"] and inp.chunk == cfg["chunk"]
    if cfg.get("init_state"):
        assert abs(float(inp.S0.std()) - 0.1) < 0.01
        assert inp.d0.min() >= 0.5 and inp.d0.max() <= 1.5
    else:
        assert inp.S0 is None and inp.d0 is None


def test_varlen_draw():
    inp = small("varlen", H=1, Dk=64, Dv=64)
    lengths = np.diff(inp.cu_seqlens)
    assert len(lengths) == 32 and inp.cu_seqlens[0] == 0
    assert lengths.min() >= 128 and lengths.max() <= 8192
    assert int(inp.cu_seqlens[-1]) == 161_577  # the total the design quotes for this seed
    assert inp.beta.shape[:2] == (1, 161_577)


def test_inputs_are_deterministic_per_seed():
    a, b = small("1p3b_apf", T=64, H=2), small("1p3b_apf", T=64, H=2)
    for x, y in ((a.q, b.q), (a.k, b.k), (a.v, b.v), (a.beta, b.beta), (a.r, b.r)):
        np.testing.assert_array_equal(x, y)
    c = small("1p3b_apf", T=64, H=2, seed=99)
    assert not np.array_equal(a.q, c.q)
