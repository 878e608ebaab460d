"""Pins for the oracle's backward pass (reverse-mode gradient of the token loop).

The pages give no backward pass, so the gradient is pinned to the forward oracle, which the
pins in test_oracle_pins.py tie to the pages: for L = <dO, o> + <dST, S_T> + <ddT, d_T>, the
directional derivative <grad_x L, delta> must equal the central difference
(L(x + eps delta) - L(x - eps delta)) / (2 eps) of the forward oracle, for every input x and
random directions delta, in fp64 (the difference's truncation error is O(eps^2), its rounding
error O(1e-16 |L| / eps)).  Planted mistakes in a copy of the backward must fail that check.
"""
import numpy as np
import pytest

from oracle import osdn_ref

EPS = 1e-6
RTOL = 1e-7


def _problem(case, seed=0):
    rng = np.random.default_rng(seed)
    B, T, H, Dk, Dv = 2, 7, 2, 4, 3
    cu = None
    if case == "packed":
        B, T = 1, 12
        cu = np.array([0, 3, 3, 12], dtype=np.int32)  # includes an empty sequence
    N = B if cu is None else len(cu) - 1
    norm = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    p = {
        "q": norm(rng.standard_normal((B, T, H, Dk))),
        "k": norm(rng.standard_normal((B, T, H, Dk))),
        "v": rng.standard_normal((B, T, H, Dv)),
        "beta": 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H)))),
        "r": 1.0 / (1.0 + np.exp(-(3.0 + rng.standard_normal((B, T, H))))),
        "d0": rng.uniform(0.5, 1.5, (N, H, Dk)),
        "S0": 0.1 * rng.standard_normal((N, H, Dv, Dk)),
    }
    kw = {"eta": 0.3, "scale": 0.7, "cu_seqlens": cu}
    p["alpha"] = None
    if case in ("gated_gdn", "gated_kda"):  # decay of a gated backbone (the oracle's fwd_gated)
        shape = (B, T, H, Dk) if case == "gated_kda" else (B, T, H)
        p["alpha"] = 1.0 / (1.0 + np.exp(-(1.0 + rng.standard_normal(shape))))
    if case == "no_apf":
        p["r"] = None
    if case == "zero_key":  # the ||k||^2 == 0 branch (gradient of the surrogate taken as 0)
        p["k"][0, 2, 1] = 0.0
        # the d update is not differentiable in k there: as k -> 0 along delta it tends to
        # eta beta (1 - beta s) delta^2 / ||delta||^2, not to the 0 taken at k = 0 itself, so
        # the k directions leave that token's key alone (every other input is still checked)
        kw["k_fixed"] = (0, 2, 1)
    up = {
        "dO": rng.standard_normal((B, T, H, Dv)),
        "dST": rng.standard_normal((N, H, Dv, Dk)),
        "ddT": rng.standard_normal((N, H, Dk)),
    }
    return p, kw, up


def _loss(ref, p, kw, up):
    args = dict(r=p["r"], eta=kw["eta"], d0=p["d0"], S0=p["S0"], scale=kw["scale"],
                cu_seqlens=kw["cu_seqlens"])
    if p["alpha"] is None:
        o, _, ST, dT = ref.fwd(p["q"], p["k"], p["v"], p["beta"], **args)
    else:
        o, _, ST, dT = ref.fwd_gated(p["q"], p["k"], p["v"], p["beta"], p["alpha"], **args)
    return (o * up["dO"]).sum() + (ST * up["dST"]).sum() + (dT * up["ddT"]).sum()


def _grads(ref, p, kw, up):
    return ref.bwd(p["q"], p["k"], p["v"], p["beta"], up["dO"], r=p["r"], eta=kw["eta"],
                   d0=p["d0"], S0=p["S0"], scale=kw["scale"], dST=up["dST"], ddT=up["ddT"],
                   cu_seqlens=kw["cu_seqlens"], alpha=p["alpha"])


def _check(ref, case, seed=0):
    """Largest relative mismatch between analytic and central-difference derivatives."""
    p, kw, up = _problem(case, seed)
    g = _grads(ref, p, kw, up)
    rng = np.random.default_rng(100 + seed)
    worst = 0.0
    names = [n for n in ("q", "k", "v", "beta", "r", "d0", "S0", "alpha") if p[n] is not None]
    for name in names + ["eta"]:
        for _ in range(2):
            if name == "eta":
                delta = 1.0
                plus = dict(kw, eta=kw["eta"] + EPS)
                minus = dict(kw, eta=kw["eta"] - EPS)
                fd = (_loss(ref, p, plus, up) - _loss(ref, p, minus, up)) / (2 * EPS)
                an = g["deta"] * delta
            else:
                delta = rng.standard_normal(p[name].shape)
                if name == "k" and "k_fixed" in kw:
                    delta[kw["k_fixed"]] = 0.0
                pp = dict(p, **{name: p[name] + EPS * delta})
                pm = dict(p, **{name: p[name] - EPS * delta})
                fd = (_loss(ref, pp, kw, up) - _loss(ref, pm, kw, up)) / (2 * EPS)
                an = (g["d" + name] * delta).sum()
            worst = max(worst, abs(fd - an) / max(abs(an), abs(fd), 1.0))
    return worst


@pytest.mark.parametrize("case", ["apf", "no_apf", "packed", "zero_key", "gated_gdn", "gated_kda"])
def test_gradient_matches_central_differences(case):
    ref = osdn_ref._oracle()
    assert _check(ref, case) <= RTOL


def test_gradient_of_a_single_token_by_hand():
    """One token, Dk = Dv = 1, S0 = 0, d0 = 1: the write key is w = d k = k and u = v, so
    o = scale beta v k q and d_T = r + eta beta (1 - beta k^2) (g a with a = n = k^2); for
    L = o + d_T every derivative has a closed form."""
    ref = osdn_ref._oracle()
    qv, kv, vv, bv, rv, eta, scale = 0.8, 0.6, 1.3, 0.4, 0.9, 0.25, 1.5
    one = lambda x: np.full((1, 1, 1, 1), x)
    g = ref.bwd(one(qv), one(kv), one(vv), np.full((1, 1, 1), bv), one(1.0),
                r=np.full((1, 1, 1), rv), eta=eta, scale=scale, dST=np.zeros((1, 1, 1, 1)),
                ddT=np.ones((1, 1, 1)))
    assert np.isclose(g["dq"].item(), scale * bv * vv * kv)
    assert np.isclose(g["dv"].item(), scale * bv * kv * qv)
    assert np.isclose(g["dk"].item(), scale * bv * vv * qv - 2 * eta * bv ** 2 * kv)
    assert np.isclose(g["dbeta"].item(), scale * vv * kv * qv + eta * (1 - 2 * bv * kv ** 2))
    assert np.isclose(g["dr"].item(), 1.0)
    assert np.isclose(g["deta"], bv * (1 - bv * kv ** 2))
    assert np.isclose(g["dd0"].item(), rv + scale * bv * vv * kv * qv - eta * bv ** 2 * kv ** 2)


# plausible mistakes in the reverse sweep, planted in a copy of the oracle's C source
MUTATIONS = {
    "beta_grad_of_g_drops_2": ("gg * eta * (1.0 - 2.0 * bt * s) / knorm2", "gg * eta * (1.0 - bt * s) / knorm2"),
    "readout_adjoint_dropped": ("gS[(int64_t)j * Dk + i] += scale * gOt[j] * qt[i];", "(void)qt;"),
    "residual_sign": ("gS[(int64_t)j * Dk + i] -= gu[j] * kt[i];", "gS[(int64_t)j * Dk + i] += gu[j] * kt[i];"),
    "gate_not_propagated": ("gdp[i] = rt * gd[i];", "gdp[i] = gd[i];"),
    "square_factor_dropped": ("2.0 * kt[i] * ga[i]", "kt[i] * ga[i]"),
    "query_grad_uses_old_state": ("acc += Sn[(int64_t)j * Dk + i] * gOt[j];", "acc += S[(int64_t)j * Dk + i] * gOt[j];"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_in_backward_is_caught(tmp_path, name):
    old, new = MUTATIONS[name]
    src = open(osdn_ref.SOURCE).read()
    assert old in src, f"mutation anchor for {name} not found"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    mutant = osdn_ref.Oracle(osdn_ref.compile_source(str(path), str(tmp_path / f"libbwd_{name}.so")))
    assert max(_check(mutant, case) for case in ("apf", "packed")) > 1e-4


# mistakes in the decay's part of the reverse sweep (Gated DeltaNet decay, one factor per token)
GATED_MUTATIONS = {
    "decay_adjoint_dropped": ("for (int64_t e = 0; e < SZ; ++e) gS[e] *= alpha[th];", "(void)0;"),
    "dalpha_from_decayed_state": ("for (int64_t e = 0; e < SZ; ++e) acc += gS[e] * Sp[e];",
                                  "for (int64_t e = 0; e < SZ; ++e) acc += gS[e] * S[e];"),
}


@pytest.mark.parametrize("name", sorted(GATED_MUTATIONS))
def test_planted_mistake_in_gated_backward_is_caught(tmp_path, name):
    old, new = GATED_MUTATIONS[name]
    src = open(osdn_ref.SOURCE).read()
    assert old in src, f"mutation anchor for {name} not found"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    mutant = osdn_ref.Oracle(osdn_ref.compile_source(str(path), str(tmp_path / f"libgbwd_{name}.so")))
    assert _check(mutant, "gated_gdn") > 1e-4
    assert _check(osdn_ref._oracle(), "gated_gdn") <= RTOL
