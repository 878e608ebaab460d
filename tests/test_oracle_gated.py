"""Pins for the oracle's gated-backbone form (OSDN on Gated DeltaNet / Kimi Delta Attention).

The pages give the gated delta rule on the Gated DeltaNet-2 page (section 1), key-major:
S_t = (I - k_t (b_t . k_t)^T) D_t S_{t-1} + k_t (w_t . v_t)^T, with D_t = Diag(alpha_t), which
is KDA when b_t = w_t = beta_t and Gated DeltaNet when alpha_t is also a scalar.  With the
preconditioner off (eta = 0, r = 1, d_0 = 1) the oracle's gated form must equal that equation,
transcribed here independently in the key-major convention; with it on, the decay must leave
the preconditioner's recurrence untouched.
"""
import numpy as np
import pytest

from oracle import osdn_ref


def _inputs(seed, B=2, T=9, H=2, Dk=5, Dv=3, per_channel=False):
    rng = np.random.default_rng(seed)
    norm = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    shape = (B, T, H, Dk) if per_channel else (B, T, H)
    return dict(
        q=norm(rng.standard_normal((B, T, H, Dk))), k=norm(rng.standard_normal((B, T, H, Dk))),
        v=rng.standard_normal((B, T, H, Dv)), beta=1 / (1 + np.exp(-rng.standard_normal((B, T, H)))),
        alpha=1 / (1 + np.exp(-(2 + rng.standard_normal(shape)))),
        r=1 / (1 + np.exp(-(3 + rng.standard_normal((B, T, H))))),
        S0=0.2 * rng.standard_normal((B, H, Dv, Dk)), d0=rng.uniform(0.5, 1.5, (B, H, Dk)))


def _gated_delta_rule_key_major(q, k, v, beta, alpha, S0, scale):
    """The Gated DeltaNet-2 page's update with b_t = w_t = beta_t, state [Dk, Dv]."""
    B, T, H, Dk = k.shape
    Dv = v.shape[-1]
    o = np.zeros((B, T, H, Dv))
    ST = np.zeros((B, H, Dv, Dk))
    for b in range(B):
        for h in range(H):
            S = S0[b, h].T.copy()  # key-major
            for t in range(T):
                kk, vv, bt = k[b, t, h], v[b, t, h], beta[b, t, h]
                D = np.diag(alpha[b, t, h]) if alpha.ndim == 4 else alpha[b, t, h] * np.eye(Dk)
                S = (np.eye(Dk) - bt * np.outer(kk, kk)) @ D @ S + bt * np.outer(kk, vv)
                o[b, t, h] = scale * S.T @ q[b, t, h]
            ST[b, h] = S.T
    return o, ST


@pytest.mark.parametrize("per_channel", [False, True])
def test_unit_decay_is_the_ungated_oracle(per_channel):
    x = _inputs(1, per_channel=per_channel)
    ones = np.ones_like(x["alpha"])
    args = (x["q"], x["k"], x["v"], x["beta"])
    kw = dict(r=x["r"], eta=0.2, d0=x["d0"], S0=x["S0"], scale=0.8)
    for a, b in zip(osdn_ref.fwd_gated(*args, ones, **kw), osdn_ref.fwd(*args, **kw)):
        np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("per_channel", [False, True])
def test_preconditioner_off_is_the_pages_gated_delta_rule(per_channel):
    x = _inputs(2, per_channel=per_channel)
    o, _, ST, _ = osdn_ref.fwd_gated(x["q"], x["k"], x["v"], x["beta"], x["alpha"], eta=0.0,
                                     S0=x["S0"], scale=0.7)
    o_ref, ST_ref = _gated_delta_rule_key_major(x["q"], x["k"], x["v"], x["beta"], x["alpha"],
                                                x["S0"], 0.7)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(ST, ST_ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("per_channel", [False, True])
def test_decay_leaves_the_preconditioner_alone(per_channel):
    x = _inputs(3, per_channel=per_channel)
    args = (x["q"], x["k"], x["v"], x["beta"])
    kw = dict(r=x["r"], eta=0.3, d0=x["d0"], S0=x["S0"])
    _, kt_g, _, dT_g = osdn_ref.fwd_gated(*args, x["alpha"], **kw)
    _, kt, _, dT = osdn_ref.fwd(*args, **kw)
    np.testing.assert_array_equal(kt_g, kt)
    np.testing.assert_array_equal(dT_g, dT)


def test_zero_key_only_decays_the_state():
    x = _inputs(4, B=1, T=1, H=1, per_channel=True)
    x["k"][:] = 0.0
    _, _, ST, _ = osdn_ref.fwd_gated(x["q"], x["k"], x["v"], x["beta"], x["alpha"], eta=0.5,
                                     S0=x["S0"])
    np.testing.assert_array_equal(ST[0, 0], x["S0"][0, 0] * x["alpha"][0, 0, 0][None, :])


MUTATIONS = {
    # the value channels decay instead of the key channels
    "decay_on_value_channels": ("alpha_per_channel ? alpha[th * Dk + i] : alpha[th]",
                                "alpha_per_channel ? alpha[th * Dk + j] : alpha[th]"),
    # the per-channel gate read as one factor per token
    "per_channel_ignored": ("alpha_per_channel ? alpha[th * Dk + i] : alpha[th]", "alpha[th]"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_in_gated_form_is_caught(tmp_path, name):
    old, new = MUTATIONS[name]
    src = open(osdn_ref.SOURCE).read()
    assert old in src
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    mutant = osdn_ref.Oracle(osdn_ref.compile_source(str(path), str(tmp_path / f"libgated_{name}.so")))
    x = _inputs(2, per_channel=True)
    o, _, _, _ = mutant.fwd_gated(x["q"], x["k"], x["v"], x["beta"], x["alpha"], eta=0.0,
                                  S0=x["S0"], scale=0.7)
    o_ref, _ = _gated_delta_rule_key_major(x["q"], x["k"], x["v"], x["beta"], x["alpha"], x["S0"], 0.7)
    assert np.abs(o - o_ref).max() > 1e-6
