"""Chunk-level algebra of the forward pass on a gated backbone, checked against the oracle.

With the key channels decaying before each write (S_t = S_{t-1} D_t + beta (v - S_{t-1} D_t k)
k~^T, D_t = Diag(alpha_t); the oracle's ``fwd_gated``), write Gamma_t = D_1 ... D_t for the
cumulative decay inside a chunk (Gamma_0 = I, t counted from the chunk's start) and rescale the
state as S~_t = S_t Gamma_t^-1.  Then
    S~_t = S~_{t-1} + beta_t (v_t - S~_{t-1} (Gamma_t k_t)) (Gamma_t^-1 k~_t)^T,
    o_t = scale S~_t (Gamma_t q_t),   S_end = S~_L Gamma_L,
which is the ungated chunk algebra with read key Gamma_t k_t, write key Gamma_t^-1 k~_t and query
Gamma_t q_t.  The Gram entries need only decay ratios between two tokens of the chunk:
    (K Gamma)(K~ Gamma^-1)^T [t, j] = sum_i k_ti k~_ji Gamma_ti / Gamma_ji   (j < t: a decay, <= 1),
    (Q Gamma)(K~ Gamma^-1)^T [t, j] likewise (j <= t),
so for Gated DeltaNet (one factor per token) they are the ungated Gram times exp(lambda_t -
lambda_j) with lambda the prefix of log alpha.  Per-channel decay (Kimi Delta Attention) needs the
ratio inside the sum; evaluating it as (K Gamma)(K~ Gamma^-1)^T overflows fp32 once a chunk's
decay passes 2^-126, which is why this statement keeps the ratio form.
"""
import numpy as np
import pytest

from oracle import osdn_ref


def _chunked_gated(q, k, kt, v, beta, alpha, S0, scale, C):
    """One (sequence, head): q, k, kt [T, Dk]; v [T, Dv]; alpha [T] or [T, Dk]."""
    T, Dk = k.shape
    a = alpha if alpha.ndim == 2 else np.repeat(alpha[:, None], Dk, axis=1)
    S = S0.copy()
    O = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, C):
        c1 = min(c0 + C, T)
        lam = np.cumsum(np.log(a[c0:c1]), axis=0)            # log Gamma_t, per key channel
        K, Kt, Q, V, b = k[c0:c1], kt[c0:c1], q[c0:c1], v[c0:c1], beta[c0:c1]
        # ratio-form Grams: sum_i x_ti y_ji exp(lam_ti - lam_ji), only for j <= t
        ratio = np.exp(np.clip(lam[:, None, :] - lam[None, :, :], None, 0.0))
        A = np.einsum("ti,ji,tji->tj", K, Kt, ratio)
        Pq = np.einsum("ti,ji,tji->tj", Q, Kt, ratio)
        G = np.exp(lam)                                       # Gamma_t (decays, <= 1)
        Tm = np.linalg.inv(np.eye(c1 - c0) + np.tril(b[:, None] * A, -1))
        W = Tm @ (b[:, None] * (V - (K * G) @ S.T))           # S~_0 = S at the chunk start
        O[c0:c1] = scale * ((Q * G) @ S.T + np.tril(Pq) @ W)
        # S_end = (S + W^T (K~ Gamma^-1)) Gamma_L = S Gamma_L + W^T (K~ Gamma_L / Gamma)
        S = S * G[-1] + W.T @ (Kt * np.exp(lam[-1] - lam))
    return O, S


@pytest.mark.parametrize("per_channel", [False, True])
@pytest.mark.parametrize("T,C", [(37, 8), (64, 16), (5, 8)])
def test_chunked_gated_forward_equals_the_oracle(per_channel, T, C):
    rng = np.random.default_rng(T * 3 + C + per_channel)
    Dk, Dv = 6, 4
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    q, k = unit(rng.standard_normal((T, Dk))), unit(rng.standard_normal((T, Dk)))
    v = rng.standard_normal((T, Dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal(T)))
    r = 1 / (1 + np.exp(-(2 + rng.standard_normal(T))))
    alpha = 1 / (1 + np.exp(-(1 + rng.standard_normal((T, Dk) if per_channel else T))))
    d0, S0 = rng.uniform(0.5, 1.5, Dk), 0.3 * rng.standard_normal((Dv, Dk))
    e4 = lambda x: x[None, :, None]
    o, kt, ST, _ = osdn_ref.fwd_gated(e4(q), e4(k), e4(v), beta[None, :, None], e4(alpha),
                                      r=r[None, :, None], eta=0.3, d0=d0[None, None],
                                      S0=S0[None, None], scale=0.9)
    # phase 1 is unchanged by the decay, so its k~ (from the oracle) feeds the chunk algebra
    O, S = _chunked_gated(q, k, kt[0, :, 0], v, beta, alpha, S0, 0.9, C)
    np.testing.assert_allclose(O, o[0, :, 0], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(S, ST[0, 0], rtol=1e-10, atol=1e-12)
