"""Chunk-level algebra of the forward kernels for bf16 with d_k = 128, stated in numpy fp64 and
checked against the oracle's token loops on the CPU.

Phase 1 in chunk form (precond_prep_kernel and precond_chain_kernel).  With a_t = k_t (.) k_t,
e_t = eta beta_t / ||k_t||^2 (0 for a zero key), c_t = e_t beta_t, R_t = prod_{i<t} r_i and
Gamma_tj = prod_{j<i<t} r_i inside a chunk, the token recurrence d_{t+1} = r_t d_t + x_t a_t with
x_t = e_t (1 - beta_t <d_t, a_t>) unrolls to
    (I + L_d) x = b,   L_d[t][j] = c_t Gamma_tj <a_t, a_j> (j < t),   b = e (.) (1 - beta (.) R (.) A d_0),
    d_C = R_C d_0 + A^T (g (.) x),   g_j = Gamma_Cj,
and k~_t = d_t (.) k_t follows from x by the token recurrence.  Gamma is evaluated from prefix sums
of log|r| and a sign parity: as a product of one factor per row and one per column when every
prefix of the chunk lies within +-80, one exponential per entry otherwise.

Phase 2 in the lookahead form (wy_prep_kernel and chunk_fwd_tc_kernel).  Per chunk c, with
T_c = (I + strict_tril(diag(beta) K_c K~_c^T))^-1, R_c = beta (.) (V_c - K_c S_c^T) and W_c = T_c R_c,
    S_{c+1} = S_c + W_c^T K~_c,    O_c = Q_c S_c^T + tril(Q_c K~_c^T) W_c,
and the product that starts chunk c + 1 is assembled before S_{c+1} exists:
    [K_{c+1}; Q_c] S_c^T + [K_{c+1} K~_c^T; tril(Q_c K~_c^T)] W_c = [K_{c+1} S_{c+1}^T; O_c].
A short last chunk is padded with zero rows (identity rows of T).

The two-term bf16 split of a computed operand (split2_bf16): Veltkamp's head hi = t - (t - x) with
t = (2^16 + 1) x in fp32 has at most 8 significant bits, so it is exactly a bf16 value (its low 16
bits are zero); the residual x - hi is exact in fp32 and keeps its upper 16 bits as the lo term,
and |x - hi - lo| <= 2^-16 |x|.
"""
import numpy as np
import pytest

from oracle import osdn_ref


def phase1_chunked(k, beta, r, eta, d0, C):
    """One (sequence, head): k [T, Dk], beta and r [T] (r None: no APF).  Returns k~, d_T and
    whether any chunk took the per-entry exponentials."""
    T, Dk = k.shape
    d = d0.copy()
    kt = np.zeros_like(k)
    per_entry = False
    for c0 in range(0, T, C):
        c1 = min(c0 + C, T)
        L = c1 - c0
        K, bt = k[c0:c1], beta[c0:c1]
        rr = np.ones(L) if r is None else r[c0:c1]
        A = K * K
        nk = A.sum(axis=1)
        e = np.where(nk > 0, eta * bt / np.where(nk > 0, nk, 1.0), 0.0)
        cc = e * bt
        lr = np.concatenate([[0.0], np.cumsum(np.log(np.abs(rr)))])  # lr[t] = sum_{i<t} log|r_i|
        sg = np.where(np.concatenate([[0], np.cumsum(rr < 0)]) % 2, -1.0, 1.0)
        # Gamma[t][j] = prod_{j<i<t} r_i = sg[t] sg[j+1] exp(lr[t] - lr[j+1]), t = 0..L, j = 0..L-1
        if np.all(np.abs(lr) < 80.0):
            Gam = (sg * np.exp(lr))[:, None] * (sg[1:] * np.exp(-lr[1:]))[None, :]
        else:
            per_entry = True
            Gam = sg[:, None] * sg[None, 1:] * np.exp(lr[:, None] - lr[None, 1:])
        Ld = np.tril(cc[:, None] * Gam[:L] * (A @ A.T), -1)
        Rt = sg[:L] * np.exp(lr[:L])
        b = e * (1.0 - bt * Rt * (A @ d))
        x = np.linalg.solve(np.eye(L) + Ld, b)
        dd = d.copy()
        for t in range(L):  # the k~ writer's token recurrence
            kt[c0 + t] = dd * K[t]
            dd = rr[t] * dd + x[t] * A[t]
        d_C = sg[L] * np.exp(lr[L]) * d + A.T @ (Gam[L] * x)
        np.testing.assert_allclose(d_C, dd, rtol=1e-10, atol=1e-14)  # the chain's d_C
        d = d_C
    return kt, d, per_entry


def phase2_lookahead(q, k, kt, v, beta, S0, scale, C):
    """One (sequence, head): q, k, kt [T, Dk]; v [T, Dv]; S0 [Dv, Dk].  Returns O, S_T."""
    T, Dk = k.shape
    nch = (T + C - 1) // C

    def tile(a, c):
        out = np.zeros((C,) + a.shape[1:])
        if c < nch:
            part = a[c * C:min((c + 1) * C, T)]
            out[:len(part)] = part
        return out

    S = S0.copy()
    O = np.zeros((T, v.shape[1]))
    D1_top = tile(k, 0) @ S.T  # D1_0: K_0 S_0^T
    for c in range(nch):
        K, Kt, Q, V, b = (tile(a, c) for a in (k, kt, q, v, beta))
        Tm = np.linalg.inv(np.eye(C) + np.tril(b[:, None] * (K @ Kt.T), -1))
        W = Tm @ (b[:, None] * (V - D1_top))  # R from the rows of D1, then W = T R
        Kn = tile(k, c + 1)
        top = Kn @ S.T + (Kn @ Kt.T) @ W      # [K_{c+1}; Q_c] S_c^T + [X_{c+1}; P_c] W_c
        bottom = Q @ S.T + np.tril(Q @ Kt.T) @ W
        S = S + W.T @ Kt                      # the state update, off the chain
        np.testing.assert_allclose(top, Kn @ S.T, rtol=1e-9, atol=1e-12)
        L = min(C, T - c * C)
        O[c * C:c * C + L] = scale * bottom[:L]
        D1_top = top
    return O, S


def _inputs(rng, T, Dk, Dv, apf=True, r_scale=3.0):
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    q, k = unit(rng.standard_normal((T, Dk))), unit(rng.standard_normal((T, Dk)))
    v = rng.standard_normal((T, Dv))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(T)))
    r = 1.0 / (1.0 + np.exp(-(r_scale + rng.standard_normal(T)))) if apf else None
    return q, k, v, beta, r


def _oracle_phase1(k, beta, r, eta, d0):
    e3 = lambda x: x[None, :, None]
    kt, dT = osdn_ref.precond_scan(e3(k), beta[None, :, None],
                                   None if r is None else r[None, :, None], eta, d0[None, None])
    return kt[0, :, 0], dT[0, 0]


@pytest.mark.parametrize("T,C,apf", [(150, 64, True), (64, 64, True), (1, 64, True),
                                     (200, 64, False), (77, 16, True)])
def test_phase1_chunk_form_equals_the_token_loop(T, C, apf):
    rng = np.random.default_rng(1000 + T + C + apf)
    _, k, _, beta, r = _inputs(rng, T, 24, 4, apf)
    k[T // 3] = 0.0  # a zero key inside a chunk: e = 0, the token only forgets
    d0 = rng.uniform(0.5, 1.5, 24)
    kt, dT, per_entry = phase1_chunked(k, beta, r, 0.3, d0, C)
    assert not per_entry
    okt, odT = _oracle_phase1(k, beta, r, 0.3, d0)
    np.testing.assert_allclose(kt, okt, rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(dT, odT, rtol=1e-10, atol=1e-14)


def test_phase1_strong_forgetting_takes_per_entry_exponentials():
    """r of a few percent over a whole chunk drives the log prefix past 80: the row-times-column
    factors would leave the fp32 range, so Gamma is evaluated one exponential per entry."""
    rng = np.random.default_rng(7)
    T, C = 192, 64
    _, k, _, beta, r = _inputs(rng, T, 16, 4)
    r[64:128] = rng.uniform(0.01, 0.05, 64)
    d0 = rng.uniform(0.5, 1.5, 16)
    kt, dT, per_entry = phase1_chunked(k, beta, r, 0.2, d0, C)
    assert per_entry
    okt, odT = _oracle_phase1(k, beta, r, 0.2, d0)
    np.testing.assert_allclose(kt, okt, rtol=1e-9, atol=1e-14)
    np.testing.assert_allclose(dT, odT, rtol=1e-9, atol=1e-14)


def test_phase1_sign_parity_of_negative_retention():
    """The recurrence as printed takes any r; the sign of Gamma is the parity of the negative
    factors between the two tokens."""
    rng = np.random.default_rng(8)
    T, C = 100, 32
    _, k, _, beta, r = _inputs(rng, T, 12, 4)
    r[rng.choice(T, 17, replace=False)] *= -1.0
    d0 = rng.uniform(0.5, 1.5, 12)
    kt, dT, _ = phase1_chunked(k, beta, r, 0.25, d0, C)
    okt, odT = _oracle_phase1(k, beta, r, 0.25, d0)
    np.testing.assert_allclose(kt, okt, rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(dT, odT, rtol=1e-10, atol=1e-14)


@pytest.mark.parametrize("T,C", [(150, 64), (64, 64), (1, 64), (130, 32), (40, 16)])
def test_phase2_lookahead_form_equals_the_token_loop(T, C):
    rng = np.random.default_rng(2000 + T + C)
    Dk, Dv = 20, 12
    q, k, v, beta, r = _inputs(rng, T, Dk, Dv)
    kt, _ = _oracle_phase1(k, beta, r, 0.2, np.ones(Dk))
    S0 = 0.2 * rng.standard_normal((Dv, Dk))
    O, S = phase2_lookahead(q, k, kt, v, beta, S0, 0.7, C)
    e4 = lambda x: x[None, :, None]
    o, ST = osdn_ref.delta_fwd(e4(q), e4(k), e4(kt), e4(v), beta[None, :, None], 0.7,
                               S0[None, None])
    np.testing.assert_allclose(O, o[0, :, 0], rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(S, ST[0, 0], rtol=1e-9, atol=1e-12)


def split2(x):
    """fp32 x -> (hi, lo) as bf16 bit patterns, by the fp32 steps of the kernels' split."""
    x = x.astype(np.float32)
    t = np.float32(65537.0) * x
    hi = t - (t - x)
    lo = x - hi
    return hi.view(np.uint32), lo.view(np.uint32)


def test_two_term_split_is_exact_to_2_pow_minus_16():
    rng = np.random.default_rng(9)
    mant = rng.uniform(1.0, 2.0, 200000)
    expo = rng.integers(-100, 100, 200000)
    sign = rng.choice([-1.0, 1.0], 200000)
    x = np.concatenate([(sign * mant * np.exp2(expo)).astype(np.float32),
                        # values next to bf16 rounding boundaries, and exact bf16 values
                        (1.0 + np.arange(256) / 256.0 + 2.0 ** -9).astype(np.float32),
                        (1.0 + np.arange(256) / 256.0).astype(np.float32),
                        np.float32([0.0, 1.0, -3.0, 2.0 ** -60, 2.0 ** 100])])
    hb, lb = split2(x)
    assert np.all(hb & 0xFFFF == 0)  # hi is exactly a bf16 value
    hi = hb.view(np.float32).astype(np.float64)
    lo = (lb & np.uint32(0xFFFF0000)).view(np.float32).astype(np.float64)  # the upper half
    err = np.abs(x.astype(np.float64) - hi - lo)
    assert np.all(err <= 2.0 ** -16 * np.abs(x.astype(np.float64)))
    # the bound is close to tight: a one-term bf16 rounding is 2^-9, the split gains 7 bits
    rel = err[x != 0] / np.abs(x[x != 0].astype(np.float64))
    assert rel.max() > 2.0 ** -18
