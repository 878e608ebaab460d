"""Pins for the fp64 oracle: each test checks it against something other than itself.

The reference is the OSDN summary pages ("OSDN: Improving Delta Rule with Provable Online
Preconditioning in Linear Attention"): section 1 defines the per-token loss f_t and the delta
rule, section 2.1 the right-preconditioned gradient step, section 2.2 the surrogate h_t (its
definition and its closed form) and the two-phase split, section 2.3 the APF gate, and
section 3 (Theorem 5.2) the gated-Newton condition beta <d*, k^2> = 1.

Independent routes used here: central finite differences of the loss and of the surrogate's
DEFINITION (both are exact quadratics, so central differences are exact up to rounding),
dense brute-force products of the per-token transition matrices, textbook delta-rule
properties, closed-form solutions of the preconditioner recurrence for repeated one-hot
keys, and a two-token example worked by hand (tests/golden/hand_two_tokens.json).
"""
import json
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_case(rng, B=1, T=1, H=1, Dk=4, Dv=3, unit=True):
    k = rng.standard_normal((B, T, H, Dk))
    q = rng.standard_normal((B, T, H, Dk))
    if unit:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, Dv))
    beta = rng.uniform(0.1, 0.95, (B, T, H))
    return q, k, v, beta


# ----------------------------------------------------------------- definitions from section 1/2
def loss(S, k, v):
    """f(S) = 1/2 ||S k - v||^2 (section 1)."""
    e = S @ k - v
    return 0.5 * float(e @ e)


def loss_grad_fd(S, k, v, eps=1e-3):
    """Gradient of f by central differences, entry by entry (exact for a quadratic)."""
    G = np.zeros_like(S)
    for idx in np.ndindex(S.shape):
        E = np.zeros_like(S)
        E[idx] = eps
        G[idx] = (loss(S + E, k, v) - loss(S - E, k, v)) / (2 * eps)
    return G


def surrogate_def(dvec, S, k, v, beta):
    """h(d) = (f(S_new) - f(S)) / ||grad f(S)||_F^2 with S_new = S - beta grad f(S) diag(d)
    (definition in section 2.2, S_new from the left-hand side of section 2.1's update)."""
    G = loss_grad_fd(S, k, v)
    S_new = S - beta * G @ np.diag(dvec)
    return (loss(S_new, k, v) - loss(S, k, v)) / float((G * G).sum())


def surrogate_grad_fd(dvec, S, k, v, beta, eps=1e-3):
    g = np.zeros_like(dvec)
    for i in range(len(dvec)):
        e = np.zeros_like(dvec)
        e[i] = eps
        g[i] = (surrogate_def(dvec + e, S, k, v, beta) -
                surrogate_def(dvec - e, S, k, v, beta)) / (2 * eps)
    return g


def one_token(ref, S, d, q, k, v, beta, r, eta):
    """Run the oracle on a single token with explicit initial state."""
    Dv, Dk = S.shape
    o, kt, ST, dT = ref.fwd(q.reshape(1, 1, 1, Dk), k.reshape(1, 1, 1, Dk), v.reshape(1, 1, 1, Dv),
                            np.array([[[beta]]]), None if r is None else np.array([[[r]]]), eta,
                            d.reshape(1, 1, Dk), S.reshape(1, 1, Dv, Dk))
    return o[0, 0, 0], kt[0, 0, 0], ST[0, 0], dT[0, 0]


# ------------------------------------------------------------------------------------ P2
def test_state_update_is_preconditioned_gradient_step(ref):
    """P2 (section 2.1): S_t = S_{t-1} - beta grad f(S_{t-1}) D_t, grad by finite differences;
    also k~ = d (.) k and o = S_t q."""
    rng = np.random.default_rng(11)
    for _ in range(50):
        S = rng.standard_normal((3, 4))
        d = rng.uniform(0.3, 2.0, 4)
        q, k, v, beta = (a.reshape(-1) if np.ndim(a) else a for a in rand_case(rng))
        beta = float(np.asarray(beta).reshape(()))
        o, kt, S1, _ = one_token(ref, S, d, q, k, v, beta, None, 0.1)
        G = loss_grad_fd(S, k, v)
        np.testing.assert_allclose(S1, S - beta * G @ np.diag(d), rtol=0, atol=1e-9)
        np.testing.assert_allclose(kt, d * k, rtol=0, atol=1e-15)
        np.testing.assert_allclose(o, S1 @ q, rtol=0, atol=1e-12)


# ------------------------------------------------------------------------------- P1/P4/P3
def test_preconditioner_step_is_descent_on_surrogate_definition(ref):
    """P4 + sign (sections 2.2/2.3): d_{t+1} = r d_t - eta grad h(d_t), with grad h taken by
    finite differences of h's DEFINITION built from explicit S; P3: h decreases."""
    rng = np.random.default_rng(12)
    descents = 0
    for trial in range(40):
        S = rng.standard_normal((3, 4))
        d = rng.uniform(0.3, 2.0, 4)
        # keys of arbitrary norm, so that the 1/||k||^2 factor is exercised
        q, k, v, beta = (a.reshape(-1) if np.ndim(a) else a
                         for a in rand_case(rng, unit=(trial % 4 == 0)))
        beta = float(np.asarray(beta).reshape(()))
        r = None if trial % 2 == 0 else float(rng.uniform(0.5, 1.0))
        eta = float(rng.uniform(0.01, 0.5))
        _, _, _, d1 = one_token(ref, S, d, q, k, v, beta, r, eta)
        g = surrogate_grad_fd(d, S, k, v, beta)
        rr = 1.0 if r is None else r
        np.testing.assert_allclose((rr * d - d1) / eta, g, rtol=1e-7, atol=1e-9)
        # h is quadratic in d with Hessian beta^2 a a^T / ||k||^2 (a = k^2) and g is parallel
        # to a, so a gradient step strictly lowers h when eta beta^2 ||a||^2 / ||k||^2 < 2.
        a = k * k
        if r is None and np.abs(g).max() > 1e-8 and eta * beta**2 * (a @ a) / (k @ k) < 2:
            assert surrogate_def(d1, S, k, v, beta) < surrogate_def(d, S, k, v, beta)
            descents += 1
    assert descents >= 5


def test_pages_closed_form_equals_definition():
    """P1 (section 2.2): the printed closed form of h equals its definition (checks our
    reading of the pages; the oracle uses the gradient of this form)."""
    rng = np.random.default_rng(13)
    for _ in range(200):
        S = rng.standard_normal((3, 4))
        d = rng.uniform(0.0, 2.0, 4)
        k = rng.standard_normal(4)
        v = rng.standard_normal(3)
        beta = float(rng.uniform(0.05, 1.0))
        closed = ((1 - beta * d @ (k * k)) ** 2 - 1) / (2 * k @ k)
        assert abs(surrogate_def(d, S, k, v, beta) - closed) <= 1e-9 * max(1.0, abs(closed))


# ------------------------------------------------------------------------------------ P9
def brute_force_states(k, kt, v, beta, S0):
    """S_t = S_0 prod_{s<=t}(I - beta_s k_s k~_s^T) + sum_s beta_s v_s k~_s^T prod_{s<u<=t}(...)
    with explicit dense matrices; returns the list of S_t."""
    T, Dk = k.shape
    out = []
    for t in range(T):
        P = np.eye(Dk)
        for s in range(t + 1):
            P = P @ (np.eye(Dk) - beta[s] * np.outer(k[s], kt[s]))
        S = S0 @ P
        for s in range(t + 1):
            tail = np.eye(Dk)
            for u in range(s + 1, t + 1):
                tail = tail @ (np.eye(Dk) - beta[u] * np.outer(k[u], kt[u]))
            S = S + beta[s] * np.outer(v[s], kt[s]) @ tail
        out.append(S)
    return out


@pytest.mark.parametrize("Dk,Dv,T", [(4, 3, 7), (8, 5, 16), (6, 6, 1)])
def test_brute_force_product(ref, Dk, Dv, T):
    """P9: the sequential oracle equals the unrolled product of (I - beta k k~^T) factors,
    for S_T and for every o_t = S_t q_t."""
    rng = np.random.default_rng(14 + T)
    q, k, v, beta = rand_case(rng, T=T, Dk=Dk, Dv=Dv)
    r = rng.uniform(0.6, 1.0, (1, T, 1))
    S0 = 0.3 * rng.standard_normal((1, 1, Dv, Dk))
    d0 = rng.uniform(0.5, 1.5, (1, 1, Dk))
    o, kt, ST, _ = ref.fwd(q, k, v, beta, r, 0.2, d0, S0)
    states = brute_force_states(k[0, :, 0], kt[0, :, 0], v[0, :, 0], beta[0, :, 0], S0[0, 0])
    np.testing.assert_allclose(ST[0, 0], states[-1], rtol=0, atol=1e-12)
    for t in range(T):
        np.testing.assert_allclose(o[0, t, 0], states[t] @ q[0, t, 0], rtol=0, atol=1e-12)


# ------------------------------------------------------------------------------------ P5
def test_eta_zero_reduces_to_deltanet(ref):
    """P5 (section 1): eta=0, r==1, d_0=1 gives k~ == k; the delta rule then writes exactly
    (beta=1, unit key: S_t k_t = v_t), and orthonormal keys from S_0=0 give S = sum v k^T."""
    rng = np.random.default_rng(15)
    q, k, v, beta = rand_case(rng, T=9, Dk=6, Dv=4)
    o, kt, ST, dT = ref.fwd(q, k, v, beta, None, 0.0)
    assert np.array_equal(kt, k)
    assert np.array_equal(dT, np.ones_like(dT))
    states = brute_force_states(k[0, :, 0], k[0, :, 0], v[0, :, 0], beta[0, :, 0], np.zeros((4, 6)))
    np.testing.assert_allclose(ST[0, 0], states[-1], atol=1e-12)
    # exact write with beta=1
    ones = np.ones_like(beta)
    for t in range(1, 9):
        _, _, St, _ = ref.fwd(q[:, :t], k[:, :t], v[:, :t], ones[:, :t], None, 0.0)
        np.testing.assert_allclose(St[0, 0] @ k[0, t - 1, 0], v[0, t - 1, 0], atol=1e-12)
    # orthonormal keys
    Qm, _ = np.linalg.qr(rng.standard_normal((6, 6)))
    ko = Qm.T[None, :, None, :].copy()  # 6 orthonormal rows
    vo = rng.standard_normal((1, 6, 1, 4))
    _, _, So, _ = ref.fwd(ko, ko, vo, np.ones((1, 6, 1)), None, 0.0)
    np.testing.assert_allclose(So[0, 0], sum(np.outer(vo[0, t, 0], ko[0, t, 0]) for t in range(6)),
                               atol=1e-12)


# ------------------------------------------------------------------------------------ P6
def test_no_apf_equals_unit_retention(ref):
    """P6 (section 2.3): r omitted == r identically 1, bit for bit."""
    rng = np.random.default_rng(16)
    q, k, v, beta = rand_case(rng, B=2, T=11, H=2, Dk=8, Dv=5)
    a = ref.fwd(q, k, v, beta, None, 0.3)
    b = ref.fwd(q, k, v, beta, np.ones_like(beta), 0.3)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    ka, da = ref.precond_scan(k, beta, None, 0.3)
    kb, db = ref.precond_scan(k, beta, np.ones_like(beta), 0.3)
    assert np.array_equal(ka, kb) and np.array_equal(da, db)


# ------------------------------------------------------------------------------------ P7
@pytest.mark.parametrize("beta,r,eta,d0", [(0.8, 1.0, 0.3, 1.0), (0.5, 1.0, 0.9, 2.5),
                                           (0.9, 0.7, 0.2, 1.0), (0.6, 0.95, 0.05, 0.2)])
def test_gated_newton_closed_form(ref, beta, r, eta, d0):
    """P7 (section 3, Theorem 5.2's gated-Newton condition beta <d*, k^2> = 1): a repeated
    one-hot key e_i with constant beta gives the scalar recurrence
    d_{t+1} = (r - eta beta^2) d_t + eta beta, solved in closed form; with r = 1 its fixed
    point is exactly 1/beta.  Other coordinates only decay by r."""
    T, Dk, i = 40, 5, 2
    k = np.zeros((1, T, 1, Dk))
    k[0, :, 0, i] = 1.0
    betas = np.full((1, T, 1), beta)
    rs = np.full((1, T, 1), r)
    d0v = np.full((1, 1, Dk), d0)
    kt, dT = ref.precond_scan(k, betas, rs, eta, d0v)
    lam = r - eta * beta * beta
    dstar = eta * beta / (1 - r + eta * beta * beta)
    for t in range(T):
        expect = dstar + (d0 - dstar) * lam ** t  # d_t
        assert abs(kt[0, t, 0, i] - expect) <= 1e-12 * max(1, abs(expect))
    assert abs(dT[0, 0, i] - (dstar + (d0 - dstar) * lam ** T)) <= 1e-12
    others = [j for j in range(Dk) if j != i]
    np.testing.assert_allclose(dT[0, 0, others], d0 * r ** T, rtol=1e-12)
    if r == 1.0:
        assert abs(dstar - 1 / beta) < 1e-15


def test_residual_ratio_closed_form(ref):
    """Section 3 residual ratio: f_t(S_t) / f_t(S_{t-1}) = (1 - beta_t <d_t, k_t^2>)^2 with
    f_t from section 1 and S_t, d_t taken from prefix runs of the oracle."""
    rng = np.random.default_rng(17)
    q, k, v, beta = rand_case(rng, T=12, Dk=6, Dv=4)
    r = rng.uniform(0.7, 1.0, (1, 12, 1))
    S_prev = np.zeros((4, 6))
    d_prev = np.ones(6)
    for t in range(12):
        _, _, St, dt1 = ref.fwd(q[:, :t + 1], k[:, :t + 1], v[:, :t + 1], beta[:, :t + 1],
                                r[:, :t + 1], 0.25)
        kk, vv, bb = k[0, t, 0], v[0, t, 0], beta[0, t, 0]
        ratio = loss(St[0, 0], kk, vv) / loss(S_prev, kk, vv)
        assert abs(ratio - (1 - bb * d_prev @ (kk * kk)) ** 2) < 1e-10
        S_prev, d_prev = St[0, 0], dt1[0, 0]


def test_rho_output_is_the_residual_ratio(ref):
    """The scan's rho output equals f_t(S_t) / f_t(S_{t-1}) built from the oracle's explicit
    states and the section-1 loss, token by token, with APF and several heads."""
    rng = np.random.default_rng(27)
    q, k, v, beta = rand_case(rng, T=9, H=2, Dk=5, Dv=3)
    r = rng.uniform(0.7, 1.0, beta.shape)
    _, _, rho = ref.precond_scan(k, beta, r, 0.3, with_rho=True)
    for h in range(2):
        S_prev = np.zeros((3, 5))
        for t in range(9):
            _, _, St, _ = ref.fwd(q[:, :t + 1], k[:, :t + 1], v[:, :t + 1], beta[:, :t + 1],
                                  r[:, :t + 1], 0.3)
            kk, vv = k[0, t, h], v[0, t, h]
            ratio = loss(St[0, h], kk, vv) / loss(S_prev, kk, vv)
            assert abs(rho[0, t, h] - ratio) < 1e-10
            S_prev = St[0, h]


def test_q_geo_is_the_geometric_mean_of_explicit_loss_ratios(ref):
    """q_geo of a (sequence, head) is the T_n-th root of the product of the token-local ratios
    f_t(S_t) / f_t(S_{t-1}) (section 3, Theorem 5.2's product; the experiments report its
    geometric mean), with the ratios built from the oracle's explicit states and the section-1
    loss, two packed sequences and two heads."""
    rng = np.random.default_rng(28)
    q, k, v, beta = rand_case(rng, T=11, H=2, Dk=5, Dv=3)
    r = rng.uniform(0.7, 1.0, beta.shape)
    cu = np.array([0, 4, 11], dtype=np.int32)
    _, _, rho = ref.precond_scan(k, beta, r, 0.3, cu_seqlens=cu, with_rho=True)
    q_geo = ref.rho_geomean(rho, cu)
    for n in range(2):
        sl = slice(cu[n], cu[n + 1])
        for h in range(2):
            S_prev = np.zeros((3, 5))
            prod, T_n = 1.0, int(cu[n + 1] - cu[n])
            for t in range(T_n):
                a = sl.start
                _, _, St, _ = ref.fwd(q[:, a:a + t + 1], k[:, a:a + t + 1], v[:, a:a + t + 1],
                                      beta[:, a:a + t + 1], r[:, a:a + t + 1], 0.3)
                kk, vv = k[0, a + t, h], v[0, a + t, h]
                prod *= loss(St[0, h], kk, vv) / loss(S_prev, kk, vv)
                S_prev = St[0, h]
            assert abs(q_geo[n, h] - prod ** (1.0 / T_n)) < 1e-12


def test_q_geo_closed_forms(ref):
    """Constant ratios give that constant; 1/4, 1, 4 give 1; a zero ratio gives 0; a sequence
    without tokens gives 1 (the empty product)."""
    rho = np.array([0.3, 0.3, 0.3, 0.25, 1.0, 4.0, 0.5, 0.0, 0.9]).reshape(1, 9, 1)
    cu = np.array([0, 3, 6, 6, 9], dtype=np.int32)
    np.testing.assert_allclose(ref.rho_geomean(rho, cu)[:, 0], [0.3, 1.0, 1.0, 0.0],
                               rtol=1e-14, atol=0)


# ------------------------------------------------------------------------------------ P8
def test_phase1_independent_of_q_v_state(ref):
    """P8 (section 2.2): the surrogate depends only on k, beta (and d), so k~ and d_T do not
    change when q, v or S_0 change."""
    rng = np.random.default_rng(18)
    q, k, v, beta = rand_case(rng, B=2, T=10, H=2, Dk=8, Dv=4)
    r = rng.uniform(0.8, 1.0, beta.shape)
    _, kt1, _, d1 = ref.fwd(q, k, v, beta, r, 0.2)
    q2, _, v2, _ = rand_case(rng, B=2, T=10, H=2, Dk=8, Dv=4)
    S0 = rng.standard_normal((2, 2, 4, 8))
    _, kt2, _, d2 = ref.fwd(q2, k, v2, beta, r, 0.2, None, S0)
    assert np.array_equal(kt1, kt2) and np.array_equal(d1, d2)


# ----------------------------------------------------------------------------- hand example
@pytest.mark.parametrize("case", ["no_apf", "apf_half"])
def test_hand_worked_example(ref, case):
    g = json.load(open(os.path.join(GOLDEN, "hand_two_tokens.json")))
    c = next(c for c in g["cases"] if c["name"] == case)
    inp = g["inputs"]
    k = np.array(inp["k"])[None, :, None, :]
    q = np.array(inp["q"])[None, :, None, :]
    v = np.array(inp["v"])[None, :, None, :]
    beta = np.array(inp["beta"])[None, :, None]
    r = None if c["r"] is None else np.array(c["r"])[None, :, None]
    o, kt, ST, dT = ref.fwd(q, k, v, beta, r, inp["eta"])
    e = c["expected"]
    np.testing.assert_allclose(kt[0, :, 0], e["k_tilde"], atol=1e-14)
    np.testing.assert_allclose(o[0, :, 0], e["o"], atol=1e-14)
    np.testing.assert_allclose(ST[0, 0], e["ST"], atol=1e-14)
    np.testing.assert_allclose(dT[0, 0], e["dT"], atol=1e-14)


# ------------------------------------------------------------------------- layout/structure
def test_heads_batches_and_packing_are_independent(ref):
    """Each (sequence, head) is its own recurrence: a multi-head, multi-batch call equals
    single-head calls on slices; packed input equals separate calls; states are indexed
    [N, H, ...]; the split phase-1 + phase-2 calls equal the one-loop form."""
    rng = np.random.default_rng(19)
    B, T, H, Dk, Dv = 2, 13, 3, 6, 5
    q, k, v, beta = rand_case(rng, B=B, T=T, H=H, Dk=Dk, Dv=Dv)
    r = rng.uniform(0.7, 1.0, (B, T, H))
    S0 = rng.standard_normal((B, H, Dv, Dk))
    d0 = rng.uniform(0.5, 1.5, (B, H, Dk))
    o, kt, ST, dT = ref.fwd(q, k, v, beta, r, 0.15, d0, S0, scale=0.7)
    for b in range(B):
        for h in range(H):
            sl = (slice(b, b + 1), slice(None), slice(h, h + 1))
            o1, kt1, ST1, dT1 = ref.fwd(q[sl], k[sl], v[sl], beta[sl], r[sl], 0.15,
                                        d0[b:b + 1, h:h + 1], S0[b:b + 1, h:h + 1], scale=0.7)
            np.testing.assert_array_equal(o1[0, :, 0], o[b, :, h])
            np.testing.assert_array_equal(ST1[0, 0], ST[b, h])
            np.testing.assert_array_equal(dT1[0, 0], dT[b, h])
    # split phases
    kt2, dT2 = ref.precond_scan(k, beta, r, 0.15, d0)
    o2, ST2 = ref.delta_fwd(q, k, kt2, v, beta, 0.7, S0)
    np.testing.assert_array_equal(kt2, kt)
    np.testing.assert_array_equal(dT2, dT)
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(ST2, ST, rtol=0, atol=1e-13)
    # scale is linear in o only
    o3, _, ST3, _ = ref.fwd(q, k, v, beta, r, 0.15, d0, S0, scale=1.4)
    np.testing.assert_allclose(o3, 2 * o, rtol=1e-13, atol=1e-14)
    np.testing.assert_array_equal(ST3, ST)
    # packing: lengths 5, 0, 8 in one row
    lens = [5, 0, 8]
    cu = np.array([0, 5, 5, 13], dtype=np.int32)
    qp, kp, vp, bp = (a[:1] for a in (q, k, v, beta))
    rp = r[:1]
    S0p = rng.standard_normal((3, H, Dv, Dk))
    d0p = rng.uniform(0.5, 1.5, (3, H, Dk))
    op, ktp, STp, dTp = ref.fwd(qp, kp, vp, bp, rp, 0.15, d0p, S0p, cu_seqlens=cu)
    for n, L in enumerate(lens):
        s = slice(cu[n], cu[n + 1])
        on, ktn, STn, dTn = ref.fwd(qp[:, s], kp[:, s], vp[:, s], bp[:, s], rp[:, s], 0.15,
                                    d0p[n:n + 1], S0p[n:n + 1])
        np.testing.assert_array_equal(op[:, s], on)
        np.testing.assert_array_equal(STp[n], STn[0])
        np.testing.assert_array_equal(dTp[n], dTn[0])
        if L == 0:
            np.testing.assert_array_equal(STp[n], S0p[n])
            np.testing.assert_array_equal(dTp[n], d0p[n])


def test_zero_key_leaves_state_and_only_decays_d(ref):
    """||k||^2 == 0: the write and the gradient vanish (reading: gradient defined as 0)."""
    rng = np.random.default_rng(20)
    S0 = rng.standard_normal((1, 1, 3, 4))
    d0 = rng.uniform(0.5, 1.5, (1, 1, 4))
    k = np.zeros((1, 1, 1, 4))
    q = rng.standard_normal((1, 1, 1, 4))
    v = rng.standard_normal((1, 1, 1, 3))
    o, kt, ST, dT = ref.fwd(q, k, v, np.array([[[0.7]]]), np.array([[[0.9]]]), 0.3, d0, S0)
    np.testing.assert_array_equal(ST, S0)
    np.testing.assert_allclose(dT, 0.9 * d0, rtol=1e-15)
    np.testing.assert_array_equal(kt, np.zeros_like(kt))
