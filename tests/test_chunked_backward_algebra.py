"""Chunk-level algebra of the backward pass, checked against the oracle's token-loop gradient.

The GPU backward is to follow the forward's structure: state-free factors for all chunks in
parallel, a short sequential chain across chunks.  This file states that algebra in numpy
(fp64, one (sequence, head) at a time) and checks it against ``oracle.osdn_ref.bwd``, so the
kernels can be written against equations that are already known to be right.

Phase 2 (delta rule with write key K~), per chunk with state S at its start, reversed over chunks:
    A = K K~^T, L = strict_tril(diag(beta) A), T = (I + L)^-1, R = diag(beta) (V - K S^T),
    W = T R, P = tril(Q K~^T), O = scale (Q S^T + P W), S' = S + W^T K~.
    Given dO and dS': dW = K~ dS'^T + scale P^T dO, dP = tril(scale dO W^T),
    dQ = scale dO S + dP K~, dK~ = W dS' + dP^T Q, dR = T^T dW, dT = dW R^T,
    dL = strict_tril(-T^T dT T^T), dbeta += rowsum(dL . A) + rowsum(dR . (V - K S^T)),
    dK += diag(beta) dL K~ - diag(beta) dR S, dK~ += dL^T diag(beta) K, dV = diag(beta) dR,
    dS = dS' + scale dO^T Q - (diag(beta) dR)^T K.
Phase 1 (the preconditioner), reversed: with a = k^2, n = ||k||^2, c = eta beta^2 / n and
d' = r d + g a (g = eta beta (1 - beta s) / n), the adjoint obeys
    dd_t = r_t dd_{t+1} - c_t y_t a_t + e_t,   y_t = <a_t, dd_{t+1}>,   e_t = dk~_t . k_t,
i.e. the transposed step matrix r I - c a a^T, which is symmetric.  Within a chunk of L tokens
ending with adjoint dd_L, with rho_{t,j} = r_t ... r_{j-1}, the y_t solve one upper-triangular
system built from the same Gram A A^T as the forward's chunk solve:
    (I + U) y = b,  U[t][j] = rho_{t+1,j} c_j <a_t, a_j>  (j > t),
    b_t = rho_{t+1,L} <a_t, dd_L> + sum_{j>t} rho_{t+1,j} <a_t, e_j>,
after which every dd_t and the per-token gradients follow without further coupling.
"""
import numpy as np
import pytest

from oracle import osdn_ref


def _phase1_forward(k, beta, r, eta, d0):
    """Token loop: d before each token [T, Dk], k~ [T, Dk], d_T."""
    T, Dk = k.shape
    d = d0.copy()
    ds, kts = np.zeros((T, Dk)), np.zeros((T, Dk))
    for t in range(T):
        a = k[t] ** 2
        n = a.sum()
        s = d @ a
        ds[t], kts[t] = d, d * k[t]
        g = eta * beta[t] * (1 - beta[t] * s) / n if n > 0 else 0.0
        d = r[t] * d + g * a
    return ds, kts, d


def _chunks(T, C):
    return [(c0, min(c0 + C, T)) for c0 in range(0, T, C)]


def _phase2_forward(q, k, kt, v, beta, S0, scale, C):
    """Chunked forward; returns O, the state at every chunk start, and S_T."""
    S = S0.copy()
    O = np.zeros((len(q), v.shape[1]))
    starts = []
    for c0, c1 in _chunks(len(q), C):
        starts.append(S.copy())
        K, Kt, Q, V, b = k[c0:c1], kt[c0:c1], q[c0:c1], v[c0:c1], beta[c0:c1]
        Tm = np.linalg.inv(np.eye(c1 - c0) + np.tril(b[:, None] * (K @ Kt.T), -1))
        W = Tm @ (b[:, None] * (V - K @ S.T))
        O[c0:c1] = scale * (Q @ S.T + np.tril(Q @ Kt.T) @ W)
        S = S + W.T @ Kt
    return O, starts, S


def _phase2_backward(q, k, kt, v, beta, scale, C, starts, dO, dST):
    """The phase-2 equations of the module docstring, chunks in reverse order."""
    dq, dk, dkt, dv = (np.zeros_like(x) for x in (q, k, kt, v))
    dbeta = np.zeros_like(beta)
    dS = dST.copy()
    for (c0, c1), S in reversed(list(zip(_chunks(len(q), C), starts))):
        K, Kt, Q, V, b, G = k[c0:c1], kt[c0:c1], q[c0:c1], v[c0:c1], beta[c0:c1], dO[c0:c1]
        A = K @ Kt.T
        Tm = np.linalg.inv(np.eye(c1 - c0) + np.tril(b[:, None] * A, -1))
        E = V - K @ S.T
        R = b[:, None] * E
        W = Tm @ R
        P = np.tril(Q @ Kt.T)
        dW = Kt @ dS.T + scale * P.T @ G
        dP = np.tril(scale * G @ W.T)
        dq[c0:c1] = scale * G @ S + dP @ Kt
        dkt[c0:c1] = W @ dS + dP.T @ Q
        dR = Tm.T @ dW
        dL = np.tril(-Tm.T @ (dW @ R.T) @ Tm.T, -1)
        dbeta[c0:c1] = (dL * A).sum(1) + (dR * E).sum(1)
        dk[c0:c1] = b[:, None] * (dL @ Kt) - b[:, None] * (dR @ S)
        dkt[c0:c1] += (b[:, None] * dL).T @ K
        dv[c0:c1] = b[:, None] * dR
        dS = dS + scale * G.T @ Q - (b[:, None] * dR).T @ K
    return dq, dk, dkt, dv, dbeta, dS


def _phase1_backward(k, beta, r, eta, ds, dkt, ddT, C):
    """The phase-1 adjoint by one triangular solve per chunk (module docstring)."""
    T, Dk = k.shape
    dk, dbeta, dr = np.zeros_like(k), np.zeros(T), np.zeros(T)
    deta = 0.0
    dd = ddT.copy()
    for c0, c1 in reversed(_chunks(T, C)):
        L = c1 - c0
        a = k[c0:c1] ** 2
        n = a.sum(1)
        ok = n > 0
        nn = np.where(ok, n, 1.0)
        b_ = beta[c0:c1]
        c = np.where(ok, eta * b_ ** 2 / nn, 0.0)
        e = dkt[c0:c1] * k[c0:c1]
        rr = r[c0:c1]
        # rho[t, j] = r_t ... r_{j-1} for j >= t (rho[t, t] = 1); index j = L is the chunk's end
        rho = np.ones((L + 1, L + 1))
        for t in range(L):
            for j in range(t + 1, L + 1):
                rho[t, j] = rho[t, j - 1] * rr[j - 1]
        Gm = a @ a.T
        U = np.zeros((L, L))
        bvec = np.zeros(L)
        for t in range(L):
            bvec[t] = rho[t + 1, L] * (a[t] @ dd)
            for j in range(t + 1, L):
                U[t, j] = rho[t + 1, j] * c[j] * Gm[t, j]
                bvec[t] += rho[t + 1, j] * (a[t] @ e[j])
        y = np.linalg.solve(np.eye(L) + U, bvec)
        f = e - (c * y)[:, None] * a                        # the per-token forcing terms
        # dd_{t+1} for every token of the chunk, and the adjoint at the chunk's start
        dnext = np.zeros((L, Dk))
        for t in range(L):
            dnext[t] = rho[t + 1, L] * dd + sum(rho[t + 1, j] * f[j] for j in range(t + 1, L))
        d_start = rho[0, L] * dd + sum(rho[0, j] * f[j] for j in range(L))
        d = ds[c0:c1]
        s = (d * a).sum(1)
        g = np.where(ok, eta * b_ * (1 - b_ * s) / nn, 0.0)
        dr[c0:c1] = (dnext * d).sum(1)
        dbeta[c0:c1] = np.where(ok, y * eta * (1 - 2 * b_ * s) / nn, 0.0)
        deta += np.where(ok, y * b_ * (1 - b_ * s) / nn, 0.0).sum()
        gs = np.where(ok, -eta * b_ ** 2 / nn, 0.0)
        gn = np.where(ok, -g / nn, 0.0)
        da = g[:, None] * dnext + (gs * y)[:, None] * d + (gn * y)[:, None]
        dk[c0:c1] = dkt[c0:c1] * d + 2 * k[c0:c1] * da
        dd = d_start
    return dk, dbeta, dr, deta, dd


def _chunked_grads(x, C):
    """All gradients of one (sequence, head) by the chunk-level algebra."""
    ds, kts, _ = _phase1_forward(x["k"], x["beta"], x["r"], x["eta"], x["d0"])
    _, starts, _ = _phase2_forward(x["q"], x["k"], kts, x["v"], x["beta"], x["S0"], x["scale"], C)
    dq, dk2, dkt, dv, db2, dS0 = _phase2_backward(x["q"], x["k"], kts, x["v"], x["beta"],
                                                  x["scale"], C, starts, x["dO"], x["dST"])
    dk1, db1, dr, deta, dd0 = _phase1_backward(x["k"], x["beta"], x["r"], x["eta"], ds, dkt,
                                               x["ddT"], C)
    return dict(dq=dq, dk=dk1 + dk2, dv=dv, dbeta=db1 + db2, dr=dr, deta=deta, dS0=dS0, dd0=dd0)


def _problem(seed, T, Dk=6, Dv=5, zero_key=False):
    rng = np.random.default_rng(seed)
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    x = dict(q=unit(rng.standard_normal((T, Dk))), k=unit(rng.standard_normal((T, Dk))),
             v=rng.standard_normal((T, Dv)), beta=1 / (1 + np.exp(-rng.standard_normal(T))),
             r=1 / (1 + np.exp(-(2 + rng.standard_normal(T)))), eta=0.4, scale=0.8,
             d0=rng.uniform(0.5, 1.5, Dk), S0=0.2 * rng.standard_normal((Dv, Dk)),
             dO=rng.standard_normal((T, Dv)), dST=rng.standard_normal((Dv, Dk)),
             ddT=rng.standard_normal(Dk))
    if zero_key:
        x["k"][T // 3] = 0.0
    return x


@pytest.mark.parametrize("T,C,zero_key", [(37, 8, False), (37, 8, True), (40, 16, False), (5, 8, False)])
def test_chunk_algebra_equals_the_oracle_gradient(T, C, zero_key):
    x = _problem(T + C, T, zero_key=zero_key)
    g = _chunked_grads(x, C)
    e4 = lambda a: a[None, :, None]  # [T, ...] -> [B=1, T, H=1, ...]
    want = osdn_ref.bwd(e4(x["q"]), e4(x["k"]), e4(x["v"]), x["beta"][None, :, None], e4(x["dO"]),
                        r=x["r"][None, :, None], eta=x["eta"], d0=x["d0"][None, None],
                        S0=x["S0"][None, None], scale=x["scale"], dST=x["dST"][None, None],
                        ddT=x["ddT"][None, None])
    for name in ("dq", "dk", "dv"):
        np.testing.assert_allclose(g[name], want[name][0, :, 0], rtol=1e-9, atol=1e-10)
    for name in ("dbeta", "dr"):
        np.testing.assert_allclose(g[name], want[name][0, :, 0], rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(g["dS0"], want["dS0"][0, 0], rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(g["dd0"], want["dd0"][0, 0], rtol=1e-9, atol=1e-10)
    assert abs(g["deta"] - want["deta"]) <= 1e-9 * max(1.0, abs(want["deta"]))
