"""The reverse mode of one stage of the write (tokens sharing one boundary, gates fixed) in
chunkwise form: every quantity the token-by-token reverse recurrence produces (the carried
gradient dQ_s, w_t = dQ_t k_t, and the token gradients of alpha_t, eta_t, u_t, k_t and q_t) from
two shared triangular solves and T x T, T x d and d x d products only, which is the form a
tensor-core backward takes.  Checked against the token recurrence in float64, including
retentions down to 1e-12.

Notation (one stage of T tokens, boundary state Q_s, d x d): c_t = prod_{m <= t} alpha_m,
g(j, t) = c_t / c_j (<= 1), s_t = Q_{t-1} u_t (forward), a_t = M0^T dy_t (readout
gradient), dQ_e = dL/dQ after the stage.  The reverse carried gradient X_t = dL/dQ_t is
  X_t = g(t, T-1) dQ_e + sum_{m >= t} g(t, m) a_m q_m^T - sum_{m > t} g(t, m-1) eta_m w_m u_m^T,
so w_t = X_t k_t solves the upper-triangular system
  w_t + sum_{m > t} g(t, m-1) eta_m (u_m . k_t) w_m = g(t, T-1) dQ_e k_t + sum_{m >= t} g(t, m) (q_m . k_t) a_m,
shared by all rows, as the forward's s_t solve a lower-triangular one."""
import numpy as np
import pytest
from scipy.linalg import solve_triangular


def token_reverse(Qs, k, u, q, al, et, a, dQe):
    """Reference: the token recurrence (what the SIMT backward kernels do)."""
    T, d = k.shape
    states = [Qs]
    for t in range(T):
        Qp = states[-1]
        states.append(al[t] * Qp - et[t] * np.outer(Qp @ u[t], k[t]))
    X = dQe.copy()
    out = {key: np.zeros((T, d)) for key in ("w", "du", "dk", "dq", "z")}
    out["dal"], out["deta"] = np.zeros(T), np.zeros(T)
    for t in reversed(range(T)):
        Qt, Qm = states[t + 1], states[t]
        X = X + np.outer(a[t], q[t])
        out["z"][t] = Qt @ q[t]
        out["dq"][t] = Qt.T @ a[t]
        w = X @ k[t]
        p = Qm @ u[t]
        out["w"][t] = w
        out["dal"][t] = np.sum(Qm * X)
        out["deta"][t] = -p @ w
        out["du"][t] = -et[t] * (Qm.T @ w)
        out["dk"][t] = -et[t] * (X.T @ p)
        X = al[t] * X - et[t] * np.outer(w, u[t])
    out["dQs"] = X
    out["Qe"] = states[-1]
    return out


def chunkwise_reverse(Qs, k, u, q, al, et, a, dQe):
    """The same quantities from triangular solves and products (no token loop over states)."""
    T, d = k.shape
    lam = np.cumsum(np.log2(al))                       # log2 c_t
    c = np.exp2(lam)
    cm1 = np.concatenate([[1.0], c[:-1]])              # c_{t-1}
    tt = np.arange(T)

    def gmat(shift):   # G[t][j] = g(j, t - shift) for j <= t - shift, else 0
        e = lam[np.clip(tt - shift, 0, None)][:, None] - lam[None, :]
        ok = (tt[None, :] <= (tt - shift)[:, None]) & ((tt - shift)[:, None] >= 0)
        full = np.where(ok, np.exp2(np.where(ok, e, 0.0)), 0.0)
        if shift == 1:   # t - 1 = -1 for t = 0: g(j, -1) has no j
            full[0] = 0.0
        return full

    g0 = gmat(0)                                       # [t][j] = g(j, t), j <= t
    g1 = gmat(1)                                       # [t][j] = g(j, t-1), j < t
    # forward: lower-triangular solve for S, then z and Q_e
    A = g1 * et[None, :] * (u @ k.T)                   # A[t][j] = g(j,t-1) eta_j (u_t . k_j)
    S = solve_triangular(np.eye(T) + A, cm1[:, None] * (u @ Qs.T), lower=True)   # rows s_t
    Z = c[:, None] * (q @ Qs.T) - (g0 * et[None, :] * (q @ k.T)) @ S
    gT = np.exp2(lam[-1] - lam)                        # g(t, T-1)
    Qe = c[-1] * Qs - (S * (gT * et)[:, None]).T @ k
    # reverse: upper-triangular solve for W (rows w_t)
    g0T, g1T = g0.T, g1.T                              # [t][m] = g(t, m) (m >= t), g(t, m-1) (m > t)
    Ahat = g1T * et[None, :] * (k @ u.T)               # [t][m] = g(t,m-1) eta_m (k_t . u_m)
    R = gT[:, None] * (k @ dQe.T) + (g0T * (k @ q.T)) @ a
    W = solve_triangular(np.eye(T) + Ahat, R, lower=False)
    deta = -np.sum(S * W, axis=1)
    # du_t = -eta_t (c_{t-1} Q_s^T w_t - sum_{j<t} g(j,t-1) eta_j (s_j . w_t) k_j)
    du = -et[:, None] * (cm1[:, None] * (W @ Qs) - (g1 * et[None, :] * (W @ S.T)) @ k)
    # dk_t = -eta_t (g(t,T-1) dQ_e^T s_t + sum_{m>=t} g(t,m) (a_m . s_t) q_m
    #                - sum_{m>t} g(t,m-1) eta_m (w_m . s_t) u_m)
    dk = -et[:, None] * (gT[:, None] * (S @ dQe) + (g0T * (S @ a.T)) @ q
                         - (g1T * et[None, :] * (S @ W.T)) @ u)
    # dq_t = c_t Q_s^T a_t - sum_{j<=t} g(j,t) eta_j (s_j . a_t) k_j
    dq = c[:, None] * (a @ Qs) - (g0 * et[None, :] * (a @ S.T)) @ k
    # dalpha_t = <Q_{t-1}, X_t>, with Q_{t-1} = c_{t-1} Q_s - sum_{j<t} g(j,t-1) eta_j s_j k_j^T
    QsdQe = np.sum(Qs * dQe)
    aQq = np.einsum("md,de,me->m", a, Qs, q)           # a_m^T Q_s q_m
    wQu = np.einsum("md,de,me->m", W, Qs, u)           # w_m^T Q_s u_m
    sdk = np.einsum("jd,de,je->j", S, dQe, k)          # s_j^T dQ_e k_j
    SA, KQ, SWm, KU = S @ a.T, k @ q.T, S @ W.T, k @ u.T
    dal = (cm1 * gT * QsdQe + cm1 * (g0T @ aQq) - cm1 * ((g1T * et[None, :]) @ wQu)
           - (g1 * et[None, :]) @ sdk * gT)
    # the double sums over j < t <= m (and m > t) as diagonals of T x T x T products
    left = g1 * et[None, :]                            # [t][j] = g(j,t-1) eta_j, j < t
    dal -= np.einsum("tj,jm,tm->t", left, SA * KQ, g0T)
    dal += np.einsum("tj,jm,tm->t", left, SWm * KU, g1T * et[None, :])
    dQs = c[-1] * dQe + (a * c[:, None]).T @ q - (W * (cm1 * et)[:, None]).T @ u
    return {"w": W, "du": du, "dk": dk, "dq": dq, "z": Z, "dal": dal, "deta": deta, "dQs": dQs, "Qe": Qe}


@pytest.mark.parametrize("T", [1, 2, 7, 23])
@pytest.mark.parametrize("retention", ["typical", "tiny"])
def test_chunkwise_stage_reverse_equals_token_recurrence(T, retention):
    rng = np.random.default_rng(40 + T)
    d = 6
    Qs = rng.normal(0, 1, (d, d))
    k = rng.normal(0, 1, (T, d))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    u = rng.normal(0, 1, (T, d))
    q = rng.normal(0, 1, (T, d))
    a = rng.normal(0, 1, (T, d))
    dQe = rng.normal(0, 1, (d, d))
    al = rng.uniform(0.3, 0.95, T)
    if retention == "tiny":
        al[::3] = 1e-12
    et = rng.uniform(0.05, 0.9, T)
    ref = token_reverse(Qs, k, u, q, al, et, a, dQe)
    got = chunkwise_reverse(Qs, k, u, q, al, et, a, dQe)
    for key in ("Qe", "z", "w", "deta", "du", "dk", "dq", "dal", "dQs"):
        scale = max(np.max(np.abs(ref[key])), 1e-300)
        np.testing.assert_allclose(got[key], ref[key], rtol=1e-9, atol=1e-10 * scale, err_msg=key)


def test_chunkwise_scan_backward_equals_oracle():
    """The whole scan's backward assembled from the chunkwise stage reverse: per chunk in
    reverse, the stage reverse above, then the gate backward, the generation adjoint and the
    boundary gradient joining the carried dQ; against the gradient oracle."""
    from oracle import srnl_grad as GR
    from oracle import srnl_oracle as O

    rng = np.random.default_rng(52)
    S_, N, d, chunk = 2, 19, 4, 6
    xs, qs, dy = rng.normal(0, 1, (S_, N, d)), rng.normal(0, 1, (S_, N, d)), rng.normal(0, 1, (S_, N, d))
    inits = dict(M_mem=rng.normal(0, .3, (S_, d, d)), M_k=rng.normal(0, .3, (S_, d, d)),
                 M_v=rng.normal(0, .4, (S_, d, d)), m_eta=rng.normal(0, .8, (S_, d)),
                 m_alpha=rng.normal(0, 1.5, (S_, d)))
    ref_x, ref_q, ref_init, _ = GR.scan_five_memory_backward(xs, qs, inits, chunk, 0.95, 1e-6, dy)
    for s in range(S_):
        M0 = inits["M_mem"][s]
        G = np.concatenate([inits["M_k"][s], inits["M_v"][s], inits["m_eta"][s][None], inits["m_alpha"][s][None]])
        bounds = list(range(0, N, chunk))
        Q, ckpt = np.eye(d), []
        for c0 in bounds:                                   # checkpoint pass (token loop is fine here)
            c1 = min(c0 + chunk, N)
            ckpt.append(Q.copy())
            gen = (G @ (Q @ xs[s, c0:c1].T)).T
            gt = O.gates(gen[:, :d], gen[:, d:2 * d], gen[:, 2 * d], gen[:, 2 * d + 1], 0.95, 1e-6)
            for j in range(c1 - c0):
                u = (1 + gt["alpha_t"][j]) * gt["k"][j] - gen[j, d:2 * d]
                Q = gt["alpha_t"][j] * Q - gt["eta"][j] * np.outer(Q @ u, gt["k"][j])
        dQ = np.zeros((d, d))
        dx, dq = np.zeros((N, d)), np.zeros((N, d))
        dM0, dG = np.zeros((d, d)), np.zeros_like(G)
        for c0, Qb in reversed(list(zip(bounds, ckpt))):
            c1 = min(c0 + chunk, N)
            X = xs[s, c0:c1]
            h = (Qb @ X.T).T
            gen = h @ G.T
            kt, vv, av, bv = gen[:, :d], gen[:, d:2 * d], gen[:, 2 * d], gen[:, 2 * d + 1]
            gt = O.gates(kt, vv, av, bv, 0.95, 1e-6)
            k, al, et = gt["k"], gt["alpha_t"], gt["eta"]
            u = (1 + al)[:, None] * k - vv
            a = dy[s, c0:c1] @ M0                            # a_t = M0^T dy_t
            st = chunkwise_reverse(Qb, k, u, qs[s, c0:c1], al, et, a, dQ)
            dq[c0:c1] = st["dq"]
            dM0 += dy[s, c0:c1].T @ st["z"]
            # through u = (1 + alpha) k - v
            dk_w = st["dk"] + (1 + al)[:, None] * st["du"]
            dal_w = st["dal"] + np.sum(k * st["du"], axis=1)
            dkt, dvv, da, db = GR.gates_backward(kt, vv, av, bv, 0.95, 1e-6, "soft", dk_w, -st["du"], dal_w,
                                                 st["deta"])
            dgen = np.concatenate([dkt, dvv, da[:, None], db[:, None]], axis=1)
            dG += dgen.T @ h
            dh = dgen @ G
            dx[c0:c1] = dh @ Qb
            dQ = st["dQs"] + dh.T @ X                        # the boundary joins the carried gradient
        np.testing.assert_allclose(dx, ref_x[s], rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(dq, ref_q[s], rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(dM0, ref_init["M_mem"][s], rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(dG[:d], ref_init["M_k"][s], rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(dG[d:2 * d], ref_init["M_v"][s], rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(dG[2 * d], ref_init["m_eta"][s], rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(dG[2 * d + 1], ref_init["m_alpha"][s], rtol=1e-9, atol=1e-12)
