"""The reverse-mode formulation the backward kernels implement (the single-product form with
checkpoints: the dQ recurrence, the per-token reductions, the generation adjoint joining dQ at
the chunk start), written here independently in numpy and checked against the gradient
oracle's reverse mode through the literal five-memory recurrence.  This pins the kernels'
algebra on the CPU; the GPU tests then pin the kernels against the oracle."""
import numpy as np
import pytest

from oracle import srnl_grad as GR
from oracle import srnl_oracle as O


def _gates(ktil, v, a, beta, alpha_max, eps, cap):
    g = O.gates(ktil, v, a, beta, alpha_max, eps, cap)
    return g["k"], g["alpha_t"], g["eta"]


def qform_backward(xs, qs, inits, chunk, alpha_max, eps, dy, cap):
    """dL/dx, dL/dq, dL/dM0 and dL/dG for sum(dy * y), y_t = M0 Q_t q_t, in the kernels' form."""
    S, N, d = xs.shape
    M0 = inits["M_mem"]
    G = np.concatenate([inits["M_k"], inits["M_v"], inits["m_eta"][:, None, :], inits["m_alpha"][:, None, :]], axis=1)
    eye = np.broadcast_to(np.eye(d), (S, d, d))
    chunks = [(c0, min(c0 + chunk, N)) for c0 in range(0, N, chunk)]
    # checkpoint pass: Q at every chunk start
    Q = eye.copy()
    ckpt = []
    for c0, c1 in chunks:
        ckpt.append(Q.copy())
        gen = np.einsum("sgd,std->stg", G, np.einsum("sij,stj->sti", Q, xs[:, c0:c1]))
        k, al, et = _gates(gen[..., :d], gen[..., d:2 * d], gen[..., 2 * d], gen[..., 2 * d + 1], alpha_max, eps, cap)
        for j in range(c1 - c0):
            u = (1 + al[:, j])[:, None] * k[:, j] - gen[:, j, d:2 * d]
            Q = al[:, j, None, None] * Q - et[:, j, None, None] * np.einsum("sij,sj->si", Q, u)[:, :, None] * k[:, j, None, :]
    dxs, dqs = np.zeros_like(xs), np.zeros_like(qs)
    dM0, dG = np.zeros_like(M0), np.zeros_like(G)
    dQ = np.zeros((S, d, d))
    for (c0, c1), Qb in reversed(list(zip(chunks, ckpt))):
        h = np.einsum("sij,stj->sti", Qb, xs[:, c0:c1])                    # w = Q_b x
        gen = np.einsum("sgd,std->stg", G, h)
        kt, vv, a, beta = gen[..., :d], gen[..., d:2 * d], gen[..., 2 * d], gen[..., 2 * d + 1]
        k, al, et = _gates(kt, vv, a, beta, alpha_max, eps, cap)
        states = [Qb]                                                       # in-chunk recompute
        for j in range(c1 - c0):
            u = (1 + al[:, j])[:, None] * k[:, j] - vv[:, j]
            Qp = states[-1]
            states.append(al[:, j, None, None] * Qp - et[:, j, None, None]
                          * np.einsum("sij,sj->si", Qp, u)[:, :, None] * k[:, j, None, :])
        Lc = c1 - c0
        dk_w, dv_w, dal_w, det_w = np.zeros((S, Lc, d)), np.zeros((S, Lc, d)), np.zeros((S, Lc)), np.zeros((S, Lc))
        for j in reversed(range(Lc)):
            t = c0 + j
            Qt, Qm = states[j + 1], states[j]
            a_t = np.einsum("sij,si->sj", M0, dy[:, t])                       # M0^T dy
            dQ = dQ + a_t[:, :, None] * qs[:, t, None, :]                        # readout
            dqs[:, t] = np.einsum("sij,si->sj", Qt, a_t)                         # Q_t^T a
            dM0 += dy[:, t, :, None] * np.einsum("sij,sj->si", Qt, qs[:, t])[:, None, :]
            u = (1 + al[:, j])[:, None] * k[:, j] - vv[:, j]
            w = np.einsum("sij,sj->si", dQ, k[:, j])                             # dQ k
            p = np.einsum("sij,sj->si", Qm, u)                                   # Q_{t-1} u
            dal_T = np.einsum("sij,sij->s", Qm, dQ)
            det = -np.sum(p * w, axis=1)
            du = -et[:, j, None] * np.einsum("sij,si->sj", Qm, w)
            dk = -et[:, j, None] * np.einsum("sij,si->sj", dQ, p)
            dQ = al[:, j, None, None] * dQ - et[:, j, None, None] * w[:, :, None] * u[:, None, :]
            # through u = (1 + alpha) k - v
            dk_w[:, j] = dk + (1 + al[:, j])[:, None] * du
            dv_w[:, j] = -du
            dal_w[:, j] = dal_T + np.sum(k[:, j] * du, axis=1)
            det_w[:, j] = det
        dkt, dvv, da, db = GR.gates_backward(kt, vv, a, beta, alpha_max, eps, cap, dk_w, dv_w, dal_w, det_w)
        dgen = np.concatenate([dkt, dvv, da[..., None], db[..., None]], axis=-1)
        dG += np.einsum("stg,std->sgd", dgen, h)
        dh = np.einsum("sgd,stg->std", G, dgen)                                  # G^T dgen
        dxs[:, c0:c1] = np.einsum("sij,sti->stj", Qb, dh)                        # Q_b^T dh
        dQ = dQ + np.einsum("sti,stj->sij", dh, xs[:, c0:c1])                   # joins at the chunk start
    return dxs, dqs, dM0, dG


@pytest.mark.parametrize("cap", ["soft", "hard"])
@pytest.mark.parametrize("chunk", [1, 3, 7])
def test_kernel_formulation_equals_oracle_gradient(cap, chunk):
    rng = np.random.default_rng(21)
    S, N, d = 3, 17, 4
    xs, qs, dy = rng.normal(0, 1, (S, N, d)), rng.normal(0, 1, (S, N, d)), rng.normal(0, 1, (S, N, d))
    inits = dict(M_mem=rng.normal(0, .3, (S, d, d)), M_k=rng.normal(0, .3, (S, d, d)),
                 M_v=rng.normal(0, .4, (S, d, d)), m_eta=rng.normal(0, .8, (S, d)),
                 m_alpha=rng.normal(0, 1.5, (S, d)))
    dxs, dqs, dM0, dG = qform_backward(xs, qs, inits, chunk, 0.95, 1e-6, dy, cap)
    ref_x, ref_q, ref_init, _ = GR.scan_five_memory_backward(xs, qs, inits, chunk, 0.95, 1e-6, dy, cap=cap)
    np.testing.assert_allclose(dxs, ref_x, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(dqs, ref_q, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(dM0, ref_init["M_mem"], rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(dG[:, :d], ref_init["M_k"], rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(dG[:, d:2 * d], ref_init["M_v"], rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(dG[:, 2 * d], ref_init["m_eta"], rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(dG[:, 2 * d + 1], ref_init["m_alpha"], rtol=1e-9, atol=1e-12)
