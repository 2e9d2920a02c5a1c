"""Pins for the float64 gradient oracle: every gradient block is checked against central
finite differences of the (separately pinned) forward oracle, the gate backward in each
of its regimes, and two gradients against closed forms that follow from linearity."""
import numpy as np
import pytest

from oracle import srnl_grad as GR
from oracle import srnl_oracle as O
from srnl_inputs import ScanConfig, make_cotangent, make_inputs, make_seq_inputs

FD_H = 1e-6
FD_TOL = 2e-6


# ---------------------------------------------------------------- gates
def _gate_regimes(rng, n=24, d=8):
    """Token batches that put each branch of the gates to work."""
    def base():
        return (rng.normal(0, 0.3, (n, d)), rng.normal(0, 0.3, (n, d)), rng.normal(0, 1, n),
                rng.normal(0, 1, n))
    out = {}
    out["generic"] = base()
    kt, v, a, b = base()
    out["series_step"] = (kt, v, np.full(n, -20.0), b)          # z < 1e-6: phi by its series
    kt, v, a, b = base()
    out["dphi_series"] = (kt, v, np.full(n, -10.0), b)         # 1e-6 <= z < 1e-3
    kt, v, a, b = base()
    out["retention_clamped"] = (kt, v, a, np.full(n, 5.0))      # sigmoid(beta) > alpha
    kt, v, a, b = base()
    khat = kt / np.sqrt(np.sum(kt * kt, axis=1, keepdims=True) + 1e-6)
    out["spectral"] = (kt, khat + rng.normal(0, 1e-4, (n, d)), np.full(n, 4.0), b)   # eta1 |k|^2 > 2
    kt, v, a, b = base()
    out["large_step"] = (kt, v, np.full(n, 3.0) + rng.normal(0, 0.1, n), b)         # cap saturates
    return out


def _gate_outputs(ktil, v, a, beta, cap):
    g = O.gates(ktil, v, a, beta, 0.95, 1e-6, cap)
    return {"k": g["k"], "alpha": g["alpha_t"], "eta": g["eta"], "v": v}


@pytest.mark.parametrize("cap", ["soft", "hard"])
def test_gate_backward_matches_finite_differences(cap):
    rng = np.random.default_rng(11)
    for regime, (kt, v, a, b) in _gate_regimes(rng).items():
        outs = _gate_outputs(kt, v, a, b, cap)
        if regime == "spectral":
            eta1 = O.gates(kt, v, a, b, 0.95, 1e-6, cap)["eta1"]
            assert np.all(eta1 * np.sum(outs["k"] ** 2, axis=1) > 2.0)
        if regime == "retention_clamped":
            assert np.all(outs["alpha"] == 0.95)
        for which in ("k", "alpha", "eta", "v"):
            w = rng.normal(0, 1, outs[which].shape)
            up = {"dk": np.zeros_like(kt), "dv": np.zeros_like(v), "dalpha": np.zeros(len(a)),
                  "deta": np.zeros(len(a))}
            up[{"k": "dk", "alpha": "dalpha", "eta": "deta", "v": "dv"}[which]] = w
            got = GR.gates_backward(kt, v, a, b, 0.95, 1e-6, cap, **up)
            for blk, (inp, g) in enumerate(zip((kt, v, a, b), got)):
                # per-token derivatives: perturb every token's input along V at once
                V = rng.normal(0, 1, inp.shape)
                h = 1e-6
                args_p = [kt, v, a, b]
                args_m = [kt, v, a, b]
                args_p[blk] = inp + h * V
                args_m[blk] = inp - h * V
                op = _gate_outputs(*args_p, cap)[which]
                fp = np.sum(w * op)
                fm = np.sum(w * _gate_outputs(*args_m, cap)[which])
                fd = (fp - fm) / (2 * h)
                an = np.sum(g * V)
                scale = np.sqrt(np.sum((g * V) ** 2)) + np.abs(an)
                # rounding floor of the difference quotient: each output carries ~eps relative error
                noise = 8 * np.finfo(np.float64).eps * np.sum(np.abs(w * op)) / h
                assert abs(fd - an) <= 1e-6 * scale + noise + 1e-13, (cap, regime, which, blk, fd, an)


def test_gate_backward_regimes_are_reached():
    rng = np.random.default_rng(11)
    reg = _gate_regimes(rng)
    kt, v, a, b = reg["series_step"]
    g = O.gates(kt, v, a, b, 0.95, 1e-6)
    assert np.all(g["eta0"] * g["gain"] / (1 - g["alpha_t"]) < 1e-6)
    kt, v, a, b = reg["dphi_series"]
    g = O.gates(kt, v, a, b, 0.95, 1e-6)
    z = g["eta0"] * g["gain"] / (1 - g["alpha_t"])
    assert np.all((z >= 1e-6) & (z < 1e-3))
    kt, v, a, b = reg["large_step"]
    g = O.gates(kt, v, a, b, 0.95, 1e-6, "hard")
    assert np.all(g["binds"])


# ---------------------------------------------------------------- operator
def _small_cfg(**kw):
    base = dict(name="fd", B=2, H=3, W=5, C=8, heads=2, d=4, alpha=0.95, chunk_row=2, chunk_col=2,
                act_dtype="f32")
    base.update(kw)
    return ScanConfig(**base)


def _op_loss(cfg, x, params, dout, cap):
    out, _, _ = O.operator_forward(x, params, alpha_max=cfg.alpha, eps=cfg.eps, chunk_row=cfg.chunk_row,
                                   chunk_col=cfg.chunk_col, heads=cfg.heads, cap=cap)
    return float(np.sum(dout * out))


def _directional_check(loss, base, grad, rng, key, h=FD_H):
    V = rng.normal(0, 1, np.shape(base[key]))
    rms = float(np.sqrt(np.mean(np.asarray(base[key], np.float64) ** 2))) or 1.0
    V *= rms
    plus = dict(base)
    minus = dict(base)
    plus[key] = np.asarray(base[key], np.float64) + h * V
    minus[key] = np.asarray(base[key], np.float64) - h * V
    fd = (loss(plus) - loss(minus)) / (2 * h)
    an = float(np.sum(grad * V))
    return fd, an


@pytest.mark.parametrize("cap", ["soft", "hard"])
@pytest.mark.parametrize("mem_scale", [0.02, 0.3])
def test_operator_backward_matches_finite_differences(cap, mem_scale):
    cfg = _small_cfg()
    inp = make_inputs(cfg, seed=3, mem_scale=mem_scale, vec_scale=0.8)
    params = {k: np.asarray(v, np.float64) for k, v in inp.params().items()}
    x = inp.x32.astype(np.float64)
    dout = make_cotangent(x.shape, seed=3).astype(np.float64)
    grads = GR.operator_backward(x, params, dout, alpha_max=cfg.alpha, eps=cfg.eps,
                                 chunk_row=cfg.chunk_row, chunk_col=cfg.chunk_col, heads=cfg.heads, cap=cap)
    rng = np.random.default_rng(5)
    base = dict(params, x=x)

    def loss(state):
        p = {k: state[k] for k in params}
        return _op_loss(cfg, state["x"], p, dout, cap)

    for key in ("x",) + GR.PARAM_KEYS:
        for _ in range(2):
            fd, an = _directional_check(loss, base, grads[key], rng, key)
            assert abs(fd - an) <= FD_TOL * max(abs(an), 1e-3), (cap, key, fd, an)


def test_hard_clamp_is_active_in_the_finite_difference_case():
    cfg = _small_cfg()
    inp = make_inputs(cfg, seed=3, mem_scale=0.3, vec_scale=0.8)
    counter = [0]
    O.operator_forward(inp.x32, inp.params(), alpha_max=cfg.alpha, chunk_row=2, chunk_col=2,
                       heads=cfg.heads, cap="hard", counter=counter)
    assert 0 < counter[0] < 4 * cfg.B * cfg.heads * cfg.N


def test_scale_gradient_is_the_one_hot_route_output():
    """The output is linear in the fusion scales: ds_r[c] = sum dout[..., c] * (the output
    with scales one on route r and zero elsewhere)[..., c]."""
    cfg = _small_cfg()
    inp = make_inputs(cfg, seed=4, mem_scale=0.3, vec_scale=0.8)
    params = inp.params()
    dout = make_cotangent(inp.x32.shape, seed=4).astype(np.float64)
    grads = GR.backward_from_inputs(inp, dout)
    for r in range(4):
        onehot = dict(params, scales=np.eye(4)[r][:, None] * np.ones((4, cfg.C)))
        out, _, _ = O.operator_forward(inp.x32, onehot, alpha_max=cfg.alpha, chunk_row=2, chunk_col=2,
                                       heads=cfg.heads)
        expect = np.einsum("bhwc,bhwc->c", dout, out)
        np.testing.assert_allclose(grads["scales"][r], expect, rtol=1e-12, atol=1e-14)


def test_query_projection_gradient_is_exact_difference():
    """The output is linear in W_q, so f(W_q + V) - f(W_q) = <dW_q, V> for any V."""
    cfg = _small_cfg()
    inp = make_inputs(cfg, seed=6, mem_scale=0.3, vec_scale=0.8)
    params = {k: np.asarray(v, np.float64) for k, v in inp.params().items()}
    dout = make_cotangent(inp.x32.shape, seed=6).astype(np.float64)
    grads = GR.backward_from_inputs(inp, dout)
    V = np.random.default_rng(1).normal(0, 1, params["W_q"].shape)
    f0 = _op_loss(cfg, inp.x32, params, dout, "soft")
    f1 = _op_loss(cfg, inp.x32, dict(params, W_q=params["W_q"] + V), dout, "soft")
    np.testing.assert_allclose(f1 - f0, np.sum(grads["W_q"] * V), rtol=1e-10)


def test_backward_forward_outputs_match_forward_oracle():
    """The backward's recomputed route outputs are the forward's."""
    rng = np.random.default_rng(8)
    S, N, d = 3, 11, 4
    xs, qs = rng.normal(0, 1, (S, N, d)), rng.normal(0, 1, (S, N, d))
    inits = dict(M_mem=rng.normal(0, .3, (S, d, d)), M_k=rng.normal(0, .3, (S, d, d)),
                 M_v=rng.normal(0, .4, (S, d, d)), m_eta=rng.normal(0, .8, (S, d)),
                 m_alpha=rng.normal(0, 1.5, (S, d)))
    y, _, _ = O.scan_five_memory(xs, qs, inits, 4, 0.95, 1e-6)
    _, _, _, y2 = GR.scan_five_memory_backward(xs, qs, inits, 4, 0.95, 1e-6, np.ones((S, N, d)))
    np.testing.assert_allclose(y2, y, rtol=0, atol=1e-15)


# ---------------------------------------------------------------- sequence layer
@pytest.mark.parametrize("with_queries", [False, True])
@pytest.mark.parametrize("cap", ["soft", "hard"])
def test_sequence_backward_matches_finite_differences(with_queries, cap):
    si = make_seq_inputs(2, 13, 8, 2, seed=2, mem_scale=0.3, vec_scale=0.8)
    params = {k: np.asarray(v, np.float64) for k, v in si.params().items()}
    x = si.x32.astype(np.float64)
    q = si.q32.astype(np.float64) if with_queries else None
    dy = make_cotangent(x.shape, seed=2).astype(np.float64)
    grads = GR.sequence_backward(x, params, dy, alpha_max=0.95, chunk=5, heads=2, queries=q, cap=cap)
    rng = np.random.default_rng(9)
    base = dict(params, x=x)
    if with_queries:
        base["queries"] = q

    def loss(state):
        p = {k: state[k] for k in params}
        y, _ = O.sequence_forward(state["x"], p, alpha_max=0.95, chunk=5, heads=2,
                                  queries=state.get("queries"), cap=cap)
        return float(np.sum(dy * y))

    keys = ["x", "M_mem0", "M_k0", "M_v0", "m_eta0", "m_alpha0"] + (["queries"] if with_queries else [])
    for key in keys:
        fd, an = _directional_check(loss, base, grads[key], rng, key)
        assert abs(fd - an) <= FD_TOL * max(abs(an), 1e-3), (key, fd, an)


def test_sequence_backward_is_route_zero_of_the_operator():
    """The sequence layer is route 0 of the operator on a 1 x T map with W_q = I and scales one on
    route 0, zero elsewhere (the forward pin); so are its gradients: dx (including the query
    path) and the initial-state gradients equal the operator's route-0 gradients, and the other
    routes' initial states get none."""
    B, T, D, heads = 2, 11, 8, 2
    d = D // heads
    rng = np.random.default_rng(31)
    x = rng.normal(0, 1, (B, T, D))
    dy = rng.normal(0, 1, (B, T, D))
    seq_p = {"M_mem0": rng.normal(0, .3, (heads, d, d)), "M_k0": rng.normal(0, .3, (heads, d, d)),
             "M_v0": rng.normal(0, .4, (heads, d, d)), "m_eta0": rng.normal(0, .8, (heads, d)),
             "m_alpha0": rng.normal(0, 1.5, (heads, d))}
    op_p = {k: np.concatenate([v[None], 0.5 * np.ones((3,) + v.shape)], axis=0) for k, v in seq_p.items()}
    op_p["W_q"] = np.eye(D)
    op_p["scales"] = np.concatenate([np.ones((1, D)), np.zeros((3, D))], axis=0)
    gs = GR.sequence_backward(x, seq_p, dy, alpha_max=0.95, chunk=4, heads=heads)
    go = GR.operator_backward(x[:, None], op_p, dy[:, None], alpha_max=0.95, chunk_row=4, heads=heads)
    np.testing.assert_allclose(go["x"][:, 0], gs["x"], rtol=1e-12, atol=1e-14)
    for key in ("M_mem0", "M_k0", "M_v0", "m_eta0", "m_alpha0"):
        np.testing.assert_allclose(go[key][0], gs[key], rtol=1e-12, atol=1e-14)
        assert np.all(go[key][1:] == 0.0), key
