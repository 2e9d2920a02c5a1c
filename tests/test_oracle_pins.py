"""Pins for the float64 oracle: each test checks it against something the pages
or the mathematics fix, not against a retyped copy of its own formulas."""
import json
import os

import numpy as np
import pytest
import torch

from oracle import srnl_oracle as O
from srnl_inputs import CONFIGS, ScanConfig, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_inits(rng, S, d, mem=0.02, vec=0.1):
    return dict(M_mem=rng.normal(0, mem, (S, d, d)), M_k=rng.normal(0, mem, (S, d, d)),
                M_v=rng.normal(0, mem, (S, d, d)), m_eta=rng.normal(0, vec, (S, d)),
                m_alpha=rng.normal(0, vec, (S, d)))


def _active_inits(rng, S, d):
    """Initial memories large enough that keys, caps and clamps all do work."""
    return dict(M_mem=rng.normal(0, 0.3, (S, d, d)), M_k=rng.normal(0, 0.3, (S, d, d)),
                M_v=rng.normal(0, 0.4, (S, d, d)), m_eta=rng.normal(0, 0.8, (S, d)),
                m_alpha=rng.normal(0, 1.5, (S, d)))


# ---------------------------------------------------------------- routes
@pytest.mark.parametrize("H,W", [(1, 1), (1, 5), (5, 1), (2, 3), (3, 2), (8, 8), (14, 20), (7, 13)])
def test_route_maps_are_permutations(H, W):
    for r in range(4):
        p = O.route_index_map(H, W, r)
        assert p.dtype == np.int64
        assert np.array_equal(np.sort(p), np.arange(H * W))


def test_route_maps_match_hand_written_2x3():
    rows = {}
    with open(os.path.join(GOLDEN, "routes_2x3.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            r, vals = line.split(":")
            rows[int(r)] = [int(v) for v in vals.split()]
    for r in range(4):
        assert O.route_index_map(2, 3, r).tolist() == rows[r]


def test_chunks_follow_rows_and_columns_14x20():
    g = json.load(open(os.path.join(GOLDEN, "chunks_14x20.json")))
    H, W = g["H"], g["W"]
    for r in range(4):
        L = O.default_chunk(H, W, r)
        assert L == (g["row_route_chunk"] if r < 2 else g["col_route_chunk"])
        p = O.route_index_map(H, W, r)
        for c0 in range(0, H * W, L):
            ii, jj = np.divmod(p[c0:c0 + L], W)
            if r < 2:   # one full image row per chunk
                assert len(set(ii.tolist())) == 1 and sorted(jj.tolist()) == list(range(W))
            else:       # one full image column per chunk
                assert len(set(jj.tolist())) == 1 and sorted(ii.tolist()) == list(range(H))


def test_readme_example_shape_preserved():
    g = json.load(open(os.path.join(GOLDEN, "chunks_14x20.json")))
    B, C, H, W = g["readme_example_shape_bchw"]
    heads = C // g["readme_example_head_dim"]
    cfg = ScanConfig("readme", B=B, H=H, W=W, C=C, heads=heads, d=C // heads, alpha=0.95, act_dtype="f32")
    inp = make_inputs(cfg, seed=3)
    out, fin, _ = O.forward_from_inputs(inp)
    assert out.shape == (B, H, W, C)
    assert fin.shape == (4, B, heads, 3 * 16 * 16 + 2 * 16)
    assert np.all(np.isfinite(out))


@pytest.mark.parametrize("H,W", [(2, 3), (5, 7), (8, 8)])
def test_gather_restore_roundtrip_bitwise(H, W):
    x = np.random.default_rng(0).standard_normal((2, H, W, 5))
    for r in range(4):
        assert np.array_equal(O.restore(O.gather(x, r), r, H, W), x)


# ---------------------------------------------------------------- gates
def test_stabilized_key_closed_form():
    rng = np.random.default_rng(1)
    for scale in (1e-6, 1e-3, 1.0, 30.0):
        kt = rng.standard_normal((50, 32)) * scale
        eps = 1e-6
        n = np.sum(kt ** 2, axis=1)
        k = O.stabilized_key(kt, eps)
        np.testing.assert_allclose(np.sum(k ** 2, axis=1), n / (n + eps), rtol=1e-13)
        # direction is preserved
        np.testing.assert_allclose(k * np.sqrt(n + eps)[:, None], kt, rtol=1e-13, atol=0)


def test_soft_cap_limits():
    rng = np.random.default_rng(2)
    eta0 = np.abs(rng.standard_normal(10000)) * 5
    g = np.abs(rng.standard_normal(10000)) * 3
    al = rng.uniform(0.0, 0.999, 10000)
    e1 = O.soft_cap(eta0, g, al)
    z = eta0 * g / (1.0 - al)
    assert np.all(e1 * g <= (1.0 - al) * (1 + 1e-14))   # inside the margin (to rounding) ...
    unsat = z < 15.0                            # ... strictly, until tanh rounds to 1.0
    assert np.all(e1[unsat] * g[unsat] < 1.0 - al[unsat])
    assert np.all(e1 <= eta0 * (1 + 1e-15))     # never raises the step
    # small steps pass nearly unchanged (smooth, no clipping): relative change ~ z^2/3
    tiny = O.soft_cap(np.full(5, 1e-5), np.full(5, 1e-3), np.full(5, 0.5))
    np.testing.assert_allclose(tiny, 1e-5, rtol=1e-15)
    # saturation: the executed injection tends to the margin
    big = O.soft_cap(np.array([1e6]), np.array([1.0]), np.array([0.9]))
    np.testing.assert_allclose(big * 1.0, 0.1, rtol=1e-12)


def test_sigmoid_closed_forms():
    """The logistic function: sigma(0) = 1/2, sigma(ln 3) = 3/4, sigma(-z) = 1 - sigma(z), and its
    asymptotes (1 - e^-z above, e^z below), without overflow at |z| = 800."""
    z = np.array([0.0, np.log(3.0), -np.log(3.0), np.log(99.0)])
    np.testing.assert_allclose(O.sigmoid(z), [0.5, 0.75, 0.25, 0.99], rtol=1e-15)
    rng = np.random.default_rng(31)
    w = rng.normal(0, 6, 1000)
    np.testing.assert_allclose(O.sigmoid(-w), 1.0 - O.sigmoid(w), atol=1e-15)
    np.testing.assert_allclose(O.sigmoid(np.array([40.0, -40.0])), [1.0 - np.exp(-40.0), np.exp(-40.0)],
                               rtol=1e-14)
    with np.errstate(over="raise"):
        big = O.sigmoid(np.array([800.0, -800.0]))
    assert big[0] == 1.0 and 0.0 <= big[1] < 1e-300


def test_softplus_closed_forms():
    """softplus(z) = log(1 + e^z): softplus(0) = ln 2, softplus(ln(e - 1)) = 1,
    softplus(z) - softplus(-z) = z, and softplus(z) -> z above, e^z below."""
    np.testing.assert_allclose(O.softplus(np.array([0.0, np.log(np.e - 1.0)])), [np.log(2.0), 1.0], rtol=1e-15)
    rng = np.random.default_rng(32)
    w = rng.normal(0, 8, 1000)
    np.testing.assert_allclose(O.softplus(w) - O.softplus(-w), w, atol=1e-13)
    np.testing.assert_allclose(O.softplus(np.array([50.0, -50.0])), [50.0, np.exp(-50.0)], rtol=1e-15)


def test_retention_clamp_values():
    """alpha_t = min(sigmoid(beta), alpha): below the cap it is the logistic of beta, above it the cap."""
    beta = np.array([np.log(3.0), -np.log(3.0), np.log(99.0), 0.0])
    np.testing.assert_allclose(O.retention(beta, 0.95), [0.75, 0.25, 0.95, 0.5], rtol=1e-15)


def test_gates_hand_computed_token():
    """One token worked by hand (d = 2, eps = 0): k~ = (3, 4), v = 0, a = 0, beta = ln 3.
    k = (3, 4) / 5; alpha_t = sigmoid(ln 3) = 3/4; eta0 = softplus(0) = ln 2; gain
    g = ||k - v|| ||k|| = 1; the soft cap's z = eta0 g / (1 - alpha_t) = 4 ln 2, and
    tanh(4 ln 2) = (16 - 1/16) / (16 + 1/16) = 255/257, so eta1 = eta0 tanh(z) / z = 255/1028;
    the spectral clamp (eta ||k||^2 <= 2) leaves it."""
    gt = O.gates(np.array([[3.0, 4.0]]), np.zeros((1, 2)), np.array([0.0]), np.array([np.log(3.0)]),
                 0.95, 0.0)
    np.testing.assert_allclose(gt["k"], [[0.6, 0.8]], rtol=1e-15)
    np.testing.assert_allclose(gt["alpha_t"], [0.75], rtol=1e-15)
    np.testing.assert_allclose(gt["eta0"], [np.log(2.0)], rtol=1e-15)
    np.testing.assert_allclose(gt["gain"], [1.0], rtol=1e-15)
    np.testing.assert_allclose(gt["eta"], [255.0 / 1028.0], rtol=1e-14)
    # a value that is not a rescaled key: v = (0, 1) gives ||k - v|| = sqrt(0.36 + 0.04)
    gt = O.gates(np.array([[3.0, 4.0]]), np.array([[0.0, 1.0]]), np.array([0.0]), np.array([np.log(3.0)]),
                 0.95, 0.0)
    np.testing.assert_allclose(gt["gain"], [np.sqrt(0.4)], rtol=1e-15)


def test_query_projection_orientation_hand_computed():
    """q = x W_q^T with W_q[o][c] (output channel o, input channel c): x = (1, 10) and
    W_q = [[1, 2], [3, 4]] give q = (1 + 20, 3 + 40) = (21, 43)."""
    x = np.array([1.0, 10.0]).reshape(1, 1, 1, 2)
    q = O.query_projection(x, np.array([[1.0, 2.0], [3.0, 4.0]]))
    assert q.shape == (1, 1, 1, 2)
    np.testing.assert_array_equal(q.reshape(2), [21.0, 43.0])


def test_spectral_clamp_bound():
    e1 = np.array([0.5, 3.0, 10.0, 0.0])
    kn2 = np.array([1.0, 1.0, 0.5, 0.0])
    e = O.spectral_clamp(e1, kn2)
    assert np.allclose(e, [0.5, 2.0, 4.0, 0.0])
    assert np.all(e * kn2 <= 2.0 + 1e-15)


def _active_trace(seed=4, S=3, N=24, d=6, chunk=5, alpha=0.95):
    rng = np.random.default_rng(seed)
    xs = rng.standard_normal((S, N, d)) * 2.0
    qs = rng.standard_normal((S, N, d))
    inits = _active_inits(rng, S, d)
    y, fin, tr = O.scan_five_memory(xs, qs, inits, chunk, alpha, 1e-6, trace=True)
    return xs, qs, inits, y, fin, tr


def test_gate_bounds_on_scans():
    for seed in range(4):
        _, _, _, _, _, tr = _active_trace(seed)
        al, eta, g = tr["alpha_t"], tr["eta"], tr["gain"]
        kn2 = np.sum(tr["k"] ** 2, axis=-1)
        assert np.all(al <= 0.95) and np.all(al > 0)
        assert np.all(eta >= 0) and np.all(eta <= tr["eta0"] * (1 + 1e-15))
        assert np.all(eta * g <= (1.0 - al) * (1 + 1e-14))
        unsat = tr["eta0"] * g / (1.0 - al) < 15.0
        assert np.all((eta * g)[unsat] < (1.0 - al)[unsat])
        assert np.all(eta * kn2 <= 2.0 + 1e-12)


def test_retained_transition_svd_brute_force():
    """sigma_max of alpha_t (I - eta k k^T) is exactly alpha_t <= alpha; the full
    right factor of the write (retained + injection) is a strict contraction."""
    for seed in range(3):
        _, _, _, _, _, tr = _active_trace(seed, S=2, N=16, d=5)
        S, N, d = tr["k"].shape
        for s in range(S):
            for t in range(N):
                k, v = tr["k"][s, t], tr["v"][s, t]
                a, e = tr["alpha_t"][s, t], tr["eta"][s, t]
                R = a * (np.eye(d) - e * np.outer(k, k))
                sv = np.linalg.svd(R, compute_uv=False)
                assert abs(sv[0] - a) < 1e-12 and sv[0] <= 0.95 + 1e-12
                T = R - e * np.outer(k - v, k)        # injection (k - v) k^T
                assert np.linalg.svd(T, compute_uv=False)[0] < 1.0


# ---------------------------------------------------------------- write rule
def test_l2_signal_is_autograd_gradient():
    rng = np.random.default_rng(5)
    S, m, d = 3, 7, 5
    X = rng.standard_normal((S, m, d))
    k = rng.standard_normal((S, d))
    v = rng.standard_normal((S, d))
    Xt = torch.tensor(X, requires_grad=True)
    kt, vt = torch.tensor(k), torch.tensor(v)
    vhat = torch.einsum("smd,sd->sm", Xt, vt).detach()          # private target, held fixed
    loss = 0.5 * ((torch.einsum("smd,sd->sm", Xt, kt) - vhat) ** 2).sum()
    loss.backward()
    np.testing.assert_allclose(O.l2_signal(X, k, v), Xt.grad.numpy(), rtol=1e-12, atol=1e-14)


def test_scan_states_follow_retained_transition_plus_gradient():
    """Every recorded state = previous @ alpha_t (I - eta k k^T) - eta * autograd gradient."""
    xs, qs, inits, y, fin, tr = _active_trace(7, S=2, N=12, d=4, chunk=5)
    st = tr["states"]
    S, N, d = tr["k"].shape
    for s in range(S):
        for t in range(N):
            X = torch.tensor(st[s, t], requires_grad=True)
            k = torch.tensor(tr["k"][s, t])
            v = torch.tensor(tr["v"][s, t])
            a, e = float(tr["alpha_t"][s, t]), float(tr["eta"][s, t])
            loss = 0.5 * ((X @ k - (X @ v).detach()) ** 2).sum()
            loss.backward()
            R = a * (torch.eye(d, dtype=torch.float64) - e * torch.outer(k, k))
            expect = X.detach() @ R - e * X.grad
            np.testing.assert_allclose(st[s, t + 1], expect.numpy(), rtol=1e-12, atol=1e-14)
            # readout after the write, from the content memory (rows 0..d-1)
            np.testing.assert_allclose(y[s, t], st[s, t + 1][:d] @ qs[s, t], rtol=1e-12, atol=1e-14)


def test_frobenius_norms_non_increasing():
    for seed in range(5):
        _, _, _, _, _, tr = _active_trace(seed, S=4, N=40, d=8, chunk=7)
        for name, fro in tr["fro"].items():
            diff = np.diff(fro, axis=1)
            assert np.all(diff <= 1e-12 * fro[:, :-1] + 1e-300), name


def test_eta_zero_and_alpha_one_keep_initial_states():
    rng = np.random.default_rng(8)
    S, N, d = 3, 17, 6
    xs, qs = rng.standard_normal((S, N, d)), rng.standard_normal((S, N, d))
    inits = _active_inits(rng, S, d)
    y, fin, _ = O.scan_five_memory(xs, qs, inits, 5, 0.95, 1e-6, eta_override=0.0, alpha_override=1.0)
    for name in O.MEMORIES:
        assert np.array_equal(fin[name], inits[name])
    # states are bit-identical (T_t = I); the readout only differs by summation order
    np.testing.assert_allclose(y, np.einsum("sij,stj->sti", inits["M_mem"], qs), rtol=1e-13, atol=1e-15)


def test_eta_zero_gives_product_of_retentions():
    rng = np.random.default_rng(9)
    S, N, d = 3, 17, 6
    xs, qs = rng.standard_normal((S, N, d)), rng.standard_normal((S, N, d))
    inits = _active_inits(rng, S, d)
    y, fin, tr = O.scan_five_memory(xs, qs, inits, 4, 0.95, 1e-6, eta_override=0.0, trace=True)
    prod = np.prod(tr["alpha_t"], axis=1)
    for name in O.MEMORIES:
        expect = inits[name] * prod.reshape((S,) + (1,) * (inits[name].ndim - 1))
        np.testing.assert_allclose(fin[name], expect, rtol=1e-13, atol=0)


# ---------------------------------------------------------------- chunking
@pytest.mark.parametrize("seed", [0, 1])
def test_chunk_one_is_tokenwise_recurrence(seed):
    rng = np.random.default_rng(seed)
    S, N, d = 3, 29, 8
    xs, qs = rng.standard_normal((S, N, d)) * 1.5, rng.standard_normal((S, N, d))
    inits = _active_inits(rng, S, d)
    y1, f1, _ = O.scan_five_memory(xs, qs, inits, 1, 0.9, 1e-6)
    y2, f2 = O.scan_tokenwise(xs, qs, inits, 0.9, 1e-6)
    np.testing.assert_allclose(y1, y2, rtol=1e-12, atol=1e-15)
    for name in O.MEMORIES:
        np.testing.assert_allclose(f1[name], f2[name], rtol=1e-12, atol=1e-15)


def test_single_chunk_generates_from_initial_states():
    rng = np.random.default_rng(10)
    S, N, d = 2, 15, 5
    xs, qs = rng.standard_normal((S, N, d)), rng.standard_normal((S, N, d))
    inits = _active_inits(rng, S, d)
    _, _, tr = O.scan_five_memory(xs, qs, inits, N, 0.95, 1e-6, trace=True)
    kt = np.einsum("sij,stj->sti", inits["M_k"], xs)
    k = kt / np.sqrt(np.sum(kt ** 2, -1, keepdims=True) + 1e-6)
    np.testing.assert_allclose(tr["k"], k, rtol=1e-12)
    np.testing.assert_allclose(tr["v"], np.einsum("sij,stj->sti", inits["M_v"], xs), rtol=1e-12)


def test_chunk_size_changes_result():
    """Changing the chunk length changes what generation sees (so it must matter)."""
    rng = np.random.default_rng(11)
    S, N, d = 2, 20, 6
    xs, qs = rng.standard_normal((S, N, d)), rng.standard_normal((S, N, d))
    inits = _active_inits(rng, S, d)
    ya, _, _ = O.scan_five_memory(xs, qs, inits, 5, 0.95, 1e-6)
    yb, _, _ = O.scan_five_memory(xs, qs, inits, 4, 0.95, 1e-6)
    assert O.rel_fro(ya, yb) > 1e-3
    # the first four tokens see the same (initial) boundary in both runs
    np.testing.assert_array_equal(ya[:, :4], yb[:, :4])


@pytest.mark.parametrize("chunk", [1, 3, 7, 24, 100])
def test_qform_equals_five_memory(chunk):
    rng = np.random.default_rng(12 + chunk)
    S, N, d = 3, 24, 7
    xs, qs = rng.standard_normal((S, N, d)) * 1.3, rng.standard_normal((S, N, d))
    inits = _active_inits(rng, S, d)
    y1, f1, _ = O.scan_five_memory(xs, qs, inits, chunk, 0.93, 1e-6)
    y2, f2 = O.scan_qform(xs, qs, inits, chunk, 0.93, 1e-6)
    assert O.rel_fro(y2, y1) < 1e-12
    for name in O.MEMORIES:
        assert O.rel_fro(f2[name], f1[name]) < 1e-12


def test_pre_write_readout_first_token_reads_initials():
    rng = np.random.default_rng(13)
    S, N, d = 2, 6, 4
    xs, qs = rng.standard_normal((S, N, d)), rng.standard_normal((S, N, d))
    inits = _active_inits(rng, S, d)
    y, _, _ = O.scan_five_memory(xs, qs, inits, 3, 0.95, 1e-6, readout="pre")
    np.testing.assert_allclose(y[:, 0], np.einsum("sij,sj->si", inits["M_mem"], qs[:, 0]), rtol=1e-14)


# ---------------------------------------------------------------- operator
def _small_params(rng, C, heads, same_routes=False, active=True):
    d = C // heads
    s_ = 0.3 if active else 0.02
    p = dict(W_q=rng.standard_normal((C, C)) / np.sqrt(C), scales=rng.uniform(0.1, 0.5, (4, C)),
             M_mem0=rng.normal(0, s_, (4, heads, d, d)), M_k0=rng.normal(0, s_, (4, heads, d, d)),
             M_v0=rng.normal(0, s_, (4, heads, d, d)), m_eta0=rng.normal(0, 0.5, (4, heads, d)),
             m_alpha0=rng.normal(0, 1.0, (4, heads, d)))
    if same_routes:
        for key in ("M_mem0", "M_k0", "M_v0", "m_eta0", "m_alpha0"):
            p[key][:] = p[key][0:1]
    return p


def _one_hot(p, r):
    q = dict(p)
    q["scales"] = np.zeros_like(p["scales"])
    q["scales"][r] = 1.0
    return q


def test_route_symmetries_rot180_and_transpose():
    rng = np.random.default_rng(14)
    B, H, W, C, heads = 2, 4, 5, 6, 2
    x = rng.standard_normal((B, H, W, C))
    p = _small_params(rng, C, heads, same_routes=True)
    kw = dict(alpha_max=0.95, heads=heads)
    out1, _, _ = O.operator_forward(x, _one_hot(p, 1), **kw)
    out0_rot, _, _ = O.operator_forward(x[:, ::-1, ::-1], _one_hot(p, 0), **kw)
    np.testing.assert_allclose(out1, out0_rot[:, ::-1, ::-1], rtol=1e-13, atol=1e-15)
    out2, _, _ = O.operator_forward(x, _one_hot(p, 2), **kw)
    out0_t, _, _ = O.operator_forward(x.transpose(0, 2, 1, 3).copy(), _one_hot(p, 0), **kw)
    np.testing.assert_allclose(out2, out0_t.transpose(0, 2, 1, 3), rtol=1e-13, atol=1e-15)
    out3, _, _ = O.operator_forward(x, _one_hot(p, 3), **kw)
    out2_rot, _, _ = O.operator_forward(x[:, ::-1, ::-1], _one_hot(p, 2), **kw)
    np.testing.assert_allclose(out3, out2_rot[:, ::-1, ::-1], rtol=1e-13, atol=1e-15)


def test_fusion_is_sum_of_one_hot_routes():
    rng = np.random.default_rng(15)
    B, H, W, C, heads = 1, 3, 4, 4, 1
    x = rng.standard_normal((B, H, W, C))
    p = _small_params(rng, C, heads)
    kw = dict(alpha_max=0.9, heads=heads)
    full, _, _ = O.operator_forward(x, p, **kw)
    parts = 0
    for r in range(4):
        o, _, _ = O.operator_forward(x, _one_hot(p, r), **kw)
        parts = parts + p["scales"][r] * o
    np.testing.assert_allclose(full, parts, rtol=1e-13, atol=1e-15)


def test_batch_permutation_equivariance():
    rng = np.random.default_rng(16)
    B, H, W, C, heads = 3, 3, 3, 4, 2
    x = rng.standard_normal((B, H, W, C))
    p = _small_params(rng, C, heads)
    kw = dict(alpha_max=0.95, heads=heads)
    o, f, _ = O.operator_forward(x, p, **kw)
    perm = [2, 0, 1]
    o2, f2, _ = O.operator_forward(x[perm], p, **kw)
    np.testing.assert_array_equal(o2, o[perm])
    np.testing.assert_array_equal(f2, f[:, perm])


def test_fresh_state_every_call():
    """Each call starts a new sequence from the learned initials (README, SRNL section)."""
    inp = make_inputs(CONFIGS["pr1_8x8"], seed=0)
    a, _, _ = O.forward_from_inputs(inp)
    b, _, _ = O.forward_from_inputs(inp)
    np.testing.assert_array_equal(a, b)


def test_pr1_config_qform_and_tokenwise_consistency():
    inp = make_inputs(CONFIGS["pr1_8x8"], seed=0)
    o1, f1, _ = O.forward_from_inputs(inp)
    o2, f2, _ = O.forward_from_inputs(inp, scan="qform")
    assert O.rel_fro(o2, o1) < 1e-12
    cfg1 = CONFIGS["pr1_8x8"].replace(chunk_row=1, chunk_col=1)
    inp1 = make_inputs(cfg1, seed=0)
    o3, _, _ = O.forward_from_inputs(inp1)
    o4, _, _ = O.forward_from_inputs(inp1, scan="tokenwise")
    assert O.rel_fro(o4, o3) < 1e-12


# ------------------------------------------------ standalone sequence layer
def _seq_params(heads, d, rng, mem_scale=0.3, vec_scale=1.0):
    return dict(M_mem0=rng.normal(0, mem_scale, (heads, d, d)), M_k0=rng.normal(0, mem_scale, (heads, d, d)),
                M_v0=rng.normal(0, mem_scale, (heads, d, d)), m_eta0=rng.normal(0, vec_scale, (heads, d)),
                m_alpha0=rng.normal(0, vec_scale, (heads, d)))


def test_sequence_chunk1_equals_tokenwise():
    rng = np.random.default_rng(11)
    x = rng.normal(size=(2, 13, 8))
    p = _seq_params(2, 4, rng)
    y1, f1 = O.sequence_forward(x, p, alpha_max=0.9, chunk=1, heads=2)
    y2, f2 = O.sequence_forward(x, p, alpha_max=0.9, chunk=1, heads=2, scan="tokenwise")
    assert np.allclose(y1, y2, rtol=1e-12, atol=1e-14) and np.allclose(f1, f2, rtol=1e-12, atol=1e-14)


def test_sequence_causal_prefix_and_default_queries():
    # README: an incomplete final chunk is allowed (257 tokens, chunks of 64); the output at
    # token t depends on tokens <= t only, so a prefix of the input gives a prefix of the output
    rng = np.random.default_rng(12)
    x = rng.normal(size=(1, 257, 8))
    q = rng.normal(size=(1, 257, 8))
    p = _seq_params(2, 4, rng)
    y, _ = O.sequence_forward(x, p, alpha_max=0.95, heads=2, queries=q)
    yp, _ = O.sequence_forward(x[:, :200], p, alpha_max=0.95, heads=2, queries=q[:, :200])
    assert np.array_equal(y[:, :200], yp)
    ya, _ = O.sequence_forward(x, p, alpha_max=0.95, heads=2)
    yb, _ = O.sequence_forward(x, p, alpha_max=0.95, heads=2, queries=x)
    assert np.array_equal(ya, yb)
    assert not np.allclose(y, ya)


def test_sequence_equals_operator_route0():
    rng = np.random.default_rng(13)
    B, T, heads, d = 2, 21, 2, 4
    D = heads * d
    x = rng.normal(size=(B, T, D))
    p = _seq_params(heads, d, rng)
    ys, fs = O.sequence_forward(x, p, alpha_max=0.9, chunk=5, heads=heads)
    op = {k: np.repeat(np.asarray(v)[None], 4, axis=0) for k, v in p.items()}
    op["W_q"] = np.eye(D)
    op["scales"] = np.zeros((4, D))
    op["scales"][0] = 1.0
    out, fin, _ = O.operator_forward(x.reshape(B, 1, T, D), op, alpha_max=0.9, chunk_row=5, chunk_col=5,
                                     heads=heads)
    assert np.allclose(out.reshape(B, T, D), ys, rtol=1e-12, atol=1e-14)
    assert np.allclose(fin[0], fs, rtol=1e-12, atol=1e-14)


# ------------------------------------------------ hard injection clamp
def test_hard_cap_bound_is_tight():
    rng = np.random.default_rng(21)
    eta0 = rng.uniform(0, 3, 2000)
    gain = rng.uniform(0.01, 2, 2000)
    al = rng.uniform(0.05, 0.95, 2000)
    e1, binds = O.hard_cap(eta0, gain, al)
    assert np.all(e1 * gain <= (1 - al) * (1 + 1e-14))
    assert np.allclose(e1[binds] * gain[binds], (1 - al[binds]), rtol=1e-13)
    assert np.array_equal(e1[~binds], eta0[~binds])
    assert 100 < np.count_nonzero(binds) < 1900


def test_hard_cap_extremes():
    # one chunk spanning the sequence: every token is generated from the initial states
    rng = np.random.default_rng(22)
    T = 24
    x = np.abs(rng.normal(size=(2, T, 8)))  # positive inputs: a = m_eta0 . x has the sign of m_eta0
    p = _seq_params(2, 4, rng)
    total = 2 * 2 * T
    for m_eta, expect in ((+5.0, "all"), (-30.0, "none")):
        p["m_eta0"] = np.full_like(p["m_eta0"], m_eta)
        cnt = [0]
        yh, _ = O.sequence_forward(x, p, alpha_max=0.9, chunk=T, heads=2, cap="hard", counter=cnt)
        ys, _ = O.sequence_forward(x, p, alpha_max=0.9, chunk=T, heads=2, cap="soft")
        if expect == "all":
            # huge steps: the clamp is active on every token (and the soft cap saturates at
            # the same margin, so both give nearly the same write)
            assert cnt[0] == total
        else:
            assert cnt[0] == 0  # tiny steps: never active, and the soft cap is eta0 (1 - O(z^2))
            assert np.allclose(yh, ys, rtol=1e-9, atol=1e-15)


def test_hard_cap_nonexpansive_and_tokenwise():
    rng = np.random.default_rng(24)
    S, N, d = 3, 30, 4
    xs = rng.normal(size=(S, N, d))
    qs = rng.normal(size=(S, N, d))
    inits = dict(M_mem=rng.normal(0, 0.5, (S, d, d)), M_k=rng.normal(0, 0.5, (S, d, d)),
                 M_v=rng.normal(0, 0.5, (S, d, d)), m_eta=rng.normal(0, 2, (S, d)), m_alpha=rng.normal(0, 2, (S, d)))
    cnt = [0]
    y, fin, tr = O.scan_five_memory(xs, qs, inits, 5, 0.9, 1e-6, trace=True, cap="hard", counter=cnt)
    for name, f in tr["fro"].items():
        assert np.all(np.diff(f, axis=1) <= 1e-12 * (1 + f[:, :-1])), name
    assert cnt[0] == int(np.count_nonzero(tr["eta0"] * tr["gain"] > 1 - tr["alpha_t"]))
    assert 0 < cnt[0] < S * N
    y1, f1, _ = O.scan_five_memory(xs, qs, inits, 1, 0.9, 1e-6, cap="hard")
    y2, f2 = O.scan_tokenwise(xs, qs, inits, 0.9, 1e-6, cap="hard")
    assert np.allclose(y1, y2, rtol=1e-11, atol=1e-13)
