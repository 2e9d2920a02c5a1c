"""Pins for the block oracle (oracle/srnl_block.py): each checks it against a closed form,
an invariant or a hand-written case, not against a retyped copy of its own formulas."""
import math

import numpy as np
import pytest

from oracle import srnl_block as K
from oracle import srnl_oracle as O
from srnl_inputs import make_block_inputs


def test_layer_norm_zero_mean_unit_variance_and_affine_invariance():
    rng = np.random.default_rng(0)
    x = rng.normal(3.0, 2.0, (5, 7, 48))
    one, zero = np.ones(48), np.zeros(48)
    y = K.layer_norm(x, one, zero, eps=0.0)
    np.testing.assert_allclose(y.mean(-1), 0.0, atol=1e-13)
    np.testing.assert_allclose((y ** 2).mean(-1), 1.0, rtol=1e-13)
    # a per-token affine change of the input leaves it unchanged (positive scale)
    a = rng.uniform(0.5, 4.0, (5, 7, 1))
    c = rng.normal(0, 3, (5, 7, 1))
    np.testing.assert_allclose(K.layer_norm(a * x + c, one, zero, eps=0.0), y, atol=1e-12)
    # scale and shift act per channel after the normalisation
    g, b = rng.normal(size=48), rng.normal(size=48)
    np.testing.assert_allclose(K.layer_norm(x, g, b, eps=0.0), y * g + b, atol=1e-12)
    # a two-channel row by hand: (1, 3) -> mean 2, variance 1 -> (-1, 1)
    np.testing.assert_allclose(K.layer_norm(np.array([[1.0, 3.0]]), np.ones(2), np.zeros(2), eps=0.0),
                               [[-1.0, 1.0]], atol=1e-15)


def test_dwconv_centre_tap_is_identity_and_off_centre_tap_is_a_shift():
    rng = np.random.default_rng(1)
    u = rng.normal(size=(2, 4, 5, 3))
    w = np.zeros((3, 3, 3))
    w[:, 1, 1] = 1.0
    np.testing.assert_array_equal(K.dwconv3x3(u, w, np.zeros(3)), u)
    # tap (di, dj) = (-1, +1): out[i, j] = u[i - 1, j + 1], zero outside the map
    w = np.zeros((3, 3, 3))
    w[:, 0, 2] = 1.0
    out = K.dwconv3x3(u, w, np.zeros(3))
    ref = np.zeros_like(u)
    ref[:, 1:, :-1] = u[:, :-1, 1:]
    np.testing.assert_array_equal(out, ref)


def test_dwconv_matches_window_sums_by_hand():
    rng = np.random.default_rng(2)
    u = rng.normal(size=(1, 3, 4, 2))
    w = rng.normal(size=(2, 3, 3))
    b = rng.normal(size=2)
    out = K.dwconv3x3(u, w, b)
    for i in range(3):
        for j in range(4):
            for c in range(2):
                acc = b[c]
                for di in (-1, 0, 1):
                    for dj in (-1, 0, 1):
                        ii, jj = i + di, j + dj
                        if 0 <= ii < 3 and 0 <= jj < 4:
                            acc += w[c, di + 1, dj + 1] * u[0, ii, jj, c]
                assert abs(out[0, i, j, c] - acc) < 1e-13


def test_gelu_closed_forms():
    assert K.gelu(np.array([0.0]))[0] == 0.0
    v = np.linspace(-6, 6, 101)
    np.testing.assert_allclose(K.gelu(v) - K.gelu(-v), v, atol=1e-14)
    phi1 = 0.5 * (1.0 + math.erf(1.0 / math.sqrt(2.0)))   # Phi(1) = 0.841344746...
    np.testing.assert_allclose(K.gelu(np.array([1.0])), [phi1], rtol=1e-15)
    np.testing.assert_allclose(phi1, 0.8413447460685429, rtol=1e-15)
    np.testing.assert_allclose(K.gelu(np.array([-10.0, 10.0])), [0.0, 10.0], atol=1e-20)


def _small(seed=3):
    return make_block_inputs(2, 4, 6, 32, 32, 16, "f32", seed=seed, mem_scale=0.3, vec_scale=0.5)


def _fwd(inp, p=None):
    return K.block_forward(inp.x32, p or inp.p, heads=inp.heads, alpha_max=0.95)


def test_zero_out_projections_make_the_block_the_identity():
    inp = _small()
    p = dict(inp.p)
    for k in ("W_out", "b_out", "W_2", "b_2"):
        p[k] = np.zeros_like(p[k])
    out, _ = _fwd(inp, p)
    np.testing.assert_array_equal(out, inp.x32.astype(np.float64))


def test_identity_mixer_reduces_to_x_plus_layer_norm():
    """W_in = I, centre-tap convolution, zero fusion scales, W_out = I, zero FFN: out = x + LN1(x)."""
    inp = _small(4)
    p = dict(inp.p)
    m = inp.m
    p["W_in"], p["b_in"] = np.eye(m), np.zeros(m)
    p["dw_w"] = np.zeros((m, 3, 3))
    p["dw_w"][:, 1, 1] = 1.0
    p["dw_b"] = np.zeros(m)
    p["scales"] = np.zeros((4, m))
    p["W_out"], p["b_out"] = np.eye(m), np.zeros(m)
    for k in ("W_2", "b_2"):
        p[k] = np.zeros_like(p[k])
    out, _ = _fwd(inp, p)
    x = inp.x32.astype(np.float64)
    mu = x.mean(-1, keepdims=True)
    sd = np.sqrt(((x - mu) ** 2).mean(-1, keepdims=True) + K.LN_EPS)
    np.testing.assert_allclose(out, x + (x - mu) / sd * p["ln1_g"] + p["ln1_b"], atol=1e-12)


def test_operator_branch_is_the_operator_on_u():
    """With a zero convolution and W_out = I, zero FFN: out - x = operator(u) + b_out."""
    inp = _small(5)
    p = dict(inp.p)
    m = inp.m
    p["dw_w"], p["dw_b"] = np.zeros((m, 3, 3)), np.zeros(m)
    p["W_out"] = np.eye(m)
    for k in ("W_2", "b_2"):
        p[k] = np.zeros_like(p[k])
    out, mids = _fwd(inp, p)
    op = {k: p[k] for k in ("W_q", "scales", "M_mem0", "M_k0", "M_v0", "m_eta0", "m_alpha0")}
    glob, _, _ = O.operator_forward(mids["u"], op, alpha_max=0.95, heads=inp.heads)
    np.testing.assert_allclose(out - inp.x32, glob + p["b_out"], atol=1e-12)


def test_block_is_equivariant_to_batch_order_and_preserves_shape():
    inp = _small(6)
    out, _ = _fwd(inp)
    assert out.shape == inp.x32.shape
    perm = [1, 0]
    out_p, _ = K.block_forward(inp.x32[perm], inp.p, heads=inp.heads, alpha_max=0.95)
    np.testing.assert_allclose(out_p, out[perm], atol=1e-12)


def test_ffn_reads_the_first_residual():
    """Identity mixer (out of the first residual y = x + LN1(x), as above) with a random FFN:
    out = y + FFN(LN2(y)), the FFN composed from the separately pinned LayerNorm, linear map and
    GELU, applied to y and not to x."""
    inp = _small(7)
    p = dict(inp.p)
    m = inp.m
    p["W_in"], p["b_in"] = np.eye(m), np.zeros(m)
    p["dw_w"] = np.zeros((m, 3, 3))
    p["dw_w"][:, 1, 1] = 1.0
    p["dw_b"] = np.zeros(m)
    p["scales"] = np.zeros((4, m))
    p["W_out"], p["b_out"] = np.eye(m), np.zeros(m)
    out, _ = _fwd(inp, p)
    x = inp.x32.astype(np.float64)
    mu = x.mean(-1, keepdims=True)
    sd = np.sqrt(((x - mu) ** 2).mean(-1, keepdims=True) + K.LN_EPS)
    y = x + (x - mu) / sd * p["ln1_g"] + p["ln1_b"]
    ffn = K.linear(K.gelu(K.linear(K.layer_norm(y, p["ln2_g"], p["ln2_b"]), p["W_1"], p["b_1"])), p["W_2"], p["b_2"])
    np.testing.assert_allclose(out, y + ffn, atol=1e-12)
