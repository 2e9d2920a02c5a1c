"""Float64 CPU oracle for the gradient of the SRNL four-direction chunked memory scan.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The GPU library never
calls it and shares no code with it.

The pages ask for the operator to be trainable end to end ([README] "SRNL and
VisionHOPE operator": the layer sits inside a backbone trained by back-propagation;
[SUMMARY] the write-rule and 2D-maps paragraphs give the forward it differentiates).
None prints a backward pass, so this module is reverse-mode differentiation of the
forward in ``srnl_oracle`` written out step by step, on the *literal five-memory*
recurrence (not on the single-product form the GPU path uses):

  * readout y_t = M_mem,t q_t (post-write): dM_mem,t += dy_t q_t^T, dq_t = M_mem,t^T dy_t;
  * write X' = alpha (X - eta (X k) k^T) - eta ((X k) - (X v)) k^T on every memory row:
    given G = dL/dX', with P = X k, R = X v, Gk = G k,
        dX     = alpha G - (1 + alpha) eta Gk k^T + eta Gk v^T
        dk    += -(1 + alpha) eta (X^T Gk + G^T P) + eta G^T R
        dv    += eta X^T Gk
        dalpha = <G, X> - eta <Gk, P>
        deta   = -(1 + alpha) <Gk, P> + <Gk, R>
    summed over all rows of the five stacked memories (they share k, v, alpha, eta);
  * gates (key normalisation, retention clamp, softplus, soft cap or hard clamp,
    spectral clamp) by the chain rule, taking the active branch of every min;
  * generation from the boundary memories: dM_{k,v,eta,alpha; b} += dgen x^T and
    dx_t = M_{..., b}^T dgen_t, added to the boundary state's gradient;
  * operator: route gather/restore are permutations (their adjoints are the inverse
    permutations), fusion out = sum_r s_r * y_r gives dy_r = s_r * dout and
    ds_r = sum dout * y_r, and q = x W_q^T gives dW_q = dq^T x, dx += dq W_q.

Chunks are recomputed from their boundary states (checkpoints), so memory stays at one
chunk of states per sequence.

Pins (tests/test_oracle_grad_pins.py): central finite differences of the *forward*
oracle along random directions, block by block (x, W_q, scales, each initial memory;
queries for the sequence layer), with the soft cap and with the hard clamp, on ragged
chunkings; the gate backward against finite differences in every regime (series
branch of the soft cap, saturated cap, retention clamp active, spectral clamp active,
hard clamp active and idle); the fusion-scale gradient against its closed form (the
operator is linear in the scales: ds_r = sum dout * (output with one-hot scales on
route r)); the query-projection gradient against the exact difference quotient (the
output is linear in W_q).
"""
from __future__ import annotations

from typing import Dict

import numpy as np

from . import srnl_oracle as F

_DPHI_SERIES_BELOW = 1e-3


# --------------------------------------------------------------------------
# Gates
# --------------------------------------------------------------------------
def _dphi(z: np.ndarray) -> np.ndarray:
    """Derivative of the soft-cap function phi(z) = tanh(z)/z as the forward evaluates it:
    the forward uses the series 1 - z^2/3 below 1e-6 (derivative -2z/3); above, the
    derivative of tanh(z)/z is (z (1 - tanh^2 z) - tanh z) / z^2, evaluated by its Taylor
    series -2z/3 + 8z^3/15 below 1e-3 where the closed form cancels."""
    z = np.asarray(z, dtype=np.float64)
    tiny = z < F._PHI_SERIES_BELOW
    small = z < _DPHI_SERIES_BELOW
    zs = np.where(small, 1.0, z)
    th = np.tanh(zs)
    closed = (zs * (1.0 - th * th) - th) / (zs * zs)
    series = -2.0 * z / 3.0 + 8.0 * z ** 3 / 15.0
    return np.where(tiny, -2.0 * z / 3.0, np.where(small, series, closed))


def gates_backward(ktil, v, a, beta, alpha_max, eps, cap, dk, dv, dalpha, deta):
    """Reverse mode through ``srnl_oracle.gates``.

    Forward (per token): k = k~ / sqrt(|k~|^2 + eps); alpha_t = min(sigmoid(beta), alpha);
    eta0 = softplus(a); g = |k - v| |k|; eta1 = soft cap or hard clamp of eta0; eta =
    min(eta1, 2 / |k|^2).  Given the gradients of the loss with respect to the gate
    outputs k, alpha_t, eta (and the value v as the write uses it directly), returns
    (dk~, dv, da, dbeta)."""
    ktil = np.asarray(ktil, np.float64)
    v = np.asarray(v, np.float64)
    n2 = np.sum(ktil * ktil, axis=-1)
    s = np.sqrt(n2 + eps)
    k = ktil / s[..., None]
    sig = F.sigmoid(np.asarray(beta, np.float64))
    clamped = sig > alpha_max
    alpha_t = np.minimum(sig, alpha_max)
    eta0 = F.softplus(np.asarray(a, np.float64))
    kn2 = np.sum(k * k, axis=-1)
    kn = np.sqrt(kn2)
    e = k - v
    ne = np.sqrt(np.sum(e * e, axis=-1))
    gain = ne * kn
    margin = 1.0 - alpha_t

    dk = np.array(dk, dtype=np.float64, copy=True)
    dv = np.array(dv, dtype=np.float64, copy=True)
    dalpha = np.array(dalpha, dtype=np.float64, copy=True)
    deta = np.asarray(deta, np.float64)

    if cap == "soft":
        eta1 = F.soft_cap(eta0, gain, alpha_t)
    else:
        eta1, binds = F.hard_cap(eta0, gain, alpha_t)
    # spectral clamp eta = min(eta1, 2 / kn2)
    over = eta1 * kn2 > 2.0
    safe_kn2 = np.where(over, kn2, 1.0)
    deta1 = np.where(over, 0.0, deta)
    dkn2 = np.where(over, -2.0 * deta / (safe_kn2 * safe_kn2), 0.0)
    # injection cap
    if cap == "soft":
        z = eta0 * gain / margin
        phi = np.where(z < F._PHI_SERIES_BELOW, 1.0 - z * z / 3.0,
                       np.tanh(np.where(z < F._PHI_SERIES_BELOW, 1.0, z)) / np.where(z < F._PHI_SERIES_BELOW, 1.0, z))
        dz = deta1 * eta0 * _dphi(z)
        deta0 = deta1 * phi + dz * gain / margin
        dgain = dz * eta0 / margin
        dalpha = dalpha + dz * eta0 * gain / (margin * margin)
    elif cap == "hard":
        safe_gain = np.where(binds, gain, 1.0)
        deta0 = np.where(binds, 0.0, deta1)
        dgain = np.where(binds, -deta1 * margin / (safe_gain * safe_gain), 0.0)
        dalpha = dalpha + np.where(binds, -deta1 / safe_gain, 0.0)
    else:
        raise ValueError(cap)
    # gain = ne * kn
    safe_ne = np.where(ne > 0.0, ne, 1.0)
    safe_kn = np.where(kn > 0.0, kn, 1.0)
    de = (dgain * kn / safe_ne)[..., None] * e
    dkn = dgain * ne
    dk = dk + de + (2.0 * dkn2 + dkn / safe_kn)[..., None] * k
    dv = dv - de
    # k = k~ / s
    dktil = dk / s[..., None] - ktil * (np.sum(ktil * dk, axis=-1) / (s ** 3))[..., None]
    da = deta0 * F.sigmoid(np.asarray(a, np.float64))
    dbeta = np.where(clamped, 0.0, dalpha * sig * (1.0 - sig))
    return dktil, dv, da, dbeta


# --------------------------------------------------------------------------
# Write and readout
# --------------------------------------------------------------------------
def retained_write_backward(Xm, k, v, eta, alpha_t, G):
    """Reverse mode through ``srnl_oracle.retained_write`` for S sequences.

    Xm: [S, m, d] memory before the write; k, v: [S, d]; eta, alpha_t: [S]; G: [S, m, d]
    gradient with respect to the memory after the write.  Returns (dX, dk, dv, dalpha,
    deta), the memory-row sums taken."""
    al = alpha_t[:, None, None]
    et = eta[:, None, None]
    P = np.matmul(Xm, k[:, :, None])[..., 0]          # [S, m]
    R = np.matmul(Xm, v[:, :, None])[..., 0]
    Gk = np.matmul(G, k[:, :, None])[..., 0]
    dX = al * G - ((1.0 + alpha_t) * eta)[:, None, None] * Gk[:, :, None] * k[:, None, :] \
        + et * Gk[:, :, None] * v[:, None, :]
    XtGk = np.matmul(np.swapaxes(Xm, 1, 2), Gk[:, :, None])[..., 0]   # [S, d]
    GtP = np.matmul(np.swapaxes(G, 1, 2), P[:, :, None])[..., 0]
    GtR = np.matmul(np.swapaxes(G, 1, 2), R[:, :, None])[..., 0]
    c1 = ((1.0 + alpha_t) * eta)[:, None]
    dk = -c1 * (XtGk + GtP) + eta[:, None] * GtR
    dv = eta[:, None] * XtGk
    GkP = np.sum(Gk * P, axis=1)
    dalpha = np.sum(G * Xm, axis=(1, 2)) - eta * GkP
    deta = -(1.0 + alpha_t) * GkP + np.sum(Gk * R, axis=1)
    return dX, dk, dv, dalpha, deta


def scan_five_memory_backward(xs, qs, inits, chunk, alpha_max, eps, dy, *, cap="soft"):
    """Gradient of sum(dy * y) for ``srnl_oracle.scan_five_memory`` (post-write readout).

    xs, qs, dy: [S, N, d]; inits as in the forward.  Returns (dxs, dqs, dinits, y): the
    gradients with respect to the memory inputs, the queries and the five initial
    memories, and the forward outputs y (for the fusion-scale gradient)."""
    xs = np.asarray(xs, np.float64)
    qs = np.asarray(qs, np.float64)
    dy = np.asarray(dy, np.float64)
    S, N, d = xs.shape
    mem = F._stack(inits, d)
    # forward pass keeping the boundary states only
    bounds = []
    for c0 in range(0, N, chunk):
        c1 = min(c0 + chunk, N)
        bounds.append((c0, c1, mem.copy()))
        ktil, v, a, beta = F._generate(mem, d, xs[:, c0:c1])
        gt = F.gates(ktil, v, a, beta, alpha_max, eps, cap)
        for j in range(c1 - c0):
            mem = F.retained_write(mem, gt["k"][:, j], v[:, j], gt["eta"][:, j], gt["alpha_t"][:, j])
    dxs = np.zeros_like(xs)
    dqs = np.zeros_like(qs)
    y = np.zeros((S, N, d))
    Gm = np.zeros_like(mem)       # dL / d(memory after the last token)
    for c0, c1, mem_b in reversed(bounds):
        Xc = xs[:, c0:c1]
        ktil, v, a, beta = F._generate(mem_b, d, Xc)
        gt = F.gates(ktil, v, a, beta, alpha_max, eps, cap)
        states = [mem_b]
        for j in range(c1 - c0):
            states.append(F.retained_write(states[-1], gt["k"][:, j], v[:, j], gt["eta"][:, j],
                                           gt["alpha_t"][:, j]))
        Lc = c1 - c0
        dk = np.zeros((S, Lc, d))
        dv = np.zeros((S, Lc, d))
        dal = np.zeros((S, Lc))
        det = np.zeros((S, Lc))
        for j in reversed(range(Lc)):
            t = c0 + j
            after = states[j + 1]
            y[:, t] = np.matmul(after[:, :d], qs[:, t, :, None])[..., 0]
            Gm[:, :d] += dy[:, t, :, None] * qs[:, t, None, :]
            dqs[:, t] = np.matmul(np.swapaxes(after[:, :d], 1, 2), dy[:, t, :, None])[..., 0]
            Gm, dk[:, j], dv[:, j], dal[:, j], det[:, j] = retained_write_backward(
                states[j], gt["k"][:, j], v[:, j], gt["eta"][:, j], gt["alpha_t"][:, j], Gm)
        dktil, dvv, da, dbeta = gates_backward(ktil, v, a, beta, alpha_max, eps, cap, dk, dv, dal, det)
        dgen = np.concatenate([dktil, dvv, da[..., None], dbeta[..., None]], axis=-1)  # [S, Lc, 2d+2]
        gen_rows = mem_b[:, d:]                                                          # [S, 2d+2, d]
        Gm[:, d:] += np.matmul(np.swapaxes(dgen, 1, 2), Xc)
        dxs[:, c0:c1] += np.matmul(dgen, gen_rows)
    return dxs, dqs, F._unstack(Gm, d), y


# --------------------------------------------------------------------------
# Operator and sequence layer
# --------------------------------------------------------------------------
PARAM_KEYS = ("W_q", "scales", "M_mem0", "M_k0", "M_v0", "m_eta0", "m_alpha0")
_INIT_KEYS = (("M_mem0", "M_mem"), ("M_k0", "M_k"), ("M_v0", "M_v"), ("m_eta0", "m_eta"),
              ("m_alpha0", "m_alpha"))


def operator_backward(x, params, dout, *, alpha_max, eps=1e-6, chunk_row=0, chunk_col=0, heads,
                      cap="soft") -> Dict[str, np.ndarray]:
    """Gradient of sum(dout * out) for ``srnl_oracle.operator_forward``.

    Returns a dict: "x" [B, H, W, C] and one entry per parameter of ``params`` (W_q [C, C],
    scales [4, C], M_mem0/M_k0/M_v0 [4, heads, d, d], m_eta0/m_alpha0 [4, heads, d])."""
    x = np.asarray(x, np.float64)
    dout = np.asarray(dout, np.float64)
    B, H, W, C = x.shape
    d = C // heads
    N = H * W
    W_q = np.asarray(params["W_q"], np.float64)
    scales = np.asarray(params["scales"], np.float64)
    q = F.query_projection(x, W_q)
    dx = np.zeros_like(x)
    dq = np.zeros_like(q)
    grads = {key: np.zeros(np.shape(params[key])) for key in PARAM_KEYS}

    def to_seq(a):   # [B, N, C] route order -> [B * heads, N, d]
        return a.reshape(B, N, heads, d).transpose(0, 2, 1, 3).reshape(B * heads, N, d)

    def from_seq(a):
        return a.reshape(B, heads, N, d).transpose(0, 2, 1, 3).reshape(B, N, C)

    for r in range(F.ROUTES):
        L = F.default_chunk(H, W, r, chunk_row, chunk_col)
        xr = to_seq(F.gather(x, r))
        qr = to_seq(F.gather(q, r))
        dyr = to_seq(F.gather(dout, r) * scales[r][None, None, :])
        inits = F._route_inits(params, r, B)
        dxs, dqs, dinit, y = scan_five_memory_backward(xr, qr, inits, L, alpha_max, eps, dyr, cap=cap)
        dx += F.restore(from_seq(dxs), r, H, W)
        dq += F.restore(from_seq(dqs), r, H, W)
        grads["scales"][r] = np.einsum("bhwc,bhwc->c", dout, F.restore(from_seq(y), r, H, W))
        for key, name in _INIT_KEYS:
            g = dinit[name]
            grads[key][r] = g.reshape((B, heads) + g.shape[1:]).sum(axis=0)
    grads["W_q"] = np.einsum("bhwo,bhwc->oc", dq, x)
    dx += np.einsum("bhwo,oc->bhwc", dq, W_q)
    grads["x"] = dx
    return grads


def sequence_backward(x, params, dy, *, alpha_max, eps=1e-6, chunk=64, heads, queries=None,
                      cap="soft") -> Dict[str, np.ndarray]:
    """Gradient of sum(dy * y) for ``srnl_oracle.sequence_forward``.

    Returns "x" [B, T, D], "queries" [B, T, D] (absent when the queries are x itself: then
    their gradient is folded into "x") and the five initial memories [heads, ...]."""
    x = np.asarray(x, np.float64)
    dy = np.asarray(dy, np.float64)
    B, T, D = x.shape
    d = D // heads
    q = x if queries is None else np.asarray(queries, np.float64)
    L = chunk if chunk > 0 else 64

    def to_seq(a):
        return a.reshape(B, T, heads, d).transpose(0, 2, 1, 3).reshape(B * heads, T, d)

    def from_seq(a):
        return a.reshape(B, heads, T, d).transpose(0, 2, 1, 3).reshape(B, T, D)

    inits = {}
    for key, name in _INIT_KEYS:
        arr = np.asarray(params[key], np.float64)
        inits[name] = np.broadcast_to(arr[None], (B,) + arr.shape).reshape((-1,) + arr.shape[1:]).copy()
    dxs, dqs, dinit, _ = scan_five_memory_backward(to_seq(x), to_seq(q), inits, L, alpha_max, eps,
                                                   to_seq(dy), cap=cap)
    out = {}
    if queries is None:
        out["x"] = from_seq(dxs) + from_seq(dqs)
    else:
        out["x"] = from_seq(dxs)
        out["queries"] = from_seq(dqs)
    for key, name in _INIT_KEYS:
        g = dinit[name]
        out[key] = g.reshape((B, heads) + g.shape[1:]).sum(axis=0)
    return out


def backward_from_inputs(inp, dout, **kw):
    """Convenience: ``operator_backward`` on a ``srnl_inputs.ScanInputs``."""
    cfg = inp.cfg
    return operator_backward(inp.x32, inp.params(), dout, alpha_max=cfg.alpha, eps=cfg.eps,
                             chunk_row=cfg.chunk_row, chunk_col=cfg.chunk_col, heads=cfg.heads, **kw)
