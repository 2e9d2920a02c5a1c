"""Float64 CPU oracle for the SRNL four-direction chunked memory scan.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The GPU library never
calls it and shares no code with it; the two meet only at the seeded inputs of
``srnl_inputs``.

Sources (web pages describing VisionHOPE; none prints an equation, so each step
below restates prose in symbols and marks the readings this oracle takes):
  [README]   "VisionHOPE" README (github PSRben/VisionHOPE): "Overview",
             "SRNL and VisionHOPE operator", "Fast inference".
  [OVERVIEW] "VisionHOPE Model Overview: Architecture, Benchmarks, and Practical
             Limits": "How VisionHOPE's Five Memories Work", "Four-Directional
             Scanning and Spatial Chunking", "Why the Stability Controls Matter".
  [SUMMARY]  "VisionHOPE: Visual Backbones as Self-Modifying Learning Systems"
             (summary of arXiv 2609.33325): the write-rule paragraph, the
             stability paragraph, the 2D-maps paragraph, the caveats paragraph.

Notation per (batch b, head h, route r): d = head dim, N = H*W tokens in route
order t = 0..N-1, chunk length L (W on row routes, H on column routes unless
overridden), memories M_mem, M_k, M_v (d x d) and m_eta, m_alpha (1 x d).

Pins (what checks this file against something other than itself), see
tests/test_oracle_pins.py:
  * route maps: bijection, gather/restore round trip, the 14x20 chunk example
    of [OVERVIEW], rot180 / transpose symmetries of whole-operator outputs;
  * stabilized key: closed form of ||k||^2;
  * gates: soft-cap margin, spectral clamp bound, brute-force SVD of every
    retained transition (sigma_max = alpha_t <= alpha), sigma_max(T_t) < 1;
  * write rule: the L2 learning signal is checked against an autograd gradient
    of its loss, and memory Frobenius norms are non-increasing;
  * eta == 0 / alpha_t == 1 overrides give the closed forms X_0 prod(alpha) / X_0;
  * chunk length 1 equals an independently written token-wise loop; one chunk
    spanning the sequence generates every token from the initial states;
  * five-memory form equals the single-product form to 1e-12;
  * one-hot fusion scales isolate routes; batch permutation equivariance;
  * hard injection clamp: eta1 g <= 1 - alpha_t with equality where it binds, eta1 =
    eta0 elsewhere; no binds for tiny steps (then it matches the soft cap to O(z^2)),
    every token binds for huge steps; norms stay non-increasing; chunk 1 equals the
    token-wise loop;
  * standalone sequence layer: chunk 1 equals the token-wise loop, outputs are causal
    (a prefix of the input gives the prefix of the output), absent queries mean x, and
    it equals route 0 of the operator with W_q = I and a one-hot route-0 scale.
The end-to-end numbers are *not* pinned by printed values (the pages print
none); they are pinned only through the properties above.
"""
from __future__ import annotations

from typing import Dict, Optional, Tuple

import numpy as np

ROUTES = 4
_PHI_SERIES_BELOW = 1e-6


# --------------------------------------------------------------------------
# Routes  ([OVERVIEW] "Four-Directional Scanning and Spatial Chunking";
#          [SUMMARY] 2D-maps paragraph)
# --------------------------------------------------------------------------
def route_index_map(H: int, W: int, route: int) -> np.ndarray:
    """Raster index p = i*W + j of the t-th token of ``route``.

    route 0: forward row-major; 1: reverse row-major; 2: forward column-major
    (t = j*H + i); 3: reverse column-major.
    """
    N = H * W
    t = np.arange(N, dtype=np.int64)
    if route == 0:
        return t
    if route == 1:
        return (N - 1) - t
    col = t // H
    row = t % H
    colmajor = row * W + col
    if route == 2:
        return colmajor
    if route == 3:
        return colmajor[::-1].copy()
    raise ValueError("route must be 0..3")


def default_chunk(H: int, W: int, route: int, chunk_row: int = 0, chunk_col: int = 0) -> int:
    """Row routes chunk by full rows (W), column routes by full columns (H)."""
    if route in (0, 1):
        return chunk_row if chunk_row > 0 else W
    return chunk_col if chunk_col > 0 else H


def gather(x: np.ndarray, route: int) -> np.ndarray:
    """[B, H, W, C] -> route order [B, N, C]."""
    B, H, W, C = x.shape
    return x.reshape(B, H * W, C)[:, route_index_map(H, W, route)]


def restore(xr: np.ndarray, route: int, H: int, W: int) -> np.ndarray:
    """Route order [B, N, C] -> [B, H, W, C] (inverse of ``gather``)."""
    B, N, C = xr.shape
    out = np.empty_like(xr)
    out[:, route_index_map(H, W, route)] = xr
    return out.reshape(B, H, W, C)


# --------------------------------------------------------------------------
# Gates ([SUMMARY] stability paragraph; [OVERVIEW] "Why the Stability Controls
# Matter")
# --------------------------------------------------------------------------
def stabilized_key(ktil: np.ndarray, eps: float) -> np.ndarray:
    """Stabilized L2 normalisation k = k~ / sqrt(||k~||^2 + eps) (keys only)."""
    n2 = np.sum(ktil * ktil, axis=-1, keepdims=True)
    return ktil / np.sqrt(n2 + eps)


def sigmoid(z: np.ndarray) -> np.ndarray:
    out = np.empty_like(z)
    pos = z >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-z[pos]))
    ez = np.exp(z[~pos])
    out[~pos] = ez / (1.0 + ez)
    return out


def softplus(z: np.ndarray) -> np.ndarray:
    return np.maximum(z, 0.0) + np.log1p(np.exp(-np.abs(z)))


def retention(beta: np.ndarray, alpha_max: float) -> np.ndarray:
    """Reading: alpha_t = min(sigmoid(beta_t), alpha); beta from the retention memory."""
    return np.minimum(sigmoid(beta), alpha_max)


def soft_cap(eta0: np.ndarray, gain: np.ndarray, alpha_t: np.ndarray) -> np.ndarray:
    """Soft injection cap: eta1 = eta0 * phi(eta0 * g / (1 - alpha_t)), phi(z) = tanh(z)/z.

    So eta1 * g = (1 - alpha_t) * tanh(eta0 * g / (1 - alpha_t)) stays strictly
    inside the retention margin, smoothly (no clipping), and eta1 ~ eta0 for
    small steps.  g = ||k - v|| * ||k|| is the key-value discrepancy gain.
    """
    z = eta0 * gain / (1.0 - alpha_t)
    small = z < _PHI_SERIES_BELOW
    zs = np.where(small, 1.0, z)
    phi = np.where(small, 1.0 - z * z / 3.0, np.tanh(zs) / zs)
    return eta0 * phi


def hard_cap(eta0: np.ndarray, gain: np.ndarray, alpha_t: np.ndarray):
    """Hard injection clamp, the ablation of the soft cap ([SUMMARY] results paragraph:
    "hard injection clamp", active on a share of token updates; [SUMMARY] stability list:
    the soft cap limits the step smoothly rather than by clipping).  Reading: clip the
    step so that eta1 * g <= 1 - alpha_t, i.e. eta1 = min(eta0, (1 - alpha_t) / g).
    Returns (eta1, binds) with binds = eta0 * g > 1 - alpha_t (the clamp is active).
    """
    margin = 1.0 - alpha_t
    binds = eta0 * gain > margin
    safe = np.where(binds, gain, 1.0)
    return np.where(binds, margin / safe, eta0), binds


def spectral_clamp(eta1: np.ndarray, knorm2: np.ndarray) -> np.ndarray:
    """eta = min(eta1, 2 / ||k||^2): then alpha_t (I - eta k k^T) has norm alpha_t."""
    over = eta1 * knorm2 > 2.0
    safe = np.where(over, knorm2, 1.0)
    return np.where(over, 2.0 / safe, eta1)


def gates(ktil, v, a, beta, alpha_max, eps, cap="soft"):
    """All per-token scalars/vectors from the generated quantities.

    Returns dict with k (normalised key), alpha_t, eta0 (proposed step), eta1
    (after the injection cap: ``cap`` = "soft" or "hard"), eta (after the spectral
    clamp), gain, and binds (where the hard clamp is active; all False for "soft").
    """
    k = stabilized_key(ktil, eps)
    alpha_t = retention(beta, alpha_max)
    eta0 = softplus(a)
    kn = np.sqrt(np.sum(k * k, axis=-1))
    gain = np.sqrt(np.sum((k - v) ** 2, axis=-1)) * kn
    if cap == "soft":
        eta1, binds = soft_cap(eta0, gain, alpha_t), np.zeros(eta0.shape, dtype=bool)
    elif cap == "hard":
        eta1, binds = hard_cap(eta0, gain, alpha_t)
    else:
        raise ValueError(cap)
    eta = spectral_clamp(eta1, kn * kn)
    return dict(k=k, alpha_t=alpha_t, eta0=eta0, eta1=eta1, eta=eta, gain=gain, binds=binds)


# --------------------------------------------------------------------------
# Retained Delta Gradient Descent write ([SUMMARY] write-rule paragraph)
# --------------------------------------------------------------------------
def l2_signal(Xm: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """Gradient of 0.5 * ||X k - vhat||^2 with the private target vhat = X v held fixed.

    Xm: [S, m, d] (m = d for a matrix memory, 1 for a vector memory, or the
    five memories stacked row-wise); k, v: [S, d].  Returns (X k - X v) k^T.
    """
    Xk = np.matmul(Xm, k[:, :, None])
    vhat = np.matmul(Xm, v[:, :, None])
    return (Xk - vhat) * k[:, None, :]


def retained_write(Xm, k, v, eta, alpha_t):
    """One write: X <- X alpha_t (I - eta k k^T) - eta * L2 signal.

    The retained transition alpha_t (I - eta k k^T) carries the residual
    correction at the current key; the signal term is the rank-one gradient
    write.  eta, alpha_t: [S].
    """
    Xk = np.matmul(Xm, k[:, :, None])
    retained = alpha_t[:, None, None] * (Xm - eta[:, None, None] * Xk * k[:, None, :])
    return retained - eta[:, None, None] * l2_signal(Xm, k, v)


MEMORIES = ("M_mem", "M_k", "M_v", "m_eta", "m_alpha")


def _stack(inits, d):
    """Five memories stacked row-wise: rows [0,d) M_mem, [d,2d) M_k, [2d,3d) M_v,
    row 3d m_eta, row 3d+1 m_alpha.  The write acts on every row of every memory
    independently (each row is a row vector times the same right factor), so
    one array holds all five without changing any arithmetic."""
    return np.concatenate([np.asarray(inits["M_mem"], np.float64), np.asarray(inits["M_k"], np.float64),
                           np.asarray(inits["M_v"], np.float64),
                           np.asarray(inits["m_eta"], np.float64)[:, None, :],
                           np.asarray(inits["m_alpha"], np.float64)[:, None, :]], axis=1)


def _unstack(mem, d):
    return {"M_mem": mem[:, 0:d], "M_k": mem[:, d:2 * d], "M_v": mem[:, 2 * d:3 * d],
            "m_eta": mem[:, 3 * d], "m_alpha": mem[:, 3 * d + 1]}


def _generate(mem, d, X):
    """Generation from the memories: k~ = M_k x, v = M_v x, a = m_eta x, beta = m_alpha x.

    One matmul of the generating rows (M_k, M_v, m_eta, m_alpha) with the chunk's tokens.
    """
    gen = np.matmul(X, np.swapaxes(mem[:, d:], 1, 2))   # [S, Lc, 2d + 2]
    return gen[..., :d], gen[..., d:2 * d], gen[..., 2 * d], gen[..., 2 * d + 1]


def scan_five_memory(xs, qs, inits, chunk, alpha_max, eps, *, readout="post",
                     eta_override=None, alpha_override=None, trace=False, cap="soft", counter=None):
    """The chunked scan over S independent sequences, literally with five memories.

    xs, qs: [S, N, d] float64 (memory input x_t and query q_t, route order).
    inits: dict M_mem, M_k, M_v [S, d, d]; m_eta, m_alpha [S, d].
    At each chunk start the *boundary* memories generate k~, v, a, beta for every
    token of the chunk ([OVERVIEW] "Four-Directional Scanning ..."; [SUMMARY]
    2D-maps paragraph); the working memories are then written in token order
    and the content memory is read after each token's write (reading: post-write
    readout).  The boundary refreshes at the end of the chunk.  The final chunk
    may be shorter than ``chunk`` ([README] "SRNL and VisionHOPE operator").

    ``cap`` selects the soft cap or the hard clamp; ``counter`` (a one-element list) collects
    the number of token updates where the hard clamp is active.
    Returns y [S, N, d], final memories dict, and a trace dict when asked.
    """
    S, N, d = xs.shape
    mem = _stack(inits, d)
    y = np.zeros((S, N, d))
    tr = None
    if trace:
        tr = {key: np.zeros((S, N)) for key in ("alpha_t", "eta0", "eta1", "eta", "gain")}
        tr["k"] = np.zeros((S, N, d))
        tr["v"] = np.zeros((S, N, d))
        tr["fro"] = {name: np.zeros((S, N + 1)) for name in MEMORIES}
        tr["states"] = np.zeros((S, N + 1) + mem.shape[1:]) if N <= 256 else None

        def record(t, m):
            parts = _unstack(m, d)
            for name in MEMORIES:
                p = parts[name]
                tr["fro"][name][:, t] = np.sqrt(np.sum(p * p, axis=tuple(range(1, p.ndim))))
            if tr["states"] is not None:
                tr["states"][:, t] = m
        record(0, mem)
    for c0 in range(0, N, chunk):
        c1 = min(c0 + chunk, N)
        ktil, v, a, beta = _generate(mem, d, xs[:, c0:c1])
        gt = gates(ktil, v, a, beta, alpha_max, eps, cap)
        if counter is not None:
            counter[0] += int(np.count_nonzero(gt["binds"]))
        eta = gt["eta"] if eta_override is None else np.full_like(gt["eta"], eta_override)
        alpha_t = gt["alpha_t"] if alpha_override is None else np.full_like(gt["alpha_t"], alpha_override)
        for j in range(c1 - c0):
            t = c0 + j
            if readout == "pre":
                y[:, t] = np.matmul(mem[:, :d], qs[:, t, :, None])[..., 0]
            mem = retained_write(mem, gt["k"][:, j], v[:, j], eta[:, j], alpha_t[:, j])
            if readout == "post":
                y[:, t] = np.matmul(mem[:, :d], qs[:, t, :, None])[..., 0]
            if trace:
                tr["alpha_t"][:, t] = alpha_t[:, j]
                tr["eta"][:, t] = eta[:, j]
                for key in ("eta0", "eta1", "gain"):
                    tr[key][:, t] = gt[key][:, j]
                tr["k"][:, t] = gt["k"][:, j]
                tr["v"][:, t] = v[:, j]
                record(t + 1, mem)
    return y, {k_: np.array(v_) for k_, v_ in _unstack(mem, d).items()}, tr


def scan_qform(xs, qs, inits, chunk, alpha_max, eps):
    """Second, independent coding of the same scan: every memory is X_0 Q_t.

    Every write right-multiplies a memory by the same matrix
    T_t = alpha_t I - eta_t u_t k_t^T with u_t = (1 + alpha_t) k_t - v_t, so the
    five memories share one product Q_t = T_1 ... T_t.  This form is derived
    from the write rule (not stated on the pages) and used only to cross-check
    ``scan_five_memory``.
    """
    S, N, d = xs.shape
    G_k = inits["M_k"].astype(np.float64)
    G_v = inits["M_v"].astype(np.float64)
    g_e = inits["m_eta"].astype(np.float64)
    g_a = inits["m_alpha"].astype(np.float64)
    M_mem = inits["M_mem"].astype(np.float64)
    Q = np.broadcast_to(np.eye(d), (S, d, d)).copy()
    y = np.zeros((S, N, d))
    eye = np.eye(d)
    for c0 in range(0, N, chunk):
        c1 = min(c0 + chunk, N)
        Xc = xs[:, c0:c1]
        Qx = np.einsum("sij,stj->sti", Q, Xc)                      # Q_b x_t
        ktil = np.einsum("sij,stj->sti", G_k, Qx)
        v = np.einsum("sij,stj->sti", G_v, Qx)
        a = np.einsum("sj,stj->st", g_e, Qx)
        beta = np.einsum("sj,stj->st", g_a, Qx)
        gt = gates(ktil, v, a, beta, alpha_max, eps)
        for j in range(c1 - c0):
            k, vv = gt["k"][:, j], v[:, j]
            al, et = gt["alpha_t"][:, j], gt["eta"][:, j]
            u = (1.0 + al)[:, None] * k - vv
            T = al[:, None, None] * eye[None] - et[:, None, None] * u[:, :, None] * k[:, None, :]
            Q = np.einsum("sij,sjk->sik", Q, T)
            y[:, c0 + j] = np.einsum("sij,sj->si", M_mem, np.einsum("sij,sj->si", Q, qs[:, c0 + j]))
    final = {
        "M_mem": M_mem @ Q, "M_k": G_k @ Q, "M_v": G_v @ Q,
        "m_eta": np.einsum("sj,sjk->sk", g_e, Q), "m_alpha": np.einsum("sj,sjk->sk", g_a, Q),
    }
    return y, final


def scan_tokenwise(xs, qs, inits, alpha_max, eps, cap="soft"):
    """Pure token-wise recurrence: every token is generated from X_{t-1}.

    Written without any chunk bookkeeping; the chunked scan with chunk length 1
    must reproduce it.
    """
    S, N, d = xs.shape
    Mm = inits["M_mem"].astype(np.float64).copy()
    Mk = inits["M_k"].astype(np.float64).copy()
    Mv = inits["M_v"].astype(np.float64).copy()
    me = inits["m_eta"].astype(np.float64).copy()
    ma = inits["m_alpha"].astype(np.float64).copy()
    y = np.zeros((S, N, d))
    for t in range(N):
        x = xs[:, t]
        ktil = np.einsum("sij,sj->si", Mk, x)
        v = np.einsum("sij,sj->si", Mv, x)
        a = np.einsum("sj,sj->s", me, x)
        beta = np.einsum("sj,sj->s", ma, x)
        k = ktil / np.sqrt(np.sum(ktil ** 2, axis=1, keepdims=True) + eps)
        al = np.minimum(sigmoid(beta), alpha_max)
        e0 = softplus(a)
        kn2 = np.sum(k ** 2, axis=1)
        g = np.sqrt(np.sum((k - v) ** 2, axis=1) * kn2)
        e1 = soft_cap(e0, g, al) if cap == "soft" else np.minimum(e0, (1.0 - al) / np.maximum(g, 1e-300))
        e = spectral_clamp(e1, kn2)

        def write(X):  # X: [S, m, d]
            Xk = np.einsum("smd,sd->sm", X, k)
            Xv = np.einsum("smd,sd->sm", X, v)
            return (al[:, None, None] * X
                    - (al * e)[:, None, None] * Xk[:, :, None] * k[:, None, :]
                    - e[:, None, None] * (Xk - Xv)[:, :, None] * k[:, None, :])

        Mm, Mk, Mv = write(Mm), write(Mk), write(Mv)
        me = write(me[:, None, :])[:, 0, :]
        ma = write(ma[:, None, :])[:, 0, :]
        y[:, t] = np.einsum("sij,sj->si", Mm, qs[:, t])
    return y, dict(M_mem=Mm, M_k=Mk, M_v=Mv, m_eta=me, m_alpha=ma)


# --------------------------------------------------------------------------
# Operator: shared query projection, four routes, restore + channel fusion
# ([README] "Overview" item 3 and "SRNL and VisionHOPE operator";
#  [OVERVIEW] "Four-Directional Scanning and Spatial Chunking";
#  [SUMMARY] 2D-maps and caveats paragraphs)
# --------------------------------------------------------------------------
def query_projection(x: np.ndarray, W_q: np.ndarray) -> np.ndarray:
    """q = x W_q^T over channels; shared by all routes, outside the recurrence."""
    return np.einsum("bhwc,oc->bhwo", x, W_q)


def _route_inits(inputs_params, route, B):
    """Per-route initial states broadcast over the batch, sequences ordered (b, head)."""
    out = {}
    for key, name in (("M_mem0", "M_mem"), ("M_k0", "M_k"), ("M_v0", "M_v"),
                      ("m_eta0", "m_eta"), ("m_alpha0", "m_alpha")):
        arr = np.asarray(inputs_params[key], dtype=np.float64)[route]  # [heads, ...]
        out[name] = np.broadcast_to(arr[None], (B,) + arr.shape).reshape((-1,) + arr.shape[1:]).copy()
    return out


def operator_forward(x, params, *, alpha_max, eps=1e-6, chunk_row=0, chunk_col=0,
                     heads, scan="five", readout="post", eta_override=None,
                     alpha_override=None, trace=False, cap="soft", counter=None):
    """Full forward of the four-direction scan.

    x: [B, H, W, C] (any float; promoted to float64).  params: dict with W_q
    [C, C], scales [4, C], M_mem0/M_k0/M_v0 [4, heads, d, d], m_eta0/m_alpha0
    [4, heads, d].  Channels-last layout; each head reads its own d-channel
    slice of x (reading: no input projection) and of q.
    Returns out [B, H, W, C], finals [4, B, heads, 3 d^2 + 2 d] (M_mem, M_k,
    M_v row-major, then m_eta, m_alpha), and per-route traces when asked.
    """
    x = np.asarray(x, dtype=np.float64)
    B, H, W, C = x.shape
    d = C // heads
    N = H * W
    q = query_projection(x, np.asarray(params["W_q"], dtype=np.float64))
    scales = np.asarray(params["scales"], dtype=np.float64)
    out = np.zeros((B, H, W, C))
    finals = np.zeros((ROUTES, B, heads, 3 * d * d + 2 * d))
    traces = []
    for r in range(ROUTES):
        L = default_chunk(H, W, r, chunk_row, chunk_col)
        xr = gather(x, r).reshape(B, N, heads, d).transpose(0, 2, 1, 3).reshape(B * heads, N, d)
        qr = gather(q, r).reshape(B, N, heads, d).transpose(0, 2, 1, 3).reshape(B * heads, N, d)
        inits = _route_inits(params, r, B)
        if scan == "five":
            y, fin, tr = scan_five_memory(xr, qr, inits, L, alpha_max, eps, readout=readout,
                                          eta_override=eta_override, alpha_override=alpha_override,
                                          trace=trace, cap=cap, counter=counter)
            traces.append(tr)
        elif scan == "qform":
            y, fin = scan_qform(xr, qr, inits, L, alpha_max, eps)
        elif scan == "tokenwise":
            y, fin = scan_tokenwise(xr, qr, inits, alpha_max, eps, cap)
        else:
            raise ValueError(scan)
        yr = y.reshape(B, heads, N, d).transpose(0, 2, 1, 3).reshape(B, N, C)
        out += scales[r][None, None, None, :] * restore(yr, r, H, W)
        flat = np.concatenate([fin["M_mem"].reshape(B * heads, -1), fin["M_k"].reshape(B * heads, -1),
                               fin["M_v"].reshape(B * heads, -1), fin["m_eta"].reshape(B * heads, -1),
                               fin["m_alpha"].reshape(B * heads, -1)], axis=1)
        finals[r] = flat.reshape(B, heads, -1)
    return out, finals, (traces if trace else None)


def sequence_forward(x, params, *, alpha_max, eps=1e-6, chunk=64, heads, queries=None, scan="five",
                     cap="soft", counter=None):
    """Standalone SRNL layer on sequences ([README] "SRNL and VisionHOPE operator": a layer
    on [batch, tokens, dim] that returns the same shape, one pass in token order, 64-token
    chunks unless told otherwise, an incomplete final chunk allowed; queries of the same shape
    may be supplied, otherwise x itself is the query; every call starts a new sequence).

    x, queries: [B, T, D].  params: M_mem0/M_k0/M_v0 [heads, d, d], m_eta0/m_alpha0
    [heads, d] (one set of initial states: a sequence has no routes).  Head h reads its own
    d-slice of x and of the queries (reading: no input or output projection).  chunk <= 0
    means 64.  Returns y [B, T, D] and finals [B, heads, 3 d^2 + 2 d].
    """
    x = np.asarray(x, dtype=np.float64)
    B, T, D = x.shape
    d = D // heads
    q = x if queries is None else np.asarray(queries, dtype=np.float64)
    L = chunk if chunk > 0 else 64
    xs = x.reshape(B, T, heads, d).transpose(0, 2, 1, 3).reshape(B * heads, T, d)
    qs = q.reshape(B, T, heads, d).transpose(0, 2, 1, 3).reshape(B * heads, T, d)
    inits = {}
    for key, name in (("M_mem0", "M_mem"), ("M_k0", "M_k"), ("M_v0", "M_v"),
                      ("m_eta0", "m_eta"), ("m_alpha0", "m_alpha")):
        arr = np.asarray(params[key], dtype=np.float64)  # [heads, ...]
        inits[name] = np.broadcast_to(arr[None], (B,) + arr.shape).reshape((-1,) + arr.shape[1:]).copy()
    if scan == "five":
        y, fin, _ = scan_five_memory(xs, qs, inits, L, alpha_max, eps, cap=cap, counter=counter)
    elif scan == "tokenwise":
        y, fin = scan_tokenwise(xs, qs, inits, alpha_max, eps, cap)
    else:
        raise ValueError(scan)
    y = y.reshape(B, heads, T, d).transpose(0, 2, 1, 3).reshape(B, T, D)
    finals = np.concatenate([fin["M_mem"].reshape(B * heads, -1), fin["M_k"].reshape(B * heads, -1),
                             fin["M_v"].reshape(B * heads, -1), fin["m_eta"].reshape(B * heads, -1),
                             fin["m_alpha"].reshape(B * heads, -1)], axis=1).reshape(B, heads, -1)
    return y, finals


def forward_from_inputs(inp, **kw):
    """Convenience: run ``operator_forward`` on a ``srnl_inputs.ScanInputs``."""
    cfg = inp.cfg
    return operator_forward(inp.x32, inp.params(), alpha_max=cfg.alpha, eps=cfg.eps,
                            chunk_row=cfg.chunk_row, chunk_col=cfg.chunk_col,
                            heads=cfg.heads, **kw)


def rel_fro(a: np.ndarray, b: np.ndarray) -> float:
    """||a - b||_F / ||b||_F (0 when both vanish)."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b.ravel())
    na = np.linalg.norm((a - b).ravel())
    if nb == 0.0:
        return 0.0 if na == 0.0 else float("inf")
    return float(na / nb)
