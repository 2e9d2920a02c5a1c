"""Float64 CPU oracle for the VisionHOPE residual block around the SRNL operator.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The GPU library never
calls it and shares no code with it.

Sources (web pages describing VisionHOPE; none prints the block's equations):
  [README]   "VisionHOPE" README: "SRNL and VisionHOPE operator" (the block takes
             image features [batch, channels, height, width], preserves the shape,
             and `mixer_dim` sets its internal width).
  [OVERVIEW] "VisionHOPE Model Overview: Architecture, Benchmarks, and Practical
             Limits": "Four-Directional Scanning and Spatial Chunking" (the residual
             blocks also contain projections, normalization, depthwise convolution
             and a feed-forward network; SRNL supplies the adaptive mixing).
  [SUMMARY]  "VisionHOPE: Visual Backbones as Self-Modifying Learning Systems",
             2D-maps paragraph (a standard two-branch residual: depthwise conv for
             local context, SRNL for long range, then an FFN).

Reading of the block (the pages fix its parts, not how they are wired):
  u   = LN1(x) W_in^T + b_in                       width dim -> m (mixer_dim)
  mix = DWConv3x3(u) + operator(u)                 the two branches, summed
  y   = x + mix W_out^T + b_out                    first residual
  out = y + GELU(LN2(y) W_1^T + b_1) W_2^T + b_2   second residual, hidden width 4 dim
LayerNorm over channels with learned scale and shift (eps 1e-6); the depthwise
convolution is 3 x 3 per channel with zero padding and a bias; GELU is the exact
form v Phi(v).  Channels-last [B, H, W, C] like the operator.

Pins (tests/test_block_oracle_pins.py): LayerNorm gives zero mean and unit
variance and is invariant to a per-row affine change of its input; the centre-tap
convolution is the identity, a single off-centre tap is a shift with zero fill, and
every output of a random convolution equals its 3 x 3 window sum written out by
hand on a small map; GELU(0) = 0, GELU(v) - GELU(-v) = v and GELU(1) = Phi(1);
zero out-projections make the block the identity; with W_in = I, a centre-tap
convolution, zero fusion scales, W_out = I and a zero FFN the block is x + LN1(x);
and the operator branch enters exactly as srnl_oracle.operator_forward on u.
"""
from __future__ import annotations

from typing import Dict

import numpy as np
from scipy.special import erf

from oracle import srnl_oracle as F

LN_EPS = 1e-6


def layer_norm(x: np.ndarray, gamma: np.ndarray, beta: np.ndarray, eps: float = LN_EPS) -> np.ndarray:
    """Normalise every token's channels to zero mean and unit variance, then scale and shift."""
    x = np.asarray(x, np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * np.asarray(gamma, np.float64) + np.asarray(beta, np.float64)


def linear(x: np.ndarray, W: np.ndarray, b: np.ndarray) -> np.ndarray:
    """x W^T + b over the last axis; W[out][in]."""
    return np.einsum("...i,oi->...o", np.asarray(x, np.float64), np.asarray(W, np.float64)) + np.asarray(b, np.float64)


def dwconv3x3(u: np.ndarray, w: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Depthwise 3 x 3 convolution with zero padding: out[.., i, j, c] = b[c] +
    sum_{di, dj in -1..1} w[c, di + 1, dj + 1] u[.., i + di, j + dj, c]."""
    u = np.asarray(u, np.float64)
    w = np.asarray(w, np.float64)
    B, H, W, C = u.shape
    pad = np.zeros((B, H + 2, W + 2, C))
    pad[:, 1:H + 1, 1:W + 1] = u
    out = np.broadcast_to(np.asarray(b, np.float64), (B, H, W, C)).copy()
    for di in range(3):
        for dj in range(3):
            out += w[:, di, dj] * pad[:, di:di + H, dj:dj + W]
    return out


def gelu(v: np.ndarray) -> np.ndarray:
    """Exact GELU: v Phi(v) with Phi the standard normal CDF, Phi(v) = (1 + erf(v / sqrt 2)) / 2."""
    v = np.asarray(v, np.float64)
    return 0.5 * v * (1.0 + erf(v / np.sqrt(2.0)))


def block_forward(x, p: Dict[str, np.ndarray], *, heads: int, alpha_max: float, eps: float = 1e-6,
                  chunk_row: int = 0, chunk_col: int = 0, ln_eps: float = LN_EPS, cap: str = "soft"):
    """One VisionHOPE residual block on channels-last x [B, H, W, dim].

    p holds ln1_g, ln1_b [dim]; W_in [m, dim], b_in [m]; dw_w [m, 3, 3], dw_b [m]; the
    operator's parameters at width m (W_q [m, m], scales [4, m], M_mem0/M_k0/M_v0
    [4, heads, d, d], m_eta0/m_alpha0 [4, heads, d]); W_out [dim, m], b_out [dim];
    ln2_g, ln2_b [dim]; W_1 [4 dim, dim], b_1 [4 dim]; W_2 [dim, 4 dim], b_2 [dim].
    Returns out [B, H, W, dim] and the intermediates (u, mix, y) for tests.
    """
    x = np.asarray(x, np.float64)
    u = linear(layer_norm(x, p["ln1_g"], p["ln1_b"], ln_eps), p["W_in"], p["b_in"])
    op_params = {k: p[k] for k in ("W_q", "scales", "M_mem0", "M_k0", "M_v0", "m_eta0", "m_alpha0")}
    glob, _, _ = F.operator_forward(u, op_params, alpha_max=alpha_max, eps=eps, chunk_row=chunk_row,
                                    chunk_col=chunk_col, heads=heads, cap=cap)
    mix = dwconv3x3(u, p["dw_w"], p["dw_b"]) + glob
    y = x + linear(mix, p["W_out"], p["b_out"])
    h = gelu(linear(layer_norm(y, p["ln2_g"], p["ln2_b"], ln_eps), p["W_1"], p["b_1"]))
    out = y + linear(h, p["W_2"], p["b_2"])
    return out, dict(u=u, mix=mix, y=y)
