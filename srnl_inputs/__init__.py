"""Seeded synthetic inputs for the SRNL four-direction scan.

This module is shared by the float64 oracle, the GPU parity tests and the
benchmark.  It only *draws* numbers and packs them; it holds none of the
method's arithmetic (no gates, no recurrence, no projection).

Workloads mirror the feature maps the VisionHOPE pages run the operator on
(VisionHOPE README, "Main results" / "Efficiency"; "VisionHOPE: Visual Backbones
as Self-Modifying Learning Systems", results paragraph): the 224x224
hierarchical backbone's stride-4 and stride-16 maps, the plain backbone's
patch-16 map, and the stride-4 map of a 800x1216 dense-prediction input.

Draw order for one config with seed s (numpy ``default_rng(s)``):
  1. x ~ N(0, 1), shape [B, H, W, C] (float32)
  2. ramp configs only: a ~ N(0, 1) of shape [B, H, C];
     x[b, i, j, c] += 0.5 * a[b, i, c] * (2 j / (W - 1) - 1)
  3. M_mem0, M_k0, M_v0 ~ N(0, 0.02^2), each [4, heads, d, d]
  4. m_eta0, m_alpha0 ~ N(0, 0.1^2), each [4, heads, d]
  5. W_q ~ N(0, 1 / C), shape [C, C]
Channel scales are the constant 0.25 ([4, C]).  For bf16 configs x is rounded
to bfloat16 (round to nearest even) and both sides receive those same values.

Long-sequence parity cases add a ``Sustain`` knob after the draws (it draws nothing and
changes the draw order of nothing): channel 0 of every head of x becomes the constant
``feature`` and ``retention_bias`` / ``step_bias`` are added to channel 0 of m_alpha0 /
m_eta0.  A retention logit that stays far above the clamp keeps alpha_t = alpha on every
token, so a retention cap close to 1 holds the memories inside fp32 range over thousands of
tokens; with the workload's own initials the memories halve every token and every chunk
after the first few is zero in fp32.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np

F32 = "f32"
BF16 = "bf16"


@dataclasses.dataclass(frozen=True)
class ScanConfig:
    name: str
    B: int
    H: int
    W: int
    C: int
    heads: int
    d: int
    alpha: float
    chunk_row: int = 0      # 0 -> W (full rows)
    chunk_col: int = 0      # 0 -> H (full columns)
    act_dtype: str = BF16
    x_kind: str = "normal"  # "normal" | "ramp"
    eps: float = 1e-6

    @property
    def N(self) -> int:
        return self.H * self.W

    def replace(self, **kw) -> "ScanConfig":
        return dataclasses.replace(self, **kw)


# The five workloads.  Sizes, alpha, chunking and value distributions follow the
# hot-path scope table; seed 0 throughout.
CONFIGS: Dict[str, ScanConfig] = {
    "pr1_8x8": ScanConfig("pr1_8x8", B=1, H=8, W=8, C=64, heads=2, d=32,
                          alpha=0.95, act_dtype=F32),
    "hier_s1_56x56": ScanConfig("hier_s1_56x56", B=32, H=56, W=56, C=64, heads=2,
                                d=32, alpha=0.95, act_dtype=BF16),
    "hier_s3_14x14": ScanConfig("hier_s3_14x14", B=64, H=14, W=14, C=256, heads=8,
                                d=32, alpha=0.95, act_dtype=BF16, x_kind="ramp"),
    "plain_14x14": ScanConfig("plain_14x14", B=128, H=14, W=14, C=384, heads=12,
                              d=32, alpha=0.90, act_dtype=BF16),
    "hires_200x304": ScanConfig("hires_200x304", B=2, H=200, W=304, C=64, heads=2,
                                d=32, alpha=0.95, act_dtype=BF16),
}


def bf16_round_bits(x32: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return uint16 bits."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bias = ((u >> 16) & 1) + 0x7FFF
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass
class ScanInputs:
    cfg: ScanConfig
    x32: np.ndarray                 # float32 [B,H,W,C]: the values both sides use
    x_bits: Optional[np.ndarray]    # uint16 [B,H,W,C] for bf16 configs, else None
    W_q: np.ndarray                 # float32 [C, C]
    scales: np.ndarray              # float32 [4, C]
    M_mem0: np.ndarray              # float32 [4, heads, d, d]
    M_k0: np.ndarray
    M_v0: np.ndarray
    m_eta0: np.ndarray              # float32 [4, heads, d]
    m_alpha0: np.ndarray

    def x_device_payload(self) -> np.ndarray:
        """The activation buffer as the device receives it (bf16 bits or float32)."""
        return self.x_bits if self.x_bits is not None else self.x32

    def params(self) -> Dict[str, np.ndarray]:
        return dict(W_q=self.W_q, scales=self.scales, M_mem0=self.M_mem0,
                    M_k0=self.M_k0, M_v0=self.M_v0, m_eta0=self.m_eta0,
                    m_alpha0=self.m_alpha0)


@dataclasses.dataclass(frozen=True)
class Sustain:
    """A constant feature on channel 0 of every head of x, and biases on channel 0 of the
    retention and step initials (parity cases on long sequences only)."""
    feature: float = 1.0
    retention_bias: float = 300.0
    step_bias: float = -7.0


def _apply_sustain(x: np.ndarray, m_eta0: np.ndarray, m_alpha0: np.ndarray, d: int, sus: Sustain) -> None:
    x.reshape(x.shape[:-1] + (x.shape[-1] // d, d))[..., 0] = np.float32(sus.feature)
    m_alpha0[..., 0] += np.float32(sus.retention_bias)
    m_eta0[..., 0] += np.float32(sus.step_bias)


def make_inputs(cfg: ScanConfig, seed: int = 0, *, x_scale: float = 1.0,
                mem_scale: float = 0.02, vec_scale: float = 0.1,
                sustain: Optional[Sustain] = None) -> ScanInputs:
    """Draw one workload.  ``*_scale`` and ``sustain`` knobs exist for extra parity cases only."""
    rng = np.random.default_rng(seed)
    B, H, W, C, nh, d = cfg.B, cfg.H, cfg.W, cfg.C, cfg.heads, cfg.d
    x = rng.standard_normal((B, H, W, C), dtype=np.float32) * np.float32(x_scale)
    if cfg.x_kind == "ramp":
        a = rng.standard_normal((B, H, C), dtype=np.float32)
        denom = max(W - 1, 1)
        ramp = (2.0 * np.arange(W, dtype=np.float32) / denom - 1.0).astype(np.float32)
        x = x + np.float32(0.5) * a[:, :, None, :] * ramp[None, None, :, None]
    elif cfg.x_kind != "normal":
        raise ValueError(f"unknown x_kind {cfg.x_kind!r}")
    x = x.astype(np.float32)
    M_mem0 = (rng.standard_normal((4, nh, d, d)) * mem_scale).astype(np.float32)
    M_k0 = (rng.standard_normal((4, nh, d, d)) * mem_scale).astype(np.float32)
    M_v0 = (rng.standard_normal((4, nh, d, d)) * mem_scale).astype(np.float32)
    m_eta0 = (rng.standard_normal((4, nh, d)) * vec_scale).astype(np.float32)
    m_alpha0 = (rng.standard_normal((4, nh, d)) * vec_scale).astype(np.float32)
    W_q = (rng.standard_normal((C, C)) / np.sqrt(C)).astype(np.float32)
    scales = np.full((4, C), 0.25, dtype=np.float32)
    if sustain is not None:
        _apply_sustain(x, m_eta0, m_alpha0, d, sustain)
    x_bits = None
    if cfg.act_dtype == BF16:
        x_bits = bf16_round_bits(x)
        x = bf16_bits_to_f32(x_bits).reshape(x.shape)
    elif cfg.act_dtype != F32:
        raise ValueError(f"unknown act_dtype {cfg.act_dtype!r}")
    return ScanInputs(cfg=cfg, x32=np.ascontiguousarray(x), x_bits=x_bits, W_q=W_q,
                      scales=scales, M_mem0=M_mem0, M_k0=M_k0, M_v0=M_v0,
                      m_eta0=m_eta0, m_alpha0=m_alpha0)


# ------------------------------------------------ standalone sequence layer
@dataclasses.dataclass
class SeqInputs:
    """Seeded inputs of the standalone sequence layer: x and queries [B, T, D] (fp32 values,
    bf16-exact when act_dtype is bf16) and one set of initial states per head."""
    B: int
    T: int
    D: int
    heads: int
    act_dtype: str
    x32: np.ndarray
    q32: np.ndarray
    x_bits: Optional[np.ndarray]
    q_bits: Optional[np.ndarray]
    M_mem0: np.ndarray
    M_k0: np.ndarray
    M_v0: np.ndarray
    m_eta0: np.ndarray
    m_alpha0: np.ndarray

    def params(self) -> Dict[str, np.ndarray]:
        return dict(M_mem0=self.M_mem0, M_k0=self.M_k0, M_v0=self.M_v0, m_eta0=self.m_eta0,
                    m_alpha0=self.m_alpha0)


def make_seq_inputs(B: int, T: int, D: int, heads: int, act_dtype: str = F32, seed: int = 0, *,
                    mem_scale: float = 0.02, vec_scale: float = 0.1,
                    sustain: Optional[Sustain] = None) -> SeqInputs:
    """Draw x, queries ~ N(0, 1) [B, T, D], then M_mem0, M_k0, M_v0 ~ N(0, mem_scale^2)
    [heads, d, d] and m_eta0, m_alpha0 ~ N(0, vec_scale^2) [heads, d], in that order; then
    apply ``sustain`` (to x only, not to the queries)."""
    rng = np.random.default_rng(seed)
    d = D // heads
    x = rng.standard_normal((B, T, D), dtype=np.float32)
    q = rng.standard_normal((B, T, D), dtype=np.float32)
    M_mem0 = (rng.standard_normal((heads, d, d)) * mem_scale).astype(np.float32)
    M_k0 = (rng.standard_normal((heads, d, d)) * mem_scale).astype(np.float32)
    M_v0 = (rng.standard_normal((heads, d, d)) * mem_scale).astype(np.float32)
    m_eta0 = (rng.standard_normal((heads, d)) * vec_scale).astype(np.float32)
    m_alpha0 = (rng.standard_normal((heads, d)) * vec_scale).astype(np.float32)
    if sustain is not None:
        _apply_sustain(x, m_eta0, m_alpha0, d, sustain)
    x_bits = q_bits = None
    if act_dtype == BF16:
        x_bits, q_bits = bf16_round_bits(x), bf16_round_bits(q)
        x = bf16_bits_to_f32(x_bits).reshape(x.shape)
        q = bf16_bits_to_f32(q_bits).reshape(q.shape)
    elif act_dtype != F32:
        raise ValueError(f"unknown act_dtype {act_dtype!r}")
    return SeqInputs(B=B, T=T, D=D, heads=heads, act_dtype=act_dtype, x32=np.ascontiguousarray(x),
                     q32=np.ascontiguousarray(q), x_bits=x_bits, q_bits=q_bits, M_mem0=M_mem0, M_k0=M_k0,
                     M_v0=M_v0, m_eta0=m_eta0, m_alpha0=m_alpha0)


# ------------------------------------------------ upstream gradients
def make_cotangent(shape, seed: int = 0, act_dtype: str = F32) -> np.ndarray:
    """Seeded upstream gradient dL/d(output) ~ N(0, 1) of the given shape (float32), drawn
    from its own stream (``default_rng([seed, 1])``) so that it never shifts the draws of
    ``make_inputs``.  For bf16 activations it is rounded to bfloat16 like x."""
    rng = np.random.default_rng([seed, 1])
    g = rng.standard_normal(tuple(shape), dtype=np.float32)
    if act_dtype == BF16:
        g = bf16_bits_to_f32(bf16_round_bits(g)).reshape(g.shape)
    elif act_dtype != F32:
        raise ValueError(f"unknown act_dtype {act_dtype!r}")
    return np.ascontiguousarray(g)


# ------------------------------------------------ residual block around the operator
@dataclasses.dataclass
class BlockInputs:
    """Seeded inputs of one VisionHOPE residual block: x [B, H, W, dim] (fp32 values, bf16-exact
    when act_dtype is bf16) and the block's parameters (fp32): two LayerNorms, the projection
    into and out of the mixer width m, the depthwise 3 x 3 convolution, the operator's
    parameters at width m, and the FFN (hidden width 4 dim)."""
    B: int
    H: int
    W: int
    dim: int
    m: int
    head_dim: int
    act_dtype: str
    x32: np.ndarray
    x_bits: Optional[np.ndarray]
    p: Dict[str, np.ndarray]

    @property
    def heads(self) -> int:
        return self.m // self.head_dim


def make_block_inputs(B: int, H: int, W: int, dim: int, m: int, head_dim: int, act_dtype: str = BF16,
                      seed: int = 0, *, mem_scale: float = 0.02, vec_scale: float = 0.1) -> BlockInputs:
    """Draw, in this order: x ~ N(0, 1) [B, H, W, dim]; ln1_g = 1 + N(0, 0.1^2), ln1_b ~ N(0, 0.1^2);
    W_in ~ N(0, 1/dim) [m, dim], b_in ~ N(0, 0.02^2); dw_w ~ N(0, 1/9) [m, 3, 3], dw_b ~ N(0, 0.02^2);
    the operator at width m as make_inputs draws it (M_mem0, M_k0, M_v0 ~ N(0, mem_scale^2),
    m_eta0, m_alpha0 ~ N(0, vec_scale^2), W_q ~ N(0, 1/m), scales 0.25); W_out ~ N(0, 1/m)
    [dim, m], b_out ~ N(0, 0.02^2); ln2_g, ln2_b as ln1; W_1 ~ N(0, 1/dim) [4 dim, dim],
    b_1 ~ N(0, 0.02^2); W_2 ~ N(0, 1/(4 dim)) [dim, 4 dim], b_2 ~ N(0, 0.02^2)."""
    rng = np.random.default_rng(seed)
    heads, d, hid = m // head_dim, head_dim, 4 * dim
    f = lambda a: np.ascontiguousarray(a, dtype=np.float32)
    x = rng.standard_normal((B, H, W, dim), dtype=np.float32)
    p = {}
    p["ln1_g"] = f(1.0 + 0.1 * rng.standard_normal(dim))
    p["ln1_b"] = f(0.1 * rng.standard_normal(dim))
    p["W_in"] = f(rng.standard_normal((m, dim)) / np.sqrt(dim))
    p["b_in"] = f(0.02 * rng.standard_normal(m))
    p["dw_w"] = f(rng.standard_normal((m, 3, 3)) / 3.0)
    p["dw_b"] = f(0.02 * rng.standard_normal(m))
    p["M_mem0"] = f(rng.standard_normal((4, heads, d, d)) * mem_scale)
    p["M_k0"] = f(rng.standard_normal((4, heads, d, d)) * mem_scale)
    p["M_v0"] = f(rng.standard_normal((4, heads, d, d)) * mem_scale)
    p["m_eta0"] = f(rng.standard_normal((4, heads, d)) * vec_scale)
    p["m_alpha0"] = f(rng.standard_normal((4, heads, d)) * vec_scale)
    p["W_q"] = f(rng.standard_normal((m, m)) / np.sqrt(m))
    p["scales"] = np.full((4, m), 0.25, dtype=np.float32)
    p["W_out"] = f(rng.standard_normal((dim, m)) / np.sqrt(m))
    p["b_out"] = f(0.02 * rng.standard_normal(dim))
    p["ln2_g"] = f(1.0 + 0.1 * rng.standard_normal(dim))
    p["ln2_b"] = f(0.1 * rng.standard_normal(dim))
    p["W_1"] = f(rng.standard_normal((hid, dim)) / np.sqrt(dim))
    p["b_1"] = f(0.02 * rng.standard_normal(hid))
    p["W_2"] = f(rng.standard_normal((dim, hid)) / np.sqrt(hid))
    p["b_2"] = f(0.02 * rng.standard_normal(dim))
    x_bits = None
    if act_dtype == BF16:
        x_bits = bf16_round_bits(x)
        x = bf16_bits_to_f32(x_bits).reshape(x.shape)
    elif act_dtype != F32:
        raise ValueError(f"unknown act_dtype {act_dtype!r}")
    return BlockInputs(B=B, H=H, W=W, dim=dim, m=m, head_dim=head_dim, act_dtype=act_dtype,
                       x32=np.ascontiguousarray(x), x_bits=x_bits, p=p)
