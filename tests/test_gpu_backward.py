"""GPU parity of the backward pass: srnl_scan_backward through the C ABI against the float64
gradient oracle (reverse mode through the literal five-memory recurrence, pinned by finite
differences), on the same seeded inputs and upstream gradients.

Tolerances (relative Frobenius error per gradient tensor):
  * 1e-4 for every gradient computed from fp32 inputs, and for the parameter gradients
    when x and dy are bf16 (both sides read the same rounded values; the GPU arithmetic is
    fp32 throughout, like the forward's fp32 path, which holds 1e-4);
  * 1e-2 for dx when it is returned in bf16: rounding each element to bf16 alone gives a
    relative error up to 2^-9 ~ 2e-3 per element.
"""
import functools

import numpy as np
import pytest
import torch

import self_referential_nested_b200 as S
from oracle import srnl_grad as GR
from oracle import srnl_oracle as O
from srnl_inputs import CONFIGS, ScanConfig, bf16_round_bits, make_cotangent, make_inputs

pytestmark = pytest.mark.gpu

TOL = 1e-4
TOL_DX_BF16 = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from self_referential_nested_b200 import build
    build.build()
    torch.cuda.set_device(0)


def _dev(a32, act):
    if act == "bf16":
        return torch.from_numpy(bf16_round_bits(a32).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a32, dtype=np.float32)).cuda()


def gpu_backward(inp, dout, act, cap="soft", keys=S.GRAD_KEYS, params=None):
    cfg = inp.cfg
    params = params or inp.params()
    h = S.srnl_scan_create(dict(B=cfg.B, H=cfg.H, W=cfg.W, C=cfg.C, heads=cfg.heads, d=cfg.d, alpha=cfg.alpha,
                                eps=cfg.eps, chunk_row=cfg.chunk_row, chunk_col=cfg.chunk_col, act_dtype=act,
                                gen_dtype="f32", injection_cap=cap), params)
    try:
        x = _dev(inp.x32, act)
        dy = _dev(dout, act)
        dx = torch.full_like(x, float("nan"))
        grads = {k: torch.full(np.shape(params[k]), float("nan"), device="cuda") for k in keys}
        S.srnl_scan_backward(h, x, dy, dx, grads)
        torch.cuda.synchronize()
        out = {k: v.cpu().numpy() for k, v in grads.items()}
        out["x"] = dx.float().cpu().numpy()
        return out
    finally:
        h.close()


def check(got, ref, act, what=""):
    for key, val in got.items():
        bound = TOL_DX_BF16 if (key == "x" and act == "bf16") else TOL
        assert np.all(np.isfinite(val)), f"{what} {key}: non-finite values"
        err = O.rel_fro(val, ref[key])
        assert err <= bound, f"{what} {key}: relative Frobenius error {err:.3e} > {bound:.0e}"


def run_case(cfg, act, cap="soft", seed=0, mem_scale=0.02, vec_scale=0.1, keys=S.GRAD_KEYS):
    inp = make_inputs(cfg.replace(act_dtype=act), seed=seed, mem_scale=mem_scale, vec_scale=vec_scale)
    dout = make_cotangent(inp.x32.shape, seed=seed, act_dtype=act)
    got = gpu_backward(inp, dout, act, cap, keys)
    ref = GR.backward_from_inputs(inp, dout, cap=cap)
    check(got, ref, act, f"{cfg.name} {act} {cap}")
    return got, ref


def _cfg(name, **kw):
    base = dict(name=name, B=1, H=8, W=8, C=64, heads=2, d=32, alpha=0.95, act_dtype="f32")
    base.update(kw)
    return ScanConfig(**base)


def test_backward_pr1_8x8_f32():
    run_case(CONFIGS["pr1_8x8"], "f32")


@pytest.mark.parametrize("act", ["f32", "bf16"])
def test_backward_ragged_chunks(act):
    """Chunk overrides that leave a short last chunk on every route, and sub-blocks that
    straddle chunk ends (7 x 13 map, row chunks of 5, column chunks of 3)."""
    run_case(_cfg("ragged", B=2, H=7, W=13, chunk_row=5, chunk_col=3), act, seed=1)


def test_backward_single_token_map():
    run_case(_cfg("one", B=2, H=1, W=1), "f32", seed=9)


def test_backward_long_chunks_span_segments():
    """Row chunks of 150 tokens: several gate segments and sub-blocks per chunk."""
    run_case(_cfg("long", B=1, H=3, W=150), "f32", seed=2)


@pytest.mark.parametrize("cap", ["soft", "hard"])
def test_backward_active_gates(cap):
    """Large initial memories: the cap saturates, the hard clamp is active on part of the
    tokens, the retention clamp acts (alpha reached) on others."""
    cfg = _cfg("active", B=2, H=6, W=10, chunk_row=4, chunk_col=0)
    inp = make_inputs(cfg, seed=3, mem_scale=0.3, vec_scale=0.8)
    counter = [0]
    O.operator_forward(inp.x32, inp.params(), alpha_max=cfg.alpha, chunk_row=4, heads=cfg.heads, cap="hard",
                       counter=counter)
    assert counter[0] > 0
    run_case(cfg, "f32", cap, seed=3, mem_scale=0.3, vec_scale=0.8)


@pytest.mark.parametrize("d", [4, 8, 16])
def test_backward_small_head_dims(d):
    run_case(_cfg(f"d{d}", B=2, H=5, W=6, C=2 * d, heads=2, d=d), "f32", seed=4, mem_scale=0.2, vec_scale=0.5)


def test_backward_s3_shape_bf16():
    run_case(CONFIGS["hier_s3_14x14"].replace(B=2), "bf16", seed=5)


def test_backward_plain_shape_bf16():
    run_case(CONFIGS["plain_14x14"].replace(B=1), "bf16", seed=6)


def test_backward_without_parameter_gradients():
    cfg = _cfg("dxonly", B=1, H=4, W=9)
    inp = make_inputs(cfg, seed=7)
    dout = make_cotangent(inp.x32.shape, seed=7)
    ref = GR.backward_from_inputs(inp, dout)
    got = gpu_backward(inp, dout, "f32", keys=())
    check(got, ref, "f32", "dx only")
    got = gpu_backward(inp, dout, "f32", keys=("M_v0", "scales"))
    check(got, ref, "f32", "two gradients")


def test_backward_repeatable():
    """Two calls on one handle give identical results (deterministic reductions)."""
    cfg = _cfg("rep", B=2, H=6, W=7)
    inp = make_inputs(cfg, seed=8)
    dout = make_cotangent(inp.x32.shape, seed=8)
    h = S.srnl_scan_create(dict(B=2, H=6, W=7, C=64, heads=2, d=32, alpha=0.95, act_dtype="f32",
                                gen_dtype="f32"), inp.params())
    try:
        x, dy = _dev(inp.x32, "f32"), _dev(dout, "f32")
        outs = []
        for _ in range(2):
            dx = torch.empty_like(x)
            g = {k: torch.empty(np.shape(inp.params()[k]), device="cuda") for k in S.GRAD_KEYS}
            S.srnl_scan_backward(h, x, dy, dx, g)
            outs.append([dx.cpu()] + [g[k].cpu() for k in S.GRAD_KEYS])
        torch.cuda.synchronize()
        for a, b in zip(*outs):
            assert torch.equal(a, b)
    finally:
        h.close()


def test_backward_rejects_bf16_generation():
    inp = make_inputs(_cfg("bf", act_dtype="bf16"), seed=0)
    h = S.srnl_scan_create(dict(B=1, H=8, W=8, C=64, heads=2, d=32, alpha=0.95, act_dtype="bf16",
                                gen_dtype="bf16"), inp.params())
    try:
        x = _dev(inp.x32, "bf16")
        with pytest.raises(S.SrnlError) as ei:
            S.srnl_scan_backward(h, x, x.clone(), torch.empty_like(x))
        assert ei.value.status == S.SRNL_E_UNSUPPORTED
    finally:
        h.close()


@functools.lru_cache(maxsize=None)
def _s1_full():
    cfg = CONFIGS["hier_s1_56x56"]
    inp = make_inputs(cfg, seed=0)
    dout = make_cotangent(inp.x32.shape, seed=0, act_dtype="bf16")
    return inp, dout


def test_backward_s1_full_size_bf16():
    """hier_s1_56x56 at B = 32 (the forward bench's workload, bf16 x and dy): every gradient
    against the oracle on the whole batch."""
    inp, dout = _s1_full()
    got = gpu_backward(inp, dout, "bf16")
    ref = GR.backward_from_inputs(inp, dout)
    check(got, ref, "bf16", "hier_s1_56x56 B=32")


# ---------------------------------------------------------------- head dim 64 (64-wide kernel)
def _cfg64(name, **kw):
    base = dict(name=name, B=2, H=5, W=9, C=128, heads=2, d=64, alpha=0.95, act_dtype="f32")
    base.update(kw)
    return ScanConfig(**base)


@pytest.mark.parametrize("act", ["f32", "bf16"])
def test_backward_d64_ragged_chunks(act):
    run_case(_cfg64("b64", chunk_row=4, chunk_col=2), act, seed=11)


def test_backward_d64_long_chunks_span_segments():
    """Row chunks of 40 tokens: three gate segments and five sub-blocks per chunk."""
    run_case(_cfg64("b64l", B=1, H=3, W=40), "f32", seed=12)


def test_backward_d64_active_gates_hard_cap():
    run_case(_cfg64("b64h", B=2, H=4, W=6, chunk_row=3), "f32", "hard", seed=13, mem_scale=0.2, vec_scale=0.6)
