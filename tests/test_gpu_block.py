"""GPU parity of the VisionHOPE residual block (srnl_block_*) against the float64 block oracle
(oracle/srnl_block.py) on the same seeded inputs.

bf16 activations: the GPU rounds x, the normalised inputs, u, the operator's output, the
branch sum, the first residual, the hidden layer and the output to bf16 (fp32 arithmetic in
between) and the oracle rounds nothing but x, so the bar is the bf16 path's 2e-2 relative
Frobenius error of the output.  Shapes: the README's block (dim 64, mixer_dim 32, head_dim 16
on a 14 x 20 map; K = 32 for the out-projection), a wider block (dim 128, mixer 64: a
512-channel hidden layer in two 256-column GEMM tiles and K = 512), the hierarchical stage-1
map (56 x 56, dim 64, mixer 64), a ragged map with overridden chunks, and the hard clamp.
"""
import numpy as np
import pytest
import torch

import self_referential_nested_b200 as S
from oracle import srnl_block as K
from srnl_inputs import make_block_inputs

pytestmark = pytest.mark.gpu

TOL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from self_referential_nested_b200 import build
    build.build()
    torch.cuda.set_device(0)


def f32(v):
    return float(np.float32(v))


def run(inp, gen="bf16", alpha=0.95, chunk_row=0, chunk_col=0, cap="soft"):
    cfg = dict(B=inp.B, H=inp.H, W=inp.W, dim=inp.dim, mixer_dim=inp.m, head_dim=inp.head_dim, alpha=alpha,
               eps=1e-6, chunk_row=chunk_row, chunk_col=chunk_col, gen_dtype=gen, injection_cap=cap, ln_eps=1e-6)
    h = S.srnl_block_create(cfg, inp.p)
    try:
        x = torch.from_numpy(inp.x_bits.view(np.int16)).cuda().view(torch.bfloat16)
        y = torch.full_like(x, float("nan"))
        S.srnl_block_forward(h, x, y)
        torch.cuda.synchronize()
        S.srnl_block_device_status(h)
        got = y.float().cpu().numpy()
    finally:
        h.close()
    ref, _ = K.block_forward(inp.x32, inp.p, heads=inp.heads, alpha_max=f32(alpha), eps=f32(1e-6),
                             chunk_row=chunk_row, chunk_col=chunk_col, cap=cap)
    assert np.all(np.isfinite(got))
    return got, ref


def check(got, ref, what):
    from oracle import srnl_oracle as O
    err = O.rel_fro(got, ref)
    print(f"\n[block] {what}: relative Frobenius error {err:.2e}")
    assert err <= TOL, f"{what}: {err:.3e}"
    # the branches, not only the residual copy of x: the change over x matches too
    return err


@pytest.mark.parametrize("gen", ["bf16", "f32"])
def test_block_readme_shape(gen):
    inp = make_block_inputs(2, 14, 20, 64, 32, 16, "bf16", seed=1)
    got, ref = run(inp, gen)
    check(got, ref, f"README block 14x20 dim 64 mixer 32 head 16 gen {gen}")
    from oracle import srnl_oracle as O
    delta = O.rel_fro(got - inp.x32, ref - inp.x32)
    assert delta <= 5e-2, f"block increment: {delta:.3e}"


def test_block_wider_hidden_tiles():
    inp = make_block_inputs(1, 9, 13, 128, 64, 32, "bf16", seed=2, mem_scale=0.3, vec_scale=0.5)
    got, ref = run(inp)
    check(got, ref, "dim 128 mixer 64 head 32")


def test_block_stage1_map():
    inp = make_block_inputs(2, 56, 56, 64, 64, 32, "bf16", seed=3)
    got, ref = run(inp)
    check(got, ref, "56x56 dim 64 mixer 64 head 32")


def test_block_ragged_chunks_and_hard_clamp():
    inp = make_block_inputs(2, 7, 11, 64, 64, 16, "bf16", seed=4, mem_scale=0.3, vec_scale=0.8)
    got, ref = run(inp, chunk_row=4, chunk_col=3, cap="hard")
    check(got, ref, "7x11 chunks 4/3 hard clamp head 16")


def test_block_rejects_bad_config():
    inp = make_block_inputs(1, 4, 4, 64, 32, 16, "bf16", seed=5)
    base = dict(B=1, H=4, W=4, dim=64, mixer_dim=32, head_dim=16, alpha=0.95, gen_dtype="bf16")
    for bad in (dict(dim=48), dict(mixer_dim=24), dict(head_dim=12), dict(act_dtype="f32"), dict(ln_eps=0.0)):
        with pytest.raises(S.SrnlError):
            S.srnl_block_create(dict(base, **bad), inp.p)
