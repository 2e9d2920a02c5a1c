"""Head dims 4, 8 and 16 ("VisionHOPE" README, "SRNL and VisionHOPE operator": head_dim 4,
8, 16, 32 or 64), run as zero-padded 32-wide heads, against the float64 oracle at the true
head dim: outputs and final states, both precision paths, operator and sequence layer."""
import numpy as np
import pytest
import torch

import self_referential_nested_b200 as S
from oracle import srnl_oracle as O
from srnl_inputs import ScanConfig, bf16_round_bits, make_inputs, make_seq_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from self_referential_nested_b200 import build
    build.build()
    torch.cuda.set_device(0)


def _x(x32, act):
    if act == "bf16":
        return torch.from_numpy(bf16_round_bits(x32).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).cuda()


def _tol(act, gen):
    return 1e-4 if (act == "f32" and gen == "f32") else 2e-2


@pytest.mark.parametrize("d", [4, 8, 16])
@pytest.mark.parametrize("path", [("f32", "f32"), ("bf16", "bf16")])
def test_operator_small_head_dims(d, path):
    act, gen = path
    cfg = ScanConfig("hd", B=2, H=6, W=9, C=3 * d, heads=3, d=d, alpha=0.9, act_dtype=act)
    inp = make_inputs(cfg, seed=d, mem_scale=0.3, vec_scale=1.0)
    h = S.srnl_scan_create(dict(B=cfg.B, H=cfg.H, W=cfg.W, C=cfg.C, heads=cfg.heads, d=d, alpha=cfg.alpha,
                                eps=cfg.eps, act_dtype=act, gen_dtype=gen), inp.params())
    try:
        x = _x(inp.x32, act)
        y = torch.empty_like(x)
        fin = torch.full((4, cfg.B, cfg.heads, 3 * d * d + 2 * d), float("nan"), device="cuda")
        S.srnl_scan_forward(h, x, y, fin)
        torch.cuda.synchronize()
        S.srnl_scan_device_status(h)
    finally:
        h.close()
    ref, ref_fin, _ = O.operator_forward(inp.x32, inp.params(), alpha_max=cfg.alpha, eps=cfg.eps, heads=cfg.heads)
    err = O.rel_fro(y.float().cpu().numpy(), ref)
    assert err <= _tol(act, gen), f"d={d} {path} y: {err:.3e}"
    if act == "f32" and np.linalg.norm(ref_fin) > 1e-30:
        err = O.rel_fro(fin.cpu().numpy(), ref_fin)
        assert err <= 1e-4, f"d={d} final states: {err:.3e}"


@pytest.mark.parametrize("d", [8, 16])
@pytest.mark.parametrize("path", [("f32", "f32"), ("bf16", "bf16")])
def test_sequence_small_head_dims(d, path):
    act, gen = path
    inp = make_seq_inputs(2, 40, 4 * d, 4, act, seed=30 + d)
    h = S.srnl_seq_create(dict(B=2, T=40, D=4 * d, heads=4, d=d, alpha=0.95, eps=1e-6, chunk=16, act_dtype=act,
                               gen_dtype=gen), inp.params())
    try:
        x = _x(inp.x32, act)
        q = _x(inp.q32, act)
        y = torch.empty_like(x)
        fin = torch.full((2, 4, 3 * d * d + 2 * d), float("nan"), device="cuda")
        S.srnl_seq_forward(h, x, y, q=q, final_states=fin)
        torch.cuda.synchronize()
    finally:
        h.close()
    ref, ref_fin = O.sequence_forward(inp.x32, inp.params(), alpha_max=0.95, eps=1e-6, chunk=16, heads=4,
                                      queries=inp.q32)
    err = O.rel_fro(y.float().cpu().numpy(), ref)
    assert err <= _tol(act, gen), f"seq d={d} {path} y: {err:.3e}"
    assert np.linalg.norm(ref_fin) > 1e-30
    err = O.rel_fro(fin.cpu().numpy(), ref_fin)
    assert err <= _tol(act, gen), f"seq d={d} {path} final states: {err:.3e}"
