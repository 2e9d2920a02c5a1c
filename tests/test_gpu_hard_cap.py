"""GPU parity of the hard injection clamp variant (injection_cap = "hard") against the
float64 oracle: outputs within the path tolerances, and the count of token updates on which
the clamp is active.  The count is an integer decided by a floating-point comparison
(eta0 g > 1 - alpha_t); the two sides make it in fp32 and fp64 from inputs that agree only to
the path's rounding, so tokens next to the threshold may fall either way: the counts must
agree within 0.1 % (fp32 path) or 1 % (bf16 path) of the token updates, plus 2."""
import numpy as np
import pytest
import torch

import self_referential_nested_b200 as S
from oracle import srnl_oracle as O
from srnl_inputs import CONFIGS, bf16_round_bits, make_inputs, make_seq_inputs

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


def _check_count(gpu, ref, total, frac):
    assert 0 < ref < total, "the case must mix active and inactive clamps"
    assert abs(gpu - ref) <= 2 + frac * total, f"active clamps {gpu} vs oracle {ref} of {total}"


@pytest.mark.parametrize("name,act,gen,B", [("pr1_8x8", "f32", "f32", 1), ("hier_s1_56x56", "bf16", "bf16", 1),
                                            ("hier_s3_14x14", "bf16", "bf16", 2)])
def test_operator_hard_cap(name, act, gen, B):
    cfg = CONFIGS[name].replace(B=B)
    inp = make_inputs(cfg)
    h = S.srnl_scan_create(dict(B=cfg.B, H=cfg.H, W=cfg.W, C=cfg.C, heads=cfg.heads, d=cfg.d, alpha=cfg.alpha,
                                eps=cfg.eps, act_dtype=act, gen_dtype=gen, injection_cap="hard"), inp.params())
    try:
        x = _x(inp.x32, act)
        y = torch.empty_like(x)
        S.srnl_scan_forward(h, x, y)
        torch.cuda.synchronize()
        S.srnl_scan_device_status(h)
        count = S.srnl_scan_cap_count(h)
    finally:
        h.close()
    cnt = [0]
    ref, _, _ = O.operator_forward(inp.x32, inp.params(), alpha_max=cfg.alpha, eps=cfg.eps, heads=cfg.heads,
                                   cap="hard", counter=cnt)
    tol = 1e-4 if (act == "f32" and gen == "f32") else 2e-2
    err = O.rel_fro(y.float().cpu().numpy(), ref)
    assert err <= tol, f"hard-cap {name} y: {err:.3e}"
    _check_count(count, cnt[0], 4 * cfg.B * cfg.H * cfg.W * cfg.heads, 1e-3 if act == "f32" else 1e-2)


@pytest.mark.parametrize("path", [("f32", "f32"), ("bf16", "bf16")])
def test_sequence_hard_cap(path):
    act, gen = path
    inp = make_seq_inputs(2, 257, 64, 2, act, seed=7)
    h = S.srnl_seq_create(dict(B=2, T=257, D=64, heads=2, d=32, alpha=0.95, eps=1e-6, chunk=0, act_dtype=act,
                               gen_dtype=gen, injection_cap="hard"), inp.params())
    try:
        x = _x(inp.x32, act)
        y = torch.empty_like(x)
        S.srnl_seq_forward(h, x, y)
        torch.cuda.synchronize()
        count = S.srnl_seq_cap_count(h)
        # the counter restarts with every forward
        S.srnl_seq_forward(h, x, y)
        assert S.srnl_seq_cap_count(h) == count
    finally:
        h.close()
    cnt = [0]
    ref, _ = O.sequence_forward(inp.x32, inp.params(), alpha_max=0.95, eps=1e-6, chunk=64, heads=2, cap="hard",
                                counter=cnt)
    tol = 1e-4 if act == "f32" else 2e-2
    err = O.rel_fro(y.float().cpu().numpy(), ref)
    assert err <= tol, f"hard-cap sequence y: {err:.3e}"
    _check_count(count, cnt[0], 2 * 257 * 2, 1e-3 if act == "f32" else 1e-2)


def test_soft_cap_counts_nothing():
    inp = make_seq_inputs(1, 64, 64, 2, "f32", seed=8)
    h = S.srnl_seq_create(dict(B=1, T=64, D=64, heads=2, d=32, alpha=0.95, eps=1e-6, chunk=0, act_dtype="f32",
                               gen_dtype="f32"), inp.params())
    try:
        x = _x(inp.x32, "f32")
        y = torch.empty_like(x)
        S.srnl_seq_forward(h, x, y)
        assert S.srnl_seq_cap_count(h) == 0
    finally:
        h.close()
