"""The pipelined host-buffer entry point: a loop of srnl_scan_forward_host_async calls, each
with its own pinned input and output, gives per step exactly what the device forward gives
for that input (the two staging slots alternate and are reused)."""
import numpy as np
import pytest
import torch

import self_referential_nested_b200 as S
from srnl_inputs import CONFIGS, bf16_round_bits, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from self_referential_nested_b200 import build
    build.build()
    torch.cuda.set_device(0)


@pytest.mark.parametrize("name", ["pr1_8x8", "hier_s3_14x14"])
def test_pipelined_host_forward_matches_device_forward(name):
    cfg = CONFIGS[name].replace(B=2) if name != "pr1_8x8" else CONFIGS[name]
    act = cfg.act_dtype
    inp = make_inputs(cfg)
    h = S.srnl_scan_create(dict(B=cfg.B, H=cfg.H, W=cfg.W, C=cfg.C, heads=cfg.heads, d=cfg.d, alpha=cfg.alpha,
                                eps=cfg.eps, act_dtype=act, gen_dtype=act), inp.params())
    try:
        rng = np.random.default_rng(1)
        xs, ys, refs = [], [], []
        for step in range(5):
            x32 = rng.standard_normal(inp.x32.shape, dtype=np.float32)
            if act == "bf16":
                xt = torch.from_numpy(bf16_round_bits(x32).view(np.int16)).view(torch.bfloat16)
            else:
                xt = torch.from_numpy(x32)
            xd = xt.cuda()
            yd = torch.empty_like(xd)
            S.srnl_scan_forward(h, xd, yd)
            torch.cuda.synchronize()
            refs.append(yd.cpu())
            xs.append(xt.pin_memory())
            ys.append(torch.empty_like(xt).pin_memory())
        for xh, yh in zip(xs, ys):
            S.srnl_scan_forward_host_async(h, xh, yh)
        S.srnl_scan_host_sync(h)
        for step, (yh, ref) in enumerate(zip(ys, refs)):
            assert torch.equal(yh, ref), f"step {step}"
    finally:
        h.close()
