"""CUDA-graph capture: the forward and (after its first call, which allocates the workspace)
the backward issue only kernel launches and asynchronous memsets on the caller's stream, so a
loop of steps can be captured once and replayed.  Replays must give bit-identical results to
eager calls (every kernel of the path is deterministic)."""
import numpy as np
import pytest
import torch

import self_referential_nested_b200 as S
from srnl_inputs import CONFIGS, bf16_round_bits, make_cotangent, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from self_referential_nested_b200 import build
    build.build()
    torch.cuda.set_device(0)


def _bf16(a32):
    return torch.from_numpy(bf16_round_bits(a32).view(np.int16)).cuda().view(torch.bfloat16)


@pytest.mark.parametrize("gen", ["bf16", "f32"])
def test_forward_graph_replay_is_bitwise_equal(gen):
    cfg = CONFIGS["hier_s1_56x56"].replace(B=2)
    inp = make_inputs(cfg, seed=0)
    h = S.srnl_scan_create(dict(B=2, H=56, W=56, C=64, heads=2, d=32, alpha=0.95, act_dtype="bf16", gen_dtype=gen),
                           inp.params())
    try:
        x = _bf16(inp.x32)
        y_eager = torch.empty_like(x)
        S.srnl_scan_forward(h, x, y_eager)
        torch.cuda.synchronize()
        y = torch.empty_like(x)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            S.srnl_scan_forward(h, x, y)          # warm-up on the capture stream
        torch.cuda.current_stream().wait_stream(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(3):
                S.srnl_scan_forward(h, x, y)
        y.zero_()
        g.replay()
        torch.cuda.synchronize()
        S.srnl_scan_device_status(h)
        assert torch.equal(y.view(torch.int16), y_eager.view(torch.int16))
        del g
    finally:
        h.close()


def test_backward_graph_replay_is_bitwise_equal():
    cfg = CONFIGS["pr1_8x8"].replace(B=2)
    inp = make_inputs(cfg, seed=1)
    params = inp.params()
    h = S.srnl_scan_create(dict(B=2, H=8, W=8, C=64, heads=2, d=32, alpha=0.95, act_dtype="f32", gen_dtype="f32"),
                           params)
    try:
        x = torch.from_numpy(inp.x32).cuda()
        dy = torch.from_numpy(make_cotangent(inp.x32.shape, seed=1)).cuda()
        dx_eager = torch.empty_like(x)
        g_eager = {k: torch.empty(np.shape(params[k]), device="cuda") for k in S.GRAD_KEYS}
        S.srnl_scan_backward(h, x, dy, dx_eager, g_eager)    # allocates the workspace
        torch.cuda.synchronize()
        dx = torch.empty_like(x)
        gr = {k: torch.empty_like(v) for k, v in g_eager.items()}
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            S.srnl_scan_backward(h, x, dy, dx, gr)
        torch.cuda.current_stream().wait_stream(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            S.srnl_scan_backward(h, x, dy, dx, gr)
        dx.zero_()
        for v in gr.values():
            v.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(dx, dx_eager)
        for k in S.GRAD_KEYS:
            assert torch.equal(gr[k], g_eager[k]), k
        del g
    finally:
        h.close()
