"""Failure detection on the GPU without a fault: the scan kernels' bounded mbarrier wait is
made to run out on a barrier that nothing completes; the kernel must give up within its
wall-time limit, report SRNL_E_TIMEOUT to the host, and leave the context usable."""
import time

import numpy as np
import pytest
import torch

import self_referential_nested_b200 as S
from oracle import srnl_oracle as O
from srnl_inputs import CONFIGS, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from self_referential_nested_b200 import build
    build.build()
    torch.cuda.set_device(0)


def test_bounded_wait_gives_up_and_the_context_survives():
    t0 = time.monotonic()
    st = S.srnl_selftest_wait_timeout(50)
    dt = time.monotonic() - t0
    assert st == S.SRNL_E_TIMEOUT, S.load_library().srnl_scan_last_error(None)
    assert dt < 10.0
    # the same context still runs the tensor-core forward correctly, with a clean status
    cfg = CONFIGS["pr1_8x8"].replace(act_dtype="bf16")
    inp = make_inputs(cfg, seed=0)
    h = S.srnl_scan_create(dict(B=1, H=8, W=8, C=64, heads=2, d=32, alpha=0.95, act_dtype="bf16",
                                gen_dtype="bf16"), inp.params())
    try:
        x = torch.from_numpy(inp.x_bits.view(np.int16)).cuda().view(torch.bfloat16)
        y = torch.empty_like(x)
        S.srnl_scan_forward(h, x, y)
        torch.cuda.synchronize()
        S.srnl_scan_device_status(h)
    finally:
        h.close()
    ref, _, _ = O.forward_from_inputs(inp)
    assert O.rel_fro(y.float().cpu().numpy(), ref) <= 2e-2
