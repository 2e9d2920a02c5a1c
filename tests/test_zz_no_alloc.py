"""The allocation-free forward against the handle-based forward (GPU).

srnl_scan_forward_noalloc exists for callers that must not call cudaMalloc:
code hosted by a framework that owns all device memory through its own pool,
and latency-critical loops where an allocation may synchronise the device.  It
keeps its scratch in a fixed device array inside the library.  It runs the
same kernels on the same packed parameters as srnl_scan_forward, so its output
must be bit-identical.  This file is named so pytest collects it last; it must
pass alone in a fresh process and after every other test.
"""
import numpy as np
import pytest
import torch

import self_referential_nested_b200 as S
from srnl_inputs import CONFIGS, ScanConfig, bf16_round_bits, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from self_referential_nested_b200 import build
    build.build()
    torch.cuda.set_device(0)


def _cfg(cfg, path, cap="soft"):
    return dict(B=cfg.B, H=cfg.H, W=cfg.W, C=cfg.C, heads=cfg.heads, d=cfg.d, alpha=cfg.alpha,
                eps=cfg.eps, chunk_row=cfg.chunk_row, chunk_col=cfg.chunk_col, act_dtype=path,
                gen_dtype=path, injection_cap=cap)


def _x(inp, path):
    if path == "bf16":
        return torch.from_numpy(bf16_round_bits(inp.x32).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(inp.x32).cuda()


def _params_dev(inp):
    return {k: torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32)).cuda() for k, v in inp.params().items()}


# The larger workload first, so that the smaller ones run on the scratch it left behind.
CASES = [
    ("bf16", CONFIGS["hier_s1_56x56"].replace(B=2), "soft"),
    ("f32", CONFIGS["pr1_8x8"], "soft"),
    ("f32", ScanConfig("ragged", B=2, H=7, W=13, C=64, heads=2, d=32, alpha=0.95,
                       chunk_row=4, chunk_col=3, act_dtype="f32"), "soft"),
    ("bf16", ScanConfig("ragged_hard", B=2, H=9, W=11, C=64, heads=2, d=32, alpha=0.95,
                        chunk_row=5, chunk_col=0, act_dtype="bf16"), "hard"),
]


def test_noalloc_matches_handle_forward_bitwise_on_two_calls():
    for path, cfg, cap in CASES:
        inp = make_inputs(cfg, seed=3, **({"mem_scale": 0.3, "vec_scale": 0.8} if cap == "hard" else {}))
        x = _x(inp, path)
        h = S.srnl_scan_create(_cfg(cfg, path, cap), inp.params())
        try:
            y_ref = torch.empty_like(x)
            S.srnl_scan_forward(h, x, y_ref)
            torch.cuda.synchronize()
        finally:
            h.close()
        params_dev = _params_dev(inp)
        for call in range(2):   # the second call runs on the scratch the first one left behind
            y = torch.full_like(x, float("nan"))
            S.srnl_scan_forward_noalloc(_cfg(cfg, path, cap), params_dev, x, y)
            S.srnl_scan_noalloc_status()
            assert torch.equal(y, y_ref), (cfg.name, path, cap, call)


def test_noalloc_reports_a_bounded_wait_that_gave_up():
    """A bounded wait that must give up records SRNL_E_TIMEOUT in the no-allocation status
    word; the status query reports it, and the next forward clears it and still matches."""
    cfg = CONFIGS["pr1_8x8"].replace(act_dtype="bf16")
    inp = make_inputs(cfg, seed=0)
    x = _x(inp, "bf16")
    params_dev = _params_dev(inp)
    S.srnl_selftest_noalloc_wait_timeout(20)
    with pytest.raises(S.SrnlError) as e:
        S.srnl_scan_noalloc_status()
    assert e.value.status == S.SRNL_E_TIMEOUT
    y = torch.empty_like(x)
    S.srnl_scan_forward_noalloc(_cfg(cfg, "bf16"), params_dev, x, y)
    S.srnl_scan_noalloc_status()
    h = S.srnl_scan_create(_cfg(cfg, "bf16"), inp.params())
    try:
        y_ref = torch.empty_like(x)
        S.srnl_scan_forward(h, x, y_ref)
        torch.cuda.synchronize()
    finally:
        h.close()
    assert torch.equal(y, y_ref)


def _real_buffers(cfg, path):
    """Real device buffers of the workload's sizes: a rejected call never reaches a kernel, but
    if it did, every address it holds is a live allocation of the right size."""
    inp = make_inputs(CONFIGS["pr1_8x8"], seed=0)
    n = cfg.B * cfg.H * cfg.W * cfg.C
    dt = torch.bfloat16 if path == "bf16" else torch.float32
    return _params_dev(inp), torch.zeros(n, dtype=dt, device="cuda"), torch.zeros(n, dtype=dt, device="cuda")


def test_noalloc_rejects_workloads_beyond_its_scratch():
    cfg = CONFIGS["hier_s1_56x56"]                        # full batch: more than the fixed scratch
    params_dev, x, y = _real_buffers(cfg, "bf16")
    d = _cfg(cfg, "bf16")
    with pytest.raises(S.SrnlError) as e:
        S.srnl_scan_forward_noalloc(d, params_dev, x, y)
    assert e.value.status == S.SRNL_E_INVAL
    assert str(S.NOALLOC_SCRATCH_BYTES) in str(e.value)


def test_noalloc_rejects_misaligned_and_host_pointers():
    params_dev, x, y = _real_buffers(CONFIGS["pr1_8x8"], "f32")
    d = _cfg(CONFIGS["pr1_8x8"], "f32")
    for key in ("W_q", "M_k0", "m_alpha0"):
        bad = dict(params_dev)
        bad[key] = params_dev[key].data_ptr() + 2
        with pytest.raises(S.SrnlError) as e:
            S.srnl_scan_forward_noalloc(d, bad, x, y)
        assert e.value.status == S.SRNL_E_INVAL and "aligned" in str(e.value), key
    host = dict(params_dev)
    host["scales"] = torch.zeros(4 * 64, dtype=torch.float32)   # host memory
    with pytest.raises(S.SrnlError) as e:
        S.srnl_scan_forward_noalloc(d, host, x, y)
    assert e.value.status == S.SRNL_E_INVAL and "scales" in str(e.value)
    with pytest.raises(S.SrnlError) as e:
        S.srnl_scan_forward_noalloc(d, params_dev, x.cpu(), y)
    assert e.value.status == S.SRNL_E_INVAL and "x" in str(e.value)
