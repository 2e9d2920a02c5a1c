"""The allocation-free forward against the handle-based forward (GPU).

srnl_scan_forward_noalloc exists for callers that must not call cudaMalloc:
code hosted by a framework that owns all device memory through its own pool,
and latency-critical loops where an allocation may synchronise the device.  It
keeps its scratch in a fixed device array inside the library.  This file is
named so pytest collects it last; it must pass alone in a fresh process and
after every other test.
"""
import numpy as np
import pytest
import torch

import self_referential_nested_b200 as S
from srnl_inputs import CONFIGS, ScanConfig, bf16_round_bits, make_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}   # the parity tolerances of the other GPU tests


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from self_referential_nested_b200 import build
    build.build()
    torch.cuda.set_device(0)


def _cfg(cfg, path):
    return dict(B=cfg.B, H=cfg.H, W=cfg.W, C=cfg.C, heads=cfg.heads, d=cfg.d, alpha=cfg.alpha,
                eps=cfg.eps, chunk_row=cfg.chunk_row, chunk_col=cfg.chunk_col, act_dtype=path,
                gen_dtype=path)


def _x(inp, path):
    if path == "bf16":
        return torch.from_numpy(bf16_round_bits(inp.x32).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(inp.x32).cuda()


def _rel(a, b):
    a, b = a.double(), b.double()
    return float(torch.linalg.vector_norm(a - b) / torch.linalg.vector_norm(b))


CASES = [
    ("f32", CONFIGS["pr1_8x8"]),
    ("bf16", CONFIGS["hier_s1_56x56"].replace(B=2)),
    ("f32", ScanConfig("ragged", B=2, H=7, W=13, C=64, heads=2, d=32, alpha=0.95,
                       chunk_row=4, chunk_col=3, act_dtype="f32")),
]


@pytest.mark.parametrize("path,cfg", CASES, ids=[c[1].name + "-" + c[0] for c in CASES])
def test_noalloc_matches_handle_forward_on_two_calls(path, cfg):
    inp = make_inputs(cfg, seed=3)
    x = _x(inp, path)
    h = S.srnl_scan_create(_cfg(cfg, path), inp.params())
    try:
        y_ref = torch.empty_like(x)
        S.srnl_scan_forward(h, x, y_ref)
        torch.cuda.synchronize()
    finally:
        h.close()
    params_dev = {k: torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32)).cuda()
                  for k, v in inp.params().items()}
    for call in range(2):   # the second call runs on the scratch the first one left behind
        y = torch.full_like(x, float("nan"))
        S.srnl_scan_forward_noalloc(_cfg(cfg, path), params_dev, x, y)
        torch.cuda.synchronize()
        assert torch.isfinite(y.float()).all(), call
        assert _rel(y.float(), y_ref.float()) <= TOL[path], call


def test_noalloc_rejects_workloads_beyond_its_scratch():
    cfg = CONFIGS["hier_s1_56x56"]           # full batch: far more than the fixed scratch
    d = _cfg(cfg, "bf16")
    fake = {k: 256 for k in ("W_q", "scales", "M_mem0", "M_k0", "M_v0", "m_eta0", "m_alpha0")}
    with pytest.raises(S.SrnlError) as e:
        S.srnl_scan_forward_noalloc(d, fake, 4096, 1 << 40)
    assert e.value.status == S.SRNL_E_INVAL
    assert str(S.NOALLOC_SCRATCH_BYTES) in str(e.value)
