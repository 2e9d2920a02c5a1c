"""GPU parity of the sequence layer's backward (srnl_seq_backward through the C ABI) against the
float64 gradient oracle (``sequence_backward``, pinned by finite differences).  Tolerances as
for the operator's backward: 1e-4 relative Frobenius error for every gradient, 1e-2 for a
gradient returned in bf16 (per-element rounding alone reaches 2^-9)."""
import numpy as np
import pytest
import torch

import self_referential_nested_b200 as S
from oracle import srnl_grad as GR
from oracle import srnl_oracle as O
from srnl_inputs import bf16_round_bits, make_cotangent, make_seq_inputs

pytestmark = pytest.mark.gpu

TOL = 1e-4
TOL_BF16_OUT = 1e-2


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


def run(B, T, D, heads, act="f32", chunk=64, queries=True, cap="soft", seed=0, mem_scale=0.02, vec_scale=0.1):
    si = make_seq_inputs(B, T, D, heads, act, seed=seed, mem_scale=mem_scale, vec_scale=vec_scale)
    d = D // heads
    params = si.params()
    dyv = make_cotangent((B, T, D), seed=seed, act_dtype=act)
    h = S.srnl_seq_create(dict(B=B, T=T, D=D, heads=heads, d=d, alpha=0.95, eps=1e-6, chunk=chunk, act_dtype=act,
                               gen_dtype="f32", injection_cap=cap), params)
    try:
        x, dy = _dev(si.x32, act), _dev(dyv, act)
        q = _dev(si.q32, act) if queries else None
        dx = torch.full_like(x, float("nan"))
        dq = torch.full_like(x, float("nan")) if queries else None
        grads = {k: torch.full(np.shape(params[k]), float("nan"), device="cuda") for k in S.SEQ_GRAD_KEYS}
        S.srnl_seq_backward(h, x, dy, dx, q=q, dq=dq, grads=grads)
        torch.cuda.synchronize()
        got = {k: v.cpu().numpy() for k, v in grads.items()}
        got["x"] = dx.float().cpu().numpy()
        if queries:
            got["queries"] = dq.float().cpu().numpy()
    finally:
        h.close()
    ref = GR.sequence_backward(si.x32, params, dyv, alpha_max=0.95, chunk=chunk, heads=heads,
                               queries=si.q32 if queries else None, cap=cap)
    for key, val in got.items():
        bound = TOL_BF16_OUT if (act == "bf16" and key in ("x", "queries")) else TOL
        assert np.all(np.isfinite(val)), key
        err = O.rel_fro(val, ref[key])
        assert err <= bound, f"{key}: relative Frobenius error {err:.3e} > {bound:.0e}"


@pytest.mark.parametrize("queries", [True, False])
def test_seq_backward_f32(queries):
    run(3, 200, 64, 2, queries=queries, seed=1)          # chunks 64, 64, 64, 8 (ragged tail)


def test_seq_backward_bf16_io():
    run(2, 130, 128, 4, act="bf16", seed=2)


def test_seq_backward_chunk_override_and_hard_cap():
    run(2, 77, 64, 2, chunk=20, cap="hard", seed=3, mem_scale=0.3, vec_scale=0.8)


def test_seq_backward_small_head_dim():
    run(2, 50, 32, 4, chunk=16, seed=4, mem_scale=0.2, vec_scale=0.5)   # d = 8, zero-padded heads


def test_seq_backward_rejects_dq_without_queries():
    si = make_seq_inputs(1, 8, 64, 2, "f32", seed=0)
    h = S.srnl_seq_create(dict(B=1, T=8, D=64, heads=2, d=32, alpha=0.95, act_dtype="f32", gen_dtype="f32"),
                          si.params())
    try:
        x = _dev(si.x32, "f32")
        with pytest.raises(S.SrnlError) as ei:
            S.srnl_seq_backward(h, x, x.clone(), torch.empty_like(x), q=None, dq=torch.empty_like(x))
        assert ei.value.status == S.SRNL_E_INVAL
    finally:
        h.close()


def test_seq_backward_head_dim_64():
    run(2, 70, 128, 2, chunk=24, seed=14)
    run(1, 33, 64, 1, chunk=0, queries=False, seed=15)


def test_seq_backward_single_token():
    run(3, 1, 64, 2, seed=16)
