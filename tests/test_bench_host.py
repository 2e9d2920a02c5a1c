"""Host-side arithmetic of bench.py against closed forms: the algorithmic bytes and flops the
roofline fractions divide by, the backward's flop count, the chain depth, and the job rate."""
import bench
from srnl_inputs import CONFIGS


def test_forward_work_model_s1():
    cfg = CONFIGS["hier_s1_56x56"]
    wm = bench.work_model(cfg)
    tokens = 32 * 56 * 56
    params = 4 * (64 * 64 + 4 * 64 + 4 * 2 * (3 * 32 * 32 + 2 * 32))
    assert wm["tokens"] == tokens and wm["route_tokens"] == 4 * tokens
    assert wm["hbm_bytes"] == 2 * tokens * 64 * 2 + params == 25807872      # x and y in bf16, fp32 params
    assert wm["gen_flops"] == 2.0 * (4 * tokens * 2) * 66 * 32
    assert wm["qproj_flops"] == 2.0 * tokens * 64 * 64


def test_backward_flops_per_token_closed_form():
    for d in (32, 64):
        gen = 2 * (2 * d + 2) * d
        assert bench.backward_flops_per_token(d) == 43 * d * d + 3 * gen
    assert bench.backward_flops_per_token(32) == 56704
    assert bench.backward_flops_per_token(64) == 226048


def test_chain_depth():
    assert bench.stages_per_sequence(CONFIGS["hier_s1_56x56"]) == 56         # one 56-token stage per row
    assert bench.stages_per_sequence(CONFIGS["pr1_8x8"]) == 8
    # 200 x 304: row chunks of 304 tokens take 5 stages of <= 64 (200 chunks); column chunks of
    # 200 take 4 (304 chunks): the column routes are the longer chain
    assert bench.stages_per_sequence(CONFIGS["hires_200x304"]) == max(200 * 5, 304 * 4)


def test_job_rate_and_single_rank_max():
    assert bench.whole_job_rate(1, 401408, 20, 11.2) == 401408 * 20 / 11.2e-3
    assert bench.whole_job_rate(4, 10, 2, 1.0) == 4 * 10 * 2 / 1e-3
    assert bench.max_over_ranks([1.5, 2.0], 1) == [1.5, 2.0]
