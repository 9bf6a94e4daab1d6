"""The bench's algorithmic bytes and ops (the numerator of every roofline
fraction it prints) against totals added up by hand from the format: codes,
scales, int8 activations with their fp32 scale, bf16 outputs."""

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


# (m, k, n, fmt) -> bytes of one iq8r_linear call, summed term by term
HAND = {
    # codes 131,072 + s1 512 + s2 512 + act 2,048 + 16 + y 2,048
    (4, 512, 256, "g256"): 136_208,
    # codes 89,128,960 + s1 348,160 + s2 34,816 + act 5,120 + 4 + y 34,816
    (1, 5120, 17408, "g256"): 89_551_876,
    # codes 89,128,960 + s1 348,160 + s2 10,240 + act 8 x 17,408 + 32 + y 81,920
    (8, 17408, 5120, "g256"): 89_708_576,
    (16, 17408, 5120, "g256"): 89_929_792,
    (128, 17408, 5120, "g256"): 93_026_816,
    # codes 777,912,320 + scales 12,154,880 + act 5,124 + y 303,872
    (1, 5120, 151936, "g128"): 790_376_196,
    (8, 5120, 151936, "g128"): 792_539_168,
    # indices 44,564,480 + scales 1,392,640 + act 5,124 + y 34,816
    (1, 5120, 17408, "cb4"): 45_997_060,
}


@pytest.mark.parametrize("shape", sorted(HAND))
def test_linear_bytes_match_hand_totals(shape):
    assert bench.linear_bytes(*shape) == HAND[shape]


def test_fused_layer_reads_bf16_activations():
    # the one-launch layer reads x (2 bytes an element) instead of xq and xs
    assert bench.fused_bytes(1, 5120, 17408, "g256") == 89_551_876 - 5_124 + 10_240


def test_prefill_ops_and_bytes():
    m, k, n = 8192, 5120, 17408
    assert 2 * m * n * k == 1_460_288_880_640
    # xq 41.9 MB + fp32 scales, weights 89.5 MB, y 285.2 MB
    assert bench.linear_bytes(m, k, n, "g256") == 41_943_040 + 32_768 + 89_511_936 + 285_212_672
    # the activation kernel: bf16 in, int8 and fp32 scales out
    assert bench.act_bytes(m, k) == 8192 * (3 * 5120 + 4) == 125_861_888


def test_bound_follows_the_ridge():
    # decode and verify stream weights (HBM); prefill is a dense contraction
    assert bench.is_hbm_bound(1, 5120, 17408, "g256")
    assert bench.is_hbm_bound(128, 17408, 5120, "g256")
    assert not bench.is_hbm_bound(8192, 5120, 17408, "g256")


def test_step_counts_one_launch_only_where_the_library_fuses():
    assert bench.one_launch(1, 5120) and bench.one_launch(2, 5120)
    assert bench.one_launch(8, 2048) and not bench.one_launch(8, 5120)
    assert not bench.one_launch(1, 5120, "cb4")
    assert bench.step_bytes(8192, 5120, 17408, "g256") == \
        bench.act_bytes(8192, 5120) + bench.linear_bytes(8192, 5120, 17408, "g256")


def test_oracle_check_reports_the_tolerance_and_bit_equality():
    """The bench's parity summary (its CPU-baseline leg): the oracle's own
    bf16 result passes with every output bit-equal; a result off by 2 % of
    the RMS in one output fails the tolerance."""
    import numpy as np

    import oracle
    from iq8r_inputs import gen_workload

    x, w = gen_workload("pr1")
    packed = oracle.pack(w, "g256", True)
    q, a = oracle.act_quant(x)
    y64 = oracle.linear(q, a, "g256", *packed)
    good = oracle.linear_bf16(y64)
    chk = {"config": "pr1", "x": x, "packed": packed, "y": good}
    r = bench.oracle_check(chk)
    # the literal ratio of a correctly rounded bf16 result is its own rounding
    # (above 1e-2 of RMS here), which the half-ulp term of the reading admits
    assert r["within_tolerance"] and r["bit_equal_frac"] == 1.0 and r["max_err_over_rms"] < 2e-2
    rms = float(np.sqrt(np.mean(y64 ** 2)))
    bad = oracle.linear_bf16(y64 + np.where(np.arange(y64.size).reshape(y64.shape) == 5, 0.02 * rms, 0.0))
    r = bench.oracle_check(dict(chk, y=bad))
    assert not r["within_tolerance"] and r["bit_equal_frac"] < 1.0


def test_timed_reps():
    # a 20-step decode region (~0.4 ms) is taken about a thousand times; a
    # prefill region three times
    assert bench.timed_reps(0.4) == 1000 and bench.timed_reps(200.0) == 3
    assert bench.timed_reps(18.0, tensor_bound=True) == 3
