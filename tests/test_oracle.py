"""The oracle against what the pages and the mathematics fix (CPU only)."""

import numpy as np
import pytest
import torch

import oracle
import pins
from iq8r_inputs import f32_to_bf16_bits
from iq8r_inputs import WORKLOADS, gen_workload


@pytest.fixture(scope="module")
def pr1():
    return gen_workload("pr1")


@pytest.fixture(scope="module")
def decode_small():
    # decode's value distribution (outlier columns and channels) at a size
    # the pure-numpy checks finish quickly
    return gen_workload("decode", m=3, n=40, k=1280, seed=101)


def test_transform_pins():
    pins.check_transform(oracle.fwht128_f32, oracle.hadamard128)


def test_transform_rounding_bound():
    pins.check_transform_rounding(oracle.fwht128_f32)


def test_transform_f64_matches_scipy():
    x = np.random.default_rng(3).standard_normal((5, 256))
    import scipy.linalg
    H = scipy.linalg.hadamard(128).astype(np.float64)
    ref = (x.reshape(5, 2, 128) @ H.T).reshape(5, 256)
    assert np.allclose(oracle.fwht128_f64(x), ref, rtol=0, atol=1e-12)


def test_transform_f32_exact_on_small_integers():
    v = np.random.default_rng(5).integers(-1000, 1001, size=(8, 256)).astype(np.float32)
    assert np.array_equal(oracle.fwht128_f32(v).astype(np.float64), oracle.fwht128_f64(v))


def test_bf16_round_nearest_matches_torch():
    rng = np.random.default_rng(9)
    v = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(37.0),
        np.float32(2.0 ** -130) * rng.standard_normal(2000).astype(np.float32),  # bf16 subnormals
        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.3895e38, -3.3896e38], np.float32),
    ])
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.bf16_round_nearest(v.astype(np.float64))
    assert np.array_equal(got, ref)


def test_bf16_round_up_is_smallest_upper_bound():
    rng = np.random.default_rng(10)
    v = np.abs(rng.standard_normal(20000).astype(np.float32)) * np.float32(1e-3)
    v = np.concatenate([v, np.float32(2.0 ** -128) * np.abs(rng.standard_normal(500)).astype(np.float32),
                        np.array([0.0, 1.0, 2.0 ** -126, 1.0078125], np.float32)])
    r = oracle.bf16_round_up(v)
    rb = r.view(np.uint32)
    assert not np.any(rb & 0xFFFF)                      # on the bf16 grid
    assert np.all(r >= v)                               # an upper bound
    below = ((rb >> 16) - 1).astype(np.uint32) << 16    # next bf16 down
    pos = r > 0
    assert np.all(below[pos].view(np.float32) < v[pos])  # and the smallest one
    assert np.all(r[v == 0] == 0)


def test_act_golden():
    pins.check_act_golden(oracle.act_quant)


def test_act_properties(pr1, decode_small):
    pins.check_act_properties(oracle.act_quant, oracle.fwht128_f64, pr1[0])
    pins.check_act_properties(oracle.act_quant, oracle.fwht128_f64, decode_small[0])


def test_act_tiny_rows():
    """Rows whose amax is below 2^-64, down to bf16 subnormals: hand-derived
    goldens, and the general properties, with no overflow or invalid
    operation anywhere in the oracle."""
    pins.check_act_tiny_golden(oracle.act_quant)
    rng = np.random.default_rng(21)
    k = 512
    x = rng.standard_normal((6, k))
    x[0] *= 1e-39                                        # bf16 subnormals, amax ~ 1e-37
    x[1] *= 2.0 ** -140                                  # mostly zeros and the smallest subnormals
    x[2] *= 2.0 ** -70                                   # prescaled, 127 / amax finite
    x[3] *= 2.0 ** -64                                   # around the threshold
    x[4] = 0.0
    x[4, 5] = 2.0 ** -133                                # a single smallest bf16 subnormal
    x[5] *= np.exp(rng.uniform(-95, -85, k))             # mixed tiny magnitudes
    bits = f32_to_bf16_bits(x.astype(np.float32))
    with np.errstate(over="raise", invalid="raise", divide="raise"):
        q, a = oracle.act_quant(bits)
        pins.check_act_properties(oracle.act_quant, oracle.fwht128_f64, bits)
    assert np.all(np.abs(q[a > 0]).max(axis=1) == 127)
    # the prescale changes no code of a row whose 127 / amax is finite: the
    # same row scaled by 2^60 (an exact bf16 exponent shift) is not prescaled
    up = pins.bf16(pins.bf16_val(bits[2]) * np.float32(2.0 ** 60)).reshape(1, k)
    assert np.array_equal(q[2], oracle.act_quant(up)[0][0])


def test_act_spike_and_zero_rows():
    pins.check_act_spike(oracle.act_quant)


def test_act_unrotated_is_plain_absmax():
    x = np.zeros((1, 128), np.float32)
    x[0, :4] = [1.0, -0.5, 0.25, 2.0]
    q, a = oracle.act_quant(pins.bf16(x).reshape(1, 128), rotate=False)
    assert list(q[0, :4]) == [64, -32, 16, 127] and np.all(q[0, 4:] == 0)  # 127/2 * x, ties to even
    assert a[0] == np.float32(2.0) / np.float32(127.0)


def test_pack_golden():
    pins.check_pack_golden(oracle.pack)


def test_pack_g256_properties(pr1, decode_small):
    pins.check_pack_g256_properties(oracle.pack, oracle.fwht128_f64, pr1[1])
    pins.check_pack_g256_properties(oracle.pack, oracle.fwht128_f64, decode_small[1])


def test_pack_g128_properties(decode_small):
    pins.check_pack_g128_properties(oracle.pack, oracle.fwht128_f64, decode_small[1])


def test_pack_zero_row_and_sizes():
    w = np.zeros((2, 512), np.uint16)
    w[1] = pins.bf16(np.full(512, 0.25, np.float32))
    codes, s1, s2 = oracle.pack(w, "g256", True)
    assert s2[0] == 0 and np.all(s1[0] == 0) and np.all(codes[0] == 0)
    assert s2[1] != 0
    assert oracle.packed_sizes("g256", 17408, 5120) == (89128960, 348160, 34816)
    assert oracle.packed_sizes("g128", 151936, 5120) == (777912320, 0, 12154880)
    g = pins.golden("format")
    assert g["trunk"]["group"] == oracle.GROUP_TRUNK and g["lm_head"]["group"] == oracle.GROUP_HEAD
    assert g["trunk"]["code_max"] == oracle.CODE_MAX == -g["trunk"]["code_min"]


def test_partials_brute_force():
    rng = np.random.default_rng(12)
    xq = rng.integers(-127, 128, size=(2, 512)).astype(np.int8)
    codes = rng.integers(-127, 128, size=(3, 512)).astype(np.int8)
    pins.check_partials_brute(oracle.partials, xq, codes, 256)
    pins.check_partials_brute(oracle.partials, xq, codes, 128)
    # extreme values: |P| reaches 256 * 127^2 exactly
    full = np.full((1, 256), 127, np.int8)
    assert oracle.partials(full, -full, 256)[0, 0, 0] == -256 * 127 * 127


def test_linear_golden():
    pins.check_linear_golden(oracle.act_quant, oracle.pack, oracle.partials, oracle.linear, oracle.linear_bf16)


def test_product_identity_trunk(pr1, decode_small):
    pins.check_product_identity(oracle.act_quant, oracle.pack, oracle.linear, pr1[0], pr1[1], "g256")
    pins.check_product_identity(oracle.act_quant, oracle.pack, oracle.linear, decode_small[0], decode_small[1], "g256")


def test_product_identity_lm_head():
    x, w = gen_workload("lm_head8", m=2, n=48, k=640, seed=104)
    pins.check_product_identity(oracle.act_quant, oracle.pack, oracle.linear, x, w, "g128")


def test_unrotated_linear_is_plain_int8_linear(pr1):
    x, w = pr1
    xq, a = oracle.act_quant(x, rotate=False)
    codes, s1, s2 = oracle.pack(w, "g256", rotate=False)
    y = oracle.linear(xq, a, "g256", codes, s1, s2, rotated=False)
    ref = (a.astype(np.float64)[:, None] * xq.astype(np.float64)) @ (
        np.repeat(pins.bf16_val(s2).astype(np.float64)[:, None] * s1, 256, axis=1) * codes).T
    assert np.allclose(y, ref, rtol=1e-12, atol=0)


def test_rotated_and_unrotated_agree(pr1):
    x, w = pr1
    ys = []
    for rot in (True, False):
        xq, a = oracle.act_quant(x, rotate=rot)
        codes, s1, s2 = oracle.pack(w, "g256", rotate=rot)
        ys.append(oracle.linear(xq, a, "g256", codes, s1, s2, rotated=rot))
    assert np.sqrt(np.mean((ys[0] - ys[1]) ** 2)) < 0.05 * np.sqrt(np.mean(ys[1] ** 2))


def test_workload_shapes_cover_the_pages_sizes():
    assert (WORKLOADS["decode"].k, WORKLOADS["decode"].n) == (5120, 17408)
    assert (WORKLOADS["verify128"].k, WORKLOADS["verify128"].n) == (17408, 5120)
    assert WORKLOADS["prefill"].m == 8192 and WORKLOADS["lm_head1"].n == 151936


# ------------------------------------------------------------- rescoring

@pytest.mark.parametrize("fmt", ["g256", "g128"])
def test_rescore_is_the_linear_at_the_candidates(fmt):
    """Rescoring (per pair, its own dot products) equals the full layer
    output gathered at the candidate rows, duplicates and the first/last row
    included; unrotated too."""
    rng = np.random.default_rng(12)
    x, w = gen_workload("decode", m=3, n=40, k=512, seed=12)
    for rotated in (True, False):
        codes, sub, scale = oracle.pack(w, fmt, rotated)
        xq, a = oracle.act_quant(x, rotated)
        y = oracle.linear(xq, a, fmt, codes, sub, scale, rotated=rotated)
        cand = rng.integers(0, 40, size=(3, 6))
        cand[0, :3] = [0, 39, 0]
        got = oracle.rescore(xq, a, fmt, codes, sub, scale, cand, rotated=rotated)
        assert np.array_equal(got, np.take_along_axis(y, cand, axis=1))


# ------------------------------------------------------- rule=search packing

def _exact_sse(vals, step):
    """Exact (rational) squared error of a group at a step, codes as packed."""
    from fractions import Fraction
    tot = Fraction(0)
    st = Fraction(float(step))
    for v in vals:
        q = max(-127, min(127, int(np.rint(np.float32(v) / np.float32(step)))))
        e = Fraction(float(v)) - q * st
        tot += e * e
    return tot


@pytest.mark.parametrize("fmt", ["g256", "g128"])
def test_pack_search_minimises_group_error(fmt):
    """Brute force: for every group of a small weight, the searched scale has
    the least exact squared error among the RTN scale and the 15 below it
    (ties to the larger); it never does worse than RTN, does better on some
    groups, and the codes are those of the chosen scale."""
    _, w = gen_workload("decode", m=1, n=6, k=512, seed=33)
    wr = oracle.fwht128_f32(oracle.bf16_to_f32(w))
    c0, s0, sc0 = oracle.pack(w, fmt, True)
    c1, s1, sc1 = oracle.pack_search(w, fmt, True)
    g = 256 if fmt == "g256" else 128
    improved = 0
    for r in range(w.shape[0]):
        for b in range(w.shape[1] // g):
            vals = wr[r, b * g:(b + 1) * g]
            if fmt == "g256":
                s2 = float(oracle.bf16_to_f32(sc0[r:r + 1])[0])
                cands = [np.float32(s2) * np.float32(s0[r, b] - i) for i in range(16) if s0[r, b] - i >= 1]
                chosen = np.float32(s2) * np.float32(s1[r, b])
            else:
                base = int(sc0[r, b])
                cands = [oracle.bf16_to_f32(np.array([base - i], np.uint16))[0] for i in range(16) if base - i >= 1]
                chosen = oracle.bf16_to_f32(sc1[r:r + 1, b])[0]
            errs = [_exact_sse(vals, c) for c in cands]
            best = min(errs)
            e_chosen = _exact_sse(vals, chosen)
            assert float(e_chosen) <= float(best) * (1 + 1e-9)
            assert e_chosen <= errs[0]
            improved += e_chosen < errs[0]
            q = np.clip(np.rint(vals / np.float32(chosen)), -127, 127).astype(np.int8)
            assert np.array_equal(c1[r, b * g:(b + 1) * g], q)
    assert improved > 0


def _exact_cb4_sse(vals, scale):
    """Exact (rational) squared error of a codebook group at a scale, each
    value at its nearest level (brute force over the 16, ties to the larger)."""
    from fractions import Fraction
    table = [-127, -97, -75, -58, -43, -30, -18, -6, 6, 18, 30, 43, 58, 75, 97, 127]
    tot = Fraction(0)
    st = Fraction(float(scale))
    for v in vals:
        t = float(np.float32(v) / np.float32(scale))
        lv = min(table, key=lambda c: (abs(t - c), -c))
        e = Fraction(float(v)) - lv * st
        tot += e * e
    return tot


def test_pack_search_cb4_minimises_group_error():
    """Brute force for the codebook format: per group, the searched bf16
    scale has the least exact squared error among the RTN scale and the 15
    next smaller bf16 values, never does worse than RTN, does better on some
    groups, and every index is the nearest level at the chosen scale."""
    _, w = gen_workload("decode", m=1, n=4, k=256, seed=35)
    wr = oracle.fwht128_f32(oracle.bf16_to_f32(w))
    _, sc0 = oracle.pack_cb4(w, True)
    p1, sub1, sc1 = oracle.pack_search(w, "cb4", True)
    assert sub1 is None
    table = [-127, -97, -75, -58, -43, -30, -18, -6, 6, 18, 30, 43, 58, 75, 97, 127]
    vals1 = oracle.decode_cb4(p1)
    improved = 0
    for r in range(w.shape[0]):
        for b in range(w.shape[1] // 128):
            vals = wr[r, b * 128:(b + 1) * 128]
            base = int(sc0[r, b])
            cands = [oracle.bf16_to_f32(np.array([base - i], np.uint16))[0] for i in range(16) if base - i >= 1]
            chosen = oracle.bf16_to_f32(sc1[r:r + 1, b])[0]
            errs = [_exact_cb4_sse(vals, c) for c in cands]
            e_chosen = _exact_cb4_sse(vals, chosen)
            assert float(e_chosen) <= float(min(errs)) * (1 + 1e-9)
            assert e_chosen <= errs[0]
            improved += e_chosen < errs[0]
            for j in range(128):
                t = float(np.float32(vals[j]) / np.float32(chosen))
                assert vals1[r, b * 128 + j] == min(table, key=lambda c: (abs(t - c), -c))
    assert improved > 0


# ------------------------------------------ the drafter's 16-level codebook

def test_cb4_nearest_level_and_layout():
    """Every index is the nearest codebook level to w'/s (ties to the larger
    level), the scale covers the group's largest value, the error is at most
    half the widest gap, and two indices share a byte, even K low."""
    _, w = gen_workload("decode", m=1, n=5, k=384, seed=41)
    packed, scale = oracle.pack_cb4(w, True)
    wr = oracle.fwht128_f32(oracle.bf16_to_f32(w))
    s = oracle.bf16_to_f32(scale)
    table = [-127, -97, -75, -58, -43, -30, -18, -6, 6, 18, 30, 43, 58, 75, 97, 127]
    vals = oracle.decode_cb4(packed)
    for r in range(5):
        for g in range(3):
            sg = np.float32(s[r, g])
            amax = np.max(np.abs(wr[r, g * 128:(g + 1) * 128]))
            assert sg * 127 >= amax
            for j in range(128):
                kk = g * 128 + j
                t = float(np.float32(wr[r, kk]) / sg)
                best = min(table, key=lambda v: (abs(t - v), -v))
                assert vals[r, kk] == best
                assert abs(float(wr[r, kk]) - float(sg) * best) <= float(sg) * 15 + 1e-12
                byte = packed[r, kk // 2]
                nib = (byte & 0x0F) if kk % 2 == 0 else (byte >> 4)
                assert table[nib] == vals[r, kk]


def test_cb4_ties_and_zero_group():
    """Hand-made groups: a value half way between two levels takes the larger
    one (-112 -> -97, 0 -> +6); an all-zero group has scale 0 and index 8."""
    s = 1.0
    grp = np.zeros(128, np.float32)
    grp[0] = 127.0 * s     # sets the scale to exactly 1 (bf16 of 127/127)
    grp[1] = -112.0        # between -127 and -97
    grp[2] = 0.0           # between -6 and +6
    grp[3] = 36.5          # 6.5 from both 30 and 43: a tie -> 43
    w = np.stack([grp, np.zeros(128, np.float32)])
    packed, scale = oracle.pack_cb4(oracle.f32_to_bf16_exact(w), rotate=False)
    v = oracle.decode_cb4(packed)
    assert oracle.bf16_to_f32(scale)[0, 0] == 1.0
    assert list(v[0, :4]) == [127, -97, 6, 43]
    assert scale[1, 0] == 0 and np.all(packed[1] == 0x88)


def test_cb4_linear_brute_force():
    """The codebook linear against a pure-Python sum on a tiny case: every
    index read from its nibble, looked up in the 16 levels, multiplied by the
    token's code, summed per 128-block with integers, then scaled."""
    table = [-127, -97, -75, -58, -43, -30, -18, -6, 6, 18, 30, 43, 58, 75, 97, 127]
    x, w = gen_workload("decode", m=2, n=3, k=256, seed=47)
    packed, scale = oracle.pack_cb4(w, True)
    q, a = oracle.act_quant(x)
    y64 = oracle.linear(q, a, "cb4", packed, None, scale, rotated=True)
    s = oracle.bf16_to_f32(scale)
    for m in range(2):
        for n in range(3):
            tot = 0.0
            for g in range(2):
                p = 0
                for kk in range(g * 128, (g + 1) * 128):
                    byte = int(packed[n, kk // 2])
                    idx = byte & 15 if kk % 2 == 0 else byte >> 4
                    p += int(q[m, kk]) * table[idx]
                tot += float(s[n, g]) * p
            want = float(np.float32(a[m])) * tot / 128.0
            assert abs(y64[m, n] - want) <= 1e-12 * max(1.0, abs(want))
