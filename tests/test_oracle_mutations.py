"""Plant plausible mistakes in the oracle (CPU only) and check a pin fails.

Each mutation is patched into the oracle module for the duration of one test,
so the oracle's own functions run with the mistake inside them.
"""

import types

import numpy as np
import pytest

import oracle
import oracle.iq8r_oracle as om
import pins
from iq8r_inputs import gen_workload

X, W = gen_workload("decode", m=3, n=40, k=1280, seed=101)


def np_proxy(**overrides):
    """A stand-in for the numpy module with some functions replaced."""
    ns = types.SimpleNamespace(**{k: getattr(np, k) for k in dir(np) if not k.startswith("__")})
    for k, v in overrides.items():
        setattr(ns, k, v)
    return ns


def fwht_sign_flipped(v):
    v = np.asarray(v, dtype=np.float32)
    x = v.reshape(-1, 128).copy()
    h = 1
    while h < 128:
        y = x.reshape(x.shape[0], 128 // (2 * h), 2, h)
        lo, hi = y[:, :, 0, :].copy(), y[:, :, 1, :].copy()
        y[:, :, 0, :] = lo - hi
        y[:, :, 1, :] = lo + hi
        h *= 2
    return x.reshape(v.shape)


def fwht_missing_stage(v):
    v = np.asarray(v, dtype=np.float32)
    x = v.reshape(-1, 128).copy()
    h = 1
    while h < 64:
        y = x.reshape(x.shape[0], 128 // (2 * h), 2, h)
        lo, hi = y[:, :, 0, :].copy(), y[:, :, 1, :].copy()
        y[:, :, 0, :] = lo + hi
        y[:, :, 1, :] = lo - hi
        h *= 2
    return x.reshape(v.shape)


def nearest_bf16_not_up(v):
    b = om.bf16_round_nearest(np.asarray(v, dtype=np.float64))
    return (b.astype(np.uint32) << 16).view(np.float32)


def fails(check):
    with pytest.raises(AssertionError):
        check()


@pytest.mark.parametrize("bad", [fwht_sign_flipped, fwht_missing_stage])
def test_broken_butterfly_is_caught(monkeypatch, bad):
    monkeypatch.setattr(om, "fwht128_f32", bad)
    fails(lambda: pins.check_transform(om.fwht128_f32, om.hadamard128))
    fails(lambda: pins.check_act_spike(om.act_quant))


def test_floor_instead_of_rint_is_caught(monkeypatch):
    monkeypatch.setattr(om, "np", np_proxy(rint=np.floor))
    fails(lambda: pins.check_act_properties(om.act_quant, om.fwht128_f64, X))
    fails(lambda: pins.check_pack_g256_properties(om.pack, om.fwht128_f64, W))


def test_floor_instead_of_ceil_for_sub_scale_is_caught(monkeypatch):
    monkeypatch.setattr(om, "np", np_proxy(ceil=np.floor))
    fails(lambda: pins.check_pack_g256_properties(om.pack, om.fwht128_f64, W))


def test_nearest_instead_of_round_up_scale_is_caught(monkeypatch):
    monkeypatch.setattr(om, "bf16_round_up", nearest_bf16_not_up)
    fails(lambda: pins.check_pack_golden(om.pack))


def test_wrong_activation_divisor_is_caught(monkeypatch):
    real = om.act_quant

    def act_128(x_bits, rotate=True):
        # codes on a 128-level grid while a still says amax / 127
        q, a = real(x_bits, rotate)
        xr = om.fwht128_f32(om.bf16_to_f32(x_bits))
        amax = np.abs(xr).max(axis=1)
        q = np.clip(np.rint(xr * (np.float32(128) / amax)[:, None]), -127, 127).astype(np.int8)
        return q, a

    fails(lambda: pins.check_act_properties(act_128, om.fwht128_f64, X))


def test_dropped_output_factor_is_caught():
    def linear_no_128(*args, **kw):
        kw["rotated"] = False
        return oracle.linear(*args, **kw)

    fails(lambda: pins.check_product_identity(oracle.act_quant, oracle.pack, linear_no_128, X, W, "g256"))


def test_misindexed_sub_scale_is_caught():
    def pack_reversed_s1(w_bits, fmt, rotate=True):
        codes, s1, s2 = oracle.pack(w_bits, fmt, rotate)
        return codes, s1[:, ::-1].copy(), s2

    fails(lambda: pins.check_product_identity(oracle.act_quant, pack_reversed_s1, oracle.linear, X, W, "g256"))


def test_shifted_block_boundary_is_caught():
    def partials_shifted(xq, codes, group):
        return oracle.partials(np.roll(xq, 1, axis=1), codes, group)

    rng = np.random.default_rng(12)
    xq = rng.integers(-127, 128, size=(2, 512)).astype(np.int8)
    codes = rng.integers(-127, 128, size=(3, 512)).astype(np.int8)
    fails(lambda: pins.check_partials_brute(partials_shifted, xq, codes, 256))


def test_transposed_weight_blocks_are_caught():
    def pack_swapped_halves(w_bits, fmt, rotate=True):
        codes, s1, s2 = oracle.pack(w_bits, fmt, rotate)
        n, k = codes.shape
        c = codes.reshape(n, k // 256, 256)[:, ::-1].reshape(n, k).copy()
        return c, s1, s2

    fails(lambda: pins.check_product_identity(oracle.act_quant, pack_swapped_halves, oracle.linear, X, W, "g256"))


def test_search_picking_the_worst_scale_is_caught(monkeypatch):
    """rule=search that keeps the largest error instead of the least."""
    import test_oracle
    real = om._group_sse
    monkeypatch.setattr(om, "_group_sse", lambda blocks, d: -real(blocks, d))
    with pytest.raises(AssertionError):
        test_oracle.test_pack_search_minimises_group_error("g128")


def test_search_with_a_misplaced_step_is_caught(monkeypatch):
    """rule=search that scores candidates at one step and keeps another."""
    import test_oracle
    real = om._group_sse
    monkeypatch.setattr(om, "_group_sse", lambda blocks, d: real(blocks, d * np.float32(1.01)))
    with pytest.raises(AssertionError):
        test_oracle.test_pack_search_minimises_group_error("g256")


def test_cb4_search_keeping_the_worst_scale_is_caught(monkeypatch):
    """The codebook's rule=search that keeps the largest error."""
    import test_oracle
    real = om._cb4_sse
    monkeypatch.setattr(om, "_cb4_sse", lambda blocks, s: -real(blocks, s))
    with pytest.raises(AssertionError):
        test_oracle.test_pack_search_cb4_minimises_group_error()


def test_cb4_swapped_nibbles_are_caught(monkeypatch):
    """The codebook's two indices a byte in the other order."""
    import test_oracle
    monkeypatch.setattr(om, "_cb4_nibbles", lambda idx: (idx[:, 1::2] | (idx[:, 0::2] << 4)).astype(np.uint8))
    with pytest.raises(AssertionError):
        test_oracle.test_cb4_nearest_level_and_layout()


def test_cb4_ties_to_the_smaller_level_are_caught(monkeypatch):
    """The codebook's nearest level with ties going down instead of up."""
    import test_oracle

    def ties_down(blocks, s):
        t = (blocks / s[..., None]).astype(np.float64)
        return np.argmin(np.abs(t[..., None] - om.CB4_TABLE.astype(np.float64)), axis=-1).astype(np.uint8)

    monkeypatch.setattr(om, "_cb4_indices", ties_down)
    with pytest.raises(AssertionError):
        test_oracle.test_cb4_ties_and_zero_group()


def test_rescore_of_the_neighbouring_row_is_caught(monkeypatch):
    """Rescoring that gathers the row after each candidate."""
    import test_oracle
    real = om.rescore

    def next_row(xq, a, fmt, codes, sub, scale_bits, cand, rotated=True):
        c = np.minimum(np.asarray(cand) + 1, np.asarray(codes).shape[0] - 1)
        return real(xq, a, fmt, codes, sub, scale_bits, c, rotated)

    monkeypatch.setattr(oracle, "rescore", next_row)
    with pytest.raises(AssertionError):
        test_oracle.test_rescore_is_the_linear_at_the_candidates("g256")


def test_cb4_scale_of_the_next_block_is_caught(monkeypatch):
    """The codebook linear scaling each block by its neighbour's scale."""
    import test_oracle
    real = om.linear

    def shifted(xq, a, fmt, codes, sub, scale_bits, rotated=True):
        if fmt == "cb4":
            scale_bits = np.roll(np.asarray(scale_bits), 1, axis=1)
        return real(xq, a, fmt, codes, sub, scale_bits, rotated)

    monkeypatch.setattr(oracle, "linear", shifted)
    with pytest.raises(AssertionError):
        test_oracle.test_cb4_linear_brute_force()


def test_dropped_tiny_row_prescale_is_caught(monkeypatch):
    """Without the 2^64 factor, 127 / amax overflows for a row of bf16
    subnormals and every code becomes +-127."""
    monkeypatch.setattr(om, "ACT_PRESCALE", np.float32(1.0))
    with np.errstate(over="ignore", invalid="ignore"):
        fails(lambda: pins.check_act_tiny_golden(om.act_quant))


def _act_prescale_variant(scale_a, scale_x):
    """The oracle's act_quant with the 2^64 prescale misapplied."""
    def act(x_bits, rotate=True):
        xr = om.fwht128_f32(om.bf16_to_f32(x_bits))
        amax = np.abs(xr).max(axis=1)
        c = np.where(amax < om.ACT_TINY, om.ACT_PRESCALE, np.float32(1.0)).astype(np.float32)
        inv = np.float32(127) / (amax * c)
        t = (xr * c[:, None] if scale_x else xr) * inv[:, None]
        q = np.clip(np.rint(t), -127, 127).astype(np.int8)
        a = ((amax * c) if scale_a else amax) / np.float32(127)
        return q, a.astype(np.float32)
    return act


def test_scale_from_the_prescaled_amax_is_caught():
    fails(lambda: pins.check_act_tiny_golden(_act_prescale_variant(scale_a=True, scale_x=True)))


def test_prescale_of_amax_only_is_caught():
    fails(lambda: pins.check_act_tiny_golden(_act_prescale_variant(scale_a=False, scale_x=False)))
