"""Checks that pin the oracle to facts outside itself.

Each check takes the oracle functions it exercises as arguments, so that the
mutation tests can hand it a deliberately broken variant and see it fail.
"""

from __future__ import annotations

import json
import os

import numpy as np
import scipy.linalg

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
U32 = 2.0 ** -24  # float32 unit roundoff


def golden(name: str):
    with open(os.path.join(GOLDEN, "hand_examples.json")) as f:
        return json.load(f)[name]


def bits(s: str) -> int:
    return int(s, 16)


def bf16(v) -> np.ndarray:
    """float values that are exactly bf16 -> bit patterns (test-side helper)."""
    u = np.asarray(v, dtype=np.float32).reshape(-1).view(np.uint32)
    assert not np.any(u & 0xFFFF)
    return (u >> 16).astype(np.uint16)


def bf16_val(b) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ------------------------------------------------------------------ transform

def check_transform(fwht128_f32, hadamard128):
    """H against scipy's Sylvester construction, H H = 128 I, and the
    closed-form images of e_j, 1 and e0 + 2 e1."""
    H = hadamard128()
    assert np.array_equal(H, scipy.linalg.hadamard(128))
    assert np.array_equal(H @ H, 128 * np.eye(128, dtype=np.int64))
    E = np.eye(128, dtype=np.float32)
    # T(e_j) is column j of H (= row j: H is symmetric)
    assert np.array_equal(fwht128_f32(E), H.T.astype(np.float32))
    ones = fwht128_f32(np.ones((1, 128), np.float32))[0]
    g = golden("fwht_ones")
    assert ones[0] == g["x_prime_0"] and np.all(ones[1:] == g["x_prime_rest"])
    g = golden("fwht_e0_plus_2e1")
    x = np.zeros((1, 128), np.float32)
    for k, v in g["x_nonzero"].items():
        x[0, int(k)] = v
    t = fwht128_f32(x)[0]
    assert np.all(t[0::2] == g["x_prime_even"]) and np.all(t[1::2] == g["x_prime_odd"])
    # T(T(v)) = 128 v exactly for small integers (all sums exact in float32)
    rng = np.random.default_rng(7)
    v = rng.integers(-50, 51, size=(4, 384)).astype(np.float32)
    assert np.array_equal(fwht128_f32(fwht128_f32(v)), 128 * v)
    # each 128 of K is rotated on its own
    w = rng.standard_normal((3, 512)).astype(np.float32)
    whole = fwht128_f32(w)
    for c in range(4):
        assert np.array_equal(whole[:, 128 * c:128 * (c + 1)], fwht128_f32(w[:, 128 * c:128 * (c + 1)]))


def check_transform_rounding(fwht128_f32):
    """The float32 butterflies agree with scipy's float64 H x within the
    rounding bound of 7 stages, 7 u sum|x| per 128-chunk."""
    Hs = scipy.linalg.hadamard(128).astype(np.float64)
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((64, 256)) * np.exp(rng.uniform(-6, 6, (64, 1)))).astype(np.float32)
    got = fwht128_f32(x).astype(np.float64)
    xc = x.astype(np.float64).reshape(64, 2, 128)
    ref = (xc @ Hs.T).reshape(64, 256)
    bound = 7.0 * U32 * np.repeat(np.abs(xc).sum(axis=2), 128, axis=1) * (1 + 1e-6)
    assert np.all(np.abs(got - ref) <= bound)


# ------------------------------------------------------------ activations

def check_act_golden(act_quant):
    g = golden("act_quant_e0_plus_2e1")
    x = np.zeros((1, g["k"]), np.float32)
    x[0, 0], x[0, 1] = 1.0, 2.0
    q, a = act_quant(bf16(x).reshape(1, -1), rotate=True)
    assert np.all(q[0, 0::2] == g["code_even"]) and np.all(q[0, 1::2] == g["code_odd"])
    assert a[0] == np.float32(3.0) / np.float32(127.0)


def check_act_properties(act_quant, fwht128_f64, x_bits):
    """Every nonzero row reaches 127; codes are the nearest integers to
    x' / a (no clipping); reconstruction within a/2 plus the transform's
    float32 rounding."""
    q, a = act_quant(x_bits, rotate=True)
    xf = bf16_val(x_bits).reshape(x_bits.shape).astype(np.float64)
    xr = fwht128_f64(xf)
    amax = np.abs(xr).max(axis=1)
    nz = amax > 0
    assert np.all(np.abs(q[nz].astype(np.int64)).max(axis=1) == 127)
    assert np.all(q[~nz] == 0) and np.all(a[~nz] == 0)
    # a = amax / 127 up to the float32 rounding of the transform and divide
    # (half a subnormal step, 2^-150, when a falls below 2^-126)
    sub = 2.0 ** -150
    assert np.all(np.abs(a[nz].astype(np.float64) - amax[nz] / 127.0) <= 1e-5 * amax[nz] / 127.0 + sub)
    # |x' - a q| <= a/2 (+ transform rounding), i.e. rint, not floor or clip;
    # a subnormal a carries up to 127 half-steps of its own rounding
    abs_chunk = np.repeat(np.abs(xf).reshape(xf.shape[0], -1, 128).sum(axis=2), 128, axis=1)
    err = np.abs(xr - a[:, None].astype(np.float64) * q)
    slack = 8 * U32 * abs_chunk + 2e-6 * amax[:, None] + 128 * sub
    assert np.all(err <= a[:, None] / 2 + slack)


def check_act_tiny_golden(act_quant):
    """Rows with amax below 2^-64: hand-derived codes and scales of a row of
    bf16 subnormals (where 127 / amax would overflow float32) and of a small
    normal row (where the exact 2^64 prescale must change no code)."""
    for name in ("act_quant_tiny_row", "act_quant_small_row_unchanged"):
        g = golden(name)
        x = np.zeros((1, g["k"]), np.uint16)
        for k, v in g["x_bits"].items():
            x[0, int(k)] = bits(v)
        q, a = act_quant(x, rotate=True)
        assert np.all(q[0, 0::2] == g["code_even"]) and np.all(q[0, 1::2] == g["code_odd"])
        assert int(np.asarray(a, np.float32).view(np.uint32)[0]) == bits(g["a_f32_bits"])


def check_act_spike(act_quant):
    """A spike c e_j rotates to +-c over its 128-chunk: all codes +-127 there,
    0 elsewhere; a zero row gives a = 0 and zero codes."""
    x = np.zeros((3, 384), np.float32)
    x[0, 128 + 7] = 3.5
    x[1, 300] = -0.125
    q, a = act_quant(bf16(x).reshape(3, 384), rotate=True)
    assert np.all(np.abs(q[0, 128:256]) == 127) and np.all(q[0, :128] == 0) and np.all(q[0, 256:] == 0)
    assert np.all(np.abs(q[1, 256:]) == 127) and np.all(q[1, :256] == 0)
    assert np.all(q[2] == 0) and a[2] == 0
    # sign pattern of the chunk follows column j of H (j = 7 has an odd
    # popcount, so a butterfly with its signs swapped would flip it)
    H = scipy.linalg.hadamard(128)
    assert np.array_equal(np.sign(q[0, 128:256]), H[:, 7])


# ---------------------------------------------------------------- pack

def check_pack_golden(pack):
    g = golden("pack_g128_half_e0")
    w = np.zeros((1, g["k"]), np.float32)
    w[0, 0] = 0.5
    codes, sub, scale = pack(bf16(w).reshape(1, -1), "g128", True)
    assert sub is None
    assert int(scale.reshape(-1)[0]) == bits(g["scale_bits"])
    assert bf16_val(scale.reshape(-1)[:1])[0] == g["scale_value"]
    assert np.all(codes == g["code_all"])
    g = golden("pack_g256_e0")
    w = np.zeros((1, g["k"]), np.float32)
    w[0, 0] = 1.0
    codes, sub, scale = pack(bf16(w).reshape(1, -1), "g256", True)
    assert int(scale.reshape(-1)[0]) == bits(g["s2_bits"])
    assert bf16_val(scale.reshape(-1)[:1])[0] == g["s2_value"]
    assert list(sub.reshape(-1)) == g["s1"]
    assert np.all(codes[0, :128] == g["codes_k0_128"]) and np.all(codes[0, 128:] == g["codes_rest"])


def check_pack_g256_properties(pack, fwht128_f64, w_bits):
    codes, s1, s2b = pack(w_bits, "g256", True)
    n, k = w_bits.shape
    ng = k // 256
    assert codes.shape == (n, k) and codes.dtype == np.int8
    assert s1.shape == (n, ng) and s1.dtype == np.uint8
    assert s2b.shape == (n,) and s2b.dtype == np.uint16
    assert codes.min() >= -127
    wr = fwht128_f64(bf16_val(w_bits).reshape(n, k).astype(np.float64))
    A = np.abs(wr).reshape(n, ng, 256).max(axis=2)
    R = A.max(axis=1)
    s2 = bf16_val(s2b).astype(np.float64)
    # s2 is R / 32385 rounded up onto the bf16 grid: within one bf16 step above
    rel = 1e-6
    assert np.all(s2 >= R / 32385.0 * (1 - rel))
    assert np.all(s2 <= R / 32385.0 * (1 + 2.0 ** -7) * (1 + rel))
    # no sub-scale clips: A <= 127 * s2 * s1 (to float32 rounding), s1 in [1, 255]
    d = s2[:, None] * s1.astype(np.float64)
    pos = A > 0
    assert np.all((s1[pos] >= 1) & (s1[pos] <= 255)) and np.all(s1[~pos] == 0)
    assert np.all(A[pos] <= 127 * d[pos] * (1 + 1e-5))
    # s1 is the smallest such integer: one less would clip
    small = pos & (s1 > 1)
    assert np.all(A[small] > 127 * s2[:, None].repeat(ng, 1)[small] * (s1[small] - 1.0) * (1 - 1e-5))
    # codes are nearest: |W' - q d| <= d/2 (+ float32 rounding of W')
    dk = np.repeat(d, 256, axis=1)
    err = np.abs(wr - codes * dk)
    slack = 8 * U32 * np.repeat(np.abs(bf16_val(w_bits).reshape(n, k // 128, 128).astype(np.float64)).sum(axis=2), 128, axis=1)
    assert np.all(err <= dk / 2 * (1 + 1e-6) + slack)
    # the block holding the row maximum reaches |code| = 127
    gmax = A.argmax(axis=1)
    blk = np.abs(codes.reshape(n, ng, 256)[np.arange(n), gmax].astype(np.int64)).max(axis=1)
    assert np.all(blk[R > 0] == 127)


def check_pack_g128_properties(pack, fwht128_f64, w_bits):
    codes, sub, sb = pack(w_bits, "g128", True)
    n, k = w_bits.shape
    ng = k // 128
    assert sub is None and sb.shape == (n, ng) and sb.dtype == np.uint16
    wr = fwht128_f64(bf16_val(w_bits).reshape(n, k).astype(np.float64))
    A = np.abs(wr).reshape(n, ng, 128).max(axis=2)
    s = bf16_val(sb).reshape(n, ng).astype(np.float64)
    assert np.all(s >= A / 127.0 * (1 - 1e-6))
    assert np.all(s <= A / 127.0 * (1 + 2.0 ** -7) * (1 + 1e-6))
    sk = np.repeat(s, 128, axis=1)
    slack = 8 * U32 * np.repeat(np.abs(bf16_val(w_bits).reshape(n, ng, 128).astype(np.float64)).sum(axis=2), 128, axis=1)
    assert np.all(np.abs(wr - codes * sk) <= sk / 2 * (1 + 1e-6) + slack)
    mx = np.abs(codes.reshape(n, ng, 128).astype(np.int64)).max(axis=2)
    assert np.all((mx[A > 0] == 126) | (mx[A > 0] == 127))


# ---------------------------------------------------------------- linear

def brute_partials(xq, codes, group):
    """Pure-Python integer sums (tiny shapes only)."""
    m, k = xq.shape
    n = codes.shape[0]
    out = np.zeros((m, n, k // group), dtype=np.int64)
    xl = xq.astype(int).tolist()
    wl = codes.astype(int).tolist()
    for i in range(m):
        for j in range(n):
            for g in range(k // group):
                out[i, j, g] = sum(xl[i][t] * wl[j][t] for t in range(g * group, (g + 1) * group))
    return out


def check_partials_brute(partials, xq, codes, group):
    assert np.array_equal(partials(xq, codes, group), brute_partials(xq, codes, group))


def check_linear_golden(act_quant, pack, partials, linear, linear_bf16):
    g = golden("linear_g256_e0")
    k = g["k"]
    x = np.zeros((1, k), np.float32)
    x[0, 0], x[0, 1] = 1.0, 2.0
    w = np.zeros((1, k), np.float32)
    w[0, 0] = 1.0
    xq, a = act_quant(bf16(x).reshape(1, k), rotate=True)
    codes, s1, s2 = pack(bf16(w).reshape(1, k), "g256", True)
    P = partials(xq, codes, 256)
    assert list(P.reshape(-1)) == g["P"]
    assert int((P[0, 0] * s1[0].astype(np.int64)).sum()) == g["S"]
    y = linear(xq, a, "g256", codes, s1, s2, rotated=True)
    assert abs(y[0, 0] - g["y_approx"]) < 1e-5
    assert abs(y[0, 0] - g["x_dot_w_exact"]) < 0.01
    assert int(linear_bf16(y).reshape(-1)[0]) == bits(g["y_bits"])


def quant_error_bound(x_bits, w_bits, fmt, xq, a, codes, sub, scale_bits):
    """Closed-form bound on |y - x W^T| from the two roundings.

    With x' = a q_x + e_x (|e_x| <= a/2) and W' = d q_w + e_w (|e_w| <= d/2),
    (a q_x).(d q_w)/128 - x.w = -(x'.e_w + e_x.W' - e_x.e_w)/128, so
    |y - x.w| <= sum_k (|x'_k| d_k / 2 + a |W'_k| / 2 + a d_k / 4) / 128.
    """
    H = scipy.linalg.hadamard(128).astype(np.float64)
    m, k = x_bits.shape
    n = w_bits.shape[0]
    xf = bf16_val(x_bits).reshape(m, k).astype(np.float64)
    wf = bf16_val(w_bits).reshape(n, k).astype(np.float64)
    xr = (xf.reshape(m, -1, 128) @ H.T).reshape(m, k)
    wr = (wf.reshape(n, -1, 128) @ H.T).reshape(n, k)
    if fmt == "g256":
        d = np.repeat(bf16_val(scale_bits).astype(np.float64)[:, None] * sub.astype(np.float64), 256, axis=1)
    else:
        d = np.repeat(bf16_val(scale_bits).reshape(n, -1).astype(np.float64), 128, axis=1)
    av = a.astype(np.float64)[:, None]
    bound = (np.abs(xr) @ d.T / 2 + av * np.abs(wr).sum(axis=1)[None, :] / 2 + av * d.sum(axis=1)[None, :] / 4) / 128
    # float32 rounding of both transforms (relative ~8u), generously
    bound += 1e-5 * (np.abs(xr) @ np.abs(wr).T) / 128
    return xf @ wf.T, bound


def check_product_identity(act_quant, pack, linear, x_bits, w_bits, fmt):
    """y from the rotated int8 path equals x W^T (unrotated, float64) within
    the closed-form quantisation bound."""
    xq, a = act_quant(x_bits, rotate=True)
    codes, sub, sc = pack(w_bits, fmt, True)
    y = linear(xq, a, fmt, codes, sub, sc, rotated=True)
    exact, bound = quant_error_bound(x_bits, w_bits, fmt, xq, a, codes, sub, sc)
    assert np.all(np.abs(y - exact) <= bound)
    # and typically far inside it: the rms error is a few percent of the rms
    # output, so a wrong scale, index or sign cannot hide under the bound
    assert np.sqrt(np.mean((y - exact) ** 2)) < 0.1 * np.sqrt(np.mean(exact ** 2))
