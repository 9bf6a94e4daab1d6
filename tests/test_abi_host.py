"""The C ABI on the host (no GPU): exports, packer parity, argument checks."""

import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import quantised_fwht128_act_b200 as iq8r
from iq8r_inputs import f32_to_bf16_bits, gen_workload

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "iq8r.h")


@pytest.fixture(scope="module")
def L():
    from quantised_fwht128_act_b200 import build
    build.build()
    return iq8r.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(iq8r_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("iq8r_pack", "iq8r_rotate_quant_act", "iq8r_linear", "iq8r_linear_partials",
                 "iq8r_packed_sizes", "iq8r_get_device_error", "iq8r_last_error"):
        assert want in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    # and they are real exported functions of this .so
    out = os.popen(f"nm -D --defined-only {iq8r.lib_path}").read()
    for name in declared_functions():
        assert re.search(rf"\bT {name}$", out, flags=re.M), name


def test_version(L):
    assert iq8r.iq8r_version() >= 100


def test_packed_sizes_match_oracle(L):
    for fmt in ("g256", "g128", "cb4"):
        for n, k in ((256, 512), (17408, 5120), (5120, 17408), (151936, 5120)):
            if fmt == "g256" and k % 256:
                continue
            assert iq8r.iq8r_packed_sizes(fmt, n, k) == oracle.packed_sizes(fmt, n, k)


def assert_pack_equal(w, fmt, rotate):
    c0, s0, sc0 = oracle.pack(w, fmt, rotate)
    c1, s1, sc1 = iq8r.iq8r_pack(w, fmt, rotate)
    assert np.array_equal(c0, c1)
    if fmt == "g256":
        assert np.array_equal(s0, s1)
    else:
        assert s1 is None
    assert np.array_equal(sc0, sc1.reshape(sc0.shape))


@pytest.mark.parametrize("fmt", ["g256", "g128"])
@pytest.mark.parametrize("rotate", [True, False])
def test_pack_byte_identical_to_oracle(L, fmt, rotate):
    _, w = gen_workload("pr1")
    assert_pack_equal(w, fmt, rotate)
    _, w = gen_workload("decode", m=1, n=300, k=5120, seed=21)
    assert_pack_equal(w, fmt, rotate)


def test_pack_edge_rows(L):
    rng = np.random.default_rng(5)
    k = 768
    w = np.zeros((8, k), np.float32)
    w[1] = 1e-38 * rng.standard_normal(k)          # scales in the bf16 subnormal range
    w[2] = 3e38 * np.sign(rng.standard_normal(k)) * 0.001
    w[3, 5] = 2.5                                   # one spike per row
    w[4] = rng.standard_normal(k) * np.exp(rng.uniform(-20, 20, k))  # wide dynamic range
    w[5, :256] = 0.0
    w[5, 256:] = 0.125                              # a zero block next to a flat one
    w[6] = -0.0
    w[7] = rng.integers(-3, 4, k)
    bits = f32_to_bf16_bits(w.astype(np.float32))
    for fmt in ("g256", "g128"):
        for rot in (True, False):
            assert_pack_equal(bits, fmt, rot)


def test_pack_thread_count_does_not_change_bytes(L):
    _, w = gen_workload("decode", m=1, n=513, k=1024, seed=22)
    a = iq8r.iq8r_pack(w, "g256", True, n_threads=1)
    b = iq8r.iq8r_pack(w, "g256", True, n_threads=7)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def status_of(fn):
    with pytest.raises(iq8r.IQ8RError) as e:
        fn()
    return e.value.status


def test_pack_rejects_bad_arguments(L):
    w = np.zeros((4, 200), np.uint16)
    assert status_of(lambda: iq8r.iq8r_pack(w, "g256", True)) == iq8r.IQ8R_ERR_INVALID_ARG
    assert "multiple of 256" in iq8r.iq8r_last_error()
    assert status_of(lambda: iq8r.iq8r_pack(np.zeros((4, 384), np.uint16), "g256")) == iq8r.IQ8R_ERR_INVALID_ARG
    assert L.iq8r_pack(7, 1, None, 1, 256, None, None, None, 0) == iq8r.IQ8R_ERR_INVALID_ARG
    assert L.iq8r_pack(0, 1, None, 1, 256, None, None, None, 0) == iq8r.IQ8R_ERR_INVALID_ARG
    assert L.iq8r_pack(0, 1, None, 0, 256, None, None, None, 0) == iq8r.IQ8R_OK  # n = 0: nothing to do


def test_gpu_calls_reject_bad_arguments_before_any_launch(L):
    # none of these reaches the GPU: every one fails host-side validation
    vp = ctypes.c_void_p
    aligned = vp(1 << 20)
    odd = vp((1 << 20) + 8)
    assert L.iq8r_rotate_quant_act(aligned, 4, 100, 1, aligned, aligned, None) == iq8r.IQ8R_ERR_INVALID_ARG
    assert L.iq8r_rotate_quant_act(aligned, -1, 128, 1, aligned, aligned, None) == iq8r.IQ8R_ERR_INVALID_ARG
    assert L.iq8r_rotate_quant_act(aligned, 4, 128, 2, aligned, aligned, None) == iq8r.IQ8R_ERR_INVALID_ARG
    assert L.iq8r_rotate_quant_act(None, 4, 128, 1, aligned, aligned, None) == iq8r.IQ8R_ERR_INVALID_ARG
    assert L.iq8r_rotate_quant_act(odd, 4, 128, 1, aligned, aligned, None) == iq8r.IQ8R_ERR_INVALID_ARG
    assert "aligned" in iq8r.iq8r_last_error()
    assert L.iq8r_rotate_quant_act(None, 0, 128, 1, None, None, None) == iq8r.IQ8R_OK  # m = 0

    def weight(**kw):
        d = dict(fmt=0, rotated=1, n=256, k=512, codes=1 << 20, sub_scale=1 << 21, scale=1 << 22)
        d.update(kw)
        return iq8r._Weight(d["fmt"], d["rotated"], d["n"], d["k"], d["codes"], d["sub_scale"], d["scale"])

    def lin(w, m=4, xq=aligned, xs=aligned, y=aligned, path=0):
        return L.iq8r_linear_ex(xq, xs, m, ctypes.byref(w), y, path, None)

    bad = [
        weight(k=384),               # trunk K must be a multiple of 256
        weight(fmt=1, k=200),        # lm_head K must be a multiple of 128
        weight(fmt=5),
        weight(rotated=3),
        weight(n=0),
        weight(codes=0),
        weight(sub_scale=0),
        weight(codes=(1 << 20) + 4),
        weight(sub_scale=(1 << 21) + 8),
    ]
    for w in bad:
        assert lin(w) == iq8r.IQ8R_ERR_INVALID_ARG, iq8r.iq8r_last_error()
    assert L.iq8r_linear_ex(aligned, aligned, 4, None, aligned, 0, None) == iq8r.IQ8R_ERR_INVALID_ARG
    assert lin(weight(), m=-2) == iq8r.IQ8R_ERR_INVALID_ARG
    assert lin(weight(), y=odd) == iq8r.IQ8R_ERR_INVALID_ARG
    assert lin(weight(), xq=None) == iq8r.IQ8R_ERR_INVALID_ARG
    assert lin(weight(), path=9) == iq8r.IQ8R_ERR_INVALID_ARG
    assert lin(weight(), path=0x200) == iq8r.IQ8R_ERR_INVALID_ARG          # an unknown flag
    assert lin(weight(), path=3 | iq8r.IQ8R_PATH_FLAG_WEIGHTS_WRITTEN) == iq8r.IQ8R_ERR_INVALID_ARG
    assert lin(weight(), m=0) == iq8r.IQ8R_OK
    w = weight()
    assert L.iq8r_linear_partials(aligned, 4, ctypes.byref(w), 10, 5, aligned, 0, None) == iq8r.IQ8R_ERR_INVALID_ARG
    assert L.iq8r_linear_partials(aligned, 4, ctypes.byref(w), 0, 257, aligned, 0, None) == iq8r.IQ8R_ERR_INVALID_ARG
    # row n0 = 1 of a K = 512 weight starts 512 bytes in: aligned, fine; odd K for lm_head is not
    assert L.iq8r_linear_partials(aligned, 4, ctypes.byref(w), 0, 256, None, 0, None) == iq8r.IQ8R_ERR_INVALID_ARG


def test_last_error_is_cleared_by_a_good_call(L):
    assert L.iq8r_pack(7, 1, None, 1, 256, None, None, None, 0) != 0
    assert iq8r.iq8r_last_error() != ""
    iq8r.iq8r_packed_sizes("g256", 4, 256)
    assert iq8r.iq8r_last_error() == ""


@pytest.mark.parametrize("fmt", ["g256", "g128"])
def test_pack_search_byte_identical_to_oracle(L, fmt):
    """rule=search: the C++ packer's chosen scales and codes are the
    oracle's, on the workload generator and on edge rows (zero, a spike,
    a constant row, tiny values)."""
    _, w = gen_workload("decode", m=1, n=120, k=1024, seed=21)
    w = w.copy()
    w[3] = 0
    w[4] = 0
    w[4, 5] = f32_to_bf16_bits(np.array([3.0], np.float32))[0]
    w[5] = f32_to_bf16_bits(np.full(1024, 0.25, np.float32))
    w[6] = f32_to_bf16_bits(np.full(1024, 1e-30, np.float32))
    got = iq8r.iq8r_pack(w, fmt, True, rule="search")
    want = oracle.pack_search(w, fmt, True)
    for g, e in zip(got, want):
        assert (g is None and e is None) or np.array_equal(g, e)


def test_pack_rule_is_checked(L):
    w = np.zeros((2, 256), np.uint16)
    codes = np.empty((2, 256), np.int8)
    sub = np.empty((2, 1), np.uint8)
    scale = np.empty((2,), np.uint16)
    st = L.iq8r_pack_ex(0, 1, 7, w.ctypes.data, 2, 256, codes.ctypes.data, sub.ctypes.data, scale.ctypes.data, 1)
    assert st == iq8r.IQ8R_ERR_INVALID_ARG


def test_pack_cb4_byte_identical_to_oracle(L):
    """The drafter's codebook: indices and scales are the oracle's, for both
    rules, on the generator and on edge rows (zero, a spike, constants, tiny
    values)."""
    _, w = gen_workload("decode", m=1, n=90, k=1024, seed=23)
    w = w.copy()
    w[3] = 0
    w[4] = 0
    w[4, 9] = f32_to_bf16_bits(np.array([-2.0], np.float32))[0]
    w[5] = f32_to_bf16_bits(np.full(1024, 0.75, np.float32))
    w[6] = f32_to_bf16_bits(np.full(1024, 1e-30, np.float32))
    for rotate in (True, False):
        codes, sub, scale = iq8r.iq8r_pack(w, "cb4", rotate)
        p, s = oracle.pack_cb4(w, rotate)
        assert sub is None and np.array_equal(codes, p) and np.array_equal(scale, s)
        codes, sub, scale = iq8r.iq8r_pack(w, "cb4", rotate, rule="search")
        p, s_none, s = oracle.pack_search(w, "cb4", rotate)
        assert sub is None and s_none is None
        assert np.array_equal(codes, p) and np.array_equal(scale, s)


def test_later_calls_reject_bad_arguments_before_any_launch(L):
    """The codebook format, rescoring, the no-allocation linear and the
    one-call layer validate on the host: none of these reaches the GPU."""
    vp = ctypes.c_void_p
    aligned = vp(1 << 20)
    odd = vp((1 << 20) + 8)

    def weight(**kw):
        d = dict(fmt=2, rotated=1, n=256, k=512, codes=1 << 20, sub_scale=0, scale=1 << 22)
        d.update(kw)
        return iq8r._Weight(d["fmt"], d["rotated"], d["n"], d["k"], d["codes"], d["sub_scale"], d["scale"])

    cb = weight()
    # the codebook format runs on its GEMV only, and needs K % 128 == 0
    assert L.iq8r_linear_ex(aligned, aligned, 4, ctypes.byref(cb), aligned, iq8r.IQ8R_PATH_TC, None) == \
        iq8r.IQ8R_ERR_UNSUPPORTED
    assert "GEMV only" in iq8r.iq8r_last_error()
    assert L.iq8r_linear_ex(aligned, aligned, 4, ctypes.byref(weight(k=200)), aligned, 0, None) == \
        iq8r.IQ8R_ERR_INVALID_ARG

    trunk = weight(fmt=0, sub_scale=1 << 21)
    cand = aligned

    def rescore(w=trunk, m=8, xq=aligned, xs=aligned, c=cand, nc=32, out=aligned):
        return L.iq8r_rescore(xq, xs, m, ctypes.byref(w), c, nc, out, None)

    assert rescore(nc=-1) == iq8r.IQ8R_ERR_INVALID_ARG
    assert rescore(nc=65535 * 32 + 1) == iq8r.IQ8R_ERR_INVALID_ARG
    assert rescore(w=weight(fmt=0, sub_scale=1 << 21, k=49408)) == iq8r.IQ8R_ERR_UNSUPPORTED
    assert rescore(w=cb) == iq8r.IQ8R_ERR_UNSUPPORTED
    assert rescore(c=None) == iq8r.IQ8R_ERR_INVALID_ARG
    assert rescore(xq=odd) == iq8r.IQ8R_ERR_INVALID_ARG
    assert rescore(m=-1) == iq8r.IQ8R_ERR_INVALID_ARG
    assert rescore(m=0) == iq8r.IQ8R_OK and rescore(nc=0) == iq8r.IQ8R_OK

    # the no-allocation linear checks like iq8r_linear
    assert L.iq8r_linear_noalloc(aligned, aligned, 4, ctypes.byref(weight(fmt=0, sub_scale=0)), aligned, None) == \
        iq8r.IQ8R_ERR_INVALID_ARG
    assert L.iq8r_linear_noalloc(aligned, aligned, 4, ctypes.byref(trunk), odd, None) == iq8r.IQ8R_ERR_INVALID_ARG
    assert L.iq8r_linear_noalloc(aligned, aligned, 0, ctypes.byref(trunk), aligned, None) == iq8r.IQ8R_OK

    # the one-call layer: beyond one launch it stages the codes, so it needs
    # xq_out and x_scale_out
    assert L.iq8r_linear_bf16(aligned, 16, ctypes.byref(trunk), aligned, None, None, None) == \
        iq8r.IQ8R_ERR_INVALID_ARG
    assert "xq_out" in iq8r.iq8r_last_error()
    assert L.iq8r_linear_bf16(None, 1, ctypes.byref(trunk), aligned, None, None, None) == iq8r.IQ8R_ERR_INVALID_ARG
    assert L.iq8r_linear_bf16(aligned, 1, ctypes.byref(trunk), odd, None, None, None) == iq8r.IQ8R_ERR_INVALID_ARG
    assert L.iq8r_linear_bf16(aligned, 0, ctypes.byref(trunk), aligned, None, None, None) == iq8r.IQ8R_OK

    # the host-buffer layer checks before its first copy
    def host(m=1, xh=aligned, xd=aligned, yd=aligned, yh=aligned, w=trunk, xq=None):
        return L.iq8r_linear_bf16_host(xh, m, ctypes.byref(w), xd, yd, yh, xq, None, None)

    assert host(xh=None) == iq8r.IQ8R_ERR_INVALID_ARG
    assert host(yh=None) == iq8r.IQ8R_ERR_INVALID_ARG
    assert host(xd=odd) == iq8r.IQ8R_ERR_INVALID_ARG
    assert host(yd=None) == iq8r.IQ8R_ERR_INVALID_ARG
    assert host(xq=odd) == iq8r.IQ8R_ERR_INVALID_ARG
    assert host(m=-1) == iq8r.IQ8R_ERR_INVALID_ARG
    assert host(w=weight(fmt=0, sub_scale=0)) == iq8r.IQ8R_ERR_INVALID_ARG
    assert host(m=0) == iq8r.IQ8R_OK

    # the self-test's limit is checked before its launch
    assert L.iq8r_selftest_wait_timeout(10, None) == iq8r.IQ8R_ERR_INVALID_ARG


def test_pack_accepts_torch_bf16_tensors(L):
    """The binding takes a CPU torch bf16 tensor as well as raw bit patterns
    and packs the same bytes."""
    import torch
    _, w = gen_workload("decode", m=1, n=24, k=512, seed=29)
    t = torch.from_numpy(w.view(np.int16)).view(torch.bfloat16)
    for fmt in ("g256", "g128", "cb4"):
        a = iq8r.iq8r_pack(w, fmt, True)
        b = iq8r.iq8r_pack(t, fmt, True)
        for x, y in zip(a, b):
            assert (x is None and y is None) or np.array_equal(x, y)
