"""CUDA path against the oracle, through the C ABI (needs a B200).

Bit-exact: activation codes and scales, per-block int32 partial sums.
Within tolerance (see tolerance.py): the bf16 outputs.
"""

import functools

import numpy as np
import pytest
import torch

import oracle
import quantised_fwht128_act_b200 as iq8r
from iq8r_inputs import WORKLOADS, f32_to_bf16_bits, gen_workload
from tolerance import check_output

pytestmark = pytest.mark.gpu


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.fixture(scope="module", autouse=True)
def built():
    from quantised_fwht128_act_b200 import build
    build.build()
    iq8r.lib()
    yield
    iq8r.iq8r_get_device_error()


@functools.lru_cache(maxsize=8)
def case(name, m=None, n=None, k=None, seed=None):
    """Inputs, oracle-packed weight and device copies for one configuration."""
    x, w = gen_workload(name, m=m, n=n, k=k, seed=seed)
    fmt = WORKLOADS[name].fmt
    codes, sub, scale = oracle.pack(w, fmt, True)
    W = iq8r.IQ8RWeight.from_packed(codes, sub, scale, fmt, True)
    return x, w, fmt, (codes, sub, scale), W


def run_act(x_bits, rotate=True):
    xq, xs = iq8r.iq8r_rotate_quant_act(dev_bf16(x_bits), rotate)
    torch.cuda.synchronize()
    return xq.cpu().numpy(), xs.cpu().numpy()


def assert_act_exact(x_bits, rotate=True):
    q0, a0 = oracle.act_quant(x_bits, rotate)
    q1, a1 = run_act(x_bits, rotate)
    assert np.array_equal(q0, q1), f"{np.sum(q0 != q1)} codes differ"
    assert np.array_equal(a0.view(np.uint32), a1.view(np.uint32))


# ------------------------------------------------------------ activations

@pytest.mark.parametrize("name", ["pr1", "decode", "verify8", "verify128", "lm_head8"])
def test_act_bit_exact_workloads(name):
    x, _ = gen_workload(name, n=8)
    assert_act_exact(x)


def test_act_bit_exact_prefill_full():
    x, _ = gen_workload("prefill", n=8)
    assert_act_exact(x)


# small M: a row spread over a cluster of CTAs; M >= 148: one CTA a row, the
# row in registers up to K = 16384, two passes above
@pytest.mark.parametrize("m,k", [(5, 128), (3, 640), (7, 2176), (1, 16384), (2, 16512), (3, 33024), (33, 1152),
                                 (16, 17408), (147, 256), (148, 5120), (160, 16512), (149, 768), (150, 2560),
                                 (152, 1152), (200, 4096), (300, 16384)])
def test_act_bit_exact_ragged_shapes(m, k):
    x, _ = gen_workload("decode", m=m, n=8, k=k, seed=m * 1000 + k)
    assert_act_exact(x)
    assert_act_exact(x, rotate=False)


def special_rows(k, seed=3):
    """Rows at the edges of the quantiser's definition: zero, a spike, large
    magnitudes, bf16 subnormals (amax below 127 / FLT_MAX, where the 2^64
    prescale defines the codes), small rows that are prescaled while
    127 / amax stays finite, exact integers and mixed magnitudes."""
    rng = np.random.default_rng(seed)
    x = np.zeros((10, k), np.float32)
    x[1, 700 % k] = -3.25                               # spike
    x[2] = rng.standard_normal(k) * 1e35                # large, transform stays finite
    x[3] = rng.standard_normal(k) * 1e-39               # bf16 subnormals
    x[4] = np.round(rng.standard_normal(k) * 4)         # exact small integers
    x[5] = rng.standard_normal(k) * np.exp(rng.uniform(-30, 30, k))
    x[6] = rng.standard_normal(k) * 2.0 ** -70          # prescaled, 127 / amax finite
    x[7] = rng.standard_normal(k) * 2.0 ** -140         # the smallest subnormals and zeros
    x[8, 0], x[8, 1] = 2.0 ** -130, 2.0 ** -129         # the hand-derived tiny golden row
    x[9] = rng.standard_normal(k) * np.exp(rng.uniform(-95, -85, k))
    return f32_to_bf16_bits(x)


def assert_act_exact_no_fp_traps(bits, rotate=True):
    with np.errstate(over="raise", invalid="raise", divide="raise"):
        assert_act_exact(bits, rotate)


@pytest.mark.parametrize("m_rep,k", [(1, 1024), (16, 1024), (16, 17408), (1, 33024)])
def test_act_special_rows(m_rep, k):
    """Each activation kernel on the special rows: a cluster of CTAs a row
    (few tokens), one CTA a row (148 tokens and up: the rows repeated), and
    the two-pass kernel (K above 16384)."""
    bits = np.tile(special_rows(k), (m_rep, 1))
    assert_act_exact_no_fp_traps(bits)
    assert_act_exact_no_fp_traps(bits, rotate=False)
    q, a = run_act(bits)
    # the golden row: codes 127 / -42 in the first chunk, scale 12385 * 2^-149
    assert np.all(q[8, 0:128:2] == 127) and np.all(q[8, 1:128:2] == -42) and np.all(q[8, 128:] == 0)
    assert a[8:9].view(np.uint32)[0] == 0x3061


def test_act_special_rows_fused_gemv_prologue():
    """The GEMV's fused prologue (iq8r_linear_bf16, one and two tokens)
    writes the same codes and scales for the special rows."""
    k, n = 1024, 64
    bits = special_rows(k)
    _, w = gen_workload("decode", m=1, n=n, k=k, seed=5)
    codes, sub, scale = oracle.pack(w, "g256", True)
    W = iq8r.IQ8RWeight.from_packed(codes, sub, scale, "g256", True)
    with np.errstate(over="raise", invalid="raise", divide="raise"):
        q0, a0 = oracle.act_quant(bits)
    for i in range(0, bits.shape[0], 2):
        xb = bits[i:i + 2]
        xq_out = torch.empty(xb.shape, dtype=torch.int8, device="cuda")
        xs_out = torch.empty((xb.shape[0],), dtype=torch.float32, device="cuda")
        iq8r.iq8r_linear_bf16(dev_bf16(xb), W, xq_out=xq_out, x_scale_out=xs_out)
        torch.cuda.synchronize()
        assert np.array_equal(xq_out.cpu().numpy(), q0[i:i + 2])
        assert np.array_equal(xs_out.cpu().numpy().view(np.uint32), a0[i:i + 2].view(np.uint32))


def test_act_empty_batch_is_a_no_op():
    x = torch.zeros((0, 256), dtype=torch.bfloat16, device="cuda")
    xq, xs = iq8r.iq8r_rotate_quant_act(x)
    assert xq.shape == (0, 256) and xs.shape == (0,)


# ------------------------------------------------------------- partials

def gpu_partials(x_bits, W, n0=0, n1=None, path=iq8r.IQ8R_PATH_AUTO):
    xq, _ = iq8r.iq8r_rotate_quant_act(dev_bf16(x_bits))
    p = iq8r.iq8r_linear_partials(xq, W, n0, n1, path=path)
    torch.cuda.synchronize()
    return p.cpu().numpy()


@pytest.mark.parametrize("name", ["pr1", "decode", "verify8"])
def test_partials_bit_exact_workloads(name):
    x, _, fmt, (codes, _, _), W = case(name)
    g = 256 if fmt == "g256" else 128
    xq, _ = oracle.act_quant(x)
    assert np.array_equal(gpu_partials(x, W), oracle.partials(xq, codes, g))


# the GEMV forced (every token-tile width 1..8), and the library's own choice
@pytest.mark.parametrize("path", ["gemv", "auto"])
@pytest.mark.parametrize("m,n,k", [(3, 1000, 768), (5, 37, 2304), (13, 64, 512), (2, 9, 4352), (8, 20, 256),
                                   (7, 300, 1024), (4, 129, 2560)])
def test_partials_bit_exact_ragged(m, n, k, path):
    x, _, _, (codes, _, _), W = case("decode", m=m, n=n, k=k, seed=7 + m + n + k)
    xq, _ = oracle.act_quant(x)
    p = iq8r.IQ8R_PATH_GEMV if path == "gemv" else iq8r.IQ8R_PATH_AUTO
    assert np.array_equal(gpu_partials(x, W, path=p), oracle.partials(xq, codes, 256))


def test_partials_lm_head_windows():
    x, _, _, (codes, _, _), W = case("lm_head8", m=8, n=4096, k=5120, seed=44)
    xq, _ = oracle.act_quant(x)
    for n0, n1 in [(0, 8), (8, 1000), (4090, 4096), (1234, 2345)]:
        got = gpu_partials(x, W, n0, n1)
        assert np.array_equal(got, oracle.partials(xq, codes[n0:n1], 128))


def test_partials_extreme_codes():
    # |P| reaches 256 * 127^2 = 4129024 when every code is +-127
    k, n = 512, 16
    x = np.zeros((2, k), np.float32)
    x[0, 0] = 1.0       # rotates to +-1 over the chunk -> codes +-127
    x[1, 128] = -2.0
    xb = f32_to_bf16_bits(x)
    codes = np.full((n, k), 127, np.int8)
    codes[1::2] = -127
    sub = np.full((n, k // 256), 255, np.uint8)
    scale = np.full((n,), 0x3C00, np.uint16)
    W = iq8r.IQ8RWeight.from_packed(codes, sub, scale, "g256", True)
    xq, _ = oracle.act_quant(xb)
    assert np.array_equal(gpu_partials(xb, W), oracle.partials(xq, codes, 256))


# ---------------------------------------------------------------- linear

def gpu_linear(x_bits, W, path=iq8r.IQ8R_PATH_AUTO):
    xq, xs = iq8r.iq8r_rotate_quant_act(dev_bf16(x_bits))
    y = iq8r.iq8r_linear_ex(xq, xs, W, path=path)
    torch.cuda.synchronize()
    return host_bits(y)


def oracle_linear(x, fmt, packed):
    codes, sub, scale = packed
    xq, a = oracle.act_quant(x)
    return oracle.linear(xq, a, fmt, codes, sub, scale, rotated=True)


@pytest.mark.parametrize("name", ["pr1", "decode", "verify8", "verify16", "verify128"])
def test_linear_within_tolerance_workloads(name):
    x, _, fmt, packed, W = case(name)
    y64 = oracle_linear(x, fmt, packed)
    st = check_output(gpu_linear(x, W), y64, oracle.linear_bf16(y64))
    assert st["bit_equal_frac"] > 0.99


@pytest.mark.parametrize("path", ["gemv", "auto"])
# (1, 300, 17408) and (2, 150, 8192): rows longer than a stage, streamed in chunks;
# (2, 7437, 2560) and (1, 7104, 4864): 48 rows a CTA or more, the last ones in
# 1 KB parts (4864: a part of 768 bytes and a half 512-byte step)
@pytest.mark.parametrize("m,n,k", [(1, 1000, 768), (3, 37, 2304), (13, 64, 512), (5, 9, 4352), (2, 333, 1280),
                                   (8, 77, 1536), (1, 300, 17408), (2, 150, 8192), (2, 7437, 2560),
                                   (1, 7104, 4864)])
def test_linear_within_tolerance_ragged(m, n, k, path):
    x, _, fmt, packed, W = case("decode", m=m, n=n, k=k, seed=11 + m + n + k)
    y64 = oracle_linear(x, fmt, packed)
    p = iq8r.IQ8R_PATH_GEMV if path == "gemv" else iq8r.IQ8R_PATH_AUTO
    check_output(gpu_linear(x, W, path=p), y64, oracle.linear_bf16(y64))


@pytest.mark.parametrize("path", ["gemv", "auto"])
def test_linear_lm_head_small(path):
    x, _, fmt, packed, W = case("lm_head8", m=8, n=2000, k=5120, seed=45)
    y64 = oracle_linear(x, fmt, packed)
    p = iq8r.IQ8R_PATH_GEMV if path == "gemv" else iq8r.IQ8R_PATH_AUTO
    check_output(gpu_linear(x, W, path=p), y64, oracle.linear_bf16(y64))


def test_linear_unrotated_weight():
    x, w = gen_workload("pr1")
    codes, sub, scale = oracle.pack(w, "g256", rotate=False)
    W = iq8r.IQ8RWeight.from_packed(codes, sub, scale, "g256", rotated=False)
    xq, xs = iq8r.iq8r_rotate_quant_act(dev_bf16(x), rotate=False)
    y = host_bits(iq8r.iq8r_linear(xq, xs, W))
    q, a = oracle.act_quant(x, rotate=False)
    y64 = oracle.linear(q, a, "g256", codes, sub, scale, rotated=False)
    check_output(y, y64)


def test_linear_zero_activation_row_gives_zero():
    x, _, fmt, packed, W = case("pr1")
    x = x.copy()
    x[2] = 0
    y = gpu_linear(x, W)
    assert np.all(y[2] == 0)


def test_prefill_full_size_sampled_rows():
    """M = 8192 through the library's launch configuration; the oracle checks
    a sample of token rows (all N outputs of each) and every act code."""
    x, _, fmt, packed, W = case("prefill")
    xq_d, xs_d = iq8r.iq8r_rotate_quant_act(dev_bf16(x))
    y = host_bits(iq8r.iq8r_linear(xq_d, xs_d, W))
    q, a = oracle.act_quant(x)
    assert np.array_equal(q, xq_d.cpu().numpy())
    rows = np.random.default_rng(0).choice(x.shape[0], 24, replace=False)
    rows = np.concatenate([rows, [0, x.shape[0] - 1]])
    codes, sub, scale = packed
    y64 = oracle.linear(q[rows], a[rows], fmt, codes, sub, scale, rotated=True)
    check_output(y[rows], y64)
    assert np.array_equal(gpu_partials(x[rows], W, 0, 17408),
                          oracle.partials(q[rows], codes, 256))


def test_lm_head_full_top32():
    """Full lm_head (N = 151936): outputs within tolerance, and the top-32
    logits agree with the oracle's: every oracle top-32 entry is within the
    output tolerance of the GPU's 32nd value and vice versa (the order of
    near-equal logits is not unique after bf16 rounding)."""
    _, w = gen_workload("lm_head8")           # the weight is drawn first: same for M = 1 and 8
    codes, sub, scale = oracle.pack(w, "g128", True)
    del w
    W = iq8r.IQ8RWeight.from_packed(codes, sub, scale, "g128", True)
    for name in ("lm_head1", "lm_head8"):
        x, _ = gen_workload(name, n=8)
        y = gpu_linear(x, W)
        y64 = oracle_linear(x, "g128", (codes, sub, scale))
        check_output(y, y64)
        yg = (y.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        tol = 1e-2 * np.sqrt(np.mean(y64 ** 2))
        for i in range(x.shape[0]):
            top_ref = np.argsort(-y64[i], kind="stable")[:32]
            top_gpu = np.argsort(-yg[i], kind="stable")[:32]
            thr_ref = y64[i, top_ref[-1]]
            thr_gpu = yg[i, top_gpu[-1]]
            ulp = 2.0 ** (np.floor(np.log2(abs(thr_gpu))) - 7)
            assert np.all(yg[i, top_ref] >= thr_gpu - tol - ulp)
            assert np.all(y64[i, top_gpu] >= thr_ref - tol - ulp)
            assert len(set(top_ref) & set(top_gpu)) >= 30
    del W
    torch.cuda.empty_cache()


def test_device_error_word_is_clear_after_the_suite_so_far():
    iq8r.iq8r_get_device_error()


def test_bounded_wait_reports_timeout_and_context_survives():
    iq8r.iq8r_get_device_error()
    iq8r.iq8r_selftest_wait_timeout(2_000_000)
    with pytest.raises(iq8r.IQ8RError) as e:
        iq8r.iq8r_get_device_error()
    assert e.value.status == iq8r.IQ8R_ERR_DEVICE_TIMEOUT
    assert "self-test" in str(e.value)
    iq8r.iq8r_get_device_error()  # cleared
    # the context still works
    x, _, fmt, packed, W = case("pr1")
    y64 = oracle_linear(x, fmt, packed)
    check_output(gpu_linear(x, W), y64)


# ------------------------------------------------------- fused bf16 entry

@pytest.mark.parametrize("name,m,n,k", [("pr1", None, None, None), ("decode", None, None, None),
                                        ("verify8", None, None, None), ("decode", 3, 1000, 768),
                                        ("decode", 5, 37, 2304), ("decode", 7, 40, 17408),
                                        ("decode", 1, 300, 17408), ("decode", 2, 100, 8192),
                                        ("decode", 2, 7437, 2560), ("decode", 1, 7104, 4864)])
def test_linear_bf16_fused_matches_two_call_path(name, m, n, k):
    """One-launch act + GEMV: codes and scales bit-exact against the oracle,
    y bit-identical to the two-call path and within tolerance of the oracle."""
    x, _, fmt, packed, W = case(name, m=m, n=n, k=k, seed=None if m is None else 31 + m + n)
    xd = dev_bf16(x)
    xq_out = torch.empty(x.shape, dtype=torch.int8, device="cuda")
    xs_out = torch.empty((x.shape[0],), dtype=torch.float32, device="cuda")
    y = iq8r.iq8r_linear_bf16(xd, W, xq_out=xq_out, x_scale_out=xs_out)
    torch.cuda.synchronize()
    q, a = oracle.act_quant(x)
    assert np.array_equal(xq_out.cpu().numpy(), q)
    assert np.array_equal(xs_out.cpu().numpy().view(np.uint32), a.view(np.uint32))
    # one launch (the GEMV with the quantiser fused) when m * k <= 16384, else
    # the activation kernel and iq8r_linear's own choice: the same arithmetic
    # as the two-call path through that kernel
    fused = x.shape[0] <= 2 or x.shape[0] * x.shape[1] <= 16384
    y2 = gpu_linear(x, W, path=iq8r.IQ8R_PATH_GEMV if fused else iq8r.IQ8R_PATH_AUTO)
    assert np.array_equal(host_bits(y), y2)
    y64 = oracle_linear(x, fmt, packed)
    check_output(host_bits(y), y64, oracle.linear_bf16(y64))


def test_linear_bf16_lm_head_and_no_outputs():
    x, _, fmt, packed, W = case("lm_head8", m=8, n=2000, k=5120, seed=45)
    y = iq8r.iq8r_linear_bf16(dev_bf16(x), W)
    torch.cuda.synchronize()
    y64 = oracle_linear(x, fmt, packed)
    check_output(host_bits(y), y64, oracle.linear_bf16(y64))


def test_linear_bf16_large_m_stages_codes():
    x, _, fmt, packed, W = case("verify16")
    xq_out = torch.empty(x.shape, dtype=torch.int8, device="cuda")
    xs_out = torch.empty((x.shape[0],), dtype=torch.float32, device="cuda")
    y = iq8r.iq8r_linear_bf16(dev_bf16(x), W, xq_out=xq_out, x_scale_out=xs_out)
    torch.cuda.synchronize()
    q, a = oracle.act_quant(x)
    assert np.array_equal(xq_out.cpu().numpy(), q)
    y64 = oracle_linear(x, fmt, packed)
    check_output(host_bits(y), y64, oracle.linear_bf16(y64))
    # without staging buffers M > 8 is refused, not silently allocated
    w = W._struct()
    import ctypes
    st = iq8r.lib().iq8r_linear_bf16(dev_bf16(x).data_ptr(), x.shape[0], ctypes.byref(w), y.data_ptr(), None, None,
                                      torch.cuda.current_stream().cuda_stream)
    assert st == iq8r.IQ8R_ERR_INVALID_ARG


# --------------------------------------------------- tensor-core path (TC)

TC_SHAPES = [(16, 128, 512), (200, 300, 768), (257, 129, 256), (33, 1000, 2304), (512, 256, 5120)]


@pytest.mark.parametrize("m,n,k", TC_SHAPES)
def test_tc_partials_bit_exact(m, n, k):
    """tcgen05 kind::i8: per-256-K int32 sums equal the oracle's exactly
    (token and weight tile tails, odd block counts, several tiles)."""
    x, _, _, (codes, _, _), W = case("decode", m=m, n=n, k=k, seed=71 + m + n + k)
    xq, _ = oracle.act_quant(x)
    got = gpu_partials(x, W, path=iq8r.IQ8R_PATH_TC)
    assert np.array_equal(got, oracle.partials(xq, codes, 256))


@pytest.mark.parametrize("m,n,k", TC_SHAPES)
def test_tc_linear_within_tolerance(m, n, k):
    x, _, fmt, packed, W = case("decode", m=m, n=n, k=k, seed=71 + m + n + k)
    y64 = oracle_linear(x, fmt, packed)
    y = gpu_linear(x, W, path=iq8r.IQ8R_PATH_TC)
    st = check_output(y, y64, oracle.linear_bf16(y64))
    assert st["bit_equal_frac"] > 0.98


def test_tc_lm_head_format():
    x, _, fmt, packed, W = case("lm_head8", m=40, n=256, k=640, seed=72)
    codes = packed[0]
    xq, _ = oracle.act_quant(x)
    assert np.array_equal(gpu_partials(x, W, path=iq8r.IQ8R_PATH_TC), oracle.partials(xq, codes, 128))
    y64 = oracle_linear(x, fmt, packed)
    check_output(gpu_linear(x, W, path=iq8r.IQ8R_PATH_TC), y64, oracle.linear_bf16(y64))


# the trunk in the earlier IQ8R format (one bf16 scale for each row and 128-wide block of K):
# the lm_head kernels at trunk shapes, through both kernels
@pytest.mark.parametrize("path", ["gemv", "tc"])
@pytest.mark.parametrize("m,n,k", [(1, 17408, 5120), (16, 512, 17408), (300, 640, 5120)])
def test_trunk_g128_format(m, n, k, path):
    x, _, fmt, packed, W = case("decode_g128", m=m, n=n, k=k, seed=61 + m)
    assert fmt == "g128"
    p = iq8r.IQ8R_PATH_GEMV if path == "gemv" else iq8r.IQ8R_PATH_TC
    xq, _ = oracle.act_quant(x)
    rows = slice(0, min(n, 2048))
    assert np.array_equal(gpu_partials(x, W, 0, rows.stop, path=p), oracle.partials(xq, packed[0][rows], 128))
    y64 = oracle_linear(x, fmt, packed)
    check_output(gpu_linear(x, W, path=p), y64, oracle.linear_bf16(y64))


# few output tiles and long K: the tile's K range is split over several CTAs
# and the fp32 partial tiles are added by the tile's last unit
TC_SPLIT_SHAPES = [(16, 256, 17408), (128, 384, 8192), (8, 200, 4096), (40, 130, 2560), (96, 1, 1024)]


@pytest.mark.parametrize("m,n,k", TC_SPLIT_SHAPES)
def test_tc_split_k_linear_within_tolerance(m, n, k):
    x, _, fmt, packed, W = case("decode", m=m, n=n, k=k, seed=81 + m + n + k)
    y64 = oracle_linear(x, fmt, packed)
    y = gpu_linear(x, W, path=iq8r.IQ8R_PATH_TC)
    st = check_output(y, y64, oracle.linear_bf16(y64))
    assert st["bit_equal_frac"] > 0.98


def test_tc_split_k_repeatable_and_lm_head():
    """Back-to-back split calls give identical bits (the arrival counters
    return to zero, the reduction order is fixed); the lm_head format splits
    the same way."""
    x, _, fmt, packed, W = case("decode", m=16, n=256, k=17408, seed=82)
    xq, xs = iq8r.iq8r_rotate_quant_act(dev_bf16(x))
    ys = [iq8r.iq8r_linear_ex(xq, xs, W, path=iq8r.IQ8R_PATH_TC) for _ in range(3)]
    torch.cuda.synchronize()
    assert all(torch.equal(ys[0], y) for y in ys[1:])
    x, _, fmt, packed, W = case("lm_head8", m=8, n=256, k=5120, seed=83)
    y64 = oracle_linear(x, fmt, packed)
    check_output(gpu_linear(x, W, path=iq8r.IQ8R_PATH_TC), y64, oracle.linear_bf16(y64))
    iq8r.iq8r_get_device_error()  # raises if a kernel reported a timeout


def test_tc_and_gemv_agree_on_partials():
    x, _, _, _, W = case("decode", m=24, n=512, k=1024, seed=73)
    a = gpu_partials(x, W, path=iq8r.IQ8R_PATH_TC)
    b = gpu_partials(x, W, path=iq8r.IQ8R_PATH_GEMV)
    assert np.array_equal(a, b)


# ------------------------------------------------------------- rescoring

def _rescore_case(name, m, n, k, seed, n_cand=32):
    x, _, fmt, packed, W = case(name, m=m, n=n, k=k, seed=seed)
    rng = np.random.default_rng(seed)
    cand = rng.integers(0, n, size=(m, n_cand)).astype(np.int32)
    cand[0, :3] = [0, n - 1, 0]  # first and last rows, a duplicate
    return x, fmt, packed, W, cand


@pytest.mark.parametrize("name,m,n,k", [("lm_head8", 8, 4096, 5120), ("decode", 5, 2000, 5120),
                                        ("decode_g128", 3, 1000, 2560), ("decode", 2, 300, 17408)])
def test_rescore_matches_oracle_and_gemv(name, m, n, k):
    """Candidate rescoring: within tolerance of the oracle, and the same bits
    as the GEMV path of the full linear at the candidate rows."""
    x, fmt, packed, W, cand = _rescore_case(name, m, n, k, seed=51 + m)
    xq, xs = iq8r.iq8r_rotate_quant_act(dev_bf16(x))
    cd = torch.from_numpy(cand).cuda()
    got = host_bits(iq8r.iq8r_rescore(xq, xs, W, cd))
    q, a = oracle.act_quant(x)
    ref64 = oracle.rescore(q, a, fmt, *packed, cand)
    check_output(got, ref64, oracle.linear_bf16(ref64))
    full = host_bits(iq8r.iq8r_linear_ex(xq, xs, W, path=iq8r.IQ8R_PATH_GEMV))
    assert np.array_equal(got, np.take_along_axis(full, cand.astype(np.int64), axis=1))
    iq8r.iq8r_get_device_error()


def test_rescore_out_of_range_candidate_is_reported():
    x, fmt, packed, W, cand = _rescore_case("lm_head8", 2, 256, 1024, seed=57, n_cand=8)
    cand[1, 4] = 256   # one past the last row
    cand[0, 7] = -1
    xq, xs = iq8r.iq8r_rotate_quant_act(dev_bf16(x))
    out = host_bits(iq8r.iq8r_rescore(xq, xs, W, torch.from_numpy(cand).cuda()))
    with pytest.raises(iq8r.IQ8RError) as err:
        iq8r.iq8r_get_device_error()
    assert err.value.status == iq8r.IQ8R_ERR_INVALID_ARG
    assert out[1, 4] == 0 and out[0, 7] == 0
    q, a = oracle.act_quant(x)
    ok = cand.copy()
    ok[1, 4] = ok[0, 7] = 0
    ref = oracle.linear_bf16(oracle.rescore(q, a, fmt, *packed, ok))
    mask = np.ones_like(cand, bool)
    mask[1, 4] = mask[0, 7] = False
    check_output(out[mask][None], oracle.rescore(q, a, fmt, *packed, ok)[mask][None], ref[mask][None])
    iq8r.iq8r_get_device_error()  # the word was cleared by the read above


# ---------------------------------------------- weights packed by rule=search

@pytest.mark.parametrize("fmt,m,n,k,path", [("g256", 1, 3000, 5120, "gemv"), ("g256", 64, 640, 2560, "tc"),
                                            ("g128", 8, 1000, 5120, "tc"), ("g128", 2, 700, 1024, "gemv")])
def test_search_packed_weights(fmt, m, n, k, path):
    """The kernels take least-error-packed weights as they are: partial sums
    exact and outputs within tolerance of the oracle on the same packing."""
    x, w = gen_workload("decode", m=m, n=n, k=k, seed=71 + m)
    codes, sub, scale = iq8r.iq8r_pack(w, fmt, True, rule="search")
    W = iq8r.IQ8RWeight.from_packed(codes, sub, scale, fmt, True)
    p = iq8r.IQ8R_PATH_GEMV if path == "gemv" else iq8r.IQ8R_PATH_TC
    q, a = oracle.act_quant(x)
    g = 256 if fmt == "g256" else 128
    assert np.array_equal(gpu_partials(x, W, path=p), oracle.partials(q, codes, g))
    y64 = oracle.linear(q, a, fmt, codes, sub, scale, rotated=True)
    check_output(gpu_linear(x, W, path=p), y64, oracle.linear_bf16(y64))


# ------------------------------------------ the drafter's 16-level codebook

def _cb4_case(m, n, k, seed):
    x, w = gen_workload("decode", m=m, n=n, k=k, seed=seed)
    packed, scale = oracle.pack_cb4(w, True)
    W = iq8r.IQ8RWeight.from_packed(packed, None, scale, "cb4", True)
    return x, packed, scale, W


@pytest.mark.parametrize("m,n,k", [(1, 17408, 5120), (3, 1000, 768), (8, 300, 17408), (13, 77, 2560),
                                   (2, 129, 128), (4, 100, 4096), (6, 200, 8192), (2, 150, 16384)])
def test_cb4_partials_and_linear(m, n, k):
    """Codebook format through its GEMV: exact per-128 partial sums of the
    levels, and outputs within tolerance of the oracle; the tensor-core path
    is refused. K = 5120, 4096, 8192 and 16384 take the instances for full
    chunks (one chunk of 5, 4 or 8 steps; two chunks of 8), the rest the
    general ones."""
    x, packed, scale, W = _cb4_case(m, n, k, seed=91 + m)
    assert W.k == k
    q, a = oracle.act_quant(x)
    vals = oracle.decode_cb4(packed)
    assert np.array_equal(gpu_partials(x, W), oracle.partials(q, vals, 128))
    y64 = oracle.linear(q, a, "cb4", packed, None, scale, rotated=True)
    check_output(gpu_linear(x, W), y64, oracle.linear_bf16(y64))
    xq, xs = iq8r.iq8r_rotate_quant_act(dev_bf16(x))
    with pytest.raises(iq8r.IQ8RError):
        iq8r.iq8r_linear_ex(xq, xs, W, path=iq8r.IQ8R_PATH_TC)
    # the whole layer from bf16 activations
    y = iq8r.iq8r_linear_bf16(dev_bf16(x), W,
                              xq_out=torch.empty(x.shape, dtype=torch.int8, device="cuda"),
                              x_scale_out=torch.empty((m,), dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    check_output(host_bits(y), y64, oracle.linear_bf16(y64))
    iq8r.iq8r_get_device_error()


@pytest.mark.parametrize("m,n,k", [(1, 257, 5120), (5, 333, 1024)])
def test_cb4_search_packed(m, n, k):
    """Codebook weights packed by the C++ rule=search: the bytes are the
    oracle's search result, the partial sums exact and the outputs within
    tolerance."""
    x, w = gen_workload("decode", m=m, n=n, k=k, seed=61 + m)
    packed, sub, scale = iq8r.iq8r_pack(w, "cb4", True, rule="search")
    want = oracle.pack_search(w, "cb4", True)
    assert sub is None and np.array_equal(packed, want[0]) and np.array_equal(scale, want[2])
    W = iq8r.IQ8RWeight.from_packed(packed, None, scale, "cb4", True)
    q, a = oracle.act_quant(x)
    assert np.array_equal(gpu_partials(x, W), oracle.partials(q, oracle.decode_cb4(packed), 128))
    y64 = oracle.linear(q, a, "cb4", packed, None, scale, rotated=True)
    check_output(gpu_linear(x, W), y64, oracle.linear_bf16(y64))


def test_cb4_partials_window():
    x, packed, scale, W = _cb4_case(4, 600, 1024, seed=97)
    q, _ = oracle.act_quant(x)
    vals = oracle.decode_cb4(packed)
    for n0, n1 in [(0, 5), (7, 300), (599, 600)]:
        assert np.array_equal(gpu_partials(x, W, n0, n1), oracle.partials(q, vals[n0:n1], 128))


# ------------------------------------------------ weights written just before

@pytest.mark.parametrize("fmt,path", [("g256", iq8r.IQ8R_PATH_GEMV), ("g256", iq8r.IQ8R_PATH_TC),
                                      ("g128", iq8r.IQ8R_PATH_GEMV), ("cb4", iq8r.IQ8R_PATH_AUTO)])
def test_weights_written_by_the_previous_kernel(fmt, path):
    """A torch kernel rewrites the packed weight immediately before the call;
    with IQ8R_PATH_FLAG_WEIGHTS_WRITTEN the kernels read the new weight (the
    weight-streaming kernels otherwise read weights ahead of the previous
    kernel's completion, see include/iq8r.h)."""
    m, n, k = (2, 1536, 5120) if path != iq8r.IQ8R_PATH_TC else (16, 1536, 5120)
    x, w_old = gen_workload("decode", m=m, n=n, k=k, seed=61)
    _, w_new = gen_workload("decode", m=1, n=n, k=k, seed=62)
    packer = (lambda w: (lambda c, s: (c, None, s))(*oracle.pack_cb4(w, True))) if fmt == "cb4" else \
        (lambda w: oracle.pack(w, fmt, True))
    old, new = packer(w_old), packer(w_new)
    W = iq8r.IQ8RWeight.from_packed(*old, fmt if fmt != "cb4" else "cb4", True)
    src = [None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in new]
    xq, xs = iq8r.iq8r_rotate_quant_act(dev_bf16(x))
    torch.cuda.synchronize()

    def rewrite(dst, s_):
        if dst is None:
            return
        if dst.dtype == torch.uint16:
            dst, s_ = dst.view(torch.int16), s_.view(torch.int16)
        torch.bitwise_or(s_, 0, out=dst)  # one elementwise kernel writes dst

    rewrite(W.scale, src[2])
    rewrite(W.sub_scale, src[1])
    rewrite(W.codes, src[0])              # the kernel right before the call
    y = iq8r.iq8r_linear_ex(xq, xs, W, path=path | iq8r.IQ8R_PATH_FLAG_WEIGHTS_WRITTEN)
    torch.cuda.synchronize()
    q, a = oracle.act_quant(x)
    y64 = oracle.linear(q, a, fmt, *new)
    check_output(host_bits(y), y64, oracle.linear_bf16(y64))
    iq8r.iq8r_get_device_error()


@pytest.mark.parametrize("m,n,k", [(1, 17408, 5120), (2, 7437, 2560), (1, 300, 17408), (2, 150, 8192)])
def test_gemv_trunk_outputs_from_exact_block_sums(m, n, k):
    """The one- and two-token GEMV's bf16 outputs, bit for bit, rebuilt from
    the oracle's exact block sums: S[m, n] = sum_g s1[n, g] * P[m, n, g] as an
    exact integer, then the kernel's stated epilogue as plain IEEE float32
    steps, ((float(S) * a[m]) * s2[n]) * (1/128), each rounded to nearest,
    and one bf16 rounding to nearest. A dropped or repeated block, a sub-scale
    from the wrong block or another token's codes change S and so the bits.
    Both entries: the codes given, and the fused one."""
    x, _, fmt, (codes, sub, scale), W = case("decode", m=m, n=n, k=k, seed=61 + m + n)
    q, a = oracle.act_quant(x)
    P = oracle.partials(q, codes, 256).astype(np.int64)  # [m, n, k / 256]
    S = np.einsum("mng,ng->mn", P, sub.astype(np.int64))
    s2 = (scale.astype(np.uint32) << 16).view(np.float32)
    yf = S.astype(np.float32) * a.astype(np.float32)[:, None]
    yf = (yf * s2[None, :]).astype(np.float32)
    yf = (yf * np.float32(0.0078125)).astype(np.float32)
    expect = oracle.bf16_round_nearest(yf.astype(np.float64))
    xd = dev_bf16(x)
    y_fused = host_bits(iq8r.iq8r_linear_bf16(xd, W))
    xq, xs = iq8r.iq8r_rotate_quant_act(xd)
    y_codes = host_bits(iq8r.iq8r_linear_ex(xq, xs, W, path=iq8r.IQ8R_PATH_GEMV))
    assert np.array_equal(y_codes, expect), f"{np.sum(y_codes != expect)} of {expect.size} outputs differ"
    assert np.array_equal(y_fused, expect), f"{np.sum(y_fused != expect)} of {expect.size} outputs differ"


def _fma32(p64: np.ndarray, acc32: np.ndarray) -> np.ndarray:
    """float32 of p + acc rounded once to nearest-even (a float32 fused
    multiply-add whose product p is exact in float64). The sum is taken
    exactly as s + err (two-sum); s rounds to float32 correctly unless s
    lies on a float32 midpoint, where the sign of err decides."""
    b = acc32.astype(np.float64)
    s = p64 + b
    bb = s - p64
    err = (p64 - (s - bb)) + (b - bb)
    r = s.astype(np.float32)
    r64 = r.astype(np.float64)
    lo = np.nextafter(r, np.float32(-np.inf))
    hi = np.nextafter(r, np.float32(np.inf))
    r = np.where((s == (r64 + hi.astype(np.float64)) / 2) & (err > 0), hi, r)
    r = np.where((s == (r64 + lo.astype(np.float64)) / 2) & (err < 0), lo, r)
    return r.astype(np.float32)


def _g128_gemv_steps(xq, a, codes, scale_bits):
    """The one- and two-token GEMV's stated lm_head arithmetic in float32 from
    exact integer dot products: lane L of a row's warp takes 16 bytes of K a
    512-byte step (K positions 512 s + 16 L ..; a step past K adds a zero
    product with the last block's scale), accumulates fma(q, s_block, acc)
    over the steps in K order, the 32 lane sums meet in a 16-8-4-2-1
    exchange of float32 adds, and y = bf16(acc * a * (1/128))."""
    m_tok, k = xq.shape
    s32 = (scale_bits.astype(np.uint32) << 16).view(np.float32)
    lanes = np.arange(32)
    out = []
    for m in range(m_tok):
        acc = np.zeros((codes.shape[0], 32), dtype=np.float32)
        for st in range(-(-k // 2560) * 5):
            kr = st * 512 + lanes * 16
            valid = kr < k
            kk = np.where(valid, kr, k - 16)
            idx = kk[:, None] + np.arange(16)[None, :]
            q = (codes[:, idx].astype(np.int64) * xq[m, idx].astype(np.int64)[None]).sum(-1)
            q = np.where(valid[None, :], q, 0)
            acc = _fma32(q.astype(np.float64) * s32[:, kk // 128].astype(np.float64), acc)
        for off in (16, 8, 4, 2, 1):
            acc = (acc + acc[:, lanes ^ off]).astype(np.float32)
        y = (acc[:, 0] * np.float32(a[m])).astype(np.float32)
        out.append((y * np.float32(0.0078125)).astype(np.float32))
    return oracle.bf16_round_nearest(np.stack(out).astype(np.float64))


@pytest.mark.parametrize("m,n,k", [(1, 4096, 5120), (2, 700, 1024), (1, 300, 4352)])
def test_gemv_g128_outputs_from_exact_dot_products(m, n, k):
    """The same for the lm_head (G128) format, whose sum over blocks is
    float32: the GEMV's outputs bit-equal to its stated summation order over
    the oracle's codes and exact 16-byte dot products. A scale taken from a
    neighbouring block (it changes 4059 of the 4096 outputs at the first
    shape), or a step dropped or summed twice, changes bits. (K = 1024 and
    4352: a row's last unit partly past its end.)"""
    x, _, fmt, (codes, sub, scale), W = case("lm_head8", m=m, n=n, k=k, seed=67 + m + n)
    q, a = oracle.act_quant(x)
    expect = _g128_gemv_steps(q, a, codes, scale)
    xd = dev_bf16(x)
    y_fused = host_bits(iq8r.iq8r_linear_bf16(xd, W))
    xq, xs = iq8r.iq8r_rotate_quant_act(xd)
    y_codes = host_bits(iq8r.iq8r_linear_ex(xq, xs, W, path=iq8r.IQ8R_PATH_GEMV))
    assert np.array_equal(y_codes, expect), f"{np.sum(y_codes != expect)} of {expect.size} outputs differ"
    assert np.array_equal(y_fused, expect), f"{np.sum(y_fused != expect)} of {expect.size} outputs differ"


@pytest.mark.parametrize("m,n,k", [(1, 17408, 5120), (2, 7437, 2560)])
def test_gemv_back_to_back_launches_agree(m, n, k):
    """Five launches queued back to back on one stream (each may start while
    the previous one drains) give the same bits as one launch alone; any
    per-launch state of the kernel must be back in place for the next one."""
    x, _, fmt, packed, W = case("decode", m=m, n=n, k=k, seed=71 + m)
    xd = dev_bf16(x)
    ref = iq8r.iq8r_linear_bf16(xd, W)
    torch.cuda.synchronize()
    ys = [iq8r.iq8r_linear_bf16(xd, W) for _ in range(5)]
    xq, xs = iq8r.iq8r_rotate_quant_act(xd)
    ys += [iq8r.iq8r_linear(xq, xs, W) for _ in range(3)]
    torch.cuda.synchronize()
    for y in ys:
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16))
    iq8r.iq8r_get_device_error()


# --------------------------------------------------------- host-buffer layer

@pytest.mark.parametrize("name,m,n,k", [("decode", 1, 4096, 5120), ("verify16", 16, 1024, 17408)])
def test_linear_bf16_host_matches_the_device_call(name, m, n, k):
    """iq8r_linear_bf16_host (pinned host x in, host y out, one call: the
    mapped-copy kernels) gives the same bits as iq8r_linear_bf16 on device
    buffers, twice in a row; so do pageable buffers (the copy calls) and an
    output whose size is not a multiple of 8 values (the copy's tail)."""
    x, _, fmt, packed, W = case(name, m=m, n=n, k=k)
    xd = dev_bf16(x)
    staged = m > 2
    xq = torch.empty(x.shape, dtype=torch.int8, device="cuda") if staged else None
    xs = torch.empty((m,), dtype=torch.float32, device="cuda") if staged else None
    ref = iq8r.iq8r_linear_bf16(xd, W, xq_out=xq, x_scale_out=xs)
    xh = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(xd)
    y_dev = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    for _ in range(2):
        yh = torch.full((m, n), 7.0, dtype=torch.bfloat16).pin_memory()
        iq8r.iq8r_linear_bf16_host(xh, W, x_dev, y_dev, yh, xq, xs)
        torch.cuda.synchronize()
        assert torch.equal(yh.view(torch.int16), ref.cpu().view(torch.int16))
    q, a = oracle.act_quant(x)
    y64 = oracle.linear(q, a, fmt, *packed)
    check_output(yh.view(torch.int16).numpy().view(np.uint16), y64, oracle.linear_bf16(y64))
    # pageable host buffers take the copy calls instead of the mapped-copy kernels
    xp = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).clone()
    yp = torch.full((m, n), 7.0, dtype=torch.bfloat16)
    assert not xp.is_pinned() and not yp.is_pinned()
    iq8r.iq8r_linear_bf16_host(xp, W, x_dev, y_dev, yp, xq, xs)
    torch.cuda.synchronize()
    assert torch.equal(yp.view(torch.int16), ref.cpu().view(torch.int16))
    # a ragged output (m * n not a multiple of 8: the copy's element tail)
    if m == 1:
        Wr = iq8r.IQ8RWeight.from_packed(*[np.ascontiguousarray(t[:n - 3]) for t in packed], fmt, True)
        ref_r = iq8r.iq8r_linear_bf16(xd, Wr)
        yr = torch.full((m, n - 3), 7.0, dtype=torch.bfloat16).pin_memory()
        yr_dev = torch.empty((m, n - 3), dtype=torch.bfloat16, device="cuda")
        iq8r.iq8r_linear_bf16_host(xh, Wr, x_dev, yr_dev, yr)
        torch.cuda.synchronize()
        assert torch.equal(yr.view(torch.int16), ref_r.cpu().view(torch.int16))
    iq8r.iq8r_get_device_error()

