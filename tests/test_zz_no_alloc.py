"""iq8r_linear_noalloc against iq8r_linear (needs a B200).

The no-allocation entry point runs the same kernels with the same split
plan as iq8r_linear, its split-K partial tiles in the library's fixed
device array instead of the allocated workspace, so its output must be the
same bits -- call after call. A plan that needs more scratch than the fixed
array holds is refused without launching anything.

The file is named to run last, after the other GPU tests have used the
allocating path, and it passes on its own as well.
"""

import numpy as np
import pytest
import torch

import quantised_fwht128_act_b200 as iq8r
from iq8r_inputs import gen_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from quantised_fwht128_act_b200 import build
    build.build()
    iq8r.lib()
    yield
    iq8r.iq8r_get_device_error()


def _layer(name, m, n, k, seed):
    x, w = gen_workload(name, m=m, n=n, k=k, seed=seed)
    fmt = "g128" if name.startswith("lm_head") else "g256"
    codes, sub, scale = iq8r.iq8r_pack(w, fmt, rotate=True)
    W = iq8r.IQ8RWeight.from_packed(codes, sub, scale, fmt, True)
    xd = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)
    xq, xs = iq8r.iq8r_rotate_quant_act(xd, True)
    return xq, xs, W


# verify-sized split K (280 partial tiles), an lm_head split, and the GEMV
# path (two tokens: the automatic choice is the weight-streaming GEMV, which
# uses no scratch at all)
@pytest.mark.parametrize("name,m,n,k", [("verify16", 16, 5120, 17408), ("lm_head8", 40, 256, 5120),
                                        ("decode", 2, 1000, 2048)])
def test_noalloc_matches_linear_two_calls_in_a_row(name, m, n, k):
    xq, xs, W = _layer(name, m, n, k, seed=90 + m)
    ref = [iq8r.iq8r_linear(xq, xs, W) for _ in range(2)]
    got = [iq8r.iq8r_linear_noalloc(xq, xs, W) for _ in range(2)]
    torch.cuda.synchronize()
    for y in ref[1:] + got:
        assert torch.equal(y.view(torch.int16), ref[0].view(torch.int16))
    iq8r.iq8r_get_device_error()


def test_noalloc_refuses_a_plan_larger_than_its_array():
    # 10 weight tiles split 14 ways at 128 tokens: 140 x 64 KiB = 8.75 MiB of
    # partial tiles, more than the fixed 8 MiB
    xq, xs, W = _layer("verify128", 128, 1280, 17408, seed=95)
    y = torch.full((128, 1280), 3.0, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(iq8r.IQ8RError) as err:
        iq8r.iq8r_linear_noalloc(xq, xs, W, y)
    assert err.value.status == iq8r.IQ8R_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert bool((y == 3.0).all())  # nothing was launched
    # the allocating entry point takes the same call
    y2 = iq8r.iq8r_linear(xq, xs, W)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(y2.float()).all())
    iq8r.iq8r_get_device_error()
