"""The linear allocates nothing, even on its first call (needs a B200).

A fresh process makes its first-ever libiq8r call at the verify shape (the
split-K plan, whose partial tiles go to the library's device-image
workspace) inside a CUDA graph capture in global mode, where any device
allocation would fail the capture. The captured graph is then replayed and
compared with an ordinary call.
"""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import numpy as np, torch
import quantised_fwht128_act_b200 as iq8r
from iq8r_inputs import gen_workload
torch.cuda.set_device(0)
x, w = gen_workload("verify16", m=16, n=1280, k=17408, seed=77)
codes, sub, scale = iq8r.iq8r_pack(w, "g256", True)
W = iq8r.IQ8RWeight.from_packed(codes, sub, scale, "g256", True)
xd = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)
xq = torch.empty((16, 17408), dtype=torch.int8, device="cuda")
xs = torch.empty((16,), dtype=torch.float32, device="cuda")
y = torch.empty((16, 1280), dtype=torch.bfloat16, device="cuda")
torch.cuda.synchronize()
g = torch.cuda.CUDAGraph()
s = torch.cuda.Stream()
with torch.cuda.graph(g, stream=s, capture_error_mode="global"):
    iq8r.iq8r_rotate_quant_act(xd, True, xq, xs)
    iq8r.iq8r_linear(xq, xs, W, y)
g.replay()
torch.cuda.synchronize()
ref = iq8r.iq8r_linear(xq, xs, W)
torch.cuda.synchronize()
assert torch.equal(y.view(torch.int16), ref.view(torch.int16)), "captured first call differs"
iq8r.iq8r_get_device_error()
print("captured-first-call ok")
"""


def test_first_linear_call_captured_in_a_graph():
    r = subprocess.run([sys.executable, "-c", SCRIPT], cwd=ROOT, capture_output=True, text=True, timeout=600,
                       env=dict(os.environ, PYTHONPATH=ROOT))
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "captured-first-call ok" in r.stdout
