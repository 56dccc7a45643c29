"""A bounded device wait that runs out reports MOE_DEVICE_ERR_TIMEOUT, the
kernel returns, and the next launch is clean.

No wait in the shipped library is meant to run out.  A separate build of the
library (MOE_TEST_HOOKS; moe_routed_experts_b200/build.py, never the shipped
libmoe_awq.so) adds one switch, moe_test_arm_stall: the streaming tile's
first consumer thread then waits, after every copy its CTA issued has
landed, on a barrier phase that nothing completes, with a 1 ms limit.  No
GPU fault, trap or endless wait is involved: the wait gives up by design and
the context stays usable.  It runs in a child process so that the two
libraries never share one.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import ctypes as C, sys
sys.path.insert(0, ROOT)
import numpy as np, torch
from moe_routed_experts_b200 import build, binding as B
build.build(test_hooks=True)
B.LIB_PATH = build.TEST_HOOKS_LIB
L = B.lib()
L.moe_test_arm_stall.restype = C.c_int32
L.moe_test_arm_stall.argtypes = [C.c_int32]
from moe_routed_experts_b200 import ffn, inputs
from moe_routed_experts_b200.configs import WORKLOADS, scaled
B.set_projection_path(1)  # the streaming tile
w = scaled(WORKLOADS["decode"], H=256, I=128, E=16)
inp = inputs.generate(w)
dev = ffn.to_device(inp)

def run():
    buf = ffn.alloc(w)
    ffn.forward(dev, buf)
    torch.cuda.synchronize()
    return int(buf.status.item()), buf.out.clone()

st0, out0 = run()
assert st0 == 0, st0
L.moe_test_arm_stall(1)
st1, _ = run()
L.moe_test_arm_stall(0)
assert st1 == 8, st1  # MOE_DEVICE_ERR_TIMEOUT, and the launch returned
st2, out2 = run()
assert st2 == 0, st2
assert torch.equal(out0, out2)
print("TIMEOUT_REPORTED_AND_RECOVERED")
""".replace("ROOT", repr(ROOT))


def test_bounded_wait_times_out_reports_and_recovers():
    r = subprocess.run([sys.executable, "-c", CHILD], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0 and "TIMEOUT_REPORTED_AND_RECOVERED" in r.stdout, r.stdout[-2000:] + r.stderr[-3000:]
