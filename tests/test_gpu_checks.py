"""The bounds-checking build of the library (libmoe_checks.so, built with
-DMOE_CHECKS and loaded by the binding when MOE_CHECKS=1).

Its kernels check the indices they compute or read before addressing memory
with them (moe_bounds_checked in include/moe.h).  The input here that only a
check can catch is a caller's pos for moe_combine pointing past the
dispatched rows: the checking build skips that read and reports it in the
device status word; a normal build would read past the buffer, so the case
runs only after the child process has confirmed which build it loaded.  The
same child runs a normal forward through the checking build against the
oracle, so the checks change nothing for valid inputs.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys
sys.path.insert(0, sys.argv[1])
sys.path.insert(0, sys.argv[1] + "/tests")
import numpy as np
import torch
import moe_inputs
import oracle
import sparse_moe_layer_top_b200 as moe
from parity import TOL, rel_l2, to_device

assert moe.lib_path.endswith("libmoe_checks.so"), moe.lib_path
assert moe.bounds_checked(), "the loaded library is not the bounds-checking build"
torch.cuda.set_device(0)

# a valid forward through the checking build matches the oracle
inp = moe_inputs.make_inputs(300, 256, 20, 4, 192, 128, act="bf16", w="bf16", seed=5)
g = to_device(inp, "cuda")
prob = moe.Problem.make(inp.T, inp.d, inp.E, inp.k, inp.I, inp.I_s, "bf16", "bf16")
ids = torch.empty((inp.T, inp.k), dtype=torch.int32, device="cuda")
tw = torch.empty((inp.T, inp.k), dtype=torch.float32, device="cuda")
y = moe.layer_forward(prob, g.x, g.w_r, None, g.wg, g.wu, g.wd, g.s_wg, g.s_wu, g.s_wd, topk_ids=ids, topk_w=tw)
s, detail = moe.device_status()
assert s == 0, hex(detail)
y_or, *_ = oracle.moe_forward(inp.x, inp.w_r, inp.wg, inp.wu, inp.wd, inp.s_wg, inp.s_wu, inp.s_wd, inp.k,
                              force_ids=ids.cpu().numpy())
assert rel_l2(y.float().cpu().numpy(), y_or) <= TOL["bf16"]

# moe_combine with one pair's row far past the dispatched rows
T, d, E, k = 8, 64, 4, 2
p = moe.Problem.make(T, d, E, k, 64, 64, "bf16", "bf16")
Rp = T * k + T
y_perm = torch.randn((Rp, d), device="cuda").to(torch.bfloat16)
ids, tw = moe_inputs.random_routing(T, E, k, seed=1)
perm = moe.permute(p, torch.randn((T, d), device="cuda").to(torch.bfloat16), ids.cuda(), tw.cuda())
pos = perm["pos"].clone()
good = moe.combine(p, y_perm, pos, tw.cuda(), perm["offs"])
assert moe.device_status()[0] == 0
pos[3, 1] = Rp + 1000
bad = moe.combine(p, y_perm, pos, tw.cuda(), perm["offs"])
s, detail = moe.device_status()
assert s == 6 and (detail & 0xffffffff) == 0x08000005, (s, hex(detail & 0xffffffff))
# the other tokens are untouched; token 3 lost only the skipped pair's term
keep = [t for t in range(T) if t != 3]
assert torch.equal(bad[keep], good[keep])
r = int(perm["pos"][3, 1])
want = good[3].float() - tw[3, 1].item() * y_perm[r].float()
assert torch.allclose(bad[3].float(), want, atol=2e-2, rtol=2e-2)
assert moe.device_status()[0] == 0  # reading cleared it
print("checks ok")
"""


def test_checking_build_catches_a_combine_row_past_the_buffer():
    lib = os.path.join(ROOT, "sparse_moe_layer_top_b200", "libmoe_checks.so")
    if not os.path.exists(lib):
        pytest.fail("libmoe_checks.so is not built (python -m sparse_moe_layer_top_b200.build --checks)")
    env = dict(os.environ, MOE_CHECKS="1")
    out = subprocess.run([sys.executable, "-c", CHILD, ROOT], capture_output=True, text=True, timeout=600,
                         env=env, cwd=ROOT)
    assert out.returncode == 0 and "checks ok" in out.stdout, out.stdout[-2000:] + out.stderr[-4000:]
