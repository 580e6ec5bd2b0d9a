"""Failure detection on the device: a pipeline wait that runs out.

Every wait in the kernels is bounded.  Here the bound is set far below the
length of the kernels' longer waits (moe_set_wait_limit), so those waits give
up on purpose -- no fault, no hang (a wait that one poll of the barrier
outlasts is not checked against the bound, so the problems are sized for
waits of many microseconds): each waiter records the timeout in the device
status word, raises its CTA's abort flag, and the kernel drains the copies
and tensor-core work it issued (with the default bound), frees its tensor
memory and returns.  The test checks that the call comes back, that
moe_device_status reports MOE_ERR_TIMEOUT with the kernel and the wait, and
that after the default bound is restored the same call on the same device
gives the same bits as before.

Only stage calls whose outputs nothing else indexes run under the short bound
(the expert GEMMs, and the router whose ids are discarded): an aborted kernel
leaves its outputs incomplete.
"""
import pytest
import torch

import moe_inputs
from parity import to_device

pytestmark = pytest.mark.gpu

MOE_ERR_TIMEOUT = 7
KERN_GEMM_TC, KERN_GEMM_SWAP = 2, 3
SHORT_CYCLES = 100


@pytest.fixture
def moe():
    import sparse_moe_layer_top_b200 as m
    torch.cuda.set_device(0)
    yield m
    m.set_wait_limit(0)
    m.set_path(0)


def _timed_out(moe, kernels):
    s, detail = moe.device_status()
    assert s == MOE_ERR_TIMEOUT, "status %d (0x%08x)" % (s, detail & 0xffffffff)
    assert (detail >> 24) & 0xff == 0x07
    assert (detail >> 8) & 0xff in kernels, hex(detail)
    assert 1 <= detail & 0xff <= 14, hex(detail)  # one of the kernels' wait sites


@pytest.mark.parametrize("path,kern", [(2, KERN_GEMM_TC), (3, KERN_GEMM_SWAP)])
def test_expert_gemm_waits_that_run_out_report_timeout_and_the_device_stays_usable(moe, path, kern):
    inp = moe_inputs.make_inputs(384, 2048, 8, 2, 512, 256, act="bf16", w="bf16", seed=3)
    g = to_device(inp, "cuda")
    ids, tw = moe_inputs.random_routing(inp.T, inp.E, inp.k, seed=3)
    prob = moe.Problem.make(inp.T, inp.d, inp.E, inp.k, inp.I, inp.I_s, "bf16", "bf16")
    moe.set_path(path)
    perm = moe.permute(prob, g.x, ids.cuda(), tw.cuda())

    def ffn():
        return moe.expert_ffn(prob, perm["x_perm"], perm["offs"], g.wg, g.wu, g.wd, g.s_wg, g.s_wu, g.s_wd)

    y_ok = ffn()
    assert moe.device_status()[0] == 0
    torch.cuda.synchronize()
    moe.set_wait_limit(SHORT_CYCLES)
    try:
        ffn()
        _timed_out(moe, (kern,))
    finally:
        moe.set_wait_limit(0)
    y_again = ffn()
    assert moe.device_status()[0] == 0
    assert torch.equal(y_again, y_ok)


def test_router_waits_that_run_out_report_timeout_and_the_device_stays_usable(moe):
    # E <= 256 with 18 row tiles: the router GEMM selects the top k in its
    # epilogue; d = 8192 makes each tile's main loop (128 K-blocks) far longer
    # than one poll of a wait, so the epilogue's wait for the accumulator runs out
    inp = moe_inputs.make_inputs(2304, 8192, 100, 6, 128, 128, act="bf16", w="bf16", bias="zipf", seed=3)
    g = to_device(inp, "cuda")
    prob = moe.Problem.make(inp.T, inp.d, inp.E, inp.k, inp.I, inp.I_s, "bf16", "bf16")
    ids_ok, w_ok = moe.router_topk(prob, g.x, g.w_r, g.bias)
    assert moe.device_status()[0] == 0
    torch.cuda.synchronize()
    moe.set_wait_limit(SHORT_CYCLES)
    try:
        moe.router_topk(prob, g.x, g.w_r, g.bias)
        _timed_out(moe, (KERN_GEMM_TC,))
    finally:
        moe.set_wait_limit(0)
    ids, w = moe.router_topk(prob, g.x, g.w_r, g.bias)
    assert moe.device_status()[0] == 0
    assert torch.equal(ids, ids_ok) and torch.equal(w, w_ok)
