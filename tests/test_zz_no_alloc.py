"""moe_router_topk_static: the router stage for callers that cannot allocate
device memory and so have no workspace to give it.

It is called through the C ABI and must reproduce moe_router_topk (the same
kernels, with the logit partials in the library's built-in array instead of
a caller workspace), on two calls in a row, since the array keeps whatever the
previous call left in it.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import moe_inputs
from parity import TOL_W

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("shape", [(300, 256, 20, 4, "bf16"), (4096, 2048, 256, 8, "bf16"),
                                   (64, 8192, 512, 10, "bf16"), (77, 96, 24, 3, "f32")])
def test_static_router_matches_workspace_router_twice(shape):
    import sparse_moe_layer_top_b200 as moe
    T, d, E, k, act = shape
    torch.cuda.set_device(0)
    x = moe_inputs.randn((T, d), "cuda", 5, moe_inputs.X, 1.0, torch.float32 if act == "f32" else torch.bfloat16)
    w_r = moe_inputs.randn((E, d), "cuda", 5, moe_inputs.W_R, 0.02, x.dtype)
    bias = moe_inputs.zipf_bias(E, "cuda")
    prob = moe.Problem.make(T, d, E, k, 64, 64, act, act)
    L = moe.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    ws = torch.empty(max(moe.stage_workspace_size(prob), 1), dtype=torch.uint8, device="cuda")
    ids_ref = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w_ref = torch.empty((T, k), dtype=torch.float32, device="cuda")
    assert L.moe_router_topk(ctypes.byref(prob), _p(x), _p(w_r), _p(bias), _p(ids_ref), _p(w_ref), _p(ws),
                             ws.numel(), stream) == 0
    torch.cuda.synchronize()

    for call in range(2):
        ids = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
        tw = torch.full((T, k), -1.0, dtype=torch.float32, device="cuda")
        rc = L.moe_router_topk_static(ctypes.byref(prob), _p(x), _p(w_r), _p(bias), _p(ids), _p(tw), stream)
        assert rc == 0, L.moe_last_error_string()
        torch.cuda.synchronize()
        assert moe.device_status()[0] == 0
        assert torch.equal(ids, ids_ref), "call %d: expert ids differ" % call
        err = (tw - w_ref).abs().max().item()
        assert err <= TOL_W[act], "call %d: weight error %.3g" % (call, err)


def test_static_router_rejects_what_does_not_fit():
    import sparse_moe_layer_top_b200 as moe
    # 157 x 2 (row block, expert block) tiles already cover the GPU, so the
    # router takes one split: 20000 x 512 fp32 logits = 41 MB > the 32 MiB
    # array.  Real buffers all the same, so that nothing could go wrong even
    # if the check let the call through.
    T, d, E, k = 20000, 8192, 512, 10
    x = torch.zeros((T, d), dtype=torch.bfloat16, device="cuda")
    w_r = torch.zeros((E, d), dtype=torch.bfloat16, device="cuda")
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    tw = torch.empty((T, k), dtype=torch.float32, device="cuda")
    prob = moe.Problem.make(T, d, E, k, 2048, 2048, "bf16", "bf16")
    L = moe.lib()
    rc = L.moe_router_topk_static(ctypes.byref(prob), _p(x), _p(w_r), None, _p(ids), _p(tw),
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    assert rc == 2
    assert b"scratch" in L.moe_last_error_string()


def test_static_router_takes_any_size_on_the_epilogue_selecting_form():
    import sparse_moe_layer_top_b200 as moe
    # E <= 256: the router selects in its GEMM epilogue, with the partial
    # logits and the lists moving through the shared memory of its 4-CTA
    # clusters -- no scratch, so a batch of 65536 tokens is taken (it would
    # not fit the built-in array in split-K form) and matches the workspace
    # router.
    T, d, E, k = 65536, 256, 256, 8
    x = moe_inputs.randn((T, d), "cuda", 7, moe_inputs.X, 1.0, torch.bfloat16)
    w_r = moe_inputs.randn((E, d), "cuda", 7, moe_inputs.W_R, 0.02, torch.bfloat16)
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    tw = torch.empty((T, k), dtype=torch.float32, device="cuda")
    prob = moe.Problem.make(T, d, E, k, 128, 128, "bf16", "bf16")
    assert moe.forward_plan(prob)["router_selects"]
    L = moe.lib()
    rc = L.moe_router_topk_static(ctypes.byref(prob), _p(x), _p(w_r), None, _p(ids), _p(tw),
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    assert rc == 0, L.moe_last_error_string()
    assert moe.device_status()[0] == 0
    ids_ref, w_ref = moe.router_topk(prob, x, w_r)
    torch.cuda.synchronize()
    assert torch.equal(ids, ids_ref)
    assert (tw - w_ref).abs().max().item() <= TOL_W["bf16"]


def _router_inputs(moe, T, d, E, k, seed):
    x = moe_inputs.randn((T, d), "cuda", seed, moe_inputs.X, 1.0, torch.bfloat16)
    w_r = moe_inputs.randn((E, d), "cuda", seed, moe_inputs.W_R, 0.02, torch.bfloat16)
    return moe.Problem.make(T, d, E, k, 64, 64, "bf16", "bf16"), x, w_r


def test_static_router_leaves_no_state_between_problems_and_allocates_nothing():
    """The built-in array keeps what the last call left: a large problem, then
    a smaller one of the same router form, must still match the workspace
    router.  Around the later calls neither the device's free memory nor the
    caching allocator's reservation moves: the entry point allocates nothing."""
    import sparse_moe_layer_top_b200 as moe
    torch.cuda.set_device(0)
    L = moe.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    big = _router_inputs(moe, 4096, 2048, 256, 8, 11)
    small = _router_inputs(moe, 1921, 512, 200, 6, 12)
    assert moe.forward_plan(big[0])["router_selects"] and moe.forward_plan(small[0])["router_selects"]
    out = {}
    for name, (prob, x, w_r) in (("big", big), ("small", small)):
        ids = torch.empty((prob.T, prob.k), dtype=torch.int32, device="cuda")
        tw = torch.empty((prob.T, prob.k), dtype=torch.float32, device="cuda")
        ref = moe.router_topk(prob, x, w_r)
        out[name] = (prob, x, w_r, ids, tw, ref)
    torch.cuda.synchronize()
    # a first call of each problem: kernel modules, the array's address
    for prob, x, w_r, ids, tw, _ in out.values():
        assert L.moe_router_topk_static(ctypes.byref(prob), _p(x), _p(w_r), None, _p(ids), _p(tw), stream) == 0
    torch.cuda.synchronize()
    for name in ("big", "small", "big", "small"):
        prob, x, w_r, ids, tw, (ids_ref, w_ref) = out[name]
        ids.fill_(-7)
        tw.fill_(-1.0)
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info()
        reserved0 = torch.cuda.memory_reserved()
        rc = L.moe_router_topk_static(ctypes.byref(prob), _p(x), _p(w_r), None, _p(ids), _p(tw), stream)
        assert rc == 0, L.moe_last_error_string()
        torch.cuda.synchronize()
        free1, _ = torch.cuda.mem_get_info()
        assert torch.cuda.memory_reserved() == reserved0, name
        assert free1 == free0, "%s: device free memory moved by %d bytes" % (name, free0 - free1)
        assert moe.device_status()[0] == 0
        assert torch.equal(ids, ids_ref), name
        assert (tw - w_ref).abs().max().item() <= TOL_W["bf16"], name
