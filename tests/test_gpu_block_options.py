"""The block's neighbours on the GPU, against the float64 oracle: the
zero-centred RMSNorm prologue (as a stage and inside the fused block) and the
sigmoid gate on the shared expert, on every kernel path."""
import numpy as np
import pytest
import torch

import moe_inputs
import oracle
from parity import TOL, TOL_W, check_routing, precision_key, rel_l2, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import sparse_moe_layer_top_b200 as m
    yield m
    m.set_path(0)


@pytest.fixture(autouse=True)
def _automatic_path_after_each_test():
    yield
    import sparse_moe_layer_top_b200 as m
    m.set_path(0)


def _no_device_errors(moe):
    s, detail = moe.device_status()
    assert s == 0, "device status %d detail 0x%08x" % (s, detail & 0xffffffff)


def _vec(d, scale, seed, dtype):
    return (torch.randn(d, generator=torch.Generator().manual_seed(seed)) * scale).to(dtype)


@pytest.mark.parametrize("act,T,d", [("bf16", 300, 256), ("bf16", 7, 8192), ("f32", 65, 136)])
def test_rmsnorm_stage_matches_oracle(moe, act, T, d):
    dt = torch.bfloat16 if act == "bf16" else torch.float32
    x = (torch.randn(T, d, generator=torch.Generator().manual_seed(T)) * 3.0).to(dt)
    x[0] = 0  # an all-zero row stays zero (eps keeps it finite)
    gamma = _vec(d, 0.2, d, dt)
    prob = moe.Problem.make(T, d, 8, 2, 64, 64, act, act)
    out = moe.rmsnorm(prob, x.cuda(), gamma.cuda(), eps=1e-6)
    torch.cuda.synchronize()
    ref = oracle.rmsnorm(x, gamma, 1e-6)
    got = out.double().cpu().numpy()
    # fp32 arithmetic: the sum of d squares carries up to d roundings of 2^-24
    # relative, halved by the square root, plus the division, the two products
    # and 1 + gamma: (d / 2 + 8) * 2^-24 relative.  bf16 output: one more
    # rounding, at most one unit in the last place (2^-8 relative).
    fp32 = (d / 2 + 8) * 2.0 ** -24
    bound = fp32 + (2.0 ** -8 if act == "bf16" else 0.0)
    assert np.all(np.abs(got - ref) <= bound * np.abs(ref) + 1e-30)
    assert np.all(got[0] == 0)


# (T, d, E, k, I, I_s, act, w, bias)
CASES = {
    "bf16": (300, 256, 20, 4, 192, 128, "bf16", "bf16", None),
    "bf16_zipf_long": (700, 512, 6, 2, 256, 256, "bf16", "bf16", "zipf"),
    "fp8": (300, 384, 12, 3, 384, 256, "bf16", "fp8", None),
    "f32": (40, 128, 16, 2, 64, 64, "f32", "f32", None),
}


@pytest.mark.parametrize("opts", ["norm", "gate", "norm_gate"])
@pytest.mark.parametrize("path", [0, 1, 2, 3, 4, 5, 6])
@pytest.mark.parametrize("case", list(CASES))
def test_block_with_options_matches_oracle(moe, case, path, opts):
    T, d, E, k, I, I_s, act, w, bias = CASES[case]
    if act == "f32" and path >= 2:
        pytest.skip("fp32 problems run on the SIMT kernels only")
    inp = moe_inputs.make_inputs(T, d, E, k, I, I_s, act=act, w=w, bias=bias, seed=11)
    dt = torch.bfloat16 if act == "bf16" else torch.float32
    norm_w = _vec(d, 0.1, 1, dt) if "norm" in opts else None
    gate_w = _vec(d, 0.05, 2, dt) if "gate" in opts else None
    moe.set_path(path)
    g = to_device(inp, "cuda")
    prob = moe.Problem.make(T, d, E, k, I, I_s, act, w)
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    tw = torch.empty((T, k), dtype=torch.float32, device="cuda")
    y = moe.block_forward(prob, g.x, g.w_r, g.bias, g.wg, g.wu, g.wd, g.s_wg, g.s_wu, g.s_wd, g.scales,
                          norm_weight=None if norm_w is None else norm_w.cuda(), norm_eps=1e-6,
                          shared_gate=None if gate_w is None else gate_w.cuda(), topk_ids=ids, topk_w=tw)
    torch.cuda.synchronize()
    _no_device_errors(moe)
    kw = dict(bias=inp.bias, scales=inp.scales, norm_weight=norm_w, norm_eps=1e-6, shared_gate=gate_w)
    y_or, ids_or, _, probs, _ = oracle.block_forward(inp.x, inp.w_r, inp.wg, inp.wu, inp.wd, inp.s_wg, inp.s_wu,
                                                     inp.s_wd, k, **kw)
    key = precision_key(inp)
    use, differ = check_routing(ids.cpu().numpy(), tw.cpu().numpy(), probs, ids_or, TOL_W[key])
    if differ:
        y_or, *_ = oracle.block_forward(inp.x, inp.w_r, inp.wg, inp.wu, inp.wd, inp.s_wg, inp.s_wu, inp.s_wd, k,
                                        force_ids=use, **kw)
    err = rel_l2(y.float().cpu().numpy(), y_or)
    assert err <= TOL[key], "rel-L2 %.3g > %.3g" % (err, TOL[key])


def test_no_options_is_the_plain_forward_bit_for_bit(moe):
    inp = moe_inputs.make_inputs(200, 256, 16, 4, 128, 128, act="bf16", w="bf16", seed=3)
    g = to_device(inp, "cuda")
    prob = moe.Problem.make(200, 256, 16, 4, 128, 128, "bf16", "bf16")
    a = moe.layer_forward(prob, g.x, g.w_r, g.bias, g.wg, g.wu, g.wd, g.s_wg, g.s_wu, g.s_wd, g.scales)
    b = moe.block_forward(prob, g.x, g.w_r, g.bias, g.wg, g.wu, g.wd, g.s_wg, g.s_wu, g.s_wd, g.scales)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_gate_without_a_shared_expert_changes_nothing(moe):
    inp = moe_inputs.make_inputs(150, 192, 12, 2, 96, 0, act="bf16", w="bf16", seed=5, shared=False)
    g = to_device(inp, "cuda")
    prob = moe.Problem.make(150, 192, 12, 2, 96, 0, "bf16", "bf16")
    a = moe.layer_forward(prob, g.x, g.w_r, g.bias, g.wg, g.wu, g.wd)
    b = moe.block_forward(prob, g.x, g.w_r, g.bias, g.wg, g.wu, g.wd,
                          shared_gate=_vec(192, 0.05, 2, torch.bfloat16).cuda())
    torch.cuda.synchronize()
    assert torch.equal(a, b)
