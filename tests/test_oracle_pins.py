"""Pins of the float64 oracle against facts that do not come from the oracle.

Each test targets a plausible mistake: a transposed operand, gate and up
swapped, a missing renormalisation, a wrong tie-break, a wrong scale index, a
non-stable dispatch order.  Sources: closed forms, invariants of the block's
definition, brute-force enumeration on tiny inputs, library routines (torch's
E4M3 conversion, numpy matmul/kron), and the parameter counts the pages print.
"""
import itertools
import json
import math
import os

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st
import pytest
import torch

import oracle
import moe_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f32(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _silu(z):
    return z / (1.0 + np.exp(-z))


def _np_expert(x, wg, wu, wd):
    """numpy matmul route to one expert (float64)."""
    x, wg, wu, wd = (np.asarray(a, np.float64) for a in (x, wg, wu, wd))
    return (_silu(x @ wg.T) * (x @ wu.T)) @ wd.T


def _tiny(T=6, d=8, E=5, k=2, I=4, I_s=3, seed=0, shared=True):
    inp = moe_inputs.make_inputs(T, d, E, k, I, I_s, act="f32", w="f32", seed=seed, shared=shared)
    # Larger weights than N(0, 0.02) so that every term matters at float64 precision.
    for name in ("w_r", "wg", "wu", "wd", "s_wg", "s_wu", "s_wd"):
        t = getattr(inp, name)
        if t is not None:
            setattr(inp, name, t * 25.0)
    return inp


def _fwd(inp, **kw):
    return oracle.moe_forward(inp.x, inp.w_r, inp.wg, inp.wu, inp.wd, inp.s_wg, inp.s_wu,
                              inp.s_wd, inp.k, bias=kw.pop("bias", inp.bias), **kw)


# --------------------------------------------------------------------------
# Parameter bookkeeping against the numbers the pages print.
# --------------------------------------------------------------------------
def test_param_counts_match_pages():
    with open(os.path.join(GOLDEN, "param_counts.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        n = c["blocks"] * oracle.param_count(c["d"], c["E"], c["k"], c["I"], c["I_s"], c["active"])
        assert abs(n - c["printed"]) <= c["rel_tol"] * c["printed"], (c["name"], n)


# --------------------------------------------------------------------------
# Element decoding.
# --------------------------------------------------------------------------
def test_e4m3_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    mine = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(mine, ref, equal_nan=True)
    assert mine[0x7E] == 448.0 and mine[0x01] == 2.0 ** -9


def test_bf16_inputs_decode_exactly():
    inp = _tiny()
    # round the same values to bf16 and feed them both ways
    conv = {n: getattr(inp, n).to(torch.bfloat16) for n in ("x", "w_r", "wg", "wu", "wd", "s_wg", "s_wu", "s_wd")}
    yb, idsb, wb, _ = oracle.moe_forward(conv["x"], conv["w_r"], conv["wg"], conv["wu"], conv["wd"],
                                         conv["s_wg"], conv["s_wu"], conv["s_wd"], 2)
    yf, idsf, wf, _ = oracle.moe_forward(*(conv[n].float() for n in ("x", "w_r", "wg", "wu", "wd", "s_wg", "s_wu", "s_wd")), 2)
    assert np.array_equal(yb, yf) and np.array_equal(idsb, idsf) and np.array_equal(wb, wf)


# --------------------------------------------------------------------------
# The expert: closed forms that fix SiLU, the gate/up roles and orientation.
# --------------------------------------------------------------------------
@pytest.mark.parametrize("x,g,u,dn,expect", [
    # dn * silu(g x) * (u x) with silu(1) = 1/(1+e^-1) = 0.7310585786300049
    (1.0, 1.0, 2.0, 3.0, 3.0 * 0.7310585786300049 * 2.0),
    # silu(-2) = -2/(1+e^2) = -0.2384058440442351; u x = -1.0
    (-1.0, 2.0, 1.0, 0.5, 0.5 * -0.2384058440442351 * -1.0),
    # gate 0 kills the expert: silu(0) = 0
    (3.0, 0.0, 7.0, 9.0, 0.0),
])
def test_single_unit_expert_closed_form(x, g, u, dn, expect):
    out = oracle.swiglu_expert(_f32([[x]]), _f32([[g]]), _f32([[u]]), _f32([[dn]]))
    assert out.shape == (1, 1)
    assert abs(out[0, 0] - expect) <= 1e-15 * max(1.0, abs(expect))


def test_expert_operand_orientation():
    # d = 2, I = 2.  W_gate picks x_1 into unit 0, W_up is the identity,
    # W_down copies unit 0 into output 1 (times 3):
    #   out = [0, 3 * silu(x_1) * x_0].  With x = [2, -1]:
    #   silu(-1) = -1/(1+e) = -0.2689414213699951  ->  out_1 = -1.6136485282199706.
    # Reading W_gate or W_down transposed gives 0 in both places.
    x = _f32([[2.0, -1.0]])
    wg = _f32([[0.0, 1.0], [0.0, 0.0]])
    wu = _f32([[1.0, 0.0], [0.0, 1.0]])
    wd = _f32([[0.0, 0.0], [3.0, 0.0]])
    out = oracle.swiglu_expert(x, wg, wu, wd)
    assert out[0, 0] == 0.0
    assert abs(out[0, 1] - (-1.6136485282199706)) < 1e-15


# --------------------------------------------------------------------------
# The router: closed forms, brute force, tie-break, invariants.
# --------------------------------------------------------------------------
def test_router_two_experts_is_a_sigmoid():
    # E = k = 2: the renormalised weights are the full softmax of two logits,
    # w_0 = 1/(1+exp(l_1-l_0)).  l = 1.5*[0.5, -0.25] = [0.75, -0.375] ->
    # w_0 = 1/(1+e^-1.125) = 0.7549149868676283 (all inputs exact in fp32).
    probs, ids, w = oracle.router(_f32([[1.5]]), _f32([[0.5], [-0.25]]), 2)
    assert list(ids[0]) == [0, 1]
    assert abs(w[0, 0] - 0.7549149868676283) < 1e-15
    assert abs(w[0, 1] - (1 - 0.7549149868676283)) < 1e-15
    assert abs(probs[0].sum() - 1.0) < 1e-15


@pytest.mark.parametrize("E,k", [(4, 1), (5, 2), (6, 3), (8, 4), (7, 7)])
def test_topk_against_brute_force_subsets(E, k):
    rng = np.random.default_rng(E * 10 + k)
    T, d = 12, 5
    x = _f32(rng.standard_normal((T, d)))
    w_r = _f32(rng.standard_normal((E, d)))
    # a token with exactly tied logits tests the tie-break too
    w_r[E - 1] = w_r[0]
    probs, ids, w = oracle.router(x, w_r, k)
    logits = x.astype(np.float64) @ w_r.astype(np.float64).T
    p = np.exp(logits - logits.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    for t in range(T):
        best, best_key = None, None
        for S in itertools.combinations(range(E), k):
            key = (round(float(p[t, list(S)].sum()), 12), tuple(-s for s in S))
            if best_key is None or key > best_key:
                best, best_key = S, key
        assert sorted(ids[t].tolist()) == list(best)
        np.testing.assert_allclose(w[t], p[t, ids[t]] / p[t, ids[t]].sum(), rtol=1e-12)
        assert abs(w[t].sum() - 1.0) < 1e-12
        # ids come out in descending probability
        assert all(p[t, ids[t][i]] >= p[t, ids[t][i + 1]] for i in range(k - 1))


def test_zero_router_ties_go_to_lower_index():
    inp = _tiny(T=4, E=6, k=3)
    inp.w_r = torch.zeros_like(inp.w_r)
    y, ids, w, probs = _fwd(inp)
    assert (ids == np.array([0, 1, 2])).all()
    np.testing.assert_allclose(w, 1.0 / 3.0, rtol=1e-15)
    np.testing.assert_allclose(probs, 1.0 / 6.0, rtol=1e-15)


def test_logit_shift_changes_nothing():
    inp = _tiny()
    y0, ids0, w0, _ = _fwd(inp)
    y1, ids1, w1, _ = _fwd(inp, bias=torch.full((inp.E,), 3.25))
    assert np.array_equal(ids0, ids1)
    np.testing.assert_allclose(w0, w1, rtol=1e-13)
    np.testing.assert_allclose(y0, y1, rtol=1e-12, atol=1e-13)


def test_bias_enters_the_softmax():
    # a large bias on one expert must put it in every token's set
    inp = _tiny(E=5, k=2)
    b = torch.zeros(5)
    b[3] = 50.0
    _, ids, w, _ = _fwd(inp, bias=b)
    assert all(3 in row for row in ids.tolist())
    assert (w[:, 0] > 0.999).all() and (ids[:, 0] == 3).all()


# --------------------------------------------------------------------------
# The whole block: invariants named by the block's definition.
# --------------------------------------------------------------------------
def test_k_equals_E_is_the_dense_mixture():
    inp = _tiny(T=5, E=4, k=4)
    y, ids, w, probs = _fwd(inp)
    x = inp.x.double().numpy()
    dense = _np_expert(x, inp.s_wg, inp.s_wu, inp.s_wd)
    logits = x @ inp.w_r.double().numpy().T
    p = np.exp(logits - logits.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    for e in range(inp.E):
        dense += p[:, e:e + 1] * _np_expert(x, inp.wg[e], inp.wu[e], inp.wd[e])
    np.testing.assert_allclose(y, dense, rtol=1e-11, atol=1e-12)


def test_zero_routed_experts_leave_the_shared_expert():
    inp = _tiny()
    inp.wd = torch.zeros_like(inp.wd)
    y, *_ = _fwd(inp)
    np.testing.assert_allclose(y, _np_expert(inp.x, inp.s_wg, inp.s_wu, inp.s_wd), rtol=1e-12, atol=1e-13)


def test_no_shared_expert_is_pure_routed_mixture():
    inp = _tiny(shared=False)
    y, ids, w, _ = _fwd(inp)
    x = inp.x.double().numpy()
    for t in range(inp.T):
        ref = sum(w[t, s] * _np_expert(x[t:t + 1], inp.wg[ids[t, s]], inp.wu[ids[t, s]], inp.wd[ids[t, s]])[0]
                  for s in range(inp.k))
        np.testing.assert_allclose(y[t], ref, rtol=1e-11, atol=1e-12)


def test_token_permutation_permutes_outputs():
    inp = _tiny(T=9)
    y0, ids0, w0, _ = _fwd(inp)
    perm = torch.tensor([4, 0, 8, 2, 7, 1, 3, 6, 5])
    inp.x = inp.x[perm].contiguous()
    y1, ids1, w1, _ = _fwd(inp)
    assert np.array_equal(ids1, ids0[perm.numpy()])
    np.testing.assert_array_equal(y1, y0[perm.numpy()])


def test_routed_part_scales_with_w_down():
    inp = _tiny()
    y1, *_ = _fwd(inp)
    shared = _np_expert(inp.x, inp.s_wg, inp.s_wu, inp.s_wd)
    inp.wd = inp.wd * 0.5          # exact in binary
    y2, *_ = _fwd(inp)
    np.testing.assert_allclose(y2 - shared, 0.5 * (y1 - shared), rtol=1e-11, atol=1e-12)


def test_forced_sets_reweight_by_their_probabilities():
    inp = _tiny(E=5, k=2)
    _, _, _, probs = _fwd(inp)
    force = np.tile(np.array([[4, 1]], np.int32), (inp.T, 1))
    y, ids, w, _ = _fwd(inp, force_ids=force)
    assert (ids == force).all()
    np.testing.assert_allclose(w[:, 0], probs[:, 4] / (probs[:, 4] + probs[:, 1]), rtol=1e-13)


# --------------------------------------------------------------------------
# Dispatch / combine stages.
# --------------------------------------------------------------------------
def test_permute_is_a_stable_sort_by_expert():
    ids, _ = moe_inputs.random_routing(37, 9, 3, seed=4)
    ids = ids.numpy()
    offs, row_tok, row_slot, pos = oracle.permute(ids, 9)
    T, k = ids.shape
    order = sorted(((ids[t, j], t, j) for t in range(T) for j in range(k)))
    assert [(t, j) for _, t, j in order] == list(zip(row_tok[:T * k].tolist(), row_slot[:T * k].tolist()))
    counts = np.bincount(ids.ravel(), minlength=9)
    assert offs[0] == 0 and (np.diff(offs[:10]) == counts).all()
    assert offs[9] == T * k and offs[10] == T * k + T
    assert (row_tok[T * k:] == np.arange(T)).all() and (row_slot[T * k:] == k).all()
    for t in range(T):
        for j in range(k):
            r = pos[t, j]
            assert row_tok[r] == t and row_slot[r] == j and offs[ids[t, j]] <= r < offs[ids[t, j] + 1]


def test_stages_chain_to_the_whole_block():
    inp = _tiny(T=11, E=6, k=3)
    y, ids, w, _ = _fwd(inp)
    offs, row_tok, _, pos = oracle.permute(ids, inp.E)
    x_perm = inp.x[torch.from_numpy(row_tok).long()].contiguous()
    y_perm = oracle.expert_ffn(x_perm, offs, inp.wg, inp.wu, inp.wd, inp.s_wg, inp.s_wu, inp.s_wd)
    y2 = oracle.combine(y_perm.astype(np.float32), pos, w.astype(np.float32), offs, inp.E)
    # y_perm and the weights were rounded to fp32 on the way: allow that rounding
    np.testing.assert_allclose(y2, y, rtol=2e-6, atol=1e-6 * np.abs(y).max())


def test_combine_indexes_rows_and_weights():
    # y_perm row r holds the constant r+1; token t's routed slots point at rows
    # pos[t] with weights w[t]; the shared row of t is offs[E] + t.
    T, E, k, d = 3, 2, 2, 4
    offs = np.array([0, 3, 6, 9], np.int32)
    pos = np.array([[0, 3], [4, 1], [2, 5]], np.int32)
    w = np.array([[0.25, 0.75], [0.5, 0.5], [1.0, 0.0]], np.float32)
    y_perm = np.repeat(np.arange(1, 10, dtype=np.float32)[:, None], d, axis=1)
    y = oracle.combine(y_perm, pos, w, offs, E)
    expect = [0.25 * 1 + 0.75 * 4 + 7, 0.5 * 5 + 0.5 * 2 + 8, 1.0 * 3 + 0.0 * 6 + 9]
    np.testing.assert_array_equal(y, np.repeat(np.array(expect)[:, None], d, axis=1))


# --------------------------------------------------------------------------
# FP8 weights: block-scale indexing.
# --------------------------------------------------------------------------
def test_fp8_block_scales_index_out_and_in_blocks():
    # d = 256 (2 column blocks), I = 128 (1 row block) for gate/up and the
    # reverse for down.  The dequantised matrix must be decode(q) times a
    # scale that is constant on each 128 x 128 block: built here with np.kron.
    rng = np.random.default_rng(3)
    d, I = 256, 128
    x = _f32(rng.standard_normal((3, d)))
    w = [torch.from_numpy(rng.standard_normal(s).astype(np.float32) * 0.05) for s in ((I, d), (I, d), (d, I))]
    qs = [moe_inputs.quantize_e4m3_blocks(m) for m in w]
    sg, su, sd = (np.array(s.numpy()) for _, s in qs)
    sg[0, 1] *= 3.0
    sd[1, 0] *= 0.25          # make every block's scale distinct from its transpose
    codes = [q.view(torch.uint8).numpy() for q, _ in qs]
    out = oracle.swiglu_expert(x, codes[0], codes[1], codes[2], sg, su, sd)
    deq = [oracle.e4m3_decode(c) * np.kron(s, np.ones((128, 128))) for c, s in zip(codes, (sg, su, sd))]
    np.testing.assert_allclose(out, _np_expert(x, *deq), rtol=1e-12, atol=1e-14)


def test_fp8_packed_scale_layout_in_the_whole_block():
    inp = moe_inputs.make_inputs(3, 256, 2, 1, 128, 128, act="bf16", w="fp8", seed=1)
    y, ids, w, _ = oracle.moe_forward(inp.x, inp.w_r, inp.wg, inp.wu, inp.wd, inp.s_wg, inp.s_wu,
                                      inp.s_wd, 1, scales=inp.scales)
    # unpack the documented layout by hand and recompute with numpy
    E, d, I, Is = 2, 256, 128, 128
    sc = inp.scales.numpy()
    n_g = E * (I // 128) * (d // 128)
    sg = sc[:n_g].reshape(E, I // 128, d // 128)
    su = sc[n_g:2 * n_g].reshape(E, I // 128, d // 128)
    sd = sc[2 * n_g:3 * n_g].reshape(E, d // 128, I // 128)
    o = 3 * n_g
    ssg = sc[o:o + 2].reshape(1, 2); ssu = sc[o + 2:o + 4].reshape(1, 2); ssd = sc[o + 4:o + 6].reshape(2, 1)

    def deq(q, s):
        return oracle.e4m3_decode(q.view(torch.uint8).numpy()) * np.kron(s, np.ones((128, 128)))

    x = inp.x.double().numpy()
    for t in range(3):
        e = ids[t, 0]
        ref = _np_expert(x[t:t + 1], deq(inp.wg[e], sg[e]), deq(inp.wu[e], su[e]), deq(inp.wd[e], sd[e]))
        ref += _np_expert(x[t:t + 1], deq(inp.s_wg, ssg), deq(inp.s_wu, ssu), deq(inp.s_wd, ssd))
        np.testing.assert_allclose(y[t], ref[0], rtol=1e-11, atol=1e-13)


# --------------------------------------------------------------------------
# The block's neighbours: zero-centred RMSNorm prologue, shared-expert gate.
# --------------------------------------------------------------------------
def test_rmsnorm_closed_form():
    # mean of squares of (3, 4) is 25/2, so the row is divided by 5/sqrt(2)
    out = oracle.rmsnorm(torch.tensor([[3.0, 4.0]]), torch.zeros(2), eps=0.0)
    np.testing.assert_allclose(out[0], [3 * math.sqrt(2) / 5, 4 * math.sqrt(2) / 5], rtol=1e-15)


def test_rmsnorm_zero_centred_scale():
    # the applied scale is 1 + gamma: gamma = -1 silences a channel, gamma = 1 doubles it
    x = torch.tensor([[3.0, 4.0, -12.0]])
    base = oracle.rmsnorm(x, torch.zeros(3), eps=0.0)
    out = oracle.rmsnorm(x, torch.tensor([-1.0, 1.0, 0.5]), eps=0.0)
    np.testing.assert_allclose(out[0], [0.0, 2 * base[0, 1], 1.5 * base[0, 2]], rtol=1e-15)


def test_rmsnorm_is_scale_invariant_and_unit_rms():
    x = torch.randn(7, 64, generator=torch.Generator().manual_seed(3))
    a = oracle.rmsnorm(x, torch.zeros(64), eps=0.0)
    b = oracle.rmsnorm(x * 4.0, torch.zeros(64), eps=0.0)
    np.testing.assert_allclose(a, b, rtol=1e-14)
    np.testing.assert_allclose((a * a).mean(axis=1), 1.0, rtol=1e-13)
    # eps keeps an all-zero row finite (and zero)
    z = oracle.rmsnorm(torch.zeros(1, 8), torch.zeros(8), eps=1e-6)
    assert np.all(z == 0.0)


def test_block_with_norm_is_the_block_on_the_normalised_rounded_input():
    inp = moe_inputs.make_inputs(9, 64, 6, 2, 32, 32, act="bf16", w="bf16", seed=4)
    gamma = (torch.randn(64, generator=torch.Generator().manual_seed(5)) * 0.1).to(torch.bfloat16)
    # numpy RMSNorm, rounded by torch's float -> bf16 conversion
    x = inp.x.double().numpy()
    xn = x / np.sqrt((x * x).mean(axis=1, keepdims=True) + 1e-6) * (1.0 + gamma.double().numpy())
    xn_bf16 = torch.from_numpy(xn).float().to(torch.bfloat16)
    y, ids, w, _, gate = oracle.block_forward(inp.x, inp.w_r, inp.wg, inp.wu, inp.wd, inp.s_wg, inp.s_wu,
                                              inp.s_wd, inp.k, norm_weight=gamma, norm_eps=1e-6)
    y2, ids2, w2, _ = oracle.moe_forward(xn_bf16, inp.w_r, inp.wg, inp.wu, inp.wd, inp.s_wg, inp.s_wu,
                                         inp.s_wd, inp.k)
    assert np.array_equal(ids, ids2)
    np.testing.assert_allclose(y, y2, rtol=1e-12, atol=1e-14)
    assert np.all(gate == 1.0)


def test_shared_gate_weights_the_shared_expert_linearly():
    inp = _tiny(T=8, d=8, E=5, k=2, I=4, I_s=3, seed=6)
    gw = torch.randn(8, generator=torch.Generator().manual_seed(7)) * 0.3
    y_full, ids, _, _ = _fwd(inp)
    y_routed, ids0, _, _ = oracle.moe_forward(inp.x, inp.w_r, inp.wg, inp.wu, inp.wd, None, None, None, inp.k)
    y, ids1, _, _, gate = oracle.block_forward(inp.x, inp.w_r, inp.wg, inp.wu, inp.wd, inp.s_wg, inp.s_wu,
                                               inp.s_wd, inp.k, shared_gate=gw)
    assert np.array_equal(ids, ids0) and np.array_equal(ids, ids1)
    g = 1.0 / (1.0 + np.exp(-(inp.x.double().numpy() @ gw.double().numpy())))
    np.testing.assert_allclose(gate, g, rtol=1e-14)
    np.testing.assert_allclose(y, y_routed + g[:, None] * (y_full - y_routed), rtol=1e-11, atol=1e-12)
    # a zero gate vector halves the shared expert
    _, _, _, _, half = oracle.block_forward(inp.x, inp.w_r, inp.wg, inp.wu, inp.wd, inp.s_wg, inp.s_wu,
                                            inp.s_wd, inp.k, shared_gate=torch.zeros(8))
    assert np.all(half == 0.5)


@settings(max_examples=300, deadline=None)
@given(st.integers(2, 9).flatmap(lambda E: st.tuples(
    st.just(E), st.integers(1, E), st.lists(st.integers(-3, 2), min_size=E, max_size=E))))
def test_topk_with_exact_ties_against_brute_force(case):
    """x = 0, so the logits are exactly the bias; a bias drawn from six values
    makes exact ties common.  The kept set maximises the summed probability,
    ties to the lexicographically smallest index set; the ids come out by
    descending probability, equal ones by ascending index."""
    E, k, levels = case
    bias = torch.tensor([0.5 * v for v in levels], dtype=torch.float32)
    x = _f32(np.zeros((2, 1)))
    w_r = _f32(np.ones((E, 1)))
    probs, ids, w = oracle.router(x, w_r, k, bias=bias)
    b = bias.double().numpy()
    p = np.exp(b - b.max())
    p /= p.sum()
    best, best_key = None, None
    for S in itertools.combinations(range(E), k):
        key = (round(float(p[list(S)].sum()), 12), tuple(-s for s in S))
        if best_key is None or key > best_key:
            best, best_key = S, key
    for t in range(2):
        got = ids[t].tolist()
        assert sorted(got) == list(best)
        assert got == sorted(got, key=lambda e: (-p[e], e))
        np.testing.assert_allclose(w[t], p[got] / p[got].sum(), rtol=1e-12)
