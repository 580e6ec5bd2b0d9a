"""Expert parallelism on the GPU.

* ep_expand_ids against numpy's repeat, and its device checks;
* the expert-parallel block (sparse_moe_layer_top_b200.ep) with G ranks
  emulated step by step in one process on one GPU: every exchange is done by
  slicing the senders' buffers, so no kernel ever waits for another rank, and
  every rank's output is checked against the oracle block over its tokens;
* one real rank of an NCCL process group through TorchExchange."""
import os
import socket

import numpy as np
import pytest
import torch

import moe_inputs
import oracle
from parity import TOL, TOL_W, check_routing, precision_key, rel_l2
from sparse_moe_layer_top_b200 import ep

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import sparse_moe_layer_top_b200 as m
    yield m
    m.set_path(0)


def _no_device_errors(moe):
    s, detail = moe.device_status()
    assert s == 0, "device status %d detail 0x%08x" % (s, detail & 0xffffffff)


@pytest.mark.parametrize("G,E_l,hi", [(1, 1, 5), (2, 128, 40), (8, 64, 40), (16, 256, 3), (3, 5, 4000)])
def test_ep_expand_ids_matches_repeat(moe, G, E_l, hi):
    rng = np.random.default_rng(G * 1000 + E_l)
    c = rng.integers(0, hi, size=G * E_l).astype(np.int32)
    c[rng.random(G * E_l) < 0.3] = 0
    R = int(c.sum())
    ids = moe.ep_expand_ids(torch.from_numpy(c).cuda(), G, E_l, R)
    torch.cuda.synchronize()
    _no_device_errors(moe)
    ref = np.repeat(np.tile(np.arange(E_l, dtype=np.int32), G), c)
    assert np.array_equal(ids.cpu().numpy(), ref)


def test_ep_expand_ids_flags_short_and_negative_counts(moe):
    # blocks (s0, e0) = 3, (s0, e1) = 0, (s1, e0) = 2, (s1, e1) = 1: 6 rows counted, 8 asked for
    c = torch.tensor([3, 0, 2, 1], dtype=torch.int32, device="cuda")
    ids = moe.ep_expand_ids(c, 2, 2, 8)
    torch.cuda.synchronize()
    s, detail = moe.device_status()
    assert s == 6 and (detail & 0xffffffff) == 0x06000002
    assert ids.cpu().tolist() == [0, 0, 0, 0, 0, 1, -1, -1]
    c = torch.tensor([2, -1], dtype=torch.int32, device="cuda")
    ids = moe.ep_expand_ids(c, 1, 2, 2)
    torch.cuda.synchronize()
    s, detail = moe.device_status()
    assert s == 6 and (detail & 0xffffffff) == 0x06000002
    assert ids.cpu().tolist() == [0, 0]


def _emulate(layers, xs):
    """One forward of G ranks, step by step in one process; each exchange
    slices the senders' buffers in rank order."""
    G, E_l, k = len(layers), layers[0].E_l, layers[0].k
    st = [L.dispatch(x) for L, x in zip(layers, xs)]
    for r, L in enumerate(layers):
        rc = []
        for s in range(G):
            rc += st[s].send_counts[r * E_l:(r + 1) * E_l]
        L.set_received(st[r], rc)

    def start(s, r):  # first row of source s bound for rank r
        return sum(st[s].send_rows[:r])

    y_recv = []
    for r, L in enumerate(layers):
        parts = [st[s].x_perm[start(s, r):start(s, r) + st[s].send_rows[r]] for s in range(G)]
        x_recv = torch.cat(parts).contiguous()
        L.shared(st[r])
        y_recv.append(L.experts(st[r], x_recv))
    for s in range(G):
        R = st[s].T * k
        chunks = []
        for r in range(G):
            off = sum(st[r].recv_rows[:s])
            chunks.append(y_recv[r][off:off + st[r].recv_rows[s]])
        if R:
            st[s].y_full[:R] = torch.cat(chunks)
    return [L.combine(s_) for L, s_ in zip(layers, st)], st


def _check_rank(inp, lo, hi, y, state):
    T = hi - lo
    if T == 0:
        assert y.shape[0] == 0
        return
    x = inp.x[lo:hi].contiguous()
    key = precision_key(inp)
    y_or, ids_or, _, probs = oracle.moe_forward(x, inp.w_r, inp.wg, inp.wu, inp.wd, inp.s_wg, inp.s_wu, inp.s_wd,
                                                inp.k, bias=inp.bias, scales=inp.scales)
    use, differ = check_routing(state.ids.cpu().numpy(), state.tw.cpu().numpy(), probs, ids_or, TOL_W[key])
    if differ:
        y_or, *_ = oracle.moe_forward(x, inp.w_r, inp.wg, inp.wu, inp.wd, inp.s_wg, inp.s_wu, inp.s_wd, inp.k,
                                      bias=inp.bias, scales=inp.scales, force_ids=use)
    err = rel_l2(y.float().cpu().numpy(), y_or)
    assert err <= TOL[key], "rel-L2 %.3g > %.3g" % (err, TOL[key])


@pytest.mark.parametrize("G,tokens,I_s", [(2, [300, 212], 128), (4, [150, 0, 333, 117], 128), (4, [64, 64, 1, 9], 0),
                                          (8, [40, 0, 17, 1, 64, 5, 33, 2], 128)])
def test_expert_parallel_ranks_emulated_on_one_gpu_match_the_oracle(moe, G, tokens, I_s):
    d, E, k, I = 256, 32, 4, 128
    inp = moe_inputs.make_inputs(sum(tokens), d, E, k, I, I_s, act="bf16", w="bf16", seed=11, shared=I_s > 0)
    g = {n: (getattr(inp, n).cuda() if getattr(inp, n) is not None else None)
         for n in ("x", "w_r", "wg", "wu", "wd", "s_wg", "s_wu", "s_wd")}
    bounds = np.concatenate([[0], np.cumsum(tokens)]).tolist()
    layers, xs = [], []
    for r in range(G):
        wg, wu, wd = ep.split_experts(r, G, g["wg"], g["wu"], g["wd"])
        layers.append(ep.EPMoELayer(r, G, d, E, k, I, I_s, g["w_r"], wg, wu, wd, g["s_wg"], g["s_wu"], g["s_wd"]))
        xs.append(g["x"][bounds[r]:bounds[r + 1]].contiguous())
    ys, st = _emulate(layers, xs)
    torch.cuda.synchronize()
    _no_device_errors(moe)
    for r in range(G):
        _check_rank(inp, bounds[r], bounds[r + 1], ys[r], st[r])


@pytest.mark.parametrize("G,tokens,I_s", [(2, [300, 212], 128), (4, [64, 0, 130, 9], 0)])
def test_expert_parallel_e4m3_ranks_emulated_on_one_gpu_match_the_oracle(moe, G, tokens, I_s):
    d, E, k, I = 256, 16, 4, 128
    inp = moe_inputs.make_inputs(sum(tokens), d, E, k, I, I_s, act="bf16", w="fp8", seed=13, shared=I_s > 0)
    g = {n: (getattr(inp, n).cuda() if getattr(inp, n) is not None else None)
         for n in ("x", "w_r", "wg", "wu", "wd", "s_wg", "s_wu", "s_wd", "scales")}
    bounds = np.concatenate([[0], np.cumsum(tokens)]).tolist()
    layers, xs = [], []
    for r in range(G):
        wg, wu, wd = ep.split_experts(r, G, g["wg"], g["wu"], g["wd"])
        sc = ep.split_scales(r, G, E, d, I, I_s, g["scales"])
        layers.append(ep.EPMoELayer(r, G, d, E, k, I, I_s, g["w_r"], wg, wu, wd, g["s_wg"], g["s_wu"], g["s_wd"],
                                    w="fp8", scales=sc))
        xs.append(g["x"][bounds[r]:bounds[r + 1]].contiguous())
    ys, st = _emulate(layers, xs)
    torch.cuda.synchronize()
    _no_device_errors(moe)
    for r in range(G):
        _check_rank(inp, bounds[r], bounds[r + 1], ys[r], st[r])


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_expert_parallel_single_nccl_rank(moe):
    import datetime
    import torch.distributed as dist
    d, E, k, I, I_s, T = 256, 16, 4, 128, 128, 200
    inp = moe_inputs.make_inputs(T, d, E, k, I, I_s, act="bf16", w="bf16", seed=12)
    g = {n: getattr(inp, n).cuda() for n in ("x", "w_r", "wg", "wu", "wd", "s_wg", "s_wu", "s_wd")}
    dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % _free_port(), rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        layer = ep.EPMoELayer(0, 1, d, E, k, I, I_s, g["w_r"], g["wg"], g["wu"], g["wd"], g["s_wg"], g["s_wu"],
                              g["s_wd"])
        st_ids = {}
        orig = layer.dispatch

        def dispatch(x):  # keep the routing for the oracle check
            s = orig(x)
            st_ids["st"] = s
            return s
        layer.dispatch = dispatch
        y = layer.forward(g["x"], ep.TorchExchange())
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    _no_device_errors(moe)
    _check_rank(inp, 0, T, y, st_ids["st"])
