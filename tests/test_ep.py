"""Expert parallelism without a GPU: the exchange logic of
sparse_moe_layer_top_b200.ep run as gloo ranks on CPU, its stage calls computed
by the oracle (tests/ep_cpu_ops.py).  Every rank's output must equal the
single-process oracle block over that rank's tokens with all E experts."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
for p in (ROOT, HERE):
    if p not in sys.path:
        sys.path.insert(0, p)

import moe_inputs  # noqa: E402
from sparse_moe_layer_top_b200 import ep  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


# d, E, k, I, I_s: small enough for the float64 oracle, ragged token counts per rank
SHAPE = dict(d=64, E=8, k=3, I=32, I_s=32)
# E4M3 weights: d, I and I_s span whole 128 x 128 scale blocks
SHAPE_FP8 = dict(d=256, E=8, k=3, I=128, I_s=128)


def _rank_tokens(rank, tokens):
    return tokens[rank] if rank < len(tokens) else 0


def _single_process(ops, prob, x, inp):
    """The same stage calls on one process over all E experts."""
    ids, tw = ops.router_topk(prob, x, inp.w_r, inp.bias)
    pm = ops.permute(prob, x, ids, tw)
    yp = ops.expert_ffn(prob, pm["x_perm"], pm["offs"], inp.wg, inp.wu, inp.wd, inp.s_wg, inp.s_wu, inp.s_wd,
                        scales=inp.scales)
    return ops.combine(prob, yp, pm["pos"], tw, pm["offs"])


def _rank(rank, world, port, tokens, I_s, q, w="f32", bias=None):
    import datetime
    import torch.distributed as dist
    import ep_cpu_ops
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        c = dict(SHAPE_FP8 if w == "fp8" else SHAPE, I_s=I_s)
        act = "bf16" if w == "fp8" else w
        T = _rank_tokens(rank, tokens)
        inp = moe_inputs.make_inputs(max(T, 1), c["d"], c["E"], c["k"], c["I"], c["I_s"], act=act, w=w,
                                     bias=bias, seed=3, x_seed=100 + rank, shared=I_s > 0)
        x = inp.x[:T].contiguous()
        wg, wu, wd = ep.split_experts(rank, world, inp.wg, inp.wu, inp.wd)
        sc = None if w != "fp8" else ep.split_scales(rank, world, c["E"], c["d"], c["I"], c["I_s"], inp.scales)
        layer = ep.EPMoELayer(rank, world, c["d"], c["E"], c["k"], c["I"], c["I_s"], inp.w_r, wg, wu, wd,
                              inp.s_wg, inp.s_wu, inp.s_wd, bias=inp.bias, act=act, w=w, ops=ep_cpu_ops, scales=sc)
        y = layer.forward(x, ep.TorchExchange())
        same = True
        if T:
            ref, _, _, _ = oracle.moe_forward(x, inp.w_r, inp.wg, inp.wu, inp.wd, inp.s_wg, inp.s_wu, inp.s_wd,
                                              c["k"], bias=inp.bias, scales=inp.scales, want_probs=False)
            err = float(np.linalg.norm(y.double().numpy() - ref) / max(np.linalg.norm(ref), 1e-30))
            prob = ep_cpu_ops.Problem.make(T, c["d"], c["E"], c["k"], c["I"], c["I_s"], act, w)
            same = torch.equal(y, _single_process(ep_cpu_ops, prob, x, inp))
        else:
            err = 0.0 if y.shape == (0, c["d"]) else float("inf")
        q.put((rank, err, None if same else "differs from the single-process stage chain"))
    except Exception as e:  # reported to the parent; the other ranks time out on their collectives
        q.put((rank, float("inf"), repr(e)))
    finally:
        dist.destroy_process_group()


def _run(world, tokens, I_s=32, w="f32", tol=2e-6, bias=None):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, tokens, I_s, q, w, bias)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    for rank, err, msg in got:
        assert msg is None, "rank %d: %s" % (rank, msg)
        # values rounded to the activation type at every stage boundary against the float64 oracle
        assert err < tol, "rank %d: rel-L2 %.3g" % (rank, err)
    for p in procs:
        assert p.exitcode == 0


@pytest.mark.parametrize("world,tokens", [(2, [37, 50]), (4, [20, 1, 33, 9])])
def test_expert_parallel_ranks_match_the_whole_block(world, tokens):
    _run(world, tokens)


def test_expert_parallel_rank_without_tokens_and_no_shared_expert():
    _run(2, [0, 41], I_s=0)


def test_expert_parallel_with_a_skewed_router_bias():
    # the replicated router adds the Zipf bias on every rank: most rows go to
    # the low experts, all held by rank 0
    _run(2, [44, 29], bias="zipf")


@pytest.mark.parametrize("world,tokens,I_s", [(2, [30, 45], 128), (4, [12, 0, 25, 7], 0)])
def test_expert_parallel_e4m3_weights(world, tokens, I_s):
    # bf16 activations between stages: the E4M3 tolerance against the oracle,
    # and bit for bit the single-process stage chain
    _run(world, tokens, I_s=I_s, w="fp8", tol=2e-2)


def test_split_scales_takes_the_rank_block_of_each_matrix():
    E, d, I, I_s, world = 4, 256, 384, 128, 2
    per = (I // 128) * (d // 128)                     # 6 blocks per expert matrix
    n_sh = 3 * (I_s // 128) * (d // 128)              # shared gate, up, down: 2 blocks each
    sc = torch.arange(3 * E * per + n_sh, dtype=torch.float32)
    r1 = ep.split_scales(1, world, E, d, I, I_s, sc)
    gate, up, down = (sc[m * E * per:(m + 1) * E * per] for m in range(3))
    want = torch.cat([gate[2 * per:4 * per], up[2 * per:4 * per], down[2 * per:4 * per], sc[3 * E * per:]])
    assert torch.equal(r1, want)
    assert r1.numel() == 3 * 2 * per + n_sh
    with pytest.raises(ValueError):
        ep.split_scales(0, world, E, d, I, I_s, sc[:-1])


def test_rejects_expert_counts_that_do_not_split():
    w = torch.zeros(3, 4, 8)
    ep.EPMoELayer(0, 2, 8, 6, 2, 4, 0, torch.zeros(6, 8), w, w, w)  # 6 experts, 3 per rank
    with pytest.raises(ValueError):
        ep.EPMoELayer(0, 3, 8, 6, 2, 4, 0, torch.zeros(6, 8), w, w, w)  # 2 per rank, but 3 given
    with pytest.raises(ValueError):
        ep.EPMoELayer(0, 4, 8, 6, 2, 4, 0, torch.zeros(6, 8), w, w, w)  # 6 experts do not split over 4
    with pytest.raises(ValueError):
        ep.EPMoELayer(2, 2, 8, 6, 2, 4, 0, torch.zeros(6, 8), w, w, w)  # rank out of range
    q = torch.zeros(3, 128, 128).to(torch.float8_e4m3fn)
    ep.EPMoELayer(0, 2, 128, 6, 2, 128, 0, torch.zeros(6, 128), q, q, q, w="fp8", scales=torch.ones(9))
    with pytest.raises(ValueError):
        ep.EPMoELayer(0, 2, 128, 6, 2, 128, 0, torch.zeros(6, 128), q, q, q, w="fp8")  # no scales
    with pytest.raises(ValueError):
        ep.EPMoELayer(0, 2, 128, 6, 2, 128, 0, torch.zeros(6, 128), q, q, q, w="fp8", scales=torch.ones(18))
    with pytest.raises(ValueError):
        ep.EPMoELayer(0, 2, 8, 6, 2, 4, 0, torch.zeros(6, 8), w, w, w, scales=torch.ones(3))  # not E4M3


def test_split_experts_takes_the_rank_block():
    wg = torch.arange(8 * 2 * 3, dtype=torch.float32).reshape(8, 2, 3)
    a, b, c = ep.split_experts(1, 4, wg, wg + 1, wg + 2)
    assert torch.equal(a, wg[2:4]) and torch.equal(b, wg[2:4] + 1) and torch.equal(c, wg[2:4] + 2)
