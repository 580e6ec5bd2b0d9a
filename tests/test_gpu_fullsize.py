"""Parity at the full workload sizes, in the launch configuration the
benchmark times (MoELayer over the whole batch).

The oracle cannot redo a whole batch at these sizes, so it recomputes sampled
tokens -- the first and last, a token of the hottest and of the coldest active
expert, and one token in each 128-token row tile (the router's and the
row-tiled GEMMs' tiles), while the experts they use fit a host budget -- from
host copies of only those experts (the renormalised weights over a token's
kept set do not depend on which other experts exist, so a compact expert list
with the set forced gives the same result).  Properties that hold at any size
are checked on every token.
"""
import gc

import numpy as np
import pytest
import torch

import moe_inputs
import oracle
from parity import TOL, TOL_W, check_routing, precision_key, rel_l2

pytestmark = pytest.mark.gpu

WORKLOADS = ["qwen36_35b_a3b_bf16", "qwen38max_decode_bf16", "qwen38max_prefill_zipf_bf16", "qwen38max_fp8"]


def _compact_scales(inp, experts):
    """The packed E4M3 scale buffer restricted to the given routed experts."""
    E, d, I, Is = inp.E, inp.d, inp.I, inp.I_s
    gd, gi, gs = d // 128, I // 128, Is // 128
    sc = inp.scales
    n = E * gi * gd
    idx = torch.as_tensor(experts, device=sc.device, dtype=torch.long)
    parts = [sc[:n].view(E, -1)[idx], sc[n:2 * n].view(E, -1)[idx], sc[2 * n:3 * n].view(E, -1)[idx],
             sc[3 * n:]]
    return torch.cat([p.reshape(-1) for p in parts]).cpu()


def _pick(t, sel):
    """Rows `sel` of a weight tensor, on the host (E4M3 tensors as raw codes)."""
    if t.dtype == torch.float8_e4m3fn:
        t = t.view(torch.uint8)
    return t[sel].cpu()


HOST_BUDGET = 16 << 30  # bytes of expert weights copied to the host for the oracle


def _sample_tokens(ids, T, per_expert_bytes):
    """First, last, hottest- and coldest-expert tokens, then one token at a
    seeded offset in every 128-token row tile, then up to 32 seeded ones, in
    that order, each kept while the union of the kept tokens' experts fits
    HOST_BUDGET (96 tokens at most)."""
    flat = ids.reshape(-1).long()
    cnt = torch.bincount(flat, minlength=int(flat.max()) + 1)
    hot = int(cnt.argmax())
    act = torch.nonzero(cnt > 0).flatten()
    cold = int(act[cnt[act].argmin()])
    tok_hot = int(torch.nonzero((ids == hot).any(1)).flatten()[0])
    tok_cold = int(torch.nonzero((ids == cold).any(1)).flatten()[-1])
    g = torch.Generator().manual_seed(1)
    tiles = [min(T - 1, r0 + int(torch.randint(0, 128, (1,), generator=g))) for r0 in range(0, T, 128)]
    more = torch.randperm(T, generator=g)[:32].tolist()  # a batch of a tile or two: more of its tokens
    ids_h = ids.cpu()
    max_experts = HOST_BUDGET // per_expert_bytes
    keep, used = [], set()
    for t in [0, T - 1, tok_hot, tok_cold] + tiles + more:
        s = set(ids_h[t].tolist())
        if t in keep or len(used | s) > max_experts or len(keep) == 96:
            continue
        keep.append(t)
        used |= s
    return sorted(keep)


@pytest.mark.parametrize("name", WORKLOADS)
def test_full_size_sampled_tokens(name):
    import sparse_moe_layer_top_b200 as moe
    torch.cuda.set_device(0)
    inp = moe_inputs.make_config(name, seed=0, device="cuda")
    T, k, E = inp.T, inp.k, inp.E
    layer = moe.MoELayer.from_inputs(inp, max_tokens=T)
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    tw = torch.empty((T, k), dtype=torch.float32, device="cuda")
    y = layer(inp.x, topk_ids=ids, topk_w=tw)
    torch.cuda.synchronize()
    s, detail = moe.device_status()
    assert s == 0, "device status %d (0x%08x)" % (s, detail & 0xffffffff)

    # properties on every token
    assert torch.isfinite(y.float()).all()
    assert ((ids >= 0) & (ids < E)).all()
    srt = ids.sort(dim=1).values
    assert (srt[:, 1:] != srt[:, :-1]).all(), "repeated expert within a token"
    assert torch.allclose(tw.sum(1), torch.ones(T, device="cuda"), atol=1e-5)
    assert (tw[:, :-1] >= tw[:, 1:] - 1e-7).all(), "weights not in descending order"

    # sampled tokens against the oracle
    per_expert = sum(t[0].numel() * t.element_size() for t in (inp.wg, inp.wu, inp.wd))
    toks = _sample_tokens(ids, T, per_expert)
    # every row tile is represented unless the host budget stopped it
    assert len(toks) >= min(T // 128 + 2, 12), toks
    key = precision_key(inp)
    x_s = inp.x[toks].cpu()
    w_r = inp.w_r.cpu()
    bias = inp.bias.cpu() if inp.bias is not None else None
    probs, ids_or, _ = oracle.router(x_s, w_r, k, bias=bias)
    use, _ = check_routing(ids[toks].cpu().numpy(), tw[toks].cpu().numpy(), probs, ids_or, TOL_W[key])
    experts = sorted(set(use.reshape(-1).tolist()))
    remap = {e: i for i, e in enumerate(experts)}
    force = np.vectorize(remap.get)(use).astype(np.int32)
    sel = torch.tensor(experts, device="cuda", dtype=torch.long)
    y_ref, *_ = oracle.moe_forward(
        x_s, w_r[experts], _pick(inp.wg, sel), _pick(inp.wu, sel), _pick(inp.wd, sel),
        inp.s_wg.cpu(), inp.s_wu.cpu(), inp.s_wd.cpu(), k,
        bias=None if bias is None else bias[experts],
        scales=_compact_scales(inp, experts) if inp.w == "fp8" else None,
        force_ids=force, want_probs=False)
    err = rel_l2(y[toks].float().cpu().numpy(), y_ref)
    assert err <= TOL[key], "%s: rel-L2 %.3g on tokens %s" % (name, err, toks)
    del inp, layer, y, ids, tw
    gc.collect()
    torch.cuda.empty_cache()
