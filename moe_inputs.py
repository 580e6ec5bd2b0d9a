"""Seeded synthetic inputs for the sparse MoE block.

The one module that both the CUDA path's tests/benchmark and the float64
oracle take their inputs from.  It draws random numbers and lays them out; it
holds none of the block's arithmetic (no routing, no softmax, no expert math).

Recipe (every tensor has its own generator, seeded from (seed, tensor index)
in the fixed order x, W_r, W_gate, W_up, W_down, shared gate, shared up,
shared down):
  * x ~ N(0, 1); every weight ~ N(0, 0.02^2); drawn in fp32, then rounded to
    the activation type (bf16 or fp32);
  * optional router-logit bias for strongly skewed loads:
    b_e = 2 * ln(1 / rank_e^1.1) = -2.2 * ln(e + 1)  (expert 0 the hottest);
  * FP8 weights: each 128 x 128 block of a bf16 weight matrix is stored as
    E4M3 codes q = RNE(w / s) clamped to +-448 with s = amax(block) / 448
    (s = 1 for an all-zero block); the fp32 scales go into one packed buffer
    (gate [E][I/128][d/128], up (same), down [E][d/128][I/128], then the
    shared expert's three in the same order).

Large weight tensors are drawn expert-chunk by expert-chunk straight on the
target device, so that no full-size fp32 temporary is ever materialised.
"""
from dataclasses import dataclass, field
import math

import torch

# The five workloads.  Shapes follow the Mixture-of-Experts keys of the two
# model families the pages describe (Qwen3.6-35B-A3B: 256 experts, 8 routed +
# 1 shared; Qwen3.8-Max config.json: 512 experts, 10 per token, intermediate
# 2048, shared intermediate 2048, hidden 8192, bf16).
CONFIGS = {
    "tiny_fp32": dict(T=32, d=128, E=16, k=2, I=64, I_s=64, act="f32", w="f32", bias=None),
    "qwen36_35b_a3b_bf16": dict(T=4096, d=2048, E=256, k=8, I=512, I_s=512, act="bf16",
                                w="bf16", bias=None),
    "qwen38max_decode_bf16": dict(T=64, d=8192, E=512, k=10, I=2048, I_s=2048, act="bf16",
                                  w="bf16", bias=None),
    "qwen38max_prefill_zipf_bf16": dict(T=8192, d=8192, E=512, k=10, I=2048, I_s=2048,
                                        act="bf16", w="bf16", bias="zipf"),
    "qwen38max_fp8": dict(T=2048, d=8192, E=512, k=10, I=2048, I_s=2048, act="bf16", w="fp8",
                          bias=None),
}

X, W_R, W_GATE, W_UP, W_DOWN, S_GATE, S_UP, S_DOWN = range(8)
FP8_MAX = 448.0
BLK = 128


@dataclass
class MoEInputs:
    T: int
    d: int
    E: int
    k: int
    I: int
    I_s: int
    act: str
    w: str
    x: torch.Tensor = None
    w_r: torch.Tensor = None
    bias: torch.Tensor = None
    wg: torch.Tensor = None
    wu: torch.Tensor = None
    wd: torch.Tensor = None
    s_wg: torch.Tensor = None
    s_wu: torch.Tensor = None
    s_wd: torch.Tensor = None
    scales: torch.Tensor = None
    extra: dict = field(default_factory=dict)

    def shape_tuple(self):
        return (self.T, self.d, self.E, self.k, self.I, self.I_s)


def _gen(device, seed, idx):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1000003 + idx)
    return g


def _act_dtype(act):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[act]


def randn(shape, device, seed, idx, std=1.0, dtype=torch.float32, chunk_rows=None):
    """N(0, std^2) drawn in fp32, rounded to dtype; chunked along dim 0."""
    g = _gen(device, seed, idx)
    out = torch.empty(shape, dtype=dtype, device=device)
    n0 = shape[0]
    step = chunk_rows or n0
    for a in range(0, n0, step):
        b = min(n0, a + step)
        t = torch.randn((b - a,) + tuple(shape[1:]), generator=g, device=device,
                        dtype=torch.float32)
        if std != 1.0:
            t.mul_(std)
        out[a:b].copy_(t)
        del t
    return out


def zipf_bias(E, device):
    """b_e = 2 ln(1/rank_e^1.1) with rank_e = e + 1."""
    r = torch.arange(1, E + 1, dtype=torch.float64)
    return (-2.2 * torch.log(r)).to(torch.float32).to(device)


def quantize_e4m3_blocks(w):
    """[..., R, C] bf16/fp32 -> (E4M3 codes [..., R, C], fp32 scales [..., R/128, C/128])."""
    R, C = w.shape[-2], w.shape[-1]
    assert R % BLK == 0 and C % BLK == 0
    lead = w.shape[:-2]
    wf = w.float().reshape(*lead, R // BLK, BLK, C // BLK, BLK)
    amax = wf.abs().amax(dim=(-3, -1))                       # [..., R/128, C/128]
    s = torch.where(amax > 0, amax / FP8_MAX, torch.ones_like(amax))
    q = (wf / s[..., :, None, :, None]).clamp_(-FP8_MAX, FP8_MAX)
    q = q.reshape(*lead, R, C).to(torch.float8_e4m3fn)
    return q, s.contiguous()


def _weights(shape, device, seed, idx, dt, quant):
    """One routed (3-D) or shared (2-D) weight tensor; for fp8 -> (codes, scales)."""
    if not quant:
        return randn(shape, device, seed, idx, 0.02, dt, chunk_rows=16 if len(shape) == 3 else None), None
    if len(shape) == 2:
        w = randn(shape, device, seed, idx, 0.02, torch.bfloat16)
        return quantize_e4m3_blocks(w)
    E, R, C = shape
    g = _gen(device, seed, idx)
    q = torch.empty(shape, dtype=torch.float8_e4m3fn, device=device)
    s = torch.empty((E, R // BLK, C // BLK), dtype=torch.float32, device=device)
    step = 16
    for a in range(0, E, step):
        b = min(E, a + step)
        t = torch.randn((b - a, R, C), generator=g, device=device, dtype=torch.float32)
        t.mul_(0.02)
        qq, ss = quantize_e4m3_blocks(t.to(torch.bfloat16))
        q[a:b].copy_(qq)
        s[a:b].copy_(ss)
        del t, qq, ss
    return q, s


def make_inputs(T, d, E, k, I, I_s, act="bf16", w="bf16", bias=None, seed=0, device="cpu",
                x_seed=None, shared=True):
    """All inputs of one block.  x_seed (default: seed) re-draws only x, e.g. one
    batch per data-parallel rank with the same weights."""
    adt = _act_dtype(act)
    quant = w == "fp8"
    wdt = adt if not quant else torch.bfloat16
    inp = MoEInputs(T, d, E, k, I, I_s if shared else 0, act, w)
    inp.x = randn((T, d), device, seed if x_seed is None else x_seed, X, 1.0, adt)
    inp.w_r = randn((E, d), device, seed, W_R, 0.02, adt)
    if bias == "zipf":
        inp.bias = zipf_bias(E, device)
    elif isinstance(bias, torch.Tensor):
        inp.bias = bias.to(device=device, dtype=torch.float32)
    inp.wg, sg = _weights((E, I, d), device, seed, W_GATE, wdt, quant)
    inp.wu, su = _weights((E, I, d), device, seed, W_UP, wdt, quant)
    inp.wd, sd = _weights((E, d, I), device, seed, W_DOWN, wdt, quant)
    ssg = ssu = ssd = None
    if shared and I_s > 0:
        inp.s_wg, ssg = _weights((I_s, d), device, seed, S_GATE, wdt, quant)
        inp.s_wu, ssu = _weights((I_s, d), device, seed, S_UP, wdt, quant)
        inp.s_wd, ssd = _weights((d, I_s), device, seed, S_DOWN, wdt, quant)
    if quant:
        parts = [sg, su, sd] + ([ssg, ssu, ssd] if ssg is not None else [])
        inp.scales = torch.cat([p.reshape(-1) for p in parts])
    return inp


def make_config(name, seed=0, device="cpu", T=None, x_seed=None):
    c = dict(CONFIGS[name])
    if T is not None:
        c["T"] = T
    return make_inputs(c["T"], c["d"], c["E"], c["k"], c["I"], c["I_s"], c["act"], c["w"],
                       c["bias"], seed=seed, device=device, x_seed=x_seed)


def random_routing(T, E, k, seed=0, device="cpu"):
    """topk_ids [T,k] int32 (k distinct experts per token, uniformly drawn) and
    topk_w [T,k] fp32 positive weights -- a synthetic router output for
    testing the later stages on their own."""
    g = _gen(device, seed, 100)
    keys = torch.rand((T, E), generator=g, device=device)
    ids = keys.argsort(dim=1)[:, :k].to(torch.int32).contiguous()
    w = torch.rand((T, k), generator=g, device=device) + 0.05
    return ids, w.to(torch.float32).contiguous()


def random_groups(E, rows_per_group, seed=0, device="cpu"):
    """Group sizes for a dispatched-row buffer: a list of E routed sizes; the
    caller appends the shared group.  Returns offs int32 [E+2] given the shared
    group size in rows_per_group[E]."""
    sizes = torch.tensor(rows_per_group, dtype=torch.int64)
    offs = torch.zeros(E + 2, dtype=torch.int64)
    offs[1:] = torch.cumsum(sizes, 0)
    return offs.to(torch.int32).to(device)
