#!/usr/bin/env python
"""Throughput of the sparse MoE block on B200 (tokens/s), one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

A step is one full forward of the block (router + top-k, dispatch, gate/up
GEMM with SwiGLU, down GEMM with the weighted combine, shared expert) over one
batch of T synthetic tokens resident in HBM.  With N > 1 (torchrun, one
process per GPU) every rank runs its own batch against its own copy of the
weights -- the block needs no exchange between batches -- so the scaling is
weak and no collective touches the data path; the step time is the maximum
over ranks.

`--impl reference` times the float64 CPU oracle on this machine's cores
instead (the reference arm): same workload, metric and unit, each step a
bounded sample of the batch's tokens.
"""
import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s at 1 B200; % HBM roofline (decode) / % bf16 TC peak (prefill)"
UNIT = "tokens/s"
DEFAULT_CONFIG = "qwen38max_prefill_zipf_bf16"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FLUSH_BYTES = 256 << 20
# Expert weights the oracle may receive on the host for the CPU baseline; a
# workload whose weights exceed it is timed on a token sample whose experts fit.
HOST_WEIGHT_BUDGET = 12 << 30
# A workload whose weights are those of another (same shapes and seed) also
# times that one in the same run, on the same resident weights: the metric's
# two regimes of the 3.8-Max-shaped block, prefill (tensor-bound) and decode
# (weight-streaming).
COMPANION = {"qwen38max_prefill_zipf_bf16": "qwen38max_decode_bf16"}
# The files that define each timed kernel (its template, the PTX wrappers it
# uses, its launch configuration): an ncu traffic figure stays valid while
# their contents hash to the value recorded with it.
KERNEL_SOURCES = {
    "gemm_tc_swiglu": ("tc_gemm.cuh", "ptx.cuh", "common.cuh", "api.cu"),
    "gemm_tc_down": ("tc_gemm.cuh", "ptx.cuh", "common.cuh", "api.cu"),
}
ALL_SOURCES = ("api.cu", "common.cuh", "permute.cuh", "ptx.cuh", "router.cuh", "simt.cuh", "tc_gemm.cuh",
               "tc_swap.cuh", "tc_swap8.cuh", "tc_pair.cuh")


# ---------------------------------------------------------------- helpers
def kernel_source_sha(files=ALL_SOURCES):
    h = hashlib.sha256()
    d = os.path.join(ROOT, "sparse_moe_layer_top_b200", "csrc")
    for f in files:
        with open(os.path.join(d, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def load_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if it still matches the kernel source."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        for e in d.get("entries", []):
            files = tuple(e.get("sources", ALL_SOURCES))
            if e["kernel"] == kernel and e["workload"] == workload and e["source_sha"] == kernel_source_sha(files):
                return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi clock/throttle samples every 200 ms while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="moe_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.Q,
                                          "--format=csv,noheader,nounits", "-lms", "200", "-f", self.path],
                                         stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    c = [x.strip() for x in line.split(",")]
                    if len(c) >= 9:
                        rows.append(c)
            os.unlink(self.path)
        except Exception:
            pass
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        loaded = [s for s in sm if s > 0.5 * (max(mx) if mx else 1)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def routing(moe, layer, x):
    """(topk_ids [T,k] on the device, rows per expert) from the block's own
    router, outside the timed region."""
    import torch
    prob = layer.problem(x.shape[0])
    w_router, bias = layer.w[0], layer.w[1]
    ids, _ = moe.router_topk(prob, x, w_router, bias)
    cnt = torch.bincount(ids.reshape(-1).long(), minlength=prob.E).cpu().tolist()
    return ids, cnt


def forward_plan(c, T):
    """The fused forward's kernel choices for workload c under the current
    path, as the library decides them (moe_forward_plan, host only)."""
    import sparse_moe_layer_top_b200 as moe
    prob = moe.Problem.make(T, c["d"], c["E"], c["k"], c["I"], c["I_s"], c["act"], c["w"])
    return moe.forward_plan(prob)


def gathers_rows(c, T):
    """Whether the fused forward's gate/up GEMM reads its rows straight from the
    token matrix."""
    return forward_plan(c, T)["gathered"]


def work_model(c, counts, T):
    """Algorithmic bytes and flops of the block and of its two expert GEMMs.

    Weights are counted for the experts that received at least one row (and
    the shared expert); each kernel's activations once in and once out (the
    gate/up GEMM reads the dispatched rows -- or, where it gathers them, the
    token matrix itself -- and writes H; the down GEMM reads H and writes the
    weighted (token, slot) rows).  For the whole block only the weights, W_r,
    x and y count: the dispatch copy, H and the slot rows are overheads."""
    d, E, k, I, I_s = c["d"], c["E"], c["k"], c["I"], c["I_s"]
    ab = 4 if c["act"] == "f32" else 2
    wb = {"f32": 4, "bf16": 2, "fp8": 1}[c["w"]]
    active = sum(1 for n in counts if n > 0)
    R = sum(counts)
    sh = 1 if I_s > 0 else 0
    w_gu = (active * 2 * d * I + sh * 2 * d * I_s) * wb
    w_dn = (active * d * I + sh * d * I_s) * wb
    h_bytes = (R * I + sh * T * I_s) * ab
    a_in = (T if gathers_rows(c, T) else R + sh * T) * d * ab
    g1 = {"bytes": w_gu + a_in + h_bytes, "flops": 4 * d * (R * I + sh * T * I_s)}
    g2 = {"bytes": w_dn + h_bytes + (R + sh * T) * d * ab, "flops": 2 * d * (R * I + sh * T * I_s)}
    layer = {"bytes": w_gu + w_dn + E * d * ab + 2 * T * d * ab,
             "flops": 2 * T * d * E + 6 * d * (R * I + sh * T * I_s)}
    if c["w"] == "fp8":
        n_sc = (E * 3 * (I // 128) * (d // 128) + sh * 3 * (I_s // 128) * (d // 128)) * 4
        layer["bytes"] += n_sc * active // max(E, 1)
    loads = sorted(n for n in counts if n > 0)
    load = {"max": loads[-1] if loads else 0, "median": loads[len(loads) // 2] if loads else 0,
            "min": loads[0] if loads else 0}
    return {"active_experts": active, "rows": R, "expert_rows": load, "gemm_gate_up": g1, "gemm_down": g2,
            "layer": layer}


# ---------------------------------------------------------------- CPU oracle timing
def oracle_sample_time(inp_cpu_fn, n_tokens):
    """Seconds the oracle takes for the first n tokens (full weights on the host)."""
    import oracle
    c = inp_cpu_fn()
    x = c["x"][:n_tokens]
    t0 = time.perf_counter()
    oracle.moe_forward(x, c["w_r"], c["wg"], c["wu"], c["wd"], c["s_wg"], c["s_wu"], c["s_wd"], c["k"],
                       bias=c["bias"], scales=c["scales"], want_probs=False)
    return time.perf_counter() - t0


def host_copy(inp):
    out = {}
    for n in ("x", "w_r", "bias", "wg", "wu", "wd", "s_wg", "s_wu", "s_wd", "scales"):
        t = getattr(inp, n)
        out[n] = None if t is None else t.detach().cpu()
    out["k"] = inp.k
    return out


def weight_bytes(inp):
    return sum(getattr(inp, n).numel() * getattr(inp, n).element_size()
               for n in ("wg", "wu", "wd") if getattr(inp, n) is not None)


def sample_tokens(ids, T, n_max):
    """Token order of a sample: a token of the hottest expert, one of the
    coldest active expert, then tokens spread evenly over the batch (so that
    every 128-token tile of it is represented once n is large enough)."""
    import torch
    flat = ids.reshape(-1).long()
    cnt = torch.bincount(flat)
    hot = int(cnt.argmax())
    act = torch.nonzero(cnt > 0).flatten()
    cold = int(act[cnt[act].argmin()])
    first = [int(torch.nonzero((ids == hot).any(1)).flatten()[0]),
             int(torch.nonzero((ids == cold).any(1)).flatten()[-1])]
    n = min(T, n_max)
    spread = [(i * T) // n + (T // n) // 2 for i in range(n)]
    out = []
    for t in first + spread:
        if t not in out:
            out.append(t)
    return out


def compact_experts(inp, experts):
    """Host copies of only the given routed experts (E4M3 as raw codes), and
    the packed E4M3 scales restricted to them."""
    import torch
    sel = torch.as_tensor(experts, device=inp.wg.device, dtype=torch.long)

    def pick(t):
        if t.dtype == torch.float8_e4m3fn:
            t = t.view(torch.uint8)
        return t[sel].cpu()

    out = {"wg": pick(inp.wg), "wu": pick(inp.wu), "wd": pick(inp.wd), "scales": None}
    if inp.w == "fp8":
        E, gd, gi = inp.E, inp.d // 128, inp.I // 128
        n = E * gi * gd
        sc = inp.scales
        parts = [sc[:n].view(E, -1)[sel], sc[n:2 * n].view(E, -1)[sel], sc[2 * n:3 * n].view(E, -1)[sel], sc[3 * n:]]
        out["scales"] = torch.cat([p.reshape(-1) for p in parts]).cpu()
    return out


def cpu_baseline_compact(inp, ids, target_s=15.0, n_max=256, budget=HOST_WEIGHT_BUDGET):
    """The oracle on a token sample of a batch whose weights do not fit the
    host budget: the sample's tokens (hottest and coldest experts' first) are
    added while the experts they use fit the budget; the oracle gets host
    copies of those experts only.  Timed: its router over all E experts, then
    the block over the compact expert list with each token's experts forced
    to the ones the device's router chose (the renormalised weights over a
    token's kept experts do not depend on the other experts)."""
    import numpy as np
    import oracle
    T, k = inp.T, inp.k
    per_expert = weight_bytes(inp) // inp.E
    max_experts = max(k, budget // max(per_expert, 1))
    ids_h = ids.cpu()
    toks, used = [], set()
    for t in sample_tokens(ids, T, n_max):
        s = set(ids_h[t].tolist())
        if len(used | s) > max_experts:
            continue
        toks.append(t)
        used |= s
        if len(toks) == n_max:
            break
    experts = sorted(used)
    remap = {e: i for i, e in enumerate(experts)}
    w = compact_experts(inp, experts)
    x_all = inp.x[toks].cpu()
    w_r = inp.w_r.cpu()
    bias = inp.bias.cpu() if inp.bias is not None else None
    force = np.vectorize(remap.get)(ids_h[toks].numpy()).astype(np.int32)
    sh = [None if t is None else t.cpu() for t in (inp.s_wg, inp.s_wu, inp.s_wd)]

    def run(n):
        t0 = time.perf_counter()
        oracle.router(x_all[:n], w_r, k, bias=bias)
        oracle.moe_forward(x_all[:n], w_r[experts], w["wg"], w["wu"], w["wd"], sh[0], sh[1], sh[2], k,
                           bias=None if bias is None else bias[experts], scales=w["scales"],
                           force_ids=force[:n], want_probs=False)
        return time.perf_counter() - t0

    probe = min(8, len(toks))
    t_probe = run(probe)
    n = int(min(len(toks), max(probe, target_s * probe / max(t_probe, 1e-6))))
    # the sample may be cut short by the host budget: it is then run again
    # until about target_s of work has been timed
    t, reps = run(n), 1
    while t < 0.5 * target_s and reps < 8:
        t += run(n)
        reps += 1
    return {"value": n * reps / t, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "%d of %d tokens of the batch (a token of the hottest and of the coldest active expert, then "
                      "tokens spread over the batch) x %d runs, float64 router over all %d experts and the block on "
                      "host copies of the %d experts those tokens use (%.1f GB), %.1f s"
                      % (n, T, reps, inp.E, len(experts), len(experts) * per_expert / 1e9, t)}


def cpu_baseline(inp, ids, target_s=15.0):
    """The oracle, as it stands, on a bounded token sample of the batch."""
    import oracle
    if weight_bytes(inp) > (8 << 30):
        return cpu_baseline_compact(inp, ids, target_s)
    host = host_copy(inp)
    probe = 16
    t_probe = oracle_sample_time(lambda: host, probe)
    n = int(max(probe, min(inp.T, target_s * probe / max(t_probe, 1e-6))))
    n = max(probe, n - n % 8)
    t = oracle_sample_time(lambda: host, n)
    return {"value": n / t, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "first %d of %d tokens of the batch, full block in float64 (%.1f s)" % (n, inp.T, t)}


# ---------------------------------------------------------------- distributed plumbing
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def aggregate(step_ms, tokens, world, device=None):
    """(max step ms over ranks, total tokens over ranks); plain values when alone."""
    if world <= 1:
        return step_ms, tokens
    import torch
    import torch.distributed as dist
    t = torch.tensor([step_ms], dtype=torch.float64, device=device)
    n = torch.tensor([float(tokens)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(n, op=dist.ReduceOp.SUM)
    return float(t.item()), int(n.item())


def barrier(world, device=None):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


E2E_MIN_STEPS = 50


def e2e_pipelined(layer, x, y, K, dev):
    import torch
    xh = [x.cpu().pin_memory() for _ in range(2)]
    yh = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(2)]
    xd = [torch.empty_like(x) for _ in range(2)]
    yd = [torch.empty_like(y) for _ in range(2)]
    s_in, s_run, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev = lambda: torch.cuda.Event()  # noqa: E731
    ran = [ev(), ev()]
    copied_out = [ev(), ev()]
    for b in range(2):  # the buffers start free
        ran[b].record(s_run)
        copied_out[b].record(s_out)

    def step(i):
        b = i % 2
        arrived = ev()
        with torch.cuda.stream(s_in):
            s_in.wait_event(ran[b])                  # x buffer b no longer read
            xd[b].copy_(xh[b], non_blocking=True)
            arrived.record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(arrived)
            s_run.wait_event(copied_out[b])          # y buffer b already copied out
            layer(xd[b], yd[b], stream=s_run)
            ran[b].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ran[b])
            yh[b].copy_(yd[b], non_blocking=True)
            copied_out[b].record(s_out)

    for i in range(4):
        step(i)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    for i in range(K):
        step(i)
    s_in.wait_stream(s_out)
    t1.record(s_in)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1) / K


# ---------------------------------------------------------------- our arm
def check_status(moe, when):
    s, detail = moe.device_status()
    if s != 0:
        raise RuntimeError("device status %d (0x%08x) %s" % (s, detail & 0xffffffff, when))


def time_steps(moe, layer, x, y, K, W, flush, world, dev, clocks=None):
    """W warm-up forwards, then K timed ones (CUDA events on the launching
    stream, L2 flushed before each outside the events) -> (mean step ms, mean
    ms per tensor-core GEMM kernel, launches per step, clock record)."""
    import torch
    for _ in range(W):
        layer(x, y)
    torch.cuda.synchronize()
    check_status(moe, "after warm-up")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    barrier(world, dev)
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.start()
    moe.profile_enable(2)  # events around the tensor-core GEMMs only
    for i in range(K):
        flush.zero_()
        ev[i][0].record()
        layer(x, y)
        ev[i][1].record()
    torch.cuda.synchronize()
    barrier(world, dev)
    launches_per_step = moe.last_launch_count()
    prof = moe.profile_read()
    moe.profile_enable(0)
    clk = clocks.stop() if clocks is not None else None
    check_status(moe, "after the timed steps")
    per = {}
    for name, ms in prof:
        per.setdefault(name, []).append(ms)
    # per step: a stage may run as more than one launch (the split form runs
    # each projection as a pair-tile and a weight-row launch)
    kern = {n: sum(v) / K for n, v in per.items()}
    # and per launch of a step, in launch order (every step launches the same sequence)
    n = len(prof) // K if K else 0
    if n and n * K == len(prof):
        kern["launches"] = [[prof[j][0], statistics.mean(prof[i * n + j][1] for i in range(K))] for j in range(n)]
    return statistics.mean(a.elapsed_time(b) for a, b in ev), kern, launches_per_step, clk


def kernel_roofline(work, kern, peaks, peak_src, workload):
    """Roofline of the dominant expert GEMM: its algorithmic bytes or flops
    over its live CUDA-event time, against the measured copy bandwidth (HBM
    bound) or the measured dense bf16 GEMM burst figure (tensor bound; the
    fraction of the sustained figure is given beside it)."""
    gemms = {"gemm_tc_swiglu": work["gemm_gate_up"], "gemm_tc_down": work["gemm_down"]}
    dom = max((n for n in gemms if n in kern), key=lambda n: kern[n], default=None)
    if dom is None:
        return None
    wk = gemms[dom]
    t_s = kern[dom] / 1e3
    hbm_t = wk["bytes"] / (peaks["hbm_gbs"] * 1e9)
    tc_t = wk["flops"] / (peaks["bf16_tflops"] * 1e12)
    if hbm_t >= tc_t:
        roof = {"bound": "hbm", "achieved": wk["bytes"] / t_s / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
        which = " copy bandwidth"
    else:
        burst, sust = peaks["bf16_tflops"], peaks["bf16_tflops_sustained"]
        ach = wk["flops"] / t_s / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": burst, "unit": "TFLOP/s", "frac_sustained": ach / sust}
        which = " bf16 dense GEMM, burst"
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = load_traffic(dom, workload)
    roof.update({"kernel": dom, "kernel_ms": kern[dom], "algorithmic_bytes": wk["bytes"],
                 "algorithmic_flops": wk["flops"], "peak_source": peak_src + which})
    return roof


def layer_roofline(work, step_ms, peaks, peak_src):
    lw = work["layer"]
    st = step_ms / 1e3
    return {"bytes": lw["bytes"], "flops": lw["flops"],
            "hbm_frac": lw["bytes"] / st / 1e9 / peaks["hbm_gbs"],
            "tc_frac": lw["flops"] / st / 1e12 / peaks["bf16_tflops"],
            "achieved_gbs": lw["bytes"] / st / 1e9, "achieved_tflops": lw["flops"] / st / 1e12,
            "active_experts": work["active_experts"], "expert_rows": work["expert_rows"],
            "peak_source": peak_src + " (tensor: burst)"}


def run_companion(args, moe, inp, flush, world, rank, dev, peaks, peak_src):
    """The companion workload on the same resident weights (its own tokens,
    its own router bias): step time, roofline and CPU baseline."""
    import moe_inputs
    import torch
    name = COMPANION[args.config]
    c = dict(moe_inputs.CONFIGS[name])
    T = c["T"]
    x = moe_inputs.randn((T, c["d"]), dev, rank, moe_inputs.X, 1.0, inp.x.dtype)
    bias = moe_inputs.zipf_bias(c["E"], dev) if c["bias"] == "zipf" else None
    layer = moe.MoELayer(inp.d, inp.E, inp.k, inp.I, inp.I_s, inp.w_r, inp.wg, inp.wu, inp.wd, inp.s_wg, inp.s_wu,
                         inp.s_wd, bias=bias, scales=inp.scales, act=inp.act, w=inp.w, max_tokens=T)
    y = torch.empty((T, c["d"]), dtype=x.dtype, device=dev)
    ids, counts = routing(moe, layer, x)
    work = work_model(c, counts, T)
    step_ms, kern, lps, _ = time_steps(moe, layer, x, y, args.steps, args.warmup, flush, world, dev)
    ms_max, tokens_all = aggregate(step_ms, T, world, dev)
    if rank != 0:
        return None
    out = {"workload": name, "value": tokens_all / (ms_max / 1e3), "unit": UNIT, "ms_per_step": ms_max,
           "T": T, "router_bias": c["bias"], "roofline": kernel_roofline(work, kern, peaks, peak_src, name),
           "layer_roofline": layer_roofline(work, ms_max, peaks, peak_src), "kernel_ms": kern,
           "launches_per_step": lps, "cpu_baseline": None}
    if world == 1 and not args.no_cpu_baseline:
        import moe_inputs as mi
        sub = mi.MoEInputs(T, inp.d, inp.E, inp.k, inp.I, inp.I_s, inp.act, inp.w, x=x, w_r=inp.w_r, bias=bias,
                           wg=inp.wg, wu=inp.wu, wd=inp.wd, s_wg=inp.s_wg, s_wu=inp.s_wu, s_wd=inp.s_wd,
                           scales=inp.scales)
        out["cpu_baseline"] = cpu_baseline(sub, ids, args.cpu_seconds)
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist

    import moe_inputs
    import sparse_moe_layer_top_b200 as moe

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=300))

    cfg = dict(moe_inputs.CONFIGS[args.config])
    inp = moe_inputs.make_config(args.config, seed=0, device=dev, x_seed=rank)
    T = inp.T
    moe.set_path(args.path)
    layer = moe.MoELayer.from_inputs(inp, max_tokens=T)
    x = inp.x
    y = torch.empty((T, inp.d), dtype=x.dtype, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    ids, counts = routing(moe, layer, x)
    work = work_model(cfg, counts, T)

    K = args.steps
    clocks = ClockSampler(local)
    step_ms, kern, launches_per_step, clk = time_steps(moe, layer, x, y, K, args.warmup, flush, world, dev, clocks)
    ms_max, tokens_all = aggregate(step_ms, T, world, dev)

    # End to end through the public API: every step copies its batch from
    # pinned host memory and its result back.  Steps are pipelined over three
    # streams with two buffers each, as a serving loop would run them: the
    # host->device copy of step i+1 and the device->host copy of step i-1
    # overlap the forward of step i.  Per-step time = whole timed region / K,
    # over at least E2E_MIN_STEPS steps, so that filling and draining the
    # pipeline (one step's copy in, one step's copy out) is spread as in a
    # serving loop.  Steps run back to back, with no L2 flush between them.
    K_e2e = max(K, E2E_MIN_STEPS)
    e2e_ms = e2e_pipelined(layer, x, y, K_e2e, dev)
    e2e_max, _ = aggregate(e2e_ms, T, world, dev)
    check_status(moe, "after the end-to-end steps")

    peaks, peak_src = load_peaks()
    regimes = {}
    if args.config in COMPANION and not args.no_companion:
        comp = run_companion(args, moe, inp, flush, world, rank, dev, peaks, peak_src)
        if comp is not None:
            regimes[comp["workload"]] = comp
    line = None
    if rank == 0:
        roof = kernel_roofline(work, kern, peaks, peak_src, args.config)
        layer_roof = layer_roofline(work, ms_max, peaks, peak_src)
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = cpu_baseline(inp, ids, args.cpu_seconds)
        resident = x.numel() * x.element_size() + y.numel() * y.element_size() + weight_bytes(inp)
        line = {
            "metric": METRIC, "value": tokens_all / (ms_max / 1e3), "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": cfg["act"], "data": "synthetic (seeded N(0,1) tokens, N(0,0.02^2) weights)",
            "config": {"workload": args.config, "T": T, "d": cfg["d"], "E": cfg["E"], "k": cfg["k"], "I": cfg["I"],
                       "I_s": cfg["I_s"], "act": cfg["act"], "weights": cfg["w"],
                       "router_bias": cfg["bias"], "global_tokens": tokens_all,
                       "parallelism": "dp%d (independent token batches per GPU, weights replicated)" % world,
                       "l2": "flushed between timed steps (256 MiB write outside the events)"},
            "roofline": roof, "layer_roofline": layer_roof, "cpu_baseline": cpu,
            "e2e": {"value": tokens_all / (e2e_max / 1e3), "unit": UNIT,
                    "h2d_bytes_per_step": x.numel() * x.element_size(),
                    "d2h_bytes_per_step": y.numel() * y.element_size(), "ms_per_step": e2e_max, "steps": K_e2e,
                    "pipelining": "host->device copy of step i+1 and device->host copy of step i-1 "
                                  "overlap the forward of step i (3 streams, 2 buffers)",
                    "l2": "no flush between steps; the step reads %.1f GB (tokens, result, weights) against "
                          "126 MB of L2" % (resident / 1e9)},
            "gpu_launches": launches_per_step * K, "launches_per_step": launches_per_step,
            "kernel_ms": kern, "expert_form": forward_plan(cfg, T)["expert_form"], "clocks": clk, "impl": "ours",
        }
        if regimes:
            line["regimes"] = regimes
    if world > 1:
        dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- reference arm
def oracle_routed_time(inp, toks, w_r, bias, budget=HOST_WEIGHT_BUDGET):
    """Seconds the oracle takes for the block on tokens `toks` of a batch
    whose weights stay on the device: its router over all E experts picks
    each token's experts, host copies of only those experts are made
    (untimed), and the block runs on them with the router's choice forced.
    Tokens whose experts would pass the host budget go in further batches."""
    import numpy as np
    import oracle
    x = inp.x[toks].cpu()
    k = inp.k
    t0 = time.perf_counter()
    _, ids, _ = oracle.router(x, w_r, k, bias=bias)
    secs = time.perf_counter() - t0
    per_expert = weight_bytes(inp) // inp.E
    max_experts = max(k, budget // max(per_expert, 1))
    sh = [None if t is None else t.cpu() for t in (inp.s_wg, inp.s_wu, inp.s_wd)]
    i = 0
    while i < len(toks):
        used, j = set(), i
        while j < len(toks) and (j == i or len(used | set(ids[j].tolist())) <= max_experts):
            used |= set(ids[j].tolist())
            j += 1
        experts = sorted(used)
        remap = {e: n for n, e in enumerate(experts)}
        w = compact_experts(inp, experts)
        force = np.vectorize(remap.get)(ids[i:j]).astype(np.int32)
        t0 = time.perf_counter()
        oracle.moe_forward(x[i:j], w_r[experts], w["wg"], w["wu"], w["wd"], sh[0], sh[1], sh[2], k,
                           bias=None if bias is None else bias[experts], scales=w["scales"], force_ids=force,
                           want_probs=False)
        secs += time.perf_counter() - t0
        del w
        i = j
    return secs


def run_reference(args):
    """The float64 oracle on the host cores, on a bounded sample per step.
    Workloads whose weights pass the host budget keep them on the device and
    give the oracle host copies of the experts each step's tokens use, chosen
    by the oracle's own router."""
    world, rank, local = dist_env()
    if rank != 0:
        return
    import torch

    import moe_inputs
    import oracle

    cfg = dict(moe_inputs.CONFIGS[args.config])
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    inp = moe_inputs.make_config(args.config, seed=0, device=dev)
    big = weight_bytes(inp) > (8 << 30)
    host = None if big else host_copy(inp)
    w_r = inp.w_r.cpu()
    bias = inp.bias.cpu() if inp.bias is not None else None
    per_step = args.ref_tokens
    samples = []
    for i in range(args.warmup + args.steps):
        lo = (i * per_step) % max(inp.T - per_step + 1, 1)
        if big:
            dt = oracle_routed_time(inp, list(range(lo, min(inp.T, lo + per_step))), w_r, bias)
        else:
            x = host["x"][lo:lo + per_step]
            t0 = time.perf_counter()
            oracle.moe_forward(x, host["w_r"], host["wg"], host["wu"], host["wd"], host["s_wg"], host["s_wu"],
                               host["s_wd"], host["k"], bias=host["bias"], scales=host["scales"], want_probs=False)
            dt = time.perf_counter() - t0
        if i >= args.warmup:
            samples.append(dt)
    ms = statistics.mean(samples) * 1e3
    n_step = min(per_step, inp.T)
    value = n_step / (ms / 1e3)
    sample = "%d tokens of the %d-token batch per step, full block in float64" % (n_step, inp.T)
    if big:
        sample += (" (router over all %d experts; the block on host copies of the experts those tokens use, "
                   "copied outside the timed region)" % inp.E)
    print(json.dumps({
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1) tokens, N(0,0.02^2) weights)",
        "config": {"workload": args.config, "T": inp.T, "d": cfg["d"], "E": cfg["E"], "k": cfg["k"],
                   "I": cfg["I"], "I_s": cfg["I_s"], "act": cfg["act"], "weights": cfg["w"],
                   "router_bias": cfg["bias"], "tokens_per_step": n_step},
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def arg_parser():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    import moe_inputs
    ap.add_argument("--config", choices=sorted(moe_inputs.CONFIGS), default=DEFAULT_CONFIG)
    ap.add_argument("--path", type=int, default=0,
                    help="expert-GEMM form (moe_set_path): 0 automatic, 2 row-tiled, 3 weight-row, 4 CTA pairs, "
                         "5 split")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-companion", action="store_true",
                    help="do not also time the workload that shares this one's weights (decode beside prefill)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-tokens", type=int, default=32)
    return ap


def main(argv=None):
    ap = arg_parser()
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world, _, _ = dist_env()
    if world != args.gpus and not (world == 1 and args.gpus == 1):
        if world == 1 and args.gpus > 1:
            ap.error("--gpus %d needs torchrun with %d processes" % (args.gpus, args.gpus))
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
