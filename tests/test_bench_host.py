"""bench.py's host-side logic without a GPU: the multi-rank aggregation (two
gloo ranks on CPU), the algorithmic work model, and the reference arm's JSON
line on the tiny workload."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    ms, tokens = bench.aggregate(step_ms=1.5 + rank, tokens=100 * (rank + 1), world=world)
    bench.barrier(world)
    dist.destroy_process_group()
    q.put((rank, ms, tokens))


def test_aggregate_takes_the_slowest_rank_and_sums_tokens():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == [(0, 2.5, 300), (1, 2.5, 300)]


def test_aggregate_alone_is_identity():
    assert bench.aggregate(3.0, 7, 1) == (3.0, 7)


def test_work_model_counts_active_experts_and_rows():
    c = dict(d=2048, E=256, k=8, I=512, I_s=512, act="bf16", w="bf16")
    counts = [128] * 255 + [0]
    w = bench.work_model(c, counts, 4096 * 8 // 8)
    assert w["active_experts"] == 255 and w["rows"] == 128 * 255
    # gate+up weights of 255 experts and the shared expert, bf16
    g1 = w["gemm_gate_up"]
    weights = (255 * 2 * 2048 * 512 + 2 * 2048 * 512) * 2
    assert g1["bytes"] >= weights
    assert g1["flops"] == 4 * 2048 * (128 * 255 * 512 + 4096 * 512)
    lw = w["layer"]
    assert lw["flops"] == 2 * 4096 * 2048 * 256 + 6 * 2048 * (128 * 255 * 512 + 4096 * 512)


def test_gate_up_input_is_the_token_matrix_where_the_gemm_gathers_it():
    c35 = dict(d=2048, E=256, k=8, I=512, I_s=512, act="bf16", w="bf16")
    pre = dict(d=8192, E=512, k=10, I=2048, I_s=2048, act="bf16", w="bf16")
    assert bench.gathers_rows(c35, 4096)            # x = 16 MiB: rows gathered
    assert bench.gathers_rows(pre, 8192)            # x = 128 MiB: gathered too (up to 256 MiB)
    assert not bench.gathers_rows(pre, 64)          # decode: the weight-row form
    assert not bench.gathers_rows(dict(c35, w="fp8"), 4096)
    assert bench.forward_plan(pre, 8192)["expert_form"] == "rows"   # the line reports it
    counts = [128] * 256
    T = 4096
    w = bench.work_model(c35, counts, T)
    weights = (256 * 2 * 2048 * 512 + 2 * 2048 * 512) * 2
    h = (128 * 256 * 512 + T * 512) * 2
    assert w["gemm_gate_up"]["bytes"] == weights + T * 2048 * 2 + h
    # prefill shape, gathered: the token matrix is the input
    counts = [160] * 512
    T = 8192
    w = bench.work_model(pre, counts, T)
    weights = (512 * 2 * 8192 * 2048 + 2 * 8192 * 2048) * 2
    h = (160 * 512 * 2048 + T * 2048) * 2
    assert w["gemm_gate_up"]["bytes"] == weights + T * 8192 * 2 + h
    # without the gather (E4M3 weights, row-tiled) the dispatched rows are the input
    pre8 = dict(pre, w="fp8")
    assert not bench.gathers_rows(pre8, 8192)


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config",
                          "tiny_fp32", "--steps", "3", "--warmup", "3"], capture_output=True, text=True,
                         timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["metric"] == bench.METRIC


def test_warmup_below_three_is_refused():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--warmup", "2"], capture_output=True,
                         text=True, timeout=300, cwd=ROOT)
    assert out.returncode != 0 and "warmup" in out.stderr


def _profile_commands(target):
    """The argument lists given to `target` in the commands of profiles/*.md."""
    import glob
    import re
    import shlex
    out = []
    for f in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        text = open(f).read().replace("\\\n", " ")
        for line in text.splitlines():
            for m in re.finditer(re.escape(target) + r"((?:\s+--?[\w-]+(?:\s+(?!-)[^\s>&|]+)?)*)", line):
                out.append((os.path.basename(f), shlex.split(m.group(1))))
    return out


def test_profile_commands_match_the_current_command_lines():
    """Every command a committed ncu summary gives for bench.py or the
    profiler target still parses: the summaries can be re-run as written."""
    from sparse_moe_layer_top_b200 import profile_case
    bench_cmds = _profile_commands("bench.py")
    case_cmds = _profile_commands("sparse_moe_layer_top_b200.profile_case")
    assert bench_cmds and case_cmds
    for name, args in bench_cmds:
        bench.arg_parser().parse_args(args)
    for name, args in case_cmds:
        profile_case.arg_parser().parse_args(args)


def _small_inputs():
    import moe_inputs
    return moe_inputs.make_inputs(48, 128, 16, 2, 64, 64, act="bf16", w="bf16", seed=0)


def test_cpu_baseline_compact_sample_fits_the_host_budget():
    """The CPU baseline of a workload too large for the host times the oracle
    on a token sample whose experts fit the budget, hottest expert first."""
    import torch

    import oracle
    inp = _small_inputs()
    _, ids, _ = oracle.router(inp.x, inp.w_r, inp.k)
    ids = torch.as_tensor(ids)
    per_expert = bench.weight_bytes(inp) // inp.E
    d = bench.cpu_baseline_compact(inp, ids, target_s=0.05, n_max=16, budget=5 * per_expert)
    assert d["value"] > 0 and d["kind"] == "oracle"
    assert "hottest" in d["sample"]
    n_exp = int(d["sample"].split("copies of the ")[1].split()[0])
    assert inp.k <= n_exp <= 5
    toks = bench.sample_tokens(ids, inp.T, 16)
    cnt = torch.bincount(ids.reshape(-1).long())
    assert int(cnt.argmax()) in ids[toks[0]].tolist()
    assert len(set(toks)) == len(toks) and all(0 <= t < inp.T for t in toks)


def test_oracle_routed_time_splits_a_step_over_the_budget():
    import oracle
    inp = _small_inputs()
    per_expert = bench.weight_bytes(inp) // inp.E
    t = bench.oracle_routed_time(inp, list(range(12)), inp.w_r, None, budget=3 * per_expert)
    assert t > 0
    # a budget below k experts still runs each token on its own
    t = bench.oracle_routed_time(inp, [0, 5], inp.w_r, None, budget=1)
    assert t > 0
