"""Run the block's forward on a synthetic problem of a chosen size, a few times.

Meant as the target of profiler runs (ncu) on sizes smaller than the
benchmark workloads:

    python -m sparse_moe_layer_top_b200.profile_case --T 64 --d 8192 --E 32 --k 10 --I 2048 --w bf16
    python -m sparse_moe_layer_top_b200.profile_case --config qwen38max_prefill_zipf_bf16 --reps 3

(--config runs a named benchmark workload at its full size instead.)

Inputs come from moe_inputs (seeded).  Exits non-zero if the device status
word reports a fault.
"""
import argparse
import os
import sys


def arg_parser():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--T", type=int, default=256)
    ap.add_argument("--d", type=int, default=8192)
    ap.add_argument("--E", type=int, default=64)
    ap.add_argument("--k", type=int, default=10)
    ap.add_argument("--I", type=int, default=2048)
    ap.add_argument("--Is", type=int, default=2048)
    ap.add_argument("--w", choices=("bf16", "fp8"), default="bf16")
    ap.add_argument("--bias", choices=("none", "zipf"), default="none")
    ap.add_argument("--path", type=int, default=0)
    ap.add_argument("--reps", type=int, default=2)
    ap.add_argument("--config", default=None, help="a named workload of moe_inputs.CONFIGS, at its full size")
    return ap


def main(argv=None):
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    if root not in sys.path:
        sys.path.insert(0, root)
    import torch

    import moe_inputs
    import sparse_moe_layer_top_b200 as moe

    a = arg_parser().parse_args(argv)
    torch.cuda.set_device(0)
    if a.config:
        inp = moe_inputs.make_config(a.config, seed=0, device="cuda")
    else:
        inp = moe_inputs.make_inputs(a.T, a.d, a.E, a.k, a.I, a.Is, act="bf16", w=a.w,
                                     bias=None if a.bias == "none" else a.bias, seed=0, device="cuda")
    moe.set_path(a.path)
    layer = moe.MoELayer.from_inputs(inp, max_tokens=inp.T)
    for _ in range(a.reps):
        y = layer(inp.x)
    torch.cuda.synchronize()
    status, detail = moe.device_status()
    if status != 0:
        raise SystemExit("device status %d (0x%08x)" % (status, detail & 0xffffffff))
    print("ok: %d launches per forward, |y| = %.4f" % (moe.last_launch_count(), float(y.float().norm())))


if __name__ == "__main__":
    main()
