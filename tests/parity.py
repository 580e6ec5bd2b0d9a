"""Comparison protocol between the CUDA path and the float64 oracle.

* Top-k sets must match exactly for every token whose oracle probability gap
  between the k-th and (k+1)-th expert exceeds 1e-4.
* A token inside that gap (a near tie) may legitimately pick another set G;
  G is accepted iff min_{e in G} p_e >= max_{e not in G} p_e - 1e-4, and the
  oracle's expected output for that token is then recomputed with G.
* Weights: |w_gpu - p_G / sum p_G| <= tol_w per entry.
* Outputs: relative L2 error ||y - y_ref|| / ||y_ref|| <= tol (1e-5 for fp32
  problems, 1e-2 for bf16, 2e-2 for FP8 weights).
"""
import numpy as np
import torch

GAP = 1e-4
TOL = {"f32": 1e-5, "bf16": 1e-2, "fp8": 2e-2}
TOL_W = {"f32": 1e-6, "bf16": 1e-3, "fp8": 1e-3}


def rel_l2(y, ref):
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(y - ref) / (den if den > 0 else 1.0))


def check_routing(gpu_ids, gpu_w, probs, oracle_ids, tol_w):
    """Validate the GPU's routing against the oracle's probabilities.

    Returns (ids to recompute the oracle with, number of near-tie tokens whose
    set differs).  Raises AssertionError on any violation."""
    gpu_ids = np.asarray(gpu_ids)
    gpu_w = np.asarray(gpu_w, np.float64)
    T, k = gpu_ids.shape
    E = probs.shape[1]
    ps = -np.sort(-probs, axis=1)
    gap = ps[:, k - 1] - ps[:, k] if k < E else np.full(T, np.inf)
    use = np.array(oracle_ids, copy=True)
    differ = 0
    for t in range(T):
        G = gpu_ids[t]
        assert len(set(G.tolist())) == k, "token %d: repeated expert ids %s" % (t, G)
        assert ((G >= 0) & (G < E)).all(), "token %d: id out of range %s" % (t, G)
        same = set(G.tolist()) == set(oracle_ids[t].tolist())
        if not same:
            assert gap[t] <= GAP, "token %d: set %s != oracle %s with gap %.3g" % (
                t, sorted(G), sorted(oracle_ids[t]), gap[t])
            out = np.ones(E, bool)
            out[G] = False
            assert probs[t, G].min() >= probs[t, out].max() - GAP, "token %d: set %s is not a near-tie choice" % (t, G)
            use[t] = G
            differ += 1
        ref_w = probs[t, G] / probs[t, G].sum()
        err = np.abs(gpu_w[t] - ref_w).max()
        assert err <= tol_w, "token %d: weight error %.3g > %.3g" % (t, err, tol_w)
    return use, differ


def to_cpu_inputs(inp):
    """A copy of a MoEInputs with every tensor on the CPU (for the oracle)."""
    import copy
    c = copy.copy(inp)
    for n in ("x", "w_r", "bias", "wg", "wu", "wd", "s_wg", "s_wu", "s_wd", "scales"):
        t = getattr(inp, n)
        if t is not None:
            setattr(c, n, t.detach().cpu())
    return c


def to_device(inp, device):
    import copy
    c = copy.copy(inp)
    for n in ("x", "w_r", "bias", "wg", "wu", "wd", "s_wg", "s_wu", "s_wd", "scales"):
        t = getattr(inp, n)
        if t is not None:
            setattr(c, n, t.to(device).contiguous())
    return c


def precision_key(inp):
    return "fp8" if inp.w == "fp8" else inp.act
