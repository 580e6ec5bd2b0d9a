"""The C ABI without a GPU: the library loads, exports every function that
include/moe.h declares, and rejects bad arguments on the host before it
touches CUDA (null or misaligned pointers, bad sizes, a short workspace)."""
import ctypes
import os
import re

import pytest

import sparse_moe_layer_top_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for f in ("moe_router_topk", "moe_permute", "moe_expert_ffn", "moe_combine", "moe_layer_forward"):
        assert f in names


def test_library_exports_every_declared_symbol():
    L = ctypes.CDLL(moe.lib_path)
    for name in _declared():
        assert hasattr(L, name), name
    assert set(_declared()) == set(moe.EXPORTS)


def test_bounds_checking_build_exports_the_same_symbols():
    """libmoe_checks.so (-DMOE_CHECKS) is the same boundary with device index
    checks compiled in; it says so through moe_bounds_checked."""
    path = os.path.join(os.path.dirname(moe.lib_path), "libmoe_checks.so")
    assert os.path.exists(path), "python -m sparse_moe_layer_top_b200.build --checks"
    L = ctypes.CDLL(path)
    for name in _declared():
        assert hasattr(L, name), name
    assert L.moe_bounds_checked() == 1
    assert ctypes.CDLL(os.path.join(os.path.dirname(moe.lib_path), "libmoe.so")).moe_bounds_checked() == 0


def P(**kw):
    base = dict(T=64, d=256, E=16, k=2, I=128, I_s=64, act="bf16", w="bf16")
    base.update(kw)
    return moe.Problem.make(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(), 0),
    (dict(T=0), 0),
    (dict(act="f32", w="f32"), 0),
    (dict(w="fp8", d=256, I=128, I_s=128), 0),
    (dict(T=-1), 1),
    (dict(k=0), 1),
    (dict(k=17, E=32), 1),
    (dict(k=5, E=4), 1),
    (dict(E=513), 2),
    (dict(d=100), 3),
    (dict(I=12), 3),
    (dict(act="f32", w="bf16"), 2),
    (dict(w="fp8", d=192), 1),
    (dict(I_s=0), 0),
])
def test_check_problem(kw, status):
    assert moe.lib().moe_check_problem(ctypes.byref(P(**kw))) == status


def test_workspace_sizes_grow_with_tokens():
    a = moe.workspace_size(P(T=64))
    b = moe.workspace_size(P(T=4096))
    assert 0 < a < b
    assert moe.workspace_size(P(k=0)) == 0
    # forward workspace holds at least the dispatched rows (shared with the
    # weighted slot rows of the down projection) and the SwiGLU activations H
    p = P(T=4096)
    Rp = 4096 * 3
    assert b >= Rp * 256 * 2 + Rp * 128 * 2
    assert moe.stage_workspace_size(p) < b


def _call_forward(prob, x=16, wr=16, y=16, ws=16, ws_bytes=None, wg=16):
    L = moe.lib()
    v = lambda a: None if a is None else ctypes.c_void_p(a)
    n = moe.workspace_size(prob) if ws_bytes is None else ws_bytes
    return L.moe_layer_forward(ctypes.byref(prob), v(x), v(wr), None, v(wg), v(16), v(16), v(16), v(16), v(16),
                               None, v(y), None, None, v(ws), n, None)


def test_host_rejects_before_any_launch():
    prob = P()
    # fake (never dereferenced) 16-byte aligned addresses; every case fails on the host
    assert _call_forward(prob, x=None) == 1
    assert _call_forward(prob, wg=None) == 1
    assert _call_forward(prob, y=0x1008) == 3
    assert _call_forward(prob, ws_bytes=moe.workspace_size(prob) - 1) == 4
    assert b"workspace" in moe.lib().moe_last_error_string()
    assert _call_forward(P(E=600)) == 2


def test_set_path_validates():
    assert moe.lib().moe_set_path(7) == 1
    assert moe.lib().moe_set_path(5) == 0
    assert moe.lib().moe_set_path(-1) == 1
    assert moe.lib().moe_set_path(0) == 0


def _call_block(prob, norm=None, eps=1e-6, gate=None, x=16):
    L = moe.lib()
    v = lambda a: None if a is None else ctypes.c_void_p(a)
    opt = moe.BlockOptions(norm, eps, gate)
    return L.moe_block_forward(ctypes.byref(prob), ctypes.byref(opt), v(x), v(16), None, v(16), v(16), v(16),
                               v(16), v(16), v(16), None, v(16), None, None, v(16), moe.workspace_size(prob), None)


def test_block_options_rejected_before_any_launch():
    prob = P()
    # every case below fails on the host (fake addresses are never dereferenced)
    assert _call_block(prob, norm=0x1008) == 3          # misaligned norm weight
    assert _call_block(prob, gate=0x1008) == 3          # misaligned gate weight
    assert _call_block(prob, norm=16, eps=-1.0) == 1    # negative eps
    assert _call_block(prob, norm=16, eps=float("nan")) == 1
    assert _call_block(prob, norm=16, x=None) == 1      # no input
    L = moe.lib()
    v = ctypes.c_void_p
    assert L.moe_rmsnorm(ctypes.byref(prob), v(16), None, 1e-6, v(16), None) == 1
    assert L.moe_rmsnorm(ctypes.byref(prob), v(16), v(16), -1.0, v(16), None) == 1
    assert L.moe_rmsnorm(ctypes.byref(prob), v(16), v(0x1008), 1e-6, v(16), None) == 3
    assert L.moe_rmsnorm(ctypes.byref(P(d=100)), v(16), v(16), 1e-6, v(16), None) == 3


def test_ep_expand_ids_rejected_before_any_launch():
    L = moe.lib()
    v = ctypes.c_void_p
    # every case fails on the host (fake addresses are never dereferenced)
    assert L.moe_ep_expand_ids(v(16), 0, 4, 10, v(16), None) == 1      # no ranks
    assert L.moe_ep_expand_ids(v(16), 2, 0, 10, v(16), None) == 1      # no experts
    assert L.moe_ep_expand_ids(v(16), 64, 65, 10, v(16), None) == 1    # 4160 blocks > 4096
    assert L.moe_ep_expand_ids(v(16), 2, 4, -1, v(16), None) == 1      # negative row count
    assert L.moe_ep_expand_ids(v(16), 2, 4, 1 << 31, v(16), None) == 1
    assert L.moe_ep_expand_ids(None, 2, 4, 10, v(16), None) == 1       # no counts
    assert L.moe_ep_expand_ids(v(16), 2, 4, 10, None, None) == 1       # no output
    assert L.moe_ep_expand_ids(v(0x1008), 2, 4, 10, v(16), None) == 3  # misaligned
    assert L.moe_ep_expand_ids(None, 2, 4, 0, None, None) == 0         # nothing to do


def test_forward_plan_on_the_host():
    # the bench workloads' plans (host only: no device needed)
    plan = lambda *a: moe.forward_plan(moe.Problem.make(*a))  # noqa: E731
    assert plan(4096, 2048, 256, 8, 512, 512, "bf16", "bf16") == \
        {"expert_form": "rows", "router_selects": True, "gathered": True}
    assert plan(8192, 8192, 512, 10, 2048, 2048, "bf16", "bf16") == \
        {"expert_form": "rows", "router_selects": False, "gathered": True}       # 512 experts; x = 128 MiB
    # the pair form from 2048 rows per expert on average; the split form only on request
    assert plan(4095, 256, 2, 1, 256, 256, "bf16", "bf16")["expert_form"] == "rows"
    assert plan(4096, 256, 2, 1, 256, 256, "bf16", "bf16")["expert_form"] == "cta_pairs"
    assert plan(64, 8192, 512, 10, 2048, 2048, "bf16", "bf16")["expert_form"] == "weight_rows"
    assert plan(2048, 8192, 512, 10, 2048, 2048, "bf16", "fp8")["expert_form"] == "weight_rows"
    assert plan(32, 128, 16, 2, 64, 64, "f32", "f32") == \
        {"expert_form": "simt", "router_selects": False, "gathered": False}
    # the router selects in its epilogue from 16 token tiles on; the gather stops above 256 MiB of x
    assert not plan(1920, 256, 64, 4, 128, 128, "bf16", "bf16")["router_selects"]
    assert plan(1921, 256, 64, 4, 128, 128, "bf16", "bf16")["router_selects"]
    assert plan(16384, 8192, 128, 8, 256, 256, "bf16", "bf16")["gathered"]      # exactly 256 MiB
    assert not plan(16385, 8192, 128, 8, 256, 256, "bf16", "bf16")["gathered"]
    # the path setting moves the form
    try:
        moe.set_path(4)
        assert plan(4096, 2048, 256, 8, 512, 512, "bf16", "bf16")["expert_form"] == "cta_pairs"
        moe.set_path(5)
        assert plan(4096, 2048, 256, 8, 512, 512, "bf16", "bf16")["expert_form"] == "split"
        assert plan(4096, 2048, 256, 8, 512, 512, "bf16", "fp8")["expert_form"] == "rows"
        moe.set_path(6)
        assert plan(4096, 2048, 256, 8, 512, 512, "bf16", "bf16") == \
            {"expert_form": "cta_pairs_tokens_n", "router_selects": True, "gathered": False}
        assert plan(4096, 2048, 256, 8, 512, 512, "bf16", "fp8")["expert_form"] == "rows"
        moe.set_path(1)
        assert plan(4096, 2048, 256, 8, 512, 512, "bf16", "bf16") == \
            {"expert_form": "simt", "router_selects": False, "gathered": False}
    finally:
        moe.set_path(0)
    assert moe.lib().moe_forward_plan(ctypes.byref(P(T=-1)), None, None, None) == 1


def _c_kind(decl):
    """Kind of one C parameter declaration: pointer, i64, i32, size or f32."""
    decl = decl.strip()
    if "*" in decl:
        return "pointer"
    t = decl.rsplit(None, 1)[0].replace("const", "").strip()
    return {"int64_t": "i64", "int32_t": "i32", "int": "i32", "size_t": "size", "float": "f32"}[t]


def _ctypes_kind(t):
    if t is ctypes.c_void_p or t is ctypes.c_char_p or hasattr(t, "_type_") and isinstance(t._type_, type):
        return "pointer"
    if t is ctypes.c_size_t:
        return "size"
    if t is ctypes.c_float:
        return "f32"
    return {8: "i64", 4: "i32"}[ctypes.sizeof(t)]


def test_binding_argument_types_follow_the_header():
    """Every declared entry point's parameters, one by one, against the ctypes
    signature the binding gives it: a mismatch would pass a value where the
    library reads a pointer (or a 32-bit value where it reads 64 bits)."""
    src = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", "moe.h")).read(), flags=re.S)
    L = moe.lib()
    seen = 0
    for m in re.finditer(r"MOE_API\s+([\w\s\*]+?)\b(moe_\w+)\s*\(([^)]*)\)\s*;", src):
        ret, name, params = m.group(1).strip(), m.group(2), m.group(3).strip()
        decls = [] if params in ("", "void") else params.split(",")
        f = getattr(L, name)
        got = [] if f.argtypes is None else [_ctypes_kind(t) for t in f.argtypes]
        assert got == [_c_kind(p) for p in decls], name
        want_ret = {"moe_status": ctypes.c_int, "int": ctypes.c_int, "size_t": ctypes.c_size_t,
                    "const char*": ctypes.c_char_p}[ret.replace(" *", "*")]
        assert f.restype is want_ret, name
        seen += 1
    assert seen == len(moe.EXPORTS)


def test_a_missing_library_fails_loudly(monkeypatch, tmp_path):
    """No fallback: without libmoe.so every call raises, on the host, before
    anything could run elsewhere."""
    import torch
    monkeypatch.setattr(moe, "lib_path", str(tmp_path / "libmoe.so"))
    monkeypatch.setattr(moe, "_lib", None)
    with pytest.raises(ImportError, match="not built"):
        moe.workspace_size(P())
    a = torch.zeros((64, 256), dtype=torch.bfloat16)
    with pytest.raises(ImportError, match="not built"):
        moe.router_topk(P(), a, torch.zeros((16, 256), dtype=torch.bfloat16))
