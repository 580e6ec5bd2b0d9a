"""Float64 CPU oracle of the sparse MoE block -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library neither imports it nor
shares any code with it.

Thin ``ctypes`` marshalling around ``moe_oracle.c`` (which carries the
citations of what each stage computes).  Arrays may be numpy arrays or CPU
torch tensors; element types are float32, bfloat16 (or its raw uint16 bits)
and float8_e4m3fn (or its raw uint8 bits).  Results come back as numpy
float64 / int32 arrays.
"""
import ctypes
import os

import numpy as np

from . import build_oracle

F32, BF16, E4M3 = 0, 1, 2

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = build_oracle.build()
        L = ctypes.CDLL(path)
        P, I64, I32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        L.oracle_router.argtypes = [I64, I32, I32, I32, I32, P, P, P, P, P, P]
        L.oracle_permute.argtypes = [I64, I32, I32, P, P, P, P, P]
        L.oracle_swiglu_expert.argtypes = [I64, I32, I32, I32, P, I64, I32, P, P, P, P, P, P, P]
        L.oracle_moe_forward.argtypes = [I64, I32, I32, I32, I32, I32, I32, I32,
                                         P, P, P, P, P, P, P, P, P, P, P, P, P, P, P]
        L.oracle_block_forward.argtypes = [I64, I32, I32, I32, I32, I32, I32, I32, P, P, ctypes.c_double, P,
                                           P, P, P, P, P, P, P, P, P, P, P, P, P, P, P]
        L.oracle_rmsnorm.argtypes = [I64, I32, I32, P, P, ctypes.c_double, P]
        L.oracle_expert_ffn.argtypes = [I32, I32, I32, I32, I32, I32, P, P, P, P, P, P, P, P, P, P]
        L.oracle_combine.argtypes = [I64, I32, I32, I32, I32, P, P, P, P, P]
        L.oracle_param_count.argtypes = [I64, I64, I64, I64, I64, I32]
        L.oracle_param_count.restype = I64
        L.oracle_e4m3_decode.argtypes = [P, I64, P]
        for f in ("oracle_router", "oracle_permute", "oracle_swiglu_expert", "oracle_moe_forward",
                  "oracle_block_forward", "oracle_rmsnorm", "oracle_expert_ffn", "oracle_combine",
                  "oracle_e4m3_decode"):
            getattr(L, f).restype = I32
        L.oracle_num_threads.restype = I32
        _lib = L
    return _lib


def _np(a):
    """(contiguous numpy array, element code) for a numpy array or CPU tensor."""
    if a is None:
        return None, None
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu().contiguous()
            if a.dtype == torch.bfloat16:
                return a.view(torch.int16).numpy().view(np.uint16), BF16
            if a.dtype == torch.float8_e4m3fn:
                return a.view(torch.uint8).numpy(), E4M3
            a = a.numpy()
    except ImportError:
        pass
    a = np.ascontiguousarray(a)
    if a.dtype == np.float32:
        return a, F32
    if a.dtype == np.uint16:
        return a, BF16
    if a.dtype == np.uint8:
        return a, E4M3
    if a.dtype == np.float64:
        return a.astype(np.float32), F32
    raise TypeError("unsupported element type %s" % a.dtype)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    if a is None:
        return None
    a, _ = _np(a)
    return np.ascontiguousarray(a, dtype=np.float32)


def _i32(a):
    a, _ = _np(a) if not isinstance(a, np.ndarray) else (a, None)
    return np.ascontiguousarray(a, dtype=np.int32)


def num_threads():
    return lib().oracle_num_threads()


def e4m3_decode(codes):
    q = np.ascontiguousarray(np.asarray(codes, dtype=np.uint8))
    out = np.empty(q.shape, dtype=np.float64)
    lib().oracle_e4m3_decode(_p(q), q.size, _p(out))
    return out


def router(x, w_r, k, bias=None):
    """-> (probs [T,E], topk_ids [T,k], topk_w [T,k])."""
    xa, adt = _np(x)
    wa, wdt = _np(w_r)
    assert adt == wdt, "router weight must be in the activation type"
    T, d = xa.shape
    E = wa.shape[0]
    b = _f32(bias)
    probs = np.empty((T, E)); ids = np.empty((T, k), np.int32); w = np.empty((T, k))
    rc = lib().oracle_router(T, d, E, k, adt, _p(xa), _p(wa), _p(b), _p(probs), _p(ids), _p(w))
    assert rc == 0
    return probs, ids, w


def permute(topk_ids, E):
    """-> (offs [E+2], row_tok [T*(k+1)], row_slot [T*(k+1)], pos [T,k])."""
    ids = _i32(topk_ids)
    T, k = ids.shape
    offs = np.empty(E + 2, np.int32)
    row_tok = np.empty(T * (k + 1), np.int32)
    row_slot = np.empty(T * (k + 1), np.int32)
    pos = np.empty((T, k), np.int32)
    rc = lib().oracle_permute(T, E, k, _p(ids), _p(offs), _p(row_tok), _p(row_slot), _p(pos))
    assert rc == 0
    return offs, row_tok, row_slot, pos


def swiglu_expert(xs, wg, wu, wd, sg=None, su=None, sd=None):
    """One expert on rows xs [n,d]; weights [I,d],[I,d],[d,I] -> [n,d] float64."""
    xa, adt = _np(xs)
    ga, wdt = _np(wg)
    ua, _ = _np(wu)
    da, _ = _np(wd)
    n, d = xa.shape
    I = ga.shape[0]
    out = np.empty((n, d))
    s = [_f32(v) for v in (sg, su, sd)]
    rc = lib().oracle_swiglu_expert(n, d, I, adt, _p(xa), d, wdt, _p(ga), _p(ua), _p(da),
                                    _p(s[0]), _p(s[1]), _p(s[2]), _p(out))
    assert rc == 0
    return out


def moe_forward(x, w_r, wg, wu, wd, s_wg, s_wu, s_wd, k, bias=None, scales=None,
                force_ids=None, want_probs=True):
    """The whole block -> (y [T,d], topk_ids [T,k], topk_w [T,k], probs [T,E] or None).

    wg, wu [E,I,d]; wd [E,d,I]; shared [I_s,d],[I_s,d],[d,I_s] (None: no shared
    expert).  scales: the packed fp32 block-scale buffer for E4M3 weights.
    """
    xa, adt = _np(x)
    ra, rdt = _np(w_r)
    assert rdt == adt
    ga, wdt = _np(wg)
    ua, _ = _np(wu)
    da, _ = _np(wd)
    T, d = xa.shape
    E, I = ga.shape[0], ga.shape[1]
    if s_wg is None:
        sga = sua = sda = None
        I_s = 0
    else:
        sga, _ = _np(s_wg)
        sua, _ = _np(s_wu)
        sda, _ = _np(s_wd)
        I_s = sga.shape[0]
    b = _f32(bias)
    sc = _f32(scales)
    fi = None if force_ids is None else _i32(force_ids)
    y = np.empty((T, d)); ids = np.empty((T, k), np.int32); w = np.empty((T, k))
    probs = np.empty((T, E)) if want_probs else None
    rc = lib().oracle_moe_forward(T, d, E, k, I, I_s, adt, wdt, _p(xa), _p(ra), _p(b), _p(ga),
                                  _p(ua), _p(da), _p(sga), _p(sua), _p(sda), _p(sc), _p(fi),
                                  _p(y), _p(ids), _p(w), _p(probs))
    assert rc == 0
    return y, ids, w, probs


def rmsnorm(x, gamma, eps=1e-6):
    """Zero-centred RMSNorm of the rows of x [T, d]: x / sqrt(mean x^2 + eps) * (1 + gamma),
    float64, not rounded (gamma [d] in x's type)."""
    xa, adt = _np(x)
    ga, gdt = _np(gamma)
    assert gdt == adt
    T, d = xa.shape
    out = np.empty((T, d))
    assert lib().oracle_rmsnorm(T, d, adt, _p(xa), _p(ga), float(eps), _p(out)) == 0
    return out


def block_forward(x, w_r, wg, wu, wd, s_wg, s_wu, s_wd, k, bias=None, scales=None, norm_weight=None,
                  norm_eps=1e-6, shared_gate=None, force_ids=None, want_probs=True):
    """The block with its optional neighbours -> (y, topk_ids, topk_w, probs, gate).

    norm_weight [d] (x's type): zero-centred RMSNorm of x first, rounded to x's type;
    shared_gate [d] (x's type): the shared expert weighted by sigmoid(x . shared_gate).
    gate [T] is that weight (1 without a gate).  The rest as moe_forward.
    """
    xa, adt = _np(x)
    ra, rdt = _np(w_r)
    assert rdt == adt
    ga, wdt = _np(wg)
    ua, _ = _np(wu)
    da, _ = _np(wd)
    T, d = xa.shape
    E, I = ga.shape[0], ga.shape[1]
    if s_wg is None:
        sga = sua = sda = None
        I_s = 0
    else:
        sga, _ = _np(s_wg)
        sua, _ = _np(s_wu)
        sda, _ = _np(s_wd)
        I_s = sga.shape[0]
    na = None if norm_weight is None else _np(norm_weight)[0]
    gwa = None if shared_gate is None else _np(shared_gate)[0]
    b = _f32(bias)
    sc = _f32(scales)
    fi = None if force_ids is None else _i32(force_ids)
    y = np.empty((T, d)); ids = np.empty((T, k), np.int32); w = np.empty((T, k)); gate = np.empty(T)
    probs = np.empty((T, E)) if want_probs else None
    rc = lib().oracle_block_forward(T, d, E, k, I, I_s, adt, wdt, _p(xa), _p(na), float(norm_eps), _p(gwa),
                                    _p(ra), _p(b), _p(ga), _p(ua), _p(da), _p(sga), _p(sua), _p(sda), _p(sc),
                                    _p(fi), _p(y), _p(ids), _p(w), _p(probs), _p(gate))
    assert rc == 0
    return y, ids, w, probs, gate


def expert_ffn(x_perm, offs, wg, wu, wd, s_wg, s_wu, s_wd, scales=None):
    """Expert stage: unweighted y_perm [R', d] for dispatched rows x_perm."""
    xa, adt = _np(x_perm)
    ga, wdt = _np(wg)
    ua, _ = _np(wu)
    da, _ = _np(wd)
    o = _i32(offs)
    E, I = ga.shape[0], ga.shape[1]
    d = xa.shape[1]
    if s_wg is None:
        sga = sua = sda = None
        I_s = 0
    else:
        sga, _ = _np(s_wg)
        sua, _ = _np(s_wu)
        sda, _ = _np(s_wd)
        I_s = sga.shape[0]
    sc = _f32(scales)
    out = np.zeros((xa.shape[0], d))
    rc = lib().oracle_expert_ffn(d, E, I, I_s, adt, wdt, _p(xa), _p(o), _p(ga), _p(ua), _p(da),
                                 _p(sga), _p(sua), _p(sda), _p(sc), _p(out))
    assert rc == 0
    return out


def combine(y_perm, pos, topk_w, offs, E):
    ya, adt = _np(y_perm)
    p = _i32(pos)
    w = _f32(topk_w)
    o = _i32(offs)
    T, k = p.shape
    d = ya.shape[1]
    y = np.empty((T, d))
    rc = lib().oracle_combine(T, d, E, k, adt, _p(ya), _p(p), _p(w), _p(o), _p(y))
    assert rc == 0
    return y


def param_count(d, E, k, I, I_s, active=False):
    return lib().oracle_param_count(d, E, k, I, I_s, 1 if active else 0)
