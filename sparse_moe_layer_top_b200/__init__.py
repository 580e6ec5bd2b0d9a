"""Python binding of libmoe.so -- the sparse MoE block on B200 (sm_100a).

Argument marshalling only: every step of the block runs in the library's CUDA
kernels.  Tensors are CUDA torch tensors (contiguous, row-major); the calls
enqueue on the current torch stream and never synchronise.  The library is
built in-tree (``python -m sparse_moe_layer_top_b200.build``) and loaded on
first use; every call raises if it is missing -- there is no fallback.
The C ABI sees only pointers, so every call first checks its tensors' element
types and sizes against the problem and raises ValueError, before any pointer
is taken, when a buffer is of the wrong type or too small for what the call
reads or writes.  The library launches on the current CUDA device and its
current stream: every call also requires all its tensors (and a stream it is
given) to be on one device, and runs with that device current.

Entry points mirror ``include/moe.h``: ``router_topk``, ``permute``,
``expert_ffn``, ``combine``, ``layer_forward``, ``block_forward``,
``rmsnorm``, ``ep_expand_ids``; ``MoELayer`` keeps a layer's weights and
workspace together; ``sparse_moe_layer_top_b200.ep`` splits the experts over
several GPUs (expert parallelism).
"""
import contextlib
import ctypes
import os

import torch

__all__ = ["MoEError", "Problem", "BlockOptions", "router_topk", "permute", "expert_ffn", "combine", "layer_forward",
           "block_forward", "rmsnorm", "ep_expand_ids", "forward_plan",
           "workspace_size", "stage_workspace_size", "set_path", "set_wait_limit", "device_status",
           "last_launch_count", "bounds_checked",
           "profile_enable", "profile_read",
           "MoELayer", "lib_path", "F32", "BF16", "FP8_E4M3_B128"]

HERE = os.path.dirname(os.path.abspath(__file__))
# MOE_CHECKS=1 loads the bounds-checking build (python -m
# sparse_moe_layer_top_b200.build --checks), whose kernels check their
# computed indices on the device (moe_bounds_checked in include/moe.h)
lib_path = os.path.join(HERE, "libmoe_checks.so" if os.environ.get("MOE_CHECKS") == "1" else "libmoe.so")

F32, BF16, FP8_E4M3_B128 = 0, 1, 2
_STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_ALIGNMENT",
           4: "MOE_ERR_WORKSPACE_TOO_SMALL", 5: "MOE_ERR_CUDA", 6: "MOE_ERR_DEVICE_CHECK", 7: "MOE_ERR_TIMEOUT"}
EXPORTS = ("moe_check_problem", "moe_workspace_size", "moe_stage_workspace_size", "moe_router_topk",
           "moe_permute", "moe_expert_ffn", "moe_combine", "moe_layer_forward", "moe_set_path",
           "moe_device_status", "moe_last_launch_count", "moe_profile_enable", "moe_profile_read",
           "moe_last_error_string", "moe_router_topk_static", "moe_block_forward", "moe_rmsnorm",
           "moe_ep_expand_ids", "moe_forward_plan", "moe_set_wait_limit", "moe_bounds_checked")


class MoEError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__("%s: %s" % (_STATUS.get(status, status), msg))
        self.status = status


class Problem(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int32), ("E", ctypes.c_int32), ("k", ctypes.c_int32),
                ("I", ctypes.c_int32), ("I_s", ctypes.c_int32), ("act_dtype", ctypes.c_int32),
                ("w_dtype", ctypes.c_int32)]

    @classmethod
    def make(cls, T, d, E, k, I, I_s, act="bf16", w="bf16"):
        codes = {"f32": F32, "bf16": BF16, "fp8": FP8_E4M3_B128}
        return cls(int(T), int(d), int(E), int(k), int(I), int(I_s), codes[act], codes[w])


class BlockOptions(ctypes.Structure):
    _fields_ = [("norm_weight", ctypes.c_void_p), ("norm_eps", ctypes.c_float), ("shared_gate", ctypes.c_void_p)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(lib_path):
            raise ImportError("libmoe.so is not built (run python -m sparse_moe_layer_top_b200.build)")
        L = ctypes.CDLL(lib_path)
        P, PP = ctypes.c_void_p, ctypes.POINTER(Problem)
        S = ctypes.c_int
        L.moe_check_problem.argtypes = [PP]
        L.moe_workspace_size.argtypes = [PP]
        L.moe_workspace_size.restype = ctypes.c_size_t
        L.moe_stage_workspace_size.argtypes = [PP]
        L.moe_stage_workspace_size.restype = ctypes.c_size_t
        L.moe_router_topk.argtypes = [PP, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.moe_router_topk_static.argtypes = [PP, P, P, P, P, P, P]
        L.moe_permute.argtypes = [PP, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.moe_expert_ffn.argtypes = [PP, P, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.moe_combine.argtypes = [PP, P, P, P, P, P, P]
        L.moe_layer_forward.argtypes = [PP, P, P, P, P, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.moe_block_forward.argtypes = [PP, ctypes.POINTER(BlockOptions), P, P, P, P, P, P, P, P, P, P, P, P, P,
                                        P, ctypes.c_size_t, P]
        L.moe_ep_expand_ids.argtypes = [P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int64, P, P]
        I32P = ctypes.POINTER(ctypes.c_int32)
        L.moe_forward_plan.argtypes = [PP, I32P, I32P, I32P]
        L.moe_rmsnorm.argtypes = [PP, P, P, ctypes.c_float, P, P]
        L.moe_set_path.argtypes = [ctypes.c_int]
        L.moe_set_wait_limit.argtypes = [ctypes.c_int64]
        L.moe_device_status.argtypes = [ctypes.POINTER(ctypes.c_int32)]
        L.moe_last_launch_count.restype = ctypes.c_int
        L.moe_bounds_checked.restype = ctypes.c_int
        L.moe_profile_enable.argtypes = [ctypes.c_int]
        L.moe_profile_enable.restype = ctypes.c_int
        L.moe_profile_read.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_float),
                                       ctypes.POINTER(ctypes.c_char_p)]
        L.moe_profile_read.restype = ctypes.c_int
        L.moe_last_error_string.restype = ctypes.c_char_p
        for f in ("moe_check_problem", "moe_router_topk", "moe_router_topk_static", "moe_permute", "moe_expert_ffn", "moe_combine",
                  "moe_layer_forward", "moe_block_forward", "moe_rmsnorm", "moe_set_path", "moe_device_status",
                  "moe_set_wait_limit"):
            getattr(L, f).restype = S
        _lib = L
    return _lib


def _check(status):
    if status != 0:
        raise MoEError(status, lib().moe_last_error_string().decode())


_F32, _I32 = (torch.float32,), (torch.int32,)
_ACT_TYPES = {F32: (torch.float32,), BF16: (torch.bfloat16,)}
_W_TYPES = {F32: (torch.float32,), BF16: (torch.bfloat16,), FP8_E4M3_B128: (torch.float8_e4m3fn, torch.uint8)}


def _need(t, name, n, dtypes, row=None):
    """t (if given) holds at least n elements of one of dtypes (None: the
    problem's type code is invalid, which the library itself reports) and, if
    it has two or more dimensions, rows of `row` elements."""
    if t is None:
        return
    if dtypes is not None and t.dtype not in dtypes:
        raise ValueError("%s: element type %s, expected %s" % (name, t.dtype, " or ".join(map(str, dtypes))))
    if t.numel() < n:
        raise ValueError("%s: %d elements, the problem needs %d" % (name, t.numel(), n))
    if row is not None and t.dim() >= 2 and t.shape[-1] != row:
        raise ValueError("%s: rows of %d elements, expected %d" % (name, t.shape[-1], row))


def _need_weights(prob, wg, wu, wd, s_wg, s_wu, s_wd, scales):
    d, E, I, I_s = prob.d, prob.E, prob.I, prob.I_s
    wt = _W_TYPES.get(prob.w_dtype)
    _need(wg, "w_gate", E * I * d, wt, d)
    _need(wu, "w_up", E * I * d, wt, d)
    _need(wd, "w_down", E * d * I, wt, I)
    if I_s > 0:
        _need(s_wg, "ws_gate", I_s * d, wt, d)
        _need(s_wu, "ws_up", I_s * d, wt, d)
        _need(s_wd, "ws_down", d * I_s, wt, I_s)
    if prob.w_dtype == FP8_E4M3_B128:
        blocks = 3 * E * (I // 128) * (d // 128) + (3 * (I_s // 128) * (d // 128) if I_s > 0 else 0)
        _need(scales, "scales", blocks, _F32)


def _nbytes(t):
    return t.numel() * t.element_size()


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _device(stream=None, **tensors):
    """The one device all given tensors are on (None if none is given); a
    given stream must belong to it.  Raises ValueError naming the tensors
    otherwise -- the library would launch on the current device with
    another device's pointers."""
    devs = {}
    for name, t in tensors.items():
        if t is not None:
            devs.setdefault(t.device, []).append(name)
    if len(devs) > 1:
        raise ValueError("tensors on different devices: " +
                         "; ".join("%s on %s" % (", ".join(n), d) for d, n in devs.items()))
    dev = next(iter(devs), None)
    if stream is not None and dev is not None and dev.type == "cuda" and stream.device != dev:
        raise ValueError("stream on %s, tensors on %s" % (stream.device, dev))
    return dev


def _current(dev):
    """A context in which `dev` is the current CUDA device (nothing to do
    for a non-CUDA device: the pointer step rejects its tensors)."""
    if dev is not None and dev.type == "cuda":
        return torch.cuda.device(dev)
    return contextlib.nullcontext()


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _act(prob):
    return torch.float32 if prob.act_dtype == F32 else torch.bfloat16


def workspace_size(prob):
    return lib().moe_workspace_size(ctypes.byref(prob))


def stage_workspace_size(prob):
    return lib().moe_stage_workspace_size(ctypes.byref(prob))


def check_problem(prob):
    _check(lib().moe_check_problem(ctypes.byref(prob)))


def set_path(path):
    """0 automatic, 1 SIMT kernels only, 2 row-tiled tensor-core expert GEMMs,
    3 weight-row tensor-core expert GEMMs, 4 row-tiled on 2-CTA clusters,
    5 split: groups of 256 rows or more on 2-CTA clusters, the others in
    weight-row form (on request only), 6 on 2-CTA clusters with the tokens as
    the MMA's N (tiles of up to 256 rows, padded to 16)."""
    _check(lib().moe_set_path(int(path)))


def set_wait_limit(cycles=0):
    """Bound, in SM cycles, of the kernels' pipeline waits on the current
    device (0: the default, about 2 s).  Synchronous; call it with no library
    work in flight."""
    _check(lib().moe_set_wait_limit(int(cycles)))


def device_status():
    """(status, detail) of the device status word, which is then cleared (synchronises)."""
    d = ctypes.c_int32(0)
    s = lib().moe_device_status(ctypes.byref(d))
    return s, d.value


def bounds_checked():
    """True when the loaded library is the bounds-checking build."""
    return bool(lib().moe_bounds_checked())


def last_launch_count():
    return lib().moe_last_launch_count()


def profile_enable(mode=1):
    """1: bracket every library kernel launch of this thread with CUDA events;
    2: only the tensor-core GEMM launches; 0: off."""
    _check(lib().moe_profile_enable(int(mode)))


def profile_read(max_launches=4096):
    """[(kernel name, device ms), ...] of the launches recorded since the last
    read (waits for them), in launch order."""
    ms = (ctypes.c_float * max_launches)()
    names = (ctypes.c_char_p * max_launches)()
    n = lib().moe_profile_read(max_launches, ms, names)
    return [(names[i].decode(), float(ms[i])) for i in range(n)]


def _ws(nbytes, device, ws):
    if ws is None:
        ws = torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)
    return ws


def router_topk(prob, x, w_router, bias=None, topk_ids=None, topk_w=None, ws=None, stream=None):
    T, k = prob.T, prob.k
    a = _ACT_TYPES.get(prob.act_dtype)
    _need(x, "x", T * prob.d, a, prob.d)
    _need(w_router, "w_router", prob.E * prob.d, a, prob.d)
    _need(bias, "router_bias", prob.E, _F32)
    _need(topk_ids, "topk_ids", T * k, _I32, k)
    _need(topk_w, "topk_w", T * k, _F32, k)
    dev = _device(stream, x=x, w_router=w_router, router_bias=bias, topk_ids=topk_ids, topk_w=topk_w, ws=ws)
    if topk_ids is None:
        topk_ids = torch.empty((T, k), dtype=torch.int32, device=x.device)
    if topk_w is None:
        topk_w = torch.empty((T, k), dtype=torch.float32, device=x.device)
    ws = _ws(stage_workspace_size(prob), x.device, ws)
    with _current(dev):
        _check(lib().moe_router_topk(ctypes.byref(prob), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(topk_ids),
                                     _ptr(topk_w), _ptr(ws), _nbytes(ws), _stream(stream)))
    return topk_ids, topk_w


def rows_total(prob):
    return prob.T * prob.k + (prob.T if prob.I_s > 0 else 0)


def permute(prob, x, topk_ids, topk_w, ws=None, stream=None):
    """-> dict(x_perm, row_tok, row_w, pos, offs)."""
    _need(x, "x", prob.T * prob.d, _ACT_TYPES.get(prob.act_dtype), prob.d)
    _need(topk_ids, "topk_ids", prob.T * prob.k, _I32, prob.k)
    _need(topk_w, "topk_w", prob.T * prob.k, _F32, prob.k)
    cur = _device(stream, x=x, topk_ids=topk_ids, topk_w=topk_w, ws=ws)
    dev = x.device
    Rp = rows_total(prob)
    out = dict(x_perm=torch.empty((Rp, prob.d), dtype=_act(prob), device=dev),
               row_tok=torch.empty(Rp, dtype=torch.int32, device=dev),
               row_w=torch.empty(Rp, dtype=torch.float32, device=dev),
               pos=torch.empty((prob.T, prob.k), dtype=torch.int32, device=dev),
               offs=torch.empty(prob.E + 2, dtype=torch.int32, device=dev))
    nbytes = stage_workspace_size(prob)
    ws = _ws(nbytes, dev, ws)
    with _current(cur):
        _check(lib().moe_permute(ctypes.byref(prob), _ptr(x), _ptr(topk_ids), _ptr(topk_w), _ptr(out["x_perm"]),
                                 _ptr(out["row_tok"]), _ptr(out["row_w"]), _ptr(out["pos"]), _ptr(out["offs"]),
                                 _ptr(ws), _nbytes(ws), _stream(stream)))
    return out


def expert_ffn(prob, x_perm, offs, wg, wu, wd, s_wg=None, s_wu=None, s_wd=None, scales=None, y_perm=None,
               ws=None, stream=None):
    a, Rp = _ACT_TYPES.get(prob.act_dtype), rows_total(prob)
    _need(x_perm, "x_perm", Rp * prob.d, a, prob.d)
    _need(offs, "offs", prob.E + 2, _I32)
    _need_weights(prob, wg, wu, wd, s_wg, s_wu, s_wd, scales)
    _need(y_perm, "y_perm", Rp * prob.d, a, prob.d)
    cur = _device(stream, x_perm=x_perm, offs=offs, w_gate=wg, w_up=wu, w_down=wd, ws_gate=s_wg, ws_up=s_wu,
                  ws_down=s_wd, scales=scales, y_perm=y_perm, ws=ws)
    dev = x_perm.device
    if y_perm is None:
        y_perm = torch.empty((x_perm.shape[0], prob.d), dtype=_act(prob), device=dev)
    ws = _ws(stage_workspace_size(prob), dev, ws)
    with _current(cur):
        _check(lib().moe_expert_ffn(ctypes.byref(prob), _ptr(x_perm), _ptr(offs), _ptr(wg), _ptr(wu), _ptr(wd),
                                    _ptr(s_wg), _ptr(s_wu), _ptr(s_wd), _ptr(scales), _ptr(y_perm), _ptr(ws),
                                    _nbytes(ws), _stream(stream)))
    return y_perm


def combine(prob, y_perm, pos, topk_w, offs, y=None, stream=None):
    a = _ACT_TYPES.get(prob.act_dtype)
    _need(y_perm, "y_perm", rows_total(prob) * prob.d, a, prob.d)
    _need(pos, "pos", prob.T * prob.k, _I32, prob.k)
    _need(topk_w, "topk_w", prob.T * prob.k, _F32, prob.k)
    _need(offs, "offs", prob.E + 2, _I32)
    _need(y, "y", prob.T * prob.d, a, prob.d)
    cur = _device(stream, y_perm=y_perm, pos=pos, topk_w=topk_w, offs=offs, y=y)
    if y is None:
        y = torch.empty((prob.T, prob.d), dtype=_act(prob), device=y_perm.device)
    with _current(cur):
        _check(lib().moe_combine(ctypes.byref(prob), _ptr(y_perm), _ptr(pos), _ptr(topk_w), _ptr(offs), _ptr(y),
                                 _stream(stream)))
    return y


def _need_params(prob, w_router, bias, wg, wu, wd, s_wg, s_wu, s_wd, scales, norm_weight=None, shared_gate=None):
    """The block's parameters (independent of the token count)."""
    a = _ACT_TYPES.get(prob.act_dtype)
    _need(w_router, "w_router", prob.E * prob.d, a, prob.d)
    _need(bias, "router_bias", prob.E, _F32)
    _need_weights(prob, wg, wu, wd, s_wg, s_wu, s_wd, scales)
    _need(norm_weight, "norm_weight", prob.d, a)
    _need(shared_gate, "shared_gate", prob.d, a)


def _need_tokens(prob, x, y, topk_ids, topk_w):
    """One call's token buffers."""
    T, d, k = prob.T, prob.d, prob.k
    a = _ACT_TYPES.get(prob.act_dtype)
    _need(x, "x", T * d, a, d)
    _need(y, "y", T * d, a, d)
    _need(topk_ids, "topk_ids", T * k, _I32, k)
    _need(topk_w, "topk_w", T * k, _F32, k)


def _forward(prob, x, w_router, bias, wg, wu, wd, s_wg, s_wu, s_wd, scales, norm_weight, norm_eps, shared_gate, y,
             topk_ids, topk_w, ws, stream, block):
    """The fused forward on checked arguments (moe_block_forward when `block`)."""
    cur = _device(stream, x=x, w_router=w_router, router_bias=bias, w_gate=wg, w_up=wu, w_down=wd, ws_gate=s_wg,
                  ws_up=s_wu, ws_down=s_wd, scales=scales, norm_weight=norm_weight, shared_gate=shared_gate, y=y,
                  topk_ids=topk_ids, topk_w=topk_w, ws=ws)
    if y is None:
        y = torch.empty((prob.T, prob.d), dtype=_act(prob), device=x.device)
    ws = _ws(workspace_size(prob), x.device, ws)
    with _current(cur):
        _forward_call(prob, x, w_router, bias, wg, wu, wd, s_wg, s_wu, s_wd, scales, norm_weight, norm_eps,
                      shared_gate, y, topk_ids, topk_w, ws, stream, block)
    return y


def _forward_call(prob, x, w_router, bias, wg, wu, wd, s_wg, s_wu, s_wd, scales, norm_weight, norm_eps, shared_gate,
                  y, topk_ids, topk_w, ws, stream, block):
    if block:
        opt = BlockOptions(_ptr(norm_weight), float(norm_eps), _ptr(shared_gate))
        _check(lib().moe_block_forward(ctypes.byref(prob), ctypes.byref(opt), _ptr(x), _ptr(w_router), _ptr(bias),
                                       _ptr(wg), _ptr(wu), _ptr(wd), _ptr(s_wg), _ptr(s_wu), _ptr(s_wd),
                                       _ptr(scales), _ptr(y), _ptr(topk_ids), _ptr(topk_w), _ptr(ws), _nbytes(ws),
                                       _stream(stream)))
    else:
        _check(lib().moe_layer_forward(ctypes.byref(prob), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(wg), _ptr(wu),
                                       _ptr(wd), _ptr(s_wg), _ptr(s_wu), _ptr(s_wd), _ptr(scales), _ptr(y),
                                       _ptr(topk_ids), _ptr(topk_w), _ptr(ws), _nbytes(ws), _stream(stream)))


def layer_forward(prob, x, w_router, bias, wg, wu, wd, s_wg=None, s_wu=None, s_wd=None, scales=None, y=None,
                  topk_ids=None, topk_w=None, ws=None, stream=None):
    _need_params(prob, w_router, bias, wg, wu, wd, s_wg, s_wu, s_wd, scales)
    _need_tokens(prob, x, y, topk_ids, topk_w)
    return _forward(prob, x, w_router, bias, wg, wu, wd, s_wg, s_wu, s_wd, scales, None, 0.0, None, y, topk_ids,
                    topk_w, ws, stream, block=False)


def block_forward(prob, x, w_router, bias, wg, wu, wd, s_wg=None, s_wu=None, s_wd=None, scales=None,
                  norm_weight=None, norm_eps=1e-6, shared_gate=None, y=None, topk_ids=None, topk_w=None, ws=None,
                  stream=None):
    """layer_forward with the block's neighbours: zero-centred RMSNorm of x
    (norm_weight [d]) and a sigmoid gate on the shared expert (shared_gate [d])."""
    _need_params(prob, w_router, bias, wg, wu, wd, s_wg, s_wu, s_wd, scales, norm_weight, shared_gate)
    _need_tokens(prob, x, y, topk_ids, topk_w)
    return _forward(prob, x, w_router, bias, wg, wu, wd, s_wg, s_wu, s_wd, scales, norm_weight, norm_eps,
                    shared_gate, y, topk_ids, topk_w, ws, stream, block=True)


def rmsnorm(prob, x, norm_weight, eps=1e-6, out=None, stream=None):
    """Zero-centred RMSNorm of the rows of x: x / sqrt(mean x^2 + eps) * (1 + norm_weight)."""
    a = _ACT_TYPES.get(prob.act_dtype)
    _need(x, "x", prob.T * prob.d, a, prob.d)
    _need(norm_weight, "norm_weight", prob.d, a)
    _need(out, "out", prob.T * prob.d, a, prob.d)
    cur = _device(stream, x=x, norm_weight=norm_weight, out=out)
    if out is None:
        out = torch.empty_like(x)
    with _current(cur):
        _check(lib().moe_rmsnorm(ctypes.byref(prob), _ptr(x), _ptr(norm_weight), float(eps), _ptr(out),
                                 _stream(stream)))
    return out


EXPERT_FORMS = ("simt", "rows", "weight_rows", "cta_pairs", "split", "cta_pairs_tokens_n")


def forward_plan(prob):
    """What the fused forward launches for `prob` under the current path,
    decided on the host: dict(expert_form, router_selects, gathered)."""
    f, r, g = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _check(lib().moe_forward_plan(ctypes.byref(prob), ctypes.byref(f), ctypes.byref(r), ctypes.byref(g)))
    return {"expert_form": EXPERT_FORMS[f.value], "router_selects": bool(r.value), "gathered": bool(g.value)}


def ep_expand_ids(counts, G, E_local, R, ids=None, stream=None):
    """Expert parallelism, receive side: the local expert (int32 [R]) of every
    received row, rows arriving as blocks (source s, local expert e) in that
    order with counts[s * E_local + e] rows each (int32, on the device)."""
    _need(counts, "counts", int(G) * int(E_local), _I32)
    _need(ids, "ids", int(R), _I32)
    cur = _device(stream, counts=counts, ids=ids)
    if ids is None:
        ids = torch.empty(max(int(R), 0), dtype=torch.int32, device=counts.device)
    with _current(cur):
        _check(lib().moe_ep_expand_ids(_ptr(counts), int(G), int(E_local), int(R), _ptr(ids), _stream(stream)))
    return ids


class MoELayer:
    """One block's weights plus a workspace sized for up to `max_tokens` tokens."""

    def __init__(self, d, E, k, I, I_s, w_router, wg, wu, wd, s_wg=None, s_wu=None, s_wd=None, bias=None,
                 scales=None, act="bf16", w="bf16", max_tokens=0, norm_weight=None, norm_eps=1e-6,
                 shared_gate=None):
        self.shape = (d, E, k, I, I_s, act, w)
        self.w = (w_router, bias, wg, wu, wd, s_wg, s_wu, s_wd, scales)
        self.opts = (norm_weight, norm_eps, shared_gate)
        # the parameters are checked once here; each call checks its token buffers
        _need_params(self.problem(0), w_router, bias, wg, wu, wd, s_wg, s_wu, s_wd, scales, norm_weight,
                     shared_gate)
        self.device = wg.device
        self.ws = None
        if max_tokens:
            self._reserve(max_tokens)

    def problem(self, T):
        d, E, k, I, I_s, act, w = self.shape
        return Problem.make(T, d, E, k, I, I_s, act, w)

    def _reserve(self, T):
        n = workspace_size(self.problem(T))
        if self.ws is None or self.ws.numel() < n:
            self.ws = torch.empty(n, dtype=torch.uint8, device=self.device)

    def __call__(self, x, y=None, topk_ids=None, topk_w=None, stream=None):
        prob = self.problem(x.shape[0])
        _need_tokens(prob, x, y, topk_ids, topk_w)
        self._reserve(x.shape[0])
        w_router, bias, wg, wu, wd, s_wg, s_wu, s_wd, scales = self.w
        norm_weight, norm_eps, shared_gate = self.opts
        block = norm_weight is not None or shared_gate is not None
        return _forward(prob, x, w_router, bias, wg, wu, wd, s_wg, s_wu, s_wd, scales, norm_weight, norm_eps,
                        shared_gate, y, topk_ids, topk_w, self.ws, stream, block)

    @classmethod
    def from_inputs(cls, inp, max_tokens=0):
        return cls(inp.d, inp.E, inp.k, inp.I, inp.I_s, inp.w_r, inp.wg, inp.wu, inp.wd, inp.s_wg, inp.s_wu,
                   inp.s_wd, bias=inp.bias, scales=inp.scales, act=inp.act, w=inp.w, max_tokens=max_tokens)
