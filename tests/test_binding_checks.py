"""The Python binding's argument checks, on the host.

The C ABI takes bare pointers, so a tensor of the wrong element type or too
few elements would have the kernels read or write past its end.  Every
binding call checks its tensors against the problem before it takes a
pointer.  Here the tensors are on the CPU: a call whose arguments pass the
checks stops at the pointer step ("must be on a CUDA device"), and a call with
a bad argument stops earlier, naming that argument."""
import pytest
import torch

import sparse_moe_layer_top_b200 as moe

ON_DEVICE = "must be on a CUDA device"


def _forward_args(act="bf16", w="bf16", T=20, d=256, E=6, k=2, I=128, I_s=128):
    at = torch.float32 if act == "f32" else torch.bfloat16
    wt = {"f32": torch.float32, "bf16": torch.bfloat16, "fp8": torch.float8_e4m3fn}[w]
    a = dict(prob=moe.Problem.make(T, d, E, k, I, I_s, act, w),
             x=torch.zeros((T, d), dtype=at), w_router=torch.zeros((E, d), dtype=at),
             bias=torch.zeros(E), wg=torch.zeros((E, I, d)).to(wt), wu=torch.zeros((E, I, d)).to(wt),
             wd=torch.zeros((E, d, I)).to(wt), s_wg=None, s_wu=None, s_wd=None, scales=None,
             y=torch.zeros((T, d), dtype=at), topk_ids=torch.zeros((T, k), dtype=torch.int32),
             topk_w=torch.zeros((T, k)))
    if I_s:
        a.update(s_wg=torch.zeros((I_s, d)).to(wt), s_wu=torch.zeros((I_s, d)).to(wt),
                 s_wd=torch.zeros((d, I_s)).to(wt))
    if w == "fp8":
        a["scales"] = torch.ones(3 * E * (I // 128) * (d // 128) + 3 * (I_s // 128) * (d // 128))
    return a


def _forward(a):
    return moe.layer_forward(a["prob"], a["x"], a["w_router"], a["bias"], a["wg"], a["wu"], a["wd"], a["s_wg"],
                             a["s_wu"], a["s_wd"], a["scales"], y=a["y"], topk_ids=a["topk_ids"],
                             topk_w=a["topk_w"])


@pytest.mark.parametrize("act,w,I_s", [("bf16", "bf16", 128), ("bf16", "fp8", 128), ("f32", "f32", 64),
                                       ("bf16", "bf16", 0), ("bf16", "fp8", 0)])
def test_well_formed_arguments_reach_the_pointer_step(act, w, I_s):
    a = _forward_args(act, w, I_s=I_s)
    with pytest.raises(ValueError, match=ON_DEVICE):
        _forward(a)
    with pytest.raises(ValueError, match=ON_DEVICE):
        moe.block_forward(a["prob"], a["x"], a["w_router"], a["bias"], a["wg"], a["wu"], a["wd"], a["s_wg"],
                          a["s_wu"], a["s_wd"], a["scales"], norm_weight=torch.zeros(256, dtype=a["x"].dtype),
                          shared_gate=torch.zeros(256, dtype=a["x"].dtype))


def _bad(name, value):
    def f(a):
        a[name] = value(a)
    return f


BAD_FORWARD = {
    "x of the wrong type": ("bf16", _bad("x", lambda a: a["x"].float()), "x: element type"),
    "x with too few rows": ("bf16", _bad("x", lambda a: a["x"][:-1]), "x: 4864 elements, the problem needs 5120"),
    "x with rows of the wrong width": ("bf16", _bad("x", lambda a: a["x"].reshape(40, 128)), "x: rows of 128"),
    "router weights too small": ("bf16", _bad("w_router", lambda a: a["w_router"][:5]), "w_router:"),
    "fp64 bias": ("bf16", _bad("bias", lambda a: a["bias"].double()), "router_bias: element type"),
    "bias too short": ("bf16", _bad("bias", lambda a: a["bias"][:5]), "router_bias:"),
    "gate weights transposed": ("bf16", _bad("wg", lambda a: a["wg"].transpose(1, 2).contiguous()),
                                "w_gate: rows of 128"),
    "down weights of one expert too few": ("bf16", _bad("wd", lambda a: a["wd"][:5]), "w_down:"),
    "bf16 weights for an fp8 problem": ("fp8", _bad("wu", lambda a: a["wu"].to(torch.bfloat16)),
                                        "w_up: element type"),
    "fp8 scales too short": ("fp8", _bad("scales", lambda a: a["scales"][:-1]), "scales:"),
    "fp8 scales in bf16": ("fp8", _bad("scales", lambda a: a["scales"].to(torch.bfloat16)), "scales: element type"),
    "shared down weights too small": ("bf16", _bad("s_wd", lambda a: a["s_wd"][:, :64].contiguous()), "ws_down:"),
    "output too small": ("bf16", _bad("y", lambda a: a["y"][:10]), "y:"),
    "int64 ids": ("bf16", _bad("topk_ids", lambda a: a["topk_ids"].long()), "topk_ids: element type"),
    "weights of the wrong width": ("bf16", _bad("topk_w", lambda a: torch.zeros((10, 4))), "topk_w: rows of 4"),
}


@pytest.mark.parametrize("case", list(BAD_FORWARD))
def test_a_bad_buffer_is_named_before_any_pointer_is_taken(case):
    w, mutate, msg = BAD_FORWARD[case]
    a = _forward_args("bf16", w)
    mutate(a)
    with pytest.raises(ValueError, match=msg):
        _forward(a)


def test_shared_weights_are_not_read_without_a_shared_expert():
    a = _forward_args(I_s=0)
    a.update(s_wg=torch.zeros(1), s_wu=torch.zeros(1, dtype=torch.int8), s_wd=torch.zeros(3))
    with pytest.raises(ValueError, match=ON_DEVICE):
        _forward(a)


def test_stage_calls_check_their_buffers():
    T, d, E, k, I, I_s = 20, 256, 6, 2, 128, 128
    prob = moe.Problem.make(T, d, E, k, I, I_s, "bf16", "bf16")
    bf = torch.bfloat16
    x = torch.zeros((T, d), dtype=bf)
    ids, tw = torch.zeros((T, k), dtype=torch.int32), torch.zeros((T, k))
    Rp = T * (k + 1)
    offs = torch.zeros(E + 2, dtype=torch.int32)
    wg, wd = torch.zeros((E, I, d), dtype=bf), torch.zeros((E, d, I), dtype=bf)
    sg, sd = torch.zeros((I_s, d), dtype=bf), torch.zeros((d, I_s), dtype=bf)

    with pytest.raises(ValueError, match="w_router:"):
        moe.router_topk(prob, x, torch.zeros((E, d - 8), dtype=bf))
    with pytest.raises(ValueError, match=ON_DEVICE):
        moe.router_topk(prob, x, torch.zeros((E, d), dtype=bf))

    with pytest.raises(ValueError, match="topk_w: element type"):
        moe.permute(prob, x, ids, tw.double())
    with pytest.raises(ValueError, match=ON_DEVICE):
        moe.permute(prob, x, ids, tw)

    # the expert stage reads and writes R' = T*k + T rows (shared group included)
    with pytest.raises(ValueError, match="x_perm: %d elements" % (T * k * d)):
        moe.expert_ffn(prob, torch.zeros((T * k, d), dtype=bf), offs, wg, wg, wd, sg, sg, sd)
    with pytest.raises(ValueError, match="offs:"):
        moe.expert_ffn(prob, torch.zeros((Rp, d), dtype=bf), offs[:E], wg, wg, wd, sg, sg, sd)
    with pytest.raises(ValueError, match="y_perm:"):
        moe.expert_ffn(prob, torch.zeros((Rp, d), dtype=bf), offs, wg, wg, wd, sg, sg, sd,
                       y_perm=torch.zeros((Rp - 1, d), dtype=bf))
    with pytest.raises(ValueError, match=ON_DEVICE):
        moe.expert_ffn(prob, torch.zeros((Rp, d), dtype=bf), offs, wg, wg, wd, sg, sg, sd)

    with pytest.raises(ValueError, match="pos: element type"):
        moe.combine(prob, torch.zeros((Rp, d), dtype=bf), ids.long(), tw, offs)
    with pytest.raises(ValueError, match="y_perm:"):
        moe.combine(prob, torch.zeros((T * k, d), dtype=bf), ids, tw, offs)
    with pytest.raises(ValueError, match=ON_DEVICE):
        moe.combine(prob, torch.zeros((Rp, d), dtype=bf), ids, tw, offs)

    with pytest.raises(ValueError, match="norm_weight:"):
        moe.rmsnorm(prob, x, torch.zeros(d - 1, dtype=bf))
    with pytest.raises(ValueError, match="norm_weight: element type"):
        moe.rmsnorm(prob, x, torch.zeros(d))
    with pytest.raises(ValueError, match=ON_DEVICE):
        moe.rmsnorm(prob, x, torch.zeros(d, dtype=bf))


def test_expert_parallel_receive_side_checks_its_buffers():
    with pytest.raises(ValueError, match="counts: element type"):
        moe.ep_expand_ids(torch.zeros(8, dtype=torch.int64), 2, 4, 10)
    with pytest.raises(ValueError, match="counts: 6 elements"):
        moe.ep_expand_ids(torch.zeros(6, dtype=torch.int32), 2, 4, 10)
    with pytest.raises(ValueError, match="ids: 9 elements"):
        moe.ep_expand_ids(torch.zeros(8, dtype=torch.int32), 2, 4, 10, ids=torch.zeros(9, dtype=torch.int32))
    with pytest.raises(ValueError, match=ON_DEVICE):
        moe.ep_expand_ids(torch.zeros(8, dtype=torch.int32), 2, 4, 10)


def test_layer_object_checks_its_weights_once_and_its_tokens_every_call():
    a = _forward_args("bf16", "fp8")
    p = a["prob"]
    args = (p.d, p.E, p.k, p.I, p.I_s, a["w_router"], a["wg"], a["wu"], a["wd"], a["s_wg"], a["s_wu"], a["s_wd"])
    with pytest.raises(ValueError, match="scales:"):
        moe.MoELayer(*args, bias=a["bias"], scales=a["scales"][:3], act="bf16", w="fp8")
    with pytest.raises(ValueError, match="shared_gate:"):
        moe.MoELayer(*args, bias=a["bias"], scales=a["scales"], act="bf16", w="fp8",
                     shared_gate=torch.zeros(p.d - 8, dtype=torch.bfloat16))
    layer = moe.MoELayer(*args, bias=a["bias"], scales=a["scales"], act="bf16", w="fp8")
    with pytest.raises(ValueError, match="x: element type"):
        layer(a["x"].float())
    with pytest.raises(ValueError, match="y:"):
        layer(a["x"], y=a["y"][:-1])
    with pytest.raises(ValueError, match=ON_DEVICE):
        layer(a["x"], y=a["y"], topk_ids=a["topk_ids"], topk_w=a["topk_w"])


def test_tensors_on_different_devices_are_rejected_before_any_pointer():
    """The library launches on the current device with the pointers it is
    given, so one call's tensors must share a device: a mix is refused,
    naming the tensors, before the pointer step (here a CPU tensor beside a
    meta tensor stands for cuda:0 beside cuda:1)."""
    a = _forward_args()
    a["w_router"] = a["w_router"].to("meta")
    with pytest.raises(ValueError, match="different devices.*w_router on meta"):
        _forward(a)
    a = _forward_args()
    p = a["prob"]
    with pytest.raises(ValueError, match="different devices"):
        moe.router_topk(p, a["x"], a["w_router"], None, topk_ids=a["topk_ids"].to("meta"))
    with pytest.raises(ValueError, match="different devices"):
        moe.combine(p, torch.zeros((p.T * (p.k + 1), p.d), dtype=torch.bfloat16), a["topk_ids"], a["topk_w"],
                    torch.zeros(p.E + 2, dtype=torch.int32), y=a["y"].to("meta"))
    layer = moe.MoELayer(p.d, p.E, p.k, 128, 128, a["w_router"], a["wg"], a["wu"], a["wd"], a["s_wg"], a["s_wu"],
                         a["s_wd"])
    with pytest.raises(ValueError, match="different devices"):
        layer(a["x"].to("meta"))
