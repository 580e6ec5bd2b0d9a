"""Stage calls with the package's signatures, computed by the oracle on the CPU.

Test infrastructure only: the expert-parallel layer (sparse_moe_layer_top_b200.ep)
takes its stage calls from an ``ops`` namespace, so the multi-rank exchange
logic can run as gloo ranks on CPU with these in place of the CUDA library.
Results are cast back to the activation type at every stage boundary, as the
library's stages store them."""
import numpy as np
import torch

import oracle
import sparse_moe_layer_top_b200 as moe

Problem = moe.Problem


def router_topk(prob, x, w_router, bias=None, **_):
    _, ids, w = oracle.router(x, w_router, prob.k, bias=bias)
    return torch.from_numpy(ids.astype(np.int32)), torch.from_numpy(w.astype(np.float32))


def permute(prob, x, topk_ids, topk_w, **_):
    offs, row_tok, _, pos = oracle.permute(topk_ids.numpy(), prob.E)
    R = prob.T * prob.k
    rows = R + (prob.T if prob.I_s > 0 else 0)
    offs[prob.E + 1] = rows  # no shared group without a shared expert, as the library writes it
    tok = torch.from_numpy(row_tok[:rows].astype(np.int64))
    return dict(x_perm=x[tok].contiguous(), row_tok=torch.from_numpy(row_tok[:rows]),
                pos=torch.from_numpy(pos), offs=torch.from_numpy(offs))


def expert_ffn(prob, x_perm, offs, wg, wu, wd, s_wg=None, s_wu=None, s_wd=None, scales=None, y_perm=None, **_):
    o_np = offs.numpy() if torch.is_tensor(offs) else np.asarray(offs, np.int32)
    out = torch.from_numpy(oracle.expert_ffn(x_perm, o_np, wg, wu, wd, s_wg, s_wu, s_wd, scales)).to(x_perm.dtype)
    if y_perm is None:
        y_perm = torch.zeros_like(out)
    o = offs.tolist() if torch.is_tensor(offs) else list(offs)
    a, b = int(o[0]), int(o[-1])  # the library writes only the rows of the groups
    y_perm[a:b] = out[a:b]
    return y_perm


def combine(prob, y_perm, pos, topk_w, offs, **_):
    y = oracle.combine(y_perm, pos.numpy(), topk_w.numpy(), offs.numpy(), prob.E)
    return torch.from_numpy(y).to(y_perm.dtype)


def ep_expand_ids(counts, G, E_local, R, **_):
    c = counts.numpy().astype(np.int64)
    ids = np.repeat(np.tile(np.arange(E_local, dtype=np.int32), G), c)
    assert ids.size == R
    return torch.from_numpy(ids)
