"""Expert parallelism: the sparse MoE block over G ranks, one process per GPU.

Rank g holds the contiguous experts [g * E_l, (g + 1) * E_l) (E_l = E / G) and
a replica of the router and of the shared expert; every rank routes its own
tokens.  One forward:

1. ``router_topk`` and ``permute`` over all E experts: the dispatch is a stable
   sort by expert, so the rows bound for rank g are the contiguous groups
   g * E_l .. (g + 1) * E_l - 1 of ``x_perm``;
2. the per-expert row counts, then the rows, go to their ranks
   (``all_to_all_single``);
3. on the receiving rank, ``ep_expand_ids`` gives each received row its local
   expert, a k = 1 ``permute`` groups the rows by expert across sources,
   ``expert_ffn`` runs the local experts, and a k = 1 ``combine`` with weight 1
   puts the results back in arrival order (exact: one value times 1);
4. the results travel back (the reverse exchange) into the routed rows of a
   [T * k (+ T), d] buffer whose shared rows the shared expert fills locally
   (``expert_ffn`` with every routed group empty);
5. ``combine`` applies the routing weights and adds the shared row.

Every arithmetic step runs in the library's kernels (through ``ops``, the
package's own calls by default).  This module moves rows between ranks
(``torch.distributed``: NCCL over NVLink on GPUs) and keeps the host-side
books: split sizes need the counts on the host, one small device-to-host copy
of the dispatch offsets and one of the received counts per forward.

The pages describe the block on one device and raise the number of GPUs only
as a chapter title (Fondations page, chapter 06, "how many GPUs for how many
parameters"); the split by contiguous expert blocks is ours.
"""
from dataclasses import dataclass, field
from typing import List, Optional

import torch


class TorchExchange:
    """Row exchange over a ``torch.distributed`` process group."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self._dist = dist
        self.group = group

    def rank(self):
        return self._dist.get_rank(self.group)

    def world(self):
        return self._dist.get_world_size(self.group)

    def all_to_all(self, out, inp, out_splits, in_splits):
        self._dist.all_to_all_single(out, inp, list(out_splits), list(in_splits), group=self.group)


@dataclass
class EPState:
    """What one rank keeps between the steps of a forward."""
    T: int
    prob: object
    x_perm: torch.Tensor
    pos: Optional[torch.Tensor]
    offs: Optional[torch.Tensor]
    ids: Optional[torch.Tensor]
    tw: Optional[torch.Tensor]
    send_counts: List[int]          # rows per expert, all E experts (host)
    send_rows: List[int]            # rows per destination rank (host)
    y_full: torch.Tensor            # [T * k (+ T), d]: routed rows come back, shared rows computed here
    recv_counts: List[int] = field(default_factory=list)  # [G * E_l]: rows from source s for local expert e
    recv_rows: List[int] = field(default_factory=list)    # rows per source rank


class EPMoELayer:
    """One rank's share of an expert-parallel MoE block.

    w_router [E, d] and the shared expert are full replicas; wg, wu [E_l, I, d]
    and wd [E_l, d, I] are this rank's experts, E_l = E / world.  With E4M3
    weights (w="fp8"), ``scales`` is this rank's packed block-scale buffer
    (``split_scales``).  ``ops`` is the namespace of stage calls (default: this
    package)."""

    def __init__(self, rank, world, d, E, k, I, I_s, w_router, wg, wu, wd, s_wg=None, s_wu=None, s_wd=None,
                 bias=None, act="bf16", w="bf16", ops=None, scales=None):
        if world < 1 or not 0 <= rank < world:
            raise ValueError("rank %d of %d" % (rank, world))
        if E % world:
            raise ValueError("E = %d experts do not split over %d ranks" % (E, world))
        if ops is None:
            import sparse_moe_layer_top_b200 as ops
        self.ops = ops
        self.rank, self.world = rank, world
        self.d, self.E, self.k, self.I, self.I_s = d, E, k, I, I_s
        self.E_l = E // world
        if wg.shape[0] != self.E_l or wu.shape[0] != self.E_l or wd.shape[0] != self.E_l:
            raise ValueError("rank weights must hold E / world = %d experts" % self.E_l)
        if w == "fp8":
            n = _scale_blocks(self.E_l, d, I, I_s)
            if scales is None or scales.numel() != n:
                raise ValueError("E4M3 weights need this rank's %d block scales (split_scales)" % n)
        elif scales is not None:
            raise ValueError("block scales are for E4M3 weights only")
        self.scales = scales
        self.w_router, self.bias = w_router, bias
        self.wg, self.wu, self.wd = wg, wu, wd
        self.s_wg, self.s_wu, self.s_wd = s_wg, s_wu, s_wd
        self.act, self.wdt = act, w

    def _prob(self, T, E, k, I_s):
        return self.ops.Problem.make(T, self.d, E, k, self.I, I_s, self.act, self.wdt)

    # -------------------------------------------------------------- step 1
    def dispatch(self, x):
        T = int(x.shape[0])
        R = T * self.k
        rows = R + (T if self.I_s > 0 else 0)
        prob = self._prob(T, self.E, self.k, self.I_s)
        y_full = torch.empty((rows, self.d), dtype=x.dtype, device=x.device)
        if T == 0:
            z = [0] * self.E
            return EPState(0, prob, x.new_empty((0, self.d)), None, None, None, None, z, [0] * self.world, y_full)
        ids, tw = self.ops.router_topk(prob, x, self.w_router, self.bias)
        perm = self.ops.permute(prob, x, ids, tw)
        offs = perm["offs"].cpu().tolist()
        counts = [offs[e + 1] - offs[e] for e in range(self.E)]
        send_rows = [sum(counts[g * self.E_l:(g + 1) * self.E_l]) for g in range(self.world)]
        return EPState(T, prob, perm["x_perm"], perm["pos"], perm["offs"], ids, tw, counts, send_rows, y_full)

    # -------------------------------------------------------------- step 3
    def set_received(self, st, recv_counts):
        """recv_counts: [G * E_l] host ints (rows from source s for local expert e)."""
        st.recv_counts = [int(c) for c in recv_counts]
        st.recv_rows = [sum(st.recv_counts[s * self.E_l:(s + 1) * self.E_l]) for s in range(self.world)]

    def experts(self, st, x_recv):
        """The local experts on the received rows, results in arrival order."""
        R_recv = int(x_recv.shape[0])
        if R_recv == 0:
            return x_recv.new_empty((0, self.d))
        counts = torch.tensor(st.recv_counts, dtype=torch.int32, device=x_recv.device)
        ids = self.ops.ep_expand_ids(counts, self.world, self.E_l, R_recv).reshape(R_recv, 1)
        ones = torch.ones((R_recv, 1), dtype=torch.float32, device=x_recv.device)
        prob = self._prob(R_recv, self.E_l, 1, 0)
        perm = self.ops.permute(prob, x_recv, ids, ones)
        y_perm = self.ops.expert_ffn(prob, perm["x_perm"], perm["offs"], self.wg, self.wu, self.wd,
                                     scales=self.scales)
        return self.ops.combine(prob, y_perm, perm["pos"], ones, perm["offs"])

    # -------------------------------------------------------------- step 4
    def shared(self, st):
        """The shared expert on this rank's tokens, into the shared rows of y_full.

        Run as a k = 1 problem over the last 2T rows of x_perm: T routed rows
        (every routed group empty, so neither read nor written) and the T shared
        rows; the output is the same window of y_full, so only its shared rows
        are written."""
        if self.I_s == 0 or st.T == 0:
            return
        T, R = st.T, st.T * self.k
        offs = torch.tensor([T] * (self.E_l + 1) + [2 * T], dtype=torch.int32, device=st.x_perm.device)
        prob = self._prob(T, self.E_l, 1, self.I_s)
        self.ops.expert_ffn(prob, st.x_perm[R - T:R + T], offs, self.wg, self.wu, self.wd, self.s_wg, self.s_wu,
                            self.s_wd, scales=self.scales, y_perm=st.y_full[R - T:R + T])

    # -------------------------------------------------------------- step 5
    def combine(self, st):
        if st.T == 0:
            return st.y_full.new_empty((0, self.d))
        return self.ops.combine(st.prob, st.y_full, st.pos, st.tw, st.offs)

    # -------------------------------------------------------------- all steps
    def forward(self, x, exchange):
        """y [T, d] for this rank's tokens x [T, d]; every rank calls it together."""
        st = self.dispatch(x)
        dev = x.device
        sc = torch.tensor(st.send_counts, dtype=torch.int32, device=dev)
        rc = torch.empty(self.world * self.E_l, dtype=torch.int32, device=dev)
        exchange.all_to_all(rc, sc, [self.E_l] * self.world, [self.E_l] * self.world)
        self.set_received(st, rc.cpu().tolist())
        R = st.T * self.k
        x_recv = torch.empty((sum(st.recv_rows), self.d), dtype=x.dtype, device=dev)
        exchange.all_to_all(x_recv, st.x_perm[:R], st.recv_rows, st.send_rows)
        self.shared(st)
        y_recv = self.experts(st, x_recv)
        exchange.all_to_all(st.y_full[:R], y_recv, st.send_rows, st.recv_rows)
        return self.combine(st)

    __call__ = forward


def split_experts(rank, world, wg, wu, wd):
    """This rank's block of the [E, ...] expert weights (contiguous views)."""
    E = wg.shape[0]
    E_l = E // world
    sl = slice(rank * E_l, (rank + 1) * E_l)
    return wg[sl].contiguous(), wu[sl].contiguous(), wd[sl].contiguous()


def _scale_blocks(E, d, I, I_s):
    """Length of the packed E4M3 scale buffer: gate, up and down of E experts,
    then the shared expert's three, one scale per 128 x 128 block each."""
    per = (I // 128) * (d // 128)
    return 3 * E * per + (3 * (I_s // 128) * (d // 128) if I_s > 0 else 0)


def split_scales(rank, world, E, d, I, I_s, scales):
    """This rank's packed E4M3 block scales from the whole block's buffer: the
    gate, up and down scales of its experts, then the shared expert's
    (replicated), in the same packed order as the whole buffer."""
    if scales.numel() != _scale_blocks(E, d, I, I_s):
        raise ValueError("scales hold %d values, not the %d of the whole block"
                         % (scales.numel(), _scale_blocks(E, d, I, I_s)))
    E_l = E // world
    per = (I // 128) * (d // 128)
    lo, hi = rank * E_l * per, (rank + 1) * E_l * per
    flat = scales.reshape(-1)
    parts = [flat[m * E * per:(m + 1) * E * per][lo:hi] for m in range(3)] + [flat[3 * E * per:]]
    return torch.cat(parts).contiguous()
