"""Expert-parallel routed MoE layer: the experts are split over ranks, the tokens travel.

The pages deploy the layer expert-parallel: EP8 with 16 of the 128 experts on each rank
(cann-recipes-infer "Gemma-4-26B-A4B 模型优化报告", §3 部署), with a double_routing AllToAll
that sends every rank the rows of its experts by the per-expert "split sizes" and a
local-expert AllReduce for decode (§6.1 方案).  Rank r holds experts [r E/G, (r+1) E/G) and
the (replicated) router.  Two ways of running one forward:

``alltoall`` (prefill; every rank brings its own tokens)
    1. route and dispatch the local tokens (library kernels);
    2. gather the routed rows in expert order (library kernel) -- the rows for rank r are then
       one contiguous block, since rank r's experts are contiguous ids;
    3. exchange the per-expert counts (AllToAll), then the rows (AllToAllv by the per-rank
       sums of those counts);
    4. run the grouped expert FFN on the received rows: one segment per (source rank, local
       expert), in the order they arrive (library kernel);
    5. send the outputs back (AllToAllv with the splits reversed): they return in the expert
       order of step 2;
    6. combine with the local weights (library kernel).

``allgather`` (decode; few tokens)
    1. AllGather the tokens of every rank;
    2. every rank routes and dispatches all of them (identically);
    3. each rank gathers and runs only the rows of its own experts;
    4. each rank combines only those rows into an fp32 partial sum (library kernel, rows
       outside its range add nothing), AllReduce sums the partials, and each rank keeps its
       own tokens' rows, rounded once to bf16.

Exchanges go through ``comm`` (``TorchComm``: torch.distributed, NCCL between GPUs); the
per-rank arithmetic goes through ``ops`` (``LibraryOps``: the C ABI of libmoe_b200.so).  Both
are parameters so that the same host logic can run between CPU processes in tests.  The
remote rows land in this rank's memory (NCCL's receive buffers) before any kernel of this
library loads them: no kernel reads another GPU's memory.
"""
from __future__ import annotations

import torch

from . import _abi


def expert_range(E: int, world: int, rank: int) -> tuple[int, int]:
    """Experts [lo, hi) held by `rank` (E divisible by the number of ranks)."""
    if E % world:
        raise ValueError(f"{E} experts do not split evenly over {world} ranks")
    per = E // world
    return rank * per, (rank + 1) * per


class TorchComm:
    """Exchanges over a torch.distributed process group (NCCL for CUDA tensors)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)

    def all_to_all_single(self, out, inp, out_splits, in_splits):
        self.dist.all_to_all_single(out, inp, out_splits, in_splits, group=self.group)

    def all_gather(self, inp):
        parts = [torch.empty_like(inp) for _ in range(self.world)]
        self.dist.all_gather(parts, inp, group=self.group)
        return torch.cat(parts, 0)

    def all_reduce_sum(self, t):
        self.dist.all_reduce(t, op=self.dist.ReduceOp.SUM, group=self.group)


class LibraryOps:
    """The per-rank steps, each one call of the library's C ABI.  Every instance owns its
    workspaces, so ranks that share a device (tests) never share scratch memory."""

    def __init__(self):
        self._ws: dict[str, torch.Tensor] = {}

    def _buf(self, name: str, nbytes: int, device) -> torch.Tensor:
        b = self._ws.get(name)
        if b is None or b.numel() < nbytes:
            b = torch.empty(max(nbytes, 1 << 16), dtype=torch.uint8, device=device)
            self._ws[name] = b
        return b

    def route(self, x, w_router, k, bias, renorm):
        L = _abi.load()
        n = L.moe_route_workspace_size(x.shape[0], x.shape[1], w_router.shape[1], k,
                                       0 if renorm else _abi.MOE_FLAG_NO_RENORM)
        return _abi.route(x, w_router, k, bias=bias, renorm=renorm,
                          workspace_buf=self._buf("route", n, x.device))

    def dispatch(self, ids, E):
        n = _abi.load().moe_dispatch_workspace_size(ids.shape[0], E, ids.shape[1])
        return _abi.dispatch(ids, E, workspace_buf=self._buf("dispatch", n, ids.device))

    def gather_rows(self, x, perm, k):
        return _abi.gather_rows(x, perm, k)

    def empty_rows(self, n, like):
        return torch.empty((n, like.shape[1]), dtype=torch.bfloat16, device=like.device)

    def expert_ffn(self, xs, seg_rows, seg_expert, w_gate, w_up, w_down, out=None):
        E, H, I = w_gate.shape
        n = _abi.load().moe_expert_ffn_workspace_size(xs.shape[0], H, E, I, seg_rows.numel())
        return _abi.expert_ffn(xs, seg_rows, seg_expert, w_gate, w_up, w_down, out=out,
                               workspace_buf=self._buf("ffn", n, xs.device))

    def combine(self, o, inv, w, row_lo=0, row_hi=None, fp32=False):
        return _abi.combine(o, inv, w, row_lo, row_hi, fp32=fp32)

    def to_output(self, y32):
        return y32.to(torch.bfloat16)


class ExpertParallelMoE:
    """One routed MoE layer with this rank's share of the experts.

    w_router [H, E] (every rank holds it), w_gate / w_up [E/G, H, I] and w_down [E/G, I, H]:
    the experts expert_range(E, G, rank) of the full layer.  forward(x) takes this rank's
    tokens x [T, H] and returns their y [T, H]; every rank must call it (collectively) with
    the same mode, and in "allgather" mode with the same T."""

    def __init__(self, w_router, w_gate, w_up, w_down, E: int, k: int, comm, bias=None,
                 renorm: bool = True, ops=None):
        self.w_router, self.w_gate, self.w_up, self.w_down = w_router, w_gate, w_up, w_down
        self.E, self.k, self.comm, self.bias, self.renorm = E, k, comm, bias, renorm
        self.ops = LibraryOps() if ops is None else ops
        self.lo, self.hi = expert_range(E, comm.world, comm.rank)
        self.El = self.hi - self.lo
        if w_gate.shape[0] != self.El:
            raise ValueError(f"rank {comm.rank} must hold {self.El} experts, got {w_gate.shape[0]}")

    # ---------------------------------------------------------------- prefill: AllToAllv
    def forward_alltoall(self, x):
        ops, comm, G, El, k = self.ops, self.comm, self.comm.world, self.El, self.k
        ids, w = ops.route(x, self.w_router, k, self.bias, self.renorm)
        counts, offsets, perm, inv = ops.dispatch(ids, self.E)
        xp = ops.gather_rows(x, perm, k)                     # rows in expert order
        # split sizes: rows for each rank, and per-expert counts for the receivers' segments
        cnt = counts.cpu()
        send = [int(cnt[r * El:(r + 1) * El].sum()) for r in range(G)]
        recv_cnt = torch.empty_like(counts)
        comm.all_to_all_single(recv_cnt, counts, [El] * G, [El] * G)
        rc = recv_cnt.cpu()
        recv = [int(rc[s * El:(s + 1) * El].sum()) for s in range(G)]
        xr = xp.new_empty((sum(recv), xp.shape[1]))
        comm.all_to_all_single(xr, xp, recv, send)
        # segments in arrival order: (source rank s, local expert e) with rc[s, e] rows
        seg_expert = torch.arange(El, dtype=torch.int32).repeat(G).to(counts.device)
        o_r = ops.expert_ffn(xr, recv_cnt, seg_expert, self.w_gate, self.w_up, self.w_down)
        o = o_r.new_empty((xp.shape[0], o_r.shape[1]))
        comm.all_to_all_single(o, o_r, send, recv)           # back in expert order
        return ops.combine(o, inv, w)

    # ---------------------------------------------------------------- decode: AllGather
    def forward_allgather(self, x):
        ops, comm, k = self.ops, self.comm, self.k
        T = x.shape[0]
        x_all = comm.all_gather(x)
        ids, w = ops.route(x_all, self.w_router, k, self.bias, self.renorm)
        counts, offsets, perm, inv = ops.dispatch(ids, self.E)
        off = offsets.cpu()
        r_lo, r_hi = int(off[self.lo]), int(off[self.hi])   # sorted rows of this rank's experts
        seg_expert = torch.arange(self.El, dtype=torch.int32).to(counts.device)
        o = ops.empty_rows(x_all.shape[0] * k, x_all)          # rows [r_lo, r_hi) used
        if r_hi > r_lo:
            xp = ops.gather_rows(x_all, perm[r_lo:r_hi], k)
            ops.expert_ffn(xp, counts[self.lo:self.hi].contiguous(), seg_expert, self.w_gate,
                           self.w_up, self.w_down, out=o[r_lo:r_hi])
        y = ops.combine(o, inv, w, r_lo, r_hi, fp32=True)   # this rank's experts only
        comm.all_reduce_sum(y)
        return ops.to_output(y[comm.rank * T:(comm.rank + 1) * T])

    def forward(self, x, mode: str = "alltoall"):
        if mode == "alltoall":
            return self.forward_alltoall(x)
        if mode == "allgather":
            return self.forward_allgather(x)
        raise ValueError("mode must be 'alltoall' or 'allgather'")
