"""Expert parallelism: the host logic of expert_routed_ffn_softmax_b200.ep.

CPU (gloo, 2 ranks): every per-rank step is done by the fp64 oracle (route, dispatch, one
expert on one row, weighted sum), so these tests check only the exchange logic -- split
sizes, the count and row AllToAlls, the segments in arrival order, the reverse exchange,
the partial-sum AllReduce -- against the oracle's single-process forward, to fp64 rounding.

GPU (one device, ranks emulated by threads that exchange through host-side copies; no kernel
waits on another): the library's kernels do every step.  The AllToAll form must give the
single-GPU forward's bytes (every output row is the same sum in the same order, and the
combine adds the same rows in the same order); the AllGather form sums fp32 partials across
ranks, so it is held to the layer's tolerance against the oracle.
"""
import os
import socket
import threading

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from expert_routed_ffn_softmax_b200 import ep
from expert_routed_ffn_softmax_b200 import workloads as wl


class OracleOps:
    """The per-rank steps in fp64 by the oracle (test stand-in for the library)."""

    def route(self, x, w_router, k, bias, renorm):
        ids, w, _ = oracle.route(x, w_router, k, bias=bias, renorm=renorm)
        return torch.from_numpy(ids), torch.from_numpy(w)

    def dispatch(self, ids, E):
        return tuple(torch.from_numpy(a) for a in oracle.dispatch(ids.numpy(), E))

    def gather_rows(self, x, perm, k):
        return x[perm.long() // k].contiguous()

    def empty_rows(self, n, like):
        return torch.zeros((n, like.shape[1]), dtype=torch.float64)

    def expert_ffn(self, xs, seg_rows, seg_expert, w_gate, w_up, w_down, out=None):
        o = torch.zeros((xs.shape[0], xs.shape[1]), dtype=torch.float64) if out is None else out
        r = 0
        for n, e in zip(seg_rows.tolist(), seg_expert.tolist()):
            for i in range(n):
                o[r + i] = torch.from_numpy(oracle.expert_ffn(xs[r + i], w_gate, w_up, w_down, e))
            r += n
        return o

    def combine(self, o, inv, w, row_lo=0, row_hi=None, fp32=False):
        T, k = w.shape
        hi = T * k if row_hi is None else row_hi
        y = torch.zeros((T, o.shape[1]), dtype=torch.float64)
        for t in range(T):
            for j in range(k):
                p = int(inv[t * k + j])
                if row_lo <= p < hi:
                    y[t] += float(w[t, j]) * o[p]
        return y

    def to_output(self, y):
        return y


def test_expert_range_partition():
    assert [ep.expert_range(128, 8, r) for r in (0, 7)] == [(0, 16), (112, 128)]
    covered = sorted(e for r in range(4) for e in range(*ep.expert_range(8, 4, r)))
    assert covered == list(range(8))
    with pytest.raises(ValueError):
        ep.expert_range(10, 4, 0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_rank(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = wl.CONFIGS["tiny"]
        w = wl.make_weights(cfg, seed=1)
        lo, hi = ep.expert_range(cfg.E, world, rank)
        x = wl.make_x(cfg, seed=10 + rank, T=6)
        bias = wl.skew_bias(cfg.E)
        layer = ep.ExpertParallelMoE(w["w_router"], w["w_gate"][lo:hi].contiguous(),
                                     w["w_up"][lo:hi].contiguous(),
                                     w["w_down"][lo:hi].contiguous(), cfg.E, cfg.k,
                                     ep.TorchComm(), bias=bias, ops=OracleOps())
        ref = oracle.forward(x, w["w_router"], w["w_gate"], w["w_up"], w["w_down"], cfg.k,
                             bias=bias)["y"]
        res = {}
        for mode in ("alltoall", "allgather"):
            y = layer.forward(x, mode).numpy()
            res[mode] = float(np.max(np.abs(y - ref)))
        out[rank] = res
    finally:
        dist.destroy_process_group()


def test_ep_two_gloo_ranks_match_the_oracle():
    """Two CPU ranks, 4 experts each, 6 tokens each, skewed router bias (so the two ranks
    send each other different numbers of rows): both forms give the oracle's y."""
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_gloo_rank, args=(world, _free_port(), out), nprocs=world,
                           start_method="spawn", join=True)
        res = dict(out)
    for r in range(world):
        assert res[r]["alltoall"] == 0.0, res        # same sums in the same order
        assert res[r]["allgather"] <= 1e-12, res     # partial sums added across ranks


class ThreadComm:
    """Ranks as threads of one process: exchanges through host-side lists and copies."""

    def __init__(self, world, rank, shared):
        self.world, self.rank, self.sh = world, rank, shared

    def _exchange(self, obj):
        self.sh["slots"][self.rank] = obj
        self.sh["barrier"].wait()
        got = list(self.sh["slots"])
        self.sh["barrier"].wait()
        return got

    def all_to_all_single(self, out, inp, out_splits, in_splits):
        torch.cuda.synchronize()
        got = self._exchange(list(torch.split(inp, in_splits)))
        out.copy_(torch.cat([got[s][self.rank] for s in range(self.world)]))
        torch.cuda.synchronize()

    def all_gather(self, inp):
        torch.cuda.synchronize()
        return torch.cat(self._exchange(inp), 0)

    def all_reduce_sum(self, t):
        torch.cuda.synchronize()
        got = self._exchange(t.clone())
        acc = got[0].clone()
        for g in got[1:]:
            acc += g
        t.copy_(acc)
        torch.cuda.synchronize()


def _run_threads(world, fn):
    shared = {"slots": [None] * world, "barrier": threading.Barrier(world, timeout=120)}
    res, errs = [None] * world, []

    def body(r):
        try:
            torch.cuda.set_device(0)
            res[r] = fn(r, ThreadComm(world, r, shared))
        except BaseException as exc:   # noqa: BLE001 -- reported below
            errs.append(exc)
            shared["barrier"].abort()

    th = [threading.Thread(target=body, args=(r,)) for r in range(world)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    if errs:
        raise errs[0]
    return res


@pytest.mark.gpu
@pytest.mark.parametrize("world", [2, 4])
def test_ep_emulated_ranks_on_one_gpu(world):
    """Gemma-shaped layer (128 experts, top-8) split over 2 or 4 ranks: 48 tokens per rank
    through the AllToAll form, 8 tokens per rank through the AllGather (decode) form."""
    import expert_routed_ffn_softmax_b200 as moe
    cfg = wl.CONFIGS["decode"]
    w = wl.make_weights(cfg)
    g = {k: v.cuda() for k, v in w.items() if v is not None}
    xs = {r: wl.make_x(cfg, seed=20 + r, T=48) for r in range(world)}

    def rank_fn(r, comm):
        lo, hi = ep.expert_range(cfg.E, world, r)
        layer = ep.ExpertParallelMoE(g["w_router"], g["w_gate"][lo:hi].contiguous(),
                                     g["w_up"][lo:hi].contiguous(),
                                     g["w_down"][lo:hi].contiguous(), cfg.E, cfg.k, comm)
        y_a2a = layer.forward(xs[r].cuda(), "alltoall")
        y_ag = layer.forward(xs[r][:8].contiguous().cuda(), "allgather")
        torch.cuda.synchronize()
        return y_a2a, y_ag

    out = _run_threads(world, rank_fn)
    assert moe.sync_status() == 0
    for r in range(world):
        y_a2a, y_ag = out[r]
        y_one = moe.forward(xs[r].cuda(), g["w_router"], g["w_gate"], g["w_up"], g["w_down"],
                            cfg.k)
        assert torch.equal(y_a2a, y_one)
        ref = oracle.forward(xs[r][:8], w["w_router"], w["w_gate"], w["w_up"], w["w_down"],
                             cfg.k)["y"]
        err = y_ag.float().cpu().numpy().astype(np.float64) - ref
        assert float(np.max(np.abs(err))) <= 2e-2
        assert float(np.linalg.norm(err) / np.linalg.norm(ref)) <= 1e-2
