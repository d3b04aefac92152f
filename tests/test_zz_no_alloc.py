"""moe_route_static: the router entry point that allocates nothing.

Some callers cannot hand the library a workspace: code running while a stream is captured
into a CUDA graph (no cudaMalloc there), plugin hosts that pass a kernel only its inputs and
outputs, runtimes with a fixed memory budget.  For them moe_route_static keeps its scratch
in an array compiled into the library.  This checks, through the C ABI, on two calls in a
row (the shared array keeps the previous call's contents), that its ids are the fp64
oracle's bit for bit and its weights within 1e-5 of the oracle's -- with and without a
router bias, with and without renormalisation -- that they equal moe_route's with its own
workspace, and that a batch whose scratch does not fit is refused.

The file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import oracle
import expert_routed_ffn_softmax_b200 as moe
from expert_routed_ffn_softmax_b200 import _abi
from expert_routed_ffn_softmax_b200 import workloads as wl

pytestmark = pytest.mark.gpu

W_ABS = 1e-5


def _static_route(lib, x, wr, bias, k, flags=0):
    T, H = x.shape
    E = wr.shape[1]
    ids = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    wts = torch.full((T, k), -1.0, dtype=torch.float32, device="cuda")
    rc = lib.moe_route_static(x.data_ptr(), wr.data_ptr(), None if bias is None else bias.data_ptr(),
                              T, H, E, k, flags, ids.data_ptr(), wts.data_ptr(),
                              torch.cuda.current_stream().cuda_stream)
    return rc, ids, wts


CASES = [("decode", 8, False, True), ("decode", 128, False, True), ("tiny", 16, False, True),
         ("decode", 64, True, True), ("decode", 8, False, False), ("tiny", 16, True, False)]


@pytest.mark.parametrize("name,T,bias,renorm", CASES,
                         ids=[f"{n}_T{t}{'_bias' if b else ''}{'' if r else '_norenorm'}"
                              for n, t, b, r in CASES])
def test_static_scratch_route_matches_oracle(name, T, bias, renorm):
    cfg = wl.CONFIGS[name]
    w = wl.make_weights(cfg)
    x_cpu = wl.make_x(cfg, seed=5, T=T)
    b_cpu = wl.skew_bias(cfg.E) if bias else None
    r_ids, r_w, _ = oracle.route(x_cpu, w["w_router"], cfg.k, bias=b_cpu, renorm=renorm)
    x = x_cpu.cuda()
    wr = w["w_router"].cuda()
    b = None if b_cpu is None else b_cpu.cuda()
    ids_ws, w_ws = moe.route(x, wr, cfg.k, bias=b, renorm=renorm, router="fp64")
    assert moe.sync_status() == 0
    lib = moe.load()
    flags = 0 if renorm else _abi.MOE_FLAG_NO_RENORM
    for _ in range(2):                      # the shared array keeps the previous contents
        rc, ids, wts = _static_route(lib, x, wr, b, cfg.k, flags)
        assert rc == _abi.MOE_OK, moe.status_string(rc)
        assert moe.sync_status() == 0
        assert np.array_equal(ids.cpu().numpy(), r_ids)
        assert float(np.max(np.abs(wts.cpu().numpy().astype(np.float64) - r_w))) <= W_ABS
        assert torch.equal(ids, ids_ws)
        assert float((wts - w_ws).abs().max()) <= W_ABS


def test_static_scratch_refuses_batches_that_do_not_fit():
    cfg = wl.CONFIGS["decode"]
    lib = moe.load()
    x = torch.zeros((4096, cfg.H), dtype=torch.bfloat16, device="cuda")
    wr = torch.zeros((cfg.H, cfg.E), dtype=torch.bfloat16, device="cuda")
    rc, _, _ = _static_route(lib, x, wr, None, cfg.k)
    assert rc == _abi.MOE_ERR_NO_WORKSPACE
