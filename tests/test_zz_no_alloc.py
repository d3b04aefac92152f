"""moe_route_static: the router entry point that allocates nothing.

Some callers cannot hand the library a workspace: code running while a stream is captured
into a CUDA graph (no cudaMalloc there), plugin hosts that pass a kernel only its inputs and
outputs, runtimes with a fixed memory budget.  For them moe_route_static keeps its scratch
in an array compiled into the library.  This checks, through the C ABI, that two calls in a
row give the same ids (bit for bit) and weights (within 1e-5) as moe_route with its own
workspace, and that a batch whose scratch does not fit is refused.

The file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import expert_routed_ffn_softmax_b200 as moe
from expert_routed_ffn_softmax_b200 import _abi
from expert_routed_ffn_softmax_b200 import workloads as wl

pytestmark = pytest.mark.gpu

W_ABS = 1e-5


def _static_route(lib, x, wr, bias, k):
    T, H = x.shape
    E = wr.shape[1]
    ids = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    wts = torch.full((T, k), -1.0, dtype=torch.float32, device="cuda")
    rc = lib.moe_route_static(x.data_ptr(), wr.data_ptr(), None if bias is None else bias.data_ptr(),
                              T, H, E, k, 0, ids.data_ptr(), wts.data_ptr(),
                              torch.cuda.current_stream().cuda_stream)
    return rc, ids, wts


@pytest.mark.parametrize("name,T", [("decode", 8), ("decode", 128), ("tiny", 16)])
def test_static_scratch_route_matches_workspace_route(name, T):
    cfg = wl.CONFIGS[name]
    w = wl.make_weights(cfg)
    x = wl.make_x(cfg, seed=5, T=T).cuda()
    wr = w["w_router"].cuda()
    ids_ref, w_ref = moe.route(x, wr, cfg.k, router="fp64")
    assert moe.sync_status() == 0
    lib = moe.load()
    for _ in range(2):                      # the shared array keeps the previous contents
        rc, ids, wts = _static_route(lib, x, wr, None, cfg.k)
        assert rc == _abi.MOE_OK, moe.status_string(rc)
        assert moe.sync_status() == 0
        assert torch.equal(ids, ids_ref)
        assert float((wts - w_ref).abs().max()) <= W_ABS


def test_static_scratch_refuses_batches_that_do_not_fit():
    cfg = wl.CONFIGS["decode"]
    lib = moe.load()
    x = torch.zeros((4096, cfg.H), dtype=torch.bfloat16, device="cuda")
    wr = torch.zeros((cfg.H, cfg.E), dtype=torch.bfloat16, device="cuda")
    rc, _, _ = _static_route(lib, x, wr, None, cfg.k)
    assert rc == _abi.MOE_ERR_NO_WORKSPACE
