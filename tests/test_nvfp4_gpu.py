"""NVFP4 experts on the GPU against the oracle.

Quantisers: the library's weight and activation quantisers take the same decisions as the
oracle's (codes, scales and tensor scales bit for bit).  Layer: moe_forward_nvfp4 with weights
quantised by the library against the oracle's NVFP4 layer with weights quantised by the oracle
(the same codes, by the first test): routing bit-exact, y within the layer's tolerance
(max-abs 2e-2, relative-L2 1e-2).  The only decisions that can differ are h's codes near a
rounding boundary (the GPU's h is an fp32 sum, the oracle's an exact one); they move y far
less than the tolerance.
"""
import numpy as np
import pytest
import torch

import oracle
import expert_routed_ffn_softmax_b200 as moe
from expert_routed_ffn_softmax_b200 import _abi
from expert_routed_ffn_softmax_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def unblock(scales: torch.Tensor, N: int, K: int) -> np.ndarray:
    """Blocked weight scales [E, ceil(N/128), K/64, 512] (include/moe.h) -> [E, N, K/16]; the
    padding rows N .. must hold 0."""
    b = scales.cpu().numpy()
    E = b.shape[0]
    n = np.arange(N)[:, None]
    g = np.arange(K // 16)[None, :]
    byte = 16 * (n % 32) + 4 * ((n % 128) // 32) + (g % 4)
    out = b[:, n // 128, g // 4, byte]
    pad = np.arange(N, b.shape[1] * 128)
    if pad.size:
        pb = 16 * (pad[:, None] % 32) + 4 * ((pad[:, None] % 128) // 32) + (g % 4)
        assert not b[:, pad[:, None] // 128, g // 4, pb].any()
    return out


def unpack(codes: torch.Tensor) -> np.ndarray:
    """Packed codes [..., K/2] (element 2b in the low nibble) -> one code per byte [..., K]."""
    b = codes.cpu().numpy()
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), np.uint8)
    out[..., 0::2] = b & 15
    out[..., 1::2] = b >> 4
    return out


@pytest.fixture(scope="module")
def gemma_fp4():
    cfg = wl.CONFIGS["decode"]
    w = wl.make_weights(cfg)
    q_gpu = _abi.nvfp4_quantize_layer(w["w_gate"].cuda(), w["w_up"].cuda(), w["w_down"].cuda())
    q_ref = oracle.quantize_expert_weights(w["w_gate"], w["w_up"], w["w_down"])
    assert moe.sync_status() == 0
    return w, q_gpu, q_ref


def check_weights(q_gpu, q_ref):
    for n in ("gate", "up", "down"):
        codes = unpack(q_gpu[f"{n}_codes"])
        assert np.array_equal(codes, q_ref[f"{n}_codes"]), n
        N, K = codes.shape[1], codes.shape[2]
        assert np.array_equal(unblock(q_gpu[f"{n}_scales"], N, K), q_ref[f"{n}_scales"]), n
        assert np.array_equal(q_gpu[f"{n}_ts"].cpu().numpy(), q_ref[f"{n}_ts"]), n


def test_weight_quantizer_matches_oracle(gemma_fp4):
    _, q_gpu, q_ref = gemma_fp4
    check_weights(q_gpu, q_ref)


def test_weight_quantizer_tiny_shape():
    cfg = wl.CONFIGS["tiny"]
    w = wl.make_weights(cfg, seed=2)
    q_gpu = _abi.nvfp4_quantize_layer(w["w_gate"].cuda(), w["w_up"].cuda(), w["w_down"].cuda())
    q_ref = oracle.quantize_expert_weights(w["w_gate"], w["w_up"], w["w_down"])
    check_weights(q_gpu, q_ref)


@pytest.mark.parametrize("ts", [1.0, 0.0078125, 0.37])
def test_rows_quantizer_matches_oracle(ts):
    x = wl.make_x(wl.CONFIGS["decode"], seed=9, T=16)
    x[3] = 0                                           # an all-zero row: scale 0, codes 0
    codes, scales = _abi.nvfp4_quantize_rows(x.cuda(), ts)
    assert moe.sync_status() == 0
    c_ref, s_ref = oracle.nvfp4_quantize(x.float().numpy(), ts)
    assert np.array_equal(unpack(codes), c_ref)
    assert np.array_equal(scales.cpu().numpy(), s_ref)


def check(y, aux, ref, E):
    assert np.array_equal(aux["topk_ids"].cpu().numpy(), ref["ids"])
    assert np.max(np.abs(aux["topk_weights"].cpu().numpy() - ref["weights"])) <= 1e-5
    counts, offsets, perm, _ = oracle.dispatch(ref["ids"], E)
    assert np.array_equal(aux["expert_counts"].cpu().numpy(), counts)
    assert np.array_equal(aux["perm"].cpu().numpy(), perm)
    err = y.float().cpu().numpy().astype(np.float64) - ref["y"]
    assert float(np.max(np.abs(err))) <= 2e-2
    assert float(np.linalg.norm(err) / np.linalg.norm(ref["y"])) <= 1e-2


@pytest.mark.parametrize("T,sx,sh", [(8, 1.0, 1.0), (1, 1.0, 1.0), (16, 0.0078125, 0.25),
                                     (5, 1.0, 1.0)])
def test_forward_nvfp4_parity_gemma(T, sx, sh, gemma_fp4):
    w, q_gpu, q_ref = gemma_fp4
    cfg = wl.CONFIGS["decode"]
    x = wl.make_x(cfg, seed=T, T=T)
    y, aux = _abi.forward_nvfp4(x.cuda(), w["w_router"].cuda(), q_gpu, cfg.k, act_scale_x=sx,
                                act_scale_h=sh, aux=True)
    assert moe.sync_status() == 0
    ref = oracle.forward_nvfp4(x, w["w_router"], q_ref, cfg.k, act_scale_x=sx, act_scale_h=sh)
    check(y, aux, ref, cfg.E)
    y2 = _abi.forward_nvfp4(x.cuda(), w["w_router"].cuda(), q_gpu, cfg.k, act_scale_x=sx,
                            act_scale_h=sh)
    assert torch.equal(y, y2)                          # deterministic


def test_forward_nvfp4_tiny_with_bias_and_no_renorm():
    cfg = wl.CONFIGS["tiny"]
    w = wl.make_weights(cfg, seed=3)
    q_gpu = _abi.nvfp4_quantize_layer(w["w_gate"].cuda(), w["w_up"].cuda(), w["w_down"].cuda())
    q_ref = oracle.quantize_expert_weights(w["w_gate"], w["w_up"], w["w_down"])
    x = wl.make_x(cfg, seed=3, T=16)
    bias = wl.skew_bias(cfg.E)
    for renorm in (True, False):
        y, aux = _abi.forward_nvfp4(x.cuda(), w["w_router"].cuda(), q_gpu, cfg.k,
                                    bias=bias.cuda(), renorm=renorm, aux=True)
        assert moe.sync_status() == 0
        ref = oracle.forward_nvfp4(x, w["w_router"], q_ref, cfg.k, bias=bias, renorm=renorm)
        check(y, aux, ref, cfg.E)


def test_forward_nvfp4_ragged_shape():
    """Shapes whose K stages and 128-row blocks do not divide evenly: H = 320 (GEMM-1 K in a
    full and a one-block stage, GEMM-2 columns in blocks of 128, 128, 64), I = 192 (GEMM-1
    features in blocks of 128 and 64, GEMM-2 K in 3 blocks)."""
    cfg = wl.MoEConfig("ragged", 5, 320, 8, 3, 192)
    w = wl.make_weights(cfg, seed=4)
    q_gpu = _abi.nvfp4_quantize_layer(w["w_gate"].cuda(), w["w_up"].cuda(), w["w_down"].cuda())
    q_ref = oracle.quantize_expert_weights(w["w_gate"], w["w_up"], w["w_down"])
    check_weights(q_gpu, q_ref)
    x = wl.make_x(cfg, seed=4, T=cfg.T)
    y, aux = _abi.forward_nvfp4(x.cuda(), w["w_router"].cuda(), q_gpu, cfg.k, act_scale_h=0.5,
                                aux=True)
    assert moe.sync_status() == 0
    ref = oracle.forward_nvfp4(x, w["w_router"], q_ref, cfg.k, act_scale_h=0.5)
    check(y, aux, ref, cfg.E)


def test_forward_nvfp4_refuses_batches_above_16(gemma_fp4):
    w, q_gpu, _ = gemma_fp4
    x = torch.zeros((17, 2816), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoEError) as ei:
        _abi.forward_nvfp4(x, w["w_router"].cuda(), q_gpu, 8)
    assert ei.value.code == _abi.MOE_ERR_UNSUPPORTED
