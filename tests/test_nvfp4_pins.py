"""Pins of the NVFP4 oracle (oracle/nvfp4_oracle.c) against things other than itself: the
format's published value set and hand-worked groups (tests/golden/nvfp4_group_example.json),
torch's float8_e4m3fn conversion (a library routine), brute-force nearest-value searches,
and the layer's composition redone with torch fp64 matmuls on the pinned pieces."""
import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from expert_routed_ffn_softmax_b200 import workloads as wl

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "nvfp4_group_example.json")))
MAGS = np.array(GOLD["e2m1_magnitudes"])


def test_e2m1_value_set_is_the_formats():
    assert [oracle.e2m1_value(c) for c in range(8)] == list(MAGS)
    for c in range(8):
        v = oracle.e2m1_value(c | 8)
        assert v == -MAGS[c] and np.signbit(v)


def test_e4m3_values_match_torch():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    mine = np.array([oracle.e4m3_value(c) for c in range(256)])
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(mine[ok], ref[ok])
    f = GOLD["e4m3_facts"]
    assert oracle.e4m3_value(126) == f["largest_finite"] and oracle.e4m3_value(1) == f["smallest_subnormal"]
    assert oracle.e4m3_value(f["one_code"]) == 1.0 and np.isnan(oracle.e4m3_value(f["nan_code"]))


def test_e4m3_round_matches_torch_including_midpoints():
    finite = np.array([oracle.e4m3_value(c) for c in range(127)])
    mids = (finite[:-1] + finite[1:]) / 2            # exact in fp32 (few significant bits)
    rng = np.random.default_rng(0)
    vals = np.concatenate([finite, mids, rng.uniform(0, 448, 4000), rng.uniform(0, 0.05, 2000)])
    vals = vals.astype(np.float32)
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).double().numpy()
    got = np.array([oracle.e4m3_value(oracle.e4m3_round(float(v))) for v in vals])
    assert np.array_equal(got, ref)
    for big in (448.0, 460.0, 1e6):                  # beyond the largest finite: saturate
        assert oracle.e4m3_round(big) == 126


def _nearest_e2m1(v):
    """All nearest signed E2M1 values of v (brute force over the published set)."""
    a = min(abs(v), 6.0)
    d = np.abs(MAGS - a)
    return set(np.flatnonzero(d == d.min()).tolist())


def test_e2m1_round_is_nearest_with_ties_to_even():
    rng = np.random.default_rng(1)
    mids = (MAGS[:-1] + MAGS[1:]) / 2
    vals = np.concatenate([MAGS, -MAGS, mids, -mids, rng.uniform(-8, 8, 5000)]).astype(np.float32)
    for v in vals:
        c = oracle.e2m1_round(float(v))
        idx = c & 7
        near = _nearest_e2m1(float(v))
        assert idx in near, (v, c)
        if len(near) == 2:                      # a midpoint: the even code
            assert idx % 2 == 0, (v, c)
        assert bool(c & 8) == bool(np.signbit(v)), (v, c)


@pytest.mark.parametrize("g", GOLD["groups"], ids=[g["name"] for g in GOLD["groups"]])
def test_hand_worked_groups(g):
    codes, scales = oracle.nvfp4_quantize(np.array([g["values"]], np.float32), g["tensor_scale"])
    assert codes[0].tolist() == g["codes"]
    assert int(scales[0, 0]) == g["scale_code"]
    dq = oracle.nvfp4_dequantize(codes, scales, g["tensor_scale"])
    assert np.array_equal(dq[0], np.array(g["dequantized"]))
    assert np.array_equal(np.signbit(dq[0]), np.signbit(np.array(g["dequantized"])))


def test_quantize_brute_force_on_small_tensors():
    """Every group: the scale is torch's E4M3 of (amax / 6) / ts (numpy fp32 steps), and every
    element takes a nearest point of the scaled grid (ties to the even code)."""
    rng = np.random.default_rng(2)
    for ts in (1.0, 0.0078125, 3.0e-5):
        v = (rng.standard_normal((6, 64)) * rng.uniform(0.01, 5.0, (6, 1)) * ts * 2000).astype(np.float32)
        v[0, :16] = 0.0                                   # an all-zero group: scale 0, codes 0
        codes, scales = oracle.nvfp4_quantize(v, ts)
        for r in range(v.shape[0]):
            for g in range(v.shape[1] // 16):
                grp = v[r, 16 * g:16 * g + 16]
                amax = np.float32(np.max(np.abs(grp)))
                s = np.float32(np.float32(amax / np.float32(6.0)) / np.float32(ts))
                # torch's cast does not saturate: the largest finite value stands for larger s
                s_ref = torch.tensor([min(s, np.float32(448.0))]).to(torch.float8_e4m3fn).double().item()
                assert oracle.e4m3_value(int(scales[r, g])) == s_ref
                S = np.float32(np.float32(s_ref) * np.float32(ts))
                for i, x in enumerate(grp):
                    c = int(codes[r, 16 * g + i])
                    if S == 0:
                        assert c & 7 == 0
                        continue
                    q = np.float32(x / S)
                    near = _nearest_e2m1(float(q))
                    assert c & 7 in near
                    if len(near) == 2:
                        assert (c & 7) % 2 == 0


def test_weight_scale_maps_the_tensor_amax_onto_the_largest_codes():
    rng = np.random.default_rng(3)
    w = (rng.standard_normal((32, 48)) * 0.02).astype(np.float32)
    ts = oracle.nvfp4_weight_scale(w)
    assert ts == np.float32(np.float32(np.max(np.abs(w))) / np.float32(2688.0))
    codes, scales = oracle.nvfp4_quantize(w, ts)
    # the group holding the tensor's amax gets the largest E4M3 scale and an E2M1 code of 6
    r, c = np.unravel_index(np.argmax(np.abs(w)), w.shape)
    assert int(scales[r, c // 16]) == 126 and int(codes[r, c]) & 7 == 7


def _torch_expert_nvfp4(x_row, dq_g, dq_u, dq_d, sx, sh):
    """The expert's composition with torch fp64 matmuls on the pinned pieces."""
    xf = x_row.float().numpy()[None]
    xq = oracle.nvfp4_dequantize(*oracle.nvfp4_quantize(xf, sx), sx)[0]
    xt = torch.from_numpy(xq)
    g = torch.from_numpy(dq_g) @ xt
    u = torch.from_numpy(dq_u) @ xt
    h = (F.gelu(g, approximate="tanh") * u).float().numpy()[None]
    hq = oracle.nvfp4_dequantize(*oracle.nvfp4_quantize(h, sh), sh)[0]
    return (torch.from_numpy(dq_d) @ torch.from_numpy(hq)).numpy()


def test_expert_ffn_nvfp4_equals_the_torch_composition():
    cfg = wl.CONFIGS["tiny"]
    w = wl.make_weights(cfg, seed=4)
    q = oracle.quantize_expert_weights(w["w_gate"], w["w_up"], w["w_down"])
    dq = oracle.dequantize_expert_weights(q)
    x = wl.make_x(cfg, seed=4, T=3)
    for t in range(3):
        for e in (0, 5):
            for sx, sh in ((1.0, 1.0), (0.0078125, 0.25)):
                mine = oracle.expert_ffn_nvfp4(x[t], dq["gate"][e], dq["up"][e], dq["down"][e], sx, sh)
                ref = _torch_expert_nvfp4(x[t], dq["gate"][e], dq["up"][e], dq["down"][e], sx, sh)
                assert np.max(np.abs(mine - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))


def test_forward_nvfp4_is_the_weighted_sum_of_its_experts():
    """The layer = routing of forward() (unchanged) + the k-sparse sum of the NVFP4 experts."""
    cfg = wl.CONFIGS["tiny"]
    w = wl.make_weights(cfg, seed=5)
    q = oracle.quantize_expert_weights(w["w_gate"], w["w_up"], w["w_down"])
    dq = oracle.dequantize_expert_weights(q)
    x = wl.make_x(cfg, seed=5, T=7)
    out = oracle.forward_nvfp4(x, w["w_router"], q, cfg.k, act_scale_x=0.5, act_scale_h=2.0)
    ids, wts, _ = oracle.route(x, w["w_router"], cfg.k)
    assert np.array_equal(out["ids"], ids) and np.array_equal(out["weights"], wts)
    for t in range(7):
        ref = sum(wts[t, j] * _torch_expert_nvfp4(x[t], dq["gate"][ids[t, j]], dq["up"][ids[t, j]],
                                                  dq["down"][ids[t, j]], 0.5, 2.0)
                  for j in range(cfg.k))
        assert np.max(np.abs(out["y"][t] - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))


def test_quantized_weights_are_close_to_the_bf16_weights():
    """Sanity of the whole quantiser on the synthetic weights: the relative error of the
    dequantised weights is what 4-bit groups give (a few percent), never more."""
    cfg = wl.CONFIGS["tiny"]
    w = wl.make_weights(cfg, seed=6)
    q = oracle.quantize_expert_weights(w["w_gate"], w["w_up"], w["w_down"])
    dq = oracle.dequantize_expert_weights(q)
    ref = w["w_gate"].double().transpose(1, 2).numpy()
    rel = np.linalg.norm(dq["gate"] - ref) / np.linalg.norm(ref)
    assert 0.02 < rel < 0.15
