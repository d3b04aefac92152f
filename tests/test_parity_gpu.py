"""GPU parity: the CUDA path through the C ABI against the fp64 CPU oracle.

Bars: topk_ids, expert counts, offsets and the permutation bit-exact; topk_weights within
1e-5 absolute; y within max-abs 2e-2 and relative-L2 1e-2 (fp64 comparison of the bf16
output against the unrounded oracle, same bf16 inputs).  Large configs compare every
token's routing and a seeded sample of y rows (the oracle computes those rows one by one).
"""
import numpy as np
import pytest
import torch

import oracle
import expert_routed_ffn_softmax_b200 as moe
from expert_routed_ffn_softmax_b200 import workloads as wl

pytestmark = pytest.mark.gpu

Y_MAX_ABS = 2e-2
Y_REL_L2 = 1e-2
W_ABS = 1e-5


@pytest.fixture(scope="session")
def gemma_w():
    cpu = wl.make_weights(wl.CONFIGS["decode"])
    gpu = {k: (v.cuda() if v is not None else None) for k, v in cpu.items()}
    gpu["bias_skew"] = wl.skew_bias(128).cuda()
    cpu["bias_skew"] = wl.skew_bias(128)
    return cpu, gpu


def layer_inputs(cfg, gemma_w, seed=0, T=None):
    T = cfg.T if T is None else T
    if (cfg.H, cfg.E, cfg.I) == (2816, 128, 704):
        cpu, gpu = gemma_w
        cpu = dict(cpu, bias=cpu["bias_skew"] if cfg.skew_bias else None)
        gpu = dict(gpu, bias=gpu["bias_skew"] if cfg.skew_bias else None)
    else:
        cpu = wl.make_weights(cfg, seed)
        gpu = {k: (v.cuda() if v is not None else None) for k, v in cpu.items()}
    x = wl.make_x(cfg, seed, T)
    return x, cpu, gpu


SCREEN_C = 2.0 ** -10     # the kernel's screen error bound, in units of |x_t| |w_e|


def gpu_forward(x, g, k, renorm=True, router="auto", tiles="auto", rows="auto"):
    y, aux = moe.forward(x.cuda(), g["w_router"], g["w_gate"], g["w_up"], g["w_down"], k,
                         bias=g["bias"], renorm=renorm, aux=True, router=router, tiles=tiles,
                         rows=rows)
    assert moe.sync_status() == 0
    st = moe.router_stats(aux)
    if st["path"] == "screen":
        # the measured screen error stays 16x inside the bound the kernel assumes
        assert st["max_screen_err_ratio"] <= SCREEN_C / 16, st
    return y, aux


def check_routing(aux, ref, E):
    ids = aux["topk_ids"].cpu().numpy()
    assert np.array_equal(ids, ref["ids"]), "topk_ids differ from the oracle"
    w = aux["topk_weights"].cpu().numpy().astype(np.float64)
    assert np.max(np.abs(w - ref["weights"])) <= W_ABS
    counts, offsets, perm, _ = oracle.dispatch(ref["ids"], E)
    assert np.array_equal(aux["expert_counts"].cpu().numpy(), counts)
    assert np.array_equal(aux["expert_offsets"].cpu().numpy(), offsets)
    assert np.array_equal(aux["perm"].cpu().numpy(), perm)


def check_y(y_gpu_rows, y_ref):
    yg = y_gpu_rows.float().cpu().numpy().astype(np.float64)
    err = yg - y_ref
    max_abs = float(np.max(np.abs(err)))
    rel = float(np.linalg.norm(err) / np.linalg.norm(y_ref))
    assert max_abs <= Y_MAX_ABS, f"max-abs {max_abs}"
    assert rel <= Y_REL_L2, f"rel-L2 {rel}"
    return max_abs, rel


def sample_tokens(T, n, seed=0):
    if T <= n:
        return np.arange(T)
    rng = np.random.default_rng(seed)
    s = rng.choice(T, size=n - 2, replace=False)
    return np.unique(np.concatenate([[0, T - 1], s]))


def run_case(cfg, gemma_w, n_sample, T=None, renorm=True, router="auto", tiles="auto",
             rows="auto"):
    x, c, g = layer_inputs(cfg, gemma_w, T=T)
    T = x.shape[0]
    y, aux = gpu_forward(x, g, cfg.k, renorm, router, tiles, rows)
    rows = sample_tokens(T, n_sample)
    ref = oracle.forward(x, c["w_router"], c["w_gate"], c["w_up"], c["w_down"], cfg.k,
                         bias=c["bias"], renorm=renorm, tokens=rows)
    check_routing(aux, ref, cfg.E)
    return check_y(y[torch.from_numpy(rows).cuda()], ref["y"])


FORWARD_CASES = [("tiny", 10**9), ("decode", 10**9), ("sweep_T1", 10**9), ("sweep_T64", 10**9),
                 ("sweep_T512", 10**9), ("prefill", 384), ("sweep_T4096", 256),
                 ("skewed", 256), ("sweep_T32768", 128)]


@pytest.mark.parametrize("name,n_sample", FORWARD_CASES, ids=[c[0] for c in FORWARD_CASES])
def test_forward_parity(name, n_sample, gemma_w):
    run_case(wl.CONFIGS[name], gemma_w, n_sample)


@pytest.mark.parametrize("T", [1, 3, 37, 129, 1000])
def test_forward_ragged_tiny(T, gemma_w):
    run_case(wl.CONFIGS["tiny"], gemma_w, 10**9, T=T)


@pytest.mark.parametrize("T", [5, 37, 300])
def test_forward_ragged_gemma(T, gemma_w):
    run_case(wl.CONFIGS["decode"], gemma_w, 64, T=T)


@pytest.mark.parametrize("name,router", [("tiny", "screen"), ("decode", "screen"),
                                         ("sweep_T512", "fp64"), ("prefill", "fp64")])
def test_forward_forced_router_path(name, router, gemma_w):
    run_case(wl.CONFIGS[name], gemma_w, 256, router=router)


@pytest.mark.parametrize("tiles", ["decode", "prefill", "fused", "unfused"])
@pytest.mark.parametrize("name,T", [("tiny", 16), ("tiny", 3), ("decode", 8), ("decode", 1),
                                    ("decode", 16)])
def test_forward_tile_families(name, T, tiles, gemma_w):
    run_case(wl.CONFIGS[name], gemma_w, 64, T=T, tiles=tiles)


# CTA-pair tiles (256 rows per pair, tcgen05 cta_group::2) and single-CTA tiles (128 rows) of
# the dynamic expert FFN, each forced at batch sizes where the other is the default.  At
# T = 65 and 300 every expert has fewer than 128 rows (the second CTA of every pair has no
# rows); at T = 2048 and 4096 experts have around 128 and 256 rows (pair tiles whose second
# half is empty, partly filled or full, and experts with an odd number of 128-row tiles);
# tiny T = 1000 has 250 rows per expert and H = 256 (one GEMM-2 block).
PAIR_CASES = [("tiny", 1000), ("decode", 65), ("decode", 300), ("prefill", 2048),
              ("sweep_T4096", 4096)]


@pytest.mark.parametrize("rows", ["gather", "copy"])
@pytest.mark.parametrize("tiles", ["pairs", "single"])
@pytest.mark.parametrize("name,T", PAIR_CASES, ids=[f"{n}_T{t}" for n, t in PAIR_CASES])
def test_forward_pair_and_single_cta_tiles(name, T, tiles, rows, gemma_w):
    """Each tile form with GEMM-1's A rows gathered inside the kernel or copied to an
    expert-sorted buffer first and loaded by TMA."""
    run_case(wl.CONFIGS[name], gemma_w, 256, T=T, tiles=tiles, rows=rows)


def test_skewed_on_cta_pairs(gemma_w):
    """The skewed batch (experts from empty to 16k rows) on 256-row CTA pairs, with rows
    gathered and with rows copied (its default, single CTAs, is in test_forward_parity)."""
    assert moe.ffn_kernel_name(16384) == "expert_ffn_dynamic_kernel<128>"
    run_case(wl.CONFIGS["skewed"], gemma_w, 128, tiles="pairs", rows="gather")
    run_case(wl.CONFIGS["skewed"], gemma_w, 128, tiles="pairs", rows="copy")


@pytest.mark.parametrize("T", [65, 300, 2048, 4096])
def test_pair_tiles_match_single_cta_tiles_bitwise(T, gemma_w):
    """Every output element is the same fp32 sum over K in the same k-step order whether its
    row sits in a 128-row single-CTA tile or in a 256-row CTA pair, and whether its A row was
    gathered in the kernel or copied first, so the bytes agree."""
    x, c, g = layer_inputs(wl.CONFIGS["decode"], gemma_w, T=T)
    x = x.cuda()
    ys = [moe.forward(x, g["w_router"], g["w_gate"], g["w_up"], g["w_down"], 8, tiles=t, rows=r)
          for t in ("pairs", "single") for r in ("gather", "copy")]
    assert moe.sync_status() == 0
    for y in ys[1:]:
        assert torch.equal(ys[0], y)


def test_forward_no_renorm(gemma_w):
    run_case(wl.CONFIGS["tiny"], gemma_w, 10**9, renorm=False)
    run_case(wl.CONFIGS["decode"], gemma_w, 10**9, renorm=False)


@pytest.mark.parametrize("router", ["auto", "fp64", "screen"])
@pytest.mark.parametrize("name", ["tiny", "decode", "prefill", "skewed", "sweep_T32768"])
def test_route_parity_all_tokens(name, router, gemma_w):
    cfg = wl.CONFIGS[name]
    x, c, g = layer_inputs(cfg, gemma_w)
    ids, w = moe.route(x.cuda(), g["w_router"], cfg.k, bias=g["bias"], router=router)
    assert moe.sync_status() == 0
    r_ids, r_w, L = oracle.route(x, c["w_router"], cfg.k, bias=c["bias"])
    assert np.array_equal(ids.cpu().numpy(), r_ids)
    assert np.max(np.abs(w.cpu().numpy() - r_w)) <= W_ABS
    srt = -np.sort(-L, axis=1)
    gap = float(np.min(srt[:, cfg.k - 1] - srt[:, cfg.k]))
    print(f"{name}: min gap between the k-th and (k+1)-th logit = {gap:.3e}")


def test_screen_select_forms_agree_bitwise(gemma_w):
    """A batch many waves deep takes the 4-CTA-per-SM form of the screen select; the same
    tokens routed in 2048-token slices take the 2-CTA form.  Routing is per token and both
    forms do the same arithmetic, so ids and weight bits agree."""
    cfg = wl.CONFIGS["sweep_T32768"]
    x, c, g = layer_inputs(cfg, gemma_w)
    xg = x.cuda()
    ids, w = moe.route(xg, g["w_router"], cfg.k, router="screen")
    parts = [moe.route(xg[s:s + 2048].contiguous(), g["w_router"], cfg.k, router="screen")
             for s in range(0, cfg.T, 2048)]
    assert moe.sync_status() == 0
    assert torch.equal(ids, torch.cat([p[0] for p in parts]))
    assert torch.equal(w.view(torch.int32), torch.cat([p[1] for p in parts]).view(torch.int32))


def test_k_equals_E_and_exact_ties():
    """k = E; duplicated router columns and all-zero rows make exact ties, which the
    kernel must resolve through its exact recomputation, in id order."""
    cfg = wl.CONFIGS["tiny"]
    w = wl.make_weights(cfg, seed=3)
    x = wl.make_x(cfg, seed=3, T=64)
    x[5:9] = 0
    w["w_router"][:, 6] = w["w_router"][:, 2]
    w["w_router"][:, 7] = w["w_router"][:, 0]
    g = {k: (v.cuda() if v is not None else None) for k, v in w.items()}
    for router in ("fp64", "screen"):
        for k in (2, cfg.E):
            y, aux = gpu_forward(x, g, k, router=router)
            ref = oracle.forward(x, w["w_router"], w["w_gate"], w["w_up"], w["w_down"], k)
            check_routing(aux, ref, cfg.E)
            check_y(y, ref["y"])
            st = moe.router_stats(aux)
            assert st["exact_recomputes"] > 0    # the ties went the exact way
            if router == "screen":               # ... through the fp64 recheck first
                assert st["fp64_rechecks"] >= st["exact_recomputes"]


def test_screen_pair_sums_settle_most_tokens(gemma_w):
    """On the Gemma-shaped batch the fp32 pair-sum recheck decides the routing (and weights)
    of most tokens; the ones it leaves go through fp64, and the result matches the oracle."""
    x, c, g = layer_inputs(wl.CONFIGS["prefill"], gemma_w)
    T = x.shape[0]
    _, aux = gpu_forward(x, g, 8, router="screen")
    st = moe.router_stats(aux)
    assert st["path"] == "screen"
    assert 8 * T <= st["candidates"] <= 32 * T, st
    assert st["fp64_rechecks"] <= T // 4, st
    ids, w_ref, _ = oracle.route(x, c["w_router"], 8)
    assert np.array_equal(aux["topk_ids"].cpu().numpy(), ids)
    w = aux["topk_weights"].cpu().numpy().astype(np.float64)
    assert np.max(np.abs(w - w_ref)) <= W_ABS


def test_determinism(gemma_w):
    x, c, g = layer_inputs(wl.CONFIGS["prefill"], gemma_w)
    y1, a1 = gpu_forward(x, g, 8)
    y2, a2 = gpu_forward(x, g, 8)
    assert torch.equal(y1, y2)
    for key in a1:
        assert torch.equal(a1[key], a2[key]), key


def test_empty_batch(gemma_w):
    _, _, g = layer_inputs(wl.CONFIGS["decode"], gemma_w)
    x = torch.empty((0, 2816), dtype=torch.bfloat16, device="cuda")
    y = moe.forward(x, g["w_router"], g["w_gate"], g["w_up"], g["w_down"], 8)
    assert y.shape == (0, 2816)
    assert moe.sync_status() == 0


def test_bounded_wait_reports_timeout_and_context_survives(gemma_w):
    lib = moe.load()
    s = torch.cuda.current_stream().cuda_stream
    assert lib.moe_debug_set_wait_limit_ns(20_000_000) == 0       # 20 ms
    try:
        assert lib.moe_debug_unsatisfied_wait(s) == 0
        assert moe.sync_status() == 5                            # MOE_ERR_TIMEOUT
        assert moe.sync_status() == 0                            # cleared
    finally:
        assert lib.moe_debug_set_wait_limit_ns(0) == 0
    run_case(wl.CONFIGS["decode"], gemma_w, 10**9)                 # context still usable


def test_graph_replay_matches_oracle_and_direct_call(gemma_w):
    """A captured moe_forward replays to the oracle's y (within the layer tolerance) and to
    the direct call's bytes, and picks up new activations copied into its input buffer."""
    x_cpu, c, g = layer_inputs(wl.CONFIGS["decode"], gemma_w)
    x = x_cpu.cuda()
    y_direct = moe.forward(x, g["w_router"], g["w_gate"], g["w_up"], g["w_down"], 8)
    fg = moe.ForwardGraph(x, g["w_router"], g["w_gate"], g["w_up"], g["w_down"], 8)
    ref = oracle.forward(x_cpu, c["w_router"], c["w_gate"], c["w_up"], c["w_down"], 8)
    for _ in range(3):
        y = fg.replay()
        assert moe.sync_status() == 0
        check_y(y, ref["y"])
        assert torch.equal(y, y_direct)
    # new activations copied into the captured input buffer are picked up by the replay
    x2_cpu = wl.make_x(wl.CONFIGS["decode"], seed=7)
    fg.x.copy_(x2_cpu.cuda())
    y2 = fg.replay()
    assert moe.sync_status() == 0
    ref2 = oracle.forward(x2_cpu, c["w_router"], c["w_gate"], c["w_up"], c["w_down"], 8)
    check_y(y2, ref2["y"])
    assert torch.equal(y2, moe.forward(x2_cpu.cuda(), g["w_router"], g["w_gate"], g["w_up"],
                                       g["w_down"], 8))


def test_forward_and_dense_mlp_on_two_streams(gemma_w):
    """The MoE layer and the dense MLP beside it, issued on two streams so that their
    kernels overlap (each persistent expert-FFN grid then finds part of the GPU taken),
    each with its own workspace: both outputs match the oracle, three times over, and the
    device status stays OK (a bounded wait that ran out would read MOE_ERR_TIMEOUT)."""
    cfg = wl.CONFIGS["prefill"]
    x_cpu, c, g = layer_inputs(cfg, gemma_w)
    wd_cpu = wl.make_dense_weights(cfg.H, wl.DENSE_I)
    gd = {k: v.cuda() for k, v in wd_cpu.items()}
    x = x_cpu.cuda()
    lib = moe.load()
    ws1 = torch.empty(moe._abi.workspace_bytes(cfg.T, cfg.H, cfg.E, cfg.I, cfg.k), dtype=torch.uint8,
                      device="cuda")
    ws2 = torch.empty(lib.moe_dense_workspace_size(cfg.T, cfg.H, wl.DENSE_I), dtype=torch.uint8,
                      device="cuda")
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    rows = sample_tokens(cfg.T, 48, seed=11)
    ref = oracle.forward(x_cpu, c["w_router"], c["w_gate"], c["w_up"], c["w_down"], cfg.k,
                         tokens=rows)
    ref_d = oracle.dense_ffn(x_cpu, wd_cpu["w_gate"], wd_cpu["w_up"], wd_cpu["w_down"],
                             rows=rows.tolist())
    torch.cuda.synchronize()
    for _ in range(3):
        with torch.cuda.stream(s1):
            y, aux = moe.forward(x, g["w_router"], g["w_gate"], g["w_up"], g["w_down"], cfg.k,
                                 aux=True, workspace_buf=ws1, stream=s1)
        with torch.cuda.stream(s2):
            yd = moe.dense_ffn(x, gd["w_gate"], gd["w_up"], gd["w_down"], workspace_buf=ws2,
                               stream=s2)
        torch.cuda.synchronize()
        assert moe.sync_status() == 0
        idx = torch.from_numpy(rows).cuda()
        check_routing(aux, ref, cfg.E)
        check_y(y[idx], ref["y"])
        check_y(yd[idx], ref_d)


def test_dispatch_three_launches_for_many_chunks(gemma_w):
    """Past 32 chunks of 2048 pairs the dispatch runs as three launches (count, scan, rank)
    instead of one; its counts, offsets and permutation must still be the oracle's for the
    ids the router chose."""
    T = 2048 * 160 // 8   # 160 chunks of 2048 pairs at k = 8
    x, c, g = layer_inputs(wl.CONFIGS["prefill"], gemma_w, T=T)
    y, aux = gpu_forward(x, g, 8)
    assert moe.last_kernel_count() == 4 + 3 + 1 + 1
    ids = aux["topk_ids"].cpu().numpy()
    counts, offsets, perm, _ = oracle.dispatch(ids, 128)
    assert np.array_equal(aux["expert_counts"].cpu().numpy(), counts)
    assert np.array_equal(aux["expert_offsets"].cpu().numpy(), offsets)
    assert np.array_equal(aux["perm"].cpu().numpy(), perm)
    assert torch.isfinite(y.float()).all()


@pytest.mark.parametrize("T,H,I,rows", [
    (16, 256, 128, None),          # tiny shape, every row
    (8, 2816, 2112, None),         # Gemma dense MLP at decode, every row
    (1, 2816, 2112, None),
    (200, 2816, 2112, "sample"),   # two row tiles, the second ragged (72 rows)
    (2048, 2816, 2112, "sample"),  # CTA pairs: 8 tiles of 256 rows
    (2500, 2816, 2112, "sample"),  # CTA pairs, the last tile 196 rows (128 + 68)
])
def test_dense_ffn_parity(T, H, I, rows):
    """The dense GEGLU MLP beside the MoE against the fp64 oracle (same bf16 inputs):
    max-abs <= 2e-2 and rel-L2 <= 1e-2 on every row, or on a seeded sample of rows; one
    kernel launch; deterministic."""
    w = wl.make_dense_weights(H, I, seed=0)
    x = wl.make_x(wl.MoEConfig("dense", T, H, 1, 1, I), seed=3)
    g = {k: v.cuda() for k, v in w.items()}
    y = moe.dense_ffn(x.cuda(), g["w_gate"], g["w_up"], g["w_down"])
    assert moe.sync_status() == 0
    assert moe.last_kernel_count() == 1
    idx = list(range(T)) if rows is None else sorted(
        set(np.random.default_rng(5).choice(T, size=24, replace=False).tolist()) | {0, T - 1})
    ref = oracle.dense_ffn(x, w["w_gate"], w["w_up"], w["w_down"], rows=idx)
    check_y(y[idx], ref)
    y2 = moe.dense_ffn(x.cuda(), g["w_gate"], g["w_up"], g["w_down"])
    assert torch.equal(y, y2)


@pytest.mark.parametrize("T,tiles,expected", [
    (8, "auto", 3),        # decode front end (router + dispatch), expert FFN, combine
    (8, "unfused", 4),     # ... with GEMM-1 and GEMM-2 as two launches
    (64, "auto", 5),       # fp64 router 2, single-CTA dispatch, expert FFN, combine
    (4096, "auto", 7),     # screen router 4, one-launch dispatch, expert FFN, combine
    (4096, "unfused", 8),  # ... with GEMM-1 and GEMM-2 as two launches
    (4096, "fused", 7),    # ... static stream-K schedule in one launch
])
def test_kernel_count_per_forward(T, tiles, expected, gemma_w):
    x, c, g = layer_inputs(wl.CONFIGS["decode"], gemma_w, T=T)
    moe.forward(x.cuda(), g["w_router"], g["w_gate"], g["w_up"], g["w_down"], 8, tiles=tiles)
    assert moe.sync_status() == 0
    assert moe.last_kernel_count() == expected
    moe.route(x.cuda(), g["w_router"], 8, router="fp64")   # partial logits + select
    assert moe.last_kernel_count() == 2


@pytest.mark.parametrize("T", [1, 8, 64, 300, 2048])
def test_fused_ffn_matches_two_launches_bitwise(T, gemma_w):
    """GEMM-1 and GEMM-2 in one persistent launch give the same bytes as two launches (same
    tiles, same stream-K split, same summation order)."""
    x, c, g = layer_inputs(wl.CONFIGS["decode"], gemma_w, T=T)
    x = x.cuda()
    y1 = moe.forward(x, g["w_router"], g["w_gate"], g["w_up"], g["w_down"], 8, tiles="fused")
    y2 = moe.forward(x, g["w_router"], g["w_gate"], g["w_up"], g["w_down"], 8, tiles="unfused")
    assert moe.sync_status() == 0
    assert torch.equal(y1, y2)


# Other layer shapes the ABI accepts: 256 experts (8 per lane in the routers), few experts,
# short hidden/intermediate sizes with ragged 128-column blocks, k from 1 to 8, every router
# path and both FFN forms.  Inputs follow the same seeded recipe.
OTHER_SHAPES = [
    wl.MoEConfig("e256_k6", 40, 512, 256, 6, 192),
    wl.MoEConfig("e256_T300", 300, 512, 256, 8, 128),
    wl.MoEConfig("e64_T300", 300, 1024, 64, 4, 256),
    wl.MoEConfig("e32_decode", 8, 2048, 32, 2, 128),
    wl.MoEConfig("e12_h768", 5, 768, 12, 3, 64),
    wl.MoEConfig("k1", 33, 1024, 16, 1, 320),
]


@pytest.mark.parametrize("router", ["auto", "fp64", "screen"])
@pytest.mark.parametrize("cfg", OTHER_SHAPES, ids=[c.name for c in OTHER_SHAPES])
def test_other_shapes(cfg, router, gemma_w):
    if router == "screen" and cfg.E % 8:
        # the screen needs 16-byte W_router rows; forcing it is refused, not run
        x, c, g = layer_inputs(cfg, gemma_w)
        with pytest.raises(moe.MoEError) as ei:
            gpu_forward(x, g, cfg.k, True, router, "auto")
        assert ei.value.code == 2   # MOE_ERR_UNSUPPORTED
        return
    run_case(cfg, gemma_w, 10**9, router=router)
    run_case(cfg, gemma_w, 10**9, router=router, tiles="unfused")
    if cfg.T > 64:
        run_case(cfg, gemma_w, 10**9, router=router, tiles="pairs")
    if router != "screen":   # the screen path renormalises only
        run_case(cfg, gemma_w, 10**9, router=router, renorm=False)
