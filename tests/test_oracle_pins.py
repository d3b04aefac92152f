"""Pins of the fp64 CPU oracle against things other than itself (CPU only).

Each test ties one part of the oracle to a closed form, exact rational arithmetic,
brute force on tiny inputs, an invariant, or a library routine, chosen so that a
plausible slip (a dropped term, a wrong sign, a transposed operand, an off-by-one in
the stable order, a mixed-up expert index) fails at least one of them.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

import oracle
from expert_routed_ffn_softmax_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
U = 2.0 ** -53


def gamma(n):
    return n * U / (1 - n * U)


def rand_bf16(rng, shape, std=1.0):
    return wl.bf16_from_f32(rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std))


def to64(t):
    return t.to(torch.float64)


# ----------------------------------------------------------------------------- shapes
def test_config_shapes_match_pages():
    g = json.load(open(os.path.join(GOLDEN, "gemma4_moe_shape.json")))
    for name in ("decode", "prefill", "skewed", "sweep_T1", "sweep_T32768"):
        c = wl.CONFIGS[name]
        assert (c.H, c.E, c.k, c.I) == (g["hidden_size"], g["num_experts"], g["top_k"],
                                        g["moe_intermediate"])
    assert (wl.CONFIGS["decode"].T, wl.CONFIGS["prefill"].T, wl.CONFIGS["skewed"].T) == (8, 2048, 16384)


# ----------------------------------------------------------------------------- GELU
def test_gelu_tanh_spot_values_and_library():
    assert oracle.gelu_tanh(0.0) == 0.0
    assert oracle.gelu_tanh(40.0) == 40.0          # -> a as a -> +inf
    assert oracle.gelu_tanh(-40.0) == 0.0          # -> 0 as a -> -inf
    a = np.linspace(-8, 8, 2001)
    ours = np.array([oracle.gelu_tanh(v) for v in a])
    ref = F.gelu(torch.from_numpy(a), approximate="tanh").numpy()
    np.testing.assert_allclose(ours, ref, rtol=0, atol=1e-12)
    # gelu(a) - gelu(-a) = a for the (1 + tanh) form
    np.testing.assert_allclose(ours - ours[::-1], a, rtol=0, atol=1e-12)
    # differs from the erf form (catches using the wrong GELU)
    erf_form = 0.5 * a * (1 + scipy.special.erf(a / math.sqrt(2)))
    assert np.max(np.abs(ours - erf_form)) > 1e-4


# ----------------------------------------------------------------------------- logits
def test_logits_exact_rational():
    rng = np.random.default_rng(1)
    T, H, E = 5, 48, 7                     # E != H: a transposed Wr would fail
    x, wr = rand_bf16(rng, (T, H)), rand_bf16(rng, (H, E), 0.02)
    b = torch.from_numpy(rng.standard_normal(E).astype(np.float32))
    L = oracle.router_logits(x, wr, b)
    xf, wf, bf = to64(x).numpy(), to64(wr).numpy(), b.double().numpy()
    for t in range(T):
        for e in range(E):
            exact = sum(Fraction(float(xf[t, h])) * Fraction(float(wf[h, e])) for h in range(H))
            exact += Fraction(float(bf[e]))
            absum = sum(abs(xf[t, h] * wf[h, e]) for h in range(H)) + abs(bf[e])
            assert abs(Fraction(L[t, e]) - exact) <= Fraction(gamma(H + 1) * absum)


def test_logits_exact_on_integers():
    rng = np.random.default_rng(2)
    T, H, E = 3, 64, 5
    x = torch.from_numpy(rng.integers(-8, 9, (T, H)).astype(np.float32)).bfloat16()
    wr = torch.from_numpy(rng.integers(-8, 9, (H, E)).astype(np.float32)).bfloat16()
    L = oracle.router_logits(x, wr)
    ref = x.double().numpy() @ wr.double().numpy()        # exact: small integers
    assert np.array_equal(L, ref)


def test_hand_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "route_hand_example.json")))
    x = torch.tensor([g["x"]], dtype=torch.bfloat16)
    wr = torch.tensor(g["w_router_rows"], dtype=torch.bfloat16)
    ids, w, L = oracle.route(x, wr, g["k"])
    assert L[0].tolist() == g["logits"]
    assert ids[0].tolist() == g["topk_ids"]
    # closed forms: softmax over the selected logits (2, 2, 1.75)
    e25 = math.exp(-0.25)
    np.testing.assert_allclose(w[0], [1 / (2 + e25), 1 / (2 + e25), e25 / (2 + e25)], atol=1e-15)
    ids2, w2, _ = oracle.route(x, wr, g["k"], renorm=False)
    z = math.exp(1) + 2 * math.exp(2) + math.exp(1.75)
    np.testing.assert_allclose(w2[0], [math.exp(2) / z, math.exp(2) / z, math.exp(1.75) / z],
                               atol=1e-15)


# ----------------------------------------------------------------------------- selection
def test_selection_brute_force_sort_with_ties():
    rng = np.random.default_rng(3)
    T, E, k = 200, 16, 5
    L = np.round(rng.standard_normal((T, E)) * 2) / 2     # coarse grid: many exact ties
    ids, _ = oracle.select(L, k)
    for t in range(T):
        ref = sorted(range(E), key=lambda e: (-L[t, e], e))[:k]
        assert ids[t].tolist() == ref


def test_zero_input_all_ties():
    E, k, H = 8, 3, 64
    x = torch.zeros(4, H, dtype=torch.bfloat16)
    wr = rand_bf16(np.random.default_rng(4), (H, E), 0.02)
    ids, w, _ = oracle.route(x, wr, k)
    assert (ids == np.arange(k)).all()
    np.testing.assert_allclose(w, 1.0 / k, atol=1e-15)
    _, w2, _ = oracle.route(x, wr, k, renorm=False)
    np.testing.assert_allclose(w2, 1.0 / E, atol=1e-15)


def test_duplicate_router_columns_prefer_lower_id():
    rng = np.random.default_rng(5)
    T, H, E, k = 300, 64, 8, 3
    x = rand_bf16(rng, (T, H))
    wr = rand_bf16(rng, (H, E), 0.02)
    wr[:, 6] = wr[:, 2]
    ids, _, L = oracle.route(x, wr, k)
    assert np.array_equal(L[:, 6], L[:, 2])
    for t in range(T):
        row = ids[t].tolist()
        if 6 in row:
            assert 2 in row and row.index(2) == row.index(6) - 1


def test_k_equals_E_is_full_argsort():
    rng = np.random.default_rng(6)
    T, H, E = 50, 32, 8
    x, wr = rand_bf16(rng, (T, H)), rand_bf16(rng, (H, E), 0.1)
    ids, w, L = oracle.route(x, wr, E)
    assert np.array_equal(ids, np.argsort(-L, axis=1, kind="stable"))
    np.testing.assert_allclose(w, np.take_along_axis(scipy.special.softmax(L, axis=1), ids, 1),
                               atol=1e-15)


# ----------------------------------------------------------------------------- weights
def test_weights_two_experts_sigmoid():
    rng = np.random.default_rng(7)
    L = rng.standard_normal((100, 2)) * 3
    ids, w = oracle.select(L, 2)
    top = L.max(1)
    other = L.min(1)
    np.testing.assert_allclose(w[:, 0], scipy.special.expit(top - other), atol=1e-15)


def test_weights_softmax_library_and_renorm_invariants():
    rng = np.random.default_rng(8)
    L = rng.standard_normal((64, 128)) * 1.1
    ids, w_raw = oracle.select(L, 8, renorm=False)
    p = scipy.special.softmax(L, axis=1)
    np.testing.assert_allclose(w_raw, np.take_along_axis(p, ids, 1), rtol=1e-13, atol=0)
    ids2, w = oracle.select(L, 8, renorm=True)
    assert np.array_equal(ids, ids2)
    assert (w > 0).all()
    np.testing.assert_allclose(w.sum(1), 1.0, atol=1e-12)
    np.testing.assert_allclose(w, w_raw / w_raw.sum(1, keepdims=True), rtol=1e-13)
    assert (np.diff(w, axis=1) <= 0).all()               # slots in descending order


# ----------------------------------------------------------------------------- dispatch
def brute_dispatch(ids, E):
    T, k = ids.shape
    perm = []
    for e in range(E):
        for t in range(T):
            for j in range(k):
                if ids[t, j] == e:
                    perm.append(t * k + j)
    counts = np.bincount(ids.ravel(), minlength=E)
    return counts, np.asarray(perm, np.int32)


@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (37, 8, 2), (100, 128, 8), (513, 16, 4)])
def test_dispatch_brute_force_and_invariants(T, E, k):
    rng = np.random.default_rng(T)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    counts, offsets, perm, inv = oracle.dispatch(ids, E)
    bc, bp = brute_dispatch(ids, E)
    assert np.array_equal(counts, bc) and np.array_equal(perm, bp)
    assert counts.sum() == T * k and offsets[0] == 0 and offsets[-1] == T * k
    assert (np.diff(offsets) == counts).all()
    assert np.array_equal(np.sort(perm), np.arange(T * k))
    assert np.array_equal(inv[perm], np.arange(T * k))
    assert (ids.ravel()[perm] == np.repeat(np.arange(E), counts)).all()


def test_dispatch_empty_and_skewed():
    ids = np.zeros((0, 4), np.int32)
    c, o, p, i = oracle.dispatch(ids, 16)
    assert c.sum() == 0 and (o == 0).all() and p.size == 0
    ids = np.tile(np.arange(4, dtype=np.int32), (50, 1))   # every token -> experts 0..3
    c, o, p, _ = oracle.dispatch(ids, 16)
    assert c[:4].tolist() == [50] * 4 and c[4:].sum() == 0
    assert p[:50].tolist() == [4 * t for t in range(50)]


# ----------------------------------------------------------------------------- experts
def dense_ffn_torch(x, wg, wu, wd):
    x, wg, wu, wd = map(to64, (x, wg, wu, wd))
    return (F.gelu(x @ wg, approximate="tanh") * (x @ wu)) @ wd


def test_single_expert_equals_dense_geglu_ffn():
    rng = np.random.default_rng(9)
    T, H, I = 6, 128, 64
    x = rand_bf16(rng, (T, H))
    wr = rand_bf16(rng, (H, 1), 0.02)
    wg, wu = rand_bf16(rng, (1, H, I), 0.02), rand_bf16(rng, (1, H, I), 0.02)
    wd = rand_bf16(rng, (1, I, H), 0.02)
    out = oracle.forward(x, wr, wg, wu, wd, k=1)
    assert (out["ids"] == 0).all() and (out["weights"] == 1.0).all()
    ref = dense_ffn_torch(x, wg[0], wu[0], wd[0]).numpy()
    np.testing.assert_allclose(out["y"], ref, rtol=1e-12, atol=1e-14)
    # gate and up are not interchangeable (catches GELU on the wrong projection)
    swapped = dense_ffn_torch(x, wu[0], wg[0], wd[0]).numpy()
    assert np.max(np.abs(out["y"] - swapped)) > 1e-3


def test_dense_mlp_oracle_is_the_library_formula():
    """The dense MLP beside the MoE: the oracle's one-expert FFN against the plain formula
    (torch fp64), on every row and on a subset of rows; gate/up swapped must differ."""
    rng = np.random.default_rng(12)
    T, H, I = 5, 128, 192
    x = rand_bf16(rng, (T, H))
    wg, wu = rand_bf16(rng, (H, I), 0.02), rand_bf16(rng, (H, I), 0.02)
    wd = rand_bf16(rng, (I, H), 0.02)
    ref = dense_ffn_torch(x, wg, wu, wd).numpy()
    np.testing.assert_allclose(oracle.dense_ffn(x, wg, wu, wd), ref, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(oracle.dense_ffn(x, wg, wu, wd, rows=[3, 0]), ref[[3, 0]],
                               rtol=1e-12, atol=1e-14)
    swapped = dense_ffn_torch(x, wu, wg, wd).numpy()
    assert np.max(np.abs(oracle.dense_ffn(x, wg, wu, wd) - swapped)) > 1e-3


def _tiny_layer(seed=10, T=16, H=256, E=8, k=2, I=128):
    rng = np.random.default_rng(seed)
    return dict(x=rand_bf16(rng, (T, H)), w_router=rand_bf16(rng, (H, E), 0.02),
                w_gate=rand_bf16(rng, (E, H, I), 0.02), w_up=rand_bf16(rng, (E, H, I), 0.02),
                w_down=rand_bf16(rng, (E, I, H), 0.02)), k


def test_whole_layer_dense_brute_force():
    d, k = _tiny_layer()
    out = oracle.forward(**d, k=k)
    x, wr = to64(d["x"]), to64(d["w_router"])
    L = (x @ wr).numpy()
    srt = np.sort(L, axis=1)[:, ::-1]
    assert np.min(srt[:, k - 1] - srt[:, k]) > 1e-9       # no near-ties in this draw
    E = L.shape[1]
    gate = np.zeros_like(L)
    for t in range(L.shape[0]):
        order = sorted(range(E), key=lambda e: (-L[t, e], e))[:k]
        p = torch.softmax(torch.from_numpy(L[t]), 0).numpy()
        gate[t, order] = p[order] / p[order].sum()
    # every expert on every token, then the k-sparse weighted sum
    y = np.zeros((L.shape[0], x.shape[1]))
    for e in range(E):
        ye = dense_ffn_torch(d["x"], d["w_gate"][e], d["w_up"][e], d["w_down"][e]).numpy()
        y += gate[:, e:e + 1] * ye
    np.testing.assert_allclose(out["y"], y, rtol=1e-10, atol=1e-13)
    assert np.array_equal(np.sort(out["ids"], 1), np.sort(np.argsort(-gate, 1)[:, :k], 1))


def test_linearity_in_w_down_and_subset_rows():
    d, k = _tiny_layer(seed=11)
    y1 = oracle.forward(**d, k=k)["y"]
    d2 = dict(d, w_down=d["w_down"] * 2)                   # exact in bf16
    y2 = oracle.forward(**d2, k=k)["y"]
    assert np.array_equal(y2, 2 * y1)
    rows = np.array([3, 0, 15, 7])
    ysub = oracle.forward(**d, k=k, tokens=rows)["y"]
    assert np.array_equal(ysub, y1[rows])


def test_expert_relabelling_invariance():
    d, k = _tiny_layer(seed=12)
    ref = oracle.forward(**d, k=k)
    rev = torch.arange(d["w_gate"].shape[0] - 1, -1, -1)
    d2 = dict(d, w_router=d["w_router"][:, rev].contiguous(), w_gate=d["w_gate"][rev].contiguous(),
              w_up=d["w_up"][rev].contiguous(), w_down=d["w_down"][rev].contiguous())
    out = oracle.forward(**d2, k=k)
    E = len(rev)
    assert np.array_equal(out["ids"], E - 1 - ref["ids"])
    # the softmax denominator sums in expert order, so only rounding may differ
    np.testing.assert_allclose(out["y"], ref["y"], rtol=1e-13, atol=1e-16)


def test_token_permutation_equivariance():
    d, k = _tiny_layer(seed=13)
    ref = oracle.forward(**d, k=k)
    p = torch.randperm(d["x"].shape[0], generator=torch.Generator().manual_seed(0))
    out = oracle.forward(**dict(d, x=d["x"][p].contiguous()), k=k)
    assert np.array_equal(out["y"], ref["y"][p.numpy()])
    assert np.array_equal(out["ids"], ref["ids"][p.numpy()])


def test_bias_enters_logits_and_shifts_routing():
    d, k = _tiny_layer(seed=14)
    E = d["w_router"].shape[1]
    b = wl.skew_bias(E)
    L0 = oracle.router_logits(d["x"], d["w_router"])
    L1 = oracle.router_logits(d["x"], d["w_router"], b)
    np.testing.assert_allclose(L1 - L0, np.broadcast_to(b.double().numpy(), L0.shape), atol=1e-13)
    ids, _ = oracle.select(L1, k)
    ids0, _ = oracle.select(L0, k)
    assert ids.mean() < ids0.mean()                        # load moves to low ids
