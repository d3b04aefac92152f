"""fp64 CPU oracle of the routed MoE FFN layer -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package.  The library never does: it shares no code with the CUDA
path, and neither side imports the other.  The arithmetic lives in ``moe_oracle.c``
(plain C, double precision, ascending-index sums); this module only builds it and
marshals numpy arrays into it.

Pinned by ``tests/test_oracle_pins.py`` and ``tests/test_nvfp4_pins.py`` against closed
forms, brute force on tiny inputs, exact rational arithmetic, library routines and a
hand-worked NVFP4 group (``tests/golden/nvfp4_group_example.json``).  Parity status of every
function: pinned (see the tests), except the Gemma-faithfulness of routing details
(no router normalisation or scaling is modelled; the pages do not describe one).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_SRC_FP4 = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

# No -ffast-math: the oracle relies on IEEE double arithmetic in source order.
CFLAGS = ["-O2", "-std=gnu11", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
          "-ffp-contract=off", "-Wall"]


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into libmoe_oracle.so next to it (gcc)."""
    srcs = [_SRC, _SRC_FP4]
    if force or not os.path.exists(_LIB) or any(os.path.getmtime(_LIB) < os.path.getmtime(f)
                                                for f in srcs):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, *srcs, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.oracle_version.restype = _I
        L.oracle_get_threads.restype = _I
        L.oracle_set_threads.argtypes = [_I]
        L.oracle_gelu_tanh.restype = ctypes.c_double
        L.oracle_gelu_tanh.argtypes = [ctypes.c_double]
        L.oracle_router_logits.argtypes = [_P, _P, _P, _I64, _I, _I, _P]
        L.oracle_select.argtypes = [_P, _I64, _I, _I, _I, _P, _P]
        L.oracle_dispatch.argtypes = [_P, _I64, _I, _I, _P, _P, _P, _P]
        L.oracle_expert_ffn.argtypes = [_P, _P, _P, _P, _I, _I, _I, _P]
        L.oracle_forward.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _I, _I, _I, _I, _I,
                                     _P, _I64, _P, _P, _P, _P]
        _F = ctypes.c_float
        L.oracle_e2m1_value.restype = ctypes.c_double
        L.oracle_e2m1_value.argtypes = [_I]
        L.oracle_e4m3_value.restype = ctypes.c_double
        L.oracle_e4m3_value.argtypes = [_I]
        L.oracle_e2m1_round.argtypes = [_F]
        L.oracle_e4m3_round.argtypes = [_F]
        L.oracle_nvfp4_weight_scale.restype = _F
        L.oracle_nvfp4_weight_scale.argtypes = [_P, _I64]
        L.oracle_nvfp4_quantize.argtypes = [_P, _I64, _I, _F, _P, _P]
        L.oracle_nvfp4_dequantize.argtypes = [_P, _P, _I64, _I, _F, _P]
        L.oracle_expert_ffn_nvfp4.argtypes = [_P, _P, _P, _P, _I, _I, _F, _F, _P]
        _lib = L
    return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data


def _u16(a) -> np.ndarray:
    """Accept a bf16 torch CPU tensor or a uint16 array of bf16 bit patterns."""
    if hasattr(a, "dtype") and str(a.dtype) == "torch.bfloat16":
        import torch  # local: only to view the bits of a torch tensor
        return a.contiguous().view(torch.int16).numpy().view(np.uint16)
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def _f32(b) -> np.ndarray | None:
    if b is None:
        return None
    if hasattr(b, "numpy"):
        b = b.numpy()
    return np.ascontiguousarray(b, dtype=np.float32)


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(lib().oracle_get_threads())


def gelu_tanh(a: float) -> float:
    return float(lib().oracle_gelu_tanh(float(a)))


def router_logits(x, w_router, bias=None) -> np.ndarray:
    x, wr, b = _u16(x), _u16(w_router), _f32(bias)
    T, H = x.shape
    E = wr.shape[1]
    out = np.empty((T, E), np.float64)
    lib().oracle_router_logits(_ptr(x), _ptr(wr), _ptr(b), T, H, E, _ptr(out))
    return out


def select(logits: np.ndarray, k: int, renorm: bool = True):
    L = np.ascontiguousarray(logits, dtype=np.float64)
    T, E = L.shape
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    lib().oracle_select(_ptr(L), T, E, k, int(bool(renorm)), _ptr(ids), _ptr(w))
    return ids, w


def route(x, w_router, k: int, bias=None, renorm: bool = True):
    """-> (topk_ids [T,k] int32, topk_weights [T,k] float64, logits [T,E] float64)."""
    L = router_logits(x, w_router, bias)
    ids, w = select(L, k, renorm)
    return ids, w, L


def dispatch(ids: np.ndarray, E: int):
    """-> (counts [E], offsets [E+1], perm [T*k], inv [T*k]) int32."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, k = ids.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(T * k, np.int32)
    inv = np.empty(T * k, np.int32)
    lib().oracle_dispatch(_ptr(ids), T, k, E, _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(inv))
    return counts, offsets, perm, inv


def expert_ffn(x_row, w_gate, w_up, w_down, e: int) -> np.ndarray:
    xr, wg, wu, wd = _u16(x_row), _u16(w_gate), _u16(w_up), _u16(w_down)
    _, H, I = wg.shape
    out = np.empty(H, np.float64)
    lib().oracle_expert_ffn(_ptr(xr), _ptr(wg), _ptr(wu), _ptr(wd), int(e), H, I, _ptr(out))
    return out


def dense_ffn(x, w_gate, w_up, w_down, rows=None) -> np.ndarray:
    """The dense MLP beside the MoE (cann-recipes-infer "Gemma-4-26B-A4B 模型优化报告",
    §1 模型概况: every layer has a dense gate/up/down MLP, intermediate 2112, GELU), read in
    the experts' GEGLU form: y[t] = (gelu_tanh(x[t] W_gate) * (x[t] W_up)) W_down, in fp64
    with no intermediate rounding -- the expert FFN with one expert.
    w_gate, w_up [H,I]; w_down [I,H] -> y [len(rows) or T, H] float64."""
    T = x.shape[0]
    rows = range(T) if rows is None else rows
    wg, wu, wd = w_gate[None], w_up[None], w_down[None]
    return np.stack([expert_ffn(x[t], wg, wu, wd, 0) for t in rows])


def forward(x, w_router, w_gate, w_up, w_down, k: int, bias=None, renorm: bool = True,
            tokens=None):
    """Whole layer in fp64.  Routes every token; computes y only for `tokens` (all if None).

    -> dict(ids, weights, logits, y) with y [len(tokens) or T, H] float64.
    """
    x, wr, wg, wu, wd, b = (_u16(x), _u16(w_router), _u16(w_gate), _u16(w_up),
                            _u16(w_down), _f32(bias))
    T, H = x.shape
    E, _, I = wg.shape
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
    n_tok = T if tok is None else len(tok)
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    L = np.empty((T, E), np.float64)
    y = np.empty((n_tok, H), np.float64)
    lib().oracle_forward(_ptr(x), _ptr(wr), _ptr(b), _ptr(wg), _ptr(wu), _ptr(wd), T, H, E, I,
                         k, int(bool(renorm)), _ptr(tok), n_tok, _ptr(ids), _ptr(w), _ptr(L),
                         _ptr(y))
    return {"ids": ids, "weights": w, "logits": L, "y": y}


# ----------------------------------------------------------------------------- NVFP4
# NVFP4 quantisation and the layer with NVFP4 experts (nvfp4_oracle.c; Gemma-4-26B-A4B-NVFP4
# Ascend verification report, §2.3 量化配置 (NVFP4): weights and activations in 4-bit float,
# group size 16).  Codes are returned one per byte (bit 3 = sign), scales as E4M3 bytes.

def e2m1_value(code: int) -> float:
    return float(lib().oracle_e2m1_value(int(code)))


def e4m3_value(code: int) -> float:
    return float(lib().oracle_e4m3_value(int(code)))


def e2m1_round(v: float) -> int:
    return int(lib().oracle_e2m1_round(float(v)))


def e4m3_round(v: float) -> int:
    return int(lib().oracle_e4m3_round(float(v)))


def nvfp4_weight_scale(v) -> float:
    """Per-tensor scale of a weight tensor: amax / (6 * 448), in fp32."""
    a = np.ascontiguousarray(v, dtype=np.float32)
    return float(lib().oracle_nvfp4_weight_scale(_ptr(a), a.size))


def nvfp4_quantize(v, tensor_scale: float):
    """v [rows, K] (fp32; K % 16 == 0) -> (codes [rows, K] uint8, scales [rows, K/16] uint8)."""
    a = np.ascontiguousarray(v, dtype=np.float32)
    rows, K = a.shape
    codes = np.empty((rows, K), np.uint8)
    scales = np.empty((rows, K // 16), np.uint8)
    lib().oracle_nvfp4_quantize(_ptr(a), rows, K, float(tensor_scale), _ptr(codes), _ptr(scales))
    return codes, scales


def nvfp4_dequantize(codes, scales, tensor_scale: float) -> np.ndarray:
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    s = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, K = c.shape
    out = np.empty((rows, K), np.float64)
    lib().oracle_nvfp4_dequantize(_ptr(c), _ptr(s), rows, K, float(tensor_scale), _ptr(out))
    return out


def quantize_expert_weights(w_gate, w_up, w_down):
    """Quantise one layer's expert weights (bf16 [E,H,I], [E,H,I], [E,I,H]) the NVFP4 way,
    groups of 16 along each projection's reduction axis (H for gate/up, I for down), one
    tensor scale per expert and projection.  Returns a dict of numpy arrays:
      {gate,up}_codes [E,I,H], {gate,up}_scales [E,I,H/16], down_codes [E,H,I],
      down_scales [E,H,I/16] (uint8), {gate,up,down}_ts [E] (fp32)."""
    import torch  # local: only to read the bf16 tensors
    out = {}
    for name, w in (("gate", w_gate), ("up", w_up), ("down", w_down)):
        wt = w.float().transpose(1, 2).contiguous().numpy()    # [E, out, K]
        E, N, K = wt.shape
        codes = np.empty((E, N, K), np.uint8)
        scales = np.empty((E, N, K // 16), np.uint8)
        ts = np.empty(E, np.float32)
        for e in range(E):
            ts[e] = nvfp4_weight_scale(wt[e])
            codes[e], scales[e] = nvfp4_quantize(wt[e], ts[e])
        out[f"{name}_codes"], out[f"{name}_scales"], out[f"{name}_ts"] = codes, scales, ts
    del torch
    return out


def dequantize_expert_weights(q: dict) -> dict:
    """-> {gate, up}: [E, I, H], down: [E, H, I] float64 (exact dequantised values)."""
    out = {}
    for name in ("gate", "up", "down"):
        c, s, ts = q[f"{name}_codes"], q[f"{name}_scales"], q[f"{name}_ts"]
        out[name] = np.stack([nvfp4_dequantize(c[e], s[e], ts[e]) for e in range(c.shape[0])])
    return out


def forward_nvfp4(x, w_router, wq: dict, k: int, bias=None, renorm: bool = True,
                  act_scale_x: float = 1.0, act_scale_h: float = 1.0, tokens=None):
    """The layer with NVFP4 expert weights (given quantised, see quantize_expert_weights) and
    NVFP4 activations (x before GEMM-1, h before GEMM-2, with fixed tensor scales).  Routing
    as forward(); y[t] = sum_j w[t,j] o_{t,j} in slot order, each o from expert_ffn_nvfp4
    (the experts are dequantised one at a time).  -> dict(ids, weights, logits, y)."""
    xb = _u16(x)
    T, H = xb.shape
    ids, w, L = route(x, w_router, k, bias=bias, renorm=renorm)
    tok = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    o = {}                                   # (row, slot) -> expert output
    for e in np.unique(ids[tok]):
        dq = [nvfp4_dequantize(wq[f"{n}_codes"][e], wq[f"{n}_scales"][e], wq[f"{n}_ts"][e])
              for n in ("gate", "up", "down")]
        for r, t in enumerate(tok):
            for j in range(k):
                if ids[t, j] == e:
                    o[(r, j)] = expert_ffn_nvfp4(xb[t], dq[0], dq[1], dq[2], act_scale_x,
                                                 act_scale_h)
    y = np.zeros((len(tok), H), np.float64)
    for r in range(len(tok)):
        for j in range(k):
            y[r] += w[tok[r], j] * o[(r, j)]
    return {"ids": ids, "weights": w, "logits": L, "y": y}


def expert_ffn_nvfp4(x_row, wg_dq, wu_dq, wd_dq, act_scale_x: float = 1.0,
                     act_scale_h: float = 1.0) -> np.ndarray:
    """One expert on one token row with NVFP4 activations: weights given dequantised,
    wg_dq / wu_dq [I, H] and wd_dq [H, I] (float64).  -> o [H] float64."""
    xr = _u16(x_row)
    g = np.ascontiguousarray(wg_dq, dtype=np.float64)
    u = np.ascontiguousarray(wu_dq, dtype=np.float64)
    d = np.ascontiguousarray(wd_dq, dtype=np.float64)
    I, H = g.shape
    out = np.empty(H, np.float64)
    lib().oracle_expert_ffn_nvfp4(_ptr(xr), _ptr(g), _ptr(u), _ptr(d), H, I, float(act_scale_x),
                                  float(act_scale_h), _ptr(out))
    return out
