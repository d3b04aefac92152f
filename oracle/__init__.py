"""fp64 CPU oracle of the routed MoE FFN layer -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package.  The library never does: it shares no code with the CUDA
path, and neither side imports the other.  The arithmetic lives in ``moe_oracle.c``
(plain C, double precision, ascending-index sums); this module only builds it and
marshals numpy arrays into it.

Pinned by ``tests/test_oracle_pins.py`` against closed forms, brute force on tiny
inputs, exact rational arithmetic and library routines.  Parity status of every
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
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

# No -ffast-math: the oracle relies on IEEE double arithmetic in source order.
CFLAGS = ["-O2", "-std=gnu11", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
          "-ffp-contract=off", "-Wall"]


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into libmoe_oracle.so next to it (gcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
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
