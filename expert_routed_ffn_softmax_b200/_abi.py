"""ctypes binding of include/moe.h (argument marshalling only).

Every step of the layer runs in libmoe_b200.so; this module checks tensor types and
shapes, owns a per-device workspace buffer, and passes raw pointers and the current
CUDA stream across the C ABI.  There is no fallback: if the library cannot be loaded,
every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_NO_WORKSPACE = 3
MOE_ERR_CUDA = 4
MOE_ERR_TIMEOUT = 5

MOE_FLAG_NO_RENORM = 1 << 0
MOE_FLAG_ROUTER_FP64 = 1 << 1
MOE_FLAG_ROUTER_SCREEN = 1 << 2
MOE_FLAG_PROFILE_STAGES = 1 << 3
MOE_FLAG_DECODE_TILES = 1 << 4
MOE_FLAG_PREFILL_TILES = 1 << 5
MOE_FLAG_UNFUSED_FFN = 1 << 6
MOE_FLAG_FUSED_FFN = 1 << 7
MOE_FLAG_FFN_PAIRS = 1 << 8
MOE_FLAG_FFN_SINGLE = 1 << 9
MOE_FLAG_FFN_ROWS_COPY = 1 << 10
MOE_FLAG_FFN_ROWS_GATHER = 1 << 11
MOE_COMBINE_F32 = 1 << 0

_ROUTER_FLAGS = {"auto": 0, "fp64": MOE_FLAG_ROUTER_FP64, "screen": MOE_FLAG_ROUTER_SCREEN}
# How GEMM-1 of the dynamic FFN gets its A rows above 64 tokens: copied into an expert-sorted
# buffer first and loaded by TMA, or gathered from x inside the FFN kernel.
_ROWS_FLAGS = {"auto": 0, "copy": MOE_FLAG_FFN_ROWS_COPY, "gather": MOE_FLAG_FFN_ROWS_GATHER}
# "auto"/"prefill": the dynamically scheduled expert FFN (one launch; CTA pairs for large
# batches); "pairs" / "single": that kernel on CTA pairs (256-row tiles) or single CTAs
# (128-row tiles) for batches of more than 64 tokens; "fused" / "unfused": the statically
# scheduled forms in one or two launches; "decode": the swap-AB decode tiles.
_TILE_FLAGS = {"auto": 0, "decode": MOE_FLAG_DECODE_TILES, "prefill": MOE_FLAG_PREFILL_TILES,
               "pairs": MOE_FLAG_FFN_PAIRS, "single": MOE_FLAG_FFN_SINGLE,
               "fused": MOE_FLAG_PREFILL_TILES | MOE_FLAG_FUSED_FFN,
               "unfused": MOE_FLAG_PREFILL_TILES | MOE_FLAG_UNFUSED_FFN}

# Every function the header declares, with (restype, argtypes).
_P, _I, _U, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint, ctypes.c_size_t
SIGNATURES = {
    "moe_abi_version": (_I, []),
    "moe_status_string": (ctypes.c_char_p, [_I]),
    "moe_route_workspace_size": (_SZ, [_I, _I, _I, _I, _U]),
    "moe_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _U]),
    "moe_route": (_I, [_P, _P, _P, _I, _I, _I, _I, _U, _P, _P, _P, _SZ, _P]),
    "moe_route_static": (_I, [_P, _P, _P, _I, _I, _I, _I, _U, _P, _P, _P]),
    "moe_forward": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _U, _P, _P, _P, _SZ, _P]),
    "moe_dense_workspace_size": (_SZ, [_I, _I, _I]),
    "moe_dense_ffn": (_I, [_P, _P, _P, _P, _I, _I, _I, _P, _P, _SZ, _P]),
    "moe_dispatch_workspace_size": (_SZ, [_I, _I, _I]),
    "moe_dispatch": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _P, _SZ, _P]),
    "moe_gather_rows": (_I, [_P, _P, _I, _I, _I, _I, _P, _P]),
    "moe_expert_ffn_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "moe_expert_ffn": (_I, [_P, _I, _P, _P, _I, _P, _P, _P, _I, _I, _I, _P, _P, _SZ, _P]),
    "moe_combine": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _U, _P, _P]),
    "moe_nvfp4_quantize_workspace_size": (_SZ, [_I]),
    "moe_nvfp4_quantize_weights": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _SZ, _P]),
    "moe_nvfp4_quantize_rows": (_I, [_P, _I, _I, ctypes.c_float, _P, _P, _P]),
    "moe_nvfp4_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _U]),
    "moe_forward_nvfp4": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _U, ctypes.c_float,
                               ctypes.c_float, _P, _P, _P, _SZ, _P]),
    "moe_sync_status": (_I, [_P]),
    "moe_ffn_kernel_name": (ctypes.c_char_p, [_I, _U]),
    "moe_last_stage_times": (_I, [ctypes.POINTER(ctypes.c_float), _I]),
    "moe_stage_name": (ctypes.c_char_p, [_I]),
    "moe_last_cuda_error": (_I, []),
    "moe_last_kernel_count": (_I, []),
    "moe_cuda_error_name": (ctypes.c_char_p, [_I]),
    "moe_debug_set_wait_limit_ns": (_I, [ctypes.c_ulonglong]),
    "moe_debug_unsatisfied_wait": (_I, [_P]),
}


class MoEError(RuntimeError):
    def __init__(self, code: int, what: str, cuda_error: int = 0):
        self.code = code
        self.cuda_error = cuda_error
        msg = f"{what}: {status_string(code)} ({code})"
        if cuda_error:
            msg += f" [{load().moe_cuda_error_name(cuda_error).decode()}]"
        super().__init__(msg)


class NVFP4Weights(ctypes.Structure):
    _fields_ = [("gate_codes", _P), ("gate_scales", _P), ("gate_ts", _P),
                ("up_codes", _P), ("up_scales", _P), ("up_ts", _P),
                ("down_codes", _P), ("down_scales", _P), ("down_ts", _P)]


class AuxOut(ctypes.Structure):
    _fields_ = [("expert_counts", _P), ("expert_offsets", _P), ("perm", _P),
                ("topk_ids", _P), ("topk_weights", _P), ("router_stats", _P)]


_lib = None
_lock = threading.Lock()


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library (once).  Raises if it is missing or incomplete."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise RuntimeError(f"{path} is missing: build it with "
                                   "`python -m expert_routed_ffn_softmax_b200.build`")
            L = ctypes.CDLL(path)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(L, name)
                fn.restype, fn.argtypes = res, args
            _lib = L
    return _lib


def status_string(code: int) -> str:
    return load().moe_status_string(code).decode()


def _check(code: int, what: str) -> None:
    if code != MOE_OK:
        raise MoEError(code, what, load().moe_last_cuda_error() if code == MOE_ERR_CUDA else 0)


def _stream_ptr(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


_ws: dict[int, torch.Tensor] = {}


def workspace(nbytes: int, device: torch.device) -> torch.Tensor:
    """A per-device scratch buffer of at least nbytes (grown on demand, 256-byte aligned)."""
    idx = device.index if device.index is not None else torch.cuda.current_device()
    buf = _ws.get(idx)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(max(nbytes, 1 << 20), dtype=torch.uint8, device=device)
        _ws[idx] = buf
    return buf


def _dev(t: torch.Tensor, name: str, dtype: torch.dtype, shape: tuple) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _flags(renorm: bool, router: str, profile: bool = False, tiles: str = "auto",
           rows: str = "auto") -> int:
    if router not in _ROUTER_FLAGS:
        raise ValueError(f"router must be one of {sorted(_ROUTER_FLAGS)}")
    if tiles not in _TILE_FLAGS:
        raise ValueError(f"tiles must be one of {sorted(_TILE_FLAGS)}")
    if rows not in _ROWS_FLAGS:
        raise ValueError(f"rows must be one of {sorted(_ROWS_FLAGS)}")
    return ((0 if renorm else MOE_FLAG_NO_RENORM) | _ROUTER_FLAGS[router] | _TILE_FLAGS[tiles]
            | _ROWS_FLAGS[rows] | (MOE_FLAG_PROFILE_STAGES if profile else 0))


def route(x: torch.Tensor, w_router: torch.Tensor, k: int, bias: torch.Tensor | None = None,
          renorm: bool = True, router: str = "auto", stream=None, workspace_buf=None):
    """Router of the MoE layer -> (topk_ids int32 [T,k], topk_weights float32 [T,k]).

    router: "auto" (tensor-core screen + fp64 recheck for T >= 256, fp64 logits below),
    "fp64" or "screen" to force a path; all give the same ids."""
    L = load()
    T, H = x.shape
    E = w_router.shape[1]
    dev = x.device
    px = _dev(x, "x", torch.bfloat16, (T, H))
    pw = _dev(w_router, "w_router", torch.bfloat16, (H, E))
    pb = None if bias is None else _dev(bias, "bias", torch.float32, (E,))
    flags = _flags(renorm, router)
    ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    wts = torch.empty((T, k), dtype=torch.float32, device=dev)
    nbytes = L.moe_route_workspace_size(T, H, E, k, flags) if T > 0 else 0
    if T > 0 and nbytes == 0:
        raise MoEError(MOE_ERR_UNSUPPORTED, "moe_route_workspace_size")
    ws = workspace(nbytes, dev) if workspace_buf is None else workspace_buf
    _check(L.moe_route(px, pw, pb, T, H, E, k, flags, ids.data_ptr(), wts.data_ptr(),
                       ws.data_ptr(), ws.numel(), _stream_ptr(stream)), "moe_route")
    return ids, wts


def forward(x: torch.Tensor, w_router: torch.Tensor, w_gate: torch.Tensor, w_up: torch.Tensor,
            w_down: torch.Tensor, k: int, bias: torch.Tensor | None = None, renorm: bool = True,
            aux: bool = False, out: torch.Tensor | None = None, profile: bool = False,
            stream=None, workspace_buf: torch.Tensor | None = None, router: str = "auto",
            tiles: str = "auto", rows: str = "auto"):
    """The routed MoE FFN layer -> y bf16 [T,H] (and a dict of routing outputs if aux).

    workspace_buf: optional caller-owned uint8 CUDA tensor used as the workspace (else a
    per-device buffer cached by this module, which may be reallocated by a later call)."""
    L = load()
    T, H = x.shape
    E, _, I = w_gate.shape
    dev = x.device
    px = _dev(x, "x", torch.bfloat16, (T, H))
    pr = _dev(w_router, "w_router", torch.bfloat16, (H, E))
    pg = _dev(w_gate, "w_gate", torch.bfloat16, (E, H, I))
    pu = _dev(w_up, "w_up", torch.bfloat16, (E, H, I))
    pd = _dev(w_down, "w_down", torch.bfloat16, (E, I, H))
    pb = None if bias is None else _dev(bias, "bias", torch.float32, (E,))
    y = torch.empty((T, H), dtype=torch.bfloat16, device=dev) if out is None else out
    py = _dev(y, "out", torch.bfloat16, (T, H))
    flags = _flags(renorm, router, profile, tiles, rows)
    a = None
    aux_d = None
    if aux:
        aux_d = {
            "expert_counts": torch.empty(E, dtype=torch.int32, device=dev),
            "expert_offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
            "perm": torch.empty(T * k, dtype=torch.int32, device=dev),
            "topk_ids": torch.empty((T, k), dtype=torch.int32, device=dev),
            "topk_weights": torch.empty((T, k), dtype=torch.float32, device=dev),
            "router_stats": torch.zeros(5, dtype=torch.int32, device=dev),
        }
        a = AuxOut(*(aux_d[n].data_ptr() for n, _ in AuxOut._fields_))
    nbytes = workspace_bytes(T, H, E, I, k, flags)
    ws = workspace(nbytes, dev) if workspace_buf is None else workspace_buf
    _check(L.moe_forward(px, pr, pb, pg, pu, pd, T, H, E, I, k, flags, py,
                         None if a is None else ctypes.byref(a), ws.data_ptr(), ws.numel(),
                         _stream_ptr(stream)), "moe_forward")
    return (y, aux_d) if aux else y


def dense_ffn(x: torch.Tensor, w_gate: torch.Tensor, w_up: torch.Tensor, w_down: torch.Tensor,
              out: torch.Tensor | None = None, stream=None,
              workspace_buf: torch.Tensor | None = None) -> torch.Tensor:
    """The dense GEGLU MLP beside the MoE -> y bf16 [T,H]:
    y = (gelu_tanh(x W_gate) * (x W_up)) W_down, W_gate/W_up [H,I], W_down [I,H]."""
    L = load()
    T, H = x.shape
    I = w_gate.shape[1]
    dev = x.device
    px = _dev(x, "x", torch.bfloat16, (T, H))
    pg = _dev(w_gate, "w_gate", torch.bfloat16, (H, I))
    pu = _dev(w_up, "w_up", torch.bfloat16, (H, I))
    pd = _dev(w_down, "w_down", torch.bfloat16, (I, H))
    y = torch.empty((T, H), dtype=torch.bfloat16, device=dev) if out is None else out
    py = _dev(y, "out", torch.bfloat16, (T, H))
    if T == 0:
        return y
    nbytes = L.moe_dense_workspace_size(T, H, I)
    if nbytes == 0:
        raise MoEError(MOE_ERR_UNSUPPORTED, "moe_dense_workspace_size")
    ws = workspace(nbytes, dev) if workspace_buf is None else workspace_buf
    _check(L.moe_dense_ffn(px, pg, pu, pd, T, H, I, py, ws.data_ptr(), ws.numel(),
                           _stream_ptr(stream)), "moe_dense_ffn")
    return y


# ----------------------------------------------------------------------------- steps alone
def dispatch(topk_ids: torch.Tensor, E: int, stream=None, workspace_buf=None):
    """moe_dispatch: topk_ids int32 [T,k] -> (counts [E], offsets [E+1], perm [T*k],
    inv [T*k]), int32 CUDA tensors."""
    L = load()
    T, k = topk_ids.shape
    dev = topk_ids.device
    pids = _dev(topk_ids, "topk_ids", torch.int32, (T, k))
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(T * k, dtype=torch.int32, device=dev)
    inv = torch.empty(T * k, dtype=torch.int32, device=dev)
    if T == 0:
        return counts.zero_(), offsets.zero_(), perm, inv
    nbytes = L.moe_dispatch_workspace_size(T, E, k)
    if nbytes == 0:
        raise MoEError(MOE_ERR_UNSUPPORTED, "moe_dispatch_workspace_size")
    ws = workspace(nbytes, dev) if workspace_buf is None else workspace_buf
    _check(L.moe_dispatch(pids, T, E, k, counts.data_ptr(), offsets.data_ptr(), perm.data_ptr(),
                          inv.data_ptr(), ws.data_ptr(), ws.numel(), _stream_ptr(stream)),
           "moe_dispatch")
    return counts, offsets, perm, inv


def gather_rows(x: torch.Tensor, perm: torch.Tensor, k: int, out: torch.Tensor | None = None,
                stream=None) -> torch.Tensor:
    """moe_gather_rows: out[r] = x[perm[r] // k] for every entry of perm (a 1-D int32 CUDA
    tensor of pair indices, possibly a slice of dispatch()'s perm)."""
    L = load()
    T, H = x.shape
    n = perm.numel()
    px = _dev(x, "x", torch.bfloat16, (T, H))
    pp = _dev(perm, "perm", torch.int32, (n,))
    xp = torch.empty((n, H), dtype=torch.bfloat16, device=x.device) if out is None else out
    po = _dev(xp, "out", torch.bfloat16, (n, H))
    if n:
        _check(L.moe_gather_rows(px, pp, n, T, H, k, po, _stream_ptr(stream)), "moe_gather_rows")
    return xp


def expert_ffn(xs: torch.Tensor, seg_rows: torch.Tensor, seg_expert: torch.Tensor,
               w_gate: torch.Tensor, w_up: torch.Tensor, w_down: torch.Tensor,
               out: torch.Tensor | None = None, stream=None, workspace_buf=None) -> torch.Tensor:
    """moe_expert_ffn: the GEGLU expert FFN of every row of xs [N,H] (bf16), whose rows form
    consecutive segments: seg_rows[i] rows of expert seg_expert[i] (int32 CUDA tensors)."""
    L = load()
    N, H = xs.shape
    E, _, I = w_gate.shape
    n_seg = seg_rows.numel()
    dev = xs.device
    px = _dev(xs, "xs", torch.bfloat16, (N, H))
    pr = _dev(seg_rows, "seg_rows", torch.int32, (n_seg,))
    pe = _dev(seg_expert, "seg_expert", torch.int32, (n_seg,))
    pg = _dev(w_gate, "w_gate", torch.bfloat16, (E, H, I))
    pu = _dev(w_up, "w_up", torch.bfloat16, (E, H, I))
    pd = _dev(w_down, "w_down", torch.bfloat16, (E, I, H))
    o = torch.empty((N, H), dtype=torch.bfloat16, device=dev) if out is None else out
    po = _dev(o, "out", torch.bfloat16, (N, H))
    if N == 0 or n_seg == 0:
        return o
    nbytes = L.moe_expert_ffn_workspace_size(N, H, E, I, n_seg)
    if nbytes == 0:
        raise MoEError(MOE_ERR_UNSUPPORTED, "moe_expert_ffn_workspace_size")
    ws = workspace(nbytes, dev) if workspace_buf is None else workspace_buf
    _check(L.moe_expert_ffn(px, N, pr, pe, n_seg, pg, pu, pd, H, E, I, po, ws.data_ptr(),
                            ws.numel(), _stream_ptr(stream)), "moe_expert_ffn")
    return o


def combine(o: torch.Tensor, inv: torch.Tensor, topk_weights: torch.Tensor, row_lo: int = 0,
            row_hi: int | None = None, fp32: bool = False, out: torch.Tensor | None = None,
            stream=None) -> torch.Tensor:
    """moe_combine: y[t] = sum_j w[t,j] o[inv[t,j]] over the slots whose sorted row lies in
    [row_lo, row_hi) -> y [T,H], bf16 (or fp32 with fp32=True)."""
    L = load()
    T, k = topk_weights.shape
    P, H = o.shape
    row_hi = T * k if row_hi is None else row_hi
    po = _dev(o, "o", torch.bfloat16, (P, H))
    pi = _dev(inv, "inv", torch.int32, (T * k,))
    pw = _dev(topk_weights, "topk_weights", torch.float32, (T, k))
    dt = torch.float32 if fp32 else torch.bfloat16
    y = torch.empty((T, H), dtype=dt, device=o.device) if out is None else out
    py = _dev(y, "out", dt, (T, H))
    if T:
        _check(L.moe_combine(po, pi, pw, T, k, H, row_lo, row_hi,
                             MOE_COMBINE_F32 if fp32 else 0, py, _stream_ptr(stream)),
               "moe_combine")
    return y


# ----------------------------------------------------------------------------- NVFP4
def nvfp4_quantize_weights(w: torch.Tensor, stream=None) -> dict:
    """moe_nvfp4_quantize_weights: bf16 w [E, K, N] (N contiguous) -> {codes uint8 [E, N, K/2],
    scales uint8 [E, ceil(N/128), K/64, 512] (the blocked scale layout of include/moe.h),
    ts float32 [E]} on w's device."""
    L = load()
    E, K, N = w.shape
    dev = w.device
    pw = _dev(w, "w", torch.bfloat16, (E, K, N))
    codes = torch.empty((E, N, K // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((E, (N + 127) // 128, K // 64, 512), dtype=torch.uint8, device=dev)
    ts = torch.empty(E, dtype=torch.float32, device=dev)
    ws = torch.empty(max(256, L.moe_nvfp4_quantize_workspace_size(E)), dtype=torch.uint8, device=dev)
    _check(L.moe_nvfp4_quantize_weights(pw, E, K, N, codes.data_ptr(), scales.data_ptr(),
                                        ts.data_ptr(), ws.data_ptr(), ws.numel(),
                                        _stream_ptr(stream)), "moe_nvfp4_quantize_weights")
    return {"codes": codes, "scales": scales, "ts": ts}


def nvfp4_quantize_layer(w_gate: torch.Tensor, w_up: torch.Tensor, w_down: torch.Tensor,
                         stream=None) -> dict:
    """The layer's expert weights (bf16, moe_forward's layout) as NVFP4: a dict of the nine
    tensors of moe_nvfp4_weights_t (gate_codes, gate_scales, gate_ts, up_..., down_...)."""
    out = {}
    for name, w in (("gate", w_gate), ("up", w_up), ("down", w_down)):
        q = nvfp4_quantize_weights(w, stream)
        out.update({f"{name}_{k}": v for k, v in q.items()})
    return out


def nvfp4_quantize_rows(x: torch.Tensor, ts: float, stream=None):
    """moe_nvfp4_quantize_rows: bf16 x [rows, K] -> (codes uint8 [rows, K/2], scales uint8
    [rows, K/16]) with tensor scale ts."""
    L = load()
    rows, K = x.shape
    px = _dev(x, "x", torch.bfloat16, (rows, K))
    codes = torch.empty((rows, K // 2), dtype=torch.uint8, device=x.device)
    scales = torch.empty((rows, K // 16), dtype=torch.uint8, device=x.device)
    _check(L.moe_nvfp4_quantize_rows(px, rows, K, float(ts), codes.data_ptr(), scales.data_ptr(),
                                     _stream_ptr(stream)), "moe_nvfp4_quantize_rows")
    return codes, scales


def forward_nvfp4(x: torch.Tensor, w_router: torch.Tensor, wq: dict, k: int,
                  bias: torch.Tensor | None = None, renorm: bool = True,
                  act_scale_x: float = 1.0, act_scale_h: float = 1.0, aux: bool = False,
                  out: torch.Tensor | None = None, profile: bool = False, stream=None,
                  workspace_buf: torch.Tensor | None = None, router: str = "auto"):
    """The routed layer with NVFP4 expert weights (wq from nvfp4_quantize_layer) and NVFP4
    activations, for T <= 16 tokens -> y bf16 [T, H] (and the routing dict if aux)."""
    L = load()
    T, H = x.shape
    E = w_router.shape[1]
    I = wq["gate_codes"].shape[1]
    dev = x.device
    px = _dev(x, "x", torch.bfloat16, (T, H))
    pr = _dev(w_router, "w_router", torch.bfloat16, (H, E))
    pb = None if bias is None else _dev(bias, "bias", torch.float32, (E,))
    sc_i = (E, (I + 127) // 128, H // 64, 512)   # blocked scales, N = I, K = H
    sc_h = (E, (H + 127) // 128, I // 64, 512)   # N = H, K = I
    shapes = {"gate_codes": ((E, I, H // 2), torch.uint8), "gate_scales": (sc_i, torch.uint8),
              "up_codes": ((E, I, H // 2), torch.uint8), "up_scales": (sc_i, torch.uint8),
              "down_codes": ((E, H, I // 2), torch.uint8), "down_scales": (sc_h, torch.uint8),
              "gate_ts": ((E,), torch.float32), "up_ts": ((E,), torch.float32),
              "down_ts": ((E,), torch.float32)}
    wstruct = NVFP4Weights(*(_dev(wq[n], n, shapes[n][1], shapes[n][0])
                             for n, _ in NVFP4Weights._fields_))
    y = torch.empty((T, H), dtype=torch.bfloat16, device=dev) if out is None else out
    py = _dev(y, "out", torch.bfloat16, (T, H))
    flags = _flags(renorm, router, profile)
    a = None
    aux_d = None
    if aux:
        aux_d = {
            "expert_counts": torch.empty(E, dtype=torch.int32, device=dev),
            "expert_offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
            "perm": torch.empty(T * k, dtype=torch.int32, device=dev),
            "topk_ids": torch.empty((T, k), dtype=torch.int32, device=dev),
            "topk_weights": torch.empty((T, k), dtype=torch.float32, device=dev),
            "router_stats": torch.zeros(5, dtype=torch.int32, device=dev),
        }
        a = AuxOut(*(aux_d[n].data_ptr() for n, _ in AuxOut._fields_))
    if T == 0:
        return (y, aux_d) if aux else y
    nbytes = L.moe_nvfp4_workspace_size(T, H, E, I, k, flags)
    if nbytes == 0:
        raise MoEError(MOE_ERR_UNSUPPORTED, "moe_nvfp4_workspace_size")
    ws = workspace(nbytes, dev) if workspace_buf is None else workspace_buf
    _check(L.moe_forward_nvfp4(px, pr, pb, ctypes.byref(wstruct), T, H, E, I, k, flags,
                               float(act_scale_x), float(act_scale_h), py,
                               None if a is None else ctypes.byref(a), ws.data_ptr(), ws.numel(),
                               _stream_ptr(stream)), "moe_forward_nvfp4")
    return (y, aux_d) if aux else y


def router_stats(aux: dict) -> dict:
    """Decode aux["router_stats"] of a forward(..., aux=True) call."""
    import struct
    v = aux["router_stats"].cpu().tolist()
    u = [x & 0xFFFFFFFF for x in v]
    return {"candidates": u[0], "exact_recomputes": u[1],
            "max_screen_err_ratio": struct.unpack("<f", struct.pack("<I", u[2]))[0],
            "path": "screen" if u[3] == 1 else "fp64", "fp64_rechecks": u[4]}


def workspace_bytes(T: int, H: int, E: int, I: int, k: int, flags: int = 0) -> int:
    if T == 0:
        return 0
    n = load().moe_workspace_size(T, H, E, I, k, flags)
    if n == 0:
        raise MoEError(MOE_ERR_UNSUPPORTED, "moe_workspace_size")
    return n


def sync_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device-side status code."""
    return load().moe_sync_status(_stream_ptr(stream))


def last_stage_times() -> dict[str, float]:
    L = load()
    buf = (ctypes.c_float * 16)()
    n = L.moe_last_stage_times(buf, 16)
    if n < 0:
        raise RuntimeError("no profiled moe_forward call yet")
    return {L.moe_stage_name(i).decode(): float(buf[i]) for i in range(n)}


def ffn_kernel_name(T: int, tiles: str = "auto", rows: str = "auto") -> str:
    """The expert-FFN kernel moe_forward launches for T tokens with this tile choice."""
    return load().moe_ffn_kernel_name(int(T), _flags(True, "auto", False, tiles, rows)).decode()


def last_kernel_count() -> int:
    """Kernels launched by this thread's most recent route/forward call."""
    return int(load().moe_last_kernel_count())


class ForwardGraph:
    """One moe_forward captured in a CUDA graph for fixed shapes and buffers.

    The layer is asynchronous, allocation-free and makes no host synchronisation on its
    call path, so a captured call replays exactly: inputs are read from, and y is written
    to, the same device buffers every replay (copy new activations into ``self.x``).  The
    library's one-time device set-up runs in the warm-up call before capture.  The graph
    owns its workspace.  profile=True records the library's stage events in every replay
    (read them with last_stage_times()).
    """

    def __init__(self, x, w_router, w_gate, w_up, w_down, k, bias=None, renorm=True,
                 profile=False, router="auto", tiles="auto", rows="auto"):
        self.x = x
        T, H = x.shape
        E, _, I = w_gate.shape
        self.y = torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
        flags = _flags(renorm, router, profile, tiles, rows)
        self.workspace = torch.empty(max(1, workspace_bytes(T, H, E, I, k, flags)),
                                     dtype=torch.uint8, device=x.device)
        self._args = (w_router, w_gate, w_up, w_down, k)
        self._kw = dict(bias=bias, renorm=renorm, profile=profile, workspace_buf=self.workspace,
                        router=router, tiles=tiles, rows=rows)
        forward(self.x, *self._args, out=self.y, **self._kw)    # set-up + workspace, uncaptured
        torch.cuda.synchronize(x.device)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            forward(self.x, *self._args, out=self.y, **self._kw)
        self.kernels_per_replay = last_kernel_count()

    def replay(self) -> torch.Tensor:
        self.graph.replay()
        return self.y
