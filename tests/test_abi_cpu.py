"""The C ABI without a GPU: the library loads, exports every function include/moe.h
declares, and rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

from expert_routed_ffn_softmax_b200 import _abi, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "moe.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*[\w\s\*]*?\b(moe_\w+)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _abi.load()


def test_header_declares_the_documented_calls():
    names = declared_functions()
    for n in ("moe_route", "moe_forward", "moe_workspace_size", "moe_route_workspace_size",
              "moe_status_string", "moe_sync_status"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert names
    for n in names:
        assert hasattr(lib, n), n
        assert n in _abi.SIGNATURES, f"binding lacks {n}"


def test_abi_version_and_status_strings(lib):
    assert lib.moe_abi_version() == 6
    assert _abi.status_string(0) == "MOE_OK"
    assert _abi.status_string(5) == "MOE_ERR_TIMEOUT"
    assert _abi.status_string(99) == "MOE_ERR_UNKNOWN"


def test_workspace_sizes(lib):
    small = lib.moe_workspace_size(8, 2816, 128, 704, 8, 0)
    big = lib.moe_workspace_size(2048, 2816, 128, 704, 8, 0)
    assert 0 < small < big
    # Hbuf + O dominate: 2 bytes x pairs x (H + I); GEMM-1 gathers its rows straight from x
    assert big >= 2 * 2048 * 8 * (2816 + 704)
    # decode tiles (at most 16 tokens) also keep a gathered copy Xp of the routed rows
    # (compared with the static single launch, which keeps no chunk partials)
    dec = lib.moe_workspace_size(8, 2816, 128, 704, 8, 1 << 4)
    static = lib.moe_workspace_size(8, 2816, 128, 704, 8, 1 << 7)
    assert dec >= static + 2 * 8 * 8 * 2816
    # the default dynamic FFN hands out whole tiles: no stream-K partial tiles
    assert small + 2 * 2 * 128 * 128 * 256 * 4 <= static
    assert lib.moe_workspace_size(8, 2816, 128, 700, 8, 0) == 0     # I % 64 != 0
    assert lib.moe_workspace_size(8, 2800, 128, 704, 8, 0) == 0     # H % 64 != 0
    assert lib.moe_workspace_size(8, 2816, 128, 704, 9, 0) == 0     # k > 8
    assert lib.moe_workspace_size(8, 2816, 260, 704, 8, 0) == 0     # E > 256
    assert lib.moe_route_workspace_size(8, 2816, 128, 8, 0) > 0
    assert lib.moe_route_workspace_size(8, 2816, 6, 8, 0) == 0      # k > E
    # the router path changes the scratch it needs: fp64 partials vs a screen buffer
    fp64 = lib.moe_workspace_size(4096, 2816, 128, 704, 8, _abi.MOE_FLAG_ROUTER_FP64)
    scr = lib.moe_workspace_size(4096, 2816, 128, 704, 8, _abi.MOE_FLAG_ROUTER_SCREEN)
    assert fp64 > 0 and scr > 0 and fp64 != scr


FAKE = 1 << 20   # an aligned non-null address; never dereferenced (host checks fail first)


def test_host_argument_checks(lib):
    f = lib.moe_forward
    ok = (FAKE, FAKE, None, FAKE, FAKE, FAKE)
    # T == 0: nothing to do
    assert f(*ok, 0, 2816, 128, 704, 8, 0, FAKE + 4096, None, FAKE, 1 << 30, None) == 0
    # null required pointer
    assert f(None, FAKE, None, FAKE, FAKE, FAKE, 8, 2816, 128, 704, 8, 0, FAKE + 4096, None,
             FAKE, 1 << 30, None) == _abi.MOE_ERR_INVALID_ARG
    # k > E, negative T, unknown flag
    assert f(*ok, 8, 2816, 4, 704, 8, 0, FAKE + 4096, None, FAKE, 1 << 30, None) == 1
    assert f(*ok, -1, 2816, 128, 704, 8, 0, FAKE + 4096, None, FAKE, 1 << 30, None) == 1
    assert f(*ok, 8, 2816, 128, 704, 8, 1 << 12, FAKE + 4096, None, FAKE, 1 << 30, None) == 1
    for both in (_abi.MOE_FLAG_ROUTER_FP64 | _abi.MOE_FLAG_ROUTER_SCREEN,   # contradictory
                 _abi.MOE_FLAG_FUSED_FFN | _abi.MOE_FLAG_UNFUSED_FFN,
                 _abi.MOE_FLAG_DECODE_TILES | _abi.MOE_FLAG_PREFILL_TILES,
                 _abi.MOE_FLAG_FFN_PAIRS | _abi.MOE_FLAG_FFN_SINGLE,
                 _abi.MOE_FLAG_FFN_PAIRS | _abi.MOE_FLAG_FUSED_FFN,
                 _abi.MOE_FLAG_FFN_SINGLE | _abi.MOE_FLAG_DECODE_TILES):
        assert f(*ok, 8, 2816, 128, 704, 8, both, FAKE + 4096, None, FAKE, 1 << 30, None) == 1
        assert lib.moe_workspace_size(8, 2816, 128, 704, 8, both) == 0
    # misaligned pointer
    assert f(FAKE + 2, *ok[1:], 8, 2816, 128, 704, 8, 0, FAKE + 4096, None, FAKE, 1 << 30,
             None) == 1
    # y aliasing x
    assert f(*ok, 8, 2816, 128, 704, 8, 0, FAKE, None, FAKE, 1 << 30, None) == 1
    # unsupported shape
    assert f(*ok, 8, 2816, 128, 700, 8, 0, FAKE + 4096, None, FAKE, 1 << 30, None) == \
        _abi.MOE_ERR_UNSUPPORTED
    # too little workspace
    assert f(*ok, 8, 2816, 128, 704, 8, 0, FAKE + 4096, None, FAKE, 1024, None) == \
        _abi.MOE_ERR_NO_WORKSPACE
    r = lib.moe_route
    assert r(FAKE, FAKE, None, 8, 2816, 128, 8, 0, FAKE, FAKE, FAKE, 16, None) == \
        _abi.MOE_ERR_NO_WORKSPACE
    assert r(FAKE, None, None, 8, 2816, 128, 8, 0, FAKE, FAKE, FAKE, 1 << 30, None) == 1


def test_dense_ffn_host_checks(lib):
    f = lib.moe_dense_ffn
    # h [T, I] bf16 plus the counters: at least 2 * T * I bytes
    assert lib.moe_dense_workspace_size(2048, 2816, 2112) >= 2 * 2048 * 2112
    assert lib.moe_dense_workspace_size(8, 2816, 2100) == 0      # I % 64 != 0
    assert lib.moe_dense_workspace_size(0, 2816, 2112) == 0
    w = (FAKE, FAKE, FAKE, FAKE)
    assert f(*w, 0, 2816, 2112, FAKE + 4096, FAKE, 1 << 30, None) == 0           # T == 0
    assert f(None, FAKE, FAKE, FAKE, 8, 2816, 2112, FAKE + 4096, FAKE, 1 << 30, None) == 1
    assert f(*w, 8, 2816, 2112, FAKE, FAKE, 1 << 30, None) == 1                   # y == x
    assert f(FAKE + 2, FAKE, FAKE, FAKE, 8, 2816, 2112, FAKE + 4096, FAKE, 1 << 30, None) == 1
    assert f(*w, 8, 2816, 2100, FAKE + 4096, FAKE, 1 << 30, None) == _abi.MOE_ERR_UNSUPPORTED
    assert f(*w, 8, 2816, 2112, FAKE + 4096, FAKE, 1024, None) == _abi.MOE_ERR_NO_WORKSPACE


def test_ffn_kernel_choice(lib):
    """Which expert-FFN kernel a batch gets: the dynamic kernel with A slots of 8..128 rows,
    single CTAs gathering their rows by default; CTA pairs and copied rows when forced above
    64 tokens."""
    assert _abi.ffn_kernel_name(1) == "expert_ffn_dynamic_kernel<8>"
    assert _abi.ffn_kernel_name(8) == "expert_ffn_dynamic_kernel<8>"
    assert _abi.ffn_kernel_name(64) == "expert_ffn_dynamic_kernel<64>"
    assert _abi.ffn_kernel_name(32768) == "expert_ffn_dynamic_kernel<128>"
    assert _abi.ffn_kernel_name(32768, "pairs") == "expert_ffn_pair_kernel"
    assert _abi.ffn_kernel_name(32768, "pairs", "copy") == "expert_ffn_pair_kernel (rows copied)"
    assert _abi.ffn_kernel_name(4096, "single", "copy") == "expert_ffn_dynamic_kernel<128> (rows copied)"
    assert _abi.ffn_kernel_name(65, "pairs") == "expert_ffn_pair_kernel"
    assert _abi.ffn_kernel_name(64, "pairs") == "expert_ffn_dynamic_kernel<64>"
    assert _abi.ffn_kernel_name(8, "decode").startswith("grouped_gemm_decode_kernel")
    assert lib.moe_ffn_kernel_name(8, _abi.MOE_FLAG_FFN_PAIRS | _abi.MOE_FLAG_FFN_SINGLE) == b""
    both_rows = _abi.MOE_FLAG_FFN_ROWS_COPY | _abi.MOE_FLAG_FFN_ROWS_GATHER
    assert lib.moe_workspace_size(4096, 2816, 128, 704, 8, both_rows) == 0
    # pair tiles of 256 rows need fewer tile-list entries; copied rows need the Xp buffer
    single = lib.moe_workspace_size(4096, 2816, 128, 704, 8, _abi.MOE_FLAG_FFN_SINGLE)
    pairs = lib.moe_workspace_size(4096, 2816, 128, 704, 8, _abi.MOE_FLAG_FFN_PAIRS)
    copy = lib.moe_workspace_size(4096, 2816, 128, 704, 8, _abi.MOE_FLAG_FFN_ROWS_COPY)
    assert 0 < pairs <= single
    assert copy >= single + 2 * 4096 * 8 * 2816


def test_nvfp4_host_checks(lib):
    """The NVFP4 calls refuse what they cannot run before touching the device."""
    ws = lib.moe_nvfp4_workspace_size
    base = lib.moe_workspace_size(8, 2816, 128, 704, 8, 0)
    fp4 = ws(8, 2816, 128, 704, 8, 0)
    # the forward's layout plus the sorted x and h codes (and their scale lines)
    assert fp4 >= base + 64 * 2816 // 2 + 64 * 704 // 2
    assert ws(16, 2816, 128, 704, 8, 0) > 0
    assert ws(17, 2816, 128, 704, 8, 0) == 0                         # T > 16
    assert ws(8, 2816, 128, 704, 8, _abi.MOE_FLAG_DECODE_TILES) == 0  # not an NVFP4 flag
    assert ws(8, 2816, 128, 704, 8, _abi.MOE_FLAG_FFN_PAIRS) == 0
    wq = _abi.NVFP4Weights(*([FAKE] * 9))
    f = lib.moe_forward_nvfp4
    args = lambda T=8, flags=0, sx=1.0, sh=1.0, x=FAKE, y=FAKE + 4096, w=ctypes.byref(wq), \
        nbytes=1 << 30: (x, FAKE, None, w, T, 2816, 128, 704, 8, flags, sx, sh, y, None, FAKE,
                         nbytes, None)
    assert f(*args(T=0)) == 0
    assert f(*args(sx=0.0)) == _abi.MOE_ERR_INVALID_ARG                 # scales must be > 0
    assert f(*args(sh=-1.0)) == _abi.MOE_ERR_INVALID_ARG
    assert f(*args(w=None)) == _abi.MOE_ERR_INVALID_ARG
    assert f(*args(y=FAKE)) == _abi.MOE_ERR_INVALID_ARG                 # y aliasing x
    assert f(*args(flags=_abi.MOE_FLAG_FUSED_FFN)) == _abi.MOE_ERR_INVALID_ARG
    assert f(*args(T=17)) == _abi.MOE_ERR_UNSUPPORTED
    assert f(*args(nbytes=1024)) == _abi.MOE_ERR_NO_WORKSPACE
    bad = _abi.NVFP4Weights(*([FAKE] * 9))
    bad.gate_scales = FAKE + 8                                          # scales 16-byte aligned
    assert f(*args(w=ctypes.byref(bad))) == _abi.MOE_ERR_INVALID_ARG
    nul = _abi.NVFP4Weights(*([FAKE] * 9))
    nul.down_ts = None
    assert f(*args(w=ctypes.byref(nul))) == _abi.MOE_ERR_INVALID_ARG
    q = lib.moe_nvfp4_quantize_weights
    big = 1 << 30
    assert q(None, 128, 2816, 704, FAKE, FAKE, FAKE, FAKE, big, None) == _abi.MOE_ERR_INVALID_ARG
    assert q(FAKE, 128, 2848, 704, FAKE, FAKE, FAKE, FAKE, big, None) == _abi.MOE_ERR_UNSUPPORTED
    assert q(FAKE, 128, 2816, 704, FAKE, FAKE, FAKE, FAKE, 16, None) == _abi.MOE_ERR_NO_WORKSPACE
    assert lib.moe_nvfp4_quantize_workspace_size(128) >= 128 * 4


def test_step_calls_host_checks(lib):
    """moe_dispatch, moe_gather_rows, moe_expert_ffn and moe_combine (the layer's steps as
    calls) refuse bad arguments on the host."""
    big = 1 << 30
    d = lib.moe_dispatch
    assert lib.moe_dispatch_workspace_size(8, 128, 8) > 0
    assert d(FAKE, 0, 128, 8, FAKE, FAKE, FAKE, FAKE, FAKE, big, None) == 0          # T == 0
    assert d(FAKE, 8, 4, 8, FAKE, FAKE, FAKE, FAKE, FAKE, big, None) == 1            # k > E
    assert d(None, 8, 128, 8, FAKE, FAKE, FAKE, FAKE, FAKE, big, None) == 1
    assert d(FAKE, 8, 128, 8, FAKE, FAKE, FAKE, FAKE, FAKE, 16, None) == _abi.MOE_ERR_NO_WORKSPACE
    g = lib.moe_gather_rows
    assert g(FAKE, FAKE, 0, 8, 2816, 8, FAKE, None) == 0                               # no rows
    assert g(FAKE + 2, FAKE, 64, 8, 2816, 8, FAKE, None) == 1                          # misaligned x
    assert g(FAKE, FAKE, 64, 8, 2812, 8, FAKE, None) == _abi.MOE_ERR_UNSUPPORTED      # H % 8
    f = lib.moe_expert_ffn
    assert lib.moe_expert_ffn_workspace_size(64, 2816, 16, 704, 16) > 0
    assert lib.moe_expert_ffn_workspace_size(64, 2816, 16, 700, 16) == 0             # I % 64
    assert lib.moe_expert_ffn_workspace_size(64, 2816, 16, 704, 2000) == 0           # segments
    w = (FAKE, FAKE, FAKE)
    assert f(FAKE, 0, FAKE, FAKE, 4, *w, 2816, 16, 704, FAKE + 4096, FAKE, big, None) == 0
    assert f(FAKE, 64, None, FAKE, 4, *w, 2816, 16, 704, FAKE + 4096, FAKE, big, None) == 1
    assert f(FAKE, 64, FAKE, FAKE, 4, *w, 2816, 16, 704, FAKE, FAKE, big, None) == 1   # out == xs
    assert f(FAKE, 64, FAKE, FAKE, 4, *w, 2816, 16, 700, FAKE + 4096, FAKE, big, None) == \
        _abi.MOE_ERR_UNSUPPORTED
    assert f(FAKE, 64, FAKE, FAKE, 4, *w, 2816, 16, 704, FAKE + 4096, FAKE, 16, None) == \
        _abi.MOE_ERR_NO_WORKSPACE
    c = lib.moe_combine
    assert c(FAKE, FAKE, FAKE, 0, 8, 2816, 0, 0, 0, FAKE, None) == 0                   # T == 0
    assert c(FAKE, FAKE, FAKE, 8, 9, 2816, 0, 64, 0, FAKE, None) == 1                  # k > 8
    assert c(FAKE, FAKE, FAKE, 8, 8, 2816, 0, 64, 4, FAKE, None) == 1                  # flag
    assert c(FAKE, FAKE, FAKE, 8, 8, 2816, 10, 5, 0, FAKE, None) == 1                  # lo > hi
    assert c(FAKE, FAKE, FAKE, 8, 8, 2816, 0, 65, 0, FAKE, None) == 1                  # hi > T k
    assert c(FAKE, FAKE, FAKE, 8, 8, 2812, 0, 64, 0, FAKE, None) == _abi.MOE_ERR_UNSUPPORTED
