"""Host-side checks of the C-ABI library that need no GPU: it loads, exports
every symbol include/sol.h declares, and rejects bad arguments synchronously
(before any CUDA call is made)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sol.h")
LIB = os.path.join(ROOT, "block_sparse_attention_sol_b200", "libsol.so")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        import importlib.util
        spec = importlib.util.spec_from_file_location("sol_build", os.path.join(os.path.dirname(LIB), "build.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
        mod.build()
    return ctypes.CDLL(LIB)


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sol_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_three_calls():
    names = declared_functions()
    for n in ("sol_qk_prologue", "sol_block_select", "sol_sparse_attn_fwd", "sol_check_device_status"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


class Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "N", "H", "D", "grid_t", "grid_h", "grid_w")]


FAKE = ctypes.c_void_p(0x10000)      # aligned, never dereferenced on the host
MISALIGNED = ctypes.c_void_p(0x10008)
OK_SHAPE = Shape(1, 1024, 2, 64, 4, 16, 16)
INVALID, UNSUPPORTED = 1, 2


def prologue(lib, shape=OK_SHAPE, split=(24, 20, 20), ptr=FAKE, theta=10000.0, eps=1e-6, dt=0):
    f = lib.sol_qk_prologue
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 6 + [Shape, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                                          ctypes.c_float, ctypes.c_int, ctypes.c_void_p]
    return f(ptr, FAKE, FAKE, FAKE, FAKE, FAKE, shape, *split, theta, eps, dt, None)


def test_prologue_argument_checks(lib):
    assert prologue(lib, ptr=None) == INVALID
    assert prologue(lib, ptr=MISALIGNED) == INVALID
    assert prologue(lib, split=(24, 20, 18)) == INVALID          # does not sum to D
    assert prologue(lib, split=(23, 21, 20)) == INVALID          # odd
    assert prologue(lib, shape=Shape(1, 1000, 2, 64, 4, 16, 16)) == INVALID   # N != grid product
    assert prologue(lib, theta=0.0) == INVALID
    assert prologue(lib, eps=-1.0) == INVALID
    assert prologue(lib, dt=7) == INVALID
    assert prologue(lib, shape=Shape(1, 1024, 2, 96, 4, 16, 16), split=(32, 32, 32)) == UNSUPPORTED


def test_select_argument_checks(lib):
    f = lib.sol_block_select
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, Shape, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    wsb = lib.sol_block_select_workspace_bytes
    wsb.restype = ctypes.c_size_t
    wsb.argtypes = [Shape, ctypes.c_int]
    need = wsb(OK_SHAPE, 64)
    assert need == 2 * 1 * 2 * 16 * 64 * 4
    assert wsb(Shape(1, 1000, 2, 64, 4, 16, 16), 64) == 0
    assert f(FAKE, FAKE, OK_SHAPE, 64, 0, 0, FAKE, None, FAKE, need, None) == INVALID        # k = 0
    assert f(FAKE, FAKE, OK_SHAPE, 64, 17, 0, FAKE, None, FAKE, need, None) == INVALID       # k > nb
    assert f(FAKE, FAKE, OK_SHAPE, 64, 4, 0, FAKE, None, FAKE, need - 4, None) == INVALID    # small workspace
    assert f(FAKE, FAKE, OK_SHAPE, 64, 4, 0, None, None, FAKE, need, None) == INVALID        # no idx_out
    assert f(FAKE, FAKE, OK_SHAPE, 0, 4, 0, FAKE, None, FAKE, need, None) == INVALID         # block 0


def test_attention_argument_checks(lib):
    f = lib.sol_sparse_attn_fwd
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 4 + [Shape, ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_int,
                                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    assert f(FAKE, FAKE, FAKE, FAKE, OK_SHAPE, 64, 0, 0.0, 0, FAKE, FAKE, None) == INVALID
    assert f(FAKE, FAKE, FAKE, FAKE, OK_SHAPE, 64, 17, 0.0, 0, FAKE, FAKE, None) == INVALID
    assert f(FAKE, FAKE, None, FAKE, OK_SHAPE, 64, 4, 0.0, 0, FAKE, FAKE, None) == INVALID
    assert f(FAKE, FAKE, FAKE, MISALIGNED, OK_SHAPE, 64, 4, 0.0, 0, FAKE, FAKE, None) == INVALID
    assert f(FAKE, FAKE, FAKE, FAKE, OK_SHAPE, 64, 4, float("nan"), 0, FAKE, FAKE, None) == INVALID


def test_selftest_limit_checked(lib):
    f = lib.sol_selftest_wait_timeout
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_uint, ctypes.c_void_p]
    assert f(0, None) == INVALID
    assert f(2_000_000, None) == INVALID


def test_status_strings(lib):
    f = lib.sol_status_string
    f.restype = ctypes.c_char_p
    f.argtypes = [ctypes.c_int]
    assert [f(i).decode() for i in range(5)] == ["SOL_OK", "SOL_ERR_INVALID_ARG", "SOL_ERR_UNSUPPORTED",
                                                 "SOL_ERR_CUDA", "SOL_ERR_TIMEOUT"]


def test_prologue_pool_argument_checks(lib):
    f = lib.sol_qk_prologue_pool
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 6 + [Shape, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                                          ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                          ctypes.c_void_p, ctypes.c_void_p]

    def call(ptr=FAKE, shape=OK_SHAPE, split=(24, 20, 20), block=64, qbar=FAKE, kbar=FAKE):
        return f(ptr, FAKE, FAKE, FAKE, FAKE, FAKE, shape, *split, 10000.0, 1e-6, 0, block, qbar, kbar, None)

    assert call(ptr=None) == INVALID                       # the prologue's own checks apply
    assert call(split=(24, 20, 18)) == INVALID
    assert call(block=0) == INVALID
    assert call(qbar=None) == INVALID
    assert call(kbar=MISALIGNED) == INVALID
    assert call(shape=Shape(1, 1024, 2, 96, 4, 16, 16), split=(32, 32, 32)) == UNSUPPORTED


def test_select_pooled_argument_checks(lib):
    f = lib.sol_block_select_pooled
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, Shape, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p]
    assert f(FAKE, FAKE, OK_SHAPE, 64, 0, FAKE, None, None) == INVALID          # k = 0
    assert f(FAKE, FAKE, OK_SHAPE, 64, 17, FAKE, None, None) == INVALID         # k > nb
    assert f(None, FAKE, OK_SHAPE, 64, 4, FAKE, None, None) == INVALID
    assert f(FAKE, MISALIGNED, OK_SHAPE, 64, 4, FAKE, None, None) == INVALID
    assert f(FAKE, FAKE, OK_SHAPE, 64, 4, None, None, None) == INVALID          # no idx_out
    assert f(FAKE, FAKE, OK_SHAPE, 64, 4, FAKE, MISALIGNED, None) == INVALID    # misaligned scores_out
    assert f(FAKE, FAKE, Shape(1, 1000, 2, 64, 4, 16, 16), 64, 4, FAKE, None, None) == INVALID
    big = Shape(1, 2049 * 64, 2, 64, 1, 2049, 64)                                 # nb = 2049 > 2048
    assert f(FAKE, FAKE, big, 64, 4, FAKE, None, None) == UNSUPPORTED


class TileStruct(ctypes.Structure):
    _fields_ = [("t", ctypes.c_int), ("h", ctypes.c_int), ("w", ctypes.c_int)]


class SelectOpts(ctypes.Structure):
    _fields_ = [("flags", ctypes.c_uint), ("top_p", ctypes.c_float), ("softmax_scale", ctypes.c_float),
                ("head_k", ctypes.c_void_p), ("tile", TileStruct)]


def test_select_pooled_ex_argument_checks(lib):
    f = lib.sol_block_select_pooled_ex
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, Shape, ctypes.c_int, ctypes.c_int,
                  ctypes.POINTER(SelectOpts), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]

    def call(opts=SelectOpts(0, 1.0, 0.0, None), k=4, counts=FAKE, shape=OK_SHAPE, idx=FAKE):
        return f(FAKE, FAKE, shape, 64, k, ctypes.byref(opts) if opts is not None else None, idx, counts, None, None)

    assert call(opts=None) == INVALID
    assert call(counts=None) == INVALID                                  # counts are required
    assert call(counts=MISALIGNED) == INVALID
    assert call(idx=None) == INVALID
    assert call(k=0) == INVALID
    assert call(k=17) == INVALID
    assert call(opts=SelectOpts(8, 1.0, 0.0, None)) == INVALID            # unknown flag
    assert call(opts=SelectOpts(4, 0.0, 0.0, None)) == INVALID            # top_p must be in (0, 1]
    assert call(opts=SelectOpts(4, 1.5, 0.0, None)) == INVALID
    assert call(opts=SelectOpts(4, float("nan"), 0.0, None)) == INVALID
    assert call(opts=SelectOpts(4, 0.5, float("inf"), None)) == INVALID
    big = Shape(1, 2049 * 64, 2, 64, 1, 2049, 64)
    assert call(shape=big) == UNSUPPORTED


def test_attention_counts_argument_checks(lib):
    f = lib.sol_sparse_attn_fwd_counts
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 5 + [Shape, ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_int,
                                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    assert f(FAKE, FAKE, FAKE, FAKE, None, OK_SHAPE, 64, 4, 0.0, 0, FAKE, FAKE, None) == INVALID   # no counts
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, OK_SHAPE, 64, 0, 0.0, 0, FAKE, FAKE, None) == INVALID
    assert f(FAKE, FAKE, None, FAKE, FAKE, OK_SHAPE, 64, 4, 0.0, 0, FAKE, FAKE, None) == INVALID
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, OK_SHAPE, 64, 4, float("nan"), 0, FAKE, FAKE, None) == INVALID


class Tile(ctypes.Structure):
    _fields_ = [("t", ctypes.c_int), ("h", ctypes.c_int), ("w", ctypes.c_int)]


def test_tiled_argument_checks(lib):
    f = lib.sol_sparse_attn_fwd_tiled
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 5 + [Shape, Tile, ctypes.c_int, ctypes.c_float, ctypes.c_int,
                                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    ok_tile = Tile(1, 8, 8)                       # 16 blocks of 64 on the 4x16x16 grid
    assert f(FAKE, FAKE, FAKE, FAKE, None, OK_SHAPE, Tile(0, 8, 8), 4, 0.0, 0, FAKE, FAKE, None) == INVALID
    assert f(FAKE, FAKE, FAKE, FAKE, None, OK_SHAPE, Tile(3, 8, 8), 4, 0.0, 0, FAKE, FAKE, None) == INVALID  # 4 % 3
    assert f(FAKE, FAKE, FAKE, FAKE, None, OK_SHAPE, Tile(1, 5, 8), 4, 0.0, 0, FAKE, FAKE, None) == INVALID
    assert f(FAKE, FAKE, FAKE, FAKE, None, OK_SHAPE, ok_tile, 17, 0.0, 0, FAKE, FAKE, None) == INVALID     # k > nb
    assert f(FAKE, FAKE, None, FAKE, None, OK_SHAPE, ok_tile, 4, 0.0, 0, FAKE, FAKE, None) == INVALID
    g = lib.sol_qk_prologue_pool_tiled
    g.restype = ctypes.c_int
    g.argtypes = [ctypes.c_void_p] * 6 + [Shape, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                                          ctypes.c_float, ctypes.c_int, Tile, ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_void_p]

    def call(tile=ok_tile, qbar=FAKE, split=(24, 20, 20)):
        return g(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, OK_SHAPE, *split, 10000.0, 1e-6, 0, tile, qbar, FAKE, None)

    assert call(tile=Tile(1, 16, 32)) == INVALID       # 16 % 32
    assert call(tile=Tile(-1, 8, 8)) == INVALID
    assert call(qbar=None) == INVALID
    assert call(split=(24, 20, 18)) == INVALID


def test_select_ex_tile_checks(lib):
    f = lib.sol_block_select_pooled_ex
    f.restype = ctypes.c_int

    class Opts(ctypes.Structure):
        _fields_ = [("flags", ctypes.c_uint), ("top_p", ctypes.c_float), ("softmax_scale", ctypes.c_float),
                    ("head_k", ctypes.c_void_p), ("tile", Tile)]

    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, Shape, ctypes.c_int, ctypes.c_int, ctypes.POINTER(Opts),
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    bad = Opts(2, 1.0, 0.0, None, Tile(1, 8, 4))       # 32 tokens per tile, but block 64
    assert f(FAKE, FAKE, OK_SHAPE, 64, 4, ctypes.byref(bad), FAKE, FAKE, None, None) == INVALID
    bad2 = Opts(2, 1.0, 0.0, None, Tile(1, 3, 8))      # does not divide the grid
    assert f(FAKE, FAKE, OK_SHAPE, 64, 4, ctypes.byref(bad2), FAKE, FAKE, None, None) == INVALID


def test_quant_exchange_argument_checks(lib):
    pack = lib.sol_quant_pack
    pack.restype = ctypes.c_int
    pack.argtypes = [ctypes.c_void_p] + [ctypes.c_int] * 7 + [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_longlong,
                                                              ctypes.c_void_p]
    # x, B, N, H, D, G, split, code, codes, scales, g_stride, stream
    assert pack(None, 1, 96, 4, 128, 2, 0, 0, FAKE, FAKE, 0, None) == INVALID
    assert pack(FAKE, 1, 96, 4, 128, 3, 0, 0, FAKE, FAKE, 0, None) == INVALID       # 4 heads over 3 ranks
    assert pack(FAKE, 1, 96, 4, 128, 5, 1, 0, FAKE, FAKE, 0, None) == INVALID       # 96 tokens over 5 ranks
    assert pack(FAKE, 1, 96, 4, 128, 2, 2, 0, FAKE, FAKE, 0, None) == INVALID       # unknown split
    assert pack(FAKE, 1, 96, 4, 128, 2, 0, 7, FAKE, FAKE, 0, None) == INVALID       # unknown code
    assert pack(FAKE, 1, 96, 4, 128, 2, 0, 0, FAKE, FAKE, 10, None) == INVALID      # slices overlap
    assert pack(MISALIGNED, 1, 96, 4, 128, 2, 0, 0, FAKE, FAKE, 0, None) == INVALID
    assert pack(FAKE, 1, 96, 4, 96, 2, 0, 0, FAKE, FAKE, 0, None) == UNSUPPORTED   # D = 96
    unpack = lib.sol_dequant_unpack
    unpack.restype = ctypes.c_int
    unpack.argtypes = [ctypes.c_void_p, ctypes.c_void_p] + [ctypes.c_int] * 7 + [ctypes.c_void_p, ctypes.c_longlong,
                                                                                 ctypes.c_void_p]
    # codes, scales, B, Nc, Hc, D, G, split, code, out, g_stride, stream
    assert unpack(FAKE, FAKE, 1, 48, 2, 128, 2, 0, 0, None, 0, None) == INVALID
    assert unpack(FAKE, FAKE, 1, 48, 2, 128, 0, 0, 0, FAKE, 0, None) == INVALID     # G = 0
    assert unpack(FAKE, FAKE, 1, 48, 2, 128, 2, 0, 0, FAKE, 95, None) == INVALID    # stride < 96 rows
    assert unpack(FAKE, FAKE, 1, 48, 2, 32, 2, 0, 0, FAKE, 0, None) == UNSUPPORTED


def test_fp8_argument_checks(lib):
    ws = lib.sol_quant_attn_fp8_workspace_bytes
    ws.restype = ctypes.c_size_t
    ws.argtypes = [Shape]
    assert ws(OK_SHAPE) == 16                                   # B * H = 2 fp32 words, rounded to 16 bytes
    q = lib.sol_quant_attn_fp8
    q.restype = ctypes.c_int
    q.argtypes = [ctypes.c_void_p] * 3 + [Shape] + [ctypes.c_void_p] * 7 + [ctypes.c_size_t, ctypes.c_void_p]
    s128 = Shape(1, 1024, 2, 128, 4, 16, 16)
    assert q(FAKE, FAKE, FAKE, s128, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, None) == INVALID     # workspace
    assert q(FAKE, FAKE, FAKE, s128, FAKE, None, FAKE, FAKE, FAKE, FAKE, FAKE, 16, None) == INVALID
    assert q(FAKE, FAKE, FAKE, s128, FAKE, ctypes.c_void_p(0x10004), FAKE, FAKE, FAKE, FAKE, FAKE, 16, None) == INVALID
    assert q(FAKE, FAKE, FAKE, OK_SHAPE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16, None) == UNSUPPORTED  # D = 64
    a = lib.sol_sparse_attn_fwd_fp8
    a.restype = ctypes.c_int
    a.argtypes = [ctypes.c_void_p] * 8 + [Shape, ctypes.c_int, ctypes.c_int, ctypes.c_float] + [ctypes.c_void_p] * 3
    assert a(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, s128, 128, 0, 0.0, FAKE, FAKE, None) == INVALID  # k = 0
    assert a(FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, None, s128, 128, 4, 0.0, FAKE, FAKE, None) == INVALID
    assert a(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, s128, 64, 4, 0.0, FAKE, FAKE, None) == UNSUPPORTED
    assert a(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, s128, 128, 4, float("inf"), FAKE, FAKE, None) == INVALID


def test_backward_argument_checks(lib):
    ws = lib.sol_sparse_attn_bwd_workspace_bytes
    ws.restype = ctypes.c_size_t
    ws.argtypes = [Shape, ctypes.c_int]
    need = ws(OK_SHAPE, 64)
    assert need == 2 * 1024 * 4 + 2 * 16 * 16 * 4 + 2 * 16 * 4        # delta, inverted index, its counts
    f = lib.sol_sparse_attn_bwd
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 8 + [Shape, ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_int] + \
        [ctypes.c_void_p] * 4 + [ctypes.c_size_t, ctypes.c_void_p]

    def call(block=64, topk=4, ws_bytes=need, dq=FAKE, dt=0, shape=OK_SHAPE):
        return f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, shape, block, topk, 0.0, dt, dq, FAKE, FAKE, FAKE,
                 ws_bytes, None)

    assert call(ws_bytes=need - 4) == INVALID
    assert call(topk=0) == INVALID
    assert call(topk=17) == INVALID
    assert call(dq=None) == INVALID
    assert call(dq=MISALIGNED) == INVALID
    assert call(dt=5) == INVALID
    assert call(shape=Shape(1, 1024, 2, 96, 4, 16, 16), ws_bytes=1 << 20) == UNSUPPORTED


def test_noalloc_select_shape_checks(lib):
    """The allocation-free selection rejects a malformed shape and one whose pooled
    means exceed its fixed 40 MiB scratch before touching the device."""
    f = lib.sol_block_select_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, Shape, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    wsb = lib.sol_block_select_workspace_bytes
    wsb.restype = ctypes.c_size_t
    wsb.argtypes = [Shape, ctypes.c_int]
    assert f(FAKE, FAKE, Shape(1, 1000, 2, 64, 4, 16, 16), 64, 4, 0, FAKE, None, None) == INVALID  # N != grid
    big = Shape(1, 16 * 68 * 120, 64, 128, 16, 68, 120)   # 64 heads at 130,560 tokens: 66.8 MB of means
    assert wsb(big, 128) > 40 * 1024 * 1024
    assert f(FAKE, FAKE, big, 128, 102, 0, FAKE, None, None) == UNSUPPORTED
