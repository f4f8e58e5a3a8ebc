"""The C ABI library loads and exports every entry point the header declares;
host-side argument checks reject bad calls before any GPU work (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn25.h")


def declared():
    text = open(HEADER).read()
    return re.findall(r"ATTN25_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


@pytest.fixture(scope="module")
def lib():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "attn25_build", os.path.join(ROOT, "tiled_attention_25_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return ctypes.CDLL(mod.build())


def test_header_declares_the_boundary():
    names = set(declared())
    assert {"attn_fwd", "attn_bwd", "build_block_mask", "attn_bwd_workspace_size",
            "attn_block_mask_bytes", "attn_block_mask_bind", "attn_get_status",
            "attn_set_wait_limit_ms", "attn_strerror"} <= names


def test_every_declared_symbol_is_exported(lib):
    for name in declared():
        assert hasattr(lib, name), name


def test_binding_names_match_header(lib):
    import tiled_attention_25_b200 as ta
    for name in declared():
        assert name in ta.EXPORTED and callable(getattr(ta, name)), name


def test_sizes(lib):
    lib.attn_block_mask_bytes.restype = ctypes.c_size_t
    lib.attn_bwd_workspace_size.restype = ctypes.c_size_t
    assert lib.attn_block_mask_bytes(0, 10, 10) == 0
    n = lib.attn_block_mask_bytes(1, 32768, 32768)
    assert n >= 256 * 256 * (1 + 4 + 4) + 256 * 4 * 2
    ws = lib.attn_bwd_workspace_size(1, 32, 32768, 128)
    assert ws >= 32 * 32768 * (128 * 4 + 8)
    assert lib.attn_bwd_workspace_size(1, 1, 1, 96) == 0  # unsupported head dim


def test_bind_lays_out_inside_the_buffer(lib):
    import tiled_attention_25_b200.abi as abi
    lib.attn_block_mask_bytes.restype = ctypes.c_size_t
    B, Sq, Skv = 2, 1000, 300
    n = lib.attn_block_mask_bytes(B, Sq, Skv)
    fake = 1 << 40  # never dereferenced: bind only computes addresses
    m = abi.CBlockMask()
    rc = lib.attn_block_mask_bind(ctypes.c_void_p(fake), ctypes.c_size_t(n), B, Sq, Skv, ctypes.byref(m))
    assert rc == 0
    ptrs = [m.tile_class, m.kv_count, m.kv_index, m.q_count, m.q_index, m.fwd_order, m.bwd_order]
    assert all(fake <= p < fake + n and p % 256 == 0 for p in ptrs)
    assert (m.nq_tiles, m.nk_tiles) == (8, 3)
    rc = lib.attn_block_mask_bind(ctypes.c_void_p(fake), ctypes.c_size_t(n - 1), B, Sq, Skv, ctypes.byref(m))
    assert rc == -4
    rc = lib.attn_block_mask_bind(ctypes.c_void_p(fake + 16), ctypes.c_size_t(n), B, Sq, Skv, ctypes.byref(m))
    assert rc == -3


def test_argument_errors_before_launch(lib):
    P, I = ctypes.c_void_p, ctypes.c_int
    lib.attn_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, I, ctypes.c_float, I, P, P, P]
    good = ctypes.c_void_p(1 << 32)
    odd = ctypes.c_void_p((1 << 32) + 8)
    args = lambda **kw: dict(dict(q=good, k=good, v=good, o=good, lse=None, B=1, Hq=4, Hkv=2, Sq=128,
                                  Skv=128, D=128, scale=0.1, mod=0, mp=None, bm=None, s=None), **kw)
    call = lambda a: lib.attn_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"], a["Sq"],
                                  a["Skv"], a["D"], a["scale"], a["mod"], a["mp"], a["bm"], a["s"])
    assert call(args(q=None)) == -1
    assert call(args(q=odd)) == -3
    assert call(args(Hkv=3)) == -1
    assert call(args(D=96)) == -2
    assert call(args(Sq=0)) == -1
    assert call(args(scale=0.0)) == -1
    assert call(args(mod=9)) == -1
    assert call(args(mod=3)) == -1   # softcap needs params
    assert call(args(mod=6)) == -1   # document mask needs offsets
    # composed codes: unknown flag bits or kinds, and the components' own parameters
    assert call(args(mod=0x1000)) == -1
    assert call(args(mod=2 | 0x1000)) == -1
    assert call(args(mod=0x800)) == -1        # bitmap flag needs the bitmap
    assert call(args(mod=7 | 0x100)) == -1
    assert call(args(mod=0x400)) == -1        # document flag needs offsets
    assert call(args(mod=2 | 0x200)) == -1    # window flag needs params
    assert call(args(mod=3 | 0x100)) == -1    # softcap component needs params


def test_strerror(lib):
    lib.attn_strerror.restype = ctypes.c_char_p
    assert b"timed out" in lib.attn_strerror(-6)
    assert lib.attn_strerror(0) == b"ok"


def test_composed_and_bitmap_argument_rules(lib):
    """Composite mod codes and bitmap fields are validated before any device
    work: a valid call gets as far as the device lookup (ATTN_ERR_DEVICE here,
    with no GPU), an invalid one stops at ATTN_ERR_ARG / ATTN_ERR_ALIGN."""
    import tiled_attention_25_b200.abi as abi
    P, I = ctypes.c_void_p, ctypes.c_int
    lib.attn_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, I, ctypes.c_float, I, P, P, P]
    lib.build_block_mask.argtypes = [I, P, I, I, I, P, P]
    good = ctypes.c_void_p(1 << 32)
    DEVICE, ARG, ALIGN = -7, -1, -3

    def params(bitmap=1 << 32, row_words=8, heads=1, head_stride=0, batch_stride=0, window=100):
        return abi.CModParams(50.0, window, 1.1, 128, None, None, 0, ctypes.c_void_p(bitmap), row_words,
                              heads, head_stride, batch_stride)

    def fwd(mod, mp, Hq=4, Skv=256, bm=None):
        return lib.attn_fwd(good, good, good, good, None, 1, Hq, 2, 256, Skv, 128, 0.1, mod,
                            None if mp is None else ctypes.byref(mp), bm, None)

    # composites that need no parameters, or get them
    assert fwd(0x100 | 2, None) == DEVICE
    assert fwd(4 | 0x400, params()) == ARG          # document flag without offsets
    assert fwd(0x200 | 3, params()) == DEVICE       # softcap + window
    assert fwd(0x200, params(window=0)) == ARG
    # the bitmap: a block mask is required for attn_fwd
    assert fwd(0x800, params()) == ARG
    n = ctypes.c_size_t(1 << 20)
    m = abi.CBlockMask()
    assert lib.attn_block_mask_bind(ctypes.c_void_p(1 << 40), n, 1, 256, 256, ctypes.byref(m)) == 0
    bm = ctypes.byref(m)
    # build_block_mask checks the bitmap fields
    build = lambda mod, mp: lib.build_block_mask(mod, ctypes.byref(mp), 1, 256, 256, bm, None)
    assert build(0x800, params()) == DEVICE
    assert build(0x800 | 0x100, params(heads=3, head_stride=256 * 8)) == DEVICE
    assert build(0x800, params(bitmap=(1 << 32) + 4)) == ALIGN
    assert build(0x800, params(row_words=4)) == ARG           # < ceil(256 / 32)
    assert build(0x800, params(row_words=10)) == ARG          # not a multiple of 4
    assert build(0x800, params(heads=0)) == ARG
    assert build(0x800, params(heads=1, head_stride=64)) == ARG
    assert build(0x800, params(batch_stride=6)) == ARG
    assert build(0x800, params(bitmap=0)) == ARG
    # the mask records the canonical code, which attn_fwd compares with its own
    m.mod_kind = 0x800 | 0x100       # what building NONE | BITMAP | CAUSAL records
    assert fwd(1 | 0x800, params(), bm=bm) == DEVICE  # causal kind with the bitmap flag: same mod
    assert fwd(0x800, params(), bm=bm) == ARG         # another mod
    # per-head bitmaps must match the call's query heads
    m.mod_kind = 0x800
    assert fwd(0x800, params(heads=4, head_stride=256 * 8), bm=bm) == DEVICE
    assert fwd(0x800, params(heads=3, head_stride=256 * 8), bm=bm) == ARG


def test_binding_marshals_bitmap_extents():
    """The binding turns a bitmap tensor's shape into the C strides, and
    refuses a tensor that does not cover the call's batch rows, heads and
    query rows (the C side cannot see its extent)."""
    import torch

    import tiled_attention_25_b200.abi as abi
    S, rw = 300, 12
    for shape, heads, hs, bs in (((1, 1, S, rw), 1, 0, 0), ((2, 1, S, rw), 1, 0, S * rw),
                                 ((2, 4, S, rw), 4, S * rw, 4 * S * rw)):
        mp = abi.ModParams(bitmap=torch.zeros(shape, dtype=torch.int32))
        c = mp.c()
        assert (c.bitmap_row_words, c.bitmap_heads, c.bitmap_head_stride, c.bitmap_batch_stride) == (rw, heads, hs, bs)
        assert c.bitmap == mp.bitmap.data_ptr()
        assert abi._mp(mp, abi.MASK_BITMAP, 2, 4, S) is not None
    bad = [((3, 1, S, rw), 2, 4, S), ((1, 3, S, rw), 2, 4, S), ((1, 1, S - 1, rw), 2, 4, S)]
    for shape, B, Hq, Sq in bad:
        mp = abi.ModParams(bitmap=torch.zeros(shape, dtype=torch.int32))
        with pytest.raises(ValueError):
            abi._mp(mp, abi.MASK_BITMAP, B, Hq, Sq)
    # without the flag the bitmap is not read, so its shape does not matter
    mp = abi.ModParams(bitmap=torch.zeros((3, 3, 1, rw), dtype=torch.int32))
    assert abi._mp(mp, abi.MOD_CAUSAL, 2, 4, S) is not None


def test_every_mod_code_is_valid_exactly_when_the_oracle_accepts_it(lib):
    """All 4096 codes below 0x1000: the C boundary and the oracle agree on which
    are mods.  Parameters are given for every component, so a valid code passes
    the checks and stops at the device lookup (ATTN_ERR_DEVICE here)."""
    import oracle
    import tiled_attention_25_b200.abi as abi
    P, I = ctypes.c_void_p, ctypes.c_int
    lib.build_block_mask.argtypes = [I, P, I, I, I, P, P]
    mp = abi.CModParams(50.0, 100, 1.1, 128, None, ctypes.c_void_p(1 << 32), 2, ctypes.c_void_p(1 << 32),
                        8, 1, 0, 0)
    m = abi.CBlockMask()
    assert lib.attn_block_mask_bind(ctypes.c_void_p(1 << 40), ctypes.c_size_t(1 << 20), 1, 256, 256,
                                    ctypes.byref(m)) == 0
    for code in range(0x1000):
        try:
            oracle.split_mod(code)
            valid = True
        except ValueError:
            valid = False
        rc = lib.build_block_mask(code, ctypes.byref(mp), 1, 256, 256, ctypes.byref(m), None)
        assert rc == (-7 if valid else -1), (hex(code), rc)
