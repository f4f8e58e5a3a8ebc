"""ctypes binding of libattn25.so — argument marshalling only.

Every function here has the name of the C entry point it calls (declared in
include/attn25.h) and does no attention work of its own: it checks tensor
metadata, turns torch tensors into device pointers and sizes, and raises
AttnError on a non-zero status.  PyTorch provides device memory and streams.
There is no fallback: if the shared library is missing or fails to load,
importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# ATTN25_LIBRARY may name the profiling build (libattn25_trace.so) instead.
LIB_PATH = os.environ.get("ATTN25_LIBRARY") or os.path.join(_HERE, "libattn25.so")

MOD_NONE = 0
MOD_CAUSAL = 1
MOD_ALIBI = 2
MOD_SOFTCAP = 3
MOD_SLIDING_WINDOW = 4
MOD_LOCAL_BOOST = 5
MOD_DOCUMENT = 6
# Mask flags ORed onto a kind to compose mods (score transform of the kind,
# AND of the masks).
MASK_CAUSAL = 0x100
MASK_SLIDING_WINDOW = 0x200
MASK_DOCUMENT = 0x400
MASK_BITMAP = 0x800
MASK_VARLEN = 0x1000

ATTN_ERR_TIMEOUT = -6


class AttnError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {code} ({attn_strerror(code)})")
        self.code = code


class CModParams(ctypes.Structure):
    _fields_ = [
        ("softcap", ctypes.c_float),
        ("window", ctypes.c_int32),
        ("boost", ctypes.c_float),
        ("boost_radius", ctypes.c_int32),
        ("alibi_slopes", ctypes.c_void_p),
        ("doc_offsets", ctypes.c_void_p),
        ("num_docs", ctypes.c_int32),
        ("bitmap", ctypes.c_void_p),
        ("bitmap_row_words", ctypes.c_int32),
        ("bitmap_heads", ctypes.c_int32),
        ("bitmap_head_stride", ctypes.c_int64),
        ("bitmap_batch_stride", ctypes.c_int64),
        ("q_offsets", ctypes.c_void_p),
        ("k_offsets", ctypes.c_void_p),
        ("num_seqs", ctypes.c_int32),
    ]


class CStrides(ctypes.Structure):
    _fields_ = [("b", ctypes.c_int64), ("h", ctypes.c_int64), ("s", ctypes.c_int64)]


class CLayouts(ctypes.Structure):
    _fields_ = [(n, CStrides) for n in ("q", "k", "v", "out", "dout", "dq", "dk", "dv")]


class CBlockMask(ctypes.Structure):
    _fields_ = [
        ("tile_class", ctypes.c_void_p),
        ("kv_count", ctypes.c_void_p),
        ("kv_index", ctypes.c_void_p),
        ("q_count", ctypes.c_void_p),
        ("q_index", ctypes.c_void_p),
        ("fwd_order", ctypes.c_void_p),
        ("bwd_order", ctypes.c_void_p),
        ("B", ctypes.c_int32),
        ("Sq", ctypes.c_int32),
        ("Skv", ctypes.c_int32),
        ("nq_tiles", ctypes.c_int32),
        ("nk_tiles", ctypes.c_int32),
        ("mod_kind", ctypes.c_int32),
    ]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python tiled_attention_25_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.attn_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, I, P, P, P]
    lib.attn_fwd.restype = I
    lib.attn_bwd.argtypes = [P, P, P, P, P, P, P, P, P, P, S, I, I, I, I, I, I, F, I, P, P, P]
    lib.attn_bwd.restype = I
    lib.attn_bwd_noalloc.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, P, P, P]
    lib.attn_bwd_noalloc.restype = I
    lib.attn_bwd_noalloc_max_workspace.argtypes = []
    lib.attn_bwd_noalloc_max_workspace.restype = S
    lib.attn_bwd_workspace_size.argtypes = [I, I, I, I]
    lib.attn_bwd_workspace_size.restype = S
    lib.attn_block_mask_bytes.argtypes = [I, I, I]
    lib.attn_block_mask_bytes.restype = S
    lib.attn_block_mask_bind.argtypes = [P, S, I, I, I, ctypes.POINTER(CBlockMask)]
    lib.attn_block_mask_bind.restype = I
    lib.build_block_mask.argtypes = [I, P, I, I, I, ctypes.POINTER(CBlockMask), P]
    lib.build_block_mask.restype = I
    lib.attn_fwd_strided.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, I, P, P, P, P]
    lib.attn_fwd_strided.restype = I
    lib.attn_bwd_strided.argtypes = [P, P, P, P, P, P, P, P, P, P, S, I, I, I, I, I, I, F, I, P, P, P, P]
    lib.attn_bwd_strided.restype = I
    lib.attn_bwd_deterministic.argtypes = [P, P, P, P, P, P, P, P, P, P, S, I, I, I, I, I, I, F, I, P, P, P]
    lib.attn_bwd_deterministic.restype = I
    lib.attn_bwd_deterministic_workspace_size.argtypes = [I, I, I, I]
    lib.attn_bwd_deterministic_workspace_size.restype = S
    lib.attn_fwd_fp8.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, P, P, P]
    lib.attn_fwd_fp8.restype = I
    lib.attn_fp8_rotate_quantize.argtypes = [P, P, P, P, I, I, I, I, P]
    lib.attn_fp8_rotate_quantize.restype = I
    lib.attn_get_status.argtypes = [P]
    lib.attn_get_status.restype = I
    lib.attn_set_wait_limit_ms.argtypes = [ctypes.c_uint32]
    lib.attn_set_wait_limit_ms.restype = None
    lib.attn_set_work_walk.argtypes = [I]
    lib.attn_set_work_walk.restype = I
    lib.attn_check_wait_timeout.argtypes = [P]
    lib.attn_check_wait_timeout.restype = I
    lib.attn_strerror.argtypes = [I]
    lib.attn_strerror.restype = ctypes.c_char_p
    if hasattr(lib, "attn_trace_read"):  # profiling build only
        lib.attn_trace_read.argtypes = [ctypes.POINTER(ctypes.c_ulonglong), I]
        lib.attn_trace_read.restype = I
        lib.attn_trace_reset.argtypes = []
        lib.attn_trace_reset.restype = I
        lib.attn_trace_window.argtypes = [I]
        lib.attn_trace_window.restype = I
    return lib


LIB = _load()

EXPORTED = ("attn_fwd", "attn_bwd", "attn_bwd_workspace_size", "attn_bwd_noalloc",
            "attn_bwd_noalloc_max_workspace", "attn_block_mask_bytes",
            "attn_block_mask_bind", "build_block_mask", "attn_get_status",
            "attn_set_wait_limit_ms", "attn_strerror", "attn_fwd_strided", "attn_bwd_strided",
            "attn_bwd_deterministic", "attn_bwd_deterministic_workspace_size", "attn_check_wait_timeout",
            "attn_fp8_rotate_quantize", "attn_fwd_fp8", "attn_set_work_walk")


def attn_strerror(code: int) -> str:
    return LIB.attn_strerror(int(code)).decode()


def _check(code: int, what: str):
    if code != 0:
        raise AttnError(code, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


class ModParams:
    """Mod scalars plus the device tensors they point at (kept alive here)."""

    def __init__(self, softcap=50.0, window=1024, boost=1.1, boost_radius=128,
                 alibi_slopes=None, doc_offsets=None, bitmap=None, q_offsets=None, k_offsets=None):
        self.softcap = float(softcap)
        self.window = int(window)
        self.boost = float(boost)
        self.boost_radius = int(boost_radius)
        self.alibi_slopes = alibi_slopes        # device fp32 [Hq] or None
        self.doc_offsets = doc_offsets          # device int32 [B][num_docs+1] or None
        if doc_offsets is not None:
            assert doc_offsets.dtype == torch.int32 and doc_offsets.is_contiguous() and doc_offsets.dim() == 2
        if alibi_slopes is not None:
            assert alibi_slopes.dtype == torch.float32 and alibi_slopes.is_contiguous()
        # device int32 [B or 1][Hq or 1][Sq][row_words] keep bits (bit j & 31 of word j >> 5)
        # device int32 [B][num_seqs + 1] each: the varlen mask's query and key offsets
        self.q_offsets, self.k_offsets = q_offsets, k_offsets
        if (q_offsets is None) != (k_offsets is None):
            raise ValueError("the varlen mask needs both query and key offsets")
        if q_offsets is not None:
            for t in (q_offsets, k_offsets):
                assert t.dtype == torch.int32 and t.is_contiguous() and t.dim() == 2
            assert q_offsets.shape == k_offsets.shape
        self.bitmap = bitmap
        if bitmap is not None:
            assert bitmap.dtype == torch.int32 and bitmap.is_contiguous() and bitmap.dim() == 4

    def c(self) -> CModParams:
        bm = self.bitmap
        if bm is None:
            bm_args = (None, 0, 0, 0, 0)
        else:
            nb, nh, sq, rw = bm.shape
            bm_args = (bm.data_ptr(), rw, nh, 0 if nh == 1 else sq * rw, 0 if nb == 1 else nh * sq * rw)
        return CModParams(self.softcap, self.window, self.boost, self.boost_radius,
                          None if self.alibi_slopes is None else self.alibi_slopes.data_ptr(),
                          None if self.doc_offsets is None else self.doc_offsets.data_ptr(),
                          0 if self.doc_offsets is None else self.doc_offsets.shape[1] - 1, *bm_args,
                          None if self.q_offsets is None else self.q_offsets.data_ptr(),
                          None if self.k_offsets is None else self.k_offsets.data_ptr(),
                          0 if self.q_offsets is None else self.q_offsets.shape[1] - 1)


class BlockMask:
    """A bound block mask: the C struct plus the device buffer that holds it."""

    def __init__(self, buffer: torch.Tensor, c: CBlockMask):
        self.buffer = buffer
        self.c = c

    def view(self, name):
        """The named array as a torch view of the buffer (for inspection and tests)."""
        c = self.c
        B, nq, nk = c.B, c.nq_tiles, c.nk_tiles
        npairs = (nq + 1) // 2
        shapes = {"tile_class": (torch.uint8, (B, nq, nk)), "kv_count": (torch.int32, (B, nq)),
                  "kv_index": (torch.int32, (B, nq, nk)), "q_count": (torch.int32, (B, nk)),
                  "q_index": (torch.int32, (B, nk, nq)), "fwd_order": (torch.int32, (B * npairs,)),
                  "bwd_order": (torch.int32, (B * nk,))}
        dtype, shape = shapes[name]
        off = getattr(c, name) - self.buffer.data_ptr()
        n = 1
        for s in shape:
            n *= s
        size = n * (1 if dtype == torch.uint8 else 4)
        return self.buffer[off:off + size].view(dtype).view(shape)


def _mp(mod_params, mod_kind, B, Hq, Sq):
    """Marshal the mod params; a bitmap tensor must cover every (b, h, row) the
    call reads (the C side cannot see its extent)."""
    if mod_params is None:
        return None
    code = int(mod_kind)
    # offsets arrays: one row per batch row (the C side cannot see their extent)
    if (code & 0xFF) == MOD_DOCUMENT or code & MASK_DOCUMENT:
        t = mod_params.doc_offsets
        if t is None or t.shape[0] < B:
            raise ValueError(f"the document mask needs doc_offsets with {B} rows")
    if code & MASK_VARLEN:
        t = mod_params.q_offsets
        if t is None or t.shape[0] < B:
            raise ValueError(f"the varlen mask needs q_offsets and k_offsets with {B} rows")
    bm = mod_params.bitmap
    if int(mod_kind) & MASK_BITMAP and bm is not None:
        nb, nh, sq, _ = bm.shape
        if nb not in (1, B) or (Hq is not None and nh not in (1, Hq)) or sq < Sq:
            raise ValueError(f"bitmap of shape {tuple(bm.shape)} does not cover B={B}, Hq={Hq}, Sq={Sq}")
    cm = mod_params.c()
    return ctypes.byref(cm), cm


def _dims(q, k, v, out):
    for t in (q, k, v, out):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError("q, k, v, out must be contiguous CUDA bf16 [B][H][S][D] tensors")
    B, Hq, Sq, D = q.shape
    Bk, Hkv, Skv, Dk = k.shape
    if tuple(v.shape) != (Bk, Hkv, Skv, Dk) or Bk != B or Dk != D or tuple(out.shape) != (B, Hq, Sq, D):
        raise ValueError("inconsistent q/k/v/out shapes")
    return B, Hq, Hkv, Sq, Skv, D


def attn_fwd(q, k, v, out, lse=None, scale=None, mod_kind=MOD_NONE, mod_params=None,
             block_mask=None, stream=None):
    B, Hq, Hkv, Sq, Skv, D = _dims(q, k, v, out)
    if lse is not None and (lse.dtype != torch.float32 or tuple(lse.shape) != (B, Hq, Sq) or not lse.is_contiguous()):
        raise ValueError("lse must be a contiguous fp32 [B][Hq][Sq] tensor")
    scale = D ** -0.5 if scale is None else float(scale)
    mp = _mp(mod_params, mod_kind, B, Hq, Sq)
    rc = LIB.attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Sq, Skv, D,
                      scale, int(mod_kind), None if mp is None else mp[0],
                      None if block_mask is None else ctypes.byref(block_mask.c), _stream(stream))
    _check(rc, "attn_fwd")


def _strides(t, shape, what):
    """Element strides (b, h, s) of a [B][H][S][D] CUDA bf16 view with D contiguous."""
    if t.dtype != torch.bfloat16 or not t.is_cuda or t.dim() != 4 or tuple(t.shape) != tuple(shape) \
            or t.stride(3) != 1:
        raise ValueError(f"{what} must be a CUDA bf16 {tuple(shape)} view with its last dimension contiguous")
    return CStrides(t.stride(0), t.stride(1), t.stride(2))


def _layouts(**views):
    lay = CLayouts()
    for name, (t, shape) in views.items():
        setattr(lay, name, _strides(t, shape, name))
    return lay


def attn_fwd_strided(q, k, v, out, lse=None, scale=None, mod_kind=MOD_NONE, mod_params=None, block_mask=None,
                     stream=None):
    """attn_fwd on [B][H][S][D] views of any strides whose last dimension is
    contiguous (e.g. x.permute(0, 2, 1, 3) of a [B][S][H][D] tensor)."""
    B, Hq, Sq, D = q.shape
    _, Hkv, Skv, _ = k.shape
    lay = _layouts(q=(q, (B, Hq, Sq, D)), k=(k, (B, Hkv, Skv, D)), v=(v, (B, Hkv, Skv, D)),
                   out=(out, (B, Hq, Sq, D)))
    if lse is not None and (lse.dtype != torch.float32 or tuple(lse.shape) != (B, Hq, Sq) or not lse.is_contiguous()):
        raise ValueError("lse must be a contiguous fp32 [B][Hq][Sq] tensor")
    scale = D ** -0.5 if scale is None else float(scale)
    mp = _mp(mod_params, mod_kind, B, Hq, Sq)
    rc = LIB.attn_fwd_strided(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Sq, Skv, D, scale,
                              int(mod_kind), None if mp is None else mp[0],
                              None if block_mask is None else ctypes.byref(block_mask.c), ctypes.byref(lay),
                              _stream(stream))
    _check(rc, "attn_fwd_strided")


def attn_bwd_strided(q, k, v, out, lse, dout, dq, dk, dv, workspace, scale=None, mod_kind=MOD_NONE,
                     mod_params=None, block_mask=None, stream=None):
    """attn_bwd on strided views (see attn_fwd_strided)."""
    B, Hq, Sq, D = q.shape
    _, Hkv, Skv, _ = k.shape
    qs, ks = (B, Hq, Sq, D), (B, Hkv, Skv, D)
    lay = _layouts(q=(q, qs), k=(k, ks), v=(v, ks), out=(out, qs), dout=(dout, qs), dq=(dq, qs), dk=(dk, ks),
                   dv=(dv, ks))
    scale = D ** -0.5 if scale is None else float(scale)
    mp = _mp(mod_params, mod_kind, B, Hq, Sq)
    rc = LIB.attn_bwd_strided(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk),
                              _ptr(dv), _ptr(workspace), workspace.numel() * workspace.element_size(), B, Hq, Hkv,
                              Sq, Skv, D, scale, int(mod_kind), None if mp is None else mp[0],
                              None if block_mask is None else ctypes.byref(block_mask.c), ctypes.byref(lay),
                              _stream(stream))
    _check(rc, "attn_bwd_strided")


def attn_fp8_rotate_quantize(x, signs, codes, scales, stream=None):
    """x: CUDA bf16 [B][H][S][D]; signs: CUDA int8 [D] of +-1; codes: CUDA uint8
    like x; scales: CUDA fp32 [B][H]."""
    if x.dtype != torch.bfloat16 or not x.is_cuda or not x.is_contiguous() or x.dim() != 4:
        raise ValueError("x must be a contiguous CUDA bf16 [B][H][S][D] tensor")
    B, H, S, D = x.shape
    if signs.dtype != torch.int8 or tuple(signs.shape) != (D,) or not signs.is_contiguous():
        raise ValueError("signs must be a contiguous int8 [D] tensor")
    if codes.dtype != torch.uint8 or tuple(codes.shape) != (B, H, S, D) or not codes.is_contiguous():
        raise ValueError("codes must be a contiguous uint8 tensor shaped like x")
    if scales.dtype != torch.float32 or tuple(scales.shape) != (B, H) or not scales.is_contiguous():
        raise ValueError("scales must be a contiguous fp32 [B][H] tensor")
    _check(LIB.attn_fp8_rotate_quantize(_ptr(x), _ptr(signs), _ptr(codes), _ptr(scales), B, H, S, D,
                                        _stream(stream)), "attn_fp8_rotate_quantize")


def attn_fwd_fp8(q8, k8, q_scales, k_scales, v, out, lse=None, scale=None, mod_kind=MOD_NONE, mod_params=None,
                 block_mask=None, stream=None):
    """The forward with e4m3 Q and K (codes from attn_fp8_rotate_quantize)."""
    for t, name in ((q8, "q8"), (k8, "k8")):
        if t.dtype != torch.uint8 or not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name} must be a contiguous CUDA uint8 [B][H][S][D] tensor")
    B, Hq, Sq, D = q8.shape
    Bk, Hkv, Skv, Dk = k8.shape
    if (Bk, Dk) != (B, D) or tuple(v.shape) != (B, Hkv, Skv, D) or tuple(out.shape) != (B, Hq, Sq, D):
        raise ValueError("inconsistent q8/k8/v/out shapes")
    for t in (v, out):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("v and out must be contiguous CUDA bf16 tensors")
    if tuple(q_scales.shape) != (B, Hq) or tuple(k_scales.shape) != (B, Hkv):
        raise ValueError("q_scales must be [B][Hq] and k_scales [B][Hkv]")
    if lse is not None and (lse.dtype != torch.float32 or tuple(lse.shape) != (B, Hq, Sq) or not lse.is_contiguous()):
        raise ValueError("lse must be a contiguous fp32 [B][Hq][Sq] tensor")
    scale = D ** -0.5 if scale is None else float(scale)
    mp = _mp(mod_params, mod_kind, B, Hq, Sq)
    rc = LIB.attn_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(q_scales), _ptr(k_scales), _ptr(v), _ptr(out), _ptr(lse),
                          B, Hq, Hkv, Sq, Skv, D, scale, int(mod_kind), None if mp is None else mp[0],
                          None if block_mask is None else ctypes.byref(block_mask.c), _stream(stream))
    _check(rc, "attn_fwd_fp8")


def attn_bwd_deterministic_workspace_size(B, Hq, Sq, D) -> int:
    return int(LIB.attn_bwd_deterministic_workspace_size(B, Hq, Sq, D))


def attn_bwd_deterministic(q, k, v, out, lse, dout, dq, dk, dv, workspace, scale=None, mod_kind=MOD_NONE,
                           mod_params=None, block_mask=None, stream=None):
    """attn_bwd with a bitwise reproducible dQ (see include/attn25.h)."""
    B, Hq, Hkv, Sq, Skv, D = _dims(q, k, v, out)
    for t in (dout, dq):
        if t.dtype != torch.bfloat16 or tuple(t.shape) != (B, Hq, Sq, D) or not t.is_contiguous():
            raise ValueError("dout/dq must be contiguous bf16 like q")
    for t in (dk, dv):
        if t.dtype != torch.bfloat16 or tuple(t.shape) != (B, Hkv, Skv, D) or not t.is_contiguous():
            raise ValueError("dk/dv must be contiguous bf16 like k")
    scale = D ** -0.5 if scale is None else float(scale)
    mp = _mp(mod_params, mod_kind, B, Hq, Sq)
    rc = LIB.attn_bwd_deterministic(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq),
                                    _ptr(dk), _ptr(dv), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), B, Hq, Hkv, Sq, Skv, D,
                                    scale, int(mod_kind), None if mp is None else mp[0],
                                    None if block_mask is None else ctypes.byref(block_mask.c), _stream(stream))
    _check(rc, "attn_bwd_deterministic")


def attn_bwd_workspace_size(B, Hq, Sq, D) -> int:
    return int(LIB.attn_bwd_workspace_size(B, Hq, Sq, D))


def attn_bwd(q, k, v, out, lse, dout, dq, dk, dv, workspace, scale=None, mod_kind=MOD_NONE,
             mod_params=None, block_mask=None, stream=None):
    B, Hq, Hkv, Sq, Skv, D = _dims(q, k, v, out)
    for t in (dout, dq):
        if t.dtype != torch.bfloat16 or tuple(t.shape) != (B, Hq, Sq, D) or not t.is_contiguous():
            raise ValueError("dout/dq must be contiguous bf16 like q")
    for t in (dk, dv):
        if t.dtype != torch.bfloat16 or tuple(t.shape) != (B, Hkv, Skv, D) or not t.is_contiguous():
            raise ValueError("dk/dv must be contiguous bf16 like k")
    scale = D ** -0.5 if scale is None else float(scale)
    mp = _mp(mod_params, mod_kind, B, Hq, Sq)
    rc = LIB.attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq),
                      _ptr(dk), _ptr(dv), _ptr(workspace), workspace.numel() * workspace.element_size(),
                      B, Hq, Hkv, Sq, Skv, D, scale, int(mod_kind), None if mp is None else mp[0],
                      None if block_mask is None else ctypes.byref(block_mask.c), _stream(stream))
    _check(rc, "attn_bwd")


def attn_bwd_noalloc(q, k, v, out, lse, dout, dq, dk, dv, scale=None, mod_kind=MOD_NONE,
                     mod_params=None, block_mask=None, stream=None):
    """attn_bwd on the library's own fixed workspace (see include/attn25.h)."""
    B, Hq, Hkv, Sq, Skv, D = _dims(q, k, v, out)
    for t in (dout, dq):
        if t.dtype != torch.bfloat16 or tuple(t.shape) != (B, Hq, Sq, D) or not t.is_contiguous():
            raise ValueError("dout/dq must be contiguous bf16 like q")
    for t in (dk, dv):
        if t.dtype != torch.bfloat16 or tuple(t.shape) != (B, Hkv, Skv, D) or not t.is_contiguous():
            raise ValueError("dk/dv must be contiguous bf16 like k")
    scale = D ** -0.5 if scale is None else float(scale)
    mp = _mp(mod_params, mod_kind, B, Hq, Sq)
    rc = LIB.attn_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq),
                              _ptr(dk), _ptr(dv), B, Hq, Hkv, Sq, Skv, D, scale, int(mod_kind),
                              None if mp is None else mp[0],
                              None if block_mask is None else ctypes.byref(block_mask.c), _stream(stream))
    _check(rc, "attn_bwd_noalloc")


def attn_bwd_noalloc_max_workspace() -> int:
    return int(LIB.attn_bwd_noalloc_max_workspace())


def attn_block_mask_bytes(B, Sq, Skv) -> int:
    return int(LIB.attn_block_mask_bytes(B, Sq, Skv))


def attn_block_mask_bind(buffer, B, Sq, Skv) -> BlockMask:
    c = CBlockMask()
    rc = LIB.attn_block_mask_bind(_ptr(buffer), buffer.numel() * buffer.element_size(), B, Sq, Skv,
                                  ctypes.byref(c))
    _check(rc, "attn_block_mask_bind")
    return BlockMask(buffer, c)


def build_block_mask(mod_kind, mod_params, B, Sq, Skv, mask: BlockMask, stream=None):
    mp = _mp(mod_params, mod_kind, B, None, Sq)
    rc = LIB.build_block_mask(int(mod_kind), None if mp is None else mp[0], B, Sq, Skv,
                              ctypes.byref(mask.c), _stream(stream))
    _check(rc, "build_block_mask")


def attn_get_status(stream=None) -> int:
    return int(LIB.attn_get_status(_stream(stream)))


def attn_set_wait_limit_ms(ms: int):
    LIB.attn_set_wait_limit_ms(int(ms))


WALK_STATIC = 0
WALK_CLUSTER_LAUNCH_CONTROL = 1
WALK_DEFAULT = WALK_CLUSTER_LAUNCH_CONTROL


def attn_set_work_walk(walk: int):
    """How the persistent kernels take their work units (see include/attn25.h)."""
    _check(LIB.attn_set_work_walk(int(walk)), "attn_set_work_walk")


def attn_check_wait_timeout(stream=None):
    """Launch the timeout self-check (see include/attn25.h); read the outcome
    with attn_get_status."""
    _check(LIB.attn_check_wait_timeout(_stream(stream)), "attn_check_wait_timeout")


def attn_trace_read(n: int = 256) -> list:
    """Per-role cycle counters of the profiling build (libattn25_trace.so)."""
    buf = (ctypes.c_ulonglong * n)()
    _check(LIB.attn_trace_read(buf, n), "attn_trace_read")
    return list(buf)


def attn_trace_reset():
    _check(LIB.attn_trace_reset(), "attn_trace_reset")


def attn_trace_window(first_step: int):
    """First backward step whose per-role event clocks the profiling build records."""
    _check(LIB.attn_trace_window(first_step), "attn_trace_window")
