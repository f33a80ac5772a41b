"""Python binding of libfbk.so (the cached block attention C ABI, include/fbk.h).

Argument marshalling only: every step of the computation runs in the CUDA
library. Tensors are torch CUDA tensors (device memory and streams come from
PyTorch); their data pointers and the current CUDA stream are passed through
ctypes. Importing this module fails loudly when the library is not built.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfbk.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m cached_block_attention_b200.build` "
        "(there is no fallback implementation)")
_lib = ctypes.CDLL(LIB_PATH)

OK = 0
BF16 = 0
FP32_CHECK = 1

DEVERR_PREFIX_LEN = 1
DEVERR_PAGE_ID = 2
DEVERR_COMMIT = 4
DEVERR_TIMEOUT = 8

EXPORTS = ("fbk_prefix_workspace_bytes", "fbk_default_num_splits", "fbk_prefix_partial",
           "fbk_block_attn_merge", "fbk_commit_block_rope_append", "fbk_full_ref_attn",
           "fbk_status_string", "fbk_prefix_partial_static_scratch", "fbk_decode_block",
           "fbk_fp8_group_quant", "fbk_facache_unchanged_rows", "fbk_prefix_partial_at",
           "fbk_facache_workspace_bytes", "fbk_facache_refresh", "fbk_facache_step", "fbk_page_means",
           "fbk_select_pages_workspace_bytes", "fbk_select_pages", "fbk_residual_capture", "fbk_residual_apply",
           "fbk_decode_block_adaptive")

STATIC_SCRATCH_BYTES = 32 << 20  # FBK_STATIC_SCRATCH_BYTES


class _Shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("block_len", ctypes.c_int32), ("softmax_scale", ctypes.c_float),
                ("rope_base", ctypes.c_double), ("mode", ctypes.c_int32)]


class _Cache(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("paged", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32),
                ("capacity_tokens", ctypes.c_int64), ("num_pages", ctypes.c_int64),
                ("page_table", ctypes.c_void_p), ("prefix_lens", ctypes.c_void_p),
                ("error_flags", ctypes.c_void_p)]


class _Partial(ctypes.Structure):
    _fields_ = [("o_unnorm", ctypes.c_void_p), ("m", ctypes.c_void_p), ("l", ctypes.c_void_p)]


class _LayerBlock(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("cache", _Cache), ("prefix", _Partial), ("out", ctypes.c_void_p),
                ("lse", ctypes.c_void_p), ("refresh_interval", ctypes.c_int32)]


_P = ctypes.POINTER
_vp = ctypes.c_void_p
_lib.fbk_prefix_workspace_bytes.argtypes = [_P(_Shape), _P(_Cache), ctypes.c_int32]
_lib.fbk_prefix_workspace_bytes.restype = ctypes.c_size_t
_lib.fbk_default_num_splits.argtypes = []
_lib.fbk_default_num_splits.restype = ctypes.c_int32
_lib.fbk_prefix_partial.argtypes = [_P(_Shape), _vp, _P(_Cache), _P(_Partial), _vp, ctypes.c_size_t,
                                    ctypes.c_int32, _vp]
_lib.fbk_prefix_partial.restype = ctypes.c_int
_lib.fbk_block_attn_merge.argtypes = [_P(_Shape), _vp, _vp, _vp, _vp, _P(_Partial), _vp, _vp, _vp]
_lib.fbk_block_attn_merge.restype = ctypes.c_int
_lib.fbk_commit_block_rope_append.argtypes = [_P(_Shape), _vp, _vp, _P(_Cache), _vp]
_lib.fbk_commit_block_rope_append.restype = ctypes.c_int
_lib.fbk_full_ref_attn.argtypes = [_P(_Shape), _vp, _vp, _vp, _P(_Cache), _vp, _vp, _vp]
_lib.fbk_full_ref_attn.restype = ctypes.c_int
_lib.fbk_prefix_partial_static_scratch.argtypes = [_P(_Shape), _vp, _P(_Cache), _P(_Partial),
                                                   ctypes.c_int32, _vp]
_lib.fbk_prefix_partial_static_scratch.restype = ctypes.c_int
_lib.fbk_decode_block.argtypes = [_P(_Shape), _P(_LayerBlock), ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                  _vp, ctypes.c_size_t, ctypes.c_int32, _vp]
_lib.fbk_decode_block.restype = ctypes.c_int


class _DriftPolicy(ctypes.Structure):
    _fields_ = [("threshold", ctypes.c_float), ("flags", ctypes.c_void_p), ("last_refresh", ctypes.c_void_p),
                ("drift", ctypes.c_void_p), ("refreshed", ctypes.c_void_p)]


_lib.fbk_decode_block_adaptive.argtypes = [_P(_Shape), _P(_LayerBlock), ctypes.c_int32, ctypes.c_int32,
                                           ctypes.c_int32, _P(_DriftPolicy), _vp, ctypes.c_size_t, ctypes.c_int32,
                                           _vp]
_lib.fbk_decode_block_adaptive.restype = ctypes.c_int
_lib.fbk_fp8_group_quant.argtypes = [_vp, ctypes.c_int64, ctypes.c_int64, _vp, _vp, _vp]
_lib.fbk_fp8_group_quant.restype = ctypes.c_int
_lib.fbk_facache_unchanged_rows.argtypes = [_P(_Shape), ctypes.c_int32, _vp, _P(_Partial), _vp, _vp, _vp, _vp,
                                            _vp, _vp]
_lib.fbk_facache_unchanged_rows.restype = ctypes.c_int
_lib.fbk_prefix_partial_at.argtypes = [_P(_Shape), _vp, _vp, _P(_Cache), _P(_Partial), _vp, ctypes.c_size_t,
                                       ctypes.c_int32, _vp]
_lib.fbk_prefix_partial_at.restype = ctypes.c_int
_lib.fbk_facache_workspace_bytes.argtypes = [_P(_Shape), ctypes.c_int32, ctypes.c_int32]
_lib.fbk_facache_workspace_bytes.restype = ctypes.c_size_t
_lib.fbk_facache_refresh.argtypes = [_P(_Shape), ctypes.c_int32, _vp, _P(ctypes.c_int32), _P(_Cache), _P(_Partial),
                                     _vp, ctypes.c_size_t, ctypes.c_int32, _vp]
_lib.fbk_facache_refresh.restype = ctypes.c_int
_lib.fbk_facache_step.argtypes = [_P(_Shape), ctypes.c_int32, _vp, _P(_Partial), _vp, _vp, _vp, _vp, _P(_Cache), _vp,
                                  _vp, _vp, _vp, _vp, ctypes.c_size_t, ctypes.c_int32, _vp]
_lib.fbk_facache_step.restype = ctypes.c_int
_lib.fbk_page_means.argtypes = [_P(_Shape), _P(_Cache), _vp, _vp]
_lib.fbk_page_means.restype = ctypes.c_int
_lib.fbk_select_pages_workspace_bytes.argtypes = [_P(_Shape), _P(_Cache)]
_lib.fbk_select_pages_workspace_bytes.restype = ctypes.c_size_t
_lib.fbk_select_pages.argtypes = [_P(_Shape), _vp, _P(_Cache), _vp, ctypes.c_int32, _vp, _vp, _vp, ctypes.c_size_t, _vp]
_lib.fbk_select_pages.restype = ctypes.c_int
_lib.fbk_residual_capture.argtypes = [_P(_Shape), _P(_Partial), _P(_Partial), _vp, _vp, _vp]
_lib.fbk_residual_capture.restype = ctypes.c_int
_lib.fbk_residual_apply.argtypes = [_P(_Shape), _P(_Partial), _vp, _vp, _P(_Partial), _vp]
_lib.fbk_residual_apply.restype = ctypes.c_int
_lib.fbk_status_string.argtypes = [ctypes.c_int]
_lib.fbk_status_string.restype = ctypes.c_char_p


class FbkError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


def status_string(status: int) -> str:
    return _lib.fbk_status_string(int(status)).decode()


@dataclass
class Shape:
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    block_len: int
    softmax_scale: float = 1.0
    rope_base: float = 1e4
    mode: int = BF16

    def c(self) -> _Shape:
        return _Shape(self.batch, self.n_q_heads, self.n_kv_heads, self.head_dim, self.block_len,
                      self.softmax_scale, self.rope_base, self.mode)


@dataclass
class KVCache:
    """Contiguous: k, v [b, Hkv, cap, d] bf16. Paged: k, v [P, Hkv, page, d] bf16 plus
    page_table int32 [b, max_pages]. prefix_lens int32 [b] on the device."""
    k: torch.Tensor
    v: torch.Tensor
    prefix_lens: torch.Tensor
    page_table: torch.Tensor | None = None
    error_flags: torch.Tensor | None = None

    @property
    def paged(self) -> bool:
        return self.page_table is not None

    def c(self) -> _Cache:
        pt = self.page_table
        return _Cache(
            self.k.data_ptr(), self.v.data_ptr(), 1 if pt is not None else 0,
            self.k.shape[2] if pt is not None else 0,
            pt.shape[1] if pt is not None else 0,
            0 if pt is not None else self.k.shape[2],
            self.k.shape[0] if pt is not None else 0,
            pt.data_ptr() if pt is not None else None,
            self.prefix_lens.data_ptr(),
            self.error_flags.data_ptr() if self.error_flags is not None else None)


@dataclass
class Partial:
    o_unnorm: torch.Tensor  # fp32 [b, Hq, B, d]
    m: torch.Tensor         # fp32 [b, Hq, B]
    l: torch.Tensor         # fp32 [b, Hq, B]

    @staticmethod
    def empty(shape: Shape, device="cuda") -> "Partial":
        b, h, B, d = shape.batch, shape.n_q_heads, shape.block_len, shape.head_dim
        return Partial(torch.empty(b, h, B, d, dtype=torch.float32, device=device),
                       torch.empty(b, h, B, dtype=torch.float32, device=device),
                       torch.empty(b, h, B, dtype=torch.float32, device=device))

    def c(self) -> _Partial:
        return _Partial(self.o_unnorm.data_ptr(), self.m.data_ptr(), self.l.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(status, what):
    if status != OK:
        raise FbkError(status, what)


def default_num_splits() -> int:
    return int(_lib.fbk_default_num_splits())


def prefix_workspace_bytes(shape: Shape, cache: KVCache | None, num_splits: int = 0) -> int:
    cs = shape.c()
    cc = cache.c() if cache is not None else None
    return int(_lib.fbk_prefix_workspace_bytes(ctypes.byref(cs), ctypes.byref(cc) if cc else None,
                                               num_splits))


def prefix_partial(shape: Shape, q_blk: torch.Tensor, cache: KVCache, out: Partial,
                   ws: torch.Tensor, num_splits: int = 0, stream=None) -> None:
    cs, cc, po = shape.c(), cache.c(), out.c()
    _check(_lib.fbk_prefix_partial(ctypes.byref(cs), _ptr(q_blk), ctypes.byref(cc), ctypes.byref(po),
                                   _ptr(ws), ws.numel() * ws.element_size(), num_splits,
                                   _stream(stream)), "fbk_prefix_partial")


def prefix_partial_at(shape: Shape, q_blk: torch.Tensor, q_pos: torch.Tensor, cache: KVCache, out: Partial,
                      ws: torch.Tensor, num_splits: int = 0, stream=None) -> None:
    """prefix_partial with the block's rows rotated at q_pos[b] + t (q_pos int32 [b] on the device)."""
    cs, cc, po = shape.c(), cache.c(), out.c()
    _check(_lib.fbk_prefix_partial_at(ctypes.byref(cs), _ptr(q_blk), _ptr(q_pos), ctypes.byref(cc), ctypes.byref(po),
                                      _ptr(ws), ws.numel() * ws.element_size(), num_splits, _stream(stream)),
           "fbk_prefix_partial_at")


def prefix_partial_static_scratch(shape: Shape, q_blk: torch.Tensor, cache: KVCache, out: Partial,
                                  num_splits: int = 0, stream=None) -> None:
    """prefix_partial using the library's built-in per-device scratch array
    (no workspace argument; calls on one device must not overlap)."""
    cs, cc, po = shape.c(), cache.c(), out.c()
    _check(_lib.fbk_prefix_partial_static_scratch(ctypes.byref(cs), _ptr(q_blk), ctypes.byref(cc),
                                                  ctypes.byref(po), num_splits, _stream(stream)),
           "fbk_prefix_partial_static_scratch")


def block_attn_merge(shape: Shape, q_blk, k_blk, v_blk, prefix_lens, prefix: Partial, out,
                     lse=None, stream=None) -> None:
    cs, po = shape.c(), prefix.c()
    _check(_lib.fbk_block_attn_merge(ctypes.byref(cs), _ptr(q_blk), _ptr(k_blk), _ptr(v_blk),
                                     _ptr(prefix_lens), ctypes.byref(po), _ptr(out), _ptr(lse),
                                     _stream(stream)), "fbk_block_attn_merge")


def commit_block_rope_append(shape: Shape, k_blk, v_blk, cache: KVCache, stream=None) -> None:
    cs, cc = shape.c(), cache.c()
    _check(_lib.fbk_commit_block_rope_append(ctypes.byref(cs), _ptr(k_blk), _ptr(v_blk),
                                             ctypes.byref(cc), _stream(stream)),
           "fbk_commit_block_rope_append")


def full_ref_attn(shape: Shape, q_blk, k_blk, v_blk, cache: KVCache, out, lse=None,
                  stream=None) -> None:
    cs, cc = shape.c(), cache.c()
    _check(_lib.fbk_full_ref_attn(ctypes.byref(cs), _ptr(q_blk), _ptr(k_blk), _ptr(v_blk),
                                  ctypes.byref(cc), _ptr(out), _ptr(lse), _stream(stream)),
           "fbk_full_ref_attn")


@dataclass
class LayerBlock:
    """One layer's buffers for decode_block: q [S, b, B, Hq, d], k / v [S, b, B, Hkv, d]
    (bf16, pre-RoPE), out [S, b, B, Hq, d], lse [S, b, Hq, B] or None, and the
    layer's cache, prefix state and cache update interval."""
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    cache: KVCache
    prefix: Partial
    out: torch.Tensor
    refresh_interval: int
    lse: torch.Tensor | None = None

    def c(self) -> _LayerBlock:
        return _LayerBlock(self.q.data_ptr(), self.k.data_ptr(), self.v.data_ptr(), self.cache.c(),
                           self.prefix.c(), self.out.data_ptr(),
                           self.lse.data_ptr() if self.lse is not None else None, self.refresh_interval)


def decode_block(shape: Shape, layers, ws: torch.Tensor, commit: bool = True, num_splits: int = 0,
                 stream=None) -> None:
    """All denoising steps of one block for every layer in `layers` (one C call):
    prefix refresh every refresh_interval steps, a step output per step, then
    (commit=True) the commit of each layer's last-step K/V."""
    steps = {int(L.q.shape[0]) for L in layers}
    if len(steps) != 1:
        raise ValueError(f"layers disagree on the number of steps: {sorted(steps)}")
    arr = (_LayerBlock * len(layers))(*[L.c() for L in layers])
    cs = shape.c()
    _check(_lib.fbk_decode_block(ctypes.byref(cs), arr, len(layers), steps.pop(), 1 if commit else 0,
                                 _ptr(ws), ws.numel() * ws.element_size(), num_splits, _stream(stream)),
           "fbk_decode_block")


@dataclass
class DriftPolicy:
    """fbk_drift_policy: threshold and the device arrays (int32 flags [2, n_layers]
    and last_refresh [n_layers] scratch; fp32 drift and int32 refreshed
    [steps, n_layers] outputs)."""
    threshold: float
    flags: torch.Tensor
    last_refresh: torch.Tensor
    drift: torch.Tensor
    refreshed: torch.Tensor

    @staticmethod
    def empty(threshold: float, n_layers: int, steps: int, device="cuda") -> "DriftPolicy":
        i32 = dict(dtype=torch.int32, device=device)
        return DriftPolicy(threshold, torch.empty(2, n_layers, **i32), torch.empty(n_layers, **i32),
                           torch.empty(steps, n_layers, dtype=torch.float32, device=device),
                           torch.empty(steps, n_layers, **i32))

    def c(self) -> _DriftPolicy:
        return _DriftPolicy(self.threshold, self.flags.data_ptr(), self.last_refresh.data_ptr(),
                            self.drift.data_ptr(), self.refreshed.data_ptr())


def decode_block_adaptive(shape: Shape, layers, policy: DriftPolicy, ws: torch.Tensor, commit: bool = True,
                          num_splits: int = 0, stream=None) -> None:
    """decode_block with the drift-triggered, depth-aware refresh of
    fbk_decode_block_adaptive (the layers' refresh_interval is ignored)."""
    steps = {int(L.q.shape[0]) for L in layers}
    if len(steps) != 1:
        raise ValueError(f"layers disagree on the number of steps: {sorted(steps)}")
    arr = (_LayerBlock * len(layers))(*[L.c() for L in layers])
    cs, cp = shape.c(), policy.c()
    _check(_lib.fbk_decode_block_adaptive(ctypes.byref(cs), arr, len(layers), steps.pop(), 1 if commit else 0,
                                          ctypes.byref(cp), _ptr(ws), ws.numel() * ws.element_size(), num_splits,
                                          _stream(stream)),
           "fbk_decode_block_adaptive")


FP8_GROUP = 128  # FBK_FP8_GROUP


def fp8_group_quant(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, stream=None) -> None:
    """Per-group FP8 (E4M3) quantisation: x bf16 [rows, cols] -> codes uint8
    [rows, cols] and scales fp32 [rows, cols // 128]."""
    if x.dim() != 2:
        raise ValueError("x must be a 2-D [rows, cols] tensor")
    rows, cols = x.shape
    _check(_lib.fbk_fp8_group_quant(_ptr(x), rows, cols, _ptr(codes), _ptr(scales), _stream(stream)),
           "fbk_fp8_group_quant")


def facache_unchanged_rows(shape: Shape, q_u: torch.Tensor, state: Partial, k_blk, v_blk, block_pos, out,
                           lse=None, stream=None) -> None:
    """FACache step of a sequence's unchanged rows: q_u [b, U, Hq, d] after RoPE,
    state [b, Hq, U, d] / [b, Hq, U], block K/V [b, B, Hkv, d] (K before RoPE),
    block_pos int32 [b] -> out [b, U, Hq, d], lse [b, Hq, U]."""
    cs, ps = shape.c(), state.c()
    _check(_lib.fbk_facache_unchanged_rows(ctypes.byref(cs), q_u.shape[1], _ptr(q_u), ctypes.byref(ps),
                                           _ptr(k_blk), _ptr(v_blk), _ptr(block_pos), _ptr(out), _ptr(lse),
                                           _stream(stream)), "fbk_facache_unchanged_rows")


def facache_workspace_bytes(shape: Shape, n_rows: int, num_splits: int = 0) -> int:
    cs = shape.c()
    return int(_lib.fbk_facache_workspace_bytes(ctypes.byref(cs), n_rows, num_splits))


def facache_refresh(shape: Shape, q_u_raw: torch.Tensor, block_pos_host, u_cache: KVCache, state: Partial,
                    ws: torch.Tensor, num_splits: int = 0, stream=None) -> None:
    """FACache's state of U's rows over U's keys: q_u_raw [b, U, Hq, d] before RoPE,
    block_pos_host a host sequence of c0 per sequence, state [b, Hq, U, d] / [b, Hq, U]."""
    pos = (ctypes.c_int32 * shape.batch)(*[int(c) for c in block_pos_host])
    cs, cc, ps = shape.c(), u_cache.c(), state.c()
    _check(_lib.fbk_facache_refresh(ctypes.byref(cs), q_u_raw.shape[1], _ptr(q_u_raw), pos, ctypes.byref(cc),
                                    ctypes.byref(ps), _ptr(ws), ws.numel() * ws.element_size(), num_splits,
                                    _stream(stream)), "fbk_facache_refresh")


def facache_step(shape: Shape, q_u_rot, state: Partial, q_blk, k_blk, v_blk, block_pos, u_cache: KVCache, out_u,
                 out_blk, ws: torch.Tensor, lse_u=None, lse_blk=None, num_splits: int = 0, stream=None) -> None:
    """One denoising step of FACache over a whole sequence: U's rows and the block's rows."""
    cs, cc, ps = shape.c(), u_cache.c(), state.c()
    _check(_lib.fbk_facache_step(ctypes.byref(cs), q_u_rot.shape[1], _ptr(q_u_rot), ctypes.byref(ps), _ptr(q_blk),
                                 _ptr(k_blk), _ptr(v_blk), _ptr(block_pos), ctypes.byref(cc), _ptr(out_u),
                                 _ptr(lse_u), _ptr(out_blk), _ptr(lse_blk), _ptr(ws), ws.numel() * ws.element_size(),
                                 num_splits, _stream(stream)), "fbk_facache_step")


def page_means(shape: Shape, cache: KVCache, means: torch.Tensor, stream=None) -> None:
    cs, cc = shape.c(), cache.c()
    _check(_lib.fbk_page_means(ctypes.byref(cs), ctypes.byref(cc), _ptr(means), _stream(stream)), "fbk_page_means")


def select_pages_workspace_bytes(shape: Shape, cache: KVCache) -> int:
    cs, cc = shape.c(), cache.c()
    return int(_lib.fbk_select_pages_workspace_bytes(ctypes.byref(cs), ctypes.byref(cc)))


def select_pages(shape: Shape, q_blk, cache: KVCache, means, k: int, kept_table, kept_lens, ws, stream=None) -> None:
    cs, cc = shape.c(), cache.c()
    _check(_lib.fbk_select_pages(ctypes.byref(cs), _ptr(q_blk), ctypes.byref(cc), _ptr(means), k, _ptr(kept_table),
                                 _ptr(kept_lens), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "fbk_select_pages")


def residual_capture(shape: Shape, dense: Partial, sparse: Partial, r_o, r_lse, stream=None) -> None:
    cs, pd, ps = shape.c(), dense.c(), sparse.c()
    _check(_lib.fbk_residual_capture(ctypes.byref(cs), ctypes.byref(pd), ctypes.byref(ps), _ptr(r_o), _ptr(r_lse),
                                     _stream(stream)), "fbk_residual_capture")


def residual_apply(shape: Shape, sparse: Partial, r_o, r_lse, ext: Partial, stream=None) -> None:
    cs, ps, pe = shape.c(), sparse.c(), ext.c()
    _check(_lib.fbk_residual_apply(ctypes.byref(cs), ctypes.byref(ps), _ptr(r_o), _ptr(r_lse), ctypes.byref(pe),
                                   _stream(stream)), "fbk_residual_apply")


# raw handles for tests of the C ABI itself
lib = _lib
CShape, CCache, CPartial, CLayerBlock = _Shape, _Cache, _Partial, _LayerBlock
CDriftPolicy = _DriftPolicy
