"""Python binding of liblf, the sm_100a hierarchical sparse attention library.

Argument marshalling only: every function below forwards to the C entry point of the
same name in ``liblf.so`` (declared in include/lf.h) with raw device pointers, host
slot lists and the current CUDA stream.  PyTorch provides device memory and streams; no
step of the attention path runs in Python or on the CPU.  If the library is missing or
does not load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

__all__ = [
    "LfError", "LfShape", "load", "make_shape", "lf_compress", "lf_select_frames",
    "lf_select_blocks", "lf_block_sparse_attn", "lf_forward_chunk",
    "lf_attn_workspace_size", "lf_forward_workspace_size", "lf_device_status",
    "lf_select_chunk", "lf_select_workspace_size", "lf_block_sparse_attn_noalloc",
    "lf_noalloc_scratch_bytes", "lf_pooled_cache_bytes", "lf_pool_frames",
    "lf_select_chunk_cached", "lf_cag_schedule", "lf_select_chunk_1d",
    "lf_status_string", "lf_abi_version", "lf_debug_configure", "lf_select_current",
    "lf_quantize_e4m3", "lf_e4m3_head_scales", "lf_block_sparse_attn_e4m3",
    "derived", "current_blocks", "LIB_PATH",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblf.so")

LF_OK = 0


class LfError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: liblf status {code} ({lf_status_string(code)})")


class LfShape(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int32), ("d", ctypes.c_int32),
                ("tokens_per_frame", ctypes.c_int32), ("block", ctypes.c_int32),
                ("n_cur_frames", ctypes.c_int32), ("n_hist", ctypes.c_int32),
                ("n_sink", ctypes.c_int32), ("n_slots", ctypes.c_int32),
                ("k_f", ctypes.c_int32), ("k_b", ctypes.c_int32), ("scale", ctypes.c_float),
                ("k_c", ctypes.c_int32)]


_lib: Optional[ctypes.CDLL] = None
_P = ctypes.c_void_p
_SZ = ctypes.c_size_t
_I32P = ctypes.POINTER(ctypes.c_int32)
_SHP = ctypes.POINTER(LfShape)

_SIGS = {
    "lf_compress": (ctypes.c_int, [_SHP, _P, _P, _I32P, _P, _P, _P, _P]),
    "lf_select_frames": (ctypes.c_int, [_SHP, _P, _P, _P, _P, _P]),
    "lf_select_blocks": (ctypes.c_int, [_SHP, _P, _P, _P, _P, _P, _P]),
    "lf_attn_workspace_size": (_SZ, [_SHP]),
    "lf_block_sparse_attn": (ctypes.c_int, [_SHP, _P, _P, _P, _P, _P, _I32P, _I32P, _P, _P,
                                            _P, _P, _P, _SZ, _P]),
    "lf_select_current": (ctypes.c_int, [_SHP, _P, _P, _P, _P, _SZ, _P]),
    "lf_forward_workspace_size": (_SZ, [_SHP]),
    "lf_select_workspace_size": (_SZ, [_SHP]),
    "lf_select_chunk": (ctypes.c_int, [_SHP, _P, _P, _I32P, _P, _P, _SZ, _P]),
    "lf_forward_chunk": (ctypes.c_int, [_SHP, _P, _P, _P, _P, _P, _I32P, _I32P, _P, _SZ, _P,
                                        _P, _P, _P, _P]),
    "lf_device_status": (ctypes.c_int, [ctypes.c_int]),
    "lf_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "lf_abi_version": (ctypes.c_int, []),
    "lf_noalloc_scratch_bytes": (_SZ, []),
    "lf_debug_configure": (ctypes.c_int, [ctypes.c_uint64, ctypes.c_int, ctypes.c_int]),
    "lf_block_sparse_attn_e4m3": (ctypes.c_int, [_SHP, _P, _P, _P, _P, _P, _P, _P, _I32P, _I32P,
                                                 _P, _P, _P, _P, _P, _SZ, _P]),
    "lf_quantize_e4m3": (ctypes.c_int, [_P, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _P,
                                        _P, _P, _P]),
    "lf_e4m3_head_scales": (ctypes.c_int, [ctypes.POINTER(ctypes.c_void_p),
                                           ctypes.POINTER(ctypes.c_int64), ctypes.c_int32,
                                           ctypes.c_int32, ctypes.c_int32, _P, _P]),
    "lf_pooled_cache_bytes": (_SZ, [_SHP]),
    "lf_cag_schedule": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, ctypes.c_float,
                                       ctypes.c_float, _I32P, ctypes.c_int32, ctypes.c_int32,
                                       ctypes.POINTER(ctypes.c_float), _I32P, _I32P]),
    "lf_pool_frames": (ctypes.c_int, [_SHP, _P, _I32P, ctypes.c_int32, _P, _P]),
    "lf_select_chunk_cached": (ctypes.c_int, [_SHP, _P, _P, _I32P, _P, _P, _SZ, _P]),
    "lf_select_chunk_1d": (ctypes.c_int, [_SHP, _P, _P, _I32P, _P, _P, _SZ, _P]),
    "lf_block_sparse_attn_noalloc": (ctypes.c_int, [_SHP, _P, _P, _P, _P, _P, _I32P, _I32P, _P,
                                                    _P, _P, _P]),
}


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads liblf.so (once) and declares its signatures.  Raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise FileNotFoundError(
                f"{path} is missing: build it with python -m block_sparse_attention_46_b200.build")
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype, fn.argtypes = res, args
        _lib = lib
    return _lib


def make_shape(s) -> LfShape:
    """lf_shape from any object with the plain size fields (H, d, T, block, ...)."""
    return LfShape(s.H, s.d, s.T, s.block, s.n_cur_frames, s.n_hist, s.n_sink, s.n_slots,
                   s.k_f, s.k_b, s.scale, getattr(s, "k_c", 0))


def derived(s):
    """(n_bpf, n_qb, kf, kb) as the library derives them (for sizing output tensors)."""
    nbpf = -(-s.T // s.block)
    kf = min(s.k_f, s.n_hist) if s.n_hist > 0 else 0
    kb = min(s.k_b, nbpf) if s.n_hist > 0 else 0
    return nbpf, s.n_cur_frames * nbpf, kf, kb


def current_blocks(s) -> int:
    """kc, the current-chunk blocks kept per query block (0: the dense current chunk)."""
    nqb = s.n_cur_frames * -(-s.T // s.block)
    k_c = getattr(s, "k_c", 0)
    return min(k_c, nqb) if k_c > 0 else 0


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor arguments must be CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("tensor arguments must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _slots(v: Sequence[int]):
    arr = (ctypes.c_int32 * max(len(v), 1))(*[int(x) for x in v])
    return ctypes.cast(arr, _I32P), arr          # keep `arr` alive during the call


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(rc: int, where: str):
    if rc != LF_OK:
        raise LfError(rc, where)


def lf_status_string(code: int) -> str:
    return load().lf_status_string(code).decode()


def lf_abi_version() -> int:
    return load().lf_abi_version()


def lf_device_status(reset: bool = True) -> int:
    return load().lf_device_status(1 if reset else 0)


def lf_debug_configure(wait_limit_ns: int = 0, stall: bool = False, tail_split: bool = True):
    """Test hook: wait limit of the device waits, a stalled first CTA, and whether the last
    partial wave of query tiles may be split (defaults restored by calling it with none)."""
    _check(load().lf_debug_configure(int(wait_limit_ns), 1 if stall else 0,
                                     1 if tail_split else 0), "lf_debug_configure")


def lf_compress(shape, q, k_cache, hist_slots, q_blk, k_blk, k_frm, stream=None):
    sh = make_shape(shape)
    hs, _keep = _slots(hist_slots)
    _check(load().lf_compress(ctypes.byref(sh), _ptr(q), _ptr(k_cache), hs, _ptr(q_blk),
                              _ptr(k_blk), _ptr(k_frm), _stream(stream)), "lf_compress")


def lf_select_frames(shape, q_blk, k_frm, frame_idx, frame_score=None, stream=None):
    sh = make_shape(shape)
    _check(load().lf_select_frames(ctypes.byref(sh), _ptr(q_blk), _ptr(k_frm), _ptr(frame_idx),
                                   _ptr(frame_score), _stream(stream)), "lf_select_frames")


def lf_select_blocks(shape, q_blk, k_blk, frame_idx, block_idx, block_score=None, stream=None):
    sh = make_shape(shape)
    _check(load().lf_select_blocks(ctypes.byref(sh), _ptr(q_blk), _ptr(k_blk), _ptr(frame_idx),
                                   _ptr(block_idx), _ptr(block_score), _stream(stream)),
           "lf_select_blocks")


def lf_select_workspace_size(shape) -> int:
    sh = make_shape(shape)
    return int(load().lf_select_workspace_size(ctypes.byref(sh)))


def lf_select_chunk(shape, q, k_cache, hist_slots, block_idx, workspace=None, stream=None):
    sh = make_shape(shape)
    hs, _keep = _slots(hist_slots)
    if workspace is None:
        workspace = torch.empty(max(lf_select_workspace_size(shape), 256), dtype=torch.uint8,
                                device=q.device)
    _check(load().lf_select_chunk(ctypes.byref(sh), _ptr(q), _ptr(k_cache), hs, _ptr(block_idx),
                                  _ptr(workspace), workspace.numel(), _stream(stream)),
           "lf_select_chunk")


def lf_select_chunk_1d(shape, q, k_cache, hist_slots, block_idx, workspace=None, stream=None):
    """One-dimensional selection (no frame stage): the kf*kb best blocks over all frames."""
    sh = make_shape(shape)
    hs, _keep = _slots(hist_slots)
    if workspace is None:
        workspace = torch.empty(max(lf_select_workspace_size(shape), 256), dtype=torch.uint8,
                                device=q.device)
    _check(load().lf_select_chunk_1d(ctypes.byref(sh), _ptr(q), _ptr(k_cache), hs,
                                     _ptr(block_idx), _ptr(workspace), workspace.numel(),
                                     _stream(stream)), "lf_select_chunk_1d")


def lf_select_current(shape, q, k_cur, cur_idx, workspace=None, stream=None):
    """Current-chunk block choice (shape.k_c >= 1): each query block's own block plus the
    k_c - 1 best-scoring other current blocks, into cur_idx [H, n_qb, kc]."""
    sh = make_shape(shape)
    if workspace is None:
        workspace = torch.empty(max(lf_forward_workspace_size(shape), 256), dtype=torch.uint8,
                                device=q.device)
    _check(load().lf_select_current(ctypes.byref(sh), _ptr(q), _ptr(k_cur), _ptr(cur_idx),
                                    _ptr(workspace), workspace.numel(), _stream(stream)),
           "lf_select_current")


def lf_pooled_cache_bytes(shape) -> int:
    sh = make_shape(shape)
    return int(load().lf_pooled_cache_bytes(ctypes.byref(sh)))


def lf_pool_frames(shape, k_cache, slots, k_pool, stream=None):
    """Block means of the keys of cache slots `slots` into the pooled-key cache k_pool
    (fp32 [n_slots, H, n_bpf, d])."""
    sh = make_shape(shape)
    sl, _keep = _slots(slots)
    _check(load().lf_pool_frames(ctypes.byref(sh), _ptr(k_cache), sl, len(slots), _ptr(k_pool),
                                 _stream(stream)), "lf_pool_frames")


def lf_select_chunk_cached(shape, q, k_pool, hist_slots, block_idx, workspace=None, stream=None):
    sh = make_shape(shape)
    hs, _keep = _slots(hist_slots)
    if workspace is None:
        workspace = torch.empty(max(lf_select_workspace_size(shape), 256), dtype=torch.uint8,
                                device=q.device)
    _check(load().lf_select_chunk_cached(ctypes.byref(sh), _ptr(q), _ptr(k_pool), hs,
                                         _ptr(block_idx), _ptr(workspace), workspace.numel(),
                                         _stream(stream)), "lf_select_chunk_cached")


def lf_cag_schedule(n_chunks, first, mean_sparsity, final_sparsity, n_hist=None, n_bpf=1,
                    kf_max=1):
    """Per-chunk keep ratios of the chunk-aware sparsity growth, and (if n_hist is given)
    the (k_f, k_b) budgets.  Host only.  Returns (keep, k_f, k_b); the last two are None
    without n_hist."""
    keep = (ctypes.c_float * n_chunks)()
    if n_hist is not None:
        nh = (ctypes.c_int32 * n_chunks)(*[int(x) for x in n_hist])
        kf = (ctypes.c_int32 * n_chunks)()
        kb = (ctypes.c_int32 * n_chunks)()
        args = (ctypes.cast(nh, _I32P), n_bpf, kf_max, keep, ctypes.cast(kf, _I32P),
                ctypes.cast(kb, _I32P))
    else:
        args = (None, n_bpf, kf_max, keep, None, None)
    _check(load().lf_cag_schedule(n_chunks, first, mean_sparsity, final_sparsity, *args),
           "lf_cag_schedule")
    if n_hist is None:
        return list(keep), None, None
    return list(keep), list(kf), list(kb)


def lf_attn_workspace_size(shape) -> int:
    sh = make_shape(shape)
    return int(load().lf_attn_workspace_size(ctypes.byref(sh)))


def lf_forward_workspace_size(shape) -> int:
    sh = make_shape(shape)
    return int(load().lf_forward_workspace_size(ctypes.byref(sh)))


def lf_block_sparse_attn(shape, q, k_cur, v_cur, k_cache, v_cache, hist_slots, sink_slots,
                         block_idx, out, lse=None, workspace=None, stream=None, cur_idx=None):
    sh = make_shape(shape)
    hs, _k1 = _slots(hist_slots)
    ss, _k2 = _slots(sink_slots)
    if workspace is None:
        workspace = torch.empty(max(lf_attn_workspace_size(shape), 256), dtype=torch.uint8,
                                device=q.device)
    _check(load().lf_block_sparse_attn(
        ctypes.byref(sh), _ptr(q), _ptr(k_cur), _ptr(v_cur), _ptr(k_cache), _ptr(v_cache), hs, ss,
        _ptr(block_idx), _ptr(cur_idx), _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
        _stream(stream)), "lf_block_sparse_attn")


def lf_quantize_e4m3(x, x8, head_scale=None, row_scale=None, stream=None):
    """e4m3 codes of x [rows, H, d] bf16 into x8 (uint8, same shape): per head with the given
    scales [H], or per (row, head) with the scales written to row_scale [rows, H]."""
    rows, H, d = x.shape
    _check(load().lf_quantize_e4m3(_ptr(x), rows, H, d, _ptr(head_scale), _ptr(x8),
                                   _ptr(row_scale), _stream(stream)), "lf_quantize_e4m3")


def lf_e4m3_head_scales(xs, head_scale, stream=None):
    """Per-head power-of-two scales over the bf16 tensors xs (each [rows, H, d])."""
    n = len(xs)
    H, d = xs[0].shape[-2], xs[0].shape[-1]
    ptrs = (ctypes.c_void_p * n)(*[x.data_ptr() for x in xs])
    rows = (ctypes.c_int64 * n)(*[x.numel() // (H * d) for x in xs])
    for x in xs:
        _ptr(x)
    _check(load().lf_e4m3_head_scales(ptrs, rows, n, H, d, _ptr(head_scale), _stream(stream)),
           "lf_e4m3_head_scales")


def lf_block_sparse_attn_e4m3(shape, q8, q_scale, k_cur8, v_cur, k_cache8, v_cache, k_scale,
                              hist_slots, sink_slots, block_idx, out, lse=None, workspace=None,
                              stream=None, cur_idx=None):
    """(d) with e4m3 queries and keys (QK^T on the FP8 tensor cores), bf16 values."""
    sh = make_shape(shape)
    hs, _k1 = _slots(hist_slots)
    ss, _k2 = _slots(sink_slots)
    if workspace is None:
        workspace = torch.empty(max(lf_attn_workspace_size(shape), 256), dtype=torch.uint8,
                                device=q8.device)
    _check(load().lf_block_sparse_attn_e4m3(
        ctypes.byref(sh), _ptr(q8), _ptr(q_scale), _ptr(k_cur8), _ptr(v_cur), _ptr(k_cache8),
        _ptr(v_cache), _ptr(k_scale), hs, ss, _ptr(block_idx), _ptr(cur_idx), _ptr(out),
        _ptr(lse), _ptr(workspace), workspace.numel(), _stream(stream)),
        "lf_block_sparse_attn_e4m3")


def lf_noalloc_scratch_bytes() -> int:
    return int(load().lf_noalloc_scratch_bytes())


def lf_block_sparse_attn_noalloc(shape, q, k_cur, v_cur, k_cache, v_cache, hist_slots,
                                 sink_slots, block_idx, out, lse=None, stream=None):
    """lf_block_sparse_attn without a workspace argument, for callers that cannot
    allocate device memory: the library's fixed scratch array is used instead (calls
    that overlap on the GPU must not share a device)."""
    sh = make_shape(shape)
    hs, _k1 = _slots(hist_slots)
    ss, _k2 = _slots(sink_slots)
    _check(load().lf_block_sparse_attn_noalloc(
        ctypes.byref(sh), _ptr(q), _ptr(k_cur), _ptr(v_cur), _ptr(k_cache), _ptr(v_cache), hs, ss,
        _ptr(block_idx), _ptr(out), _ptr(lse), _stream(stream)), "lf_block_sparse_attn_noalloc")


def lf_forward_chunk(shape, q, k_cur, v_cur, k_cache, v_cache, hist_slots, sink_slots,
                     out, lse=None, block_idx_out=None, workspace=None, stream=None,
                     cur_idx_out=None):
    sh = make_shape(shape)
    hs, _k1 = _slots(hist_slots)
    ss, _k2 = _slots(sink_slots)
    if workspace is None:
        workspace = torch.empty(max(lf_forward_workspace_size(shape), 256), dtype=torch.uint8,
                                device=q.device)
    _check(load().lf_forward_chunk(
        ctypes.byref(sh), _ptr(q), _ptr(k_cur), _ptr(v_cur), _ptr(k_cache), _ptr(v_cache), hs, ss,
        _ptr(workspace), workspace.numel(), _ptr(out), _ptr(lse), _ptr(block_idx_out),
        _ptr(cur_idx_out), _stream(stream)), "lf_forward_chunk")
