"""The C ABI without a GPU: the library loads, exports every symbol include/lf.h declares,
and rejects invalid arguments before touching the device."""
import ctypes
import os
import re

import pytest

import block_sparse_attention_46_b200 as lf
import lf_workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "lf.h")).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(lf_\w+)\s*\(", src, re.M)))


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_46_b200 import build
    build.build()
    return lf.load()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert "lf_forward_chunk" in names and "lf_block_sparse_attn" in names
    raw = ctypes.CDLL(lf.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), n
    assert lf.lf_abi_version() == 2


def _shape(**kw):
    base = dict(H=2, d=64, T=256, block=64, n_cur_frames=1, n_hist=4, n_sink=0, n_slots=4,
                k_f=2, k_b=2, scale=0.125)
    base.update(kw)
    return W.Shape(**base)


FAKE = ctypes.c_void_p(1 << 20)       # never dereferenced: validation fails first


def _attn(lib, shape, hist=(0, 1, 2, 3), sinks=(), ws=1 << 20, wsptr=FAKE, bidx=FAKE,
          cidx=FAKE):
    sh = lf.make_shape(shape)
    h = (ctypes.c_int32 * max(len(hist), 1))(*hist)
    s = (ctypes.c_int32 * max(len(sinks), 1))(*sinks)
    return lib.lf_block_sparse_attn(ctypes.byref(sh), FAKE, FAKE, FAKE, FAKE, FAKE,
                                     ctypes.cast(h, ctypes.POINTER(ctypes.c_int32)),
                                     ctypes.cast(s, ctypes.POINTER(ctypes.c_int32)), bidx, cidx,
                                     FAKE, None, wsptr, ws, None)


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), 2), (dict(d=256), 2), (dict(block=32), 2), (dict(H=0), 1),
    (dict(n_cur_frames=0), 1), (dict(T=0), 1), (dict(T=20000), 2), (dict(n_hist=-1), 1),
    (dict(k_f=0), 1), (dict(k_b=0), 1), (dict(scale=0.0), 1), (dict(scale=float("nan")), 1),
    (dict(n_hist=300, n_slots=300), 2),
    # one past each size limit of the header
    (dict(T=16385), 2),                                                    # LF_MAX_T
    (dict(n_hist=250, n_sink=7, n_slots=257, k_f=1), 2),                   # LF_MAX_FRAMES
    (dict(T=1600, n_hist=41, n_slots=41, k_f=41, k_b=25), 2),              # LF_MAX_SELECTED
    (dict(T=1600, n_hist=40, n_sink=4, n_slots=44, k_f=40, k_b=25), 2),    # LF_MAX_PLAN
])
def test_shape_validation(lib, kw, code):
    assert _attn(lib, _shape(**kw), hist=tuple(range(min(kw.get("n_hist", 4), 256)))
                 if kw.get("n_hist", 4) > 0 else ()) == code


def test_slot_and_workspace_validation(lib):
    assert _attn(lib, _shape(), hist=(0, 1, 2, 4)) == 1                # slot >= n_slots
    assert _attn(lib, _shape(), hist=(0, 1, -1, 2)) == 1
    assert _attn(lib, _shape(n_sink=1, n_slots=5), hist=(0, 1, 2, 3), sinks=(9,)) == 1
    assert _attn(lib, _shape(), ws=16) == 5                            # workspace too small
    assert _attn(lib, _shape(), wsptr=None) == 5
    assert _attn(lib, _shape(), bidx=None) == 1                        # needs block_idx


def test_misaligned_pointer_rejected(lib):
    sh = lf.make_shape(_shape())
    h = (ctypes.c_int32 * 4)(0, 1, 2, 3)
    odd = ctypes.c_void_p((1 << 20) + 2)
    rc = lib.lf_compress(ctypes.byref(sh), odd, FAKE, ctypes.cast(h, ctypes.POINTER(ctypes.c_int32)),
                         FAKE, FAKE, FAKE, None)
    assert rc == 1


def test_workspace_sizes(lib):
    s480 = W.p480_shape()
    attn = lf.lf_attn_workspace_size(s480)
    fwd = lf.lf_forward_workspace_size(s480)
    # 38 tiles x 12 heads x (2 x 72) plan entries + counts, and the pooled tensors
    assert attn >= 38 * 12 * 144 * 4
    assert fwd >= attn + 12 * 18 * 25 * 128 * 4
    assert lf.lf_attn_workspace_size(_shape(d=96)) == 0


def test_status_strings(lib):
    assert lf.lf_status_string(0) == "ok"
    assert "timed out" in lf.lf_status_string(4)


def _i32(vals):
    arr = (ctypes.c_int32 * max(len(vals), 1))(*vals)
    return ctypes.cast(arr, ctypes.POINTER(ctypes.c_int32)), arr


def test_pooled_cache_validation(lib):
    sh = lf.make_shape(_shape())
    slots, _k = _i32([0, 3])
    bad, _k2 = _i32([0, 4])                                             # slot >= n_slots
    assert lib.lf_pool_frames(ctypes.byref(sh), FAKE, slots, 0, FAKE, None) == 0   # nothing
    assert lib.lf_pool_frames(ctypes.byref(sh), FAKE, bad, 2, FAKE, None) == 1
    assert lib.lf_pool_frames(ctypes.byref(sh), FAKE, slots, -1, FAKE, None) == 1
    assert lib.lf_pool_frames(ctypes.byref(sh), FAKE, slots, 257, FAKE, None) == 1
    assert lib.lf_pool_frames(ctypes.byref(sh), None, slots, 2, FAKE, None) == 1
    assert lib.lf_pool_frames(ctypes.byref(sh), FAKE, slots, 2, ctypes.c_void_p((1 << 20) + 4),
                              None) == 1                                # misaligned cache
    hist, _k3 = _i32([0, 1, 2, 3])
    assert lib.lf_select_chunk_cached(ctypes.byref(sh), FAKE, FAKE, hist, FAKE, None, 0,
                                      None) == 5                        # no workspace
    assert lib.lf_select_chunk_cached(ctypes.byref(sh), FAKE, None, hist, FAKE, FAKE, 1 << 30,
                                      None) == 1                        # no pooled cache
    nh = lf.make_shape(_shape(n_hist=0, n_slots=0))
    assert lib.lf_select_chunk_cached(ctypes.byref(nh), FAKE, FAKE, hist, FAKE, FAKE, 1 << 30,
                                      None) == 1                        # needs history
    # the cache holds one fp32 row of d channels per (slot, head, block)
    s480 = W.p480_shape()
    assert lf.lf_pooled_cache_bytes(s480) == s480.n_slots * 12 * 25 * 128 * 4


def test_select_1d_block_limit(lib):
    # 40 history frames x 64 blocks = 2560 candidate blocks: beyond the 1-D selector
    sh = lf.make_shape(_shape(H=1, T=4096, n_hist=40, n_slots=40))
    hist, _k = _i32(list(range(40)))
    assert lib.lf_select_chunk_1d(ctypes.byref(sh), FAKE, FAKE, hist, FAKE, FAKE, 1 << 40,
                                  None) == 2
    small = lf.make_shape(_shape())
    h4, _k2 = _i32([0, 1, 2, 3])
    assert lib.lf_select_chunk_1d(ctypes.byref(small), FAKE, FAKE, h4, FAKE, None, 0,
                                  None) == 5


def test_debug_configure_validates_and_restores(lib):
    assert lib.lf_debug_configure(30_000_000_000, 0, 1) == 1          # above 20 s
    assert lib.lf_debug_configure(20_000_000, 0, 0) == 0
    assert lib.lf_debug_configure(0, 0, 1) == 0                       # defaults


def test_sparse_current_chunk_validation(lib):
    assert _attn(lib, _shape(k_c=-1)) == 1                             # negative k_c
    assert _attn(lib, _shape(k_c=2), cidx=None) == 1                   # needs cur_idx
    assert _attn(lib, _shape(k_c=2), ws=16) == 5                       # lists fine, ws small
    # n_qb = 3 * ceil(16384 / 64) = 768 current blocks: above LF_MAX_CUR_BLOCKS
    assert _attn(lib, _shape(T=16384, n_cur_frames=3, n_hist=0, n_slots=0, k_c=4),
                 hist=()) == 2
    # the fixed-scratch variant takes no current-chunk list
    sh = lf.make_shape(_shape(k_c=2))
    h = (ctypes.c_int32 * 4)(0, 1, 2, 3)
    rc = lib.lf_block_sparse_attn_noalloc(ctypes.byref(sh), FAKE, FAKE, FAKE, FAKE, FAKE,
                                          ctypes.cast(h, ctypes.POINTER(ctypes.c_int32)), None,
                                          FAKE, FAKE, None, None)
    assert rc == 1
    # lf_select_current needs k_c >= 1
    rc = lib.lf_select_current(ctypes.byref(lf.make_shape(_shape())), FAKE, FAKE, FAKE, FAKE,
                               1 << 20, None)
    assert rc == 1


def test_e4m3_entry_points_validate(lib):
    sh = lf.make_shape(_shape(d=64))
    h = (ctypes.c_int32 * 4)(0, 1, 2, 3)
    hp = ctypes.cast(h, ctypes.POINTER(ctypes.c_int32))
    rc = lib.lf_block_sparse_attn_e4m3(ctypes.byref(sh), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                       hp, None, FAKE, None, FAKE, None, FAKE, 1 << 20, None)
    assert rc == 2                                                    # d = 64: unsupported
    sh = lf.make_shape(_shape(d=128))
    rc = lib.lf_block_sparse_attn_e4m3(ctypes.byref(sh), FAKE, None, FAKE, FAKE, FAKE, FAKE, FAKE,
                                       hp, None, FAKE, None, FAKE, None, FAKE, 1 << 20, None)
    assert rc == 1                                                    # no query scales
    assert lib.lf_quantize_e4m3(FAKE, 10, 2, 96, None, FAKE, FAKE, None) == 1     # d = 96
    assert lib.lf_quantize_e4m3(FAKE, 10, 2, 64, None, FAKE, None, None) == 1     # no row_scale
    assert lib.lf_quantize_e4m3(FAKE, 0, 2, 64, None, FAKE, FAKE, None) == 0      # nothing to do
    assert lib.lf_e4m3_head_scales(None, None, 0, 2, 64, FAKE, None) == 1
