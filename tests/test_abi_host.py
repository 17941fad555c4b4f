"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
symbol ``include/sgqa.h`` declares, sizes workspaces, and rejects bad arguments
before enqueuing anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sgqa.h")


@pytest.fixture(scope="module")
def lib():
    from sparse_long_context_sgqa_b200 import build
    path = build.build_library()
    return ctypes.CDLL(path)


@pytest.fixture(scope="module")
def bd(lib):
    from sparse_long_context_sgqa_b200 import binding
    return binding


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"\b(sgqa_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_four_calls():
    syms = declared_symbols()
    for s in ("sgqa_merge_blocks", "sgqa_index_topk", "sgqa_sparse_attn", "sgqa_forward"):
        assert s in syms


def test_library_exports_every_declared_symbol(lib):
    for s in declared_symbols():
        assert hasattr(lib, s), s


def test_version_and_no_error(bd):
    assert "sm_100a" in bd.version()


def _p(bd, **kw):
    return bd.Params(**kw).c()


def test_workspace_size(bd):
    p = bd.Params()
    small = bd.sgqa_workspace_size(p, 1, 8192, 8192)
    big = bd.sgqa_workspace_size(p, 1, 8192, 131072)
    assert 0 < small < big
    # index scores dominate: nq * G * ceil64((ctx-1)/B) * 4 bytes
    assert big >= 8192 * 4 * 16384 * 4
    dec = bd.sgqa_workspace_size(p, 16, 1, 262144)
    assert dec > 0


@pytest.mark.parametrize("field,value,code", [("head_dim", 128, 2), ("idx_heads", 3, 2), ("block_size", 16, 2),
                                               ("topk", 4096, 2), ("topk", 0, 1), ("merge_in_f32", 2, 1)])
def test_bad_params_rejected(bd, field, value, code):
    kw = {field: value}
    with pytest.raises(bd.SgqaError) as e:
        bd.sgqa_workspace_size(bd.Params(**kw), 1, 16, 16)
    assert e.value.code == code


def test_null_and_range_checks_before_any_launch(lib, bd):
    p = _p(bd)
    st = ctypes.c_void_p(0)
    # NULL inputs
    rc = lib.sgqa_merge_blocks(ctypes.byref(p), ctypes.c_int64(1), ctypes.c_int64(64), None, None,
                               ctypes.c_int64(0), ctypes.c_int64(8), None, None, st)
    assert rc == 1
    assert b"NULL" in ctypes.string_at(lib.sgqa_last_error())
    # incomplete block range
    dummy = ctypes.c_void_p(4096)
    rc = lib.sgqa_merge_blocks(ctypes.byref(p), ctypes.c_int64(1), ctypes.c_int64(60), dummy, dummy,
                               ctypes.c_int64(0), ctypes.c_int64(8), None, dummy, st)
    assert rc == 1
    # cache smaller than the queries
    rc = lib.sgqa_sparse_attn(ctypes.byref(p), ctypes.c_int64(1), ctypes.c_int64(100), ctypes.c_int64(50),
                              dummy, ctypes.c_int64(120), ctypes.c_int64(120), dummy, dummy, dummy, dummy,
                              dummy, dummy, ctypes.c_size_t(1 << 30), st)
    assert rc == 1
    # workspace too small / misaligned
    rc = lib.sgqa_index_topk(ctypes.byref(p), ctypes.c_int64(1), ctypes.c_int64(0), ctypes.c_int64(64),
                             dummy, dummy, ctypes.c_int64(64), dummy, dummy, dummy, dummy,
                             ctypes.c_size_t(16), st)
    assert rc == 3
    rc = lib.sgqa_index_topk(ctypes.byref(p), ctypes.c_int64(1), ctypes.c_int64(0), ctypes.c_int64(64),
                             dummy, dummy, ctypes.c_int64(64), dummy, dummy, dummy, ctypes.c_void_p(4096 + 16),
                             ctypes.c_size_t(1 << 30), st)
    assert rc == 3
    # a misaligned gate is refused before any launch (gated attention and forward)
    odd = ctypes.c_void_p(4096 + 1)
    rc = lib.sgqa_sparse_attn_gated(ctypes.byref(p), ctypes.c_int64(1), ctypes.c_int64(0), ctypes.c_int64(64),
                                    dummy, ctypes.c_int64(64), ctypes.c_int64(64), dummy, dummy, dummy, dummy, odd,
                                    dummy, dummy, ctypes.c_size_t(1 << 30), st)
    assert rc == 1
    assert b"gate" in ctypes.string_at(lib.sgqa_last_error())
    rc = lib.sgqa_forward_gated(ctypes.byref(p), ctypes.c_int64(1), ctypes.c_int64(0), ctypes.c_int64(64), dummy,
                                dummy, dummy, ctypes.c_int64(64), ctypes.c_int64(64), dummy, dummy, dummy, dummy, None,
                                dummy, dummy, dummy, odd, dummy, dummy, ctypes.c_size_t(1 << 30), st)
    assert rc == 1
    assert b"gate" in ctypes.string_at(lib.sgqa_last_error())
    # paged decode: decode-sized calls with B = 8 only, a page table that covers cache_len
    def paged(nq, max_pages, cache_len=4096, pt=dummy):
        return lib.sgqa_sparse_attn_paged(ctypes.byref(p), ctypes.c_int64(1), ctypes.c_int64(4000), ctypes.c_int64(nq),
                                          dummy, dummy, dummy, ctypes.c_int64(300), pt, ctypes.c_int64(max_pages),
                                          ctypes.c_int64(cache_len), dummy, dummy, None, dummy, st)
    assert paged(33, 256) == 2
    assert paged(4, 255) == 1 and b"max_pages" in ctypes.string_at(lib.sgqa_last_error())
    assert paged(4, 256, pt=ctypes.c_void_p(4096 + 2)) == 1
    p.block_size = 4
    assert paged(4, 256) == 2
    p.block_size = 8
    # nothing to do is not an error
    rc = lib.sgqa_forward(ctypes.byref(p), ctypes.c_int64(1), ctypes.c_int64(0), ctypes.c_int64(0), None, None,
                          None, ctypes.c_int64(0), ctypes.c_int64(0), None, None, None, None, None, None, None,
                          None, None, None, ctypes.c_size_t(0), st)
    assert rc == 0
