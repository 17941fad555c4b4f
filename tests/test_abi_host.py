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
    # paged: B = 8 only, a page table that covers cache_len, a workspace for more than 32 queries
    def paged(nq, max_pages, cache_len=4096, pt=dummy):
        return lib.sgqa_sparse_attn_paged(ctypes.byref(p), ctypes.c_int64(1), ctypes.c_int64(4000), ctypes.c_int64(nq),
                                          dummy, dummy, dummy, ctypes.c_int64(300), pt, ctypes.c_int64(max_pages),
                                          ctypes.c_int64(cache_len), dummy, dummy, None, dummy, None,
                                          ctypes.c_size_t(0), st)
    assert paged(33, 256, cache_len=4033) == 3 and b"workspace" in ctypes.string_at(lib.sgqa_last_error())
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


def test_wait_limit_above_the_maximum_is_rejected(bd):
    """Validated on the host before the device variable is touched (no GPU needed)."""
    with pytest.raises(bd.SgqaError) as err:
        bd.sgqa_set_wait_limit_ns(3_000_000_000)
    assert err.value.code == 1


def test_workspace_stays_bounded_at_1m_context(bd):
    """Long rows never materialise FP32 score rows: the index workspace of an
    8192-query chunk at a 1M-token context is the filtered path's lists, the
    sample and the fallback's per-CTA rows, or the score rows of the longest
    chunk that still takes them (16384 candidates), whichever is larger."""
    b8 = bd.sgqa_workspace_size(bd.Params(), 1, 8192, 1 << 20)
    rows_path = 8192 * 4 * 16384 * 4  # score rows of 16384 candidates
    assert rows_path <= b8 < rows_path + (1 << 30), b8
    b1 = bd.sgqa_workspace_size(bd.Params(block_size=1, topk=2048), 1, 8192, 1 << 20)
    assert b1 < 6 * (1 << 30), b1
