"""The C-ABI library loads and exports every entry point its header declares,
and its host-side checks reject bad arguments before touching a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "s5attn.h")


@pytest.fixture(scope="module")
def s5():
    from block_sparse_gqa_indexer_b200 import build
    build.build()
    from block_sparse_gqa_indexer_b200 import s5 as mod
    return mod


def _declared():
    text = open(HEADER).read()
    return set(re.findall(r"^\s*(?:s5_status|const char \*|int32_t)\s*(s5_\w+)\s*\(", text, re.M))


def test_header_declarations_match_binding(s5):
    assert _declared() == set(s5.SYMBOLS)


def test_every_declared_symbol_is_exported(s5):
    lib = ctypes.CDLL(s5.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name


def test_status_strings_and_version(s5):
    assert s5.s5_abi_version() == s5.ABI_VERSION
    m = re.search(r"#define S5_ABI_VERSION (\d+)", open(HEADER).read())
    assert m and int(m.group(1)) == s5.ABI_VERSION
    for code in range(7):
        assert s5.s5_status_string(code).startswith("S5_")
    assert s5.s5_status_string(99) == "S5_ERR_UNKNOWN"


def _batch(**kw):
    fake = 0x1000
    d = dict(page_table=fake, ctx_lens=fake, cu_q=fake, batch=2, max_pages=4, total_q=2, max_q=1, max_len=200)
    d.update(kw)
    from block_sparse_gqa_indexer_b200 import s5
    return s5.BatchDesc(**d)


def test_workspace_size_is_host_only(s5):
    n = ctypes.c_size_t(0)
    b = _batch()
    assert s5._lib.s5_workspace_size(ctypes.byref(b), 512, ctypes.byref(n)) == 0
    assert n.value >= 256
    # the headline batch: 64 rows, 131,073 tokens each
    b = _batch(batch=64, total_q=64, max_pages=2049, max_len=131073)
    assert s5._lib.s5_workspace_size(ctypes.byref(b), 512, ctypes.byref(n)) == 0
    fixed = 256 + 16384                      # error record + partition counters
    scores = 64 * 16384 * 4                  # one fp32 score per history block and row
    parts = 64 * 64 * 2 * (192 + 1) * 4      # <= 2 partitions: one wave of 2 CTAs on <= 256 SMs
    assert n.value >= fixed + max(scores, parts)
    assert n.value < fixed + max(scores, parts) + 4096


@pytest.mark.parametrize("field,val,code", [
    ("batch", 0, 1), ("max_pages", 0, 1), ("total_q", -1, 1), ("max_len", (1 << 21) + 1, 2),
    ("max_len", 4 * 64 + 1, 1), ("page_table", 0, 1),
])
def test_bad_batch_rejected(s5, field, val, code):
    n = ctypes.c_size_t(0)
    b = _batch(**{field: val})
    assert s5._lib.s5_workspace_size(ctypes.byref(b), 512, ctypes.byref(n)) == code


def test_bad_descriptors_rejected_before_launch(s5):
    fake = ctypes.c_void_p(0x1000)
    b = _batch()
    kv = s5.KvDesc(0x1000, 0x1000, 8, 64, 4, 128)  # head_dim 128: not this build
    assert s5._lib.s5_sparse_gqa_attn(ctypes.byref(kv), ctypes.byref(b), fake, fake, fake, 512, 0.1, fake, None,
                                      fake, 1 << 30, None) == s5.S5_ERR_UNSUPPORTED
    kv = s5.KvDesc(0x1000, 0x1000, 8, 64, 4, 192)
    assert s5._lib.s5_sparse_gqa_attn(ctypes.byref(kv), ctypes.byref(b), fake, fake, fake, 513, 0.1, fake, None,
                                      fake, 1 << 30, None) == s5.S5_ERR_INVALID_ARG
    assert s5._lib.s5_swa_gqa_attn(ctypes.byref(kv), ctypes.byref(b), fake, 0, 0.1, fake, None, fake, 1 << 30,
                                   None) == s5.S5_ERR_INVALID_ARG
    assert s5._lib.s5_sparse_gqa_attn(ctypes.byref(kv), ctypes.byref(b), fake, fake, fake, 512, 0.1, fake, None,
                                      fake, 16, None) == s5.S5_ERR_WORKSPACE
    ix = s5.IndexDesc(0x1000, 8, 128)
    assert s5._lib.s5_index_score_topk(ctypes.byref(ix), ctypes.byref(b), fake, 512, fake, fake, fake, 1 << 30,
                                       None) == s5.S5_ERR_UNSUPPORTED
    ix = s5.IndexDesc(0x1000, 8, 256)
    assert s5._lib.s5_index_score_topk(ctypes.byref(ix), ctypes.byref(b), fake, 0, fake, fake, fake, 1 << 30,
                                       None) == s5.S5_ERR_INVALID_ARG
    assert s5._lib.s5_index_score_topk(ctypes.byref(ix), ctypes.byref(b), fake, 512, fake, fake, None, 1 << 30,
                                       None) == s5.S5_ERR_WORKSPACE


def test_workspace_covers_shared_set_tiles(s5):
    # multi-token batches also hold the tile kernel's union lists (8 rows per
    # tile, 8 x topk + 8 entries each), per-tile path flags and per-row skip
    # flags above the per-row partials; single-token batches do not
    n1, n4 = ctypes.c_size_t(0), ctypes.c_size_t(0)
    one = _batch(batch=64, total_q=64, max_q=1, max_pages=2049, max_len=131073)
    four = _batch(batch=64, total_q=256, max_q=4, max_pages=2049, max_len=131076)
    assert s5._lib.s5_workspace_size(ctypes.byref(one), 0, ctypes.byref(n1)) == 0
    assert s5._lib.s5_workspace_size(ctypes.byref(four), 0, ctypes.byref(n4)) == 0
    union = 64 * (8 * 512 + 8) * 4
    flags = 64 * 4 + 256 * 4
    assert n4.value >= 256 + 16384 + union + flags
    assert n4.value > n1.value
    # more rows per sequence never need less
    prev = 0
    for max_q in (2, 8, 9, 64, 65, 1000):
        b = _batch(batch=4, total_q=4 * max_q, max_q=max_q, max_pages=300, max_len=19000)
        n = ctypes.c_size_t(0)
        assert s5._lib.s5_workspace_size(ctypes.byref(b), 512, ctypes.byref(n)) == 0
        assert n.value >= prev
        prev = n.value


def test_append_rejects_bad_arguments_before_launch(s5):
    fake = ctypes.c_void_p(0x1000)
    odd = ctypes.c_void_p(0x1008)
    b = _batch()
    kv = s5.KvDesc(0x1000, 0x1000, 8, 64, 4, 192)
    ix = s5.IndexDesc(0x1000, 8, 256)
    big = 1 << 20
    ap = s5._lib.s5_append_kv
    # unsupported geometry
    bad_kv = s5.KvDesc(0x1000, 0x1000, 8, 64, 4, 128)
    assert ap(ctypes.byref(bad_kv), None, ctypes.byref(b), fake, fake, None, fake, big, None) == s5.S5_ERR_UNSUPPORTED
    bad_ix = s5.IndexDesc(0x1000, 8, 128)
    assert ap(ctypes.byref(kv), ctypes.byref(bad_ix), ctypes.byref(b), fake, fake, fake, fake, big,
              None) == s5.S5_ERR_UNSUPPORTED
    # missing or misaligned new rows, missing keys with a key pool
    assert ap(ctypes.byref(kv), None, ctypes.byref(b), None, fake, None, fake, big, None) == s5.S5_ERR_INVALID_ARG
    assert ap(ctypes.byref(kv), None, ctypes.byref(b), fake, odd, None, fake, big, None) == s5.S5_ERR_INVALID_ARG
    assert ap(ctypes.byref(kv), ctypes.byref(ix), ctypes.byref(b), fake, fake, None, fake, big,
              None) == s5.S5_ERR_INVALID_ARG
    # workspace: the error record and counters at least
    assert ap(ctypes.byref(kv), None, ctypes.byref(b), fake, fake, None, fake, 256, None) == s5.S5_ERR_WORKSPACE
    assert ap(ctypes.byref(kv), None, ctypes.byref(b), fake, fake, None, None, big, None) == s5.S5_ERR_WORKSPACE
    # bad batch
    assert ap(ctypes.byref(kv), None, ctypes.byref(_batch(batch=0)), fake, fake, None, fake, big,
              None) == s5.S5_ERR_INVALID_ARG
    # nothing to append: OK with nothing enqueued (null rows allowed)
    assert ap(ctypes.byref(kv), ctypes.byref(ix), ctypes.byref(_batch(total_q=0)), None, None, None, fake, big,
              None) == s5.S5_OK


def test_grouped_workspace_and_limits(s5):
    # one selection per KV group: four score rows per token
    n1, n4 = ctypes.c_size_t(0), ctypes.c_size_t(0)
    b = _batch(batch=64, total_q=64, max_q=1, max_pages=2049, max_len=131073)
    assert s5._lib.s5_workspace_size(ctypes.byref(b), 0, ctypes.byref(n1)) == 0
    assert s5._lib.s5_workspace_size_grouped(ctypes.byref(b), 0, ctypes.byref(n4)) == 0
    assert n4.value >= 256 + 16384 + 4 * 64 * 16384 * 4
    assert n4.value >= n1.value
    # small histories with many rows: the shared call's histograms may need more
    # than the grouped scores; the grouped size still covers every call
    b = _batch(batch=2, total_q=512, max_q=256, max_pages=20, max_len=1200)
    assert s5._lib.s5_workspace_size(ctypes.byref(b), 512, ctypes.byref(n1)) == 0
    assert s5._lib.s5_workspace_size_grouped(ctypes.byref(b), 512, ctypes.byref(n4)) == 0
    assert n4.value >= n1.value
    fake = ctypes.c_void_p(0x1000)
    ix = s5.IndexDesc(0x1000, 8, 256)
    # selections over more than 16,384 blocks: at most 65,535 (token, group) rows
    big = _batch(batch=1, total_q=20000, max_q=20000, max_pages=32768, max_len=(1 << 21))
    assert s5._lib.s5_index_score_topk_grouped(ctypes.byref(ix), ctypes.byref(big), fake, 512, fake, fake, fake,
                                               1 << 40, None) == s5.S5_ERR_UNSUPPORTED
    kv = s5.KvDesc(0x1000, 0x1000, 8, 64, 4, 192)
    assert s5._lib.s5_sparse_gqa_attn_grouped(ctypes.byref(kv), ctypes.byref(_batch()), fake, None, fake, 512, 0.1,
                                              fake, None, fake, 1 << 30, None) == s5.S5_ERR_INVALID_ARG
    assert s5._lib.s5_index_score_topk_grouped(ctypes.byref(ix), ctypes.byref(_batch()), fake, 512, fake, fake,
                                               None, 1 << 30, None) == s5.S5_ERR_WORKSPACE


def test_fp8_key_entry_checks(s5):
    fake = ctypes.c_void_p(0x1000)
    ix = s5.IndexDesc(0x1000, 8, 128)
    assert s5._lib.s5_index_score_topk_fp8(ctypes.byref(ix), ctypes.byref(_batch()), fake, 512, fake, fake, fake,
                                           1 << 30, None) == s5.S5_ERR_UNSUPPORTED
    ix = s5.IndexDesc(0x1008, 8, 256)  # not 16-byte aligned
    assert s5._lib.s5_index_score_topk_fp8(ctypes.byref(ix), ctypes.byref(_batch()), fake, 512, fake, fake, fake,
                                           1 << 30, None) == s5.S5_ERR_INVALID_ARG


def test_grouped_and_fp8_entries_validate_like_the_shared_ones(s5):
    fake = ctypes.c_void_p(0x1000)
    b = _batch()
    kv = s5.KvDesc(0x1000, 0x1000, 8, 64, 4, 192)
    # non-finite softmax scale, top-k out of range, short workspace
    assert s5._lib.s5_sparse_gqa_attn_grouped(ctypes.byref(kv), ctypes.byref(b), fake, fake, fake, 512,
                                              float("nan"), fake, None, fake, 1 << 30, None) == s5.S5_ERR_INVALID_ARG
    assert s5._lib.s5_sparse_gqa_attn_grouped(ctypes.byref(kv), ctypes.byref(b), fake, fake, fake, 0, 0.1, fake,
                                              None, fake, 1 << 30, None) == s5.S5_ERR_INVALID_ARG
    assert s5._lib.s5_sparse_gqa_attn_grouped(ctypes.byref(kv), ctypes.byref(b), fake, fake, fake, 512, 0.1, fake,
                                              None, fake, 16, None) == s5.S5_ERR_WORKSPACE
    ix = s5.IndexDesc(0x1000, 8, 256)
    for f in (s5._lib.s5_index_score_topk_grouped, s5._lib.s5_index_score_topk_fp8):
        assert f(ctypes.byref(ix), ctypes.byref(b), fake, 513, fake, fake, fake, 1 << 30, None) == s5.S5_ERR_INVALID_ARG
        assert f(ctypes.byref(ix), ctypes.byref(b), None, 512, fake, fake, fake, 1 << 30, None) == s5.S5_ERR_INVALID_ARG
        assert f(ctypes.byref(ix), ctypes.byref(b), fake, 512, fake, fake, fake, 16, None) == s5.S5_ERR_WORKSPACE
        # an empty batch enqueues nothing
        assert f(ctypes.byref(ix), ctypes.byref(_batch(total_q=0)), None, 512, None, None, fake, 16,
                 None) == s5.S5_OK
    n = ctypes.c_size_t(0)
    assert s5._lib.s5_workspace_size_grouped(ctypes.byref(b), -1, ctypes.byref(n)) == s5.S5_ERR_INVALID_ARG


def test_workspace_constants_match_header(s5):
    text = open(HEADER).read()
    m = re.search(r"#define S5_WS_FIXED_BYTES \((\d+) \+ (\d+)\)", text)
    assert m and int(m.group(1)) + int(m.group(2)) == s5.S5_WS_FIXED_BYTES
    m = re.search(r"#define S5_WS_TEST_STALL_OFFSET (\d+)", text)
    assert m and int(m.group(1)) == s5.S5_WS_TEST_STALL_OFFSET
    # the hook lies in the zeroed header, clear of the error record (bytes 0..7)
    assert 8 <= s5.S5_WS_TEST_STALL_OFFSET and s5.S5_WS_TEST_STALL_OFFSET + 8 <= 256


def test_fp8_kv_entry_checks(s5):
    fake = ctypes.c_void_p(0x1000)
    b = _batch()
    kv = s5.KvDesc(0x1000, 0x1000, 8, 64, 4, 192)
    f = s5._lib.s5_sparse_gqa_attn_fp8kv
    # non-finite scales (or an overflowing sm_scale * k_scale), bad top-k, short workspace, unaligned pool
    for ks, vs, sm in [(float("nan"), 1.0, 0.1), (1.0, float("inf"), 0.1), (1e38, 1.0, 1e3)]:
        assert f(ctypes.byref(kv), ctypes.byref(b), fake, fake, fake, 512, sm, ks, vs, fake, None, fake, 1 << 30,
                 None) == s5.S5_ERR_INVALID_ARG
    assert f(ctypes.byref(kv), ctypes.byref(b), fake, fake, fake, 0, 0.1, 1.0, 1.0, fake, None, fake, 1 << 30,
             None) == s5.S5_ERR_INVALID_ARG
    assert f(ctypes.byref(kv), ctypes.byref(b), fake, fake, fake, 512, 0.1, 1.0, 1.0, fake, None, fake, 16,
             None) == s5.S5_ERR_WORKSPACE
    kv_bad = s5.KvDesc(0x1008, 0x1000, 8, 64, 4, 192)
    assert f(ctypes.byref(kv_bad), ctypes.byref(b), fake, fake, fake, 512, 0.1, 1.0, 1.0, fake, None, fake, 1 << 30,
             None) == s5.S5_ERR_INVALID_ARG
    kv_geo = s5.KvDesc(0x1000, 0x1000, 8, 64, 4, 128)
    assert f(ctypes.byref(kv_geo), ctypes.byref(b), fake, fake, fake, 512, 0.1, 1.0, 1.0, fake, None, fake, 1 << 30,
             None) == s5.S5_ERR_UNSUPPORTED


def test_fp8_append_rejects_bad_scales_before_launch(s5):
    fake = ctypes.c_void_p(0x1000)
    kv = s5.KvDesc(0x1000, 0x1000, 8, 64, 4, 192)
    f = s5._lib.s5_append_kv_fp8
    for ks, vs in [(0.0, 1.0), (1.0, float("nan")), (float("inf"), 1.0), (1e-45, 1.0)]:
        assert f(ctypes.byref(kv), None, ctypes.byref(_batch()), fake, fake, None, ks, vs, fake, 1 << 20,
                 None) == s5.S5_ERR_INVALID_ARG
    assert f(ctypes.byref(kv), None, ctypes.byref(_batch()), fake, fake, None, 1.0, 1.0, fake, 16,
             None) == s5.S5_ERR_WORKSPACE


def test_noalloc_limits_checked_before_anything_is_enqueued(s5):
    # every case returns from the host checks, before the entry point looks up
    # its scratch array or enqueues anything
    fake = ctypes.c_void_p(0x1000)
    ix = s5.IndexDesc(0x1000, 8, 256)

    def call(b, topk=512, index=ix, q=fake):
        return s5._lib.s5_index_score_topk_noalloc(ctypes.byref(index), ctypes.byref(b), q, topk, fake, fake, None)

    # the scoring grid: 4-row tiles of one sequence on grid.z (<= 65,535), one sequence per grid.y
    # step; histories of 3 blocks (stride 4) let the 8 MiB scratch hold 262,141 rows
    assert call(_batch(batch=1, total_q=262141, max_q=262141, max_pages=1, max_len=32)) == s5.S5_ERR_UNSUPPORTED
    assert call(_batch(batch=65536, total_q=65536, max_q=1, max_pages=1, max_len=32)) == s5.S5_ERR_UNSUPPORTED
    # scores beyond the scratch: 130 rows x 16,376 fp32 = 8.5 MB > 8 MiB
    assert call(_batch(batch=2, total_q=130, max_q=65, max_pages=2048, max_len=131000)) == s5.S5_ERR_WORKSPACE
    # more than 16,384 history blocks need the two-stage select: max_len 131,081 is the first such length
    assert call(_batch(batch=1, total_q=1, max_q=1, max_pages=2049, max_len=131081)) == s5.S5_ERR_WORKSPACE
    assert call(_batch(batch=1, total_q=1, max_q=1, max_pages=2188, max_len=140000)) == s5.S5_ERR_WORKSPACE
    # argument checks shared with the workspace entry point
    b = _batch()
    assert call(b, topk=0) == s5.S5_ERR_INVALID_ARG
    assert call(b, topk=513) == s5.S5_ERR_INVALID_ARG
    assert call(b, index=s5.IndexDesc(0x1000, 8, 128)) == s5.S5_ERR_UNSUPPORTED
    assert call(b, index=s5.IndexDesc(0x1008, 8, 256)) == s5.S5_ERR_INVALID_ARG
    assert call(b, q=None) == s5.S5_ERR_INVALID_ARG
    assert call(b, q=ctypes.c_void_p(0x1004)) == s5.S5_ERR_INVALID_ARG
    assert call(_batch(max_len=4 * 64 + 1)) == s5.S5_ERR_INVALID_ARG  # pages cannot hold max_len
    # an empty batch enqueues nothing
    assert s5._lib.s5_index_score_topk_noalloc(ctypes.byref(ix), ctypes.byref(_batch(total_q=0)), None, 512, None,
                                               None, None) == s5.S5_OK
