"""The indexer entry point that allocates nothing.

Some callers cannot allocate device memory (a host framework that owns every
device allocation and hands over only inputs and outputs, or a fixed
device-memory budget), so s5_index_score_topk_noalloc keeps its scratch in a
fixed array inside the library.  Its selections must equal those of
s5_index_score_topk with a caller workspace, on two calls in a row (the
second call must not be affected by what the first left in the array).
This file is collected last so that a stop-at-first-failure run has already
run every other test; it also passes alone in a fresh process.
"""
import pytest
import torch

from block_sparse_gqa_indexer_b200 import synth as S

pytestmark = pytest.mark.gpu


def _inputs(lib, ctx, nq, seed):
    w = S.Workload(ctx=ctx, nq=nq, seed=seed)
    pt = w.page_table()
    key_pool = w.index_pool("cuda", pt)
    _, qx = w.queries("cuda")
    batch = lib.Batch.from_host(pt, w.ctx, w.nq, "cuda")
    return w, key_pool, qx, batch


def _reference(lib, key_pool, batch, qx):
    ws = lib.new_workspace(batch)
    sel = torch.empty((batch.total_q, S.TOPK), dtype=torch.int32, device="cuda")
    cnt = torch.empty((batch.total_q,), dtype=torch.int32, device="cuda")
    lib.s5_index_score_topk(key_pool, batch, qx, S.TOPK, sel, cnt, ws)
    code, _ = lib.s5_get_device_error(ws)
    assert code == 0
    return sel, cnt


def test_noalloc_matches_workspace_path_twice(lib):
    # varlen batches with short and long histories, a verify row group and a
    # chunk row, called back to back
    cases = [([20000, 300, 9000, 131072], [1, 1, 4, 1], 31),
             ([50000, 4500, 70000], [2, 1, 3], 32),
             # a chunk row: 200 new tokens of one sequence (more than 16 row
             # tiles of the scoring grid; the workspace path scores these on
             # the tensor cores instead)
             ([6000, 300], [200, 1], 35)]
    for ctx, nq, seed in cases:
        w, key_pool, qx, batch = _inputs(lib, ctx, nq, seed)
        want_sel, want_cnt = _reference(lib, key_pool, batch, qx)
        sel = torch.full_like(want_sel, -5)
        cnt = torch.full_like(want_cnt, -5)
        lib.s5_index_score_topk_noalloc(key_pool, batch, qx, S.TOPK, sel, cnt)
        torch.cuda.synchronize()
        assert torch.equal(sel, want_sel)
        assert torch.equal(cnt, want_cnt)


def test_noalloc_rejects_oversized_requests(lib):
    # 130 rows of 16,375 history blocks need 8.5 MB of scores: more than the 8 MiB scratch
    w, key_pool, qx, batch = _inputs(lib, [131000] * 130, [1] * 130, 33)
    sel = torch.empty((batch.total_q, S.TOPK), dtype=torch.int32, device="cuda")
    cnt = torch.empty((batch.total_q,), dtype=torch.int32, device="cuda")
    with pytest.raises(lib.S5Error) as e:
        lib.s5_index_score_topk_noalloc(key_pool, batch, qx, S.TOPK, sel, cnt)
    assert e.value.code == lib.S5_ERR_WORKSPACE
    # a history above 16,384 blocks needs the two-stage select, which has no fixed scratch here
    w, key_pool, qx, batch = _inputs(lib, [140000], [1], 34)
    sel = torch.empty((1, S.TOPK), dtype=torch.int32, device="cuda")
    cnt = torch.empty((1,), dtype=torch.int32, device="cuda")
    with pytest.raises(lib.S5Error) as e:
        lib.s5_index_score_topk_noalloc(key_pool, batch, qx, S.TOPK, sel, cnt)
    assert e.value.code == lib.S5_ERR_WORKSPACE
