"""Cache append (``s5_append_kv``) on the GPU, through the C ABI.

The append is a copy, so the bar is bit-exact: the pools it leaves must equal
the CPU oracle's and the generator's pools of the whole batch.  A decode step
that appends and then attends, eagerly and as a CUDA graph, must match the
oracle on the tokens it has just written.
"""
import numpy as np
import pytest
import torch

from block_sparse_gqa_indexer_b200 import synth as S
from oracle import s5_oracle as O
from tests.harness import LSE_ABS, assert_attn_close, oracle_selection, oracle_sparse, oracle_swa

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.contiguous().cpu().view(torch.int16).numpy()


class AppendInputs:
    """Prefix pools (the cache before the batch's new tokens) on the device,
    the new rows, and the pools of the whole batch to compare against."""

    def __init__(self, w: S.Workload, s5, with_index=True, junk_keys=True):
        self.w = w
        self.pt = w.page_table()
        self.k_pool, self.v_pool = w.kv_pools("cuda", self.pt, upto=w.ctx)
        self.key_pool = w.index_pool("cuda", self.pt, upto=w.ctx) if with_index else None
        kn, vn, xn = w.new_tokens("cuda")
        if junk_keys and w.total_q:
            # rows that complete no block: the append must not read their key
            _, pos = w.query_seq_pos()
            junk = torch.tensor([p % S.BLOCK != S.BLOCK - 1 for p in pos], device="cuda")
            xn = torch.where(junk.view(-1, 1), torch.full_like(xn, -3.5), xn)
        self.k_new, self.v_new, self.key_new = kn, vn, xn.contiguous()
        self.batch = s5.Batch.from_host(self.pt, w.ctx, w.nq, "cuda")
        self.ws = s5.new_workspace(self.batch, window=S.WINDOW, device="cuda")

    def append(self, s5, stream=None):
        s5.s5_append_kv(self.k_pool, self.v_pool, self.key_pool, self.batch, self.k_new, self.v_new,
                        self.key_new if self.key_pool is not None else None, self.ws, stream)


def _no_error(lib, ws):
    code, info = lib.s5_get_device_error(ws)
    assert code == 0, (lib.s5_status_string(code), info)


APPEND_CASES = [
    # page and block edges on both sides of the new tokens, an empty sequence,
    # a fresh sequence, several pages of new tokens
    ([0, 5, 63, 64, 130, 1000, 7, 40], [3, 9, 1, 64, 70, 17, 0, 200]),
    ([131072] * 2, [1] * 2),        # decode at 128K
    ([4090, 4095, 4096, 12345], [4, 4, 4, 4]),  # verify: 4 tokens each
]


@pytest.mark.parametrize("ctx,nq", APPEND_CASES)
def test_append_matches_oracle_and_generator(lib, ctx, nq):
    w = S.Workload(ctx=ctx, nq=nq, seed=31)
    a = AppendInputs(w, lib)
    before = (_bits(a.k_pool), _bits(a.v_pool), _bits(a.key_pool))
    a.append(lib)
    torch.cuda.synchronize()
    _no_error(lib, a.ws)
    got = (_bits(a.k_pool), _bits(a.v_pool), _bits(a.key_pool))
    want = O.append_to_paged_cache(*before, a.pt.numpy(), w.ctx, w.nq, _bits(a.k_new), _bits(a.v_new),
                                   _bits(a.key_new))
    for g, o in zip(got, want):
        assert np.array_equal(g, o)
    k1, v1 = w.kv_pools("cuda", a.pt)
    assert torch.equal(a.k_pool, k1) and torch.equal(a.v_pool, v1)
    assert torch.equal(a.key_pool, w.index_pool("cuda", a.pt))


def test_append_without_key_pool_window_only_cache(lib):
    # a sliding-window layer's cache: no block keys, and pages wholly before
    # every window unmapped (the append never touches them)
    w = S.Workload(ctx=[3000, 70, 9000], nq=[1, 5, 2], seed=32)
    a = AppendInputs(w, lib, with_index=False)
    for s in range(w.batch):
        first = max(0, w.ctx[s] - S.WINDOW + 1)
        for p in range(first // S.PAGE):
            a.pt[s, p] = -1
    a.batch.page_table.copy_(a.pt.cuda())
    a.k_pool, a.v_pool = w.kv_pools("cuda", w.page_table(), window_only=S.WINDOW, upto=w.ctx)
    before = (_bits(a.k_pool), _bits(a.v_pool))
    a.append(lib)
    torch.cuda.synchronize()
    _no_error(lib, a.ws)
    ko, vo, _ = O.append_to_paged_cache(*before, None, a.pt.numpy(), w.ctx, w.nq, _bits(a.k_new), _bits(a.v_new),
                                        None)
    assert np.array_equal(_bits(a.k_pool), ko) and np.array_equal(_bits(a.v_pool), vo)
    k1, v1 = w.kv_pools("cuda", w.page_table(), window_only=S.WINDOW)
    assert torch.equal(a.k_pool, k1) and torch.equal(a.v_pool, v1)


@pytest.mark.slow
def test_append_prefill_chunk_16k(lib):
    # a 16,384-token prefill chunk appended at offset 114,688: every CTA loops
    # over many rows; the result must be the generator's whole-batch cache
    w = S.Workload(ctx=[114688], nq=[16384], seed=33)
    a = AppendInputs(w, lib)
    a.append(lib)
    torch.cuda.synchronize()
    _no_error(lib, a.ws)
    k1, v1 = w.kv_pools("cuda", a.pt)
    assert torch.equal(a.k_pool, k1) and torch.equal(a.v_pool, v1)
    assert torch.equal(a.key_pool, w.index_pool("cuda", a.pt))


def test_append_unmapped_page_is_reported_and_skipped(lib):
    w = S.Workload(ctx=[100, 200, 300], nq=[1, 1, 1], seed=34)
    a = AppendInputs(w, lib)
    a.batch.page_table[1, 200 // S.PAGE] = -1  # row 1's page is unmapped
    lib.s5_reset_device_error(a.ws)
    a.append(lib)
    code, info = lib.s5_get_device_error(a.ws)
    assert code == lib.S5_ERR_DEVICE_BOUNDS and info == 1
    # the other rows were written
    k1, _ = w.kv_pools("cuda", a.pt)
    for s in (0, 2):
        t = w.ctx[s]
        p = int(a.pt[s, t // S.PAGE])
        assert torch.equal(a.k_pool[p, :, t % S.PAGE], k1[p, :, t % S.PAGE])


def test_append_then_attend_decode_step_in_cuda_graph(lib):
    # one hybrid decode step: a sparse layer appends its tokens and completed
    # block keys, scores, selects and attends; a sliding-window layer appends
    # and attends.  Eager and CUDA-graph replays give the same bits, and the
    # results match the oracle on the tokens just written.
    # sequence 1's third draft token (t = 9007) completes block 1125, which its
    # last two draft tokens already score in the same step
    ctx, nq = [5003, 9005, 303, 3000, 20479], [1, 5, 1, 5, 1]
    ws_ = S.Workload(ctx=ctx, nq=nq, seed=35)
    ww = S.Workload(ctx=ctx, nq=nq, seed=35, layer=1)
    sp = AppendInputs(ws_, lib)
    sw = AppendInputs(ww, lib, with_index=False)
    q, qx = ws_.queries("cuda")
    q_w, _ = ww.queries("cuda")
    tq = ws_.total_q
    sel = torch.full((tq, S.TOPK), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((tq,), -7, dtype=torch.int32, device="cuda")
    out = torch.empty((tq, 64, 192), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((tq, 64), dtype=torch.float32, device="cuda")
    out_w, lse_w = torch.empty_like(out), torch.empty_like(lse)
    prefix = [t.clone() for t in (sp.k_pool, sp.v_pool, sp.key_pool, sw.k_pool, sw.v_pool)]

    def step():
        sp.append(lib)
        lib.s5_index_score_topk(sp.key_pool, sp.batch, qx, S.TOPK, sel, cnt, sp.ws)
        lib.s5_sparse_gqa_attn(sp.k_pool, sp.v_pool, sp.batch, q, sel, cnt, S.TOPK, O.DEFAULT_SM_SCALE, out, lse,
                               sp.ws)
        sw.append(lib)
        lib.s5_swa_gqa_attn(sw.k_pool, sw.v_pool, sw.batch, q_w, S.WINDOW, O.DEFAULT_SM_SCALE, out_w, lse_w, sw.ws)

    def restore():
        for dst, src in zip((sp.k_pool, sp.v_pool, sp.key_pool, sw.k_pool, sw.v_pool), prefix):
            dst.copy_(src)

    results = (sel, cnt, out, lse, out_w, lse_w)
    step()
    torch.cuda.synchronize()
    eager = [t.clone() for t in results]
    restore()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for t in results:
        t.zero_()
    g.replay()
    torch.cuda.synchronize()
    for a_, b_ in zip(eager, results):
        assert torch.equal(a_, b_)
    _no_error(lib, sp.ws)
    _no_error(lib, sw.ws)

    rows = list(range(tq))
    want_sel = oracle_selection(ws_, rows)
    assert np.array_equal(sel.cpu().numpy(), want_sel)
    want, want_lse = oracle_sparse(ws_, rows, want_sel)
    assert_attn_close(out.float().cpu().numpy(), want, "sparse layer after append")
    assert np.abs(lse.cpu().numpy() - want_lse).max() <= LSE_ABS
    want_w, want_lse_w = oracle_swa(ww, rows)
    assert_attn_close(out_w.float().cpu().numpy(), want_w, "sliding-window layer after append")
    assert np.abs(lse_w.cpu().numpy() - want_lse_w).max() <= LSE_ABS
    del g
