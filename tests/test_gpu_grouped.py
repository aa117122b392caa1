"""Per-KV-group selection on the GPU against the CPU oracle, through the C ABI.

Each token carries one indexer query per KV group; every (token, group)
selection must match the oracle bit-exactly, and the attention of head h must
follow its group's selection within the attention tolerances.
"""
import numpy as np
import pytest
import torch

from block_sparse_gqa_indexer_b200 import synth as S
from oracle import s5_oracle as O
from tests.harness import LSE_ABS, LazyRows, assert_attn_close, oracle_selection_grouped, sample_rows

pytestmark = pytest.mark.gpu


class GroupedInputs:
    def __init__(self, w: S.Workload, s5):
        self.w = w
        self.pt = w.page_table()
        self.k_pool, self.v_pool = w.kv_pools("cuda", self.pt)
        self.key_pool = w.index_pool("cuda", self.pt)
        rows = torch.arange(w.total_q, dtype=torch.int64)
        self.q = w.q_rows(rows, "cuda")
        self.qx = w.qx_group_rows(rows, "cuda").contiguous()
        self.batch = s5.Batch.from_host(self.pt, w.ctx, w.nq, "cuda")
        self.ws = s5.new_workspace(self.batch, window=S.WINDOW, device="cuda", grouped=True)
        tq = w.total_q
        self.sel = torch.full((tq, S.N_KV, S.TOPK), -7, dtype=torch.int32, device="cuda")
        self.cnt = torch.full((tq, S.N_KV), -7, dtype=torch.int32, device="cuda")
        self.out = torch.full((tq, 64, 192), float("nan"), dtype=torch.bfloat16, device="cuda")
        self.lse = torch.full((tq, 64), float("nan"), dtype=torch.float32, device="cuda")

    def run(self, s5):
        s5.s5_index_score_topk_grouped(self.key_pool, self.batch, self.qx, S.TOPK, self.sel, self.cnt, self.ws)
        s5.s5_sparse_gqa_attn_grouped(self.k_pool, self.v_pool, self.batch, self.q, self.sel, self.cnt, S.TOPK,
                                      O.DEFAULT_SM_SCALE, self.out, self.lse, self.ws)


def _no_error(lib, ws):
    code, info = lib.s5_get_device_error(ws)
    assert code == 0, (lib.s5_status_string(code), info)


def _check_selections(g: GroupedInputs, rows=None):
    """Every listed row's four selections and counts, bit for bit (default: all rows)."""
    rows = list(range(g.w.total_q)) if rows is None else list(rows)
    want = oracle_selection_grouped(g.w, rows)
    sel = g.sel.cpu().numpy()[rows]
    cnt = g.cnt.cpu().numpy()[rows]
    bad = np.nonzero(~np.all(sel == want, axis=(1, 2)))[0]
    assert bad.size == 0, f"{bad.size} rows with a differing group selection, first {[rows[i] for i in bad[:8]]}"
    assert np.array_equal(cnt, (want >= 0).sum(axis=2)), "selection counts differ"
    return want


def _check(lib, g: GroupedInputs, rows, all_selections=False):
    torch.cuda.synchronize()
    _no_error(lib, g.ws)
    w = g.w
    seqs, pos = w.query_seq_pos()
    rows = list(rows)
    q = w.q_rows(torch.as_tensor(rows, dtype=torch.int64)).double().numpy()
    if all_selections:
        want_sel = _check_selections(g)[rows]
    else:
        want_sel = _check_selections(g, rows)
    want_o, want_l = [], []
    for i, r in enumerate(rows):
        s, t = seqs[r], pos[r]
        want = want_sel[i]
        o, l = O.sparse_attention_query_grouped(q[i], want, t, LazyRows(w, s, "k"), LazyRows(w, s, "v"))
        want_o.append(O.round_bf16(o))
        want_l.append(l)
    got = g.out.float().cpu().numpy()[rows]
    assert_attn_close(got, np.array(want_o), "grouped sparse attention")
    assert np.abs(g.lse.cpu().numpy()[rows] - np.array(want_l)).max() <= LSE_ABS


GROUPED_SMALL = [
    ([0, 5, 4095, 4104, 6000, 20001], [1, 1, 1, 1, 1, 1]),   # below / at / above 512 blocks
    ([5000, 4090, 12345], [4, 4, 4]),                         # verify: 4 tokens x 4 groups per sequence
    ([3, 4200, 777, 16383, 9000], [2, 3, 1, 4, 0]),           # varlen, an empty sequence
]


@pytest.mark.parametrize("ctx,nq", GROUPED_SMALL)
def test_grouped_small_all_rows(lib, ctx, nq):
    g = GroupedInputs(S.Workload(ctx=ctx, nq=nq, seed=41), lib)
    g.run(lib)
    _check(lib, g, range(g.w.total_q))


def test_grouped_prefill_sized_tensor_core_scores(lib):
    # 40 tokens x 4 groups = 160 indexer rows per sequence: scored by the
    # tcgen05 GEMM, rows token-major and group-minor
    g = GroupedInputs(S.Workload(ctx=[9000, 6007], nq=[40, 33], seed=42), lib)
    g.run(lib)
    # every row's selection, attention on sampled rows
    _check(lib, g, sample_rows(g.w.total_q, 12, 1), all_selections=True)


def test_grouped_more_than_1024_selection_rows(lib):
    # 20 x 16 tokens x 4 groups = 1,280 rows: the select runs two CTAs per SM
    # and builds each row's histogram in shared memory
    g = GroupedInputs(S.Workload(ctx=[7000 + 37 * i for i in range(20)], nq=[16] * 20, seed=43), lib)
    g.run(lib)
    _check(lib, g, sample_rows(g.w.total_q, 10, 2), all_selections=True)


def test_grouped_history_beyond_16k_blocks(lib):
    # rows of more than 16,384 history blocks: per-segment top-k, then a merge
    g = GroupedInputs(S.Workload(ctx=[140000, 9000, 200003], nq=[1, 2, 1], seed=46), lib)
    g.run(lib)
    _check(lib, g, range(g.w.total_q))


def test_grouped_equal_selections_match_the_shared_call_bit_for_bit(lib):
    # decode rows take the same per-row kernel either way: handing every group
    # the shared selection must reproduce the shared call exactly
    w = S.Workload(ctx=[9000, 30000, 4100, 131072], nq=[1, 1, 1, 1], seed=44)
    g = GroupedInputs(w, lib)
    _, qx = w.queries("cuda")
    sel1 = torch.empty((w.total_q, S.TOPK), dtype=torch.int32, device="cuda")
    cnt1 = torch.empty((w.total_q,), dtype=torch.int32, device="cuda")
    lib.s5_index_score_topk(g.key_pool, g.batch, qx, S.TOPK, sel1, cnt1, g.ws)
    out1, lse1 = torch.empty_like(g.out), torch.empty_like(g.lse)
    lib.s5_sparse_gqa_attn(g.k_pool, g.v_pool, g.batch, g.q, sel1, cnt1, S.TOPK, O.DEFAULT_SM_SCALE, out1, lse1, g.ws)
    sel4 = sel1.unsqueeze(1).repeat(1, S.N_KV, 1).contiguous()
    cnt4 = cnt1.unsqueeze(1).repeat(1, S.N_KV).contiguous()
    lib.s5_sparse_gqa_attn_grouped(g.k_pool, g.v_pool, g.batch, g.q, sel4, cnt4, S.TOPK, O.DEFAULT_SM_SCALE, g.out,
                                   g.lse, g.ws)
    torch.cuda.synchronize()
    _no_error(lib, g.ws)
    assert torch.equal(out1, g.out) and torch.equal(lse1, g.lse)


def test_grouped_bad_count_in_a_later_group_is_reported(lib):
    w = S.Workload(ctx=[9000, 5000], nq=[1, 1], seed=45)
    g = GroupedInputs(w, lib)
    lib.s5_index_score_topk_grouped(g.key_pool, g.batch, g.qx, S.TOPK, g.sel, g.cnt, g.ws)
    g.cnt[1, 3] = S.TOPK + 1  # row 1, group 3: more than topk
    lib.s5_reset_device_error(g.ws)
    lib.s5_sparse_gqa_attn_grouped(g.k_pool, g.v_pool, g.batch, g.q, g.sel, g.cnt, S.TOPK, O.DEFAULT_SM_SCALE,
                                   g.out, g.lse, g.ws)
    code, info = lib.s5_get_device_error(g.ws)
    assert code == lib.S5_ERR_DEVICE_BOUNDS and info == 1


@pytest.mark.slow
def test_grouped_decode_b64_128k(lib):
    (w0,) = S.config_workloads(0)
    g = GroupedInputs(w0, lib)
    g.run(lib)
    # all 64 x 4 selections; attention on sampled rows
    _check(lib, g, sample_rows(w0.total_q, 3, 3), all_selections=True)
