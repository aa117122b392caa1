"""CUDA path against the CPU oracle, through the C ABI.

Selections must match bit-exactly (integer-valued indexer inputs make the fp32
scores exact); attention outputs must be within max-abs 2e-2 and rel-RMS 5e-3
of the float64 oracle (rounded to bf16), lse within 1e-3.
"""
import numpy as np
import pytest
import torch

from block_sparse_gqa_indexer_b200 import synth as S
from oracle import s5_oracle as O
from tests.harness import (DeviceInputs, LSE_ABS, assert_attn_close, check_all_selections, oracle_selection,
                           oracle_sparse, oracle_swa, sample_rows)

pytestmark = pytest.mark.gpu


def _run_index(lib, d: DeviceInputs):
    lib.s5_index_score_topk(d.key_pool, d.batch, d.qx, S.TOPK, d.sel, d.sel_count, d.ws)


def _run_sparse(lib, d: DeviceInputs, sel=None, sm_scale=O.DEFAULT_SM_SCALE):
    lib.s5_sparse_gqa_attn(d.k_pool, d.v_pool, d.batch, d.q, d.sel if sel is None else sel, d.sel_count, S.TOPK,
                           sm_scale, d.out, d.lse, d.ws)


def _check_no_device_error(lib, d):
    code, info = lib.s5_get_device_error(d.ws)
    assert code == 0, (lib.s5_status_string(code), info)


def _check_selection(lib, d, rows):
    torch.cuda.synchronize()
    want = oracle_selection(d.w, rows)
    got = d.sel.cpu().numpy()[rows]
    cnt = d.sel_count.cpu().numpy()[rows]
    for i, r in enumerate(rows):
        assert np.array_equal(got[i], want[i]), f"row {r}: selection differs"
        assert cnt[i] == O.selection_count(want[i])
    return want


def _check_sparse_out(d, rows, sel_rows, what):
    want, want_lse = oracle_sparse(d.w, rows, sel_rows)
    got = d.out.float().cpu().numpy()[rows]
    assert_attn_close(got, want, what)
    lse = d.lse.cpu().numpy()[rows]
    assert np.abs(lse - want_lse).max() <= LSE_ABS


# ------------------------------------------------------------------ small cases (every row checked)

SMALL_SPARSE = [
    # ctx per sequence, nq per sequence: history below / at / above 512 blocks, ragged tails
    ([0, 5, 7, 8, 100], [1, 1, 1, 1, 1]),
    ([4095, 4096, 4103, 4104, 4111], [1, 1, 1, 1, 1]),
    ([6000, 9999, 20001], [1, 1, 1]),
    ([5000, 4090, 12345], [4, 4, 4]),            # verify: 4 tokens each, crossing block edges
    ([3, 4200, 777, 16383, 9000], [2, 3, 1, 4, 0]),  # varlen, an empty sequence
]


@pytest.mark.parametrize("ctx,nq", SMALL_SPARSE)
def test_sparse_small_all_rows(lib, ctx, nq):
    w = S.Workload(ctx=ctx, nq=nq, seed=11)
    d = DeviceInputs(w, lib)
    _run_index(lib, d)
    _run_sparse(lib, d)
    rows = list(range(w.total_q))
    want_sel = _check_selection(lib, d, rows)
    _check_sparse_out(d, rows, want_sel, f"sparse ctx={ctx} nq={nq}")
    _check_no_device_error(lib, d)


@pytest.mark.parametrize("ctx,nq,window", [
    ([0, 1, 300, 511, 512, 513, 1000], [1] * 7, 512),
    ([7000, 65, 2047], [4, 2, 1], 512),
    ([2500, 100], [1, 3], 64),
    ([900, 33], [1, 1], 4096),  # window covers everything: full causal attention
])
def test_swa_small_all_rows(lib, ctx, nq, window):
    w = S.Workload(ctx=ctx, nq=nq, seed=12)
    d = DeviceInputs(w, lib, with_index=False)
    lib.s5_swa_gqa_attn(d.k_pool, d.v_pool, d.batch, d.q, window, O.DEFAULT_SM_SCALE, d.out, d.lse, d.ws)
    rows = list(range(w.total_q))
    want, want_lse = oracle_swa(w, rows, window)
    assert_attn_close(d.out.float().cpu().numpy(), want, f"swa ctx={ctx} W={window}")
    assert np.abs(d.lse.cpu().numpy() - want_lse).max() <= LSE_ABS
    _check_no_device_error(lib, d)


def test_sparse_equals_swa_when_history_fits(lib):
    # c <= 512 selects every history block: sparse == sliding window with W >= length
    w = S.Workload(ctx=[1000, 4000, 4095], nq=[1, 2, 1], seed=13)
    d = DeviceInputs(w, lib)
    _run_index(lib, d)
    _run_sparse(lib, d)
    torch.cuda.synchronize()
    sparse_out = d.out.clone()
    lib.s5_swa_gqa_attn(d.k_pool, d.v_pool, d.batch, d.q, 1 << 20, O.DEFAULT_SM_SCALE, d.out, d.lse, d.ws)
    assert_attn_close(sparse_out.float().cpu().numpy(), d.out.float().cpu().numpy(), "sparse vs full")


def test_sparse_block_order_invariance(lib):
    w = S.Workload(ctx=[30000, 7777], nq=[1, 2], seed=14)
    d = DeviceInputs(w, lib)
    _run_index(lib, d)
    _run_sparse(lib, d)
    torch.cuda.synchronize()
    ref = d.out.float().cpu().numpy()
    g = torch.Generator().manual_seed(3)
    sel = d.sel.cpu()
    perm = sel.clone()
    for r in range(sel.shape[0]):
        n = int(d.sel_count[r])
        perm[r, :n] = sel[r, :n][torch.randperm(n, generator=g)]
    _run_sparse(lib, d, sel=perm.cuda())
    assert_attn_close(d.out.float().cpu().numpy(), ref, "permuted selection")


def test_deterministic_across_runs(lib):
    w = S.Workload(ctx=[20000] * 6, nq=[1] * 6, seed=15)
    d = DeviceInputs(w, lib)
    outs = []
    for _ in range(3):
        _run_index(lib, d)
        _run_sparse(lib, d)
        torch.cuda.synchronize()
        outs.append((d.sel.clone(), d.out.clone(), d.lse.clone()))
    for o in outs[1:]:
        assert torch.equal(o[0], outs[0][0]) and torch.equal(o[1], outs[0][1]) and torch.equal(o[2], outs[0][2])


def test_softmax_weights_sum_to_one(lib):
    # with every V row equal to 1, each output is the sum of the softmax weights
    w = S.Workload(ctx=[9000, 300], nq=[1, 1], seed=16)
    d = DeviceInputs(w, lib)
    d.v_pool.fill_(1.0)
    _run_index(lib, d)
    _run_sparse(lib, d)
    torch.cuda.synchronize()
    # P is rounded to bf16 for the PV product while the denominator sums it in fp32
    assert float((d.out.float() - 1.0).abs().max()) <= 2 ** -8


def test_tie_heavy_selection(lib):
    # all block keys equal: every score ties, the first 512 blocks win
    w = S.Workload(ctx=[50000, 8 * 600 + 3], nq=[1, 2], seed=17)
    d = DeviceInputs(w, lib)
    d.key_pool.fill_(1.0)
    _run_index(lib, d)
    torch.cuda.synchronize()
    for r in range(w.total_q):
        assert d.sel[r].tolist() == list(range(512))


def test_bad_page_is_reported_not_read(lib):
    w = S.Workload(ctx=[20000], nq=[1], seed=18)
    d = DeviceInputs(w, lib)
    d.batch.page_table[0, 5] = -1  # an unmapped page in the history
    lib.s5_reset_device_error(d.ws)
    _run_index(lib, d)
    _run_sparse(lib, d)
    code, info = lib.s5_get_device_error(d.ws)
    assert code == lib.S5_ERR_DEVICE_BOUNDS and info == 0
    assert torch.isfinite(d.out.float()).all()


def test_host_validation(lib):
    w = S.Workload(ctx=[100], nq=[1], seed=19)
    d = DeviceInputs(w, lib)
    with pytest.raises(lib.S5Error) as e:
        lib.s5_sparse_gqa_attn(d.k_pool, d.v_pool, d.batch, d.q, d.sel, d.sel_count, S.TOPK, float("nan"), d.out,
                               d.lse, d.ws)
    assert e.value.code == lib.S5_ERR_INVALID_ARG
    with pytest.raises(lib.S5Error) as e:
        lib.s5_swa_gqa_attn(d.k_pool, d.v_pool, d.batch, d.q, 0, 0.1, d.out, d.lse, d.ws)
    assert e.value.code == lib.S5_ERR_INVALID_ARG
    with pytest.raises(lib.S5Error) as e:
        lib.s5_sparse_gqa_attn(d.k_pool, d.v_pool, d.batch, d.q, d.sel, d.sel_count, S.TOPK, 0.1, d.out, d.lse,
                               d.ws[:64])
    assert e.value.code == lib.S5_ERR_WORKSPACE


# ------------------------------------------------------------------ the configurations (sampled rows)

def _config_sparse(lib, which, n_rows, seed=0):
    # every row's selection bit for bit; attention on sampled rows
    (w,) = S.config_workloads(which)
    d = DeviceInputs(w, lib)
    lib.s5_reset_device_error(d.ws)
    _run_index(lib, d)
    _run_sparse(lib, d)
    torch.cuda.synchronize()
    want_all = check_all_selections(w, d.sel, d.sel_count)
    rows = sample_rows(w.total_q, n_rows, seed)
    _check_sparse_out(d, rows, want_all[rows], f"config {which}")
    _check_no_device_error(lib, d)
    return d


@pytest.mark.slow
def test_config1_sparse_decode_b1_16k(lib):
    _config_sparse(lib, 1, 1)


@pytest.mark.slow
def test_config3_sparse_verify_b64x4(lib):
    _config_sparse(lib, 3, 8)


@pytest.mark.slow
def test_headline_sparse_decode_b64_128k(lib):
    _config_sparse(lib, 0, 4)


@pytest.mark.slow
def test_config2_swa_decode_b64(lib):
    (w,) = S.config_workloads(2)
    d = DeviceInputs(w, lib, window_only=S.WINDOW, with_index=False)
    lib.s5_swa_gqa_attn(d.k_pool, d.v_pool, d.batch, d.q, S.WINDOW, O.DEFAULT_SM_SCALE, d.out, d.lse, d.ws)
    rows = sample_rows(w.total_q, 8)
    want, want_lse = oracle_swa(w, rows)
    assert_attn_close(d.out.float().cpu().numpy()[rows], want, "config 2")
    assert np.abs(d.lse.cpu().numpy()[rows] - want_lse).max() <= LSE_ABS
    _check_no_device_error(lib, d)


@pytest.mark.slow
def test_config4_sparse_prefill_16k(lib):
    _config_sparse(lib, 4, 6)


@pytest.mark.slow
def test_config5_hybrid_1m(lib):
    layers = S.config_workloads(5)
    for li, w in enumerate(layers):
        if li < 3:
            d = DeviceInputs(w, lib, window_only=S.WINDOW, with_index=False)
            lib.s5_swa_gqa_attn(d.k_pool, d.v_pool, d.batch, d.q, S.WINDOW, O.DEFAULT_SM_SCALE, d.out, d.lse, d.ws)
            rows = sample_rows(w.total_q, 2, li)
            want, _ = oracle_swa(w, rows)
            assert_attn_close(d.out.float().cpu().numpy()[rows], want, f"config 5 swa layer {li}")
            _check_no_device_error(lib, d)
        else:
            d = DeviceInputs(w, lib)
            _run_index(lib, d)
            _run_sparse(lib, d)
            torch.cuda.synchronize()
            want_sel = check_all_selections(w, d.sel, d.sel_count)  # all 4 rows
            rows = sample_rows(w.total_q, 2, li)
            _check_sparse_out(d, rows, want_sel[rows], "config 5 sparse layer")
            _check_no_device_error(lib, d)
        del d
        torch.cuda.empty_cache()


def test_swa_many_rows_wide_window_separate_merge(lib):
    # > 1,024 rows whose windows need two partitions each: partitions merge in
    # the standalone kernel instead of inside the attention kernel
    w = S.Workload(ctx=[8000], nq=[1100], seed=20)
    d = DeviceInputs(w, lib, with_index=False)
    d.ws = lib.new_workspace(d.batch, window=8192)
    lib.s5_swa_gqa_attn(d.k_pool, d.v_pool, d.batch, d.q, 8192, O.DEFAULT_SM_SCALE, d.out, d.lse, d.ws)
    rows = sample_rows(w.total_q, 6, 5)
    want, want_lse = oracle_swa(w, rows, 8192)
    assert_attn_close(d.out.float().cpu().numpy()[rows], want, "swa W=8192, 1100 rows")
    assert np.abs(d.lse.cpu().numpy()[rows] - want_lse).max() <= LSE_ABS
    _check_no_device_error(lib, d)


@pytest.mark.parametrize("ctx,nq", [
    ([3000, 70000], [300, 200]),    # more than 64 rows per sequence: tensor-core scoring
    ([100, 20000, 9], [129, 1, 70]),
])
def test_prefill_sized_batches_all_selections(lib, ctx, nq):
    w = S.Workload(ctx=ctx, nq=nq, seed=22)
    d = DeviceInputs(w, lib)
    _run_index(lib, d)
    _run_sparse(lib, d)
    rows = list(range(w.total_q))
    want_sel = _check_selection(lib, d, rows)
    some = sample_rows(w.total_q, 8, 3)
    _check_sparse_out(d, some, want_sel[some], f"prefill-sized ctx={ctx} nq={nq}")
    _check_no_device_error(lib, d)


def test_tile_late_max_rescale(lib):
    # verify rows (4 per sequence, block-coherent indexer queries so the tiles
    # take the shared-set tensor-core path): the keys of the last
    # block read (the current block, highest index) are made to align strongly
    # with head 0 of every group, so that row maximum jumps late and the
    # accumulated output must be rescaled
    w = S.Workload(ctx=[9000, 20000], nq=[4, 4], seed=23, qx_coherent=64)
    d = DeviceInputs(w, lib)
    seqs, pos = w.query_seq_pos()
    q_cpu = d.q.float().cpu()
    k_cpu = {}
    for r in range(w.total_q):
        s, t = seqs[r], pos[r]
        for tok in range((t // 8) * 8, t + 1):
            page = int(d.pt[s, tok // 64])
            for g in range(4):
                vec = (6.0 * q_cpu[r, 16 * g]).to(torch.bfloat16)
                d.k_pool[page, g, tok % 64] = vec.to(d.k_pool.device)
                k_cpu[(s, tok, g)] = vec.double().numpy()
    _run_index(lib, d)
    _run_sparse(lib, d)
    torch.cuda.synchronize()
    sel = d.sel.cpu().numpy()
    got = d.out.float().cpu().numpy()
    for r in range(w.total_q):
        s, t = seqs[r], pos[r]
        T = O.sparse_token_set(sel[r], t)
        K = w.k_tokens(s, torch.as_tensor(T)).double().numpy()
        for i, tok in enumerate(T.tolist()):
            for g in range(4):
                if (s, tok, g) in k_cpu:
                    K[i, g] = k_cpu[(s, tok, g)]
        V = w.v_tokens(s, torch.as_tensor(T)).double().numpy()
        want, _ = O.gqa_attention(q_cpu[r].double().numpy(), K, V, O.DEFAULT_SM_SCALE)
        assert_attn_close(got[r], O.round_bf16(want), f"row {r}")
    _check_no_device_error(lib, d)


def _tiles_by_path(w, sel):
    """(shared-set tiles, per-row tiles) of a batch under the library's
    crossover rule: an 8-row tile takes the shared set when its union of blocks
    (selected + current) is at most 70 % of the blocks its rows read one by one."""
    seqs, pos = w.query_seq_pos()
    shared = per_row = 0
    r = 0
    for s in range(w.batch):
        for k in range(0, w.nq[s], 8):
            rows = range(r + k, r + min(k + 8, w.nq[s]))
            union, total = set(), 0
            for i in rows:
                blocks = set(int(b) for b in sel[i] if b >= 0) | {pos[i] // 8}
                union |= blocks
                total += len(blocks)
            if 100 * len(union) <= 70 * total:
                shared += 1
            else:
                per_row += 1
        r += w.nq[s]
    return shared, per_row


@pytest.mark.parametrize("ctx,nq,coherent,need_per_row", [
    ([20000, 3000, 70000], [300, 77, 45], 64, False),  # block-coherent queries: shared-set tiles
    ([9000, 4000, 100000], [40, 9, 23], 0, True),      # independent queries: both paths in one batch
])
def test_prefill_both_paths(lib, ctx, nq, coherent, need_per_row):
    w = S.Workload(ctx=ctx, nq=nq, seed=24, qx_coherent=coherent)
    d = DeviceInputs(w, lib)
    lib.s5_reset_device_error(d.ws)
    _run_index(lib, d)
    _run_sparse(lib, d)
    rows = list(range(w.total_q))
    want_sel = _check_selection(lib, d, rows)
    shared, per_row = _tiles_by_path(w, want_sel)
    assert shared > 0 and (per_row > 0 or not need_per_row), (shared, per_row)
    some = sample_rows(w.total_q, 16, 4)
    _check_sparse_out(d, some, want_sel[some], f"prefill ctx={ctx} nq={nq} coherent={coherent}")
    _check_no_device_error(lib, d)


@pytest.mark.slow
def test_config6_block_coherent_prefill_16k(lib):
    _config_sparse(lib, 6, 6)


def test_tile_batches_beyond_the_compacted_list(lib):
    # more than 4,096 tiles (520 sequences x 8 tiles of 8 rows): the tile
    # kernel walks every tile instead of a compacted list of shared-set tiles
    ctx = [int(x) for x in S.uniform_lengths(25, 520, 0, 300)]
    w = S.Workload(ctx=ctx, nq=[64] * 520, seed=25)
    d = DeviceInputs(w, lib)
    lib.s5_reset_device_error(d.ws)
    _run_index(lib, d)
    _run_sparse(lib, d)
    rows = sample_rows(w.total_q, 12, 6)
    want_sel = _check_selection(lib, d, rows)
    _check_sparse_out(d, rows, want_sel, "4,160 tiles")
    _check_no_device_error(lib, d)


@pytest.mark.parametrize("sm_scale", [0.0, -0.04, 0.3])
def test_softmax_scale_sign_and_zero_both_paths(lib, sm_scale):
    # a zero or negative scale turns the row maximum into the scores' minimum
    # (or makes every weight equal): shared-set tiles (8 rows at a short
    # history) and per-row decode rows in one batch
    w = S.Workload(ctx=[2000, 7000, 150], nq=[8, 1, 3], seed=26)
    d = DeviceInputs(w, lib)
    _run_index(lib, d)
    _run_sparse(lib, d, sm_scale=sm_scale)
    rows = list(range(w.total_q))
    want_sel = _check_selection(lib, d, rows)
    want, want_lse = oracle_sparse(w, rows, want_sel, sm_scale)
    assert_attn_close(d.out.float().cpu().numpy(), want, f"sm_scale={sm_scale}")
    assert np.abs(d.lse.cpu().numpy() - want_lse).max() <= LSE_ABS
    _check_no_device_error(lib, d)


def test_cuda_graph_replay_matches_eager(lib):
    # the entry points allocate nothing and never synchronise, so a whole
    # layer step (indexer, sparse attention with both tile paths, and a
    # sliding-window call) captures into a CUDA graph and replays to the same
    # bits as eager calls
    w = S.Workload(ctx=[5003, 9000, 300, 3000], nq=[1, 2, 1, 8], seed=27)
    d = DeviceInputs(w, lib)
    out_swa, lse_swa = torch.empty_like(d.out), torch.empty_like(d.lse)

    def step():
        _run_index(lib, d)
        _run_sparse(lib, d)
        lib.s5_swa_gqa_attn(d.k_pool, d.v_pool, d.batch, d.q, S.WINDOW, O.DEFAULT_SM_SCALE, out_swa, lse_swa, d.ws)

    results = (d.sel, d.sel_count, d.out, d.lse, out_swa, lse_swa)
    step()
    torch.cuda.synchronize()
    eager = [t.clone() for t in results]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for t in results:
        t.zero_()
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    for a, b in zip(eager, results):
        assert torch.equal(a, b)
    _check_no_device_error(lib, d)


@pytest.mark.parametrize("topk", [1, 64, 300])
def test_smaller_topk_both_paths(lib, topk):
    # k below 512: decode rows, a verify group and an 8-token chunk (tile
    # path candidates), histories below and above k blocks
    w = S.Workload(ctx=[5, 700, 3000, 9000, 12000], nq=[1, 1, 4, 1, 8], seed=47)
    d = DeviceInputs(w, lib)
    sel = torch.full((w.total_q, topk), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((w.total_q,), -7, dtype=torch.int32, device="cuda")
    lib.s5_index_score_topk(d.key_pool, d.batch, d.qx, topk, sel, cnt, d.ws)
    lib.s5_sparse_gqa_attn(d.k_pool, d.v_pool, d.batch, d.q, sel, cnt, topk, O.DEFAULT_SM_SCALE, d.out, d.lse, d.ws)
    torch.cuda.synchronize()
    _check_no_device_error(lib, d)
    rows = list(range(w.total_q))
    want = oracle_selection(w, rows, topk)
    assert np.array_equal(sel.cpu().numpy(), want)
    assert np.array_equal(cnt.cpu().numpy(), [O.selection_count(x) for x in want])
    _check_sparse_out(d, rows, want, f"topk {topk}")
