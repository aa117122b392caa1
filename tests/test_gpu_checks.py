"""GPU checks beside parity: no write lands outside an output, a verify row
agrees with the same row computed as a single-token decode, and a bounded
wait that runs out is reported and leaves the library usable.

Canary guards stand in for a memory checker: every output (out, lse, sel,
sel_count, and the pools the cache append writes) sits inside a larger byte
buffer whose margins are filled with a sentinel, and the margins must be
unchanged after the call.
"""
import numpy as np
import pytest
import torch

from block_sparse_gqa_indexer_b200 import synth as S
from oracle import s5_oracle as O
from tests.harness import (LSE_ABS, MAX_ABS, REL_RMS, DeviceInputs, assert_attn_close, oracle_selection,
                           oracle_sparse, sample_rows)

pytestmark = pytest.mark.gpu

GUARD = 4096  # bytes of sentinel on each side
SENTINEL = 0xA5


class Guarded:
    """A tensor of `shape` / `dtype` inside a byte buffer with sentinel margins."""

    def __init__(self, shape, dtype, device="cuda"):
        n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        self.n = n
        self.flat = torch.full((n + 2 * GUARD,), SENTINEL, dtype=torch.uint8, device=device)
        self.t = self.flat[GUARD:GUARD + n].view(dtype).view(shape)

    def intact(self) -> bool:
        return bool((self.flat[:GUARD] == SENTINEL).all()) and bool((self.flat[GUARD + self.n:] == SENTINEL).all())


def _no_error(lib, ws):
    code, info = lib.s5_get_device_error(ws)
    assert code == 0, (lib.s5_status_string(code), info)


def _guarded_outputs(w, topk=S.TOPK):
    return (Guarded((w.total_q, topk), torch.int32), Guarded((w.total_q,), torch.int32),
            Guarded((w.total_q, 64, 192), torch.bfloat16), Guarded((w.total_q, 64), torch.float32))


@pytest.mark.parametrize("ctx,nq,coherent", [
    ([20000, 300, 9000], [1, 1, 1], 0),           # decode rows, partitions merged in the kernel
    ([5000, 4090, 12345], [4, 4, 4], 0),          # verify rows: union kernel, per-row kernel
    ([20000, 3000], [16, 9], 64),                 # shared-set tiles on the tensor cores (+ a ragged tile)
    ([3000, 70000], [100, 70], 0),                # tensor-core indexer GEMM; tiles of both kinds
    ([140000, 9000], [1, 2], 0),                  # two-stage select beyond 16,384 blocks
])
def test_sparse_outputs_stay_inside_their_buffers(lib, ctx, nq, coherent):
    w = S.Workload(ctx=ctx, nq=nq, seed=71, qx_coherent=coherent)
    d = DeviceInputs(w, lib)
    sel, cnt, out, lse = _guarded_outputs(w)
    lib.s5_index_score_topk(d.key_pool, d.batch, d.qx, S.TOPK, sel.t, cnt.t, d.ws)
    lib.s5_sparse_gqa_attn(d.k_pool, d.v_pool, d.batch, d.q, sel.t, cnt.t, S.TOPK, O.DEFAULT_SM_SCALE, out.t,
                           lse.t, d.ws)
    torch.cuda.synchronize()
    _no_error(lib, d.ws)
    for name, g in (("sel", sel), ("sel_count", cnt), ("out", out), ("lse", lse)):
        assert g.intact(), f"a write landed outside {name}"
    # and the guarded buffers hold the same results as plain ones
    lib.s5_index_score_topk(d.key_pool, d.batch, d.qx, S.TOPK, d.sel, d.sel_count, d.ws)
    lib.s5_sparse_gqa_attn(d.k_pool, d.v_pool, d.batch, d.q, d.sel, d.sel_count, S.TOPK, O.DEFAULT_SM_SCALE,
                           d.out, d.lse, d.ws)
    torch.cuda.synchronize()
    assert torch.equal(sel.t, d.sel) and torch.equal(cnt.t, d.sel_count)
    assert torch.equal(out.t, d.out) and torch.equal(lse.t, d.lse)


def test_swa_standalone_merge_stays_inside(lib):
    # > 1,024 rows with two partitions each: the standalone merge kernel writes out / lse
    w = S.Workload(ctx=[8000], nq=[1100], seed=72)
    d = DeviceInputs(w, lib, with_index=False)
    ws = lib.new_workspace(d.batch, window=8192)
    _, _, out, lse = _guarded_outputs(w)
    lib.s5_swa_gqa_attn(d.k_pool, d.v_pool, d.batch, d.q, 8192, O.DEFAULT_SM_SCALE, out.t, lse.t, ws)
    torch.cuda.synchronize()
    _no_error(lib, ws)
    assert out.intact() and lse.intact()


def test_fp8kv_and_grouped_outputs_stay_inside(lib):
    w = S.Workload(ctx=[20000, 300, 9000], nq=[1, 4, 1], seed=73)
    d = DeviceInputs(w, lib)
    _, _, out, lse = _guarded_outputs(w)
    lib.s5_index_score_topk(d.key_pool, d.batch, d.qx, S.TOPK, d.sel, d.sel_count, d.ws)
    k8, v8 = w.kv_pools("cuda", d.pt, fp8=True)
    lib.s5_sparse_gqa_attn_fp8kv(k8, v8, d.batch, d.q, d.sel, d.sel_count, S.TOPK, O.DEFAULT_SM_SCALE, 1.0, 1.0,
                                 out.t, lse.t, d.ws)
    torch.cuda.synchronize()
    _no_error(lib, d.ws)
    assert out.intact() and lse.intact()
    # grouped: selections [total_q][4][topk], attention per group
    wsg = lib.new_workspace(d.batch, window=S.WINDOW, grouped=True)
    qxg = w.qx_group_rows(torch.arange(w.total_q), "cuda").contiguous()
    selg = Guarded((w.total_q, 4, S.TOPK), torch.int32)
    cntg = Guarded((w.total_q, 4), torch.int32)
    _, _, out2, lse2 = _guarded_outputs(w)
    lib.s5_index_score_topk_grouped(d.key_pool, d.batch, qxg, S.TOPK, selg.t, cntg.t, wsg)
    lib.s5_sparse_gqa_attn_grouped(d.k_pool, d.v_pool, d.batch, d.q, selg.t, cntg.t, S.TOPK, O.DEFAULT_SM_SCALE,
                                   out2.t, lse2.t, wsg)
    torch.cuda.synchronize()
    _no_error(lib, wsg)
    assert selg.intact() and cntg.intact() and out2.intact() and lse2.intact()


def test_append_writes_stay_inside_the_pools(lib):
    # pools with a guard page on each side: the append may write only the pages of the pool
    w = S.Workload(ctx=[60, 5000, 0, 130], nq=[9, 3, 70, 1], seed=74)
    pt = w.page_table()
    n = w.num_pages
    k_full = torch.full((n + 2, 4, 64, 192), -3.0, dtype=torch.bfloat16, device="cuda")
    v_full = torch.full_like(k_full, -3.0)
    x_full = torch.full((n + 2, 8, 256), -3.0, dtype=torch.bfloat16, device="cuda")
    kp, vp, xp = k_full[1:n + 1], v_full[1:n + 1], x_full[1:n + 1]
    kp.copy_(w.kv_pools("cuda", pt, upto=w.ctx)[0])
    vp.copy_(w.kv_pools("cuda", pt, upto=w.ctx)[1])
    xp.copy_(w.index_pool("cuda", pt, upto=w.ctx))
    batch = lib.Batch.from_host(pt, w.ctx, w.nq, "cuda")
    ws = lib.new_workspace(batch)
    kn, vn, xn = w.new_tokens("cuda")
    lib.s5_append_kv(kp, vp, xp, batch, kn, vn, xn, ws)
    torch.cuda.synchronize()
    _no_error(lib, ws)
    for full in (k_full, v_full, x_full):
        assert bool((full[0] == -3.0).all()) and bool((full[n + 1] == -3.0).all()), "a write left the pool"
    k_want, v_want = w.kv_pools("cuda", pt)
    assert torch.equal(kp, k_want) and torch.equal(vp, v_want) and torch.equal(xp, w.index_pool("cuda", pt))


def test_verify_rows_match_single_token_decode(lib):
    # verify tiles of 8 rows with block-coherent indexer queries take the
    # shared-set tensor-core path; the same rows, each run as a one-token
    # decode with the same selection and position, take the per-row kernel
    w = S.Workload(ctx=[9000, 20000, 4000], nq=[8, 8, 8], seed=75, qx_coherent=64)
    d = DeviceInputs(w, lib)
    lib.s5_index_score_topk(d.key_pool, d.batch, d.qx, S.TOPK, d.sel, d.sel_count, d.ws)
    lib.s5_sparse_gqa_attn(d.k_pool, d.v_pool, d.batch, d.q, d.sel, d.sel_count, S.TOPK, O.DEFAULT_SM_SCALE,
                           d.out, d.lse, d.ws)
    torch.cuda.synchronize()
    _no_error(lib, d.ws)
    seqs, pos = w.query_seq_pos()
    sel = d.sel.cpu().numpy()
    # the tiles really take the shared set (union <= 70% of the rows' blocks)
    shared = 0
    for s in range(w.batch):
        rows = range(w.cu_q[s], w.cu_q[s + 1])
        union, total = set(), 0
        for r in rows:
            b = set(int(x) for x in sel[r] if x >= 0) | {pos[r] // 8}
            union |= b
            total += len(b)
        shared += 100 * len(union) <= 70 * total
    assert shared == w.batch
    # one single-token sequence per verify row: same pages, cached = t, one query
    pt_rows = d.pt[torch.as_tensor(seqs)]
    one = lib.Batch.from_host(pt_rows, pos, [1] * w.total_q, "cuda")
    ws1 = lib.new_workspace(one)
    out1 = torch.empty_like(d.out)
    lse1 = torch.empty_like(d.lse)
    lib.s5_sparse_gqa_attn(d.k_pool, d.v_pool, one, d.q, d.sel, d.sel_count, S.TOPK, O.DEFAULT_SM_SCALE, out1,
                           lse1, ws1)
    torch.cuda.synchronize()
    _no_error(lib, ws1)
    a, b = d.out.float().cpu().numpy(), out1.float().cpu().numpy()
    diff = np.abs(a - b)
    print(f"verify (tensor-core tiles) vs single-token decode (per-row kernel): bit-equal elements "
          f"{float((diff == 0).mean()):.4f}, max_abs={diff.max():.3e}, "
          f"lse max_abs={float((d.lse - lse1).abs().max()):.3e}")
    # not bit-exact (different tiles, accumulation orders and rescaling), so
    # each must match the other within the attention tolerance
    assert_attn_close(a, b, "verify vs decode")
    assert float((d.lse - lse1).abs().max()) <= LSE_ABS


@pytest.mark.parametrize("wide", [False, True])
@pytest.mark.parametrize("fp8", [False, True])
def test_expired_wait_is_reported_and_the_next_call_succeeds(lib, fp8, wide):
    # the workspace's test hook makes every attention CTA's first block wait
    # also wait 200 us on a barrier nothing arrives on: the kernel records
    # S5_ERR_TIMEOUT, drains its copies in flight and returns.  Three rows
    # launch fewer CTAs than there are SMs (the deeper-ring variant); forty
    # rows launch more (the default variant).
    if wide:
        w = S.Workload(ctx=[5000 + 97 * i for i in range(40)], nq=[1] * 40, seed=77)
    else:
        w = S.Workload(ctx=[20000, 9000, 300], nq=[1, 1, 1], seed=76)
    d = DeviceInputs(w, lib)
    lib.s5_index_score_topk(d.key_pool, d.batch, d.qx, S.TOPK, d.sel, d.sel_count, d.ws)
    if fp8:
        k_pool, v_pool = w.kv_pools("cuda", d.pt, fp8=True)

    def attend():
        if fp8:
            lib.s5_sparse_gqa_attn_fp8kv(k_pool, v_pool, d.batch, d.q, d.sel, d.sel_count, S.TOPK,
                                         O.DEFAULT_SM_SCALE, 1.0, 1.0, d.out, d.lse, d.ws)
        else:
            lib.s5_sparse_gqa_attn(d.k_pool, d.v_pool, d.batch, d.q, d.sel, d.sel_count, S.TOPK,
                                   O.DEFAULT_SM_SCALE, d.out, d.lse, d.ws)

    torch.cuda.synchronize()
    _no_error(lib, d.ws)
    off = lib.S5_WS_TEST_STALL_OFFSET
    d.ws[off:off + 8] = torch.tensor([200_000], dtype=torch.int64).view(torch.uint8).to(d.ws.device)
    attend()
    code, info = lib.s5_get_device_error(d.ws)
    assert code == lib.S5_ERR_TIMEOUT, lib.s5_status_string(code)
    assert 0 <= info < w.total_q
    # the context stays usable: clear the hook and the record, run again
    lib.s5_reset_device_error(d.ws)
    attend()
    torch.cuda.synchronize()
    _no_error(lib, d.ws)
    rows = list(range(w.total_q))
    want_sel = oracle_selection(w, rows)
    if fp8:
        from tests.test_gpu_fp8kv import oracle_fp8kv
        want, want_lse = oracle_fp8kv(w, rows, want_sel, 1.0, 1.0)
    else:
        want, want_lse = oracle_sparse(w, rows, want_sel)
    assert_attn_close(d.out.float().cpu().numpy(), want, "after an expired wait")
    assert np.abs(d.lse.cpu().numpy() - want_lse).max() <= LSE_ABS
