"""Sparse attention over one-byte (E4M3) KV on the GPU against the CPU oracle,
through the C ABI.

The oracle decodes every stored K / V byte to its exact E4M3 value, multiplies
by the call's k_scale / v_scale and evaluates the same attention in float64.
The GPU widens the same bytes exactly, so the tolerance is the bf16 layer's
(max-abs 2e-2, rel-RMS 5e-3, lse 1e-3).  The lossy step, rounding the values
to E4M3, is measured separately against the bf16-KV oracle.
"""
import numpy as np
import pytest
import torch

from block_sparse_gqa_indexer_b200 import synth as S
from oracle import s5_oracle as O
from tests.harness import (LSE_ABS, LazyRows, assert_attn_close, check_all_selections, oracle_selection,
                           oracle_sparse, sample_rows)

pytestmark = pytest.mark.gpu


class LazyCodes:
    """Oracle view of a sequence's one-byte K or V: the stored E4M3 bytes [n][4][192]."""

    def __init__(self, w: S.Workload, s: int, which: str):
        self.w, self.s, self.which = w, s, which

    def __getitem__(self, pos):
        pos = torch.as_tensor(np.asarray(pos, dtype=np.int64))
        f = self.w.k_tokens if self.which == "k" else self.w.v_tokens
        return S.to_e4m3_codes(f(self.s, pos)).numpy()


class Fp8Inputs:
    def __init__(self, w: S.Workload, lib):
        self.w = w
        self.pt = w.page_table()
        self.k8, self.v8 = w.kv_pools("cuda", self.pt, fp8=True)
        self.key_pool = w.index_pool("cuda", self.pt)
        self.q, self.qx = w.queries("cuda")
        self.batch = lib.Batch.from_host(self.pt, w.ctx, w.nq, "cuda")
        self.ws = lib.new_workspace(self.batch, window=S.WINDOW, device="cuda")
        tq = w.total_q
        self.sel = torch.full((tq, S.TOPK), -7, dtype=torch.int32, device="cuda")
        self.cnt = torch.full((tq,), -7, dtype=torch.int32, device="cuda")
        self.out = torch.full((tq, 64, 192), float("nan"), dtype=torch.bfloat16, device="cuda")
        self.lse = torch.full((tq, 64), float("nan"), dtype=torch.float32, device="cuda")

    def run(self, lib, k_scale=1.0, v_scale=1.0, sm_scale=O.DEFAULT_SM_SCALE, sel=None):
        lib.s5_index_score_topk(self.key_pool, self.batch, self.qx, S.TOPK, self.sel, self.cnt, self.ws)
        lib.s5_sparse_gqa_attn_fp8kv(self.k8, self.v8, self.batch, self.q, self.sel if sel is None else sel,
                                     self.cnt, S.TOPK, sm_scale, k_scale, v_scale, self.out, self.lse, self.ws)
        torch.cuda.synchronize()
        code, info = lib.s5_get_device_error(self.ws)
        assert code == 0, (lib.s5_status_string(code), info)


def oracle_fp8kv(w, rows, sel_rows, k_scale, v_scale, sm_scale=O.DEFAULT_SM_SCALE):
    seqs, pos = w.query_seq_pos()
    q = w.q_rows(torch.as_tensor(list(rows), dtype=torch.int64)).double().numpy()
    outs, lses = [], []
    for i, r in enumerate(rows):
        s = seqs[r]
        o, l = O.sparse_attention_query_fp8kv(q[i], sel_rows[i], pos[r], LazyCodes(w, s, "k"), LazyCodes(w, s, "v"),
                                              k_scale, v_scale, sm_scale)
        outs.append(O.round_bf16(o))
        lses.append(l)
    return np.array(outs), np.array(lses)


def _check(d: Fp8Inputs, rows, sel_rows, k_scale, v_scale, what, sm_scale=O.DEFAULT_SM_SCALE):
    want, want_lse = oracle_fp8kv(d.w, rows, sel_rows, k_scale, v_scale, sm_scale)
    got = d.out.float().cpu().numpy()[rows]
    assert_attn_close(got, want, what)
    assert np.abs(d.lse.cpu().numpy()[rows] - want_lse).max() <= LSE_ABS


@pytest.mark.parametrize("ctx,nq", [
    ([0, 5, 7, 8, 100], [1, 1, 1, 1, 1]),              # tiny histories, partial current blocks
    ([4095, 4096, 4103, 4104, 4111], [1, 1, 1, 1, 1]),  # history at the 512-block edge
    ([6000, 9999, 20001], [1, 1, 1]),
    ([5000, 4090, 12345], [4, 4, 4]),                  # verify rows (all on the per-row kernel)
    ([3, 4200, 777, 16383, 9000], [2, 3, 1, 4, 0]),    # varlen, an empty sequence
])
@pytest.mark.parametrize("k_scale,v_scale", [(1.0, 1.0), (0.37, 1.9)])
def test_fp8kv_small_all_rows(lib, ctx, nq, k_scale, v_scale):
    d = Fp8Inputs(S.Workload(ctx=ctx, nq=nq, seed=61), lib)
    d.run(lib, k_scale, v_scale)
    rows = list(range(d.w.total_q))
    want_sel = check_all_selections(d.w, d.sel, d.cnt)
    _check(d, rows, want_sel, k_scale, v_scale, f"fp8 kv ctx={ctx} nq={nq} scales={k_scale},{v_scale}")


def test_fp8kv_block_order_invariance_and_repeatability(lib):
    d = Fp8Inputs(S.Workload(ctx=[30000, 7777], nq=[1, 2], seed=62), lib)
    d.run(lib)
    ref = d.out.clone()
    d.run(lib)
    assert torch.equal(ref, d.out)  # bit-identical repeat
    g = torch.Generator().manual_seed(5)
    sel = d.sel.cpu()
    perm = sel.clone()
    for r in range(sel.shape[0]):
        n = int(d.cnt[r])
        perm[r, :n] = sel[r, :n][torch.randperm(n, generator=g)]
    d.run(lib, sel=perm.cuda())
    assert_attn_close(d.out.float().cpu().numpy(), ref.float().cpu().numpy(), "permuted selection")


def test_fp8kv_host_validation(lib):
    d = Fp8Inputs(S.Workload(ctx=[100], nq=[1], seed=63), lib)
    for ks, vs in [(float("nan"), 1.0), (1.0, float("inf")), (1e38, 1.0)]:
        with pytest.raises(lib.S5Error) as e:
            lib.s5_sparse_gqa_attn_fp8kv(d.k8, d.v8, d.batch, d.q, d.sel, d.cnt, S.TOPK, 1e3, ks, vs, d.out, d.lse,
                                         d.ws)
        assert e.value.code == lib.S5_ERR_INVALID_ARG


@pytest.mark.slow
def test_fp8kv_headline_decode_b64_128k(lib):
    (w,) = S.config_workloads(0)
    d = Fp8Inputs(w, lib)
    d.run(lib, 1.0, 1.0)
    rows = sample_rows(w.total_q, 6, 7)
    want_sel = oracle_selection(w, rows)
    assert np.array_equal(d.sel.cpu().numpy()[rows], want_sel)
    _check(d, rows, want_sel, 1.0, 1.0, "fp8 kv headline")


def test_fp8kv_accuracy_against_bf16_kv(lib):
    # the lossy step: E4M3 storage of ~N(0,1) K/V against the bf16 layer on the
    # unrounded values.  E4M3 keeps 3 mantissa bits (relative rounding error
    # <= 2^-4); both the weights and the averaged values move by a few percent,
    # so the output is bounded here at 10% relative RMS (measured: about 5%)
    w = S.Workload(ctx=[20000, 60000, 131072], nq=[1, 1, 1], seed=64)
    d = Fp8Inputs(w, lib)
    d.run(lib)
    rows = list(range(w.total_q))
    want_sel = oracle_selection(w, rows)
    want_bf16, _ = oracle_sparse(w, rows, want_sel)
    got = d.out.float().cpu().numpy()
    err = got - want_bf16
    rel_rms = float(np.sqrt((err ** 2).sum() / (want_bf16 ** 2).sum()))
    print(f"fp8 KV vs bf16 KV: max_abs={np.abs(err).max():.3e} rel_rms={rel_rms:.3e}")
    assert rel_rms < 0.10


# ---------------------------------------------------------------- the one-byte cache append

def _fp8_append_inputs(lib, w):
    pt = w.page_table()
    k0, v0 = w.kv_pools("cuda", pt, upto=w.ctx, fp8=True)
    x0 = w.index_pool("cuda", pt, upto=w.ctx)
    kn, vn, xn = w.new_tokens("cuda")
    batch = lib.Batch.from_host(pt, w.ctx, w.nq, "cuda")
    ws = lib.new_workspace(batch)
    return pt, k0, v0, x0, kn, vn, xn, batch, ws


@pytest.mark.parametrize("ctx,nq", [
    ([60, 5000, 0, 130], [9, 3, 70, 1]),   # page and block edges on both sides, a fresh sequence
    ([131072, 7, 4095], [1, 4, 2]),        # decode / verify rows
    ([2000], [300]),                       # a prefill chunk
])
def test_fp8_append_matches_the_oracle_and_the_generator(lib, ctx, nq):
    w = S.Workload(ctx=ctx, nq=nq, seed=65)
    pt, k0, v0, x0, kn, vn, xn, batch, ws = _fp8_append_inputs(lib, w)
    # unit scales: the codes the generator draws for the whole batch
    k1, v1, x1 = k0.clone(), v0.clone(), x0.clone()
    lib.s5_append_kv_fp8(k1, v1, x1, batch, kn, vn, xn, 1.0, 1.0, ws)
    torch.cuda.synchronize()
    code, info = lib.s5_get_device_error(ws)
    assert code == 0, (lib.s5_status_string(code), info)
    kw, vw = w.kv_pools("cuda", pt, fp8=True)
    assert torch.equal(k1, kw) and torch.equal(v1, vw)
    assert torch.equal(x1, w.index_pool("cuda", pt))
    # other scales: the oracle's codes of x * fl32(1 / scale), bit for bit
    if w.num_pages <= 4096:
        k2, v2, x2 = k0.clone(), v0.clone(), x0.clone()
        lib.s5_append_kv_fp8(k2, v2, x2, batch, kn, vn, xn, 0.37, 1.9, ws)
        torch.cuda.synchronize()
        ko, vo, xo = O.append_to_paged_cache_fp8(k0.cpu().numpy(), v0.cpu().numpy(), x0.double().cpu().numpy(),
                                                 pt.numpy(), w.ctx, w.nq, kn.double().cpu().numpy(),
                                                 vn.double().cpu().numpy(), xn.double().cpu().numpy(), 0.37, 1.9)
        assert np.array_equal(k2.cpu().numpy(), ko) and np.array_equal(v2.cpu().numpy(), vo)
        assert np.array_equal(x2.double().cpu().numpy(), xo)


def test_fp8_append_reports_an_unmapped_page(lib):
    w = S.Workload(ctx=[100, 700], nq=[2, 1], seed=66)
    pt, k0, v0, x0, kn, vn, xn, batch, ws = _fp8_append_inputs(lib, w)
    batch.page_table[1, 700 // 64] = -1
    lib.s5_reset_device_error(ws)
    lib.s5_append_kv_fp8(k0, v0, None, batch, kn, vn, None, 1.0, 1.0, ws)
    code, info = lib.s5_get_device_error(ws)
    assert code == lib.S5_ERR_DEVICE_BOUNDS and info == 2


def test_fp8_append_then_attend_matches_the_oracle(lib):
    # one decode / verify step on a one-byte cache: append (scales 0.5, 2),
    # score and select, attend with the same scales
    w = S.Workload(ctx=[9000, 20000, 300], nq=[1, 4, 2], seed=67)
    pt, k0, v0, x0, kn, vn, xn, batch, ws = _fp8_append_inputs(lib, w)
    ks, vs = 0.5, 2.0
    lib.s5_append_kv_fp8(k0, v0, x0, batch, kn, vn, xn, ks, vs, ws)
    _, qx = w.queries("cuda")
    q = w.q_rows(torch.arange(w.total_q), "cuda")
    sel = torch.empty((w.total_q, S.TOPK), dtype=torch.int32, device="cuda")
    cnt = torch.empty((w.total_q,), dtype=torch.int32, device="cuda")
    out = torch.empty((w.total_q, 64, 192), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.total_q, 64), dtype=torch.float32, device="cuda")
    lib.s5_index_score_topk(x0, batch, qx, S.TOPK, sel, cnt, ws)
    lib.s5_sparse_gqa_attn_fp8kv(k0, v0, batch, q, sel, cnt, S.TOPK, O.DEFAULT_SM_SCALE, ks, vs, out, lse, ws)
    torch.cuda.synchronize()
    code, info = lib.s5_get_device_error(ws)
    assert code == 0, (lib.s5_status_string(code), info)
    rows = list(range(w.total_q))
    want_sel = oracle_selection(w, rows)
    assert np.array_equal(sel.cpu().numpy(), want_sel)
    # the oracle reads the codes its own append stores: cached tokens carry the
    # generator's unit-scale codes, new tokens the scaled ones
    seqs, pos = w.query_seq_pos()
    new_at = {(seqs[r], pos[r]): r for r in rows}
    kn_np, vn_np = kn.double().cpu().numpy(), vn.double().cpu().numpy()

    class Codes:
        def __init__(self, s, which):
            self.s, self.which = s, which

        def __getitem__(self, ps):
            ps = np.asarray(ps, dtype=np.int64)
            f = w.k_tokens if self.which == "k" else w.v_tokens
            out_c = S.to_e4m3_codes(f(self.s, torch.as_tensor(ps))).numpy()
            for i, p in enumerate(ps.tolist()):
                if (self.s, p) in new_at:
                    x = (kn_np if self.which == "k" else vn_np)[new_at[(self.s, p)]]
                    out_c[i] = O.quantize_kv_e4m3(x, ks if self.which == "k" else vs)
            return out_c

    q_np = q.double().cpu().numpy()
    want, want_l = [], []
    for r in rows:
        s = seqs[r]
        o, l = O.sparse_attention_query_fp8kv(q_np[r], want_sel[r], pos[r], Codes(s, "k"), Codes(s, "v"), ks, vs)
        want.append(O.round_bf16(o))
        want_l.append(l)
    assert_attn_close(out.float().cpu().numpy(), np.array(want), "append then attend, one-byte KV")
    assert np.abs(lse.cpu().numpy() - np.array(want_l)).max() <= LSE_ABS
