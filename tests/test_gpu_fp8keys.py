"""One-byte (E4M3) block keys on the GPU against the CPU oracle, through the C ABI.

The oracle scores the exact E4M3 value of every stored key byte; with the
integer-valued keys and queries of these inputs every score is exact, so the
selections must match bit for bit, and must equal the selections made from
the same keys stored as bf16.
"""
import numpy as np
import pytest
import torch

from block_sparse_gqa_indexer_b200 import synth as S
from tests.harness import oracle_selection

pytestmark = pytest.mark.gpu


def _select(lib, w: S.Workload, fp8: bool):
    pt = w.page_table()
    pool = w.index_pool("cuda", pt, fp8=fp8)
    _, qx = w.queries("cuda")
    batch = lib.Batch.from_host(pt, w.ctx, w.nq, "cuda")
    ws = lib.new_workspace(batch, window=S.WINDOW, device="cuda")
    sel = torch.full((w.total_q, S.TOPK), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((w.total_q,), -7, dtype=torch.int32, device="cuda")
    f = lib.s5_index_score_topk_fp8 if fp8 else lib.s5_index_score_topk
    f(pool, batch, qx, S.TOPK, sel, cnt, ws)
    code, info = lib.s5_get_device_error(ws)
    assert code == 0, (lib.s5_status_string(code), info)
    return sel.cpu().numpy(), cnt.cpu().numpy()


def _check_oracle(w, sel, cnt):
    # every row, against the oracle scoring the exact E4M3 value of each stored key byte
    want = oracle_selection(w, range(w.total_q), fp8=True)
    bad = np.nonzero(~np.all(sel == want, axis=1))[0]
    assert bad.size == 0, f"{bad.size} rows differ, first {bad[:8].tolist()}"
    assert np.array_equal(cnt, (want >= 0).sum(axis=1))


@pytest.mark.parametrize("ctx,nq", [
    ([0, 5, 4095, 4104, 6000, 20001], [1, 1, 1, 1, 1, 1]),   # below / at / above 512 blocks
    ([5000, 4090, 12345], [4, 4, 4]),                         # verify
    ([3, 4200, 777, 16383, 9000], [2, 3, 1, 4, 0]),           # varlen, an empty sequence
    ([9000, 6007], [100, 70]),                                # prefill-sized: keys widened for the GEMM
    ([140000, 9000], [1, 2]),                                 # beyond 16,384 blocks: segment + merge
])
def test_fp8_keys_select_like_the_oracle(lib, ctx, nq):
    w = S.Workload(ctx=ctx, nq=nq, seed=51)
    sel, cnt = _select(lib, w, fp8=True)
    _check_oracle(w, sel, cnt)
    sel2, cnt2 = _select(lib, w, fp8=False)
    assert np.array_equal(sel, sel2) and np.array_equal(cnt, cnt2)


@pytest.mark.slow
def test_fp8_keys_headline_decode_b64_128k(lib):
    (w,) = S.config_workloads(0)
    sel, cnt = _select(lib, w, fp8=True)
    sel2, cnt2 = _select(lib, w, fp8=False)
    assert np.array_equal(sel, sel2) and np.array_equal(cnt, cnt2)
    _check_oracle(w, sel, cnt)
