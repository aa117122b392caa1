"""Shared test plumbing: seeded inputs for both sides, oracle wrappers, tolerances.

The device side gets paged pools built by the generator module; the oracle
gets logical values drawn from the same counters, on the CPU.  Nothing here
holds attention or indexer arithmetic.
"""
import numpy as np
import torch

from block_sparse_gqa_indexer_b200 import synth as S
from oracle import s5_oracle as O

# bf16 attention outputs against the float64 oracle
MAX_ABS = 2e-2
REL_RMS = 5e-3
LSE_ABS = 1e-3


class LazyRows:
    """Numpy-style fancy indexing over the K or V rows of one sequence, drawn on demand."""

    def __init__(self, w: S.Workload, s: int, which: str):
        self.w, self.s, self.which = w, s, which

    def __getitem__(self, pos):
        pos = torch.as_tensor(np.asarray(pos, dtype=np.int64))
        f = self.w.k_tokens if self.which == "k" else self.w.v_tokens
        return f(self.s, pos).double().numpy()


class LazyKeys:
    def __init__(self, w: S.Workload, s: int):
        self.w, self.s = w, s

    def __getitem__(self, blocks):
        b = torch.as_tensor(np.asarray(blocks, dtype=np.int64))
        return self.w.kx_blocks(self.s, b).double().numpy()


class DeviceInputs:
    """Everything the CUDA path needs for one layer, resident on the device."""

    def __init__(self, w: S.Workload, s5, device="cuda", window_only=None, with_index=True):
        self.w = w
        self.pt = w.page_table()
        self.k_pool, self.v_pool = w.kv_pools(device, self.pt, window_only=window_only)
        self.key_pool = w.index_pool(device, self.pt) if with_index else None
        self.q, self.qx = w.queries(device)
        self.batch = s5.Batch.from_host(self.pt, w.ctx, w.nq, device)
        self.ws = s5.new_workspace(self.batch, window=S.WINDOW, device=device)
        tq = w.total_q
        self.sel = torch.full((tq, S.TOPK), -7, dtype=torch.int32, device=device)
        self.sel_count = torch.full((tq,), -7, dtype=torch.int32, device=device)
        self.out = torch.full((tq, 64, 192), float("nan"), dtype=torch.bfloat16, device=device)
        self.lse = torch.full((tq, 64), float("nan"), dtype=torch.float32, device=device)


def oracle_selection(w: S.Workload, rows, topk=S.TOPK):
    seqs, pos = w.query_seq_pos()
    qx = w.qx_rows(torch.as_tensor(list(rows), dtype=torch.int64)).double().numpy()
    out = []
    for i, r in enumerate(rows):
        out.append(O.index_topk_query(qx[i], LazyKeys(w, seqs[r]), pos[r], topk))
    return np.array(out)


def oracle_sparse(w: S.Workload, rows, sel_rows, sm_scale=O.DEFAULT_SM_SCALE):
    seqs, pos = w.query_seq_pos()
    q = w.q_rows(torch.as_tensor(list(rows), dtype=torch.int64)).double().numpy()
    outs, lses = [], []
    for i, r in enumerate(rows):
        s = seqs[r]
        o, l = O.sparse_attention_query(q[i], sel_rows[i], pos[r], LazyRows(w, s, "k"), LazyRows(w, s, "v"),
                                        sm_scale)
        outs.append(O.round_bf16(o))
        lses.append(l)
    return np.array(outs), np.array(lses)


def oracle_swa(w: S.Workload, rows, window=S.WINDOW, sm_scale=O.DEFAULT_SM_SCALE):
    seqs, pos = w.query_seq_pos()
    q = w.q_rows(torch.as_tensor(list(rows), dtype=torch.int64)).double().numpy()
    outs, lses = [], []
    for i, r in enumerate(rows):
        s = seqs[r]
        o, l = O.swa_attention_query(q[i], pos[r], LazyRows(w, s, "k"), LazyRows(w, s, "v"), window, sm_scale)
        outs.append(O.round_bf16(o))
        lses.append(l)
    return np.array(outs), np.array(lses)


def assert_attn_close(got, want, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = got - want
    max_abs = float(np.abs(err).max())
    rel_rms = float(np.sqrt((err ** 2).sum() / max((want ** 2).sum(), 1e-300)))
    assert max_abs <= MAX_ABS and rel_rms <= REL_RMS, f"{what}: max_abs={max_abs:.3e} rel_rms={rel_rms:.3e}"
    return max_abs, rel_rms


def sample_rows(n_rows, k, seed=0):
    """A few spread rows: first, last, and seeded picks."""
    if n_rows <= k:
        return list(range(n_rows))
    g = np.random.default_rng(seed)
    picks = set([0, n_rows - 1]) | set(g.choice(n_rows, k - 2, replace=False).tolist())
    return sorted(picks)
