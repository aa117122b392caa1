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


class DeviceInputs:
    """Everything the CUDA path needs for one layer, resident on the device.

    ``draw`` is where the generator runs (default: on ``device``; "cpu" draws
    on the host and copies the tensors over once)."""

    def __init__(self, w: S.Workload, s5, device="cuda", window_only=None, with_index=True, draw=None):
        self.w = w
        self.pt = w.page_table()
        draw = device if draw is None else draw
        k_pool, v_pool = w.kv_pools(draw, self.pt, window_only=window_only)
        self.k_pool, self.v_pool = k_pool.to(device), v_pool.to(device)
        self.key_pool = w.index_pool(draw, self.pt).to(device) if with_index else None
        q, qx = w.queries(draw)
        self.q, self.qx = q.to(device), qx.to(device)
        self.batch = s5.Batch.from_host(self.pt, w.ctx, w.nq, device)
        self.ws = s5.new_workspace(self.batch, window=S.WINDOW, device=device)
        tq = w.total_q
        self.sel = torch.full((tq, S.TOPK), -7, dtype=torch.int32, device=device)
        self.sel_count = torch.full((tq,), -7, dtype=torch.int32, device=device)
        self.out = torch.full((tq, 64, 192), float("nan"), dtype=torch.bfloat16, device=device)
        self.lse = torch.full((tq, 64), float("nan"), dtype=torch.float32, device=device)


def seq_keys(w: S.Workload, s: int, n_blocks: int, fp8: bool = False, chunk: int = 16384) -> np.ndarray:
    """Block keys 0 .. n_blocks-1 of sequence s as float64 [n_blocks][256], drawn
    once on the CPU (with ``fp8``: the exact E4M3 value of each stored byte)."""
    out = np.empty((n_blocks, S.INDEX_DIM), dtype=np.float64)
    for b0 in range(0, n_blocks, chunk):
        b = torch.arange(b0, min(n_blocks, b0 + chunk), dtype=torch.int64)
        if fp8:
            out[b0:b0 + len(b)] = O.decode_e4m3(w.kx_blocks(s, b, fp8=True).numpy())
        else:
            out[b0:b0 + len(b)] = w.kx_blocks(s, b).double().numpy()
    return out


def oracle_selection(w: S.Workload, rows, topk=S.TOPK, qx=None, fp8=False, chunk=1024):
    """Oracle selections [len(rows)][topk] of the given query rows.

    ``qx`` [len(rows)][256] overrides the workload's indexer queries (one
    per row).  Each sequence's keys are drawn once and all of its rows are
    selected against them."""
    rows = list(rows)
    seqs, pos = w.query_seq_pos()
    if qx is None:
        qx = w.qx_rows(torch.as_tensor(rows, dtype=torch.int64)).double().numpy()
    qx = np.asarray(qx, dtype=np.float64)
    out = np.full((len(rows), topk), -1, dtype=np.int64)
    by_seq = {}
    for i, r in enumerate(rows):
        by_seq.setdefault(seqs[r], []).append(i)
    for s, idx in by_seq.items():
        idx = np.array(idx)
        p = np.array([pos[rows[i]] for i in idx], dtype=np.int64)
        c_max = int((p // S.BLOCK).max())
        keys = seq_keys(w, s, c_max, fp8) if c_max > topk else np.zeros((0, S.INDEX_DIM))
        for k in range(0, len(idx), chunk):
            part = idx[k:k + chunk]
            out[part] = O.index_topk_rows(qx[part], keys, p[k:k + chunk], topk)
    return out


def oracle_selection_grouped(w: S.Workload, rows, topk=S.TOPK):
    """Per-KV-group oracle selections [len(rows)][4][topk]: each (row, group)
    pair is selected from that group's indexer query."""
    rows = list(rows)
    qx = w.qx_group_rows(torch.as_tensor(rows, dtype=torch.int64)).double().numpy()
    flat = [r for r in rows for _ in range(S.N_KV)]  # row-major, group-minor, as qx
    return oracle_selection(w, flat, topk, qx=qx.reshape(-1, S.INDEX_DIM)).reshape(len(rows), S.N_KV, topk)


def check_all_selections(w: S.Workload, sel_dev, cnt_dev, topk=S.TOPK, fp8=False):
    """Every row's selection and count against the oracle, bit for bit."""
    rows = list(range(w.total_q))
    want = oracle_selection(w, rows, topk, fp8=fp8)
    got = sel_dev.cpu().numpy()
    cnt = cnt_dev.cpu().numpy()
    bad = np.nonzero(~np.all(got == want, axis=1))[0]
    assert bad.size == 0, f"{bad.size} of {len(rows)} rows differ, first {bad[:8].tolist()}"
    assert np.array_equal(cnt, (want >= 0).sum(axis=1)), "selection counts differ"
    return want


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
