"""CPU oracle for the Step 5 Preview sparse and sliding-window attention layers.

TEST INFRASTRUCTURE ONLY.  This module exists to check the CUDA library.  Only
the test suite, the package smoke check and the benchmark's CPU-baseline leg
may import it; the library itself never calls it and has no CPU fallback.  It
shares no code with the CUDA path: it does not import the package, and the
package does not import it.  Its inputs are plain numpy arrays (or any object
that supports numpy-style fancy indexing on the first axis, for lazily drawn
key/value rows).

Everything here is the plain definition, evaluated in float64:

* block scoring and top-512 selection: a full stable sort on the composite key
  (score descending, block index ascending);
* attention: the softmax over an explicit token set, one head at a time, with
  head h reading KV group h // 16.

Sources (the pages give prose and a configuration table, no formulas or code):

[HA]  SGLang day-0 blog "Step 5 Preview: Day-0 Inference and RL Support with
      SGLang and Miles", section "Hybrid Attention": a sliding-window layer
      attends to a 512-token window and is followed (after two more such
      layers) by a sparse layer; the sparse layer rates each 8-token block of
      history through a per-block summary, keeps no more than 512 blocks,
      and reads the tokens of those blocks as well as the tokens of the block
      that holds the query.
[KS]  same page, section "Kernels from StepFun": the indexer rates each query
      against the compressed (per-block) history held in the paged cache;
      decode cuts a long selection into partitions and combines their partial
      results.
[CFG] StepFun open-weights blog, section "What the config says": the head
      geometry (64 query heads over 4 KV groups of dimension 192), the 256-wide
      block key for each block of 8 tokens, the selection size (512 blocks,
      4,096 tokens) and the window width (512).
[SAV] same blog, section "What sparse attention does and doesn't save": every
      history block is scored; the attention side reads at most 512 selected
      blocks and the query's own block.
[GS]  SGLang day-0 blog, section "Get Started": the cache is paged, 64 tokens
      per page, and stored in bf16.

Readings taken where the pages are silent (each the plainest one):

* history of a query at absolute position t: the complete blocks 0 .. c-1 with
  c = t // 8; the current block c is always read, causally (tokens 8c .. t);
* block score = plain dot product of the 256-dim indexer query with the block
  key (no normalisation; any monotone map leaves the selection unchanged);
* selection shared by all four KV groups; ties go to the lower block index;
  selected indices are reported in ascending order, -1 padded;
* softmax scale ``sm_scale`` (1/sqrt(192) by default), natural exponent;
* the sliding window covers positions max(0, t - W + 1) .. t (the query
  included);
* outputs rounded to bf16 with round-to-nearest-even directly from float64;
* cache append: token t of a sequence lives in slot t % 64 of the page that
  holds its logical page t // 64; a block's key is stored, in slot
  (t % 64) // 8 of the same page, when its last token t (t % 8 == 7) arrives,
  since only complete blocks are ever scored.

Per-KV-group selection (the StepFun open-weights blog, section "What sparse
attention does and doesn't save", has each KV group pick its own blocks):
reading taken here, since the configuration gives a single 256-wide key per
block, the block keys are shared and the indexer query differs per group;
group g's selection is made exactly as the shared one, from group g's query,
and heads 16g .. 16g+15 attend over group g's selected blocks and the current
block.

One-byte block keys (the StepFun blog, section "What sparse attention does and
doesn't save", sizes the indexer read for keys of one or two bytes per value
without naming the one-byte format): reading taken here, the 8-bit float
E4M3 of the OCP 8-bit floating point specification (1 sign bit, 4 exponent
bits with bias 7, 3 mantissa bits, subnormals, no infinities, S.1111.111 is
NaN); a key byte stands for its exact E4M3 value and scores are then formed
as for two-byte keys.

One-byte KV for the sparse layer (the StepFun open-weights blog, section
"Fitting it on a node", notes that SGLang can hold the full-attention layers'
KV cache in FP8, a lossy format to be re-checked, and "What I'd check before
deploying it" asks for speed and accuracy with and without it; the pages name
neither the 8-bit format nor a scale): reading taken here, the same E4M3 format as the
one-byte block keys, with one scale for K and one for V per layer; a stored K
byte b stands for k_scale * E4M3(b) and a V byte for v_scale * E4M3(b), and
attention is then defined exactly as for bf16 KV on those values.

Parity status: the cache append is pinned by rebuilding the seeded pools of
a whole batch from the pools of its cached prefix;
block selection is pinned by brute force, tie cases and the
subset characterisation of top-k (the multi-row form also by brute force on
tiny inputs, by history masking and by agreement with the one-row form); the attention functions are pinned by closed
forms (one token, identical keys, two tokens), the reduction of sparse and
sliding-window attention to full causal attention, weight normalisation and
invariance to the order of the selected blocks.  The pages print no worked
numerical example, so attention values beyond these properties are pinned only
by them.
"""
from __future__ import annotations

import math

import numpy as np

N_HEADS = 64
N_KV = 4
HEADS_PER_GROUP = N_HEADS // N_KV
HEAD_DIM = 192
PAGE = 64
BLOCK = 8
INDEX_DIM = 256
TOPK = 512
WINDOW = 512
DEFAULT_SM_SCALE = 1.0 / math.sqrt(HEAD_DIM)


# ----------------------------------------------------------------------------
# rounding
# ----------------------------------------------------------------------------

def round_bf16(x) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (ties to even), returned
    as float64.  bf16 keeps 8 significant bits; rounding is done once, from
    float64, never through float32.  Finite values in the normal range only
    (attention outputs are bounded by the values they average)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                # x = m * 2**e, 0.5 <= |m| < 1
    r = np.rint(m * 256.0)            # 8 significant bits; rint rounds halves to even
    return np.ldexp(r / 256.0, e)


# ----------------------------------------------------------------------------
# indexer: block scores and top-k selection   [HA], [KS], [CFG], [SAV]
# ----------------------------------------------------------------------------

def current_block(t: int) -> int:
    """Index of the block that holds position t; blocks before it are history."""
    return t // BLOCK


def block_scores(qx, kx) -> np.ndarray:
    """score[b] = sum_d qx[d] * kx[b, d] in float64.

    Exact for the integer-valued inputs used in the parity tests (|score| is
    far below 2**53)."""
    qx = np.asarray(qx, dtype=np.float64)
    kx = np.asarray(kx, dtype=np.float64)
    return kx @ qx


def select_topk(scores, topk: int = TOPK) -> np.ndarray:
    """The ``topk`` largest scores, ties to the lower index, as ascending indices.

    With fewer than ``topk`` candidates every index is returned.  The result is
    padded with -1 to length ``topk``."""
    scores = np.asarray(scores, dtype=np.float64)
    c = scores.shape[0]
    out = np.full(topk, -1, dtype=np.int64)
    if c <= topk:
        out[:c] = np.arange(c)
        return out
    idx = np.arange(c)
    order = np.lexsort((idx, -scores))  # primary: -score ascending; secondary: index ascending
    out[:] = np.sort(order[:topk])
    return out


def index_topk_query(qx, kx_seq, t: int, topk: int = TOPK) -> np.ndarray:
    """Selection for one query at absolute position t.

    ``kx_seq[b]`` is the 256-dim key of block b of the query's sequence; only
    blocks 0 .. t//8 - 1 are scored."""
    c = current_block(t)
    if c <= topk:
        return select_topk(np.zeros(c), topk)
    return select_topk(block_scores(qx, kx_seq[np.arange(c)]), topk)


def index_topk_rows(qx_rows, kx_seq, positions, topk: int = TOPK) -> np.ndarray:
    """Selections [len(positions)][topk] of several query rows of ONE sequence.

    Row i has indexer query ``qx_rows[i]`` and absolute position
    ``positions[i]``; ``kx_seq`` is an array [>= c_max][256] of the sequence's
    block keys.  Each row's result is exactly ``index_topk_query`` of that row:
    the scores of the row's history blocks 0 .. c_i - 1 (c_i = t_i // 8), the
    stable sort on descending score (which keeps equal scores in ascending
    block order, i.e. the lower block wins a tie), the first ``topk``, reported
    ascending and -1 padded.  The scores of all rows come from one product of
    the stacked queries with the keys; blocks at or past a row's current block
    are set to -inf for that row, so they sort after every history block and a
    row with more than ``topk`` history blocks never selects one."""
    qx_rows = np.asarray(qx_rows, dtype=np.float64).reshape(-1, INDEX_DIM)
    positions = np.asarray(positions, dtype=np.int64).reshape(-1)
    n = positions.shape[0]
    out = np.full((n, topk), -1, dtype=np.int64)
    if n == 0:
        return out
    c = positions // BLOCK
    short = c <= topk
    for i in np.nonzero(short)[0]:
        out[i, :c[i]] = np.arange(c[i])
    long_rows = np.nonzero(~short)[0]
    if long_rows.size == 0:
        return out
    c_max = int(c[long_rows].max())
    kx = np.asarray(kx_seq[np.arange(c_max)], dtype=np.float64)
    scores = qx_rows[long_rows] @ kx.T                     # [rows][c_max]
    scores[np.arange(c_max)[None, :] >= c[long_rows][:, None]] = -np.inf
    order = np.argsort(-scores, axis=1, kind="stable")     # ties keep ascending block order
    out[long_rows] = np.sort(order[:, :topk], axis=1)
    return out


def selection_count(sel) -> int:
    sel = np.asarray(sel)
    return int((sel >= 0).sum())


# ----------------------------------------------------------------------------
# token sets   [HA], [SAV]
# ----------------------------------------------------------------------------

def sparse_token_set(sel, t: int) -> np.ndarray:
    """Positions read by a sparse-layer query at t: the 8 tokens of every
    selected block plus tokens 8c .. t of the current block c = t // 8."""
    sel = np.asarray(sel, dtype=np.int64)
    sel = sel[sel >= 0]
    c = current_block(t)
    hist = (sel[:, None] * BLOCK + np.arange(BLOCK)[None, :]).reshape(-1)
    cur = np.arange(c * BLOCK, t + 1)
    return np.concatenate([hist, cur])


def swa_token_set(t: int, window: int = WINDOW) -> np.ndarray:
    """Positions read by a sliding-window query at t: max(0, t - W + 1) .. t."""
    return np.arange(max(0, t - window + 1), t + 1)


# ----------------------------------------------------------------------------
# attention over an explicit token set   [HA], [CFG]
# ----------------------------------------------------------------------------

def gqa_attention(q, k_rows, v_rows, sm_scale: float = DEFAULT_SM_SCALE, return_weights: bool = False):
    """Grouped-query attention of one query token over an explicit token set.

    q        [64][192]      (head h reads KV group h // 16)
    k_rows   [n][4][192]    keys of the n tokens of the set
    v_rows   [n][4][192]    values of the same tokens
    returns  out float64 [64][192] (not rounded), lse float64 [64]
             (natural log of the softmax denominator, scores included), and,
             with ``return_weights``, the softmax weights [64][n].
    """
    q = np.asarray(q, dtype=np.float64)
    k_rows = np.asarray(k_rows, dtype=np.float64)
    v_rows = np.asarray(v_rows, dtype=np.float64)
    n = k_rows.shape[0]
    out = np.zeros((N_HEADS, HEAD_DIM))
    lse = np.full(N_HEADS, -np.inf)
    weights = np.zeros((N_HEADS, n))
    if n == 0:
        return (out, lse, weights) if return_weights else (out, lse)
    for h in range(N_HEADS):
        g = h // HEADS_PER_GROUP
        s = sm_scale * (k_rows[:, g, :] @ q[h])   # s_j = scale * q . k_j
        m = s.max()
        w = np.exp(s - m)
        l = w.sum()
        p = w / l
        out[h] = p @ v_rows[:, g, :]
        lse[h] = m + math.log(l)
        weights[h] = p
    return (out, lse, weights) if return_weights else (out, lse)


def sparse_attention_query(q, sel, t: int, k_seq, v_seq, sm_scale: float = DEFAULT_SM_SCALE):
    """Sparse-layer attention of one query at t over its selected blocks and
    current block.  ``k_seq[pos]`` / ``v_seq[pos]`` give [4][192] rows of the
    query's sequence (fancy indexing on positions)."""
    T = sparse_token_set(sel, t)
    return gqa_attention(q, k_seq[T], v_seq[T], sm_scale)


def swa_attention_query(q, t: int, k_seq, v_seq, window: int = WINDOW, sm_scale: float = DEFAULT_SM_SCALE):
    """Sliding-window attention of one query at t."""
    T = swa_token_set(t, window)
    return gqa_attention(q, k_seq[T], v_seq[T], sm_scale)


def sparse_attention_query_fp8kv(q, sel, t: int, k_codes_seq, v_codes_seq, k_scale: float, v_scale: float,
                                 sm_scale: float = DEFAULT_SM_SCALE):
    """Sparse-layer attention of one query at t over one-byte KV.

    ``k_codes_seq[pos]`` / ``v_codes_seq[pos]`` give the stored E4M3 bytes
    (uint8 [4][192]) of the query's sequence; a K byte stands for
    k_scale * E4M3(byte), a V byte for v_scale * E4M3(byte).  The token set is
    the sparse layer's (selected blocks + current block)."""
    T = sparse_token_set(sel, t)
    k_rows = float(k_scale) * decode_e4m3(k_codes_seq[T])
    v_rows = float(v_scale) * decode_e4m3(v_codes_seq[T])
    return gqa_attention(q, k_rows, v_rows, sm_scale)


# ----------------------------------------------------------------------------
# per-KV-group selection and attention; row positions of a varlen batch
# ----------------------------------------------------------------------------

def index_topk_query_grouped(qx_groups, kx_seq, t: int, topk: int = TOPK) -> np.ndarray:
    """Per-KV-group selections of one query at t: ``qx_groups`` [4][256] holds
    one indexer query per KV group; returns [4][topk] (each row as
    index_topk_query)."""
    return np.stack([index_topk_query(qx_groups[g], kx_seq, t, topk) for g in range(N_KV)])


def sparse_attention_query_grouped(q, sel_groups, t: int, k_seq, v_seq, sm_scale: float = DEFAULT_SM_SCALE):
    """Sparse-layer attention with a selection per KV group: head h (group
    g = h // 16) reads the tokens of sel_groups[g] plus the current block.
    Returns (out [64][192], lse [64])."""
    out = np.zeros((N_HEADS, HEAD_DIM))
    lse = np.zeros(N_HEADS)
    for g in range(N_KV):
        T = sparse_token_set(sel_groups[g], t)
        o, l = gqa_attention(q, k_seq[T], v_seq[T], sm_scale)
        heads = slice(g * HEADS_PER_GROUP, (g + 1) * HEADS_PER_GROUP)
        out[heads] = o[heads]
        lse[heads] = l[heads]
    return out, lse


def query_positions(ctx, nq):
    """(sequence, position) of every query row, rows ordered by sequence."""
    rows = []
    for s, (c, n) in enumerate(zip(ctx, nq)):
        for j in range(n):
            rows.append((s, c + j))
    return rows


# ----------------------------------------------------------------------------
# cache append: new tokens and completed block keys into the paged cache
# [KS], [GS], [CFG]
# ----------------------------------------------------------------------------

def append_to_paged_cache(k_pool, v_pool, key_pool, page_table, ctx, nq, k_new, v_new, key_new):
    """The paged pools after appending the new tokens of a varlen batch (copies).

    k_pool, v_pool  [num_pages][4][64][192]   K / V of page p, group g, slot i
    key_pool        [num_pages][8][256] or None (a cache without block keys)
    page_table      [batch][max_pages]        logical page -> physical page
    k_new, v_new    [total_q][4][192]         row r = token t = ctx[s] + j
    key_new         [total_q][256]            key of the block row r completes

    Token t goes to slot t % 64 of physical page page_table[s][t // 64], for
    all four groups.  If t is the last token of its block (t % 8 == 7),
    key_new[r] becomes the key of block t // 8: slot (t % 64) // 8 of that
    page.  Other rows of key_new are not read.  An unmapped page (-1) or a
    page id outside the pool raises ValueError."""
    k_out = np.array(k_pool, copy=True)
    v_out = np.array(v_pool, copy=True)
    key_out = None if key_pool is None else np.array(key_pool, copy=True)
    page_table = np.asarray(page_table)
    for r, (s, t) in enumerate(query_positions(ctx, nq)):
        logical = t // PAGE
        if logical >= page_table.shape[1]:
            raise ValueError(f"row {r}: position {t} beyond the page table")
        p = int(page_table[s, logical])
        if p < 0 or p >= k_out.shape[0]:
            raise ValueError(f"row {r}: page {p} not in the pool")
        slot = t % PAGE
        for g in range(N_KV):
            k_out[p, g, slot, :] = k_new[r][g]
            v_out[p, g, slot, :] = v_new[r][g]
        if key_out is not None and t % BLOCK == BLOCK - 1:
            if p >= key_out.shape[0]:
                raise ValueError(f"row {r}: page {p} not in the key pool")
            key_out[p, slot // BLOCK, :] = key_new[r]
    return k_out, v_out, key_out


# ----------------------------------------------------------------------------
# one-byte block keys: the E4M3 value of each byte   [SAV]
# ----------------------------------------------------------------------------

def encode_e4m3(x) -> np.ndarray:
    """E4M3 code (uint8) of each value: the nearest E4M3 value, ties to the
    code with an even last mantissa bit; magnitudes beyond the largest finite
    value (448) saturate to it; NaN gives the NaN code 0x7F.  -0.0 keeps its
    sign (0x80).  Values are compared exactly in float64 against the 127
    non-negative finite codes listed by ``decode_e4m3``."""
    x = np.asarray(x, dtype=np.float64)
    grid = decode_e4m3(np.arange(0x7F, dtype=np.uint8))  # codes 0x00 .. 0x7E, ascending values
    mag = np.minimum(np.abs(x), grid[-1])
    hi = np.clip(np.searchsorted(grid, mag, side="left"), 0, len(grid) - 1)  # first grid value >= mag
    lo = np.maximum(hi - 1, 0)
    d_lo = mag - grid[lo]
    d_hi = grid[hi] - mag
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.int64)
    code = np.where(mag == grid[hi], hi, code)  # exact hits (including 0)
    code = code | np.where(np.signbit(x), 0x80, 0)
    return np.where(np.isnan(x), 0x7F, code).astype(np.uint8)


def quantize_kv_e4m3(x, scale: float) -> np.ndarray:
    """One-byte codes stored for values x with a per-layer scale: the E4M3
    code of the fp32 product x * fl32(1 / scale) (one fp32 rounding, then
    encode_e4m3), so that a code stands for about x / scale."""
    inv = np.float32(1.0) / np.float32(scale)
    prod = np.asarray(x, dtype=np.float32) * inv  # IEEE fp32 multiply
    return encode_e4m3(prod.astype(np.float64))


def append_to_paged_cache_fp8(k_pool, v_pool, key_pool, page_table, ctx, nq, k_new, v_new, key_new,
                              k_scale: float, v_scale: float):
    """The pools after appending the new tokens of a varlen batch to a cache
    with one-byte K / V: row r's values are stored as
    quantize_kv_e4m3(k_new[r], k_scale) and quantize_kv_e4m3(v_new[r], v_scale)
    at the slots the bf16 append uses; block keys (bf16, key_pool may be None)
    are stored exactly as by append_to_paged_cache."""
    k_codes = quantize_kv_e4m3(np.asarray(k_new, dtype=np.float64), k_scale)
    v_codes = quantize_kv_e4m3(np.asarray(v_new, dtype=np.float64), v_scale)
    return append_to_paged_cache(k_pool, v_pool, key_pool, page_table, ctx, nq, k_codes, v_codes, key_new)


def decode_e4m3(b) -> np.ndarray:
    """Exact float64 value of each E4M3 byte (uint8 array of any shape).

    bits: s eeee mmm.  e = 0: (-1)^s * 2^-6 * m/8 (subnormal, zero when m = 0);
    e = 1..15: (-1)^s * 2^(e-7) * (1 + m/8), except e = 15, m = 7: NaN.
    Largest finite magnitude 448 (e = 15, m = 6)."""
    b = np.asarray(b, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 0x7).astype(np.float64)
    normal = np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))
    sub = np.ldexp(m / 8.0, -6)
    v = sign * np.where(e == 0, sub, normal)
    return np.where((e == 15) & (b & 0x7 == 7), np.nan, v)
