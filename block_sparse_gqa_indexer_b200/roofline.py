"""Algorithmic bytes and FLOPs of the sparse and sliding-window layers.

These are the roofline numerators: the bytes a perfect implementation must
move (each selected KV token once, each scored block key once, queries and
outputs once), never the dense KV cache, and the useful FLOPs of the
attention contractions.

The per-token figures reproduce the KV arithmetic of the StepFun open-weights
blog ("Why GQA, and what it costs": 3,072 bytes per token per full-attention
layer, ~70.7 KB per token over 23 layers, ~9.3 GB at 128K and ~74 GB at 1M
tokens, ~109 MB for 69 sliding-window layers, index keys ~2% extra at two
bytes per value) and its read-volume estimate ("What sparse attention does and
doesn't save": ~290 MB of selected blocks over 23 sparse layers and ~0.8-1.5 GB
of indexer keys per decode step at 1M context).
"""
from __future__ import annotations

N_HEADS = 64
N_KV = 4
HEAD_DIM = 192
BLOCK = 8
INDEX_DIM = 256
TOPK = 512
WINDOW = 512
BF16 = 2

# full-model layer counts (SGLang day-0 blog, "Overview": 3 sliding-window + 1 sparse, 92 layers)
N_LAYERS = 92
N_SPARSE_LAYERS = N_LAYERS // 4
N_SWA_LAYERS = N_LAYERS - N_SPARSE_LAYERS


def kv_bytes_per_token(kv_bytes_per_value: int = BF16) -> int:
    """K and V of all KV groups for one token of one layer."""
    return 2 * N_KV * HEAD_DIM * kv_bytes_per_value


def index_key_bytes(key_bytes_per_value: int = BF16) -> int:
    """One block key."""
    return INDEX_DIM * key_bytes_per_value


def q_bytes() -> int:
    return N_HEADS * HEAD_DIM * BF16


def out_bytes(with_lse: bool = True) -> int:
    return N_HEADS * HEAD_DIM * BF16 + (N_HEADS * 4 if with_lse else 0)


def sparse_tokens(t: int, topk: int = TOPK) -> int:
    """Tokens a sparse query at position t reads: min(topk, c) blocks of 8 plus
    the 1..8 tokens of its current block."""
    c = t // BLOCK
    return BLOCK * min(topk, c) + (t - BLOCK * c + 1)


def swa_tokens(t: int, window: int = WINDOW) -> int:
    return min(window, t + 1)


def scored_blocks(t: int, topk: int = TOPK) -> int:
    """Blocks whose keys must be read to select for a query at t (none when
    every history block is selected anyway)."""
    c = t // BLOCK
    return c if c > topk else 0


def attn_flops(n_tokens: int) -> int:
    """QK^T and PV for all 64 heads over n_tokens keys (2 FLOPs per MAC)."""
    return 4 * N_HEADS * HEAD_DIM * n_tokens


def index_flops(n_blocks: int) -> int:
    return 2 * INDEX_DIM * n_blocks


def sparse_decode_bytes(ctx, nq, unique_tokens=None, topk: int = TOPK) -> dict:
    """Algorithmic bytes of one sparse layer step over a varlen batch.

    Keys are read once per sequence (the largest history among its queries).
    KV tokens are counted per query unless ``unique_tokens`` (per sequence,
    the size of the union of its queries' token sets) is given."""
    kv = keys = qio = 0
    for s, (c0, n) in enumerate(zip(ctx, nq)):
        if n == 0:
            continue
        last = c0 + n - 1
        keys += scored_blocks(last, topk) * index_key_bytes()
        if unique_tokens is not None:
            kv += unique_tokens[s] * kv_bytes_per_token()
        else:
            kv += sum(sparse_tokens(c0 + j, topk) for j in range(n)) * kv_bytes_per_token()
        qio += n * (q_bytes() + out_bytes() + index_key_bytes())
    return {"kv": kv, "keys": keys, "qio": qio, "total": kv + keys + qio}


def swa_decode_bytes(ctx, nq, window: int = WINDOW) -> dict:
    """Algorithmic bytes of one sliding-window layer step (union of each
    sequence's windows counted once)."""
    kv = qio = 0
    for c0, n in zip(ctx, nq):
        if n == 0:
            continue
        last = c0 + n - 1
        first = max(0, c0 - window + 1)
        kv += (last - first + 1) * kv_bytes_per_token()
        qio += n * (q_bytes() + out_bytes())
    return {"kv": kv, "keys": 0, "qio": qio, "total": kv + qio}


def append_bytes(ctx, nq, with_keys: bool = True) -> dict:
    """Algorithmic bytes of one cache append: each new token's K/V read once
    and written once; with block keys, each key of a block the batch
    completes read once and written once."""
    kv = keys = 0
    for c0, n in zip(ctx, nq):
        kv += 2 * n * kv_bytes_per_token()
        if with_keys:
            keys += 2 * ((c0 + n) // BLOCK - c0 // BLOCK) * index_key_bytes()
    return {"kv": kv, "keys": keys, "total": kv + keys}


def sparse_flops(ctx, nq, topk: int = TOPK) -> dict:
    attn = index = 0
    for c0, n in zip(ctx, nq):
        for j in range(n):
            t = c0 + j
            attn += attn_flops(sparse_tokens(t, topk))
            index += index_flops(scored_blocks(t, topk))
    return {"attn": attn, "index": index, "total": attn + index}


# ---------------- whole-model arithmetic (the blog's figures) ----------------

def model_kv_bytes_per_token(n_layers: int = N_SPARSE_LAYERS) -> int:
    return n_layers * kv_bytes_per_token()


def session_kv_bytes(tokens: int) -> int:
    return tokens * model_kv_bytes_per_token()


def swa_resident_bytes(n_layers: int = N_SWA_LAYERS, window: int = WINDOW) -> int:
    return n_layers * window * kv_bytes_per_token()


def selected_bytes_per_step(n_layers: int = N_SPARSE_LAYERS, topk: int = TOPK) -> int:
    """Full 8-token current block (the upper end)."""
    return n_layers * (topk * BLOCK + BLOCK) * kv_bytes_per_token()


def indexer_bytes_per_step(context: int, key_bytes_per_value: int = BF16,
                           n_layers: int = N_SPARSE_LAYERS) -> int:
    return n_layers * (context // BLOCK) * INDEX_DIM * key_bytes_per_value


def index_key_overhead(key_bytes_per_value: int = BF16) -> float:
    return index_key_bytes(key_bytes_per_value) / (BLOCK * kv_bytes_per_token())
