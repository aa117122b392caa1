"""Seeded synthetic inputs for the sparse / sliding-window attention layers.

This module only draws numbers and lays them out; it holds none of the
attention or indexer arithmetic.  It serves both sides of every parity check:
the CUDA path receives paged device pools built here, and the CPU oracle
receives logical (per-sequence, per-position) values drawn here from the same
counters.  Every value is a pure function of (seed, tensor id, element
counter), so any element can be regenerated anywhere without materialising a
whole pool.

Generator (stated here so either side could be re-implemented from it):

* stream keys: three 32-bit words from SplitMix64 (Steele, Lea & Flood,
  "Fast splittable pseudorandom number generators", OOPSLA 2014) run on the
  64-bit value ``seed * 2**20 + tensor_id``;
* counter hash: with ``lo``/``hi`` the 32-bit halves of the element counter,
  ``h1 = fmix32(lo ^ k0)``, ``h2 = fmix32(h1 ^ hi ^ k1)``,
  ``h3 = fmix32(h2 ^ k2)``, where fmix32 is the MurmurHash3 32-bit finaliser
  (Appleby, MurmurHash3, public domain);
* uniform integers in ``[lo, hi]``: ``lo + (h2 * (hi - lo + 1)) >> 32``;
* approximately N(0, 1): the Irwin-Hall sum of the four 16-bit halves of
  ``h2`` and ``h3``, centred and scaled by sqrt(3)/65536 in fp32, then rounded
  to bf16 (round to nearest even).

Only integer operations and one correctly rounded fp32 multiply are used, so
torch on the CPU and on a GPU produce bit-identical tensors.  All integer
arithmetic runs in int64 with every intermediate below 2**49 (32-bit
multiplies are split into 16-bit halves), so nothing overflows.

Workload shapes follow the Step 5 Preview attention configuration (the
StepFun open-weights blog, "What the config says": 64 query heads sharing 4
KV groups of dimension 192, and a 256-wide index key for each 8-token block)
and the serving setup of the SGLang day-0 blog ("Get Started": 64-token pages
and a bf16 KV cache).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import torch

# geometry (StepFun open-weights blog, "What the config says"; SGLang day-0 blog, "Get Started")
N_HEADS = 64
N_KV = 4
HEAD_DIM = 192
PAGE = 64
BLOCK = 8
BLOCKS_PER_PAGE = PAGE // BLOCK
INDEX_DIM = 256
TOPK = 512
WINDOW = 512

# counter layout: positions and blocks of sequence s live at s * MAX_TOKENS + pos
MAX_TOKENS = 1 << 21
MAX_BLOCKS = MAX_TOKENS // BLOCK

# tensor ids (one stream per tensor kind, per layer: id + 16 * layer)
TID_Q, TID_QX, TID_K, TID_V, TID_KX, TID_LEN, TID_PERM, TID_QXN, TID_QXG = 1, 2, 3, 4, 5, 6, 7, 8, 9

_M32 = 0xFFFFFFFF
_M64 = (1 << 64) - 1


def _splitmix64(x: int) -> int:
    x = (x + 0x9E3779B97F4A7C15) & _M64
    z = x
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def stream_keys(seed: int, tensor_id: int) -> tuple:
    """Three 32-bit stream keys for (seed, tensor_id)."""
    s = _splitmix64(((seed & 0xFFFFFFFFFFF) << 20) + (tensor_id & 0xFFFFF))
    t = _splitmix64(s)
    return (s & _M32, (s >> 32) & _M32, t & _M32)


def _mul32(a: torch.Tensor, b: int) -> torch.Tensor:
    """(a * b) mod 2**32 for int64 ``a`` in [0, 2**32) and constant ``b`` < 2**32."""
    b_lo = b & 0xFFFF
    b_hi = b >> 16
    hi = torch.bitwise_and(a * b_hi, 0xFFFF)
    hi.bitwise_left_shift_(16)
    r = a * b_lo
    r.add_(hi)
    return r.bitwise_and_(_M32)


def _fmix32(h: torch.Tensor) -> torch.Tensor:
    h = h ^ (h >> 16)
    h = _mul32(h, 0x85EBCA6B)
    h ^= h >> 13
    h = _mul32(h, 0xC2B2AE35)
    h ^= h >> 16
    return h


def _hash_pair(idx: torch.Tensor, keys: tuple):
    k0, k1, k2 = keys
    lo = torch.bitwise_and(idx, _M32)
    hi = idx >> 32
    h1 = _fmix32(lo ^ k0)
    h2 = _fmix32(h1 ^ hi ^ k1)
    h3 = _fmix32(h2 ^ k2)
    return h2, h3


def uniform_int(seed: int, tensor_id: int, idx: torch.Tensor, lo: int, hi: int) -> torch.Tensor:
    """Uniform integers in [lo, hi] (int64) for int64 counters ``idx``."""
    h2, _ = _hash_pair(idx, stream_keys(seed, tensor_id))
    return ((h2 * (hi - lo + 1)) >> 32) + lo


_IH_SCALE = torch.tensor(math.sqrt(3.0) / 65536.0, dtype=torch.float32)


def normal_bf16(seed: int, tensor_id: int, idx: torch.Tensor) -> torch.Tensor:
    """Approximately N(0,1) bf16 values (Irwin-Hall of four 16-bit uniforms)."""
    h2, h3 = _hash_pair(idx, stream_keys(seed, tensor_id))
    s = torch.bitwise_and(h2, 0xFFFF)
    s += h2 >> 16
    s += torch.bitwise_and(h3, 0xFFFF)
    s += h3 >> 16
    s -= 131070  # 4 * 65535 / 2: centre of the sum of four (u + 0.5) / 65536
    f = s.to(torch.float32)
    f.mul_(_IH_SCALE.to(f.device))
    return f.to(torch.bfloat16)


def to_e4m3_codes(x: torch.Tensor) -> torch.Tensor:
    """One-byte E4M3 codes (uint8) of the values of x, rounded by torch's
    float8_e4m3fn conversion (exact for integers of magnitude <= 16)."""
    return x.to(torch.float8_e4m3fn).view(torch.uint8)


def small_int_bf16(seed: int, tensor_id: int, idx: torch.Tensor, lim: int = 4) -> torch.Tensor:
    """Integer-valued bf16 in [-lim, lim] (exact in bf16)."""
    return uniform_int(seed, tensor_id, idx, -lim, lim).to(torch.bfloat16)


# ----------------------------------------------------------------------------
# workload description
# ----------------------------------------------------------------------------


@dataclasses.dataclass
class Workload:
    """One layer's batch: per sequence s, ``ctx[s]`` cached tokens precede
    ``nq[s]`` new query tokens, whose K/V are already in the cache, so the
    cache holds ``ctx[s] + nq[s]`` tokens of sequence s."""

    ctx: list
    nq: list
    seed: int = 1
    layer: int = 0
    index_int: bool = True  # integer-valued indexer inputs (exact fp32 scores)
    perm_pages: bool = True  # shuffle physical pages
    seq_base: int = 0  # global id of sequence 0 (a shard of a larger batch)
    row_base: int = 0  # global id of query row 0
    # 0: independent indexer queries per token.  W > 0: "block-coherent"
    # indexer queries: the tokens of each W-token window of a sequence share
    # one base query, and each token adds +-1 to about 1/16 of its
    # dimensions, so neighbouring tokens select mostly the same blocks.
    qx_coherent: int = 0

    def __post_init__(self):
        assert len(self.ctx) == len(self.nq)
        assert self.qx_coherent <= 0 or self.index_int, "block-coherent indexer queries are integer-valued"
        for c, n in zip(self.ctx, self.nq):
            assert c >= 0 and n >= 0 and c + n <= MAX_TOKENS

    @property
    def batch(self) -> int:
        return len(self.ctx)

    @property
    def lens(self) -> list:
        return [c + n for c, n in zip(self.ctx, self.nq)]

    @property
    def cu_q(self) -> list:
        out = [0]
        for n in self.nq:
            out.append(out[-1] + n)
        return out

    @property
    def total_q(self) -> int:
        return sum(self.nq)

    @property
    def max_q(self) -> int:
        return max(self.nq) if self.nq else 0

    @property
    def max_len(self) -> int:
        return max(self.lens) if self.nq else 0

    def pages_of(self, s: int) -> int:
        return (self.lens[s] + PAGE - 1) // PAGE

    @property
    def max_pages(self) -> int:
        return max([self.pages_of(s) for s in range(self.batch)] + [1])

    @property
    def num_pages(self) -> int:
        return max(1, sum(self.pages_of(s) for s in range(self.batch)))

    def tid(self, base: int) -> int:
        return base + 16 * self.layer

    def query_seq_pos(self):
        """(sequence, absolute position) of every query row, in row order."""
        seqs, pos = [], []
        for s in range(self.batch):
            for j in range(self.nq[s]):
                seqs.append(s)
                pos.append(self.ctx[s] + j)
        return seqs, pos

    # ---------------- page table ----------------
    def page_table(self) -> torch.Tensor:
        """int32 [batch][max_pages]; -1 marks unmapped entries."""
        n = self.num_pages
        if self.perm_pages:
            g = torch.Generator().manual_seed(self.seed * 1000003 + self.tid(TID_PERM))
            perm = torch.randperm(n, generator=g)
        else:
            perm = torch.arange(n)
        pt = torch.full((self.batch, self.max_pages), -1, dtype=torch.int32)
        k = 0
        for s in range(self.batch):
            m = self.pages_of(s)
            pt[s, :m] = perm[k:k + m].to(torch.int32)
            k += m
        return pt

    # ---------------- logical values (any device) ----------------
    def q_rows(self, rows: torch.Tensor, device="cpu") -> torch.Tensor:
        """Attention queries, bf16 [len(rows)][64][192]."""
        rows = rows.to(device=device, dtype=torch.int64) + self.row_base
        idx = (rows.view(-1, 1, 1) * N_HEADS + torch.arange(N_HEADS, device=device).view(1, -1, 1)) * HEAD_DIM \
            + torch.arange(HEAD_DIM, device=device).view(1, 1, -1)
        return normal_bf16(self.seed, self.tid(TID_Q), idx)

    def row_seq_pos(self, rows: torch.Tensor):
        """(sequence, absolute position) of local query rows ``rows`` (int64 tensors)."""
        dev = rows.device
        cu = torch.tensor(self.cu_q, dtype=torch.int64, device=dev)
        seq = torch.searchsorted(cu[1:], rows, right=True)
        ctx = torch.tensor(self.ctx, dtype=torch.int64, device=dev)
        return seq, ctx[seq] + rows - cu[seq]

    def qx_rows(self, rows: torch.Tensor, device="cpu") -> torch.Tensor:
        """Indexer queries, bf16 [len(rows)][256] (one per query token, shared by all heads)."""
        rows = rows.to(device=device, dtype=torch.int64)
        dims = torch.arange(INDEX_DIM, device=device).view(1, -1)
        grows = rows + self.row_base
        idx = grows.view(-1, 1) * INDEX_DIM + dims
        if self.qx_coherent <= 0:
            if self.index_int:
                return small_int_bf16(self.seed, self.tid(TID_QX), idx)
            return normal_bf16(self.seed, self.tid(TID_QX), idx)
        seq, pos = self.row_seq_pos(rows)
        windows = MAX_TOKENS // self.qx_coherent + 1
        bidx = ((seq + self.seq_base) * windows + pos // self.qx_coherent).view(-1, 1) * INDEX_DIM + dims
        base = uniform_int(self.seed, self.tid(TID_QX), bidx, -4, 4)
        u = uniform_int(self.seed, self.tid(TID_QXN), idx, 0, 31)
        noise = (u == 0).to(torch.int64) - (u == 1).to(torch.int64)
        return (base + noise).to(torch.bfloat16)

    def qx_group_rows(self, rows: torch.Tensor, device="cpu") -> torch.Tensor:
        """Per-KV-group indexer queries, bf16 [len(rows)][4][256]: one query per
        token and KV group, for a selection made separately by each group."""
        rows = rows.to(device=device, dtype=torch.int64) + self.row_base
        idx = (rows.view(-1, 1, 1) * N_KV + torch.arange(N_KV, device=device).view(1, -1, 1)) * INDEX_DIM \
            + torch.arange(INDEX_DIM, device=device).view(1, 1, -1)
        if self.index_int:
            return small_int_bf16(self.seed, self.tid(TID_QXG), idx)
        return normal_bf16(self.seed, self.tid(TID_QXG), idx)

    def kx_blocks(self, s: int, blocks: torch.Tensor, device="cpu", fp8: bool = False) -> torch.Tensor:
        """Block keys of sequence s, bf16 [len(blocks)][256]; with ``fp8``, the
        same values as one-byte E4M3 codes, uint8 [len(blocks)][256]."""
        blocks = blocks.to(device=device, dtype=torch.int64)
        idx = ((self.seq_base + s) * MAX_BLOCKS + blocks.view(-1, 1)) * INDEX_DIM + torch.arange(INDEX_DIM, device=device).view(1, -1)
        if self.index_int:
            vals = small_int_bf16(self.seed, self.tid(TID_KX), idx)
        else:
            vals = normal_bf16(self.seed, self.tid(TID_KX), idx)
        return to_e4m3_codes(vals) if fp8 else vals

    def _kv_tokens(self, tid: int, s: int, pos: torch.Tensor, device) -> torch.Tensor:
        pos = pos.to(device=device, dtype=torch.int64)
        idx = (((self.seq_base + s) * MAX_TOKENS + pos.view(-1, 1, 1)) * N_KV + torch.arange(N_KV, device=device).view(1, -1, 1)) \
            * HEAD_DIM + torch.arange(HEAD_DIM, device=device).view(1, 1, -1)
        return normal_bf16(self.seed, self.tid(tid), idx)

    def k_tokens(self, s: int, pos: torch.Tensor, device="cpu") -> torch.Tensor:
        """Keys of sequence s at positions ``pos``, bf16 [len(pos)][4][192]."""
        return self._kv_tokens(TID_K, s, pos, device)

    def v_tokens(self, s: int, pos: torch.Tensor, device="cpu") -> torch.Tensor:
        """Values of sequence s at positions ``pos``, bf16 [len(pos)][4][192]."""
        return self._kv_tokens(TID_V, s, pos, device)

    # ---------------- paged device pools ----------------
    def _page_owner(self, pt: torch.Tensor):
        """For each physical page: (sequence, logical page), -1 where unused."""
        n = self.num_pages
        own_s = torch.full((n,), -1, dtype=torch.int64)
        own_p = torch.full((n,), -1, dtype=torch.int64)
        for s in range(self.batch):
            m = self.pages_of(s)
            phys = pt[s, :m].to(torch.int64)
            own_s[phys] = s
            own_p[phys] = torch.arange(m, dtype=torch.int64)
        return own_s, own_p

    def kv_pools(self, device, pt: Optional[torch.Tensor] = None, pages_per_chunk: int = 2048,
                 window_only: Optional[int] = None, upto: Optional[Sequence[int]] = None, fp8: bool = False):
        """K and V pools, bf16 [num_pages][4][64][192] each, filled through the page table.

        With ``fp8`` the pools hold the same values as one-byte E4M3 codes
        (uint8, same shape; rounded by torch's float8_e4m3fn conversion).

        With ``window_only = W`` only pages that can hold one of the last W
        tokens before any query of the sequence are filled (the rest stay
        zero): a sliding-window layer never reads older pages.  With ``upto``
        only positions below ``upto[s]`` of sequence s are filled (e.g.
        ``upto = ctx``: the cache before the new tokens are appended); the
        page table and pool size stay those of the whole batch."""
        if pt is None:
            pt = self.page_table()
        own_s, own_p = self._page_owner(pt)
        n = self.num_pages
        k_pool = torch.zeros((n, N_KV, PAGE, HEAD_DIM), dtype=torch.bfloat16, device=device)
        v_pool = torch.zeros_like(k_pool)
        lens = torch.tensor(self.lens if upto is None else list(upto), dtype=torch.int64)
        keep = own_s >= 0
        if window_only is not None:
            ctx = torch.tensor(self.ctx, dtype=torch.int64)
            first_tok = torch.clamp(ctx - window_only + 1, min=0)  # earliest position any query can see
            s_safe = torch.clamp(own_s, min=0)
            keep &= (own_p + 1) * PAGE > first_tok[s_safe]
        ar_g = torch.arange(N_KV, device=device).view(1, -1, 1, 1)
        ar_t = torch.arange(PAGE, device=device).view(1, 1, -1, 1)
        ar_d = torch.arange(HEAD_DIM, device=device).view(1, 1, 1, -1)
        for p0 in range(0, n, pages_per_chunk):
            p1 = min(n, p0 + pages_per_chunk)
            sel = keep[p0:p1]
            if not bool(sel.any()):
                continue
            s = own_s[p0:p1].clamp(min=0).to(device).view(-1, 1, 1, 1)
            lp = own_p[p0:p1].clamp(min=0).to(device).view(-1, 1, 1, 1)
            pos = lp * PAGE + ar_t
            idx = (((self.seq_base + s) * MAX_TOKENS + pos) * N_KV + ar_g) * HEAD_DIM + ar_d
            valid = (sel.to(device).view(-1, 1, 1, 1)) & (pos < lens.to(device)[s.view(-1)].view(-1, 1, 1, 1))
            kv = normal_bf16(self.seed, self.tid(TID_K), idx)
            k_pool[p0:p1] = torch.where(valid, kv, torch.zeros((), dtype=torch.bfloat16, device=device))
            del kv
            kv = normal_bf16(self.seed, self.tid(TID_V), idx)
            v_pool[p0:p1] = torch.where(valid, kv, torch.zeros((), dtype=torch.bfloat16, device=device))
            del kv, idx, valid
        if fp8:
            return to_e4m3_codes(k_pool), to_e4m3_codes(v_pool)
        return k_pool, v_pool

    def index_pool(self, device, pt: Optional[torch.Tensor] = None, pages_per_chunk: int = 16384,
                   upto: Optional[Sequence[int]] = None, fp8: bool = False):
        """Block-key pool, bf16 [num_pages][8][256]; slot j of page p holds the key
        of block 8 * (logical page) + j.  Only complete blocks carry a key: those
        that end at or below ``upto[s]`` tokens (default: the whole sequence).
        With ``fp8`` the pool holds the same keys as one-byte E4M3 codes (uint8;
        exact for the integer-valued keys)."""
        if fp8:
            return to_e4m3_codes(self.index_pool(device, pt, pages_per_chunk, upto))
        if pt is None:
            pt = self.page_table()
        own_s, own_p = self._page_owner(pt)
        n = self.num_pages
        pool = torch.zeros((n, BLOCKS_PER_PAGE, INDEX_DIM), dtype=torch.bfloat16, device=device)
        nblk = torch.tensor([L // BLOCK for L in (self.lens if upto is None else list(upto))], dtype=torch.int64)
        ar_j = torch.arange(BLOCKS_PER_PAGE, device=device).view(1, -1, 1)
        ar_d = torch.arange(INDEX_DIM, device=device).view(1, 1, -1)
        tid = self.tid(TID_KX)
        for p0 in range(0, n, pages_per_chunk):
            p1 = min(n, p0 + pages_per_chunk)
            used = own_s[p0:p1] >= 0
            if not bool(used.any()):
                continue
            s = own_s[p0:p1].clamp(min=0).to(device).view(-1, 1, 1)
            lp = own_p[p0:p1].clamp(min=0).to(device).view(-1, 1, 1)
            blk = lp * BLOCKS_PER_PAGE + ar_j
            idx = ((self.seq_base + s) * MAX_BLOCKS + blk) * INDEX_DIM + ar_d
            valid = used.to(device).view(-1, 1, 1) & (blk < nblk.to(device)[s.view(-1)].view(-1, 1, 1))
            if self.index_int:
                vals = small_int_bf16(self.seed, tid, idx)
            else:
                vals = normal_bf16(self.seed, tid, idx)
            pool[p0:p1] = torch.where(valid, vals, torch.zeros((), dtype=torch.bfloat16, device=device))
        return pool

    def new_tokens(self, device="cpu") -> tuple:
        """Inputs of a cache append of every query row (sequence s, position t):
        ``(k_new, v_new)`` bf16 [total_q][4][192], the values the pools hold at
        t, and ``key_new`` bf16 [total_q][256], the key of block t // 8 (an
        append stores it only for a token that completes its block)."""
        ks, vs, xs = [], [], []
        for s in range(self.batch):
            if self.nq[s] == 0:
                continue
            pos = torch.arange(self.ctx[s], self.lens[s], dtype=torch.int64)
            ks.append(self.k_tokens(s, pos, device))
            vs.append(self.v_tokens(s, pos, device))
            xs.append(self.kx_blocks(s, pos // BLOCK, device))
        if not ks:
            e = torch.zeros((0, N_KV, HEAD_DIM), dtype=torch.bfloat16, device=device)
            return e, e.clone(), torch.zeros((0, INDEX_DIM), dtype=torch.bfloat16, device=device)
        return torch.cat(ks), torch.cat(vs), torch.cat(xs)

    def queries(self, device) -> tuple:
        """(q bf16 [total_q][64][192], qx bf16 [total_q][256]) for every query row."""
        rows = torch.arange(self.total_q, dtype=torch.int64)
        return self.q_rows(rows, device), self.qx_rows(rows, device)


def shard(w: Workload, rank: int, world: int) -> Workload:
    """The rank-th of `world` contiguous shards of w's sequences.  Values are
    drawn with global sequence and row ids, so the shards of a batch hold
    exactly the data of the whole batch."""
    n = w.batch
    lo, hi = rank * n // world, (rank + 1) * n // world
    rows_before = sum(w.nq[:lo])
    return dataclasses.replace(w, ctx=list(w.ctx[lo:hi]), nq=list(w.nq[lo:hi]), seq_base=w.seq_base + lo,
                               row_base=w.row_base + rows_before)


def uniform_lengths(seed: int, n: int, lo: int, hi: int) -> list:
    """n seeded integer lengths uniform in [lo, hi]."""
    idx = torch.arange(n, dtype=torch.int64)
    return [int(x) for x in uniform_int(seed, TID_LEN, idx, lo, hi)]


# ----------------------------------------------------------------------------
# the five workloads (shapes of the Step 5 Preview serving setup)
# ----------------------------------------------------------------------------


def config_workloads(which: int, seed: Optional[int] = None) -> list:
    """Workloads of the numbered configurations; a list of layers.

    1  sparse decode, B=1, 16,384 cached tokens, one query;
    2  sliding-window decode, B=64, lengths U[1K, 128K], one query each;
    3  sparse multi-token verify, B=64, lengths U[32K, 128K], 4 queries each;
    4  sparse chunked prefill, 16,384 queries appended at offset 114,688;
    5  hybrid group (3 sliding-window layers + 1 sparse layer), B=4, 1,048,576 cached tokens.
    0  the headline: sparse decode, B=64, 131,072 cached tokens each, one query;
    6  config 4 with block-coherent indexer queries (64-token windows share a
       base query), a labelled secondary input on which neighbouring queries'
       selections overlap as the shared-set prefill design expects.
    """
    sd = (0x5E5 + which) if seed is None else seed
    if which == 0:
        return [Workload(ctx=[131072] * 64, nq=[1] * 64, seed=sd)]
    if which == 1:
        return [Workload(ctx=[16384], nq=[1], seed=sd)]
    if which == 2:
        return [Workload(ctx=uniform_lengths(sd, 64, 1024, 131072), nq=[1] * 64, seed=sd)]
    if which == 3:
        return [Workload(ctx=uniform_lengths(sd, 64, 32768, 131072), nq=[4] * 64, seed=sd)]
    if which == 4:
        return [Workload(ctx=[114688], nq=[16384], seed=sd)]
    if which == 5:
        return [Workload(ctx=[1048576] * 4, nq=[1] * 4, seed=sd, layer=l) for l in range(4)]
    if which == 6:
        return [Workload(ctx=[114688], nq=[16384], seed=sd, qx_coherent=64)]
    raise ValueError(which)


