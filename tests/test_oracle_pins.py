"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: brute force,
an independent characterisation, a closed form, an invariant, or a value the
pages print.  A plausible mistake in the oracle (a dropped term, a wrong sign,
a wrong head-to-group map, an off-by-one in the window or the current block,
a wrong tie-break) fails at least one of them.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

from oracle import s5_oracle as O

RNG = np.random.default_rng(12345)


# ---------------------------------------------------------------- rounding

def test_round_bf16_ties_and_double_rounding():
    one = 1.0
    assert O.round_bf16(one) == 1.0
    # halfway between 1 and 1 + 2**-7 -> even (1.0)
    assert O.round_bf16(1 + 2 ** -8) == 1.0
    # halfway between 1 + 2**-7 and 1 + 2**-6 -> even (1 + 2**-6)
    assert O.round_bf16(1 + 3 * 2 ** -8) == 1 + 2 ** -6
    # just above the halfway point: rounding through float32 would drop the
    # 2**-30 and tie to 1.0; rounding once from float64 goes up
    assert O.round_bf16(1 + 2 ** -8 + 2 ** -30) == 1 + 2 ** -7
    assert O.round_bf16(-(1 + 2 ** -8 + 2 ** -30)) == -(1 + 2 ** -7)
    assert O.round_bf16(0.0) == 0.0


def test_round_bf16_matches_library_on_float32_values():
    # for values already in float32, one rounding to bf16 is what torch does
    x = (RNG.standard_normal(20000) * 10.0 ** RNG.uniform(-3, 3, 20000)).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.round_bf16(x.astype(np.float64)), ref)


# ---------------------------------------------------------------- selection

def _naive_topk(scores, k):
    """Repeated max extraction, scanning in index order with a strict '>'
    so the lower index wins a tie."""
    scores = list(scores)
    taken = [False] * len(scores)
    out = []
    for _ in range(min(k, len(scores))):
        best = -1
        for i, s in enumerate(scores):
            if taken[i]:
                continue
            if best < 0 or s > scores[best]:
                best = i
        taken[best] = True
        out.append(best)
    return sorted(out)


def _subset_characterisation(scores, k):
    """The unique k-subset S with: every member beats every non-member
    (higher score, or equal score and lower index)."""
    c = len(scores)
    found = []
    for S in itertools.combinations(range(c), k):
        inside = set(S)
        ok = all((scores[x] > scores[y]) or (scores[x] == scores[y] and x < y)
                 for x in inside for y in range(c) if y not in inside)
        if ok:
            found.append(list(S))
    assert len(found) == 1
    return found[0]


@pytest.mark.parametrize("trial", range(40))
def test_select_topk_brute_force(trial):
    c = int(RNG.integers(1, 40))
    k = int(RNG.choice([1, 3, 8]))
    scores = RNG.integers(-3, 4, c).astype(np.float64)  # many ties
    got = O.select_topk(scores, k)
    want = _naive_topk(scores, k)
    assert list(got[:len(want)]) == want
    assert np.all(got[len(want):] == -1)


@pytest.mark.parametrize("trial", range(25))
def test_select_topk_subset_definition(trial):
    c = int(RNG.integers(5, 12))
    k = int(RNG.integers(1, 5))
    scores = RNG.integers(-2, 3, c).astype(np.float64)
    got = O.select_topk(scores, k)
    assert list(got) == _subset_characterisation(list(scores), k)


def test_select_topk_tie_cases():
    # all equal -> the first 512 blocks
    assert list(O.select_topk(np.zeros(2000), 512)) == list(range(512))
    # strictly decreasing -> the first 512
    assert list(O.select_topk(-np.arange(2000.0), 512)) == list(range(512))
    # strictly increasing -> the last 512
    assert list(O.select_topk(np.arange(2000.0), 512)) == list(range(1488, 2000))
    # a tie straddling the cut: 500 clear winners, then ties broken by index
    s = np.zeros(3000)
    winners = RNG.choice(3000, 500, replace=False)
    s[winners] = 10
    got = O.select_topk(s, 512)
    rest = [i for i in range(3000) if i not in set(winners.tolist())][:12]
    assert list(got) == sorted(winners.tolist() + rest)


def test_select_topk_short_history_takes_all():
    for c in [0, 1, 7, 511, 512]:
        got = O.select_topk(RNG.standard_normal(c), 512)
        assert list(got[:c]) == list(range(c))
        assert np.all(got[c:] == -1)


def test_index_topk_scores_only_history_blocks():
    # blocks at or after the current block must never be scored
    c_t = 600  # t in block 600
    t = c_t * 8 + 5
    kx = RNG.integers(-4, 5, (c_t + 10, 256)).astype(np.float64)
    qx = RNG.integers(-4, 5, 256).astype(np.float64)
    kx[c_t:] = 4 * np.sign(qx)  # make the future/current blocks score highest
    sel = O.index_topk_query(qx, kx, t, 512)
    assert sel.max() < c_t and len(set(sel.tolist())) == 512
    scores = kx[:c_t] @ qx
    assert list(sel) == _naive_topk(scores, 512)


def test_block_scores_exact_integers():
    kx = RNG.integers(-4, 5, (1000, 256))
    qx = RNG.integers(-4, 5, 256)
    want = kx.astype(np.int64) @ qx.astype(np.int64)
    got = O.block_scores(qx.astype(np.float64), kx.astype(np.float64))
    assert np.array_equal(got, want.astype(np.float64))


# ---------------------------------------------------------------- token sets

@pytest.mark.parametrize("trial", range(20))
def test_sparse_token_set_membership(trial):
    t = int(RNG.integers(0, 6000))
    c = t // 8
    n = min(512, c)
    sel = np.sort(RNG.choice(c, n, replace=False)) if c else np.zeros(0, np.int64)
    T = set(O.sparse_token_set(sel, t).tolist())
    sset = set(sel.tolist())
    for p in range(0, t + 20):
        inside = (p // 8 in sset) or (p // 8 == c and p <= t)
        assert (p in T) == inside, (p, t)
    assert len(T) == len(O.sparse_token_set(sel, t))  # no duplicates


def test_swa_token_set_edges():
    assert list(O.swa_token_set(0, 512)) == [0]
    assert list(O.swa_token_set(511, 512)) == list(range(0, 512))
    assert list(O.swa_token_set(512, 512)) == list(range(1, 513))
    assert len(O.swa_token_set(100000, 512)) == 512


# ---------------------------------------------------------------- attention closed forms

def _rand(*shape):
    return RNG.standard_normal(shape)


def test_single_token_returns_its_value():
    q = _rand(64, 192)
    k = _rand(1, 4, 192)
    v = _rand(1, 4, 192)
    out, lse = O.gqa_attention(q, k, v, 0.1)
    for h in range(64):
        assert np.allclose(out[h], v[0, h // 16], atol=0, rtol=0)
        assert math.isclose(lse[h], 0.1 * float(q[h] @ k[0, h // 16]), rel_tol=1e-14, abs_tol=1e-14)


def test_identical_keys_average_values():
    q = _rand(64, 192)
    k1 = _rand(1, 4, 192)
    k = np.repeat(k1, 37, axis=0)
    v = _rand(37, 4, 192)
    out, lse = O.gqa_attention(q, k, v, 0.07)
    for h in range(64):
        g = h // 16
        assert np.allclose(out[h], v[:, g].mean(axis=0), rtol=1e-13, atol=1e-13)
        assert math.isclose(lse[h], 0.07 * float(q[h] @ k1[0, g]) + math.log(37), rel_tol=1e-13)


def test_two_tokens_sigmoid_weights():
    # k0 = e_0, k1 = 0; q_h = x_h * e_0 -> weight of token 0 is sigmoid(scale * x_h)
    q = np.zeros((64, 192))
    x = RNG.uniform(-5, 5, 64)
    q[:, 0] = x
    k = np.zeros((2, 4, 192))
    k[0, :, 0] = 1.0
    v = np.zeros((2, 4, 192))
    v[0] = 1.0
    scale = 0.3
    out, lse = O.gqa_attention(q, k, v, scale)
    sig = 1.0 / (1.0 + np.exp(-scale * x))
    assert np.allclose(out, np.repeat(sig[:, None], 192, axis=1), rtol=1e-13, atol=1e-15)
    assert np.allclose(lse, np.log(np.exp(scale * x) + 1.0), rtol=1e-13)


def test_head_reads_group_h_div_16():
    # each group's values are the constant g + 1; head h must return g(h) + 1
    q = _rand(64, 192)
    k = _rand(9, 4, 192)
    v = np.zeros((9, 4, 192))
    for g in range(4):
        v[:, g] = g + 1
    out, _ = O.gqa_attention(q, k, v, 0.1)
    for h in range(64):
        assert np.allclose(out[h], h // 16 + 1, rtol=1e-14)


def test_weights_sum_to_one_and_positive():
    q = _rand(64, 192)
    k = _rand(300, 4, 192)
    v = _rand(300, 4, 192)
    _, _, w = O.gqa_attention(q, k, v, O.DEFAULT_SM_SCALE, return_weights=True)
    assert np.all(w > 0)
    assert np.allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-12)


def test_zero_scale_is_uniform_average():
    q = _rand(64, 192)
    k = _rand(50, 4, 192)
    v = _rand(50, 4, 192)
    out, lse = O.gqa_attention(q, k, v, 0.0)
    for h in range(64):
        assert np.allclose(out[h], v[:, h // 16].mean(axis=0), rtol=1e-13, atol=1e-14)
    assert np.allclose(lse, math.log(50), rtol=1e-14)


def test_lse_is_log_sum_exp_of_scores():
    q = _rand(64, 192) * 0.1
    k = _rand(20, 4, 192)
    v = _rand(20, 4, 192)
    _, lse = O.gqa_attention(q, k, v, 0.5)
    for h in range(64):
        s = 0.5 * (k[:, h // 16] @ q[h])
        assert math.isclose(lse[h], math.log(sum(math.exp(x) for x in s)), rel_tol=1e-12)


def test_scale_shift_invariance():
    # adding the same amount to every score leaves the output unchanged
    q = _rand(64, 192)
    k = _rand(40, 4, 192)
    v = _rand(40, 4, 192)
    out1, lse1 = O.gqa_attention(q, k, v, 0.1)
    kb = k + 0.0
    # shift every key by a vector orthogonal to nothing in particular: use q-dependent shift
    # per group, k_j + u_g changes s_j by scale * q_h . u_g, the same for all j
    u = _rand(4, 192)
    kb = k + u[None]
    out2, lse2 = O.gqa_attention(q, kb, v, 0.1)
    assert np.allclose(out1, out2, rtol=1e-11, atol=1e-12)
    for h in range(64):
        assert math.isclose(lse2[h] - lse1[h], 0.1 * float(q[h] @ u[h // 16]), rel_tol=1e-9, abs_tol=1e-11)


# ---------------------------------------------------------------- invariants of the layers

def _full_causal(q, k_seq, v_seq, t, scale):
    """Full causal attention over positions 0..t, written with the group map
    applied by repeating KV groups to heads (a different formulation)."""
    K = np.repeat(k_seq[: t + 1], 16, axis=1)   # [n][64][192]
    V = np.repeat(v_seq[: t + 1], 16, axis=1)
    s = scale * np.einsum("hd,nhd->hn", q, K)
    w = np.exp(s)
    w /= w.sum(axis=1, keepdims=True)
    return np.einsum("hn,nhd->hd", w, V)


@pytest.mark.parametrize("t", [0, 5, 7, 8, 63, 64, 200, 4095])
def test_sparse_equals_full_when_history_fits(t):
    # c = t // 8 <= 512: every history block is selected
    L = t + 1
    k_seq = _rand(L, 4, 192)
    v_seq = _rand(L, 4, 192)
    q = _rand(64, 192)
    kx = RNG.integers(-4, 5, (L // 8 + 1, 256)).astype(np.float64)
    qx = RNG.integers(-4, 5, 256).astype(np.float64)
    sel = O.index_topk_query(qx, kx, t, 512)
    out, _ = O.sparse_attention_query(q, sel, t, k_seq, v_seq, 0.08)
    assert np.allclose(out, _full_causal(q, k_seq, v_seq, t, 0.08), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("t,window", [(0, 512), (100, 512), (511, 512), (700, 701), (50, 4096)])
def test_swa_equals_full_when_window_covers(t, window):
    k_seq = _rand(t + 1, 4, 192)
    v_seq = _rand(t + 1, 4, 192)
    q = _rand(64, 192)
    out, _ = O.swa_attention_query(q, t, k_seq, v_seq, window, 0.08)
    assert np.allclose(out, _full_causal(q, k_seq, v_seq, t, 0.08), rtol=1e-11, atol=1e-12)


def test_swa_excludes_tokens_outside_window():
    t, W = 900, 512
    k_seq = _rand(t + 1, 4, 192)
    v_seq = _rand(t + 1, 4, 192)
    q = _rand(64, 192)
    out1, _ = O.swa_attention_query(q, t, k_seq, v_seq, W, 0.1)
    k2, v2 = k_seq.copy(), v_seq.copy()
    k2[: t - W + 1] = 50.0  # would dominate if read
    v2[: t - W + 1] = 1e6
    out2, _ = O.swa_attention_query(q, t, k2, v2, W, 0.1)
    assert np.array_equal(out1, out2)
    # and the oldest in-window token is read
    k3 = k_seq.copy()
    k3[t - W + 1] = 3.0 * q.mean(axis=0) / 16
    out3, _ = O.swa_attention_query(q, t, k3, v_seq, W, 0.1)
    assert not np.allclose(out1, out3)


def test_sparse_order_invariance():
    t = 8 * 3000 + 3
    L = t + 1
    k_seq = _rand(L, 4, 192)
    v_seq = _rand(L, 4, 192)
    q = _rand(64, 192)
    sel = np.sort(RNG.choice(3000, 512, replace=False))
    out1, lse1 = O.sparse_attention_query(q, sel, t, k_seq, v_seq, 0.07)
    perm = RNG.permutation(sel)
    out2, lse2 = O.sparse_attention_query(q, perm, t, k_seq, v_seq, 0.07)
    assert np.allclose(out1, out2, rtol=1e-12, atol=1e-12)
    assert np.allclose(lse1, lse2, rtol=1e-12, atol=1e-12)


def test_sparse_causal_within_current_block():
    t = 8 * 700 + 2  # three tokens of the current block are visible
    L = t + 6
    k_seq = _rand(L, 4, 192)
    v_seq = _rand(L, 4, 192)
    q = _rand(64, 192)
    sel = np.sort(RNG.choice(700, 512, replace=False))
    out1, _ = O.sparse_attention_query(q, sel, t, k_seq, v_seq, 0.1)
    k2, v2 = k_seq.copy(), v_seq.copy()
    k2[t + 1:] = 40.0
    v2[t + 1:] = 1e6
    out2, _ = O.sparse_attention_query(q, sel, t, k2, v2, 0.1)
    assert np.array_equal(out1, out2)
    # an unselected history block is never read
    unsel = sorted(set(range(700)) - set(sel.tolist()))[0]
    k2[unsel * 8: unsel * 8 + 8] = 40.0
    v2[unsel * 8: unsel * 8 + 8] = 1e6
    out3, _ = O.sparse_attention_query(q, sel, t, k2, v2, 0.1)
    assert np.array_equal(out1, out3)


def test_batch_driver_rows():
    ctx, nq = [20, 5000], [2, 3]
    rows = O.query_positions(ctx, nq)
    assert rows == [(0, 20), (0, 21), (1, 5000), (1, 5001), (1, 5002)]


# ---------------------------------------------------------------- the pages' arithmetic

def _golden(name):
    path = os.path.join(os.path.dirname(__file__), "golden", name)
    out = {}
    for line in open(path):
        if line.startswith("#") or not line.strip():
            continue
        parts = [p.strip() for p in line.split("|")]
        out[parts[0]] = (float(parts[1]), float(parts[3]))
    return out


def test_bytes_model_reproduces_pages():
    from block_sparse_gqa_indexer_b200 import roofline as R
    g = _golden("pages_byte_arithmetic.txt")
    got = {
        "kv_bytes_per_token_layer": R.kv_bytes_per_token(),
        "kv_bytes_per_token_23": R.model_kv_bytes_per_token(),
        "session_128k": R.session_kv_bytes(128 * 1024),
        "session_1m": R.session_kv_bytes(1 << 20),
        "swa_69_layers": R.swa_resident_bytes(),
        "index_key_overhead": R.index_key_overhead(),
        "selected_1m_23_layers": R.selected_bytes_per_step(),
        "blocks_per_layer_1m": (1 << 20) // 8,
        "indexer_1m_1byte": R.indexer_bytes_per_step(1 << 20, 1),
        "indexer_1m_2byte": R.indexer_bytes_per_step(1 << 20, 2),
        "dense_1m": R.session_kv_bytes(1 << 20),
    }
    assert set(got) == set(g)
    for k, (val, tol) in g.items():
        assert abs(got[k] - val) <= tol * val + 1e-9, (k, got[k], val)


def test_sparse_tokens_bounds():
    from block_sparse_gqa_indexer_b200 import roofline as R
    # a query reads 4,097 .. 4,104 tokens once 512 history blocks exist
    assert {R.sparse_tokens(8 * 5000 + j) for j in range(8)} == set(range(4097, 4105))
    assert R.sparse_tokens(0) == 1
    assert R.scored_blocks(8 * 512 + 7) == 0 and R.scored_blocks(8 * 513) == 513


def test_append_bytes_count_written_keys():
    from block_sparse_gqa_indexer_b200 import roofline as R
    # a token is 3,072 bytes of K and V, read once and written once; a key is
    # moved only for blocks the batch completes: 7 -> 8 completes block 0,
    # 8 -> 9 completes none, 5 -> 22 completes blocks 0 and 1
    assert R.append_bytes([7], [1]) == {"kv": 6144, "keys": 1024, "total": 7168}
    assert R.append_bytes([8], [1])["keys"] == 0
    assert R.append_bytes([5], [17])["keys"] == 2 * 1024
    assert R.append_bytes([7], [1], with_keys=False)["total"] == 6144
    # the prefix-to-whole check of the oracle counts the same blocks
    w = _append_case()
    _, pos = w.query_seq_pos()
    completing = sum(1 for t in pos if t % 8 == 7)
    assert R.append_bytes(w.ctx, w.nq)["keys"] == completing * 1024


# ---------------------------------------------------------------- cache append

def _bits(t):
    """bf16 tensor -> int16 numpy bit patterns (exact comparisons)."""
    return t.contiguous().view(torch.int16).numpy()


def _append_case():
    from block_sparse_gqa_indexer_b200 import synth as S
    # page and block boundaries on both sides of the new tokens, an empty
    # sequence, a fresh sequence, several pages of new tokens
    return S.Workload(ctx=[0, 5, 63, 64, 130, 1000, 7, 40], nq=[3, 9, 1, 64, 70, 17, 0, 200], seed=11)


def test_append_rebuilds_the_seeded_cache_from_its_prefix():
    # The generator's pool builder fills positions below `upto` through the
    # page table on its own; appending the new tokens (and the keys of the
    # blocks they complete) to the prefix pools must give the whole batch's
    # pools bit for bit.
    w = _append_case()
    pt = w.page_table()
    k0, v0 = w.kv_pools("cpu", pt, upto=w.ctx)
    x0 = w.index_pool("cpu", pt, upto=w.ctx)
    k1, v1 = w.kv_pools("cpu", pt)
    x1 = w.index_pool("cpu", pt)
    kn, vn, xn = w.new_tokens("cpu")
    # rows that complete no block carry junk: the append must not read them
    _, pos = w.query_seq_pos()
    junk = torch.tensor([p % 8 != 7 for p in pos])
    xn = xn.clone()
    xn[junk] = torch.tensor(-3.5, dtype=torch.bfloat16)
    ko, vo, xo = O.append_to_paged_cache(_bits(k0), _bits(v0), _bits(x0), pt.numpy(), w.ctx, w.nq, _bits(kn),
                                         _bits(vn), _bits(xn))
    assert np.array_equal(ko, _bits(k1)) and np.array_equal(vo, _bits(v1)) and np.array_equal(xo, _bits(x1))
    # the prefix really differed (the append did the work)
    assert not np.array_equal(_bits(k0), _bits(k1)) and not np.array_equal(_bits(x0), _bits(x1))


def test_append_without_block_keys_and_empty_batch():
    w = _append_case()
    pt = w.page_table()
    k0, v0 = w.kv_pools("cpu", pt, upto=w.ctx)
    k1, v1 = w.kv_pools("cpu", pt)
    kn, vn, _ = w.new_tokens("cpu")
    ko, vo, xo = O.append_to_paged_cache(_bits(k0), _bits(v0), None, pt.numpy(), w.ctx, w.nq, _bits(kn),
                                         _bits(vn), None)
    assert xo is None and np.array_equal(ko, _bits(k1)) and np.array_equal(vo, _bits(v1))
    # no new tokens: nothing changes
    z = np.zeros((0, 4, 192), dtype=np.int16)
    ke, ve, xe = O.append_to_paged_cache(_bits(k0), _bits(v0), None, pt.numpy(), w.ctx, [0] * w.batch, z, z, None)
    assert np.array_equal(ke, _bits(k0)) and np.array_equal(ve, _bits(v0))


def test_append_rejects_unmapped_pages():
    w = _append_case()
    pt = w.page_table()
    k0, v0 = w.kv_pools("cpu", pt, upto=w.ctx)
    kn, vn, xn = w.new_tokens("cpu")
    bad = pt.numpy().copy()
    bad[4, 2] = -1  # sequence 4 appends positions 130..199: logical pages 2 and 3
    with pytest.raises(ValueError):
        O.append_to_paged_cache(_bits(k0), _bits(v0), None, bad, w.ctx, w.nq, _bits(kn), _bits(vn), None)


# ---------------------------------------------------------------- per-KV-group selection

def test_grouped_selection_follows_each_groups_query():
    # Group g's query is a unit vector on dimension d_g, and exactly the 512
    # blocks of a known set S_g have a 1 there (0 elsewhere): each group must
    # select its own S_g, whatever the other dimensions hold.
    rng = np.random.default_rng(7)
    c = 700
    dims = [3, 77, 140, 255]
    kx = rng.integers(-4, 5, size=(c, 256)).astype(np.float64)
    qx = np.zeros((4, 256))
    sets = []
    for g, d in enumerate(dims):
        qx[g, d] = 1.0
        S_g = np.sort(rng.choice(c, 512, replace=False))
        kx[:, d] = 0.0
        kx[S_g, d] = 1.0
        sets.append(S_g)
    sel = O.index_topk_query_grouped(qx, kx, 8 * c + 5)
    assert sel.shape == (4, 512)
    for g in range(4):
        assert np.array_equal(sel[g], sets[g]), g


def test_grouped_attention_routes_heads_to_their_groups_selection():
    # Zero keys give uniform weights, so head h returns the mean of its
    # group's values over that group's token set; values encode (position,
    # group), which pins the token set of each group and the head-to-group map.
    t = 8 * 40 + 3
    rng = np.random.default_rng(8)
    sels = [np.sort(rng.choice(40, 5 + 3 * g, replace=False)) for g in range(4)]
    k_seq = np.zeros((t + 1, 4, 192))
    pos = np.arange(t + 1, dtype=np.float64)
    v_seq = np.zeros((t + 1, 4, 192))
    for g in range(4):
        v_seq[:, g, :] = (pos + 1000.0 * g)[:, None]
    q = rng.standard_normal((64, 192))
    out, lse = O.sparse_attention_query_grouped(q, sels, t, k_seq, v_seq)
    for h in range(64):
        g = h // 16
        toks = np.concatenate([(sels[g][:, None] * 8 + np.arange(8)).ravel(), np.arange(8 * 40, t + 1)])
        assert np.allclose(out[h], toks.mean() + 1000.0 * g, rtol=0, atol=1e-9), h
        assert abs(lse[h] - math.log(len(toks))) < 1e-12


def test_grouped_attention_with_equal_selections_is_the_shared_layer():
    rng = np.random.default_rng(9)
    t = 8 * 600 + 2
    k_seq = rng.standard_normal((t + 1, 4, 192))
    v_seq = rng.standard_normal((t + 1, 4, 192))
    q = rng.standard_normal((64, 192))
    sel = np.sort(rng.choice(600, 512, replace=False))
    o1, l1 = O.sparse_attention_query(q, sel, t, k_seq, v_seq)
    o4, l4 = O.sparse_attention_query_grouped(q, [sel] * 4, t, k_seq, v_seq)
    assert np.array_equal(o1, o4) and np.array_equal(l1, l4)


# ---------------------------------------------------------------- one-byte (E4M3) block keys

def test_e4m3_values_the_format_fixes():
    d = lambda x: float(O.decode_e4m3(np.array([x], dtype=np.uint8))[0])
    assert d(0x38) == 1.0 and d(0x40) == 2.0 and d(0xB8) == -1.0
    assert d(0x7E) == 448.0                  # largest finite: e = 15, m = 6
    assert d(0x08) == 2.0 ** -6              # smallest normal
    assert d(0x01) == 2.0 ** -9 and d(0x07) == 7 * 2.0 ** -9   # subnormals
    assert d(0x00) == 0.0 and d(0x80) == 0.0 and math.copysign(1, d(0x80)) == -1
    assert math.isnan(d(0x7F)) and math.isnan(d(0xFF))
    assert d(0x77) == 240.0                  # e = 14, m = 7: 2^7 * 1.875
    # positive codes increase strictly up to the largest finite value
    v = O.decode_e4m3(np.arange(0x7F, dtype=np.uint8))
    assert np.all(np.diff(v) > 0)


def test_e4m3_matches_the_library_type_on_every_byte():
    b = np.arange(256, dtype=np.uint8)
    ours = O.decode_e4m3(b)
    lib = torch.from_numpy(b).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(lib))
    assert np.array_equal(ours[~np.isnan(ours)], lib[~np.isnan(lib)])


# ---------------------------------------------------------------- multi-row selection

@pytest.mark.parametrize("trial", range(12))
def test_index_topk_rows_brute_force_tiny(trial):
    # tiny histories with heavy ties: every row against repeated max extraction
    # over its own history only
    c_max = int(RNG.integers(2, 40))
    k = int(RNG.choice([1, 3, 8]))
    kx = RNG.integers(-2, 3, (c_max + 3, 256)).astype(np.float64)
    pos = RNG.integers(0, 8 * c_max + 8, 7)
    qx = RNG.integers(-2, 3, (7, 256)).astype(np.float64)
    got = O.index_topk_rows(qx, kx, pos, k)
    for i, t in enumerate(pos.tolist()):
        c = t // 8
        if c <= k:
            want = list(range(c))
        else:
            want = _naive_topk([float(kx[b] @ qx[i]) for b in range(c)], k)
        assert list(got[i][:len(want)]) == want, (i, t)
        assert np.all(got[i][len(want):] == -1)


def test_index_topk_rows_masks_each_rows_future():
    # rows of one sequence at different positions: blocks at or after a row's
    # current block score highest, yet no row may select them
    c_hi = 900
    kx = RNG.integers(-4, 5, (c_hi, 256)).astype(np.float64)
    qx = np.tile(RNG.integers(-4, 5, 256).astype(np.float64), (4, 1))
    kx[600:] = 4 * np.sign(qx[0])
    pos = np.array([600 * 8, 600 * 8 + 7, 700 * 8 + 3, 899 * 8 + 1])
    got = O.index_topk_rows(qx, kx, pos, 512)
    for i, t in enumerate(pos.tolist()):
        c = t // 8
        assert got[i].max() < c and len(set(got[i].tolist())) == 512
    # a row whose history holds the strong blocks takes all of them that fit
    assert set(range(600, 700)) <= set(got[2].tolist())


def test_index_topk_rows_agrees_with_one_row_form():
    kx = RNG.integers(-4, 5, (3000, 256)).astype(np.float64)
    pos = RNG.integers(0, 3000 * 8, 40)
    qx = RNG.integers(-4, 5, (40, 256)).astype(np.float64)
    got = O.index_topk_rows(qx, kx, pos, 512)
    for i, t in enumerate(pos.tolist()):
        assert np.array_equal(got[i], O.index_topk_query(qx[i], kx, t, 512))


# ---------------------------------------------------------------- one-byte (E4M3) KV

def _codes(x):
    return torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_fp8kv_single_token_returns_scaled_value():
    # one readable token (t = 0, nothing selected): every head returns that
    # token's V of its group, decoded and multiplied by v_scale, whatever K is
    vals = RNG.integers(-16, 17, (1, 4, 192)).astype(np.float64)
    kc = _codes(RNG.standard_normal((1, 4, 192)))
    vc = _codes(vals)
    q = RNG.standard_normal((64, 192))
    out, lse = O.sparse_attention_query_fp8kv(q, np.full(512, -1), 0, kc, vc, 0.7, 2.5)
    for h in range(64):
        assert np.array_equal(out[h], 2.5 * vals[0, h // 16])


def test_fp8kv_identical_keys_average_scaled_values():
    # every key equal: uniform weights, so out = v_scale * mean of the decoded values
    t = 8 * 600 + 3
    kc = np.tile(_codes(RNG.standard_normal((1, 4, 192))), (t + 1, 1, 1))
    vals = RNG.integers(-8, 9, (t + 1, 4, 192)).astype(np.float64) / 4.0  # exact in E4M3
    vc = _codes(vals)
    sel = np.sort(RNG.choice(600, 512, replace=False))
    q = RNG.standard_normal((64, 192))
    out, _ = O.sparse_attention_query_fp8kv(q, sel, t, kc, vc, 1.3, 0.5)
    T = O.sparse_token_set(sel, t)
    for h in range(64):
        assert np.allclose(out[h], 0.5 * vals[T, h // 16].mean(axis=0), rtol=0, atol=1e-12)


def test_fp8kv_two_tokens_weights_follow_k_scale():
    # two tokens: the weight of the second is sigmoid(sm_scale * k_scale * q.(k1 - k0))
    k = np.zeros((2, 4, 192))
    k[0, :, 0] = 1.0
    k[1, :, 0] = 3.0
    v = np.zeros((2, 4, 192))
    v[1, :, :] = 1.0  # out = weight of token 1
    q = np.zeros((64, 192))
    q[:, 0] = np.linspace(-2, 2, 64)
    for k_scale in (0.25, 1.0, 3.0):
        out, lse = O.sparse_attention_query_fp8kv(q, np.full(512, -1), 1, _codes(k), _codes(v), k_scale, 1.0, 0.5)
        z = 0.5 * k_scale * q[:, 0] * (3.0 - 1.0)
        assert np.allclose(out[:, 5], 1.0 / (1.0 + np.exp(-z)), rtol=0, atol=1e-12)
        s0, s1 = 0.5 * k_scale * q[:, 0] * 1.0, 0.5 * k_scale * q[:, 0] * 3.0
        assert np.allclose(lse, np.logaddexp(s0, s1), rtol=0, atol=1e-12)


def test_fp8kv_equals_bf16_attention_on_representable_values():
    # values exactly representable in E4M3 (and bf16): with unit scales the
    # one-byte layer is the two-byte layer on the same values; with scales
    # a, b it is the two-byte layer on a*K and b*V
    t = 8 * 700 + 6
    kv_vals = RNG.integers(-16, 17, (2, t + 1, 4, 192)).astype(np.float64) / 8.0
    kc, vc = _codes(kv_vals[0]), _codes(kv_vals[1])
    assert np.array_equal(O.decode_e4m3(kc), kv_vals[0]) and np.array_equal(O.decode_e4m3(vc), kv_vals[1])
    sel = np.sort(RNG.choice(700, 512, replace=False))
    q = RNG.standard_normal((64, 192))
    o8, l8 = O.sparse_attention_query_fp8kv(q, sel, t, kc, vc, 1.0, 1.0)
    o2, l2 = O.sparse_attention_query(q, sel, t, kv_vals[0], kv_vals[1])
    assert np.allclose(o8, o2, rtol=0, atol=1e-12) and np.allclose(l8, l2, rtol=0, atol=1e-12)
    o8s, l8s = O.sparse_attention_query_fp8kv(q, sel, t, kc, vc, 0.75, 3.0)
    o2s, l2s = O.sparse_attention_query(q, sel, t, 0.75 * kv_vals[0], 3.0 * kv_vals[1])
    assert np.allclose(o8s, o2s, rtol=0, atol=1e-12) and np.allclose(l8s, l2s, rtol=0, atol=1e-12)


def test_fp8kv_reads_only_the_sparse_token_set():
    # bytes outside the selected blocks and past t never change the result
    t = 8 * 650 + 2
    kc = _codes(RNG.standard_normal((t + 9, 4, 192)))
    vc = _codes(RNG.standard_normal((t + 9, 4, 192)))
    sel = np.sort(RNG.choice(650, 512, replace=False))
    q = RNG.standard_normal((64, 192))
    o1, _ = O.sparse_attention_query_fp8kv(q, sel, t, kc, vc, 1.0, 1.0)
    unsel = sorted(set(range(650)) - set(sel.tolist()))[0]
    kc2, vc2 = kc.copy(), vc.copy()
    kc2[unsel * 8:unsel * 8 + 8] = 0x7E  # 448
    vc2[unsel * 8:unsel * 8 + 8] = 0x7E
    kc2[t + 1:] = 0x7E
    vc2[t + 1:] = 0x7E
    o2, _ = O.sparse_attention_query_fp8kv(q, sel, t, kc2, vc2, 1.0, 1.0)
    assert np.array_equal(o1, o2)


# ---------------------------------------------------------------- E4M3 encoding (one-byte KV append)

def test_e4m3_encode_round_trips_every_finite_code():
    b = np.arange(256, dtype=np.uint8)
    v = O.decode_e4m3(b)
    fin = ~np.isnan(v)
    assert np.array_equal(O.encode_e4m3(v[fin]), b[fin])  # -0.0 -> 0x80 included


def test_e4m3_encode_ties_saturation_nan():
    # midpoints go to the code with an even mantissa: 1.0 = 0x38, 1.125 = 0x39, 1.25 = 0x3A
    assert O.encode_e4m3(1.0625) == 0x38
    assert O.encode_e4m3(1.1875) == 0x3A
    assert O.encode_e4m3(-1.0625) == 0xB8
    # smallest subnormal 2^-9: half of it ties to zero, just above rounds up
    assert O.encode_e4m3(2.0 ** -10) == 0x00 and O.encode_e4m3(2.0 ** -10 * 1.0001) == 0x01
    # beyond 448 (0x7E) saturates; NaN keeps the NaN code
    assert O.encode_e4m3(500.0) == 0x7E and O.encode_e4m3(-1e9) == 0xFE
    assert O.encode_e4m3(float("nan")) == 0x7F


def test_e4m3_encode_matches_the_library_conversion():
    # an independent implementation: torch's float8_e4m3fn conversion, in range
    g = np.random.default_rng(5)
    x = (g.standard_normal(100000) * np.exp(g.uniform(-9, 6, 100000))).astype(np.float32)
    x = x[np.abs(x) < 440]
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.encode_e4m3(x.astype(np.float64)), want)


def test_quantize_kv_scale_is_one_fp32_product():
    g = np.random.default_rng(6)
    x = torch.from_numpy(g.standard_normal(5000).astype(np.float32)).to(torch.bfloat16).double().numpy()
    assert np.array_equal(O.quantize_kv_e4m3(x, 1.0), O.encode_e4m3(x))
    assert np.array_equal(O.quantize_kv_e4m3(x, 4.0), O.encode_e4m3(x / 4.0))  # power of two: exact
    # a general scale: the fp32 product, not the exact quotient, is encoded
    s = 0.37
    prod = (x.astype(np.float32) * (np.float32(1.0) / np.float32(s))).astype(np.float64)
    assert np.array_equal(O.quantize_kv_e4m3(x, s), O.encode_e4m3(prod))


def test_fp8_append_rebuilds_the_seeded_one_byte_cache():
    # appending the new tokens' values (scale 1) to the one-byte pools of the
    # cached prefix gives the whole batch's one-byte pools, as the generator
    # draws them independently through the page table
    from block_sparse_gqa_indexer_b200 import synth as S
    w = S.Workload(ctx=[60, 130, 0], nq=[9, 2, 70], seed=21)
    pt = w.page_table()
    k0, v0 = w.kv_pools("cpu", pt, upto=w.ctx, fp8=True)
    x0 = w.index_pool("cpu", pt, upto=w.ctx)
    kn, vn, xn = w.new_tokens("cpu")
    k1, v1, x1 = O.append_to_paged_cache_fp8(k0.numpy(), v0.numpy(), x0.double().numpy(), pt.numpy(), w.ctx, w.nq,
                                             kn.double().numpy(), vn.double().numpy(), xn.double().numpy(), 1.0, 1.0)
    kw, vw = w.kv_pools("cpu", pt, fp8=True)
    assert np.array_equal(k1, kw.numpy()) and np.array_equal(v1, vw.numpy())
    assert np.array_equal(x1, w.index_pool("cpu", pt).double().numpy())
