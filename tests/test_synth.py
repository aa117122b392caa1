"""Host checks of the seeded input generator and the paged layout it builds."""
import numpy as np
import torch

from block_sparse_gqa_indexer_b200 import synth as S


def test_counter_hash_reference_values():
    # mul32 against Python's exact integers
    a = torch.tensor([0, 1, 0xFFFFFFFF, 0x12345678, 0xDEADBEEF], dtype=torch.int64)
    for b in [0x85EBCA6B, 0xC2B2AE35, 1, 0xFFFFFFFF]:
        got = S._mul32(a, b).tolist()
        assert got == [(int(x) * b) & 0xFFFFFFFF for x in a.tolist()]


def _fmix32_py(h):
    h ^= h >> 16
    h = (h * 0x85EBCA6B) & 0xFFFFFFFF
    h ^= h >> 13
    h = (h * 0xC2B2AE35) & 0xFFFFFFFF
    h ^= h >> 16
    return h


def test_fmix32_matches_definition():
    xs = [0, 1, 2, 0x7FFFFFFF, 0x80000000, 0xFFFFFFFF, 123456789]
    got = S._fmix32(torch.tensor(xs, dtype=torch.int64)).tolist()
    assert got == [_fmix32_py(x) for x in xs]
    assert _fmix32_py(0) == 0 and _fmix32_py(1) == 0x514E28B7  # MurmurHash3 fmix32(1)


def test_uniform_and_normal_moments():
    idx = torch.arange(1 << 20, dtype=torch.int64)
    u = S.uniform_int(9, 2, idx, -4, 4)
    assert int(u.min()) == -4 and int(u.max()) == 4
    counts = torch.bincount(u + 4).double()
    assert float((counts / counts.mean() - 1).abs().max()) < 0.02
    x = S.normal_bf16(9, 3, idx).double()
    assert abs(float(x.mean())) < 0.01 and abs(float(x.std()) - 1) < 0.01
    assert float(x.abs().max()) < 3.5  # Irwin-Hall(4) support is +-sqrt(12)


def test_generator_is_deterministic_and_seed_dependent():
    idx = torch.arange(5000, dtype=torch.int64)
    a = S.normal_bf16(1, 3, idx)
    assert torch.equal(a, S.normal_bf16(1, 3, idx))
    assert not torch.equal(a, S.normal_bf16(2, 3, idx))
    assert not torch.equal(a, S.normal_bf16(1, 4, idx))


def test_paged_pools_hold_logical_values():
    w = S.Workload(ctx=[130, 0, 77], nq=[3, 2, 1], seed=5)
    pt = w.page_table()
    assert sorted(pt[pt >= 0].tolist()) == list(range(w.num_pages))
    k, v = w.kv_pools("cpu", pt)
    ip = w.index_pool("cpu", pt)
    for s in range(w.batch):
        L = w.lens[s]
        pos = torch.arange(L)
        kk, vv = w.k_tokens(s, pos), w.v_tokens(s, pos)
        for p in range(L):
            page = int(pt[s, p // 64])
            assert torch.equal(k[page, :, p % 64], kk[p])
            assert torch.equal(v[page, :, p % 64], vv[p])
        blocks = torch.arange(L // 8)
        kb = w.kx_blocks(s, blocks)
        for b in range(L // 8):
            assert torch.equal(ip[int(pt[s, b // 8]), b % 8], kb[b])
    # index values are small integers
    assert set(torch.unique(ip.float()).tolist()) <= set(range(-4, 5))


def test_config_shapes():
    assert S.config_workloads(1)[0].ctx == [16384]
    w2 = S.config_workloads(2)[0]
    assert w2.batch == 64 and all(1024 <= c <= 131072 for c in w2.ctx)
    w3 = S.config_workloads(3)[0]
    assert w3.total_q == 256 and all(32768 <= c <= 131072 for c in w3.ctx)
    w4 = S.config_workloads(4)[0]
    assert w4.ctx == [114688] and w4.nq == [16384]
    w5 = S.config_workloads(5)
    assert len(w5) == 4 and w5[0].ctx == [1 << 20] * 4
    # different layers draw different values
    assert not torch.equal(w5[0].k_tokens(0, torch.arange(4)), w5[1].k_tokens(0, torch.arange(4)))


def test_block_coherent_indexer_queries():
    # tokens of one 64-token window share a base query and differ from it by
    # +-1 in about 1/16 of the dimensions; windows draw independent bases
    w = S.Workload(ctx=[1000, 130], nq=[200, 64], seed=9, qx_coherent=64)
    rows = torch.arange(w.total_q)
    qx = w.qx_rows(rows).float()
    seq, pos = w.row_seq_pos(rows)
    assert torch.equal(seq[:200], torch.zeros(200, dtype=torch.int64))
    assert torch.equal(pos[:200], torch.arange(1000, 1200))
    assert torch.equal(pos[200:], torch.arange(130, 194))
    assert qx.abs().max() <= 5 and torch.equal(qx, qx.round())
    same = pos[:200] // 64 == 1000 // 64  # rows of the window holding position 1000
    a, b = qx[:200][same][0], qx[:200][same][1]
    frac = (a != b).float().mean().item()  # two tokens differ where either was perturbed
    assert 0.0 < frac < 0.3
    far = qx[0] != qx[150]  # positions 1000 and 1150: different windows
    assert far.float().mean().item() > 0.5
    # deterministic, a pure function of (seed, sequence, position): the second
    # sequence drawn alone gives the same values
    w2 = S.Workload(ctx=[130], nq=[64], seed=9, qx_coherent=64, seq_base=1, row_base=200)
    assert torch.equal(w2.qx_rows(torch.arange(64)), w.qx_rows(torch.arange(200, 264)))
    assert torch.equal(S.shard(w, 1, 2).qx_rows(torch.arange(64)), w.qx_rows(torch.arange(200, 264)))
    # independent queries are unchanged by the option's existence
    w0 = S.Workload(ctx=[1000, 130], nq=[200, 64], seed=9)
    assert not torch.equal(w0.qx_rows(rows), w.qx_rows(rows))


def test_config6_is_config4_with_coherent_queries():
    (w4,), (w6,) = S.config_workloads(4), S.config_workloads(6)
    assert w6.ctx == w4.ctx and w6.nq == w4.nq and w6.qx_coherent == 64 and w4.qx_coherent == 0


def test_grouped_indexer_queries():
    w = S.Workload(ctx=[100, 9000], nq=[3, 2], seed=5)
    rows = torch.arange(w.total_q)
    qg = w.qx_group_rows(rows)
    assert qg.shape == (5, 4, 256) and qg.dtype == torch.bfloat16
    v = qg.float()
    assert torch.equal(v, v.round()) and v.abs().max() <= 4
    # four different queries per token, and a stream of their own
    assert not torch.equal(qg[:, 0], qg[:, 1])
    assert not torch.equal(qg[:, 0], w.qx_rows(rows))
    # a shard draws the same values for its rows
    sh = S.shard(w, 1, 2)
    assert torch.equal(sh.qx_group_rows(torch.arange(sh.total_q)), qg[3:])


def test_one_byte_keys_hold_the_same_integer_values():
    from oracle import s5_oracle as O
    w = S.Workload(ctx=[3000, 700], nq=[1, 2], seed=6)
    pt = w.page_table()
    codes = w.index_pool("cpu", pt, fp8=True)
    vals = w.index_pool("cpu", pt)
    assert codes.dtype == torch.uint8 and codes.shape == vals.shape
    assert (O.decode_e4m3(codes.numpy()) == vals.double().numpy()).all()
    blk = torch.arange(100)
    assert torch.equal(w.kx_blocks(1, blk, fp8=True), S.to_e4m3_codes(w.kx_blocks(1, blk)))
