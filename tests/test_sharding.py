"""Spreading a decode batch over ranks, on CPU: the oracle's attention state
and state merge pinned against closed forms and library routines, the host
logic that splits pages and heads, and the exchange of states between two
gloo ranks.

Decode of rank r's page range (a plain shorter sequence) leaves, per row, the
normalised output o_r and its log-sum-exp lse_r; merging the ranks' states by
log-sum-exp gives the attention over the whole sequence (the split-KV
recombination of xiaodao.ai "HPC-Ops TPOT -48.8%", Attention section)."""
from __future__ import annotations

import math
import os
import socket

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

import oracle
from mixed_length_paged_b200 import HpaError, workloads as W
from mixed_length_paged_b200 import sharding as SH
from tests.helpers import bf16_values, bits16, dense_kv


def _tiny(seed, lens, Hq=8, Hkv=2, D=64):
    return W.make_batch(W.DecodeShape("s", Hq, Hkv, D), list(lens), seed=seed)


def _arrays(batch):
    return (bits16(batch.q), bits16(batch.k_cache), bits16(batch.v_cache),
            batch.page_table.numpy(), batch.seq_lens.numpy())


# ---------------------------------------------------------------- oracle: state and merge

def test_attention_state_matches_dense_logsumexp():
    batch = _tiny(11, (37, 200, 1))
    q, kc, vc, pt, sl = _arrays(batch)
    qv, kv, vv = bf16_values(q), bf16_values(kc), bf16_values(vc)
    scale = 1 / 8
    for b, L in enumerate(sl):
        K, V = dense_kv(kv, pt, b, int(L)), dense_kv(vv, pt, b, int(L))
        for h in (0, 3, 7):
            o, lse = oracle.attention_state(q, kc, vc, pt, 2, scale, b, h, 0, int(L))
            s = scale * (K[:, h // 4, :] @ qv[b, h])          # [L] logits
            assert lse == pytest.approx(logsumexp(s), abs=1e-12)
            p = np.exp(s - logsumexp(s))
            np.testing.assert_allclose(o, p @ V[:, h // 4, :], atol=1e-12)
            if L == 1:  # one key: its logit and its value
                assert lse == pytest.approx(s[0], abs=1e-15)
                np.testing.assert_array_equal(o, V[0, h // 4, :])


def test_attention_state_zero_query_and_empty_range():
    batch = _tiny(12, (37, 200))
    batch.q.zero_()
    q, kc, vc, pt, _ = _arrays(batch)
    o, lse = oracle.attention_state(q, kc, vc, pt, 2, 1 / 8, 1, 2, 0, 200)
    assert lse == pytest.approx(math.log(200), abs=1e-13)   # all logits 0
    o, lse = oracle.attention_state(q, kc, vc, pt, 2, 1 / 8, 1, 2, 50, 50)
    assert lse == -math.inf and not o.any()


def test_merge_states_of_split_equals_unsplit():
    batch = _tiny(13, (37, 200))
    q, kc, vc, pt, sl = _arrays(batch)
    rng = np.random.default_rng(14)
    for b, L in enumerate(sl):
        L = int(L)
        whole = oracle.attention_state(q, kc, vc, pt, 2, 1 / 8, b, 5, 0, L)
        for nsplit in (1, 2, 4, 9):
            cuts = np.sort(rng.choice(np.arange(1, L), size=nsplit - 1, replace=False))
            edges = [0, *cuts.tolist(), L]
            st = [oracle.attention_state(q, kc, vc, pt, 2, 1 / 8, b, 5, a, e)
                  for a, e in zip(edges[:-1], edges[1:])]
            o, lse = oracle.merge_states([s[0] for s in st], [s[1] for s in st])
            np.testing.assert_allclose(o, whole[0], atol=1e-12)
            assert lse == pytest.approx(whole[1], abs=1e-12)
            # the merged log-sum-exp is the library's log-sum-exp of the parts'
            assert lse == pytest.approx(logsumexp([s[1] for s in st]), abs=1e-12)


def test_merge_states_special_cases():
    rng = np.random.default_rng(15)
    o = rng.standard_normal((3, 16))
    # one state: the identity
    m, l = oracle.merge_states(o[:1], [0.7])
    np.testing.assert_array_equal(m, o[0])
    assert l == 0.7
    # equal weights: the mean, and log(n) added
    m, l = oracle.merge_states(o, [2.0, 2.0, 2.0])
    np.testing.assert_allclose(m, o.mean(axis=0), atol=1e-15)
    assert l == pytest.approx(2.0 + math.log(3), abs=1e-15)
    # -inf states are ignored, even holding NaN
    bad = o.copy()
    bad[1] = np.nan
    m, l = oracle.merge_states(bad, [1.0, -math.inf, 1.0])
    np.testing.assert_allclose(m, (o[0] + o[2]) / 2, atol=1e-15)
    # a dominant state wins; all -inf merges to (0, -inf)
    m, l = oracle.merge_states(o, [0.0, 800.0, 0.0])
    np.testing.assert_allclose(m, o[1], atol=1e-15)
    m, l = oracle.merge_states(o, [-math.inf] * 3)
    assert l == -math.inf and not m.any()


# ---------------------------------------------------------------- host logic

def _tiles_by_rule(n, start, N):
    """Tile t of a sequence of n tiles goes to rank (start + t) mod N: the
    tiles of each rank, listed by walking the tiles once."""
    held = [[] for _ in range(N)]
    for t in range(n):
        held[(start + t) % N].append(t)
    return held


@pytest.mark.parametrize("N", [1, 2, 3, 4, 8])
def test_page_shard_covers_every_token_once(N):
    rng = np.random.default_rng(20 + N)
    lens = np.concatenate([[0, 1, 63, 64, 65, 128, 4096], rng.integers(0, 3000, 40)]).astype(np.int32)
    pts = int((lens.max() + 63) // 64) + 1
    pt = rng.permutation(len(lens) * pts).reshape(len(lens), pts).astype(np.int32)
    start = rng.integers(0, N, len(lens))
    for st in (None, start):
        shards = [SH.page_shard(torch.from_numpy(lens), torch.from_numpy(pt), N, r,
                                start=None if st is None else torch.from_numpy(st))
                  for r in range(N)]
        total = sum(s[0].numpy().astype(np.int64) for s in shards)
        np.testing.assert_array_equal(total, lens)
        for b, L in enumerate(lens):
            n = (int(L) + 63) // 64
            held = _tiles_by_rule(n, b % N if st is None else int(st[b]), N)
            for r, (lr, ptr) in enumerate(shards):
                lr, ptr = int(lr[b]), ptr.numpy()
                k = (lr + 63) // 64
                assert ptr.shape == pt.shape
                assert k == len(held[r])
                assert ptr[b, :k].tolist() == [int(pt[b, t]) for t in held[r]]
                assert not ptr[b, k:].any()
                # every tile but the sequence's last is full
                if n - 1 not in held[r]:
                    assert lr == 64 * k
                else:
                    assert lr == 64 * (k - 1) + (int(L) - 64 * (n - 1))
            # within one tile of even
            sizes = [len(h) for h in held]
            assert max(sizes) - min(sizes) <= 1


def test_page_shard_is_stable_as_sequences_grow():
    """200 decode steps, every sequence growing by one token a step (crossing
    page boundaries): no page that was written ever changes rank, and each
    rank's page list at a step is a prefix of its list at the next step (so
    its cache layout only grows at the end)."""
    N = 3
    rng = np.random.default_rng(5)
    base = np.array([0, 1, 63, 64, 127, 300, 1000], dtype=np.int64)
    steps = 200
    final = base + steps
    pts = int((final.max() + 63) // 64)
    pt = rng.permutation(len(base) * pts).reshape(len(base), pts).astype(np.int32)
    start = torch.from_numpy(rng.integers(0, N, len(base)))
    owner, lists = {}, None
    for s in range(steps + 1):
        L = torch.from_numpy((base + s).astype(np.int32))
        shares = [SH.page_shard(L, torch.from_numpy(pt), N, r, start=start) for r in range(N)]
        now = []
        for r, (lr, ptr) in enumerate(shares):
            per_seq = []
            for b in range(len(base)):
                k = (int(lr[b]) + 63) // 64
                pages = ptr.numpy()[b, :k].tolist()
                per_seq.append(pages)
                for p in pages:
                    assert owner.setdefault(p, r) == r, (s, b, p)
            now.append(per_seq)
        if lists is not None:
            for r in range(N):
                for b in range(len(base)):
                    prev = lists[r][b]
                    assert now[r][b][:len(prev)] == prev, (s, r, b)
        lists = now
    # every page of the final lengths was handed out, each to one rank
    assert len(owner) == int(((final + 63) // 64).sum())


def test_page_shard_rejects_bad_input():
    lens, pt = torch.tensor([130], dtype=torch.int32), torch.zeros(1, 2, dtype=torch.int32)
    with pytest.raises(HpaError):
        SH.page_shard(lens, pt, 2, 0)            # 3 tiles in a 2-entry table
    with pytest.raises(HpaError):
        SH.page_shard(torch.tensor([5]), pt, 2, 2)
    with pytest.raises(HpaError):
        SH.page_shard(torch.tensor([-1]), pt, 1, 0)
    with pytest.raises(HpaError):
        SH.page_shard(torch.tensor([5]), pt, 2, 0, start=torch.tensor([2]))  # start >= N
    with pytest.raises(HpaError):
        SH.page_shard(torch.tensor([5]), pt, 2, 0, start=torch.tensor([0, 1]))


@pytest.mark.parametrize("N", [1, 2, 3, 5])
def test_page_shard_then_merge_equals_whole_sequence(N):
    lens = (0, 1, 37, 200, 129)
    batch = _tiny(30 + N, lens)
    q, kc, vc, pt, sl = _arrays(batch)
    whole = oracle.paged_decode(q, kc, vc, pt, sl, 2, 1 / 8)
    per = [SH.page_shard(batch.seq_lens, batch.page_table, N, r) for r in range(N)]
    for b in range(len(lens)):
        for h in (0, 6):
            st = [oracle.attention_state(q, kc, vc, ptr.numpy(), 2, 1 / 8, b, h, 0, int(lr[b]))
                  for lr, ptr in per]
            o, lse = oracle.merge_states([s[0] for s in st], [s[1] for s in st])
            np.testing.assert_allclose(o, whole[b, h], atol=1e-12)
            if lens[b] == 0:
                assert lse == -math.inf


def test_head_shard_keeps_groups_whole():
    for Hq, Hkv, N in [(64, 8, 1), (64, 8, 2), (64, 8, 8), (32, 8, 4), (8, 2, 2)]:
        G = Hq // Hkv
        seen_g, seen_h = [], []
        for r in range(N):
            (g0, g1), (h0, h1) = SH.head_shard(Hq, Hkv, N, r)
            assert (h0, h1) == (g0 * G, g1 * G)
            seen_g += list(range(g0, g1))
            seen_h += list(range(h0, h1))
        assert seen_g == list(range(Hkv)) and seen_h == list(range(Hq))
    with pytest.raises(HpaError):
        SH.head_shard(64, 8, 3, 0)
    with pytest.raises(HpaError):
        SH.head_shard(64, 8, 2, 2)


# ---------------------------------------------------------------- two gloo ranks

def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_worker(rank: int, world: int, port: int, q):
    import sys
    from datetime import timedelta
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle as O
    from mixed_length_paged_b200 import sharding as S
    from mixed_length_paged_b200 import workloads as WL
    from tests.helpers import bits16 as b16
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        lens = (0, 1, 37, 200, 129)
        batch = WL.make_batch(WL.DecodeShape("s", 8, 2, 64), list(lens), seed=40)
        qb, kc, vc = b16(batch.q), b16(batch.k_cache), b16(batch.v_cache)
        lr, ptr = S.page_shard(batch.seq_lens, batch.page_table, world, rank)
        o = torch.zeros(len(lens), 8, 64, dtype=torch.float64)
        lse = torch.full((len(lens), 8), -math.inf, dtype=torch.float64)
        for b in range(len(lens)):
            for h in range(8):
                ob, lb = O.attention_state(qb, kc, vc, ptr.numpy(), 2, 1 / 8, b, h, 0, int(lr[b]))
                o[b, h] = torch.from_numpy(ob)
                lse[b, h] = lb
        o_all, lse_all = S.gather_states(o, lse)
        assert len(o_all) == world
        whole = O.paged_decode(qb, kc, vc, batch.page_table.numpy(), batch.seq_lens.numpy(), 2,
                               1 / 8)
        err = 0.0
        for b in range(len(lens)):
            for h in range(8):
                m, _ = O.merge_states([x[b, h].numpy() for x in o_all],
                                      [float(x[b, h]) for x in lse_all])
                err = max(err, float(np.abs(m - whole[b, h]).max()))
        # the local state arrived unchanged at its own slot
        assert torch.equal(o_all[rank], o) and torch.equal(lse_all[rank], lse)
        # the same exchange into receive buffers allocated beforehand
        ob = [torch.full_like(o, float("nan")) for _ in range(world)]
        lb = [torch.full_like(lse, float("nan")) for _ in range(world)]
        o2, l2 = S.gather_states(o, lse, o_all=ob, lse_all=lb)
        assert o2 is ob and l2 is lb
        assert all(torch.equal(x, y) for x, y in zip(ob, o_all))
        assert all(torch.equal(x, y) for x, y in zip(lb, lse_all))
        dist.barrier()
        q.put((rank, err))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_page_sharded_decode_equals_whole():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gloo_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1]
    assert max(r[1] for r in res) <= 1e-12, res


def _growing_worker(rank: int, world: int, port: int, q):
    """Several decode steps on gloo ranks while the sequences grow across page
    boundaries: each step, every rank takes its share by the stable page rule,
    computes its states with the oracle, all-gathers them and merges; the
    result must equal the whole-sequence oracle, and a rank's page list may
    only grow at its end."""
    import sys
    from datetime import timedelta
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle as O
    from mixed_length_paged_b200 import sharding as S
    from mixed_length_paged_b200 import workloads as WL
    from tests.helpers import bits16 as b16
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        base = np.array([62, 127, 1, 190, 0, 63])
        steps = 6
        # the cache already holds every token the steps will reach
        batch = WL.make_batch(WL.DecodeShape("g", 8, 2, 64), list(base + steps), seed=42)
        qb, kc, vc = b16(batch.q), b16(batch.k_cache), b16(batch.v_cache)
        pt = batch.page_table.numpy()
        start = torch.tensor([1, 0, 1, 1, 0, 0])
        err, prev = 0.0, None
        for s in range(steps + 1):
            L = torch.from_numpy((base + s).astype(np.int32))
            lr, ptr = S.page_shard(L, batch.page_table, world, rank, start=start)
            pages = [ptr.numpy()[b, :(int(lr[b]) + 63) // 64].tolist() for b in range(len(base))]
            if prev is not None:
                assert all(pages[b][:len(prev[b])] == prev[b] for b in range(len(base)))
            prev = pages
            o = torch.zeros(len(base), 8, 64, dtype=torch.float64)
            lse = torch.full((len(base), 8), -math.inf, dtype=torch.float64)
            for b in range(len(base)):
                for h in range(8):
                    ob, lb = O.attention_state(qb, kc, vc, ptr.numpy(), 2, 1 / 8, b, h, 0,
                                               int(lr[b]))
                    o[b, h] = torch.from_numpy(ob)
                    lse[b, h] = lb
            o_all, lse_all = S.gather_states(o, lse)
            whole = O.paged_decode(qb, kc, vc, pt, L.numpy(), 2, 1 / 8)
            for b in range(len(base)):
                for h in range(8):
                    m, _ = O.merge_states([x[b, h].numpy() for x in o_all],
                                          [float(x[b, h]) for x in lse_all])
                    err = max(err, float(np.abs(m - whole[b, h]).max()))
        dist.barrier()
        q.put((rank, err))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_page_sharded_decode_while_sequences_grow():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_growing_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1]
    assert max(r[1] for r in res) <= 1e-12, res


def test_gather_states_outside_a_process_group_is_the_local_state():
    o, l = torch.ones(2, 3, 4), torch.zeros(2, 3)
    oa, la = SH.gather_states(o, l)
    assert len(oa) == 1 and oa[0] is o and la[0] is l


def _decoder_worker(rank: int, world: int, port: int, q):
    """PageShardedDecoder's host logic on gloo: its GPU step and merge are
    replaced by the oracle (the decoder's own code still allocates the
    receive buffers, gathers the states in rank order and hands them on)."""
    import sys
    from datetime import timedelta
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle as O
    from mixed_length_paged_b200 import sharding as S
    from mixed_length_paged_b200 import workloads as WL
    from tests.helpers import bits16 as b16
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        lens = (0, 1, 37, 200, 129, 700)
        B, Hq, Hkv, D = len(lens), 8, 2, 64
        batch = WL.make_batch(WL.DecodeShape("s", Hq, Hkv, D), list(lens), seed=41)
        qb, kc, vc = b16(batch.q), b16(batch.k_cache), b16(batch.v_cache)
        calls = []

        class FakeDecoder:  # the local decode step, computed by the oracle
            def __init__(self, *a, **kw):
                self.device = torch.device("cpu")

            def step(self, q, k, v, pt, sl, out, scale, *, k_scale=None, v_scale=None, lse=None):
                calls.append("step")
                for b in range(B):
                    for h in range(Hq):
                        o, l = O.attention_state(qb, kc, vc, pt.numpy(), Hkv, scale, b, h, 0,
                                                 int(sl[b]))
                        out[b, h] = torch.from_numpy(o)
                        lse[b, h] = l
                return out

        def fake_merge(o_parts, l_parts, out, lse_out=None):
            calls.append(("merge", len(o_parts)))
            for b in range(B):
                for h in range(Hq):
                    m, _ = O.merge_states([x[b, h].double().numpy() for x in o_parts],
                                          [float(x[b, h]) for x in l_parts])
                    out[b, h] = torch.from_numpy(m)
            return out

        S.PagedDecoder = FakeDecoder
        S.merge_states = fake_merge
        dec = S.PageShardedDecoder(B, Hq, Hkv, D, batch.pt_stride)
        assert len(dec.o_all) == world and len(dec.lse_all) == world
        lr, ptr = S.page_shard(batch.seq_lens, batch.page_table, world, rank)
        out = torch.full((B, Hq, D), float("nan"), dtype=torch.float32)
        for _ in range(2):  # a second step reuses the same receive buffers
            bufs = [id(x) for x in dec.o_all]
            dec.step(batch.q, batch.k_cache, batch.v_cache, ptr, lr, out, 1 / 8)
            assert [id(x) for x in dec.o_all] == bufs
        whole = O.paged_decode(qb, kc, vc, batch.page_table.numpy(), batch.seq_lens.numpy(),
                               Hkv, 1 / 8)
        err = float(np.abs(out.double().numpy() - whole).max())
        assert calls == ["step", ("merge", world)] * 2, calls
        dist.barrier()
        q.put((rank, err))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_page_sharded_decoder_host_logic():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_decoder_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # fp32 states merged: within fp32 rounding of the fp64 whole-batch result
    assert max(r[1] for r in res) <= 1e-5, res
