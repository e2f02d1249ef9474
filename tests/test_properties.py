"""Property-based checks (hypothesis) of the oracle planner and the host-side
page split, on random batches: the invariants the plan kinds promise, which
the parametrised pins check on fixed cases."""
from __future__ import annotations

import numpy as np
import torch
from hypothesis import given, settings, strategies as st

import oracle
from mixed_length_paged_b200 import sharding as SH
from tests.test_oracle_pins import _check_plan_invariants, _units

lens_st = st.lists(st.integers(min_value=0, max_value=3000), min_size=1, max_size=24)


@settings(max_examples=60, deadline=None)
@given(lens=lens_st, Hkv=st.sampled_from([1, 2, 4, 8]), P=st.integers(1, 300),
       m=st.integers(1, 12), q=st.integers(1, 4), e=st.integers(0, 4))
def test_length_aware_plan_properties(lens, Hkv, P, m, q, e):
    """The length-aware plan moves each cut of the dynamic plan of the same
    shape (tail and cost weights) by less than m units, keeps segments of
    fewer than 2m tiles whole, and leaves the end pieces of a cut segment at
    least m tiles long."""
    sl = np.array(lens, dtype=np.int32)
    cap = max(64, max(lens))
    la = oracle.plan(sl, Hkv, kind=3, num_ctas=P, param=m, capacity_tokens=cap, tail=(8, 4, 0),
                     cost=(q, e))
    dyn = oracle.plan(sl, Hkv, kind=0, num_ctas=P, capacity_tokens=cap, tail=(8, 4, 0),
                      cost=(q, e))
    # coverage, contiguity, consecutive holders and partial slots
    _check_plan_invariants(la, lens, Hkv, 3)
    assert la["ranges"] == dyn["ranges"]
    units = _units(lens, Hkv)
    seg_n = {}
    for (b, g, t) in units:
        seg_n[(b, g)] = seg_n.get((b, g), 0) + 1
    pieces = {}
    for c in range(la["ranges"]):
        a, e = int(la["cta"][c, 0]), int(la["cta"][c, 1])
        assert abs(a - int(dyn["cta"][c, 0])) < m and abs(e - int(dyn["cta"][c, 1])) < m
        for u in range(a, e):
            key = units[u][:2]
            if u == a or units[u - 1][:2] != key:
                pieces.setdefault(key, []).append(0)
            pieces[key][-1] += 1
    for key, ps in pieces.items():
        if seg_n[key] < 2 * m:
            assert len(ps) == 1
        if len(ps) > 1:
            assert ps[0] >= m and ps[-1] >= m
    # never more pieces than the dynamic plan cuts the segment into
    for s in range(len(lens) * Hkv):
        assert la["split_count"][s] <= dyn["split_count"][s]


@settings(max_examples=60, deadline=None)
@given(lens=lens_st, N=st.integers(1, 9), extra=st.integers(0, 3), seed=st.integers(0, 99))
def test_page_shard_properties(lens, N, extra, seed):
    L = np.array(lens, dtype=np.int32)
    pts = int((L.max() + 63) // 64) + extra + 1
    pt = np.arange(len(lens) * pts, dtype=np.int32).reshape(len(lens), pts)
    start = np.random.default_rng(seed).integers(0, N, len(lens))
    shares = [SH.page_shard(torch.from_numpy(L), torch.from_numpy(pt), N, r,
                            start=torch.from_numpy(start)) for r in range(N)]
    np.testing.assert_array_equal(sum(s[0].numpy().astype(np.int64) for s in shares), L)
    for b in range(len(lens)):
        n = (int(L[b]) + 63) // 64
        got = {}
        for r, (lr, ptr) in enumerate(shares):
            k = (int(lr[b]) + 63) // 64
            for p in ptr.numpy()[b, :k].tolist():
                got[p] = r
        # every page once, on the rank the rule names
        assert sorted(got) == pt[b, :n].tolist()
        for t in range(n):
            assert got[int(pt[b, t])] == (int(start[b]) + t) % N
        sizes = [(int(lr[b]) + 63) // 64 for lr, _ in shares]
        assert max(sizes) - min(sizes) <= 1        # shares even to within a tile


@settings(max_examples=60, deadline=None)
@given(lens=lens_st, Hkv=st.sampled_from([1, 2, 4, 8]), P=st.integers(1, 300),
       kind=st.sampled_from([0, 1, 2]), param=st.integers(0, 9),
       den=st.integers(0, 40), k=st.integers(1, 4), mn=st.integers(0, 40),
       q=st.integers(1, 4), e=st.integers(0, 4))
def test_plan_kinds_properties(lens, Hkv, P, kind, param, den, k, mn, q, e):
    """Every plan kind covers each unit exactly once with contiguous ranges,
    consecutive holders per segment and distinct partial slots; a dynamic plan
    of any tail shape (den, k, mn) and cost weights (q, e) has the primary
    ranges of even cost and the even tail chunks of that shape."""
    sl = np.array(lens, dtype=np.int32)
    cap = max(64, max(lens))
    p = oracle.plan(sl, Hkv, kind=kind, num_ctas=P, param=param if kind else 0,
                    max_seq_len=max(lens), capacity_tokens=cap, tail=(den, k, mn), cost=(q, e))
    _check_plan_invariants(p, lens, Hkv, kind, (den, k, mn), (q, e))
    assert p["n_units"] == len(_units(lens, Hkv))


@settings(max_examples=60, deadline=None)
@given(lens=lens_st, Hkv=st.sampled_from([1, 2, 4, 8]), P=st.integers(1, 300),
       den=st.integers(1, 40), k=st.integers(1, 4))
def test_dynamic_tail_covers_the_last_units_evenly(lens, Hkv, P, den, k):
    """Whatever the tail shape, the tail chunks are the last units of the list,
    in order, each within one unit of the others, and the primary ranges the
    units before them, also within one unit of each other."""
    sl = np.array(lens, dtype=np.int32)
    p = oracle.plan(sl, Hkv, kind=0, num_ctas=P, capacity_tokens=max(64, max(lens)),
                    tail=(den, k, 0))
    U, R = p["n_units"], p["ranges"]
    if U <= P:
        return
    sizes = [int(e - a) for a, e in p["cta"]]
    prim, chunks = sizes[:P], sizes[P:]
    assert min(prim) >= 1 and max(prim) - min(prim) <= 1
    assert sum(prim) + sum(chunks) == U
    if chunks:
        assert min(chunks) >= 1 and max(chunks) - min(chunks) <= 1
        assert int(p["cta"][P][0]) == sum(prim) and int(p["cta"][R - 1][1]) == U
