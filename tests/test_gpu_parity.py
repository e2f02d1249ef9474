"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Tolerances (bf16 output): max-abs <= 2e-2, mean-abs <= 2e-3; FP8 caches:
max-abs <= 5e-2.  Split schedules must agree with one another within 1e-3 in
fp32 output; plans and slot writes are compared bit for bit.
"""
from __future__ import annotations

import copy
import math
import zlib

import numpy as np
import pytest
import torch

import oracle
import mixed_length_paged_b200 as hpa
from mixed_length_paged_b200 import workloads as W
from tests.helpers import (bf16_values, bits16, check_rows_relative, compact_rows, errors,
                           gpu_decode, gpu_decode_multi, oracle_decode, quantize_fp8, to_device)

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS, FP8_MAX_ABS, SCHED_TOL = 2e-2, 2e-3, 5e-2, 1e-3


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixed_length_paged_b200 import build
    build.build()
    hpa.lib()


def _check(out, ref, max_abs=MAX_ABS, mean_abs=MEAN_ABS, rows=None):
    if rows is not None:
        out, ref = out[list(rows)], ref[list(rows)]
    assert torch.isfinite(out.float()).all()
    mx, mn = errors(out, ref)
    assert mx <= max_abs and mn <= mean_abs, (mx, mn)
    return mx, mn


# ---------------------------------------------------------------- plan

def _read_plan(ws, kind, B, Hkv, Hq, D, grid):
    lay = hpa.workspace_layout(kind, B, Hkv, Hq, D, grid)
    w = ws.cpu().numpy()

    def i32(off, n):
        return w[off:off + 4 * n].view(np.int32)

    S = B * Hkv
    header = i32(lay["header"], 32)
    V = int(header[10])
    return {
        "header": header, "lens": i32(lay["lens"], B),
        "tile_start": i32(lay["tile_start"], B + 1),
        "cta": i32(lay["cta_desc"], 8 * V).reshape(V, 8),
        "seg": i32(lay["seg_desc"], 2 * S).reshape(S, 2),
    }


# The library's member of the dynamic plan family (hpa.h: HPA_TAIL_*_DEFAULT,
# HPA_COST_*_DEFAULT); other members are called with hpa_decode_plan_shape.
LIB_TAIL = (8, 4, 32)
LIB_COST = (hpa.COST_UNIT_DEFAULT, hpa.COST_END_DEFAULT)


@pytest.mark.parametrize("lens,Hkv,P", [
    ([131072] + [4096] * 31, 8, 148), ([512] * 64, 8, 148), ([37, 200], 2, 148),
    ([37, 200], 2, 3), ([0, 5, 0, 64, 65, 3000, 1], 4, 7), ([1], 1, 148), ([0, 0], 2, 5),
    (list(range(1, 3000, 7)), 2, 148),
    # cost weights on: a range's share below a segment end's cost, so the
    # plan falls back to the even split of the units
    ([65, 65], 8, 27),
    # beyond 12K sequences the tile offsets need more than 48 KiB of shared memory
    ([int(x) for x in np.random.default_rng(3).integers(0, 300, 20000)], 2, 148),
    ([int(x) for x in np.random.default_rng(4).integers(1, 100, 32768)], 1, 148),  # the maximum
])
@pytest.mark.parametrize("kind,param,tail,cost", [
    (0, 0, None, None), (1, 0, None, None), (1, 3, None, None), (2, 0, None, None),
    (2, 5, None, None), (3, 0, None, None), (3, 2, None, None), (3, 9, None, None),
    (0, 0, (0, 1, 0), None), (0, 0, (8, 4, 0), None), (0, 0, (3, 1, 0), None),
    (0, 0, (16, 2, 3), None), (0, 0, (1, 4, 0), None), (3, 4, (0, 1, 0), None),
    (3, 2, (5, 3, 0), None),
    (0, 0, (0, 1, 0), (1, 0)), (0, 0, (0, 1, 0), (1, 1)), (0, 0, (8, 4, 0), (2, 1)),
    (0, 0, (8, 4, 32), (4, 3)), (0, 0, (0, 1, 0), (1, 4)), (0, 0, (3, 1, 0), (3, 0)),
    (0, 0, None, (2, 1)), (3, 2, (8, 4, 0), (2, 1)), (3, 4, (0, 1, 0), (1, 2))])
def test_plan_is_bit_exact(lens, Hkv, P, kind, param, tail, cost):
    """tail and cost None: hpa_decode_plan (the library's default shape,
    LIB_TAIL and LIB_COST); else hpa_decode_plan_shape with that tail shape
    ((0, 1, 0) = no tail) and cost weights ((1, 0) = units split evenly), the
    default for whichever is None."""
    B, Hq, D = len(lens), Hkv * 2, 64
    cap = max(64, max(lens))
    pts = (cap + 63) // 64
    maxlen = max(lens)
    grid = hpa.plan_grid(kind, B, Hkv, P, param, maxlen)
    ref = oracle.plan(np.array(lens, dtype=np.int32), Hkv, kind=kind, num_ctas=P, param=param,
                      max_seq_len=maxlen, capacity_tokens=pts * 64,
                      tail=LIB_TAIL if tail is None else tail,
                      cost=LIB_COST if cost is None else cost)
    assert grid == ref["grid"]
    ws = torch.full((hpa.decode_workspace_size(kind, B, Hkv, Hq, D, grid),), 0xAB,
                    dtype=torch.uint8, device="cuda")
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    g = hpa.decode_plan(sl, num_kv_heads=Hkv, num_q_heads=Hq, head_dim=D, pt_stride=pts,
                        workspace=ws, kind=kind, num_ctas=P, param=param, max_seq_len=maxlen,
                        tail=tail, cost=cost)
    torch.cuda.synchronize()
    assert g == grid
    got = _read_plan(ws, kind, B, Hkv, Hq, D, grid)
    assert got["header"][10] == ref["ranges"]
    np.testing.assert_array_equal(got["lens"], ref["lens"])
    np.testing.assert_array_equal(got["tile_start"], ref["tile_start"])
    np.testing.assert_array_equal(got["cta"][:, :2], ref["cta"])
    assert not got["cta"][:, 6:].any()
    # start state (b, g, t, tiles of b) of each CTA's first unit, from the oracle's offsets
    ts = ref["tile_start"].astype(np.int64)
    for c in range(ref["ranges"]):
        ub, ue = int(ref["cta"][c, 0]), int(ref["cta"][c, 1])
        if ub == ue:
            continue
        b0 = int(np.searchsorted(ts * Hkv, ub, side="right") - 1)
        n0 = int(ts[b0 + 1] - ts[b0])
        rem = ub - int(ts[b0]) * Hkv
        assert tuple(got["cta"][c, [2, 3, 4, 5]]) == (b0, rem // n0, rem % n0, n0), c
    np.testing.assert_array_equal(got["seg"][:, 0], ref["first_slot"])
    np.testing.assert_array_equal(got["seg"][:, 1], ref["split_count"])
    h = got["header"]
    assert h[2] == ref["n_units"] and h[3] == grid and h[1] == 0
    # the tail shape the plan was made with, recorded in the header
    want = (LIB_TAIL if tail is None else tail) if kind in (0, 3) else (0, 0, 0)
    assert (int(h[13]), int(h[14]), int(h[15])) == want
    want = (LIB_COST if cost is None else cost) if kind in (0, 3) else (0, 0)
    assert (int(h[19]), int(h[20])) == want


def test_plan_flags_clamped_lengths():
    sl = torch.tensor([-3, 100, 10_000], dtype=torch.int32, device="cuda")
    ws = torch.zeros(hpa.decode_workspace_size(0, 3, 2, 4, 64, 148), dtype=torch.uint8,
                     device="cuda")
    hpa.decode_plan(sl, num_kv_heads=2, num_q_heads=4, head_dim=64, pt_stride=4, workspace=ws,
                    num_ctas=148)
    assert hpa.read_status(ws) & hpa.DEVICE_LEN_CLAMPED
    got = _read_plan(ws, 0, 3, 2, 4, 64, 148)
    np.testing.assert_array_equal(got["lens"], [0, 100, 256])


# ---------------------------------------------------------------- small cases

SMALL = [
    # name, lens, Hq, Hkv, D
    ("tiny", [37, 200], 8, 2, 64),
    ("ragged_g4_d128", [1, 63, 64, 65, 300, 1000, 2047, 5000], 16, 4, 128),
    ("g8", [129, 1, 700, 64], 64, 8, 128),
    ("g1", [90, 257], 4, 4, 128),
    ("g2_d64", [33, 400, 1], 8, 4, 64),
    ("g16", [200, 1500], 32, 2, 128),
    ("b1", [3333], 8, 1, 128),
    # group sizes that are not powers of two (rows padded to n-tiles of 8)
    ("g7", [300, 64, 4100], 28, 4, 128),
    ("g12", [129, 2000], 96, 8, 128),
    ("g3_d64", [65, 1, 777], 6, 2, 64),
    ("g5", [5000], 5, 1, 128),
]


@pytest.mark.parametrize("name,lens,Hq,Hkv,D", SMALL)
@pytest.mark.parametrize("num_ctas", [None, 7, 1])
def test_decode_matches_oracle_small(name, lens, Hq, Hkv, D, num_ctas):
    batch = W.make_batch(W.DecodeShape(name, Hq, Hkv, D), lens, seed=zlib.crc32(name.encode()) % 1000)
    ref = oracle_decode(batch)
    to_device(batch)
    out = gpu_decode(batch, num_ctas=num_ctas)
    _check(out, ref)
    out32 = gpu_decode(batch, num_ctas=num_ctas, out_dtype=torch.float32)
    mx, _ = errors(out32, ref)
    assert mx <= 5e-3, mx


def test_tiny_workload_exact_config():
    batch = W.build("tiny")
    ref = oracle_decode(batch)
    out = gpu_decode(to_device(batch))
    _check(out, ref)


def test_length_one_returns_v_row():
    batch = W.make_batch(W.DecodeShape("l1", 16, 2, 128), [1, 1, 1], seed=5)
    out = gpu_decode(to_device(batch), out_dtype=torch.float32).cpu()
    vv = batch.v_cache.float().cpu()
    pt = batch.page_table.cpu()
    for b in range(3):
        for h in range(16):
            torch.testing.assert_close(out[b, h], vv[pt[b, 0], h // 8, 0], rtol=0, atol=0)


def test_zero_length_sequence_gives_zeros():
    batch = W.make_batch(W.DecodeShape("z", 8, 2, 64), [0, 100, 0], seed=6)
    ref = oracle_decode(batch)
    out = gpu_decode(to_device(batch))
    assert torch.all(out[0] == 0) and torch.all(out[2] == 0)
    _check(out, ref)


def test_page_permutation_invariance_on_gpu():
    batch = W.make_batch(W.DecodeShape("perm", 16, 4, 128), [700, 33, 2000], seed=8)
    to_device(batch)
    out1 = gpu_decode(batch, out_dtype=torch.float32)
    perm = torch.randperm(batch.num_pages, generator=torch.Generator().manual_seed(1)).cuda()
    k2 = torch.empty_like(batch.k_cache)
    v2 = torch.empty_like(batch.v_cache)
    k2[perm] = batch.k_cache
    v2[perm] = batch.v_cache
    pt = batch.page_table.clone()
    m = pt >= 0
    pt[m] = perm[pt[m].long()].int()
    batch.k_cache, batch.v_cache, batch.page_table = k2, v2, pt
    out2 = gpu_decode(batch, out_dtype=torch.float32)
    assert torch.equal(out1, out2)


def test_repeated_steps_are_deterministic():
    batch = W.make_batch(W.DecodeShape("rep", 64, 8, 128), [5000, 64, 9000, 1], seed=9)
    to_device(batch)
    outs = [gpu_decode(batch, num_ctas=37, out_dtype=torch.float32) for _ in range(3)]
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])


# ---------------------------------------------------------------- schedules

@pytest.mark.parametrize("lens", [[131072 // 8] + [4096 // 8] * 31, [1, 63, 64, 65, 300, 5000]])
def test_split_schedules_agree(lens):
    batch = W.make_batch(W.DecodeShape("sched", 64, 8, 128), lens, seed=10)
    ref = oracle_decode(batch)
    to_device(batch)
    U = sum((L + 63) // 64 for L in lens) * 8
    plans = [(0, None, 0), (0, 1, 0), (0, U, 0), (0, 37, 0), (1, None, 0), (1, None, 3),
             (2, None, 0), (2, None, 1), (2, None, 7), (3, None, 0), (3, 37, 2), (3, None, 16),
             (3, U, 3)]
    outs = []
    for kind, nc, param in plans:
        o = gpu_decode(batch, kind=kind, num_ctas=nc, param=param, out_dtype=torch.float32)
        mx, _ = errors(o, ref)
        assert mx <= 5e-3, (kind, nc, param, mx)
        outs.append(o)
    for o in outs[1:]:
        assert (o - outs[0]).abs().max().item() <= SCHED_TOL


def test_length_aware_plan_with_unit_pieces_is_the_dynamic_plan():
    # smallest piece 1 tile: no cut moves, so the same ranges, partials and bits
    batch = W.make_batch(W.DecodeShape("la1", 64, 8, 128), [9000, 64, 1, 700, 2047, 0], seed=11)
    to_device(batch)
    a = gpu_decode(batch, kind=hpa.PLAN_DYNAMIC, out_dtype=torch.float32)
    b = gpu_decode(batch, kind=hpa.PLAN_LENGTH_AWARE, param=1, out_dtype=torch.float32)
    assert torch.equal(a, b)


@pytest.mark.parametrize("name,lens", [
    ("uniform_small", [512] * 64),
    ("mixed", [1, 63, 64, 65, 300, 5000, 129, 4096, 0, 7]),
])
@pytest.mark.parametrize("param", [0, 3])
def test_length_aware_plan_matches_oracle(name, lens, param):
    batch = W.make_batch(W.DecodeShape(name, 64, 8, 128), lens, seed=12)
    ref = oracle_decode(batch)
    to_device(batch)
    out = gpu_decode(batch, kind=hpa.PLAN_LENGTH_AWARE, param=param)
    _check(out, ref)
    ws = gpu_decode(batch, kind=hpa.PLAN_LENGTH_AWARE, param=param, return_ws=True)[1]
    assert hpa.read_status(ws) == 0


# ---------------------------------------------------------------- named workloads

def test_uniform_workload():
    batch = W.build("uniform")
    ref = oracle_decode(batch)
    out = gpu_decode(to_device(batch))
    _check(out, ref)


def _bench_step(batch, out_dtype=torch.bfloat16):
    """The benchmark's launch: hpa_decode_step (plan inside the decode kernel)
    over the persistent CTA count hpa_decode_num_ctas gives."""
    B, Hq, D = batch.batch, batch.shape.num_q_heads, batch.shape.head_dim
    Hkv = batch.shape.num_kv_heads
    dec = hpa.PagedDecoder(B, Hq, Hkv, D, batch.pt_stride)
    out = torch.full((B, Hq, D), float("nan"), dtype=out_dtype, device="cuda")
    dec.step(batch.q, batch.k_cache, batch.v_cache, batch.page_table, batch.seq_lens, out,
             1.0 / math.sqrt(D))
    torch.cuda.synchronize()
    assert dec.status() == 0
    return out


def test_skewed_workload_all_rows():
    """The whole skewed batch (1 x 131072 + 31 x 4096) against the oracle, every
    row, in the benchmark's launch and through plan + run; each row also
    within 5 % of its own magnitude, so a wrong 128K row cannot hide under the
    absolute tolerance."""
    batch = W.build("skewed", device="cuda")
    ref = oracle_decode(batch)
    for out in (_bench_step(batch), gpu_decode(batch)):
        _check(out, ref)
        check_rows_relative(out, ref)
    outA = gpu_decode(batch, kind=1, out_dtype=torch.float32)
    outD = gpu_decode(batch, out_dtype=torch.float32)
    assert (outA - outD).abs().max().item() <= SCHED_TOL


def test_needle_in_the_128k_sequence_full_batch():
    """Needle pin of the page mapping at scale, on the full skewed batch in the
    benchmark's launch: for one query head h of every kv group g, the key at a
    random position j_g of the 131072-token sequence is set to
    40 q_h / |q_h| (a logit of ~40 against N(0, 1) logits), so head h's output
    is V[j_g] to within bf16 rounding while the other heads of the group stay
    far from it.  The sequence is spread over ~74 CTAs per kv head, so this
    checks the tile-to-page mapping, the split and the merge together."""
    batch = W.build("skewed", device="cuda")
    G, D = batch.shape.group, batch.shape.head_dim
    rng = np.random.default_rng(2024)
    planted = []
    for g in range(batch.shape.num_kv_heads):
        h = g * G + int(rng.integers(0, G))
        j = int(rng.integers(0, 131072))
        qh = batch.q[0, h].float()
        batch.k_cache[int(batch.page_table[0, j // 64]), g, j % 64] = \
            (40.0 * qh / qh.norm()).to(torch.bfloat16)
        planted.append((g, h, j))
    for out in (_bench_step(batch), gpu_decode(batch, num_ctas=37)):
        o = out[0].float()
        for g, h, j in planted:
            v = batch.v_cache[int(batch.page_table[0, j // 64]), g, j % 64].float()
            assert (o[h] - v).abs().max().item() <= MAX_ABS, (g, h, j)
            for h2 in range(g * G, (g + 1) * G):
                if h2 != h:
                    assert (o[h2] - v).abs().max().item() > 0.5, (g, h2, j)


def test_fp8_small():
    shape = W.DecodeShape("f8", 64, 8, 128, kv_dtype="fp8_e4m3")
    batch = W.make_batch(shape, [1, 63, 64, 65, 700, 3000], seed=12)
    fp8 = quantize_fp8(batch)
    ref = oracle_decode(batch, fp8=fp8)
    to_device(batch)
    for nc in (None, 5):
        out = gpu_decode(batch, fp8=fp8, num_ctas=nc)
        _check(out, ref, max_abs=FP8_MAX_ABS, mean_abs=MEAN_ABS)


def test_fp8_workload_sampled_rows():
    batch = W.build("fp8", device="cuda")
    fp8 = quantize_fp8(batch)
    out = gpu_decode(batch, fp8=fp8)
    L = batch.seq_lens.cpu().numpy()
    rows = [int(np.argmax(L)), int(np.argmin(L)), 0, 100, 255]
    ref = oracle_decode(batch, fp8=fp8, rows=np.array(rows, dtype=np.int32))
    _check(out, ref, max_abs=FP8_MAX_ABS, rows=rows)


# ---------------------------------------------------------------- prologue

def _prologue_case(lens, Hq=32, Hkv=8, D=128, seed=13, device="cpu"):
    shape = W.DecodeShape("pro", Hq, Hkv, D, prologue=True)
    return W.make_batch(shape, lens, seed=seed, device=device)


def _run_prologue(batch):
    B, Hq, D = batch.q_raw.shape
    q_out = torch.empty_like(batch.q_raw)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    hpa.kv_prologue(batch.q_raw, batch.k_raw, batch.v_raw, batch.q_gamma, batch.k_gamma,
                    batch.positions, batch.page_table, batch.k_cache, batch.v_cache, q_out,
                    eps=1e-6, rope_theta=10000.0, status=status)
    torch.cuda.synchronize()
    return q_out, int(status.item())


@pytest.mark.parametrize("D", [64, 128])
def test_prologue_slot_writes_and_attention(D):
    lens = [0, 63, 64, 127, 1000, 4095]
    batch = _prologue_case(lens, Hq=16, Hkv=4, D=D)
    kc, vc = bits16(batch.k_cache).copy(), bits16(batch.v_cache).copy()
    pt = batch.page_table.numpy()
    q64 = oracle.prologue(bits16(batch.q_raw), bits16(batch.k_raw), bits16(batch.v_raw),
                          batch.q_gamma.numpy(), batch.k_gamma.numpy(), 1e-6, 1e4,
                          batch.positions.numpy(), pt, kc, vc)
    to_device(batch)
    q_out, status = _run_prologue(batch)
    assert status == 0
    gk, gv = bits16(batch.k_cache), bits16(batch.v_cache)
    # V slots and every untouched byte: bit-exact
    np.testing.assert_array_equal(gv, vc)
    diff = gk != kc
    # K slots: equal up to one bf16 ulp (fp32 vs fp64 rounding at a tie)
    touched = np.zeros(diff.shape[:3], dtype=bool)
    for b, pos in enumerate(lens):
        touched[pt[b, pos // 64], :, pos % 64] = True
    assert not diff[~touched].any()
    a, b_ = gk[touched].astype(np.int32), kc[touched].astype(np.int32)
    assert np.all(np.abs(a - b_) <= 1)
    # q_out against the oracle's fp64 prologue
    qg = bf16_values(bits16(q_out))
    assert np.abs(qg - q64).max() <= np.abs(q64).max() * 2.0 ** -8 + 1e-6
    # attention over the appended token
    ref = oracle.paged_decode(q64, kc, vc, pt, batch.seq_lens.cpu().numpy(), 4, 1 / math.sqrt(D))
    out = gpu_decode(batch, q=q_out)
    _check(out, ref)


def test_prologue_bad_position_is_flagged_not_written():
    batch = _prologue_case([10, 20], Hq=8, Hkv=2, D=64)
    batch.positions[1] = 10_000  # beyond the page table
    before = bits16(batch.k_cache).copy()
    to_device(batch)
    _, status = _run_prologue(batch)
    assert status & hpa.DEVICE_BAD_POSITION
    after = bits16(batch.k_cache)
    changed = np.argwhere((after != before).any(axis=-1))
    assert len(changed) == 2  # sequence 0's K row for its two kv heads only


def test_mix_prologue_workload_all_rows():
    """The whole 128-sequence continuous-batching mix with the prologue, every
    row against the oracle's prologue + attention, in the benchmark's launch
    (hpa_decode_step_prologue) and as prologue kernel + plan + run; each row
    also within 5 % of its own magnitude."""
    batch = W.build("mix_prologue", device="cuda")
    host = copy.copy(batch)
    for name in ("q_raw", "k_raw", "v_raw", "positions", "page_table", "seq_lens"):
        setattr(host, name, getattr(batch, name).cpu())
    kc, vc = bits16(batch.k_cache).copy(), bits16(batch.v_cache).copy()
    q64 = oracle.prologue(bits16(host.q_raw), bits16(host.k_raw), bits16(host.v_raw),
                          batch.q_gamma.cpu().numpy(), batch.k_gamma.cpu().numpy(), 1e-6, 1e4,
                          host.positions.numpy(), host.page_table.numpy(), kc, vc)
    ref = oracle.paged_decode(q64, kc, vc, host.page_table.numpy(), host.seq_lens.numpy(), 8,
                              1 / math.sqrt(128))
    del kc, vc
    B, Hq, D = batch.q_raw.shape
    kc0, vc0 = batch.k_cache.clone(), batch.v_cache.clone()
    # 1. the benchmark's launch: the whole step in two launches
    dec = hpa.PagedDecoder(B, Hq, 8, D, batch.pt_stride)
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    dec.step_prologue(batch.q_raw, batch.k_raw, batch.v_raw, batch.q_gamma, batch.k_gamma,
                      batch.k_cache, batch.v_cache, batch.page_table, batch.seq_lens, out,
                      1 / math.sqrt(D), eps=1e-6, rope_theta=1e4)
    torch.cuda.synchronize()
    assert dec.status() == 0
    _check(out, ref)
    check_rows_relative(out, ref)
    # 2. prologue kernel, then plan + run, on fresh copies of the caches
    batch.k_cache.copy_(kc0)
    batch.v_cache.copy_(vc0)
    del kc0, vc0
    q_out, status = _run_prologue(batch)
    assert status == 0
    out2 = gpu_decode(batch, q=q_out)
    _check(out2, ref)
    check_rows_relative(out2, ref)


# ---------------------------------------------------------------- multi-token decode

# pre-step lengths: new tokens straddling a page edge, a sequence exactly T
# long, one shorter than T (its first queries see nothing), an empty one,
# several pages, a long one
MT_LENS = [65, 200, 2, 0, 1000, 64, 4097, 130]


@pytest.mark.parametrize("Hq,Hkv,D,T", [(64, 8, 128, 2), (32, 8, 128, 4), (8, 4, 64, 8),
                                        (4, 4, 128, 16), (16, 2, 64, 2), (12, 4, 128, 5)])
@pytest.mark.parametrize("kind,num_ctas", [(0, None), (0, 5), (1, None), (2, 7), (3, None),
                                            (3, 5)])
def test_multi_token_decode_matches_oracle(Hq, Hkv, D, T, kind, num_ctas):
    batch = W.make_batch(W.DecodeShape("mt", Hq, Hkv, D, q_tokens=T), MT_LENS, seed=31)
    ref = oracle.paged_decode_multi(bits16(batch.q), bits16(batch.k_cache),
                                    bits16(batch.v_cache), batch.page_table.numpy(),
                                    batch.seq_lens.numpy(), Hkv, 1 / math.sqrt(D))
    out = gpu_decode_multi(batch, kind=kind, num_ctas=num_ctas, out_dtype=torch.float32)
    _check(out, ref)


@pytest.mark.parametrize("Hq,Hkv,D,T,fp8", [
    (64, 8, 128, 4, False),   # G = 8, four query tokens: 32 rows
    (32, 2, 128, 2, False),   # G = 16, two tokens
    (24, 2, 64, 2, False),    # 24 rows: padded to four n-tiles
    (64, 8, 128, 3, True),    # 24 rows, FP8 KV
    (32, 1, 128, 1, False),   # one kv head for 32 query heads, single token
    (24, 1, 64, 1, False),
])
@pytest.mark.parametrize("kind,num_ctas", [(0, None), (0, 7), (1, None), (2, None), (3, None)])
def test_wide_query_groups_match_oracle(Hq, Hkv, D, T, fp8, kind, num_ctas):
    """17..32 query rows per kv head (G x T): one warp per MMA n-tile over the
    whole tile, two CTAs per SM (one per SM for small grids), against the
    oracle on every plan kind."""
    shape = W.DecodeShape("wide", Hq, Hkv, D, kv_dtype="fp8_e4m3" if fp8 else "bf16",
                          q_tokens=T)
    batch = W.make_batch(shape, MT_LENS, seed=35)
    q8 = quantize_fp8(batch) if fp8 else None
    kc, vc = (bits16(batch.k_cache), bits16(batch.v_cache)) if q8 is None else (q8[0], q8[2])
    kw = {} if q8 is None else dict(kv_fp8=True, k_scale=q8[1], v_scale=q8[3])
    if T == 1:
        ref = oracle.paged_decode(bits16(batch.q), kc, vc, batch.page_table.numpy(),
                                  batch.seq_lens.numpy(), Hkv, 1 / math.sqrt(D), **kw)
        to_device(batch)
        out = gpu_decode(batch, kind=kind, num_ctas=num_ctas, out_dtype=torch.float32, fp8=q8)
    else:
        ref = oracle.paged_decode_multi(bits16(batch.q), kc, vc, batch.page_table.numpy(),
                                        batch.seq_lens.numpy(), Hkv, 1 / math.sqrt(D), **kw)
        out = gpu_decode_multi(batch, kind=kind, num_ctas=num_ctas, out_dtype=torch.float32,
                               fp8=q8)
    _check(out, ref, max_abs=FP8_MAX_ABS if fp8 else MAX_ABS)


def test_decode_num_ctas_matches_residency():
    two = hpa.default_num_ctas()
    # 8 rows per kv head, 16 (two n-tiles, warps split by n-tile) and 17..32
    # (four n-tiles, one deposit buffer): 2 CTAs / SM
    for args in ((64, 8, 1), (64, 8, 2), (32, 2, 1), (8, 2, 2), (64, 8, 3), (64, 8, 4),
                 (32, 1, 1), (24, 2, 2)):
        assert hpa.decode_num_ctas(*args) == two, args


def test_multi_token_fp8_and_bf16_out():
    shape = W.DecodeShape("mt8", 32, 8, 128, kv_dtype="fp8_e4m3", q_tokens=2)
    batch = W.make_batch(shape, [1, 63, 64, 65, 700, 3000], seed=32)
    fp8 = quantize_fp8(batch)
    kc, ks, vc, vs = fp8
    ref = oracle.paged_decode_multi(bits16(batch.q), kc, vc, batch.page_table.numpy(),
                                    batch.seq_lens.numpy(), 8, 1 / math.sqrt(128), kv_fp8=True,
                                    k_scale=ks, v_scale=vs)
    out = gpu_decode_multi(batch, fp8=fp8)
    _check(out, ref, max_abs=FP8_MAX_ABS)


def test_length_aware_plan_fp8():
    shape = W.DecodeShape("la8", 64, 8, 128, kv_dtype="fp8_e4m3")
    batch = W.make_batch(shape, [1, 63, 64, 65, 700, 3000, 511, 512, 513], seed=34)
    fp8 = quantize_fp8(batch)
    ref = oracle_decode(batch, fp8=fp8)
    to_device(batch)
    for param, nc in ((0, None), (3, 7)):
        out = gpu_decode(batch, kind=hpa.PLAN_LENGTH_AWARE, param=param, num_ctas=nc, fp8=fp8)
        _check(out, ref, max_abs=FP8_MAX_ABS, mean_abs=MEAN_ABS)


def test_multi_token_one_token_equals_single_token_run():
    # q_tokens = 1 through the multi-token entry is the regular run, bit for bit
    batch = W.make_batch(W.DecodeShape("mt1", 64, 8, 128, q_tokens=1), [100, 5000, 3], seed=33)
    to_device(batch)
    single = gpu_decode(batch, out_dtype=torch.float32)
    batch.q = batch.q.unsqueeze(1)
    multi = gpu_decode_multi(batch, out_dtype=torch.float32)
    assert torch.equal(single, multi[:, 0])


def test_multi_token_workload_sampled_rows():
    batch = W.build("skewed_mtp2", device="cuda")
    out = gpu_decode_multi(batch)
    rows = [0, 1, 31]
    small = compact_rows(batch, rows)
    small.q = batch.q[rows].cpu()
    ref = oracle.paged_decode_multi(bits16(small.q), bits16(small.k_cache),
                                    bits16(small.v_cache), small.page_table.numpy(),
                                    small.seq_lens.numpy(), 8, 1 / math.sqrt(128))
    _check(out[rows], ref)


# ---------------------------------------------------------------- fused prologue

def _separate_and_fused(batch, *, kind=0, num_ctas=None, param=0, out_dtype=torch.bfloat16,
                        with_q_out=True):
    """The same step twice on copies of the caches: prologue kernel -> plan ->
    run, and plan -> run with the prologue fused in."""
    B, Hq, D = batch.q_raw.shape
    Hkv = batch.k_raw.shape[1]
    n = num_ctas or hpa.default_num_ctas()
    maxlen = int(batch.seq_lens.max().item())
    grid = hpa.plan_grid(kind, B, Hkv, n, param, maxlen)
    res = []
    for fused in (False, True):
        kc, vc = batch.k_cache.clone(), batch.v_cache.clone()
        q_out = torch.full_like(batch.q_raw, float("nan")) if (with_q_out or not fused) else None
        ws = torch.zeros(hpa.decode_workspace_size(kind, B, Hkv, Hq, D, grid), dtype=torch.uint8,
                         device="cuda")
        out = torch.full((B, Hq, D), float("nan"), dtype=out_dtype, device="cuda")
        if not fused:
            hpa.kv_prologue(batch.q_raw, batch.k_raw, batch.v_raw, batch.q_gamma, batch.k_gamma,
                            batch.positions, batch.page_table, kc, vc, q_out, eps=1e-6,
                            rope_theta=10000.0)
        hpa.decode_plan(batch.seq_lens, num_kv_heads=Hkv, num_q_heads=Hq, head_dim=D,
                        pt_stride=batch.pt_stride, workspace=ws, kind=kind, num_ctas=n,
                        param=param, max_seq_len=maxlen)
        if fused:
            hpa.decode_run_prologue(batch.q_raw, batch.k_raw, batch.v_raw, batch.q_gamma,
                                    batch.k_gamma, kc, vc, batch.page_table, out, ws, grid,
                                    1.0 / math.sqrt(D), q_out=q_out, eps=1e-6, rope_theta=1e4,
                                    kind=kind)
        else:
            hpa.decode_run(q_out, kc, vc, batch.page_table, out, ws, grid, 1.0 / math.sqrt(D),
                           kind=kind)
        torch.cuda.synchronize()
        assert hpa.read_status(ws) == 0
        res.append((out, kc, vc, q_out))
    return res


@pytest.mark.parametrize("D,Hq,Hkv", [(128, 32, 8), (64, 16, 4), (128, 16, 1), (128, 32, 2)])
@pytest.mark.parametrize("kind,num_ctas", [(0, None), (0, 5), (1, None), (2, 7), (3, 7)])
def test_fused_prologue_bitwise_equals_separate(D, Hq, Hkv, kind, num_ctas):
    # pre-append lengths: a first token, page edges, several pages, one long
    lens = [0, 63, 64, 127, 1000, 4095, 1]
    batch = _prologue_case(lens, Hq=Hq, Hkv=Hkv, D=D)
    to_device(batch)
    (oa, ka, va, qa), (ob, kb, vb, qb) = _separate_and_fused(batch, kind=kind, num_ctas=num_ctas)
    # same bits: the caches (new slots and every other byte), q_out, and the output
    assert torch.equal(bits_t(ka), bits_t(kb)) and torch.equal(bits_t(va), bits_t(vb))
    assert torch.equal(bits_t(qa), bits_t(qb))
    assert torch.equal(bits_t(oa), bits_t(ob))


@pytest.mark.parametrize("D,Hq,Hkv,num_ctas", [(128, 32, 8, None), (64, 16, 4, 5),
                                                (128, 16, 1, None), (128, 32, 2, 7)])
def test_step_prologue_bitwise_equals_separate(D, Hq, Hkv, num_ctas):
    """The whole step in two launches (prologue + plan inside the decode
    kernel) against prologue kernel -> plan kernel -> run: same bits in the
    output, q_out and both caches."""
    lens = [0, 63, 64, 127, 1000, 4095, 1]
    batch = _prologue_case(lens, Hq=Hq, Hkv=Hkv, D=D)
    to_device(batch)
    (oa, ka, va, qa), _ = _separate_and_fused(batch, num_ctas=num_ctas)
    B = batch.batch
    n = num_ctas or hpa.default_num_ctas()
    kc, vc = batch.k_cache.clone(), batch.v_cache.clone()
    q_out = torch.full_like(batch.q_raw, float("nan"))
    ws = torch.zeros(hpa.decode_workspace_size(0, B, Hkv, Hq, D, n), dtype=torch.uint8,
                     device="cuda")
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    hpa.decode_step_prologue(batch.seq_lens, batch.q_raw, batch.k_raw, batch.v_raw,
                             batch.q_gamma, batch.k_gamma, kc, vc, batch.page_table, out, ws, n,
                             1.0 / math.sqrt(D), q_out=q_out, eps=1e-6, rope_theta=1e4)
    torch.cuda.synchronize()
    assert hpa.read_status(ws) == 0
    assert torch.equal(bits_t(out), bits_t(oa)) and torch.equal(bits_t(q_out), bits_t(qa))
    assert torch.equal(bits_t(kc), bits_t(ka)) and torch.equal(bits_t(vc), bits_t(va))


def test_fused_prologue_against_oracle_f32_out_no_q_out():
    lens = [5, 200, 3000, 64]
    batch = _prologue_case(lens, Hq=32, Hkv=8, D=128)
    kc, vc = bits16(batch.k_cache).copy(), bits16(batch.v_cache).copy()
    pt = batch.page_table.numpy()
    q64 = oracle.prologue(bits16(batch.q_raw), bits16(batch.k_raw), bits16(batch.v_raw),
                          batch.q_gamma.numpy(), batch.k_gamma.numpy(), 1e-6, 1e4,
                          batch.positions.numpy(), pt, kc, vc)
    ref = oracle.paged_decode(q64, kc, vc, pt, batch.seq_lens.numpy(), 8, 1 / math.sqrt(128))
    to_device(batch)
    (oa, *_), (ob, kb, vb, qb) = _separate_and_fused(batch, out_dtype=torch.float32,
                                                     with_q_out=False)
    assert qb is None
    _check(ob, ref)
    assert torch.equal(oa, ob)


def test_fused_prologue_mix_workload_bitwise():
    batch = W.build("mix_prologue", device="cuda")
    (oa, ka, va, qa), (ob, kb, vb, qb) = _separate_and_fused(batch)
    assert torch.equal(bits_t(oa), bits_t(ob)) and torch.equal(bits_t(qa), bits_t(qb))
    assert torch.equal(bits_t(ka), bits_t(kb)) and torch.equal(bits_t(va), bits_t(vb))


def bits_t(t: torch.Tensor) -> torch.Tensor:
    """Bit pattern of a bf16/f32 tensor (NaN-safe equality)."""
    return t.view(torch.int16 if t.dtype == torch.bfloat16 else torch.int32)


# ---------------------------------------------------------------- in-kernel plan (decode_step)

def _plan_and_run(batch, num_ctas, out_dtype=torch.float32, fp8=None):
    """Reference: hpa_decode_plan + hpa_decode_run(_multi) on a fresh workspace
    (for an e4m3 cache hpa_decode_plan_shape with the in-kernel plans' e4m3
    cost weights)."""
    q = batch.q
    T = q.shape[1] if q.dim() == 4 else 1
    B, Hq, D = q.shape[0], q.shape[-2], q.shape[-1]
    Hkv = batch.k_cache.shape[1]
    ws = torch.zeros(hpa.decode_workspace_size(0, B, Hkv, Hq * T, D, num_ctas), dtype=torch.uint8,
                     device="cuda")
    hpa.decode_plan(batch.seq_lens, num_kv_heads=Hkv, num_q_heads=Hq * T, head_dim=D,
                    pt_stride=batch.pt_stride, workspace=ws, num_ctas=num_ctas,
                    cost=None if fp8 is None else (hpa.COST_UNIT_DEFAULT, hpa.COST_END_DEFAULT_FP8))
    out = torch.full(q.shape, float("nan"), dtype=out_dtype, device="cuda")
    kw = {}
    kc, vc = batch.k_cache, batch.v_cache
    if fp8 is not None:
        kc, ks, vc, vs = (torch.from_numpy(x).cuda() for x in fp8)
        kw = dict(k_scale=ks, v_scale=vs)
    run = hpa.decode_run_multi if q.dim() == 4 else hpa.decode_run
    run(q, kc, vc, batch.page_table, out, ws, num_ctas, 1 / math.sqrt(D), **kw)
    return out, ws


def _step(batch, num_ctas, ws=None, out_dtype=torch.float32, fp8=None):
    q = batch.q
    T = q.shape[1] if q.dim() == 4 else 1
    B, Hq, D = q.shape[0], q.shape[-2], q.shape[-1]
    Hkv = batch.k_cache.shape[1]
    if ws is None:
        ws = torch.zeros(hpa.decode_workspace_size(0, B, Hkv, Hq * T, D, num_ctas),
                         dtype=torch.uint8, device="cuda")
    out = torch.full(q.shape, float("nan"), dtype=out_dtype, device="cuda")
    kw = {}
    kc, vc = batch.k_cache, batch.v_cache
    if fp8 is not None:
        kc, ks, vc, vs = (torch.from_numpy(x).cuda() for x in fp8)
        kw = dict(k_scale=ks, v_scale=vs)
    hpa.decode_step(batch.seq_lens, q, kc, vc, batch.page_table, out, ws, num_ctas,
                    1 / math.sqrt(D), **kw)
    return out, ws


STEP_CASES = [
    # name, lens, Hq, Hkv, D, T, num_ctas
    ("skewed_small", [8192] + [512] * 15, 64, 8, 128, 1, None),
    ("few_units", [37, 200], 8, 2, 64, 1, None),          # U <= P: one unit per CTA
    ("ragged", [0, 1, 63, 64, 65, 700, 3000, 2], 32, 8, 128, 1, 7),
    ("g16", [129, 2000, 5], 32, 2, 128, 1, None),
    ("mt2", [65, 300, 2, 4097], 64, 8, 128, 2, None),
    ("mt4_d64", [130, 64, 1000], 16, 4, 64, 4, 5),
    ("max_batch", [int(x) for x in np.random.default_rng(7).integers(0, 400, 512)], 8, 2, 64, 1,
     None),
    ("g32", [129, 2000, 5, 64], 32, 1, 128, 1, None),      # 32 rows: four n-tiles
    ("mt4_g8", [65, 300, 2, 4097], 64, 8, 128, 4, None),  # 32 rows of four query tokens
]


@pytest.mark.parametrize("name,lens,Hq,Hkv,D,T,num_ctas", STEP_CASES)
def test_step_equals_plan_and_run_bitwise(name, lens, Hq, Hkv, D, T, num_ctas):
    batch = W.make_batch(W.DecodeShape(name, Hq, Hkv, D, q_tokens=T), lens,
                         seed=zlib.crc32(name.encode()) % 1000)
    to_device(batch)
    n = num_ctas or hpa.default_num_ctas()
    ref, ws_ref = _plan_and_run(batch, n)
    got, ws = _step(batch, n)
    torch.cuda.synchronize()
    assert hpa.read_status(ws) == 0
    assert torch.equal(got, ref)
    # the segment descriptors and the plan fields of the header, as the plan writes them
    lay = hpa.workspace_layout(0, batch.batch, Hkv, Hq * T, D, n)
    S = batch.batch * Hkv
    a, b = ws.cpu().numpy(), ws_ref.cpu().numpy()
    sd = slice(lay["seg_desc"], lay["seg_desc"] + 8 * S)
    np.testing.assert_array_equal(a[sd], b[sd])
    hdr_a = a[lay["header"]:lay["header"] + 64].view(np.int32)
    hdr_b = b[lay["header"]:lay["header"] + 64].view(np.int32)
    for f in (0, 2, 3, 4, 5, 6, 7, 8, 9, 10):  # magic, units, grid, kind, shapes, tiles, ranges
        assert hdr_a[f] == hdr_b[f], f
    assert hdr_a[11] == 0 and hdr_a[12] == 0  # run-time counters back at zero


@pytest.mark.parametrize("lens", [
    [1, 63, 64, 65, 700, 3000],
    # many single-tile sequences: the e4m3 cost weights move the cuts
    [64] * 100 + [4000] * 20 + [1, 130] * 10,
    # 480 sequences, a sixth of them empty: the scan's non-empty counts cross
    # all six warps' slices and the cost prefix skips the empty sequences
    ([64] * 3 + [0, 1, 2000]) * 80,
    # 320 units over 296 CTAs at cost 640 < 3 x 296: the fallback to the
    # even split of the units
    [65] * 20,
])
def test_step_fp8_equals_plan_and_run(lens):
    """The e4m3 in-kernel plan weighs segment ends (COST_END_DEFAULT_FP8): it
    equals hpa_decode_plan_shape with those weights, bit for bit, and the plan
    fields of the header record them."""
    shape = W.DecodeShape("st8", 64, 8, 128, kv_dtype="fp8_e4m3")
    batch = W.make_batch(shape, lens, seed=44)
    fp8 = quantize_fp8(batch)
    to_device(batch)
    n = hpa.default_num_ctas()
    ref, ws_ref = _plan_and_run(batch, n, fp8=fp8)
    got, ws = _step(batch, n, fp8=fp8)
    assert torch.equal(got, ref)
    lay = hpa.workspace_layout(0, batch.batch, 8, 64, 128, n)
    S = batch.batch * 8
    a, b = ws.cpu().numpy(), ws_ref.cpu().numpy()
    sd = slice(lay["seg_desc"], lay["seg_desc"] + 8 * S)
    np.testing.assert_array_equal(a[sd], b[sd])
    hdr = a[lay["header"]:lay["header"] + 128].view(np.int32)
    assert (int(hdr[19]), int(hdr[20])) == (hpa.COST_UNIT_DEFAULT, hpa.COST_END_DEFAULT_FP8)
    ref64 = oracle_decode(batch, fp8=fp8)
    mx, _ = errors(got, ref64)
    assert mx <= FP8_MAX_ABS, mx


def test_step_repeated_with_changing_lengths_and_mixed_calls():
    """One workspace through several steps whose lengths change, with plain
    plan + run calls in between: every step must find the run-time counters
    at zero."""
    n = hpa.default_num_ctas()
    steps = [[5000, 64, 1], [300] * 9, [1, 2, 3], [20000, 7, 4000, 640]]
    # one buffer for all steps: each call lays the workspace out for its own
    # batch size; the header (with the counters) sits at offset 0 for all
    size = max(hpa.decode_workspace_size(0, len(l), 8, 32, 128, n) for l in steps)
    ws = torch.zeros(size, dtype=torch.uint8, device="cuda")
    for i, lens in enumerate(steps):
        batch = W.make_batch(W.DecodeShape("rep", 32, 8, 128), lens, seed=50 + i)
        to_device(batch)
        ref, _ = _plan_and_run(batch, n)
        got, _ = _step(batch, n, ws=ws)
        assert torch.equal(got, ref), i
        # a plain dynamic plan + run on the same workspace in between
        hpa.decode_plan(batch.seq_lens, num_kv_heads=8, num_q_heads=32, head_dim=128,
                        pt_stride=batch.pt_stride, workspace=ws, num_ctas=n)
        out = torch.empty_like(ref)
        hpa.decode_run(batch.q, batch.k_cache, batch.v_cache, batch.page_table, out, ws, n,
                       1 / math.sqrt(128))
        assert torch.equal(out, ref), i
    torch.cuda.synchronize()
    assert hpa.read_status(ws) == 0


def test_step_flags_clamped_lengths():
    batch = W.make_batch(W.DecodeShape("clamp", 8, 2, 64), [100, 300], seed=45)
    batch.seq_lens[1] = 100_000  # past the page table
    to_device(batch)
    _, ws = _step(batch, hpa.default_num_ctas())
    torch.cuda.synchronize()
    assert hpa.read_status(ws) & hpa.DEVICE_LEN_CLAMPED


# ---------------------------------------------------------------- canaries

@pytest.mark.parametrize("kind,num_ctas,T,Hq", [(0, None, 1, 32), (0, 5, 1, 32), (1, None, 1, 32),
                                                (2, 7, 1, 32), (0, None, 2, 32),
                                                (0, None, 4, 64), (1, None, 1, 256)])
def test_writes_stay_inside_out_and_workspace(kind, num_ctas, T, Hq):
    """Guard bytes around the output and the workspace, and the whole KV
    cache, are unchanged by plan + run (compute-sanitizer is not available,
    so out-of-range writes are looked for this way); the last two cases run
    the four-n-tile kernel (32 query rows per kv head)."""
    Hkv, D = 8, 128
    batch = W.make_batch(W.DecodeShape("canary", Hq, Hkv, D, q_tokens=T),
                         [0, 1, 64, 65, 4000, 300], seed=41)
    to_device(batch)
    B = batch.batch
    n = num_ctas or hpa.default_num_ctas()
    maxlen = int(batch.seq_lens.max().item())
    grid = hpa.plan_grid(kind, B, Hkv, n, 0, maxlen)
    ws_bytes = hpa.decode_workspace_size(kind, B, Hkv, Hq * T, D, grid)
    guard = 4096
    ws_all = torch.full((ws_bytes + 2 * guard,), 0x5A, dtype=torch.uint8, device="cuda")
    ws = ws_all[guard:guard + ws_bytes]
    out_shape = (B, T, Hq, D) if T > 1 else (B, Hq, D)
    numel = B * T * Hq * D
    out_all = torch.full((numel + 2 * guard,), 12345.0, dtype=torch.float32, device="cuda")
    out = out_all[guard:guard + numel].view(out_shape)
    kc, vc = bits16(batch.k_cache).copy(), bits16(batch.v_cache).copy()
    hpa.decode_plan(batch.seq_lens, num_kv_heads=Hkv, num_q_heads=Hq * T, head_dim=D,
                    pt_stride=batch.pt_stride, workspace=ws, kind=kind, num_ctas=n,
                    max_seq_len=maxlen)
    run = hpa.decode_run_multi if T > 1 else hpa.decode_run
    run(batch.q, batch.k_cache, batch.v_cache, batch.page_table, out, ws, grid,
        1 / math.sqrt(D), kind=kind)
    torch.cuda.synchronize()
    assert hpa.read_status(ws) == 0
    assert torch.all(ws_all[:guard] == 0x5A) and torch.all(ws_all[guard + ws_bytes:] == 0x5A)
    assert torch.all(out_all[:guard] == 12345.0) and torch.all(out_all[guard + numel:] == 12345.0)
    assert torch.isfinite(out).all()
    np.testing.assert_array_equal(bits16(batch.k_cache), kc)
    np.testing.assert_array_equal(bits16(batch.v_cache), vc)


def test_fused_prologue_writes_only_the_new_slots():
    lens = [0, 63, 64, 1000]
    batch = _prologue_case(lens, Hq=32, Hkv=8, D=128)
    kc, vc = bits16(batch.k_cache).copy(), bits16(batch.v_cache).copy()
    to_device(batch)
    _, (_, ka, va, _) = _separate_and_fused(batch)  # the fused path's caches
    pt = batch.page_table.cpu().numpy()
    touched = np.zeros(kc.shape[:3], dtype=bool)
    for b, pos in enumerate(lens):
        touched[pt[b, pos // 64], :, pos % 64] = True
    gk, gv = bits16(ka), bits16(va)
    assert not (gk != kc)[~touched].any() and not (gv != vc)[~touched].any()


# ---------------------------------------------------------------- device-side checks

def test_bad_page_id_is_flagged():
    batch = W.make_batch(W.DecodeShape("bad", 8, 2, 64), [100, 300], seed=14)
    batch.page_table[1, 2] = batch.num_pages + 5
    to_device(batch)
    out, ws, _ = gpu_decode(batch, return_ws=True)
    assert hpa.read_status(ws) & hpa.DEVICE_BAD_PAGE


def test_run_without_plan_is_flagged():
    batch = W.make_batch(W.DecodeShape("np", 8, 2, 64), [100], seed=15)
    to_device(batch)
    grid = 148
    ws = torch.zeros(hpa.decode_workspace_size(0, 1, 2, 8, 64, grid), dtype=torch.uint8,
                     device="cuda")
    out = torch.zeros(1, 8, 64, dtype=torch.bfloat16, device="cuda")
    hpa.decode_run(batch.q, batch.k_cache, batch.v_cache, batch.page_table, out, ws, grid, 0.125)
    assert hpa.read_status(ws) & hpa.DEVICE_BAD_PLAN


def test_status_clean_on_normal_run():
    batch = W.make_batch(W.DecodeShape("ok", 16, 4, 128), [700, 33], seed=16)
    to_device(batch)
    _, ws, _ = gpu_decode(batch, return_ws=True)
    assert hpa.read_status(ws) == 0


# ---------------------------------------------------------------- per-CTA trace

@pytest.mark.parametrize("name,lens,kind", [
    ("skewed_small", [8192] + [512] * 31, 0), ("uniform_small", [512] * 64, 0),
    ("mixed", [1, 63, 64, 65, 300, 5000, 129, 4096, 0, 7], 0),
    ("mixed_static", [1, 63, 64, 65, 300, 5000, 129, 4096, 0, 7], 1)])
def test_cta_times_account_for_every_unit(name, lens, kind):
    """hpa_read_cta_times: every CTA's stamps are ordered (start <= producer
    done <= epilogue done, within one launch) and the units the CTAs report
    streaming add up to the plan's units, each streamed once."""
    batch = W.make_batch(W.DecodeShape(name, 64, 8, 128), lens, seed=5)
    to_device(batch)
    B, Hkv = batch.batch, 8
    dec = hpa.PagedDecoder(B, 64, Hkv, 128, batch.pt_stride, kind=kind,
                           max_seq_len=max(lens))
    out = torch.empty(B, 64, 128, dtype=torch.bfloat16, device="cuda")
    for _ in range(2):
        dec.step(batch.q, batch.k_cache, batch.v_cache, batch.page_table, batch.seq_lens, out,
                 1 / math.sqrt(128))
    t = dec.cta_times()
    assert t.shape == (dec.grid, 4)
    assert torch.all(t[:, 0] <= t[:, 1]) and torch.all(t[:, 1] <= t[:, 2])
    assert int(t[:, 2].max() - t[:, 0].min()) < 1_000_000_000  # one launch, not stale values
    U = sum((L + 63) // 64 for L in lens) * Hkv
    assert int(t[:, 3].sum()) == U
    ti = hpa.tail_idle(t)
    assert 0.0 <= ti["idle_fraction"] < 1.0 and ti["span_us"] > 0


# ---------------------------------------------------------------- random sweep

def _random_case(seed):
    rng = np.random.default_rng(1000 + seed)
    D = int(rng.choice([64, 128]))
    fp8 = D == 128 and rng.random() < 0.3
    Hkv = int(rng.choice([1, 2, 4, 8]))
    G = int(rng.integers(1, 33))
    T = int(rng.integers(1, 32 // G + 1)) if rng.random() < 0.4 else 1
    B = int(rng.integers(1, 12))
    lens = [int(x) for x in rng.choice([0, 1, 63, 64, 65, 127, 129, 700, 2000, 5000], B)]
    lens = [L + int(rng.integers(0, 3)) for L in lens]
    lens = [max(L, T) if rng.random() < 0.9 else L for L in lens]
    kind = int(rng.choice([0, 0, 1, 2, 3]))
    param = int(rng.integers(0, 5)) if kind else 0
    tail = [(8, 4, 32), (0, 1, 0), (3, 2, 0), (16, 4, 4)][int(rng.integers(0, 4))] \
        if kind in (0, 3) else None
    num_ctas = int(rng.choice([1, 5, 37, 148, 296]))
    out_dtype = torch.float32 if rng.random() < 0.5 else torch.bfloat16
    cost = [None, (1, 0), (1, 1), (2, 1), (4, 4)][int(rng.integers(0, 5))] \
        if kind in (0, 3) else None
    return dict(D=D, fp8=fp8, Hkv=Hkv, G=G, T=T, lens=lens, kind=kind, param=param, tail=tail,
                cost=cost, num_ctas=num_ctas, out_dtype=out_dtype)


@pytest.mark.parametrize("seed", range(24))
def test_random_configurations_match_oracle(seed):
    """Seeded random shapes through plan + run (plan kinds, tail shapes, cost
    weights, CTA counts, group sizes 1..32, head_dim 64/128, up to 32 query rows per kv
    head, bf16 or FP8 KV, bf16 or fp32 output) against the oracle."""
    c = _random_case(seed)
    D, Hkv, G, T = c["D"], c["Hkv"], c["G"], c["T"]
    Hq = G * Hkv
    shape = W.DecodeShape(f"rnd{seed}", Hq, Hkv, D, kv_dtype="fp8_e4m3" if c["fp8"] else "bf16",
                          q_tokens=T)
    batch = W.make_batch(shape, c["lens"], seed=2000 + seed)
    fp8 = quantize_fp8(batch) if c["fp8"] else None
    if T == 1:
        ref = oracle_decode(batch, fp8=fp8)
    else:
        kc, vc = (bits16(batch.k_cache), bits16(batch.v_cache)) if fp8 is None else (fp8[0], fp8[2])
        kw = {} if fp8 is None else dict(kv_fp8=True, k_scale=fp8[1], v_scale=fp8[3])
        ref = oracle.paged_decode_multi(bits16(batch.q), kc, vc, batch.page_table.numpy(),
                                        batch.seq_lens.numpy(), Hkv, 1 / math.sqrt(D), **kw)
    to_device(batch)
    B = batch.batch
    maxlen = max(max(c["lens"]), 1)
    grid = hpa.plan_grid(c["kind"], B, Hkv, c["num_ctas"], c["param"], maxlen)
    ws = torch.zeros(hpa.decode_workspace_size(c["kind"], B, Hkv, Hq * T, D, grid),
                     dtype=torch.uint8, device="cuda")
    g = hpa.decode_plan(batch.seq_lens, num_kv_heads=Hkv, num_q_heads=Hq * T, head_dim=D,
                        pt_stride=batch.pt_stride, workspace=ws, kind=c["kind"],
                        num_ctas=c["num_ctas"], param=c["param"], max_seq_len=maxlen,
                        tail=c["tail"], cost=c["cost"])
    out = torch.full(batch.q.shape, float("nan"), dtype=c["out_dtype"], device="cuda")
    kw = {}
    kc, vc = batch.k_cache, batch.v_cache
    if fp8 is not None:
        kc, ks, vc, vs = (torch.from_numpy(x).cuda() for x in fp8)
        kw = dict(k_scale=ks, v_scale=vs)
    if T == 1:
        hpa.decode_run(batch.q, kc, vc, batch.page_table, out, ws, g, 1 / math.sqrt(D),
                       kind=c["kind"], **kw)
    else:
        hpa.decode_run_multi(batch.q, kc, vc, batch.page_table, out, ws, g, 1 / math.sqrt(D),
                             kind=c["kind"], **kw)
    torch.cuda.synchronize()
    assert hpa.read_status(ws) == 0, c
    assert torch.isfinite(out.float()).all(), c
    mx, mn = errors(out, ref)
    assert mx <= (FP8_MAX_ABS if fp8 is not None else MAX_ABS) and mn <= MEAN_ABS, (c, mx, mn)
