"""Pins for the fp64 oracle: closed forms, library routines, brute force and
invariants -- never the oracle against itself.

Each test names the plain fact it checks.  A plausible slip in the oracle (a
dropped term, a wrong sign or index, a transposed operand, a wrong page or
head mapping, a wrong rounding rule) fails at least one of them.
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from mixed_length_paged_b200 import workloads as W
from tests.helpers import bf16_values, bits16, dense_attention, dense_kv

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- bf16 codec

def test_bf16_decode_matches_float32_view():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 1 << 16, size=4096, dtype=np.uint32).astype(np.uint16)
    ours = oracle.bf16_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(ours[ok], ref[ok])


def test_bf16_round_matches_torch_rne_on_float32_values():
    # For values exactly representable in fp32, fp64->bf16 RNE equals torch's
    # fp32->bf16 RNE cast (a library routine).
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(3000).astype(np.float32),
                        (rng.standard_normal(500) * 1e-38).astype(np.float32),   # subnormal range
                        (rng.standard_normal(500) * 1e30).astype(np.float32)])
    ours = oracle.bf16_from_f64(x.astype(np.float64))
    ref = bits16(torch.from_numpy(x).to(torch.bfloat16))
    np.testing.assert_array_equal(ours, ref)


def test_bf16_round_ties_to_even():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7 -> even mantissa (1.0).
    assert oracle.bf16_from_f64(1.0 + 2.0 ** -8) == 0x3F80
    # 1 + 3*2^-8 is halfway between 1+2^-7 (odd) and 1+2^-6 (even) -> 1+2^-6
    assert oracle.bf16_from_f64(1.0 + 3 * 2.0 ** -8) == 0x3F82
    # just above the tie rounds up
    assert oracle.bf16_from_f64(1.0 + 2.0 ** -8 + 2.0 ** -30) == 0x3F81


# ---------------------------------------------------------------- e4m3 codec

def _golden_e4m3():
    rows = []
    with open(os.path.join(GOLDEN, "e4m3_table.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            kind, code, val = line.split()
            rows.append((kind, int(code, 16), float(val)))
    return rows


def test_e4m3_golden_table():
    for kind, code, val in _golden_e4m3():
        if kind == "decode":
            got = oracle.e4m3_decode([code])[0]
            if math.isnan(val):
                assert math.isnan(got), hex(code)
            else:
                assert got == val and math.copysign(1, got) == math.copysign(1, val), hex(code)
        else:
            assert oracle.e4m3_encode([val])[0] == code, (val, hex(code))


def test_e4m3_decode_all_codes_closed_form():
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.e4m3_decode(codes)
    for c in range(256):
        s, e, m = c >> 7, (c >> 3) & 15, c & 7
        if e == 15 and m == 7:
            assert math.isnan(got[c])
            continue
        mag = m * 2.0 ** -9 if e == 0 else (8 + m) * 2.0 ** (e - 10)
        assert got[c] == (-mag if s else mag), hex(c)


def test_e4m3_decode_matches_torch_float8():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_decode(codes)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])


def test_e4m3_encode_roundtrips_every_finite_code():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = oracle.e4m3_decode(codes)
    np.testing.assert_array_equal(oracle.e4m3_encode(vals), codes)


def test_e4m3_encode_midpoints_brute_force():
    # Every midpoint between adjacent non-negative finite values rounds to the
    # neighbour with an even code (even mantissa); just off the midpoint rounds
    # to the nearer one.
    pos = [c for c in range(0x7F)]
    vals = oracle.e4m3_decode(np.array(pos, dtype=np.uint8))
    for a, b in zip(pos[:-1], pos[1:]):
        va, vb = vals[a], vals[b]
        mid = (va + vb) / 2
        even = a if a % 2 == 0 else b
        assert oracle.e4m3_encode([mid])[0] == even, (hex(a), hex(b))
        eps = (vb - va) * 1e-6
        assert oracle.e4m3_encode([mid - eps])[0] == a
        assert oracle.e4m3_encode([mid + eps])[0] == b
        assert oracle.e4m3_encode([-(mid + eps)])[0] == (0x80 | b)


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.standard_normal(4000) * 50, rng.standard_normal(1000) * 0.01])
    x = np.clip(x, -448, 448).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(x.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_quantizer_scale_and_error_bound():
    shape = W.DecodeShape("q", 4, 2, 16, kv_dtype="fp8_e4m3")
    batch = W.make_batch(shape, [70, 5], seed=3)
    vals = batch.k_cache.numpy()
    live = batch.live.numpy()
    codes, scales = oracle.quantize_kv_e4m3(vals, live, dead_code=0x7F)
    for p in range(vals.shape[0]):
        for g in range(vals.shape[1]):
            n = live[p]
            if n == 0:
                assert scales[p, g] == 1.0
                assert np.all(codes[p, g] == 0x7F)
                continue
            blk = vals[p, g, :n].astype(np.float64)
            amax = np.abs(blk).max()
            assert scales[p, g] == np.float32(amax / 448.0)
            dec = oracle.e4m3_decode(codes[p, g, :n]) * float(scales[p, g])
            # RNE with 3 mantissa bits: relative error <= 2^-4 for normals,
            # absolute error <= 2^-10 * scale in the subnormal range.
            err = np.abs(dec - blk)
            bound = np.maximum(np.abs(blk) * 2.0 ** -4, 2.0 ** -10 * float(scales[p, g]))
            assert np.all(err <= bound * (1 + 1e-12))
            # the amax element lands on +-448
            i = np.unravel_index(np.abs(blk).argmax(), blk.shape)
            assert abs(oracle.e4m3_decode([codes[p, g][i]])[0]) == 448.0
            assert np.all(codes[p, g, n:] == 0x7F)


# ---------------------------------------------------------------- RMSNorm / RoPE

def test_rmsnorm_closed_form():
    # x = (3, 4): mean square 12.5, y = x / sqrt(12.5) * gamma
    y = oracle.rmsnorm([3.0, 4.0], [1.0, 2.0], 0.0)
    np.testing.assert_allclose(y, [3 * math.sqrt(2) / 5, 2 * 4 * math.sqrt(2) / 5], rtol=1e-15)


def test_rmsnorm_unit_rms_scale_invariance_and_eps():
    rng = np.random.default_rng(4)
    x = rng.standard_normal(128)
    y = oracle.rmsnorm(x, np.ones(128), 0.0)
    assert abs(math.sqrt(np.mean(y * y)) - 1.0) < 1e-14
    np.testing.assert_allclose(oracle.rmsnorm(7.5 * x, np.ones(128), 0.0), y, rtol=1e-14)
    ms = np.mean(x * x)
    ye = oracle.rmsnorm(x, np.ones(128), 1e-6)
    assert abs(math.sqrt(np.mean(ye * ye)) - math.sqrt(ms / (ms + 1e-6))) < 1e-14
    g = rng.uniform(0.5, 1.5, 128)
    np.testing.assert_allclose(oracle.rmsnorm(x, g, 0.0), y * g, rtol=1e-14)


def test_rope_position_zero_is_identity():
    x = np.random.default_rng(5).standard_normal(128)
    np.testing.assert_array_equal(oracle.rope(x, 0, 10000.0), x)


def test_rope_matches_complex_rotation():
    # Rotate-half RoPE == multiplying z_i = x_i + i x_{i+D/2} by e^{i pos w_i},
    # w_i = theta^(-2i/D), evaluated with numpy's complex exponential.
    rng = np.random.default_rng(6)
    D, theta = 128, 10000.0
    x = rng.standard_normal(D)
    for pos in [1, 7, 4095, 65536]:
        i = np.arange(D // 2)
        w = theta ** (-2.0 * i / D)
        z = (x[:D // 2] + 1j * x[D // 2:]) * np.exp(1j * pos * w)
        y = oracle.rope(x, pos, theta)
        np.testing.assert_allclose(y[:D // 2], z.real, atol=1e-12)
        np.testing.assert_allclose(y[D // 2:], z.imag, atol=1e-12)


def test_rope_quarter_turn_and_invariants():
    # D = 2: one pair with w_0 = 1; pos = pi/2 maps (a, b) to (-b, a).
    y = oracle.rope([0.3, -1.7], math.pi / 2, 10000.0)
    np.testing.assert_allclose(y, [1.7, 0.3], atol=1e-15)
    rng = np.random.default_rng(7)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    for m, n, t in [(5, 2, 11), (1000, 37, 4096), (65536, 3, 17)]:
        yq = oracle.rope(q, m, 10000.0)
        # every (i, i+D/2) pair keeps its norm
        np.testing.assert_allclose(yq[:32] ** 2 + yq[32:] ** 2, q[:32] ** 2 + q[32:] ** 2,
                                   rtol=1e-12)
        # <R(m)q, R(n)k> depends only on m - n
        a = np.dot(yq, oracle.rope(k, n, 10000.0))
        b = np.dot(oracle.rope(q, m + t, 10000.0), oracle.rope(k, n + t, 10000.0))
        assert abs(a - b) < 1e-10


# ---------------------------------------------------------------- attention

def _tiny(seed=0, lens=(37, 200), Hq=8, Hkv=2, D=64):
    shape = W.DecodeShape("t", Hq, Hkv, D)
    return W.make_batch(shape, list(lens), seed=seed)


def _run(batch, **kw):
    D = batch.shape.head_dim
    return oracle.paged_decode(bits16(batch.q), bits16(batch.k_cache), bits16(batch.v_cache),
                               batch.page_table.numpy(), batch.seq_lens.numpy(),
                               batch.shape.num_kv_heads, 1.0 / math.sqrt(D), **kw)


def test_attention_golden_equal_logits():
    with open(os.path.join(GOLDEN, "attention_equal_logits.json")) as f:
        g = json.load(f)

    def arr(x):
        return np.array(x, dtype=np.float64)

    q = arr(g["q"])
    kc = oracle.bf16_from_f64(arr(g["k_cache"]))
    vc = oracle.bf16_from_f64(arr(g["v_cache"]))
    out = oracle.paged_decode(q, kc, vc, np.array(g["page_table"], dtype=np.int32),
                              np.array(g["seq_lens"], dtype=np.int32), g["num_kv_heads"],
                              g["scale"], page_size=g["page_size"])
    np.testing.assert_allclose(out, arr(g["expected"]), rtol=1e-15, atol=0)


@pytest.mark.parametrize("seed,lens,Hq,Hkv,D", [
    (0, (37, 200), 8, 2, 64),
    (1, (1, 64, 65, 129), 8, 8, 32),
    (2, (300, 7), 16, 2, 128),
    (3, (128,), 4, 1, 16),
])
def test_attention_matches_dense_brute_force(seed, lens, Hq, Hkv, D):
    batch = _tiny(seed, lens, Hq, Hkv, D)
    out = _run(batch)
    kv = bf16_values(bits16(batch.k_cache))
    vv = bf16_values(bits16(batch.v_cache))
    qv = bf16_values(bits16(batch.q))
    pt = batch.page_table.numpy()
    for b, L in enumerate(lens):
        ref = dense_attention(qv[b], dense_kv(kv, pt, b, L), dense_kv(vv, pt, b, L),
                              1.0 / math.sqrt(D))
        np.testing.assert_allclose(out[b], ref, rtol=0, atol=1e-12)


def test_attention_length_one_returns_v():
    batch = _tiny(4, (1, 1), 8, 2, 64)
    out = _run(batch)
    vv = bf16_values(bits16(batch.v_cache))
    pt = batch.page_table.numpy()
    for b in range(2):
        for h in range(8):
            np.testing.assert_array_equal(out[b, h], vv[pt[b, 0], h // 4, 0])


def test_attention_zero_query_is_mean_of_v():
    batch = _tiny(5, (37, 200), 8, 2, 64)
    batch.q.zero_()
    out = _run(batch)
    vv = bf16_values(bits16(batch.v_cache))
    pt = batch.page_table.numpy()
    for b, L in enumerate((37, 200)):
        V = dense_kv(vv, pt, b, L)
        for h in range(8):
            np.testing.assert_allclose(out[b, h], V[:, h // 4, :].mean(axis=0), atol=1e-14)


def test_attention_invariant_under_page_permutation():
    batch = _tiny(6, (37, 200), 8, 2, 64)
    out = _run(batch)
    rng = np.random.default_rng(99)
    P = batch.num_pages
    perm = rng.permutation(P)               # new physical id of old page p
    kc = np.empty_like(bits16(batch.k_cache))
    vc = np.empty_like(kc)
    kc[perm] = bits16(batch.k_cache)
    vc[perm] = bits16(batch.v_cache)
    pt = batch.page_table.numpy().copy()
    pt[pt >= 0] = perm[pt[pt >= 0]]
    out2 = oracle.paged_decode(bits16(batch.q), kc, vc, pt, batch.seq_lens.numpy(), 2, 1 / 8)
    np.testing.assert_array_equal(out, out2)


def test_split_and_lse_merge_equals_unsplit():
    batch = _tiny(7, (37, 200), 8, 2, 64)
    out = _run(batch)
    q, kc, vc = bits16(batch.q), bits16(batch.k_cache), bits16(batch.v_cache)
    pt = batch.page_table.numpy()
    rng = np.random.default_rng(8)
    for b, L in enumerate((37, 200)):
        for h in (0, 5):
            for nsplit in (1, 2, 3, 7):
                cuts = np.sort(rng.choice(np.arange(1, L), size=nsplit - 1, replace=False)) \
                    if nsplit > 1 else np.array([], dtype=int)
                edges = [0, *cuts.tolist(), L]
                parts = [oracle.partial(q, kc, vc, pt, 2, 1 / 8, b, h, a, e)
                         for a, e in zip(edges[:-1], edges[1:])]
                acc = np.stack([p[0] for p in parts])
                m = np.array([p[1] for p in parts])
                l = np.array([p[2] for p in parts])
                np.testing.assert_allclose(oracle.lse_merge(acc, m, l), out[b, h], atol=1e-12)
            # an empty partial contributes nothing
            a0, m0, l0 = oracle.partial(q, kc, vc, pt, 2, 1 / 8, b, h, 0, 0)
            assert m0 == -math.inf and l0 == 0.0
            a1, m1, l1 = oracle.partial(q, kc, vc, pt, 2, 1 / 8, b, h, 0, L)
            np.testing.assert_allclose(
                oracle.lse_merge(np.stack([a0, a1]), [m0, m1], [l0, l1]), out[b, h], atol=1e-15)


def test_needle_in_128k_tokens():
    # A key planted as c * q / |q| at a random position of a 131072-token
    # sequence takes essentially all the softmax mass: o ~= V[needle].
    D, Hkv, Hq, L = 128, 1, 2, 131072
    shape = W.DecodeShape("needle", Hq, Hkv, D)
    batch = W.make_batch(shape, [L], seed=9, spare_pages=1)
    q = bf16_values(bits16(batch.q))[0, 0]
    j = int(np.random.default_rng(10).integers(0, L))
    pt = batch.page_table.numpy()
    page, slot = pt[0, j // 64], j % 64
    batch.k_cache[page, 0, slot] = torch.from_numpy(40.0 * q / np.linalg.norm(q)).to(torch.bfloat16)
    out = _run(batch, num_threads=0)
    vv = bf16_values(bits16(batch.v_cache))
    np.testing.assert_allclose(out[0, 0], vv[page, 0, slot], atol=1e-6)
    # the other head of the group does not see the needle
    assert np.abs(out[0, 1] - vv[page, 0, slot]).max() > 0.1


def test_zero_length_sequence_gives_zero_output():
    batch = _tiny(11, (0, 5), 8, 2, 64)
    out = _run(batch)
    assert np.all(out[0] == 0.0)
    assert np.all(np.isfinite(out[1]))


def test_rows_subset_matches_full():
    batch = _tiny(12, (37, 200, 90), 8, 2, 64)
    full = _run(batch)
    sub = _run(batch, rows=np.array([2, 0], dtype=np.int32))
    np.testing.assert_array_equal(sub[[0, 2]], full[[0, 2]])
    assert np.all(sub[1] == 0)


def test_fp8_attention_matches_dense_on_dequantised_values():
    shape = W.DecodeShape("f", 8, 2, 64, kv_dtype="fp8_e4m3")
    lens = (70, 130)
    batch = W.make_batch(shape, list(lens), seed=13)
    kcode, ks = oracle.quantize_kv_e4m3(batch.k_cache.numpy(), batch.live.numpy())
    vcode, vs = oracle.quantize_kv_e4m3(batch.v_cache.numpy(), batch.live.numpy())
    pt = batch.page_table.numpy()
    out = oracle.paged_decode(bits16(batch.q), kcode, vcode, pt, batch.seq_lens.numpy(), 2,
                              1 / 8, kv_fp8=True, k_scale=ks, v_scale=vs)
    # dequantise with torch's float8 decoder (library) and the scales
    kd = torch.from_numpy(kcode).view(torch.float8_e4m3fn).to(torch.float64).numpy() \
        * ks[:, :, None, None]
    vd = torch.from_numpy(vcode).view(torch.float8_e4m3fn).to(torch.float64).numpy() \
        * vs[:, :, None, None]
    qv = bf16_values(bits16(batch.q))
    for b, L in enumerate(lens):
        ref = dense_attention(qv[b], dense_kv(kd, pt, b, L), dense_kv(vd, pt, b, L), 1 / 8)
        np.testing.assert_allclose(out[b], ref, atol=1e-12)


# ---------------------------------------------------------------- prologue

def test_prologue_slot_write_and_values():
    shape = W.DecodeShape("p", 8, 2, 64, prologue=True)
    lens = [63, 64, 130, 0]
    batch = W.make_batch(shape, lens, seed=14)
    kc0, vc0 = bits16(batch.k_cache), bits16(batch.v_cache)
    kc, vc = kc0.copy(), vc0.copy()
    pt = batch.page_table.numpy()
    eps, theta = 1e-6, 10000.0
    q_out = oracle.prologue(bits16(batch.q_raw), bits16(batch.k_raw), bits16(batch.v_raw),
                            batch.q_gamma.numpy(), batch.k_gamma.numpy(), eps, theta,
                            batch.positions.numpy(), pt, kc, vc)
    touched = np.zeros(kc.shape[:3], dtype=bool)
    qg = batch.q_gamma.numpy().astype(np.float64)
    kg = batch.k_gamma.numpy().astype(np.float64)
    for b, pos in enumerate(lens):
        page, slot = pt[b, pos // 64], pos % 64
        for g in range(2):
            touched[page, g, slot] = True
            kraw = bf16_values(bits16(batch.k_raw))[b, g]
            # RMSNorm (closed form, numpy) then rotation (numpy complex form)
            x = kraw / math.sqrt(np.mean(kraw * kraw) + eps) * kg
            w = theta ** (-2.0 * np.arange(32) / 64)
            z = (x[:32] + 1j * x[32:]) * np.exp(1j * pos * w)
            ref = np.concatenate([z.real, z.imag])
            got = bf16_values(kc[page, g, slot])
            # fp64 RNE of nearly the same value: equal, or 1 ulp apart at a tie
            ulp = np.abs(got) * 2.0 ** -7
            assert np.all(np.abs(got - ref) <= ulp * 0.5000001 + 1e-300)
            np.testing.assert_array_equal(vc[page, g, slot], bits16(batch.v_raw)[b, g])
        for h in range(8):
            qraw = bf16_values(bits16(batch.q_raw))[b, h]
            x = qraw / math.sqrt(np.mean(qraw * qraw) + eps) * qg
            w = theta ** (-2.0 * np.arange(32) / 64)
            z = (x[:32] + 1j * x[32:]) * np.exp(1j * pos * w)
            np.testing.assert_allclose(q_out[b, h], np.concatenate([z.real, z.imag]), atol=1e-12)
    # nothing else in either cache changed (NaN-aware byte comparison)
    np.testing.assert_array_equal(kc[~touched], kc0[~touched])
    np.testing.assert_array_equal(vc[~touched], vc0[~touched])


# ---------------------------------------------------------------- planner

def _units(lens, Hkv):
    """Global unit list (b, g, t) in seq-major, kv-head, tile order."""
    out = []
    for b, L in enumerate(lens):
        n = (max(0, L) + 63) // 64
        for g in range(Hkv):
            for t in range(n):
                out.append((b, g, t))
    return out


def _check_plan_invariants(p, lens, Hkv, kind, tail=None, cost=(1, 0)):
    units = _units(lens, Hkv)
    U = len(units)
    assert p["n_units"] == U
    cta = p["cta"]
    R = p["ranges"]
    # ordered, contiguous, disjoint, covering [0, U) exactly once
    cover = np.zeros(U, dtype=int)
    prev_end = 0
    for c in range(R):
        a, e = int(cta[c, 0]), int(cta[c, 1])
        assert 0 <= a <= e <= U
        if a < e:
            assert a == prev_end
            prev_end = e
        cover[a:e] += 1
    assert prev_end == U and np.all(cover == 1)
    # split counts and partial slots, recounted with Python lists: range c
    # keeps the piece of its first segment in slot 2c and that of its last in
    # 2c + 1; the ranges holding a segment are consecutive
    seg_units = {}
    for (b, g, t) in units:
        seg_units[b * Hkv + g] = seg_units.get(b * Hkv + g, 0) + 1
    holders, pieces = {}, {}
    for c in range(R):
        a, e = int(cta[c, 0]), int(cta[c, 1])
        segs = []
        for u in range(a, e):
            s = units[u][0] * Hkv + units[u][1]
            if not segs or segs[-1][0] != s:
                segs.append([s, 0])
            segs[-1][1] += 1
        for i, (s, n) in enumerate(segs):
            holders.setdefault(s, []).append(c)
            if n < seg_units[s]:
                # a cut piece is the range's first or last segment
                assert i == 0 or i == len(segs) - 1
                pieces.setdefault(s, []).append(2 * c + (0 if i == 0 else 1))
    S = len(lens) * Hkv
    for s in range(S):
        hs = holders.get(s, [])
        assert p["split_count"][s] == len(hs)
        assert hs == list(range(hs[0], hs[0] + len(hs))) if hs else True
        if len(hs) > 1:
            ps = pieces[s]
            assert len(ps) == len(hs) and p["first_slot"][s] == ps[0]
            assert ps[1:] == [2 * c for c in hs[1:]]
        else:
            assert p["first_slot"][s] == -1 and s not in pieces
    # no slot is used twice
    used = [x for ps in pieces.values() for x in ps]
    assert len(used) == len(set(used)) and all(0 <= x < 2 * R for x in used)
    if kind == 0:
        _check_dynamic_family(p, U, tail, _unit_costs(units, cost))


def _even_ranges(n, m):
    """Unit list [0, n) cut into m contiguous ranges as evenly as possible,
    enumerated from scratch: scale the list onto m equal ranges and give unit
    u the range in which its right end (u + 1) * m / n falls, with each range
    closed on the right.  Exact rational arithmetic; returns [(begin, end)]."""
    owner = [math.ceil(Fraction((u + 1) * m, n)) - 1 for u in range(n)]
    out = []
    for c in range(m):
        us = [u for u in range(n) if owner[u] == c]
        if us:
            assert us == list(range(us[0], us[-1] + 1))
            out.append((us[0], us[-1] + 1))
        else:
            b = out[-1][1] if out else 0
            out.append((b, b))
    return out


def _unit_costs(units, cost):
    """Cost of every unit of the list under cost weights (q, e): q, plus e
    for the last unit of its (sequence, kv head) segment."""
    q, e = cost
    out = []
    for i, (b, g, t) in enumerate(units):
        last = i + 1 == len(units) or units[i + 1][:2] != (b, g)
        out.append(q + (e if last else 0))
    return out


def _cost_ranges(costs, m):
    """Units with the given costs cut into m contiguous ranges of even cost,
    enumerated from scratch: lay the units end to end on a line, each as long
    as its cost, scale the line onto m equal ranges and give unit u the range
    in which its right end falls, each range closed on the right (with unit
    costs this is _even_ranges).  Exact rational arithmetic."""
    right, acc = [], 0
    for c in costs:
        acc += c
        right.append(acc)
    owner = [math.ceil(Fraction(r * m, acc)) - 1 for r in right]
    out = []
    for c in range(m):
        us = [u for u in range(len(costs)) if owner[u] == c]
        if us:
            assert us == list(range(us[0], us[-1] + 1))
            out.append((us[0], us[-1] + 1))
        else:
            b = out[-1][1] if out else 0
            out.append((b, b))
    return out


def _check_dynamic_family(p, U, tail, costs=None):
    """A dynamic plan of the family (den, k, mn; q, e): the primary ranges
    cut the first U1 units into P ranges of even cost (every unit q, a
    segment's last unit e more: `costs`, None = all equal) if that cost is at
    least the largest unit cost times P, else of even unit count (so that no
    primary range is empty), and the tail chunks
    are the even partition of the last Ut units over M chunks, where Ut is the
    largest tail with Ut <= U / den that still leaves every primary range a
    unit (no tail for den = 0 or when U < mn P) and M the largest chunk count
    with M <= k P and M <= Ut."""
    den, k, mn = tail
    P = p["grid"]
    R = p["ranges"]
    cta = [(int(a), int(e)) for a, e in p["cta"]]
    if U <= P:
        # one unit per CTA, no tail
        assert R == P and cta == [(min(c, U), min(c + 1, U)) for c in range(P)]
        return
    M = R - P
    Ut = U - cta[P - 1][1] if M else 0
    if den == 0 or U < mn * P:
        assert Ut == 0 and M == 0
    else:
        assert Ut * den <= U and U - Ut >= P
        assert (Ut + 1) * den > U or U - Ut == P      # no larger tail would do
        if Ut:
            assert 1 <= M <= k * P and M <= Ut
            assert M == k * P or M == Ut
        else:
            assert M == 0
    prim = costs[:U - Ut] if costs is not None else None
    if prim is None or sum(prim) < max(costs) * P:
        assert cta[:P] == _even_ranges(U - Ut, P)
    else:
        assert cta[:P] == _cost_ranges(prim, P)
    assert all(a < e for a, e in cta[:P])  # no primary range is empty
    assert [(a - (U - Ut), e - (U - Ut)) for a, e in cta[P:]] == (_even_ranges(Ut, M) if M else [])


@pytest.mark.parametrize("lens,Hkv,P", [
    ([131072] + [4096] * 31, 8, 148),
    ([512] * 64, 8, 148),
    ([37, 200], 2, 148),
    ([37, 200], 2, 3),
    ([0, 5, 0, 64, 65], 4, 7),
    ([1], 1, 148),
    ([0, 0], 2, 5),
])
@pytest.mark.parametrize("kind,tail", [(0, (8, 4, 32)), (0, (8, 4, 0)), (0, (0, 1, 0)),
                                       (0, (3, 1, 0)), (0, (16, 2, 5)), (0, (1, 4, 0)),
                                       (1, (8, 4, 32)), (2, (8, 4, 32))])
def test_planner_invariants(lens, Hkv, P, kind, tail):
    p = oracle.plan(np.array(lens, dtype=np.int32), Hkv, kind=kind, num_ctas=P,
                    max_seq_len=max(lens), capacity_tokens=max(64, max(lens)), tail=tail)
    _check_plan_invariants(p, lens, Hkv, kind, tail)


def test_even_ranges_enumerator_hand_cases():
    # the enumerator the dynamic-plan pins compare with, on cases worked by hand
    assert _even_ranges(7, 3) == [(0, 2), (2, 4), (4, 7)]
    assert _even_ranges(3, 5) == [(0, 0), (0, 1), (1, 1), (1, 2), (2, 3)]
    assert _even_ranges(6, 3) == [(0, 2), (2, 4), (4, 6)]
    assert _even_ranges(10, 4) == [(0, 2), (2, 5), (5, 7), (7, 10)]
    # with costs: unit costs give the even ranges; costs (1, 1, 3, 1) over 2
    # ranges: right ends 1, 2, 5, 6 scaled by 2/6 -> 1/3, 2/3, 5/3, 2
    assert _cost_ranges([1] * 7, 3) == _even_ranges(7, 3)
    assert _cost_ranges([1, 1, 3, 1], 2) == [(0, 2), (2, 4)]
    # (5, 1, 1, 1): right ends 5..8 of 8 all lie past the midpoint 4, so
    # every unit goes to range 1 and range 0 is empty
    assert _cost_ranges([5, 1, 1, 1], 2) == [(0, 0), (0, 4)]


# A batch worked by hand: lens (5, 64, 700, 0, 1, 3000, 130) tokens are
# (1, 1, 11, 0, 1, 47, 3) tiles; with 2 kv heads the 128 units form 12
# segments whose last units are 0, 1, 2, 3, 14, 25, 26, 27, 74, 121, 124,
# 127.  Seven CTAs, no tail.
#   cost (1, 1): K(x) = x + (segment ends before x), K(128) = 140; cut c is
#     the largest x with K(x) <= 20 c: K(15) = 15 + 5 = 20, K(32) = 32 + 8 =
#     40, K(52) = 60, K(72) = 80, K(91) = 91 + 9 = 100, K(111) = 120.
#   cost (2, 1): K(x) = 2x + ends, K(128) = 268, cut c at K(x) <= floor(268
#     c / 7) = 38, 76, 114, 153, 191, 229: x = 16 (K 37), 34 (76), 53 (114),
#     72 (152), 91 (191), 110 (229).
_HAND_LENS = [5, 64, 700, 0, 1, 3000, 130]
_HAND_CUTS = {
    (1, 0): [0, 18, 36, 54, 73, 91, 109, 128],
    (1, 1): [0, 15, 32, 52, 72, 91, 111, 128],
    (2, 1): [0, 16, 34, 53, 72, 91, 110, 128],
}


@pytest.mark.parametrize("cost", sorted(_HAND_CUTS))
def test_cost_weighted_cuts_hand_case(cost):
    p = oracle.plan(np.array(_HAND_LENS, dtype=np.int32), 2, kind=0, num_ctas=7,
                    capacity_tokens=4096, tail=(0, 1, 0), cost=cost)
    cuts = _HAND_CUTS[cost]
    assert p["n_units"] == 128 and p["ranges"] == 7
    assert [(int(a), int(e)) for a, e in p["cta"]] == list(zip(cuts[:-1], cuts[1:]))


@pytest.mark.parametrize("lens,Hkv,P", [
    ([131072] + [4096] * 31, 8, 148),
    ([512] * 64, 8, 148),
    ([37, 200], 2, 3),
    ([0, 5, 0, 64, 65, 3000, 1], 4, 7),
    ([1, 63, 64, 65, 300, 5000, 129, 4096, 0, 7] * 3, 8, 296),
    ([64] * 40 + [6400] * 3, 2, 37),
])
@pytest.mark.parametrize("tail,cost", [((0, 1, 0), (1, 1)), ((0, 1, 0), (2, 1)),
                                       ((8, 4, 0), (4, 3)), ((8, 4, 32), (1, 4)),
                                       ((3, 2, 0), (3, 2))])
def test_cost_weighted_plan_invariants(lens, Hkv, P, tail, cost):
    """Cost-weighted primary ranges: coverage, slots and split counts as for
    any plan, and the primary cuts those of the from-scratch enumerator."""
    p = oracle.plan(np.array(lens, dtype=np.int32), Hkv, kind=0, num_ctas=P,
                    capacity_tokens=max(64, max(lens)), tail=tail, cost=cost)
    _check_plan_invariants(p, lens, Hkv, 0, tail, cost)


@pytest.mark.parametrize("lens,Hkv,P", [([64] * 500, 4, 148), ([1, 30, 64] * 70, 2, 37),
                                        ([10] * 7, 1, 3)])
@pytest.mark.parametrize("cost", [(1, 1), (2, 1), (3, 4)])
def test_cost_weights_do_not_move_cuts_when_all_units_cost_the_same(lens, Hkv, P, cost):
    """Every segment a single tile: every unit costs q + e, so the cost split
    is the even split of the units, the plan of cost (1, 0)."""
    kw = dict(kind=0, num_ctas=P, capacity_tokens=64, tail=(8, 4, 0))
    a = oracle.plan(np.array(lens, dtype=np.int32), Hkv, cost=cost, **kw)
    b = oracle.plan(np.array(lens, dtype=np.int32), Hkv, cost=(1, 0), **kw)
    np.testing.assert_array_equal(a["cta"], b["cta"])


@pytest.mark.parametrize("lens,Hkv,P,cost", [
    ([65, 65], 8, 27, (1, 1)),     # 16 two-unit segments of cost 3: 48 / 27 < 2
    ([65, 65], 8, 27, (2, 4)),
    ([1] * 5 + [130], 4, 30, (1, 3)),  # cost 104 < 4 x 30, 32 units
])
def test_cost_weights_fall_back_to_the_even_split_when_a_range_could_be_empty(lens, Hkv, P, cost):
    """When a range's share of the cost, K(U1) / P, is below the largest unit
    cost q + e, a cut could leave a range empty inside a split segment (and
    break the consecutive holders the partial slots need): the plan then
    splits the units evenly.  The first case is the one a random search
    found before the rule existed."""
    p = oracle.plan(np.array(lens, dtype=np.int32), Hkv, kind=0, num_ctas=P,
                    capacity_tokens=max(64, max(lens)), tail=(0, 1, 0), cost=cost)
    U = p["n_units"]
    costs = _unit_costs(_units(lens, Hkv), cost)
    assert sum(costs) < (cost[0] + cost[1]) * P < (cost[0] + cost[1]) * U
    assert [(int(a), int(e)) for a, e in p["cta"]] == _even_ranges(U, P)
    _check_plan_invariants(p, lens, Hkv, 0, (0, 1, 0), cost)


@pytest.mark.parametrize("q", [1, 2, 3, 4])
def test_end_cost_zero_is_the_even_split_for_any_unit_cost(q):
    lens = [1, 63, 64, 65, 300, 5000, 129, 4096, 0, 7]
    kw = dict(kind=0, num_ctas=37, capacity_tokens=5056, tail=(8, 4, 0))
    a = oracle.plan(np.array(lens, dtype=np.int32), 8, cost=(q, 0), **kw)
    b = oracle.plan(np.array(lens, dtype=np.int32), 8, cost=(1, 0), **kw)
    np.testing.assert_array_equal(a["cta"], b["cta"])


def test_cost_weighted_ranges_are_balanced_in_cost():
    """Each primary range's cost is within one unit's largest cost (q + e) of
    the mean, and a range of many short segments holds fewer units than one
    inside a long segment."""
    lens = [64] * 300 + [64 * 900]
    q, e = 2, 3
    P = 50
    p = oracle.plan(np.array(lens, dtype=np.int32), 1, kind=0, num_ctas=P, capacity_tokens=64 * 900,
                    tail=(0, 1, 0), cost=(q, e))
    costs = _unit_costs(_units(lens, 1), (q, e))
    K1 = sum(costs)
    sizes = []
    for a, b in p["cta"]:
        c = sum(costs[int(a):int(b)])
        assert abs(c - K1 / P) < q + e
        sizes.append(int(b - a))
    # 300 single-tile segments cost 5 each (1500), the long one 2 per unit (1803)
    assert sizes[0] < sizes[-1]


@pytest.mark.parametrize("U,P", [(5, 5), (6, 5), (7, 3), (100, 7), (32256, 148), (4096, 296),
                                 (301, 300), (1000, 1)])
def test_dynamic_plan_without_tail_is_the_even_partition(U, P):
    """With no run-time tail (den = 0) the dynamic plan is the plain even
    partition of the unit list over the CTAs: range c holds units
    [floor(cU/P), floor((c+1)U/P))."""
    # U units as one sequence of U tiles with one kv head
    p = oracle.plan(np.array([64 * U], dtype=np.int32), 1, kind=0, num_ctas=P,
                    capacity_tokens=64 * U, tail=(0, 1, 0))
    assert p["ranges"] == P
    assert [(int(a), int(e)) for a, e in p["cta"]] == _even_ranges(U, P)
    # one split count and consecutive slots, recounted
    _check_plan_invariants(p, [64 * U], 1, 0, (0, 1, 0))


@pytest.mark.parametrize("lens,Hkv,P", [
    ([131072] + [4096] * 31, 8, 148),
    ([512] * 64, 8, 148),
    ([37, 200], 2, 148),
    ([37, 200], 2, 3),
    ([0, 5, 0, 64, 65], 4, 7),
    ([1, 63, 64, 65, 300, 5000, 129, 4096, 0, 7], 8, 296),
    ([0, 0], 2, 5),
])
@pytest.mark.parametrize("m", [1, 2, 4, 9])
def test_length_aware_planner(lens, Hkv, P, m):
    """The length-aware plan: every cut point of the dynamic plan that would
    leave a piece of fewer than m tiles at a segment's end moves to that end."""
    sl = np.array(lens, dtype=np.int32)
    cap = max(64, max(lens))
    la = oracle.plan(sl, Hkv, kind=3, num_ctas=P, param=m, capacity_tokens=cap, tail=(8, 4, 0))
    dyn = oracle.plan(sl, Hkv, kind=0, num_ctas=P, capacity_tokens=cap, tail=(8, 4, 0))
    _check_plan_invariants(la, lens, Hkv, 3)
    assert la["grid"] == P and la["ranges"] == dyn["ranges"]
    units = _units(lens, Hkv)
    seg_n = {}
    for (b, g, t) in units:
        seg_n[(b, g)] = seg_n.get((b, g), 0) + 1
    # pieces of every segment, from the ranges
    pieces = {}
    for c in range(la["ranges"]):
        a, e = int(la["cta"][c, 0]), int(la["cta"][c, 1])
        for u in range(a, e):
            key = units[u][:2]
            if u == a or units[u - 1][:2] != key:
                pieces.setdefault(key, []).append(0)
            pieces[key][-1] += 1
    for key, ps in pieces.items():
        assert sum(ps) == seg_n[key]
        if len(ps) > 1:
            assert ps[0] >= m and ps[-1] >= m, (key, ps)   # no end piece below m tiles
        if seg_n[key] < 2 * m:
            assert len(ps) == 1, (key, ps)            # short segments stay whole
    # every cut moved by less than m, and only where a piece would be short
    for c in range(la["ranges"]):
        for j in (0, 1):
            x, xd = int(la["cta"][c, j]), int(dyn["cta"][c, j])
            assert abs(x - xd) < m
            if 0 < xd < len(units) and units[xd][2] > 0:
                t, n = units[xd][2], seg_n[units[xd][:2]]
                if t >= m and n - t >= m:
                    assert x == xd
                else:
                    assert x in (xd - t, xd + n - t)   # an end of the segment
    if m == 1:
        for k in ("cta", "split_count", "first_slot"):
            np.testing.assert_array_equal(la[k], dyn[k])


def test_length_aware_planner_hand_cases():
    # 2 tiles, 1 kv head, 2 CTAs: the dynamic plan gives each CTA one tile;
    # with m = 2 the cut after tile 1 leaves 1 tile on each side (a tie) and
    # moves to the segment's start, so the second range holds the whole segment
    p = oracle.plan(np.array([128], dtype=np.int32), 1, kind=3, num_ctas=2, param=2,
                    capacity_tokens=128, tail=(8, 4, 0))
    np.testing.assert_array_equal(p["cta"], [[0, 0], [0, 2]])
    assert p["split_count"][0] == 1 and p["first_slot"][0] == -1
    # 3 tiles, 3 CTAs, m = 2: the cut after tile 1 (a=1, r=2) moves to the
    # start, the cut after tile 2 (a=2, r=1) to the end: one whole range
    p = oracle.plan(np.array([192], dtype=np.int32), 1, kind=3, num_ctas=3, param=2,
                    capacity_tokens=192, tail=(8, 4, 0))
    np.testing.assert_array_equal(p["cta"], [[0, 0], [0, 3], [3, 3]])
    # 8 tiles, 2 CTAs, tail (8, 4, 0): the dynamic plan has primary ranges
    # [0, 3), [3, 7) and one tail chunk [7, 8).  m = 2 keeps the cut at 3 (a=3, r=5) and moves
    # the one at 7 (r=1) to the end; m = 4 also moves the cut at 3 (a=3 < 4)
    for m, want in ((2, [[0, 3], [3, 8], [8, 8]]), (4, [[0, 0], [0, 8], [8, 8]])):
        p = oracle.plan(np.array([512], dtype=np.int32), 1, kind=3, num_ctas=2, param=m,
                        capacity_tokens=512, tail=(8, 4, 0))
        np.testing.assert_array_equal(p["cta"], want)


def test_planner_static_shapes():
    lens = [131072] + [4096] * 31
    pA = oracle.plan(np.array(lens, dtype=np.int32), 8, kind=1, num_ctas=148, max_seq_len=131072,
                     capacity_tokens=131072, tail=(8, 4, 0))
    assert pA["grid"] == 32 * 8  # ceil(148 / 256) = 1 split per (seq, kv head)
    pB = oracle.plan(np.array(lens, dtype=np.int32), 8, kind=2, num_ctas=148, max_seq_len=131072,
                     capacity_tokens=131072, tail=(8, 4, 0))
    # chunk = ceil(2048 / ceil(148 / 8)) = 108 tiles; 19 chunks per segment
    assert pB["grid"] == 32 * 8 * 19
    sizes = pB["cta"][:, 1] - pB["cta"][:, 0]
    assert sizes.max() == 108 and (sizes == 0).sum() == 31 * 8 * 18


def test_planner_clamps_lengths_to_capacity():
    p = oracle.plan(np.array([-5, 1000, 64], dtype=np.int32), 2, kind=0, num_ctas=4,
                    capacity_tokens=128, tail=(8, 4, 0))
    np.testing.assert_array_equal(p["lens"], [0, 128, 64])
    np.testing.assert_array_equal(p["tile_start"], [0, 0, 2, 3])


# ---------------------------------------------------------------- multi-token decode

@pytest.mark.parametrize("seed,lens,T,Hq,Hkv,D", [
    # tokens straddling a page edge (65 with T = 3), a sequence exactly T long,
    # one shorter than T (its first query sees nothing), an empty one
    (5, (65, 200, 3, 2, 0), 3, 8, 2, 32),
    (6, (130, 64, 17), 2, 16, 2, 64),
    (7, (300,), 4, 4, 1, 16),
])
def test_multi_token_decode_matches_causal_masked_dense(seed, lens, T, Hq, Hkv, D):
    """Query token i of a sequence of L tokens sits at position L - T + i and
    sees positions 0 .. L - T + i: written here as a dense [T x L] score
    matrix with an explicit causal mask, one numpy softmax per head."""
    shape = W.DecodeShape("mt", Hq, Hkv, D, q_tokens=T)
    batch = W.make_batch(shape, list(lens), seed=seed)
    kv = bf16_values(bits16(batch.k_cache))
    vv = bf16_values(bits16(batch.v_cache))
    qv = bf16_values(bits16(batch.q))          # [B][T][Hq][D]
    pt = batch.page_table.numpy()
    scale = 1.0 / math.sqrt(D)
    out = oracle.paged_decode_multi(bits16(batch.q), bits16(batch.k_cache),
                                    bits16(batch.v_cache), pt, batch.seq_lens.numpy(), Hkv,
                                    scale)
    G = Hq // Hkv
    for b, L in enumerate(lens):
        K = dense_kv(kv, pt, b, L)               # [L][Hkv][D]
        V = dense_kv(vv, pt, b, L)
        pos = L - T + np.arange(T)               # position of each query token
        visible = np.arange(L)[None, :] <= pos[:, None]  # [T][L]
        for h in range(Hq):
            g = h // G
            S = (qv[b, :, h, :] @ K[:, g, :].T) * scale  # [T][L]
            for i in range(T):
                if not visible[i].any():
                    np.testing.assert_array_equal(out[b, i, h], 0.0)
                    continue
                s = np.where(visible[i], S[i], -np.inf)
                p = np.exp(s - s.max())
                p /= p.sum()
                np.testing.assert_allclose(out[b, i, h], p @ V[:, g, :], rtol=0, atol=1e-12)


def test_multi_token_last_query_equals_single_token_decode():
    """The last of T query tokens sees the whole sequence: it is the
    single-token decode of that query (a different entry point of the oracle
    computes it)."""
    shape = W.DecodeShape("mt", 8, 2, 64, q_tokens=3)
    batch = W.make_batch(shape, [100, 3, 70], seed=9)
    args = (bits16(batch.k_cache), bits16(batch.v_cache), batch.page_table.numpy(),
            batch.seq_lens.numpy(), 2, 0.125)
    multi = oracle.paged_decode_multi(bits16(batch.q), *args)
    single = oracle.paged_decode(np.ascontiguousarray(bits16(batch.q)[:, -1]), *args)
    np.testing.assert_array_equal(multi[:, -1], single)


@pytest.mark.parametrize("U,P,has_tail", [(4096, 296, False), (9471, 296, False),
                                          (9472, 296, True), (32256, 296, True)])
def test_tail_needs_enough_units_per_cta(U, P, has_tail):
    """mn = 32: no run-time tail below 32 units per CTA (U < 32 P), the tail of
    den = 8 from there on."""
    p = oracle.plan(np.array([64 * U], dtype=np.int32), 1, kind=0, num_ctas=P,
                    capacity_tokens=64 * U, tail=(8, 4, 32))
    assert (p["ranges"] > P) == has_tail
    if not has_tail:
        assert [(int(a), int(e)) for a, e in p["cta"]] == _even_ranges(U, P)
    else:
        assert int(p["cta"][P][0]) == U - U // 8
