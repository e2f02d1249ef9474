"""GPU parity of the calls that let a batch be spread over GPUs: the decode
step's log-sum-exp output, the state merge, and both decompositions (by page
range with a merge, by kv head) run shard after shard on one GPU, through the
C ABI, against the fp64 oracle and against the unsharded step.

One GPU holds every shard here: the shards' decodes are separate launches that
never wait on one another, and the merge reads their states from local memory.

Tolerances as in the decode parity tests: bf16 output max-abs <= 2e-2,
mean-abs <= 2e-3 against the oracle; fp32 outputs of different schedules
(sharded vs unsharded) within 1e-3; log-sum-exps within 1e-3.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
import mixed_length_paged_b200 as hpa
from mixed_length_paged_b200 import sharding as SH
from mixed_length_paged_b200 import workloads as W
from tests.helpers import bits16, errors, oracle_decode, quantize_fp8, to_device

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS, FP8_MAX_ABS, SCHED_TOL, LSE_TOL = 2e-2, 2e-3, 5e-2, 1e-3, 1e-3


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixed_length_paged_b200 import build
    build.build()
    hpa.lib()


def _oracle_lse(batch, fp8=None):
    """[B][Hq] log-sum-exp of every row from the oracle's attention state."""
    q, pt, sl = bits16(batch.q), batch.page_table.cpu().numpy(), batch.seq_lens.cpu().numpy()
    B, Hq, D = batch.q.shape
    Hkv = batch.shape.num_kv_heads
    if fp8 is None:
        kc, vc, kw = bits16(batch.k_cache), bits16(batch.v_cache), {}
    else:
        kc, ks, vc, vs = fp8
        kw = dict(kv_fp8=True, k_scale=ks, v_scale=vs)
    out = np.empty((B, Hq))
    for b in range(B):
        for h in range(Hq):
            out[b, h] = oracle.attention_state(q, kc, vc, pt, Hkv, 1.0 / math.sqrt(D), b, h, 0,
                                               int(sl[b]), **kw)[1]
    return out


def _step(batch, *, out_dtype=torch.float32, lse=True, fp8=None, num_ctas=None, q=None,
          k_cache=None, v_cache=None, seq_lens=None, page_table=None):
    q = batch.q if q is None else q
    B, Hq, D = q.shape
    kc = batch.k_cache if k_cache is None else k_cache
    vc = batch.v_cache if v_cache is None else v_cache
    Hkv = kc.shape[1]
    pt = batch.page_table if page_table is None else page_table
    sl = batch.seq_lens if seq_lens is None else seq_lens
    kw = {}
    if fp8 is not None:
        kc, ks, vc, vs = (torch.from_numpy(x).cuda() for x in fp8)
        kw = dict(k_scale=ks, v_scale=vs)
    dec = hpa.PagedDecoder(B, Hq, Hkv, D, pt.shape[1], num_ctas=num_ctas)
    out = torch.full((B, Hq, D), float("nan"), dtype=out_dtype, device="cuda")
    l = torch.full((B, Hq), float("nan"), dtype=torch.float32, device="cuda") if lse else None
    dec.step(q, kc, vc, pt, sl, out, 1.0 / math.sqrt(D), lse=l, **kw)
    torch.cuda.synchronize()
    assert hpa.read_status(dec.workspace) == 0
    return out, l


CASES = [
    ("mixed", 64, 8, 128, [16384, 64, 4096, 1, 700, 2047, 0, 129]),
    ("skewed_small", 64, 8, 128, [32768] + [1024] * 7),
    ("d64_g4", 16, 4, 64, [37, 5000, 129, 0, 64]),
    ("g1", 8, 8, 128, [300, 1, 65]),
]


@pytest.mark.parametrize("name,Hq,Hkv,D,lens", CASES)
@pytest.mark.parametrize("num_ctas", [None, 5])
def test_step_lse_matches_oracle_and_plain_step(name, Hq, Hkv, D, lens, num_ctas):
    batch = to_device(W.make_batch(W.DecodeShape(name, Hq, Hkv, D), lens, seed=50))
    out, lse = _step(batch, num_ctas=num_ctas)
    plain, _ = _step(batch, lse=False, num_ctas=num_ctas)
    # the log-sum-exp output leaves the attention output bit for bit as it was
    assert torch.equal(out, plain)
    mx, mn = errors(out, oracle_decode(batch))
    assert mx <= MAX_ABS and mn <= MEAN_ABS, (mx, mn)
    ref = _oracle_lse(batch)
    got = lse.cpu().numpy().astype(np.float64)
    empty = batch.seq_lens.cpu().numpy() == 0
    assert np.isneginf(got[empty]).all()
    assert np.abs(got[~empty] - ref[~empty]).max() <= LSE_TOL
    # bf16 output: the same log-sum-exps
    out16, lse16 = _step(batch, out_dtype=torch.bfloat16, num_ctas=num_ctas)
    assert torch.equal(lse16, lse)


def test_step_lse_fp8():
    batch = W.make_batch(W.DecodeShape("f8", 64, 8, 128, kv_dtype="fp8_e4m3"), [3000, 1, 640, 77],
                         seed=51)
    fp8 = quantize_fp8(batch)
    to_device(batch)
    out, lse = _step(batch, fp8=fp8)
    mx, _ = errors(out, oracle_decode(batch, fp8=fp8))
    assert mx <= FP8_MAX_ABS, mx
    ref = _oracle_lse(batch, fp8=fp8)
    assert np.abs(lse.cpu().numpy() - ref).max() <= LSE_TOL


def test_step_lse_multi_token():
    B, T, Hq, Hkv, D = 3, 2, 16, 2, 128
    batch = to_device(W.make_batch(W.DecodeShape("mt", Hq, Hkv, D), [900, 1, 2], seed=52))
    q = torch.randn(B, T, Hq, D, generator=torch.Generator().manual_seed(53)).to(torch.bfloat16).cuda()
    dec = hpa.PagedDecoder(B, Hq, Hkv, D, batch.pt_stride, q_tokens=T)
    out = torch.empty(B, T, Hq, D, dtype=torch.float32, device="cuda")
    lse = torch.empty(B, T, Hq, dtype=torch.float32, device="cuda")
    dec.step(q, batch.k_cache, batch.v_cache, batch.page_table, batch.seq_lens, out, D ** -0.5,
             lse=lse)
    torch.cuda.synchronize()
    qb, kc, vc = bits16(q), bits16(batch.k_cache), bits16(batch.v_cache)
    pt, sl = batch.page_table.cpu().numpy(), batch.seq_lens.cpu().numpy()
    for b in range(B):
        for i in range(T):
            # query token i sits at position L - T + i and sees tokens [0, L - T + i]
            n = int(sl[b]) - T + i + 1
            for h in (0, 9, 15):
                o, l = oracle.attention_state(qb[:, i], kc, vc, pt, Hkv, D ** -0.5, b, h, 0, n)
                if n <= 0:
                    assert lse[b, i, h].item() == -math.inf and not out[b, i, h].any()
                    continue
                assert abs(lse[b, i, h].item() - l) <= LSE_TOL
                assert np.abs(out[b, i, h].cpu().numpy() - o).max() <= MAX_ABS


# ---------------------------------------------------------------- merge_states

@pytest.mark.parametrize("n", [1, 2, 5, 16])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_merge_states_matches_oracle(n, D, out_dtype):
    g = torch.Generator().manual_seed(60 + n + D)
    rows = 1000 + 37                                  # several warps' worth and a ragged tail
    o = torch.randn(n, rows, D, generator=g)
    lse = torch.randn(n, rows, generator=g) * 4.0
    lse[:, 5] = -math.inf                             # a row no state saw
    if n > 1:
        lse[0, 7:200] = -math.inf                     # state 0 empty on some rows ...
        o[0, 7:200] = float("nan")                    # ... and never read there
        lse[1, 300] = 90.0                            # a dominant state
    o_d, l_d = o.cuda(), lse.cuda()
    out = torch.full((rows, D), float("nan"), dtype=out_dtype, device="cuda")
    lse_out = torch.full((rows,), float("nan"), device="cuda")
    hpa.merge_states(list(o_d), list(l_d), out, lse_out)
    torch.cuda.synchronize()
    got, gl = out.float().cpu().numpy(), lse_out.cpu().numpy()
    tol = 1e-5 if out_dtype == torch.float32 else 1e-2
    for r in range(rows):
        ro, rl = oracle.merge_states(o[:, r].double().numpy(), lse[:, r].double().numpy())
        assert np.abs(got[r] - ro).max() <= tol * max(1.0, np.abs(ro).max()), r
        if rl == -math.inf:
            assert gl[r] == -math.inf
        else:
            assert abs(gl[r] - rl) <= 1e-5 * max(1.0, abs(rl)), r
    if n == 1 and out_dtype == torch.float32:
        # one state: the identity, bit for bit
        finite = ~torch.isneginf(lse[0])
        assert torch.equal(out.cpu()[finite], o[0][finite])
        assert torch.equal(lse_out.cpu()[finite], lse[0][finite])


# ---------------------------------------------------------------- decompositions

SHARD_CASES = [
    ("mixed", 64, 8, 128, [16384, 64, 4096, 1, 700, 2047, 0, 129]),
    ("d64", 16, 4, 64, [37, 5000, 129, 0, 64, 1]),
]


@pytest.mark.parametrize("name,Hq,Hkv,D,lens", SHARD_CASES)
@pytest.mark.parametrize("N", [2, 3, 4, 8])
def test_page_sharded_decode_equals_unsharded(name, Hq, Hkv, D, lens, N):
    batch = to_device(W.make_batch(W.DecodeShape(name, Hq, Hkv, D), lens, seed=70 + N))
    whole, whole_lse = _step(batch)
    o_parts, l_parts = [], []
    for r in range(N):
        lr, ptr = SH.page_shard(batch.seq_lens, batch.page_table, N, r)
        o, l = _step(batch, seq_lens=lr.cuda(), page_table=ptr.cuda())
        o_parts.append(o)
        l_parts.append(l)
    out = torch.full_like(whole, float("nan"))
    lse = torch.full_like(whole_lse, float("nan"))
    hpa.merge_states(o_parts, l_parts, out, lse)
    out16 = torch.empty(whole.shape, dtype=torch.bfloat16, device="cuda")
    hpa.merge_states(o_parts, l_parts, out16)
    torch.cuda.synchronize()
    assert (out - whole).abs().max().item() <= SCHED_TOL
    fin = torch.isfinite(whole_lse)
    assert torch.equal(torch.isneginf(lse), ~fin)
    assert (lse[fin] - whole_lse[fin]).abs().max().item() <= LSE_TOL
    mx, mn = errors(out16, oracle_decode(batch))
    assert mx <= MAX_ABS and mn <= MEAN_ABS, (mx, mn)


@pytest.mark.parametrize("N", [2, 4, 8])
def test_head_sharded_decode_equals_unsharded(N):
    Hq, Hkv, D = 64, 8, 128
    batch = to_device(W.make_batch(W.DecodeShape("hs", Hq, Hkv, D), [9000, 1, 640, 0, 77],
                                   seed=80 + N))
    whole, whole_lse = _step(batch)
    outs, lses = [], []
    for r in range(N):
        (g0, g1), (h0, h1) = SH.head_shard(Hq, Hkv, N, r)
        o, l = _step(batch, q=batch.q[:, h0:h1].contiguous(),
                     k_cache=batch.k_cache[:, g0:g1].contiguous(),
                     v_cache=batch.v_cache[:, g0:g1].contiguous())
        outs.append(o)
        lses.append(l)
    out, lse = torch.cat(outs, dim=1), torch.cat(lses, dim=1)
    assert (out - whole).abs().max().item() <= SCHED_TOL
    fin = torch.isfinite(whole_lse)
    assert (lse[fin] - whole_lse[fin]).abs().max().item() <= LSE_TOL
    mx, mn = errors(out, oracle_decode(batch))
    assert mx <= MAX_ABS and mn <= MEAN_ABS, (mx, mn)


def test_page_sharded_decoder_single_rank_is_the_plain_step():
    # outside a process group the sharded decoder is the local step plus a
    # one-state merge, which is the identity: the same bits as the plain step
    Hq, Hkv, D = 64, 8, 128
    batch = to_device(W.make_batch(W.DecodeShape("one", Hq, Hkv, D), [4096, 33, 0, 700], seed=90))
    plain, _ = _step(batch, out_dtype=torch.bfloat16, lse=False)
    dec = SH.PageShardedDecoder(4, Hq, Hkv, D, batch.pt_stride)
    out = torch.full_like(plain, float("nan"))
    dec.step(batch.q, batch.k_cache, batch.v_cache, batch.page_table, batch.seq_lens, out,
             D ** -0.5)
    torch.cuda.synchronize()
    assert torch.equal(out, plain)


def test_page_sharded_skewed_workload_full_size():
    # the benchmark's skewed batch (1 x 131072 + 31 x 4096 tokens) over 8 page
    # shares: every row against the unsharded step, sampled rows against the
    # oracle (the 128K-token sequence among them)
    from tests.helpers import compact_rows
    batch = W.build("skewed", device="cuda")
    whole, whole_lse = _step(batch)
    R = 8
    o_parts, l_parts = [], []
    for r in range(R):
        lr, ptr = SH.page_shard(batch.seq_lens, batch.page_table, R, r)
        o, l = _step(batch, seq_lens=lr.cuda(), page_table=ptr.cuda())
        o_parts.append(o)
        l_parts.append(l)
    out = torch.empty(whole.shape, dtype=torch.bfloat16, device="cuda")
    out32 = torch.empty_like(whole)
    lse = torch.empty_like(whole_lse)
    hpa.merge_states(o_parts, l_parts, out32, lse)
    hpa.merge_states(o_parts, l_parts, out)
    torch.cuda.synchronize()
    assert (out32 - whole).abs().max().item() <= SCHED_TOL
    assert (lse - whole_lse).abs().max().item() <= LSE_TOL
    rows = [0, 1, 17, 31]
    ref = oracle_decode(compact_rows(batch, rows))
    mx, mn = errors(out[rows], ref)
    assert mx <= MAX_ABS and mn <= MEAN_ABS, (mx, mn)


def test_merge_states_refuses_unreachable_pointers():
    """A pageable host buffer passed as a state or as the output is refused
    on the host with HPA_ERR_INVALID_ARG and nothing is launched; device and
    mapped pinned buffers are accepted."""
    import ctypes as C
    rows, D = 8, 64
    o = torch.randn(rows, D, device="cuda")
    lse = torch.randn(rows, device="cuda")
    out = torch.empty(rows, D, device="cuda")
    host_o = torch.randn(rows, D)                       # pageable host memory
    host_out = torch.empty(rows, D)
    L = hpa.lib()

    def call(o_ptrs, lse_ptrs, out_ptr):
        op = (C.c_void_p * len(o_ptrs))(*o_ptrs)
        lp = (C.c_void_p * len(lse_ptrs))(*lse_ptrs)
        return L.hpa_merge_states(op, lp, len(o_ptrs), rows, D, out_ptr, 1, None, None)

    assert call([o.data_ptr(), host_o.data_ptr()], [lse.data_ptr()] * 2, out.data_ptr()) == 1
    assert call([o.data_ptr()], [lse.data_ptr()], host_out.data_ptr()) == 1
    pinned = torch.randn(rows, D).pin_memory()
    assert call([o.data_ptr(), pinned.data_ptr()], [lse.data_ptr()] * 2, out.data_ptr()) == 0
    torch.cuda.synchronize()
    assert call([o.data_ptr()], [lse.data_ptr()], out.data_ptr()) == 0
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out.cpu().numpy(), o.cpu().numpy())  # one state: identity
