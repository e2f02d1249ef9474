"""The allocation-free decode entry point (hpa_decode_noalloc).

Some callers cannot allocate device memory where they issue a decode step:
code running inside a device memory pool that must not grow after start-up,
code whose allocator belongs to another framework and is not reachable from
there, or a C program that keeps cudaMalloc off its hot path.  For them the
library keeps its scratch in a static 16 MiB device array.  These tests check
that this entry point gives the same bits as the regular workspace-based plan
+ run over the same CTA count, on calls in a row of both of its forms (the
plan inside the decode kernel up to 512 sequences, the plan kernel above) in
both orders -- a call must not be disturbed by what the one before left in the
shared array -- with bf16 and FP8 caches and head_dim 64 and 128; that it
matches the fp64 oracle; that a bad page id shows in the array's status word;
and that an oversized request is refused on the host.

This file is named so that pytest collects it last.
"""
from __future__ import annotations

import ctypes as C
import math

import numpy as np
import pytest
import torch

import mixed_length_paged_b200 as hpa
from mixed_length_paged_b200 import workloads as W
from tests.helpers import errors, oracle_decode, quantize_fp8

MAX_ABS, MEAN_ABS, FP8_MAX_ABS = 2e-2, 2e-3, 5e-2


@pytest.fixture(scope="module")
def L():
    from mixed_length_paged_b200 import build
    build.build()
    return hpa.lib()


def _sms():
    return torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count


def _fp8_tensors(fp8):
    kc, ks, vc, vs = (torch.from_numpy(x).cuda() for x in fp8)
    return kc, vc, dict(k_scale=ks, v_scale=vs)


def _reference(batch, out_dtype, fp8=None):
    """The existing entry points over the CTA count noalloc uses by default
    (one per SM): caller-allocated workspace, plan + run."""
    dev = batch.q.device
    B, Hq, D = batch.q.shape
    Hkv = batch.k_cache.shape[1]
    n = _sms()
    ws = torch.empty(hpa.decode_workspace_size(hpa.PLAN_DYNAMIC, B, Hkv, Hq, D, n),
                     dtype=torch.uint8, device=dev)
    # (an e4m3 cache: the cost weights noalloc's plan uses for it)
    grid = hpa.decode_plan(batch.seq_lens, num_kv_heads=Hkv, num_q_heads=Hq, head_dim=D,
                           pt_stride=batch.pt_stride, workspace=ws, num_ctas=n,
                           cost=None if fp8 is None
                           else (hpa.COST_UNIT_DEFAULT, hpa.COST_END_DEFAULT_FP8))
    out = torch.empty(B, Hq, D, dtype=out_dtype, device=dev)
    kc, vc, kw = (batch.k_cache, batch.v_cache, {}) if fp8 is None else _fp8_tensors(fp8)
    hpa.decode_run(batch.q, kc, vc, batch.page_table, out, ws, grid, 1.0 / math.sqrt(D), **kw)
    torch.cuda.synchronize()
    assert hpa.read_status(ws) == 0
    return out


def _noalloc(batch, out_dtype, fp8=None):
    B, Hq, D = batch.q.shape
    out = torch.full((B, Hq, D), float("nan"), dtype=out_dtype, device=batch.q.device)
    kc, vc, kw = (batch.k_cache, batch.v_cache, {}) if fp8 is None else _fp8_tensors(fp8)
    hpa.decode_noalloc(batch.q, kc, vc, batch.page_table, batch.seq_lens, out,
                       1.0 / math.sqrt(D), **kw)
    torch.cuda.synchronize()
    return out


def _on_gpu(batch):
    for name in ["seq_lens", "page_table", "k_cache", "v_cache", "q"]:
        setattr(batch, name, getattr(batch, name).cuda())
    return batch


def _large_batch(seed):
    # more sequences than the in-kernel plan holds: the plan kernel runs first
    lens = np.random.default_rng(seed).integers(0, 400, 600).tolist()
    return W.make_batch(W.DecodeShape("na_big", 16, 4, 64), lens, seed=seed)


@pytest.mark.gpu
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_noalloc_matches_workspace_path_on_two_calls(L, out_dtype):
    first = W.make_batch(W.DecodeShape("na1", 64, 8, 128), [16384, 64, 4096, 1, 700, 2047],
                         seed=21)
    second = W.make_batch(W.DecodeShape("na2", 16, 4, 128), [37, 5000, 129], seed=22)
    refs = [oracle_decode(b) for b in (first, second)]
    hpa.noalloc_read_status(clear=True)
    for batch, ref in zip((_on_gpu(first), _on_gpu(second)), refs):
        got = _noalloc(batch, out_dtype)
        assert torch.equal(got, _reference(batch, out_dtype))
        mx, mn = errors(got, ref)
        assert mx <= MAX_ABS and mn <= MEAN_ABS, (mx, mn)
    assert hpa.noalloc_read_status() == 0


@pytest.mark.gpu
def test_noalloc_both_plan_forms_in_both_orders(L):
    """Above 512 sequences the plan kernel writes the array's plan; up to 512
    the decode kernel plans itself and shares the header counters at offset 0.
    Calls alternate large, small, large, small and each equals plan + run."""
    big = _on_gpu(_large_batch(24))
    small = _on_gpu(W.make_batch(W.DecodeShape("na_s", 16, 4, 64), [3000, 1, 64, 65, 900],
                                 seed=25))
    refs = {id(big): _reference(big, torch.float32), id(small): _reference(small, torch.float32)}
    for batch in (big, small, big, small):
        assert torch.equal(_noalloc(batch, torch.float32), refs[id(batch)])
    ref = oracle_decode(big)
    mx, mn = errors(refs[id(big)], ref)
    assert mx <= MAX_ABS and mn <= MEAN_ABS, (mx, mn)


@pytest.mark.gpu
@pytest.mark.parametrize("lens", [
    [1, 63, 64, 65, 700, 3000],
    [64] * 100 + [4000] * 20 + [1, 130] * 10,   # the e4m3 cost weights move the cuts
    [64] * 500 + [3000] * 20,                    # above 512 sequences: the plan kernel
])
def test_noalloc_fp8_cache(L, lens):
    shape = W.DecodeShape("na_f8", 64, 8, 128, kv_dtype="fp8_e4m3")
    batch = W.make_batch(shape, lens, seed=26)
    fp8 = quantize_fp8(batch)
    ref64 = oracle_decode(batch, fp8=fp8)
    _on_gpu(batch)
    got = _noalloc(batch, torch.bfloat16, fp8=fp8)
    assert torch.equal(got, _reference(batch, torch.bfloat16, fp8=fp8))
    mx, _ = errors(got, ref64)
    assert mx <= FP8_MAX_ABS, mx


@pytest.mark.gpu
def test_noalloc_repeated_call_is_stable(L):
    batch = _on_gpu(W.make_batch(W.DecodeShape("na3", 32, 8, 128), [9000, 100], seed=23))
    a = _noalloc(batch, torch.float32).clone()
    b = _noalloc(batch, torch.float32)
    assert torch.equal(a, b)


@pytest.mark.gpu
def test_noalloc_status_word_shows_a_bad_page(L):
    """A page id outside the cache is skipped by the kernel (no access is
    made) and flagged in the array's status word, which the caller reads and
    clears without allocating."""
    batch = _on_gpu(W.make_batch(W.DecodeShape("na4", 16, 4, 64), [200, 70], seed=27))
    hpa.noalloc_read_status(clear=True)
    _noalloc(batch, torch.float32)
    assert hpa.noalloc_read_status() == 0
    batch.page_table[1, 1] = batch.k_cache.shape[0] + 5   # past the last page
    _noalloc(batch, torch.float32)
    assert hpa.noalloc_read_status(clear=True) & hpa.DEVICE_BAD_PAGE
    assert hpa.noalloc_read_status() == 0


def test_noalloc_refuses_oversized_request_on_host(L):
    # 2,000,000 sequences x 8 kv heads of per-segment plan data cannot fit in
    # the static array; refused before any CUDA call, so this runs without a GPU.
    need = hpa.decode_workspace_size(hpa.PLAN_DYNAMIC, 2_000_000, 8, 64, 128, 148)
    assert need > hpa.NOALLOC_SCRATCH_BYTES
    rc = L.hpa_decode_noalloc(256, 256, 256, None, None, 0, 256, 4, 8, 256, 256, 0, 2_000_000, 64,
                              8, 128, C.c_float(0.088), 148, None)
    assert rc == 3  # HPA_ERR_WORKSPACE
    # bad arguments are refused before anything is enqueued, too
    rc = L.hpa_decode_noalloc(None, 256, 256, None, None, 0, 256, 4, 8, 256, 256, 0, 2, 8, 2, 64,
                              C.c_float(0.125), 148, None)
    assert rc == 1
    assert L.hpa_noalloc_read_status(None, 0, None) == 1
