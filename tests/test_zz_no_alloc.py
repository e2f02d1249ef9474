"""The allocation-free decode entry point (hpa_decode_noalloc).

Some callers cannot allocate device memory where they issue a decode step:
code running inside a device memory pool that must not grow after start-up,
code whose allocator belongs to another framework and is not reachable from
there, or a C program that keeps cudaMalloc off its hot path.  For them the
library keeps its scratch in a static 16 MiB device array.  These tests check
that this entry point gives the same result as the regular workspace-based
plan + run on two calls in a row (the second call must not be disturbed by
what the first left in the shared array), and that an oversized request is
refused on the host.

This file is named so that pytest collects it last.
"""
from __future__ import annotations

import ctypes as C
import math

import pytest
import torch

import mixed_length_paged_b200 as hpa
from mixed_length_paged_b200 import workloads as W

SCHED_TOL = 1e-3  # schedules/entry points must agree within this in fp32 output


@pytest.fixture(scope="module")
def L():
    from mixed_length_paged_b200 import build
    build.build()
    return hpa.lib()


def _reference(batch, out_dtype):
    """The existing entry points: caller-allocated workspace, plan + run."""
    dev = batch.q.device
    B, Hq, D = batch.q.shape
    Hkv = batch.k_cache.shape[1]
    n = hpa.default_num_ctas(dev.index)
    ws = torch.empty(hpa.decode_workspace_size(hpa.PLAN_DYNAMIC, B, Hkv, Hq, D, n),
                     dtype=torch.uint8, device=dev)
    grid = hpa.decode_plan(batch.seq_lens, num_kv_heads=Hkv, num_q_heads=Hq, head_dim=D,
                           pt_stride=batch.pt_stride, workspace=ws, num_ctas=n)
    out = torch.empty(B, Hq, D, dtype=out_dtype, device=dev)
    hpa.decode_run(batch.q, batch.k_cache, batch.v_cache, batch.page_table, out, ws, grid,
                   1.0 / math.sqrt(D))
    return out


def _noalloc(batch, out_dtype):
    B, Hq, D = batch.q.shape
    out = torch.full((B, Hq, D), float("nan"), dtype=out_dtype, device=batch.q.device)
    return hpa.decode_noalloc(batch.q, batch.k_cache, batch.v_cache, batch.page_table,
                              batch.seq_lens, out, 1.0 / math.sqrt(D))


def _on_gpu(batch):
    for name in ["seq_lens", "page_table", "k_cache", "v_cache", "q"]:
        setattr(batch, name, getattr(batch, name).cuda())
    return batch


@pytest.mark.gpu
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_noalloc_matches_workspace_path_on_two_calls(L, out_dtype):
    first = _on_gpu(W.make_batch(W.DecodeShape("na1", 64, 8, 128),
                                 [16384, 64, 4096, 1, 700, 2047], seed=21))
    second = _on_gpu(W.make_batch(W.DecodeShape("na2", 16, 4, 128),
                                  [37, 5000, 129], seed=22))
    results = []
    for batch in (first, second):
        got = _noalloc(batch, out_dtype)
        torch.cuda.synchronize()
        ref = _reference(batch, out_dtype)
        torch.cuda.synchronize()
        assert torch.isfinite(got.float()).all()
        results.append((got.float() - ref.float()).abs().max().item())
    # the same kernels on the same plan: agreement within the schedule tolerance
    assert max(results) <= SCHED_TOL, results


@pytest.mark.gpu
def test_noalloc_repeated_call_is_stable(L):
    batch = _on_gpu(W.make_batch(W.DecodeShape("na3", 32, 8, 128), [9000, 100], seed=23))
    a = _noalloc(batch, torch.float32).clone()
    b = _noalloc(batch, torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


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
