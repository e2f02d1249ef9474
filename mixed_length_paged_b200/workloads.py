"""Seeded synthetic decode workloads: the inputs of one decode step.

This module draws random numbers and lays them out; it holds none of the
attention, normalisation, rotary or quantisation arithmetic.  Both the CUDA
path's tests/benchmark and the fp64 oracle consume what it returns.

Workload shapes follow the batch shapes reported for the HPC-Ops dynamic
decode scheduler (xiaodao.ai "HPC-Ops TPOT -48.8%", section on Attention:
uniform 64 x 0.5K, skewed 1 x 128K + 31 x 4K, and continuous-batching mixes
of 1K..64K lengths) and the paged layout of the schematic attention call
(openai-hub.com news/688, the illustrative ``kv_cache_layout="paged"``
example).

Physical layout (shared by every consumer):
  k_cache, v_cache : [num_pages][Hkv][PAGE_SIZE][D]   (bf16, or e4m3 codes)
  page_table       : [B][pt_stride] int32, -1 past a sequence's last page
  seq_lens         : [B] int32 (tokens attended this step)
Slots past a sequence's length in its last page, and a few spare physical
pages that no table entry references, are filled with NaN so that any read
of them shows up in the output.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

PAGE_SIZE = 64


@dataclass(frozen=True)
class DecodeShape:
    """Head geometry and cache dtype of one workload."""

    name: str
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    kv_dtype: str = "bf16"  # "bf16" or "fp8_e4m3"
    prologue: bool = False
    q_tokens: int = 1       # query tokens per sequence (multi-token decode if > 1)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads


SHAPES = {
    "tiny": DecodeShape("tiny", 8, 2, 64),
    "uniform": DecodeShape("uniform", 64, 8, 128),
    "skewed": DecodeShape("skewed", 64, 8, 128),
    # the skewed shape at a quarter of the lengths (264 MB of KV, above the
    # 126 MB L2): the size used for detailed profiler captures
    "skewed_quarter": DecodeShape("skewed_quarter", 64, 8, 128),
    "mix_prologue": DecodeShape("mix_prologue", 32, 8, 128, prologue=True),
    "fp8": DecodeShape("fp8", 64, 8, 128, kv_dtype="fp8_e4m3"),
    # the first 64 sequences of the fp8 batch (~0.3 GB of e4m3 KV, above the
    # L2): the size used for detailed profiler captures of the FP8 kernel
    "fp8_quarter": DecodeShape("fp8_quarter", 64, 8, 128, kv_dtype="fp8_e4m3"),
    # the skewed batch with two query tokens per sequence (a draft token to
    # verify, or a multi-token-prediction head): 8 heads x 2 tokens per kv head
    "skewed_mtp2": DecodeShape("skewed_mtp2", 64, 8, 128, q_tokens=2),
    # four query tokens per sequence: 32 query rows per kv head (four MMA n-tiles)
    "skewed_mtp4": DecodeShape("skewed_mtp4", 64, 8, 128, q_tokens=4),
}


def cache_lengths(name: str, seed: int = 0) -> np.ndarray:
    """KV lengths held in the cache before the step (int64, one per sequence).

    For the prologue workload the step appends one token, so attention runs
    over ``cache_lengths + 1`` tokens; for every other workload attention runs
    over exactly these lengths.
    """
    rng = np.random.default_rng(seed)
    if name == "tiny":
        return np.array([37, 200], dtype=np.int64)
    if name == "uniform":
        return np.full(64, 512, dtype=np.int64)
    if name in ("skewed", "skewed_mtp2", "skewed_mtp4"):
        return np.array([131072] + [4096] * 31, dtype=np.int64)
    if name == "skewed_quarter":
        return np.array([32768] + [1024] * 31, dtype=np.int64)
    if name == "mix_prologue":
        u = rng.uniform(math.log(256.0), math.log(65536.0), size=128)
        return np.rint(np.exp(u)).astype(np.int64)
    if name in ("fp8", "fp8_quarter"):
        g = rng.geometric(1.0 / 2048.0, size=256)
        g = g if name == "fp8" else g[:64]
        return np.clip(g, 1, 16384).astype(np.int64)
    raise KeyError(name)


@dataclass
class DecodeBatch:
    """All inputs of one decode step, on one device."""

    shape: DecodeShape
    seq_lens: torch.Tensor          # [B] int32, attention lengths
    page_table: torch.Tensor        # [B][pt_stride] int32
    num_pages: int
    k_cache: torch.Tensor           # [num_pages][Hkv][64][D] bf16 (or fp32 values for fp8, see below)
    v_cache: torch.Tensor
    q: torch.Tensor | None = None   # [B][Hq][D] bf16 (no prologue); [B][T][Hq][D] if q_tokens > 1
    # fp8 workloads: k_cache/v_cache hold fp32 N(0,1) values; a quantiser turns
    # them into e4m3 codes + per-(page, kv-head) scales.  live[p] counts the
    # live tokens in physical page p.
    live: torch.Tensor | None = None
    # prologue workloads: the new token's raw projections and norm weights.
    q_raw: torch.Tensor | None = None   # [B][Hq][D] bf16
    k_raw: torch.Tensor | None = None   # [B][Hkv][D] bf16
    v_raw: torch.Tensor | None = None   # [B][Hkv][D] bf16
    q_gamma: torch.Tensor | None = None  # [D] fp32
    k_gamma: torch.Tensor | None = None  # [D] fp32
    positions: torch.Tensor | None = None  # [B] int32, pre-append lengths
    extra: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return int(self.seq_lens.shape[0])

    @property
    def pt_stride(self) -> int:
        return int(self.page_table.shape[1])


def _normal(shape, gen, device, dtype):
    """N(0,1) samples: numpy PCG64 on the host, torch Philox on a GPU."""
    if gen["kind"] == "numpy":
        x = gen["rng"].standard_normal(size=shape, dtype=np.float32)
        return torch.from_numpy(x).to(dtype=dtype).to(device)
    return torch.randn(shape, generator=gen["torch"], device=device, dtype=torch.float32).to(dtype)


def _uniform(shape, lo, hi, gen, device):
    if gen["kind"] == "numpy":
        x = gen["rng"].uniform(lo, hi, size=shape).astype(np.float32)
        return torch.from_numpy(x).to(device)
    return torch.empty(shape, device=device, dtype=torch.float32).uniform_(lo, hi, generator=gen["torch"])


def make_batch(shape: DecodeShape, cache_lens, *, seed: int = 0, device="cpu",
               spare_pages: int = 3, pt_pad: int = 1, dead_fill: float = float("nan"),
               value_source: str | None = None) -> DecodeBatch:
    """Build the inputs of one decode step.

    ``cache_lens`` are the tokens already in the cache.  Without a prologue the
    step attends exactly those tokens; with one it appends a token at position
    ``cache_lens[b]`` and attends ``cache_lens[b] + 1`` tokens, so the page
    table has room for it.  Physical pages are a seeded random permutation.
    ``value_source`` picks the generator for tensor values: "numpy" (host,
    identical everywhere) or "torch" (Philox on ``device``); the default is
    numpy on the host and torch on a GPU.
    """
    cache_lens = np.asarray(cache_lens, dtype=np.int64)
    B = int(cache_lens.shape[0])
    D, Hkv, Hq = shape.head_dim, shape.num_kv_heads, shape.num_q_heads
    attn_lens = cache_lens + (1 if shape.prologue else 0)
    pages_per_seq = (attn_lens + PAGE_SIZE - 1) // PAGE_SIZE
    total_pages = int(pages_per_seq.sum())
    num_pages = total_pages + spare_pages
    pt_stride = int(max(1, pages_per_seq.max(initial=0))) + pt_pad

    rng = np.random.default_rng([seed, 1])
    perm = rng.permutation(num_pages)[:total_pages].astype(np.int32)
    page_table = np.full((B, pt_stride), -1, dtype=np.int32)
    off = 0
    for b in range(B):
        n = int(pages_per_seq[b])
        page_table[b, :n] = perm[off:off + n]
        off += n

    device = torch.device(device)
    if value_source is None:
        value_source = "numpy" if device.type == "cpu" else "torch"
    if value_source == "numpy":
        gen = {"kind": "numpy", "rng": np.random.default_rng([seed, 2])}
    else:
        g = torch.Generator(device=device)
        g.manual_seed(seed)
        gen = {"kind": "torch", "torch": g}

    fp8 = shape.kv_dtype == "fp8_e4m3"
    store = torch.float32 if fp8 else torch.bfloat16
    cache_shape = (num_pages, Hkv, PAGE_SIZE, D)
    k_cache = _normal(cache_shape, gen, device, store)
    v_cache = _normal(cache_shape, gen, device, store)

    # live tokens per physical page (cache contents before the step)
    live = np.zeros(num_pages, dtype=np.int32)
    for b in range(B):
        L = int(cache_lens[b])
        for t in range(int(pages_per_seq[b])):
            live[page_table[b, t]] = max(0, min(PAGE_SIZE, L - t * PAGE_SIZE))
    live_t = torch.from_numpy(live).to(device)
    slot = torch.arange(PAGE_SIZE, device=device).view(1, PAGE_SIZE)
    dead = (slot >= live_t.view(-1, 1)).view(num_pages, 1, PAGE_SIZE, 1)
    if fp8:
        k_cache = k_cache.masked_fill(dead, 0.0)
        v_cache = v_cache.masked_fill(dead, 0.0)
    else:
        k_cache = k_cache.masked_fill(dead, dead_fill)
        v_cache = v_cache.masked_fill(dead, dead_fill)

    batch = DecodeBatch(
        shape=shape,
        seq_lens=torch.from_numpy(attn_lens.astype(np.int32)).to(device),
        page_table=torch.from_numpy(page_table).to(device),
        num_pages=num_pages,
        k_cache=k_cache.contiguous(),
        v_cache=v_cache.contiguous(),
        live=live_t if fp8 else None,
    )
    if shape.prologue:
        batch.q_raw = _normal((B, Hq, D), gen, device, torch.bfloat16)
        batch.k_raw = _normal((B, Hkv, D), gen, device, torch.bfloat16)
        batch.v_raw = _normal((B, Hkv, D), gen, device, torch.bfloat16)
        batch.q_gamma = _uniform((D,), 0.5, 1.5, gen, device)
        batch.k_gamma = _uniform((D,), 0.5, 1.5, gen, device)
        batch.positions = torch.from_numpy(cache_lens.astype(np.int32)).to(device)
    elif shape.q_tokens > 1:
        # the q_tokens new tokens are the last q_tokens of each sequence
        batch.q = _normal((B, shape.q_tokens, Hq, D), gen, device, torch.bfloat16)
    else:
        batch.q = _normal((B, Hq, D), gen, device, torch.bfloat16)
    return batch


def build(name: str, *, seed: int = 0, device="cpu", **kw) -> DecodeBatch:
    """One of the named workloads (tiny, uniform, skewed, skewed_quarter, mix_prologue, fp8,
    fp8_quarter, skewed_mtp2, skewed_mtp4)."""
    return make_batch(SHAPES[name], cache_lengths(name, seed), seed=seed, device=device, **kw)


def live_kv_bytes(seq_lens, num_kv_heads: int, head_dim: int, elt_bytes: int) -> int:
    """Bytes of live K and V one decode step must read: sum_b L_b * 2 * Hkv * D * elt."""
    total_tokens = int(np.asarray(seq_lens, dtype=np.int64).sum())
    return total_tokens * 2 * num_kv_heads * head_dim * elt_bytes
