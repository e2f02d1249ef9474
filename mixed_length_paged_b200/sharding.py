"""One decode batch spread over the ranks of a process group.

The pages put the attention kernels in tensor- and expert-parallel serving
on one node, where cross-GPU communication and its overlap with compute set
the throughput (openai-hub.com news/688).  Decode attention splits over GPUs
in two ways that need no exchange inside the attention itself:

* by kv head: rank r of N holds kv heads [r Hkv/N, (r+1) Hkv/N) of every page
  and the q heads of their groups.  Its decode is the plain decode of that
  head slice; the ranks' outputs are disjoint head ranges of the full output
  (what a tensor-parallel layer's output projection consumes as it is).
* by page: tile t of sequence b (tokens [64 t, 64 t + 64)) is held by rank
  (s_b + t) mod N, where s_b is the sequence's start rank.  A single-token
  query attends every earlier token, so a rank's share of a sequence -- its
  tiles in order, only the sequence's last tile possibly partial -- is an
  ordinary shorter sequence.  Each rank computes its rows' normalised outputs
  and log-sum-exps (hpa_decode_step_lse); the ranks all-gather them
  (B Hq (D + 1) fp32 per rank) and every rank combines them with the
  log-sum-exp merge (hpa_merge_states) -- the split-KV recombination of
  xiaodao.ai "HPC-Ops TPOT -48.8%" (Attention section) carried across GPUs.

The page rule is stable under decode: a tile's rank depends only on its index
and the sequence's start rank, so as a sequence grows no page that has been
written ever changes rank, and each rank's page list only grows at its end.
A new page goes to the rank after the one holding the previous tile, so
every sequence stays spread within one tile of even, and start ranks that
differ between sequences (by default s_b = b mod N) spread the batch's odd
tiles over the ranks.  (Cutting each sequence into N contiguous runs would
keep a rank's tokens contiguous, but every new page would shift the run
boundaries and move written pages between ranks.)

The split of pages and heads is host logic run when a cache is laid out and
when a sequence gets a new page; the per-step work runs in the library's
kernels plus one collective.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (HpaError, MAX_MERGE_STATES, MAX_STEP_BATCH, PAGE_SIZE, PagedDecoder,
               merge_states)

__all__ = ["head_shard", "page_owner", "page_shard", "gather_states", "PageShardedDecoder"]


def head_shard(num_q_heads: int, num_kv_heads: int, num_shards: int, shard: int):
    """((g0, g1), (h0, h1)): the kv heads and q heads rank ``shard`` of
    ``num_shards`` holds when the heads are split evenly (GQA groups stay
    whole: q head h belongs to kv head h // (num_q_heads / num_kv_heads))."""
    if num_shards < 1 or not 0 <= shard < num_shards:
        raise HpaError(f"head_shard: shard {shard} of {num_shards}")
    if num_kv_heads % num_shards or num_q_heads % num_kv_heads:
        raise HpaError(f"head_shard: {num_kv_heads} kv heads / {num_q_heads} q heads do not "
                       f"split over {num_shards} ranks")
    per = num_kv_heads // num_shards
    G = num_q_heads // num_kv_heads
    g0, g1 = shard * per, (shard + 1) * per
    return (g0, g1), (g0 * G, g1 * G)


def page_owner(tile, start, num_shards: int):
    """Rank holding tile ``tile`` of a sequence whose start rank is ``start``
    (scalars or arrays): (start + tile) mod num_shards."""
    return (np.asarray(start, dtype=np.int64) + np.asarray(tile, dtype=np.int64)) % num_shards


def page_shard(seq_lens, page_table, num_shards: int, shard: int, start=None):
    """(lens_r, page_table_r), int32 CPU tensors: rank ``shard``'s share of
    every sequence when tile t of sequence b is held by rank
    page_owner(t, start[b], N) = (start[b] + t) mod N.  ``start`` [B] gives
    each sequence's start rank (default b mod N; keep it with the sequence
    for as long as it lives).  page_table_r[b] lists the rank's pages in tile
    order and keeps the input's width (unused entries are 0 and never read);
    lens_r[b] counts the tokens in them: 64 per tile, less the unfilled part
    of the sequence's last tile if the rank holds it (that tile is then last
    in its list, so only a list's last page is ever partial)."""
    if num_shards < 1 or not 0 <= shard < num_shards:
        raise HpaError(f"page_shard: shard {shard} of {num_shards}")
    L = np.asarray(torch.as_tensor(seq_lens).cpu(), dtype=np.int64)
    pt = np.asarray(torch.as_tensor(page_table).cpu(), dtype=np.int32)
    if L.ndim != 1 or pt.ndim != 2 or pt.shape[0] != L.shape[0]:
        raise HpaError("page_shard: seq_lens [B] and page_table [B][pt_stride] expected")
    if (L < 0).any():
        raise HpaError("page_shard: negative length")
    B = L.shape[0]
    st = np.arange(B, dtype=np.int64) % num_shards if start is None else \
        np.asarray(torch.as_tensor(start).cpu(), dtype=np.int64)
    if st.shape != (B,) or (st < 0).any() or (st >= num_shards).any():
        raise HpaError("page_shard: start ranks [B] in [0, num_shards) expected")
    n = (L + PAGE_SIZE - 1) // PAGE_SIZE
    if (n > pt.shape[1]).any():
        raise HpaError("page_shard: a sequence needs more pages than page_table holds")
    first = (shard - st) % num_shards                      # this rank's first tile of b
    count = np.where(n > first, (n - first + num_shards - 1) // num_shards, 0)
    holds_last = (n > 0) & (page_owner(n - 1, st, num_shards) == shard)
    lens = count * PAGE_SIZE - np.where(holds_last, n * PAGE_SIZE - L, 0)
    out = np.zeros_like(pt)
    for b in range(B):
        out[b, :count[b]] = pt[b, first[b]:n[b]:num_shards]
    return torch.from_numpy(lens.astype(np.int32)), torch.from_numpy(out)


def _world(group) -> int:
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return 1
    return dist.get_world_size(group)


def gather_states(o_local: torch.Tensor, lse_local: torch.Tensor, group=None, *,
                  o_all=None, lse_all=None):
    """Every rank's (o, lse) state, in rank order, on every rank: an
    all-gather over ``group`` (one collective per tensor), or the local pair
    alone outside a process group of several ranks.  ``o_all`` / ``lse_all``:
    optional lists of receive tensors (one per rank, shaped like the local
    ones), so that a step allocates nothing."""
    import torch.distributed as dist
    n = _world(group)
    if n == 1:
        return [o_local], [lse_local]
    if n > MAX_MERGE_STATES:
        raise HpaError(f"gather_states: at most {MAX_MERGE_STATES} ranks merge in one call")
    if o_all is None:
        o_all = [torch.empty_like(o_local) for _ in range(n)]
    if lse_all is None:
        lse_all = [torch.empty_like(lse_local) for _ in range(n)]
    if len(o_all) != n or len(lse_all) != n:
        raise HpaError("gather_states: one receive tensor per rank")
    dist.all_gather(o_all, o_local, group=group)
    dist.all_gather(lse_all, lse_local, group=group)
    return o_all, lse_all


class PageShardedDecoder:
    """Single-token decode of a batch whose sequences' pages are spread over
    the ranks of ``group`` as ``page_shard`` lays them out: the local decode
    with log-sum-exps, an all-gather of the ranks' states, and the merge, all
    on the current stream.  Every rank calls ``step`` with its own share
    (lengths, page table, caches) and gets the whole output."""

    def __init__(self, batch: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                 pt_stride: int, *, group=None, num_ctas: int | None = None, device=None):
        if batch > MAX_STEP_BATCH:
            raise HpaError(f"PageShardedDecoder: batch <= {MAX_STEP_BATCH}")
        world = _world(group)
        if world > MAX_MERGE_STATES:
            raise HpaError(f"PageShardedDecoder: at most {MAX_MERGE_STATES} ranks")
        self.group = group
        self.dec = PagedDecoder(batch, num_q_heads, num_kv_heads, head_dim, pt_stride,
                                num_ctas=num_ctas, device=device)
        dev = self.dec.device
        self.o_local = torch.empty(batch, num_q_heads, head_dim, dtype=torch.float32, device=dev)
        self.lse_local = torch.empty(batch, num_q_heads, dtype=torch.float32, device=dev)
        # receive buffers of the all-gather, allocated once
        self.o_all = [torch.empty_like(self.o_local) for _ in range(world)] if world > 1 else None
        self.lse_all = [torch.empty_like(self.lse_local) for _ in range(world)] if world > 1 else None

    def step(self, q, k_cache, v_cache, page_table, seq_lens, out, softmax_scale, *,
             k_scale=None, v_scale=None, lse_out=None):
        self.dec.step(q, k_cache, v_cache, page_table, seq_lens, self.o_local, softmax_scale,
                      k_scale=k_scale, v_scale=v_scale, lse=self.lse_local)
        o_all, lse_all = gather_states(self.o_local, self.lse_local, self.group,
                                       o_all=self.o_all, lse_all=self.lse_all)
        return merge_states(o_all, lse_all, out, lse_out)
