"""Context-parallel decode: one sequence's latent cache spread over ranks.

Each rank holds one page-aligned window of every sequence, positions
``[start, start + count)``, in its own page pool.  A decode step runs on every
rank over its window (``mla.decode_cp_partial``: the normalised latent sum and
the base-2 log-sum-exp of every new token's scores, per head), exchanges those
partials with one all-gather, and merges them (``mla.decode_cp_combine``:
log-sum-exp weights, then the W_UV up-projection).  The result is the
attention over the whole sequence, since the softmax denominators of disjoint
key sets add up.

This module is host logic only: the window plan, the per-rank page tables and
the exchange.  Every computation runs in libmla's kernels.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import numpy as np


@dataclass
class Window:
    """One rank's share of every sequence."""
    start: np.ndarray   # [B] int32, first position held (a multiple of the page size)
    count: np.ndarray   # [B] int32, positions held from there (0: none)


def shard_windows(kv_len: np.ndarray, n_ranks: int, page_size: int = 64) -> List[Window]:
    """Splits each sequence's pages into ``n_ranks`` contiguous runs of as
    equal a length as the page count allows (rank r takes pages
    ``[floor(r P / n), floor((r + 1) P / n))`` of a sequence with P pages), so
    the windows of a sequence are page-aligned, disjoint and cover
    ``[0, kv_len)``.  A rank may hold nothing of a short sequence."""
    if n_ranks <= 0:
        raise ValueError("n_ranks must be positive")
    kv = np.asarray(kv_len, dtype=np.int64)
    pages = (kv + page_size - 1) // page_size
    out = []
    for r in range(n_ranks):
        p0 = (r * pages) // n_ranks
        p1 = ((r + 1) * pages) // n_ranks
        start = p0 * page_size
        count = np.clip(np.minimum(kv, p1 * page_size) - start, 0, None)
        out.append(Window(start.astype(np.int32), count.astype(np.int32)))
    return out


@dataclass
class RankPages:
    """A rank's page pool for its window.

    ``local`` [B, max_local_pages] maps the window's i-th page to a physical
    page (what the attention reads); ``by_position`` [B, max_global_pages]
    maps a sequence's global page index to the same physical pages and holds
    -1 outside the window (what the append writes through, so that the RoPE
    key is rotated by the token's global position)."""
    local: np.ndarray
    by_position: np.ndarray
    num_pages: int


def rank_pages(win: Window, kv_len: np.ndarray, page_size: int = 64, order: Optional[np.ndarray] = None,
               spare_pages: int = 0) -> RankPages:
    """Page tables of one rank: the window's pages handed out in ``order``
    (a permutation of the pool; identity when None)."""
    need = (win.count.astype(np.int64) + page_size - 1) // page_size
    total = int(need.sum()) + spare_pages
    if order is None:
        order = np.arange(total)
    if len(order) != total:
        raise ValueError("order must be a permutation of the rank's page pool")
    B = len(need)
    max_local = max(1, int(need.max()) if B else 1)
    max_global = max(1, int(((np.asarray(kv_len, np.int64) + page_size - 1) // page_size).max()) if B else 1)
    local = np.full((B, max_local), -1, np.int32)
    by_pos = np.full((B, max_global), -1, np.int32)
    k = 0
    for b in range(B):
        n = int(need[b])
        local[b, :n] = order[k:k + n]
        g0 = int(win.start[b]) // page_size
        by_pos[b, g0:g0 + n] = order[k:k + n]
        k += n
    return RankPages(local, by_pos, total)


def gather_partials(obar_local, lse_local, group=None):
    """All-gathers every rank's partials: returns ``(obar_parts, lse_parts)``
    of shapes ``[world, *obar_local.shape]`` and ``[world, *lse_local.shape]``
    in rank order (NCCL over NVLink on GPUs, gloo on CPU)."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    out = []
    for t in (obar_local, lse_local):
        t = t.contiguous()
        # Concatenated along the first dimension (the form every backend
        # takes), then viewed per rank.
        buf = torch.empty((world * t.shape[0],) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
        dist.all_gather_into_tensor(buf, t, group=group)
        out.append(buf.view((world,) + tuple(t.shape)))
    return out[0], out[1]


def decode_cp(w, h_q, kv_len, window_start, window_count, page_table, num_pages: int, cache, out,
              max_kv_len: int, workspace, group=None):
    """One context-parallel decode step on this rank: its window's partials,
    the exchange, and the merge into ``out`` [B, n_q, n_h, d_v] (fp32, the
    same on every rank).  ``page_table`` is the rank's local table.  The
    kernels and the all-gather run on torch's current stream, in that order."""
    import torch
    from . import mla
    d = w.dims
    B, n_q = h_q.shape[0], h_q.shape[1]
    obar = torch.empty((B, n_q, d.n_h, d.d_c), dtype=h_q.dtype, device=h_q.device)
    lse = torch.empty((B, n_q, d.n_h), dtype=torch.float32, device=h_q.device)
    mla.decode_cp_partial(w, h_q, kv_len, window_start, window_count, page_table, num_pages, cache, obar, lse,
                          max_kv_len, workspace)
    obar_parts, lse_parts = gather_partials(obar, lse, group)
    mla.decode_cp_combine(w, obar_parts, lse_parts, out, workspace)
    return obar_parts, lse_parts
