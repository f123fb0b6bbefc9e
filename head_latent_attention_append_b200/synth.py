"""Seeded synthetic inputs shared by the tests, the smoke run and the benchmark.

This module holds workload shapes and random-number recipes only; none of the
attention arithmetic lives here.  Host-side draws use NumPy's PCG64 seeded by a
``SeedSequence([seed, workload_id, stream, ...])`` so any one tensor can be
regenerated on its own; values are rounded to bfloat16 (round to nearest even)
for the bf16 workloads so that the CPU and the GPU see identical inputs.

Recipe (the pages use no dataset; every workload is synthetic):
  * weights  W ~ N(0,1)/sqrt(fan_in), drawn in the order
    W_DKV, W_KR, W_DQ, W_UQ, W_QR, W_UK, W_UV (stream 0);
  * hidden states h ~ N(0,1), one stream per sequence (stream 1, b);
  * ragged cached lengths ~ U{1..32768} (stream 2);
  * physical page order: a random permutation of the page pool (stream 3);
  * cache history of sequences no check looks at: filled on the device with
    N(0,1) bf16 values, the distribution the append path produces for
    h ~ N(0,1) and these weights (each latent/key entry is a sum of D terms of
    variance 1/D), seeded through a CUDA torch.Generator.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

BASE_SEED = 20261202
PAGE_SIZE = 64


@dataclass(frozen=True)
class Workload:
    name: str
    wid: int
    n_h: int
    d_h: int
    d_v: int
    d_c: int
    d_r: int
    d_model: int
    d_cq: int
    dtype: str              # "f32" or "bf16"
    mode: str               # "decode" or "prefill"
    B: int
    n_q: int                # new query tokens per sequence (decode); S for prefill
    cached: int             # cached tokens per sequence before the queries (uniform workloads)
    ragged: bool = False
    max_cached: int = 0     # ragged: lengths drawn from U{1..max_cached}
    rope_base: float = 10000.0
    materialised: bool = False  # prefill through expanded per-head keys and values
    rope_per_head: bool = False  # one RoPE key per head in every cache row instead of one shared

    @property
    def d_cr(self) -> int:
        """Cache row width: the latent, then one shared RoPE key or n_h of them."""
        return self.d_c + (self.n_h if self.rope_per_head else 1) * self.d_r

    def flops_per_pair(self) -> int:
        """Algorithmic flops per causal (query, key) pair, all heads: the
        absorbed form scores each head over d_c + d_r columns (its own RoPE key
        in the per-head layout) and sums d_c latent columns; the materialised
        form scores over d_h + d_r and sums d_v."""
        if self.materialised:
            return self.n_h * (2 * (self.d_h + self.d_r) + 2 * self.d_v)
        return self.n_h * (2 * (self.d_c + self.d_r) + 2 * self.d_c)


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny_fp32_decode", 1, 4, 32, 32, 64, 16, 128, 0, "f32", "decode", 1, 1, 128),
        Workload("page_bf16_decode", 2, 16, 128, 128, 256, 32, 2048, 0, "bf16", "decode", 8, 1, 4096),
        Workload("dsv2_bf16_decode", 3, 128, 128, 128, 512, 64, 5120, 1536, "bf16", "decode", 64, 1, 8192),
        Workload("dsv2_bf16_prefill", 4, 128, 128, 128, 512, 64, 5120, 1536, "bf16", "prefill", 4, 4096, 0),
        Workload("dsv2_ragged_decode", 5, 128, 128, 128, 512, 64, 5120, 1536, "bf16", "decode", 128, 2, 0,
                 ragged=True, max_cached=32768),
        # Multi-token (speculative-style) decode: 4 new tokens per sequence over ragged histories.
        Workload("dsv2_spec4_decode", 6, 128, 128, 128, 512, 64, 5120, 1536, "bf16", "decode", 64, 4, 0,
                 ragged=True, max_cached=32768),
        # Config 2's model with one 32-dim RoPE key per head (cache row 256 + 16 x 32 = 768).
        Workload("page_bf16_decode_rph", 8, 16, 128, 128, 256, 32, 2048, 0, "bf16", "decode", 8, 1, 4096,
                 rope_per_head=True),
        # The causal prefill of config 4 (same seeds, same inputs) in the materialised form.
        Workload("dsv2_bf16_prefill_mat", 4, 128, 128, 128, 512, 64, 5120, 1536, "bf16", "prefill", 4, 4096, 0,
                 materialised=True),
    ]
}


def rng_for(wl_id: int, *stream: int, seed: int = BASE_SEED) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, wl_id, *stream])))


def round_bf16(x: np.ndarray) -> np.ndarray:
    """float32 -> nearest bfloat16 (ties to even), returned as float32 values."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    u = (u + (((u >> 16) & 1) + np.uint32(0x7FFF))) & np.uint32(0xFFFF0000)
    return u.view(np.float32)


def _finish(a: np.ndarray, dtype: str) -> np.ndarray:
    return round_bf16(a) if dtype == "bf16" else a.astype(np.float32)


@dataclass
class HostWeights:
    W_DKV: np.ndarray
    W_KR: np.ndarray
    W_DQ: Optional[np.ndarray]
    W_UQ: np.ndarray
    W_QR: np.ndarray
    W_UK: np.ndarray
    W_UV: np.ndarray

    def as_dict(self):
        return {k: getattr(self, k) for k in ("W_DKV", "W_KR", "W_DQ", "W_UQ", "W_QR", "W_UK", "W_UV")}


def make_weights(wl: Workload, seed: int = BASE_SEED) -> HostWeights:
    rng = rng_for(wl.wid, 0, seed=seed)
    d_in = wl.d_cq if wl.d_cq > 0 else wl.d_model

    def draw(rows, fan_in):
        return _finish(rng.standard_normal((rows, fan_in), dtype=np.float32) / np.float32(math.sqrt(fan_in)),
                       wl.dtype)

    W_DKV = draw(wl.d_c, wl.d_model)
    W_KR = draw(wl.d_r * (wl.n_h if wl.rope_per_head else 1), wl.d_model)
    W_DQ = draw(wl.d_cq, wl.d_model) if wl.d_cq > 0 else None
    W_UQ = draw(wl.n_h * wl.d_h, d_in)
    W_QR = draw(wl.n_h * wl.d_r, d_in)
    W_UK = draw(wl.n_h * wl.d_h, wl.d_c)
    W_UV = draw(wl.n_h * wl.d_v, wl.d_c)
    return HostWeights(W_DKV, W_KR, W_DQ, W_UQ, W_QR, W_UK, W_UV)


def make_hidden(wl: Workload, b: int, n_tokens: int, seed: int = BASE_SEED) -> np.ndarray:
    """Hidden states of sequence ``b``: [n_tokens, d_model], token t at position t."""
    rng = rng_for(wl.wid, 1, b, seed=seed)
    return _finish(rng.standard_normal((n_tokens, wl.d_model), dtype=np.float32), wl.dtype)


def cached_lengths(wl: Workload, seed: int = BASE_SEED) -> np.ndarray:
    """Tokens already in the cache per sequence (before the new query tokens)."""
    if wl.ragged:
        return rng_for(wl.wid, 2, seed=seed).integers(1, wl.max_cached, endpoint=True,
                                                      size=wl.B).astype(np.int32)
    if wl.mode == "prefill":
        return np.zeros(wl.B, np.int32)
    return np.full(wl.B, wl.cached, np.int32)


def kv_lengths(wl: Workload, seed: int = BASE_SEED) -> np.ndarray:
    """Keys per sequence once the new tokens are appended."""
    return cached_lengths(wl, seed) + np.int32(wl.n_q)


@dataclass
class PageLayout:
    page_table: np.ndarray      # [B, max_pages] int32, -1 where unused
    num_pages: int
    max_pages: int


def page_layout(kv_len: np.ndarray, page_size: int = PAGE_SIZE, shuffle: bool = True,
                wl_id: int = 0, seed: int = BASE_SEED, spare_pages: int = 0) -> PageLayout:
    """A page pool with exactly sum(ceil(kv_len/page)) pages (+ spares), the
    pages handed out to sequences in a random (or identity) order."""
    need = [(int(L) + page_size - 1) // page_size for L in kv_len]
    total = int(sum(need)) + spare_pages
    order = rng_for(wl_id, 3, seed=seed).permutation(total) if shuffle else np.arange(total)
    max_pages = max(need) if need else 1
    pt = np.full((len(need), max_pages), -1, np.int32)
    k = 0
    for b, n in enumerate(need):
        pt[b, :n] = order[k:k + n]
        k += n
    return PageLayout(pt, total, max_pages)


def checked_sequences(wl: Workload, lengths: np.ndarray, count: int) -> List[int]:
    """Sequences whose outputs a full-size parity run compares with the oracle:
    for ragged workloads the shortest, the longest, one with length = 63 mod 64,
    one with length = 0 mod 64 and random others; for uniform ones a seeded
    random subset."""
    B = len(lengths)
    rng = rng_for(wl.wid, 4)
    if not wl.ragged:
        return sorted(rng.choice(B, size=min(count, B), replace=False).tolist())
    picks = [int(np.argmin(lengths)), int(np.argmax(lengths))]
    for r in (63, 0):
        cand = [b for b in range(B) if (int(lengths[b]) + wl.n_q) % 64 == r and b not in picks]
        if cand:
            picks.append(cand[0])
    rest = [b for b in rng.permutation(B).tolist() if b not in picks]
    picks += rest[:max(0, count - len(picks))]
    return sorted(set(picks))


def device_fill_normal_(t, seed: int):
    """Fill a CUDA tensor with seeded N(0,1) values (used for cache history no
    check reads)."""
    import torch
    g = torch.Generator(device=t.device)
    g.manual_seed(int(seed))
    t.normal_(0.0, 1.0, generator=g)
    return t
