"""Device-resident setup of the named synthetic workloads (see synth.py).

Builds the absorbed weights, a shuffled page pool, the latent cache history
and the new tokens of one decode step (or the tokens of one prefill) on a CUDA
device, and runs one step through the C ABI.  Used by the tests, the smoke
run and the benchmark; it computes nothing itself.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np
import torch

from . import mla, synth

TORCH_DTYPE = {"bf16": torch.bfloat16, "f32": torch.float32}


def dims_of(wl: synth.Workload, softmax_scale: float = 0.0) -> mla.Dims:
    return mla.make_dims(wl.n_h, wl.d_h, wl.d_v, wl.d_c, wl.d_r, wl.d_model, wl.d_cq, wl.rope_base,
                         softmax_scale, synth.PAGE_SIZE, mla.BF16 if wl.dtype == "bf16" else mla.F32,
                         wl.rope_per_head)


def upload_weights(wl: synth.Workload, hw: synth.HostWeights, device) -> Dict[str, torch.Tensor]:
    dt = TORCH_DTYPE[wl.dtype]
    return {k: (None if v is None else torch.from_numpy(v).to(device=device, dtype=dt))
            for k, v in hw.as_dict().items()}


@dataclass
class Setup:
    wl: synth.Workload
    dims: mla.Dims
    host_weights: synth.HostWeights
    weights: mla.Weights
    kv_len_host: np.ndarray
    layout: synth.PageLayout
    kv_len: torch.Tensor
    page_table: torch.Tensor
    cache: torch.Tensor
    h_new: torch.Tensor               # decode: [B, n_q, D]; prefill: [B, S, D]
    seq_idx: Optional[torch.Tensor]   # decode: sequence of each new token
    pos: Optional[torch.Tensor]       # decode: position of each new token
    out: torch.Tensor
    ws_append: Optional[torch.Tensor]
    ws: torch.Tensor
    checked: List[int]
    host_hidden: Dict[int, np.ndarray] = field(default_factory=dict)

    @property
    def max_kv_len(self) -> int:
        return int(self.kv_len_host.max())

    def cache_bytes_read(self) -> int:
        """Latent-cache bytes the attention kernel streams: every key of every
        query token's row block once (each query token is its own row block,
        so a sequence with n_q new tokens is read n_q times)."""
        wl = self.wl
        esz = 2 if wl.dtype == "bf16" else 4
        if wl.mode == "prefill":
            S = wl.n_q
            keys = wl.B * S * (S + 1) // 2
        else:
            keys = int(sum(int(L) - wl.n_q + 1 + q for L in self.kv_len_host for q in range(wl.n_q)))
        return keys * wl.d_cr * esz

    def cache_bytes_unique(self) -> int:
        """Latent-cache bytes of every sequence's history, counted once: the
        least a step's attention must read, however many query tokens a
        sequence brings."""
        wl = self.wl
        esz = 2 if wl.dtype == "bf16" else 4
        keys = wl.B * wl.n_q if wl.mode == "prefill" else int(self.kv_len_host.sum())
        return keys * wl.d_cr * esz

    def attention_pairs(self) -> int:
        """Causal (query, key) pairs of one step."""
        wl = self.wl
        if wl.mode == "prefill":
            return wl.B * wl.n_q * (wl.n_q + 1) // 2
        return int(sum(int(L) - wl.n_q + 1 + q for L in self.kv_len_host for q in range(wl.n_q)))

    def attention_flops(self) -> int:
        """The step's algorithmic attention flops in its own form (absorbed or
        materialised)."""
        return Setup.attention_pairs(self) * self.wl.flops_per_pair()


def setup(name: str, device="cuda", checked_count: int = 4, check_all: Optional[bool] = None,
          seed: int = synth.BASE_SEED, build_history: bool = True, softmax_scale: float = 0.0) -> Setup:
    """``softmax_scale`` 0 selects the library default 1/sqrt(d_h + d_r)."""
    wl = synth.WORKLOADS[name]
    dev = torch.device(device)
    dt = TORCH_DTYPE[wl.dtype]
    dims = dims_of(wl, softmax_scale)
    hw = synth.make_weights(wl, seed)
    W = upload_weights(wl, hw, dev)
    weights = mla.Weights(dims, W)
    del W

    kv = synth.kv_lengths(wl, seed)
    layout = synth.page_layout(kv, synth.PAGE_SIZE, shuffle=(wl.dtype == "bf16"), wl_id=wl.wid, seed=seed)
    page_table = torch.from_numpy(layout.page_table).to(dev)
    kv_len = torch.from_numpy(kv).to(dev)
    cache = torch.empty((layout.num_pages, synth.PAGE_SIZE, wl.d_cr), dtype=dt, device=dev)
    if check_all is None:
        check_all = wl.B * int(kv.max()) * wl.d_model <= 80_000_000
    checked = list(range(wl.B)) if check_all else synth.checked_sequences(wl, kv - wl.n_q, checked_count)

    host_hidden: Dict[int, np.ndarray] = {}
    if wl.mode == "prefill":
        S = wl.n_q
        h_new = torch.empty((wl.B, S, wl.d_model), dtype=dt, device=dev)
        for b in range(wl.B):
            if b in checked:
                host_hidden[b] = synth.make_hidden(wl, b, S, seed)
                h_new[b] = torch.from_numpy(host_hidden[b]).to(dev, dt)
            else:
                synth.device_fill_normal_(h_new[b], seed * 1000 + b)
        cache.zero_()
        out = torch.empty((wl.B, S, wl.n_h, wl.d_v), dtype=torch.float32, device=dev)
        nws = (mla.prefill_materialised_workspace_bytes(dims, wl.B, S) if wl.materialised
               else mla.prefill_workspace_bytes(dims, wl.B, S))
        ws = torch.empty(nws, dtype=torch.uint8, device=dev)
        return Setup(wl, dims, hw, weights, kv, layout, kv_len, page_table, cache, h_new, None, None, out, None,
                     ws, checked, host_hidden)

    # Decode: history of unchecked sequences is N(0,1) cache rows; checked
    # sequences get their whole history through the append path.
    synth.device_fill_normal_(cache, seed + 17)
    h_new = torch.empty((wl.B, wl.n_q, wl.d_model), dtype=dt, device=dev)
    ws_app = None
    for b in range(wl.B):
        if b in checked:
            H = synth.make_hidden(wl, b, int(kv[b]), seed)
            host_hidden[b] = H
            h_new[b] = torch.from_numpy(H[-wl.n_q:]).to(dev, dt)
        else:
            synth.device_fill_normal_(h_new[b], seed * 1000 + b)
    if build_history:
        for b in checked:
            L = int(kv[b]) - wl.n_q
            if L <= 0:
                continue
            for p0 in range(0, L, 8192):
                p1 = min(L, p0 + 8192)
                hb = torch.from_numpy(host_hidden[b][p0:p1]).to(dev, dt)
                si = torch.full((p1 - p0,), b, dtype=torch.int32, device=dev)
                ps = torch.arange(p0, p1, dtype=torch.int32, device=dev)
                need = mla.append_workspace_bytes(dims, p1 - p0)
                if ws_app is None or ws_app.numel() < need:
                    ws_app = torch.empty(need, dtype=torch.uint8, device=dev)
                mla.append_latent(weights, hb, si, ps, page_table, layout.num_pages, cache, ws_app)
    seq_idx = torch.arange(wl.B, dtype=torch.int32, device=dev).repeat_interleave(wl.n_q)
    pos = torch.from_numpy(np.concatenate([np.arange(int(L) - wl.n_q, int(L)) for L in kv]).astype(np.int32)).to(dev)
    need = mla.append_workspace_bytes(dims, wl.B * wl.n_q)
    if ws_app is None or ws_app.numel() < need:
        ws_app = torch.empty(need, dtype=torch.uint8, device=dev)
    out = torch.empty((wl.B, wl.n_q, wl.n_h, wl.d_v), dtype=torch.float32, device=dev)
    ws = torch.empty(mla.decode_step_workspace_bytes(dims, wl.B, wl.n_q, int(kv.max())), dtype=torch.uint8,
                     device=dev)
    return Setup(wl, dims, hw, weights, kv, layout, kv_len, page_table, cache, h_new, seq_idx, pos, out, ws_app,
                 ws, checked, host_hidden)


def step(s: Setup, stream=None, fused: bool = True) -> int:
    """One pass of the hot path: append the new tokens, then attend (decode:
    one mla_decode_step call, or with fused=False mla_append_latent then
    mla_decode), or append every token and attend causally (prefill).  Returns
    the number of kernels libmla launched."""
    if s.wl.mode == "prefill":
        fn = mla.prefill_materialised if s.wl.materialised else mla.prefill
        fn(s.weights, s.h_new, s.page_table, s.layout.num_pages, s.cache, s.out, s.ws, stream)
        return mla.last_launch_count()
    wl = s.wl
    if fused:
        mla.decode_step(s.weights, s.h_new, s.kv_len, s.page_table, s.layout.num_pages, s.cache, s.out,
                        s.max_kv_len, s.ws, stream)
        return mla.last_launch_count()
    mla.append_latent(s.weights, s.h_new.view(wl.B * wl.n_q, wl.d_model), s.seq_idx, s.pos, s.page_table,
                      s.layout.num_pages, s.cache, s.ws_append, stream)
    n = mla.last_launch_count()
    mla.decode(s.weights, s.h_new, s.kv_len, s.page_table, s.layout.num_pages, s.cache, s.out, s.max_kv_len,
               s.ws, stream)
    return n + mla.last_launch_count()
