"""GPU parity of context-parallel decode through the C ABI.

The ranks are emulated one after another on one GPU (no kernel waits for
another): each has its own page pool, filled through mla_append_latent at the
tokens' global positions, and runs mla_decode_cp_partial over its window; the
stacked partials go through mla_decode_cp_combine.  Checked against the fp64
oracle: every rank's (obar_r, lse_r) against the oracle's window partial, and
the merged output against the oracle's decode (2e-2, bf16 inputs with fp32
accumulation), plus the single-GPU decode of the same inputs.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle as O  # noqa: E402
from head_latent_attention_append_b200 import cp, synth  # noqa: E402

TOL = 2e-2
LSE_TOL = 0.1  # log2 units; a base-e/base-2 mix-up or a missing max is off by whole units


def _mods():
    from head_latent_attention_append_b200 import mla, workload
    return mla, workload


def case(lengths, n_q, seed=5):
    mla, workload = _mods()
    base = synth.WORKLOADS["page_bf16_decode"]
    wl = synth.Workload("cp", 9, base.n_h, base.d_h, base.d_v, base.d_c, base.d_r, base.d_model, base.d_cq,
                        "bf16", "decode", len(lengths), n_q, 0)
    dev = torch.device("cuda")
    dims = workload.dims_of(wl)
    hw = synth.make_weights(wl, seed)
    weights = mla.Weights(dims, workload.upload_weights(wl, hw, dev))
    kv = np.asarray(lengths, np.int32) + n_q
    H = {b: synth.make_hidden(wl, b, int(kv[b]), seed) for b in range(len(lengths))}
    return dict(wl=wl, dims=dims, hw=hw, weights=weights, kv=kv, H=H, dev=dev)


def run_cp(c, n_ranks):
    mla, _ = _mods()
    wl, dev, kv, H = c["wl"], c["dev"], c["kv"], c["H"]
    B, n_q = wl.B, wl.n_q
    wins = cp.shard_windows(kv, n_ranks, 64)
    hq = torch.from_numpy(np.stack([H[b][-n_q:] for b in range(B)])).to(dev, torch.bfloat16)
    kv_dev = torch.from_numpy(kv).to(dev)
    obar_parts = torch.empty((n_ranks, B, n_q, wl.n_h, wl.d_c), dtype=torch.bfloat16, device=dev)
    lse_parts = torch.empty((n_ranks, B, n_q, wl.n_h), dtype=torch.float32, device=dev)
    ws = torch.empty(mla.decode_cp_workspace_bytes(c["dims"], B, n_q), dtype=torch.uint8, device=dev)
    for r, win in enumerate(wins):
        pool = int(((win.count.astype(np.int64) + 63) // 64).sum()) + 1
        rp = cp.rank_pages(win, kv, 64, order=np.random.default_rng(100 + r).permutation(pool), spare_pages=1)
        # Unwritten slots hold NaN: only the window's keys may reach a result.
        cache = torch.full((rp.num_pages, 64, wl.d_cr), float("nan"), dtype=torch.bfloat16, device=dev)
        toks = [(b, p) for b in range(B) for p in range(int(win.start[b]), int(win.start[b]) + int(win.count[b]))]
        if toks:
            h = torch.from_numpy(np.stack([H[b][p] for b, p in toks])).to(dev, torch.bfloat16)
            si = torch.tensor([b for b, _ in toks], dtype=torch.int32, device=dev)
            ps = torch.tensor([p for _, p in toks], dtype=torch.int32, device=dev)
            wsa = torch.empty(mla.append_workspace_bytes(c["dims"], len(toks)), dtype=torch.uint8, device=dev)
            mla.append_latent(c["weights"], h, si, ps, torch.from_numpy(rp.by_position).to(dev), rp.num_pages,
                              cache, wsa)
            assert mla.get_error(wsa) == mla.MLA_OK
        mla.decode_cp_partial(c["weights"], hq, kv_dev, torch.from_numpy(win.start).to(dev),
                              torch.from_numpy(win.count).to(dev), torch.from_numpy(rp.local).to(dev),
                              rp.num_pages, cache, obar_parts[r], lse_parts[r], int(kv.max()), ws)
        torch.cuda.synchronize()
        assert mla.get_error(ws) == mla.MLA_OK, r
    out = torch.empty((B, n_q, wl.n_h, wl.d_v), dtype=torch.float32, device=dev)
    mla.decode_cp_combine(c["weights"], obar_parts, lse_parts, out, ws)
    torch.cuda.synchronize()
    assert mla.get_error(ws) == mla.MLA_OK
    return out.cpu().numpy(), obar_parts.float().cpu().numpy(), lse_parts.cpu().numpy(), wins


def rel_err(got, ref):
    return float(np.abs(got - ref).max() / np.abs(ref).max())


# (ranks, new tokens per sequence, cached lengths): windows that hold nothing
# of a short sequence, windows cut inside the new tokens (126 cached + 4 new
# over 3 ranks: the last window holds positions 128, 129 only, which the first
# two new tokens may not see), and ragged lengths around page boundaries.
CASES = [(2, 1, [0, 1, 63, 64, 200, 700, 1000]), (3, 2, [0, 1, 63, 64, 200, 700, 1000]),
         (4, 1, [0, 1, 130, 64]), (3, 4, [126, 3, 300])]


@pytest.mark.parametrize("n_ranks,n_q,lengths", CASES)
def test_context_parallel_decode_matches_oracle(n_ranks, n_q, lengths):
    mla, _ = _mods()
    c = case(lengths, n_q)
    out, obar, lse, wins = run_cp(c, n_ranks)
    dims = O.Dims(c["wl"].n_h, c["wl"].d_h, c["wl"].d_v, c["wl"].d_c, c["wl"].d_r, c["wl"].d_model,
                  c["wl"].d_cq, c["wl"].rope_base)
    w = O.Weights(**c["hw"].as_dict())
    for b in range(len(lengths)):
        ref = O.mla_decode(dims, w, c["H"][b], n_q)
        assert rel_err(out[b], ref) <= TOL, (b, lengths[b])
        for r, win in enumerate(wins):
            o_ref, l_ref = O.window_partial(dims, w, c["H"][b], n_q, int(win.start[b]), int(win.count[b]))
            empty = np.isneginf(l_ref)
            np.testing.assert_array_equal(np.isneginf(lse[r, b]), empty)
            if (~empty).any():
                assert np.abs(lse[r, b][~empty] - l_ref[~empty]).max() <= LSE_TOL, (b, r)
                seen = ~empty.all(axis=1)  # query tokens with a key in this window
                assert rel_err(obar[r, b][seen], o_ref[seen]) <= TOL, (b, r)

    # The same inputs through the single-GPU decode.
    from test_gpu_parity import run_small, small_case
    s = small_case(lengths, n_q)
    single, _, e1, e2 = run_small(s)
    assert e1 == 0 and e2 == 0
    assert rel_err(out, single) <= TOL


def test_fp32_context_parallel_is_unsupported():
    mla, workload = _mods()
    wl = synth.WORKLOADS["tiny_fp32_decode"]
    dims = workload.dims_of(wl)
    weights = mla.Weights(dims, workload.upload_weights(wl, synth.make_weights(wl), torch.device("cuda")))
    assert mla.decode_cp_workspace_bytes(dims, 1, 1) == 0
    dev = torch.device("cuda")
    z = torch.zeros(1, dtype=torch.int32, device=dev)
    buf = torch.zeros(1 << 16, dtype=torch.float32, device=dev)
    with pytest.raises(mla.MlaError) as e:
        mla.decode_cp_partial(weights, buf.view(1, 1, -1), z, z, z, z.view(1, 1), 1, buf, buf, buf, 1, buf)
    assert e.value.code == -2
