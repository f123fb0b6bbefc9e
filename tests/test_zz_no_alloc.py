"""The workspace-free append (mla_append_latent_noalloc), through the C ABI,
against the regular mla_append_latent and against the oracle's cache rows.

It is meant for callers that cannot allocate device memory where they append
(an engine that owns all of HBM through its own pool, code under stream
capture); its scratch lives in a fixed array inside libmla.  This file is named
to be collected last so that a run stopping at the first failure has already
run every other test."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle as O  # noqa: E402
from head_latent_attention_append_b200 import synth  # noqa: E402

TOL = {"bf16": 2e-2, "f32": 1e-4}   # the parity bounds (max |err| / max |ref|)


def _case(dtype="bf16"):
    from head_latent_attention_append_b200 import mla, workload
    base = synth.WORKLOADS["page_bf16_decode" if dtype == "bf16" else "tiny_fp32_decode"]
    wl = synth.Workload("noalloc", 11, base.n_h, base.d_h, base.d_v, base.d_c, base.d_r, base.d_model, base.d_cq,
                        dtype, "decode", 3, 1, 0)
    dev = torch.device("cuda")
    tdt = workload.TORCH_DTYPE[dtype]
    dims = workload.dims_of(wl)
    hw = synth.make_weights(wl, 7)
    weights = mla.Weights(dims, workload.upload_weights(wl, hw, dev))
    kv = np.array([150, 37, 213], np.int32)
    # Two spare pages that no sequence uses: they must stay untouched.
    lay = synth.page_layout(kv, 64, shuffle=True, wl_id=11, seed=7, spare_pages=2)
    H = {b: synth.make_hidden(wl, b, int(kv[b]), 7) for b in range(3)}
    h = torch.from_numpy(np.concatenate([H[b] for b in range(3)])).to(dev, tdt)
    si = torch.from_numpy(np.concatenate([np.full(int(L), b, np.int32) for b, L in enumerate(kv)])).to(dev)
    ps = torch.from_numpy(np.concatenate([np.arange(int(L), dtype=np.int32) for L in kv])).to(dev)
    pt = torch.from_numpy(lay.page_table).to(dev)
    return dict(mla=mla, wl=wl, hw=hw, weights=weights, kv=kv, lay=lay, H=H, h=h, si=si, ps=ps, pt=pt, tdt=tdt)


def _oracle_rows(c):
    """The oracle's cache rows [c_t | RoPE_t(W_KR h_t)] of every token, by sequence."""
    wl = c["wl"]
    w = O.Weights(**c["hw"].as_dict())
    f = O.rope_frequencies(wl.d_r, wl.rope_base)
    out = {}
    for b, L in enumerate(c["kv"]):
        cc, kr = O.cache_entries(w, c["H"][b], np.arange(int(L)), f)
        out[b] = np.concatenate([cc, kr], axis=1)
    return out


def _rows(cache_np, lay, b, L):
    return np.stack([cache_np[lay.page_table[b, p // 64], p % 64] for p in range(L)])


def _rel(got, ref):
    return float(np.abs(got - ref).max() / np.abs(ref).max())


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_append_matches_workspace_append_and_oracle_on_two_calls_in_a_row(dtype):
    c = _case(dtype)
    mla, wl, lay, h, si, ps, pt = c["mla"], c["wl"], c["lay"], c["h"], c["si"], c["ps"], c["pt"]
    dev = h.device
    T = h.shape[0]                    # 400 tokens, appended in two calls of 200
    half = T // 2
    ref = torch.zeros((lay.num_pages, 64, wl.d_cr), dtype=c["tdt"], device=dev)
    got = torch.zeros_like(ref)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    for lo, hi in ((0, half), (half, T)):
        ws = torch.empty(mla.append_workspace_bytes(c["weights"].dims, hi - lo), dtype=torch.uint8, device=dev)
        mla.append_latent(c["weights"], h[lo:hi], si[lo:hi], ps[lo:hi], pt, lay.num_pages, ref, ws)
        mla.append_latent_noalloc(c["weights"], h[lo:hi], si[lo:hi], ps[lo:hi], pt, lay.num_pages, got, err)
        torch.cuda.synchronize()
        assert mla.get_error(ws) == mla.MLA_OK
        assert int(err.item()) == 0
        a = ref.float().cpu().numpy()
        b = got.float().cpu().numpy()
        assert np.abs(b - a).max() <= TOL[dtype] * np.abs(a).max()
    # Every token's row against the oracle (fp64), through the page table.
    got_np = got.float().cpu().numpy()
    orows = _oracle_rows(c)
    for b, L in enumerate(c["kv"]):
        assert _rel(_rows(got_np, lay, b, int(L)), orows[b]) <= TOL[dtype], (dtype, b)
    # Pages no sequence owns are never written.
    used = set(int(p) for p in lay.page_table.ravel() if p >= 0)
    for p in range(lay.num_pages):
        if p not in used:
            assert not got_np[p].any(), p


def test_noalloc_append_reports_a_bad_page_id_through_device_error():
    c = _case("bf16")
    mla, wl, lay, h, si, ps = c["mla"], c["wl"], c["lay"], c["h"], c["si"], c["ps"]
    bad = lay.page_table.copy()
    bad[0, 1] = lay.num_pages + 5            # positions 64..127 of sequence 0 point outside the pool
    pt = torch.from_numpy(bad).to(h.device)
    cache = torch.zeros((lay.num_pages, 64, wl.d_cr), dtype=torch.bfloat16, device=h.device)
    err = torch.zeros(1, dtype=torch.int32, device=h.device)
    mla.append_latent_noalloc(c["weights"], h[:150], si[:150], ps[:150], pt, lay.num_pages, cache, err)
    torch.cuda.synchronize()
    assert int(err.item()) & 1                # the bounds condition, OR-ed in as 1
    # The tokens with valid pages were still written.
    got_np = cache.float().cpu().numpy()
    orow = _oracle_rows(c)[0]
    rows = np.stack([got_np[bad[0, p // 64], p % 64] for p in range(64)])
    assert _rel(rows, orow[:64]) <= TOL["bf16"]


def test_noalloc_append_rejects_more_than_its_fixed_capacity():
    c = _case("bf16")
    mla, wl, lay, h, si, ps, pt = c["mla"], c["wl"], c["lay"], c["h"], c["si"], c["ps"], c["pt"]
    cache = torch.zeros((lay.num_pages, 64, wl.d_cr), dtype=torch.bfloat16, device=h.device)
    T = mla.APPEND_NOALLOC_MAX_T + 1
    with pytest.raises(mla.MlaError) as ei:
        mla.append_latent_noalloc(c["weights"], h[:T], si[:T], ps[:T], pt, lay.num_pages, cache)
    assert ei.value.code == -3  # MLA_ERR_WORKSPACE
