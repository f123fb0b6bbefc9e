"""The workspace-free append (mla_append_latent_noalloc) against the regular
mla_append_latent, through the C ABI.

It is meant for callers that cannot allocate device memory where they append
(an engine that owns all of HBM through its own pool, code under stream
capture); its scratch lives in a fixed array inside libmla.  This file is named
to be collected last so that a run stopping at the first failure has already
run every other test."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from head_latent_attention_append_b200 import synth  # noqa: E402

TOL_BF16 = 2e-2   # same bound as the bf16 parity tests (max |err| / max |ref|)


def _case():
    from head_latent_attention_append_b200 import mla, workload
    base = synth.WORKLOADS["page_bf16_decode"]
    wl = synth.Workload("noalloc", 11, base.n_h, base.d_h, base.d_v, base.d_c, base.d_r, base.d_model, base.d_cq,
                        "bf16", "decode", 3, 1, 0)
    dev = torch.device("cuda")
    dims = workload.dims_of(wl)
    hw = synth.make_weights(wl, 7)
    weights = mla.Weights(dims, workload.upload_weights(wl, hw, dev))
    kv = np.array([150, 37, 213], np.int32)
    lay = synth.page_layout(kv, 64, shuffle=True, wl_id=11, seed=7)
    H = {b: synth.make_hidden(wl, b, int(kv[b]), 7) for b in range(3)}
    h = torch.from_numpy(np.concatenate([H[b] for b in range(3)])).to(dev, torch.bfloat16)
    si = torch.from_numpy(np.concatenate([np.full(int(L), b, np.int32) for b, L in enumerate(kv)])).to(dev)
    ps = torch.from_numpy(np.concatenate([np.arange(int(L), dtype=np.int32) for L in kv])).to(dev)
    pt = torch.from_numpy(lay.page_table).to(dev)
    return mla, wl, weights, lay, h, si, ps, pt


def test_noalloc_append_matches_workspace_append_on_two_calls_in_a_row():
    mla, wl, weights, lay, h, si, ps, pt = _case()
    dev = h.device
    T = h.shape[0]                    # 400 tokens, appended in two calls of 200
    half = T // 2
    ref = torch.zeros((lay.num_pages, 64, wl.d_cr), dtype=torch.bfloat16, device=dev)
    got = torch.zeros_like(ref)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    for lo, hi in ((0, half), (half, T)):
        ws = torch.empty(mla.append_workspace_bytes(weights.dims, hi - lo), dtype=torch.uint8, device=dev)
        mla.append_latent(weights, h[lo:hi], si[lo:hi], ps[lo:hi], pt, lay.num_pages, ref, ws)
        mla.append_latent_noalloc(weights, h[lo:hi], si[lo:hi], ps[lo:hi], pt, lay.num_pages, got, err)
        torch.cuda.synchronize()
        assert mla.get_error(ws) == mla.MLA_OK
        assert int(err.item()) == 0
        a = ref.float().cpu().numpy()
        b = got.float().cpu().numpy()
        assert np.abs(b - a).max() <= TOL_BF16 * np.abs(a).max()
    assert torch.count_nonzero(got) > 0


def test_noalloc_append_rejects_more_than_its_fixed_capacity():
    mla, wl, weights, lay, h, si, ps, pt = _case()
    cache = torch.zeros((lay.num_pages, 64, wl.d_cr), dtype=torch.bfloat16, device=h.device)
    T = mla.APPEND_NOALLOC_MAX_T + 1
    with pytest.raises(mla.MlaError) as ei:
        mla.append_latent_noalloc(weights, h[:T], si[:T], ps[:T], pt, lay.num_pages, cache)
    assert ei.value.code == -3  # MLA_ERR_WORKSPACE
