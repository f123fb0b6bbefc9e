"""GPU parity of the materialised causal prefill (mla_prefill_materialised):
per-head keys K_C = W_UK,h c and values V = W_UV,h c expanded from the latent,
then causal multi-head attention on [K_C | k_R] and V ("Multi-Head Latent
Attention" (talalahmed), "Compress first, expand later").  Compared element
by element with the fp64 oracle (max |out - ref| / max |ref| <= 2e-2 for bf16),
and with the absorbed prefill: equal to rounding, not bit for bit
("ropeabsorb", "Absorption is exact")."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle as O  # noqa: E402
from head_latent_attention_append_b200 import synth  # noqa: E402

TOL = 2e-2


def rel_err(got, ref):
    return float(np.abs(got - ref).max() / np.abs(ref).max())


def _small(B, S, d_h=128, d_v=128, seed=3, cache_fill=float("nan")):
    """A small prefill (16 heads, d_c = 256, d_r = 64, hidden 2048, no query
    latent) with a shuffled page table; unused cache slots hold `cache_fill`."""
    from head_latent_attention_append_b200 import mla, workload
    wl = synth.Workload("matp", 21, 16, d_h, d_v, 256, 64, 2048, 0, "bf16", "prefill", B, S, 0)
    dev = torch.device("cuda")
    dims = workload.dims_of(wl)
    hw = synth.make_weights(wl, seed)
    weights = mla.Weights(dims, workload.upload_weights(wl, hw, dev))
    lay = synth.page_layout(np.full(B, S, np.int32), 64, shuffle=True, wl_id=21, seed=seed, spare_pages=3)
    H = {b: synth.make_hidden(wl, b, S, seed) for b in range(B)}
    h = torch.from_numpy(np.stack([H[b] for b in range(B)])).to(dev, torch.bfloat16)
    pt = torch.from_numpy(lay.page_table).to(dev)

    def run(fn, wsize):
        cache = torch.full((lay.num_pages, 64, wl.d_cr), cache_fill, dtype=torch.bfloat16, device=dev)
        out = torch.empty((B, S, wl.n_h, wl.d_v), dtype=torch.float32, device=dev)
        ws = torch.empty(wsize(dims, B, S), dtype=torch.uint8, device=dev)
        fn(weights, h, pt, lay.num_pages, cache, out, ws)
        torch.cuda.synchronize()
        assert mla.get_error(ws) == mla.MLA_OK
        return out.cpu().numpy(), cache

    return wl, hw, H, run, mla


@pytest.mark.parametrize("S", [1, 63, 100, 128, 129, 300])
def test_materialised_prefill_matches_oracle_small(S):
    wl, hw, H, run, mla = _small(3, S)
    out, _ = run(mla.prefill_materialised, mla.prefill_materialised_workspace_bytes)
    assert np.isfinite(out).all()
    dims = O.Dims(wl.n_h, wl.d_h, wl.d_v, wl.d_c, wl.d_r, wl.d_model, wl.d_cq, wl.rope_base)
    w = O.Weights(**hw.as_dict())
    for b in range(3):
        ref = O.mla_sequence(dims, w, H[b], list(range(S)))
        e = rel_err(out[b], ref)
        assert e <= TOL, (S, b, e)


def test_materialised_prefill_narrow_heads_match_oracle():
    """d_h = d_v = 64: two score chunks (content + RoPE) and one value chunk."""
    wl, hw, H, run, mla = _small(2, 200, d_h=64, d_v=64)
    out, _ = run(mla.prefill_materialised, mla.prefill_materialised_workspace_bytes)
    dims = O.Dims(wl.n_h, wl.d_h, wl.d_v, wl.d_c, wl.d_r, wl.d_model, wl.d_cq, wl.rope_base)
    w = O.Weights(**hw.as_dict())
    for b in range(2):
        assert rel_err(out[b], O.mla_sequence(dims, w, H[b], list(range(200)))) <= TOL


def test_materialised_and_absorbed_prefill_agree_to_rounding_not_bitwise():
    wl, hw, H, run, mla = _small(2, 257)
    out_m, cache_m = run(mla.prefill_materialised, mla.prefill_materialised_workspace_bytes)
    out_a, cache_a = run(mla.prefill, mla.prefill_workspace_bytes)
    # Both append the same cache rows through the same path.
    assert torch.equal(torch.nan_to_num(cache_m, nan=7.0), torch.nan_to_num(cache_a, nan=7.0))
    assert not np.array_equal(out_m, out_a)
    assert rel_err(out_m, out_a) <= TOL


def test_materialised_prefill_is_deterministic():
    wl, hw, H, run, mla = _small(2, 190)
    a, _ = run(mla.prefill_materialised, mla.prefill_materialised_workspace_bytes)
    b, _ = run(mla.prefill_materialised, mla.prefill_materialised_workspace_bytes)
    np.testing.assert_array_equal(a, b)


def test_materialised_prefill_full_size_matches_oracle_on_sampled_positions():
    """Config 4 (B=4, S=4096, 128 heads, d_c=512, d_r=64) in the materialised
    form, 512 seeded query positions of one sequence including 0, 63, 64 and
    4095; and the same positions of the absorbed prefill within 2e-2."""
    from head_latent_attention_append_b200 import mla, workload
    s = workload.setup("dsv2_bf16_prefill_mat", checked_count=1, check_all=False)
    workload.step(s)
    torch.cuda.synchronize()
    assert mla.get_error(s.ws) == mla.MLA_OK
    wl = s.wl
    b = s.checked[0]
    rng = np.random.default_rng(0)
    fixed = [0, 63, 64, 4095]
    rows = sorted(fixed + [r for r in rng.permutation(wl.n_q).tolist() if r not in fixed][:512 - len(fixed)])
    dims = O.Dims(wl.n_h, wl.d_h, wl.d_v, wl.d_c, wl.d_r, wl.d_model, wl.d_cq, wl.rope_base)
    ref = O.mla_sequence(dims, O.Weights(**s.host_weights.as_dict()), s.host_hidden[b], rows)
    got = s.out[b, rows].float().cpu().numpy()
    e = rel_err(got, ref)
    print(f"materialised prefill: max rel err {e:.3e} over {len(rows)} positions")
    assert e <= TOL
    assert torch.isfinite(s.out).all()


def test_unsupported_dims_are_refused():
    from head_latent_attention_append_b200 import mla, workload
    wl = synth.WORKLOADS["page_bf16_decode"]          # d_r = 32: not this kernel's RoPE width
    assert mla.prefill_materialised_workspace_bytes(workload.dims_of(wl), 2, 64) == 0
