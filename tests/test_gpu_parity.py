"""GPU parity: libmla through its C ABI against the fp64 oracle.

Tolerance (max |out - ref| / max |ref| over the checked outputs): 1e-4 for the
fp32 workload, 2e-2 for bf16 inputs with fp32 accumulation.  Indexing, paging
and causal masking are checked bit for bit.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle as O  # noqa: E402
from head_latent_attention_append_b200 import synth  # noqa: E402

TOL = {"f32": 1e-4, "bf16": 2e-2}


def _mods():
    from head_latent_attention_append_b200 import mla, workload
    return mla, workload


def oracle_dims(wl):
    return O.Dims(wl.n_h, wl.d_h, wl.d_v, wl.d_c, wl.d_r, wl.d_model, wl.d_cq, wl.rope_base,
                  rope_per_head=wl.rope_per_head)


def oracle_weights(s):
    return O.Weights(**s.host_weights.as_dict())


def rel_err(got, ref):
    return float(np.abs(got - ref).max() / np.abs(ref).max())


def check_decode(s, tol, scale=None):
    wl = s.wl
    dims, w = oracle_dims(wl), oracle_weights(s)
    out = s.out.float().cpu().numpy()
    worst = 0.0
    for b in s.checked:
        ref = O.mla_decode(dims, w, s.host_hidden[b], wl.n_q, scale=scale)
        e = rel_err(out[b], ref)
        worst = max(worst, e)
        assert e <= tol, f"sequence {b}: rel err {e:.3e} > {tol}"
    return worst


@pytest.mark.parametrize("name,count", [("tiny_fp32_decode", 1), ("page_bf16_decode", 8),
                                        ("dsv2_bf16_decode", 4), ("dsv2_ragged_decode", 8),
                                        ("dsv2_spec4_decode", 4)])
def test_decode_matches_oracle(name, count):
    mla, workload = _mods()
    s = workload.setup(name, checked_count=count)
    workload.step(s)
    torch.cuda.synchronize()
    assert mla.get_error(s.ws) == mla.MLA_OK
    assert mla.get_error(s.ws_append) == mla.MLA_OK
    assert torch.isfinite(s.out).all()
    err = check_decode(s, TOL[s.wl.dtype])
    print(f"{name}: max rel err {err:.3e} over sequences {s.checked}")


def test_prefill_matches_oracle_on_sampled_positions():
    mla, workload = _mods()
    s = workload.setup("dsv2_bf16_prefill", checked_count=1, check_all=False)
    workload.step(s)
    torch.cuda.synchronize()
    assert mla.get_error(s.ws) == mla.MLA_OK
    wl = s.wl
    b = s.checked[0]
    rng = np.random.default_rng(0)
    fixed = [0, 63, 64, 4095]
    rest = [r for r in rng.permutation(wl.n_q).tolist() if r not in fixed][:512 - len(fixed)]
    rows = sorted(fixed + rest)      # 512 seeded query positions
    assert len(rows) == 512
    ref = O.mla_sequence(oracle_dims(wl), oracle_weights(s), s.host_hidden[b], rows)
    got = s.out[b, rows].float().cpu().numpy()
    e = rel_err(got, ref)
    print(f"prefill: max rel err {e:.3e} over {len(rows)} positions")
    assert e <= TOL["bf16"]


# ------------------------------------------------------ small custom cases --
def small_case(lengths, n_q, shuffle=True, dtype="bf16", spare=2, seed=5, d_c=None, d_r=None, softmax_scale=0.0,
               rope_per_head=False):
    """A page_bf16_decode-shaped problem with the given cached lengths
    (optionally another latent width d_c or RoPE-key width d_r, or a softmax
    scale other than the default 1/sqrt(d_h + d_r))."""
    mla, workload = _mods()
    base = synth.WORKLOADS["page_bf16_decode" if dtype == "bf16" else "tiny_fp32_decode"]
    wl = synth.Workload("custom", 9, base.n_h, base.d_h, base.d_v, d_c or base.d_c, d_r or base.d_r, base.d_model,
                        base.d_cq, dtype, "decode", len(lengths), n_q, 0, rope_per_head=rope_per_head)
    dev = torch.device("cuda")
    dt = workload.TORCH_DTYPE[dtype]
    dims = workload.dims_of(wl, softmax_scale)
    hw = synth.make_weights(wl, seed)
    weights = mla.Weights(dims, workload.upload_weights(wl, hw, dev))
    kv = np.asarray(lengths, np.int32) + n_q
    lay = synth.page_layout(kv, 64, shuffle=shuffle, wl_id=9, seed=seed, spare_pages=spare)
    H = {b: synth.make_hidden(wl, b, int(kv[b]), seed) for b in range(len(lengths))}
    return dict(wl=wl, dims=dims, hw=hw, weights=weights, kv=kv, lay=lay, H=H, dev=dev, dt=dt)


def run_small(c, page_table=None, cache_fill=0.0, cache=None):
    mla, _ = _mods()
    wl, dev, dt = c["wl"], c["dev"], c["dt"]
    lay = c["lay"]
    pt = torch.from_numpy(lay.page_table if page_table is None else page_table).to(dev)
    if cache is None:
        cache = torch.full((lay.num_pages, 64, wl.d_cr), cache_fill, dtype=dt, device=dev)
    T = int(c["kv"].sum())
    h = torch.from_numpy(np.concatenate([c["H"][b] for b in range(wl.B)])).to(dev, dt)
    si = torch.from_numpy(np.concatenate([np.full(int(L), b, np.int32) for b, L in enumerate(c["kv"])])).to(dev)
    ps = torch.from_numpy(np.concatenate([np.arange(int(L), dtype=np.int32) for L in c["kv"]])).to(dev)
    wsa = torch.empty(mla.append_workspace_bytes(c["dims"], T), dtype=torch.uint8, device=dev)
    mla.append_latent(c["weights"], h, si, ps, pt, lay.num_pages, cache, wsa)
    hq = torch.from_numpy(np.stack([c["H"][b][-wl.n_q:] for b in range(wl.B)])).to(dev, dt)
    out = torch.empty((wl.B, wl.n_q, wl.n_h, wl.d_v), dtype=torch.float32, device=dev)
    ws = torch.empty(mla.decode_workspace_bytes(c["dims"], wl.B, wl.n_q, int(c["kv"].max())), dtype=torch.uint8,
                     device=dev)
    mla.decode(c["weights"], hq, torch.from_numpy(c["kv"]).to(dev), pt, lay.num_pages, cache, out,
               int(c["kv"].max()), ws)
    torch.cuda.synchronize()
    return out.cpu().numpy(), cache, mla.get_error(ws), mla.get_error(wsa)


EDGE_LENGTHS = [0, 1, 62, 63, 64, 127, 128, 129, 1000]


@pytest.mark.parametrize("n_q", [1, 2, 3, 4, 8])
def test_edge_lengths_match_oracle(n_q):
    c = small_case(EDGE_LENGTHS, n_q)
    out, _, e1, e2 = run_small(c)
    assert e1 == 0 and e2 == 0
    dims = oracle_dims(c["wl"])
    w = O.Weights(**c["hw"].as_dict())
    for b in range(len(EDGE_LENGTHS)):
        ref = O.mla_decode(dims, w, c["H"][b], n_q)
        assert rel_err(out[b], ref) <= TOL["bf16"], (b, EDGE_LENGTHS[b])


@pytest.mark.parametrize("d_c,d_r", [(256, 16), (256, 48), (128, 64), (384, 64), (384, 32)])
def test_rope_share_and_latent_width_variants_match_oracle(d_c, d_r):
    """The two CTAs split the RoPE-key columns 16 * (d_r / 32) : the rest, so
    d_r = 16 leaves rank 0 without any and d_r = 48 gives the ranks 16 and 32
    columns (boxes swizzled to 32 and 64 bytes in one launch); d_c = 128 gives
    each CTA a single latent chunk and d_c = 384 three."""
    c = small_case([0, 1, 63, 64, 200, 700], 2, d_c=d_c, d_r=d_r)
    out, _, e1, e2 = run_small(c)
    assert e1 == 0 and e2 == 0
    dims = oracle_dims(c["wl"])
    w = O.Weights(**c["hw"].as_dict())
    for b in range(6):
        ref = O.mla_decode(dims, w, c["H"][b], 2)
        assert rel_err(out[b], ref) <= TOL["bf16"], (d_c, d_r, b)


def test_fp32_edge_lengths_match_oracle():
    c = small_case([0, 5, 64, 130], 2, dtype="f32")
    out, _, e1, e2 = run_small(c)
    assert e1 == 0 and e2 == 0
    dims = oracle_dims(c["wl"])
    w = O.Weights(**c["hw"].as_dict())
    for b in range(4):
        ref = O.mla_decode(dims, w, c["H"][b], 2)
        assert rel_err(out[b], ref) <= TOL["f32"]


def test_page_order_does_not_change_results_bitwise():
    c = small_case([300, 64, 7], 2, shuffle=True)
    out_shuf, _, _, _ = run_small(c)
    ident = synth.page_layout(c["kv"], 64, shuffle=False, spare_pages=2)
    out_id, _, _, _ = run_small(c, page_table=ident.page_table)
    np.testing.assert_array_equal(out_shuf, out_id)


def test_poisoned_unused_slots_do_not_change_results_bitwise():
    c = small_case([300, 64, 7], 2)
    clean, _, _, _ = run_small(c, cache_fill=0.0)
    poisoned, _, _, _ = run_small(c, cache_fill=float("nan"))
    np.testing.assert_array_equal(clean, poisoned)


def test_two_runs_are_bitwise_identical():
    c = small_case([1000, 77], 2)
    a, _, _, _ = run_small(c)
    b, _, _, _ = run_small(c)
    np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("lengths,n_q", [([9000], 1), ([9000, 5], 2), ([100] * 19 + [20000], 2)])
def test_one_long_row_block_split_over_every_worker_matches_oracle(lengths, n_q):
    """One long sequence: its row blocks are cut into a piece per worker (one
    per CTA pair).  With few row blocks the combine kernel merges the pieces;
    with 40 (at least half as many as workers) the attention kernel's last
    piece of each row block merges them all, here 30-odd pieces."""
    c = small_case(lengths, n_q)
    out, _, e1, e2 = run_small(c)
    assert e1 == 0 and e2 == 0
    dims = oracle_dims(c["wl"])
    w = O.Weights(**c["hw"].as_dict())
    for b in range(len(lengths)):
        ref = O.mla_decode(dims, w, c["H"][b], n_q)
        assert rel_err(out[b], ref) <= TOL["bf16"], b
    again, _, _, _ = run_small(c)
    np.testing.assert_array_equal(out, again)


@pytest.mark.parametrize("n_q,j", [(2, 1), (4, 2)])
def test_later_new_token_does_not_reach_earlier_query(n_q, j):
    mla, _ = _mods()
    c = small_case([200, 64], n_q)
    out, cache, _, _ = run_small(c)
    # Overwrite the cache row of new token j of sequence 0 and decode again
    # without re-appending: the queries before j must not change, query j and
    # the later ones must, and sequence 1 must not.
    wl, lay = c["wl"], c["lay"]
    pos = int(c["kv"][0]) - n_q + j
    page = int(lay.page_table[0, pos // 64])
    cache2 = cache.clone()
    cache2[page, pos % 64] = 7.0
    hq = torch.from_numpy(np.stack([c["H"][b][-n_q:] for b in range(2)])).to(c["dev"], c["dt"])
    out2 = torch.empty_like(torch.from_numpy(out)).to(c["dev"])
    ws = torch.empty(mla.decode_workspace_bytes(c["dims"], 2, n_q, int(c["kv"].max())), dtype=torch.uint8,
                     device=c["dev"])
    pt = torch.from_numpy(lay.page_table).to(c["dev"])
    mla.decode(c["weights"], hq, torch.from_numpy(c["kv"]).to(c["dev"]), pt, lay.num_pages, cache2, out2,
               int(c["kv"].max()), ws)
    torch.cuda.synchronize()
    out2 = out2.cpu().numpy()
    for q in range(n_q):
        if q < j:
            np.testing.assert_array_equal(out[0, q], out2[0, q])
        else:
            assert not np.array_equal(out[0, q], out2[0, q]), q
    np.testing.assert_array_equal(out[1], out2[1])


def test_append_writes_oracle_cache_rows_and_paging_is_exact():
    c = small_case([150, 3], 1)
    _, cache, _, e = run_small(c)
    assert e == 0
    wl, lay = c["wl"], c["lay"]
    w = O.Weights(**c["hw"].as_dict())
    f = O.rope_frequencies(wl.d_r, wl.rope_base)
    cache_h = cache.float().cpu().numpy()
    for b in range(wl.B):
        L = int(c["kv"][b])
        rows = np.stack([cache_h[lay.page_table[b, p // 64], p % 64] for p in range(L)])
        cc, kr = O.cache_entries(w, c["H"][b], np.arange(L), f)
        ref = np.concatenate([cc, kr], axis=1)
        assert rel_err(rows, ref) <= 1e-2
    # Same tokens through an identity page table land in the same values.
    ident = synth.page_layout(c["kv"], 64, shuffle=False, spare_pages=2)
    _, cache_id, _, _ = run_small(c, page_table=ident.page_table)
    cid = cache_id.float().cpu().numpy()
    for b in range(wl.B):
        for p in range(int(c["kv"][b])):
            np.testing.assert_array_equal(cache_h[lay.page_table[b, p // 64], p % 64],
                                          cid[ident.page_table[b, p // 64], p % 64])


def test_out_of_range_page_id_is_reported_not_faulted():
    mla, _ = _mods()
    c = small_case([100], 1)
    bad = c["lay"].page_table.copy()
    bad[0, 1] = c["lay"].num_pages + 5
    _, _, e_dec, e_app = run_small(c, page_table=bad)
    assert e_app == -5  # MLA_ERR_DEVICE_BOUNDS
    assert e_dec == -5


# ------------------------------------------------ peaked softmax (large logits)
def max_abs_logit(wl, hw, H, n_q, scale):
    """Largest |a_t| (natural-log units) any new token of this sequence sees,
    from the oracle's own cache entries and queries."""
    dims, w = oracle_dims(wl), O.as_f64(O.Weights(**hw.as_dict()))
    T = H.shape[0]
    f = O.rope_frequencies(wl.d_r, wl.rope_base)
    pos = np.arange(T, dtype=np.float64)
    c, k_r = O.cache_entries(w, H, pos, f)
    rows = np.arange(T - n_q, T)
    q_c, q_r = O.queries(w, dims, H[rows], pos[rows], f)
    q_abs = np.einsum("qhd,hdc->qhc", q_c, w.W_UK.reshape(wl.n_h, wl.d_h, wl.d_c))
    a = (np.einsum("qhc,tc->qht", q_abs, c) + np.einsum("qhr,tr->qht", q_r, k_r)) * scale
    return float(np.abs(a).max())


@pytest.mark.parametrize("mult", [4.0, 8.0])
def test_peaked_softmax_matches_oracle(mult):
    """Logits of magnitude up to ~37 (x8 the default scale: the softmax near
    one-hot): the scores the two CTAs of a pair add must keep their precision
    where a few keys carry all the weight (the decoupled-RoPE page's score:
    content + position term).  Beyond this regime the bf16 cache rows
    themselves (before any kernel arithmetic) move the output by more than
    2e-2 against the fp64 oracle, e.g. 2.4e-2 at x16 with every later step
    exact, so x16 and up are not held to the bf16 bar."""
    base = synth.WORKLOADS["page_bf16_decode"]
    scale = mult / np.sqrt(base.d_h + base.d_r)
    c = small_case([0, 63, 64, 700, 2000, 4096], 2, softmax_scale=scale)
    out, _, e1, e2 = run_small(c)
    assert e1 == 0 and e2 == 0
    assert np.isfinite(out).all()
    dims = oracle_dims(c["wl"])
    w = O.Weights(**c["hw"].as_dict())
    worst, amax = 0.0, 0.0
    for b in range(c["wl"].B):
        ref = O.mla_decode(dims, w, c["H"][b], 2, scale=scale)
        worst = max(worst, rel_err(out[b], ref))
        amax = max(amax, max_abs_logit(c["wl"], c["hw"], c["H"][b], 2, scale))
    print(f"peaked x{mult}: max |logit| {amax:.1f}, max rel err {worst:.3e}")
    assert amax >= 10.0
    assert worst <= TOL["bf16"], (mult, worst)


@pytest.mark.parametrize("name,count", [("dsv2_bf16_decode", 2), ("dsv2_ragged_decode", 4)])
def test_peaked_softmax_full_size_matches_oracle(name, count):
    """Logits of magnitude ~20 (x4 the default scale) at the DeepSeek-V2-like
    dimensions (d_c = 512, d_r = 64, 128 heads, up to 32K keys), uniform and
    ragged.  (At x8 the longest ragged sequence reaches |a| ~ 44, where the
    bf16 rounding of the query latent, the absorbed query and the cache rows
    alone put the output ~2e-2 from the fp64 oracle, with every later step
    exact.)"""
    mla, workload = _mods()
    wl = synth.WORKLOADS[name]
    scale = 4.0 / np.sqrt(wl.d_h + wl.d_r)
    s = workload.setup(name, checked_count=count, softmax_scale=scale)
    workload.step(s)
    torch.cuda.synchronize()
    assert mla.get_error(s.ws) == mla.MLA_OK
    assert torch.isfinite(s.out).all()
    err = check_decode(s, TOL["bf16"], scale=scale)
    amax = max(max_abs_logit(wl, s.host_weights, s.host_hidden[b], wl.n_q, scale) for b in s.checked[:2])
    print(f"{name} x4 scale: max |logit| {amax:.1f}, max rel err {err:.3e} over sequences {s.checked}")
    assert amax >= 10.0


# ------------------------------------------------ per-head RoPE keys (NEXT) --
@pytest.mark.parametrize("dtype,n_q", [("bf16", 1), ("bf16", 3), ("f32", 2)])
def test_per_head_rope_keys_match_oracle(dtype, n_q):
    """One RoPE key per head ("Multi-Head Latent Attention", "A concrete size
    comparison"): cache rows of d_c + n_h * d_r, append rotating every head's
    key, attention scoring each head against its own key."""
    c = small_case([0, 1, 63, 64, 200, 700], n_q, dtype=dtype, rope_per_head=True)
    out, cache, e1, e2 = run_small(c)
    assert e1 == 0 and e2 == 0
    wl = c["wl"]
    assert cache.shape[-1] == wl.d_c + wl.n_h * wl.d_r
    dims = oracle_dims(wl)
    w = O.Weights(**c["hw"].as_dict())
    for b in range(wl.B):
        ref = O.mla_decode(dims, w, c["H"][b], n_q)
        assert rel_err(out[b], ref) <= TOL[dtype], (dtype, b)


def test_per_head_rope_key_cache_rows_match_oracle():
    c = small_case([150, 3], 1, rope_per_head=True)
    _, cache, _, e = run_small(c)
    assert e == 0
    wl, lay = c["wl"], c["lay"]
    w = O.Weights(**c["hw"].as_dict())
    f = O.rope_frequencies(wl.d_r, wl.rope_base)
    cache_h = cache.float().cpu().numpy()
    for b in range(wl.B):
        L = int(c["kv"][b])
        rows = np.stack([cache_h[lay.page_table[b, p // 64], p % 64] for p in range(L)])
        cc, kr = O.cache_entries(w, c["H"][b], np.arange(L), f)
        assert kr.shape == (L, wl.n_h, wl.d_r)
        ref = np.concatenate([cc, kr.reshape(L, -1)], axis=1)
        assert rel_err(rows, ref) <= 1e-2


def test_per_head_rope_keys_full_size_match_oracle():
    """The page-scale model (16 heads, d_c = 256, 32-dim keys: the page's
    768-number row) at B = 8, 4096 cached tokens, every sequence checked."""
    mla, workload = _mods()
    s = workload.setup("page_bf16_decode_rph", checked_count=8)
    assert s.cache.shape[-1] == 768
    workload.step(s)
    torch.cuda.synchronize()
    assert mla.get_error(s.ws) == mla.MLA_OK
    err = check_decode(s, TOL["bf16"])
    print(f"per-head RoPE keys: max rel err {err:.3e}")

@pytest.mark.parametrize("n_q", [1, 3])
def test_decode_step_equals_append_then_decode(n_q):
    """mla_decode_step (the append on the side stream beside the query
    projections) writes the same cache rows and outputs, bit for bit, as
    mla_append_latent of the new tokens followed by mla_decode."""
    mla, _ = _mods()
    c = small_case([0, 1, 63, 64, 300, 1000], n_q)
    wl, dev, dt, lay = c["wl"], c["dev"], c["dt"], c["lay"]
    pt = torch.from_numpy(lay.page_table).to(dev)
    kv = c["kv"]
    # History (every token but the new ones) appended into one cache; two copies of it.
    T = int((kv - n_q).sum())
    base = torch.full((lay.num_pages, 64, wl.d_cr), float("nan"), dtype=dt, device=dev)
    if T:
        h = torch.from_numpy(np.concatenate([c["H"][b][:int(L) - n_q] for b, L in enumerate(kv)])).to(dev, dt)
        si = torch.from_numpy(np.concatenate([np.full(int(L) - n_q, b, np.int32) for b, L in enumerate(kv)])).to(dev)
        ps = torch.from_numpy(np.concatenate([np.arange(int(L) - n_q, dtype=np.int32) for L in kv])).to(dev)
        wsa = torch.empty(mla.append_workspace_bytes(c["dims"], T), dtype=torch.uint8, device=dev)
        mla.append_latent(c["weights"], h, si, ps, pt, lay.num_pages, base, wsa)
    cache_a, cache_b = base.clone(), base.clone()
    hq = torch.from_numpy(np.stack([c["H"][b][-n_q:] for b in range(wl.B)])).to(dev, dt)
    kvd = torch.from_numpy(kv).to(dev)
    maxkv = int(kv.max())
    # Two calls.
    si = torch.arange(wl.B, dtype=torch.int32, device=dev).repeat_interleave(n_q)
    ps = torch.from_numpy(np.concatenate([np.arange(int(L) - n_q, int(L)) for L in kv]).astype(np.int32)).to(dev)
    wsa = torch.empty(mla.append_workspace_bytes(c["dims"], wl.B * n_q), dtype=torch.uint8, device=dev)
    mla.append_latent(c["weights"], hq.view(wl.B * n_q, -1), si, ps, pt, lay.num_pages, cache_a, wsa)
    out_a = torch.empty((wl.B, n_q, wl.n_h, wl.d_v), dtype=torch.float32, device=dev)
    ws = torch.empty(mla.decode_workspace_bytes(c["dims"], wl.B, n_q, maxkv), dtype=torch.uint8, device=dev)
    mla.decode(c["weights"], hq, kvd, pt, lay.num_pages, cache_a, out_a, maxkv, ws)
    # One call.
    out_b = torch.empty_like(out_a)
    wss = torch.empty(mla.decode_step_workspace_bytes(c["dims"], wl.B, n_q, maxkv), dtype=torch.uint8, device=dev)
    mla.decode_step(c["weights"], hq, kvd, pt, lay.num_pages, cache_b, out_b, maxkv, wss)
    torch.cuda.synchronize()
    assert mla.get_error(ws) == 0 and mla.get_error(wss) == 0 and mla.get_error(wsa) == 0
    assert torch.equal(torch.nan_to_num(cache_a, nan=7.0), torch.nan_to_num(cache_b, nan=7.0))
    assert torch.equal(out_a, out_b)
    # And against the oracle.
    dims = oracle_dims(wl)
    w = O.Weights(**c["hw"].as_dict())
    got = out_b.cpu().numpy()
    for b in range(wl.B):
        assert rel_err(got[b], O.mla_decode(dims, w, c["H"][b], n_q)) <= TOL["bf16"]
