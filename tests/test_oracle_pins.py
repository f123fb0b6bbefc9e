"""Pins for the fp64 oracle against what the pages and the mathematics fix.

None of these re-types the oracle's own formula: each checks it against an
independent route (a rotation matrix, complex multiplication, a scalar brute
force, a library attention routine), an invariant the pages state, a closed
form, or a number the pages print.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle as O
from head_latent_attention_append_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_weights(rng, dims: O.Dims) -> O.Weights:
    d_in = dims.d_in

    def g(r, c):
        return rng.standard_normal((r, c)) / math.sqrt(c)

    return O.Weights(
        W_DKV=g(dims.d_c, dims.d_model), W_KR=g(dims.d_r, dims.d_model),
        W_DQ=g(dims.d_cq, dims.d_model) if dims.d_cq else None,
        W_UQ=g(dims.n_h * dims.d_h, d_in), W_QR=g(dims.n_h * dims.d_r, d_in),
        W_UK=g(dims.n_h * dims.d_h, dims.d_c), W_UV=g(dims.n_h * dims.d_v, dims.d_c))


TINY = O.Dims(n_h=2, d_h=3, d_v=5, d_c=4, d_r=2, d_model=6)
TINY_Q = O.Dims(n_h=3, d_h=4, d_v=2, d_c=5, d_r=4, d_model=7, d_cq=3)
SMALL = O.Dims(n_h=4, d_h=8, d_v=6, d_c=16, d_r=8, d_model=24, d_cq=10)


# ---------------------------------------------------------------- RoPE -----
def test_default_scale_reading():
    # One factor 1/sqrt(d_h + d_r) on both score terms (the reading taken).
    d = O.Dims(n_h=128, d_h=128, d_v=128, d_c=512, d_r=64, d_model=5120, d_cq=1536)
    assert d.default_scale() == pytest.approx(1 / math.sqrt(192), rel=1e-15)


def test_rope_frequencies_reading():
    f = O.rope_frequencies(64, 10000.0)
    assert f.shape == (32,)
    assert f[0] == 1.0
    np.testing.assert_allclose(f[-1], 10000.0 ** (-62 / 64), rtol=1e-15)
    assert np.all(np.diff(f) < 0)


def test_rope_matrix_is_a_rotation_and_identity_at_zero():
    f = O.rope_frequencies(16, 10000.0)
    np.testing.assert_array_equal(O.rope_rotation_matrix(0, f), np.eye(16))
    for p in (1, 7, 129, 32769):
        R = O.rope_rotation_matrix(p, f)
        np.testing.assert_allclose(R.T @ R, np.eye(16), atol=1e-14)
        assert abs(np.linalg.det(R) - 1.0) < 1e-12


@pytest.mark.parametrize("m,t", [(0, 5), (3, 3), (128, 17), (32768, 1), (4095, 32769), (20000, 31000)])
def test_rope_relative_property(m, t):
    # R_m^T R_t = R_{t-m}: decoupled-RoPE page, relative property; notion page Step 3.
    f = O.rope_frequencies(64, 10000.0)
    lhs = O.rope_rotation_matrix(m, f).T @ O.rope_rotation_matrix(t, f)
    rhs = O.rope_rotation_matrix(t - m, f)
    np.testing.assert_allclose(lhs, rhs, atol=5e-11)


def test_rope_apply_matches_matrix_and_complex_multiplication():
    rng = np.random.default_rng(1)
    f = O.rope_frequencies(16, 10000.0)
    x = rng.standard_normal((9, 16))
    pos = rng.integers(0, 40000, size=9)
    y = O.rope_apply(x, pos, f)
    for i in range(9):
        np.testing.assert_allclose(y[i], O.rope_rotation_matrix(pos[i], f) @ x[i], atol=1e-13)
    z = (x[:, 0::2] + 1j * x[:, 1::2]) * np.exp(1j * pos[:, None] * f[None, :])
    np.testing.assert_allclose(y[:, 0::2], z.real, atol=1e-12)
    np.testing.assert_allclose(y[:, 1::2], z.imag, atol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)


# ------------------------------------------------------- whole pipeline -----
@pytest.mark.parametrize("dims", [TINY, TINY_Q])
def test_brute_force_tiny(dims):
    rng = np.random.default_rng(2)
    w = rand_weights(rng, dims)
    H = rng.standard_normal((6, dims.d_model))
    rows = [0, 3, 5]
    ref = O.brute_force_sequence(dims, w, H, rows)
    got = O.mla_sequence(dims, w, H, rows)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-13 * np.abs(ref).max())


def test_brute_force_tiny_fp32_decode_workload():
    wl = synth.WORKLOADS["tiny_fp32_decode"]
    dims = O.Dims(wl.n_h, wl.d_h, wl.d_v, wl.d_c, wl.d_r, wl.d_model, wl.d_cq)
    hw = synth.make_weights(wl)
    w = O.Weights(**hw.as_dict())
    H = synth.make_hidden(wl, 0, wl.cached + wl.n_q)
    ref = O.brute_force_sequence(dims, w, H, [wl.cached])
    got = O.mla_decode(dims, w, H, 1)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-13 * np.abs(ref).max())


def test_matches_library_attention_routine():
    """Concatenated per-head vectors [q_C | q_R] . [K_C | k_R] through torch's
    scaled_dot_product_attention (fp64, explicit mask and scale) agree with the
    oracle: a dot product of concatenations is the sum of the halves' products
    ("Latent Attention Meets RoPE", the content/position split)."""
    torch = pytest.importorskip("torch")
    dims = SMALL
    rng = np.random.default_rng(3)
    w = rand_weights(rng, dims)
    T = 11
    H = rng.standard_normal((T, dims.d_model))
    rows = [4, 9, 10]
    pos = np.arange(T, dtype=np.float64)
    f = O.rope_frequencies(dims.d_r, dims.rope_base)
    c, kr = O.cache_entries(w, H, pos, f)
    qc, qr = O.queries(w, dims, H[rows], pos[rows], f)
    n_h = dims.n_h
    K_C = np.einsum("hdc,tc->htd", w.W_UK.reshape(n_h, dims.d_h, dims.d_c), c)
    V = np.einsum("hvc,tc->htv", w.W_UV.reshape(n_h, dims.d_v, dims.d_c), c)
    q = np.concatenate([qc.transpose(1, 0, 2), qr.transpose(1, 0, 2)], axis=-1)       # [h, Q, dh+dr]
    k = np.concatenate([K_C, np.broadcast_to(kr, (n_h,) + kr.shape)], axis=-1)       # [h, T, dh+dr]
    mask = torch.tensor(np.arange(T)[None, :] <= np.asarray(rows)[:, None])
    o = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q), torch.tensor(k), torch.tensor(V), attn_mask=mask,
        scale=1.0 / math.sqrt(dims.d_h + dims.d_r)).numpy().transpose(1, 0, 2)
    got = O.mla_sequence(dims, w, H, rows)
    np.testing.assert_allclose(got, o, rtol=0, atol=1e-12 * np.abs(o).max())


@pytest.mark.parametrize("dims", [SMALL, TINY_Q])
def test_absorbed_equals_materialised(dims):
    # "ropeabsorb" README, "Absorption is exact": agreement to about 2e-13 in
    # fp64, but the two evaluation orders are different reductions.
    rng = np.random.default_rng(4)
    w = rand_weights(rng, dims)
    H = rng.standard_normal((40, dims.d_model))
    rows = [0, 17, 39]
    a = O.mla_sequence(dims, w, H, rows, absorbed=True)
    m = O.mla_sequence(dims, w, H, rows, absorbed=False)
    err = np.abs(a - m).max() / np.abs(m).max()
    assert err <= 1e-12
    assert not np.array_equal(a, m)


def test_common_position_shift_leaves_outputs_unchanged():
    # Relative property => scores depend only on t - m.
    dims = SMALL
    rng = np.random.default_rng(5)
    w = rand_weights(rng, dims)
    H = rng.standard_normal((20, dims.d_model))
    rows = [7, 19]
    base = O.mla_sequence(dims, w, H, rows)
    for delta in (1000, 12345):
        shifted = O.mla_sequence(dims, w, H, rows, positions=np.arange(20) + delta)
        assert np.abs(shifted - base).max() / np.abs(base).max() <= 1e-10
    stretched = O.mla_sequence(dims, w, H, rows, positions=np.arange(20) * 3)
    assert np.abs(stretched - base).max() / np.abs(base).max() > 1e-4


def test_zero_frequency_control_ignores_positions():
    # "ropeabsorb" README, no-RoPE control: with every frequency zero the
    # position operator is constant, so only visibility depends on position.
    dims = SMALL
    rng = np.random.default_rng(6)
    w = rand_weights(rng, dims)
    H = rng.standard_normal((15, dims.d_model))
    zero = np.zeros(dims.d_r // 2)
    a = O.mla_sequence(dims, w, H, [14], freqs=zero)
    b = O.mla_sequence(dims, w, H, [14], freqs=zero, positions=np.arange(15) * 7 + 3)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-14)


def test_single_key_gives_value_of_that_key():
    # With one visible key the softmax weight is 1, so o_h = W_UV,h c_0.
    dims = TINY_Q
    rng = np.random.default_rng(7)
    w = rand_weights(rng, dims)
    H = rng.standard_normal((3, dims.d_model))
    o = O.mla_sequence(dims, w, H, [0])[0]
    c0 = w.W_DKV @ H[0]
    expect = (w.W_UV @ c0).reshape(dims.n_h, dims.d_v)
    np.testing.assert_allclose(o, expect, rtol=1e-13, atol=1e-14)


def test_equal_keys_split_attention_evenly():
    # Two tokens with the same hidden state and W_QR = 0: both scores are
    # equal, alpha = (1/2, 1/2), and o = W_UV c.
    dims = TINY
    rng = np.random.default_rng(8)
    w = rand_weights(rng, dims)
    w.W_QR[:] = 0.0
    h = rng.standard_normal(dims.d_model)
    o = O.mla_sequence(dims, w, np.stack([h, h]), [1])[0]
    expect = (w.W_UV @ (w.W_DKV @ h)).reshape(dims.n_h, dims.d_v)
    np.testing.assert_allclose(o, expect, rtol=1e-13, atol=1e-14)


def test_later_tokens_do_not_reach_earlier_queries():
    dims = SMALL
    rng = np.random.default_rng(9)
    w = rand_weights(rng, dims)
    H = rng.standard_normal((12, dims.d_model))
    a = O.mla_decode(dims, w, H, 2)[0]
    H2 = H.copy()
    H2[-1] += 5.0
    b = O.mla_decode(dims, w, H2, 2)[0]
    np.testing.assert_array_equal(a, b)


def test_materialised_keys_have_rank_d_c():
    # "ropeabsorb" README: the materialised key matrix factors through the
    # latent, so it has rank exactly d_c (a cliff in the singular values).
    dims = O.Dims(n_h=8, d_h=8, d_v=8, d_c=6, d_r=2, d_model=30)
    rng = np.random.default_rng(10)
    w = rand_weights(rng, dims)
    H = rng.standard_normal((50, dims.d_model))
    c = H @ w.W_DKV.T
    K = c @ w.W_UK.T                    # [T, n_h*d_h] = 50 x 64
    s = np.linalg.svd(K, compute_uv=False)
    assert s[dims.d_c - 1] / s[0] > 1e-3
    assert s[dims.d_c] / s[0] < 1e-13


def test_naive_rope_on_the_content_key_cannot_be_absorbed():
    # "Latent Attention Meets RoPE", why RoPE breaks absorption: rotating the
    # content key by its position makes q.k depend on the rotation, so the
    # position-free absorbed score q~.c no longer equals it.
    rng = np.random.default_rng(11)
    d = 8
    W_UK = rng.standard_normal((d, 5))
    q = rng.standard_normal(d)
    c = rng.standard_normal(5)
    f = O.rope_frequencies(d, 10000.0)
    absorbed = (W_UK.T @ q) @ c
    rotated = q @ (O.rope_rotation_matrix(9, f) @ (W_UK @ c))
    assert abs(absorbed - rotated) > 1e-3
    assert abs(absorbed - q @ (O.rope_rotation_matrix(0, f) @ (W_UK @ c))) < 1e-12


# ------------------------------------------------------------ cache sizes ---
def test_cache_sizes_printed_on_the_pages():
    with open(os.path.join(GOLDEN, "cache_sizes.json")) as fh:
        gold = json.load(fh)["entries"]
    for e in gold:
        mha, mla = O.cache_numbers_per_token(e["n_h"], e["d_h"], e["d_v"], e["d_c"], e["d_r"],
                                             e["shared_rope_key"])
        assert (mha, mla) == (e["mha"], e["mla"]), e["cite"]
        if "ratio" in e:
            assert round(mha / mla) == pytest.approx(e["ratio"], abs=1.0)
        if "reduction" in e:
            assert 1 - mla / mha == pytest.approx(e["reduction"], abs=0.01)


# --------------------------------------------- per-head position keys -----
# The 16-head example of "Multi-Head Latent Attention" (talalahmed), "A
# concrete size comparison", caches one RoPE key per head.
import dataclasses  # noqa: E402

TINY_PH = dataclasses.replace(TINY, rope_per_head=True)
SMALL_PH = dataclasses.replace(SMALL, rope_per_head=True)


def per_head_weights(rng, dims):
    w = rand_weights(rng, dataclasses.replace(dims, rope_per_head=False))
    w.W_KR = rng.standard_normal((dims.n_h * dims.d_r, dims.d_model)) / math.sqrt(dims.d_model)
    return w


def test_per_head_keys_reduce_to_the_shared_key_when_every_block_is_the_same():
    rng = np.random.default_rng(20)
    w = rand_weights(rng, SMALL)
    H = rng.standard_normal((25, SMALL.d_model))
    rows = [0, 12, 24]
    w_ph = dataclasses.replace(w, W_KR=np.tile(w.W_KR, (SMALL.n_h, 1)))
    shared = O.mla_sequence(SMALL, w, H, rows)
    per_head = O.mla_sequence(SMALL_PH, w_ph, H, rows)
    np.testing.assert_allclose(per_head, shared, rtol=0, atol=1e-13 * np.abs(shared).max())


def test_per_head_keys_brute_force_tiny():
    rng = np.random.default_rng(21)
    w = per_head_weights(rng, TINY_PH)
    H = rng.standard_normal((6, TINY_PH.d_model))
    rows = [0, 2, 5]
    ref = O.brute_force_sequence(TINY_PH, w, H, rows)
    got = O.mla_sequence(TINY_PH, w, H, rows)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-13 * np.abs(ref).max())


def test_per_head_keys_absorbed_equals_materialised():
    rng = np.random.default_rng(22)
    w = per_head_weights(rng, SMALL_PH)
    H = rng.standard_normal((30, SMALL_PH.d_model))
    a = O.mla_sequence(SMALL_PH, w, H, [3, 29], absorbed=True)
    m = O.mla_sequence(SMALL_PH, w, H, [3, 29])
    assert np.abs(a - m).max() / np.abs(m).max() <= 1e-12
    assert not np.array_equal(a, m)


def test_per_head_keys_keep_the_relative_property():
    rng = np.random.default_rng(23)
    w = per_head_weights(rng, SMALL_PH)
    H = rng.standard_normal((18, SMALL_PH.d_model))
    base = O.mla_sequence(SMALL_PH, w, H, [17])
    shifted = O.mla_sequence(SMALL_PH, w, H, [17], positions=np.arange(18) + 4321)
    assert np.abs(shifted - base).max() / np.abs(base).max() <= 1e-10


def test_per_head_keys_use_each_heads_own_block():
    """Distinct blocks change every head's scores: the result differs from the
    shared-key result built from head 0's block, and head h's output depends
    only on block h (replacing block 1 leaves head 0 unchanged)."""
    rng = np.random.default_rng(24)
    w = per_head_weights(rng, SMALL_PH)
    H = rng.standard_normal((22, SMALL_PH.d_model))
    got = O.mla_sequence(SMALL_PH, w, H, [21])
    w0 = dataclasses.replace(w, W_KR=w.W_KR[:SMALL.d_r])
    assert np.abs(got - O.mla_sequence(SMALL, w0, H, [21])).max() / np.abs(got).max() > 1e-3
    W2 = w.W_KR.copy()
    W2[SMALL.d_r:2 * SMALL.d_r] = rng.standard_normal((SMALL.d_r, SMALL.d_model))
    got2 = O.mla_sequence(SMALL_PH, dataclasses.replace(w, W_KR=W2), H, [21])
    np.testing.assert_array_equal(got2[:, 0], got[:, 0])
    assert not np.allclose(got2[:, 1], got[:, 1])


def test_per_head_cache_row_matches_the_pages_16_head_example():
    """cache_entries of the 16-head example stores d_c + n_h * d_r = 768
    numbers per token: the per-head size the page prints."""
    with open(os.path.join(GOLDEN, "cache_sizes.json")) as fh:
        ent = [e for e in json.load(fh)["entries"] if not e["shared_rope_key"]][0]
    dims = O.Dims(n_h=ent["n_h"], d_h=ent["d_h"], d_v=ent["d_v"], d_c=ent["d_c"], d_r=ent["d_r"], d_model=40,
                  rope_per_head=True)
    rng = np.random.default_rng(25)
    w = per_head_weights(rng, dims)
    c, k_r = O.cache_entries(O.as_f64(w), rng.standard_normal((3, 40)), np.arange(3),
                             O.rope_frequencies(dims.d_r, dims.rope_base))
    assert k_r.shape == (3, dims.n_h, dims.d_r)
    assert c.shape[1] + k_r[0].size == ent["mla"] == 768
