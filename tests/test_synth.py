"""The seeded input recipe shared by the oracle and the CUDA path (CPU): bf16
rounding, page pools, ragged lengths, checked-sequence picks and weight
scales."""
import math

import numpy as np
import pytest

from head_latent_attention_append_b200 import synth

torch = pytest.importorskip("torch")


def test_round_bf16_is_round_to_nearest_even():
    rng = np.random.default_rng(3)
    x = np.concatenate([
        rng.standard_normal(100_000).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 30, 100_000),
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38, 1e-40, np.inf, -np.inf], np.float32),
    ]).astype(np.float32)
    # Exact ties: the dropped 16 bits are 0x8000, the kept part odd or even.
    ties = (rng.integers(0x0080, 0x7F00, 2000, dtype=np.uint32) << 16 | 0x8000).astype(np.uint32).view(np.float32)
    x = np.concatenate([x, ties, -ties])
    ours = synth.round_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(ours.view(np.uint32), ref.view(np.uint32))
    # Rounded values are bf16 already: rounding again changes nothing.
    np.testing.assert_array_equal(synth.round_bf16(ours).view(np.uint32), ours.view(np.uint32))


@pytest.mark.parametrize("shuffle", [True, False])
def test_page_pool_holds_every_sequence_exactly(shuffle):
    kv = np.array([1, 63, 64, 65, 128, 1000, 4097], np.int32)
    lay = synth.page_layout(kv, 64, shuffle=shuffle, wl_id=5, seed=9, spare_pages=3)
    need = [-(-int(L) // 64) for L in kv]
    assert lay.num_pages == sum(need) + 3 and lay.max_pages == max(need)
    used = []
    for b, n in enumerate(need):
        row = lay.page_table[b]
        assert (row[:n] >= 0).all() and (row[n:] == -1).all()
        used += row[:n].tolist()
    assert len(set(used)) == len(used) and max(used) < lay.num_pages
    if not shuffle:
        assert used == list(range(len(used)))
    again = synth.page_layout(kv, 64, shuffle=shuffle, wl_id=5, seed=9, spare_pages=3)
    np.testing.assert_array_equal(lay.page_table, again.page_table)


@pytest.mark.parametrize("name", ["dsv2_ragged_decode", "dsv2_spec4_decode"])
def test_ragged_lengths_are_seeded_and_in_range(name):
    wl = synth.WORKLOADS[name]
    kv = synth.kv_lengths(wl)
    assert kv.shape == (wl.B,) and kv.dtype == np.int32
    assert kv.min() >= 1 + wl.n_q and kv.max() <= wl.max_cached + wl.n_q
    np.testing.assert_array_equal(kv, synth.kv_lengths(wl))
    assert not np.array_equal(kv, synth.kv_lengths(wl, seed=synth.BASE_SEED + 1))


def test_checked_sequences_cover_the_length_extremes():
    wl = synth.WORKLOADS["dsv2_ragged_decode"]
    cached = synth.cached_lengths(wl)
    picks = synth.checked_sequences(wl, cached, 8)
    assert len(picks) == 8 and picks == sorted(set(picks))
    assert int(np.argmin(cached)) in picks and int(np.argmax(cached)) in picks
    residues = {(int(cached[b]) + wl.n_q) % 64 for b in picks}
    assert {63, 0} <= residues


@pytest.mark.parametrize("name", ["page_bf16_decode", "tiny_fp32_decode"])
def test_weights_follow_the_recipe(name):
    wl = synth.WORKLOADS[name]
    hw = synth.make_weights(wl)
    d_in = wl.d_cq if wl.d_cq > 0 else wl.d_model
    shapes = {"W_DKV": (wl.d_c, wl.d_model), "W_KR": (wl.d_r, wl.d_model), "W_UQ": (wl.n_h * wl.d_h, d_in),
              "W_QR": (wl.n_h * wl.d_r, d_in), "W_UK": (wl.n_h * wl.d_h, wl.d_c),
              "W_UV": (wl.n_h * wl.d_v, wl.d_c)}
    for k, shp in shapes.items():
        W = getattr(hw, k)
        assert W.shape == shp and W.dtype == np.float32
        # N(0, 1) / sqrt(fan_in): the sample std is within a few percent.
        assert abs(W.std() * math.sqrt(shp[1]) - 1.0) < 0.06, k
        if wl.dtype == "bf16":
            np.testing.assert_array_equal(synth.round_bf16(W), W)
    assert (hw.W_DQ is None) == (wl.d_cq == 0)
    h = synth.make_hidden(wl, 2, 5)
    np.testing.assert_array_equal(h, synth.make_hidden(wl, 2, 5))
    assert not np.array_equal(h, synth.make_hidden(wl, 3, 5))
