"""The benchmark's accounting (CPU): unique and streamed cache bytes and the
attention flops of a step, against brute-force counting of (query, key) pairs
and the per-step figures of the decode and prefill workloads."""
import types

import numpy as np
import pytest

from head_latent_attention_append_b200 import synth

pytest.importorskip("torch")
from head_latent_attention_append_b200 import workload  # noqa: E402


def _setup(wl, kv):
    return types.SimpleNamespace(wl=wl, kv_len_host=np.asarray(kv, np.int32))


def _brute(wl, kv):
    """Pairs and streamed keys by enumeration: new token q of a sequence with
    L keys sits at L - n_q + q and sees every key at a position <= its own."""
    pairs = 0
    for L in kv:
        for q in range(wl.n_q):
            pos = int(L) - wl.n_q + q
            pairs += sum(1 for t in range(int(L)) if t <= pos)
    return pairs


@pytest.mark.parametrize("n_q", [1, 2, 4])
def test_decode_accounting_matches_enumeration(n_q):
    base = synth.WORKLOADS["page_bf16_decode"]
    wl = synth.Workload("acct", 12, base.n_h, base.d_h, base.d_v, base.d_c, base.d_r, base.d_model, base.d_cq,
                        "bf16", "decode", 5, n_q, 0)
    kv = np.array([1, 63, 64, 65, 300]) + n_q
    s = _setup(wl, kv)
    pairs = _brute(wl, kv)
    assert workload.Setup.cache_bytes_unique(s) == int(kv.sum()) * wl.d_cr * 2
    assert workload.Setup.cache_bytes_read(s) == pairs * wl.d_cr * 2
    assert workload.Setup.attention_flops(s) == pairs * wl.n_h * (2 * wl.d_cr + 2 * wl.d_c)


def test_prefill_accounting_counts_causal_pairs():
    wl = synth.Workload("acct_p", 13, 4, 8, 8, 128, 16, 64, 0, "bf16", "prefill", 3, 70, 0)
    s = _setup(wl, np.zeros(3, np.int32))
    pairs = 3 * sum(t + 1 for t in range(70))
    assert workload.Setup.attention_flops(s) == pairs * wl.n_h * (2 * wl.d_cr + 2 * wl.d_c)
    assert workload.Setup.cache_bytes_read(s) == pairs * wl.d_cr * 2


def test_headline_figures_of_the_decode_and_prefill_workloads():
    wl = synth.WORKLOADS["dsv2_bf16_decode"]
    s = _setup(wl, synth.kv_lengths(wl))
    assert workload.Setup.cache_bytes_unique(s) == 604_053_504          # 64 x 8193 keys x 1152 B
    assert workload.Setup.attention_flops(s) == 64 * 8193 * 278_528       # 146.05 GFLOP
    wp = synth.WORKLOADS["dsv2_bf16_prefill"]
    sp = _setup(wp, np.zeros(wp.B, np.int32))
    assert workload.Setup.attention_flops(sp) == 33_562_624 * 278_528     # 9.348 TFLOP over the causal pairs


def test_materialised_prefill_counts_its_own_flops():
    """The materialised twin of the prefill workload scores over d_h + d_r
    columns and sums d_v: 640 flops per pair and head instead of 2176."""
    wm = synth.WORKLOADS["dsv2_bf16_prefill_mat"]
    wp = synth.WORKLOADS["dsv2_bf16_prefill"]
    assert wm.materialised and not wp.materialised
    assert (wm.B, wm.n_q, wm.wid) == (wp.B, wp.n_q, wp.wid)         # the same inputs
    sm = _setup(wm, np.zeros(wm.B, np.int32))
    assert wm.flops_per_pair() == 128 * (2 * (128 + 64) + 2 * 128) == 81_920
    assert workload.Setup.attention_flops(sm) == 33_562_624 * 81_920      # 2.749 TFLOP
