"""Context-parallel decode on the host: the window plan and page tables, the
oracle's window partials and merge pinned against the materialised oracle,
and the exchange on two gloo ranks (CPU)."""
import os
import socket
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

import oracle as O  # noqa: E402
from head_latent_attention_append_b200 import cp, synth  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("n_ranks", [1, 2, 3, 4, 8])
def test_windows_partition_every_sequence(n_ranks):
    rng = np.random.default_rng(7)
    kv = np.concatenate([[1, 2, 63, 64, 65, 128, 129], rng.integers(1, 5000, 20)]).astype(np.int32)
    wins = cp.shard_windows(kv, n_ranks, 64)
    assert len(wins) == n_ranks
    for b, L in enumerate(kv):
        pos = 0
        for win in wins:
            s, c = int(win.start[b]), int(win.count[b])
            assert s % 64 == 0 and c >= 0
            if c:
                assert s == pos, (b, s, pos)   # contiguous, in rank order
                pos += c
        assert pos == L                          # every key exactly once
        pages = -(-int(L) // 64)
        held = [-(-int(w.count[b]) // 64) for w in wins]
        assert max(held) - min(held) <= 1 or pages < n_ranks


def test_rank_page_tables_agree():
    kv = np.array([1, 200, 64, 700], np.int32)
    for win in cp.shard_windows(kv, 3, 64):
        order = np.random.default_rng(1).permutation(int(((win.count + 63) // 64).sum()) + 2)
        rp = cp.rank_pages(win, kv, 64, order=order, spare_pages=2)
        used = rp.local[rp.local >= 0]
        assert len(set(used.tolist())) == used.size and used.max(initial=-1) < rp.num_pages
        for b in range(len(kv)):
            n = -(-int(win.count[b]) // 64)
            g0 = int(win.start[b]) // 64
            np.testing.assert_array_equal(rp.by_position[b, g0:g0 + n], rp.local[b, :n])
            assert (rp.local[b, n:] == -1).all()
            assert (np.delete(rp.by_position[b], np.arange(g0, g0 + n)) == -1).all()


def _small(d_cq):
    wl = synth.Workload("cp_pin", 11, 4, 8, 8, 16, 4, 32, d_cq, "f32", "decode", 1, 1, 0)
    dims = O.Dims(wl.n_h, wl.d_h, wl.d_v, wl.d_c, wl.d_r, wl.d_model, wl.d_cq, wl.rope_base)
    return wl, dims, O.Weights(**synth.make_weights(wl).as_dict())


@pytest.mark.parametrize("d_cq", [0, 12])
@pytest.mark.parametrize("n_q", [1, 3])
def test_merged_window_partials_equal_the_materialised_decode(d_cq, n_q):
    """Windows of any split, merged by their base-2 log-sum-exp and projected
    by W_UV, give the materialised oracle's output; a window the queries
    cannot see has lse = -inf; one window covering everything has the
    log-sum-exp of the whole softmax."""
    wl, dims, w = _small(d_cq)
    T = 150
    H = synth.make_hidden(wl, 0, T)
    ref = O.mla_decode(dims, w, H, n_q)
    splits = [[(0, T)], [(0, 64), (64, T - 64)], [(0, 16), (16, 48), (64, 64), (128, 22)],
              [(0, T - 2), (T - 2, 2)], [(0, 0), (0, 96), (96, 54)]]
    whole = O.window_partial(dims, w, H, n_q, 0, T)
    for split in splits:
        parts = [O.window_partial(dims, w, H, n_q, s, c) for s, c in split]
        out = O.latent_output(dims, w, O.merge_windows(parts))
        assert np.abs(out - ref).max() <= 1e-12 * np.abs(ref).max(), split
        lse = np.stack([p[1] for p in parts])
        with np.errstate(divide="ignore"):
            total = np.log2(np.exp2(lse).sum(axis=0))
        np.testing.assert_allclose(total, whole[1], rtol=0, atol=1e-12)
    # The window [T-2, T) holds only the last two new tokens: the first new
    # token (position T-n_q) sees none of it when n_q = 3.
    o_last, lse_last = O.window_partial(dims, w, H, n_q, T - 2, 2)
    if n_q == 3:
        assert np.all(lse_last[0] == -np.inf) and np.all(o_last[0] == 0)
        assert np.all(np.isfinite(lse_last[1:]))
    # One key: the partial is that key's latent, its lse the key's score.
    o1, l1 = O.window_partial(dims, w, H, 1, T - 1, 1)
    c_last, _ = O.cache_entries(O.as_f64(w), H[T - 1:], np.array([T - 1.0]), O.rope_frequencies(dims.d_r,
                                                                                               dims.rope_base))
    np.testing.assert_allclose(o1[0], np.broadcast_to(c_last[0], o1[0].shape), rtol=0, atol=1e-12)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, q):
    sys.path.insert(0, ROOT)
    import oracle as Ow
    from head_latent_attention_append_b200 import cp as cpw
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        _exchange(rank, ws, q, Ow, cpw)
    except Exception as e:  # report instead of leaving the parent waiting
        q.put((rank, float("inf"), repr(e)))
    finally:
        dist.destroy_process_group()


def _exchange(rank, ws, q, Ow, cpw):
    wl, dims, w = _small(12)
    T, n_q = 150, 2
    H = synth.make_hidden(wl, 0, T)
    win = cpw.shard_windows(np.array([T], np.int32), ws, 16)[rank]
    o_bar, lse = Ow.window_partial(dims, w, H, n_q, int(win.start[0]), int(win.count[0]))
    ob, ls = cpw.gather_partials(torch.from_numpy(o_bar), torch.from_numpy(lse))
    parts = [(ob[r].numpy(), ls[r].numpy()) for r in range(ws)]
    out = Ow.latent_output(dims, w, Ow.merge_windows(parts))
    ref = Ow.mla_decode(dims, w, H, n_q)
    # The gathered partials are in rank order: rank r's slot is its own.
    own = np.array_equal(ob[rank].numpy(), o_bar) and np.array_equal(ls[rank].numpy(), lse)
    q.put((rank, float(np.abs(out - ref).max() / np.abs(ref).max()), own))
    dist.barrier()


def test_exchange_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    for rank, err, own in res:
        assert own is True, (rank, own)
        assert err <= 1e-12, (rank, err)


def _orchestration_worker(rank, ws, port, q):
    """cp.decode_cp on one gloo rank, with libmla's two calls stood in for by
    the oracle (test-only fakes): checks the step's buffers, the exchange
    and the hand-off to the merge."""
    sys.path.insert(0, ROOT)
    import types
    import oracle as Ow
    from head_latent_attention_append_b200 import cp as cpw
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        wl, dims, w = _small(0)
        n_q, lengths = 2, [150, 40, 1]
        kv = np.asarray(lengths, np.int32) + n_q
        H = [synth.make_hidden(wl, b, int(kv[b])) for b in range(len(lengths))]
        win = cpw.shard_windows(kv, ws, 16)[rank]

        def fake_partial(wt, h_q, kv_len, start, count, pt, num_pages, cache, obar_out, lse_out, max_kv_len,
                         workspace, stream=None):
            for b in range(h_q.shape[0]):
                o, ls = Ow.window_partial(dims, w, H[b], n_q, int(start[b]), int(count[b]))
                obar_out[b] = torch.from_numpy(o)
                lse_out[b] = torch.from_numpy(ls)

        def fake_combine(wt, obar_parts, lse_parts, out, workspace, stream=None):
            for b in range(out.shape[0]):
                parts = [(obar_parts[r, b].numpy(), lse_parts[r, b].double().numpy())
                         for r in range(obar_parts.shape[0])]
                out[b] = torch.from_numpy(Ow.latent_output(dims, w, Ow.merge_windows(parts)))

        fake_mla = types.SimpleNamespace(decode_cp_partial=fake_partial, decode_cp_combine=fake_combine)
        import head_latent_attention_append_b200 as pkg
        sys.modules["head_latent_attention_append_b200.mla"] = fake_mla
        pkg.mla = fake_mla
        h_q = torch.from_numpy(np.stack([H[b][-n_q:] for b in range(len(lengths))]).astype(np.float64))
        out = torch.empty((len(lengths), n_q, dims.n_h, dims.d_v), dtype=torch.float64)
        wts = types.SimpleNamespace(dims=dims)
        obar_parts, lse_parts = cpw.decode_cp(wts, h_q, torch.from_numpy(kv), torch.from_numpy(win.start),
                                              torch.from_numpy(win.count), None, 0, None, out, int(kv.max()), None)
        err = max(float(np.abs(out[b].numpy() - Ow.mla_decode(dims, w, H[b], n_q)).max()
                        / np.abs(Ow.mla_decode(dims, w, H[b], n_q)).max()) for b in range(len(lengths)))
        q.put((rank, err, tuple(obar_parts.shape), tuple(lse_parts.shape)))
        dist.barrier()
    except Exception as e:  # report instead of leaving the parent waiting
        q.put((rank, float("inf"), repr(e), None))
    finally:
        dist.destroy_process_group()


def test_decode_step_orchestration_on_three_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ws = 3
    procs = [ctx.Process(target=_orchestration_worker, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    for rank, err, oshape, lshape in res:
        assert err <= 1e-6, (rank, err, oshape)   # lse travels as fp32
        assert oshape == (ws, 3, 2, 4, 16) and lshape == (ws, 3, 2, 4), (oshape, lshape)
