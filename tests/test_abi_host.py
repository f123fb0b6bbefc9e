"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/mla.h declares, sizes its buffers, and rejects bad
arguments before anything is launched."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def mla():
    from head_latent_attention_append_b200 import build
    build.build()
    from head_latent_attention_append_b200 import mla as m
    return m


def declared_functions():
    with open(os.path.join(ROOT, "include", "mla.h")) as fh:
        text = fh.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(mla):
    names = declared_functions()
    assert len(names) >= 12
    lib = ctypes.CDLL(mla.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(mla.EXPORTED)


def dims3(mla, **kw):
    d = dict(n_h=128, d_h=128, d_v=128, d_c=512, d_r=64, d_model=5120, d_cq=1536)
    d.update(kw)
    return mla.make_dims(**d)


def test_size_queries(mla):
    d = dims3(mla)
    assert mla.absorbed_weights_bytes(d) >= 2 * (576 * 5120 + 1536 * 5120 + 128 * 192 * 1536 + 2 * 128 * 128 * 512)
    assert mla.decode_workspace_bytes(d, 64, 1, 8193) > 0
    assert mla.prefill_workspace_bytes(d, 4, 4096) > mla.decode_workspace_bytes(d, 64, 1, 8193)
    assert mla.append_workspace_bytes(d, 64) > 0
    # Invalid or unsupported dimensions size to 0.
    assert mla.absorbed_weights_bytes(dims3(mla, d_r=63)) == 0
    assert mla.absorbed_weights_bytes(dims3(mla, page_size=32)) == 0
    assert mla.absorbed_weights_bytes(dims3(mla, n_h=0)) == 0
    assert mla.decode_workspace_bytes(d, 0, 1, 10) == 0
    assert mla.decode_workspace_bytes(d, 4, 2, 1) == 0
    # Context-parallel partials: one partial slot per segment (more row blocks
    # than the decode path's slots need a larger workspace); bf16 only.
    assert mla.decode_cp_workspace_bytes(d, 64, 1) >= mla.decode_workspace_bytes(d, 64, 1, 8193)
    assert mla.decode_cp_workspace_bytes(d, 1024, 1) > mla.decode_workspace_bytes(d, 1024, 1, 8193)
    assert mla.decode_cp_workspace_bytes(dims3(mla, dtype=mla.F32), 4, 1) == 0
    assert mla.decode_cp_workspace_bytes(d, 0, 1) == 0
    # Per-head RoPE keys: cache rows of d_c + n_h * d_r up to 1024 (the 16-head, 32-dim page example: 768);
    # the absorbed weights hold n_h RoPE-key projections; no context-parallel or materialised path.
    page = dict(n_h=16, d_h=128, d_v=128, d_c=256, d_r=32, d_model=2048, d_cq=0)
    shared, per_head = dims3(mla, **page), dims3(mla, rope_key_per_head=1, **page)
    assert mla.absorbed_weights_bytes(per_head) - mla.absorbed_weights_bytes(shared) >= 2 * 15 * 32 * 2048
    assert mla.absorbed_weights_bytes(dims3(mla, rope_key_per_head=1)) == 0       # 512 + 128 * 64 > 1024
    assert mla.absorbed_weights_bytes(dims3(mla, rope_key_per_head=2)) == 0
    assert mla.decode_cp_workspace_bytes(per_head, 4, 1) == 0
    assert mla.prefill_materialised_workspace_bytes(dims3(mla, rope_key_per_head=1, n_h=8), 2, 64) == 0
    # Materialised prefill: bf16, d_r = 64, d_h and d_v in {64, 128}; it holds the expanded K_C and V.
    assert mla.prefill_materialised_workspace_bytes(d, 4, 4096) >= 2 * 4 * 4096 * 128 * (128 + 128)
    assert mla.prefill_materialised_workspace_bytes(dims3(mla, d_r=32), 4, 4096) == 0
    assert mla.prefill_materialised_workspace_bytes(dims3(mla, d_h=96), 4, 4096) == 0
    assert mla.prefill_materialised_workspace_bytes(dims3(mla, dtype=mla.F32), 4, 4096) == 0
    assert mla.prefill_materialised_workspace_bytes(d, 0, 4096) == 0


def test_status_strings(mla):
    for code, name in mla.STATUS.items():
        assert mla.status_string(code) == name


FAKE = 0x100000  # aligned, never dereferenced: every call below returns before any CUDA call


def test_bad_arguments_are_rejected_before_launch(mla):
    lib = mla.lib
    d = dims3(mla)
    h = ctypes.c_void_p()
    P = ctypes.c_void_p
    # Null weights.
    assert lib.mla_absorb_weights(ctypes.byref(d), None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                  1 << 40, ctypes.byref(h), None) == -1
    # W_DQ given although d_cq == 0.
    d0 = dims3(mla, d_cq=0)
    assert lib.mla_absorb_weights(ctypes.byref(d0), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                  1 << 40, ctypes.byref(h), None) == -1
    # Buffer too small / misaligned.
    assert lib.mla_absorb_weights(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                  1024, ctypes.byref(h), None) == -3
    assert lib.mla_absorb_weights(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 8,
                                  1 << 40, ctypes.byref(h), None) == -1
    # Unsupported dims.
    dbad = dims3(mla, d_r=7)
    assert lib.mla_absorb_weights(ctypes.byref(dbad), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                  1 << 40, ctypes.byref(h), None) == -2
    # Calls with a null handle.
    assert lib.mla_decode(None, FAKE, FAKE, FAKE, 4, 4, FAKE, FAKE, 1, 1, 10, FAKE, 1 << 30, None) == -1
    assert lib.mla_append_latent(None, FAKE, FAKE, FAKE, FAKE, 1, 4, 4, FAKE, 1, FAKE, 1 << 30, None) == -1
    assert lib.mla_prefill(None, FAKE, FAKE, 4, 4, FAKE, FAKE, 1, 8, FAKE, 1 << 30, None) == -1
    assert lib.mla_decode_cp_partial(None, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 4, FAKE, FAKE, FAKE, 1, 1, 10, FAKE,
                                     1 << 30, None) == -1
    assert lib.mla_decode_cp_combine(None, 2, FAKE, FAKE, FAKE, 1, 1, FAKE, 1 << 30, None) == -1
    assert lib.mla_get_error(None, None) == -1
    assert lib.mla_weights_dims(None, ctypes.byref(d)) == -1
    # The timeout self-test hook: null or misaligned workspace, limit out of range.
    assert lib.mla_selftest_wait_timeout(None, 1000, None) == -1
    assert lib.mla_selftest_wait_timeout(FAKE + 8, 1000, None) == -1
    assert lib.mla_selftest_wait_timeout(FAKE, 0, None) == -1
    assert lib.mla_selftest_wait_timeout(FAKE, 1000001, None) == -1


def test_handle_arguments_checked_before_launch(mla):
    """A handle built from host-side fakes: argument checks and workspace
    checks must fire before any CUDA call."""
    lib = mla.lib
    # mla_absorb_weights launches copies, so forge no handle; check the
    # workspace and size arguments of the calls through a decode with a null
    # workspace instead.
    d = dims3(mla)
    assert mla.decode_workspace_bytes(d, 2, 1, 100) > 4096


def test_binding_fails_loudly_without_the_library(mla, monkeypatch, tmp_path):
    """No fallback: with libmla.so absent the binding refuses to load."""
    monkeypatch.setattr(mla, "LIB_PATH", str(tmp_path / "libmla.so"))
    with pytest.raises(ImportError, match="libmla.so not built"):
        mla._load()
