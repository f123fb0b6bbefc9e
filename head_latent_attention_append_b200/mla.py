"""Thin ctypes binding over libmla's C ABI (include/mla.h).

Argument marshalling only: tensors are passed as raw device pointers, the
stream as the raw CUDA stream handle.  Every computation runs in libmla's
kernels; importing this module fails loudly when libmla.so is missing.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import Dict, Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmla.so")

MLA_OK = 0
STATUS = {0: "MLA_OK", -1: "MLA_ERR_INVALID_ARG", -2: "MLA_ERR_UNSUPPORTED", -3: "MLA_ERR_WORKSPACE",
          -4: "MLA_ERR_CUDA", -5: "MLA_ERR_DEVICE_BOUNDS", -6: "MLA_ERR_TIMEOUT"}
F32, BF16 = 0, 1

EXPORTED = [
    "mla_absorbed_weights_bytes", "mla_absorb_weights", "mla_release_weights", "mla_weights_dims",
    "mla_append_workspace_bytes", "mla_append_latent", "mla_decode_workspace_bytes", "mla_decode",
    "mla_prefill_workspace_bytes", "mla_prefill", "mla_get_error", "mla_status_string",
    "mla_last_launch_count", "mla_profile_begin", "mla_profile_end", "mla_append_latent_noalloc",
    "mla_decode_cp_workspace_bytes", "mla_decode_cp_partial", "mla_decode_cp_combine",
    "mla_selftest_wait_timeout", "mla_prefill_materialised_workspace_bytes", "mla_prefill_materialised",
    "mla_decode_step_workspace_bytes", "mla_decode_step",
]
APPEND_NOALLOC_MAX_T = 256


class MlaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)}")
        self.code = code


class Dims(ctypes.Structure):
    _fields_ = [("n_h", ctypes.c_int), ("d_h", ctypes.c_int), ("d_v", ctypes.c_int), ("d_c", ctypes.c_int),
                ("d_r", ctypes.c_int), ("d_model", ctypes.c_int), ("d_cq", ctypes.c_int),
                ("rope_base", ctypes.c_float), ("softmax_scale", ctypes.c_float), ("page_size", ctypes.c_int),
                ("dtype", ctypes.c_int), ("rope_key_per_head", ctypes.c_int)]


def make_dims(n_h, d_h, d_v, d_c, d_r, d_model, d_cq=0, rope_base=10000.0, softmax_scale=0.0,
              page_size=64, dtype=BF16, rope_key_per_head=0) -> Dims:
    return Dims(n_h, d_h, d_v, d_c, d_r, d_model, d_cq, rope_base, softmax_scale, page_size, dtype,
                int(rope_key_per_head))


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libmla.so not built ({LIB_PATH}); run head_latent_attention_append_b200/build.py")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, Z, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_int
    D = ctypes.POINTER(Dims)
    sig = {
        "mla_absorbed_weights_bytes": (Z, [D]),
        "mla_absorb_weights": (S, [D, P, P, P, P, P, P, P, P, Z, ctypes.POINTER(P), P]),
        "mla_release_weights": (None, [P]),
        "mla_weights_dims": (S, [P, D]),
        "mla_append_workspace_bytes": (Z, [D, I]),
        "mla_append_latent": (S, [P, P, P, P, P, I, I, I, P, I, P, Z, P]),
        "mla_decode_workspace_bytes": (Z, [D, I, I, I]),
        "mla_decode": (S, [P, P, P, P, I, I, P, P, I, I, I, P, Z, P]),
        "mla_decode_step_workspace_bytes": (Z, [D, I, I, I]),
        "mla_decode_step": (S, [P, P, P, P, I, I, P, P, I, I, I, P, Z, P]),
        "mla_prefill_workspace_bytes": (Z, [D, I, I]),
        "mla_prefill": (S, [P, P, P, I, I, P, P, I, I, P, Z, P]),
        "mla_get_error": (S, [P, P]),
        "mla_status_string": (ctypes.c_char_p, [S]),
        "mla_last_launch_count": (I, []),
        "mla_profile_begin": (S, [I]),
        "mla_append_latent_noalloc": (S, [P, P, P, P, P, I, I, I, P, I, P, P]),
        "mla_profile_end": (S, [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int)]),
        "mla_decode_cp_workspace_bytes": (Z, [D, I, I]),
        "mla_decode_cp_partial": (S, [P, P, P, P, P, P, I, I, P, P, P, I, I, I, P, Z, P]),
        "mla_decode_cp_combine": (S, [P, I, P, P, P, I, I, P, Z, P]),
        "mla_selftest_wait_timeout": (S, [P, I, P]),
        "mla_prefill_materialised_workspace_bytes": (Z, [D, I, I]),
        "mla_prefill_materialised": (S, [P, P, P, I, I, P, P, I, I, P, Z, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


lib = _load()


def _check(fn: str, code: int):
    if code != MLA_OK:
        raise MlaError(fn, code)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def absorbed_weights_bytes(dims: Dims) -> int:
    return lib.mla_absorbed_weights_bytes(ctypes.byref(dims))


def append_workspace_bytes(dims: Dims, T: int) -> int:
    return lib.mla_append_workspace_bytes(ctypes.byref(dims), T)


def decode_workspace_bytes(dims: Dims, B: int, n_q: int, max_kv_len: int) -> int:
    return lib.mla_decode_workspace_bytes(ctypes.byref(dims), B, n_q, max_kv_len)


def decode_step_workspace_bytes(dims: Dims, B: int, n_q: int, max_kv_len: int) -> int:
    return lib.mla_decode_step_workspace_bytes(ctypes.byref(dims), B, n_q, max_kv_len)


def prefill_workspace_bytes(dims: Dims, B: int, S: int) -> int:
    return lib.mla_prefill_workspace_bytes(ctypes.byref(dims), B, S)


def last_launch_count() -> int:
    return lib.mla_last_launch_count()


def profile_begin(max_launches: int):
    _check("mla_profile_begin", lib.mla_profile_begin(max_launches))


def profile_end():
    """Returns (summed attention-kernel milliseconds, timed launches)."""
    ms, n = ctypes.c_double(), ctypes.c_int()
    _check("mla_profile_end", lib.mla_profile_end(ctypes.byref(ms), ctypes.byref(n)))
    return ms.value, n.value


class Weights:
    """Absorbed weights: a caller-owned device buffer plus libmla's handle."""

    def __init__(self, dims: Dims, W: Dict[str, "torch.Tensor"], stream=None):
        import torch
        self.dims = dims
        nbytes = absorbed_weights_bytes(dims)
        if nbytes == 0:
            raise MlaError("mla_absorbed_weights_bytes", -2)
        dev = W["W_DKV"].device
        self.buffer = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        h = ctypes.c_void_p()
        _check("mla_absorb_weights", lib.mla_absorb_weights(
            ctypes.byref(dims), _ptr(W["W_DKV"]), _ptr(W["W_KR"]), _ptr(W.get("W_DQ")), _ptr(W["W_UQ"]),
            _ptr(W["W_QR"]), _ptr(W["W_UK"]), _ptr(W["W_UV"]), self.buffer.data_ptr(), nbytes, ctypes.byref(h),
            _stream(stream)))
        self.handle = h

    def close(self):
        if self.handle:
            lib.mla_release_weights(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def append_latent(w: Weights, h, seq_idx, pos, page_table, num_pages: int, cache, workspace, stream=None):
    T = h.shape[0]
    num_seqs, max_pages = page_table.shape
    _check("mla_append_latent", lib.mla_append_latent(
        w.handle, _ptr(h), _ptr(seq_idx), _ptr(pos), _ptr(page_table), num_seqs, max_pages, num_pages,
        _ptr(cache), T, _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def append_latent_noalloc(w: Weights, h, seq_idx, pos, page_table, num_pages: int, cache, device_error=None,
                          stream=None):
    """mla_append_latent without a workspace (scratch inside libmla; T <= 256)."""
    T = h.shape[0]
    num_seqs, max_pages = page_table.shape
    _check("mla_append_latent_noalloc", lib.mla_append_latent_noalloc(
        w.handle, _ptr(h), _ptr(seq_idx), _ptr(pos), _ptr(page_table), num_seqs, max_pages, num_pages,
        _ptr(cache), T, _ptr(device_error), _stream(stream)))


def decode(w: Weights, h_q, kv_len, page_table, num_pages: int, cache, out, max_kv_len: int, workspace,
           stream=None):
    B, n_q = h_q.shape[0], h_q.shape[1]
    _check("mla_decode", lib.mla_decode(
        w.handle, _ptr(h_q), _ptr(kv_len), _ptr(page_table), page_table.shape[1], num_pages, _ptr(cache),
        _ptr(out), B, n_q, max_kv_len, _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))


def decode_step(w: Weights, h, kv_len, page_table, num_pages: int, cache, out, max_kv_len: int, workspace,
                stream=None):
    """Append the new tokens' latent rows, then decode them (one call)."""
    B, n_q = h.shape[0], h.shape[1]
    _check("mla_decode_step", lib.mla_decode_step(
        w.handle, _ptr(h), _ptr(kv_len), _ptr(page_table), page_table.shape[1], num_pages, _ptr(cache),
        _ptr(out), B, n_q, max_kv_len, _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))


def prefill(w: Weights, h, page_table, num_pages: int, cache, out, workspace, stream=None):
    B, S = h.shape[0], h.shape[1]
    _check("mla_prefill", lib.mla_prefill(
        w.handle, _ptr(h), _ptr(page_table), page_table.shape[1], num_pages, _ptr(cache), _ptr(out), B, S,
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def prefill_materialised_workspace_bytes(dims: Dims, B: int, S: int) -> int:
    return lib.mla_prefill_materialised_workspace_bytes(ctypes.byref(dims), B, S)


def prefill_materialised(w: Weights, h, page_table, num_pages: int, cache, out, workspace, stream=None):
    """Causal prefill through expanded per-head keys and values (include/mla.h)."""
    B, S = h.shape[0], h.shape[1]
    _check("mla_prefill_materialised", lib.mla_prefill_materialised(
        w.handle, _ptr(h), _ptr(page_table), page_table.shape[1], num_pages, _ptr(cache), _ptr(out), B, S,
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def decode_cp_workspace_bytes(dims: Dims, B: int, n_q: int) -> int:
    return lib.mla_decode_cp_workspace_bytes(ctypes.byref(dims), B, n_q)


def decode_cp_partial(w: Weights, h_q, kv_len, window_start, window_count, page_table, num_pages: int, cache,
                      obar_out, lse_out, max_kv_len: int, workspace, stream=None):
    """This rank's share of a context-parallel decode step (include/mla.h)."""
    B, n_q = h_q.shape[0], h_q.shape[1]
    _check("mla_decode_cp_partial", lib.mla_decode_cp_partial(
        w.handle, _ptr(h_q), _ptr(kv_len), _ptr(window_start), _ptr(window_count), _ptr(page_table),
        page_table.shape[1], num_pages, _ptr(cache), _ptr(obar_out), _ptr(lse_out), B, n_q, max_kv_len,
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def decode_cp_combine(w: Weights, obar_parts, lse_parts, out, workspace, stream=None):
    """Merges all ranks' partials [n_ranks, B, n_q, ...] into out [B, n_q, n_h, d_v]."""
    n_ranks, B, n_q = obar_parts.shape[0], obar_parts.shape[1], obar_parts.shape[2]
    _check("mla_decode_cp_combine", lib.mla_decode_cp_combine(
        w.handle, n_ranks, _ptr(obar_parts), _ptr(lse_parts), _ptr(out), B, n_q, _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def selftest_wait_timeout(workspace, limit_us: int, stream=None):
    """Test hook: a bounded wait that nothing satisfies (include/mla.h)."""
    _check("mla_selftest_wait_timeout", lib.mla_selftest_wait_timeout(_ptr(workspace), limit_us, _stream(stream)))


def get_error(workspace, stream=None) -> int:
    return lib.mla_get_error(_ptr(workspace), _stream(stream))


def status_string(code: int) -> str:
    return lib.mla_status_string(code).decode()
