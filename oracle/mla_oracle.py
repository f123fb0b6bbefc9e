"""fp64 CPU oracle for multi-head latent attention with decoupled RoPE.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only the tests under ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may use it.  It
shares no code with the CUDA library (no kernels, headers, tables or helpers);
it takes plain NumPy arrays and computes in float64.

What it computes, and where the pages define it (pages are named by title and
section):

* Cache entries.  "ai-decoupled-rope-mla" (operatorworld), section on the
  decoupled RoPE solution: the latent is ``c_t = W_DKV h_t`` and the position
  key is ``k_R,t = W_KR h_t`` with RoPE applied.  "Latent Attention Meets RoPE"
  (sahipadhai), section "Two small, telling details": the position key is one
  vector shared by every head, and only the latent and that key are cached.
* Queries.  "Detailed Illustration of the Problem" (notion), Step 1: the query
  latent ``c^Q = W_DQ h`` and ``q = W_UQ c^Q``.  The decoupled-RoPE page gives
  the content query ``q^C`` and the position query ``q^R``, the latter rotated
  by the query's own position.
* Score.  Same decoupled-RoPE page, score equation: a content term plus a
  position term.  The scale is one shared factor ``1/sqrt(d_h + d_r)`` on both
  terms (the two pages disagree on the scale; this is the reading taken, and
  the scale is an argument).
* Output.  The materialised form of "Multi-Head Latent Attention"
  (talalahmed), section "Compress first, expand later": ``K^C = W_UK c`` and
  ``V = W_UV c`` are rebuilt per head and ordinary softmax attention is run.
  The absorbed form (decoupled-RoPE page, "absorption saves cache" equations:
  ``q~ = W_UK^T q`` and ``W_UV sum_t alpha_t c_t``) is provided separately as a
  self-check, never as the oracle's answer.
* Context-parallel decode (``window_partial``, ``merge_windows``,
  ``latent_output``).  The pages do not split a sequence over devices; these
  state the softmax-over-disjoint-key-sets identity a split relies on.
* Per-head position keys (``rope_per_head``).  The 16-head example of
  "Multi-Head Latent Attention" (talalahmed), section "A concrete size
  comparison", caches one 32-dim RoPE key per head instead of one shared key:
  ``k_R,h,t = RoPE_t(W_KR,h h_t)`` with ``W_KR`` then ``[n_h*d_r, D]`` (rows
  ``h*d_r ..`` for head ``h``), and head ``h``'s position term is
  ``q_R,h . k_R,h,t``.  Everything else is unchanged.
* RoPE.  Pairs ``(2i, 2i+1)`` rotated by angle ``pos * theta_i`` with
  ``theta_i = base^(-2i/d_r)``; the pages print only the rotation family and its
  relative property ``R_m^T R_t = R_{t-m}`` ("ai-decoupled-rope-mla", decoupled
  RoPE section; "Detailed Illustration of the Problem", Step 3), so the
  frequencies and the interleaved pairing are a reading (the RoFormer
  convention behind the pages' ``R_Theta`` notation).

Weight orientation is column-vector (``y = W x``): ``W_DKV`` is ``[d_c, D]``,
``W_KR`` ``[d_r, D]``, ``W_DQ`` ``[d_cq, D]``, ``W_UQ`` ``[n_h*d_h, d_in]``,
``W_QR`` ``[n_h*d_r, d_in]``, ``W_UK`` ``[n_h*d_h, d_c]``, ``W_UV``
``[n_h*d_v, d_c]`` where ``d_in = d_cq`` if a query latent exists, else ``D``.
Row ``h*d_h + i`` of ``W_UK`` belongs to head ``h``.

Parity status: every function here is pinned by a test under ``tests/``
(closed forms, invariants, a scalar brute force, a library attention routine);
none is "parity unpinned".
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np


# ----------------------------------------------------------------------------
# Dimensions and weights
# ----------------------------------------------------------------------------
@dataclass(frozen=True)
class Dims:
    n_h: int
    d_h: int
    d_v: int
    d_c: int
    d_r: int
    d_model: int
    d_cq: int = 0           # 0: the query is projected straight from h
    rope_base: float = 10000.0
    rope_per_head: bool = False  # one RoPE key per head (W_KR is [n_h*d_r, D]) instead of one shared

    @property
    def d_in(self) -> int:
        return self.d_cq if self.d_cq > 0 else self.d_model

    def default_scale(self) -> float:
        # One shared factor on both score terms (a reading; see module doc).
        return 1.0 / math.sqrt(self.d_h + self.d_r)


@dataclass
class Weights:
    W_DKV: np.ndarray
    W_KR: np.ndarray
    W_DQ: Optional[np.ndarray]
    W_UQ: np.ndarray
    W_QR: np.ndarray
    W_UK: np.ndarray
    W_UV: np.ndarray


def _f64(a):
    return None if a is None else np.asarray(a, dtype=np.float64)


def as_f64(w: Weights) -> Weights:
    return Weights(*(_f64(getattr(w, f)) for f in
                     ("W_DKV", "W_KR", "W_DQ", "W_UQ", "W_QR", "W_UK", "W_UV")))


# ----------------------------------------------------------------------------
# RoPE
# ----------------------------------------------------------------------------
def rope_frequencies(d_r: int, base: float) -> np.ndarray:
    """theta_i = base^(-2i/d_r), i = 0 .. d_r/2 - 1 (the reading taken for the
    frequencies the pages leave unprinted)."""
    assert d_r % 2 == 0
    i = np.arange(d_r // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * i / d_r)


def rope_rotation_matrix(pos: float, freqs: np.ndarray) -> np.ndarray:
    """The d_r x d_r block-diagonal rotation R_pos: block i is the 2x2 rotation
    by pos*theta_i acting on components (2i, 2i+1)."""
    d_r = 2 * len(freqs)
    R = np.zeros((d_r, d_r))
    for i, th in enumerate(freqs):
        a = float(pos) * float(th)
        c, s = math.cos(a), math.sin(a)
        R[2 * i, 2 * i] = c
        R[2 * i, 2 * i + 1] = -s
        R[2 * i + 1, 2 * i] = s
        R[2 * i + 1, 2 * i + 1] = c
    return R


def rope_apply(x: np.ndarray, pos: np.ndarray, freqs: np.ndarray) -> np.ndarray:
    """R_pos x for each vector in ``x[..., d_r]``; ``pos`` broadcasts against
    ``x.shape[:-1]``.  This is ``rope_rotation_matrix(pos) @ x`` written out per
    2x2 block, with the angle formed in fp64."""
    x = np.asarray(x, dtype=np.float64)
    pos = np.asarray(pos, dtype=np.float64)
    ang = pos[..., None] * freqs                     # [..., d_r/2]
    c, s = np.cos(ang), np.sin(ang)
    x0 = x[..., 0::2]
    x1 = x[..., 1::2]
    out = np.empty(np.broadcast_shapes(x.shape, ang.shape[:-1] + (x.shape[-1],)))
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


# ----------------------------------------------------------------------------
# Projections
# ----------------------------------------------------------------------------
def cache_entries(w: Weights, H: np.ndarray, pos: np.ndarray, freqs: np.ndarray):
    """The two cached quantities per token: the latent ``c_t = W_DKV h_t`` and
    the already rotated position key ``RoPE_t(W_KR h_t)``: one shared key
    ``[T, d_r]`` when ``W_KR`` has ``d_r`` rows, else one per head
    ``[T, n_h, d_r]`` (``W_KR`` with ``n_h*d_r`` rows, head ``h`` at rows
    ``h*d_r ..``)."""
    H = np.asarray(H, dtype=np.float64)
    c = H @ w.W_DKV.T
    d_r = 2 * len(freqs)
    k = H @ np.asarray(w.W_KR, np.float64).T
    if k.shape[1] == d_r:
        return c, rope_apply(k, pos, freqs)
    k = k.reshape(H.shape[0], k.shape[1] // d_r, d_r)
    return c, rope_apply(k, np.asarray(pos)[:, None], freqs)


def _position_term(q_r, k_r):
    """``q_R,h . k_R,t`` for every query, head and key: ``[Q, n_h, T]``; the key
    is shared ``[T, d_r]`` or per head ``[T, n_h, d_r]``."""
    if k_r.ndim == 2:
        return np.matmul(q_r, k_r.T)
    return np.einsum("qhr,thr->qht", q_r, k_r)


def queries(w: Weights, dims: Dims, H: np.ndarray, pos: np.ndarray, freqs: np.ndarray):
    """Content query ``q_C`` [T, n_h, d_h] and rotated position query ``q_R``
    [T, n_h, d_r].  With a query latent, both come from ``c_Q = W_DQ h``;
    without one, both come from ``h`` directly."""
    H = np.asarray(H, dtype=np.float64)
    src = H @ w.W_DQ.T if dims.d_cq > 0 else H
    T = H.shape[0]
    q_c = (src @ w.W_UQ.T).reshape(T, dims.n_h, dims.d_h)
    q_r_pre = (src @ w.W_QR.T).reshape(T, dims.n_h, dims.d_r)
    q_r = rope_apply(q_r_pre, np.asarray(pos)[:, None], freqs)
    return q_c, q_r


# ----------------------------------------------------------------------------
# Attention: materialised (the oracle) and absorbed (a self-check)
# ----------------------------------------------------------------------------
def _softmax(a: np.ndarray) -> np.ndarray:
    m = a.max(axis=-1, keepdims=True)
    e = np.exp(a - m)
    return e / e.sum(axis=-1, keepdims=True)


def attend_materialised(dims: Dims, w: Weights, q_c, q_r, c, k_r, q_pos, k_pos,
                        scale: float, head_chunk: int = 16) -> np.ndarray:
    """Materialised attention: rebuild ``K_C = W_UK,h c_t`` and
    ``V = W_UV,h c_t`` per head, score ``scale*(q_C.k_C + q_R.k_R)``, softmax
    over the keys whose position is <= the query's, and sum the values.

    q_c [Q, n_h, d_h], q_r [Q, n_h, d_r], c [T, d_c], k_r [T, d_r];
    returns o [Q, n_h, d_v].
    """
    n_h, d_h, d_v, d_c = dims.n_h, dims.d_h, dims.d_v, dims.d_c
    W_UK = w.W_UK.reshape(n_h, d_h, d_c)
    W_UV = w.W_UV.reshape(n_h, d_v, d_c)
    q_pos = np.asarray(q_pos)
    k_pos = np.asarray(k_pos)
    visible = k_pos[None, :] <= q_pos[:, None]                    # [Q, T]
    out = np.empty((q_c.shape[0], n_h, d_v))
    pos_term = _position_term(q_r, k_r)                           # [Q, n_h, T]
    for h0 in range(0, n_h, head_chunk):
        hs = slice(h0, min(n_h, h0 + head_chunk))
        k_c = np.matmul(c[None], W_UK[hs].transpose(0, 2, 1))     # [h, T, d_h]  (K_C = W_UK,h c_t)
        v = np.matmul(c[None], W_UV[hs].transpose(0, 2, 1))       # [h, T, d_v]  (V = W_UV,h c_t)
        content = np.matmul(q_c[:, hs].transpose(1, 0, 2), k_c.transpose(0, 2, 1))  # [h, Q, T]
        a = (content.transpose(1, 0, 2) + pos_term[:, hs]) * scale
        a = np.where(visible[:, None, :], a, -np.inf)
        alpha = _softmax(a)                                       # [Q, h, T]
        out[:, hs] = np.matmul(alpha.transpose(1, 0, 2), v).transpose(1, 0, 2)
    return out


def attend_absorbed(dims: Dims, w: Weights, q_c, q_r, c, k_r, q_pos, k_pos,
                    scale: float) -> np.ndarray:
    """Absorbed attention, used only to check the oracle: ``q~ = W_UK,h^T q_C``
    scores against the latent directly, the softmax-weighted latent sum
    ``o_bar = sum_t alpha_t c_t`` is formed, then ``o = W_UV,h o_bar``."""
    n_h, d_h, d_v, d_c = dims.n_h, dims.d_h, dims.d_v, dims.d_c
    W_UK = w.W_UK.reshape(n_h, d_h, d_c)
    W_UV = w.W_UV.reshape(n_h, d_v, d_c)
    q_abs = np.einsum("qhd,hdc->qhc", q_c, W_UK)
    a = (np.einsum("qhc,tc->qht", q_abs, c) + _position_term(q_r, k_r)) * scale
    visible = np.asarray(k_pos)[None, :] <= np.asarray(q_pos)[:, None]
    a = np.where(visible[:, None, :], a, -np.inf)
    alpha = _softmax(a)
    o_bar = np.einsum("qht,tc->qhc", alpha, c)
    return np.einsum("qhc,hvc->qhv", o_bar, W_UV)


# ----------------------------------------------------------------------------
# Whole-sequence entry points
# ----------------------------------------------------------------------------
def mla_sequence(dims: Dims, w: Weights, H: np.ndarray, query_rows: Sequence[int],
                 scale: Optional[float] = None, positions: Optional[np.ndarray] = None,
                 freqs: Optional[np.ndarray] = None, absorbed: bool = False) -> np.ndarray:
    """Attention outputs for the tokens ``query_rows`` of one sequence.

    ``H`` [T, D] holds the hidden states of every token of the sequence (cached
    ones and the queries); token ``t`` sits at ``positions[t]`` (default
    ``t``).  Each query attends to every token whose position is <= its own,
    itself included.  Returns o [len(query_rows), n_h, d_v].
    """
    w = as_f64(w)
    H = np.asarray(H, dtype=np.float64)
    T = H.shape[0]
    pos = np.arange(T, dtype=np.float64) if positions is None else np.asarray(positions, np.float64)
    freqs = rope_frequencies(dims.d_r, dims.rope_base) if freqs is None else freqs
    scale = dims.default_scale() if scale is None else scale
    rows = np.asarray(query_rows, dtype=np.int64)
    c, k_r = cache_entries(w, H, pos, freqs)
    q_c, q_r = queries(w, dims, H[rows], pos[rows], freqs)
    fn = attend_absorbed if absorbed else attend_materialised
    return fn(dims, w, q_c, q_r, c, k_r, pos[rows], pos, scale)


def mla_decode(dims: Dims, w: Weights, H: np.ndarray, n_q: int, **kw) -> np.ndarray:
    """Decode for one sequence of ``len(H)`` tokens whose last ``n_q`` tokens
    are the new queries (each appended to the cache before it attends)."""
    T = H.shape[0]
    return mla_sequence(dims, w, H, list(range(T - n_q, T)), **kw)


# ----------------------------------------------------------------------------
# Decode over a window of the keys (context-parallel split)
# ----------------------------------------------------------------------------
# The pages never split one sequence's keys across devices.  What such a split
# needs is the plain identity for a softmax over a union of disjoint key sets:
# with Z_j = sum over set j of exp(a_t), the full softmax-weighted latent sum is
# sum_j (Z_j / sum_k Z_k) * (the softmax-weighted latent sum over set j).  The
# functions below state it in base 2 (log2 Z_j), the form the library
# exchanges between ranks.
def window_partial(dims: Dims, w: Weights, H: np.ndarray, n_q: int, start: int, count: int,
                   scale: Optional[float] = None):
    """One window's share of a decode step of one sequence.

    ``H`` [T, D] holds every token of the sequence; the last ``n_q`` are the
    new queries at positions T-n_q .. T-1.  Keys are limited to positions
    ``[start, start + count)`` and, per query, to positions <= its own.
    Returns ``(o_bar [n_q, n_h, d_c], lse2 [n_q, n_h])``: the softmax-weighted
    latent sum over those keys (scores against the latent with the absorbed
    query ``q~ = W_UK,h^T q_C``) and ``log2 sum_t exp(a_t)``.  A query with no
    such key gets ``o_bar = 0`` and ``lse2 = -inf``."""
    assert not dims.rope_per_head, "window partials are stated for the shared position key"
    w = as_f64(w)
    H = np.asarray(H, dtype=np.float64)
    T = H.shape[0]
    n_h, d_h, d_c = dims.n_h, dims.d_h, dims.d_c
    scale = dims.default_scale() if scale is None else scale
    freqs = rope_frequencies(dims.d_r, dims.rope_base)
    pos = np.arange(T, dtype=np.float64)
    rows = np.arange(T - n_q, T)
    keys = np.arange(max(0, start), min(T, start + count))
    o_bar = np.zeros((n_q, n_h, d_c))
    lse2 = np.full((n_q, n_h), -np.inf)
    if keys.size == 0:
        return o_bar, lse2
    c, k_r = cache_entries(w, H[keys], pos[keys], freqs)
    q_c, q_r = queries(w, dims, H[rows], pos[rows], freqs)
    q_abs = np.einsum("qhd,hdc->qhc", q_c, w.W_UK.reshape(n_h, d_h, d_c))
    a = (np.einsum("qhc,tc->qht", q_abs, c) + np.einsum("qhr,tr->qht", q_r, k_r)) * scale
    visible = keys[None, :] <= rows[:, None]                      # [Q, K]
    for qi in range(n_q):
        if not visible[qi].any():
            continue
        aq = a[qi][:, visible[qi]]                                 # [n_h, K']
        m = aq.max(axis=1, keepdims=True)
        e = np.exp(aq - m)
        z = e.sum(axis=1)
        o_bar[qi] = (e @ c[visible[qi]]) / z[:, None]
        lse2[qi] = (m[:, 0] + np.log(z)) / math.log(2.0)
    return o_bar, lse2


def merge_windows(parts):
    """Merges window partials ``[(o_bar_j, lse2_j), ...]`` of the same queries
    into the latent sum over the union of the windows: weights
    ``2^(lse2_j - L)`` with ``L = log2 sum_j 2^lse2_j`` (windows with
    ``lse2 = -inf`` weigh nothing)."""
    lse = np.stack([p[1] for p in parts])                         # [J, Q, n_h]
    L = np.log2(np.sum(np.exp2(lse - lse.max(axis=0)), axis=0)) + lse.max(axis=0)
    wts = np.exp2(lse - L)                                        # [J, Q, n_h]
    return sum(wts[j][..., None] * parts[j][0] for j in range(len(parts)))


def latent_output(dims: Dims, w: Weights, o_bar: np.ndarray) -> np.ndarray:
    """``o_h = W_UV,h o_bar_h`` for o_bar [Q, n_h, d_c]; returns [Q, n_h, d_v]."""
    W_UV = np.asarray(w.W_UV, np.float64).reshape(dims.n_h, dims.d_v, dims.d_c)
    return np.einsum("qhc,hvc->qhv", np.asarray(o_bar, np.float64), W_UV)


# ----------------------------------------------------------------------------
# Pure-Python scalar brute force (tiny sizes only)
# ----------------------------------------------------------------------------
def brute_force_sequence(dims: Dims, w: Weights, H, query_rows, scale=None):
    """The same definition as ``mla_sequence`` in scalar Python loops with no
    NumPy arithmetic, indexing the weights element by element."""
    n_h, d_h, d_v, d_c, d_r, D = dims.n_h, dims.d_h, dims.d_v, dims.d_c, dims.d_r, dims.d_model
    scale = 1.0 / math.sqrt(d_h + d_r) if scale is None else scale
    Wl = {k: (None if getattr(w, k) is None else np.asarray(getattr(w, k), np.float64).tolist())
          for k in ("W_DKV", "W_KR", "W_DQ", "W_UQ", "W_QR", "W_UK", "W_UV")}
    Hl = np.asarray(H, np.float64).tolist()
    T = len(Hl)
    theta = [float(dims.rope_base) ** (-2.0 * i / d_r) for i in range(d_r // 2)]

    def matvec(W, x):
        return [sum(W[r][k] * x[k] for k in range(len(x))) for r in range(len(W))]

    def rot(x, p):
        y = list(x)
        for i in range(d_r // 2):
            a = p * theta[i]
            y[2 * i] = x[2 * i] * math.cos(a) - x[2 * i + 1] * math.sin(a)
            y[2 * i + 1] = x[2 * i] * math.sin(a) + x[2 * i + 1] * math.cos(a)
        return y

    c = [matvec(Wl["W_DKV"], Hl[t]) for t in range(T)]
    kr_all = [matvec(Wl["W_KR"], Hl[t]) for t in range(T)]

    def key(t, h):
        """Head h's rotated position key of token t (shared or its own)."""
        base = h * d_r if dims.rope_per_head else 0
        return rot(kr_all[t][base:base + d_r], t)
    out = []
    for m in query_rows:
        src = matvec(Wl["W_DQ"], Hl[m]) if dims.d_cq > 0 else Hl[m]
        qc_all = matvec(Wl["W_UQ"], src)
        qr_all = matvec(Wl["W_QR"], src)
        per_head = []
        for h in range(n_h):
            qc = qc_all[h * d_h:(h + 1) * d_h]
            qr = rot(qr_all[h * d_r:(h + 1) * d_r], m)
            scores, vals = [], []
            for t in range(m + 1):
                kc = [sum(Wl["W_UK"][h * d_h + i][j] * c[t][j] for j in range(d_c)) for i in range(d_h)]
                v = [sum(Wl["W_UV"][h * d_v + i][j] * c[t][j] for j in range(d_c)) for i in range(d_v)]
                kr = key(t, h)
                s = sum(qc[i] * kc[i] for i in range(d_h)) + sum(qr[i] * kr[i] for i in range(d_r))
                scores.append(s * scale)
                vals.append(v)
            mx = max(scores)
            e = [math.exp(s - mx) for s in scores]
            z = sum(e)
            per_head.append([sum(e[t] * vals[t][i] for t in range(len(e))) / z for i in range(d_v)])
        out.append(per_head)
    return np.asarray(out)


# ----------------------------------------------------------------------------
# Per-token cache size arithmetic
# ----------------------------------------------------------------------------
def cache_numbers_per_token(n_h: int, d_h: int, d_v: int, d_c: int, d_r: int,
                            shared_rope_key: bool = True):
    """Numbers stored per token and layer: (multi-head attention, latent cache).

    Multi-head attention stores a key and a value per head.  The latent cache
    stores the latent plus the RoPE key: one shared key, or one per head in the
    per-head variant of the 16-head example in "Multi-Head Latent Attention",
    section "A concrete size comparison"."""
    mha = n_h * d_h + n_h * d_v
    mla = d_c + (d_r if shared_rope_key else n_h * d_r)
    return mha, mla
