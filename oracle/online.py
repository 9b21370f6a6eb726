"""Tiled online-softmax attention and its associative merge, float64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

This is the running-state form of "Online softmax: divide once, at the end"
in the FlashAttention case-study slides (nmj0.github.io): for each tile of keys,

    m_new = max(m, max_tile s),   alpha = exp(m - m_new),
    l     = alpha * l + sum_tile exp(s - m_new),
    o     = alpha * o + sum_tile exp(s - m_new) v,

and after the last tile O = o / l.  ``merge`` is the same update written as a
binary operator on states (m, l, o), the "secretly associative" operation of
the digest "Mastering FlashAttention: The Algebraic Foundation" (setupai.cc),
with identity (-inf, 0, 0).  The one guard the pages do not print: when both
maxima are -inf (nothing visible yet) the rescale factor is taken as 0 rather
than exp(-inf - (-inf)).

Used only to pin the two-pass oracle: the result must not depend on how the
keys are cut into tiles nor on the order the tiles are visited.
"""
from __future__ import annotations

import numpy as np

NEG_INF = -np.inf


def _scores(q, k, key_bias_row, causal, scale, Nq, Nk):
    """S = scale * Q K^T + mask for one head (Nq x Nk), float64."""
    s = scale * (q @ k.T)
    if key_bias_row is not None:
        s = s + key_bias_row[None, :]
    if causal:
        i = np.arange(Nq)[:, None]
        j = np.arange(Nk)[None, :]
        s = np.where(j <= i + (Nk - Nq), s, NEG_INF)
    return s


def _rescale(m_old, m_new):
    """exp(m_old - m_new), with 0 where m_old is -inf (nothing seen yet)."""
    out = np.zeros_like(m_old)
    ok = m_old != NEG_INF
    out[ok] = np.exp(m_old[ok] - m_new[ok])
    return out


def identity_state(rows, D):
    return (np.full(rows, NEG_INF), np.zeros(rows), np.zeros((rows, D)))


def tile_state(s_tile, v_tile):
    """State (m, l, o) of one tile of scores s_tile [rows, t] and values [t, D]."""
    m = s_tile.max(axis=1) if s_tile.shape[1] else np.full(s_tile.shape[0], NEG_INF)
    m_safe = np.where(m == NEG_INF, 0.0, m)
    e = np.exp(s_tile - m_safe[:, None])        # exp(-inf) = 0 on masked entries
    return m, e.sum(axis=1), e @ v_tile


def merge(a, b):
    """(m_a, l_a, o_a) (+) (m_b, l_b, o_b): the associative softmax merge."""
    m_a, l_a, o_a = a
    m_b, l_b, o_b = b
    m = np.maximum(m_a, m_b)
    ca = _rescale(m_a, m)
    cb = _rescale(m_b, m)
    return m, ca * l_a + cb * l_b, ca[:, None] * o_a + cb[:, None] * o_b


def online_update(state, s_tile, v_tile):
    """One step of the slides' running update (m, l, o) <- tile."""
    m, l, o = state
    m_tile = s_tile.max(axis=1) if s_tile.shape[1] else np.full(m.shape, NEG_INF)
    m_new = np.maximum(m, m_tile)
    alpha = _rescale(m, m_new)
    m_use = np.where(m_new == NEG_INF, 0.0, m_new)
    e = np.exp(s_tile - m_use[:, None])
    return m_new, alpha * l + e.sum(axis=1), alpha[:, None] * o + e @ v_tile


def finish(state):
    """O = o / l and LSE = m + ln l; rows with l = 0 give O = 0, LSE = -inf."""
    m, l, o = state
    ok = l > 0
    out = np.zeros_like(o)
    out[ok] = o[ok] / l[ok, None]
    lse = np.full(m.shape, NEG_INF)
    lse[ok] = m[ok] + np.log(l[ok])
    return out, lse


def fwd_online(q, k, v, key_bias=None, causal=False, scale=None,
               tile_sizes=None, order=None):
    """Attention of one head by the online update over key tiles.

    q [Nq,D], k/v [Nk,D], key_bias [Nk] or None.  ``tile_sizes`` cut the keys
    into consecutive tiles (default: one tile); ``order`` is the order in which
    those tiles are visited (default: ascending).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    Nq, D = q.shape
    Nk = k.shape[0]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    s = _scores(q, k, None if key_bias is None else np.asarray(key_bias, np.float64),
                causal, scale, Nq, Nk)
    if tile_sizes is None:
        tile_sizes = [Nk]
    assert sum(tile_sizes) == Nk
    bounds = np.cumsum([0] + list(tile_sizes))
    tiles = [(bounds[t], bounds[t + 1]) for t in range(len(tile_sizes))]
    if order is None:
        order = range(len(tiles))
    state = identity_state(Nq, D)
    for t in order:
        a, b = tiles[t]
        state = online_update(state, s[:, a:b], v[a:b])
    return finish(state)
