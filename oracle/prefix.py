"""Associative (affine-map) evaluations of the selective recurrence, numpy.

TEST INFRASTRUCTURE ONLY (see the package docstring). These evaluate the same
recurrence as the sequential oracle by a different route, so the tests can pin
the oracle against the algebra rather than against itself.

Each step t is the affine map f_t(h) = a_t * h + w_t (elementwise over the
state), with a_t = exp(delta_t * A) and w_t = delta_t * B_t * x_t. Two maps
compose as (a2, w2) o (a1, w1) = (a2 * a1, a2 * w1 + w2): "later after
earlier". This is the algebra of the page "mamba, from scratch | khushi
keswani", section "the scan", and of the page "Mamba: Linear-Time Sequence
Modeling with Selective State Spaces" (www.abhik.ai/papers/mamba), section
"Compose the updates instead of waiting for every state" and row "3. Compose
chronological affine updates". The operation is associative but not
commutative, so every bracketing of the chronological product gives the same
map, and swapping two maps generally does not.
"""
from __future__ import annotations

import functools

import numpy as np


def _softplus_default(v):
    # PyTorch F.softplus defaults: identity above the threshold 20.
    v = np.asarray(v, dtype=np.float64)
    return np.where(v > 20.0, v, np.log1p(np.exp(np.minimum(v, 20.0))))


def affine_pairs(x, delta, A_log, B, delta_bias=None, delta_softplus=True):
    """Per-step maps: (a, w), each [b, L, E, N], float64."""
    x = np.asarray(x, dtype=np.float64)
    raw = np.asarray(delta, dtype=np.float64)
    if delta_bias is not None:
        raw = raw + np.asarray(delta_bias, dtype=np.float64)[None, None, :]
    step = _softplus_default(raw) if delta_softplus else raw
    A = -np.exp(np.asarray(A_log, dtype=np.float64))          # [E, N]
    Bf = np.asarray(B, dtype=np.float64)                        # [b, L, N]
    a = np.exp(step[..., None] * A[None, None, :, :])
    w = step[..., None] * Bf[:, :, None, :] * x[..., None]
    return a, w


def compose(later, earlier):
    """(a2, w2) o (a1, w1) = (a2 a1, a2 w1 + w2): apply earlier, then later."""
    a2, w2 = later
    a1, w1 = earlier
    return a2 * a1, a2 * w1 + w2


def hillis_steele_prefix(a, w, h0=None):
    """Inclusive prefix of the maps over axis 1 by snapshot rounds.

    Round r combines position t with position t - 2**r, reading only the
    previous round's arrays (a snapshot), so the dependency depth is
    ceil(log2 L). Returns every state [b, L, E, N] after applying the prefix
    map of each position to the incoming state h0 (zeros when None).
    """
    cur_a, cur_w = np.array(a, copy=True), np.array(w, copy=True)
    L = cur_a.shape[1]
    stride = 1
    while stride < L:
        prev_a, prev_w = cur_a, cur_w
        nxt_a, nxt_w = prev_a.copy(), prev_w.copy()
        na, nw = compose((prev_a[:, stride:], prev_w[:, stride:]),
                         (prev_a[:, :-stride], prev_w[:, :-stride]))
        nxt_a[:, stride:] = na
        nxt_w[:, stride:] = nw
        cur_a, cur_w = nxt_a, nxt_w
        stride *= 2
    if h0 is None:
        h0 = np.zeros((a.shape[0], a.shape[2], a.shape[3]))
    return cur_a * np.asarray(h0, dtype=np.float64)[:, None] + cur_w


def bracketings(lo, hi):
    """Every full binary bracketing of the maps lo..hi-1 (chronological).

    Yields nested tuples: an int is a single step, (left, right) means
    "left happens first, then right". There are Catalan(hi-lo-1) of them.
    """
    if hi - lo == 1:
        yield lo
        return
    for mid in range(lo + 1, hi):
        for left in bracketings(lo, mid):
            for right in bracketings(mid, hi):
                yield (left, right)


def evaluate_bracketing(tree, a, w):
    """Compose the maps of a bracketing tree; a, w are per-step arrays."""
    @functools.lru_cache(maxsize=None)
    def ev(node):
        if isinstance(node, int):
            return a[node], w[node]
        left, right = node
        return compose(ev(right), ev(left))
    return ev(tree)


def readout(states, x, C, D=None, z=None):
    """y = sum_n C[t, n] h[t, n] (+ D x) then * SiLU(z); [b, L, E]."""
    states = np.asarray(states, dtype=np.float64)
    xf = np.asarray(x, dtype=np.float64)
    y = np.einsum("blen,bln->ble", states, np.asarray(C, dtype=np.float64))
    if D is not None:
        y = y + np.asarray(D, dtype=np.float64)[None, None, :] * xf
    if z is not None:
        zf = np.asarray(z, dtype=np.float64)
        y = y * (zf / (1.0 + np.exp(-zf)))
    return y
