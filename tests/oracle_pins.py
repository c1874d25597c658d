"""Pins for the float64 oracle: facts the pages and the mathematics fix.

Each ``pin_*`` function takes an oracle object (``oracle.OracleLib`` or the
module ``oracle`` itself: anything with ``scan``, ``step_size`` and
``retention``) and raises AssertionError when the oracle disagrees with the
fact. ``test_oracle_pins.py`` runs them on the real oracle;
``test_oracle_mutants.py`` runs them on copies of the oracle with planted
mistakes and requires each mistake to be caught.

Pages cited:
  [abhik]   "Mamba: Linear-Time Sequence Modeling with Selective State Spaces"
            (www.abhik.ai/papers/mamba)
  [keswani] "mamba, from scratch | khushi keswani"
            (khushikeswani.vercel.app/work/mamba)
  [nadeem]  "Mamba: Linear-Time Sequence Modeling with Selective State Spaces"
            (nadeemcite.github.io/research-papers/100_mamba-...), the summary
  [s4]      the sailikhithk/mamba-from-scratch README (S4 section)
"""
from __future__ import annotations

import math
import os

import numpy as np

from oracle import prefix as P

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden_rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f
                if ln.strip() and not ln.lstrip().startswith("#")]


def incoming_memory():
    """[abhik] "A small state has to choose what survives": h0 of the demo."""
    return np.array([float(v) for v in _golden_rows(
        "abhik_incoming_memory.txt")[0]])


def tolerance(dtype="float64"):
    """[abhik] "Original paper, equations and runnable CPU code": the
    self-check's (atol, rtol)."""
    for row in _golden_rows("abhik_selfcheck_tolerances.txt"):
        if row[0] == dtype:
            return float(row[1]), float(row[2])
    raise KeyError(dtype)


def toy_steps():
    """[keswani] "the scan": length of the sequential-vs-prefix toy run."""
    for row in _golden_rows("keswani_toy_scan.txt"):
        if row[0] == "steps":
            return int(row[1])
    raise KeyError("steps")


def random_case(seed, b, L, E, N, gate=True, D=True, bias=True, h0=True):
    rng = np.random.default_rng(seed)
    case = dict(
        x=rng.standard_normal((b, L, E)),
        delta=rng.normal(0.0, 0.7, (b, L, E)),
        A_log=rng.normal(0.0, 0.6, (E, N)),
        B=rng.standard_normal((b, L, N)),
        C=rng.standard_normal((b, L, N)),
        D=rng.standard_normal(E) if D else None,
        z=rng.standard_normal((b, L, E)) if gate else None,
        delta_bias=rng.normal(-0.5, 0.5, E) if bias else None,
        h0=rng.standard_normal((b, E, N)) if h0 else None,
    )
    return case


def _softplus(v):
    # log(1 + e^v) written out, for the test side's closed forms
    # (the cases here keep v well below the identity threshold 20).
    return np.log1p(np.exp(v))


def _close(actual, expected, atol, rtol, what):
    actual = np.asarray(actual, dtype=np.float64)
    expected = np.asarray(expected, dtype=np.float64)
    assert actual.shape == expected.shape, (what, actual.shape,
                                            expected.shape)
    ok = np.abs(actual - expected) <= atol + rtol * np.abs(expected)
    if not np.all(ok):
        i = np.unravel_index(np.argmax(~ok), ok.shape)
        raise AssertionError("%s: mismatch at %s: %r vs %r" % (
            what, i, actual[i], expected[i]))


def _scaled_close(actual, expected, scale, rel, what):
    """|actual - expected| <= rel * scale, elementwise (scale >= 0)."""
    err = np.abs(np.asarray(actual) - np.asarray(expected))
    bad = err > rel * np.asarray(scale) + 1e-300
    if np.any(bad):
        i = np.unravel_index(np.argmax(bad), bad.shape)
        raise AssertionError("%s: mismatch at %s: %r vs %r (scale %r)" % (
            what, i, np.asarray(actual)[i], np.asarray(expected)[i],
            np.asarray(scale)[i]))


# ---------------------------------------------------------------- pin 1
def pin_associative_prefix(o):
    """Sequential states equal the associative-prefix states.

    [keswani] "the scan" and [abhik] "Compose the updates instead of waiting
    for every state" / "3. Compose chronological affine updates": steps are
    affine maps composed by (a2,w2)o(a1,w1) = (a2 a1, a2 w1 + w2), which is
    associative, so (i) the snapshot Hillis-Steele prefix and (ii) every
    bracketing of each chronological prefix give the sequential states.
    Compared at the page's float64 self-check tolerance.
    """
    atol, rtol = tolerance("float64")
    cases = [
        # the page's demo: one channel, three state coordinates, six inputs,
        # with its printed incoming memory
        (dict(random_case(11, 1, 6, 1, 3), h0=incoming_memory()[None, None, :]),
         True),
        # the length of the toy run on [keswani]
        (random_case(12, 1, toy_steps(), 2, 2), True),
        (random_case(13, 2, 7, 3, 4), True),
        (random_case(14, 2, 7, 2, 3, gate=False, D=False, bias=False,
                     h0=False), False),
    ]
    for case, softplus in cases:
        y, h_last, states = o.scan(**case, delta_softplus=softplus,
                                   return_states=True)
        a, w = P.affine_pairs(case["x"], case["delta"], case["A_log"],
                              case["B"], case["delta_bias"], softplus)
        h0 = case["h0"]
        hs = P.hillis_steele_prefix(a, w, h0)
        _close(states, hs, atol, rtol, "states vs Hillis-Steele prefix")
        _close(h_last, hs[:, -1], atol, rtol, "h_last vs prefix")
        y_ref = P.readout(hs, case["x"], case["C"], case["D"], case["z"])
        _close(y, y_ref, atol, rtol, "y vs prefix readout")
        # every bracketing of every chronological prefix
        L = a.shape[1]
        a_t = [a[:, t] for t in range(L)]
        w_t = [w[:, t] for t in range(L)]
        h0v = np.zeros_like(a_t[0]) if h0 is None else np.asarray(h0)
        for m in range(1, L + 1):
            for tree in P.bracketings(0, m):
                am, wm = P.evaluate_bracketing(tree, a_t, w_t)
                _close(states[:, m - 1], am * h0v + wm, atol, rtol,
                       "state %d vs bracketing %r" % (m - 1, tree))


# ---------------------------------------------------------------- pin 2
def pin_lti_convolution(o):
    """Constant step and constant B, C reduce the scan to a convolution.

    [s4] (recurrent and convolutional views agree) and [abhik] "The input
    changes the coefficients, while A stays learned" (fixed coefficients
    unroll into a fixed convolution kernel): with a = exp(delta A) fixed,
        y_k = sum_{j<=k} K_j x_{k-j} + D x_k + sum_n C_n a_n^(k+1) h0_n,
        K_j = sum_n C_n a_n^j delta B_n,
    then the gate multiplies elementwise.
    """
    rng = np.random.default_rng(21)
    b, L, E, N = 2, 40, 3, 5
    raw_e = rng.normal(-1.0, 0.5, E)
    bias = rng.normal(0.0, 0.3, E)
    delta = np.broadcast_to(raw_e, (b, L, E)).copy()
    Bc = rng.standard_normal((b, N))
    Cc = rng.standard_normal((b, N))
    case = dict(
        x=rng.standard_normal((b, L, E)), delta=delta,
        A_log=rng.normal(0.0, 0.6, (E, N)),
        B=np.repeat(Bc[:, None, :], L, axis=1),
        C=np.repeat(Cc[:, None, :], L, axis=1),
        D=rng.standard_normal(E), z=rng.standard_normal((b, L, E)),
        delta_bias=bias, h0=rng.standard_normal((b, E, N)))
    y, h_last = o.scan(**case, delta_softplus=True)

    step = _softplus(raw_e + bias)                          # [E]
    a = np.exp(step[:, None] * -np.exp(case["A_log"]))      # [E, N]
    x, D, z, h0 = case["x"], case["D"], case["z"], case["h0"]
    expect = np.zeros((b, L, E))
    scale = np.zeros((b, L, E))
    h_expect = np.zeros((b, E, N))
    for bb in range(b):
        for e in range(E):
            powers = a[e][None, :] ** np.arange(L + 1)[:, None]    # [L+1, N]
            K = (powers[:L] * (Cc[bb] * step[e] * Bc[bb])[None, :]).sum(1)
            Kabs = (powers[:L] * np.abs(Cc[bb] * step[e] * Bc[bb])).sum(1)
            for k in range(L):
                conv = np.dot(K[:k + 1], x[bb, k::-1, e])
                free = np.dot(Cc[bb] * powers[k + 1], h0[bb, e])
                pre = conv + D[e] * x[bb, k, e] + free
                g = z[bb, k, e] / (1.0 + math.exp(-z[bb, k, e]))
                expect[bb, k, e] = pre * g
                scale[bb, k, e] = abs(g) * (
                    np.dot(Kabs[:k + 1], np.abs(x[bb, k::-1, e]))
                    + abs(D[e] * x[bb, k, e])
                    + np.dot(np.abs(Cc[bb]) * powers[k + 1],
                             np.abs(h0[bb, e])))
            # final state: sum_j a^j delta B x_{L-1-j} + a^L h0
            h_expect[bb, e] = (powers[:L] * step[e] * Bc[bb][None, :]
                               * x[bb, ::-1, e][:, None]).sum(0) \
                + powers[L] * h0[bb, e]
    _scaled_close(y, expect, scale + 1e-300, 1e-12, "y vs LTI convolution")
    _close(h_last, h_expect, 1e-12, 1e-10, "h_last vs LTI closed form")


# ---------------------------------------------------------------- pin 3
def pin_forgetting(o):
    """A very negative A forgets everything but the current write.

    [nadeem] "Core Idea" (a large step resets the state and focuses on the
    current input) and [abhik] "The input changes the coefficients": with
    A_log = 50, a = exp(delta A) underflows to exactly 0, so
    h_t = delta_t B_t x_t and y_t = delta_t x_t sum_n C_t B_t + D x_t, gated;
    the incoming state has no effect at all.
    """
    case = random_case(31, 2, 9, 3, 4)
    case["A_log"] = np.full_like(case["A_log"], 50.0)
    y, h_last = o.scan(**case, delta_softplus=True)
    y0, h_last0 = o.scan(**dict(case, h0=None), delta_softplus=True)
    assert np.array_equal(y, y0) and np.array_equal(h_last, h_last0), \
        "incoming state leaked through a fully forgetting scan"
    step = _softplus(case["delta"] + case["delta_bias"][None, None, :])
    x, B, C, D, z = (case[k] for k in ("x", "B", "C", "D", "z"))
    cb = (C * B).sum(-1)[:, :, None]
    cb_abs = np.abs(C * B).sum(-1)[:, :, None]
    g = z / (1.0 + np.exp(-z))
    expect = (step * x * cb + D * x) * g
    scale = (np.abs(step * x) * cb_abs + np.abs(D * x)) * np.abs(g)
    _scaled_close(y, expect, scale, 1e-13, "y vs forgetting closed form")
    last_w = step[:, -1, :, None] * B[:, -1, None, :] * x[:, -1, :, None]
    _close(h_last, last_w, 0.0, 1e-14, "h_last vs last write")


# ---------------------------------------------------------------- pin 4
def pin_freezing(o):
    """A zero step freezes the state.

    [nadeem] "Core Idea" (a small step keeps the state and ignores the input):
    delta = 0 exactly gives a = 1 and a zero write, so every state equals h0
    bitwise and y_t = sum_n C_t h0 + D x_t. With softplus on and raw = -60 the
    step is ~1e-26 and the state moves by less than 1e-20.
    """
    case = random_case(41, 2, 11, 3, 4, gate=False, bias=False)
    case["delta"] = np.zeros_like(case["delta"])
    y, h_last, states = o.scan(**case, delta_softplus=False,
                               return_states=True)
    assert np.array_equal(h_last, case["h0"]), "state moved with zero step"
    assert np.array_equal(states, np.broadcast_to(
        case["h0"][:, None], states.shape)), "a state moved with zero step"
    expect = np.einsum("bln,ben->ble", case["C"], case["h0"]) \
        + case["D"] * case["x"]
    scale = np.einsum("bln,ben->ble", np.abs(case["C"]), np.abs(case["h0"])) \
        + np.abs(case["D"] * case["x"])
    _scaled_close(y, expect, scale, 1e-14, "y with frozen state")
    case2 = dict(case, delta=np.full_like(case["delta"], -60.0))
    _, h_last2 = o.scan(**case2, delta_softplus=True)
    assert np.max(np.abs(h_last2 - case["h0"])) <= 1e-20, \
        "state moved with softplus(-60) step"


# ---------------------------------------------------------------- pin 5
def pin_retention_bounds(o):
    """0 <= a <= 1, and 0 < a < 1 for moderate delta * A.

    [abhik] "The input changes the coefficients, while A stays learned": A is
    negative and delta positive, so each retention lies between zero and one.
    In floating point the ends are reachable (underflow, rounding to 1); the
    strict bounds are checked where delta * A is in [-700, -1e-15]. Checked on
    the retention function and through the scan itself (B = 0, h0 = 1: the
    states are the running products of retentions).
    """
    for step in (0.0, 1e-300, 1e-15, 1e-6, 1e-3, 0.1, 1.0, 7.0, 1e3):
        for a_log in (-50.0, -5.0, -1.0, 0.0, 1.5, 3.0, 6.5, 50.0):
            r = o.retention(step, a_log)
            assert 0.0 <= r <= 1.0, (step, a_log, r)
            arg = step * -math.exp(a_log)
            if -700.0 <= arg <= -1e-15:
                assert 0.0 < r < 1.0, (step, a_log, r)
            assert abs(r - math.exp(arg)) <= 1e-15 * max(r, 1e-300) + 1e-300
    case = random_case(51, 2, 25, 3, 6, gate=False, D=False)
    case["B"] = np.zeros_like(case["B"])
    case["h0"] = np.ones_like(case["h0"])
    _, _, states = o.scan(**case, delta_softplus=True, return_states=True)
    assert np.all(states >= 0.0) and np.all(states <= 1.0)
    assert np.all(states[:, 0] < 1.0)
    assert np.all(np.diff(states, axis=1) <= 0.0), "a retention exceeded 1"


# ---------------------------------------------------------------- pin 6
def pin_continuation(o):
    """Processing a prefix, then the rest from its final state, is the same.

    [abhik] "2. Retain, write and read each channel's state" (an optional
    incoming state describes continuation from an earlier prefix) and "The
    selective operator is one part of the Mamba block" (full-sequence and
    token-at-a-time results agree). The sequential oracle must agree bitwise.
    """
    for seed, N, h0 in ((61, 5, None), (62, 3, "demo")):
        case = random_case(seed, 2, 37, 3, N, h0=False)
        if h0 == "demo":
            case["h0"] = np.broadcast_to(incoming_memory(), (2, 3, 3)).copy()
        y, h_last = o.scan(**case, delta_softplus=True)
        for m in (1, 5, 16, 17, 36):
            head = {k: (v[:, :m] if k in ("x", "delta", "z", "B", "C")
                        and v is not None else v) for k, v in case.items()}
            tail = {k: (v[:, m:] if k in ("x", "delta", "z", "B", "C")
                        and v is not None else v) for k, v in case.items()}
            y1, h1 = o.scan(**head, delta_softplus=True)
            tail["h0"] = h1
            y2, h2 = o.scan(**tail, delta_softplus=True)
            assert np.array_equal(np.concatenate([y1, y2], 1), y), m
            assert np.array_equal(h2, h_last), m
        # token at a time
        h = case["h0"]
        for t in range(37):
            one = {k: (v[:, t:t + 1] if k in ("x", "delta", "z", "B", "C")
                       and v is not None else v) for k, v in case.items()}
            one["h0"] = h
            yt, h = o.scan(**one, delta_softplus=True)
            assert np.array_equal(yt[:, 0], y[:, t]), t
        assert np.array_equal(h, h_last)


# ---------------------------------------------------------------- pin 7
def pin_decode_step(o):
    """L = 1 is the decode step.

    [abhik] "6. Carry both buffers to the next token": one token updates the
    [b, E, N] state as exp(delta A) * state + delta B x, reads
    (state * C).sum + D x, and the gate multiplies by SiLU(z).
    """
    case = random_case(71, 3, 1, 4, 5)
    y, h_last = o.scan(**case, delta_softplus=True)
    step = _softplus(case["delta"][:, 0] + case["delta_bias"])      # [b, E]
    A = -np.exp(case["A_log"])
    state = np.exp(step[..., None] * A) * case["h0"] \
        + step[..., None] * case["B"][:, 0, None, :] * case["x"][:, 0, :, None]
    read = (state * case["C"][:, 0, None, :]).sum(-1) \
        + case["D"] * case["x"][:, 0]
    zz = case["z"][:, 0]
    out = read * zz / (1.0 + np.exp(-zz))
    _close(h_last, state, 1e-15, 1e-13, "decode state")
    _close(y[:, 0], out, 1e-14, 1e-12, "decode output")


# ---------------------------------------------------------------- pin 8
def pin_linearity(o):
    """For fixed steps and B, C the ungated scan is linear in (x, h0).

    [abhik] "2. Retain, write and read each channel's state": the state
    update and readout are linear in the state and the input once delta,
    B and C are fixed (here delta is given directly, softplus off).
    """
    rng = np.random.default_rng(81)
    b, L, E, N = 2, 19, 3, 4
    base = random_case(82, b, L, E, N, gate=False)
    base["delta"] = np.abs(base["delta"]) + 0.01
    base["delta_bias"] = None
    x1, x2 = rng.standard_normal((2, b, L, E))
    g1, g2 = rng.standard_normal((2, b, E, N))
    al, be = 0.75, -1.25
    ya, ha = o.scan(**dict(base, x=x1, h0=g1), delta_softplus=False)
    yb, hb = o.scan(**dict(base, x=x2, h0=g2), delta_softplus=False)
    yc, hc = o.scan(**dict(base, x=al * x1 + be * x2, h0=al * g1 + be * g2),
                    delta_softplus=False)
    scale_y = np.abs(al * ya) + np.abs(be * yb) + 1.0
    _scaled_close(yc, al * ya + be * yb, scale_y, 1e-12, "linearity y")
    scale_h = np.abs(al * ha) + np.abs(be * hb) + 1.0
    _scaled_close(hc, al * ha + be * hb, scale_h, 1e-12, "linearity h")


# ---------------------------------------------------------------- pin 9
def pin_independence(o):
    """Channels and batches never interact.

    [abhik] "The input changes the coefficients": A is per channel, B and C
    are shared across the expanded channels, the state is [b, E, N]. So
    permuting channels (with their A_log, D, bias, steps, x, z, h0) permutes
    the outputs, and changing one batch leaves the others untouched.
    """
    case = random_case(91, 3, 13, 5, 4)
    y, h = o.scan(**case, delta_softplus=True)
    perm = np.array([3, 0, 4, 1, 2])
    pc = dict(case)
    for k in ("x", "delta", "z"):
        pc[k] = case[k][..., perm]
    pc["A_log"] = case["A_log"][perm]
    pc["D"] = case["D"][perm]
    pc["delta_bias"] = case["delta_bias"][perm]
    pc["h0"] = case["h0"][:, perm]
    yp, hp = o.scan(**pc, delta_softplus=True)
    assert np.array_equal(yp, y[..., perm]), "channel permutation"
    assert np.array_equal(hp, h[:, perm]), "channel permutation (state)"
    other = random_case(92, 3, 13, 5, 4)
    mixed = {k: (None if v is None else v.copy()) for k, v in case.items()}
    for k in ("x", "delta", "z", "B", "C", "h0"):
        mixed[k][1] = other[k][1]
    ym, hm = o.scan(**mixed, delta_softplus=True)
    for bb in (0, 2):
        assert np.array_equal(ym[bb], y[bb]), "batch %d changed" % bb
        assert np.array_equal(hm[bb], h[bb]), "batch %d state changed" % bb
    assert not np.array_equal(ym[1], y[1])


# ---------------------------------------------------------------- pin 10
def pin_degenerate(o):
    """Zero write or zero readout leaves only the direct path; gate limits.

    [abhik] "2. Retain, write and read each channel's state" and "The
    selective operator is one part of the Mamba block" (D x is a direct path
    inside the scan output; the z branch multiplies through SiLU): B = 0 with
    a zero incoming state, or C = 0, gives y = D x * SiLU(z); D absent equals
    D = 0; z = 0 gives exactly 0; the gate scales by z / (1 + exp(-z)).
    """
    case = random_case(101, 2, 12, 3, 4, h0=False)
    x, D, z = case["x"], case["D"], case["z"]
    g = z / (1.0 + np.exp(-z))
    yB, _ = o.scan(**dict(case, B=np.zeros_like(case["B"])))
    _close(yB, D * x * g, 0.0, 1e-15, "B = 0")
    yC, _ = o.scan(**dict(case, C=np.zeros_like(case["C"]),
                          h0=np.ones((2, 3, 4))))
    _close(yC, D * x * g, 0.0, 1e-15, "C = 0")
    yN, hN = o.scan(**dict(case, D=None))
    yZ, hZ = o.scan(**dict(case, D=np.zeros(3)))
    assert np.array_equal(yN, yZ) and np.array_equal(hN, hZ), "D absent"
    y0, _ = o.scan(**dict(case, z=np.zeros_like(z)))
    assert np.all(y0 == 0.0), "z = 0 must zero the output"
    yu, hu = o.scan(**dict(case, z=None))
    yg, hg = o.scan(**case)
    assert np.array_equal(hu, hg), "the gate must not touch the state"
    _close(yg, yu * g, 1e-300, 1e-14, "gate = SiLU(z)")
    yl, _ = o.scan(**dict(case, z=np.full_like(z, 40.0)))
    _close(yl, yu * 40.0, 0.0, 1e-14, "gate at z = 40")


# ---------------------------------------------------------------- zero-order hold
def pin_zoh_lti(o):
    """Exact zero-order hold: constant step and B, C give a convolution with
    Bbar_n = expm1(delta A_n) / A_n * B_n.

    "Mamba: Linear-Time Sequence Modeling with Selective State Spaces"
    (nadeemcite summary), section "Core Idea": Abar = exp(delta A) and
    Bbar = (delta A)^-1 (exp(delta A) - I) delta B; with A diagonal, each
    state's input map is expm1(delta A_n) / A_n * B_n. With those fixed, the
    recurrence unrolls into y_k = sum_j K_j x_{k-j} (+ D x_k + the decayed h0),
    K_j = sum_n C_n Abar_n^j Bbar_n.
    """
    rng = np.random.default_rng(23)
    b, L, E, N = 1, 30, 2, 4
    raw_e = rng.normal(0.0, 0.5, E)
    Bc = rng.standard_normal((b, N))
    Cc = rng.standard_normal((b, N))
    case = dict(
        x=rng.standard_normal((b, L, E)),
        delta=np.broadcast_to(raw_e, (b, L, E)).copy(),
        A_log=rng.normal(0.0, 0.6, (E, N)),
        B=np.repeat(Bc[:, None, :], L, axis=1),
        C=np.repeat(Cc[:, None, :], L, axis=1),
        D=rng.standard_normal(E), h0=rng.standard_normal((b, E, N)))
    y, h_last = o.scan(**case, delta_softplus=True, write_zoh=True)
    step = _softplus(raw_e)
    A = -np.exp(case["A_log"])
    abar = np.exp(step[:, None] * A)
    bbar = np.expm1(step[:, None] * A) / A * Bc[0][None, :]     # [E, N]
    x, D, h0 = case["x"], case["D"], case["h0"]
    for e in range(E):
        powers = abar[e][None, :] ** np.arange(L + 1)[:, None]
        K = (powers[:L] * Cc[0] * bbar[e]).sum(1)
        scale = (powers[:L] * np.abs(Cc[0] * bbar[e])).sum(1)
        for k in range(L):
            want = np.dot(K[:k + 1], x[0, k::-1, e]) + D[e] * x[0, k, e] \
                + np.dot(Cc[0] * powers[k + 1], h0[0, e])
            tol = 1e-12 * (np.dot(scale[:k + 1], np.abs(x[0, k::-1, e]))
                           + abs(D[e] * x[0, k, e])
                           + np.dot(np.abs(Cc[0]) * powers[k + 1],
                                    np.abs(h0[0, e]))) + 1e-300
            assert abs(y[0, k, e] - want) <= tol, (e, k, y[0, k, e], want)


def pin_zoh_fixed_point(o):
    """Exact zero-order hold keeps the continuous system's equilibrium.

    Same page and section: the discretization is exact for inputs held
    constant over each step, so with constant x and B the state settles at
    the fixed point of h' = A h + B x, that is h = -B x / A, whatever the
    step size. (The delta * B write instead settles at delta B x / (1 - Abar),
    which depends on delta.)
    """
    for raw in (-1.0, 0.8):
        b, L, E, N = 1, 4000, 2, 3
        rng = np.random.default_rng(29)
        xv = rng.standard_normal(E)
        Bv = rng.standard_normal(N)
        case = dict(x=np.broadcast_to(xv, (b, L, E)).copy(),
                    delta=np.full((b, L, E), raw),
                    A_log=rng.normal(0.0, 0.3, (E, N)),
                    B=np.broadcast_to(Bv, (b, L, N)).copy(),
                    C=rng.standard_normal((b, L, N)))
        _, h_last = o.scan(**case, delta_softplus=True, write_zoh=True)
        A = -np.exp(case["A_log"])
        want = -Bv[None, :] * xv[:, None] / A
        _close(h_last[0], want, 1e-12, 1e-10, "ZOH fixed point")


def pin_zoh_small_step(o):
    """Zero-order hold tends to the delta * B write as delta -> 0.

    expm1(delta A) / A = delta (1 + delta A / 2 + ...), so for delta ~ 1e-9
    the two writes agree to about 1e-9 relative ("There is a discretization
    detail worth keeping explicit" on the abhik page contrasts the two).
    """
    case = random_case(37, 2, 20, 3, 4, gate=False, bias=False)
    case["delta"] = np.full_like(case["delta"], 1e-9)
    yz, hz = o.scan(**case, delta_softplus=False, write_zoh=True)
    yd, hd = o.scan(**case, delta_softplus=False, write_zoh=False)
    _scaled_close(yz, yd, np.abs(yd) + 1e-6, 1e-7, "ZOH small step y")
    _scaled_close(hz, hd, np.abs(hd) + 1e-9, 1e-7, "ZOH small step h")
    assert not np.array_equal(yz, yd)


# ---------------------------------------------------------------- decode step
def pin_step_matches_scan(o):
    """Decoding one token at a time reproduces the full scan, bitwise.

    [abhik] "6. Carry both buffers to the next token" updates the [b, E, N]
    state exactly as the scan does for one step, and "The selective operator
    is one part of the Mamba block" asks the full sequence and token-by-token
    results to agree. Checked without the convolution, for both writes.
    """
    for zoh in (False, True):
        case = random_case(43, 2, 17, 3, 4)
        y, h_last = o.scan(**case, delta_softplus=True, write_zoh=zoh)
        state = case["h0"].copy()
        for t in range(17):
            yt, state, _ = o.step(case["x"][:, t], case["delta"][:, t],
                                  case["A_log"], case["B"][:, t],
                                  case["C"][:, t], state, D=case["D"],
                                  z=case["z"][:, t],
                                  delta_bias=case["delta_bias"],
                                  delta_softplus=True, write_zoh=zoh)
            assert np.array_equal(yt, y[:, t]), (zoh, t)
        assert np.array_equal(state, h_last), zoh


def pin_step_causal_convolution(o):
    """The step's convolution is the causal depthwise convolution + SiLU.

    [abhik] "4. Add causal local context before selecting coefficients":
    x_t = SiLU(b + sum_k q_k v_{t-K+1+k}) with zeros before the start, and
    "6. Carry both buffers" keeps K samples including the newest. With B = 0,
    D = 1 and no gate the step outputs that x, which must equal numpy's full
    convolution with the reversed kernel, cut to the causal part.
    """
    rng = np.random.default_rng(47)
    b, E, N, K, L = 2, 3, 2, 4, 12
    v = rng.standard_normal((b, L, E))
    w = rng.standard_normal((E, K))
    bias = rng.standard_normal(E)
    conv = np.zeros((b, E, K))
    state = np.zeros((b, E, N))
    for t in range(L):
        yt, state, conv = o.step(v[:, t], np.zeros((b, E)),
                                 np.zeros((E, N)), np.zeros((b, N)),
                                 rng.standard_normal((b, N)), state,
                                 conv_state=conv, conv_weight=w,
                                 conv_bias=bias, D=np.ones(E),
                                 delta_softplus=False)
        for bb in range(b):
            for e in range(E):
                full = np.convolve(v[bb, :t + 1, e], w[e, ::-1])[:t + 1]
                pre = full[t] + bias[e]
                want = pre / (1.0 + math.exp(-pre))
                assert abs(yt[bb, e] - want) <= 1e-13 * (1 + abs(want)), \
                    (t, bb, e, yt[bb, e], want)
        # the buffer holds the last K inputs, oldest first, zeros before
        for k in range(K):
            src = t - (K - 1) + k
            want = v[:, src] if src >= 0 else np.zeros((b, E))
            assert np.array_equal(conv[:, :, k], want), (t, k)


def pin_step_conv_feeds_scan(o):
    """With the convolution on, decoding equals the scan of the convolved
    input.

    [abhik] "5. Put the selective operator inside the complete mixer": the
    scan runs on x = SiLU(CausalDWConv(v)), with D x and the gate on that x;
    "6. Carry both buffers" decodes the same thing token by token. The
    convolved input is formed here with numpy's convolution, then the scan
    oracle (pinned above) gives the expected outputs and final state.
    """
    rng = np.random.default_rng(53)
    b, E, N, K, L = 2, 3, 4, 3, 15
    case = random_case(59, b, L, E, N)
    v = rng.standard_normal((b, L, E))
    w = rng.standard_normal((E, K))
    cbias = rng.standard_normal(E)
    xc = np.empty_like(v)
    for bb in range(b):
        for e in range(E):
            pre = np.convolve(v[bb, :, e], w[e, ::-1])[:L] + cbias[e]
            xc[bb, :, e] = pre / (1.0 + np.exp(-pre))
    y, h_last = o.scan(**dict(case, x=xc), delta_softplus=True)
    state = case["h0"].copy()
    conv = np.zeros((b, E, K))
    for t in range(L):
        yt, state, conv = o.step(v[:, t], case["delta"][:, t], case["A_log"],
                                 case["B"][:, t], case["C"][:, t], state,
                                 conv_state=conv, conv_weight=w,
                                 conv_bias=cbias, D=case["D"],
                                 z=case["z"][:, t],
                                 delta_bias=case["delta_bias"])
        _close(yt, y[:, t], 1e-12, 1e-10, "decode with conv, step %d" % t)
    _close(state, h_last, 1e-12, 1e-10, "decode with conv, state")


def pin_scan_conv(o):
    """The scan with the causal convolution in front.

    [abhik] "4. Add causal local context before selecting coefficients" and
    "5. Put the selective operator inside the complete mixer": the scan runs
    on x = SiLU(CausalDWConv(v)) with left zero padding. Checked against (i)
    the pinned scan of x formed with numpy's convolution, and (ii) decoding
    the sequence token by token through the conv buffer ("6. Carry both
    buffers").
    """
    rng = np.random.default_rng(61)
    b, L, E, N, K = 2, 21, 3, 4, 4
    case = random_case(67, b, L, E, N)
    v = rng.standard_normal((b, L, E))
    w = rng.standard_normal((E, K))
    cb = rng.standard_normal(E)
    y, h = o.scan_conv(v, w, case["delta"], case["A_log"], case["B"],
                       case["C"], conv_bias=cb, D=case["D"], z=case["z"],
                       delta_bias=case["delta_bias"], h0=case["h0"])
    xc = np.empty_like(v)
    for bb in range(b):
        for e in range(E):
            pre = np.convolve(v[bb, :, e], w[e, ::-1])[:L] + cb[e]
            xc[bb, :, e] = pre / (1.0 + np.exp(-pre))
    y2, h2 = o.scan(**dict(case, x=xc), delta_softplus=True)
    _close(y, y2, 1e-12, 1e-10, "scan_conv vs scan of numpy conv")
    _close(h, h2, 1e-12, 1e-10, "scan_conv state")
    state, conv = case["h0"].copy(), np.zeros((b, E, K))
    for t in range(L):
        yt, state, conv = o.step(v[:, t], case["delta"][:, t], case["A_log"],
                                 case["B"][:, t], case["C"][:, t], state,
                                 conv_state=conv, conv_weight=w, conv_bias=cb,
                                 D=case["D"], z=case["z"][:, t],
                                 delta_bias=case["delta_bias"])
        _close(yt, y[:, t], 1e-12, 1e-10, "decode vs scan_conv step %d" % t)


# ---------------------------------------------------------------- softplus
def pin_step_size(o):
    """delta = softplus(raw + bias), PyTorch default softplus.

    [abhik] "1. Produce coefficients from the locally mixed input" (softplus
    of the projection plus its bias gives a positive time scale) and [keswani]
    "from ssm to selective ssm" (numerically stable softplus). F.softplus'
    default threshold 20 returns the input itself above 20.
    """
    assert abs(o.step_size(0.0) - math.log(2.0)) <= 1e-16
    for v in (20.5, 25.0, 100.0, 1e6):
        assert o.step_size(v) == v, v
    for v in (-40.0, -60.0, -700.0):
        assert abs(o.step_size(v) - math.exp(v)) <= 1e-15 * math.exp(v), v
    for v in (-3.0, -0.5, 0.7, 4.0, 19.5):
        # the test side's log(1 + e^v) rounds 1 + e^v first: ~2 ulp of 1
        assert abs(o.step_size(v) - math.log(1.0 + math.exp(v))) <= \
            5e-16 + 4e-16 * abs(math.log(1.0 + math.exp(v))), v
    assert o.step_size(0.3, -0.8) == o.step_size(-0.5)
    assert o.step_size(0.3, -0.8, softplus=False) == 0.3 + -0.8
    prev = 0.0
    for v in np.linspace(-30.0, 30.0, 121):
        cur = o.step_size(float(v))
        assert cur > 0.0 and cur >= prev
        prev = cur


# ---------------------------------------------------------------- backward
def pin_backward_finite_differences(o):
    """Every gradient of the backward oracle equals a central finite
    difference of the (pinned) forward oracle.

    The loss is sum(dy * y) + sum(dh * h_last) for random dy, dh; each input
    entry is moved by +-eps and the loss recomputed by the forward oracle
    ([abhik] rows 1, 2 and 5 and "Compose the updates instead of waiting for
    every state", which trains through the scan). Central differences are
    exact to O(eps^2) ~ 1e-12 here, so a dropped term, a wrong sign or a
    transposed index shows as an O(1e-2..1) mismatch. Covered: both writes,
    gate on and off, softplus on and off, with and without D and the bias.
    """
    variants = [dict(write_zoh=False), dict(write_zoh=True),
                dict(write_zoh=False, gate=False, D=False, bias=False),
                dict(write_zoh=True, softplus=False)]
    for k, var in enumerate(variants):
        zoh = var["write_zoh"]
        softplus = var.get("softplus", True)
        b, L, E, N = 2, 6, 3, 3
        case = random_case(71 + k, b, L, E, N, gate=var.get("gate", True),
                           D=var.get("D", True), bias=var.get("bias", True))
        if not softplus:   # positive raw steps
            case["delta"] = np.abs(case["delta"]) * 0.5 + 0.05
            case["delta_bias"] = None
        rng = np.random.default_rng(90 + k)
        dy = rng.standard_normal((b, L, E))
        dh = rng.standard_normal((b, E, N))

        def loss(c):
            y, h = o.scan(**c, delta_softplus=softplus, write_zoh=zoh)
            return float(np.sum(dy * y) + np.sum(dh * h))

        g = o.scan_bwd(case["x"], case["delta"], case["A_log"], case["B"],
                       case["C"], dy, D=case["D"], z=case["z"],
                       delta_bias=case["delta_bias"], delta_softplus=softplus,
                       h0=case["h0"], dh_last=dh, write_zoh=zoh)
        names = {"x": "dx", "delta": "ddelta", "A_log": "dA_log", "B": "dB",
                 "C": "dC", "D": "dD", "z": "dz", "delta_bias": "ddelta_bias",
                 "h0": "dh0"}
        for key, gname in names.items():
            if case[key] is None:
                assert g[gname] is None or gname == "dh0", gname
                continue
            arr = case[key]
            fd = np.empty_like(arr)
            for idx in np.ndindex(arr.shape):
                eps = 1e-6 * max(1.0, abs(arr[idx]))
                c1 = dict(case)
                c1[key] = arr.copy()
                c1[key][idx] += eps
                up = loss(c1)
                c1[key][idx] -= 2 * eps
                fd[idx] = (up - loss(c1)) / (2 * eps)
            _close(g[gname], fd, 1e-6, 1e-6,
                   "backward %s (variant %d)" % (gname, k))


ALL_PINS = (pin_associative_prefix, pin_lti_convolution, pin_forgetting,
            pin_freezing, pin_retention_bounds, pin_continuation,
            pin_decode_step, pin_linearity, pin_independence, pin_degenerate,
            pin_step_size, pin_zoh_lti, pin_zoh_fixed_point, pin_zoh_small_step,
            pin_step_matches_scan, pin_step_causal_convolution,
            pin_step_conv_feeds_scan, pin_scan_conv,
            pin_backward_finite_differences)
