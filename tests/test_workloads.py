"""Seeded input generator: determinism, bf16 rounding, recipe (CPU only)."""
import numpy as np
import torch

import oracle
from selective_state_space_51_b200 import workloads as W


def test_deterministic_and_seed_sensitive():
    a, b = W.make(0), W.make(0)
    for k in a.dev:
        if a.dev[k] is None:
            assert b.dev[k] is None
        else:
            assert np.array_equal(a.dev[k], b.dev[k]), k
    c = W.make(0, seed=123)
    assert not np.array_equal(a.dev["x"], c.dev["x"])


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    vals = np.concatenate([
        rng.standard_normal(100000).astype(np.float32),
        # exact ties between two bfloat16 values, both parities
        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8),
                  0.0, -0.0, 3.0e38, 1e-40], dtype=np.float32)])
    ours = W.round_to_bf16_bits(vals)
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy()
    assert np.array_equal(ours.view(np.int16), ref)
    back = W.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(vals).to(torch.bfloat16)
                          .to(torch.float32).numpy())


def test_shapes_and_options():
    for idx in range(5):
        w = W.make(idx, batch=2, seqlen=33, dim=24)
        N = W.SHAPES[idx][4]
        assert w.dev["x"].shape == (2, 33, 24)
        assert w.dev["B"].shape == (2, 33, N)
        assert w.dev["A_log"].shape == (24, N)
        assert (w.dev["z"] is not None) == W.SHAPES[idx][6]
        assert (w.dev["h0"] is not None) == (idx == 4)
        assert (w.dev["delta_bias"] is None) == (idx == 4)
        if w.dtype == W.BF16:
            assert w.dev["x"].dtype == np.uint16
            assert w.values("x").dtype == np.float32
        assert np.array_equal(w.dev["A_log"][3],
                              np.log(np.arange(1, N + 1)).astype(np.float32))


def test_step_bias_recipe():
    """softplus(0 + bias) recovers dt in [1e-3, 1e-1] (float32 bias)."""
    w = W.make(0, dim=64)
    steps = np.array([oracle.step_size(0.0, float(b)) for b in
                      w.dev["delta_bias"]])
    assert np.all(steps >= 1e-3 * (1 - 1e-5)) and np.all(steps <= 0.1 * (1 + 1e-5))
    assert np.unique(np.round(np.log10(steps), 1)).size > 5   # spread out


def test_long_memory_recipe():
    w = W.make(4, seqlen=4096, dim=64)
    raw = w.dev["delta"]
    assert abs(float(raw.mean()) + 2.0) < 0.02 and abs(float(raw.std()) - 1) < 0.02
    assert abs(float(w.dev["h0"].std()) - 0.1) < 0.01


def test_per_channel_A_jitter_keeps_other_draws():
    """a_jitter draws a distinct A row per channel after every other draw,
    so the other arrays are unchanged and the rows differ channel to
    channel."""
    base = W.make(2, batch=2, seqlen=40, dim=32)
    jit = W.make(2, batch=2, seqlen=40, dim=32, a_jitter=0.5)
    for k in base.dev:
        if k == "A_log" or base.dev[k] is None:
            continue
        assert np.array_equal(base.dev[k], jit.dev[k]), k
    A = jit.dev["A_log"]
    assert A.dtype == np.float32 and A.shape == (32, 16)
    assert len({A[e].tobytes() for e in range(32)}) == 32
    dev = A - base.dev["A_log"]
    assert 0.35 < float(dev.std()) < 0.65
