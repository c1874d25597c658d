"""GPU tests of split sequences: pieces scanned concurrently and joined by a
decoupled look-back over their affine aggregates, then a replay of each
piece's start for its carried-in state. Compared with the float64 oracle
and with the unsplit scan; the bounded wait is made to run out on purpose
(a piece that never publishes) and must report a timeout, not hang."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_51_b200 as S
from selective_state_space_51_b200 import workloads as W
from gpu_helpers import assert_close, oracle_inputs, rel_err, run, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def scan():
    s = S.SelectiveScan(0)
    yield s
    s.close()


def _set(scan, segments, tb=0, variant=S.SSM_VARIANT_CHUNKED):
    scan.set_variant(variant, segments)
    S.library().ssm_scan_set_time_blocks(scan.handle, tb)


def _reset(scan):
    _set(scan, 0, 0, S.SSM_VARIANT_AUTO)
    S.library().ssm_scan_set_debug(scan.handle, 0, 0)


@pytest.mark.parametrize("jitter", [0.0, 0.5], ids=["A_stated",
                                                    "A_per_channel"])
@pytest.mark.parametrize("tb", [1, 2])
@pytest.mark.parametrize("segments", [2, 3, 7])
@pytest.mark.parametrize("idx,size", [
    (4, dict(seqlen=9000, dim=32)),
    (3, dict(batch=2, seqlen=3000, dim=24, with_h0=True)),
    (1, dict(batch=2, seqlen=2500, dim=40, with_h0=True)),
], ids=["long_f32", "layer_bf16", "classifier_f32"])
def test_split_parity(scan, idx, size, segments, tb, jitter):
    wl = W.make(idx, a_jitter=jitter, **size)
    _set(scan, segments, tb)
    try:
        y, h = run(scan, wl)
        v, segs = scan.last_variant()
        assert v == S.SSM_VARIANT_CHUNKED and segs == segments
    finally:
        _reset(scan)
    yo, ho = oracle.scan(**oracle_inputs(wl))
    assert_close(y, yo, wl.dtype, "y")
    assert_close(h, ho, wl.dtype, "h_last")


def test_split_slow_decay_replays_whole_piece(scan):
    """Tiny steps keep the carried-in state alive through a whole piece, so
    the replay cannot stop early. Split and unsplit must agree at the float32
    bar, and both must meet it against the float64 oracle. The input is the
    float32 worst case: the same retention (a ~ 1 - 6e-6) repeats for 4000
    steps, so any bias in its rounding compounds linearly; the float32
    kernels take retentions this close to 1 from a polynomial rounded once,
    not from the SFU's exp2."""
    wl = W.make(4, seqlen=4000, dim=16)
    wl.dev["delta"] = np.full_like(wl.dev["delta"], -12.0)   # delta ~ 6e-6
    t = to_device(wl)
    try:
        _set(scan, 4, 1)
        y, h = run(scan, wl, t=t)
        _set(scan, 1, 1)
        y1, h1 = run(scan, wl, t=t)
    finally:
        _reset(scan)
    assert_close(y, y1, wl.dtype, "y split vs unsplit")
    assert_close(h, h1, wl.dtype, "h_last split vs unsplit")
    yo, ho = oracle.scan(**oracle_inputs(wl))
    assert_close(y, yo, wl.dtype, "y against the oracle")
    assert_close(h, ho, wl.dtype, "h_last against the oracle")
    assert_close(y1, yo, wl.dtype, "unsplit y against the oracle")


def test_split_matches_unsplit(scan):
    wl = W.make(4, seqlen=12000, dim=32)
    t = to_device(wl)
    _set(scan, 1, 1)
    try:
        y1, h1 = run(scan, wl, t=t)
        _set(scan, 6, 1)
        y6, h6 = run(scan, wl, t=t)
    finally:
        _reset(scan)
    assert_close(y6, y1, W.F32, "y split vs unsplit")
    assert_close(h6, h1, W.F32, "h_last split vs unsplit")


def test_auto_splits_long_few_channel_sequences(scan):
    wl = W.make(4, seqlen=131072, dim=64)
    run(scan, wl)
    v, segs = scan.last_variant()
    assert v == S.SSM_VARIANT_CHUNKED and segs > 1


def test_bounded_wait_times_out_and_recovers(scan):
    """The first piece never publishes; its successor gives up after a short
    bounded wait, the call reports SSM_ERR_TIMEOUT, and the next call on the
    same handle and context is correct."""
    wl = W.make(4, seqlen=6000, dim=32)
    t = to_device(wl)
    _set(scan, 3, 1)
    lib = S.library()
    try:
        assert lib.ssm_scan_set_debug(scan.handle, 1, 2000) == S.SSM_OK
        scan(t["x"], t["delta"], t["A_log"], t["B"], t["C"], D=t["D"],
             z=t["z"], delta_bias=t["delta_bias"], h0=t["h0"])
        assert scan.sync_status() == S.SSM_ERR_TIMEOUT
        assert scan.sync_status() == S.SSM_OK          # status was reset
        lib.ssm_scan_set_debug(scan.handle, 0, 0)
        y, h = run(scan, wl, t=t)
    finally:
        _reset(scan)
    yo, ho = oracle.scan(**oracle_inputs(wl))
    assert_close(y, yo, wl.dtype, "y after recovery")
    assert_close(h, ho, wl.dtype, "h_last after recovery")
