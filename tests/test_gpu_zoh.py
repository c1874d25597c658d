"""GPU parity of the exact zero-order-hold write (SSM_WRITE_ZOH): the write
expm1(delta A) / A * B * x, against the float64 oracle's write_zoh path."""
import numpy as np
import pytest

import oracle
import selective_state_space_51_b200 as S
from selective_state_space_51_b200 import workloads as W
from gpu_helpers import assert_close, oracle_inputs, run, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def scan():
    s = S.SelectiveScan(0)
    yield s
    s.close()


def _set(scan, variant, tb=0, segments=0):
    scan.set_variant(variant, segments)
    S.library().ssm_scan_set_time_blocks(scan.handle, tb)


CASES = {
    "classifier_f32": (1, dict(batch=2, seqlen=700, dim=72)),
    "layer_bf16": (3, dict(batch=2, seqlen=1500, dim=40, with_h0=True)),
    "long_f32": (4, dict(seqlen=6000, dim=32)),
    "tiny_n4": (0, dict()),
    "n8_bf16": (2, dict(batch=2, seqlen=900, dim=48, dstate=8)),
}


@pytest.mark.parametrize("variant", [(S.SSM_VARIANT_AUTO, 0, 0),
                                     (S.SSM_VARIANT_SEQUENTIAL, 0, 0),
                                     (S.SSM_VARIANT_CHUNKED, 1, 1),
                                     (S.SSM_VARIANT_CHUNKED, 1, 3)],
                         ids=["auto", "sequential", "chunked", "chunked_split3"])
@pytest.mark.parametrize("jitter", [0.0, 0.5], ids=["A_stated",
                                                    "A_per_channel"])
@pytest.mark.parametrize("name", sorted(CASES))
def test_zoh_parity(scan, name, variant, jitter):
    idx, size = CASES[name]
    wl = W.make(idx, a_jitter=jitter, **size)
    _set(scan, *variant)
    try:
        y, h = run(scan, wl, write_zoh=True)
    finally:
        _set(scan, S.SSM_VARIANT_AUTO)
    yo, ho = oracle.scan(**oracle_inputs(wl), write_zoh=True)
    assert_close(y, yo, wl.dtype, "y")
    assert_close(h, ho, wl.dtype, "h_last")


def test_zoh_differs_from_default_write(scan):
    wl = W.make(4, seqlen=2000, dim=32)
    t = to_device(wl)
    y0, _ = run(scan, wl, t=t)
    y1, _ = run(scan, wl, t=t, write_zoh=True)
    assert np.max(np.abs(y1 - y0)) > 1e-3


def test_zoh_with_two_time_blocks_is_refused(scan):
    wl = W.make(1, batch=1, seqlen=64, dim=32)
    t = to_device(wl)
    _set(scan, S.SSM_VARIANT_CHUNKED, 2)
    try:
        with pytest.raises(S.SsmScanError) as ei:
            scan(t["x"], t["delta"], t["A_log"], t["B"], t["C"], D=t["D"],
                 z=t["z"], delta_bias=t["delta_bias"], write_zoh=True)
        assert ei.value.status == S.SSM_ERR_UNSUPPORTED
    finally:
        _set(scan, S.SSM_VARIANT_AUTO)
