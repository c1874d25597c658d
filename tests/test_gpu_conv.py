"""GPU parity of the scan with the causal depthwise convolution + SiLU fused
in front (ssm_scan_fwd_conv), against the float64 oracle's scan_conv."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_51_b200 as S
from selective_state_space_51_b200 import workloads as W
from gpu_helpers import assert_close, oracle_inputs, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def scan():
    s = S.SelectiveScan(0)
    yield s
    s.close()


def _set(scan, variant, tb=0, segments=0):
    scan.set_variant(variant, segments)
    S.library().ssm_scan_set_time_blocks(scan.handle, tb)


def _run(scan, wl, w, cb, write_zoh=False, t=None):
    t = to_device(wl) if t is None else t
    y, h = scan(t["x"], t["delta"], t["A_log"], t["B"], t["C"], D=t["D"],
                z=t["z"], delta_bias=t["delta_bias"], h0=t["h0"],
                write_zoh=write_zoh,
                conv_weight=torch.from_numpy(w).cuda(),
                conv_bias=None if cb is None else torch.from_numpy(cb).cuda())
    torch.cuda.synchronize()
    assert scan.sync_status() == S.SSM_OK
    return (y.float().cpu().numpy().astype(np.float64),
            h.cpu().numpy().astype(np.float64))


def _oracle(wl, w, cb, write_zoh=False):
    inp = oracle_inputs(wl)
    v = inp.pop("x")
    return oracle.scan_conv(v, w, conv_bias=cb, write_zoh=write_zoh, **inp)


# sizes span several windows with a ragged tail
CASES = {
    "classifier_f32": (1, dict(batch=2, seqlen=700, dim=72)),
    "layer_bf16": (3, dict(batch=2, seqlen=1500, dim=40, with_h0=True)),
    "long_f32": (4, dict(seqlen=6000, dim=32)),
    "tiny_n4": (0, dict()),
    "n8_bf16": (2, dict(batch=2, seqlen=900, dim=48, dstate=8)),
    "n4_f32_ragged": (0, dict(batch=3, seqlen=333, dim=24)),
}
VARIANTS = [(S.SSM_VARIANT_AUTO, 0, 0), (S.SSM_VARIANT_SEQUENTIAL, 0, 0),
            (S.SSM_VARIANT_CHUNKED, 1, 1), (S.SSM_VARIANT_CHUNKED, 1, 3)]
VARIANT_IDS = ["auto", "sequential", "chunked", "chunked_split3"]


@pytest.mark.parametrize("jitter", [0.0, 0.5], ids=["A_stated",
                                                    "A_per_channel"])
@pytest.mark.parametrize("variant", VARIANTS, ids=VARIANT_IDS)
@pytest.mark.parametrize("name", sorted(CASES))
def test_conv_parity(scan, name, variant, jitter):
    idx, size = CASES[name]
    wl = W.make(idx, a_jitter=jitter, **size)
    w, cb = W.conv_params(wl.dim, 4)
    _set(scan, *variant)
    try:
        y, h = _run(scan, wl, w, cb)
    finally:
        _set(scan, S.SSM_VARIANT_AUTO)
    yo, ho = _oracle(wl, w, cb)
    assert_close(y, yo, wl.dtype, "y")
    assert_close(h, ho, wl.dtype, "h_last")


@pytest.mark.parametrize("variant", VARIANTS, ids=VARIANT_IDS)
@pytest.mark.parametrize("width", [1, 2, 3])
@pytest.mark.parametrize("idx,dtype", [(1, W.F32), (3, W.BF16), (0, W.F32)],
                         ids=["n16_f32", "n16_bf16", "n4_f32"])
def test_conv_widths(scan, width, idx, dtype, variant):
    wl = W.make(idx, batch=2, seqlen=400, dim=64, dtype=dtype, a_jitter=0.5)
    w, cb = W.conv_params(wl.dim, width, seed=7 + width)
    _set(scan, *variant)
    try:
        y, h = _run(scan, wl, w, cb)
    finally:
        _set(scan, S.SSM_VARIANT_AUTO)
    yo, ho = _oracle(wl, w, cb)
    assert_close(y, yo, wl.dtype, "y")
    assert_close(h, ho, wl.dtype, "h_last")


@pytest.mark.parametrize("variant", VARIANTS, ids=VARIANT_IDS)
def test_conv_with_zoh_and_no_bias(scan, variant):
    wl = W.make(3, batch=2, seqlen=1100, dim=40, with_h0=True, a_jitter=0.5)
    w, _ = W.conv_params(wl.dim, 4, seed=3)
    _set(scan, *variant)
    try:
        y, h = _run(scan, wl, w, None, write_zoh=True)
    finally:
        _set(scan, S.SSM_VARIANT_AUTO)
    yo, ho = _oracle(wl, w, None, write_zoh=True)
    assert_close(y, yo, wl.dtype, "y")
    assert_close(h, ho, wl.dtype, "h_last")


@pytest.mark.parametrize("segments", [2, 5, 16])
def test_conv_split_boundaries(scan, segments):
    """Pieces of a split sequence take their convolution history from the
    piece before; a wide filter with large taps makes any lost halo show."""
    wl = W.make(4, seqlen=5000, dim=32, a_jitter=0.5)
    w, cb = W.conv_params(wl.dim, 4, seed=11)
    w *= 4
    _set(scan, S.SSM_VARIANT_CHUNKED, 1, segments)
    try:
        y, h = _run(scan, wl, w, cb)
    finally:
        _set(scan, S.SSM_VARIANT_AUTO)
    yo, ho = _oracle(wl, w, cb)
    assert_close(y, yo, wl.dtype, "y")
    assert_close(h, ho, wl.dtype, "h_last")


@pytest.mark.parametrize("idx", [3, 4])
def test_conv_full_size_sampled(scan, idx):
    """Full workload sizes in the launch configuration the bench times with
    the convolution; a sample of channels is checked at every step."""
    wl = W.make(idx)
    t = to_device(wl)
    w, cb = W.conv_params(wl.dim, 4)
    y, h = scan(t["x"], t["delta"], t["A_log"], t["B"], t["C"], D=t["D"],
                z=t["z"], delta_bias=t["delta_bias"], h0=t["h0"],
                conv_weight=torch.from_numpy(w).cuda(),
                conv_bias=torch.from_numpy(cb).cuda())
    torch.cuda.synchronize()
    assert scan.sync_status() == S.SSM_OK
    rng = np.random.default_rng(idx)
    ch = np.unique(np.concatenate([[0, wl.dim - 1],
                                   rng.choice(wl.dim, 6, replace=False)]))
    sel = torch.from_numpy(ch).cuda()
    ych = y[..., sel].float().cpu().numpy()
    hch = h[:, sel].cpu().numpy()
    del y, h, t
    inp = oracle_inputs(wl)
    v = inp.pop("x")
    yo, ho = oracle.scan_conv_channels(ch, v, w, conv_bias=cb, **inp)
    assert_close(ych, yo, wl.dtype, "y (sampled channels)")
    assert_close(hch, ho, wl.dtype, "h_last (sampled channels)")


def test_conv_is_not_the_plain_scan(scan):
    """The fused path really convolves: its output differs from the scan of
    the raw input."""
    wl = W.make(1, batch=2, seqlen=300, dim=64)
    t = to_device(wl)
    w, cb = W.conv_params(wl.dim, 4)
    y1, _ = _run(scan, wl, w, cb, t=t)
    y0, _ = scan(t["x"], t["delta"], t["A_log"], t["B"], t["C"], D=t["D"],
                 z=t["z"], delta_bias=t["delta_bias"])
    assert np.max(np.abs(y1 - y0.cpu().numpy())) > 1e-2


def test_conv_argument_errors(scan):
    b, L, E, N = 1, 32, 16, 4
    x = torch.zeros((b, L, E), device="cuda")
    A = torch.zeros((E, N), device="cuda")
    Bm = torch.zeros((b, L, N), device="cuda")
    y = torch.empty_like(x)
    w5 = torch.zeros((E, 5), device="cuda")
    w4 = torch.zeros((E, 4), device="cuda")
    dims = (b, L, E, N)

    def call(w, width):
        return S.ssm_scan_fwd_conv(scan.handle, x, w, None, width, x, A, Bm,
                                   Bm, None, None, None, 1, None, y, None,
                                   dims, S.SSM_F32, check=False)
    assert call(w5, 5) == S.SSM_ERR_INVALID
    assert call(w4, 0) == S.SSM_ERR_INVALID
    assert call(None, 4) == S.SSM_ERR_INVALID
    assert call(w4, 4) == S.SSM_OK
    torch.cuda.synchronize()


@pytest.mark.parametrize("width", [4, 2])
@pytest.mark.parametrize("idx,size", [
    (3, dict(batch=2, seqlen=1024, dim=64)),
    (3, dict(batch=4, seqlen=96, dim=4736)),   # enough tiles for 16-ch ones
    (1, dict(batch=2, seqlen=512, dim=64)),
], ids=["bf16", "bf16_many_tiles", "f32"])
def test_conv_whole_tiles_and_windows(scan, idx, size, width):
    """Shapes of whole channel tiles and windows, gated, softplus: the fused
    convolution on the specialised kernel (halo carried across windows with
    one barrier per window). Per-channel A; against the oracle."""
    wl = W.make(idx, a_jitter=0.5, **size)
    w, cb = W.conv_params(wl.dim, width, seed=5 + width)
    y, h = _run(scan, wl, w, cb)
    yo, ho = _oracle(wl, w, cb)
    assert_close(y, yo, wl.dtype, "y")
    assert_close(h, ho, wl.dtype, "h_last")
