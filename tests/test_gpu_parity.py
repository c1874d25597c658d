"""GPU parity: the CUDA library (through its C ABI) against the float64 oracle.

Bar: max |gpu - oracle| / (1 + |oracle|) <= 1e-4 for float32 activations and
<= 2e-2 for bfloat16 activations (the oracle reads the same bfloat16-rounded
inputs), for y and for h_last.
"""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_51_b200 as S
from selective_state_space_51_b200 import workloads as W
from gpu_helpers import TOL, assert_close, oracle_inputs, run, to_device

pytestmark = pytest.mark.gpu

# (variant, time blocks per channel for the chunked variant)
VARIANTS = [(S.SSM_VARIANT_AUTO, 0), (S.SSM_VARIANT_SEQUENTIAL, 0),
            (S.SSM_VARIANT_CHUNKED, 1), (S.SSM_VARIANT_CHUNKED, 2)]
VARIANT_IDS = ["auto", "sequential", "chunked_tb1", "chunked_tb2"]

# Small cases with each workload's distributions: several tiles, ragged
# sequence ends and ragged channel tiles.
SMALL = {
    0: dict(),                                            # full tiny shape
    1: dict(batch=3, seqlen=700, dim=72),
    2: dict(batch=2, seqlen=1500, dim=48),
    3: dict(batch=2, seqlen=2100, dim=40),
    4: dict(seqlen=5000, dim=24),
}


@pytest.fixture(scope="module")
def scan():
    s = S.SelectiveScan(0)
    yield s
    s.close()


def _with_variant(scan, variant, segments=0):
    if isinstance(variant, tuple):
        variant, tb = variant
    else:
        tb = 0
    scan.set_variant(variant, segments)
    S.library().ssm_scan_set_time_blocks(scan.handle, tb)


# a_jitter 0: the stated A_log = log(n + 1) for every channel; 0.5: every
# channel draws its own A row (A is a learned [E, N] parameter), so a read of
# the wrong channel's A cannot pass
JITTER = [0.0, 0.5]


@pytest.mark.parametrize("jitter", JITTER, ids=["A_stated", "A_per_channel"])
@pytest.mark.parametrize("variant", VARIANTS, ids=VARIANT_IDS)
@pytest.mark.parametrize("idx", sorted(SMALL), ids=lambda i: "shape%d" % i)
def test_small_parity(scan, idx, variant, jitter):
    wl = W.make(idx, a_jitter=jitter, **SMALL[idx])
    _with_variant(scan, variant)
    try:
        y, h = run(scan, wl)
    finally:
        _with_variant(scan, S.SSM_VARIANT_AUTO)
    yo, ho = oracle.scan(**oracle_inputs(wl), delta_softplus=True)
    assert_close(y, yo, wl.dtype, "y")
    assert_close(h, ho, wl.dtype, "h_last")


def _sample_channels(E, k, seed):
    rng = np.random.default_rng(seed)
    pick = set([0, 1, E - 1, E // 2]) | set(
        rng.choice(E, size=min(k, E), replace=False).tolist())
    return np.array(sorted(pick))


@pytest.mark.parametrize("idx", [1, 2, 3, 4], ids=lambda i: "shape%d" % i)
def test_full_size_sampled(scan, idx):
    """Full workload sizes, the launch configuration the bench times;
    every step of a sample of channels is checked against the oracle."""
    wl = W.make(idx)
    t = to_device(wl)
    y, h_last = scan(t["x"], t["delta"], t["A_log"], t["B"], t["C"],
                     D=t["D"], z=t["z"], delta_bias=t["delta_bias"],
                     h0=t["h0"])
    torch.cuda.synchronize()
    assert scan.sync_status() == S.SSM_OK
    ch = _sample_channels(wl.dim, 12 if idx != 4 else 6, 7 + idx)
    ych = y[..., torch.from_numpy(ch).cuda()].float().cpu().numpy()
    hch = h_last[:, torch.from_numpy(ch).cuda()].cpu().numpy()
    del t, y, h_last
    yo, ho = oracle.scan_channels(ch, **oracle_inputs(wl), delta_softplus=True)
    assert_close(ych, yo, wl.dtype, "y (sampled channels)")
    assert_close(hch, ho, wl.dtype, "h_last (sampled channels)")
    assert np.all(np.isfinite(ych))


@pytest.mark.parametrize("N", [1, 2, 3, 5, 8, 32, 64])
def test_state_sizes(scan, N):
    wl = W.make(1, batch=2, seqlen=300, dim=40, dstate=N, a_jitter=0.5)
    y, h = run(scan, wl)
    yo, ho = oracle.scan(**oracle_inputs(wl))
    assert_close(y, yo, wl.dtype, "y")
    assert_close(h, ho, wl.dtype, "h_last")


@pytest.mark.parametrize("variant", VARIANTS[2:], ids=VARIANT_IDS[2:])
@pytest.mark.parametrize("N,dtype", [(4, W.F32), (8, W.F32), (8, W.BF16),
                                     (16, W.F32), (16, W.BF16)])
def test_chunked_state_sizes(scan, N, dtype, variant):
    wl = W.make(2, batch=3, seqlen=333, dim=72, dstate=N, dtype=dtype,
                with_h0=True, a_jitter=0.5)
    _with_variant(scan, variant)
    try:
        y, h = run(scan, wl)
        assert scan.last_variant()[0] == S.SSM_VARIANT_CHUNKED
    finally:
        _with_variant(scan, S.SSM_VARIANT_AUTO)
    yo, ho = oracle.scan(**oracle_inputs(wl))
    assert_close(y, yo, wl.dtype, "y")
    assert_close(h, ho, wl.dtype, "h_last")


@pytest.mark.parametrize("variant", VARIANTS, ids=VARIANT_IDS)
@pytest.mark.parametrize("L", [1, 2, 31, 33, 257])
def test_short_and_ragged_lengths(scan, L, variant):
    wl = W.make(3, batch=2, seqlen=L, dim=24, with_h0=True)
    _with_variant(scan, variant)
    try:
        y, h = run(scan, wl)
    finally:
        _with_variant(scan, S.SSM_VARIANT_AUTO)
    yo, ho = oracle.scan(**oracle_inputs(wl))
    assert_close(y, yo, wl.dtype, "y")
    assert_close(h, ho, wl.dtype, "h_last")


@pytest.mark.parametrize("opts", [
    dict(gate=False), dict(D=False), dict(bias=False), dict(h0=True),
    dict(softplus=False), dict(gate=False, D=False, bias=False)],
    ids=["no_gate", "no_D", "no_bias", "h0", "no_softplus", "bare"])
@pytest.mark.parametrize("dtype", [W.F32, W.BF16])
def test_optional_inputs(scan, opts, dtype):
    wl = W.make(1, batch=2, seqlen=520, dim=48, dtype=dtype,
                gated=opts.get("gate", True), with_D=opts.get("D", True),
                with_h0=opts.get("h0", False))
    if not opts.get("bias", True):
        wl.dev["delta_bias"] = None
    softplus = opts.get("softplus", True)
    if not softplus:
        # without softplus the step is raw + bias as given: keep it positive
        # and moderate (the recipe's bias is negative, made for softplus)
        d = np.abs(wl.values("delta")) * np.float32(0.1)
        wl.dev["delta"] = (W.round_to_bf16_bits(d) if dtype == W.BF16 else d)
        wl.dev["delta_bias"] = np.full(48, 0.01, dtype=np.float32)
    y, h = run(scan, wl, softplus=softplus)
    yo, ho = oracle.scan(**oracle_inputs(wl), delta_softplus=softplus)
    assert_close(y, yo, dtype, "y")
    assert_close(h, ho, dtype, "h_last")


def test_explicit_zero_state_equals_null(scan):
    wl = W.make(2, batch=2, seqlen=600, dim=32)
    t = to_device(wl)
    y0, h0 = run(scan, wl, t=t)
    t["h0"] = torch.zeros((2, 32, 16), dtype=torch.float32, device="cuda")
    y1, h1 = run(scan, wl, t=t)
    assert np.array_equal(y0, y1) and np.array_equal(h0, h1)


def test_deterministic(scan):
    wl = W.make(3, batch=2, seqlen=1000, dim=64)
    t = to_device(wl)
    a = run(scan, wl, t=t)
    b = run(scan, wl, t=t)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_continuation_on_gpu(scan):
    """scan(L) == scan(first m) then scan(rest, h0 = its final state)."""
    wl = W.make(4, seqlen=3000, dim=16)
    t = to_device(wl)
    y, h = run(scan, wl, t=t)
    for m in (1, 255, 256, 257, 1024, 2999):
        head = {k: (v[:, :m].contiguous() if k in ("x", "delta", "z", "B", "C")
                    and v is not None else v) for k, v in t.items()}
        tail = {k: (v[:, m:].contiguous() if k in ("x", "delta", "z", "B", "C")
                    and v is not None else v) for k, v in t.items()}
        y1, h1 = run(scan, wl, t=head)
        tail["h0"] = torch.from_numpy(h1.astype(np.float32)).cuda()
        y2, h2 = run(scan, wl, t=tail)
        assert_close(np.concatenate([y1, y2], 1), y, W.F32, "y m=%d" % m)
        assert_close(h2, h, W.F32, "h_last m=%d" % m)


def test_freezing_is_exact(scan):
    """A zero step keeps the state bitwise (retention exactly 1, zero write)."""
    wl = W.make(1, batch=2, seqlen=300, dim=32, with_h0=True)
    wl.dev["delta"] = np.zeros_like(wl.dev["delta"])
    wl.dev["delta_bias"] = None
    y, h = run(scan, wl, softplus=False)
    assert np.array_equal(h, wl.dev["h0"].astype(np.float64))


def test_forgetting(scan):
    wl = W.make(1, batch=2, seqlen=300, dim=32, with_h0=True)
    wl.dev["A_log"] = np.full_like(wl.dev["A_log"], 50.0)
    y, h = run(scan, wl)
    yo, ho = oracle.scan(**oracle_inputs(wl))
    assert_close(y, yo, W.F32, "y")
    assert_close(h, ho, W.F32, "h_last")


def test_channel_permutation(scan):
    """Permuting the channels of every per-channel input (x, raw step, z, A
    rows, D, step bias) permutes the outputs bit for bit. Every channel has
    its own A row, so a read of another channel's A would show."""
    wl = W.make(3, batch=2, seqlen=700, dim=48, a_jitter=0.5)
    assert len({r.tobytes() for r in wl.dev["A_log"]}) == 48
    t = to_device(wl)
    y, h = run(scan, wl, t=t)
    perm = torch.from_numpy(np.random.default_rng(3).permutation(48)).cuda()
    tp = dict(t)
    for k in ("x", "delta", "z"):
        tp[k] = t[k][..., perm].contiguous()
    for k in ("A_log", "D", "delta_bias"):
        tp[k] = t[k][perm].contiguous()
    yp, hp = run(scan, wl, t=tp)
    pn = perm.cpu().numpy()
    assert np.array_equal(yp, y[..., pn]) and np.array_equal(hp, h[:, pn])


@pytest.mark.parametrize("N", [4, 16])
def test_sequential_shape_huge_A_freezes_and_forgets(scan, N):
    """A shape only the sequential variant runs (E * 4 bytes not a multiple
    of 16) with A_log = 100, so -exp(A_log) overflows float32 to -inf. A zero
    step must keep the state bitwise (retention 1, not 0 * -inf = NaN); a
    positive step must forget it (retention 0)."""
    wl = W.make(1, batch=2, seqlen=90, dim=42, dstate=N, with_h0=True)
    wl.dev["A_log"] = np.full_like(wl.dev["A_log"], 100.0)
    wl.dev["A_log"][::3] = 0.5                     # some channels ordinary
    wl.dev["delta"] = np.zeros_like(wl.dev["delta"])
    wl.dev["delta_bias"] = None
    y, h = run(scan, wl, softplus=False)
    assert scan.last_variant()[0] == S.SSM_VARIANT_SEQUENTIAL
    assert np.array_equal(h, wl.dev["h0"].astype(np.float64))
    yo, ho = oracle.scan(**oracle_inputs(wl), delta_softplus=False)
    assert_close(y, yo, W.F32, "y (zero step)")
    # positive steps: channels with A_log = 100 forget everything at once
    wl.dev["delta"] = np.full_like(wl.dev["delta"], 0.05)
    y, h = run(scan, wl, softplus=False)
    yo, ho = oracle.scan(**oracle_inputs(wl), delta_softplus=False)
    assert np.all(np.isfinite(y)) and np.all(np.isfinite(h))
    assert_close(y, yo, W.F32, "y (forgetting)")
    assert_close(h, ho, W.F32, "h_last (forgetting)")


def test_chunked_unsupported_shapes(scan):
    """A forced chunked variant reports shapes it cannot tile; AUTO falls
    back to the sequential variant for them."""
    wl = W.make(1, batch=1, seqlen=100, dim=42, dstate=16)   # E*4 % 16 != 0
    t = to_device(wl)
    _with_variant(scan, (S.SSM_VARIANT_CHUNKED, 1))
    try:
        with pytest.raises(S.SsmScanError) as ei:
            scan(t["x"], t["delta"], t["A_log"], t["B"], t["C"], D=t["D"],
                 z=t["z"], delta_bias=t["delta_bias"])
        assert ei.value.status == S.SSM_ERR_UNSUPPORTED
    finally:
        _with_variant(scan, S.SSM_VARIANT_AUTO)
    y, h = run(scan, wl, t=t)
    assert scan.last_variant()[0] == S.SSM_VARIANT_SEQUENTIAL
    yo, ho = oracle.scan(**oracle_inputs(wl))
    assert_close(y, yo, wl.dtype, "y")


def test_argument_errors(scan):
    wl = W.make(0)
    t = to_device(wl)
    h = scan.handle
    dims = (1, 64, 16, 4)
    args = lambda **kw: dict(dict(  # noqa: E731
        x=t["x"], delta=t["delta"], A_log=t["A_log"], B=t["B"], C=t["C"],
        D=t["D"], z=t["z"], delta_bias=t["delta_bias"], flags=1, h0=None,
        y=torch.empty_like(t["x"]), h_last=None, dims=dims,
        dtype=S.SSM_F32), **kw)

    def call(**kw):
        a = args(**kw)
        return S.ssm_scan_fwd(h, a["x"], a["delta"], a["A_log"], a["B"],
                              a["C"], a["D"], a["z"], a["delta_bias"],
                              a["flags"], a["h0"], a["y"], a["h_last"],
                              a["dims"], a["dtype"], check=False)
    assert call() == S.SSM_OK
    assert call(x=None) == S.SSM_ERR_INVALID
    assert call(y=None) == S.SSM_ERR_INVALID
    assert call(A_log=None) == S.SSM_ERR_INVALID
    assert call(dims=(0, 64, 16, 4)) == S.SSM_ERR_INVALID
    assert call(dims=(1, 0, 16, 4)) == S.SSM_ERR_INVALID
    assert call(dims=(1, 64, 16, 65)) == S.SSM_ERR_UNSUPPORTED
    assert call(dtype=7) == S.SSM_ERR_UNSUPPORTED
    assert call(flags=1 << 6) == S.SSM_ERR_INVALID            # unknown flag
    assert call(flags=S.SSM_REUSE_CHECKPOINTS) == S.SSM_ERR_INVALID  # bwd's
    assert call(x=t["x"].data_ptr() + 2) == S.SSM_ERR_ALIGN
    assert call(h0=t["A_log"].data_ptr() + 1) == S.SSM_ERR_ALIGN
    torch.cuda.synchronize()
    assert scan.sync_status() == S.SSM_OK


@pytest.mark.parametrize("idx,size", [
    (3, dict(batch=2, seqlen=1024, dim=64)),
    (3, dict(batch=4, seqlen=96, dim=4736)),   # enough tiles for 16-ch ones
    (2, dict(batch=3, seqlen=640, dim=96, dstate=8)),
    (1, dict(batch=2, seqlen=512, dim=64)),
    (0, dict(batch=2, seqlen=256, dim=32)),
], ids=["bf16_n16", "bf16_n16_many_tiles", "bf16_n8", "f32_n16", "f32_n4"])
@pytest.mark.parametrize("h0", [False, True], ids=["zero_state", "h0"])
def test_whole_tiles_and_windows(scan, idx, size, h0):
    """Shapes of whole channel tiles and whole windows with a gate and the
    softplus step: the launch takes the specialised kernel that tests none
    of those at run time. Per-channel A; against the oracle."""
    wl = W.make(idx, a_jitter=0.5, with_h0=h0, **size)
    y, h = run(scan, wl)
    assert tuple(scan.last_variant()) == (S.SSM_VARIANT_CHUNKED, 1)
    yo, ho = oracle.scan(**oracle_inputs(wl))
    assert_close(y, yo, wl.dtype, "y")
    assert_close(h, ho, wl.dtype, "h_last")
