"""The training pair: a forward that keeps the backward's state checkpoints
(SSM_SAVE_CHECKPOINTS) and a backward that starts from them
(SSM_REUSE_CHECKPOINTS). The forward's outputs are checked against the
float64 oracle, and the reused backward against both the oracle and the
backward that recomputes its own checkpoints."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_51_b200 as S
from selective_state_space_51_b200 import workloads as W
from gpu_helpers import TOL, oracle_inputs, rel_err, to_device

pytestmark = pytest.mark.gpu

SUMMED = ("dB", "dC", "dA_log", "dD", "ddelta_bias")


@pytest.fixture(scope="module")
def scan():
    s = S.SelectiveScan(0)
    yield s
    s.close()


def _incoming(wl, seed):
    """Seeded dy (activation dtype, rounded like the inputs) and dh_last."""
    b, L, E, N = wl.batch, wl.seqlen, wl.dim, wl.dstate
    rng = np.random.Generator(np.random.PCG64(seed))
    dy = rng.standard_normal((b, L, E), dtype=np.float32)
    dh = rng.standard_normal((b, E, N), dtype=np.float32)
    if wl.dtype == W.BF16:
        bits = W.round_to_bf16_bits(dy)
        dyt = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
        return dyt, W.bf16_bits_to_f32(bits), dh
    return torch.from_numpy(dy).cuda(), dy, dh


def _fwd(scan, t, zoh, save):
    y, hl = scan(t["x"], t["delta"], t["A_log"], t["B"], t["C"], D=t["D"],
                 z=t["z"], delta_bias=t["delta_bias"], h0=t["h0"],
                 write_zoh=zoh, save_checkpoints=save)
    return y, hl


def _bwd(scan, t, dyt, dht, zoh, reuse, det=False):
    return scan.backward(t["x"], t["delta"], t["A_log"], t["B"], t["C"], dyt,
                         D=t["D"], z=t["z"], delta_bias=t["delta_bias"],
                         h0=t["h0"], dh_last=dht, write_zoh=zoh,
                         reuse_checkpoints=reuse, deterministic=det)


def _host(g):
    return {k: v.float().cpu().numpy() for k, v in g.items() if v is not None}


def _same_gradients(a, b):
    """Per-element gradients bit for bit; the channel and step sums, added
    with float32 atomics in a varying order, to 1e-5 relative."""
    assert a.keys() == b.keys()
    for k in a:
        if k in SUMMED:
            assert rel_err(b[k], a[k]) <= 1e-5, k
        else:
            assert np.array_equal(b[k], a[k]), k


# whole tiles and windows with a gate (the specialised kernels), ragged
# shapes, both writes, N = 4, 8, 16, per-channel A
CASES = {
    "layer_bf16_whole": (3, dict(batch=2, seqlen=256, dim=64, a_jitter=0.5)),
    "layer_bf16_ragged": (3, dict(batch=2, seqlen=203, dim=40, with_h0=True)),
    "classifier_f32": (1, dict(batch=2, seqlen=150, dim=72, a_jitter=0.5)),
    "n8_bf16": (2, dict(batch=2, seqlen=96, dim=48, dstate=8)),
    "n4_f32_no_gate": (0, dict(batch=2, seqlen=100, dim=36, dstate=4,
                               gated=False)),
}


@pytest.mark.parametrize("zoh", [False, True], ids=["dtBx", "zoh"])
@pytest.mark.parametrize("name", sorted(CASES))
def test_train_pair(scan, name, zoh):
    idx, size = CASES[name]
    wl = W.make(idx, **size)
    t = to_device(wl)
    dyt, dy_val, dh = _incoming(wl, 17)
    dht = torch.from_numpy(dh).cuda()
    inp = oracle_inputs(wl)

    # the forward that keeps its checkpoints still returns the forward
    y, hl = _fwd(scan, t, zoh, save=True)
    torch.cuda.synchronize()
    ref_y, ref_h = oracle.scan(inp["x"], inp["delta"], inp["A_log"],
                               inp["B"], inp["C"], D=inp["D"], z=inp["z"],
                               delta_bias=inp["delta_bias"], h0=inp["h0"],
                               write_zoh=zoh)
    assert rel_err(y.float().cpu().numpy(), ref_y) <= TOL[wl.dtype]
    assert rel_err(hl.cpu().numpy(), ref_h) <= TOL[wl.dtype]

    g = _host(_bwd(scan, t, dyt, dht, zoh, reuse=True))
    ref = oracle.scan_bwd(inp["x"], inp["delta"], inp["A_log"], inp["B"],
                          inp["C"], dy_val, D=inp["D"], z=inp["z"],
                          delta_bias=inp["delta_bias"], h0=inp["h0"],
                          dh_last=dh, write_zoh=zoh)
    for k, v in g.items():
        assert rel_err(v, ref[k]) <= TOL[wl.dtype], k
    # the backward with its own checkpointing forward gives the same
    _same_gradients(g, _host(_bwd(scan, t, dyt, dht, zoh, reuse=False)))
    # and with deterministic sums, every gradient is the same bit for bit
    own = _host(scan.backward(t["x"], t["delta"], t["A_log"], t["B"],
                              t["C"], dyt, D=t["D"], z=t["z"],
                              delta_bias=t["delta_bias"], h0=t["h0"],
                              dh_last=dht, write_zoh=zoh, deterministic=True))
    _fwd(scan, t, zoh, save=True)
    reused = _host(scan.backward(t["x"], t["delta"], t["A_log"], t["B"],
                                 t["C"], dyt, D=t["D"], z=t["z"],
                                 delta_bias=t["delta_bias"], h0=t["h0"],
                                 dh_last=dht, write_zoh=zoh,
                                 reuse_checkpoints=True, deterministic=True))
    for k in own:
        assert np.array_equal(reused[k], own[k]), k


def test_train_pair_full_size(scan):
    """The Mamba-2.8B layer as the bench runs it: the reused backward equals
    the self-contained one bit for bit, every gradient (with deterministic
    sums: at this size the atomic sums of 320 channel tiles spread by about
    1e-5 run to run), and the forward's y equals the plain forward's bit for
    bit (same kernel arithmetic, checkpoints on the side)."""
    wl = W.make(3)
    t = to_device(wl)
    dyt, _, dh = _incoming(wl, 23)
    dht = torch.from_numpy(dh).cuda()
    y0, h0 = _fwd(scan, t, False, save=False)
    y0, h0 = y0.clone(), h0.clone()
    own = _host(_bwd(scan, t, dyt, dht, False, reuse=False, det=True))
    y1, h1 = _fwd(scan, t, False, save=True)
    torch.cuda.synchronize()
    assert torch.equal(y1, y0) and torch.equal(h1, h0)
    reused = _host(_bwd(scan, t, dyt, dht, False, reuse=True, det=True))
    assert own.keys() == reused.keys()
    for k in own:
        assert np.array_equal(reused[k], own[k]), k


def test_reuse_needs_matching_checkpoints(scan):
    """SSM_REUSE_CHECKPOINTS is refused (SSM_ERR_INVALID) without a saving
    forward for the same shape, dtype and flags, and after a backward
    without it has overwritten the checkpoints."""
    s = S.SelectiveScan(0)   # a fresh handle: nothing saved yet
    try:
        wl = W.make(1, batch=2, seqlen=64, dim=32)
        t = to_device(wl)
        dyt, _, dh = _incoming(wl, 3)
        dht = torch.from_numpy(dh).cuda()

        def refused(**kw):
            with pytest.raises(S.SsmScanError) as e:
                s.backward(t["x"], t["delta"], t["A_log"], t["B"], t["C"],
                           dyt, D=t["D"], z=t["z"],
                           delta_bias=t["delta_bias"], h0=t["h0"],
                           dh_last=dht, reuse_checkpoints=True, **kw)
            assert e.value.status == S.SSM_ERR_INVALID

        refused()                                  # nothing saved
        _fwd(s, t, False, save=True)
        refused(write_zoh=True)                    # other flags
        refused(delta_softplus=False)
        _bwd(s, t, dyt, dht, False, reuse=True)    # accepted
        _bwd(s, t, dyt, dht, False, reuse=False)   # overwrites them
        refused()
        # another shape
        _fwd(s, t, False, save=True)
        wl2 = W.make(1, batch=2, seqlen=48, dim=32)
        t2 = to_device(wl2)
        dy2, _, _ = _incoming(wl2, 4)
        with pytest.raises(S.SsmScanError) as e:
            s.backward(t2["x"], t2["delta"], t2["A_log"], t2["B"], t2["C"],
                       dy2, D=t2["D"], z=t2["z"],
                       delta_bias=t2["delta_bias"], h0=t2["h0"],
                       reuse_checkpoints=True)
        assert e.value.status == S.SSM_ERR_INVALID
        torch.cuda.synchronize()
    finally:
        s.close()


def test_save_checkpoints_argument_errors(scan):
    """The saving forward rejects the fused convolution (SSM_ERR_INVALID)
    and a forced sequential variant (SSM_ERR_UNSUPPORTED)."""
    wl = W.make(1, batch=1, seqlen=32, dim=32)
    t = to_device(wl)
    b, L, E, N = wl.batch, wl.seqlen, wl.dim, wl.dstate
    y = torch.empty_like(t["x"])
    w = torch.zeros((E, 4), device="cuda", dtype=torch.float32)
    flags = S.SSM_DELTA_SOFTPLUS | S.SSM_SAVE_CHECKPOINTS
    rc = S.ssm_scan_fwd_conv(scan.handle, t["x"], w, None, 4, t["delta"],
                             t["A_log"], t["B"], t["C"], t["D"], t["z"],
                             t["delta_bias"], flags, None, y, None,
                             (b, L, E, N), S.SSM_F32, check=False)
    assert rc == S.SSM_ERR_INVALID
    s = S.SelectiveScan(0)
    try:
        s.set_variant(S.SSM_VARIANT_SEQUENTIAL)
        rc = S.ssm_scan_fwd(s.handle, t["x"], t["delta"], t["A_log"],
                            t["B"], t["C"], t["D"], t["z"], t["delta_bias"],
                            flags, None, y, None, (b, L, E, N), S.SSM_F32,
                            check=False)
        assert rc == S.SSM_ERR_UNSUPPORTED
    finally:
        s.close()
    torch.cuda.synchronize()
