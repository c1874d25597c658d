"""GPU parity of the backward pass (ssm_scan_bwd) against the float64
oracle's scan_bwd (itself pinned by finite differences of the forward)."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_51_b200 as S
from selective_state_space_51_b200 import workloads as W
from gpu_helpers import TOL, oracle_inputs, rel_err, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def scan():
    s = S.SelectiveScan(0)
    yield s
    s.close()


def _grads(dtype, shape, seed):
    """Seeded incoming gradients: dy in the activation dtype (rounded like
    the inputs), dh_last in float32."""
    rng = np.random.Generator(np.random.PCG64(seed))
    dy = rng.standard_normal(shape[0], dtype=np.float32)
    dh = rng.standard_normal(shape[1], dtype=np.float32)
    if dtype == W.BF16:
        bits = W.round_to_bf16_bits(dy)
        return bits, W.bf16_bits_to_f32(bits), dh
    return dy, dy, dh


def _dev(a):
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(a).cuda()


def _check(scan, wl, write_zoh=False, with_dh=True, seed=5):
    t = to_device(wl)
    b, L, E, N = wl.batch, wl.seqlen, wl.dim, wl.dstate
    dy_dev, dy_val, dh = _grads(wl.dtype, ((b, L, E), (b, E, N)), seed)
    dyt = _dev(dy_dev)
    dht = torch.from_numpy(dh).cuda() if with_dh else None
    g = scan.backward(t["x"], t["delta"], t["A_log"], t["B"], t["C"], dyt,
                      D=t["D"], z=t["z"], delta_bias=t["delta_bias"],
                      h0=t["h0"], dh_last=dht, write_zoh=write_zoh)
    torch.cuda.synchronize()
    inp = oracle_inputs(wl)
    ref = oracle.scan_bwd(inp["x"], inp["delta"], inp["A_log"], inp["B"],
                          inp["C"], dy_val, D=inp["D"], z=inp["z"],
                          delta_bias=inp["delta_bias"], h0=inp["h0"],
                          dh_last=dh if with_dh else None,
                          write_zoh=write_zoh)
    errs = {}
    for k, v in g.items():
        if v is None:
            assert ref[k] is None, k
            continue
        got = v.float().cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(got)), "%s has non-finite values" % k
        errs[k] = rel_err(got, ref[k])
    bad = {k: e for k, e in errs.items() if e > TOL[wl.dtype]}
    assert not bad, "gradients off: %s (all: %s)" % (bad, errs)
    return errs


# several 16-step windows, a ragged tail and a ragged channel tile
CASES = {
    "classifier_f32": (1, dict(batch=2, seqlen=203, dim=72)),
    "layer_bf16": (3, dict(batch=2, seqlen=333, dim=40, with_h0=True)),
    "long_f32": (4, dict(seqlen=1500, dim=32)),
    "tiny_n4_f32": (0, dict()),
    "n8_bf16": (2, dict(batch=2, seqlen=150, dim=48, dstate=8)),
    "n8_f32_ragged": (1, dict(batch=3, seqlen=17, dim=24, dstate=8)),
    "n4_f32_ragged": (0, dict(batch=2, seqlen=100, dim=36, dstate=4)),
}


@pytest.mark.parametrize("jitter", [0.0, 0.5], ids=["A_stated",
                                                    "A_per_channel"])
@pytest.mark.parametrize("zoh", [False, True], ids=["dtBx", "zoh"])
@pytest.mark.parametrize("name", sorted(CASES))
def test_bwd_parity(scan, name, zoh, jitter):
    idx, size = CASES[name]
    _check(scan, W.make(idx, a_jitter=jitter, **size), write_zoh=zoh)


@pytest.mark.parametrize("idx,size", [
    (3, dict(batch=2, seqlen=4096, dim=2048)),
    (1, dict(batch=2, seqlen=2048, dim=2048)),
], ids=["layer_bf16_E2048_L4096", "classifier_f32_E2048_L2048"])
def test_bwd_channel_sums_many_tiles(scan, idx, size):
    """dB and dC sum over every channel, dA_log, dD and the step-bias
    gradient over every step and sequence: here 128 channel tiles add into
    each dB/dC row and 2 x L steps into each parameter gradient. All of them,
    and every per-element gradient, against the oracle at the parity bar."""
    errs = _check(scan, W.make(idx, a_jitter=0.5, **size), seed=21)
    for k in ("dB", "dC", "dA_log", "dD", "ddelta_bias"):
        assert k in errs, k


def test_bwd_run_to_run(scan):
    """The per-element gradients are the same bit for bit on every run. The
    summed ones (dB, dC, dA_log, dD, step bias) are added with float32
    atomics, whose order varies from run to run: their spread is bounded
    far inside the parity bar."""
    wl = W.make(3, batch=2, seqlen=2048, dim=1024, a_jitter=0.5)
    t = to_device(wl)
    b, L, E, N = wl.batch, wl.seqlen, wl.dim, wl.dstate
    dy_dev, _, dh = _grads(wl.dtype, ((b, L, E), (b, E, N)), 3)
    dyt, dht = _dev(dy_dev), torch.from_numpy(dh).cuda()
    runs = []
    for _ in range(3):
        g = scan.backward(t["x"], t["delta"], t["A_log"], t["B"], t["C"],
                          dyt, D=t["D"], z=t["z"], delta_bias=t["delta_bias"],
                          h0=t["h0"], dh_last=dht)
        torch.cuda.synchronize()
        runs.append({k: v.float().cpu().numpy() for k, v in g.items()
                     if v is not None})
    for k in runs[0]:
        for r in runs[1:]:
            if k in ("dB", "dC", "dA_log", "dD", "ddelta_bias"):
                assert rel_err(r[k], runs[0][k]) <= 1e-5, k
            else:
                assert np.array_equal(r[k], runs[0][k]), k


@pytest.mark.parametrize("opts", [dict(gated=False), dict(with_D=False),
                                  dict(with_h0=False)],
                         ids=["no_gate", "no_D", "no_h0"])
def test_bwd_optional_inputs(scan, opts):
    wl = W.make(1, batch=2, seqlen=130, dim=40, **opts)
    _check(scan, wl)


def test_bwd_no_dh_last_no_bias(scan):
    wl = W.make(4, seqlen=300, dim=32)     # no step bias, no gate
    _check(scan, wl, with_dh=False)


@pytest.mark.parametrize("L", [1, 15, 16, 17])
def test_bwd_short_sequences(scan, L):
    _check(scan, W.make(1, batch=2, seqlen=L, dim=32))


def test_bwd_full_size_sampled(scan):
    """The Mamba-2.8B layer at full size: the per-channel gradients of a
    sample of channels against the oracle on those channels (channels are
    independent). dB and dC, sums over every channel, are finite here; they
    are compared with the oracle where 128 channel tiles add into them in
    test_bwd_channel_sums_many_tiles."""
    wl = W.make(3)
    t = to_device(wl)
    b, L, E, N = wl.batch, wl.seqlen, wl.dim, wl.dstate
    dy_dev, dy_val, dh = _grads(wl.dtype, ((b, L, E), (b, E, N)), 9)
    dyt = _dev(dy_dev)
    g = scan.backward(t["x"], t["delta"], t["A_log"], t["B"], t["C"], dyt,
                      D=t["D"], z=t["z"], delta_bias=t["delta_bias"],
                      h0=t["h0"], dh_last=torch.from_numpy(dh).cuda())
    torch.cuda.synchronize()
    ch = np.array([0, 1, 777, 2500, E - 1])
    sel = torch.from_numpy(ch).cuda()
    got = {k: g[k][..., sel].float().cpu().numpy()
           for k in ("dx", "ddelta", "dz")}
    got["dA_log"] = g["dA_log"][sel].cpu().numpy()
    got["dD"] = g["dD"][sel].cpu().numpy()
    got["ddelta_bias"] = g["ddelta_bias"][sel].cpu().numpy()
    got["dh0"] = g["dh0"][:, sel].cpu().numpy()
    assert torch.isfinite(g["dB"]).all() and torch.isfinite(g["dC"]).all()
    del g, t
    inp = oracle_inputs(wl)
    cut = lambda a: None if a is None else np.asarray(a)[..., ch]  # noqa
    ref = oracle.scan_bwd(cut(inp["x"]), cut(inp["delta"]),
                          inp["A_log"][ch], inp["B"], inp["C"],
                          dy_val[..., ch], D=inp["D"][ch], z=cut(inp["z"]),
                          delta_bias=inp["delta_bias"][ch],
                          h0=None, dh_last=dh[:, ch])
    for k, v in got.items():
        assert rel_err(v, ref[k]) <= TOL[wl.dtype], k


def test_bwd_argument_errors(scan):
    b, L, E, N = 1, 32, 16, 4
    f = dict(device="cuda", dtype=torch.float32)
    x = torch.zeros((b, L, E), **f)
    A = torch.zeros((E, N), **f)
    Bm = torch.zeros((b, L, N), **f)
    dA = torch.empty((E, N), **f)
    dB = torch.empty((b, L, N), **f)
    out = torch.empty_like(x)
    dims = (b, L, E, N)

    def call(**kw):
        a = dict(x=x, z=None, D=None, dz=None, dD=None, dy=x, dims=dims,
                 dtype=S.SSM_F32, dB=dB)
        a.update(kw)
        return S.ssm_scan_bwd(scan.handle, a["x"], x, A, Bm, Bm, a["D"],
                              a["z"], None, 1, None, a["dy"], None, out, out,
                              dA, a["dB"], dB.clone(), a["dD"], a["dz"], None,
                              None, a["dims"], a["dtype"], check=False)
    assert call() == S.SSM_OK
    assert call(dy=None) == S.SSM_ERR_INVALID
    assert call(z=x) == S.SSM_ERR_INVALID              # z without dz
    assert call(D=torch.zeros(E, **f)) == S.SSM_ERR_INVALID  # D without dD
    assert call(dims=(b, L, E, 5)) == S.SSM_ERR_UNSUPPORTED
    assert call(dims=(b, L, 6, N)) == S.SSM_ERR_UNSUPPORTED  # 24-byte rows
    assert call(dtype=S.SSM_BF16) == S.SSM_ERR_UNSUPPORTED   # N=4 bf16
    # dB and dC take 16-byte atomic adds: rejected before any launch
    assert call(dB=dB.data_ptr() + 4) == S.SSM_ERR_ALIGN
    torch.cuda.synchronize()


DET_CASES = {
    "layer_bf16_whole": (3, dict(batch=2, seqlen=256, dim=64, a_jitter=0.5)),
    "layer_bf16_ragged": (3, dict(batch=2, seqlen=203, dim=40, with_h0=True)),
    "classifier_f32": (1, dict(batch=2, seqlen=203, dim=72, a_jitter=0.5)),
    "n8_bf16": (2, dict(batch=2, seqlen=150, dim=48, dstate=8)),
    "n4_f32_ragged": (0, dict(batch=2, seqlen=100, dim=36, dstate=4)),
}


@pytest.mark.parametrize("zoh", [False, True], ids=["dtBx", "zoh"])
@pytest.mark.parametrize("name", sorted(DET_CASES))
def test_bwd_deterministic(scan, name, zoh):
    """SSM_DETERMINISTIC: every gradient, the channel and step sums
    included, is the same bit for bit on every run; the gradients match the
    oracle at the parity bar, and the per-element ones equal the atomic
    path's bit for bit."""
    idx, size = DET_CASES[name]
    wl = W.make(idx, **size)
    t = to_device(wl)
    b, L, E, N = wl.batch, wl.seqlen, wl.dim, wl.dstate
    dy_dev, dy_val, dh = _grads(wl.dtype, ((b, L, E), (b, E, N)), 31)
    dyt, dht = _dev(dy_dev), torch.from_numpy(dh).cuda()

    def run(det):
        g = scan.backward(t["x"], t["delta"], t["A_log"], t["B"], t["C"],
                          dyt, D=t["D"], z=t["z"], delta_bias=t["delta_bias"],
                          h0=t["h0"], dh_last=dht, write_zoh=zoh,
                          deterministic=det)
        torch.cuda.synchronize()
        return {k: v.float().cpu().numpy() for k, v in g.items()
                if v is not None}

    runs = [run(True) for _ in range(3)]
    for k in runs[0]:
        for r in runs[1:]:
            assert np.array_equal(r[k], runs[0][k]), k
    inp = oracle_inputs(wl)
    ref = oracle.scan_bwd(inp["x"], inp["delta"], inp["A_log"], inp["B"],
                          inp["C"], dy_val, D=inp["D"], z=inp["z"],
                          delta_bias=inp["delta_bias"], h0=inp["h0"],
                          dh_last=dh, write_zoh=zoh)
    for k, v in runs[0].items():
        assert rel_err(v, ref[k]) <= TOL[wl.dtype], k
    atomic = run(False)
    for k, v in runs[0].items():
        if k in ("dB", "dC", "dA_log", "dD", "ddelta_bias"):
            assert rel_err(v, atomic[k]) <= 1e-5, k
        else:
            assert np.array_equal(v, atomic[k]), k


def test_bwd_deterministic_many_tiles(scan):
    """64 channel tiles per sum: the deterministic sums repeat bit for bit
    and agree with the atomic ones to 1e-5."""
    wl = W.make(3, batch=2, seqlen=2048, dim=1024, a_jitter=0.5)
    t = to_device(wl)
    b, L, E, N = wl.batch, wl.seqlen, wl.dim, wl.dstate
    dy_dev, _, dh = _grads(wl.dtype, ((b, L, E), (b, E, N)), 3)
    dyt, dht = _dev(dy_dev), torch.from_numpy(dh).cuda()
    runs = []
    for det in (True, True, False):
        g = scan.backward(t["x"], t["delta"], t["A_log"], t["B"], t["C"],
                          dyt, D=t["D"], z=t["z"], delta_bias=t["delta_bias"],
                          h0=t["h0"], dh_last=dht, deterministic=det)
        torch.cuda.synchronize()
        runs.append({k: v.float().cpu().numpy() for k, v in g.items()
                     if v is not None})
    for k in runs[0]:
        assert np.array_equal(runs[1][k], runs[0][k]), k
        assert rel_err(runs[0][k], runs[2][k]) <= 1e-5, k
