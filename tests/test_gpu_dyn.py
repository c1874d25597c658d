"""The specialised scan on persistent blocks: where the channel tiles do not
divide evenly over the SM schedulers, blocks take (tile, chunk of steps)
units in ticket order and hand the exact state from chunk to chunk. Its
results must equal the one-block-per-tile scan bit for bit (the arithmetic
per step is the same, and the carried state is stored and loaded as it is),
and the float64 oracle at the parity bar. A test hook forces the path on
small shapes with 64-step chunks."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_51_b200 as S
from selective_state_space_51_b200 import workloads as W
from gpu_helpers import TOL, oracle_inputs, rel_err, to_device

pytestmark = pytest.mark.gpu

FORCE_DYN = 1 << 2   # kDebugForceDyn: persistent blocks, 64-step chunks
NO_DYN = 1 << 3      # kDebugNoDyn: one block per tile
NO_PUBLISH = 1 << 0  # the first chunk of every tile leaves its state unpublished


@pytest.fixture(scope="module")
def scan():
    s = S.SelectiveScan(0)
    yield s
    s.close()


def _debug(scan, flags, spin=0):
    assert S.library().ssm_scan_set_debug(scan.handle, flags, spin) == S.SSM_OK


def _run(scan, t, flags):
    _debug(scan, flags)
    try:
        y, h = scan(t["x"], t["delta"], t["A_log"], t["B"], t["C"],
                    D=t["D"], z=t["z"], delta_bias=t["delta_bias"],
                    h0=t["h0"])
        torch.cuda.synchronize()
        assert scan.sync_status() == S.SSM_OK
        return y.clone(), h.clone()
    finally:
        _debug(scan, 0)


# whole 16-channel tiles and 32-step windows with a gate (the specialised
# path); lengths that end in a partial chunk; per-channel A; h0
CASES = {
    "bf16_L992": (3, dict(batch=2, seqlen=992, dim=64, a_jitter=0.5)),
    "bf16_L1024_h0": (3, dict(batch=3, seqlen=1024, dim=48, with_h0=True)),
    "bf16_n8_L480": (2, dict(batch=2, seqlen=480, dim=64, dstate=8)),
    "f32_L608": (1, dict(batch=2, seqlen=608, dim=64, a_jitter=0.5)),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_forced_chunks_match_one_block_per_tile_and_oracle(scan, name):
    idx, size = CASES[name]
    wl = W.make(idx, **size)
    t = to_device(wl)
    y1, h1 = _run(scan, t, NO_DYN)
    y2, h2 = _run(scan, t, FORCE_DYN)
    assert torch.equal(y2, y1) and torch.equal(h2, h1)
    inp = oracle_inputs(wl)
    ref_y, ref_h = oracle.scan(inp["x"], inp["delta"], inp["A_log"],
                               inp["B"], inp["C"], D=inp["D"], z=inp["z"],
                               delta_bias=inp["delta_bias"], h0=inp["h0"])
    assert rel_err(y2.float().cpu().numpy(), ref_y) <= TOL[wl.dtype]
    assert rel_err(h2.cpu().numpy(), ref_h) <= TOL[wl.dtype]


def test_uneven_tiles_take_the_persistent_path(scan):
    """8 sequences x 150 tiles = 1200 units for 148 x 8 two-warp workers:
    the shape the path is for, with its default chunks. Bitwise equal to one
    block per tile, and to the oracle on sampled channels."""
    wl = W.make(3, batch=8, seqlen=2048, dim=2400, a_jitter=0.5)
    t = to_device(wl)
    y1, h1 = _run(scan, t, NO_DYN)
    y2, h2 = _run(scan, t, 0)
    assert torch.equal(y2, y1) and torch.equal(h2, h1)
    ch = np.array([0, 15, 16, 1201, 2399])
    inp = oracle_inputs(wl)
    cut = lambda a: None if a is None else np.asarray(a)[..., ch]  # noqa
    ref_y, ref_h = oracle.scan(cut(inp["x"]), cut(inp["delta"]),
                               inp["A_log"][ch], inp["B"], inp["C"],
                               D=inp["D"][ch], z=cut(inp["z"]),
                               delta_bias=inp["delta_bias"][ch], h0=None)
    got = y2[..., torch.from_numpy(ch).cuda()].float().cpu().numpy()
    assert rel_err(got, ref_y) <= TOL[wl.dtype]
    assert rel_err(h2[:, torch.from_numpy(ch).cuda()].cpu().numpy(),
                   ref_h) <= TOL[wl.dtype]


def test_unpublished_chunk_times_out_and_recovers(scan):
    """With the first chunk of every tile unpublished, each successor's
    bounded wait runs out: the call reports SSM_ERR_TIMEOUT (and returns);
    the next call, without the hook, is correct again."""
    wl = W.make(3, batch=2, seqlen=256, dim=32)
    t = to_device(wl)
    y_ok, h_ok = _run(scan, t, NO_DYN)
    _debug(scan, FORCE_DYN | NO_PUBLISH, 2000)
    try:
        scan(t["x"], t["delta"], t["A_log"], t["B"], t["C"], D=t["D"],
             z=t["z"], delta_bias=t["delta_bias"])
        torch.cuda.synchronize()
        assert scan.sync_status() == S.SSM_ERR_TIMEOUT
    finally:
        _debug(scan, 0)
    y, h = _run(scan, t, FORCE_DYN)
    assert torch.equal(y, y_ok) and torch.equal(h, h_ok)


def test_forced_chunks_replay_in_a_graph(scan):
    """A persistent-block call captured once and replayed with new inputs
    matches the one-block-per-tile scan of each replay's inputs: the ticket
    and the hand-over flags are cleared on the stream before every launch."""
    wl = W.make(3, batch=2, seqlen=512, dim=64)
    t = to_device(wl)
    _debug(scan, FORCE_DYN)
    try:
        y = torch.empty_like(t["x"])
        h = torch.empty((wl.batch, wl.dim, wl.dstate), device="cuda")
        args = lambda: scan(t["x"], t["delta"], t["A_log"], t["B"], t["C"],  # noqa
                            D=t["D"], z=t["z"], delta_bias=t["delta_bias"],
                            y=y, h_last=h)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            args()                      # grows the workspace, outside capture
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            args()
        rng = np.random.Generator(np.random.PCG64(7))
        for _ in range(3):
            t["x"].copy_(torch.from_numpy(rng.standard_normal(
                tuple(t["x"].shape), dtype=np.float32)).to(t["x"].dtype))
            g.replay()
            torch.cuda.synchronize()
            assert scan.sync_status() == S.SSM_OK
            y_dyn, h_dyn = y.clone(), h.clone()
            y_ref, h_ref = _run(scan, t, NO_DYN)
            _debug(scan, FORCE_DYN)
            assert torch.equal(y_dyn, y_ref) and torch.equal(h_dyn, h_ref)
        del g
    finally:
        _debug(scan, 0)


def test_forced_chunks_with_the_fused_convolution(scan):
    """The convolution's 3-step halo comes from the previous chunk's inputs:
    the chunked run equals one block per tile bit for bit, and the oracle."""
    wl = W.make(3, batch=2, seqlen=992, dim=64, a_jitter=0.5)
    t = to_device(wl)
    w, cb = W.conv_params(wl.dim, 4)
    wt, cbt = torch.from_numpy(w).cuda(), torch.from_numpy(cb).cuda()
    outs = []
    for flags in (NO_DYN, FORCE_DYN):
        _debug(scan, flags)
        try:
            y, h = scan(t["x"], t["delta"], t["A_log"], t["B"], t["C"],
                        D=t["D"], z=t["z"], delta_bias=t["delta_bias"],
                        conv_weight=wt, conv_bias=cbt)
            torch.cuda.synchronize()
            assert scan.sync_status() == S.SSM_OK
            outs.append((y.clone(), h.clone()))
        finally:
            _debug(scan, 0)
    assert torch.equal(outs[1][0], outs[0][0])
    assert torch.equal(outs[1][1], outs[0][1])
    inp = oracle_inputs(wl)
    ref_y, ref_h = oracle.scan_conv(inp["x"], w, inp["delta"],
                                    inp["A_log"], inp["B"], inp["C"],
                                    conv_bias=cb, D=inp["D"], z=inp["z"],
                                    delta_bias=inp["delta_bias"])
    assert rel_err(outs[1][0].float().cpu().numpy(), ref_y) <= TOL[wl.dtype]
    assert rel_err(outs[1][1].cpu().numpy(), ref_h) <= TOL[wl.dtype]


def test_forced_chunks_keep_the_training_checkpoints(scan):
    """The checkpoint-saving forward on persistent blocks writes the same
    checkpoints: the backward that reuses them gives the gradients of the
    self-contained backward bit for bit (deterministic sums)."""
    wl = W.make(3, batch=2, seqlen=512, dim=64, a_jitter=0.5)
    t = to_device(wl)
    rng = np.random.Generator(np.random.PCG64(5))
    dy = torch.from_numpy(rng.standard_normal(
        (wl.batch, wl.seqlen, wl.dim), dtype=np.float32)).to(t["x"].dtype)
    dy = dy.cuda()
    kw = dict(D=t["D"], z=t["z"], delta_bias=t["delta_bias"],
              deterministic=True)
    own = scan.backward(t["x"], t["delta"], t["A_log"], t["B"], t["C"], dy,
                        **kw)
    own = {k: v.clone() for k, v in own.items() if v is not None}
    _debug(scan, FORCE_DYN)
    try:
        y, h = scan(t["x"], t["delta"], t["A_log"], t["B"], t["C"],
                    D=t["D"], z=t["z"], delta_bias=t["delta_bias"],
                    save_checkpoints=True)
        torch.cuda.synchronize()
        assert scan.sync_status() == S.SSM_OK
    finally:
        _debug(scan, 0)
    y_ref, h_ref = _run(scan, t, NO_DYN)
    assert torch.equal(y, y_ref) and torch.equal(h, h_ref)
    g = scan.backward(t["x"], t["delta"], t["A_log"], t["B"], t["C"], dy,
                      reuse_checkpoints=True, **kw)
    torch.cuda.synchronize()
    for k, v in own.items():
        assert torch.equal(g[k], v), k


BWD_CASES = {
    "bf16_L256": (3, dict(batch=2, seqlen=256, dim=64, a_jitter=0.5)),
    "f32_L160_h0": (1, dict(batch=2, seqlen=160, dim=64, with_h0=True)),
    "bf16_n8_L192": (2, dict(batch=2, seqlen=192, dim=64, dstate=8)),
}


def _bwd_all(scan, t, dy, dh, flags, zoh=False, det=True):
    _debug(scan, flags)
    try:
        g = scan.backward(t["x"], t["delta"], t["A_log"], t["B"], t["C"], dy,
                          D=t["D"], z=t["z"], delta_bias=t["delta_bias"],
                          h0=t["h0"], dh_last=dh, write_zoh=zoh,
                          deterministic=det)
        torch.cuda.synchronize()
        assert scan.sync_status() == S.SSM_OK
        return {k: v.clone() for k, v in g.items() if v is not None}
    finally:
        _debug(scan, 0)


def _incoming(wl, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    dy = rng.standard_normal((wl.batch, wl.seqlen, wl.dim), dtype=np.float32)
    dh = rng.standard_normal((wl.batch, wl.dim, wl.dstate), dtype=np.float32)
    if wl.dtype == W.BF16:
        bits = W.round_to_bf16_bits(dy)
        return (torch.from_numpy(bits.view(np.int16)).cuda()
                .view(torch.bfloat16), W.bf16_bits_to_f32(bits), dh)
    return torch.from_numpy(dy).cuda(), dy, dh


@pytest.mark.parametrize("zoh", [False, True], ids=["dtBx", "zoh"])
@pytest.mark.parametrize("name", sorted(BWD_CASES))
def test_backward_chunks_match_one_block_per_tile_and_oracle(scan, name, zoh):
    """The reverse sweep on persistent blocks (forced 4-window chunks, the
    sweep's adjoint and sums handed from each chunk to the earlier one):
    every gradient equal bit for bit to one block per tile (deterministic
    sums in both), and the oracle at the parity bar."""
    idx, size = BWD_CASES[name]
    wl = W.make(idx, **size)
    t = to_device(wl)
    dy, dy_val, dh = _incoming(wl, 41)
    dht = torch.from_numpy(dh).cuda()
    ref_gpu = _bwd_all(scan, t, dy, dht, NO_DYN, zoh)
    got = _bwd_all(scan, t, dy, dht, FORCE_DYN, zoh)
    assert got.keys() == ref_gpu.keys()
    for k in got:
        assert torch.equal(got[k], ref_gpu[k]), k
    inp = oracle_inputs(wl)
    ref = oracle.scan_bwd(inp["x"], inp["delta"], inp["A_log"], inp["B"],
                          inp["C"], dy_val, D=inp["D"], z=inp["z"],
                          delta_bias=inp["delta_bias"], h0=inp["h0"],
                          dh_last=dh, write_zoh=zoh)
    for k, v in got.items():
        assert rel_err(v.float().cpu().numpy(), ref[k]) <= TOL[wl.dtype], k


def test_backward_uneven_tiles_take_the_persistent_path(scan):
    """1200 tiles for 148 x 8 workers, default chunks: bit for bit the
    gradients of one block per tile (deterministic sums)."""
    wl = W.make(3, batch=8, seqlen=2048, dim=2400, a_jitter=0.5)
    t = to_device(wl)
    dy, _, dh = _incoming(wl, 43)
    dht = torch.from_numpy(dh).cuda()
    ref_gpu = _bwd_all(scan, t, dy, dht, NO_DYN)
    got = _bwd_all(scan, t, dy, dht, 0)
    for k in got:
        assert torch.equal(got[k], ref_gpu[k]), k


def test_backward_unpublished_chunk_times_out_and_recovers(scan):
    wl = W.make(3, batch=2, seqlen=256, dim=32)
    t = to_device(wl)
    dy, _, dh = _incoming(wl, 47)
    dht = torch.from_numpy(dh).cuda()
    ok = _bwd_all(scan, t, dy, dht, NO_DYN)
    _debug(scan, FORCE_DYN | NO_PUBLISH, 2000)
    try:
        scan.backward(t["x"], t["delta"], t["A_log"], t["B"], t["C"], dy,
                      D=t["D"], z=t["z"], delta_bias=t["delta_bias"],
                      dh_last=dht, deterministic=True)
        torch.cuda.synchronize()
        assert scan.sync_status() == S.SSM_ERR_TIMEOUT
    finally:
        _debug(scan, 0)
    again = _bwd_all(scan, t, dy, dht, FORCE_DYN)
    for k in ok:
        assert torch.equal(again[k], ok[k]), k
