"""GPU parity of the batched decode step (ssm_scan_step) against the float64
oracle's decode step, over several consecutive tokens, and against the
chunked scan of the same sequence."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_51_b200 as S
from selective_state_space_51_b200 import workloads as W
from gpu_helpers import TOL, assert_close, rel_err, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def scan():
    s = S.SelectiveScan(0)
    yield s
    s.close()


def _dev(a, dtype):
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()
    return t.to(torch.bfloat16) if dtype == W.BF16 else t


def _host(t):
    return t.float().cpu().numpy().astype(np.float64)


# N = 4, 8, 16 run the bulk-copy kernel unless the per-thread-load kernel is
# asked for (debug flag 2); the other N always run the per-thread kernel.
KERNELS = {"bulk": 0, "per_thread": 2}


@pytest.mark.parametrize("kernel", sorted(KERNELS))
@pytest.mark.parametrize("dtype", [W.F32, W.BF16])
@pytest.mark.parametrize("N", [1, 3, 4, 8, 16, 32, 64])
@pytest.mark.parametrize("conv,zoh,gate", [(4, False, True), (0, False, True),
                                           (3, True, False), (1, False, False)],
                         ids=["conv4", "noconv", "conv3_zoh", "conv1_nogate"])
def test_step_parity(scan, dtype, N, conv, zoh, gate, kernel):
    if kernel == "per_thread" and N not in (4, 8, 16):
        pytest.skip("only one kernel runs this state size")
    S.library().ssm_scan_set_debug(scan.handle, KERNELS[kernel], 0)
    try:
        _step_parity(scan, dtype, N, conv, zoh, gate)
    finally:
        S.library().ssm_scan_set_debug(scan.handle, 0, 0)


def _step_parity(scan, dtype, N, conv, zoh, gate):
    rng = np.random.default_rng(N * 7 + conv)
    b, E, T = 5, 40, 6
    # every channel has its own A row (A is a learned [E, N] parameter)
    wl = W.make(3, batch=b, seqlen=T, dim=E, dstate=N, dtype=dtype,
                gated=gate, with_h0=True, a_jitter=0.5)
    vals = {k: wl.values(k) for k in ("x", "delta", "z", "B", "C")}
    state_h = wl.dev["h0"].astype(np.float64)
    state = torch.from_numpy(wl.dev["h0"].copy()).cuda()
    cw = rng.standard_normal((E, conv)).astype(np.float32) if conv else None
    cb = rng.standard_normal(E).astype(np.float32) if conv else None
    conv_h = rng.standard_normal((b, E, conv)) if conv else None
    if conv:   # the buffer lives in the activation type
        conv_h = conv_h.astype(np.float32).astype(np.float64)
        if dtype == W.BF16:
            conv_h = W.bf16_bits_to_f32(W.round_to_bf16_bits(
                conv_h.astype(np.float32))).astype(np.float64)
    conv_t = _dev(conv_h, dtype) if conv else None
    A_log = torch.from_numpy(wl.dev["A_log"]).cuda()
    D = torch.from_numpy(wl.dev["D"]).cuda()
    bias = torch.from_numpy(wl.dev["delta_bias"]).cuda()
    cw_t = torch.from_numpy(cw).cuda() if conv else None
    cb_t = torch.from_numpy(cb).cuda() if conv else None
    for t in range(T):
        xt = _dev(vals["x"][:, t], dtype)
        dt = _dev(vals["delta"][:, t], dtype)
        zt = _dev(vals["z"][:, t], dtype) if gate else None
        Bt = _dev(vals["B"][:, t], dtype)
        Ct = _dev(vals["C"][:, t], dtype)
        y = scan.step(xt, dt, A_log, Bt, Ct, state, conv_state=conv_t,
                      conv_weight=cw_t, conv_bias=cb_t, D=D, z=zt,
                      delta_bias=bias, write_zoh=zoh)
        torch.cuda.synchronize()
        yo, state_h, conv_h = oracle.step(
            vals["x"][:, t], vals["delta"][:, t], wl.dev["A_log"],
            vals["B"][:, t], vals["C"][:, t], state_h, conv_state=conv_h,
            conv_weight=cw, conv_bias=cb, D=wl.dev["D"],
            z=vals["z"][:, t] if gate else None,
            delta_bias=wl.dev["delta_bias"], write_zoh=zoh)
        assert_close(_host(y), yo, dtype, "y token %d" % t)
        assert_close(state.cpu().numpy(), state_h, dtype, "state token %d" % t)
        if conv:
            # the buffer holds copies of the inputs: exact
            assert np.array_equal(_host(conv_t), conv_h), "conv buffer %d" % t


def test_decoding_matches_the_scan(scan):
    """Token-by-token decoding (no convolution) equals the chunked scan."""
    wl = W.make(1, batch=3, seqlen=200, dim=64, with_h0=True, a_jitter=0.5)
    t = to_device(wl)
    y_scan, h_scan = scan(t["x"], t["delta"], t["A_log"], t["B"], t["C"],
                          D=t["D"], z=t["z"], delta_bias=t["delta_bias"],
                          h0=t["h0"])
    state = t["h0"].clone()
    ys = []
    for k in range(200):
        ys.append(scan.step(t["x"][:, k].contiguous(),
                            t["delta"][:, k].contiguous(), t["A_log"],
                            t["B"][:, k].contiguous(),
                            t["C"][:, k].contiguous(), state, D=t["D"],
                            z=t["z"][:, k].contiguous(),
                            delta_bias=t["delta_bias"]))
    torch.cuda.synchronize()
    y_dec = torch.stack(ys, 1)
    assert rel_err(_host(y_dec), _host(y_scan)) <= TOL[W.F32]
    assert rel_err(_host(state), _host(h_scan)) <= TOL[W.F32]


def test_step_argument_errors(scan):
    b, E, N = 2, 8, 4
    x = torch.zeros((b, E), device="cuda")
    st = torch.zeros((b, E, N), device="cuda")
    A = torch.zeros((E, N), device="cuda")
    Bm = torch.zeros((b, N), device="cuda")
    y = torch.empty_like(x)
    conv = torch.zeros((b, E, 4), device="cuda")
    w = torch.zeros((E, 4), device="cuda")
    h = scan.handle

    def call(**kw):
        a = dict(x_new=x, conv_state=None, conv_weight=None, conv_bias=None,
                 conv_width=0, delta=x, delta_bias=None, A_log=A, B=Bm, C=Bm,
                 D=None, z=None, flags=1, state=st, y=y, dims=(b, 1, E, N),
                 dtype=S.SSM_F32)
        a.update(kw)
        return S.ssm_scan_step(h, a["x_new"], a["conv_state"],
                               a["conv_weight"], a["conv_bias"],
                               a["conv_width"], a["delta"], a["delta_bias"],
                               a["A_log"], a["B"], a["C"], a["D"], a["z"],
                               a["flags"], a["state"], a["y"], a["dims"],
                               a["dtype"], check=False)
    assert call() == S.SSM_OK
    assert call(state=None) == S.SSM_ERR_INVALID
    assert call(dims=(b, 2, E, N)) == S.SSM_ERR_INVALID
    assert call(conv_state=conv, conv_width=4) == S.SSM_ERR_INVALID
    assert call(conv_state=conv, conv_weight=w, conv_width=9) == \
        S.SSM_ERR_INVALID
    assert call(conv_state=conv, conv_weight=w, conv_width=4) == S.SSM_OK
    assert call(flags=4) == S.SSM_ERR_INVALID
    assert call(dims=(b, 1, E, 65)) == S.SSM_ERR_UNSUPPORTED
    assert call(state=st.data_ptr() + 2) == S.SSM_ERR_ALIGN
    torch.cuda.synchronize()
    assert scan.sync_status() == S.SSM_OK


@pytest.mark.parametrize("dtype", [W.F32, W.BF16])
def test_step_bulk_many_rows_and_ragged_channels(scan, dtype):
    """The bulk-copy kernel over more batch rows than resident blocks (each
    block walks several rows through its two buffers) and a ragged last
    block of channels (E not a multiple of 128): two tokens against the
    oracle, and against the per-thread-load kernel (the state bit for bit;
    y differs only in the order of the readout sum)."""
    b, E, N = 300, 200, 16
    wl = W.make(3, batch=b, seqlen=2, dim=E, dstate=N, dtype=dtype,
                with_h0=True, a_jitter=0.5)
    vals = {k: wl.values(k) for k in ("x", "delta", "z", "B", "C")}
    A_log = torch.from_numpy(wl.dev["A_log"]).cuda()
    D = torch.from_numpy(wl.dev["D"]).cuda()
    bias = torch.from_numpy(wl.dev["delta_bias"]).cuda()
    outs = {}
    for kernel, flag in KERNELS.items():
        S.library().ssm_scan_set_debug(scan.handle, flag, 0)
        try:
            state = torch.from_numpy(wl.dev["h0"].copy()).cuda()
            state_h = wl.dev["h0"].astype(np.float64)
            ys = []
            for t in range(2):
                y = scan.step(_dev(vals["x"][:, t], dtype),
                              _dev(vals["delta"][:, t], dtype), A_log,
                              _dev(vals["B"][:, t], dtype),
                              _dev(vals["C"][:, t], dtype), state, D=D,
                              z=_dev(vals["z"][:, t], dtype), delta_bias=bias)
                torch.cuda.synchronize()
                assert scan.sync_status() == S.SSM_OK
                yo, state_h, _ = oracle.step(
                    vals["x"][:, t], vals["delta"][:, t], wl.dev["A_log"],
                    vals["B"][:, t], vals["C"][:, t], state_h, D=wl.dev["D"],
                    z=vals["z"][:, t], delta_bias=wl.dev["delta_bias"])
                assert_close(_host(y), yo, dtype, "%s y token %d" % (kernel, t))
                assert_close(state.cpu().numpy(), state_h, dtype,
                             "%s state token %d" % (kernel, t))
                ys.append(_host(y))
            outs[kernel] = (ys, state.cpu().numpy())
        finally:
            S.library().ssm_scan_set_debug(scan.handle, 0, 0)
    for t in range(2):
        assert rel_err(outs["bulk"][0][t], outs["per_thread"][0][t]) <= \
            TOL[dtype]
    assert np.array_equal(outs["bulk"][1], outs["per_thread"][1])


def test_step_bulk_short_wait_limit_reports_and_recovers(scan):
    """With the bounded wait cut to a single poll, a wait for a state copy
    may give up: the call then reports SSM_ERR_TIMEOUT through the status
    word (the block drains its copies before it exits) and the context stays
    usable: the next call with the normal limit is correct."""
    b, E, N = 512, 1024, 16
    wl = W.make(3, batch=b, seqlen=1, dim=E, dstate=N, with_h0=True)
    t = {k: (None if v is None else v) for k, v in to_device(wl).items()}
    flat = {k: t[k][:, 0].contiguous() for k in ("x", "delta", "z", "B", "C")}
    state = t["h0"].clone()
    S.library().ssm_scan_set_debug(scan.handle, 0, 1)
    try:
        scan.step(flat["x"], flat["delta"], t["A_log"], flat["B"], flat["C"],
                  state, D=t["D"], z=flat["z"], delta_bias=t["delta_bias"])
        rc = scan.sync_status()
        assert rc in (S.SSM_OK, S.SSM_ERR_TIMEOUT)
    finally:
        S.library().ssm_scan_set_debug(scan.handle, 0, 0)
    assert scan.sync_status() == S.SSM_OK
    state = t["h0"].clone()
    y = scan.step(flat["x"], flat["delta"], t["A_log"], flat["B"], flat["C"],
                  state, D=t["D"], z=flat["z"], delta_bias=t["delta_bias"])
    torch.cuda.synchronize()
    assert scan.sync_status() == S.SSM_OK
    vals = {k: wl.values(k)[:, 0] for k in ("x", "delta", "z", "B", "C")}
    yo, so, _ = oracle.step(vals["x"], vals["delta"], wl.dev["A_log"],
                            vals["B"], vals["C"],
                            wl.dev["h0"].astype(np.float64), D=wl.dev["D"],
                            z=vals["z"], delta_bias=wl.dev["delta_bias"])
    assert_close(_host(y), yo, wl.dtype, "y after recovery")
    assert_close(state.cpu().numpy(), so, wl.dtype, "state after recovery")
