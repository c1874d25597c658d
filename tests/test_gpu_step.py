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


@pytest.mark.parametrize("dtype", [W.F32, W.BF16])
@pytest.mark.parametrize("N", [1, 3, 4, 8, 16, 32, 64])
@pytest.mark.parametrize("conv,zoh,gate", [(4, False, True), (0, False, True),
                                           (3, True, False), (1, False, False)],
                         ids=["conv4", "noconv", "conv3_zoh", "conv1_nogate"])
def test_step_parity(scan, dtype, N, conv, zoh, gate):
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
