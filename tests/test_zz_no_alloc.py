"""ssm_scan_fwd_static_scratch: the entry point for callers that cannot
allocate device memory (its split-sequence workspace is a fixed device array
of the library). Checked through the C ABI against the handle-based
ssm_scan_fwd on the same inputs, on two calls in a row, within the tolerance
of the parity tests. It lives in a file of its own that pytest collects last,
and passes alone in a fresh process as well as after the other tests."""
import numpy as np
import pytest
import torch

import selective_state_space_51_b200 as S
from selective_state_space_51_b200 import workloads as W
from gpu_helpers import TOL, rel_err, to_device

pytestmark = pytest.mark.gpu


def _handle_reference(t, wl, segments):
    scan = S.SelectiveScan(0)
    try:
        scan.set_variant(S.SSM_VARIANT_CHUNKED, segments)
        y, h = scan(t["x"], t["delta"], t["A_log"], t["B"], t["C"], D=t["D"],
                    z=t["z"], delta_bias=t["delta_bias"], h0=t["h0"])
        torch.cuda.synchronize()
        assert scan.sync_status() == S.SSM_OK
        return y.float().cpu().numpy(), h.cpu().numpy()
    finally:
        scan.close()


@pytest.mark.parametrize("idx,size,segments", [
    (4, dict(seqlen=20000, dim=64), 4),
    (3, dict(batch=2, seqlen=6000, dim=48, with_h0=True), 3),
    (4, dict(seqlen=5000, dim=32), 0),
], ids=["long_f32_4pieces", "layer_bf16_3pieces", "long_f32_auto"])
def test_static_scratch_matches_fwd_twice(idx, size, segments):
    wl = W.make(idx, **size)
    t = to_device(wl)
    y_ref, h_ref = _handle_reference(t, wl, segments)
    dtype = S.SSM_F32 if wl.dtype == W.F32 else S.SSM_BF16
    dims = (wl.batch, wl.seqlen, wl.dim, wl.dstate)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    for call in range(2):
        y = torch.empty_like(t["x"])
        h = torch.empty((wl.batch, wl.dim, wl.dstate), dtype=torch.float32,
                        device="cuda")
        S.ssm_scan_fwd_static_scratch(
            0, t["x"], t["delta"], t["A_log"], t["B"], t["C"], t["D"],
            t["z"], t["delta_bias"], S.SSM_DELTA_SOFTPLUS, t["h0"], y, h,
            dims, dtype, segments=segments, status=status, stream=stream)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, "a bounded wait gave up"
        yv, hv = y.float().cpu().numpy(), h.cpu().numpy()
        assert np.all(np.isfinite(yv))
        assert rel_err(yv, y_ref) <= TOL[wl.dtype], "call %d y" % call
        assert rel_err(hv, h_ref) <= TOL[wl.dtype], "call %d h_last" % call


def test_static_scratch_rejects_what_does_not_fit():
    """Asking for more pieces than the fixed array can hold is refused on the
    host with SSM_ERR_UNSUPPORTED (buffers are full size all the same)."""
    b, L, E, N = 1, 16 * 16 * 64, 4096, 16        # 16 pieces need ~12.6 MB
    x = torch.zeros((b, L, E), dtype=torch.float32, device="cuda")
    dl = torch.zeros_like(x)
    y = torch.empty_like(x)
    Bm = torch.zeros((b, L, N), dtype=torch.float32, device="cuda")
    A_log = torch.zeros((E, N), dtype=torch.float32, device="cuda")
    rc = S.ssm_scan_fwd_static_scratch(
        0, x, dl, A_log, Bm, Bm, None, None, None, S.SSM_DELTA_SOFTPLUS,
        None, y, None, (b, L, E, N), S.SSM_F32, segments=16, check=False)
    assert rc == S.SSM_ERR_UNSUPPORTED
    torch.cuda.synchronize()
