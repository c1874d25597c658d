"""ssm_scan_fwd_static_scratch: the entry point for callers that cannot
allocate device memory, such as code running after a serving engine has
handed the whole device to its own memory pool, or a plug-in whose host fixes
its memory budget up front. Its split-sequence workspace is a fixed device
array of the library, so it never calls the allocator.

Each case calls it twice in a row through the C ABI and compares both calls
with the handle-based ssm_scan_fwd on the same inputs and with the float64
oracle, within the tolerance of the parity tests. The file is collected last,
and passes alone in a fresh process as well as after the other tests."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_51_b200 as S
from selective_state_space_51_b200 import workloads as W
from gpu_helpers import TOL, oracle_inputs, rel_err, to_device

pytestmark = pytest.mark.gpu


def _handle_reference(t, segments, flags):
    scan = S.SelectiveScan(0)
    try:
        scan.set_variant(S.SSM_VARIANT_CHUNKED, segments)
        y, h = scan(t["x"], t["delta"], t["A_log"], t["B"], t["C"], D=t["D"],
                    z=t["z"], delta_bias=t["delta_bias"], h0=t["h0"],
                    write_zoh=bool(flags & S.SSM_WRITE_ZOH))
        torch.cuda.synchronize()
        assert scan.sync_status() == S.SSM_OK
        return y.float().cpu().numpy(), h.cpu().numpy()
    finally:
        scan.close()


CASES = {
    # name: (workload, sizes, segments, caller status word, write flags)
    "long_f32_4pieces": (4, dict(seqlen=20000, dim=64), 4, True, 0),
    "layer_bf16_3pieces": (3, dict(batch=2, seqlen=6000, dim=48,
                                   with_h0=True), 3, True, 0),
    "long_f32_auto": (4, dict(seqlen=5000, dim=32), 0, True, 0),
    "n8_bf16_2pieces": (2, dict(batch=2, seqlen=4000, dim=32, dstate=8), 2,
                        True, 0),
    "n8_f32_3pieces": (1, dict(batch=1, seqlen=5000, dim=24, dstate=8), 3,
                       True, 0),
    "n4_f32_5pieces": (0, dict(batch=2, seqlen=6000, dim=16), 5, True, 0),
    "zoh_f32_3pieces": (4, dict(seqlen=7000, dim=32), 3, True,
                        S.SSM_WRITE_ZOH),
    "no_status_never_splits": (4, dict(seqlen=6000, dim=32), 0, False, 0),
    "unsplit_bf16": (3, dict(batch=2, seqlen=1500, dim=40), 1, True, 0),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_static_scratch_matches_fwd_and_oracle_twice(name):
    idx, size, segments, with_status, write = CASES[name]
    wl = W.make(idx, a_jitter=0.5, **size)
    t = to_device(wl)
    flags = S.SSM_DELTA_SOFTPLUS | write
    # with no status word the call runs unsplit: compare with that
    y_ref, h_ref = _handle_reference(t, segments if with_status else 1, flags)
    yo, ho = oracle.scan(**oracle_inputs(wl), delta_softplus=True,
                         write_zoh=bool(write))
    dtype = S.SSM_F32 if wl.dtype == W.F32 else S.SSM_BF16
    dims = (wl.batch, wl.seqlen, wl.dim, wl.dstate)
    status = (torch.zeros(1, dtype=torch.int32, device="cuda")
              if with_status else None)
    stream = torch.cuda.current_stream()
    for call in range(2):
        y = torch.empty_like(t["x"])
        h = torch.empty((wl.batch, wl.dim, wl.dstate), dtype=torch.float32,
                        device="cuda")
        S.ssm_scan_fwd_static_scratch(
            0, t["x"], t["delta"], t["A_log"], t["B"], t["C"], t["D"],
            t["z"], t["delta_bias"], flags, t["h0"], y, h, dims, dtype,
            segments=segments, status=status, stream=stream)
        torch.cuda.synchronize()
        if status is not None:
            assert int(status.item()) == 0, "a bounded wait gave up"
        yv, hv = y.float().cpu().numpy(), h.cpu().numpy()
        assert np.all(np.isfinite(yv)) and np.all(np.isfinite(hv))
        tol = TOL[wl.dtype]
        assert rel_err(yv, y_ref) <= tol, "call %d y vs ssm_scan_fwd" % call
        assert rel_err(hv, h_ref) <= tol, "call %d h_last vs ssm_scan_fwd" % call
        assert rel_err(yv, yo) <= tol, "call %d y vs oracle" % call
        assert rel_err(hv, ho) <= tol, "call %d h_last vs oracle" % call


def test_static_scratch_rejects_what_does_not_fit():
    """Asking for more pieces than the fixed array can hold is refused on the
    host with SSM_ERR_UNSUPPORTED (buffers are full size all the same); a
    forced split with no status word to report a given-up wait, and the
    checkpoint-saving flag, are refused with SSM_ERR_INVALID."""
    b, L, E, N = 1, 16 * 16 * 64, 4096, 16        # 16 pieces need ~12.6 MB
    x = torch.zeros((b, L, E), dtype=torch.float32, device="cuda")
    dl = torch.zeros_like(x)
    y = torch.empty_like(x)
    Bm = torch.zeros((b, L, N), dtype=torch.float32, device="cuda")
    A_log = torch.zeros((E, N), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = S.ssm_scan_fwd_static_scratch(
        0, x, dl, A_log, Bm, Bm, None, None, None, S.SSM_DELTA_SOFTPLUS,
        None, y, None, (b, L, E, N), S.SSM_F32, segments=16, status=status,
        check=False)
    assert rc == S.SSM_ERR_UNSUPPORTED
    rc = S.ssm_scan_fwd_static_scratch(
        0, x, dl, A_log, Bm, Bm, None, None, None, S.SSM_DELTA_SOFTPLUS,
        None, y, None, (b, L, E, N), S.SSM_F32, segments=2, status=None,
        check=False)
    assert rc == S.SSM_ERR_INVALID
    # no handle to keep checkpoints in
    rc = S.ssm_scan_fwd_static_scratch(
        0, x, dl, A_log, Bm, Bm, None, None, None,
        S.SSM_DELTA_SOFTPLUS | S.SSM_SAVE_CHECKPOINTS, None, y, None,
        (b, L, E, N), S.SSM_F32, segments=1, status=status, check=False)
    assert rc == S.SSM_ERR_INVALID
    torch.cuda.synchronize()
