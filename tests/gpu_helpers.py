"""Shared helpers for the GPU parity tests: move a workload to the device,
run the library through its C ABI binding, compare with the oracle."""
import numpy as np
import torch

import selective_state_space_51_b200 as S
from selective_state_space_51_b200 import workloads as W

# Tolerances on max |gpu - oracle| / (1 + |oracle|), for y and h_last:
# 1e-4 for float32 activations, 2e-2 for bfloat16 (oracle on the same
# bfloat16-rounded inputs).
TOL = {W.F32: 1e-4, W.BF16: 2e-2}


def to_device(wl, device="cuda"):
    out = {}
    for k, v in wl.dev.items():
        if v is None:
            out[k] = None
        elif v.dtype == np.uint16:
            out[k] = torch.from_numpy(v.view(np.int16)).to(device).view(
                torch.bfloat16)
        else:
            out[k] = torch.from_numpy(np.ascontiguousarray(v)).to(device)
    return out


def run(scan, wl, t=None, softplus=None, with_h_last=True, write_zoh=False):
    t = to_device(wl) if t is None else t
    y, h_last = scan(t["x"], t["delta"], t["A_log"], t["B"], t["C"],
                     D=t["D"], z=t["z"], delta_bias=t["delta_bias"],
                     delta_softplus=wl.delta_softplus if softplus is None
                     else softplus,
                     h0=t["h0"], return_last_state=True, write_zoh=write_zoh)
    torch.cuda.synchronize()
    assert scan.sync_status() == S.SSM_OK
    yf = y.float().cpu().numpy().astype(np.float64)
    hf = h_last.cpu().numpy().astype(np.float64)
    return yf, hf


def oracle_inputs(wl):
    return dict(x=wl.values("x"), delta=wl.values("delta"),
                A_log=wl.dev["A_log"], B=wl.values("B"), C=wl.values("C"),
                D=wl.dev["D"], z=wl.values("z"),
                delta_bias=wl.dev["delta_bias"], h0=wl.dev["h0"])


def rel_err(a, ref):
    a = np.asarray(a, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(a - ref) / (1.0 + np.abs(ref))))


def assert_close(a, ref, dtype, what):
    err = rel_err(a, ref)
    assert np.all(np.isfinite(a)), "%s has non-finite values" % what
    assert err <= TOL[dtype], "%s: max rel err %.3e > %.1e" % (
        what, err, TOL[dtype])
    return err
