"""CUDA-graph capture of the library's calls: a decode loop (the step with
its conv buffer) and an unsplit forward scan, captured once with
torch.cuda.graph and replayed, give the same bits as eager calls. The step
and unsplit scan entry points make no allocating or synchronising call, so a
serving loop can replay them without per-token launch overhead."""
import numpy as np
import pytest
import torch

import selective_state_space_51_b200 as S
from selective_state_space_51_b200 import workloads as W
from gpu_helpers import to_device

pytestmark = pytest.mark.gpu


def _decode_inputs(T=8, b=3, E=64, N=16, seed=5):
    wl = W.make(3, batch=b, seqlen=T, dim=E, dstate=N, with_h0=True, seed=seed)
    t = to_device(wl)
    w, cb = W.conv_params(E, 4)
    return wl, t, torch.from_numpy(w).cuda(), torch.from_numpy(cb).cuda()


def test_decode_loop_graph_replay_matches_eager():
    scan = S.SelectiveScan(0)
    try:
        T = 8
        wl, t, w, cb = _decode_inputs(T)
        b, E, N = wl.batch, wl.dim, wl.dstate
        per_t = {k: [t[k][:, i].contiguous() for i in range(T)]
                 for k in ("x", "delta", "z", "B", "C")}

        def run(state, conv, ys):
            for i in range(T):
                scan.step(per_t["x"][i], per_t["delta"][i], t["A_log"],
                          per_t["B"][i], per_t["C"][i], state, conv_state=conv,
                          conv_weight=w, conv_bias=cb, D=t["D"],
                          z=per_t["z"][i], delta_bias=t["delta_bias"],
                          y=ys[i])

        # eager
        st_e = t["h0"].clone()
        cv_e = torch.zeros((b, E, 4), dtype=torch.bfloat16, device="cuda")
        ys_e = [torch.empty((b, E), dtype=torch.bfloat16, device="cuda")
                for _ in range(T)]
        run(st_e, cv_e, ys_e)
        torch.cuda.synchronize()
        # captured once, replayed from the same starting buffers
        st_g = t["h0"].clone()
        cv_g = torch.zeros_like(cv_e)
        ys_g = [torch.empty_like(y) for y in ys_e]
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            run(st_g, cv_g, ys_g)
        st_g.copy_(t["h0"])
        cv_g.zero_()
        graph.replay()
        torch.cuda.synchronize()
        for i in range(T):
            assert torch.equal(ys_g[i], ys_e[i]), i
        assert torch.equal(st_g, st_e)
        assert torch.equal(cv_g, cv_e)
        # a second replay continues the sequence from the carried buffers
        graph.replay()
        run(st_e, cv_e, ys_e)
        torch.cuda.synchronize()
        assert torch.equal(st_g, st_e)
    finally:
        scan.close()


def test_scan_graph_replay_matches_eager():
    scan = S.SelectiveScan(0)
    try:
        scan.set_variant(S.SSM_VARIANT_CHUNKED, 1)  # unsplit: no workspace
        wl = W.make(1, batch=4, seqlen=700, dim=128)
        t = to_device(wl)
        y_e, h_e = scan(t["x"], t["delta"], t["A_log"], t["B"], t["C"],
                        D=t["D"], z=t["z"], delta_bias=t["delta_bias"])
        torch.cuda.synchronize()
        y_g = torch.empty_like(y_e)
        h_g = torch.empty_like(h_e)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            scan(t["x"], t["delta"], t["A_log"], t["B"], t["C"], D=t["D"],
                 z=t["z"], delta_bias=t["delta_bias"], y=y_g, h_last=h_g)
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(y_g, y_e) and torch.equal(h_g, h_e)
        assert scan.sync_status() == S.SSM_OK
    finally:
        scan.close()


def test_split_scan_graph_replays_with_new_inputs():
    """A split call (pieces joined by the look-back over publication flags)
    captured once and replayed after its input buffers were refilled: every
    replay must match the oracle on the inputs it saw, so no publication of
    an earlier replay can be taken for one of the current replay."""
    import oracle
    from gpu_helpers import assert_close, oracle_inputs
    scan = S.SelectiveScan(0)
    try:
        scan.set_variant(S.SSM_VARIANT_CHUNKED, 4)
        wls = [W.make(4, seqlen=6000, dim=32, a_jitter=0.5, seed=s)
               for s in (101, 202)]
        ts = [to_device(wl) for wl in wls]
        buf = {k: (None if v is None else v.clone())
               for k, v in ts[0].items()}
        y = torch.empty_like(buf["x"])
        h = torch.empty((1, 32, 16), dtype=torch.float32, device="cuda")

        def call():
            scan(buf["x"], buf["delta"], buf["A_log"], buf["B"], buf["C"],
                 D=buf["D"], z=buf["z"], delta_bias=buf["delta_bias"],
                 h0=buf["h0"], y=y, h_last=h)
        call()                       # grows the workspace before capture
        torch.cuda.synchronize()
        assert tuple(scan.last_variant()) == (S.SSM_VARIANT_CHUNKED, 4)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            call()
        for k in (1, 0, 1):
            for name, v in ts[k].items():
                if v is not None:
                    buf[name].copy_(v)
            graph.replay()
            torch.cuda.synchronize()
            assert scan.sync_status() == S.SSM_OK
            yo, ho = oracle.scan(**oracle_inputs(wls[k]))
            assert_close(y.cpu().numpy(), yo, W.F32, "y replay (inputs %d)" % k)
            assert_close(h.cpu().numpy(), ho, W.F32,
                         "h_last replay (inputs %d)" % k)
        del graph
    finally:
        scan.close()
