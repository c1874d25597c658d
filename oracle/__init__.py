"""Float64 CPU oracle for the selective-scan forward pass.

TEST INFRASTRUCTURE ONLY. Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package. The product path
(the CUDA library and its Python binding) never imports, links or calls it,
and it shares no code with that path.

What it computes: the sequential recurrence of the page "Mamba: Linear-Time
Sequence Modeling with Selective State Spaces" (www.abhik.ai/papers/mamba),
section "Original paper, equations and runnable CPU code", rows "1. Produce
coefficients from the locally mixed input", "2. Retain, write and read each
channel's state" and "5. Put the selective operator inside the complete mixer".
The loop itself is plain C (``ssm_oracle.c``), compiled with gcc at -O2 without
fast-math, run in float64 on inputs widened exactly from float32 or bfloat16.

Beyond the scan it holds, from the same page: the scan with the causal
depthwise convolution and SiLU in front (rows "4. Add causal local context
before selecting coefficients" and 5), the batched decode step with its conv
buffer (row "6. Carry both buffers to the next token"), the exact
zero-order-hold write option, and the backward pass (reverse-mode gradients of
the scan, recomputing each channel's states).

Every function here is pinned by ``tests/test_oracle_pins.py`` to facts the
pages and the mathematics fix (associative-prefix agreement over every
bracketing, the LTI convolution closed form, forgetting and freezing limits,
retention bounds, continuation, the one-token decode step, linearity, channel
independence, degenerate skips, the zero-order-hold closed forms, numpy's
causal convolution, and central finite differences of the forward for every
gradient).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssm_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libssm_oracle.so")
_lock = threading.Lock()
_default = None


def build(force: bool = False, source: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the C oracle into a shared library (gcc, OpenMP, no fast-math)."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(source)):
        return out
    tmp = out + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
           "-shared", "-fPIC", "-std=c11", "-o", tmp, source, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def _f64(a, shape, name):
    """Widen to a contiguous float64 array (exact for float32/bfloat16)."""
    if a is None:
        return None
    arr = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    if tuple(arr.shape) != tuple(shape):
        raise ValueError("%s has shape %s, expected %s"
                         % (name, arr.shape, tuple(shape)))
    return arr


def _ptr(a):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


class OracleLib:
    """One compiled copy of the C oracle (the tests also load mutated copies
    to show that the pins catch planted mistakes)."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        d = ctypes.POINTER(ctypes.c_double)
        i64 = ctypes.c_int64
        lib.ssm_oracle_scan.restype = ctypes.c_int
        lib.ssm_oracle_scan.argtypes = [i64, i64, i64, i64, d, d, d, d, d, d,
                                        d, d, ctypes.c_int, d, d, d, d,
                                        ctypes.c_int]
        lib.ssm_oracle_scan_ex.restype = ctypes.c_int
        lib.ssm_oracle_scan_ex.argtypes = [i64, i64, i64, i64, d, d, d, d, d,
                                           d, d, d, ctypes.c_int, ctypes.c_int,
                                           d, d, d, d, ctypes.c_int]
        lib.ssm_oracle_scan_conv.restype = ctypes.c_int
        lib.ssm_oracle_scan_conv.argtypes = [i64, i64, i64, i64, i64, d, d, d,
                                             d, d, d, d, d, d, d,
                                             ctypes.c_int, ctypes.c_int, d, d,
                                             d, ctypes.c_int]
        lib.ssm_oracle_scan_bwd.restype = ctypes.c_int
        lib.ssm_oracle_scan_bwd.argtypes = [i64, i64, i64, i64] + [d] * 8 + [
            ctypes.c_int, ctypes.c_int] + [d] * 12 + [ctypes.c_int]
        lib.ssm_oracle_step.restype = ctypes.c_int
        lib.ssm_oracle_step.argtypes = [i64, i64, i64, i64, d, d, d, d, d, d,
                                        ctypes.c_int, ctypes.c_int, d, d, d, d,
                                        d, d, d]
        lib.ssm_oracle_step_size.restype = ctypes.c_double
        lib.ssm_oracle_step_size.argtypes = [ctypes.c_double, ctypes.c_double,
                                             ctypes.c_int]
        lib.ssm_oracle_retention.restype = ctypes.c_double
        lib.ssm_oracle_retention.argtypes = [ctypes.c_double, ctypes.c_double]
        lib.ssm_oracle_max_threads.restype = ctypes.c_int
        lib.ssm_oracle_max_threads.argtypes = []
        self.lib = lib
        self.path = path

    def max_threads(self) -> int:
        return int(self.lib.ssm_oracle_max_threads())

    def step_size(self, raw, bias=0.0, softplus=True) -> float:
        return float(self.lib.ssm_oracle_step_size(raw, bias,
                                                   int(bool(softplus))))

    def retention(self, step, a_log) -> float:
        return float(self.lib.ssm_oracle_retention(step, a_log))

    def scan(self, x, delta, A_log, B, C, D=None, z=None, delta_bias=None,
             delta_softplus=True, h0=None, return_states=False, nthreads=0,
             write_zoh=False):
        xa = np.asarray(x)
        if xa.ndim != 3:
            raise ValueError("x must be [batch, seqlen, dim]")
        b, L, E = xa.shape
        N = np.asarray(A_log).shape[-1]
        x64 = _f64(xa, (b, L, E), "x")
        dt64 = _f64(delta, (b, L, E), "delta")
        al64 = _f64(A_log, (E, N), "A_log")
        B64 = _f64(B, (b, L, N), "B")
        C64 = _f64(C, (b, L, N), "C")
        D64 = _f64(D, (E,), "D")
        z64 = _f64(z, (b, L, E), "z")
        bias64 = _f64(delta_bias, (E,), "delta_bias")
        h064 = _f64(h0, (b, E, N), "h0")
        y = np.empty((b, L, E), dtype=np.float64)
        h_last = np.empty((b, E, N), dtype=np.float64)
        states = (np.empty((b, L, E, N), dtype=np.float64)
                  if return_states else None)
        rc = self.lib.ssm_oracle_scan_ex(b, L, E, N, _ptr(x64), _ptr(dt64),
                                         _ptr(al64), _ptr(B64), _ptr(C64),
                                         _ptr(D64), _ptr(z64), _ptr(bias64),
                                         int(bool(delta_softplus)),
                                         int(bool(write_zoh)), _ptr(h064),
                                         _ptr(y), _ptr(h_last), _ptr(states),
                                         int(nthreads))
        if rc != 0:
            raise ValueError("oracle rejected its arguments (rc=%d)" % rc)
        if return_states:
            return y, h_last, states
        return y, h_last


    def scan_conv(self, v, conv_weight, delta, A_log, B, C, conv_bias=None,
                  D=None, z=None, delta_bias=None, delta_softplus=True,
                  h0=None, write_zoh=False, nthreads=0):
        """The scan of x = SiLU(causal_conv(v)) (left zero padding). Returns
        (y [b, L, E], h_last [b, E, N])."""
        va = np.asarray(v)
        b, L, E = va.shape
        N = np.asarray(A_log).shape[-1]
        K = np.asarray(conv_weight).shape[-1]
        y = np.empty((b, L, E), dtype=np.float64)
        h_last = np.empty((b, E, N), dtype=np.float64)
        rc = self.lib.ssm_oracle_scan_conv(
            b, L, E, N, K, _ptr(_f64(va, (b, L, E), "v")),
            _ptr(_f64(conv_weight, (E, K), "conv_weight")),
            _ptr(_f64(conv_bias, (E,), "conv_bias")),
            _ptr(_f64(delta, (b, L, E), "delta")),
            _ptr(_f64(A_log, (E, N), "A_log")), _ptr(_f64(B, (b, L, N), "B")),
            _ptr(_f64(C, (b, L, N), "C")), _ptr(_f64(D, (E,), "D")),
            _ptr(_f64(z, (b, L, E), "z")),
            _ptr(_f64(delta_bias, (E,), "delta_bias")),
            int(bool(delta_softplus)), int(bool(write_zoh)),
            _ptr(_f64(h0, (b, E, N), "h0")), _ptr(y), _ptr(h_last),
            int(nthreads))
        if rc != 0:
            raise ValueError("oracle rejected its arguments (rc=%d)" % rc)
        return y, h_last

    def scan_bwd(self, x, delta, A_log, B, C, dy, D=None, z=None,
                 delta_bias=None, delta_softplus=True, h0=None, dh_last=None,
                 write_zoh=False, nthreads=0):
        """Gradients of sum(dy * y) + sum(dh_last * h_last) with respect to
        every input of scan(). Returns a dict: dx, ddelta, dz (or None), dB,
        dC, dA_log, dD (or None), ddelta_bias (or None), dh0."""
        xa = np.asarray(x)
        b, L, E = xa.shape
        N = np.asarray(A_log).shape[-1]
        out = {k: np.empty(sh, dtype=np.float64) for k, sh in (
            ("dx", (b, L, E)), ("ddelta", (b, L, E)), ("dA_log", (E, N)),
            ("dB", (b, L, N)), ("dC", (b, L, N)), ("dh0", (b, E, N)))}
        out["dz"] = np.empty((b, L, E)) if z is not None else None
        out["dD"] = np.empty(E) if D is not None else None
        out["ddelta_bias"] = np.empty(E) if delta_bias is not None else None
        rc = self.lib.ssm_oracle_scan_bwd(
            b, L, E, N, _ptr(_f64(xa, (b, L, E), "x")),
            _ptr(_f64(delta, (b, L, E), "delta")),
            _ptr(_f64(A_log, (E, N), "A_log")), _ptr(_f64(B, (b, L, N), "B")),
            _ptr(_f64(C, (b, L, N), "C")), _ptr(_f64(D, (E,), "D")),
            _ptr(_f64(z, (b, L, E), "z")),
            _ptr(_f64(delta_bias, (E,), "delta_bias")),
            int(bool(delta_softplus)), int(bool(write_zoh)),
            _ptr(_f64(h0, (b, E, N), "h0")), _ptr(_f64(dy, (b, L, E), "dy")),
            _ptr(_f64(dh_last, (b, E, N), "dh_last")), _ptr(out["dx"]),
            _ptr(out["ddelta"]), _ptr(out["dA_log"]), _ptr(out["dB"]),
            _ptr(out["dC"]), _ptr(out["dD"]), _ptr(out["dz"]),
            _ptr(out["ddelta_bias"]), _ptr(out["dh0"]), int(nthreads))
        if rc != 0:
            raise ValueError("oracle rejected its arguments (rc=%d)" % rc)
        return out

    def step(self, x_new, delta, A_log, B, C, state, conv_state=None,
             conv_weight=None, conv_bias=None, D=None, z=None,
             delta_bias=None, delta_softplus=True, write_zoh=False):
        """One decode step. Returns (y [b, E], new state [b, E, N], new
        conv_state [b, E, K] or None); the inputs are not modified."""
        xa = np.asarray(x_new)
        b, E = xa.shape
        N = np.asarray(A_log).shape[-1]
        K = 0 if conv_state is None else np.asarray(conv_state).shape[-1]
        st = _f64(state, (b, E, N), "state").copy()
        cs = None if conv_state is None else \
            _f64(conv_state, (b, E, K), "conv_state").copy()
        cw = _f64(conv_weight, (E, K), "conv_weight") if K else None
        cb = _f64(conv_bias, (E,), "conv_bias") if K else None
        y = np.empty((b, E), dtype=np.float64)
        rc = self.lib.ssm_oracle_step(
            b, E, N, K, _ptr(_f64(xa, (b, E), "x_new")), _ptr(cs), _ptr(cw),
            _ptr(cb), _ptr(_f64(delta, (b, E), "delta")),
            _ptr(_f64(delta_bias, (E,), "delta_bias")),
            int(bool(delta_softplus)), int(bool(write_zoh)),
            _ptr(_f64(A_log, (E, N), "A_log")), _ptr(_f64(B, (b, N), "B")),
            _ptr(_f64(C, (b, N), "C")), _ptr(_f64(D, (E,), "D")),
            _ptr(_f64(z, (b, E), "z")), _ptr(st), _ptr(y))
        if rc != 0:
            raise ValueError("oracle rejected its arguments (rc=%d)" % rc)
        return y, st, cs


def _load() -> OracleLib:
    global _default
    with _lock:
        if _default is None:
            _default = OracleLib(build())
    return _default


def max_threads() -> int:
    """Threads an OpenMP region of the oracle uses by default."""
    return _load().max_threads()


def step_size(raw: float, bias: float = 0.0, softplus: bool = True) -> float:
    """delta = softplus(raw + bias) (or raw + bias with softplus off)."""
    return _load().step_size(raw, bias, softplus)


def retention(step: float, a_log: float) -> float:
    """a = exp(step * A) with A = -exp(A_log)."""
    return _load().retention(step, a_log)


def scan(x, delta, A_log, B, C, D=None, z=None, delta_bias=None,
         delta_softplus=True, h0=None, return_states=False, nthreads=0,
         write_zoh=False):
    """Run the float64 oracle (write_zoh: exact zero-order-hold write).

    Shapes: x, delta, z: [b, L, E]; B, C: [b, L, N]; A_log: [E, N];
    D, delta_bias: [E]; h0: [b, E, N]. Returns (y [b,L,E], h_last [b,E,N])
    and, with return_states, also every state [b, L, E, N].
    """
    return _load().scan(x, delta, A_log, B, C, D=D, z=z,
                        delta_bias=delta_bias, delta_softplus=delta_softplus,
                        h0=h0, return_states=return_states, nthreads=nthreads,
                        write_zoh=write_zoh)


def scan_conv(v, conv_weight, delta, A_log, B, C, conv_bias=None, D=None,
              z=None, delta_bias=None, delta_softplus=True, h0=None,
              write_zoh=False, nthreads=0):
    """The scan of SiLU(causal_conv(v)) (see OracleLib.scan_conv)."""
    return _load().scan_conv(v, conv_weight, delta, A_log, B, C,
                             conv_bias=conv_bias, D=D, z=z,
                             delta_bias=delta_bias,
                             delta_softplus=delta_softplus, h0=h0,
                             write_zoh=write_zoh, nthreads=nthreads)


def scan_bwd(x, delta, A_log, B, C, dy, D=None, z=None, delta_bias=None,
             delta_softplus=True, h0=None, dh_last=None, write_zoh=False,
             nthreads=0):
    """Gradients of the scan (see OracleLib.scan_bwd)."""
    return _load().scan_bwd(x, delta, A_log, B, C, dy, D=D, z=z,
                            delta_bias=delta_bias,
                            delta_softplus=delta_softplus, h0=h0,
                            dh_last=dh_last, write_zoh=write_zoh,
                            nthreads=nthreads)


def step(x_new, delta, A_log, B, C, state, conv_state=None, conv_weight=None,
         conv_bias=None, D=None, z=None, delta_bias=None, delta_softplus=True,
         write_zoh=False):
    """One batched decode step (see OracleLib.step)."""
    return _load().step(x_new, delta, A_log, B, C, state,
                        conv_state=conv_state, conv_weight=conv_weight,
                        conv_bias=conv_bias, D=D, z=z, delta_bias=delta_bias,
                        delta_softplus=delta_softplus, write_zoh=write_zoh)


def scan_conv_channels(channels, v, conv_weight, delta, A_log, B, C,
                       conv_bias=None, D=None, z=None, delta_bias=None,
                       delta_softplus=True, h0=None, nthreads=0,
                       write_zoh=False):
    """scan_conv on a subset of channels. The convolution is depthwise (one
    filter per channel), so channels stay independent as in scan_channels."""
    ch = np.asarray(channels, dtype=np.int64)
    sel = lambda a: None if a is None else np.asarray(a)[..., ch]  # noqa: E731
    h0s = None if h0 is None else np.asarray(h0)[:, ch, :]
    return scan_conv(sel(v), np.asarray(conv_weight)[ch], sel(delta),
                     np.asarray(A_log)[ch], B, C,
                     conv_bias=None if conv_bias is None
                     else np.asarray(conv_bias)[ch],
                     D=None if D is None else np.asarray(D)[ch], z=sel(z),
                     delta_bias=None if delta_bias is None
                     else np.asarray(delta_bias)[ch],
                     delta_softplus=delta_softplus, h0=h0s,
                     write_zoh=write_zoh, nthreads=nthreads)


def scan_channels(channels, x, delta, A_log, B, C, D=None, z=None,
                  delta_bias=None, delta_softplus=True, h0=None, nthreads=0,
                  write_zoh=False):
    """Oracle on a subset of channels (every batch, the full length).

    Channels never interact (A, D and the bias are per channel; B and C are
    shared read-only), so the result equals the full oracle's columns
    ``channels``. Returns (y [b, L, len(channels)], h_last [b, len, N]).
    """
    ch = np.asarray(channels, dtype=np.int64)
    sel = lambda a: None if a is None else np.asarray(a)[..., ch]  # noqa: E731
    h0s = None if h0 is None else np.asarray(h0)[:, ch, :]
    return scan(sel(x), sel(delta), np.asarray(A_log)[ch], B, C,
                D=None if D is None else np.asarray(D)[ch], z=sel(z),
                delta_bias=None if delta_bias is None
                else np.asarray(delta_bias)[ch],
                delta_softplus=delta_softplus, h0=h0s, nthreads=nthreads,
                write_zoh=write_zoh)
