"""Seeded synthetic inputs for the selective-scan forward pass.

This module only draws inputs; it holds none of the scan's arithmetic. The
same arrays feed the CUDA library and the float64 oracle: bfloat16 inputs are
rounded once here (round to nearest even) and the oracle reads exactly those
rounded values, widened.

Five workload shapes, with the value distributions they are stated with:

  0 tiny           b=1,  L=64,     E=16,   N=4,  fp32, gate on
  1 classifier     b=64, L=512,    E=512,  N=16, fp32, gate on, x / sqrt(E)
                   (the width of a four-block d_model=256 classifier)
  2 130M layer     b=8,  L=2048,   E=1536, N=16, bf16 activations, gate on
  3 2.8B layer     b=4,  L=8192,   E=5120, N=16, bf16 activations, gate on
  4 long sequence  b=1,  L=262144, E=2048, N=16, fp32, no gate, h0 ~ N(0, .1^2)

Recipe (shapes 0-3): x, z, B, C ~ N(0, 1); raw step ~ N(0, 0.5^2); D ~ N(0, 1);
A_log[e, n] = log(n + 1) (the S4D-Real initialisation A[n] = -(n + 1)); the
per-channel step bias is the inverse softplus of dt, dt log-uniform in
[1e-3, 1e-1]; softplus on; h0 absent (a zero state). Shape 4: raw step
~ N(-2, 1) before softplus (mostly small steps, long memory), no step bias,
D ~ N(0, 1), h0 ~ N(0, 0.1^2), no gate.

Every draw comes from numpy's PCG64 seeded with 51000 + shape index (or an
explicit seed), in float32, in the fixed order x, raw step, z, B, C, D, dt,
h0. Sizes may be overridden (batch, seqlen, dim, dstate) to make smaller cases
with the same distributions for parity tests.

``a_jitter`` (tests only) gives every channel its own A: A_log[e, n] =
log(n + 1) + a_jitter * N(0, 1), drawn after all the draws above so that
they stay the same. The stated workloads use a_jitter = 0.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np

F32 = "f32"
BF16 = "bf16"

# name, batch, seqlen, dim, dstate, activation dtype, gated, long-memory recipe
SHAPES = (
    ("tiny", 1, 64, 16, 4, F32, True, False),
    ("classifier", 64, 512, 512, 16, F32, True, False),
    ("mamba130m_layer", 8, 2048, 1536, 16, BF16, True, False),
    ("mamba2p8b_layer", 4, 8192, 5120, 16, BF16, True, False),
    ("long_sequence", 1, 262144, 2048, 16, F32, False, True),
)


def shape_description(index: int) -> str:
    name, b, L, E, N, dt, gated, _ = SHAPES[index]
    return "%s b=%d L=%d E=%d N=%d %s%s" % (name, b, L, E, N, dt,
                                            " gated" if gated else "")


def round_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> float32 values (exact)."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32)
            << np.uint32(16)).view(np.float32)


@dataclasses.dataclass
class Workload:
    """Host arrays of one problem.

    ``dev`` holds each activation in its storage form (float32, or uint16
    bfloat16 bits); ``values(name)`` returns the float32 values those stand
    for. Optional inputs absent from the workload are None.
    """
    name: str
    batch: int
    seqlen: int
    dim: int
    dstate: int
    dtype: str
    delta_softplus: bool
    dev: Dict[str, Optional[np.ndarray]]

    ACTIVATIONS = ("x", "delta", "z", "B", "C")

    def values(self, key: str) -> Optional[np.ndarray]:
        a = self.dev[key]
        if a is None:
            return None
        if self.dtype == BF16 and key in self.ACTIVATIONS:
            return bf16_bits_to_f32(a)
        return a

    @property
    def elements(self) -> int:
        """Scan elements b * L * E * N (one retention exp each)."""
        return self.batch * self.seqlen * self.dim * self.dstate


def _log_uniform(rng, lo, hi, n):
    u = rng.random(n, dtype=np.float32)
    return np.exp(np.float32(np.log(lo)) +
                  u * np.float32(np.log(hi) - np.log(lo))).astype(np.float32)


def make(index: int, seed: Optional[int] = None, batch: Optional[int] = None,
         seqlen: Optional[int] = None, dim: Optional[int] = None,
         dstate: Optional[int] = None, dtype: Optional[str] = None,
         gated: Optional[bool] = None, with_h0: Optional[bool] = None,
         with_D: bool = True, a_jitter: float = 0.0) -> Workload:
    """Draw workload ``index`` (0-4), optionally with other sizes or options."""
    name, b0, L0, E0, N0, dt0, gated0, long_memory = SHAPES[index]
    b = b0 if batch is None else int(batch)
    L = L0 if seqlen is None else int(seqlen)
    E = E0 if dim is None else int(dim)
    N = N0 if dstate is None else int(dstate)
    act = dt0 if dtype is None else dtype
    gate = gated0 if gated is None else bool(gated)
    h0_on = long_memory if with_h0 is None else bool(with_h0)
    rng = np.random.Generator(np.random.PCG64(51000 + index
                                              if seed is None else seed))
    normal = lambda *shape: rng.standard_normal(shape, dtype=np.float32)  # noqa

    x = normal(b, L, E)
    if index == 1:
        x *= np.float32(1.0 / np.sqrt(E))
    raw = normal(b, L, E)
    if long_memory:
        raw -= np.float32(2.0)
    else:
        raw *= np.float32(0.5)
    z = normal(b, L, E) if gate else None
    Bm = normal(b, L, N)
    Cm = normal(b, L, N)
    D = normal(E) if with_D else None
    dt = _log_uniform(rng, 1e-3, 1e-1, E)
    h0 = (normal(b, E, N) * np.float32(0.1)) if h0_on else None

    # Inverse softplus of dt: the bias that makes softplus(0 + bias) == dt.
    bias = None
    if not long_memory:
        dt64 = dt.astype(np.float64)
        bias = (dt64 + np.log(-np.expm1(-dt64))).astype(np.float32)
    A_log = np.log(np.arange(1, N + 1, dtype=np.float64))
    A_log = np.ascontiguousarray(np.broadcast_to(A_log, (E, N)),
                                 dtype=np.float32)
    if a_jitter:
        # per-channel A (A is a learned [E, N] parameter): the last draw
        A_log = (A_log + np.float32(a_jitter) * normal(E, N)).astype(
            np.float32)

    dev = dict(x=x, delta=raw, z=z, B=Bm, C=Cm)
    if act == BF16:
        dev = {k: (None if v is None else round_to_bf16_bits(v))
               for k, v in dev.items()}
    dev.update(A_log=A_log, D=D, delta_bias=bias, h0=h0)
    return Workload(name=name, batch=b, seqlen=L, dim=E, dstate=N, dtype=act,
                    delta_softplus=True, dev=dev)


def conv_params(dim: int, width: int = 4, seed: int = 51100):
    """Weights [dim, width] and bias [dim] (float32) of a causal depthwise
    convolution in front of the scan, drawn uniform in +-1/sqrt(width) (the
    fan-in bound of a freshly initialised depthwise filter), weights first,
    from PCG64(seed). When a convolution is used, the workload's x array is
    its input v."""
    rng = np.random.Generator(np.random.PCG64(seed))
    bound = np.float32(1.0 / np.sqrt(width))
    w = (rng.random((dim, width), dtype=np.float32) * 2 - 1) * bound
    bias = (rng.random(dim, dtype=np.float32) * 2 - 1) * bound
    return np.ascontiguousarray(w), np.ascontiguousarray(bias)
