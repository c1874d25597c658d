"""Planted mistakes in the oracle must each fail at least one pin.

Each mutant is a copy of the C oracle with one plausible slip (a dropped
term, a wrong sign or index, a transposed operand), compiled on the CPU and
run through every pin. A mutant that passes all pins would mean the pins
cannot tell that slip from the real oracle.
"""
import os
import shutil
import tempfile

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "ssm_oracle.c")

# (name, [(text in ssm_oracle.c, replacement), ...])
MUTANTS = [
    ("A not negated", [("A[n] = -exp(A_log[c * dstate + n]);",
                        "A[n] = exp(A_log[c * dstate + n]);")]),
    ("retention exp(step)*A", [("exp(step * A[n])", "(exp(step) * A[n])")]),
    ("retention without step", [("exp(step * A[n])", "exp(A[n])")]),
    ("D term dropped", [("out += D[c] * xv;", "out += 0.0 * xv;")]),
    ("B and C transposed", [(": step) * B[r + n] * xv", ": step) * C[r + n] * xv"),
                            ("out += C[r + n] * h[n];",
                             "out += B[r + n] * h[n];")]),
    ("write uses previous B row",
     [(": step) * B[r + n] * xv",
       ": step) * B[(t ? r - dstate : r) + n] * xv")]),
    ("write without x", [(": step) * B[r + n] * xv;", ": step) * B[r + n];")]),
    ("decode buffer shifted the wrong way",
     [("buf[k] = buf[k + 1];", "buf[k + 1] = buf[k];")]),
    ("decode convolution without its bias",
     [("double acc = conv_bias ? conv_bias[c] : 0.0;", "double acc = 0.0;")]),
    ("decode write uses the raw input, not the convolved one",
     [("* B[b * dstate + n]\n                    * xv;",
       "* B[b * dstate + n]\n                    * x_new[i];")]),
    ("backward adjoint not carried through the retention",
     [("                            lam[n] *= a;\n", "")]),
    ("backward dB without x",
     [("pB[t * N + n] += lam[n] * s * xv;", "pB[t * N + n] += lam[n] * s;")]),
    ("backward step gradient without the softplus slope",
     [("delta_softplus ? ds / (1.0 + exp(-v)) : ds;", "ds;")]),
    ("backward gate gradient without the SiLU slope",
     [("dz[i] = g * pre * sg * (1.0 + z[i] * (1.0 - sg));",
       "dz[i] = g * pre * sg;")]),
    ("backward readout gradient uses the previous state",
     [("pC[t * N + n] += dy * h[n];", "pC[t * N + n] += dy * hp[n];")]),
    ("scan convolution reads the future",
     [("const int64_t s = t - width + 1 + k;", "const int64_t s = t + k;")]),
    ("scan convolution without SiLU",
     [("x[(b * seqlen + t) * dim + c] = silu(acc);",
       "x[(b * seqlen + t) * dim + c] = acc;")]),
    ("zero-order hold without dividing by A",
     [("return expm1(step * A) / A;", "return expm1(step * A);")]),
    ("zero-order hold with exp instead of expm1",
     [("return expm1(step * A) / A;", "return exp(step * A) / A;")]),
    ("x from the wrong channel",
     [("const double xv = x[i];",
       "const double xv = x[(b * seqlen + t) * dim + (dim - 1 - c)];")]),
    ("softplus skipped", [("delta_softplus ? softplus_default(v) : v",
                           "delta_softplus ? v : v")]),
    ("softplus without log1p", [("return log1p(exp(v));",
                                 "return log(exp(v));")]),
    ("bias dropped", [("const double bias = delta_bias ? delta_bias[c] : 0.0;",
                       "const double bias = 0.0;")]),
    ("gate sigmoid instead of SiLU", [("return z / (1.0 + exp(-z));",
                                       "return 1.0 / (1.0 + exp(-z));")]),
    ("incoming state ignored",
     [("h[n] = h0 ? h0[(b * dim + c) * dstate + n] : 0.0;", "h[n] = 0.0;")]),
    ("readout skips n = 0",
     [("for (int64_t n = 0; n < dstate; ++n)\n                out += C",
       "for (int64_t n = 1; n < dstate; ++n)\n                out += C")]),
    ("retention applied twice",
     [("h[n] = retention * h[n] + write;",
       "h[n] = retention * (retention * h[n] + write);")]),
]


@pytest.fixture(scope="module")
def workdir():
    d = tempfile.mkdtemp(prefix="oracle_mutants_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


@pytest.mark.parametrize("name,edits", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, edits, workdir):
    with open(SRC) as f:
        text = f.read()
    for old, new in edits:
        assert text.count(old) >= 1, "mutation site missing: %r" % old
        text = text.replace(old, new)
    tag = "".join(c if c.isalnum() else "_" for c in name)
    src = os.path.join(workdir, tag + ".c")
    with open(src, "w") as f:
        f.write(text)
    lib = oracle.OracleLib(oracle.build(force=True, source=src,
                                        out=os.path.join(workdir,
                                                         tag + ".so")))
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(lib)
        except (AssertionError, FloatingPointError, ValueError) as exc:
            caught.append((pin.__name__, str(exc)[:80]))
    assert caught, "mutant %r passed every pin" % name
