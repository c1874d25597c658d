"""The C-ABI library loads, exports every declared symbol, and rejects bad
arguments on the host (no GPU needed)."""
import ctypes
import glob
import os
import re

import pytest

import selective_state_space_51_b200 as S
from selective_state_space_51_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return S.library()


def declared_symbols():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names += re.findall(r"SSM_API\s+[\w\s\*]*?\b(ssm_\w+)\s*\(", text)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert "ssm_scan_fwd" in names and "ssm_scan_create" in names
    for n in names:
        assert hasattr(lib, n), n


def declared_arity():
    """Number of parameters of each SSM_API function in include/*.h."""
    out = {}
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        for m in re.finditer(r"SSM_API\s+[\w\s\*]*?\b(ssm_\w+)\s*\(([^)]*)\)",
                             text):
            params = [q for q in m.group(2).split(",") if q.strip()]
            if len(params) == 1 and params[0].strip() == "void":
                params = []
            out[m.group(1)] = len(params)
    return out


def test_binding_signatures_match_the_header(lib):
    """Every function the binding declares to ctypes takes exactly the
    header's parameter count."""
    arity = declared_arity()
    checked = 0
    for name, n in arity.items():
        fn = getattr(lib, name)
        if fn.argtypes is not None:
            assert len(fn.argtypes) == n, (name, len(fn.argtypes), n)
            checked += 1
    assert checked >= 8


def test_library_built_for_sm100a():
    assert "arch=compute_100a,code=sm_100a" in " ".join(B.NVCC_FLAGS)


def test_status_strings(lib):
    for code in range(-7, 1):
        assert S.ssm_scan_status_string(code) != "unknown status"
    assert S.ssm_scan_status_string(-99) == "unknown status"


def test_null_handle_rejected_on_host(lib):
    dims = S.ssm_scan_dims(1, 4, 8, 4)
    rc = lib.ssm_scan_fwd(None, 16, 16, 16, 16, 16, None, None, None, 1,
                          None, 16, None, dims, S.SSM_F32, None)
    assert rc == S.SSM_ERR_INVALID
    assert lib.ssm_scan_set_variant(None, 0, 0) == S.SSM_ERR_INVALID
    assert lib.ssm_scan_last_variant(None, None, None) == S.SSM_ERR_INVALID
    assert lib.ssm_scan_sync_status(None, None) == S.SSM_ERR_INVALID
    assert lib.ssm_scan_destroy(None) == S.SSM_OK
    assert lib.ssm_scan_create(None, 0) == S.SSM_ERR_INVALID


def test_create_without_a_gpu_fails_cleanly(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    h = ctypes.c_void_p()
    rc = lib.ssm_scan_create(ctypes.byref(h), 0)
    assert rc in (S.SSM_ERR_CUDA, S.SSM_ERR_INVALID)
    assert not h.value


def declared_enums():
    """Every `SSM_NAME = value` enumerator of include/*.h (values written as
    integers, negative integers or `1u << k`)."""
    out = {}
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        for body in re.findall(r"enum\s*\{([^}]*)\}", text):
            body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
            for name, val in re.findall(r"(SSM_\w+)\s*=\s*([^,]+)", body):
                val = val.strip()
                m = re.fullmatch(r"1u\s*<<\s*(\d+)", val)
                out[name] = (1 << int(m.group(1))) if m else int(val)
    return out


def test_binding_constants_match_the_header():
    """The binding's flag, dtype, status and variant constants carry the
    header's values, so a flag added to one side cannot drift."""
    enums = declared_enums()
    for name in ("SSM_DELTA_SOFTPLUS", "SSM_WRITE_ZOH", "SSM_SAVE_CHECKPOINTS",
                 "SSM_REUSE_CHECKPOINTS", "SSM_DETERMINISTIC", "SSM_F32",
                 "SSM_BF16", "SSM_OK", "SSM_ERR_INVALID", "SSM_ERR_TIMEOUT",
                 "SSM_VARIANT_CHUNKED"):
        assert name in enums, name
    for name, val in enums.items():
        if hasattr(S, name):
            assert getattr(S, name) == val, name
    flags = [enums[n] for n in ("SSM_DELTA_SOFTPLUS", "SSM_WRITE_ZOH",
                                "SSM_SAVE_CHECKPOINTS",
                                "SSM_REUSE_CHECKPOINTS", "SSM_DETERMINISTIC")]
    assert len(set(flags)) == len(flags)           # distinct bits
    assert all(f & (f - 1) == 0 for f in flags)    # one bit each
