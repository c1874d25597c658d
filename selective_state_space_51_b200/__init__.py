"""Python binding of libssmscan.so, the B200 selective-scan library.

Argument marshalling only: every step of the scan runs in the CUDA kernels of
the shared library; PyTorch supplies device memory and streams. The functions
carry the C ABI's names (include/ssm_scan.h) and its semantics; status codes
other than SSM_OK raise ``SsmScanError``. If the library has not been built,
importing works but the first call raises: there is no fallback path.

    from selective_state_space_51_b200 import SelectiveScan
    scan = SelectiveScan(device=0)
    # forward (optionally write_zoh=True, or conv_weight=/conv_bias= to fuse
    # the causal depthwise convolution + SiLU that forms x)
    y, h_last = scan(x, delta, A_log, B, C, D=D, z=z, delta_bias=bias)
    # one decode token for a batch, updating state and conv buffer in place
    y_t = scan.step(x_t, delta_t, A_log, B_t, C_t, state, conv_state=buf,
                    conv_weight=w, conv_bias=cb, D=D, z=z_t, delta_bias=bias)
    # gradients of sum(dy * y) + sum(dh_last * h_last)
    grads = scan.backward(x, delta, A_log, B, C, dy, D=D, z=z,
                          delta_bias=bias)
    # a training step: the forward keeps the backward's checkpoints
    y, h_last = scan(x, delta, A_log, B, C, D=D, z=z, delta_bias=bias,
                     save_checkpoints=True)
    grads = scan.backward(x, delta, A_log, B, C, dy, D=D, z=z,
                          delta_bias=bias, reuse_checkpoints=True)
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIBRARY_PATH = os.path.join(_HERE, "libssmscan.so")

SSM_F32 = 0
SSM_BF16 = 1
SSM_DELTA_SOFTPLUS = 1
SSM_WRITE_ZOH = 2
SSM_SAVE_CHECKPOINTS = 4
SSM_REUSE_CHECKPOINTS = 8
SSM_DETERMINISTIC = 16

SSM_OK = 0
SSM_ERR_INVALID = -1
SSM_ERR_UNSUPPORTED = -2
SSM_ERR_ALIGN = -3
SSM_ERR_ARCH = -4
SSM_ERR_CUDA = -5
SSM_ERR_TIMEOUT = -6
SSM_ERR_NOMEM = -7

SSM_VARIANT_AUTO = 0
SSM_VARIANT_SEQUENTIAL = 1
SSM_VARIANT_CHUNKED = 2


class ssm_scan_dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64),
                ("dim", ctypes.c_int64), ("dstate", ctypes.c_int64)]


class SsmScanError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s failed: %s (status %d)" % (
            where, ssm_scan_status_string(status), status))


_lock = threading.Lock()
_lib = None


def library() -> ctypes.CDLL:
    """Load libssmscan.so (built in-tree); raise if it is missing."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIBRARY_PATH):
                raise RuntimeError(
                    "libssmscan.so is not built (expected at %s); run "
                    "`python -m selective_state_space_51_b200.build`"
                    % LIBRARY_PATH)
            lib = ctypes.CDLL(LIBRARY_PATH)
            vp, i32, u32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint32
            lib.ssm_scan_create.argtypes = [ctypes.POINTER(vp), i32]
            lib.ssm_scan_create.restype = i32
            lib.ssm_scan_destroy.argtypes = [vp]
            lib.ssm_scan_destroy.restype = i32
            lib.ssm_scan_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                         u32, vp, vp, vp, ssm_scan_dims, i32,
                                         vp]
            lib.ssm_scan_fwd.restype = i32
            lib.ssm_scan_fwd_conv.argtypes = [vp, vp, vp, vp, i32, vp, vp, vp,
                                              vp, vp, vp, vp, u32, vp, vp, vp,
                                              ssm_scan_dims, i32, vp]
            lib.ssm_scan_fwd_conv.restype = i32
            lib.ssm_scan_bwd.argtypes = [vp] * 9 + [u32] + [vp] * 12 + [
                ssm_scan_dims, i32, vp]
            lib.ssm_scan_bwd.restype = i32
            lib.ssm_scan_set_variant.argtypes = [vp, i32, i32]
            lib.ssm_scan_set_variant.restype = i32
            lib.ssm_scan_last_variant.argtypes = [vp, ctypes.POINTER(i32),
                                                  ctypes.POINTER(i32)]
            lib.ssm_scan_last_variant.restype = i32
            lib.ssm_scan_sync_status.argtypes = [vp, vp]
            lib.ssm_scan_sync_status.restype = i32
            lib.ssm_scan_step.argtypes = [vp, vp, vp, vp, vp, i32, vp, vp, vp,
                                          vp, vp, vp, vp, u32, vp, vp,
                                          ssm_scan_dims, i32, vp]
            lib.ssm_scan_step.restype = i32
            lib.ssm_scan_fwd_static_scratch.argtypes = [
                i32, vp, vp, vp, vp, vp, vp, vp, vp, u32, vp, vp, vp,
                ssm_scan_dims, i32, i32, vp, vp]
            lib.ssm_scan_fwd_static_scratch.restype = i32
            lib.ssm_measure_ex2_rate.argtypes = [i32,
                                                 ctypes.POINTER(ctypes.c_double)]
            lib.ssm_measure_ex2_rate.restype = i32
            lib.ssm_scan_status_string.argtypes = [i32]
            lib.ssm_scan_status_string.restype = ctypes.c_char_p
            _lib = lib
    return _lib


def _ptr(a):
    """Device address of a tensor (or an int address, or None -> NULL)."""
    if a is None:
        return None
    if isinstance(a, int):
        return a
    return a.data_ptr()


def _stream(s):
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(status: int, where: str) -> int:
    if status != SSM_OK:
        raise SsmScanError(status, where)
    return status


def ssm_measure_ex2_rate(device: int = 0) -> float:
    """Measured MUFU exp2 operations per second on ``device`` (see
    include/ssm_scan.h)."""
    out = ctypes.c_double(0.0)
    _check(library().ssm_measure_ex2_rate(int(device), ctypes.byref(out)),
           "ssm_measure_ex2_rate")
    return out.value


def ssm_scan_status_string(status: int) -> str:
    return library().ssm_scan_status_string(int(status)).decode()


def ssm_scan_create(device: int = 0) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check(library().ssm_scan_create(ctypes.byref(h), int(device)),
           "ssm_scan_create")
    return h


def ssm_scan_destroy(h) -> int:
    return _check(library().ssm_scan_destroy(h), "ssm_scan_destroy")


def ssm_scan_set_variant(h, variant: int, segments: int = 0) -> int:
    return _check(library().ssm_scan_set_variant(h, int(variant),
                                                 int(segments)),
                  "ssm_scan_set_variant")


def ssm_scan_last_variant(h):
    v, s = ctypes.c_int(), ctypes.c_int()
    _check(library().ssm_scan_last_variant(h, ctypes.byref(v),
                                           ctypes.byref(s)),
           "ssm_scan_last_variant")
    return v.value, s.value


def ssm_scan_sync_status(h, stream=None) -> int:
    """Status code (not raised): SSM_OK, SSM_ERR_TIMEOUT or SSM_ERR_CUDA."""
    return library().ssm_scan_sync_status(h, _stream(stream))


def ssm_scan_fwd(h, x, delta, A_log, B, C, D, z, delta_bias, flags, h0, y,
                 h_last, dims, dtype, stream=None, check=True) -> int:
    """Call ssm_scan_fwd with tensors (or raw addresses) and a dims tuple
    (batch, seqlen, dim, dstate). Returns the status; raises unless
    ``check`` is False."""
    if not isinstance(dims, ssm_scan_dims):
        dims = ssm_scan_dims(*[int(d) for d in dims])
    rc = library().ssm_scan_fwd(h, _ptr(x), _ptr(delta), _ptr(A_log), _ptr(B),
                                _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
                                int(flags), _ptr(h0), _ptr(y), _ptr(h_last),
                                dims, int(dtype), _stream(stream))
    return _check(rc, "ssm_scan_fwd") if check else rc


def ssm_scan_fwd_conv(h, v, conv_weight, conv_bias, conv_width, delta, A_log,
                      B, C, D, z, delta_bias, flags, h0, y, h_last, dims,
                      dtype, stream=None, check=True) -> int:
    """Call ssm_scan_fwd_conv: the scan of SiLU(causal depthwise conv of v)
    (see include/ssm_scan.h). dims is (batch, seqlen, dim, dstate)."""
    if not isinstance(dims, ssm_scan_dims):
        dims = ssm_scan_dims(*[int(d) for d in dims])
    rc = library().ssm_scan_fwd_conv(
        h, _ptr(v), _ptr(conv_weight), _ptr(conv_bias), int(conv_width),
        _ptr(delta), _ptr(A_log), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
        _ptr(delta_bias), int(flags), _ptr(h0), _ptr(y), _ptr(h_last), dims,
        int(dtype), _stream(stream))
    return _check(rc, "ssm_scan_fwd_conv") if check else rc


def ssm_scan_bwd(h, x, delta, A_log, B, C, D, z, delta_bias, flags, h0, dy,
                 dh_last, dx, ddelta, dA_log, dB, dC, dD, dz, ddelta_bias,
                 dh0, dims, dtype, stream=None, check=True) -> int:
    """Call ssm_scan_bwd (gradients of the scan; see include/ssm_scan.h)."""
    if not isinstance(dims, ssm_scan_dims):
        dims = ssm_scan_dims(*[int(d) for d in dims])
    rc = library().ssm_scan_bwd(
        h, _ptr(x), _ptr(delta), _ptr(A_log), _ptr(B), _ptr(C), _ptr(D),
        _ptr(z), _ptr(delta_bias), int(flags), _ptr(h0), _ptr(dy),
        _ptr(dh_last), _ptr(dx), _ptr(ddelta), _ptr(dA_log), _ptr(dB),
        _ptr(dC), _ptr(dD), _ptr(dz), _ptr(ddelta_bias), _ptr(dh0), dims,
        int(dtype), _stream(stream))
    return _check(rc, "ssm_scan_bwd") if check else rc


def ssm_scan_step(h, x_new, conv_state, conv_weight, conv_bias, conv_width,
                  delta, delta_bias, A_log, B, C, D, z, flags, state, y, dims,
                  dtype, stream=None, check=True) -> int:
    """Call ssm_scan_step (one batched decode step; see include/ssm_scan.h).
    dims is (batch, 1, dim, dstate)."""
    if not isinstance(dims, ssm_scan_dims):
        dims = ssm_scan_dims(*[int(d) for d in dims])
    rc = library().ssm_scan_step(
        h, _ptr(x_new), _ptr(conv_state), _ptr(conv_weight), _ptr(conv_bias),
        int(conv_width), _ptr(delta), _ptr(delta_bias), _ptr(A_log), _ptr(B),
        _ptr(C), _ptr(D), _ptr(z), int(flags), _ptr(state), _ptr(y), dims,
        int(dtype), _stream(stream))
    return _check(rc, "ssm_scan_step") if check else rc


def ssm_scan_fwd_static_scratch(device, x, delta, A_log, B, C, D, z,
                                delta_bias, flags, h0, y, h_last, dims, dtype,
                                segments=0, status=None, stream=None,
                                check=True) -> int:
    """Call ssm_scan_fwd_static_scratch (no handle, allocates nothing; see
    include/ssm_scan.h). Returns the status; raises unless ``check`` is
    False."""
    if not isinstance(dims, ssm_scan_dims):
        dims = ssm_scan_dims(*[int(d) for d in dims])
    rc = library().ssm_scan_fwd_static_scratch(
        int(device), _ptr(x), _ptr(delta), _ptr(A_log), _ptr(B), _ptr(C),
        _ptr(D), _ptr(z), _ptr(delta_bias), int(flags), _ptr(h0), _ptr(y),
        _ptr(h_last), dims, int(dtype), int(segments), _ptr(status),
        _stream(stream))
    return _check(rc, "ssm_scan_fwd_static_scratch") if check else rc


class SelectiveScan:
    """Owns one library handle on a device and runs the fused forward pass.

    Tensors must already be on that device, contiguous, with the layouts of
    include/ssm_scan.h: x, delta, z: [b, L, E]; B, C: [b, L, N]; A_log: [E, N]
    float32; D, delta_bias: [E] float32; h0: [b, E, N] float32. Activations
    are all float32 or all bfloat16; y comes back in the same dtype.
    """

    def __init__(self, device: int = 0):
        import torch
        self.device = torch.device("cuda", device)
        with torch.cuda.device(self.device):
            self.handle = ssm_scan_create(device)

    def close(self):
        if getattr(self, "handle", None) is not None:
            ssm_scan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_variant(self, variant: int, segments: int = 0):
        ssm_scan_set_variant(self.handle, variant, segments)

    def last_variant(self):
        return ssm_scan_last_variant(self.handle)

    def sync_status(self, stream=None) -> int:
        import torch
        if stream is None:
            stream = torch.cuda.current_stream(self.device)
        return ssm_scan_sync_status(self.handle, stream)

    def backward(self, x, delta, A_log, B, C, dy, D=None, z=None,
                 delta_bias=None, delta_softplus=True, h0=None, dh_last=None,
                 write_zoh=False, stream=None, reuse_checkpoints=False,
                 deterministic=False):
        """Gradients of sum(dy * y) + sum(dh_last * h_last) for the scan of
        these inputs. Returns a dict: dx, ddelta, dz (activation dtype; dz
        None without z), dB, dC, dA_log, dD, ddelta_bias, dh0 (float32; dD /
        ddelta_bias None without D / delta_bias). reuse_checkpoints: start
        from the checkpoints of this handle's last forward called with
        save_checkpoints=True on these same inputs. deterministic: the summed
        gradients bitwise reproducible (fixed-order sums of per-block
        partials instead of atomics)."""
        import torch
        if x.dtype == torch.float32:
            dtype = SSM_F32
        elif x.dtype == torch.bfloat16:
            dtype = SSM_BF16
        else:
            raise TypeError("activations must be float32 or bfloat16")
        b, L, E = x.shape
        N = A_log.shape[-1]
        f32 = dict(dtype=torch.float32, device=self.device)
        g = {"dx": torch.empty_like(x), "ddelta": torch.empty_like(x),
             "dz": torch.empty_like(x) if z is not None else None,
             "dB": torch.empty((b, L, N), **f32),
             "dC": torch.empty((b, L, N), **f32),
             "dA_log": torch.empty((E, N), **f32),
             "dD": torch.empty((E,), **f32) if D is not None else None,
             "ddelta_bias": torch.empty((E,), **f32)
             if delta_bias is not None else None,
             "dh0": torch.empty((b, E, N), **f32)}
        if stream is None:
            stream = torch.cuda.current_stream(self.device)
        flags = (SSM_DELTA_SOFTPLUS if delta_softplus else 0) | \
            (SSM_WRITE_ZOH if write_zoh else 0) | \
            (SSM_REUSE_CHECKPOINTS if reuse_checkpoints else 0) | \
            (SSM_DETERMINISTIC if deterministic else 0)
        ssm_scan_bwd(self.handle, x, delta, A_log, B, C, D, z, delta_bias,
                     flags, h0, dy, dh_last, g["dx"], g["ddelta"], g["dA_log"],
                     g["dB"], g["dC"], g["dD"], g["dz"], g["ddelta_bias"],
                     g["dh0"], (b, L, E, N), dtype, stream)
        return g

    def step(self, x_new, delta, A_log, B, C, state, conv_state=None,
             conv_weight=None, conv_bias=None, D=None, z=None,
             delta_bias=None, delta_softplus=True, write_zoh=False, y=None,
             stream=None):
        """One decode step; state (and conv_state) are updated in place.
        Returns y [batch, dim]."""
        import torch
        dtype = SSM_F32 if x_new.dtype == torch.float32 else SSM_BF16
        b, E = x_new.shape
        N = A_log.shape[-1]
        K = 0 if conv_state is None else conv_state.shape[-1]
        if y is None:
            y = torch.empty_like(x_new)
        if stream is None:
            stream = torch.cuda.current_stream(self.device)
        flags = (SSM_DELTA_SOFTPLUS if delta_softplus else 0) | \
            (SSM_WRITE_ZOH if write_zoh else 0)
        ssm_scan_step(self.handle, x_new, conv_state, conv_weight, conv_bias,
                      K, delta, delta_bias, A_log, B, C, D, z, flags, state, y,
                      (b, 1, E, N), dtype, stream)
        return y

    def __call__(self, x, delta, A_log, B, C, D=None, z=None, delta_bias=None,
                 delta_softplus=True, h0=None, y=None, h_last=None,
                 return_last_state=True, stream=None, write_zoh=False,
                 conv_weight=None, conv_bias=None, save_checkpoints=False):
        """The forward scan. With conv_weight ([E, K] float32) x is the input
        of the causal depthwise convolution + SiLU fused in front. With
        save_checkpoints the handle keeps the state checkpoints a following
        backward(..., reuse_checkpoints=True) starts from."""
        import torch
        if x.dtype == torch.float32:
            dtype = SSM_F32
        elif x.dtype == torch.bfloat16:
            dtype = SSM_BF16
        else:
            raise TypeError("activations must be float32 or bfloat16")
        b, L, E = x.shape
        N = A_log.shape[-1]
        for name, t in (("x", x), ("delta", delta), ("B", B), ("C", C),
                        ("z", z)):
            if t is not None and (t.dtype != x.dtype or not t.is_contiguous()
                                  or t.device != self.device):
                raise ValueError("%s must be a contiguous %s tensor on %s"
                                 % (name, x.dtype, self.device))
        for name, t in (("A_log", A_log), ("D", D),
                        ("delta_bias", delta_bias), ("h0", h0),
                        ("conv_weight", conv_weight),
                        ("conv_bias", conv_bias)):
            if t is not None and (t.dtype != torch.float32
                                  or not t.is_contiguous()
                                  or t.device != self.device):
                raise ValueError("%s must be a contiguous float32 tensor on %s"
                                 % (name, self.device))
        if y is None:
            y = torch.empty_like(x)
        if h_last is None and return_last_state:
            h_last = torch.empty((b, E, N), dtype=torch.float32,
                                 device=self.device)
        if stream is None:
            stream = torch.cuda.current_stream(self.device)
        flags = (SSM_DELTA_SOFTPLUS if delta_softplus else 0) | \
            (SSM_WRITE_ZOH if write_zoh else 0) | \
            (SSM_SAVE_CHECKPOINTS if save_checkpoints else 0)
        if conv_weight is not None:
            ssm_scan_fwd_conv(self.handle, x, conv_weight, conv_bias,
                              conv_weight.shape[-1], delta, A_log, B, C, D, z,
                              delta_bias, flags, h0, y, h_last, (b, L, E, N),
                              dtype, stream)
        else:
            ssm_scan_fwd(self.handle, x, delta, A_log, B, C, D, z,
                         delta_bias, flags, h0, y, h_last, (b, L, E, N),
                         dtype, stream)
        return (y, h_last) if return_last_state else y
