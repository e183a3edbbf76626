"""B200 (sm_100a) selective state-space scan (S6): Python binding.

A thin ctypes layer over ``libssm_scan_b200.so`` (declared in
``include/ssm_scan.h``).  It checks tensor dtypes, devices and contiguity and
passes raw device pointers and the current CUDA stream; every step of the
scan runs in the library's CUDA kernels.  PyTorch is used only to hold device
memory and to name the stream.

The library must have been built (``python -m selective_state_space_38_b200.build``);
the first call without it raises ImportError -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libssm_scan_b200.so")

SSM_F32, SSM_BF16 = 0, 1
DSTATE = 16


class SSMError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"ssm_scan error {code}: {msg}")
        self.code = code


class SsdDims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("heads", ctypes.c_int64),
                ("headdim", ctypes.c_int64), ("groups", ctypes.c_int64), ("dstate", ctypes.c_int64),
                ("act_dtype", ctypes.c_int32)]


class Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("dim", ctypes.c_int64),
                ("dstate", ctypes.c_int64), ("act_dtype", ctypes.c_int32)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m selective_state_space_38_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I = ctypes.c_void_p, ctypes.c_int
    DP = ctypes.POINTER(Dims)
    S = ctypes.c_size_t
    lib.ssm_scan_fwd_workspace_size.argtypes = [DP, I, ctypes.POINTER(S)]
    lib.ssm_scan_fwd_workspace_size.restype = I
    lib.ssm_scan_fwd.argtypes = [P, P, P, I, P, P, P, P, P, P, P, P, P, S, DP, P]
    lib.ssm_scan_fwd.restype = I
    lib.ssm_scan_fwd_status.argtypes = [P, P]
    lib.ssm_scan_fwd_status.restype = I
    lib.ssm_scan_fwd_noalloc.argtypes = [P, P, P, I, P, P, P, P, P, P, P, P, DP, P]
    lib.ssm_scan_fwd_noalloc.restype = I
    lib.ssm_debug_fwd_flag_timeout.argtypes = [P, P, P, I, P, P, P, P, P, P, P, P, P, S, ctypes.c_uint32, DP, P]
    lib.ssm_debug_fwd_flag_timeout.restype = I
    lib.ssm_conv_scan_fwd.argtypes = [P, P, P, I, P, P, P, P, I, P, P, P, P, P, P, P, P, P, S, DP, P]
    lib.ssm_conv_scan_fwd.restype = I
    lib.ssm_conv_scan_step.argtypes = [P, P, P, P, P, I, P, P, I, P, P, P, P, P, P, DP, P]
    lib.ssm_conv_scan_step.restype = I
    lib.ssm_trap_scan_fwd.argtypes = [P, P, P, I, P, P, P, P, P, P, P, P, P, P, P, P, S, DP, P]
    lib.ssm_trap_scan_fwd.restype = I
    lib.ssm_trap_scan_step.argtypes = [P, P, P, P, I, P, P, P, P, P, P, P, P, P, DP, P]
    lib.ssm_trap_scan_step.restype = I
    lib.ssm_scan_bwd_workspace_size.argtypes = [DP, ctypes.POINTER(S)]
    lib.ssm_scan_bwd_workspace_size.restype = I
    lib.ssm_scan_bwd.argtypes = [P, P, P, I, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, S, DP, P]
    lib.ssm_scan_bwd.restype = I
    lib.ssm_ssd_fwd_workspace_size.argtypes = [ctypes.POINTER(SsdDims), I, ctypes.POINTER(S)]
    lib.ssm_ssd_fwd_workspace_size.restype = I
    lib.ssm_ssd_fwd.argtypes = [P, P, P, I, P, P, P, P, P, P, P, P, S, ctypes.POINTER(SsdDims), P]
    lib.ssm_debug_ssd_flag_timeout.argtypes = [P, P, P, I, P, P, P, P, P, P, P, P, S, ctypes.c_uint32,
                                               ctypes.POINTER(SsdDims), P]
    lib.ssm_debug_ssd_flag_timeout.restype = I
    lib.ssm_ssd_fwd.restype = I
    lib.ssm_scan_step.argtypes = [P, P, P, P, I, P, P, P, P, P, P, DP, P]
    lib.ssm_scan_step.restype = I
    lib.ssm_strerror.argtypes = [I]
    lib.ssm_strerror.restype = ctypes.c_char_p
    lib.ssm_version.argtypes = []
    lib.ssm_version.restype = I
    return lib


_lib = None


def get_lib():
    """The loaded CUDA library (loaded on first use; ImportError if not built)."""
    global _lib
    if _lib is None:
        _lib = _load()
    return _lib


EXPORTS = ("ssm_scan_fwd_workspace_size", "ssm_scan_fwd", "ssm_scan_fwd_status", "ssm_scan_step",
           "ssm_conv_scan_fwd", "ssm_conv_scan_step", "ssm_trap_scan_fwd", "ssm_trap_scan_step",
           "ssm_scan_bwd_workspace_size", "ssm_scan_bwd", "ssm_ssd_fwd_workspace_size", "ssm_ssd_fwd",
           "ssm_scan_fwd_noalloc",
           "ssm_debug_fwd_flag_timeout", "ssm_debug_ssd_flag_timeout",
           "ssm_strerror", "ssm_version")


def ssm_strerror(code: int) -> str:
    return get_lib().ssm_strerror(int(code)).decode()


def ssm_version() -> int:
    return int(get_lib().ssm_version())


_ws_sizes = {}


def ssm_scan_fwd_workspace_size(batch: int, seqlen: int, dim: int, device=None, sm_count: int = 0) -> int:
    """Workspace bytes ssm_scan_fwd needs for this shape (on `device`, or on a
    GPU with `sm_count` SMs when that is given)."""
    key = (batch, seqlen, dim, sm_count, None if sm_count > 0 else torch.device(device or "cuda").index)
    n = _ws_sizes.get(key)
    if n is None:
        out = ctypes.c_size_t(0)
        dims = Dims(batch, seqlen, dim, DSTATE, SSM_BF16)
        if sm_count > 0:
            rc = get_lib().ssm_scan_fwd_workspace_size(ctypes.byref(dims), int(sm_count), ctypes.byref(out))
        else:
            with torch.cuda.device(device):
                rc = get_lib().ssm_scan_fwd_workspace_size(ctypes.byref(dims), 0, ctypes.byref(out))
        _check(rc)
        n = _ws_sizes[key] = int(out.value)
    return n


def ssm_scan_fwd_status(workspace=None, stream=None, device=None) -> int:
    """Block until `stream` is done and return the status code of the last
    forward call on `workspace` (a uint8 CUDA tensor; None: the last
    ssm_scan_fwd_noalloc call): 0, or 5 when a bounded device wait gave up."""
    dev = workspace.device if workspace is not None else torch.device(device or "cuda")
    with torch.cuda.device(dev):
        return int(get_lib().ssm_scan_fwd_status(
            None if workspace is None else workspace.data_ptr(), _stream_ptr(stream, dev)))


def _act_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SSM_BF16
    if t.dtype == torch.float32:
        return SSM_F32
    raise TypeError(f"activations must be bfloat16 or float32, got {t.dtype}")


def _ptr(t, *, dtype=None, device=None, shape=None, name=""):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream_ptr(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream


def _check(rc):
    if rc != 0:
        raise SSMError(rc, ssm_strerror(rc))


def ssm_scan_fwd(x, delta, delta_bias, softplus, A, B, C, D=None, z=None, h0=None,
                 out=None, h_last=None, return_last_state=True, stream=None, workspace=None,
                 check=False):
    """Forward selective scan.

    x, delta, z: [batch, dim, L]; B, C: [batch, 16, L] (all bfloat16 or all
    float32, on one CUDA device); A: [dim, 16], D, delta_bias: [dim], h0:
    [batch, dim, 16] float32.  Returns (out, h_last); h_last is None when
    ``return_last_state`` is False and no buffer is given.  ``workspace`` is
    a uint8 CUDA tensor of at least ssm_scan_fwd_workspace_size bytes (taken
    from torch's caching allocator when None).  ``check=True`` waits for the
    call and raises SSMError when a bounded device wait gave up.
    """
    if x.device.type != "cuda":
        raise ValueError("ssm_scan_fwd needs CUDA tensors")
    dev = x.device
    batch, dim, L = x.shape
    code = _act_code(x)
    act = x.dtype
    f32 = torch.float32
    ptrs = dict(
        x=_ptr(x, dtype=act, device=dev, name="x"),
        delta=_ptr(delta, dtype=act, device=dev, shape=x.shape, name="delta"),
        z=_ptr(z, dtype=act, device=dev, shape=x.shape, name="z"),
        B=_ptr(B, dtype=act, device=dev, shape=(batch, DSTATE, L), name="B"),
        C=_ptr(C, dtype=act, device=dev, shape=(batch, DSTATE, L), name="C"),
        A=_ptr(A, dtype=f32, device=dev, shape=(dim, DSTATE), name="A"),
        D=_ptr(D, dtype=f32, device=dev, shape=(dim,), name="D"),
        delta_bias=_ptr(delta_bias, dtype=f32, device=dev, shape=(dim,), name="delta_bias"),
        h0=_ptr(h0, dtype=f32, device=dev, shape=(batch, dim, DSTATE), name="h0"),
    )
    if out is None:
        out = torch.empty_like(x)
    if h_last is None and return_last_state:
        h_last = torch.empty((batch, dim, DSTATE), dtype=f32, device=dev)
    po = _ptr(out, dtype=act, device=dev, shape=x.shape, name="out")
    ph = _ptr(h_last, dtype=f32, device=dev, shape=(batch, dim, DSTATE), name="h_last")
    dims = Dims(batch, L, dim, DSTATE, code)
    if workspace is None:
        workspace = torch.empty(ssm_scan_fwd_workspace_size(batch, L, dim, dev), dtype=torch.uint8,
                                device=dev)
    pw = _ptr(workspace, dtype=torch.uint8, device=dev, name="workspace")
    sp = _stream_ptr(stream, dev)
    with torch.cuda.device(dev):
        rc = get_lib().ssm_scan_fwd(ptrs["x"], ptrs["delta"], ptrs["delta_bias"], int(bool(softplus)),
                                    ptrs["A"], ptrs["B"], ptrs["C"], ptrs["D"], ptrs["z"], ptrs["h0"],
                                    po, ph, pw, workspace.numel(), ctypes.byref(dims), sp)
        _check(rc)
        if check:
            _check(get_lib().ssm_scan_fwd_status(pw, sp))
    return out, h_last


def ssm_conv_scan_fwd(x, conv_w, conv_bias, conv_state, delta, delta_bias, softplus, A, B, C, D=None,
                      z=None, h0=None, out=None, h_last=None, conv_state_out=None, return_conv_state=True,
                      stream=None, workspace=None, check=False):
    """Causal convolution (width conv_w.shape[1] <= 4) + silu fused in front of
    the forward scan.  x is the raw input [batch, dim, L]; conv_w [dim, K] and
    conv_bias [dim] float32; conv_state [batch, dim, K-1] in x's dtype (None:
    zeros).  Returns (out, h_last, conv_state_out); the new convolution state
    is written into ``conv_state_out`` (may be ``conv_state``) or a new tensor."""
    if x.device.type != "cuda":
        raise ValueError("ssm_conv_scan_fwd needs CUDA tensors")
    dev = x.device
    batch, dim, L = x.shape
    code = _act_code(x)
    act = x.dtype
    f32 = torch.float32
    K = int(conv_w.shape[1])
    ptrs = dict(
        x=_ptr(x, dtype=act, device=dev, name="x"),
        w=_ptr(conv_w, dtype=f32, device=dev, shape=(dim, K), name="conv_w"),
        cb=_ptr(conv_bias, dtype=f32, device=dev, shape=(dim,), name="conv_bias"),
        cs=_ptr(conv_state, dtype=act, device=dev, shape=(batch, dim, K - 1), name="conv_state"),
        delta=_ptr(delta, dtype=act, device=dev, shape=x.shape, name="delta"),
        z=_ptr(z, dtype=act, device=dev, shape=x.shape, name="z"),
        B=_ptr(B, dtype=act, device=dev, shape=(batch, DSTATE, L), name="B"),
        C=_ptr(C, dtype=act, device=dev, shape=(batch, DSTATE, L), name="C"),
        A=_ptr(A, dtype=f32, device=dev, shape=(dim, DSTATE), name="A"),
        D=_ptr(D, dtype=f32, device=dev, shape=(dim,), name="D"),
        delta_bias=_ptr(delta_bias, dtype=f32, device=dev, shape=(dim,), name="delta_bias"),
        h0=_ptr(h0, dtype=f32, device=dev, shape=(batch, dim, DSTATE), name="h0"),
    )
    if out is None:
        out = torch.empty_like(x)
    if h_last is None:
        h_last = torch.empty((batch, dim, DSTATE), dtype=f32, device=dev)
    if conv_state_out is None and return_conv_state and K > 1:
        conv_state_out = torch.empty((batch, dim, K - 1), dtype=act, device=dev)
    po = _ptr(out, dtype=act, device=dev, shape=x.shape, name="out")
    ph = _ptr(h_last, dtype=f32, device=dev, shape=(batch, dim, DSTATE), name="h_last")
    pcs = _ptr(conv_state_out, dtype=act, device=dev, shape=(batch, dim, K - 1), name="conv_state_out")
    dims = Dims(batch, L, dim, DSTATE, code)
    if workspace is None:
        workspace = torch.empty(ssm_scan_fwd_workspace_size(batch, L, dim, dev), dtype=torch.uint8,
                                device=dev)
    pw = _ptr(workspace, dtype=torch.uint8, device=dev, name="workspace")
    sp = _stream_ptr(stream, dev)
    with torch.cuda.device(dev):
        rc = get_lib().ssm_conv_scan_fwd(ptrs["x"], ptrs["w"], ptrs["cb"], K, ptrs["cs"], pcs, ptrs["delta"],
                                         ptrs["delta_bias"], int(bool(softplus)), ptrs["A"], ptrs["B"], ptrs["C"],
                                         ptrs["D"], ptrs["z"], ptrs["h0"], po, ph, pw, workspace.numel(),
                                         ctypes.byref(dims), sp)
        _check(rc)
        if check:
            _check(get_lib().ssm_scan_fwd_status(pw, sp))
    return out, h_last, conv_state_out


def ssm_conv_scan_step(conv_state, state, x, conv_w, conv_bias, delta, delta_bias, softplus, A, B, C,
                       D=None, z=None, out=None, stream=None):
    """One decode step of convolution + scan; ``conv_state`` ([batch, dim,
    K-1], x's dtype) and ``state`` ([batch, dim, 16] float32) are updated in
    place.  Returns out [batch, dim]."""
    if x.device.type != "cuda":
        raise ValueError("ssm_conv_scan_step needs CUDA tensors")
    dev = x.device
    batch, dim = x.shape
    code = _act_code(x)
    act = x.dtype
    f32 = torch.float32
    K = int(conv_w.shape[1])
    pcs = _ptr(conv_state, dtype=act, device=dev, shape=(batch, dim, K - 1), name="conv_state")
    ps = _ptr(state, dtype=f32, device=dev, shape=(batch, dim, DSTATE), name="state")
    px = _ptr(x, dtype=act, device=dev, name="x")
    pw = _ptr(conv_w, dtype=f32, device=dev, shape=(dim, K), name="conv_w")
    pcb = _ptr(conv_bias, dtype=f32, device=dev, shape=(dim,), name="conv_bias")
    pd = _ptr(delta, dtype=act, device=dev, shape=x.shape, name="delta")
    pz = _ptr(z, dtype=act, device=dev, shape=x.shape, name="z")
    pB = _ptr(B, dtype=act, device=dev, shape=(batch, DSTATE), name="B")
    pC = _ptr(C, dtype=act, device=dev, shape=(batch, DSTATE), name="C")
    pA = _ptr(A, dtype=f32, device=dev, shape=(dim, DSTATE), name="A")
    pD = _ptr(D, dtype=f32, device=dev, shape=(dim,), name="D")
    pb = _ptr(delta_bias, dtype=f32, device=dev, shape=(dim,), name="delta_bias")
    if out is None:
        out = torch.empty_like(x)
    po = _ptr(out, dtype=act, device=dev, shape=x.shape, name="out")
    dims = Dims(batch, 1, dim, DSTATE, code)
    with torch.cuda.device(dev):
        rc = get_lib().ssm_conv_scan_step(pcs, ps, px, pw, pcb, K, pd, pb, int(bool(softplus)), pA, pB, pC,
                                          pD, pz, po, ctypes.byref(dims), _stream_ptr(stream, dev))
    _check(rc)
    return out


def ssm_trap_scan_fwd(x, delta, delta_bias, softplus, lam, A, B, C, D=None, z=None, h0=None, x_prev=None,
                      B_prev=None, out=None, h_last=None, stream=None, workspace=None, check=False):
    """Forward scan with the exponential-trapezoidal rule.  lam: [batch, dim, L]
    in x's dtype; x_prev [batch, dim] and B_prev [batch, 16]: the input before
    t = 0 (the previous call's last x and B).  Returns (out, h_last)."""
    if x.device.type != "cuda":
        raise ValueError("ssm_trap_scan_fwd needs CUDA tensors")
    dev = x.device
    batch, dim, L = x.shape
    code = _act_code(x)
    act = x.dtype
    f32 = torch.float32
    ptrs = dict(
        x=_ptr(x, dtype=act, device=dev, name="x"),
        delta=_ptr(delta, dtype=act, device=dev, shape=x.shape, name="delta"),
        lam=_ptr(lam, dtype=act, device=dev, shape=x.shape, name="lam"),
        z=_ptr(z, dtype=act, device=dev, shape=x.shape, name="z"),
        B=_ptr(B, dtype=act, device=dev, shape=(batch, DSTATE, L), name="B"),
        C=_ptr(C, dtype=act, device=dev, shape=(batch, DSTATE, L), name="C"),
        A=_ptr(A, dtype=f32, device=dev, shape=(dim, DSTATE), name="A"),
        D=_ptr(D, dtype=f32, device=dev, shape=(dim,), name="D"),
        delta_bias=_ptr(delta_bias, dtype=f32, device=dev, shape=(dim,), name="delta_bias"),
        h0=_ptr(h0, dtype=f32, device=dev, shape=(batch, dim, DSTATE), name="h0"),
        x_prev=_ptr(x_prev, dtype=act, device=dev, shape=(batch, dim), name="x_prev"),
        B_prev=_ptr(B_prev, dtype=act, device=dev, shape=(batch, DSTATE), name="B_prev"),
    )
    if out is None:
        out = torch.empty_like(x)
    if h_last is None:
        h_last = torch.empty((batch, dim, DSTATE), dtype=f32, device=dev)
    po = _ptr(out, dtype=act, device=dev, shape=x.shape, name="out")
    ph = _ptr(h_last, dtype=f32, device=dev, shape=(batch, dim, DSTATE), name="h_last")
    dims = Dims(batch, L, dim, DSTATE, code)
    if workspace is None:
        workspace = torch.empty(ssm_scan_fwd_workspace_size(batch, L, dim, dev), dtype=torch.uint8,
                                device=dev)
    pw = _ptr(workspace, dtype=torch.uint8, device=dev, name="workspace")
    sp = _stream_ptr(stream, dev)
    with torch.cuda.device(dev):
        rc = get_lib().ssm_trap_scan_fwd(ptrs["x"], ptrs["delta"], ptrs["delta_bias"], int(bool(softplus)),
                                         ptrs["lam"], ptrs["A"], ptrs["B"], ptrs["C"], ptrs["D"], ptrs["z"],
                                         ptrs["h0"], ptrs["x_prev"], ptrs["B_prev"], po, ph, pw, workspace.numel(),
                                         ctypes.byref(dims), sp)
        _check(rc)
        if check:
            _check(get_lib().ssm_scan_fwd_status(pw, sp))
    return out, h_last


def ssm_trap_scan_step(state, x, delta, delta_bias, softplus, lam, A, B, C, D=None, z=None, x_prev=None,
                       B_prev=None, out=None, stream=None):
    """One trapezoidal decode step; ``state`` is updated in place.  lam:
    [batch, dim]; x_prev [batch, dim], B_prev [batch, 16]: the previous token's."""
    if x.device.type != "cuda":
        raise ValueError("ssm_trap_scan_step needs CUDA tensors")
    dev = x.device
    batch, dim = x.shape
    code = _act_code(x)
    act = x.dtype
    f32 = torch.float32
    args = [_ptr(state, dtype=f32, device=dev, shape=(batch, dim, DSTATE), name="state"),
            _ptr(x, dtype=act, device=dev, name="x"),
            _ptr(delta, dtype=act, device=dev, shape=x.shape, name="delta"),
            _ptr(delta_bias, dtype=f32, device=dev, shape=(dim,), name="delta_bias"), int(bool(softplus)),
            _ptr(lam, dtype=act, device=dev, shape=x.shape, name="lam"),
            _ptr(A, dtype=f32, device=dev, shape=(dim, DSTATE), name="A"),
            _ptr(B, dtype=act, device=dev, shape=(batch, DSTATE), name="B"),
            _ptr(C, dtype=act, device=dev, shape=(batch, DSTATE), name="C"),
            _ptr(D, dtype=f32, device=dev, shape=(dim,), name="D"),
            _ptr(z, dtype=act, device=dev, shape=x.shape, name="z"),
            _ptr(x_prev, dtype=act, device=dev, shape=x.shape, name="x_prev"),
            _ptr(B_prev, dtype=act, device=dev, shape=(batch, DSTATE), name="B_prev")]
    if out is None:
        out = torch.empty_like(x)
    args.append(_ptr(out, dtype=act, device=dev, shape=x.shape, name="out"))
    dims = Dims(batch, 1, dim, DSTATE, code)
    with torch.cuda.device(dev):
        rc = get_lib().ssm_trap_scan_step(*args, ctypes.byref(dims), _stream_ptr(stream, dev))
    _check(rc)
    return out


def ssm_scan_bwd(x, delta, delta_bias, softplus, A, B, C, D, z, h0, dout, dh_last=None, stream=None,
                 workspace=None):
    """Backward pass of ssm_scan_fwd.  Returns a dict: dx, ddelta, dz (None
    without z) in x's dtype [batch, dim, L]; dB, dC float32 [batch, 16, L];
    dA float32 [dim, 16]; dD, dbias float32 [dim]; dh0 float32 [batch, dim, 16]."""
    if x.device.type != "cuda":
        raise ValueError("ssm_scan_bwd needs CUDA tensors")
    dev = x.device
    batch, dim, L = x.shape
    code = _act_code(x)
    act = x.dtype
    f32 = torch.float32
    ins = [_ptr(x, dtype=act, device=dev, name="x"),
           _ptr(delta, dtype=act, device=dev, shape=x.shape, name="delta"),
           _ptr(delta_bias, dtype=f32, device=dev, shape=(dim,), name="delta_bias"), int(bool(softplus)),
           _ptr(A, dtype=f32, device=dev, shape=(dim, DSTATE), name="A"),
           _ptr(B, dtype=act, device=dev, shape=(batch, DSTATE, L), name="B"),
           _ptr(C, dtype=act, device=dev, shape=(batch, DSTATE, L), name="C"),
           _ptr(D, dtype=f32, device=dev, shape=(dim,), name="D"),
           _ptr(z, dtype=act, device=dev, shape=x.shape, name="z"),
           _ptr(h0, dtype=f32, device=dev, shape=(batch, dim, DSTATE), name="h0"),
           _ptr(dout, dtype=act, device=dev, shape=x.shape, name="dout"),
           _ptr(dh_last, dtype=f32, device=dev, shape=(batch, dim, DSTATE), name="dh_last")]
    g = dict(dx=torch.empty_like(x), ddelta=torch.empty_like(x), dz=torch.empty_like(x) if z is not None else None,
             dB=torch.empty((batch, DSTATE, L), dtype=f32, device=dev),
             dC=torch.empty((batch, DSTATE, L), dtype=f32, device=dev),
             dA=torch.empty((dim, DSTATE), dtype=f32, device=dev), dD=torch.empty(dim, dtype=f32, device=dev),
             dbias=torch.empty(dim, dtype=f32, device=dev),
             dh0=torch.empty((batch, dim, DSTATE), dtype=f32, device=dev))
    dims = Dims(batch, L, dim, DSTATE, code)
    if workspace is None:
        n = ctypes.c_size_t(0)
        _check(get_lib().ssm_scan_bwd_workspace_size(ctypes.byref(dims), ctypes.byref(n)))
        workspace = torch.empty(int(n.value), dtype=torch.uint8, device=dev)
    outs = [None if g[k] is None else g[k].data_ptr()
            for k in ("dx", "ddelta", "dz", "dB", "dC", "dA", "dD", "dbias", "dh0")]
    pw = _ptr(workspace, dtype=torch.uint8, device=dev, name="workspace")
    with torch.cuda.device(dev):
        rc = get_lib().ssm_scan_bwd(*ins, *outs, pw, workspace.numel(), ctypes.byref(dims),
                                    _stream_ptr(stream, dev))
    _check(rc)
    return g


def ssm_ssd_fwd_workspace_size(batch: int, heads: int, device=None, sm_count: int = 0) -> int:
    """Workspace bytes with which ssm_ssd_fwd balances batch * heads sequences
    over the device's SMs (``sm_count`` > 0 sizes it without a device)."""
    dims = SsdDims(batch, 1, heads, 64, 1, 128, SSM_BF16)
    out = ctypes.c_size_t(0)
    if sm_count > 0:
        _check(get_lib().ssm_ssd_fwd_workspace_size(ctypes.byref(dims), int(sm_count), ctypes.byref(out)))
    else:
        with torch.cuda.device(torch.device(device or "cuda")):
            _check(get_lib().ssm_ssd_fwd_workspace_size(ctypes.byref(dims), 0, ctypes.byref(out)))
    return int(out.value)


def ssm_ssd_fwd(x, dt, dt_bias, softplus, A, B, C, D=None, h0=None, y=None, h_last=None, stream=None,
                workspace=None, check=False):
    """Mamba-2 SSD forward on the tensor cores.  x [batch, L, heads, 64],
    dt [batch, L, heads], B, C [batch, L, groups, 128] bf16; A, dt_bias, D
    [heads] float32; h0 [batch, heads, 64, 128] float32.  Returns (y, h_last)."""
    if x.device.type != "cuda":
        raise ValueError("ssm_ssd_fwd needs CUDA tensors")
    dev = x.device
    batch, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    act = torch.bfloat16
    f32 = torch.float32
    args = [_ptr(x, dtype=act, device=dev, name="x"),
            _ptr(dt, dtype=act, device=dev, shape=(batch, L, H), name="dt"),
            _ptr(dt_bias, dtype=f32, device=dev, shape=(H,), name="dt_bias"), int(bool(softplus)),
            _ptr(A, dtype=f32, device=dev, shape=(H,), name="A"),
            _ptr(B, dtype=act, device=dev, shape=(batch, L, G, N), name="B"),
            _ptr(C, dtype=act, device=dev, shape=(batch, L, G, N), name="C"),
            _ptr(D, dtype=f32, device=dev, shape=(H,), name="D"),
            _ptr(h0, dtype=f32, device=dev, shape=(batch, H, P, N), name="h0")]
    if y is None:
        y = torch.empty_like(x)
    if h_last is None:
        h_last = torch.empty((batch, H, P, N), dtype=f32, device=dev)
    args += [_ptr(y, dtype=act, device=dev, shape=x.shape, name="y"),
             _ptr(h_last, dtype=f32, device=dev, shape=(batch, H, P, N), name="h_last")]
    dims = SsdDims(batch, L, H, P, G, N, SSM_BF16)
    if workspace is None:
        workspace = torch.empty(ssm_ssd_fwd_workspace_size(batch, H, dev), dtype=torch.uint8, device=dev)
    pw = _ptr(workspace, dtype=torch.uint8, device=dev, name="workspace")
    sp = _stream_ptr(stream, dev)
    with torch.cuda.device(dev):
        _check(get_lib().ssm_ssd_fwd(*args, pw, workspace.numel(), ctypes.byref(dims), sp))
        if check:
            _check(get_lib().ssm_scan_fwd_status(pw, sp))
    return y, h_last


def ssm_scan_step(state, x, delta, delta_bias, softplus, A, B, C, D=None, z=None, out=None,
                  stream=None):
    """One recurrent decode step; ``state`` ([batch, dim, 16] float32) is
    updated in place.  x, delta, z: [batch, dim]; B, C: [batch, 16].
    Returns out [batch, dim]."""
    if x.device.type != "cuda":
        raise ValueError("ssm_scan_step needs CUDA tensors")
    dev = x.device
    batch, dim = x.shape
    code = _act_code(x)
    act = x.dtype
    f32 = torch.float32
    ps = _ptr(state, dtype=f32, device=dev, shape=(batch, dim, DSTATE), name="state")
    px = _ptr(x, dtype=act, device=dev, name="x")
    pd = _ptr(delta, dtype=act, device=dev, shape=x.shape, name="delta")
    pz = _ptr(z, dtype=act, device=dev, shape=x.shape, name="z")
    pB = _ptr(B, dtype=act, device=dev, shape=(batch, DSTATE), name="B")
    pC = _ptr(C, dtype=act, device=dev, shape=(batch, DSTATE), name="C")
    pA = _ptr(A, dtype=f32, device=dev, shape=(dim, DSTATE), name="A")
    pD = _ptr(D, dtype=f32, device=dev, shape=(dim,), name="D")
    pb = _ptr(delta_bias, dtype=f32, device=dev, shape=(dim,), name="delta_bias")
    if out is None:
        out = torch.empty_like(x)
    po = _ptr(out, dtype=act, device=dev, shape=x.shape, name="out")
    dims = Dims(batch, 1, dim, DSTATE, code)
    with torch.cuda.device(dev):
        rc = get_lib().ssm_scan_step(ps, px, pd, pb, int(bool(softplus)), pA, pB, pC, pD, pz, po,
                               ctypes.byref(dims), _stream_ptr(stream, dev))
    _check(rc)
    return out


__all__ = ["ssm_scan_fwd", "ssm_scan_fwd_workspace_size", "ssm_scan_fwd_status", "ssm_scan_step",
           "ssm_conv_scan_fwd", "ssm_conv_scan_step", "ssm_trap_scan_fwd", "ssm_trap_scan_step", "ssm_scan_bwd",
           "ssm_ssd_fwd", "ssm_ssd_fwd_workspace_size", "SsdDims", "ssm_strerror", "ssm_version", "SSMError", "Dims", "LIB_PATH", "get_lib"]
