"""Float64 CPU oracle for the selective state-space scan (S6).

TEST INFRASTRUCTURE ONLY.  The product path (the CUDA library and its Python
binding) never imports this package.  Only ``tests/``, the package smoke check
and the benchmark's CPU-baseline leg use it.

The arithmetic lives in ``ssm_ref.c`` (plain C, double precision, sequential
in time).  This module compiles it with gcc and marshals numpy arrays to it.
Activations are passed as stored: ``float32`` arrays, or bfloat16 given as
``uint16`` bit patterns; the C code widens each value exactly to double.

Sources: the Mamba pages' description of the selection mechanism (input-
dependent dt, B, C), the ZOH + Euler discretisation named in the "Mamba3"
post, the recurrent one-step mode, and Gu & Dao Appendix D ("Speed": chunks
continue from the carried state).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssm_ref.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libssm_ref.so")

_lib = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the C oracle into a shared library and return its path.

    No fast-math and no FMA contraction: the double-precision arithmetic is
    evaluated exactly as written.
    """
    os.makedirs(os.path.dirname(out), exist_ok=True)
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", "-o", out, src, "-lm"]
        subprocess.check_call(cmd)
    return out


class Oracle:
    """ctypes handle on one compiled copy of the oracle library."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        P, I, L = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        lib.ssm_ref_fwd.argtypes = [P, P, P, I, P, P, P, P, P, P, I, L, L, L, L, P, P, I]
        lib.ssm_ref_fwd.restype = I
        lib.ssm_ref_fwd_channels.argtypes = [P, P, P, I, P, P, P, P, P, P, I, L, L, L, L,
                                             P, L, P, P, I]
        lib.ssm_ref_fwd_channels.restype = I
        lib.ssm_ref_step.argtypes = [P, P, P, P, I, P, P, P, P, P, I, L, L, L, P, I]
        lib.ssm_ref_step.restype = I
        lib.ssm_ref_conv1d.argtypes = [P, P, P, L, P, I, I, L, L, L, P, P, I]
        lib.ssm_ref_conv1d.restype = I
        lib.ssm_ref_conv_fwd.argtypes = [P, P, P, L, P, P, P, I, P, P, P, P, P, P, I, L, L, L, L,
                                         P, P, P, I]
        lib.ssm_ref_conv_fwd.restype = I
        lib.ssm_ref_conv_step.argtypes = [P, P, P, P, P, L, P, P, I, P, P, P, P, P, I, L, L, L, P, I]
        lib.ssm_ref_conv_step.restype = I
        lib.ssm_ref_trap_fwd.argtypes = [P, P, P, I, P, P, P, P, P, P, P, P, P, I, L, L, L, L, P, P, I]
        lib.ssm_ref_trap_fwd.restype = I
        lib.ssm_ref_trap_step.argtypes = [P, P, P, P, I, P, P, P, P, P, P, P, P, I, L, L, L, P, I]
        lib.ssm_ref_trap_step.restype = I
        lib.ssm_ref_bwd.argtypes = [P, P, P, I, P, P, P, P, P, P, P, P, I, L, L, L, L,
                                    P, P, P, P, P, P, P, P, P, I]
        lib.ssm_ref_bwd.restype = I
        lib.ssm_ref_ssd_fwd.argtypes = [P, P, P, I, P, P, P, P, P, I, L, L, L, L, L, L, P, P, I]
        lib.ssm_ref_ssd_fwd.restype = I
        self._lib = lib

    # -- marshalling helpers ---------------------------------------------
    @staticmethod
    def _act(a, dtype_code):
        if a is None:
            return None
        a = np.ascontiguousarray(a)
        want = np.uint16 if dtype_code == 1 else np.float32
        if a.dtype != want:
            raise TypeError(f"activation dtype {a.dtype}, expected {want}")
        return a

    @staticmethod
    def _f32(a):
        if a is None:
            return None
        return np.ascontiguousarray(a, dtype=np.float32)

    @staticmethod
    def _ptr(a):
        return None if a is None else a.ctypes.data

    @staticmethod
    def _dtype_code(x):
        if x.dtype == np.uint16:
            return 1
        if x.dtype == np.float32:
            return 0
        raise TypeError(f"activations must be float32 or bf16 bits (uint16), got {x.dtype}")

    # -- entry points -----------------------------------------------------
    def fwd(self, x, delta, delta_bias, softplus, A, B, C, D, z, h0, threads=0,
            want_h_last=True):
        """Full scan.  Returns (out [b,d,L] float64, h_last [b,d,N] float64 or None)."""
        code = self._dtype_code(x)
        x, delta, B, C, z = (self._act(t, code) for t in (x, delta, B, C, z))
        A, D, delta_bias, h0 = (self._f32(t) for t in (A, D, delta_bias, h0))
        batch, dim, L = x.shape
        N = A.shape[1]
        out = np.empty((batch, dim, L), np.float64)
        hl = np.empty((batch, dim, N), np.float64) if want_h_last else None
        rc = self._lib.ssm_ref_fwd(self._ptr(x), self._ptr(delta), self._ptr(delta_bias),
                                   int(bool(softplus)), self._ptr(A), self._ptr(B), self._ptr(C),
                                   self._ptr(D), self._ptr(z), self._ptr(h0), code,
                                   batch, L, dim, N, self._ptr(out), self._ptr(hl), int(threads))
        if rc != 0:
            raise ValueError("oracle rejected the arguments")
        return out, hl

    def fwd_channels(self, x, delta, delta_bias, softplus, A, B, C, D, z, h0, channels,
                     threads=0):
        """Scan of selected channels (flat index b*dim + d).

        Returns (out [nsel, L] float64, h_last [nsel, N] float64)."""
        code = self._dtype_code(x)
        x, delta, B, C, z = (self._act(t, code) for t in (x, delta, B, C, z))
        A, D, delta_bias, h0 = (self._f32(t) for t in (A, D, delta_bias, h0))
        batch, dim, L = x.shape
        N = A.shape[1]
        chan = np.ascontiguousarray(channels, dtype=np.int64)
        out = np.empty((chan.size, L), np.float64)
        hl = np.empty((chan.size, N), np.float64)
        rc = self._lib.ssm_ref_fwd_channels(
            self._ptr(x), self._ptr(delta), self._ptr(delta_bias), int(bool(softplus)),
            self._ptr(A), self._ptr(B), self._ptr(C), self._ptr(D), self._ptr(z), self._ptr(h0),
            code, batch, L, dim, N, self._ptr(chan), chan.size, self._ptr(out), self._ptr(hl),
            int(threads))
        if rc != 0:
            raise ValueError("oracle rejected the arguments")
        return out, hl

    def step(self, state, x, delta, delta_bias, softplus, A, B, C, D, z, threads=0):
        """One decode step.  `state` ([b,d,N] float64) is updated in place.

        Token tensors: x, delta, z [b,d]; B, C [b,N].  Returns out [b,d] float64."""
        if state.dtype != np.float64 or not state.flags.c_contiguous:
            raise TypeError("state must be a contiguous float64 array")
        code = self._dtype_code(x)
        x, delta, B, C, z = (self._act(t, code) for t in (x, delta, B, C, z))
        A, D, delta_bias = (self._f32(t) for t in (A, D, delta_bias))
        batch, dim = x.shape
        N = A.shape[1]
        out = np.empty((batch, dim), np.float64)
        rc = self._lib.ssm_ref_step(self._ptr(state), self._ptr(x), self._ptr(delta),
                                    self._ptr(delta_bias), int(bool(softplus)), self._ptr(A),
                                    self._ptr(B), self._ptr(C), self._ptr(D), self._ptr(z), code,
                                    batch, dim, N, self._ptr(out), int(threads))
        if rc != 0:
            raise ValueError("oracle rejected the arguments")
        return out


    # -- the short causal convolution in front of the scan -----------------
    def conv1d(self, x, w, bias, conv_state=None, silu=True, threads=0):
        """Causal depthwise convolution of width K = w.shape[1] (then silu).

        x: [b,d,L] stored activations; w: [d,K]; bias: [d] or None;
        conv_state: [b,d,K-1] stored activations or None (zeros).
        Returns (xc [b,d,L] float64, new state [b,d,K-1] float64)."""
        code = self._dtype_code(x)
        x, conv_state = (self._act(t, code) for t in (x, conv_state))
        w, bias = self._f32(w), self._f32(bias)
        batch, dim, L = x.shape
        K = w.shape[1]
        xc = np.empty((batch, dim, L), np.float64)
        st = np.empty((batch, dim, K - 1), np.float64)
        rc = self._lib.ssm_ref_conv1d(self._ptr(x), self._ptr(w), self._ptr(bias), K,
                                      self._ptr(conv_state), int(bool(silu)), code, batch, L, dim,
                                      self._ptr(xc), self._ptr(st), int(threads))
        if rc != 0:
            raise ValueError("oracle rejected the arguments")
        return xc, st

    def conv_fwd(self, x, w, cbias, conv_state, delta, delta_bias, softplus, A, B, C, D, z, h0,
                 threads=0):
        """Convolution + silu, then the scan on its output.

        Returns (out [b,d,L], h_last [b,d,N], new conv state [b,d,K-1]), float64."""
        code = self._dtype_code(x)
        x, conv_state, delta, B, C, z = (self._act(t, code) for t in (x, conv_state, delta, B, C, z))
        w, cbias, A, D, delta_bias, h0 = (self._f32(t) for t in (w, cbias, A, D, delta_bias, h0))
        batch, dim, L = x.shape
        N, K = A.shape[1], w.shape[1]
        out = np.empty((batch, dim, L), np.float64)
        hl = np.empty((batch, dim, N), np.float64)
        st = np.empty((batch, dim, K - 1), np.float64)
        rc = self._lib.ssm_ref_conv_fwd(
            self._ptr(x), self._ptr(w), self._ptr(cbias), K, self._ptr(conv_state), self._ptr(delta),
            self._ptr(delta_bias), int(bool(softplus)), self._ptr(A), self._ptr(B), self._ptr(C),
            self._ptr(D), self._ptr(z), self._ptr(h0), code, batch, L, dim, N, self._ptr(out),
            self._ptr(hl), self._ptr(st), int(threads))
        if rc != 0:
            raise ValueError("oracle rejected the arguments")
        return out, hl, st

    def conv_step(self, conv_state, state, x, w, cbias, delta, delta_bias, softplus, A, B, C, D, z,
                  threads=0):
        """One decode step of convolution + scan.  conv_state ([b,d,K-1]) and
        state ([b,d,N]), both contiguous float64, are updated in place.
        Returns out [b,d] float64."""
        for name, a in (("conv_state", conv_state), ("state", state)):
            if a.dtype != np.float64 or not a.flags.c_contiguous:
                raise TypeError(f"{name} must be a contiguous float64 array")
        code = self._dtype_code(x)
        x, delta, B, C, z = (self._act(t, code) for t in (x, delta, B, C, z))
        w, cbias, A, D, delta_bias = (self._f32(t) for t in (w, cbias, A, D, delta_bias))
        batch, dim = x.shape
        N, K = A.shape[1], w.shape[1]
        out = np.empty((batch, dim), np.float64)
        rc = self._lib.ssm_ref_conv_step(
            self._ptr(conv_state), self._ptr(state), self._ptr(x), self._ptr(w), self._ptr(cbias), K,
            self._ptr(delta), self._ptr(delta_bias), int(bool(softplus)), self._ptr(A), self._ptr(B),
            self._ptr(C), self._ptr(D), self._ptr(z), code, batch, dim, N, self._ptr(out), int(threads))
        if rc != 0:
            raise ValueError("oracle rejected the arguments")
        return out


    # -- the exponential-trapezoidal rule (Mamba-3) -------------------------
    def trap_fwd(self, x, delta, delta_bias, softplus, lam, A, B, C, D, z, h0, x_prev=None, B_prev=None,
                 threads=0):
        """Scan with the exponential-trapezoidal discretisation.  lam: [b,d,L]
        stored activations; x_prev [b,d] and B_prev [b,N]: the input before
        t = 0 (None: zero).  Returns (out [b,d,L], h_last [b,d,N]), float64."""
        code = self._dtype_code(x)
        x, delta, lam, B, C, z, x_prev, B_prev = (self._act(t, code) for t in
                                                  (x, delta, lam, B, C, z, x_prev, B_prev))
        A, D, delta_bias, h0 = (self._f32(t) for t in (A, D, delta_bias, h0))
        batch, dim, L = x.shape
        N = A.shape[1]
        out = np.empty((batch, dim, L), np.float64)
        hl = np.empty((batch, dim, N), np.float64)
        rc = self._lib.ssm_ref_trap_fwd(
            self._ptr(x), self._ptr(delta), self._ptr(delta_bias), int(bool(softplus)), self._ptr(lam),
            self._ptr(A), self._ptr(B), self._ptr(C), self._ptr(D), self._ptr(z), self._ptr(h0),
            self._ptr(x_prev), self._ptr(B_prev), code, batch, L, dim, N, self._ptr(out), self._ptr(hl),
            int(threads))
        if rc != 0:
            raise ValueError("oracle rejected the arguments")
        return out, hl

    def trap_step(self, state, x, delta, delta_bias, softplus, lam, A, B, C, D, z, x_prev=None,
                  B_prev=None, threads=0):
        """One trapezoidal decode step; `state` ([b,d,N] float64) is updated in
        place.  x_prev [b,d], B_prev [b,N]: the previous token's.  Returns out."""
        if state.dtype != np.float64 or not state.flags.c_contiguous:
            raise TypeError("state must be a contiguous float64 array")
        code = self._dtype_code(x)
        x, delta, lam, B, C, z, x_prev, B_prev = (self._act(t, code) for t in
                                                  (x, delta, lam, B, C, z, x_prev, B_prev))
        A, D, delta_bias = (self._f32(t) for t in (A, D, delta_bias))
        batch, dim = x.shape
        N = A.shape[1]
        out = np.empty((batch, dim), np.float64)
        rc = self._lib.ssm_ref_trap_step(
            self._ptr(state), self._ptr(x), self._ptr(delta), self._ptr(delta_bias), int(bool(softplus)),
            self._ptr(lam), self._ptr(A), self._ptr(B), self._ptr(C), self._ptr(D), self._ptr(z),
            self._ptr(x_prev), self._ptr(B_prev), code, batch, dim, N, self._ptr(out), int(threads))
        if rc != 0:
            raise ValueError("oracle rejected the arguments")
        return out


    # -- the backward pass ---------------------------------------------------
    def bwd(self, x, delta, delta_bias, softplus, A, B, C, D, z, h0, dout, dh_last=None, threads=0):
        """Derivatives of a loss L through the forward scan, given dout =
        dL/dout (stored activations, like x) and dh_last = dL/dh_last (float32
        [b,d,N] or None).  Returns a dict of float64 arrays: dx, ddelta, dz
        (None without z) [b,d,L]; dB, dC [b,N,L]; dA [d,N]; dD, dbias [d];
        dh0 [b,d,N]."""
        code = self._dtype_code(x)
        x, delta, B, C, z, dout = (self._act(t, code) for t in (x, delta, B, C, z, dout))
        A, D, delta_bias, h0, dh_last = (self._f32(t) for t in (A, D, delta_bias, h0, dh_last))
        batch, dim, L = x.shape
        N = A.shape[1]
        r = dict(dx=np.empty((batch, dim, L)), ddelta=np.empty((batch, dim, L)),
                 dz=np.empty((batch, dim, L)) if z is not None else None,
                 dB=np.empty((batch, N, L)), dC=np.empty((batch, N, L)), dA=np.empty((dim, N)),
                 dD=np.empty(dim), dbias=np.empty(dim), dh0=np.empty((batch, dim, N)))
        rc = self._lib.ssm_ref_bwd(
            self._ptr(x), self._ptr(delta), self._ptr(delta_bias), int(bool(softplus)), self._ptr(A),
            self._ptr(B), self._ptr(C), self._ptr(D), self._ptr(z), self._ptr(h0), self._ptr(dout),
            self._ptr(dh_last), code, batch, L, dim, N,
            *(self._ptr(r[k]) for k in ("dx", "ddelta", "dz", "dB", "dC", "dA", "dD", "dbias", "dh0")),
            int(threads))
        if rc != 0:
            raise ValueError("oracle rejected the arguments")
        return r


    # -- Mamba-2 SSD (scalar-times-identity transition) ------------------------
    def ssd_fwd(self, x, dt, dt_bias, softplus, A, B, C, D, h0, threads=0):
        """x [b,L,H,P], dt [b,L,H], B and C [b,L,G,N] stored activations; A, dt_bias,
        D [H]; h0 [b,H,P,N] float32 or None.  Returns (y [b,L,H,P], h_last
        [b,H,P,N]), float64."""
        code = self._dtype_code(x)
        x, dt, B, C = (self._act(t, code) for t in (x, dt, B, C))
        A, dt_bias, D, h0 = (self._f32(t) for t in (A, dt_bias, D, h0))
        batch, L, H, P = x.shape
        G, N = B.shape[2], B.shape[3]
        y = np.empty((batch, L, H, P), np.float64)
        hl = np.empty((batch, H, P, N), np.float64)
        rc = self._lib.ssm_ref_ssd_fwd(self._ptr(x), self._ptr(dt), self._ptr(dt_bias), int(bool(softplus)),
                                       self._ptr(A), self._ptr(B), self._ptr(C), self._ptr(D), self._ptr(h0), code,
                                       batch, L, H, P, G, N, self._ptr(y), self._ptr(hl), int(threads))
        if rc != 0:
            raise ValueError("oracle rejected the arguments")
        return y, hl


def load(path: str | None = None) -> Oracle:
    """Build (if needed) and load the oracle library; cached per process."""
    global _lib
    if path is not None:
        return Oracle(path)
    if _lib is None:
        _lib = Oracle(build())
    return _lib


def fwd(*args, **kw):
    return load().fwd(*args, **kw)


def fwd_channels(*args, **kw):
    return load().fwd_channels(*args, **kw)


def step(*args, **kw):
    return load().step(*args, **kw)


def conv1d(*args, **kw):
    return load().conv1d(*args, **kw)


def conv_fwd(*args, **kw):
    return load().conv_fwd(*args, **kw)


def conv_step(*args, **kw):
    return load().conv_step(*args, **kw)


def trap_fwd(*args, **kw):
    return load().trap_fwd(*args, **kw)


def trap_step(*args, **kw):
    return load().trap_step(*args, **kw)


def bwd(*args, **kw):
    return load().bwd(*args, **kw)


def ssd_fwd(*args, **kw):
    return load().ssd_fwd(*args, **kw)
