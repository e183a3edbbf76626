"""Checks that pin the float64 oracle to facts other than its own loop.

Each pin takes an oracle handle (``oracle.Oracle``) and raises AssertionError
when the oracle disagrees with what the mathematics fixes.  The expected values
are computed here by independent routes: closed forms, numpy/scipy library
routines, the convolutional mode of an LTI system, chunk-split invariance and
brute-force evaluation of every bracketing of the associative combine.

The mutation test runs every pin against deliberately broken copies of the
oracle and requires each copy to fail at least one pin.
"""
from __future__ import annotations

import itertools
import math
from functools import lru_cache

import numpy as np
from scipy.special import expit

RTOL = 1e-11


def _rng(seed):
    return np.random.default_rng(seed)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _close(got, want, rtol=RTOL, atol=1e-13, what=""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    err = np.abs(got - want)
    lim = atol + rtol * np.abs(want)
    bad = err > lim
    assert not bad.any(), f"{what}: max err {err.max():.3e} at {np.argwhere(bad)[0]}"


def _rand_case(seed, b=2, d=3, n=4, L=5, h0=True, z=True, Dskip=True, bias=True):
    r = _rng(seed)
    return dict(
        x=_f32(r.standard_normal((b, d, L))),
        delta=_f32(r.standard_normal((b, d, L)) * 0.5),
        z=_f32(r.standard_normal((b, d, L))) if z else None,
        B=_f32(r.standard_normal((b, n, L))),
        C=_f32(r.standard_normal((b, n, L))),
        A=_f32(-r.uniform(0.2, 2.0, (d, n))),
        D=_f32(r.standard_normal(d)) if Dskip else None,
        delta_bias=_f32(r.standard_normal(d) * 0.3) if bias else None,
        h0=_f32(r.standard_normal((b, d, n))) if h0 else None,
        softplus=True,
    )


def _call(orc, c, **over):
    a = dict(c)
    a.update(over)
    return orc.fwd(a["x"], a["delta"], a["delta_bias"], a["softplus"], a["A"], a["B"], a["C"],
                   a["D"], a["z"], a["h0"])


def _softplus_lib(v):
    # numpy's log(exp(0) + exp(v)) is softplus without our formula
    return np.logaddexp(0.0, v)


# ---------------------------------------------------------------------------
def pin_single_step_closed_form(orc):
    """(a) L = 1: one ZOH/Euler step from h0, readout, D skip and silu gate,
    written as one vectorised expression (no loop over t or n)."""
    for seed, sp in ((1, True), (2, False)):
        c = _rand_case(seed, L=1)
        c["softplus"] = sp
        x, v = c["x"].astype(np.float64), c["delta"].astype(np.float64)
        v = v + c["delta_bias"].astype(np.float64)[None, :, None]
        dt = _softplus_lib(v) if sp else v                       # [b,d,1]
        A = c["A"].astype(np.float64)                              # [d,n]
        Bm, Cm = c["B"].astype(np.float64), c["C"].astype(np.float64)  # [b,n,1]
        h0 = c["h0"].astype(np.float64)                            # [b,d,n]
        h1 = np.exp(dt * A[None]) * h0 + dt * x * np.transpose(Bm, (0, 2, 1))
        y = np.einsum("bdn,bn->bd", h1, Cm[:, :, 0])[..., None] + c["D"][None, :, None] * x
        zz = c["z"].astype(np.float64)
        want = y * zz * expit(zz)
        out, hl = _call(orc, c)
        _close(out, want, what="L=1 out")
        _close(hl, h1, what="L=1 h_last")


def pin_hand_values(orc):
    """(a') Exactly representable single step worked by hand: softplus off,
    dt = ln 2 and A = -1 give Abar = 1/2; x = 2, B = 3, C = 5, D = 0.5,
    h0 = 4, no gate.  h1 = 2 + 6 ln 2, y = 5 h1 + 1."""
    ln2 = math.log(2.0)
    one = lambda v: np.full((1, 1, 1), v, np.float32)
    c = dict(x=one(2.0), delta=_f32(np.full((1, 1, 1), ln2)), z=None, B=one(3.0), C=one(5.0),
             A=_f32([[-1.0]]), D=_f32([0.5]), delta_bias=None, h0=one(4.0), softplus=False)
    dt = float(np.float32(ln2))
    out, hl = _call(orc, c)
    h1 = math.exp(-dt) * 4.0 + dt * 6.0
    _close(hl[0, 0, 0], h1, rtol=1e-15, what="hand h1")
    _close(out[0, 0, 0], 5.0 * h1 + 1.0, rtol=1e-15, what="hand y")
    assert abs(hl[0, 0, 0] - (2.0 + 6.0 * ln2)) < 1e-6


def pin_geometric_sum(orc):
    """(b) dt, B, C, x (and z) constant over t: h_t = a^(t+1) h0 + u B (1 - a^(t+1)) / (1 - a),
    a = exp(dt A), u = dt x; y_t = C.h_t + D x, gated."""
    r = _rng(3)
    b, d, n, L = 2, 3, 5, 40
    xv = r.standard_normal((b, d, 1))
    vv = r.standard_normal((b, d, 1)) * 0.5
    zv = r.standard_normal((b, d, 1))
    Bv = r.standard_normal((b, n, 1))
    Cv = r.standard_normal((b, n, 1))
    c = dict(x=_f32(np.repeat(xv, L, 2)), delta=_f32(np.repeat(vv, L, 2)),
             z=_f32(np.repeat(zv, L, 2)), B=_f32(np.repeat(Bv, L, 2)), C=_f32(np.repeat(Cv, L, 2)),
             A=_f32(-r.uniform(0.1, 1.5, (d, n))), D=_f32(r.standard_normal(d)),
             delta_bias=_f32(r.standard_normal(d) * 0.2), h0=_f32(r.standard_normal((b, d, n))),
             softplus=True)
    dt = _softplus_lib(c["delta"][:, :, :1].astype(np.float64) + c["delta_bias"][None, :, None])
    a = np.exp(dt * c["A"][None].astype(np.float64))                     # [b,d,n]
    u = dt * c["x"][:, :, :1].astype(np.float64)                           # [b,d,1]
    Bn = np.transpose(c["B"][:, :, :1].astype(np.float64), (0, 2, 1))      # [b,1,n]
    Cn = np.transpose(c["C"][:, :, :1].astype(np.float64), (0, 2, 1))
    t = np.arange(L)[None, None, None, :] + 1.0                            # [1,1,1,L]
    ap = a[..., None] ** t                                                 # [b,d,n,L]
    h = ap * c["h0"].astype(np.float64)[..., None] + (u * Bn)[..., None] * (1 - ap) / (1 - a)[..., None]
    y = np.einsum("bdnl,bdn->bdl", h, np.broadcast_to(Cn, a.shape)) + \
        c["D"][None, :, None] * c["x"].astype(np.float64)
    zz = c["z"].astype(np.float64)
    want = y * zz * expit(zz)
    out, hl = _call(orc, c)
    _close(out, want, rtol=1e-10, what="geometric out")
    _close(hl, h[..., -1], rtol=1e-10, what="geometric h_last")


def pin_convolution_mode(orc):
    """(c) Input-independent dt, B, C with h0 = 0 make the system LTI, so the
    scan equals the convolutional mode y = K * x + D x with kernel
    K_k = sum_n C_n Abar_n^k dt B_n (computed with numpy.convolve)."""
    r = _rng(4)
    b, d, n, L = 2, 3, 6, 64
    vv = r.standard_normal((1, d, 1)) * 0.5
    Bv = r.standard_normal((b, n, 1))
    Cv = r.standard_normal((b, n, 1))
    x = _f32(r.standard_normal((b, d, L)))
    c = dict(x=x, delta=_f32(np.repeat(np.repeat(vv, b, 0), L, 2)), z=None,
             B=_f32(np.repeat(Bv, L, 2)), C=_f32(np.repeat(Cv, L, 2)),
             A=_f32(-r.uniform(0.05, 1.0, (d, n))), D=_f32(r.standard_normal(d)),
             delta_bias=_f32(r.standard_normal(d) * 0.2), h0=None, softplus=True)
    out, _ = _call(orc, c)
    dt = _softplus_lib(c["delta"][0, :, 0].astype(np.float64) + c["delta_bias"])   # [d]
    k = np.arange(L)
    for bi in range(b):
        for di in range(d):
            abar = np.exp(dt[di] * c["A"][di].astype(np.float64))                # [n]
            K = ((c["C"][bi, :, 0].astype(np.float64) * dt[di] * c["B"][bi, :, 0])[:, None]
                 * abar[:, None] ** k[None, :]).sum(0)
            xs = x[bi, di].astype(np.float64)
            want = np.convolve(xs, K)[:L] + c["D"][di] * xs
            _close(out[bi, di], want, rtol=1e-10, atol=1e-12, what=f"conv b{bi} d{di}")


def pin_chunk_split(orc):
    """(d) Scanning [0, m) and then [m, L) from the carried state equals the
    full scan, for several split points m."""
    c = _rand_case(5, b=2, d=3, n=4, L=37)
    out, hl = _call(orc, c)
    seq_keys = ("x", "delta", "z", "B", "C")
    for m in (1, 5, 16, 36):
        first = {k: (np.ascontiguousarray(v[..., :m]) if k in seq_keys else v) for k, v in c.items()}
        second = {k: (np.ascontiguousarray(v[..., m:]) if k in seq_keys else v) for k, v in c.items()}
        o1, h1 = _call(orc, first)
        second["h0"] = _f32(h1)
        o2, h2 = _call(orc, second)
        # the carried state is rounded to float32 between the two calls
        _close(o1, out[..., :m], rtol=1e-12, what=f"split m={m} first")
        _close(o2, out[..., m:], rtol=2e-5, atol=2e-5, what=f"split m={m} second")
        _close(h2, hl, rtol=2e-5, atol=2e-5, what=f"split m={m} h_last")


def pin_segment_summaries(orc):
    """(d') The identity behind the time-parallel schedule: scanning segment s
    from a zero state gives e_s, the decays of the segment multiply to
    P_s[n] = exp(A[d, n] sum_t dt_t), and the state at the end of segment s is
    P_s h_s + e_s, where h_s is the state entering it (h_0 = h0).  P_s is
    computed here from its closed form (softplus by numpy's logaddexp), not by
    the oracle, so a wrong decay or a wrong state carry fails."""
    c = _rand_case(13, b=2, d=3, n=4, L=40)
    seq_keys = ("x", "delta", "z", "B", "C")
    dt = np.logaddexp(0.0, c["delta"].astype(np.float64) + c["delta_bias"].astype(np.float64)[None, :, None])
    A = c["A"].astype(np.float64)
    h = c["h0"].astype(np.float64)
    for lo in range(0, 40, 8):
        hi = lo + 8
        seg = {k: (np.ascontiguousarray(v[..., lo:hi]) if k in seq_keys else v) for k, v in c.items()}
        _, e = _call(orc, seg, h0=None)
        P = np.exp(A[None, :, :] * dt[..., lo:hi].sum(-1)[..., None])
        h = P * h + e
        prefix = {k: (np.ascontiguousarray(v[..., :hi]) if k in seq_keys else v) for k, v in c.items()}
        _, want = _call(orc, prefix)
        _close(h, want, rtol=1e-11, atol=1e-13, what=f"segment summaries up to t={hi}")


@lru_cache(maxsize=None)
def _bracketings(lo, hi):
    """All full bracketings of the elements lo..hi-1 as nested tuples."""
    if hi - lo == 1:
        return [lo]
    res = []
    for m in range(lo + 1, hi):
        for left in _bracketings(lo, m):
            for right in _bracketings(m, hi):
                res.append((left, right))
    return res


def _eval_bracket(tree, pairs):
    """Combine affine maps h -> a h + b, earlier map first:
    (a1, b1) then (a2, b2) gives (a2 a1, a2 b1 + b2)."""
    if isinstance(tree, int):
        return pairs[tree]
    a1, b1 = _eval_bracket(tree[0], pairs)
    a2, b2 = _eval_bracket(tree[1], pairs)
    return a2 * a1, a2 * b1 + b2


def pin_associative_brute_force(orc):
    """(e) On tiny L, every bracketing of the associative combine of the
    per-step pairs (Abar_t, Bbar_t x_t) gives the state the oracle reaches; the
    prefix of each t gives y_t.  This is the algebra a parallel scan relies on."""
    for L in (1, 2, 3, 5, 6):
        c = _rand_case(10 + L, b=1, d=2, n=3, L=L)
        out, hl = _call(orc, c)
        dt = _softplus_lib(c["delta"].astype(np.float64) + c["delta_bias"][None, :, None])  # [1,d,L]
        for di in range(2):
            for ni in range(3):
                pairs = [(math.exp(dt[0, di, t] * float(c["A"][di, ni])),
                          dt[0, di, t] * float(c["B"][0, ni, t]) * float(c["x"][0, di, t]))
                         for t in range(L)]
                h0 = float(c["h0"][0, di, ni])
                for tree in _bracketings(0, L):
                    a, bb = _eval_bracket(tree, pairs)
                    assert abs(a * h0 + bb - hl[0, di, ni]) <= 1e-12 * (1 + abs(hl[0, di, ni])), \
                        (L, di, ni, tree)
        # outputs from prefixes, bracketed right-to-left
        for di in range(2):
            for t in range(L):
                y = float(c["D"][di]) * float(c["x"][0, di, t])
                for ni in range(3):
                    pairs = [(math.exp(dt[0, di, s] * float(c["A"][di, ni])),
                              dt[0, di, s] * float(c["B"][0, ni, s]) * float(c["x"][0, di, s]))
                             for s in range(t + 1)]
                    tree = _bracketings(0, t + 1)[-1]
                    a, bb = _eval_bracket(tree, pairs)
                    y += float(c["C"][0, ni, t]) * (a * float(c["h0"][0, di, ni]) + bb)
                zz = float(c["z"][0, di, t])
                y *= zz * expit(zz)
                assert abs(y - out[0, di, t]) <= 1e-11 * (1 + abs(y)), (L, di, t)


def pin_degenerate(orc):
    """Special cases: dt = 0 keeps h = h0; A -> -inf makes the system
    memoryless (h_t = dt B_t x_t); optional inputs absent mean zero / identity."""
    c = _rand_case(20, L=7)
    c0 = dict(c, delta=np.zeros_like(c["delta"]), delta_bias=None, softplus=False)
    out, hl = _call(orc, c0)
    _close(hl, c["h0"], rtol=0, atol=0, what="dt=0 state")
    D64, x64 = c["D"].astype(np.float64), c["x"].astype(np.float64)
    y = np.einsum("bdn,bnl->bdl", c["h0"].astype(np.float64), c["C"].astype(np.float64)) + \
        D64[None, :, None] * x64
    zz = c["z"].astype(np.float64)
    _close(out, y * zz * expit(zz), rtol=1e-12, what="dt=0 out")

    cinf = dict(c, A=np.full_like(c["A"], -1e30))
    out, hl = _call(orc, cinf)
    dt = _softplus_lib(c["delta"].astype(np.float64) + c["delta_bias"][None, :, None])
    ht = dt[:, :, None, :] * c["B"].astype(np.float64)[:, None] * x64[:, :, None, :]
    y = np.einsum("bdnl,bnl->bdl", ht, c["C"].astype(np.float64)) + D64[None, :, None] * x64
    _close(out, y * zz * expit(zz), rtol=1e-12, what="memoryless out")
    _close(hl, ht[..., -1], rtol=1e-12, what="memoryless h_last")

    # no h0 / D / z / bias equals passing zeros / no gate
    cn = dict(c, h0=None, D=None, z=None, delta_bias=None)
    cz = dict(c, h0=np.zeros_like(c["h0"]), D=np.zeros_like(c["D"]), z=None,
              delta_bias=np.zeros_like(c["delta_bias"]))
    o1, h1 = _call(orc, cn)
    o2, h2 = _call(orc, cz)
    _close(o1, o2, rtol=0, atol=0, what="optional args")
    _close(h1, h2, rtol=0, atol=0, what="optional args h")


def pin_softplus_extremes(orc):
    """dt = softplus(v) is read back through A = 0, h0 = 0, B = x = 1, L = 1
    (then h1 = dt): compare with math.log1p(math.exp(v)) and its limits."""
    vs = np.array([-80.0, -20.0, -3.0, 0.0, 0.5, 8.0, 30.0, 300.0], np.float32)
    d = vs.size
    c = dict(x=np.ones((1, d, 1), np.float32), delta=vs.reshape(1, d, 1).copy(), z=None,
             B=np.ones((1, 1, 1), np.float32), C=np.ones((1, 1, 1), np.float32),
             A=np.zeros((d, 1), np.float32), D=None, delta_bias=None, h0=None, softplus=True)
    _, hl = _call(orc, c)
    for i, v in enumerate(vs.astype(np.float64)):
        want = math.log1p(math.exp(v))  # the definition; no overflow for these v
        assert abs(hl[0, i, 0] - want) <= 1e-14 * max(1.0, abs(want)) + 1e-300, (v, hl[0, i, 0])
    assert hl[0, 0, 0] > 0.0  # softplus(-80) = 1.8e-35 is not flushed to zero


def pin_bf16_widening(orc):
    """bf16 inputs are widened exactly: the oracle on bf16 bit patterns equals
    the oracle on the same values given as float32."""
    c = _rand_case(30, L=9)
    def bits(a):
        u = np.ascontiguousarray(a, np.float32).view(np.uint32)
        return (u >> 16).astype(np.uint16)  # truncation: any bf16 value will do
    cb = {k: (bits(v) if k in ("x", "delta", "z", "B", "C") else v) for k, v in c.items()}
    cf = {k: ((bits(v).astype(np.uint32) << 16).view(np.float32) if k in ("x", "delta", "z", "B", "C")
              else v) for k, v in c.items()}
    o1, h1 = _call(orc, cb)
    o2, h2 = _call(orc, cf)
    _close(o1, o2, rtol=0, atol=0, what="bf16 widening")
    _close(h1, h2, rtol=0, atol=0, what="bf16 widening h")


def pin_step_equals_scan(orc):
    """The recurrent mode: T single steps from h0 equal one scan over T tokens;
    channel-subset entry equals the full scan on those channels."""
    c = _rand_case(40, b=2, d=3, n=4, L=6)
    out, hl = _call(orc, c)
    state = c["h0"].astype(np.float64).copy()
    for t in range(6):
        tok = {k: np.ascontiguousarray(c[k][..., t]) for k in ("x", "delta", "z", "B", "C")}
        o = orc.step(state, tok["x"], tok["delta"], c["delta_bias"], True, c["A"], tok["B"], tok["C"],
                     c["D"], tok["z"])
        _close(o, out[..., t], rtol=1e-13, what=f"step t={t}")
    _close(state, hl, rtol=1e-13, what="step state")
    sel = np.array([5, 0, 3])
    o, h = orc.fwd_channels(c["x"], c["delta"], c["delta_bias"], True, c["A"], c["B"], c["C"],
                            c["D"], c["z"], c["h0"], sel)
    _close(o, out.reshape(6, 6)[sel], rtol=0, atol=0, what="channel subset out")
    _close(h, hl.reshape(6, 4)[sel], rtol=0, atol=0, what="channel subset h")


# ---------------------------------------------------------------------------
# The short causal convolution in front of the scan (convolution, activation,
# then the scan: Mamba, Appendix D "Memory").

def _conv_case(seed, b=2, d=3, n=4, L=11, K=4, state=True):
    r = _rng(seed)
    c = _rand_case(seed, b=b, d=d, n=n, L=L)
    c["w"] = _f32(r.standard_normal((d, K)) * 0.7)
    c["cbias"] = _f32(r.standard_normal(d) * 0.3)
    c["conv_state"] = _f32(r.standard_normal((b, d, K - 1))) if (state and K > 1) else None
    return c


def _conv_fwd(orc, c, **over):
    a = dict(c)
    a.update(over)
    return orc.conv_fwd(a["x"], a["w"], a["cbias"], a["conv_state"], a["delta"], a["delta_bias"],
                        a["softplus"], a["A"], a["B"], a["C"], a["D"], a["z"], a["h0"])


def pin_conv_numpy_convolve(orc):
    """The convolution is numpy.convolve of the state-padded row with the
    reversed taps (the last tap multiplies the current input), plus the bias,
    then silu (scipy's expit); the new state is the last K-1 inputs."""
    for K, L, state in ((4, 11, True), (4, 2, True), (3, 9, False), (1, 5, False), (2, 1, True)):
        c = _conv_case(50 + K + L, K=K, L=L, state=state)
        xc, st = orc.conv1d(c["x"], c["w"], c["cbias"], c["conv_state"], silu=True)
        pre, _ = orc.conv1d(c["x"], c["w"], c["cbias"], c["conv_state"], silu=False)
        b, d, _ = c["x"].shape
        for bi in range(b):
            for di in range(d):
                hist = (c["conv_state"][bi, di].astype(np.float64) if c["conv_state"] is not None
                        else np.zeros(K - 1))
                row = np.concatenate([hist, c["x"][bi, di].astype(np.float64)])
                want = np.convolve(row, c["w"][di, ::-1].astype(np.float64), mode="valid") + c["cbias"][di]
                _close(pre[bi, di], want, rtol=1e-13, atol=1e-14, what=f"conv K={K} L={L}")
                _close(xc[bi, di], want * expit(want), rtol=1e-13, atol=1e-14, what=f"conv silu K={K}")
                _close(st[bi, di], row[len(row) - (K - 1):], rtol=0, atol=0, what=f"conv state K={K} L={L}")


def pin_conv_impulse(orc):
    """Brute force on the tap order: a unit impulse at step s, zero bias and
    no silu, gives w[d, K-1-j] at step s+j for j < K and zero elsewhere; an
    impulse held in the state (j steps before the call) appears at t = K-2-j."""
    K, L = 4, 9
    w = _f32(np.arange(1, 2 * K + 1, dtype=np.float32).reshape(2, K))
    for s in range(L):
        x = np.zeros((1, 2, L), np.float32)
        x[0, :, s] = 1.0
        pre, _ = orc.conv1d(x, w, None, None, silu=False)
        for di in range(2):
            want = np.zeros(L)
            for j in range(K):
                if s + j < L:
                    want[s + j] = w[di, K - 1 - j]
            _close(pre[0, di], want, rtol=0, atol=0, what=f"impulse at {s}")
    for j in range(K - 1):
        st = np.zeros((1, 2, K - 1), np.float32)
        st[0, :, K - 2 - j] = 1.0  # the input j steps before t = 0
        pre, _ = orc.conv1d(np.zeros((1, 2, L), np.float32), w, None, st, silu=False)
        for di in range(2):
            want = np.zeros(L)
            for t in range(L):
                k = K - 1 - (t + 1 + j)  # the impulse sits at s = -1 - j
                if 0 <= k < K:
                    want[t] = w[di, k]
            _close(pre[0, di], want, rtol=0, atol=0, what=f"state impulse {j}")


def pin_conv_feeds_scan(orc):
    """The fused path is the composition of the convolution (pinned above) and
    the scan (pinned by the pins before): conv_fwd equals fwd run on the
    convolution's output, up to the float32 rounding of that output."""
    for K in (4, 1):
        c = _conv_case(60 + K, K=K, L=13)
        out, hl, st = _conv_fwd(orc, c)
        xc, st2 = orc.conv1d(c["x"], c["w"], c["cbias"], c["conv_state"], silu=True)
        o2, h2 = _call(orc, c, x=_f32(xc))
        _close(out, o2, rtol=1e-6, atol=1e-6, what=f"conv then scan K={K}")
        _close(hl, h2, rtol=1e-6, atol=1e-6, what=f"conv then scan h K={K}")
        _close(st, st2, rtol=0, atol=0, what=f"conv then scan state K={K}")


def pin_conv_split(orc):
    """Two calls continue one: [0, m) and then [m, L) with the new convolution
    state and h_last carried over equal one call over [0, L), including splits
    shorter than the convolution window."""
    c = _conv_case(70, L=17, K=4)
    out, hl, st = _conv_fwd(orc, c)
    seq_keys = ("x", "delta", "z", "B", "C")
    for m in (1, 2, 3, 8, 16):
        first = {k: (np.ascontiguousarray(v[..., :m]) if k in seq_keys else v) for k, v in c.items()}
        second = {k: (np.ascontiguousarray(v[..., m:]) if k in seq_keys else v) for k, v in c.items()}
        o1, h1, s1 = _conv_fwd(orc, first)
        second["h0"] = _f32(h1)
        second["conv_state"] = _f32(s1)  # raw float32 inputs: exact
        o2, h2, s2 = _conv_fwd(orc, second)
        _close(o1, out[..., :m], rtol=1e-12, what=f"conv split m={m} first")
        _close(o2, out[..., m:], rtol=2e-5, atol=2e-5, what=f"conv split m={m} second")
        _close(h2, hl, rtol=2e-5, atol=2e-5, what=f"conv split m={m} h_last")
        _close(s2, st, rtol=0, atol=0, what=f"conv split m={m} state")


def pin_conv_step_equals_fwd(orc):
    """The recurrent mode of the block: T single steps (convolution window from
    the carried inputs, then the SSM step) equal one call over T tokens."""
    c = _conv_case(80, L=7, K=4)
    out, hl, st = _conv_fwd(orc, c)
    cs = c["conv_state"].astype(np.float64).copy()
    state = c["h0"].astype(np.float64).copy()
    for t in range(7):
        tok = {k: np.ascontiguousarray(c[k][..., t]) for k in ("x", "delta", "z", "B", "C")}
        o = orc.conv_step(cs, state, tok["x"], c["w"], c["cbias"], tok["delta"], c["delta_bias"], True,
                          c["A"], tok["B"], tok["C"], c["D"], tok["z"])
        _close(o, out[..., t], rtol=1e-13, atol=1e-15, what=f"conv step t={t}")
    _close(state, hl, rtol=1e-13, what="conv step state")
    _close(cs, st, rtol=0, atol=0, what="conv step window")


# ---------------------------------------------------------------------------
# The exponential-trapezoidal discretisation ("Mamba3" posts: both ends of the
# interval, mixed by a data-dependent lambda; second order).

def _trap_case(seed, b=2, d=3, n=4, L=9, prev=True):
    r = _rng(seed)
    c = _rand_case(seed, b=b, d=d, n=n, L=L)
    c["lam"] = _f32(r.uniform(0.0, 1.0, (b, d, L)))
    c["x_prev"] = _f32(r.standard_normal((b, d))) if prev else None
    c["B_prev"] = _f32(r.standard_normal((b, n))) if prev else None
    return c


def _trap(orc, c, **over):
    a = dict(c)
    a.update(over)
    return orc.trap_fwd(a["x"], a["delta"], a["delta_bias"], a["softplus"], a["lam"], a["A"], a["B"],
                        a["C"], a["D"], a["z"], a["h0"], a["x_prev"], a["B_prev"])


def pin_trap_lambda_one_is_euler(orc):
    """lambda = 1 drops the interval's start: the rule is Mamba-1's Euler
    input step, whatever the previous input."""
    c = _trap_case(90, L=12)
    out, hl = _trap(orc, c, lam=np.ones_like(c["lam"]))
    o2, h2 = _call(orc, c)
    _close(out, o2, rtol=1e-13, atol=1e-14, what="trap lambda=1 out")
    _close(hl, h2, rtol=1e-13, atol=1e-14, what="trap lambda=1 h_last")


def pin_trap_constant_inputs(orc):
    """Constant dt, lambda, B, x: h_0 = alpha h0 + beta v_prev + gamma v and
    h_t = alpha h_{t-1} + (beta + gamma) v after it, a geometric sum; v = B x,
    alpha = exp(dt A), beta = (1 - lambda) dt alpha, gamma = lambda dt."""
    r = _rng(91)
    b, d, n, L = 2, 3, 4, 30
    rep = lambda a: _f32(np.repeat(a, L, -1))
    c = dict(x=rep(r.standard_normal((b, d, 1))), delta=rep(r.standard_normal((b, d, 1)) * 0.4),
             z=None, B=rep(r.standard_normal((b, n, 1))), C=rep(r.standard_normal((b, n, 1))),
             A=_f32(-r.uniform(0.1, 1.5, (d, n))), D=None, delta_bias=_f32(r.standard_normal(d) * 0.2),
             h0=_f32(r.standard_normal((b, d, n))), softplus=True,
             lam=rep(r.uniform(0, 1, (b, d, 1))), x_prev=_f32(r.standard_normal((b, d))),
             B_prev=_f32(r.standard_normal((b, n))))
    dt = np.logaddexp(0.0, c["delta"][..., :1].astype(np.float64) + c["delta_bias"][None, :, None])  # [b,d,1]
    lam = c["lam"][..., :1].astype(np.float64)
    al = np.exp(dt * c["A"][None].astype(np.float64))                                             # [b,d,n]
    be, ga = (1 - lam) * dt * al, lam * dt
    v = c["x"][..., :1].astype(np.float64) * np.transpose(c["B"][..., :1], (0, 2, 1)).astype(np.float64)
    vp = c["x_prev"][..., None].astype(np.float64) * c["B_prev"][:, None, :].astype(np.float64)
    h_first = al * c["h0"] + be * vp + ga * v
    t = np.arange(L)[None, None, None, :]
    ap = al[..., None] ** t
    h = ap * h_first[..., None] + ((be + ga) * v)[..., None] * (1 - ap) / (1 - al)[..., None]
    y = np.einsum("bdnl,bn->bdl", h, c["C"][..., 0].astype(np.float64))
    out, hl = _trap(orc, c)
    _close(out, y, rtol=1e-10, atol=1e-12, what="trap constant out")
    _close(hl, h[..., -1], rtol=1e-10, atol=1e-12, what="trap constant h_last")


def pin_trap_second_order(orc):
    """The rule is second order for lambda = 1/2 and first order for lambda = 1.
    The scalar system h' = a h + b cos(w s), h(0) = 0, has the exact solution
    h(T) = b (a e^{aT} - a cos wT + w sin wT) / (a^2 + w^2); n steps of
    dt = T / n with x_t = cos(w (t+1) dt) and x_prev = cos(0) approximate it,
    and halving dt divides the error by about 4 (lambda = 1/2) or 2 (lambda = 1)."""
    a, bb, w, T = -0.7, 1.3, 2.0, 3.0
    exact = bb * (a * math.exp(a * T) - a * math.cos(w * T) + w * math.sin(w * T)) / (a * a + w * w)

    def err(n, lam):
        dtv = T / n
        s = (np.arange(n) + 1) * dtv
        c = dict(x=_f32(np.cos(w * s)).reshape(1, 1, n), delta=_f32(np.full((1, 1, n), dtv)), z=None,
                 B=_f32(np.full((1, 1, n), bb)), C=np.zeros((1, 1, n), np.float32), A=_f32([[a]]), D=None,
                 delta_bias=None, h0=None, softplus=False, lam=_f32(np.full((1, 1, n), lam)),
                 x_prev=_f32([[1.0]]), B_prev=_f32([[bb]]))
        _, hl = _trap(orc, c)
        return abs(hl[0, 0, 0] - exact)

    for lam, lo, hi in ((0.5, 3.6, 4.4), (1.0, 1.8, 2.2)):
        errs = [err(n, lam) for n in (32, 64, 128)]
        for e1, e2 in zip(errs, errs[1:]):
            assert lo < e1 / e2 < hi, (lam, errs)
    assert err(128, 0.5) < 1e-3 * err(128, 1.0) ** 0.5


def pin_trap_convolution_mode(orc):
    """LTI case (constant dt, lambda, B, C; h0 = 0; nothing before t = 0):
    y = K * x + D x with K_0 = sum_n C_n gamma B_n and
    K_k = sum_n C_n alpha_n^(k-1) (alpha_n gamma + beta_n) B_n for k >= 1."""
    r = _rng(92)
    b, d, n, L = 1, 2, 5, 40
    c = _trap_case(92, b=b, d=d, n=n, L=L, prev=False)
    vv = r.standard_normal((1, d, 1)) * 0.4
    c.update(delta=_f32(np.repeat(vv, L, 2)), B=_f32(np.repeat(r.standard_normal((b, n, 1)), L, 2)),
             C=_f32(np.repeat(r.standard_normal((b, n, 1)), L, 2)), h0=None, z=None,
             lam=_f32(np.repeat(r.uniform(0, 1, (1, d, 1)), L, 2)))
    out, _ = _trap(orc, c)
    dt = np.logaddexp(0.0, c["delta"][0, :, 0].astype(np.float64) + c["delta_bias"].astype(np.float64))
    for di in range(d):
        lam = float(c["lam"][0, di, 0])
        al = np.exp(dt[di] * c["A"][di].astype(np.float64))
        be, ga = (1 - lam) * dt[di] * al, lam * dt[di]
        Bn, Cn = c["B"][0, :, 0].astype(np.float64), c["C"][0, :, 0].astype(np.float64)
        K = np.empty(L)
        K[0] = (Cn * ga * Bn).sum()
        for k in range(1, L):
            K[k] = (Cn * al ** (k - 1) * (al * ga + be) * Bn).sum()
        xs = c["x"][0, di].astype(np.float64)
        want = np.convolve(xs, K)[:L] + c["D"][di] * xs
        _close(out[0, di], want, rtol=1e-10, atol=1e-12, what=f"trap conv mode d{di}")


def pin_trap_split_and_step(orc):
    """Two calls continue one when h_last and the last token's x and B are
    carried over; T decode steps (each given the previous token) equal one call."""
    c = _trap_case(93, L=15)
    out, hl = _trap(orc, c)
    seq = ("x", "delta", "z", "B", "C", "lam")
    for m in (1, 6, 14):
        first = {k: (np.ascontiguousarray(v[..., :m]) if k in seq else v) for k, v in c.items()}
        second = {k: (np.ascontiguousarray(v[..., m:]) if k in seq else v) for k, v in c.items()}
        o1, h1 = _trap(orc, first)
        second.update(h0=_f32(h1), x_prev=np.ascontiguousarray(c["x"][..., m - 1]),
                      B_prev=np.ascontiguousarray(c["B"][..., m - 1]))
        o2, h2 = _trap(orc, second)
        _close(o1, out[..., :m], rtol=1e-12, what=f"trap split m={m} first")
        _close(o2, out[..., m:], rtol=2e-5, atol=2e-5, what=f"trap split m={m} second")
        _close(h2, hl, rtol=2e-5, atol=2e-5, what=f"trap split m={m} h_last")
    state = c["h0"].astype(np.float64).copy()
    xp, bp = c["x_prev"], c["B_prev"]
    for t in range(15):
        tok = {k: np.ascontiguousarray(c[k][..., t]) for k in seq}
        o = orc.trap_step(state, tok["x"], tok["delta"], c["delta_bias"], True, tok["lam"], c["A"], tok["B"],
                          tok["C"], c["D"], tok["z"], xp, bp)
        _close(o, out[..., t], rtol=1e-13, atol=1e-15, what=f"trap step t={t}")
        xp, bp = tok["x"], tok["B"]
    _close(state, hl, rtol=1e-13, what="trap step state")


# ---------------------------------------------------------------------------
# The backward pass (reverse-mode derivatives of the forward scan).

def _bwd(orc, c, dout, dh_last=None, **over):
    a = dict(c)
    a.update(over)
    return orc.bwd(a["x"], a["delta"], a["delta_bias"], a["softplus"], a["A"], a["B"], a["C"], a["D"],
                   a["z"], a["h0"], dout, dh_last)


def pin_bwd_finite_differences(orc):
    """Every derivative against central differences of the forward oracle:
    the loss is L = sum(dout * out) + sum(dh_last * h_last); each input element
    is moved by +-2^-12 (as far as float32 storage allows; the quotient uses
    the stored values), so the derivative is pinned to ~1e-7 by the forward
    definition alone."""
    for softplus, zgate in ((True, True), (False, False)):
        c = _rand_case(100 + softplus, b=2, d=3, n=4, L=6, z=zgate)
        c["softplus"] = softplus
        if not softplus:
            c["delta"] = _f32(np.abs(c["delta"]) * 0.3)
        r = _rng(101)
        dout = _f32(r.standard_normal(c["x"].shape))
        dhl = _f32(r.standard_normal(c["h0"].shape))
        g = _bwd(orc, c, dout, dhl)

        def loss(cc):
            out, hl = _call(orc, cc)
            return float((dout.astype(np.float64) * out).sum() + (dhl.astype(np.float64) * hl).sum())

        names = [("x", "dx"), ("delta", "ddelta"), ("B", "dB"), ("C", "dC"), ("A", "dA"), ("D", "dD"),
                 ("delta_bias", "dbias"), ("h0", "dh0")] + ([("z", "dz")] if zgate else [])
        for key, gk in names:
            base = c[key]
            fd = np.empty(base.shape)
            for idx in np.ndindex(base.shape):
                up, dn = base.copy(), base.copy()
                up[idx] = np.float32(float(base[idx]) + 2.0 ** -12)
                dn[idx] = np.float32(float(base[idx]) - 2.0 ** -12)
                fd[idx] = (loss(dict(c, **{key: up})) - loss(dict(c, **{key: dn}))) / \
                    (float(up[idx]) - float(dn[idx]))
            _close(g[gk], fd, rtol=2e-5, atol=2e-6, what=f"d{key} (softplus={softplus})")


def pin_bwd_split(orc):
    """The chain rule across a split: the backward of [m, L) gives dh0, which
    is the dh_last of [0, m); the two halves' derivatives are the full ones
    (the sums over time of dA, dD, dbias add up)."""
    c = _rand_case(110, b=2, d=3, n=4, L=13)
    r = _rng(111)
    dout = _f32(r.standard_normal(c["x"].shape))
    dhl = _f32(r.standard_normal(c["h0"].shape))
    full = _bwd(orc, c, dout, dhl)
    seq = ("x", "delta", "z", "B", "C")
    for m in (1, 5, 12):
        first = {k: (np.ascontiguousarray(v[..., :m]) if k in seq else v) for k, v in c.items()}
        second = {k: (np.ascontiguousarray(v[..., m:]) if k in seq else v) for k, v in c.items()}
        _, h_mid = _call(orc, first)
        second["h0"] = _f32(h_mid)  # the state between the halves, rounded to float32 storage
        g2 = _bwd(orc, second, np.ascontiguousarray(dout[..., m:]), dhl)
        g1 = _bwd(orc, first, np.ascontiguousarray(dout[..., :m]), _f32(g2["dh0"]))
        for k in ("dx", "ddelta", "dz"):
            _close(np.concatenate([g1[k], g2[k]], -1), full[k], rtol=1e-5, atol=1e-6, what=f"split {k} m={m}")
        for k in ("dB", "dC"):
            _close(np.concatenate([g1[k], g2[k]], -1), full[k], rtol=1e-5, atol=1e-6, what=f"split {k} m={m}")
        for k in ("dA", "dD", "dbias"):
            _close(g1[k] + g2[k], full[k], rtol=1e-5, atol=1e-6, what=f"split {k} m={m}")
        _close(g1["dh0"], full["dh0"], rtol=1e-5, atol=1e-6, what=f"split dh0 m={m}")


# ---------------------------------------------------------------------------
# Mamba-2 SSD: scalar-times-identity transition, multi-dimensional heads.

def _ssd_case(seed, b=2, L=9, H=4, P=3, G=2, N=5, h0=True):
    r = _rng(seed)
    return dict(x=_f32(r.standard_normal((b, L, H, P))), dt=_f32(r.standard_normal((b, L, H)) * 0.5),
                dt_bias=_f32(r.standard_normal(H) * 0.3), softplus=True, A=_f32(-r.uniform(0.2, 2.0, H)),
                B=_f32(r.standard_normal((b, L, G, N))), C=_f32(r.standard_normal((b, L, G, N))),
                D=_f32(r.standard_normal(H)), h0=_f32(r.standard_normal((b, H, P, N))) if h0 else None)


def _ssd(orc, c, **over):
    a = dict(c)
    a.update(over)
    return orc.ssd_fwd(a["x"], a["dt"], a["dt_bias"], a["softplus"], a["A"], a["B"], a["C"], a["D"], a["h0"])


def pin_ssd_semiseparable_form(orc):
    """The attention-like dual: y = M x + D x with the lower-triangular
    (semiseparable) matrix M[t, s] = (C_t . B_s) exp(A sum_{r=s+1..t} dt_r) dt_s,
    plus the h0 term C_t . (exp(A sum_{r<=t} dt_r) h0); built with numpy einsum
    and cumulative sums, no recurrence."""
    c = _ssd_case(120)
    y, hl = _ssd(orc, c)
    b, L, H, P = c["x"].shape
    G, N = c["B"].shape[2:]
    dt = np.logaddexp(0.0, c["dt"].astype(np.float64) + c["dt_bias"][None, None, :])   # [b,L,H]
    cum = np.cumsum(dt * c["A"][None, None, :], axis=1)                                  # [b,L,H]
    grp = np.arange(H) // (H // G)
    Bh = c["B"].astype(np.float64)[:, :, grp, :]                                         # [b,L,H,N]
    Ch = c["C"].astype(np.float64)[:, :, grp, :]
    CB = np.einsum("bthn,bshn->bhts", Ch, Bh)
    dec = np.exp(cum.transpose(0, 2, 1)[:, :, :, None] - cum.transpose(0, 2, 1)[:, :, None, :])  # [b,H,t,s]
    mask = np.tril(np.ones((L, L)))[None, None]
    M = CB * dec * mask * dt.transpose(0, 2, 1)[:, :, None, :]
    want = np.einsum("bhts,bshp->bthp", M, c["x"].astype(np.float64))
    want += c["D"].astype(np.float64)[None, None, :, None] * c["x"].astype(np.float64)
    h0 = c["h0"].astype(np.float64)
    want += np.einsum("bthn,bhpn,bth->bthp", Ch, h0, np.exp(cum))
    _close(y, want, rtol=1e-11, atol=1e-12, what="ssd semiseparable form")
    hw = np.einsum("bhs,bshp,bshn->bhpn", (np.exp(cum[:, -1:, :] - cum) * dt).transpose(0, 2, 1),
                   c["x"].astype(np.float64), Bh) + np.exp(cum[:, -1, :])[:, :, None, None] * h0
    _close(hl, hw, rtol=1e-11, atol=1e-12, what="ssd semiseparable h_last")


def pin_ssd_reduces_to_s6(orc):
    """P = N = 1, one head: the SSD recurrence is the selective scan of one
    channel with a one-dimensional state (the S6 oracle, no gate)."""
    c = _ssd_case(121, b=2, L=11, H=1, P=1, G=1, N=1)
    y, hl = _ssd(orc, c)
    s6 = dict(x=np.ascontiguousarray(c["x"][:, :, 0, 0][:, None, :]), delta=np.ascontiguousarray(c["dt"][:, :, 0][:, None, :]),
              z=None, B=np.ascontiguousarray(c["B"][:, :, 0, 0][:, None, :]), C=np.ascontiguousarray(c["C"][:, :, 0, 0][:, None, :]),
              A=_f32(c["A"].reshape(1, 1)), D=c["D"], delta_bias=c["dt_bias"],
              h0=_f32(c["h0"].reshape(2, 1, 1)), softplus=True)
    o2, h2 = _call(orc, s6)
    _close(y[:, :, 0, 0], o2[:, 0, :], rtol=1e-13, atol=1e-14, what="ssd vs s6 out")
    _close(hl.reshape(2, 1), h2.reshape(2, 1), rtol=1e-13, atol=1e-14, what="ssd vs s6 state")


def pin_ssd_split(orc):
    """Two calls continue one when h_last is carried."""
    c = _ssd_case(122, L=14)
    y, hl = _ssd(orc, c)
    for m in (1, 7, 13):
        first = dict(c, x=np.ascontiguousarray(c["x"][:, :m]), dt=np.ascontiguousarray(c["dt"][:, :m]),
                     B=np.ascontiguousarray(c["B"][:, :m]), C=np.ascontiguousarray(c["C"][:, :m]))
        y1, h1 = _ssd(orc, first)
        second = dict(c, x=np.ascontiguousarray(c["x"][:, m:]), dt=np.ascontiguousarray(c["dt"][:, m:]),
                      B=np.ascontiguousarray(c["B"][:, m:]), C=np.ascontiguousarray(c["C"][:, m:]), h0=_f32(h1))
        y2, h2 = _ssd(orc, second)
        _close(y1, y[:, :m], rtol=1e-12, what=f"ssd split m={m} first")
        _close(y2, y[:, m:], rtol=2e-5, atol=2e-5, what=f"ssd split m={m} second")
        _close(h2, hl, rtol=2e-5, atol=2e-5, what=f"ssd split m={m} state")


ALL_PINS = [
    pin_single_step_closed_form,
    pin_hand_values,
    pin_geometric_sum,
    pin_convolution_mode,
    pin_chunk_split,
    pin_segment_summaries,
    pin_associative_brute_force,
    pin_degenerate,
    pin_softplus_extremes,
    pin_bf16_widening,
    pin_step_equals_scan,
    pin_conv_numpy_convolve,
    pin_conv_impulse,
    pin_conv_feeds_scan,
    pin_conv_split,
    pin_conv_step_equals_fwd,
    pin_trap_lambda_one_is_euler,
    pin_trap_constant_inputs,
    pin_trap_second_order,
    pin_trap_convolution_mode,
    pin_trap_split_and_step,
    pin_bwd_finite_differences,
    pin_bwd_split,
    pin_ssd_semiseparable_form,
    pin_ssd_reduces_to_s6,
    pin_ssd_split,
]
