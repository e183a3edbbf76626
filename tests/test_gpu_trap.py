"""GPU parity of the exponential-trapezoidal scan (ssm_trap_scan_fwd) and of
its decode step (ssm_trap_scan_step) against the float64 oracle, element by
element on the same stored inputs.

The rule ("Mamba3" posts, section on the new discretisation scheme) mixes
both ends of each step's interval by a data-dependent lambda; the kernel
carries h~_t = h_t - lam_t dt_t x_t B_t so that each state costs as much as
the Euler rule, and turns it back into h at the end of the sequence."""
import numpy as np
import pytest
import torch

import workloads
from helpers import check, to_dev, to_np64

pytestmark = pytest.mark.gpu


def _trap_inputs(batch, L, dim, dtype="bf16", seed=0, has_h0=True, prev=True):
    inp = workloads.custom_inputs(batch, L, dim, 16, dtype=dtype, seed=seed, has_h0=has_h0)
    rng = np.random.default_rng(seed + 500)
    lam = rng.uniform(0.0, 1.0, (batch, dim, L)).astype(np.float32)
    xp = rng.standard_normal((batch, dim)).astype(np.float32)
    bp = rng.standard_normal((batch, 16)).astype(np.float32)
    cvt = (lambda a: a) if dtype == "f32" else workloads.f32_to_bf16_bits
    inp["lam"] = cvt(lam)
    inp["x_prev"] = cvt(xp) if prev else None
    inp["B_prev"] = cvt(bp) if prev else None
    return inp


def _gpu(inp, h0=None, ws=None):
    import selective_state_space_38_b200 as ssm
    t = {k: to_dev(v) for k, v in inp.items() if isinstance(v, np.ndarray)}
    out, hl = ssm.ssm_trap_scan_fwd(t["x"], t["delta"], t["delta_bias"], True, t["lam"], t["A"], t["B"], t["C"],
                                    t["D"], t["z"], to_dev(h0) if h0 is not None else t.get("h0"),
                                    t.get("x_prev"), t.get("B_prev"), workspace=ws, check=True)
    torch.cuda.synchronize()
    return out, hl


def _ref(orc, inp):
    return orc.trap_fwd(inp["x"], inp["delta"], inp["delta_bias"], True, inp["lam"], inp["A"], inp["B"], inp["C"],
                        inp["D"], inp["z"], inp["h0"], inp["x_prev"], inp["B_prev"])


def _dt(inp):
    return "f32" if inp["x"].dtype == np.float32 else "bf16"


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("L", [1, 2, 7, 33, 64, 255, 257, 1000])
def test_small_shapes(orc, dtype, L):
    inp = _trap_inputs(2, L, 130, dtype=dtype, seed=L, prev=(L % 2 == 1), has_h0=(L % 3 != 0))
    out, hl = _gpu(inp)
    ref_out, ref_hl = _ref(orc, inp)
    check(to_np64(out), ref_out, _dt(inp), f"trap out L={L}")
    check(to_np64(hl), ref_hl, _dt(inp), f"trap h_last L={L}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_general_A(orc, dtype):
    inp = _trap_inputs(1, 300, 96, dtype=dtype, seed=7)
    inp["A"] = -np.random.default_rng(70).uniform(0.05, 3.0, size=inp["A"].shape).astype(np.float32)
    out, hl = _gpu(inp)
    ref_out, ref_hl = _ref(orc, inp)
    check(to_np64(out), ref_out, _dt(inp), "trap general A out")
    check(to_np64(hl), ref_hl, _dt(inp), "trap general A h_last")


def test_lambda_one_equals_euler_scan():
    """lam = 1: the same outputs as ssm_scan_fwd (within the parity tolerance)."""
    import selective_state_space_38_b200 as ssm
    inp = _trap_inputs(2, 777, 200, seed=8)
    inp["lam"] = workloads.f32_to_bf16_bits(np.ones_like(workloads.bf16_bits_to_f32(inp["lam"])))
    out, hl = _gpu(inp)
    t = {k: to_dev(v) for k, v in inp.items() if isinstance(v, np.ndarray)}
    o2, h2 = ssm.ssm_scan_fwd(t["x"], t["delta"], t["delta_bias"], True, t["A"], t["B"], t["C"], t["D"], t["z"],
                              t["h0"])
    check(to_np64(out), to_np64(o2), "bf16", "trap lam=1 vs Euler out")
    check(to_np64(hl), to_np64(h2), "bf16", "trap lam=1 vs Euler h_last")


@pytest.mark.parametrize("A_kind", ["s4d", "general"])
@pytest.mark.parametrize("L", [4000, 4001])
def test_time_parallel_schedule(orc, A_kind, L):
    """Few groups: segments start mid-sequence, where the step before the
    segment (x, lam, dt, B) comes from the inputs themselves; the two-pass
    schedule combines the carried h~ states."""
    inp = _trap_inputs(1, L, 40, seed=L)
    if A_kind == "general":
        inp["A"] = -np.random.default_rng(L).uniform(0.05, 3.0, size=inp["A"].shape).astype(np.float32)
    out, hl = _gpu(inp)
    ref_out, ref_hl = _ref(orc, inp)
    check(to_np64(out), ref_out, "bf16", f"trap time-parallel out {A_kind} L={L}")
    check(to_np64(hl), ref_hl, "bf16", f"trap time-parallel h_last {A_kind} L={L}")


def test_chained_segments_and_split(orc):
    """Many groups (chained schedule, 512-step segments) and a split into two
    calls carrying h_last and the last token's x and B."""
    inp = _trap_inputs(2, 1500, 600, seed=9)
    out, hl = _gpu(inp)
    ref_out, ref_hl = _ref(orc, inp)
    check(to_np64(out), ref_out, "bf16", "trap chained out")
    check(to_np64(hl), ref_hl, "bf16", "trap chained h_last")
    m = 700
    seq = ("x", "delta", "z", "B", "C", "lam")
    a = {k: (np.ascontiguousarray(v[..., :m]) if k in seq else v) for k, v in inp.items()}
    b = {k: (np.ascontiguousarray(v[..., m:]) if k in seq else v) for k, v in inp.items()}
    o1, h1 = _gpu(a)
    b["h0"] = None
    b["x_prev"] = np.ascontiguousarray(inp["x"][..., m - 1])
    b["B_prev"] = np.ascontiguousarray(inp["B"][..., m - 1])
    o2, h2 = _gpu(b, h0=h1.cpu().numpy())
    check(to_np64(torch.cat([o1, o2], -1)), ref_out, "bf16", "trap split out")
    check(to_np64(h2), ref_hl, "bf16", "trap split h_last")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_step_against_oracle_and_fwd(orc, dtype):
    import selective_state_space_38_b200 as ssm
    T = 10
    inp = _trap_inputs(3, T, 200, dtype=dtype, seed=11)
    t = {k: to_dev(v) for k, v in inp.items() if isinstance(v, np.ndarray)}
    fwd_out, fwd_hl = ssm.ssm_trap_scan_fwd(t["x"], t["delta"], t["delta_bias"], True, t["lam"], t["A"], t["B"],
                                            t["C"], t["D"], t["z"], t["h0"], t["x_prev"], t["B_prev"])
    st = t["h0"].clone()
    st64 = inp["h0"].astype(np.float64)
    xp, bp = inp["x_prev"], inp["B_prev"]
    outs = []
    for s in range(T):
        tok = {k: np.ascontiguousarray(inp[k][..., s]) for k in ("x", "delta", "z", "B", "C", "lam")}
        o = ssm.ssm_trap_scan_step(st, to_dev(tok["x"]), to_dev(tok["delta"]), t["delta_bias"], True,
                                   to_dev(tok["lam"]), t["A"], to_dev(tok["B"]), to_dev(tok["C"]), t["D"],
                                   to_dev(tok["z"]), to_dev(xp), to_dev(bp))
        r = orc.trap_step(st64, tok["x"], tok["delta"], inp["delta_bias"], True, tok["lam"], inp["A"], tok["B"],
                          tok["C"], inp["D"], tok["z"], xp, bp)
        torch.cuda.synchronize()
        check(to_np64(o), r, _dt(inp), f"trap step {s} out")
        outs.append(o)
        xp, bp = tok["x"], tok["B"]
    check(to_np64(st), st64, _dt(inp), "trap step state")
    check(to_np64(torch.stack(outs, -1)), to_np64(fwd_out), _dt(inp), "trap steps vs fwd out")
    check(to_np64(st), to_np64(fwd_hl), _dt(inp), "trap steps vs fwd state")


def test_mamba2p8b_layer_trap_full(orc):
    """The Mamba-2.8B mixer-layer shape (4 x 4096 x 5120, bf16) with a
    lambda ~ U(0, 1) per token and channel, against the oracle on every channel."""
    c = workloads.CONFIGS[2]
    inp = workloads.make_inputs(2)
    rng = np.random.default_rng(2002)
    inp["lam"] = workloads.f32_to_bf16_bits(rng.uniform(0, 1, inp["x"].shape).astype(np.float32))
    inp["x_prev"] = None
    inp["B_prev"] = None
    out, hl = _gpu(inp)
    out_all, hl_all = out.view(c.channels, -1), hl.view(c.channels, -1)
    slab = 1024
    for s0 in range(0, c.channels, slab):
        b0, d0 = s0 // c.dim, s0 % c.dim
        sub = dict(inp)
        for k in ("x", "delta", "z", "lam"):
            sub[k] = np.ascontiguousarray(inp[k][b0:b0 + 1, d0:d0 + slab])
        for k in ("B", "C"):
            sub[k] = np.ascontiguousarray(inp[k][b0:b0 + 1])
        for k in ("A", "D", "delta_bias"):
            sub[k] = np.ascontiguousarray(inp[k][d0:d0 + slab])
        ro, rh = _ref(orc, sub)
        check(to_np64(out_all[s0:s0 + slab]), ro.reshape(slab, -1), "bf16", f"trap layer out {s0}")
        check(to_np64(hl_all[s0:s0 + slab]), rh.reshape(slab, -1), "bf16", f"trap layer h_last {s0}")
