"""GPU parity of ssm_scan_fwd against the float64 oracle (element by element,
same stored inputs).  Every shape is compared in full: every channel, every
step, and h_last; the large configs in slabs of channels so that the float64
copies stay small.  Every call also checks that no bounded device wait gave
up (ssm_scan_fwd_status)."""
import ctypes

import numpy as np
import pytest
import torch

import workloads
from helpers import check, to_dev, to_np64

pytestmark = pytest.mark.gpu


def _gpu_fwd(inp, want_state=True, h0=None):
    import selective_state_space_38_b200 as ssm
    t = {k: to_dev(v) for k, v in inp.items() if isinstance(v, np.ndarray)}
    out, hl = ssm.ssm_scan_fwd(t["x"], t["delta"], t.get("delta_bias"), inp["softplus"], t["A"],
                               t["B"], t["C"], t.get("D"), t.get("z"),
                               to_dev(h0) if h0 is not None else t.get("h0"),
                               return_last_state=want_state, check=True)
    torch.cuda.synchronize()
    return out, hl


def _oracle(orc, inp, channels=None):
    args = (inp["x"], inp["delta"], inp.get("delta_bias"), inp["softplus"], inp["A"], inp["B"],
            inp["C"], inp.get("D"), inp.get("z"), inp.get("h0"))
    if channels is None:
        return orc.fwd(*args)
    return orc.fwd_channels(*args, channels)


def _dt(inp):
    return "f32" if inp["x"].dtype == np.float32 else "bf16"


SMALL_L = [1, 7, 31, 33, 64, 255, 257, 1000]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("L", SMALL_L)
def test_small_shapes(orc, dtype, L):
    inp = workloads.custom_inputs(2, L, 130, 16, dtype=dtype, seed=L, has_h0=(L % 2 == 1))
    out, hl = _gpu_fwd(inp)
    ref_out, ref_hl = _oracle(orc, inp)
    check(to_np64(out), ref_out, dtype, f"out L={L}")
    check(to_np64(hl), ref_hl, dtype, f"h_last L={L}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_optional_inputs_absent(orc, dtype):
    inp = workloads.custom_inputs(1, 300, 200, 16, dtype=dtype, seed=5)
    inp.update(z=None, D=None, delta_bias=None, h0=None)
    inp["delta"] = inp["delta"]  # raw delta without bias; softplus keeps dt > 0
    out, hl = _gpu_fwd(inp)
    ref_out, ref_hl = _oracle(orc, inp)
    check(to_np64(out), ref_out, dtype, "out (no z/D/bias/h0)")
    check(to_np64(hl), ref_hl, dtype, "h_last (no z/D/bias/h0)")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_softplus_off(orc, dtype):
    inp = workloads.custom_inputs(2, 129, 64, 16, dtype=dtype, seed=6)
    inp["softplus"] = False
    # dt = delta + bias must stay positive and small: use |delta| as stored values
    if dtype == "f32":
        inp["delta"] = np.abs(inp["delta"]) * np.float32(0.1)
    else:
        inp["delta"] = inp["delta"] & np.uint16(0x7FFF)  # clear the sign bit
    inp["delta_bias"] = np.full_like(inp["delta_bias"], 0.01)
    out, hl = _gpu_fwd(inp)
    ref_out, ref_hl = _oracle(orc, inp)
    check(to_np64(out), ref_out, dtype, "out softplus=0")
    check(to_np64(hl), ref_hl, dtype, "h_last softplus=0")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_general_A(orc, dtype):
    """A without the S4D-real structure takes the per-state exp path."""
    inp = workloads.custom_inputs(2, 200, 96, 16, dtype=dtype, seed=7, has_h0=True)
    rng = np.random.default_rng(70)
    inp["A"] = -rng.uniform(0.05, 3.0, size=inp["A"].shape).astype(np.float32)
    out, hl = _gpu_fwd(inp)
    ref_out, ref_hl = _oracle(orc, inp)
    check(to_np64(out), ref_out, dtype, "out general A")
    check(to_np64(hl), ref_hl, dtype, "h_last general A")


def test_mixed_A_rows(orc):
    """Some channels S4D-structured, some not, within one warp."""
    inp = workloads.custom_inputs(1, 100, 64, 16, dtype="bf16", seed=8)
    inp["A"][5] = -np.linspace(0.3, 4.0, 16, dtype=np.float32)
    out, hl = _gpu_fwd(inp)
    ref_out, ref_hl = _oracle(orc, inp)
    check(to_np64(out), ref_out, "bf16", "out mixed A")
    check(to_np64(hl), ref_hl, "bf16", "h_last mixed A")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("A_kind", ["s4d", "general", "mixed"])
@pytest.mark.parametrize("L", [4000, 4001])
def test_time_parallel_schedule(orc, dtype, A_kind, L):
    """Few channel groups over a long sequence take the time-parallel schedule:
    every segment is summarised from a zero state, the summaries are combined
    into start states, and every segment runs again from its own.  Here 2 groups
    (40 channels, the second ragged) over 4000 or 4001 steps, which the schedule
    cuts into 16 segments of 256 with a ragged last one, from a random h0; 4001
    also takes the element-wise (unaligned) loads."""
    inp = workloads.custom_inputs(1, L, 40, 16, dtype=dtype, seed=L + len(A_kind), has_h0=True)
    rng = np.random.default_rng(L)
    if A_kind == "general":
        inp["A"] = -rng.uniform(0.05, 3.0, size=inp["A"].shape).astype(np.float32)
    elif A_kind == "mixed":
        inp["A"][3] = -np.linspace(0.3, 4.0, 16, dtype=np.float32)
    out, hl = _gpu_fwd(inp)
    ref_out, ref_hl = _oracle(orc, inp)
    check(to_np64(out), ref_out, dtype, f"out time-parallel {A_kind} L={L}")
    check(to_np64(hl), ref_hl, dtype, f"h_last time-parallel {A_kind} L={L}")


def test_extreme_dt(orc):
    """dt spanning 1e-6..50: state decay from ~1 (memory) to exactly 0 (reset)."""
    inp = workloads.custom_inputs(1, 257, 64, 16, dtype="bf16", seed=9, has_h0=True)
    bias = np.linspace(-14.0, 50.0, 64).astype(np.float32)
    inp["delta_bias"] = bias
    out, hl = _gpu_fwd(inp)
    ref_out, ref_hl = _oracle(orc, inp)
    check(to_np64(out), ref_out, "bf16", "out extreme dt")
    check(to_np64(hl), ref_hl, "bf16", "h_last extreme dt")


@pytest.mark.parametrize("dim,L", [(130, 96), (40, 4000)])
def test_h_last_in_place_over_h0(orc, dim, L):
    """h_last written over h0.  130 channels x 96 steps runs the chained
    schedule; 40 channels x 4000 steps the time-parallel one, whose second
    pass starts every segment, the first included, from the combined start
    states rather than from h0."""
    import selective_state_space_38_b200 as ssm
    inp = workloads.custom_inputs(2 if dim == 130 else 1, L, dim, 16, dtype="bf16", seed=10 + L,
                                  has_h0=True)
    t = {k: to_dev(v) for k, v in inp.items() if isinstance(v, np.ndarray)}
    h = t["h0"].clone()
    out, hl = ssm.ssm_scan_fwd(t["x"], t["delta"], t["delta_bias"], True, t["A"], t["B"], t["C"],
                               t["D"], t["z"], h, h_last=h, check=True)
    torch.cuda.synchronize()
    assert hl.data_ptr() == h.data_ptr()
    ref_out, ref_hl = _oracle(orc, inp)
    check(to_np64(out), ref_out, "bf16", "out in-place")
    check(to_np64(h), ref_hl, "bf16", "h_last in-place")


def test_workspace_reused_across_shapes(orc):
    """One workspace serves calls of different shapes and schedules in a row:
    every call re-arms its queue and flags."""
    import selective_state_space_38_b200 as ssm
    ws = torch.empty(ssm.ssm_scan_fwd_workspace_size(1, 4000, 40), dtype=torch.uint8, device="cuda")
    cases = [workloads.custom_inputs(1, 4000, 40, 16, seed=31, has_h0=True),   # time-parallel
             workloads.custom_inputs(2, 700, 96, 16, seed=32),                 # chained, 2 segments
             workloads.custom_inputs(1, 4000, 40, 16, seed=33)]
    for i, inp in enumerate(cases):
        assert ws.numel() >= ssm.ssm_scan_fwd_workspace_size(*inp["x"].shape[:1], inp["x"].shape[2],
                                                             inp["x"].shape[1])
        t = {k: to_dev(v) for k, v in inp.items() if isinstance(v, np.ndarray)}
        out, hl = ssm.ssm_scan_fwd(t["x"], t["delta"], t["delta_bias"], True, t["A"], t["B"], t["C"],
                                   t["D"], t["z"], t.get("h0"), workspace=ws, check=True)
        ref_out, ref_hl = _oracle(orc, inp)
        check(to_np64(out), ref_out, "bf16", f"shared workspace call {i} out")
        check(to_np64(hl), ref_hl, "bf16", f"shared workspace call {i} h_last")


@pytest.mark.parametrize("spin_limit", [0, 2000])
def test_wait_timeout_is_reported(orc, spin_limit):
    """A bounded device wait that gives up is reported, and the kernels still
    end.  The test entry point makes every segment after the first wait for a
    flag value that nothing writes; with a bound of 0 (or 2000 polls, about
    0.1 ms) the wait gives up, the kernels run to their end, and the status
    call returns SSM_ERR_TIMEOUT.  The next ordinary call on the same
    workspace is correct and reports success."""
    import selective_state_space_38_b200 as ssm
    lib = ssm.get_lib()
    inp = workloads.custom_inputs(1, 2048, 64, 16, seed=41, has_h0=True)  # 2 groups x 4 segments
    t = {k: to_dev(v) for k, v in inp.items() if isinstance(v, np.ndarray)}
    ws = torch.empty(ssm.ssm_scan_fwd_workspace_size(1, 2048, 64), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(t["x"])
    hl = torch.empty_like(t["h0"])
    dims = ssm.Dims(1, 2048, 64, 16, ssm.SSM_BF16)
    stream = torch.cuda.current_stream()
    rc = lib.ssm_debug_fwd_flag_timeout(
        t["x"].data_ptr(), t["delta"].data_ptr(), t["delta_bias"].data_ptr(), 1, t["A"].data_ptr(),
        t["B"].data_ptr(), t["C"].data_ptr(), t["D"].data_ptr(), t["z"].data_ptr(), t["h0"].data_ptr(),
        out.data_ptr(), hl.data_ptr(), ws.data_ptr(), ws.numel(), spin_limit, ctypes.byref(dims),
        stream.cuda_stream)
    assert rc == 0, ssm.ssm_strerror(rc)
    assert ssm.ssm_scan_fwd_status(ws, stream) == 5
    torch.cuda.synchronize()  # the context is still usable
    out2, hl2 = ssm.ssm_scan_fwd(t["x"], t["delta"], t["delta_bias"], True, t["A"], t["B"], t["C"],
                                 t["D"], t["z"], t["h0"], workspace=ws)
    assert ssm.ssm_scan_fwd_status(ws, stream) == 0
    ref_out, ref_hl = _oracle(orc, inp)
    check(to_np64(out2), ref_out, "bf16", "out after a timed-out call")
    check(to_np64(hl2), ref_hl, "bf16", "h_last after a timed-out call")


def test_chunk_split_matches_full_gpu_scan():
    """Scanning [0, m) then [m, L) from the carried state equals one call."""
    inp = workloads.custom_inputs(2, 1000, 200, 16, dtype="bf16", seed=11, has_h0=True)
    out, hl = _gpu_fwd(inp)
    for m in (1, 333, 512, 999):
        a = {k: (np.ascontiguousarray(v[..., :m]) if k in ("x", "delta", "z", "B", "C") else v)
             for k, v in inp.items()}
        b = {k: (np.ascontiguousarray(v[..., m:]) if k in ("x", "delta", "z", "B", "C") else v)
             for k, v in inp.items()}
        o1, h1 = _gpu_fwd(a)
        b["h0"] = None
        o2, h2 = _gpu_fwd(b, h0=h1.cpu().numpy())
        got = torch.cat([o1, o2], dim=-1)
        check(to_np64(got), to_np64(out), "bf16", f"split m={m} out")
        check(to_np64(h2), to_np64(hl), "bf16", f"split m={m} h_last")


def test_output_guard_bands():
    """The kernel writes exactly [batch][dim][L] and h_last: the bytes
    around both stay untouched (NaN canary)."""
    import selective_state_space_38_b200 as ssm
    inp = workloads.custom_inputs(1, 77, 130, 16, dtype="bf16", seed=12)
    t = {k: to_dev(v) for k, v in inp.items() if isinstance(v, np.ndarray)}
    n_out = 130 * 77
    guard = 64
    big = torch.full((n_out + 2 * guard,), float("nan"), dtype=torch.bfloat16, device="cuda")
    out = big[guard:guard + n_out].view(1, 130, 77)
    hbig = torch.full((130 * 16 + 2 * guard,), float("nan"), dtype=torch.float32, device="cuda")
    hl = hbig[guard:guard + 130 * 16].view(1, 130, 16)
    ssm.ssm_scan_fwd(t["x"], t["delta"], t["delta_bias"], True, t["A"], t["B"], t["C"], t["D"],
                     t["z"], None, out=out, h_last=hl)
    torch.cuda.synchronize()
    assert torch.isnan(big[:guard].float()).all() and torch.isnan(big[-guard:].float()).all()
    assert torch.isnan(hbig[:guard]).all() and torch.isnan(hbig[-guard:]).all()
    assert torch.isfinite(out.float()).all() and torch.isfinite(hl).all()


# ---- the configs ---------------------------------------------------------------
def test_tiny_fp32_full(orc):
    inp = workloads.make_inputs(0)
    out, hl = _gpu_fwd(inp)
    ref_out, ref_hl = _oracle(orc, inp)
    check(to_np64(out), ref_out, "f32", "tiny fp32 out")
    check(to_np64(hl), ref_hl, "f32", "tiny fp32 h_last")


def test_mamba130m_layer_full(orc):
    inp = workloads.make_inputs(1)
    out, hl = _gpu_fwd(inp)
    ref_out, ref_hl = _oracle(orc, inp)
    check(to_np64(out), ref_out, "bf16", "mamba-130m layer out")
    check(to_np64(hl), ref_hl, "bf16", "mamba-130m layer h_last")


def _full_in_slabs(orc, cfg, slab):
    """The whole config against the oracle, `slab` channels at a time."""
    inp = workloads.make_inputs(cfg)
    out, hl = _gpu_fwd(inp)
    c = workloads.CONFIGS[cfg]
    out_all = out.view(c.channels, -1)
    hl_all = hl.view(c.channels, -1)
    worst = 0.0
    for s0 in range(0, c.channels, slab):
        chan = np.arange(s0, min(c.channels, s0 + slab))
        ref_out, ref_hl = _oracle(orc, inp, chan)
        st = check(to_np64(out_all[s0:s0 + len(chan)]), ref_out, "bf16",
                   f"{c.name} out, channels {s0}..{s0 + len(chan) - 1}")
        check(to_np64(hl_all[s0:s0 + len(chan)]), ref_hl, "bf16",
              f"{c.name} h_last, channels {s0}..{s0 + len(chan) - 1}")
        worst = max(worst, st["worst_ratio"])
    return inp, out, hl


def test_mamba2p8b_layer_full(orc):
    _full_in_slabs(orc, 2, 2048)


def test_long_sequence_full_and_split(orc):
    inp, out, hl = _full_in_slabs(orc, 3, 256)
    # state carry across two calls at a non-aligned split point
    m = 65536 + 777
    a = {k: (np.ascontiguousarray(v[..., :m]) if k in ("x", "delta", "z", "B", "C") else v)
         for k, v in inp.items()}
    o1, h1 = _gpu_fwd(a)
    del a
    b = {k: (np.ascontiguousarray(v[..., m:]) if k in ("x", "delta", "z", "B", "C") else v)
         for k, v in inp.items()}
    b["h0"] = None
    o2, h2 = _gpu_fwd(b, h0=h1.cpu().numpy())
    check(to_np64(o1), to_np64(out[..., :m]), "bf16", "long sequence split, first part")
    check(to_np64(o2), to_np64(out[..., m:]), "bf16", "long sequence split, second part")
    check(to_np64(h2), to_np64(hl), "bf16", "long sequence split h_last")
