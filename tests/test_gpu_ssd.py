"""GPU parity of the Mamba-2 SSD forward (ssm_ssd_fwd, tensor cores) against
the float64 oracle's recurrence, element by element on the same stored inputs.

The kernel computes each 128-step chunk through its semiseparable (attention-
like) form as dense products on tcgen05; the oracle runs the plain recurrence
H_t = exp(dt_t A) H_{t-1} + (dt_t x_t) B_t^T, y_t = H_t C_t + D x_t."""
import numpy as np
import pytest
import torch

import workloads
from helpers import check, to_dev, to_np64

pytestmark = pytest.mark.gpu


def ssd_inputs(batch, L, H, G, seed=0, h0=True, P=64, N=128):
    rng = np.random.default_rng(seed)
    bf = workloads.f32_to_bf16_bits
    dt0 = np.exp(rng.uniform(np.log(1e-3), np.log(1e-1), H))
    return dict(x=bf(rng.standard_normal((batch, L, H, P)).astype(np.float32)),
                dt=bf((rng.standard_normal((batch, L, H)) * 0.1).astype(np.float32)),
                dt_bias=np.log(np.expm1(dt0)).astype(np.float32),
                A=-rng.uniform(1.0, 16.0, H).astype(np.float32),
                B=bf(rng.standard_normal((batch, L, G, N)).astype(np.float32)),
                C=bf(rng.standard_normal((batch, L, G, N)).astype(np.float32)),
                D=np.ones(H, np.float32),
                h0=rng.standard_normal((batch, H, P, N)).astype(np.float32) if h0 else None)


def _gpu(inp, softplus=True):
    import selective_state_space_38_b200 as ssm
    t = {k: to_dev(v) for k, v in inp.items() if isinstance(v, np.ndarray)}
    y, hl = ssm.ssm_ssd_fwd(t["x"], t["dt"], t["dt_bias"], softplus, t["A"], t["B"], t["C"], t.get("D"), t.get("h0"),
                            check=True)
    torch.cuda.synchronize()
    return y, hl


def _ref(orc, inp, softplus=True):
    return orc.ssd_fwd(inp["x"], inp["dt"], inp["dt_bias"], softplus, inp["A"], inp["B"], inp["C"], inp.get("D"),
                       inp.get("h0"))


@pytest.mark.parametrize("L", [1, 100, 128, 129, 300, 1000])
def test_small_shapes(orc, L):
    inp = ssd_inputs(2, L, 4, 2, seed=L, h0=(L % 2 == 0))
    y, hl = _gpu(inp)
    ry, rh = _ref(orc, inp)
    check(to_np64(y), ry, "bf16", f"ssd y L={L}")
    check(to_np64(hl), rh, "bf16", f"ssd h_last L={L}")


def test_no_skip_and_one_group(orc):
    inp = ssd_inputs(1, 400, 6, 1, seed=7)
    inp["D"] = None
    y, hl = _gpu(inp)
    ry, rh = _ref(orc, inp)
    check(to_np64(y), ry, "bf16", "ssd no D y")
    check(to_np64(hl), rh, "bf16", "ssd no D h_last")


def test_mamba2_layer_shape_all_heads(orc):
    """The Mamba-2 2.7B-like layer shape (4 x 4096, 80 heads of 64, one group,
    state 128): every batch, step and head against the oracle."""
    inp = ssd_inputs(4, 4096, 80, 1, seed=2, h0=False)
    y, hl = _gpu(inp)
    ry, rh = _ref(orc, inp)
    check(to_np64(y), ry, "bf16", "ssd layer y")
    check(to_np64(hl), rh, "bf16", "ssd layer h_last")


@pytest.mark.parametrize("step", [0.002, 2.0])
def test_decay_ranges(orc, step):
    """Small steps keep every |running sum of dt A| of a chunk below 80, where the
    kernel forms exp(cs_i - cs_j) as exp(cs_i) exp(-cs_j); large steps (sums in
    the thousands) take the per-element exponential.  Both against the oracle."""
    inp = ssd_inputs(2, 300, 4, 2, seed=11, h0=True)
    inp["dt_bias"] = np.log(np.expm1(np.full(4, step))).astype(np.float32)
    y, hl = _gpu(inp)
    ry, rh = _ref(orc, inp)
    check(to_np64(y), ry, "bf16", f"ssd decay step {step} y")
    check(to_np64(hl), rh, "bf16", f"ssd decay step {step} h_last")


def test_softplus_off(orc):
    """dt used as given (dt + dt_bias, no softplus), positive."""
    inp = ssd_inputs(2, 200, 4, 1, seed=12, h0=True)
    rng = np.random.default_rng(13)
    inp["dt"] = workloads.f32_to_bf16_bits(rng.uniform(0.001, 0.05, inp["dt"].shape).astype(np.float32))
    inp["dt_bias"] = np.full(4, 0.01, np.float32)
    y, hl = _gpu(inp, softplus=False)
    ry, rh = _ref(orc, inp, softplus=False)
    check(to_np64(y), ry, "bf16", "ssd softplus off y")
    check(to_np64(hl), rh, "bf16", "ssd softplus off h_last")


@pytest.mark.parametrize("L", [100, 300])
def test_split_sequences(orc, L):
    """More sequences (3 x 64 heads) than SMs: with the sized workspace the CTAs
    walk equal numbers of chunks and hand the state of a split sequence on
    through the workspace (ragged last chunk at L = 300); with a 256-byte
    workspace every sequence gets its own CTA.  Both against the oracle."""
    import selective_state_space_38_b200 as ssm
    inp = ssd_inputs(3, L, 64, 2, seed=20 + L, h0=True)
    t = {k: to_dev(v) for k, v in inp.items() if isinstance(v, np.ndarray)}
    ry, rh = _ref(orc, inp)
    sized = ssm.ssm_ssd_fwd_workspace_size(3, 64, t["x"].device)
    assert sized > 256
    got = []
    for nbytes in (sized, 256):
        ws = torch.empty(nbytes, dtype=torch.uint8, device=t["x"].device)
        y, hl = ssm.ssm_ssd_fwd(t["x"], t["dt"], t["dt_bias"], True, t["A"], t["B"], t["C"], t["D"], t["h0"],
                                workspace=ws, check=True)
        torch.cuda.synchronize()
        check(to_np64(y), ry, "bf16", f"ssd split y L={L} ws={nbytes}")
        check(to_np64(hl), rh, "bf16", f"ssd split h_last L={L} ws={nbytes}")
        got.append((y, hl))
    # a chunk's arithmetic does not depend on which CTA runs it, and the handed-on
    # state is the float32 state itself: both launches agree bit for bit
    assert torch.equal(got[0][0], got[1][0]) and torch.equal(got[0][1], got[1][1])


@pytest.mark.parametrize("spin_limit", [0, 2000])
def test_handoff_wait_timeout_is_reported(orc, spin_limit):
    """A hand-off wait of the split launch that gives up is reported, and the
    kernel still ends.  The test entry point makes every CTA that continues a
    split sequence wait for a flag value that nothing writes; with a bound of
    0 (or 2000 polls) the wait gives up, the status call returns
    SSM_ERR_TIMEOUT, and the next ordinary call on the same workspace is
    correct and reports success."""
    import ctypes
    import selective_state_space_38_b200 as ssm
    if torch.cuda.get_device_properties(0).multi_processor_count >= 3 * 64:
        pytest.skip("the launch splits sequences only with more sequences than SMs")
    lib = ssm.get_lib()
    inp = ssd_inputs(3, 300, 64, 2, seed=51, h0=True)
    t = {k: to_dev(v) for k, v in inp.items() if isinstance(v, np.ndarray)}
    ws = torch.empty(ssm.ssm_ssd_fwd_workspace_size(3, 64, t["x"].device), dtype=torch.uint8, device="cuda")
    y = torch.empty_like(t["x"])
    hl = torch.empty(t["h0"].shape, dtype=torch.float32, device="cuda")
    dims = ssm.SsdDims(3, 300, 64, 64, 2, 128, ssm.SSM_BF16)
    stream = torch.cuda.current_stream()
    rc = lib.ssm_debug_ssd_flag_timeout(
        t["x"].data_ptr(), t["dt"].data_ptr(), t["dt_bias"].data_ptr(), 1, t["A"].data_ptr(), t["B"].data_ptr(),
        t["C"].data_ptr(), t["D"].data_ptr(), t["h0"].data_ptr(), y.data_ptr(), hl.data_ptr(), ws.data_ptr(),
        ws.numel(), spin_limit, ctypes.byref(dims), stream.cuda_stream)
    assert rc == 0, ssm.ssm_strerror(rc)
    assert ssm.ssm_scan_fwd_status(ws, stream) == 5
    torch.cuda.synchronize()  # the context is still usable
    y2, hl2 = ssm.ssm_ssd_fwd(t["x"], t["dt"], t["dt_bias"], True, t["A"], t["B"], t["C"], t["D"], t["h0"],
                              workspace=ws, check=True)
    torch.cuda.synchronize()
    ry, rh = _ref(orc, inp)
    check(to_np64(y2), ry, "bf16", "ssd y after a timed-out call")
    check(to_np64(hl2), rh, "bf16", "ssd h_last after a timed-out call")
