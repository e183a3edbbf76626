"""GPU parity of the backward pass (ssm_scan_bwd) against the float64 oracle,
every derivative compared element by element on the same stored inputs.

The backward pass stores the state at chunk starts only and recomputes the
states chunk by chunk (Mamba, Appendix D "Memory"); lanes of a warp run
across time, with warp-shuffle scans for the states and for the adjoint."""
import numpy as np
import pytest
import torch

import workloads
from helpers import check, to_dev, to_np64

pytestmark = pytest.mark.gpu

KEYS = ("dx", "ddelta", "dz", "dB", "dC", "dA", "dD", "dbias", "dh0")


def _case(batch, L, dim, dtype="bf16", seed=0, has_h0=True, dh_last=True):
    inp = workloads.custom_inputs(batch, L, dim, 16, dtype=dtype, seed=seed, has_h0=has_h0)
    rng = np.random.default_rng(seed + 7000)
    dout = rng.standard_normal(inp["x"].shape).astype(np.float32)
    inp["dout"] = dout if dtype == "f32" else workloads.f32_to_bf16_bits(dout)
    inp["dh_last"] = rng.standard_normal((batch, dim, 16)).astype(np.float32) if dh_last else None
    return inp


def _run(orc, inp, what):
    import selective_state_space_38_b200 as ssm
    t = {k: to_dev(v) for k, v in inp.items() if isinstance(v, np.ndarray)}
    g = ssm.ssm_scan_bwd(t["x"], t["delta"], t.get("delta_bias"), inp["softplus"], t["A"], t["B"], t["C"],
                         t.get("D"), t.get("z"), t.get("h0"), t["dout"], t.get("dh_last"))
    torch.cuda.synchronize()
    ref = orc.bwd(inp["x"], inp["delta"], inp.get("delta_bias"), inp["softplus"], inp["A"], inp["B"], inp["C"],
                  inp.get("D"), inp.get("z"), inp.get("h0"), inp["dout"], inp.get("dh_last"))
    dt = "f32bwd" if inp["x"].dtype == np.float32 else "bf16"
    for k in KEYS:
        if ref[k] is None:
            assert inp.get("z") is None and k == "dz"
            continue
        check(to_np64(g[k]), ref[k], dt, f"{what} {k}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
# 17, 48, 49: a last chunk of 17, 16 and 17 steps around the checkpoint inside a
# 32-step chunk (bf16), and segments of one step
@pytest.mark.parametrize("L", [1, 7, 17, 48, 49, 128, 129, 300, 1000])
def test_small_shapes(orc, dtype, L):
    """Ragged chunks (L not a multiple of 128) and a ragged channel block (70
    channels = 2 blocks of 32 + 6)."""
    _run(orc, _case(2, L, 70, dtype=dtype, seed=L, has_h0=(L % 2 == 1), dh_last=(L % 3 != 0)), f"L={L}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_general_A_and_mixed_rows(orc, dtype):
    inp = _case(1, 400, 64, dtype=dtype, seed=5)
    rng = np.random.default_rng(50)
    inp["A"] = -rng.uniform(0.05, 3.0, size=inp["A"].shape).astype(np.float32)
    inp["A"][3] = -(np.arange(16, dtype=np.float32) + 1) * 0.5  # one S4D-structured row
    _run(orc, inp, "general A")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_optional_inputs_absent(orc, dtype):
    inp = _case(2, 260, 40, dtype=dtype, seed=6, has_h0=False, dh_last=False)
    inp.update(z=None, D=None, delta_bias=None)
    _run(orc, inp, "no z/D/bias/h0/dh_last")


def test_softplus_off(orc):
    inp = _case(2, 200, 40, dtype="f32", seed=7)
    inp["softplus"] = False
    inp["delta"] = np.abs(inp["delta"]) * np.float32(0.1)
    inp["delta_bias"] = np.full_like(inp["delta_bias"], 0.01)
    _run(orc, inp, "softplus off")


def test_mamba130m_layer_shape(orc):
    """The Mamba-130M mixer-layer shape (8 x 2048 x 1536, bf16) in full."""
    inp = workloads.make_inputs(1)
    rng = np.random.default_rng(1001)
    inp["dout"] = workloads.f32_to_bf16_bits(rng.standard_normal(inp["x"].shape).astype(np.float32))
    inp["dh_last"] = None
    _run(orc, inp, "mamba-130m layer")


def test_mamba2p8b_layer_shape(orc):
    """The Mamba-2.8B mixer-layer shape (4 x 4096 x 5120, bf16) in full: every
    derivative of every channel, and dB, dC summed over all 5120 channels."""
    inp = workloads.make_inputs(2)
    rng = np.random.default_rng(2001)
    inp["dout"] = workloads.f32_to_bf16_bits(rng.standard_normal(inp["x"].shape).astype(np.float32))
    inp["dh_last"] = None
    _run(orc, inp, "mamba-2.8b layer")
