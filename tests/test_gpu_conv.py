"""GPU parity of the fused causal convolution + silu in front of the scan
(ssm_conv_scan_fwd) and of its decode step (ssm_conv_scan_step) against the
float64 oracle, element by element on the same stored inputs.

The block runs input projection, convolution, activation, scan (Mamba,
Appendix D "Memory"); the inference cache holds the convolution window beside
the SSM state.  Every output is compared in full: out, h_last and the new
convolution window."""
import numpy as np
import pytest
import torch

import workloads
from helpers import check, to_dev, to_np64

pytestmark = pytest.mark.gpu


def _conv_inputs(batch, L, dim, K=4, dtype="bf16", seed=0, has_h0=True, has_state=True):
    inp = workloads.custom_inputs(batch, L, dim, 16, dtype=dtype, seed=seed, has_h0=has_h0)
    rng = np.random.default_rng(seed + 1000)
    inp["conv_w"] = (rng.standard_normal((dim, K)) * 0.5).astype(np.float32)
    inp["conv_bias"] = (rng.standard_normal(dim) * 0.2).astype(np.float32)
    inp["conv_state"] = None
    if has_state and K > 1:
        st = rng.standard_normal((batch, dim, K - 1)).astype(np.float32)
        inp["conv_state"] = st if dtype == "f32" else workloads.f32_to_bf16_bits(st)
    return inp


def _gpu(inp, h0=None, conv_state=None, in_place=False):
    import selective_state_space_38_b200 as ssm
    t = {k: to_dev(v) for k, v in inp.items() if isinstance(v, np.ndarray)}
    cs = to_dev(conv_state) if conv_state is not None else t.get("conv_state")
    out, hl, cso = ssm.ssm_conv_scan_fwd(
        t["x"], t["conv_w"], t.get("conv_bias"), cs, t["delta"], t["delta_bias"], True, t["A"], t["B"], t["C"],
        t["D"], t["z"], to_dev(h0) if h0 is not None else t.get("h0"),
        conv_state_out=cs if (in_place and cs is not None) else None, check=True)
    torch.cuda.synchronize()
    return out, hl, cso


def _ref(orc, inp):
    return orc.conv_fwd(inp["x"], inp["conv_w"], inp["conv_bias"], inp["conv_state"], inp["delta"],
                        inp["delta_bias"], True, inp["A"], inp["B"], inp["C"], inp["D"], inp["z"], inp["h0"])


def _dt(inp):
    return "f32" if inp["x"].dtype == np.float32 else "bf16"


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("L", [1, 2, 3, 7, 33, 64, 257, 1000])
@pytest.mark.parametrize("K", [4, 2])
def test_small_shapes(orc, dtype, L, K):
    inp = _conv_inputs(2, L, 130, K=K, dtype=dtype, seed=L + 10 * K, has_state=(L % 2 == 1))
    out, hl, cso = _gpu(inp)
    ref_out, ref_hl, ref_st = _ref(orc, inp)
    d = _dt(inp)
    check(to_np64(out), ref_out, d, f"conv out L={L} K={K}")
    check(to_np64(hl), ref_hl, d, f"conv h_last L={L} K={K}")
    assert np.array_equal(to_np64(cso), ref_st), "new convolution window differs"


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_width_one_and_no_bias(orc, dtype):
    inp = _conv_inputs(1, 300, 64, K=1, dtype=dtype, seed=3, has_state=False)
    inp["conv_bias"] = None
    out, hl, cso = _gpu(inp)
    ref_out, ref_hl, _ = _ref(orc, inp)
    assert cso is None
    check(to_np64(out), ref_out, _dt(inp), "conv K=1 out")
    check(to_np64(hl), ref_hl, _dt(inp), "conv K=1 h_last")


@pytest.mark.parametrize("L", [4000, 4001])
def test_time_parallel_schedule(orc, L):
    """Few channel groups over a long sequence: segments start in the middle of
    the sequence, where the convolution's window comes from x itself."""
    inp = _conv_inputs(1, L, 40, seed=L)
    out, hl, cso = _gpu(inp)
    ref_out, ref_hl, ref_st = _ref(orc, inp)
    check(to_np64(out), ref_out, "bf16", f"conv time-parallel out L={L}")
    check(to_np64(hl), ref_hl, "bf16", f"conv time-parallel h_last L={L}")
    assert np.array_equal(to_np64(cso), ref_st)


def test_window_in_place_and_split(orc):
    """Two calls, each carrying the window (written over the old one) and the
    state, equal one call, also when the first part is shorter than the window."""
    inp = _conv_inputs(2, 1000, 96, seed=21)
    ref_out, ref_hl, ref_st = _ref(orc, inp)
    for m in (2, 333, 512):
        a = {k: (np.ascontiguousarray(v[..., :m]) if k in ("x", "delta", "z", "B", "C") else v)
             for k, v in inp.items()}
        b = {k: (np.ascontiguousarray(v[..., m:]) if k in ("x", "delta", "z", "B", "C") else v)
             for k, v in inp.items()}
        o1, h1, c1 = _gpu(a, in_place=True)
        b["h0"] = None
        b["conv_state"] = None
        o2, h2, c2 = _gpu(b, h0=h1.cpu().numpy(), conv_state=c1.cpu().view(torch.int16).numpy().view(np.uint16),
                          in_place=True)
        check(to_np64(torch.cat([o1, o2], -1)), ref_out, "bf16", f"conv split m={m} out")
        check(to_np64(h2), ref_hl, "bf16", f"conv split m={m} h_last")
        assert np.array_equal(to_np64(c2), ref_st)


def test_mamba2p8b_layer_with_conv_full(orc):
    """The Mamba-2.8B mixer-layer shape (4 x 4096 x 5120, bf16) with a width-4
    convolution in front, against the oracle on every channel."""
    c = workloads.CONFIGS[2]
    inp = workloads.make_inputs(2)
    rng = np.random.default_rng(2000)
    inp["conv_w"] = (rng.standard_normal((c.dim, 4)) * 0.5).astype(np.float32)
    inp["conv_bias"] = (rng.standard_normal(c.dim) * 0.2).astype(np.float32)
    inp["conv_state"] = None
    out, hl, cso = _gpu(inp)
    out_all, hl_all = out.view(c.channels, -1), hl.view(c.channels, -1)
    slab = 1024  # divides dim: a slab never crosses a sequence
    for s0 in range(0, c.channels, slab):
        sl = slice(s0, s0 + slab)
        sub = dict(inp)
        b0, d0 = s0 // c.dim, s0 % c.dim
        for k in ("x", "delta", "z"):
            sub[k] = np.ascontiguousarray(inp[k][b0:b0 + 1, d0:d0 + slab])
        for k in ("B", "C"):
            sub[k] = np.ascontiguousarray(inp[k][b0:b0 + 1])
        for k in ("A", "conv_w", "D", "delta_bias", "conv_bias"):
            sub[k] = np.ascontiguousarray(inp[k][d0:d0 + slab])
        ro, rh, rs = _ref(orc, sub)
        check(to_np64(out_all[sl]), ro.reshape(slab, -1), "bf16", f"conv layer out {s0}")
        check(to_np64(hl_all[sl]), rh.reshape(slab, -1), "bf16", f"conv layer h_last {s0}")
        assert np.array_equal(to_np64(cso.view(c.channels, -1)[sl]), rs.reshape(slab, -1))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("K", [4, 3, 1])
def test_step_against_oracle_and_fwd(orc, dtype, K):
    """Decode steps with the window in the cache: against the oracle's step
    on every channel, and T steps against one fused forward call."""
    import selective_state_space_38_b200 as ssm
    T = 12
    inp = _conv_inputs(3, T, 200, K=K, dtype=dtype, seed=40 + K, has_state=True)
    t = {k: to_dev(v) for k, v in inp.items() if isinstance(v, np.ndarray)}
    ref_out, ref_hl, ref_st = _ref(orc, inp)
    fwd_out, fwd_hl, fwd_st = ssm.ssm_conv_scan_fwd(
        t["x"], t["conv_w"], t["conv_bias"], t.get("conv_state"), t["delta"], t["delta_bias"], True, t["A"],
        t["B"], t["C"], t["D"], t["z"], t["h0"])
    cs = t["conv_state"].clone() if K > 1 else None
    st = t["h0"].clone()
    cs64 = (inp["conv_state"].astype(np.float64) if dtype == "f32" else
            to_np64(t["conv_state"])) if K > 1 else np.zeros((3, 200, 0))
    cs64 = np.ascontiguousarray(cs64)
    st64 = inp["h0"].astype(np.float64)
    outs = []
    for s in range(T):
        tok = {k: np.ascontiguousarray(inp[k][..., s]) for k in ("x", "delta", "z", "B", "C")}
        o = ssm.ssm_conv_scan_step(cs, st, to_dev(tok["x"]), t["conv_w"], t["conv_bias"], to_dev(tok["delta"]),
                                   t["delta_bias"], True, t["A"], to_dev(tok["B"]), to_dev(tok["C"]), t["D"],
                                   to_dev(tok["z"]))
        r = orc.conv_step(cs64, st64, tok["x"], inp["conv_w"], inp["conv_bias"], tok["delta"], inp["delta_bias"],
                          True, inp["A"], tok["B"], tok["C"], inp["D"], tok["z"])
        torch.cuda.synchronize()
        check(to_np64(o), r, _dt(inp), f"conv step {s} out")
        outs.append(o)
    check(to_np64(st), st64, _dt(inp), "conv step state")
    check(to_np64(torch.stack(outs, -1)), ref_out, _dt(inp), "conv steps vs oracle fwd")
    check(to_np64(torch.stack(outs, -1)), to_np64(fwd_out), _dt(inp), "conv steps vs fused fwd")
    check(to_np64(st), to_np64(fwd_hl), _dt(inp), "conv step state vs fused fwd")
    if K > 1:
        assert np.array_equal(to_np64(cs), ref_st)
        assert np.array_equal(to_np64(cs), to_np64(fwd_st))
