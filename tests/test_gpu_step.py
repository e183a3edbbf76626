"""GPU parity of ssm_scan_step (recurrent decode) against the float64 oracle."""
import numpy as np
import pytest
import torch

import workloads
from helpers import check, to_dev, to_np64

pytestmark = pytest.mark.gpu


def _step(state, tok, prm):
    import selective_state_space_38_b200 as ssm
    return ssm.ssm_scan_step(state, tok["x"], tok["delta"], prm["delta_bias"], prm["softplus"],
                             prm["A"], tok["B"], tok["C"], prm["D"], tok.get("z"))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("batch,dim", [(1, 1), (3, 7), (5, 130), (2, 1000)])
def test_step_small(orc, dtype, batch, dim):
    rng = np.random.default_rng(batch * 1000 + dim)
    inp = workloads.custom_inputs(batch, 5, dim, 16, dtype=dtype, seed=batch + dim, has_h0=True)
    state64 = inp["h0"].astype(np.float64)
    state = to_dev(inp["h0"]).clone()
    prm = {k: to_dev(inp[k]) for k in ("A", "D", "delta_bias")}
    prm["softplus"] = True
    for t in range(5):
        tok_np = {k: np.ascontiguousarray(inp[k][..., t]) for k in ("x", "delta", "z", "B", "C")}
        out = _step(state, {k: to_dev(v) for k, v in tok_np.items()}, prm)
        ref = orc.step(state64, tok_np["x"], tok_np["delta"], inp["delta_bias"], True, inp["A"],
                       tok_np["B"], tok_np["C"], inp["D"], tok_np["z"])
        torch.cuda.synchronize()
        check(to_np64(out), ref, dtype, f"step {t} out")
        check(to_np64(state), state64, dtype, f"step {t} state")
    assert rng is not None


def test_steps_equal_fwd_scan():
    """T decode steps from h0 equal one forward scan over the same T tokens."""
    import selective_state_space_38_b200 as ssm
    inp = workloads.custom_inputs(4, 40, 300, 16, dtype="bf16", seed=21, has_h0=True)
    t = {k: to_dev(v) for k, v in inp.items() if isinstance(v, np.ndarray)}
    out, hl = ssm.ssm_scan_fwd(t["x"], t["delta"], t["delta_bias"], True, t["A"], t["B"], t["C"],
                               t["D"], t["z"], t["h0"])
    state = t["h0"].clone()
    prm = dict(A=t["A"], D=t["D"], delta_bias=t["delta_bias"], softplus=True)
    outs = []
    for s in range(40):
        tok = {k: t[k][..., s].contiguous() for k in ("x", "delta", "z", "B", "C")}
        outs.append(_step(state, tok, prm))
    torch.cuda.synchronize()
    check(to_np64(torch.stack(outs, -1)), to_np64(out), "bf16", "steps vs fwd out")
    check(to_np64(state), to_np64(hl), "bf16", "steps vs fwd state")


def decode_prefill_state(orc, cfg=4):
    """The decode workload's initial state: 64 oracle steps from zero on the
    prefill tokens, rounded to float32."""
    c = workloads.CONFIGS[cfg]
    prm = workloads.decode_params(cfg)
    state64 = np.zeros((c.batch, c.dim, c.dstate), np.float64)
    for k in range(c.prefill_steps):
        tok = workloads.decode_tokens(cfg, k, phase=0)
        orc.step(state64, tok["x"], tok["delta"], prm["delta_bias"], True, prm["A"], tok["B"],
                 tok["C"], prm["D"], tok["z"])
    return state64.astype(np.float32)


def test_decode_batch_256x5120(orc):
    """256 sequences x 5120 channels x 16 fp32 states, 1024 consecutive steps
    from the 64-step prefill state.  Every step: out of all 256 sequences
    against the oracle.  After steps 1, 2, 64 and 1024: the whole state."""
    c = workloads.CONFIGS[4]
    prm_np = workloads.decode_params(4)
    state0 = decode_prefill_state(orc)
    state = to_dev(state0)
    prm = {k: to_dev(prm_np[k]) for k in ("A", "D", "delta_bias")}
    prm["softplus"] = True
    ref_state = state0.astype(np.float64)
    for s in range(c.decode_steps):
        tok_np = workloads.decode_tokens(4, s)
        out = _step(state, {k: to_dev(v) for k, v in tok_np.items()}, prm)
        ref = orc.step(ref_state, tok_np["x"], tok_np["delta"], prm_np["delta_bias"], True,
                       prm_np["A"], tok_np["B"], tok_np["C"], prm_np["D"], tok_np["z"])
        check(to_np64(out), ref, "bf16", f"decode step {s + 1} out (all sequences)")
        if s + 1 in (1, 2, 64, c.decode_steps):
            check(to_np64(state), ref_state, "bf16", f"decode step {s + 1} state (all sequences)")
