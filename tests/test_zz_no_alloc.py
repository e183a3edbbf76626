"""The allocation-free forward scan, ssm_scan_fwd_noalloc.

It exists for callers that cannot allocate any device memory while they run
the scan, not even a workspace: code inside an allocator or memory-pool
callback, runtimes that reserve all device memory up front.  Its output must
match the float64 oracle, and ssm_scan_fwd, within the parity tolerance of
the other GPU tests, on two calls in a row (the fixed scratch array keeps the
previous call's contents and must be re-armed); a warmed call must leave the
device's free memory and torch's allocations unchanged; and shapes whose work
queue does not fit the fixed array must be rejected before anything runs.
This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

import workloads
from helpers import check, to_dev, to_np64


def _lib():
    import selective_state_space_38_b200 as ssm
    return ssm.get_lib(), ssm


def test_noalloc_rejects_shapes_beyond_its_scratch():
    lib, ssm = _lib()
    fake = [ctypes.c_void_p((i + 1) << 36) for i in range(8)]  # 64 GiB apart: no overlaps
    # batch * ceil(dim / 32) = 64 * 160 groups: far beyond the fixed array
    dims = ssm.Dims(64, 4096, 5120, 16, ssm.SSM_BF16)
    rc = lib.ssm_scan_fwd_noalloc(fake[0], fake[1], None, 1, fake[2], fake[3], fake[4], None, None, None,
                                  fake[5], None, ctypes.byref(dims), None)
    assert rc == 2, ssm.ssm_strerror(rc)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,L", [("bf16", 1500), ("f32", 777), ("bf16", 2048), ("f32", 1024)])
def test_noalloc_matches_oracle_and_fwd_twice(orc, dtype, L):
    """L = 1500 (bf16) and 777 (f32) take the element-wise loads, 2048 and 1024
    the TMA path; each runs two calls in a row on the shared array."""
    import torch
    lib, ssm = _lib()
    inp = workloads.custom_inputs(2, L, 600, 16, dtype=dtype, seed=99 + L, has_h0=True)
    t = {k: to_dev(v) for k, v in inp.items() if isinstance(v, np.ndarray)}
    ref_out, ref_hl = orc.fwd(inp["x"], inp["delta"], inp["delta_bias"], True, inp["A"], inp["B"],
                              inp["C"], inp["D"], inp["z"], inp["h0"])
    fwd_out, fwd_hl = ssm.ssm_scan_fwd(t["x"], t["delta"], t["delta_bias"], True, t["A"], t["B"], t["C"],
                                       t["D"], t["z"], t["h0"], check=True)
    torch.cuda.synchronize()
    dims = ssm.Dims(2, L, 600, 16, ssm.SSM_BF16 if dtype == "bf16" else ssm.SSM_F32)
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        out = torch.full_like(t["x"], float("nan"))
        hl = torch.full_like(t["h0"], float("nan"))
        rc = lib.ssm_scan_fwd_noalloc(t["x"].data_ptr(), t["delta"].data_ptr(), t["delta_bias"].data_ptr(), 1,
                                      t["A"].data_ptr(), t["B"].data_ptr(), t["C"].data_ptr(), t["D"].data_ptr(),
                                      t["z"].data_ptr(), t["h0"].data_ptr(), out.data_ptr(), hl.data_ptr(),
                                      ctypes.byref(dims), stream)
        assert rc == 0, ssm.ssm_strerror(rc)
        assert lib.ssm_scan_fwd_status(None, stream) == 0
        check(to_np64(out), ref_out, dtype, f"noalloc out vs oracle, call {call}")
        check(to_np64(hl), ref_hl, dtype, f"noalloc h_last vs oracle, call {call}")
        check(to_np64(out), to_np64(fwd_out), dtype, f"noalloc out vs ssm_scan_fwd, call {call}")
        check(to_np64(hl), to_np64(fwd_hl), dtype, f"noalloc h_last vs ssm_scan_fwd, call {call}")


@pytest.mark.gpu
def test_noalloc_allocates_nothing():
    """After a first (warming) call, further calls change neither the device's
    free memory nor torch's allocation counters."""
    import torch
    lib, ssm = _lib()
    inp = workloads.custom_inputs(1, 2048, 256, 16, seed=5)
    t = {k: to_dev(v) for k, v in inp.items() if isinstance(v, np.ndarray)}
    out = torch.empty_like(t["x"])
    dims = ssm.Dims(1, 2048, 256, 16, ssm.SSM_BF16)
    stream = torch.cuda.current_stream().cuda_stream

    def call():
        rc = lib.ssm_scan_fwd_noalloc(t["x"].data_ptr(), t["delta"].data_ptr(), t["delta_bias"].data_ptr(), 1,
                                      t["A"].data_ptr(), t["B"].data_ptr(), t["C"].data_ptr(), t["D"].data_ptr(),
                                      t["z"].data_ptr(), None, out.data_ptr(), None, ctypes.byref(dims), stream)
        assert rc == 0, ssm.ssm_strerror(rc)

    call()
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    allocs0 = torch.cuda.memory_stats().get("allocation.all.allocated", 0)
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert torch.cuda.memory_stats().get("allocation.all.allocated", 0) == allocs0
