"""Host-side tests of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments before launching anything.  These
run without a GPU: every rejected call returns before any CUDA call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssm_scan.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ssm_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    import selective_state_space_38_b200 as m
    return m.get_lib()


def test_header_declares_entry_points():
    names = _declared()
    for n in ("ssm_scan_fwd_workspace_size", "ssm_scan_fwd", "ssm_scan_fwd_status", "ssm_scan_step",
              "ssm_scan_fwd_noalloc", "ssm_debug_fwd_flag_timeout", "ssm_strerror", "ssm_version"):
        assert n in names
    import selective_state_space_38_b200 as m
    assert sorted(m.EXPORTS) == names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), f"{name} declared in ssm_scan.h but not exported"


def test_strerror_and_version(lib):
    import selective_state_space_38_b200 as m
    for code in range(0, 6):
        assert m.ssm_strerror(code)
    assert m.ssm_strerror(99) == "unknown error code"
    assert m.ssm_version() >= 10000


# fake, suitably aligned device addresses: validation fails before any use
def _p(i):
    return ctypes.c_void_p(0x10000000 + i * 0x1000000)


def _dims(m, batch=2, L=64, dim=128, N=16, dt=1):
    return ctypes.byref(m.Dims(batch, L, dim, N, dt))


WS = 1 << 20  # bytes of the fake workspace (enough for the default shape)


def _fwd(lib, m, fn="ssm_scan_fwd", **over):
    a = dict(x=_p(1), delta=_p(2), bias=None, sp=1, A=_p(3), B=_p(4), C=_p(5), D=None, z=_p(6),
             h0=None, out=_p(7), hl=None, ws=_p(9), wsb=WS, dims=_dims(m))
    a.update(over)
    args = [a["x"], a["delta"], a["bias"], a["sp"], a["A"], a["B"], a["C"], a["D"], a["z"], a["h0"],
            a["out"], a["hl"]]
    if fn == "ssm_scan_fwd_noalloc":
        return lib.ssm_scan_fwd_noalloc(*args, a["dims"], None)
    if fn == "ssm_debug_fwd_flag_timeout":
        return lib.ssm_debug_fwd_flag_timeout(*args, a["ws"], a["wsb"], 0, a["dims"], None)
    return lib.ssm_scan_fwd(*args, a["ws"], a["wsb"], a["dims"], None)


def test_fwd_rejects_bad_arguments(lib):
    import selective_state_space_38_b200 as m
    assert _fwd(lib, m, x=None) == 1
    assert _fwd(lib, m, out=None) == 1
    assert _fwd(lib, m, A=None) == 1
    assert _fwd(lib, m, dims=None) == 1
    assert _fwd(lib, m, dims=_dims(m, batch=0)) == 1
    assert _fwd(lib, m, dims=_dims(m, L=0)) == 1
    assert _fwd(lib, m, dims=_dims(m, dim=-3)) == 1
    assert _fwd(lib, m, dims=_dims(m, N=8)) == 2
    assert _fwd(lib, m, dims=_dims(m, dt=7)) == 2
    assert _fwd(lib, m, x=ctypes.c_void_p(0x10000002)) == 3
    assert _fwd(lib, m, hl=ctypes.c_void_p(0x10000008)) == 3
    # out overlapping an input
    assert _fwd(lib, m, out=_p(1)) == 1
    assert _fwd(lib, m, out=ctypes.c_void_p(0x11000000 + 0x100)) == 1
    # h_last overlapping an activation input
    assert _fwd(lib, m, hl=_p(2)) == 1
    # the workspace: required, 16-byte aligned, large enough, disjoint from every buffer
    assert _fwd(lib, m, ws=None) == 1
    assert _fwd(lib, m, ws=ctypes.c_void_p(0x19000008)) == 3
    assert _fwd(lib, m, wsb=100) == 1
    assert _fwd(lib, m, ws=_p(3)) == 1
    assert _fwd(lib, m, ws=ctypes.c_void_p(0x17000000 - 0x100)) == 1  # runs into out
    # sizes beyond the kernels' 32-bit coordinates
    assert _fwd(lib, m, dims=_dims(m, batch=1, L=1 << 31, dim=1)) == 2
    assert _fwd(lib, m, dims=_dims(m, batch=1, L=8, dim=1 << 31)) == 2


@pytest.mark.parametrize("fn", ["ssm_scan_fwd_noalloc", "ssm_debug_fwd_flag_timeout"])
def test_other_fwd_entries_share_the_checks(lib, fn):
    import selective_state_space_38_b200 as m
    assert _fwd(lib, m, fn, x=None) == 1
    assert _fwd(lib, m, fn, dims=_dims(m, N=8)) == 2
    assert _fwd(lib, m, fn, x=ctypes.c_void_p(0x10000002)) == 3
    assert _fwd(lib, m, fn, out=_p(1)) == 1
    assert _fwd(lib, m, fn, dims=_dims(m, batch=1, L=1 << 31, dim=1)) == 2
    if fn == "ssm_debug_fwd_flag_timeout":
        assert _fwd(lib, m, fn, ws=None) == 1


def test_workspace_size_query(lib):
    """Sizes for a given SM count, computed on the host: 16 KB of header and
    flags plus a 2 KB carry per 32-channel group; the two-pass schedule adds
    6 KB per (group, segment) when groups are fewer than half of 4 x SMs."""
    import selective_state_space_38_b200 as m

    def size(batch, L, dim, sms=148):
        out = ctypes.c_size_t(0)
        rc = lib.ssm_scan_fwd_workspace_size(ctypes.byref(m.Dims(batch, L, dim, 16, 1)), sms,
                                             ctypes.byref(out))
        assert rc == 0, m.ssm_strerror(rc)
        return out.value

    def flag_bytes(groups):
        return (256 + 4 * groups + 255) // 256 * 256

    groups = 4 * 160  # the Mamba-2.8B layer: 640 groups >= 592 / 2: chained
    assert size(4, 4096, 5120) == flag_bytes(groups) + groups * 2048
    groups = 64       # the long sequence: 64 groups, 4 x 592 / 64 = 37 segments of 3552 steps
    segs = -(-131072 // 3552)
    assert size(1, 131072, 2048) == flag_bytes(groups) + groups * 2048 + groups * segs * 6144
    assert size(1, 64, 2048) == flag_bytes(groups) + groups * 2048  # too short to split
    bad = ctypes.c_size_t(0)
    assert lib.ssm_scan_fwd_workspace_size(None, 148, ctypes.byref(bad)) == 1
    assert lib.ssm_scan_fwd_workspace_size(ctypes.byref(m.Dims(1, 8, 8, 8, 1)), 148, ctypes.byref(bad)) == 2


def test_step_rejects_bad_arguments(lib):
    import selective_state_space_38_b200 as m

    def step(**over):
        a = dict(st=_p(0), x=_p(1), delta=_p(2), bias=None, sp=1, A=_p(3), B=_p(4), C=_p(5), D=None,
                 z=None, out=_p(7), dims=_dims(m))
        a.update(over)
        return lib.ssm_scan_step(a["st"], a["x"], a["delta"], a["bias"], a["sp"], a["A"], a["B"],
                                 a["C"], a["D"], a["z"], a["out"], a["dims"], None)
    assert step(st=None) == 1
    assert step(out=None) == 1
    assert step(dims=_dims(m, dim=0)) == 1
    assert step(dims=_dims(m, N=32)) == 2
    assert step(st=ctypes.c_void_p(0x10000004)) == 3
    assert step(out=_p(0)) == 1  # out overlapping the state
    # B and C are read as 16-byte vectors: an element-aligned but not 16-byte
    # aligned B or C is refused (it would be a misaligned vector load)
    assert step(B=ctypes.c_void_p(0x14000004)) == 3
    assert step(C=ctypes.c_void_p(0x15000008)) == 3
    assert step(B=ctypes.c_void_p(0x14000002), dims=_dims(m, dt=1)) == 3
    assert step(A=ctypes.c_void_p(0x13000004)) == 3


def test_python_binding_refuses_cpu_tensors():
    import torch
    import selective_state_space_38_b200 as m
    x = torch.zeros(1, 4, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        m.ssm_scan_fwd(x, x, None, True, torch.zeros(4, 16), x, x)


def test_conv_entries_reject_bad_arguments(lib):
    """The fused convolution entries share the forward and step checks and add
    their own: taps required, width 1..4, the new window disjoint from every
    other buffer (it may only be the old window itself)."""
    import selective_state_space_38_b200 as m

    def fwd(**over):
        a = dict(x=_p(1), w=_p(10), cb=None, k=4, cs=None, cso=_p(11), delta=_p(2), bias=None, sp=1, A=_p(3),
                 B=_p(4), C=_p(5), D=None, z=_p(6), h0=None, out=_p(7), hl=None, ws=_p(9), wsb=WS,
                 dims=_dims(m))
        a.update(over)
        return lib.ssm_conv_scan_fwd(a["x"], a["w"], a["cb"], a["k"], a["cs"], a["cso"], a["delta"], a["bias"],
                                     a["sp"], a["A"], a["B"], a["C"], a["D"], a["z"], a["h0"], a["out"], a["hl"],
                                     a["ws"], a["wsb"], a["dims"], None)
    assert fwd(w=None) == 1
    assert fwd(k=5) == 2
    assert fwd(k=0) == 2
    assert fwd(w=ctypes.c_void_p(0x1A000002)) == 3
    assert fwd(cso=ctypes.c_void_p(0x1B000001)) == 3      # bf16 window at an odd byte
    assert fwd(cso=_p(1)) == 1                            # new window over x
    assert fwd(cso=_p(7)) == 1                            # ... over out
    assert fwd(cso=_p(10)) == 1                           # ... over the taps
    assert fwd(cs=_p(12), cso=ctypes.c_void_p(0x1C000002)) == 1  # partly over the old window
    assert fwd(out=_p(10)) == 1                           # out over the taps
    assert fwd(ws=None) == 1

    def step(**over):
        a = dict(cs=_p(12), st=_p(0), x=_p(1), w=_p(10), cb=None, k=4, delta=_p(2), bias=None, sp=1, A=_p(3),
                 B=_p(4), C=_p(5), D=None, z=None, out=_p(7), dims=_dims(m))
        a.update(over)
        return lib.ssm_conv_scan_step(a["cs"], a["st"], a["x"], a["w"], a["cb"], a["k"], a["delta"], a["bias"],
                                      a["sp"], a["A"], a["B"], a["C"], a["D"], a["z"], a["out"], a["dims"], None)
    assert step(cs=None) == 1                             # the window is required for K > 1
    assert step(w=None) == 1
    assert step(k=7) == 2
    assert step(cs=_p(0)) == 1                            # window over the state
    assert step(cs=_p(1)) == 1                            # window over x
    assert step(B=ctypes.c_void_p(0x14000004)) == 3


def test_trap_entries_reject_bad_arguments(lib):
    """The trapezoidal entries share the forward and step checks; lam is
    required, and lam, x_prev and B_prev are inputs that no output may overlap."""
    import selective_state_space_38_b200 as m

    def fwd(**over):
        a = dict(x=_p(1), delta=_p(2), bias=None, sp=1, lam=_p(13), A=_p(3), B=_p(4), C=_p(5), D=None, z=_p(6),
                 h0=None, xp=None, bp=None, out=_p(7), hl=None, ws=_p(9), wsb=WS, dims=_dims(m))
        a.update(over)
        return lib.ssm_trap_scan_fwd(a["x"], a["delta"], a["bias"], a["sp"], a["lam"], a["A"], a["B"], a["C"],
                                     a["D"], a["z"], a["h0"], a["xp"], a["bp"], a["out"], a["hl"], a["ws"],
                                     a["wsb"], a["dims"], None)
    assert fwd(lam=None) == 1
    assert fwd(lam=ctypes.c_void_p(0x1D000008)) == 3
    assert fwd(xp=ctypes.c_void_p(0x1E000001)) == 3
    assert fwd(out=_p(13)) == 1
    assert fwd(hl=_p(14), xp=ctypes.c_void_p(0x1E000000 + 0x20)) == 1  # h_last over x_prev
    assert fwd(ws=None) == 1

    def step(**over):
        a = dict(st=_p(0), x=_p(1), delta=_p(2), bias=None, sp=1, lam=_p(13), A=_p(3), B=_p(4), C=_p(5), D=None,
                 z=None, xp=_p(14), bp=_p(15), out=_p(7), dims=_dims(m))
        a.update(over)
        return lib.ssm_trap_scan_step(a["st"], a["x"], a["delta"], a["bias"], a["sp"], a["lam"], a["A"], a["B"],
                                      a["C"], a["D"], a["z"], a["xp"], a["bp"], a["out"], a["dims"], None)
    assert step(lam=None) == 1
    assert step(bp=ctypes.c_void_p(0x1F000004)) == 3  # B_prev is read as vectors
    assert step(out=_p(14)) == 1
    assert step(st=_p(15)) == 1


def test_bwd_rejects_bad_arguments(lib):
    """The backward entry: required inputs and outputs, dz with z, alignment,
    a large enough workspace, and no output over an input or another output."""
    import selective_state_space_38_b200 as m
    need = ctypes.c_size_t(0)
    assert lib.ssm_scan_bwd_workspace_size(_dims(m), ctypes.byref(need)) == 0
    # the checkpoint pass's forward scratch (sized for 256 SMs), then one 64-byte
    # state per channel and 16-step segment
    fwd = ctypes.c_size_t(0)
    assert lib.ssm_scan_fwd_workspace_size(_dims(m), 256, ctypes.byref(fwd)) == 0
    segments = -(-64 // 16)
    assert need.value == (fwd.value + 255) // 256 * 256 + (2 * 128 * segments * 16 * 4 + 255) // 256 * 256

    def bwd(**over):
        a = dict(x=_p(1), delta=_p(2), bias=None, sp=1, A=_p(3), B=_p(4), C=_p(5), D=None, z=_p(6), h0=None,
                 dout=_p(16), dhl=None, dx=_p(17), ddelta=_p(18), dz=_p(19), dB=_p(20), dC=_p(21), dA=_p(22),
                 dD=None, dbias=None, dh0=None, ws=_p(23), wsb=need.value, dims=_dims(m))
        a.update(over)
        return lib.ssm_scan_bwd(a["x"], a["delta"], a["bias"], a["sp"], a["A"], a["B"], a["C"], a["D"], a["z"],
                                a["h0"], a["dout"], a["dhl"], a["dx"], a["ddelta"], a["dz"], a["dB"], a["dC"],
                                a["dA"], a["dD"], a["dbias"], a["dh0"], a["ws"], a["wsb"], a["dims"], None)
    assert bwd(dout=None) == 1
    assert bwd(dx=None) == 1
    assert bwd(dA=None) == 1
    assert bwd(dz=None) == 1                       # z is given, so dz is required
    assert bwd(ws=None) == 1
    assert bwd(wsb=need.value - 1) == 1
    assert bwd(dims=_dims(m, N=8)) == 2
    assert bwd(dx=ctypes.c_void_p(0x11000008)) == 3
    assert bwd(dD=ctypes.c_void_p(0x1A000002)) == 3
    assert bwd(dx=_p(1)) == 1                      # dx over x
    assert bwd(dB=_p(17)) == 1                     # dB over dx
    assert bwd(ws=_p(16)) == 1                     # workspace over dout


def test_ssd_rejects_bad_arguments(lib):
    """The SSD entry: head dim 64, state 128, bf16; heads a multiple of groups;
    alignment; outputs disjoint from inputs."""
    import selective_state_space_38_b200 as m

    def ssd(**over):
        a = dict(x=_p(1), dt=_p(2), bias=None, sp=1, A=_p(3), B=_p(4), C=_p(5), D=None, h0=None, y=_p(7),
                 hl=None, ws=_p(9), wsb=256, dims=ctypes.byref(m.SsdDims(2, 256, 8, 64, 2, 128, 1)))
        a.update(over)
        return lib.ssm_ssd_fwd(a["x"], a["dt"], a["bias"], a["sp"], a["A"], a["B"], a["C"], a["D"], a["h0"],
                               a["y"], a["hl"], a["ws"], a["wsb"], a["dims"], None)
    assert ssd(x=None) == 1
    assert ssd(ws=None) == 1
    assert ssd(wsb=100) == 1
    assert ssd(dims=ctypes.byref(m.SsdDims(2, 256, 8, 64, 3, 128, 1))) == 1   # 8 heads, 3 groups
    assert ssd(dims=ctypes.byref(m.SsdDims(2, 256, 8, 32, 2, 128, 1))) == 2   # head dim
    assert ssd(dims=ctypes.byref(m.SsdDims(2, 256, 8, 64, 2, 64, 1))) == 2    # state dim
    assert ssd(dims=ctypes.byref(m.SsdDims(2, 256, 8, 64, 2, 128, 0))) == 2   # float32
    assert ssd(x=ctypes.c_void_p(0x11000008)) == 3
    assert ssd(dt=ctypes.c_void_p(0x12000001)) == 3
    assert ssd(y=_p(1)) == 1
    assert ssd(hl=_p(4)) == 1


def test_ssd_workspace_size(lib):
    """Split sequences need 2048 bytes plus one 32 KB state per CTA (at most one
    per SM, at most 448); without more sequences than SMs, 256 bytes."""
    import selective_state_space_38_b200 as m
    n = ctypes.c_size_t(0)

    def size(batch, heads, sms):
        assert lib.ssm_ssd_fwd_workspace_size(ctypes.byref(m.SsdDims(batch, 4096, heads, 64, 1, 128, 1)), sms,
                                              ctypes.byref(n)) == 0
        return n.value
    assert size(4, 80, 148) == 2048 + 148 * 32768
    assert size(1, 148, 148) == 256
    assert size(1, 149, 148) == 2048 + 148 * 32768
    assert size(4, 200, 1000) == 2048 + 448 * 32768
    assert m.ssm_ssd_fwd_workspace_size(4, 80, sm_count=132) == 2048 + 132 * 32768
    assert lib.ssm_ssd_fwd_workspace_size(None, 148, ctypes.byref(n)) == 1
    assert lib.ssm_ssd_fwd_workspace_size(ctypes.byref(m.SsdDims(0, 1, 1, 64, 1, 128, 1)), 148,
                                          ctypes.byref(n)) == 1
