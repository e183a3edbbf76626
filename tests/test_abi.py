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
    for n in ("ssm_scan_fwd", "ssm_scan_step", "ssm_strerror", "ssm_version"):
        assert n in names


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


def _fwd(lib, m, **over):
    a = dict(x=_p(1), delta=_p(2), bias=None, sp=1, A=_p(3), B=_p(4), C=_p(5), D=None, z=_p(6),
             h0=None, out=_p(7), hl=None, dims=_dims(m))
    a.update(over)
    return lib.ssm_scan_fwd(a["x"], a["delta"], a["bias"], a["sp"], a["A"], a["B"], a["C"], a["D"],
                            a["z"], a["h0"], a["out"], a["hl"], a["dims"], None)


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


def test_python_binding_refuses_cpu_tensors():
    import torch
    import selective_state_space_38_b200 as m
    x = torch.zeros(1, 4, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        m.ssm_scan_fwd(x, x, None, True, torch.zeros(4, 16), x, x)
