"""The C-ABI library without a GPU: it loads, exports every symbol the header
declares, its structs match the binding's mirrors, and host-side validation
rejects bad arguments before touching CUDA."""
import ctypes
import os
import re
import subprocess

import pytest

import selective_state_space_27_b200 as ms
from selective_state_space_27_b200 import build as msbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mambascan.h")


@pytest.fixture(scope="module")
def lib():
    msbuild.build()
    return ms.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(mamba_[a-z_0-9]+)\s*\(",
                       text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for want in ("mamba_scan_fwd", "mamba_state_update", "mamba_scan_workspace_size", "mamba_conv_scan_fwd",
                 "mamba_conv_state_update", "mamba_ssd_fwd",
                 "mamba_status_string", "mamba_last_error", "mamba_abi_version"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", ms.library_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert hasattr(lib, n)


def test_struct_layout_matches_binding(tmp_path):
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "mambascan.h"\n'
        "int main(void){printf(\"%zu %zu %zu %zu %zu %zu\\n\", sizeof(ms_scan_args),"
        " offsetof(ms_scan_args, y), offsetof(ms_scan_args, force_segments), sizeof(ms_update_args),"
        " offsetof(ms_update_args, y), offsetof(ms_update_args, delta_bias)); return 0;}\n")
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c11", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)])
    got = [int(v) for v in subprocess.check_output([str(exe)], text=True).split()]
    want = [ctypes.sizeof(ms.ScanArgs), ms.ScanArgs.y.offset, ms.ScanArgs.force_segments.offset,
            ctypes.sizeof(ms.UpdateArgs), ms.UpdateArgs.y.offset, ms.UpdateArgs.delta_bias.offset]
    assert got == want


def test_abi_version_and_status_strings(lib):
    assert lib.mamba_abi_version() == 2
    for code, name in ms.STATUS.items():
        assert lib.mamba_status_string(code).decode() == name
    assert lib.mamba_status_string(99).decode() == "MS_UNKNOWN_STATUS"


def _valid_scan_args():
    """Arguments that pass validation; pointers are fake (never dereferenced
    here: every case below fails before any CUDA call)."""
    a = ms.ScanArgs()
    a.batch, a.dim, a.dstate, a.seqlen = 2, 8, 16, 64
    a.in_dtype, a.delta_softplus = ms.MS_BF16, 1
    base = 1 << 20
    a.u, a.u_batch_stride, a.u_dim_stride = base, 8 * 64, 64
    a.delta, a.delta_batch_stride, a.delta_dim_stride = base * 2, 8 * 64, 64
    a.B, a.B_batch_stride, a.B_state_stride = base * 3, 16 * 64, 64
    a.C, a.C_batch_stride, a.C_state_stride = base * 4, 16 * 64, 64
    a.y, a.y_batch_stride, a.y_dim_stride = base * 5, 8 * 64, 64
    a.A = base * 6
    return a


@pytest.mark.parametrize("field,value,status", [
    ("batch", 0, 1), ("dim", -1, 1), ("dstate", 0, 1), ("seqlen", 0, 1),
    ("in_dtype", 7, 1), ("reserved", 1, 1), ("force_segments", -2, 1),
    ("u", None, 1), ("A", None, 1), ("y", None, 1),
    ("u_dim_stride", -64, 1), ("dstate", 17, 2), ("batch", 70000, 2),
    ("u", (1 << 20) + 1, 3), ("A", (1 << 20) * 6 + 2, 3),
])
def test_scan_validation_rejects(lib, field, value, status):
    a = _valid_scan_args()
    setattr(a, field, value)
    n = ctypes.c_size_t(123)
    rc = lib.mamba_scan_workspace_size(ctypes.byref(a), ctypes.byref(n))
    assert rc == status, (rc, lib.mamba_last_error())
    assert n.value == 0
    rc = lib.mamba_scan_fwd(ctypes.byref(a), None, 0, None)
    assert rc == status
    assert lib.mamba_last_error().decode() != ""


def test_scan_null_args(lib):
    assert lib.mamba_scan_fwd(None, None, 0, None) == 1
    n = ctypes.c_size_t(0)
    assert lib.mamba_scan_workspace_size(None, ctypes.byref(n)) == 1
    assert lib.mamba_scan_workspace_size(ctypes.byref(_valid_scan_args()), None) == 1


def _valid_update_args():
    a = ms.UpdateArgs()
    a.batch, a.dim, a.dstate = 4, 8, 16
    a.in_dtype, a.delta_softplus = ms.MS_BF16, 1
    base = 1 << 20
    a.state, a.state_batch_stride, a.state_dim_stride = base, 8 * 16, 16
    a.x, a.x_batch_stride = base * 2, 8
    a.delta, a.delta_batch_stride = base * 3, 8
    a.B, a.B_batch_stride = base * 4, 16
    a.C, a.C_batch_stride = base * 5, 16
    a.y, a.y_batch_stride = base * 6, 8
    a.A = base * 7
    return a


@pytest.mark.parametrize("field,value,status", [
    ("batch", 0, 1), ("dstate", -3, 1), ("in_dtype", 2, 1), ("state", None, 1), ("x", None, 1),
    ("C", None, 1), ("x_batch_stride", -1, 1), ("dstate", 32, 2), ("batch", 70000, 2),
    ("state", (1 << 20) + 2, 3),
    ("x", (1 << 20) * 2 + 1, 3),
])
def test_update_validation_rejects(lib, field, value, status):
    a = _valid_update_args()
    setattr(a, field, value)
    assert lib.mamba_state_update(ctypes.byref(a), None) == status
    assert lib.mamba_state_update(None, None) == 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(ms, "_lib", None)
    monkeypatch.setattr(ms, "_LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="not built"):
        ms.load_library()


def _valid_conv():
    c = ms.Conv1dArgs()
    c.weight, c.bias, c.width, c.silu = (1 << 20) * 9, (1 << 20) * 10, 4, 1
    return c


@pytest.mark.parametrize("field,value,status", [
    ("weight", None, 1), ("width", 0, 1), ("width", 5, 2), ("silu", 2, 1), ("weight", (1 << 20) * 9 + 2, 3),
    ("bias", (1 << 20) * 10 + 1, 3),
])
def test_conv_scan_validation_rejects(lib, field, value, status):
    c = _valid_conv()
    setattr(c, field, value)
    assert lib.mamba_conv_scan_fwd(ctypes.byref(_valid_scan_args()), ctypes.byref(c), None, None) == status
    assert lib.mamba_last_error().decode() != ""


def test_conv_scan_null_and_segments(lib):
    assert lib.mamba_conv_scan_fwd(ctypes.byref(_valid_scan_args()), None, None, None) == 1
    a = _valid_scan_args()
    a.force_segments = 2
    assert lib.mamba_conv_scan_fwd(ctypes.byref(a), ctypes.byref(_valid_conv()), None, None) == 2
    a = _valid_scan_args()
    a.dstate = 0
    assert lib.mamba_conv_scan_fwd(ctypes.byref(a), ctypes.byref(_valid_conv()), None, None) == 1


@pytest.mark.parametrize("state,sb,sd,status", [
    (None, 32, 4, 1), ((1 << 20) * 11, -1, 4, 1), ((1 << 20) * 11, 32, -4, 1), ((1 << 20) * 11 + 1, 32, 4, 3),
])
def test_conv_state_update_validation_rejects(lib, state, sb, sd, status):
    rc = lib.mamba_conv_state_update(ctypes.byref(_valid_update_args()), ctypes.byref(_valid_conv()), state,
                                     sb, sd, None)
    assert rc == status
    assert lib.mamba_conv_state_update(ctypes.byref(_valid_update_args()), None, (1 << 20) * 11, 32, 4, None) == 1


@pytest.mark.parametrize("lam,sb,sd,segments,status", [
    (None, 512, 64, 0, 1), ((1 << 20) * 12, -1, 64, 0, 1), ((1 << 20) * 12 + 1, 512, 64, 0, 3),
    ((1 << 20) * 12, 512, 64, 2, 2),
])
def test_trap_scan_validation_rejects(lib, lam, sb, sd, segments, status):
    a = _valid_scan_args()
    a.force_segments = segments
    assert lib.mamba_trap_scan_fwd(ctypes.byref(a), lam, sb, sd, None, None) == status
    assert lib.mamba_last_error().decode() != ""


def test_bwd_struct_layout_matches_binding(tmp_path):
    src = tmp_path / "bwd_layout.c"
    src.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "mambascan.h"\n'
        "int main(void){printf(\"%zu %zu %zu %zu\\n\", sizeof(ms_scan_bwd_args), offsetof(ms_scan_bwd_args, dz),"
        " offsetof(ms_scan_bwd_args, dA), offsetof(ms_scan_bwd_args, dinitial_state)); return 0;}\n")
    exe = tmp_path / "bwd_layout"
    subprocess.check_call(["gcc", "-std=c11", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)])
    got = [int(v) for v in subprocess.check_output([str(exe)], text=True).split()]
    want = [ctypes.sizeof(ms.ScanBwdArgs), ms.ScanBwdArgs.dz.offset, ms.ScanBwdArgs.dA.offset,
            ms.ScanBwdArgs.dinitial_state.offset]
    assert got == want


def _valid_bwd():
    g = ms.ScanBwdArgs()
    base = 1 << 20
    g.dy, g.dy_batch_stride, g.dy_dim_stride = base * 20, 512, 64
    g.du, g.du_batch_stride, g.du_dim_stride = base * 21, 512, 64
    g.ddelta, g.ddelta_batch_stride, g.ddelta_dim_stride = base * 22, 512, 64
    g.dA, g.dB, g.dC = base * 23, base * 24, base * 25
    return g


@pytest.mark.parametrize("field,value,status", [
    ("dy", None, 1), ("du", None, 1), ("dA", None, 1), ("dy_batch_stride", -1, 1),
    ("dy", (1 << 20) * 20 + 1, 3), ("dB", (1 << 20) * 24 + 2, 3),
])
def test_bwd_validation_rejects(lib, field, value, status):
    g = _valid_bwd()
    setattr(g, field, value)
    assert lib.mamba_scan_bwd(ctypes.byref(_valid_scan_args()), ctypes.byref(g), (1 << 20) * 30, 1 << 30,
                              None) == status


def test_checkpoint_calls_validate_before_launching(lib):
    """The checkpointed forward and backward refuse a missing, short or
    misaligned checkpoint buffer with no device work (CPU: nothing launches)."""
    a = _valid_scan_args()
    n = ctypes.c_size_t(0)
    assert lib.mamba_scan_bwd_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0
    base = (1 << 20) * 40
    assert lib.mamba_scan_fwd_checkpointed(ctypes.byref(a), None, n.value, None, 0, None) == 1
    assert lib.mamba_scan_fwd_checkpointed(ctypes.byref(a), base, n.value - 1, None, 0, None) == 6
    assert lib.mamba_scan_fwd_checkpointed(ctypes.byref(a), base + 16, n.value, None, 0, None) == 3
    assert lib.mamba_scan_bwd_checkpointed(ctypes.byref(a), ctypes.byref(_valid_bwd()), None, n.value, None) == 1
    assert lib.mamba_scan_bwd_checkpointed(ctypes.byref(a), ctypes.byref(_valid_bwd()), base, n.value - 1,
                                           None) == 6


def test_bwd_needs_workspace_and_matching_gradients(lib):
    a = _valid_scan_args()
    assert lib.mamba_scan_bwd(ctypes.byref(a), None, None, 0, None) == 1
    assert lib.mamba_scan_bwd(ctypes.byref(a), ctypes.byref(_valid_bwd()), None, 0, None) == 6
    n = ctypes.c_size_t(0)
    assert lib.mamba_scan_bwd_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0
    assert n.value == 2 * 8 * 8 * 16 * 4      # batch x dim x ceil(64 / 8) checkpoints x 16 states, float32
    a.D = (1 << 20) * 7                      # D given: dD required
    assert lib.mamba_scan_bwd(ctypes.byref(a), ctypes.byref(_valid_bwd()), (1 << 20) * 30, 1 << 30, None) == 1


def test_ssd_struct_layout_matches_binding(tmp_path):
    src = tmp_path / "ssd_layout.c"
    src.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "mambascan.h"\n'
        "int main(void){printf(\"%zu %zu %zu %zu %zu\\n\", sizeof(ms_ssd_args), offsetof(ms_ssd_args, x),"
        " offsetof(ms_ssd_args, z_token_stride), offsetof(ms_ssd_args, A), offsetof(ms_ssd_args, final_state));"
        " return 0;}\n")
    exe = tmp_path / "ssd_layout"
    subprocess.check_call(["gcc", "-std=c11", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)])
    got = [int(v) for v in subprocess.check_output([str(exe)], text=True).split()]
    want = [ctypes.sizeof(ms.SsdArgs), ms.SsdArgs.x.offset, ms.SsdArgs.z_token_stride.offset, ms.SsdArgs.A.offset,
            ms.SsdArgs.final_state.offset]
    assert got == want


def _valid_ssd_args():
    a = ms.SsdArgs()
    base = 1 << 20
    a.batch, a.seqlen, a.nheads, a.ngroups = 2, 300, 4, 1
    a.in_dtype, a.dt_softplus = ms.MS_BF16, 1
    a.x, a.x_batch_stride, a.x_token_stride = base * 1, 300 * 256, 256
    a.dt, a.dt_batch_stride, a.dt_token_stride = base * 2, 1200, 4
    a.B, a.B_batch_stride, a.B_token_stride = base * 3, 300 * 128, 128
    a.C, a.C_batch_stride, a.C_token_stride = base * 4, 300 * 128, 128
    a.y, a.y_batch_stride, a.y_token_stride = base * 5, 300 * 256, 256
    a.A = base * 6
    return a


@pytest.mark.parametrize("field,value,status", [
    ("x", None, 1), ("A", None, 1), ("seqlen", 0, 1), ("ngroups", 3, 1), ("x_token_stride", 200, 1),
    ("B_token_stride", 64, 1), ("dt_token_stride", 2, 1), ("y_batch_stride", -8, 1),
    ("in_dtype", 0, 2), ("in_dtype", 7, 1),
    ("x_token_stride", 260, 3), ("B_batch_stride", 300 * 128 + 4, 3), ("x", (1 << 20) + 8, 3),
    ("dt", (1 << 20) * 2 + 1, 3), ("A", (1 << 20) * 6 + 2, 3),
])
def test_ssd_validation_rejects(lib, field, value, status):
    a = _valid_ssd_args()
    setattr(a, field, value)
    assert lib.mamba_ssd_fwd(ctypes.byref(a), (1 << 20) * 9, 256, None) == status


def test_ssd_needs_args_and_workspace(lib):
    assert lib.mamba_ssd_fwd(None, (1 << 20) * 9, 256, None) == 1
    a = _valid_ssd_args()
    assert lib.mamba_ssd_fwd(ctypes.byref(a), None, 0, None) == 6
    assert lib.mamba_ssd_fwd(ctypes.byref(a), (1 << 20) * 9, 128, None) == 6
    assert lib.mamba_ssd_fwd(ctypes.byref(a), (1 << 20) * 9 + 4, 256, None) == 3


# The workspace entry points (and their size queries) validate exactly as the
# plain ones, before any device query or launch.

@pytest.mark.parametrize("field,value,status", [
    ("weight", None, 1), ("width", 0, 1), ("width", 5, 2), ("silu", 2, 1), ("weight", (1 << 20) * 9 + 2, 3),
])
def test_conv_scan_ws_entries_validate(lib, field, value, status):
    c = _valid_conv()
    setattr(c, field, value)
    n = ctypes.c_size_t(7)
    a = _valid_scan_args()
    assert lib.mamba_conv_scan_workspace_size(ctypes.byref(a), ctypes.byref(c), None, ctypes.byref(n)) == status
    assert n.value == 0
    assert lib.mamba_conv_scan_fwd_ws(ctypes.byref(a), ctypes.byref(c), None, None, 0, None) == status


@pytest.mark.parametrize("lam,sb,sd,segments,status", [
    (None, 512, 64, 0, 1), ((1 << 20) * 12, -1, 64, 0, 1), ((1 << 20) * 12 + 1, 512, 64, 0, 3),
    ((1 << 20) * 12, 512, 64, 2, 2),
])
def test_trap_scan_ws_entries_validate(lib, lam, sb, sd, segments, status):
    a = _valid_scan_args()
    a.force_segments = segments
    n = ctypes.c_size_t(7)
    assert lib.mamba_trap_scan_workspace_size(ctypes.byref(a), lam, sb, sd, None, ctypes.byref(n)) == status
    assert n.value == 0
    assert lib.mamba_trap_scan_fwd_ws(ctypes.byref(a), lam, sb, sd, None, None, 0, None) == status


@pytest.mark.parametrize("field,value,status", [
    ("batch", 0, 1), ("ngroups", 3, 1), ("in_dtype", 0, 2), ("x_token_stride", 260, 3),
])
def test_ssd_workspace_size_validates(lib, field, value, status):
    a = _valid_ssd_args()
    setattr(a, field, value)
    n = ctypes.c_size_t(7)
    assert lib.mamba_ssd_workspace_size(ctypes.byref(a), ctypes.byref(n)) == status
    assert n.value == 0


def test_workspace_queries_need_their_arguments(lib):
    a, c = _valid_scan_args(), _valid_conv()
    n = ctypes.c_size_t(0)
    assert lib.mamba_conv_scan_workspace_size(ctypes.byref(a), ctypes.byref(c), None, None) == 1
    assert lib.mamba_conv_scan_workspace_size(ctypes.byref(a), None, None, ctypes.byref(n)) == 1
    assert lib.mamba_trap_scan_workspace_size(ctypes.byref(a), (1 << 20) * 12, 512, 64, None, None) == 1
    assert lib.mamba_ssd_workspace_size(ctypes.byref(_valid_ssd_args()), None) == 1
    assert lib.mamba_ssd_workspace_size(None, ctypes.byref(n)) == 1
