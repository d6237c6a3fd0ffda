"""The C ABI without a GPU: the library loads, exports every function rdt.h declares, and
rejects bad arguments before touching a device."""
import ctypes
import os
import re

import pytest

import recurrent_depth_transformer_b200 as R
from recurrent_depth_transformer_b200.build import build
from workloads import WORKLOADS

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "rdt.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return R.load_library()


def declared_functions():
    src = open(HDR).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return set(re.findall(r"^\s*(?:rdt_status|const char\*|void)\s+(rdt_\w+)\s*\(", src, flags=re.M))


def test_header_declares_the_boundary():
    fns = declared_functions()
    for f in ("rdt_create", "rdt_attn_forward", "rdt_moe_forward", "rdt_loop_forward"):
        assert f in fns
    assert fns == set(R.EXPORTED)


def test_every_declared_symbol_is_exported(lib):
    for f in declared_functions():
        assert hasattr(lib, f), f


def test_status_strings(lib):
    assert lib.rdt_status_string(0) == b"ok"
    assert b"rho" in lib.rdt_status_string(4)
    assert lib.rdt_status_string(99) == b"unknown status"


def test_create_rejects_bad_config_before_any_device_call(lib):
    cfg = R.make_config(WORKLOADS[1])
    w = R.RdtWeights()
    h = ctypes.c_void_p()
    bad = R.make_config(WORKLOADS[1])
    bad.top_k = bad.n_experts + 1
    assert lib.rdt_create(ctypes.byref(bad), ctypes.byref(w), None, ctypes.byref(h)) == 1
    assert b"top_k" in lib.rdt_last_error()
    bad = R.make_config(WORKLOADS[1])
    bad.dim = 1000
    assert lib.rdt_create(ctypes.byref(bad), ctypes.byref(w), None, ctypes.byref(h)) == 2
    bad = R.make_config(WORKLOADS[1], max_loops=0)
    assert lib.rdt_create(ctypes.byref(bad), ctypes.byref(w), None, ctypes.byref(h)) == 1
    assert lib.rdt_create(ctypes.byref(cfg), None, None, ctypes.byref(h)) == 1
    # missing weight pointers are caught before the device is queried
    assert lib.rdt_create(ctypes.byref(cfg), ctypes.byref(w), None, ctypes.byref(h)) == 1
    assert b"NULL" in lib.rdt_last_error()
    assert h.value is None


def test_calls_reject_null_handle(lib):
    assert lib.rdt_loop_forward(None, None, None, 1, None, None) == 1
    assert lib.rdt_set_trace(None, None, None, None) == 1
    assert lib.rdt_set_act(None, None, 0.0, 0.99, None) == 1
    assert lib.rdt_loop_forward_act(None, None, None, 1, None, None, None) == 1
    lib.rdt_destroy(None)


def test_configs_of_all_workloads_validate_shapes():
    for wl in WORKLOADS:
        c = R.make_config(wl, max_loops=max(wl.loops))
        assert c.batch * c.seq == wl.tokens


def test_ctypes_structs_match_the_header(tmp_path):
    """Every field offset and struct size of the ctypes mirrors in the binding equals the C
    compiler's for include/rdt.h (a field added on one side only would shift the others)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    mirrors = {"rdt_config": R.RdtConfig, "rdt_weights": R.RdtWeights, "rdt_diag": R.RdtDiag,
               "rdt_kernel_stat": R.RdtKernelStat}
    lines = ['#include <stdio.h>', '#include <stddef.h>', f'#include "{HDR}"', "int main(void) {"]
    for cname, py in mirrors.items():
        lines.append(f'    printf("{cname} size %zu\\n", sizeof({cname}));')
        for field, _ in py._fields_:
            lines.append(f'    printf("{cname} {field} %zu\\n", offsetof({cname}, {field}));')
    lines += ["    return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-std=c11", str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    got = {tuple(l.split()[:2]): int(l.split()[2]) for l in out if l.strip()}
    for cname, py in mirrors.items():
        assert got[(cname, "size")] == ctypes.sizeof(py), cname
        for field, _ in py._fields_:
            assert got[(cname, field)] == getattr(py, field).offset, (cname, field)
