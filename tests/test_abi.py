"""The C-ABI library loads and exports every symbol include/gtr_gla.h declares (CPU only).

No compute call is made here; host-only queries that need no GPU are exercised.
"""
import ctypes
import os
import re
import subprocess

import pytest

from recurrent_vision_backbone_b200 import build, gla

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", n) for n in sorted(os.listdir(os.path.join(ROOT, "include")))
           if n.endswith(".h")]


def declared_functions():
    names = set()
    for h in HEADERS:
        names |= set(re.findall(r"\b(gtr_[a-z_]+)\s*\(", open(h).read()))
    return sorted(names)


@pytest.fixture(scope="module")
def lib_path():
    return build.build()


def test_header_declares_the_boundary():
    names = declared_functions()
    assert "gtr_gla_fwd" in names and "gtr_gla_device_status" in names
    assert set(names) == set(gla.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol(lib_path):
    out = subprocess.run(["nm", "-D", "--defined-only", lib_path], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (gtr_\w+)", out))
    missing = set(declared_functions()) - exported
    assert not missing, f"not exported: {missing}"


def test_library_loads_and_answers_host_queries(lib_path):
    lib = gla.load(lib_path)
    assert gla.version().count(".") == 2
    assert gla.status_str(gla.GTR_ERR_TIMEOUT) == "device-side wait timed out"
    assert lib.gtr_status_str(99) == b"unknown status"


def test_library_is_built_for_sm100a(lib_path):
    # the fat binary must carry sm_100a code (cuobjdump-free check: nvcc's -gencode is in
    # the build command and the ELF has an .nv_fatbin section)
    assert "arch=compute_100a,code=sm_100a" in " ".join(build.nvcc_cmd())
    out = subprocess.run(["readelf", "-S", lib_path], capture_output=True, text=True).stdout
    assert ".nv_fatbin" in out


def test_header_compiles_as_c(tmp_path):
    src = tmp_path / "t.c"
    src.write_text('#include "gtr_gla.h"\nint main(void){ return (int)GTR_OK; }\n')
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(tmp_path / "t")], check=True)


def test_binding_refuses_host_tensors(lib_path):
    """No CPU fallback: every entry of the binding refuses tensors that are not on a
    CUDA device before it calls the library."""
    import torch
    gla.load(lib_path)
    h = lambda *s: torch.zeros(s, dtype=torch.float16)  # noqa: E731
    q = h(1, 4, 2, 64)
    with pytest.raises(ValueError):
        gla.gtr_gla_fwd(q, q, q, q, 2, 2, 0)
    with pytest.raises(ValueError):
        gla.gtr_gla_fwd_z(q, q, q, q, 16.0, 2, 2, 0)
    with pytest.raises(ValueError):
        gla.gtr_gla_bwd(q, q, q, q, q, 2, 2, 0)
