"""Host-only checks of the C-ABI library (no kernel is launched)."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fipa.h")


@pytest.fixture(scope="module")
def lib():
    from protein_structure_models_b200 import build, fipa
    build.build()
    return fipa.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fipa_[a-z_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("fipa_create", "fipa_workspace_size", "fipa_forward", "fipa_sync_status",
              "fipa_status_string", "fipa_last_error", "fipa_destroy"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_library_exports_nothing_else(lib):
    import subprocess
    from protein_structure_models_b200 import fipa
    out = subprocess.run(["nm", "-D", "--defined-only", fipa.library_path()], capture_output=True,
                         text=True).stdout
    exported = sorted({ln.split()[-1] for ln in out.splitlines() if " T " in ln})
    assert exported == declared_functions()


def test_status_strings(lib):
    for code in range(7):
        s = lib.fipa_status_string(code)
        assert isinstance(s, bytes) and len(s) > 0
    assert lib.fipa_status_string(99) == b"unknown status"


def test_null_handles_are_safe(lib):
    assert lib.fipa_destroy(None) == 0
    assert lib.fipa_last_error(None) == b""
    from protein_structure_models_b200.fipa import FipaDims
    n = ctypes.c_size_t()
    assert lib.fipa_workspace_size(None, ctypes.byref(FipaDims(*[1] * 10)), ctypes.byref(n)) == 1
    assert lib.fipa_create(None, None, 1, 0) == 1


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU failure path")
def test_create_without_gpu_fails_cleanly(lib):
    h = ctypes.c_void_p()
    st = lib.fipa_create(ctypes.byref(h), None, 1, 0)
    assert st != 0
    assert not h.value


def test_binding_raises_without_library(monkeypatch, tmp_path):
    from protein_structure_models_b200 import fipa
    monkeypatch.setattr(fipa, "_lib", None)
    monkeypatch.setattr(fipa, "_LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="not found"):
        fipa.load_library()
