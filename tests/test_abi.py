"""The C-ABI library builds, loads and exports what include/muon.h declares (no GPU needed)."""
import ctypes
import os
import re

import pytest

import spectral_optimizer_state_b200 as sos
from spectral_optimizer_state_b200 import binding
from spectral_optimizer_state_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return sos.load_library()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "muon.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(muon_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert len(names) >= 21
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(binding.EXPORTS) == names


def test_status_strings(lib):
    for code, name in binding.STATUS_NAMES.items():
        assert lib.muon_status_string(code).decode() == name
    assert lib.muon_abi_version() == 2


def test_argument_errors_need_no_device(lib):
    # Every one of these is rejected on the host before any CUDA call.
    assert lib.muon_create(None, 0) == 1
    assert lib.muon_set_coeffs(None, None, 5) == 1
    assert lib.muon_get_coeffs(None, None, None) == 1
    hp = binding.Hparams(0.02, 0.95, 0.1, 1e-7, 1, 0, 1.0)
    assert lib.muon_step(None, None, None, None, 1, 8, 8, 0, ctypes.byref(hp), None) == 1
    assert lib.muon_step_groups(None, None, 1, ctypes.byref(hp), None) == 1
    assert lib.muon_ns_orthogonalize(None, None, None, 1, 8, 8, 0, 1e-7, None) == 1
    assert lib.muon_get_status(None, None, 0, None) == 1
    assert lib.muon_workspace_bytes(None) == 0
    assert lib.muon_destroy(None) == 0


def test_create_without_gpu_reports_no_device(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    h = ctypes.c_void_p()
    assert lib.muon_create(ctypes.byref(h), 0) == 7
    with pytest.raises(sos.MuonError):
        sos.Muon(0)


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(ImportError):
        binding.load_library(str(tmp_path / "nope.so"))


def test_binding_validates_before_calling():
    import torch
    with pytest.raises(TypeError):
        binding._dtype_code(torch.zeros(2, 2, dtype=torch.float16))
    with pytest.raises(ValueError):
        binding._check_same([torch.zeros(2, 3)], (2, 2), torch.float32, "cpu", "W")


def declared_arities():
    """name -> number of parameters, from the prototypes in include/muon.h."""
    text = open(os.path.join(ROOT, "include", "muon.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = {}
    for m in re.finditer(r"\b(muon_[a-z_]+)\s*\(([^;{]*?)\)\s*;", text, flags=re.S):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_argtypes_match_the_prototypes(lib):
    arities = declared_arities()
    assert sorted(arities) == declared_symbols()
    for name, n in arities.items():
        fn = getattr(lib, name)
        assert fn.argtypes is not None and len(fn.argtypes) == n, (name, n, fn.argtypes)
