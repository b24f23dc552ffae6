"""The C-ABI library loads and exports every symbol include/*.h declares (CPU only).

No compute call is made here: only calls that return before touching a GPU.
"""
import ctypes
import glob
import os
import re

import pytest

from vla_flow_matching_b200 import build as B
from vla_flow_matching_b200 import pi0x

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return pi0x.load()


def declared_symbols():
    names = set()
    for hdr in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(hdr).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b(pi0x_[a-z0-9_]+)\s*\(", text):
            names.add(m.group(1))
    return sorted(names)


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert "pi0x_sample" in names and "pi0x_create" in names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    assert set(pi0x.EXPORTED) <= set(names)


def test_status_strings_and_version(lib):
    for code in range(7):
        s = lib.pi0x_status_string(code)
        assert s and s != b"unknown status"
    assert lib.pi0x_status_string(99) == b"unknown status"
    assert lib.pi0x_version() >= 100


def test_null_arguments_are_rejected_without_a_gpu(lib):
    h = ctypes.c_void_p()
    assert lib.pi0x_create(None, None, ctypes.byref(h)) == pi0x.PI0X_EINVAL
    assert lib.pi0x_sample(None, None, None, None, 1, 1, None, None, 1, None, None) == pi0x.PI0X_EINVAL
    assert lib.pi0x_sync_status(None) == pi0x.PI0X_EINVAL
    assert lib.pi0x_set_variant(None, 0, 0, 0) == pi0x.PI0X_EINVAL
    assert lib.pi0x_launch_count(None, 1, 1, 1) == -1
    lib.pi0x_destroy(None)


def test_unsupported_dims_are_rejected_before_device_use(lib):
    cfg = pi0x.Config(512, 18, 4096, 8, 1, 256, 50, 32, 32, 0)
    w = pi0x.Weights()
    layers = (pi0x.LayerWeights * 1)()
    w.layers = ctypes.cast(layers, ctypes.POINTER(pi0x.LayerWeights))
    h = ctypes.c_void_p()
    assert lib.pi0x_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h)) == pi0x.PI0X_EUNSUPPORTED
    cfg = pi0x.Config(1024, 0, 4096, 8, 1, 256, 50, 32, 32, 0)
    assert lib.pi0x_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h)) == pi0x.PI0X_EINVAL


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "vla_flow_matching_b200")
    for path in glob.glob(os.path.join(pkg, "**", "*.*"), recursive=True):
        if path.endswith((".py", ".cu", ".cuh", ".h")):
            text = open(path).read()
            assert not re.search(r"^\s*(import|from)\s+oracle\b|pi0_oracle|oracle/", text, re.M), path
