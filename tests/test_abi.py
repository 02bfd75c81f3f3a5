"""The C ABI library builds, loads without a GPU and exports every symbol that
include/mpe.h declares; the binding's error path works without a device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from mixed_precision_expert_b200.build import build
    build()
    import mixed_precision_expert_b200 as mpe
    return mpe.lib()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "mpe.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mpe_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_binding_exports():
    import mixed_precision_expert_b200 as mpe
    assert declared_symbols() == sorted(mpe.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_version_and_argument_errors_without_gpu(lib):
    import mixed_precision_expert_b200 as mpe
    assert lib.mpe_version() == 100
    # invalid arguments are rejected before any device work
    assert lib.mpe_create(None, None) == -1
    cfg = mpe.Config(0, 256, 512, 0, 0, 0, 0, 0, None)
    h = ctypes.c_void_p()
    assert lib.mpe_create(ctypes.byref(h), ctypes.byref(cfg)) == -1
    assert b"E=0" in lib.mpe_last_error_global()
    cfg = mpe.Config(8, 200, 512, 0, 0, 0, 0, 0, None)
    assert lib.mpe_create(ctypes.byref(h), ctypes.byref(cfg)) == -1
    with pytest.raises(mpe.MpeError):
        mpe.allocate_bits([0.5, 0.5], [10, 0], 100)      # W_e = 0
    with pytest.raises(mpe.MpeError) as ei:
        mpe.allocate_bits([0.5, 0.5], [10, 10], 59)      # below 3 bits per weight
    assert ei.value.code == -2


def test_beyond_path_argument_errors_without_gpu(lib):
    import numpy as np

    import mixed_precision_expert_b200 as mpe
    # the loss-table program validates its table before any device work
    with pytest.raises(mpe.MpeError) as ei:
        mpe.allocate_bits_table([0.5, 0.5], np.array([[1e-3, 1e-4, np.nan], [1e-3, 1e-4, 1e-6]]),
                                [10, 10], 100)
    assert ei.value.code == -1
    with pytest.raises(ValueError):
        mpe.allocate_bits_table([0.5, 0.5], np.zeros((3, 3)), [10, 10], 100)
    with pytest.raises(mpe.MpeError) as ei:
        mpe.allocate_bits_table([0.5, 0.5], np.full((2, 3), 1e-3), [10, 10], 59)
    assert ei.value.code == -2
    with pytest.raises(mpe.MpeError):
        mpe.allocate_bits_proportional([0.5, -0.5], [10, 10], 100)  # p < 0
    # the channel choice and the layered store reject bad sizes up front
    out = ctypes.c_void_p(1)
    assert lib.mpe_select_salient(ctypes.c_void_p(1), 4, 64, 0, out, None) == -1
    assert lib.mpe_select_salient(ctypes.c_void_p(1), 4, 64, 257, out, None) == -1
    assert lib.mpe_select_salient(None, 0, 64, 8, None, None) == 0   # no rows: nothing to do
    h = ctypes.c_void_p()
    cfg = mpe.Config(4, 100, 256, 0, 0, 0, 0, 0, None)
    assert lib.mpe_prefix_create(ctypes.byref(h), ctypes.byref(cfg)) == -1
    cfg = mpe.Config(4, 256, 256, 1000, 0, 0, 0, 0, None)
    assert lib.mpe_prefix_create(ctypes.byref(h), ctypes.byref(cfg)) == -1
    assert lib.mpe_prefix_quantize(None, None, None) == -1
    assert lib.mpe_set_compensation(None, 8, 0) == -1
    assert lib.mpe_selftest_wait(None, 1000) == -1
