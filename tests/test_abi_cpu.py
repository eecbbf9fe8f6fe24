"""CPU-only checks of the C ABI: the library loads without a GPU and exports
every function include/ttt.h declares; host-side validation answers without
touching the device."""
import ctypes
import os
import re

import pytest

from weight_long_context_b200 import ttt

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "ttt.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ttt_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from weight_long_context_b200 import build
    build.build()
    return ttt.load_library()


def test_header_declares_the_entry_points():
    names = declared_functions()
    assert set(names) == set(ttt.EXPORTED), names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    assert ttt.ttt_status_string(0) == "ok"
    assert ttt.ttt_status_string(2) == "invalid shape"
    assert ttt.ttt_status_string(99) == "unknown status"


def _create(lib, cfg):
    h = ctypes.c_void_p()
    dummy = ctypes.c_void_p(16)  # never dereferenced: validation rejects first
    return lib.ttt_create(ctypes.byref(cfg), dummy, dummy, None, ctypes.byref(h))


def test_config_validation_is_host_side(lib):
    C = ttt.ttt_config
    assert _create(lib, C(30, 32, 32, 1, 0, 0, 0, 0, 1e-6)) == 3        # d % 16
    assert _create(lib, C(32, 32, 32, 1, 7, 0, 0, 0, 1e-6)) == 1        # bad mlp
    assert _create(lib, C(32, 32, 32, 1, 0, 0, 5, 0, 1e-6)) == 1        # bad precision
    assert _create(lib, C(32, 32, 32, 0, 0, 0, 0, 0, 1e-6)) == 2        # n_blocks
    assert _create(lib, C(32, 32, 32, 1, 0, 0, 0, 0, float("nan"))) == 1
    assert _create(lib, C(32, 32, 32, 1, 0, 1, 0, 0, 1e-6)) == 1        # static_w NULL with has_static
    assert b"NULL" in lib.ttt_last_error()


def test_scalar_kernels_shape_validation(lib):
    z = ctypes.c_void_p(16)
    for rule in (0, 1):   # E2TTT, LaCT
        assert lib.ttt_scalar_kernels(rule, 1, 10, 3, z, z, z, z, z, z, None) == 2
        assert lib.ttt_scalar_kernels(rule, 1, 10, 0, z, z, z, z, z, z, None) == 2
        assert lib.ttt_scalar_kernels(rule, 0, 0, 4, z, z, z, z, z, z, None) == 0
    assert lib.ttt_scalar_kernels(2, 0, 0, 4, z, z, z, z, z, z, None) == 1   # unknown rule


def test_create_rejects_unknown_update_rule(lib):
    C = ttt.ttt_config
    assert _create(lib, C(32, 32, 32, 1, 0, 0, 0, 0, 1e-6, 2)) == 1
    assert b"update_rule" in lib.ttt_last_error()


def test_scalar_heads_validation(lib):
    z = ctypes.c_void_p(16)
    args = lambda d, tau: (1, 4, d, z, z, 0.0, 0.0, 0.0, 0.01, 1.0, tau, z, z, z, None)
    assert lib.ttt_scalar_heads(*args(6, 16.0)) == 2          # d % 4
    assert lib.ttt_scalar_heads(*args(8, 0.0)) == 1           # tau <= 0
    assert lib.ttt_scalar_heads(*args(8, float("inf"))) == 1
    assert lib.ttt_scalar_heads(0, 0, 8, z, z, 0.0, 0.0, 0.0, 0.01, 1.0, 16.0, z, z, z, None) == 0


def test_recon_head_config_validation(lib):
    C = ttt.ttt_config
    assert _create(lib, C(32, 32, 32, 1, 0, 0, 0, 0, 1e-6, 0, 2)) == 1        # unknown head
    assert _create(lib, C(32, 32, 0, 2, 0, 0, 0, 0, 1e-6, 0, 1)) == 3         # recon: one block only
    assert _create(lib, C(32, 32, 0, 1, 0, 1, 0, 0, 1e-6, 0, 1)) == 3         # recon: no static MLP
    assert lib.ttt_prefill_recon(None, 1, 8, 4, *([None] * 10), None, 0, None) == 1   # NULL handle


def test_prefill_rejects_null_handle(lib):
    n = ctypes.c_size_t()
    assert lib.ttt_workspace_size(None, 1, 8, 4, ctypes.byref(n)) == 1


def test_predict_rejects_null_handle(lib):
    assert lib.ttt_predict(None, 1, 8, 4, *([None] * 5), None, 0, None) == 1
    assert b"NULL" in lib.ttt_last_error()


def test_set_attention_rejects_null_handle(lib):
    assert lib.ttt_set_attention(None, 4, 8, None, None, None, 1e-5) == 1
    assert b"NULL" in lib.ttt_last_error()
