"""CPU-side checks of the C ABI: the library loads without a GPU and exports every
function include/sage_fp4.h declares; host-side argument checks need no device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "sage_fp4.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sage_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    from microscaling_fp4_quantized_b200 import build
    build.build()
    import microscaling_fp4_quantized_b200 as sage
    return sage.lib()


def test_header_declares_entry_points():
    names = _declared()
    assert "sage_fp4_attn_fwd" in names and "sage_fp4_quantize_qkv" in names


def test_library_exports_every_declared_symbol(L):
    for name in _declared():
        assert hasattr(L, name), name


def test_binding_names_match_header():
    import microscaling_fp4_quantized_b200 as sage
    assert sorted(sage.EXPORTED) == _declared()


def test_host_side_argument_checks(L):
    import microscaling_fp4_quantized_b200 as sage
    assert sage.sizes(2, 3, 300, 128)["q_fp4"] == 6 * 384 * 64
    assert sage.sizes(2, 3, 300, 128)["vt_sf"] == 6 * 3 * 1024
    assert sage.sizes(0, 3, 300, 64)["q_fp4"] == 0
    with pytest.raises(sage.SageError) as e:
        sage.sizes(1, 1, 128, 80)
    assert e.value.status == sage.SAGE_ERR_UNSUPPORTED
    with pytest.raises(sage.SageError) as e:
        sage.sizes(1, -1, 128, 64)
    assert e.value.status == sage.SAGE_ERR_INVALID_ARG
    # null pointers are rejected before anything touches a device
    st = L.sage_fp4_attn_fwd_quantized(None, None, None, None, None, None, None, 0, 1, 1, 128, 64, 0,
                                       ctypes.c_float(0.0), None)
    assert st == sage.SAGE_ERR_INVALID_ARG
    st = L.sage_fp4_quantize_qkv(None, None, None, 0, 1, 1, 128, 64, 1, None, None, None, None, None,
                                 None, None, None, 0, None)
    assert st == sage.SAGE_ERR_INVALID_ARG
    # empty problems are a successful no-op
    assert L.sage_fp4_attn_fwd(None, None, None, None, 0, 4, 128, 64, 0, ctypes.c_float(0.0), None) == 0
    assert L.sage_status_string(4) == b"SAGE_ERR_TIMEOUT"
    assert sage.workspace_bytes(1, 24, 32768, 128) > 0
