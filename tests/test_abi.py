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


def _dense_pr(sage, **kw):
    args = dict(B=2, Hq=8, Hkv=2, D=128, Nq=300, Nk=500, dtype=__import__("torch").bfloat16,
                q_stride=(8 * 300 * 128, 300 * 128, 128), k_stride=(2 * 500 * 128, 500 * 128, 128),
                v_stride=(2 * 500 * 128, 500 * 128, 128), o_stride=(8 * 300 * 128, 300 * 128, 128))
    args.update(kw)
    return sage.make_problem(**args)


def test_general_problem_sizes_on_host(L):
    import microscaling_fp4_quantized_b200 as sage
    z = sage.problem_sizes(_dense_pr(sage))
    # padded rows: B * round128(Nq) per query head, B * round128(Nk) per key/value head
    assert z["q_fp4"] == 8 * 2 * 384 * 64 and z["q_sf"] == 8 * 2 * 384 * 8
    assert z["k_fp4"] == 2 * 2 * 512 * 64 and z["vt_fp4"] == z["k_fp4"]
    assert z["vt_sf"] == 2 * 2 * 4 * 1024 and z["k_mean"] == 2 * 2 * 128 * 4
    assert z["amax"] == 3 * 2 * 8 * 4 and z["seq"] == 0
    assert z["workspace"] >= sum(z[n] for n in ("q_fp4", "q_sf", "k_fp4", "k_sf", "vt_fp4", "vt_sf"))
    zg = sage.problem_sizes(_dense_pr(sage, gscale="head"))
    assert zg["scratch"] > z["scratch"]
    # packed: bounded by both B * round128(max length) and total + 127 * B
    torch = __import__("torch")
    cu = torch.zeros(4, dtype=torch.int32)  # only its address is passed; nothing is read on the host
    pr = _dense_pr(sage, B=3, Nq=1000, Nk=1000, cu_seqlens_q=cu, cu_seqlens_k=cu, total_q=1100,
                   total_k=1100, q_stride=(0, 128, 8 * 128), k_stride=(0, 128, 2 * 128),
                   v_stride=(0, 128, 2 * 128), o_stride=(0, 128, 8 * 128))
    zp = sage.problem_sizes(pr)
    rows = min(3 * 1024, (1100 + 127 * 3) // 128 * 128)
    assert zp["q_fp4"] == 8 * rows * 64 and zp["seq"] == (2 * 4 + 4) * 4


@pytest.mark.parametrize("bad,status", [
    (dict(Hkv=3), 1),                                  # Hq not a multiple of Hkv
    (dict(D=96), 2),                                   # unsupported head dimension
    (dict(q_stride=(8 * 300 * 128, 300 * 128, 100)), 1),  # token stride not 16-byte granular
    (dict(gscale="none", sm_scale=float("inf")), 1),
    (dict(Nq=-1), 1),
])
def test_general_problem_rejections(L, bad, status):
    import microscaling_fp4_quantized_b200 as sage
    with pytest.raises(sage.SageError) as e:
        sage.problem_sizes(_dense_pr(sage, **bad))
    assert e.value.status == status


def test_packed_problem_needs_both_tables(L):
    import microscaling_fp4_quantized_b200 as sage
    torch = __import__("torch")
    cu = torch.zeros(4, dtype=torch.int32)
    with pytest.raises(sage.SageError) as e:
        sage.problem_sizes(_dense_pr(sage, cu_seqlens_q=cu, total_q=10, total_k=10))
    assert e.value.status == sage.SAGE_ERR_INVALID_ARG


def test_8bit_problem_sizes_and_refusals(L):
    import microscaling_fp4_quantized_b200 as sage
    z = sage.problem_sizes(_dense_pr(sage, precision="8bit"))
    # one byte per element, one float per 128-row tile, float channel scales for V
    assert z["q_fp4"] == 8 * 2 * 384 * 128 and z["q_sf"] == 8 * 2 * 3 * 4
    assert z["k_fp4"] == 2 * 2 * 512 * 128 and z["vt_fp4"] == z["k_fp4"] and z["k_sf"] == 2 * 2 * 4 * 4
    assert z["vt_sf"] == 2 * 2 * 128 * 4 and z["amax"] == 0 and z["qk_bias"] == 0
    for bad in (dict(gscale="tensor"), dict(smooth_q=True)):
        with pytest.raises(sage.SageError) as e:
            sage.problem_sizes(_dense_pr(sage, precision="8bit", **bad))
        assert e.value.status == sage.SAGE_ERR_UNSUPPORTED


def test_bounds_checked_build_loads_and_reports_itself():
    """The bounds-checked variant exports the same entry points and says it is checked;
    the regular build says it is not, and refuses the checked build's test switch."""
    import ctypes
    from microscaling_fp4_quantized_b200 import build as b
    path = b.build(checks=True)
    C = ctypes.CDLL(path)
    for name in _declared():
        assert hasattr(C, name), name
    assert C.sage_fp4_bounds_checked() == 1
    R = ctypes.CDLL(b.build())
    assert R.sage_fp4_bounds_checked() == 0
    R.sage_fp4_set_debug_flags.argtypes = [ctypes.c_uint32]
    C.sage_fp4_set_debug_flags.argtypes = [ctypes.c_uint32]
    assert R.sage_fp4_set_debug_flags(2) == 2       # SAGE_ERR_UNSUPPORTED
    assert C.sage_fp4_set_debug_flags(2) == 0 and C.sage_fp4_set_debug_flags(0) == 0
    assert R.sage_fp4_set_debug_flags(4) == 1       # SAGE_ERR_INVALID_ARG
