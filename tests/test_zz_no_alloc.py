"""The allocation-free forward entry point (sage_fp4_attn_fwd_noalloc).

It serves callers that cannot allocate device memory; its scratch is a fixed device
array inside the library. Two consecutive calls (different shapes, so the second runs on
what the first left in the shared array) must each match the regular workspace entry
point within the attention tolerance of the other GPU tests. This file is named so that
pytest collects it last.
"""
import numpy as np
import pytest
import torch

from microscaling_fp4_quantized_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sage():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import microscaling_fp4_quantized_b200 as s
    s.lib()
    return s


def _close(sage, got, ref, v):
    g = got.float().cpu().numpy().ravel().astype(np.float64)
    r = ref.float().cpu().numpy().ravel().astype(np.float64)
    vmax = float(v.float().abs().max())
    max_abs = float(np.abs(g - r).max())
    cos = float((g * r).sum() / np.sqrt((g * g).sum() * (r * r).sum()))
    assert max_abs <= 1e-2 * vmax, max_abs
    assert cos >= 0.999, cos


def test_noalloc_matches_workspace_entry_point_two_calls(sage):
    for wl in (workloads.MEDIUM, workloads.custom(1, 2, 300, 128, causal=True, seed=51)):
        q, k, v = workloads.make_inputs(wl, device="cuda")
        ref = sage.attn(q, k, v, causal=wl.causal, sm_scale=wl.sm_scale)
        got = sage.attn_noalloc(q, k, v, causal=wl.causal, sm_scale=wl.sm_scale)
        torch.cuda.synchronize()
        assert sage.device_error() == 0
        _close(sage, got, ref, v)


def test_noalloc_rejects_problems_beyond_its_scratch(sage):
    q = torch.zeros((1, 32, 4096, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.full_like(q, 7.0)
    with pytest.raises(sage.SageError) as e:
        sage.attn_noalloc(q, q, q, out=out)
    assert e.value.status == sage.SAGE_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())  # nothing was launched
