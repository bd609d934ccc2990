"""The allocation-free forward entry point (sage_fp4_attn_fwd_noalloc).

It serves callers that cannot allocate device memory; its scratch is a fixed device
array inside the library. Two consecutive calls (different shapes, so the second runs on
what the first left in the shared array) must each match the regular workspace entry
point within the attention tolerance of the other GPU tests, and the second call is
also held to the oracle's emulation of the method (the bar of the parity tests), so a
fault shared by both entry points cannot pass. This file is named so that pytest
collects it last.
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


def _close(oracle_mod, got, ref, v):
    m = oracle_mod.metrics(np.asarray(got, np.float64), np.asarray(ref, np.float64))
    vmax = float(np.abs(v).max())
    assert m["max_abs"] <= 1e-2 * vmax, m
    assert m["cos"] >= 0.999, m


def test_noalloc_matches_workspace_entry_point_two_calls(sage, oracle_mod):
    for i, wl in enumerate((workloads.MEDIUM, workloads.custom(1, 2, 300, 128, causal=True, seed=51))):
        q, k, v = workloads.make_inputs(wl, device="cuda")
        ref = sage.attn(q, k, v, causal=wl.causal, sm_scale=wl.sm_scale)
        got = sage.attn_noalloc(q, k, v, causal=wl.causal, sm_scale=wl.sm_scale)
        torch.cuda.synchronize()
        assert sage.device_error() == 0
        BH = wl.B * wl.H
        f = lambda t: t.float().cpu().numpy().reshape(BH, wl.N, wl.D)  # noqa: E731
        _close(oracle_mod, f(got), f(ref), f(v))
        if i == 1:
            # The second call, made on what the first left in the shared array, against the
            # oracle's emulation of the whole method.
            em, _ = oracle_mod.attention(f(q), f(k), f(v), wl.causal, wl.sm_scale, Bk=128)
            _close(oracle_mod, f(got), em, f(v))


def test_noalloc_rejects_problems_beyond_its_scratch(sage):
    q = torch.zeros((1, 32, 4096, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.full_like(q, 7.0)
    with pytest.raises(sage.SageError) as e:
        sage.attn_noalloc(q, q, q, out=out)
    assert e.value.status == sage.SAGE_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())  # nothing was launched
