"""Failure detection without a GPU fault.

The test switch makes the attention kernel issue no loads, so every bounded wait in the
other roles runs out (50 ms here). The kernel must drain, release its tensor memory and
return; the host must read a timeout from the device error word; and the same context
must then run a normal forward that matches the oracle.
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


# A causal problem with fewer work items than SMs (one item per CTA) and a short dense
# non-causal D = 128 problem with many (sequence, head, query tile) items per CTA, so that
# the abort reaches CTAs in the middle of their walk (drains of the last Q/K/V loads and
# of both MMA issuers with several items behind them).
CASES = [workloads.custom(1, 2, 384, 128, causal=True, seed=61),
         workloads.custom(8, 32, 1024, 128, causal=False, seed=62)]


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_bounded_wait_reports_timeout_and_context_survives(sage, oracle_mod, wl):
    q, k, v = workloads.make_inputs(wl, device="cuda")
    assert sage.device_error() == 0
    sage.set_wait_timeout_ns(50_000_000)
    sage.set_debug_flags(1)
    try:
        sage.attn(q, k, v, causal=wl.causal, sm_scale=wl.sm_scale)
        torch.cuda.synchronize()
    finally:
        sage.set_debug_flags(0)
        sage.set_wait_timeout_ns(0)
    word = sage.device_error()
    assert word & 1, f"expected the timeout bit, got {word:#x}"
    assert sage.device_error() == 0  # reading clears it

    out = sage.attn(q, k, v, causal=wl.causal, sm_scale=wl.sm_scale)
    torch.cuda.synchronize()
    assert sage.device_error() == 0
    BH = wl.B * wl.H
    heads = sorted({0, 1, BH - 1})
    f = lambda t: t.float().cpu().numpy().reshape(BH, wl.N, wl.D)[heads]  # noqa: E731
    em, _ = oracle_mod.attention(f(q), f(k), f(v), wl.causal, wl.sm_scale)
    m = oracle_mod.metrics(f(out), em)
    assert m["cos"] >= 0.999 and m["max_abs"] <= 1e-2 * float(np.abs(f(v)).max()), m


def test_debug_flags_reject_unknown_bits(sage):
    with pytest.raises(sage.SageError) as e:
        sage.set_debug_flags(4)
    assert e.value.status == sage.SAGE_ERR_INVALID_ARG
    if not sage.lib().sage_fp4_bounds_checked():
        # the output-extent switch exists in the bounds-checked build only
        with pytest.raises(sage.SageError) as e:
            sage.set_debug_flags(2)
        assert e.value.status == sage.SAGE_ERR_UNSUPPORTED
