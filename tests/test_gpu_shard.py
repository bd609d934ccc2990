"""GPU check of the B*H partition: the forward of each rank's slice of (batch, head) pairs
equals the same pairs of the whole problem, bit for bit (every pair is an independent
problem). Ranks are emulated as slices on one GPU; nothing here waits on another rank."""
import pytest
import torch

from microscaling_fp4_quantized_b200 import shard, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sage():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import microscaling_fp4_quantized_b200 as s
    s.lib()
    return s


@pytest.mark.parametrize("N,causal", [(2048, False), (512, True)])
def test_slices_equal_the_whole_problem(sage, N, causal):
    wl = workloads.custom(2, 5, N, 128, causal=causal, seed=91)
    q, k, v = workloads.make_inputs(wl, device="cuda")
    whole = sage.attn(q, k, v, causal=causal, sm_scale=wl.sm_scale)
    BH = wl.B * wl.H
    flat = lambda t: t.reshape(BH, wl.N, wl.D)  # noqa: E731
    for world in (2, 3):
        parts = []
        for r in range(world):
            lo, hi = shard.head_slice(BH, world, r)
            parts.append(shard.attn_slice(flat(q)[lo:hi].contiguous(), flat(k)[lo:hi].contiguous(),
                                          flat(v)[lo:hi].contiguous(), causal=causal, sm_scale=wl.sm_scale))
        torch.cuda.synchronize()
        assert sage.device_error() == 0
        assert torch.equal(torch.cat(parts, 0), flat(whole)), world
