"""The B*H partition of one attention problem across ranks (shard.py): the slice
arithmetic covers every (batch, head) pair exactly once in contiguous, balanced slices,
and the optional all-gather reassembles the slices in order. Two gloo ranks on
127.0.0.1, no GPU; the GPU check that a slice's forward equals the same heads of the
whole problem is in test_gpu_shard.py."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from microscaling_fp4_quantized_b200 import shard  # noqa: E402


@pytest.mark.parametrize("n", [0, 1, 5, 24, 128, 1001])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_head_slices_partition_the_pairs(n, world):
    covered = []
    sizes = shard.slice_sizes(n, world)
    for r in range(world):
        lo, hi = shard.head_slice(n, world, r)
        assert 0 <= lo <= hi <= n
        covered.extend(range(lo, hi))
        if r > 0:
            assert lo == shard.head_slice(n, world, r - 1)[1]  # contiguous, in rank order
    assert covered == list(range(n))
    assert max(sizes) - min(sizes) <= 1 and sum(sizes) == n


def test_bad_partition_rejected():
    with pytest.raises(ValueError):
        shard.head_slice(4, 0, 0)
    with pytest.raises(ValueError):
        shard.head_slice(4, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, n_pairs, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from microscaling_fp4_quantized_b200 import shard as sh
    lo, hi = sh.head_slice(n_pairs, world, rank)
    # A stand-in for this rank's attention output: every element of pair i holds i.
    out_r = torch.arange(lo, hi, dtype=torch.float32).view(-1, 1, 1).expand(hi - lo, 3, 2).contiguous()
    full = sh.gather_heads(out_r, n_pairs)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, full.tolist()))


@pytest.mark.parametrize("n_pairs", [5, 8])
def test_gather_reassembles_in_pair_order(n_pairs):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, n_pairs, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    want = torch.arange(n_pairs, dtype=torch.float32).view(-1, 1, 1).expand(n_pairs, 3, 2).tolist()
    for _ in range(2):
        rank, full = q.get(timeout=10)
        assert full == want, rank


def _attn_worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import numpy as np
    import oracle
    from microscaling_fp4_quantized_b200 import shard as sh
    n_pairs, N, D = 5, 96, 64
    g = np.random.default_rng(7)                       # every rank draws the same whole problem
    qq, kk, vv = (g.standard_normal((n_pairs, N, D)) for _ in range(3))
    lo, hi = sh.head_slice(n_pairs, world, rank)
    o_r, _ = oracle.attention(qq[lo:hi], kk[lo:hi], vv[lo:hi], True, D ** -0.5)
    full = sh.gather_heads(torch.from_numpy(np.ascontiguousarray(o_r)), n_pairs)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, full.numpy()))


@pytest.mark.parametrize("world", [2, 3])
def test_sliced_forward_equals_whole_problem(world):
    """Each rank runs the (oracle) FP4 forward on its slice of 5 pairs and gathers: every
    rank must hold exactly the whole problem's result, pair order kept."""
    import numpy as np
    import oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_attn_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    g = np.random.default_rng(7)
    qq, kk, vv = (g.standard_normal((5, 96, 64)) for _ in range(3))
    want, _ = oracle.attention(qq, kk, vv, True, 64 ** -0.5)
    for rank, full in got:
        assert full.shape == want.shape, rank
        assert np.array_equal(full, want), rank
