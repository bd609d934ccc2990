"""GPU parity of the fused FP4 attention forward against the emulated oracle.

Bar (per configuration): max |O_gpu - O_oracle| <= 1e-2 * max|V| and cosine similarity
>= 0.999 against the oracle's emulation of the same quantization (same key-tile width,
128). P~ codes are not unique (the GPU's S is FP32 with its own summation order and
exp2 is approximate), so the output is judged by tolerance; cos / relative L1 / RMSE
against exact binary64 attention are printed for information only.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import f32, heads_view, sample_rows
from microscaling_fp4_quantized_b200 import workloads

pytestmark = pytest.mark.gpu

MAX_ABS_FRAC = 1e-2
MIN_COS = 0.999


@pytest.fixture(scope="module")
def sage():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import microscaling_fp4_quantized_b200 as s
    s.lib()
    return s


def _check(sage, oracle_mod, wl, heads=None, rows_per_head=None, entry="attn"):
    q, k, v = workloads.make_inputs(wl, device="cuda")
    if entry == "attn":
        out = sage.attn(q, k, v, causal=wl.causal, sm_scale=wl.sm_scale)
    elif entry == "library_ws":
        out = sage.attn_bf16_library_workspace(q, k, v, causal=wl.causal, sm_scale=wl.sm_scale)
    else:
        out = sage.attn_quantized(sage.quantize_qkv(q, k, v), causal=wl.causal, sm_scale=wl.sm_scale)
    torch.cuda.synchronize()
    assert sage.device_error() == 0
    BH = wl.B * wl.H
    hs = list(range(BH)) if heads is None else list(heads)
    qo, ko, vo = heads_view(q, hs), heads_view(k, hs), heads_view(v, hs)
    og = f32(out.reshape(BH, wl.N, wl.D))[hs]
    assert np.isfinite(og).all()
    if rows_per_head is None:
        rows = None
        got = og.reshape(-1, wl.D)
    else:
        rr = [sample_rows(wl.N, rows_per_head, seed=h) for h in range(len(hs))]
        rows = np.concatenate([np.stack([np.full(len(r), i), r], 1) for i, r in enumerate(rr)])
        got = og[rows[:, 0], rows[:, 1]]
    em, _ = oracle_mod.attention(qo, ko, vo, wl.causal, wl.sm_scale, Bk=128, rows=rows)
    em = em.reshape(-1, wl.D)
    ex = oracle_mod.attn_exact(qo, ko, vo, wl.causal, wl.sm_scale, rows=rows).reshape(-1, wl.D)
    m_em = oracle_mod.metrics(got, em)
    m_ex = oracle_mod.metrics(got, ex)
    vmax = float(np.abs(vo).max())
    print(f"\n{wl.name}: vs emulated {m_em}  vs exact {m_ex}  max|V| {vmax:.3f}")
    assert m_em["max_abs"] <= MAX_ABS_FRAC * vmax, m_em
    assert m_em["cos"] >= MIN_COS, m_em
    return m_em, m_ex


@pytest.mark.parametrize("wl", [
    workloads.TINY,
    workloads.custom(1, 2, 256, 64, causal=True, dtype=torch.float16, seed=31),
    workloads.custom(1, 2, 300, 128, seed=32),                     # ragged, several tiles
    workloads.custom(1, 2, 300, 128, causal=True, seed=33),
    workloads.custom(2, 1, 200, 64, causal=True, seed=34),
    workloads.custom(1, 1, 1, 128, seed=35),                       # a single token
    workloads.custom(1, 1, 130, 64, seed=36),
    workloads.custom(1, 2, 1024, 128, causal=True, seed=37, outliers=True),
], ids=lambda w: w.name)
def test_attn_small_all_rows(sage, oracle_mod, wl):
    _check(sage, oracle_mod, wl)


def test_attn_quantized_entry_matches(sage, oracle_mod):
    _check(sage, oracle_mod, workloads.custom(1, 2, 384, 128, causal=True, seed=38), entry="quantized")


def test_attn_library_workspace_entry(sage, oracle_mod):
    _check(sage, oracle_mod, workloads.custom(1, 2, 512, 128, seed=39), entry="library_ws")


def test_attn_medium_sampled(sage, oracle_mod):
    _check(sage, oracle_mod, workloads.MEDIUM, heads=[0, 7, 15], rows_per_head=256)


@pytest.mark.parametrize("wl", [workloads.LLM_CAUSAL, workloads.LONG], ids=lambda w: w.name)
def test_attn_full_size_sampled(sage, oracle_mod, wl):
    BH = wl.B * wl.H
    _check(sage, oracle_mod, wl, heads=[0, BH - 1], rows_per_head=48)


@pytest.mark.parametrize("wl", workloads.SWEEP, ids=lambda w: w.name)
def test_attn_sweep_sampled(sage, oracle_mod, wl):
    BH = wl.B * wl.H
    _check(sage, oracle_mod, wl, heads=[BH // 3], rows_per_head=24)


def test_empty_problem_is_a_noop(sage):
    q = torch.empty((0, 2, 128, 64), dtype=torch.bfloat16, device="cuda")
    out = sage.attn(q, q, q)
    assert out.shape == q.shape
    q = torch.empty((1, 2, 0, 128), dtype=torch.bfloat16, device="cuda")
    assert sage.attn(q, q, q).shape == q.shape


def test_argument_errors(sage):
    q = torch.randn((1, 1, 128, 96), device="cuda", dtype=torch.bfloat16)
    with pytest.raises(sage.SageError) as e:
        sage.attn(q, q, q)
    assert e.value.status == sage.SAGE_ERR_UNSUPPORTED
    base = torch.zeros(1 * 1 * 128 * 64 + 8, device="cuda", dtype=torch.bfloat16)
    mis = base[1:1 + 128 * 64].view(1, 1, 128, 64)  # 2-byte offset: not 16-byte aligned
    with pytest.raises(sage.SageError) as e:
        sage.attn(mis, mis, mis)
    assert e.value.status == sage.SAGE_ERR_INVALID_ARG


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_attn_alternating_tile_maxima(sage, oracle_mod, causal):
    """Key tiles whose score level alternates between far above and far below the others
    (plus a drift across tiles): consecutive key tiles go to different softmax warpgroups,
    so their lazy reference maxima differ by far more than the rescale threshold and the
    correction re-bases every tile's contribution and moves its own reference often."""
    B, H, N, D = 1, 2, 1280, 128
    g = torch.Generator(device="cpu")
    g.manual_seed(61)
    u = torch.randn(D, generator=g)
    u = u / u.norm()
    q = torch.randn((B, H, N, D), generator=g) * 0.5 + 3.0 * u
    k = torch.randn((B, H, N, D), generator=g) * 0.5
    v = torch.randn((B, H, N, D), generator=g)
    tiles = torch.arange(N) // 128
    level = torch.where(tiles % 2 == 0, 1.0, -1.0) * 20.0 + 2.5 * tiles.float()
    k = k + level[None, None, :, None] * u
    q, k, v = (t.to(torch.bfloat16).cuda() for t in (q, k, v))
    sm = 1.0 / np.sqrt(D)
    out = sage.attn(q, k, v, causal=causal, sm_scale=sm)
    torch.cuda.synchronize()
    assert sage.device_error() == 0
    hs = list(range(B * H))
    qo, ko, vo = heads_view(q, hs), heads_view(k, hs), heads_view(v, hs)
    got = f32(out.reshape(B * H, N, D)).reshape(-1, D)
    assert np.isfinite(got).all()
    em, _ = oracle_mod.attention(qo, ko, vo, causal, sm, Bk=128)
    m_em = oracle_mod.metrics(got, em.reshape(-1, D))
    vmax = float(np.abs(vo).max())
    print(f"\nalternating tile maxima ({'causal' if causal else 'full'}): vs emulated {m_em}")
    assert m_em["max_abs"] <= MAX_ABS_FRAC * vmax, m_em
    assert m_em["cos"] >= MIN_COS, m_em


def test_attn_short_dense_many_items_per_cta(sage, oracle_mod):
    """Square dense non-causal D = 128, short rows: 2 x 96 heads x 8 query tiles = 1536
    work items over one CTA per SM (about ten items each, consecutive items of a CTA in
    different heads), with a ragged last tile."""
    wl = workloads.custom(2, 96, 1000, 128, seed=62)
    _check(sage, oracle_mod, wl, heads=[0, 95, 191], rows_per_head=40)


@pytest.mark.parametrize("D", [128, 64])
def test_attn_causal_walk_partial_reversed_round(sage, oracle_mod, D):
    """Causal rows walk their work items heaviest first over all (sequence, head) pairs,
    odd rounds in reverse CTA order. 2 x 104 heads x 8 query tiles = 1664 items over the
    148 CTAs of a B200 is 11 full rounds and a partial 12th, which is an odd (reversed)
    round: it holds the lightest items, query tile 0 of pairs 172-207, taken by the last
    CTAs. Every row of the pairs on either side of that boundary is checked, and the last
    query tile (the ragged one) of the first pair."""
    wl = workloads.custom(2, 104, 1000, D, causal=True, seed=63)
    _check(sage, oracle_mod, wl, heads=[0, 171, 172, 207])
