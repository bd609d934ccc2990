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
