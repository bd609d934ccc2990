"""GPU parity of the 8-bit path (INT8 Q/K per 128-token tile, E4M3 V per channel, E4M3 P~
with s1 = rowmax / 448): quantization bit for bit against the oracle (K mean within 1 ulp,
fed to the oracle), attention within the FP4 path's bar against the oracle's 8-bit
emulation, and the accuracy the 8 bits buy over FP4 on the same inputs."""
import numpy as np
import pytest
import torch

from gpu_helpers import canonical8, f32
from microscaling_fp4_quantized_b200 import workloads as W
from test_gpu_general import _out_per_seq, _per_seq

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


def _problem(sage, w, x, out):
    if w.packed:
        return sage.sageattn_varlen_problem(x["q"], x["k"], x["v"], out, x["cu_seqlens_q"], x["cu_seqlens_k"],
                                            max(w.lens_q), max(w.lens_k), w.causal, None, True, "none", False,
                                            "8bit")
    return sage.sageattn_problem(x["q"], x["k"], x["v"], out, w.layout, w.causal, None, True, "none", False, "8bit")


def _run(sage, w, x, precision="8bit"):
    if w.packed:
        return sage.sageattn_varlen(x["q"], x["k"], x["v"], x["cu_seqlens_q"], x["cu_seqlens_k"], max(w.lens_q),
                                    max(w.lens_k), is_causal=w.causal, precision=precision)
    return sage.sageattn(x["q"], x["k"], x["v"], tensor_layout=w.layout, is_causal=w.causal, precision=precision)


CASES = [
    W.general("i8_gqa_dense_causal", 4, 2, 128, (300, 300), causal=True, packed=False, seed=81, precision="8bit"),
    W.general("i8_nhd_fp16_d64", 3, 3, 64, (333, 333), packed=False, layout="NHD", dtype=torch.float16, seed=82,
              precision="8bit"),
    W.general("i8_packed_gqa", 4, 2, 64, (5, 0, 300, 128, 1, 1000), causal=True, seed=83, precision="8bit"),
    W.general("i8_packed_cross", 2, 1, 128, (100, 37, 513, 0), (300, 37, 129, 50), causal=True, seed=84,
              precision="8bit"),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_8bit_quant_bit_exact(sage, oracle_mod, w):
    x = W.make_general_inputs(w, "cuda")
    out = torch.empty(x["q"].shape, dtype=x["q"].dtype, device="cuda")
    qz = sage.quantize(_problem(sage, w, x, out), x["q"], x["k"], x["v"])
    torch.cuda.synchronize()
    assert sage.device_error() == 0
    can = canonical8(qz, w.lens_q, w.lens_k, w.Hq, w.Hkv, w.D)
    for b, ((qs, ks, vs), c) in enumerate(zip(_per_seq(w, x), can)):
        assert c["pads_zero"], f"sequence {b}: padding not zero"
        if ks.shape[1]:
            km = oracle_mod.kmean(ks)
            ulp = np.abs(c["k_mean"].view(np.int32).astype(np.int64) - km.view(np.int32).astype(np.int64))
            assert ulp.max() <= 1
        o = oracle_mod.quantize8(qs, ks, vs, smooth_k=True, kmean_in=c["k_mean"], heads=(1, w.Hq, w.Hkv))
        for name in ("q8", "q_scale", "k8", "k_scale", "vt8", "v_scale"):
            got, want = c[name], o[name]
            if want.size == 0 and got.size == 0:
                continue
            assert got.shape == want.shape, (name, got.shape, want.shape)
            bad = np.argwhere(got != want)
            assert bad.size == 0, f"sequence {b} {name}: {len(bad)} mismatches, first {bad[:4].tolist()}"


def _check_attention8(sage, oracle_mod, w, rows_per_seq=None):
    x = W.make_general_inputs(w, "cuda")
    out = _run(sage, w, x)
    torch.cuda.synchronize()
    assert sage.device_error() == 0
    got_all = _out_per_seq(w, x, out)
    qz = sage.quantize(_problem(sage, w, x, torch.empty_like(out)), x["q"], x["k"], x["v"])
    torch.cuda.synchronize()
    can = canonical8(qz, w.lens_q, w.lens_k, w.Hq, w.Hkv, w.D)
    worst = None
    for b, ((qs, ks, vs), got) in enumerate(zip(_per_seq(w, x), got_all)):
        Lq = qs.shape[1]
        if Lq == 0:
            continue
        assert np.isfinite(got).all()
        if ks.shape[1] == 0:
            assert not got.any()
            continue
        rows = None
        if rows_per_seq is not None:
            rng = np.random.default_rng(b)
            rr = np.unique(np.concatenate([[0, Lq - 1], rng.choice(Lq, min(Lq, rows_per_seq), replace=False)]))
            rows = np.array([(h, i) for h in sorted({0, w.Hq - 1}) for i in rr], np.int64)
        em, _ = oracle_mod.attention8(qs, ks, vs, w.causal, w.sm_scale, rows=rows, kmean_in=can[b]["k_mean"],
                                      heads=(1, w.Hq, w.Hkv))
        g = got.reshape(-1, w.D) if rows is None else got[rows[:, 0], rows[:, 1]]
        e = em.reshape(-1, w.D)
        m = oracle_mod.metrics(g, e)
        assert m["cos"] >= MIN_COS, (b, m)
        # Every row within the max-abs bar: the 8-bit scores are exact integers, so no
        # score rounding can move a P~ code here.
        assert m["max_abs"] <= MAX_ABS_FRAC * float(np.abs(vs).max()), (b, m)
        worst = m if worst is None or m["cos"] < worst["cos"] else worst
    print(f"\n{w.name}: worst sequence vs 8-bit emulation {worst}")


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_8bit_attention(sage, oracle_mod, w):
    _check_attention8(sage, oracle_mod, w)


def test_8bit_full_size_sampled(sage, oracle_mod):
    w = W.general("i8_video_long", 24, 24, 128, (32768,), packed=False, seed=3, bias_sigma=4.0, precision="8bit")
    _check_attention8(sage, oracle_mod, w, rows_per_seq=32)


def test_8bit_is_closer_to_exact_than_fp4(sage, oracle_mod):
    w = W.general("i8_vs_fp4", 4, 4, 128, (1024,), packed=False, seed=85)
    x = W.make_general_inputs(w, "cuda")
    (qs, ks, vs), = _per_seq(w, x)
    ex = oracle_mod.attn_exact(qs, ks, vs, False, w.sm_scale)
    err = {}
    for prec in ("fp4", "8bit"):
        got = _out_per_seq(w, x, _run(sage, w, x, precision=prec))[0]
        torch.cuda.synchronize()
        err[prec] = oracle_mod.metrics(got, ex)["rel_l1"]
    print(f"\nrelative L1 vs exact attention: {err}")
    assert err["8bit"] < 0.5 * err["fp4"], err
