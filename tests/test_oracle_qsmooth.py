"""Pins for smoothing Q (the SageAttention2 abstract's "smooth Q", read as the counterpart
of smoothing K): Q is quantized as q - mu_q, mu_q its per-(sequence, head) channel mean
over tokens, and mu_q . k' returns as a per-key score bias computed from the
unquantized smoothed keys k'.

  * decomposition: on inputs where q, q - mu_q and k are all exactly representable in
    the block format, both ways of forming S are exact, so smoothed and unsmoothed
    emulations agree to rounding; dropping the bias breaks the agreement;
  * the bias equals a float64 einsum of mu_q and fp32(k - mu_k); mu_q equals numpy's mean;
  * grouped heads with smoothing equal the problem with K/V heads repeated;
  * on queries with a large shared component, smoothing shrinks the error against exact
    attention.
"""
import numpy as np
import pytest


def _rand(shape, seed, scale=1.0, bias=0.0):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal(shape) * scale + bias).astype(np.float32)


def _exact_case():
    # 8 queries, 16 channels: each channel holds 1.5 in four rows and 3 in the other four
    # (mean 2.25, q - mean = -+0.75: every block scale and code exact before and after).
    rng = np.random.default_rng(3)
    q = np.empty((1, 8, 16), np.float32)
    for c in range(16):
        col = np.array([1.5] * 4 + [3.0] * 4, np.float32)
        q[0, :, c] = rng.permutation(col)
    # 16 keys in +- pairs (channel means exactly 0), values on the E2M1 grid x 0.5 with a
    # 3 (= 6 x 0.5) in every row so that each row's block scale is exactly 0.5.
    grid = np.array([0.0, 0.25, 0.5, 0.75, 1.0, 1.5, 2.0, 3.0], np.float32)
    half = grid[rng.integers(0, 8, (8, 16))] * np.where(rng.integers(0, 2, (8, 16)) > 0, 1, -1)
    half[:, 0] = 3.0
    k = np.concatenate([half, -half])[None].astype(np.float32)
    v = _rand((1, 16, 16), 4)
    return q, k, v


def test_smoothing_is_lossless_on_exact_inputs(oracle_mod):
    q, k, v = _exact_case()
    assert np.array_equal(oracle_mod.kmean(k), np.zeros((1, 16), np.float32))
    for causal in (False, True):
        plain, _ = oracle_mod.attention(q, k, v, causal, 0.125)
        smooth, qz = oracle_mod.attention(q, k, v, causal, 0.125, smooth_q=True)
        assert np.array_equal(qz["q_mean"], np.full((1, 16), 2.25, np.float32))
        assert np.max(np.abs(smooth - plain)) <= 1e-12
        # The bias carries real weight: without it the scores lose mu_q . k.
        qz["qk_bias"] = np.zeros_like(qz["qk_bias"])
        nobias = oracle_mod.attn_emulated(qz, causal, 0.125)
        assert np.max(np.abs(nobias - plain)) > 1e-2


def test_bias_and_mean_match_numpy(oracle_mod):
    q, k = _rand((2, 40, 32), 5, bias=1.0), _rand((2, 50, 32), 6, bias=-2.0)
    v = _rand((2, 50, 32), 7)
    qz = oracle_mod.quantize_qkv(q, k, v, smooth_q=True)
    mq = q.astype(np.float64).mean(axis=1).astype(np.float32)
    assert np.array_equal(qz["q_mean"], mq)
    kp = (k - qz["k_mean"][:, None, :]).astype(np.float32)
    want = np.einsum("hd,hjd->hj", mq.astype(np.float64), kp.astype(np.float64))
    assert np.max(np.abs(qz["qk_bias"] - want)) <= 1e-12 * np.max(np.abs(want))


@pytest.mark.parametrize("causal", [False, True])
def test_smoothing_with_grouped_heads(oracle_mod, causal):
    B, Hq, Hkv, N, D = 2, 4, 2, 70, 64
    q = _rand((B * Hq, N, D), 8, bias=2.0)
    k, v = _rand((B * Hkv, N, D), 9, bias=0.5), _rand((B * Hkv, N, D), 10)
    got, _ = oracle_mod.attention(q, k, v, causal, 0.125, heads=(B, Hq, Hkv), smooth_q=True)
    rep = lambda t: np.repeat(t.reshape(B, Hkv, N, D), Hq // Hkv, axis=1).reshape(B * Hq, N, D)  # noqa: E731
    want, _ = oracle_mod.attention(q, rep(k), rep(v), causal, 0.125, smooth_q=True)
    assert np.array_equal(got, want)


def test_smoothing_reduces_error_on_shifted_queries(oracle_mod):
    # A large channel offset shared by all queries dominates Q's block scales; removing
    # it leaves the varying part to the FP4 grid and adds the offset back exactly.
    q = _rand((2, 128, 64), 11) + _rand((2, 1, 64), 12, scale=8.0)
    k, v = _rand((2, 128, 64), 13, bias=0.3), _rand((2, 128, 64), 14)
    ex = oracle_mod.attn_exact(q, k, v, False, 0.125)
    plain, _ = oracle_mod.attention(q, k, v, False, 0.125)
    smooth, _ = oracle_mod.attention(q, k, v, False, 0.125, smooth_q=True)
    e_plain = oracle_mod.metrics(plain, ex)["rel_l1"]
    e_smooth = oracle_mod.metrics(smooth, ex)["rel_l1"]
    assert e_smooth < 0.7 * e_plain, (e_smooth, e_plain)
