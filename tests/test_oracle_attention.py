"""Pins for the oracle's attention, K mean and quantize/layout functions.

What each test holds the oracle to (never the oracle's own formula retyped):
  * the online-softmax recurrence equals two-pass softmax (the reply to Q3 of the
    SageAttention review thread: "ensure equivalent computation");
  * exact attention equals torch's scaled_dot_product_attention in float64;
  * softmax shift invariance behind smoothing K (reply to W1: smoothing K);
  * identical keys give the mean of V; causal row 0 gives v_0; one key gives v^_0;
  * hand-derived closed forms of the two-level P~ quantization (per-row factor, then
    per-16 E4M3 scales) and of the cross-tile recurrence;
  * the K mean equals numpy's float64 mean rounded to float32.
"""
import math

import numpy as np
import pytest
import torch

from microscaling_fp4_quantized_b200 import workloads


def _rand(shape, seed, bias=0.0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(shape).astype(np.float32)
    return x + np.float32(bias)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,Bk", [(37, 16), (128, 128), (300, 128), (64, 32)])
def test_online_equals_two_pass(oracle_mod, causal, N, Bk):
    BH, D = 2, 32
    q, k, v = _rand((BH, N, D), 1), _rand((BH, N, D), 2), _rand((BH, N, D), 3)
    a = oracle_mod.attn_online(q, k, v, causal, 0.3, Bk=Bk)
    b = oracle_mod.attn_exact(q, k, v, causal, 0.3)
    assert np.max(np.abs(a - b)) <= 1e-12 * max(1.0, np.max(np.abs(b)))


@pytest.mark.parametrize("causal", [False, True])
def test_exact_matches_torch_sdpa(oracle_mod, causal):
    BH, N, D = 3, 70, 64
    q, k, v = _rand((BH, N, D), 4), _rand((BH, N, D), 5), _rand((BH, N, D), 6)
    got = oracle_mod.attn_exact(q, k, v, causal, 1 / 8.0)
    t = [torch.from_numpy(a).double()[None] for a in (q, k, v)]
    want = torch.nn.functional.scaled_dot_product_attention(*t, is_causal=causal, scale=1 / 8.0)[0].numpy()
    assert np.max(np.abs(got - want)) <= 1e-12


def test_kmean_matches_numpy(oracle_mod):
    k = _rand((3, 257, 64), 7, bias=1.5)
    got = oracle_mod.kmean(k)
    want = k.astype(np.float64).mean(axis=1).astype(np.float32)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("causal", [False, True])
def test_smoothing_k_is_softmax_invariant(oracle_mod, causal):
    # Subtracting a per-channel constant c from every key changes each score of a row by
    # the same q.c, which softmax cancels. Keys on a 2^-10 grid with |k| < 16 make k - c
    # exact in binary32 for c on the same grid, so the two outputs agree to rounding.
    BH, N, D = 2, 96, 64
    q, v = _rand((BH, N, D), 8), _rand((BH, N, D), 10)
    k = np.round(np.clip(_rand((BH, N, D), 9, bias=3.0), -15, 15) * 1024) / 1024
    c = np.round(_rand((BH, 1, D), 17) * 1024) / 1024
    a = oracle_mod.attn_exact(q, k.astype(np.float32), v, causal, 0.125)
    b = oracle_mod.attn_exact(q, (k - c).astype(np.float32), v, causal, 0.125)
    assert np.array_equal((k - c).astype(np.float32).astype(np.float64), k - c)
    assert np.max(np.abs(a - b)) <= 1e-12


def test_identical_keys_give_mean_of_v(oracle_mod):
    BH, N, D = 1, 48, 32
    q, v = _rand((BH, N, D), 11), _rand((BH, N, D), 12)
    k = np.repeat(_rand((BH, 1, D), 13), N, axis=1)
    ex = oracle_mod.attn_exact(q, k, v, False, 0.2)
    assert np.max(np.abs(ex - v.astype(np.float64).mean(axis=1, keepdims=True))) <= 1e-12
    # Emulated path: after smoothing every K' row is 0, so S = 0, P~ = 1, s1 = 1/2688,
    # P2 = 2688 -> scale 448, code 7 -> p^ = 2688 exactly; O = mean of the dequantized V^.
    out, qz = oracle_mod.attention(q, k, v, causal=False, sm_scale=0.2)
    vt = oracle_mod.unpack_fp4(qz["vt_codes"])[:, :, :N]
    vdeq = oracle_mod.e2m1_decode(vt) * np.repeat(oracle_mod.e4m3_decode(qz["vt_sf"]), 16, axis=2)[:, :, :N]
    want = vdeq.mean(axis=2)  # [BH, D]
    assert np.max(np.abs(out - want[:, None, :])) <= 1e-12


def test_causal_row0_is_v0(oracle_mod):
    BH, N, D = 2, 40, 32
    q, k, v = _rand((BH, N, D), 14), _rand((BH, N, D), 15), _rand((BH, N, D), 16)
    ex = oracle_mod.attn_exact(q, k, v, True, 0.2)
    assert np.array_equal(ex[:, 0, :], v[:, 0, :].astype(np.float64))


def _two_level_case(oracle_mod, key_scales, v_rows, Bk):
    """q = [6, 0...] (FP4-exact), key j = [-6 * key_scales[j], 0...] (FP4-exact: scale
    key_scales[j], code -6), sm_scale = ln2/12 so S_j = -3*ln2*key_scales[j]."""
    D = 16
    N = len(key_scales)
    q = np.zeros((1, N, D), np.float32)
    q[0, :, 0] = 6.0
    k = np.zeros((1, N, D), np.float32)
    k[0, :, 0] = -6.0 * np.asarray(key_scales, np.float32)
    v = np.asarray(v_rows, np.float32).reshape(1, N, D)
    qz = oracle_mod.quantize_qkv(q, k, v, smooth_k=False)
    return oracle_mod.attn_emulated(qz, False, math.log(2) / 12, Bk=Bk, rows=[(0, 0)])[0]


def _exact_v(seed, N, D=16):
    # V columns whose 16-token blocks are FP4-exact (values e2m1 * 1 with a 6 present);
    # returned as float64 (every value is exact in binary32 too).
    rng = np.random.default_rng(seed)
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float32)
    v = mags[rng.integers(0, 8, (N, D))] * np.where(rng.integers(0, 2, (N, D)) > 0, 1, -1)
    for b0 in range(0, N, 16):
        v[b0, :] = 6.0
    return v.astype(np.float64)


def test_two_level_p_quantization_closed_form(oracle_mod):
    # Keys: k0 = 0 (S=0, P~=1), k1 with S = -3 ln2 (P~ = 1/8). Row factor s1 = 1/2688,
    # P2 = [2688, 336]; block scale = 2688/6 = 448 (E4M3 exact); 336/448 = 0.75 is a
    # tie between E2M1 0.5 and 1.0 -> 1.0, so p^_1 = 448 = 2688/6. The sum l uses the
    # unquantized P~: l = 1 + 1/8. Hence O = (v0 + v1/6) / (9/8).
    v = _exact_v(20, 2)
    out = _two_level_case(oracle_mod, [0.0, 1.0], v, Bk=16)
    want = (v[0].astype(np.float64) + v[1] / 6.0) / (9.0 / 8.0)
    assert np.max(np.abs(out - want)) <= 1e-12


def test_two_level_lossless_when_representable(oracle_mod):
    # S = [0, -ln2 * 3 * 1/3 ...]: use key scale 1/3? Not E4M3-exact; instead S1 = -3 ln2 * 0.5
    # is not a power of two. Keys with S = 0 and S = -3*ln2*(1/3) are avoided; use the
    # representable P2 = 2688 * 2^-1 via key scale... here with two keys at S=0 and one at
    # S = -3 ln2 * 2 (P~ = 1/64): P2 = 42 -> 42/448 = 0.09375 -> below 0.25 -> code 0.
    v = _exact_v(21, 3)
    out = _two_level_case(oracle_mod, [0.0, 0.0, 2.0], v, Bk=16)
    want = (v[0].astype(np.float64) + v[1] + 0.0 * v[2]) / (2.0 + 1.0 / 64.0)
    assert np.max(np.abs(out - want)) <= 1e-12


def test_cross_tile_recurrence_closed_form(oracle_mod):
    # Tile 0 (16 keys): S = -3 ln2 (P~ relative to the running max), tile 1 (16 keys): S = 0.
    # Tile 0 alone: m = -3ln2, P~ = 1, l = 16, O = sum v (p^ exact: 2688 -> code 7, s 448).
    # Tile 1: m' = 0, alpha = 1/8, l = 16/8 + 16 = 18, O = O/8 + sum v(tile 1).
    # Within each tile every P2 = 2688, so quantization is exact.
    v = _exact_v(22, 32)
    ks = [1.0] * 16 + [0.0] * 16
    out = _two_level_case(oracle_mod, ks, v, Bk=16)
    want = (v[:16].astype(np.float64).sum(0) / 8 + v[16:].sum(0)) / 18.0
    assert np.max(np.abs(out - want)) <= 1e-12
    # Reverse order: tile 1 has the lower max; its row factor r = 1/8 maps its P2 back
    # to 2688, still exact: O = (sum v(t0) + sum v(t1)/8) / (16 + 2).
    out = _two_level_case(oracle_mod, ks[16:] + ks[:16], np.concatenate([v[16:], v[:16]]), Bk=16)
    want = (v[16:].astype(np.float64).sum(0) + v[:16].sum(0) / 8) / 18.0
    assert np.max(np.abs(out - want)) <= 1e-12


def test_mixed_tile_rounds_to_nearest_code(oracle_mod):
    # One tile, keys S = [-3ln2, -6ln2 x 15]: m = -3ln2, r = 1, P2 = [2688, 336 x 15];
    # block scale 448; 336/448 = 0.75 -> 1.0: weights [1, 1/6 x 15] times s1 = 1/2688 * 2688
    # -> O = (v0 + sum_{j>0} v_j / 6) / (1 + 15/8).
    v = _exact_v(23, 16)
    out = _two_level_case(oracle_mod, [1.0] + [2.0] * 15, v, Bk=16)
    want = (v[0].astype(np.float64) + v[1:].sum(0) / 6.0) / (1.0 + 15.0 / 8.0)
    assert np.max(np.abs(out - want)) <= 1e-12


def test_single_key_returns_dequantized_v(oracle_mod):
    q, k, v = _rand((1, 1, 64), 30), _rand((1, 1, 64), 31), _rand((1, 1, 64), 32)
    out, qz = oracle_mod.attention(q, k, v, causal=True, sm_scale=0.125)
    vdeq = oracle_mod.e2m1_decode(oracle_mod.unpack_fp4(qz["vt_codes"])[0, :, 0]) * oracle_mod.e4m3_decode(qz["vt_sf"][0, :, 0])
    assert np.max(np.abs(out[0, 0] - vdeq)) <= 1e-12


def test_quantize_layouts_match_block_rule(oracle_mod):
    BH, N, D = 2, 40, 64  # ragged: N not a multiple of 16
    q, k, v = _rand((BH, N, D), 40), _rand((BH, N, D), 41, bias=2.0), _rand((BH, N, D), 42)
    qz = oracle_mod.quantize_qkv(q, k, v)
    c, s = oracle_mod.quant_block16(q.reshape(BH, N, D // 16, 16))
    assert np.array_equal(oracle_mod.unpack_fp4(qz["q_codes"]), c.reshape(BH, N, D))
    assert np.array_equal(qz["q_sf"], s)
    kp = k - oracle_mod.kmean(k)[:, None, :]
    c, s = oracle_mod.quant_block16(kp.reshape(BH, N, D // 16, 16))
    assert np.array_equal(oracle_mod.unpack_fp4(qz["k_codes"]), c.reshape(BH, N, D))
    assert np.array_equal(qz["k_sf"], s)
    Np = 48
    vt = np.zeros((BH, D, Np), np.float32)
    vt[:, :, :N] = v.transpose(0, 2, 1)
    c, s = oracle_mod.quant_block16(vt.reshape(BH, D, Np // 16, 16))
    assert np.array_equal(oracle_mod.unpack_fp4(qz["vt_codes"]), c.reshape(BH, D, Np))
    assert np.array_equal(qz["vt_sf"], s)


def test_emulated_close_to_exact_on_tiny_workload(oracle_mod):
    # Not a pin (the pages print no FP4 accuracy figure): a sanity bound only.
    w = workloads.TINY
    q, k, v = [t.float().reshape(w.B * w.H, w.N, w.D).numpy() for t in workloads.make_inputs(w)]
    em, _ = oracle_mod.attention(q, k, v, w.causal, w.sm_scale)
    ex = oracle_mod.attn_exact(q, k, v, w.causal, w.sm_scale)
    m = oracle_mod.metrics(em, ex)
    # Random Gaussian inputs give near-uniform attention whose output is a heavily
    # cancelling average, so FP4 error is large relative to |O|: Q,K,V quantization
    # alone measures cos ~0.985 here. 0.97 only guards against gross breakage.
    assert m["cos"] > 0.97, m


@pytest.mark.parametrize("causal,Nq,Nk,gscale", [(False, 130, 300, "none"), (True, 300, 300, "head"),
                                                  (True, 100, 260, "none"), (True, 260, 100, "tensor")])
def test_attn_from_scores_equals_emulation(oracle_mod, causal, Nq, Nk, gscale):
    # The emulation's tile walk applied to given scores: fed the emulation's own scores
    # (formed here in numpy from the dequantized codes; products of E2M1 codes and E4M3
    # scales are exact in binary64, and so are their sums at these sizes), it must give
    # the emulated rows bit for bit, for grouped heads and masks. With a second-level
    # scale the products carry a 24-bit factor and are rounded in another order, so the
    # rows agree to binary64 rounding instead.
    Hq, Hkv, D, sm = 4, 2, 64, 0.125
    rng = np.random.default_rng(Nq + Nk)
    q = rng.standard_normal((Hq, Nq, D)).astype(np.float32)
    k = (rng.standard_normal((Hkv, Nk, D)) + 1.5).astype(np.float32)
    v = rng.standard_normal((Hkv, Nk, D)).astype(np.float32)
    em, qz = oracle_mod.attention(q, k, v, causal, sm, gscale=gscale, heads=(1, Hq, Hkv))
    dec = lambda c, s: oracle_mod.e2m1_decode(oracle_mod.unpack_fp4(c)) * np.repeat(oracle_mod.e4m3_decode(s), 16, -1)  # noqa: E731
    qd, kd = dec(qz["q_codes"], qz["q_sf"]), dec(qz["k_codes"], qz["k_sf"])
    gq = np.ones(Hq) if qz["gq"] is None else qz["gq"].astype(np.float64)
    gk = np.ones(Hkv) if qz["gk"] is None else qz["gk"].astype(np.float64)
    for h in range(Hq):
        hk = h // (Hq // Hkv)
        S = sm * np.einsum("id,jd->ij", qd[h] * gq[h], kd[hk] * gk[hk])
        n_keys = [min(i + Nk - Nq, Nk - 1) + 1 if causal else Nk for i in range(Nq)]
        n_keys = [max(n, 0) for n in n_keys]
        got = oracle_mod.attn_from_scores(S, [hk] * Nq, n_keys, qz)
        if gscale == "none":
            assert np.array_equal(got, em[h]), h
        else:
            assert np.abs(got - em[h]).max() <= 1e-12 * np.abs(v).max(), h
