"""Pins for the oracle's general problem: second-level (per-tensor / per-head) scales,
grouped key/value heads, different query and key lengths with the causal mask aligned
to the last key, and packed variable-length sequences.

Each pin holds the oracle to something other than itself:
  * closed forms of the second-level scale (a group maximum of 2688 * 2^k gives the
    scale 2^k exactly, the block holding the maximum gets scale byte 448 and code 6);
  * powers of two commute with the block rule, so the two-level path on x equals the
    one-level path on x / 2^k, and the two-level codes do not change when x is scaled;
  * saturation: a block maximum above 2688 is clipped by the one-level rule and kept by
    the two-level rule;
  * grouped heads equal the same problem with key/value heads repeated (and torch's
    float64 scaled_dot_product_attention on the repeated heads);
  * the causal mask for Nq < Nk equals the last Nq rows of the square problem, and
    matches torch with an explicit mask; rows that see no key are 0;
  * packed sequences equal torch on each sequence.
"""
import math

import numpy as np
import pytest
import torch


def _rand(shape, seed, scale=1.0, bias=0.0):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal(shape) * scale + bias).astype(np.float32)


# ------------------------------------------------------------ second-level scale --

def test_second_level_scale_closed_forms(oracle_mod):
    amax = np.array([2688.0, 2688.0 * 8, 2688.0 / 32, 0.0, 2688.0 * 3], np.float32)
    g = oracle_mod.second_level_scale(amax)
    assert g.tolist() == [1.0, 8.0, 1.0 / 32, 1.0, 3.0]


def test_group_amax_matches_numpy(oracle_mod):
    x = _rand((3, 50, 32), 1, bias=2.0)
    mu = _rand((3, 32), 2)
    want = np.abs(x - mu[:, None, :]).max(axis=(1, 2))
    assert np.array_equal(oracle_mod.group_amax(x, mu), want)
    assert np.array_equal(oracle_mod.group_amax(x), np.abs(x).max(axis=(1, 2)))


@pytest.mark.parametrize("k", [3, -5])
def test_power_of_two_scale_equals_prescaled_one_level(oracle_mod, k):
    # Plant the group maximum 2688 * 2^k so that the second-level scale is exactly 2^k;
    # dividing by it is exact, so the codes must be those of the one-level rule on x/2^k.
    x = _rand((2, 40, 64), 30 + k, scale=2.0 ** k)
    x[0, 7, 5] = 2688.0 * 2.0 ** k
    x[1, 0, 63] = -2688.0 * 2.0 ** k
    g = oracle_mod.second_level_scale(oracle_mod.group_amax(x))
    assert g.tolist() == [2.0 ** k, 2.0 ** k]
    c2, s2 = oracle_mod.quantize_rows(x, None, g)
    c1, s1 = oracle_mod.quantize_rows(np.ldexp(x, -k).astype(np.float32))
    assert np.array_equal(c2, c1) and np.array_equal(s2, s1)
    # The block with the maximum: scale byte 0x7E (448), element code 7 (6) with its sign.
    assert s2[0, 7, 0] == 0x7E and oracle_mod.unpack_fp4(c2)[0, 7, 5] == 0x7
    assert s2[1, 0, 3] == 0x7E and oracle_mod.unpack_fp4(c2)[1, 0, 63] == 0xF
    vc2, vs2 = oracle_mod.quantize_vt(x, g)
    vc1, vs1 = oracle_mod.quantize_vt(np.ldexp(x, -k).astype(np.float32))
    assert np.array_equal(vc2, vc1) and np.array_equal(vs2, vs1)


def test_two_level_codes_are_scale_equivariant(oracle_mod):
    x = _rand((2, 48, 64), 7)
    base = oracle_mod.quantize_qkv(x, x, x, gscale="head")
    for k in (-6, 9):
        xs = np.ldexp(x, k).astype(np.float32)
        got = oracle_mod.quantize_qkv(xs, xs, xs, gscale="head")
        for n in ("q_codes", "q_sf", "k_codes", "k_sf", "vt_codes", "vt_sf"):
            assert np.array_equal(got[n], base[n]), n
        assert np.array_equal(got["gq"], np.ldexp(base["gq"], k))


def test_two_level_keeps_values_above_2688(oracle_mod):
    x = np.zeros((1, 1, 16), np.float32)
    x[0, 0, 0] = 10000.0
    c1, s1 = oracle_mod.quantize_rows(x)
    one = oracle_mod.e2m1_decode(oracle_mod.unpack_fp4(c1))[0, 0, 0] * oracle_mod.e4m3_decode(s1)[0, 0, 0]
    assert one == 2688.0  # clipped: scale 448, code 6
    g = oracle_mod.second_level_scale(oracle_mod.group_amax(x))
    c2, s2 = oracle_mod.quantize_rows(x, None, g)
    two = oracle_mod.e2m1_decode(oracle_mod.unpack_fp4(c2))[0, 0, 0] * oracle_mod.e4m3_decode(s2)[0, 0, 0] * float(g[0])
    assert abs(two - 10000.0) <= 1e-3


def test_tensor_mode_uses_the_largest_head(oracle_mod):
    q = _rand((3, 32, 64), 8)
    q[1] *= 50
    qz = oracle_mod.quantize_qkv(q, q, q, gscale="tensor", smooth_k=False)
    want = np.float32(np.abs(q).max()) / np.float32(2688.0)
    assert np.all(qz["gq"] == want) and np.all(qz["gv"] == want)
    qh = oracle_mod.quantize_qkv(q, q, q, gscale="head", smooth_k=False)
    assert qh["gq"][1] == want and qh["gq"][0] < want


def test_attention_with_power_of_two_scales(oracle_mod):
    # q~ = code * s * g: with g = 2^a, 2^b, 2^c the emulated output on (q, k, v) equals
    # 2^c times the output without second-level scales on (q/2^a, k/2^b, v/2^c) with
    # sm_scale * 2^(a+b). (K unsmoothed here so that its maximum can be planted; the
    # smoothed path's scaling is pinned by the equivariance test above.)
    a, b, c = 2, -3, 4
    q, k, v = _rand((2, 70, 64), 9), _rand((2, 70, 64), 10, scale=0.01), _rand((2, 70, 64), 11)
    q[:, 3, 1] = 2688.0 * 2.0 ** a
    k[:, 9, 4] = -2688.0 * 2.0 ** b
    v[:, 5, 2] = 2688.0 * 2.0 ** c
    qz = oracle_mod.quantize_qkv(q, k, v, gscale="head", smooth_k=False)
    assert qz["gq"].tolist() == [2.0 ** a] * 2 and qz["gk"].tolist() == [2.0 ** b] * 2
    assert qz["gv"].tolist() == [2.0 ** c] * 2
    for causal in (False, True):
        got = oracle_mod.attn_emulated(qz, causal, 0.125)
        ref, _ = oracle_mod.attention(np.ldexp(q, -a), np.ldexp(k, -b), np.ldexp(v, -c), causal,
                                      0.125 * 2.0 ** (a + b), smooth_k=False)
        assert np.max(np.abs(got - ref * 2.0 ** c)) <= 1e-12 * np.max(np.abs(got))


# ------------------------------------------------------------------ grouped heads --

@pytest.mark.parametrize("gscale", ["none", "head"])
@pytest.mark.parametrize("causal", [False, True])
def test_grouped_heads_equal_repeated_heads(oracle_mod, causal, gscale):
    B, Hq, Hkv, N, D = 2, 4, 2, 90, 64
    q = _rand((B * Hq, N, D), 12)
    k, v = _rand((B * Hkv, N, D), 13, bias=0.5), _rand((B * Hkv, N, D), 14)
    got, _ = oracle_mod.attention(q, k, v, causal, 0.125, heads=(B, Hq, Hkv), gscale=gscale)
    rep = lambda t: np.repeat(t.reshape(B, Hkv, N, D), Hq // Hkv, axis=1).reshape(B * Hq, N, D)  # noqa: E731
    want, _ = oracle_mod.attention(q, rep(k), rep(v), causal, 0.125, gscale=gscale)
    assert np.array_equal(got, want)


def test_grouped_heads_exact_matches_torch(oracle_mod):
    B, Hq, Hkv, Nq, Nk, D = 2, 6, 2, 33, 51, 32
    q = _rand((B * Hq, Nq, D), 15)
    k, v = _rand((B * Hkv, Nk, D), 16), _rand((B * Hkv, Nk, D), 17)
    got = oracle_mod.attn_exact(q, k, v, False, 0.2, heads=(B, Hq, Hkv))
    tq = torch.from_numpy(q).double().reshape(B, Hq, Nq, D)
    tk = torch.from_numpy(k).double().reshape(B, Hkv, Nk, D).repeat_interleave(Hq // Hkv, dim=1)
    tv = torch.from_numpy(v).double().reshape(B, Hkv, Nk, D).repeat_interleave(Hq // Hkv, dim=1)
    want = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=0.2)
    assert np.max(np.abs(got - want.reshape(B * Hq, Nq, D).numpy())) <= 1e-12


# ------------------------------------------------------- different lengths, causal --

@pytest.mark.parametrize("Nq", [1, 37, 130])
def test_causal_last_rows_equal_square_problem(oracle_mod, Nq):
    # Causal with the mask aligned to the last key: the Nq queries are the last Nq
    # positions of an Nk x Nk causal problem; Q rows are quantized independently, so the
    # emulated outputs agree bit for bit.
    Nk, D = 300, 64
    qf = _rand((2, Nk, D), 18)
    k, v = _rand((2, Nk, D), 19, bias=1.0), _rand((2, Nk, D), 20)
    full, _ = oracle_mod.attention(qf, k, v, True, 0.125)
    part, _ = oracle_mod.attention(qf[:, Nk - Nq:], k, v, True, 0.125)
    assert np.array_equal(part, full[:, Nk - Nq:])


@pytest.mark.parametrize("Nq,Nk", [(20, 45), (45, 20)])
def test_causal_different_lengths_match_torch_mask(oracle_mod, Nq, Nk):
    D = 32
    q, k, v = _rand((2, Nq, D), 21), _rand((2, Nk, D), 22), _rand((2, Nk, D), 23)
    got = oracle_mod.attn_exact(q, k, v, True, 0.3)
    i = np.arange(Nq)[:, None]
    j = np.arange(Nk)[None, :]
    mask = torch.from_numpy(j <= i + (Nk - Nq))
    t = [torch.from_numpy(a).double() for a in (q, k, v)]
    want = torch.nn.functional.scaled_dot_product_attention(*t, attn_mask=mask, scale=0.3).numpy()
    seen = (Nk - Nq) + np.arange(Nq) >= 0
    assert np.max(np.abs(got[:, seen] - want[:, seen])) <= 1e-12
    assert not got[:, ~seen].any()
    em, _ = oracle_mod.attention(q, k, v, True, 0.3)
    assert not em[:, ~seen].any() and np.isfinite(em).all()


# ----------------------------------------------------------- packed sequences --

def test_varlen_exact_matches_torch_per_sequence(oracle_mod):
    Hq, Hkv, D = 4, 2, 32
    lq, lk = [5, 0, 70, 33], [9, 4, 70, 1]
    cu_q, cu_k = np.concatenate([[0], np.cumsum(lq)]), np.concatenate([[0], np.cumsum(lk)])
    q = _rand((cu_q[-1], Hq, D), 24)
    k, v = _rand((cu_k[-1], Hkv, D), 25), _rand((cu_k[-1], Hkv, D), 26)
    for causal in (False, True):
        got = oracle_mod.attn_exact_varlen(q, k, v, cu_q, cu_k, causal, 0.25)
        for b in range(len(lq)):
            if lq[b] == 0:
                continue
            tq = torch.from_numpy(q[cu_q[b]:cu_q[b + 1]]).double().permute(1, 0, 2)
            tk = torch.from_numpy(k[cu_k[b]:cu_k[b + 1]]).double().permute(1, 0, 2).repeat_interleave(2, 0)
            tv = torch.from_numpy(v[cu_k[b]:cu_k[b + 1]]).double().permute(1, 0, 2).repeat_interleave(2, 0)
            i = np.arange(lq[b])[:, None]
            j = np.arange(lk[b])[None, :]
            mask = torch.from_numpy((j <= i + lk[b] - lq[b]) if causal else np.ones((lq[b], lk[b]), bool))
            want = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=0.25)
            want = want.permute(1, 0, 2).numpy()
            seen = (lk[b] - lq[b] + np.arange(lq[b]) >= 0) if causal else np.ones(lq[b], bool)
            seg = got[cu_q[b]:cu_q[b + 1]]
            assert np.max(np.abs(seg[seen] - want[seen]), initial=0.0) <= 1e-12
            assert not seg[~seen].any()


def test_varlen_tensor_scale_spans_all_sequences(oracle_mod):
    Hq, D = 2, 64
    lq = [40, 17]
    cu = np.concatenate([[0], np.cumsum(lq)])
    q = _rand((cu[-1], Hq, D), 27)
    q[cu[1] + 3, 1, 7] = 900.0
    out, qzs = oracle_mod.attention_varlen(q, q, q, cu, cu, False, 0.125, gscale="tensor", smooth_k=False)
    want = np.float32(900.0) / np.float32(2688.0)
    assert all(np.all(z["gq"] == want) for z in qzs)
    # sampled rows equal the full result
    rows = np.array([[0, 0], [cu[1] + 3, 1], [cu[2] - 1, 0]])
    part, _ = oracle_mod.attention_varlen(q, q, q, cu, cu, False, 0.125, gscale="tensor",
                                          smooth_k=False, rows=rows)
    assert np.array_equal(part, out[rows[:, 0], rows[:, 1]])
    assert math.isfinite(float(np.abs(out).max()))


def _separate_sequences(lq, lk, Hq, Hkv, D, seed):
    """Each sequence drawn on its own as [H, L, D] arrays (never sliced from a packed
    tensor), then packed by concatenation along tokens into [T, H, D]."""
    rng = np.random.default_rng(seed)
    seqs = []
    for b, (a, c) in enumerate(zip(lq, lk)):
        q = rng.standard_normal((Hq, a, D)).astype(np.float32)
        k = (rng.standard_normal((Hkv, c, D)) + rng.normal(0, 2, (Hkv, 1, D))).astype(np.float32)
        v = rng.standard_normal((Hkv, c, D)).astype(np.float32)
        seqs.append((q, k, v))
    pack = lambda i, H: np.concatenate([s[i].transpose(1, 0, 2) for s in seqs], 0).reshape(-1, H, D)  # noqa: E731
    cu_q = np.concatenate([[0], np.cumsum(lq)]).astype(np.int64)
    cu_k = np.concatenate([[0], np.cumsum(lk)]).astype(np.int64)
    return seqs, pack(0, Hq), pack(1, Hkv), pack(2, Hkv), cu_q, cu_k


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("gscale,smooth_q", [("none", False), ("head", False), ("none", True)])
def test_varlen_equals_each_sequence_alone(oracle_mod, causal, gscale, smooth_q):
    # Every sequence is its own problem with its own K mean (and query mean, and
    # per-(sequence, head) scales): the packed result must equal oracle.attention on each
    # separately drawn sequence, bit for bit, and zero rows for a sequence with no keys.
    Hq, Hkv, D = 4, 2, 64
    lq, lk = [130, 1, 0, 77, 40], [200, 5, 3, 77, 0]
    seqs, q, k, v, cu_q, cu_k = _separate_sequences(lq, lk, Hq, Hkv, D, 31)
    got, _ = oracle_mod.attention_varlen(q, k, v, cu_q, cu_k, causal, 0.125, gscale=gscale,
                                         smooth_q=smooth_q)
    for b, (qs, ks, vs) in enumerate(seqs):
        seg = got[cu_q[b]:cu_q[b + 1]]
        if lq[b] == 0:
            assert seg.shape[0] == 0
            continue
        if lk[b] == 0:
            assert not seg.any()
            continue
        want, _ = oracle_mod.attention(qs, ks, vs, causal, 0.125, gscale=gscale, heads=(1, Hq, Hkv),
                                       smooth_q=smooth_q)
        assert np.array_equal(seg.transpose(1, 0, 2), want), b
    # Sampled (token, head) rows equal the same rows of the full result.
    rows = np.array([[0, 0], [129, 3], [130, 1], [131 + 76, 2], [131 + 77 + 39, 0]])
    part, _ = oracle_mod.attention_varlen(q, k, v, cu_q, cu_k, causal, 0.125, gscale=gscale,
                                          smooth_q=smooth_q, rows=rows)
    assert np.array_equal(part, got[rows[:, 0], rows[:, 1]])


def test_varlen_equal_lengths_equal_dense_batches(oracle_mod):
    # With every length equal, the packed problem is the dense [B, H, N, D] problem: the
    # dense oracle indexes batches itself (per-(batch, head) K means inside the C code),
    # the packed one slices sequences in Python, and they must agree bit for bit.
    B, Hq, Hkv, N, D = 3, 4, 2, 150, 64
    seqs, q, k, v, cu_q, cu_k = _separate_sequences([N] * B, [N] * B, Hq, Hkv, D, 32)
    got, _ = oracle_mod.attention_varlen(q, k, v, cu_q, cu_k, True, 0.125)
    qd = np.concatenate([s[0] for s in seqs], 0)
    kd = np.concatenate([s[1] for s in seqs], 0)
    vd = np.concatenate([s[2] for s in seqs], 0)
    dense, _ = oracle_mod.attention(qd, kd, vd, True, 0.125, heads=(B, Hq, Hkv))
    assert np.array_equal(got.reshape(B, N, Hq, D).transpose(0, 2, 1, 3).reshape(B * Hq, N, D), dense)


def test_varlen_tensor_scale_is_the_plain_maximum(oracle_mod):
    # The per-tensor second-level maxima are max |x| over every sequence and head (K after
    # subtracting its own sequence's mean), computed here directly with numpy.
    Hq, Hkv, D = 2, 1, 64
    lq, lk = [60, 33], [50, 90]
    seqs, q, k, v, cu_q, cu_k = _separate_sequences(lq, lk, Hq, Hkv, D, 33)
    a = oracle_mod.varlen_amax(q, k, v, cu_q, cu_k)
    want_q = max(np.abs(s[0]).max() for s in seqs)
    want_v = max(np.abs(s[2]).max() for s in seqs)
    want_k = 0.0
    for _, ks, _ in seqs:
        mu = (ks.astype(np.float64).sum(1) / ks.shape[1]).astype(np.float32)
        want_k = max(want_k, float(np.abs((ks - mu[:, None, :]).astype(np.float32)).max()))
    assert a["q"] == np.float32(want_q) and a["v"] == np.float32(want_v) and a["k"] == np.float32(want_k)
