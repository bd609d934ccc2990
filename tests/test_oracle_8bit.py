"""Pins for the oracle's 8-bit path (INT8 Q/K per 128-token block, E4M3 V per channel,
E4M3 P~ with the per-row factor rowmax / 448 per key tile).

  * INT8 blocks: integer grids round-trip with scale absmax / 127; ties go to the even
    integer; an all-zero block gives scale 0 and codes 0; each block takes its own
    maximum (ragged last block); the K mean is subtracted first;
  * E4M3 channels: representable columns round-trip with scale absmax / 448;
  * attention closed forms: identical keys give the mean of the dequantized V; scores at
    multiples of -ln 2 make every P~ a power of two (exact in E4M3 relative to 448), so
    the emulation equals exact attention on the dequantized inputs, across key tiles and
    a change of running maximum; a P~ of 0.3 becomes the E4M3 value 128/448 = 2/7.
"""
import math

import numpy as np
import pytest


def _rand(shape, seed, scale=1.0, bias=0.0):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal(shape) * scale + bias).astype(np.float32)


def test_int8_grid_round_trip_and_ties(oracle_mod):
    rng = np.random.default_rng(1)
    c = rng.integers(-127, 128, (1, 200, 32)).astype(np.float32)
    c[0, 5, 3] = 127.0
    c[0, 150, 0] = -127.0
    x = (c * 0.125).astype(np.float32)
    codes, sc = oracle_mod.quant_int8_rows(x, block=128)
    assert sc.tolist() == [[0.125, 0.125]]
    assert np.array_equal(codes.astype(np.float32), c)
    # ties: block absmax 127 -> scale 1; 2.5 -> 2, -3.5 -> -4, 0.5 -> 0, 126.5 -> 126
    t = np.zeros((1, 4, 16), np.float32)
    t[0, 0, :5] = [127.0, 2.5, -3.5, 0.5, 126.5]
    codes, sc = oracle_mod.quant_int8_rows(t, block=4)
    assert sc[0, 0] == 1.0 and codes[0, 0, :5].tolist() == [127, 2, -4, 0, 126]


def test_int8_zero_block_ragged_blocks_and_mean(oracle_mod):
    x = _rand((2, 300, 64), 2)
    x[1, 128:256] = 0.0
    codes, sc = oracle_mod.quant_int8_rows(x, block=128)
    assert sc.shape == (2, 3) and sc[1, 1] == 0.0 and not codes[1, 128:256].any()
    for g in range(2):
        for b, (n0, n1) in enumerate([(0, 128), (128, 256), (256, 300)]):
            assert sc[g, b] == np.float32(np.abs(x[g, n0:n1]).max()) / np.float32(127.0)
    mu = _rand((2, 64), 3)
    c1, s1 = oracle_mod.quant_int8_rows(x, block=128, mean=mu)
    c2, s2 = oracle_mod.quant_int8_rows((x - mu[:, None, :]).astype(np.float32), block=128)
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)


def test_e4m3_channels_round_trip(oracle_mod):
    rng = np.random.default_rng(4)
    G, N, D = 2, 40, 16
    codes = rng.integers(0, 0x7F, (G, N, D)).astype(np.uint8)  # finite positive bytes
    codes[:, 0, :] = 0x7E                                       # 448 in every channel
    sign = np.where(rng.integers(0, 2, (G, N, D)) > 0, 1.0, -1.0)
    v = (oracle_mod.e4m3_decode(codes) * sign * 2.0 ** -7).astype(np.float32)
    vt, sc = oracle_mod.quant_e4m3_channels(v)
    assert np.all(sc == np.float32(2.0 ** -7))
    back = oracle_mod.e4m3_decode(vt) * sc[:, :, None]
    assert np.array_equal(back, v.transpose(0, 2, 1).astype(np.float64))
    z = np.zeros((1, 8, 16), np.float32)
    vt, sc = oracle_mod.quant_e4m3_channels(z)
    assert not vt.any() and not sc.any()


def test_identical_keys_give_mean_of_v(oracle_mod):
    q, v = _rand((1, 64, 32), 5), _rand((1, 64, 32), 6)
    k = np.repeat(_rand((1, 1, 32), 7), 64, axis=1)
    out, qz = oracle_mod.attention8(q, k, v, False, 0.2)
    assert not qz["k8"].any()
    vdeq = oracle_mod.e4m3_decode(qz["vt8"]) * qz["v_scale"][:, :, None]   # [1, D, N]
    assert np.max(np.abs(out - vdeq.mean(axis=2)[:, None, :])) <= 1e-12


def _power_of_two_case(ts, seed):
    """q = [127, 0...]; key j = [-t_j, 0...] plus one key [0, 127, 0...] that pins K's
    block scale to 1; sm_scale = ln 2 / 127 makes S_j = -t_j ln 2. V columns are E4M3 grid
    values times 2^-7, each with a +-3.5 (= 448 * 2^-7) so that every scale is 2^-7."""
    N, D = len(ts) + 1, 16
    q = np.zeros((1, 1, D), np.float32)
    q[0, 0, 0] = 127.0
    k = np.zeros((1, N, D), np.float32)
    k[0, :-1, 0] = -np.asarray(ts, np.float32)
    k[0, -1, 1] = 127.0
    rng = np.random.default_rng(seed)
    grid = np.array([0.0, 0.25, 0.5, 1.0, 1.5, 2.0, 3.0, 3.5], np.float32)
    v = grid[rng.integers(0, 8, (1, N, D))] * np.where(rng.integers(0, 2, (1, N, D)) > 0, 1, -1)
    v[0, 0, :] = 3.5
    return q, k, v.astype(np.float32), math.log(2.0) / 127.0


@pytest.mark.parametrize("Bk", [16, 128])
def test_power_of_two_weights_are_lossless(oracle_mod, Bk):
    ts = [2, 0, 1, 3, 0, 2, 1, 1] * 4 + [0, 3, 3, 1]          # 36 keys, maxima move across tiles
    q, k, v, sm = _power_of_two_case(ts, 8)
    out, qz = oracle_mod.attention8(q, k, v, False, sm, Bk=Bk, smooth_k=False)
    assert qz["k_scale"].tolist() == [[1.0]] and qz["q_scale"].tolist() == [[1.0]]
    assert np.all(qz["v_scale"] == np.float32(2.0 ** -7))
    ex = oracle_mod.attn_exact(q, k, v, False, sm)
    assert np.max(np.abs(out - ex)) <= 1e-12


def test_p_rounds_to_nearest_e4m3(oracle_mod):
    # Two keys: S = 0 and S = ln 0.3. P2 = [448, 134.4]; 134.4 rounds to 128 (E4M3 spacing
    # 16 in [128, 256)), so the weights are 1 and 128/448 = 2/7 while l = 1.3.
    N, D = 2, 16
    q = np.zeros((1, 1, D), np.float32)
    q[0, 0, 0] = 127.0
    k = np.zeros((1, N, D), np.float32)
    k[0, 1, 0] = -1.0
    k[0, 0, 1] = 127.0                                          # block scale 1
    v = np.zeros((1, N, D), np.float32)
    v[0, :, 0] = [3.5, -1.5]
    v[0, :, 1] = [0.5, 3.5]
    sm = math.log(0.3) / -127.0
    out, _ = oracle_mod.attention8(q, k, v, False, sm, smooth_k=False)
    vd = v[0].astype(np.float64)
    want = (vd[0] + (2.0 / 7.0) * vd[1]) / 1.3
    assert np.max(np.abs(out[0, 0] - want)) <= 1e-12
