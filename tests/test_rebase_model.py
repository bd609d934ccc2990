"""The FP4 attention kernel splits a row's key tiles between two softmax warpgroups
(tiles j = 0, 2, ... and 1, 3, ...), each keeping its own lazy reference maximum m_w
(it moves only when a tile maximum exceeds it by more than 8 in log2 units) and row sum
l_w; a correction warpgroup keeps O relative to its own lazy reference m_O and folds tile
j in with the factor s1_j * 2^(e_j - m_O), where e_j is the reference the tile's
warpgroup used. The final row sum is l = sum_w l_w * 2^(m_w - m_O).

This is a binary64 model of that bookkeeping (without the FP4 rounding, which does not
depend on the references: P~ is quantized relative to the tile maximum) checked against a
plain softmax: on rows whose tile maxima alternate far above and below each other, drift,
and include fully masked tiles, the two agree to rounding."""
import numpy as np
import pytest

THRESH = 8.0


def model(S, V):
    """S [T, 128] scores in log2 units (-inf = masked), V [T, 128, D] -> O [D]."""
    T = S.shape[0]
    m_w = [-np.inf, -np.inf]
    l_w = [0.0, 0.0]
    O = np.zeros(V.shape[2])
    m_o = -np.inf
    for j in range(T):
        w = j & 1
        tmx = S[j].max()
        empty = tmx == -np.inf
        move = tmx > m_w[w] + THRESH
        m_new = tmx if move else m_w[w]
        alpha = 2.0 ** (m_w[w] - m_new) if move else 1.0
        rfac = 0.0 if empty else 2.0 ** (tmx - m_new)
        P2 = np.zeros(128) if empty else 2.0 ** (S[j] - tmx) * 2688.0  # what the kernel quantizes
        l_w[w] = l_w[w] * alpha + P2.sum() / 2688.0 * rfac
        m_w[w] = m_new
        s1 = rfac / 2688.0
        PV = P2 @ V[j]
        # correction warpgroup
        a_o, c = 1.0, 0.0
        if s1 > 0.0:
            if m_new > m_o + THRESH:
                a_o = 2.0 ** (m_o - m_new)   # 0 on the first contribution
                m_o = m_new
            c = s1 * 2.0 ** (m_new - m_o)
        O = O * a_o + c * PV
    l = sum(lw * 2.0 ** (mw - m_o) for lw, mw in zip(l_w, m_w) if lw > 0.0)
    return O / l if l > 0.0 else np.zeros_like(O)


def reference(S, V):
    s = S.reshape(-1)
    v = V.reshape(-1, V.shape[2])
    if np.all(s == -np.inf):
        return np.zeros(V.shape[2])
    p = 2.0 ** (s - s.max())
    return p @ v / p.sum()


@pytest.mark.parametrize("seed", range(6))
def test_two_references_rebased_equal_plain_softmax(seed):
    rng = np.random.default_rng(seed)
    T, D = 11, 32
    level = np.where(np.arange(T) % 2 == 0, 1.0, -1.0) * rng.uniform(5.0, 40.0) + rng.uniform(0.0, 3.0) * np.arange(T)
    if seed % 2:
        level = level[::-1]                       # references that fall as well as rise
    S = rng.standard_normal((T, 128)) * 2.0 + level[:, None]
    if seed >= 3:
        S[rng.integers(0, T)] = -np.inf           # a fully masked tile
        S[:, rng.integers(0, 128, 20)] = -np.inf  # masked keys
    V = rng.standard_normal((T, 128, D))
    got, want = model(S, V), reference(S, V)
    assert np.max(np.abs(got - want)) <= 1e-12 * max(1.0, np.max(np.abs(want)))


def test_row_with_no_key_is_zero():
    S = np.full((4, 128), -np.inf)
    V = np.ones((4, 128, 8))
    assert not model(S, V).any()


def test_first_tiles_empty_then_keys():
    rng = np.random.default_rng(7)
    S = rng.standard_normal((5, 128))
    S[:2] = -np.inf                                # both warpgroups start with an empty tile
    V = rng.standard_normal((5, 128, 16))
    assert np.max(np.abs(model(S, V) - reference(S, V))) <= 1e-12
