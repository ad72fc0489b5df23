"""The index arithmetic of the streaming FWHT kernel, restated on the CPU.

The kernel (act_quant_fwht_stream_kernel) transforms a token of K = 2^LOGK elements in
two register phases around one shared-memory transpose:
  phase 0: thread t holds elements t + (r << TLOG), r < 2^ELOG, and transforms element
           bits TLOG..LOGK-1;
  phase 1: thread t holds elements t * 2^ELOG + r and transforms bits 0..TLOG-1;
with ELOG = ceil(LOGK / 2), TLOG = LOGK - ELOG, and element i stored at shared-memory
word i ^ (((i >> ELOG) & 7) << 2).  These checks restate that arithmetic and verify
what the kernel relies on: the word map is a bijection, the phase-0 word stores of a
warp hit 32 distinct banks, the phase-1 16-byte loads of each quarter warp hit 8
distinct 16-byte bank groups and keep their four elements contiguous, and the two
phases compose to the Sylvester-ordered Walsh-Hadamard transform (the v2 page's
fast_hadamard_transform without its per-stage scaling).
"""
import numpy as np
import pytest


def shape(logk):
    elog = (logk + 1) // 2
    return elog, 1 << elog, logk - elog, 1 << (logk - elog)


def word(i, elog):
    return i ^ (((i >> elog) & 7) << 2)


@pytest.mark.parametrize("logk", [11, 12, 13, 14])
def test_word_map_is_a_bijection_and_conflict_free(logk):
    elog, E, tlog, T = shape(logk)
    K = 1 << logk
    i = np.arange(K)
    w = word(i, elog)
    assert np.array_equal(np.sort(w), i)
    # phase-0 stores: for each warp and register, 32 lanes -> 32 distinct banks
    lanes = np.arange(min(32, T))
    for warp in range(max(1, T // 32)):
        t = warp * 32 + lanes
        for r in range(E):
            banks = word(t + (r << tlog), elog) % 32
            assert len(np.unique(banks)) == len(lanes)
    # phase-1 16-byte loads: quarter warps of 8 lanes, distinct bank groups, contiguous units
    for t0 in range(0, T, 8):
        t = np.arange(t0, min(t0 + 8, T))
        for u in range(E // 4):
            base = word(t * E + 4 * u, elog)
            assert np.all(base % 4 == 0)
            for k in range(4):
                assert np.array_equal(word(t * E + 4 * u + k, elog), base + k)
            assert len(np.unique((base // 4) % 8)) == len(t)
            # the kernel reads unit u of thread t at t*E + 4 * ((u & ~7) | ((u ^ t) & 7))
            assert np.array_equal(base, t * E + 4 * ((u & ~7) | ((u ^ t) & 7)))


@pytest.mark.parametrize("logk", [11, 12])
def test_two_phases_compose_to_the_hadamard_transform(logk):
    elog, E, tlog, T = shape(logk)
    K = 1 << logk
    x = np.random.default_rng(logk).standard_normal(K)
    smem = np.zeros(K)
    r = np.arange(E)
    for t in range(T):
        v = x[t + (r << tlog)].copy()
        for b in range(elog):  # register bit b = element bit tlog + b
            lo = r[(r >> b) & 1 == 0]
            a, c = v[lo].copy(), v[lo | (1 << b)].copy()
            v[lo], v[lo | (1 << b)] = a + c, a - c
        smem[word(t + (r << tlog), elog)] = v
    z = np.zeros(K)
    for t in range(T):
        v = smem[word(t * E + r, elog)].copy()
        for b in range(tlog):  # register bit b = element bit b
            lo = r[(r >> b) & 1 == 0]
            a, c = v[lo].copy(), v[lo | (1 << b)].copy()
            v[lo], v[lo | (1 << b)] = a + c, a - c
        z[t * E + r] = v
    idx = np.arange(K)
    parity = np.vectorize(lambda a: bin(a).count("1") & 1)(np.bitwise_and.outer(idx, idx))
    H = 1.0 - 2.0 * parity  # Sylvester order: H[i][j] = (-1)^popcount(i & j)
    np.testing.assert_allclose(z, H @ x, rtol=0, atol=1e-9)
