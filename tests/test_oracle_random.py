"""Randomised structure checks of the CPU oracle (both exponent coders): small tensors with
random lengths, exponent spreads, chunk sizes, group sizes and table sizes.  Each case
checks the round trip and properties fixed by the container rules: the size rule, the
index (chunk lengths summing to their group's span, group starts summing to the total),
the Huffman stream length (the sum of the code lengths) and the tANS chunk floor (a
chunk with elements holds at least its start state)."""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle


def tensor(n: int, spread: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    e = (120 + rng.integers(0, spread, size=n)).astype(np.uint16)
    low = rng.integers(0, 128, size=n, dtype=np.uint16)
    sign = rng.integers(0, 2, size=n, dtype=np.uint16) << 15
    return (sign | (e << 7) | low).astype(np.uint16)


def index_of(c: np.ndarray, gbase_off: int):
    ng = int(c[44:48].view(np.uint32)[0])
    nc = int(c[40:44].view(np.uint32)[0])
    gbase = c[gbase_off: gbase_off + 8 * (ng + 1)].view(np.uint64).astype(np.int64)
    off_clen = (gbase_off + 8 * (ng + 1) + 15) // 16 * 16
    clen = c[off_clen: off_clen + 2 * nc].view(np.uint16).astype(np.int64)
    return ng, gbase, clen


def check_index(c: np.ndarray, gbase_off: int, G: int):
    ng, gbase, clen = index_of(c, gbase_off)
    total_bits = int(c[16:24].view(np.uint64)[0])
    assert gbase[0] == 0 and gbase[-1] == total_bits
    for g in range(ng):
        assert gbase[g + 1] - gbase[g] == clen[g * G:(g + 1) * G].sum()
    return clen


cases = st.tuples(st.integers(0, 700), st.integers(1, 40), st.integers(0, 2 ** 31 - 1),
                  st.sampled_from([8, 16, 24, 64]), st.integers(1, 5))


@settings(max_examples=60, deadline=None)
@given(cases)
def test_huffman_random(case):
    n, spread, seed, K, G = case
    w = tensor(n, spread, seed)
    c = oracle.encode(w, K=K, G=G)
    assert np.array_equal(oracle.decode(c), w)
    total_bits = int(c[16:24].view(np.uint64)[0])
    assert c.size == oracle.container_bytes(n, K, G, total_bits)
    lens = oracle.code_lengths(oracle.histogram(w))
    assert total_bits == int(lens[(w >> 7) & 0xFF].astype(np.int64).sum())
    check_index(c, 320, G)


@settings(max_examples=60, deadline=None)
@given(cases, st.integers(6, 12))
def test_tans_random(case, R):
    n, spread, seed, K, G = case
    w = tensor(n, spread, seed)
    c = oracle.encode_tans(w, K=K, G=G, table_log=R)
    assert np.array_equal(oracle.decode(c), w)
    total_bits = int(c[16:24].view(np.uint64)[0])
    assert c.size == oracle.tans_container_bytes(n, K, G, total_bits)
    clen = check_index(c, 576, G)
    f = c[64:576].view(np.uint16)
    assert int(f.sum()) == (1 << R if n else 0)
    # a chunk has bits exactly when it has elements, and then at least its R-bit state
    ng = int(c[44:48].view(np.uint32)[0])
    for g in range(ng):
        for lane in range(G):
            has = g * G * K + lane * 8 < n
            cl = int(clen[g * G + lane])
            assert (cl >= R) if has else (cl == 0)
