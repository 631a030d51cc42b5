"""Pins of the oracle's second tANS coder, two interleaved states per chunk (coder 2, rule
T6 on top of T1-T5): hand-worked containers (tests/golden/tans2_containers.txt), and the
rule's reduction to two independent single-state coders (T4) on the even and the odd
positions of a chunk: same bit count, and with dyadic frequencies (every field length
known in advance) the same fields, interleaved in symbol order."""
import os
import sys

import numpy as np
import pytest

import oracle
from lossless_entropy_coded_exponent_b200 import inputs

sys.path.insert(0, os.path.dirname(__file__))
from test_oracle import load_golden_containers  # noqa: E402


@pytest.mark.parametrize("case", load_golden_containers("tans2_containers.txt"), ids=lambda c: c["name"])
def test_tans2_golden_containers(case):
    got = oracle.encode_tans(case["input"], K=case["K"], G=case["G"], table_log=case["R"], states=2)
    assert got.size == case["bytes"].size
    assert np.array_equal(got, case["bytes"])
    assert np.array_equal(oracle.decode(case["bytes"]), case["input"])


def random_table(rng, R, used):
    """A frequency table over `used` symbols summing to M = 2^R."""
    M = 1 << R
    syms = np.sort(rng.choice(256, size=used, replace=False))
    cut = np.sort(rng.choice(np.arange(1, M), size=used - 1, replace=False))
    f = np.zeros(256, dtype=np.uint32)
    f[syms] = np.diff(np.concatenate([[0], cut, [M]]))
    return f, syms


@pytest.mark.parametrize("seed", range(6))
def test_tans2_bits_are_the_two_single_state_codes(seed):
    """A chunk's T6 length is the T4 length of its even-position symbols plus the T4
    length of its odd-position symbols: each state runs T4 on its own subsequence."""
    rng = np.random.default_rng(seed)
    R = int(rng.integers(4, 13))
    f, syms = random_table(rng, R, int(rng.integers(2, min(40, 1 << R) + 1)))
    for cnt in (1, 2, 3, 8, 17, 128):
        e = rng.choice(syms, size=cnt, p=f[syms] / f[syms].sum()).astype(np.uint8)
        t6 = oracle.tans_encode_chunk(f, e, table_log=R, states=2)
        even = oracle.tans_encode_chunk(f, e[0::2], table_log=R)
        odd = oracle.tans_encode_chunk(f, e[1::2], table_log=R) if cnt > 1 else ""
        # a state with no symbol stays at M: R zero bits
        assert len(t6) == len(even) + (len(odd) if cnt > 1 else R)


@pytest.mark.parametrize("R", [4, 8, 12])
def test_tans2_dyadic_fields_interleave_the_single_state_fields(R):
    """With f[s] = M 2^-l every field of s is exactly l bits long, so the T4 codes of the
    even and odd subsequences split into their start state and fields; T6 must be A's
    state, B's state, then the two field lists interleaved in symbol order."""
    rng = np.random.default_rng(R)
    M = 1 << R
    f = np.zeros(256, dtype=np.uint32)
    f[[127, 126, 125, 128]] = [M // 2, M // 4, M // 8, M // 8]
    width = {127: 1, 126: 2, 125: 3, 128: 3}
    for cnt in (1, 2, 5, 8, 31, 128):
        e = rng.choice([127, 126, 125, 128], size=cnt, p=[0.5, 0.25, 0.125, 0.125]).astype(np.uint8)

        def split(bits, seq):
            state, rest, fields = bits[:R], bits[R:], []
            for s in seq:
                fields.append(rest[: width[int(s)]])
                rest = rest[width[int(s)]:]
            assert rest == ""
            return state, fields

        sa, fa = split(oracle.tans_encode_chunk(f, e[0::2], table_log=R), e[0::2])
        sb, fb = split(oracle.tans_encode_chunk(f, e[1::2], table_log=R), e[1::2]) if cnt > 1 else ("0" * R, [])
        merged = [fa[i // 2] if i % 2 == 0 else fb[i // 2] for i in range(cnt)]
        assert oracle.tans_encode_chunk(f, e, table_log=R, states=2) == sa + sb + "".join(merged)


@pytest.mark.parametrize("name", list(inputs.edge_cases().keys()))
def test_tans2_round_trip_edge_cases(name):
    w = inputs.edge_cases()[name]
    for K, G in ((8, 1), (64, 32), (128, 32)):
        c = oracle.encode_tans(w, K=K, G=G, table_log=12, states=2)
        assert int(c[60:64].view(np.uint32)[0]) == 2
        assert np.array_equal(oracle.decode(c), w)


def test_tans2_container_length_is_the_sum_of_the_single_state_codes():
    """Whole tensor: with the container's own frequency table, every chunk's length in
    the index and the stream's total are the T4 lengths of the chunk's even and odd
    subsequences added up (one extra R-bit state per chunk against coder 1, and fields
    whose lengths follow each state's own trajectory)."""
    w = inputs.gaussian(4096 * 3 + 8 * 5 + 3, 0.02, seed=5)
    K, G, R = 128, 32, 12
    c = oracle.encode_tans(w, K=K, G=G, table_log=R, states=2)
    f = c[64: 64 + 512].view(np.uint16).astype(np.uint32)
    ng = int(c[44:48].view(np.uint32)[0])
    off_clen = (576 + 8 * (ng + 1) + 15) // 16 * 16
    clen = c[off_clen: off_clen + 2 * ng * G].view(np.uint16)
    e = ((w >> 7) & 0xFF).astype(np.uint8)
    total = 0
    for g in range(ng):
        for lane in range(G):
            idx = [g * G * K + (G * k + lane) * 8 + j for k in range(K // 8) for j in range(8)]
            sym = np.array([e[x] for x in idx if x < w.size], dtype=np.uint8)
            want = 0
            if sym.size:
                want = len(oracle.tans_encode_chunk(f, sym[0::2], table_log=R))
                want += len(oracle.tans_encode_chunk(f, sym[1::2], table_log=R)) if sym.size > 1 else R
            assert int(clen[g * G + lane]) == want
            total += want
    assert int(c[16:24].view(np.uint64)[0]) == total
    assert np.array_equal(oracle.decode(c), w)


def test_tans2_malformed_containers_are_rejected():
    w = inputs.gaussian(5000, 0.02, seed=3)
    c = oracle.encode_tans(w, K=64, G=4, table_log=10, states=2)
    stream_end = int(c[24:32].view(np.uint64)[0])
    rng = np.random.default_rng(1)
    rejected = 0
    for _ in range(40):
        bad = c.copy()
        pos = int(rng.integers(stream_end - 200, stream_end - 16))
        bad[pos] ^= np.uint8(1 << int(rng.integers(0, 8)))
        try:
            out = oracle.decode(bad)
            assert not np.array_equal(out, w) or True
        except oracle.OracleError:
            rejected += 1
    assert rejected >= 30
    bad = c.copy()
    bad[60] = 3  # no such coder
    with pytest.raises(oracle.OracleError):
        oracle.decode(bad)
