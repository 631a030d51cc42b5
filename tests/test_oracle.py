"""Pins for the CPU oracle: checks against things other than the oracle itself.

* the BF16 field split, against the IEEE value of every one of the 65 536 patterns;
* hand-worked containers and tie-rule vectors (tests/golden, derived by hand);
* brute-force optimality of the code lengths on tiny alphabets;
* equality with the textbook (heap) Huffman cost when the tree fits the limit;
* an independent dynamic program for the length-limited optimum (Fibonacci clamp);
* Kraft equality, the entropy bound, canonical-code prefix-freedom;
* exhaustive and edge-case round trips, and rejection of malformed containers;
* for the tANS exponent coder: hand-worked containers and frequency vectors, the
  state-numbering and tiling properties of its tables, exact field lengths on dyadic
  distributions (equal to the package-merge code's), a rate within a hair of the
  entropy, round trips and rejection of malformed containers.
"""
import heapq
import itertools
import math
import os
from functools import lru_cache

import numpy as np
import pytest

import oracle
from lossless_entropy_coded_exponent_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- helpers

def textbook_huffman(counts):
    """Heap Huffman: (total cost, tree depth).  Independent of package-merge."""
    items = [(c, i, 0) for i, c in enumerate(counts) if c > 0]
    if len(items) < 2:
        return (sum(c for c, _, _ in items), 1 if items else 0)
    heapq.heapify(items)
    cost, uid = 0, len(counts)
    while len(items) > 1:
        a = heapq.heappop(items)
        b = heapq.heappop(items)
        cost += a[0] + b[0]
        heapq.heappush(items, (a[0] + b[0], uid, max(a[2], b[2]) + 1))
        uid += 1
    return cost, items[0][2]


def brute_force_min_cost(counts, L):
    used = [c for c in counts if c > 0]
    best = None
    for lens in itertools.product(range(1, L + 1), repeat=len(used)):
        if sum(2.0 ** -l for l in lens) <= 1.0 + 1e-12:
            cost = sum(c * l for c, l in zip(used, lens))
            best = cost if best is None else min(best, cost)
    return best


def dp_length_limited_cost(counts, L):
    """Optimal cost of a prefix code with lengths <= L by a level-by-level DP:
    heavier symbols take shallower leaves; at depth d with `a` open nodes,
    choose how many become leaves, the rest split into 2 nodes each."""
    w = sorted((c for c in counts if c > 0), reverse=True)
    m = len(w)
    prefix = [0]
    for x in w:
        prefix.append(prefix[-1] + x)

    @lru_cache(maxsize=None)
    def f(d, i, a):
        if i == m:
            return 0
        if d > L or a == 0:
            return math.inf
        best = math.inf
        for k in range(0, min(a, m - i) + 1):
            rest = min(2 * (a - k), m - i - k)
            best = min(best, d * (prefix[i + k] - prefix[i]) + f(d + 1, i + k, rest))
        return best

    return f(1, 0, 2)


def cost_of(counts, lens):
    return int(sum(int(c) * int(l) for c, l in zip(counts, lens)))


def kraft24(lens):
    return sum(1 << (24 - int(l)) for l in lens if l > 0)


def load_golden_containers(name="tiny_containers.txt"):
    cases, cur = [], None
    with open(os.path.join(GOLDEN, name)) as fh:
        for raw in fh:
            line = raw.split("#", 1)[0].strip()
            if not line:
                continue
            if line.startswith("case "):
                parts = line.split()
                kv = dict(p.split("=") for p in parts[2:])
                cur = {"name": parts[1], "K": int(kv["K"]), "G": int(kv["G"]), "R": int(kv.get("R", 0)),
                       "bytes": np.zeros(int(kv["total"]), dtype=np.uint8)}
                cases.append(cur)
            elif line.startswith("input"):
                words = []
                for t in line.split()[1:]:
                    wv, _, rep = t.partition("*")
                    words += [int(wv, 16)] * (int(rep) if rep else 1)
                cur["input"] = np.array(words, dtype=np.uint16)
            else:
                off, hexes = line.split(":")
                vals = [int(t, 16) for t in hexes.split()]
                cur["bytes"][int(off): int(off) + len(vals)] = vals
    return cases


def load_tie_rules():
    rows = []
    with open(os.path.join(GOLDEN, "tie_rule.txt")) as fh:
        for raw in fh:
            line = raw.split("#", 1)[0].strip()
            if not line:
                continue
            L, cnt, exp = (p.strip() for p in line.split("|"))
            counts = np.zeros(256, dtype=np.uint64)
            for t in cnt.split():
                s, c = t.split(":")
                counts[int(s)] = int(c)
            expected = np.zeros(256, dtype=np.uint8)
            for t in exp.split():
                s, l = t.split(":")
                expected[int(s)] = int(l)
            rows.append((int(L), counts, expected))
    return rows


# ---------------------------------------------------------------- the split

def test_split_matches_ieee_fields_for_every_pattern():
    # every pattern, each with a partner drawn from the patterns (a seeded
    # permutation): the byte is the pattern's mantissa above the partner's sign
    w = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    q = w[np.random.default_rng(5).permutation(w.size)]
    x = (w.astype(np.uint32) << 16).view(np.float32)
    xq = (q.astype(np.uint32) << 16).view(np.float32)
    e_or = np.array([oracle.exponent(int(v)) for v in w], dtype=np.int64)
    m_or = np.array([oracle.sign_mantissa(int(v), int(u)) for v, u in zip(w, q)], dtype=np.int64)
    mq_or = np.array([oracle.sign_mantissa(int(u), int(v)) for v, u in zip(w, q)], dtype=np.int64)
    with np.errstate(all="ignore"):
        finite = np.isfinite(x)
        a = np.abs(x.astype(np.float64))
        normal = finite & (a >= 2.0 ** -126)
        sub = finite & (a > 0) & ~normal
        frac, ex = np.frexp(a)
    exp_e = np.where(normal, ex + 126, 0)
    exp_e = np.where(finite, exp_e, 255)
    mant = np.zeros_like(exp_e)
    mant = np.where(normal, np.rint((frac * 2 - 1) * 128), mant)
    mant = np.where(sub, np.rint(a / 2.0 ** -133), mant).astype(np.int64)
    sign_q = np.signbit(xq).astype(np.int64)
    nan = np.isnan(x)
    assert np.array_equal(e_or, exp_e)
    ok = ~nan
    assert np.array_equal(m_or[ok], (mant[ok] << 1) | sign_q[ok])
    assert np.all((m_or[nan] >> 1) != 0) and np.array_equal(m_or & 1, sign_q)
    assert np.mean(np.signbit(x) != np.signbit(xq)) > 0.4  # the partner's sign is really another bit
    back = np.array([oracle.merge(int(e), int(m), int(mq)) for e, m, mq in zip(e_or, m_or, mq_or)], dtype=np.uint16)
    assert np.array_equal(back, w)


def test_partners_are_even_odd_pairs():
    assert [oracle.partner(x, 6) for x in range(6)] == [1, 0, 3, 2, 5, 4]
    assert [oracle.partner(x, 5) for x in range(5)] == [1, 0, 3, 2, 4]  # the odd last element keeps its own sign
    assert oracle.partner(0, 1) == 0


# ---------------------------------------------------------------- code lengths

@pytest.mark.parametrize("row", load_tie_rules(), ids=lambda r: str(r[0]))
def test_tie_rule_golden(row):
    L, counts, expected = row
    assert np.array_equal(oracle.code_lengths(counts, L), expected)


def test_brute_force_optimality_tiny_alphabets():
    rng = np.random.default_rng(123)
    trials = 0
    for m in range(2, 8):
        for L in (3, 4, 5):
            if (1 << L) < m:
                continue
            for _ in range(6 if m < 7 else 2):
                syms = rng.choice(256, size=m, replace=False)
                counts = np.zeros(256, dtype=np.uint64)
                counts[syms] = rng.integers(1, 40, size=m)
                lens = oracle.code_lengths(counts, L)
                assert lens.max() <= L and kraft24(lens) == 1 << 24
                assert np.all((lens > 0) == (counts > 0))
                assert cost_of(counts, lens) == brute_force_min_cost(counts, L)
                trials += 1
    assert trials > 50


def test_matches_textbook_huffman_when_tree_fits():
    w = inputs.small_gaussian()
    counts = oracle.histogram(w)
    hcost, depth = textbook_huffman([int(c) for c in counts])
    assert depth <= 24
    lens = oracle.code_lengths(counts, 24)
    assert cost_of(counts, lens) == hcost
    rng = np.random.default_rng(5)
    for _ in range(20):
        counts = np.zeros(256, dtype=np.uint64)
        k = int(rng.integers(2, 257))
        counts[rng.choice(256, size=k, replace=False)] = rng.integers(1, 10_000, size=k)
        hcost, depth = textbook_huffman([int(c) for c in counts])
        if depth <= 24:
            assert cost_of(counts, oracle.code_lengths(counts, 24)) == hcost


def test_fibonacci_counts_force_the_clamp():
    fib = inputs.fibonacci_counts(28)
    counts = np.zeros(256, dtype=np.uint64)
    counts[100:128] = fib
    hcost, depth = textbook_huffman([int(c) for c in counts])
    assert depth == 27
    lens = oracle.code_lengths(counts, 24)
    assert lens.max() == 24 and kraft24(lens) == 1 << 24
    cost = cost_of(counts, lens)
    assert cost > hcost
    assert cost == dp_length_limited_cost([int(c) for c in counts], 24)


@pytest.mark.parametrize("n_values", [2, 65, 129, 200])
def test_exponent_spread_sets_the_leaf_count(n_values):
    """The generator behind the GPU code-book cases: exactly n_values distinct exponents, all
    of them given a code by the oracle (a complete prefix code), and a lossless round trip."""
    w = inputs.exponent_spread(20_000, n_values, seed=7)
    e = ((w >> 7) & 0xFF).astype(np.int64)
    assert np.unique(e).size == n_values
    counts = np.bincount(e, minlength=256).astype(np.uint64)
    lens = oracle.code_lengths(counts, 24)
    assert int((lens > 0).sum()) == n_values and kraft24(lens) == 1 << 24
    assert np.array_equal(oracle.decode(oracle.encode(w, K=128)), w)


def test_dp_agrees_on_random_limited_cases():
    rng = np.random.default_rng(9)
    for _ in range(10):
        m = int(rng.integers(9, 20))
        L = int(rng.integers(5, 9))
        counts = np.zeros(256, dtype=np.uint64)
        counts[rng.choice(256, size=m, replace=False)] = np.maximum(1, (2.0 ** rng.uniform(0, 14, size=m)).astype(np.int64))
        lens = oracle.code_lengths(counts, L)
        assert lens.max() <= L and kraft24(lens) == 1 << 24
        assert cost_of(counts, lens) == dp_length_limited_cost([int(c) for c in counts], L)


def test_kraft_equality_and_entropy_bound():
    for w in (inputs.small_gaussian(), inputs.projection_with_outliers()):
        counts = oracle.histogram(w)
        lens = oracle.code_lengths(counts, 24)
        assert kraft24(lens) == 1 << 24
        p = counts[counts > 0].astype(np.float64) / w.size
        H = float(-(p * np.log2(p)).sum())
        mean = cost_of(counts, lens) / w.size
        assert H <= mean <= H + 1


def test_canonical_codes_prefix_free_and_ordered():
    for w in (inputs.small_gaussian(), inputs.fibonacci_clamp_tensor(27), inputs.uniform_patterns(1 << 16, 3)):
        lens = oracle.code_lengths(oracle.histogram(w), 24)
        code = oracle.canonical_codes(lens)
        used = [s for s in range(256) if lens[s] > 0]
        order = sorted(used, key=lambda s: (int(lens[s]), s))
        left = [int(code[s]) << (24 - int(lens[s])) for s in order]
        assert left == sorted(left) and len(set(left)) == len(left)
        for a, b in zip(order, order[1:]):
            la, lb = int(lens[a]), int(lens[b])
            # b's code must not start with a's code
            assert (int(code[b]) >> (lb - la)) != int(code[a])
        assert int(code[order[0]]) == 0
        last = order[-1]
        assert int(code[last]) == (1 << int(lens[last])) - 1  # complete code ends in all ones


# ---------------------------------------------------------------- containers

@pytest.mark.parametrize("case", load_golden_containers(), ids=lambda c: c["name"])
def test_golden_containers(case):
    got = oracle.encode(case["input"], K=case["K"], G=case["G"])
    assert got.size == case["bytes"].size
    assert np.array_equal(got, case["bytes"])
    assert np.array_equal(oracle.decode(case["bytes"]), case["input"])


def test_round_trip_every_bit_pattern():
    w = inputs.all_patterns_shuffled(26)
    c = oracle.encode(w)
    assert np.array_equal(oracle.decode(c), w)


@pytest.mark.parametrize("name", list(inputs.edge_cases().keys()))
def test_round_trip_edge_cases(name):
    w = inputs.edge_cases()[name]
    for K, G in ((64, 32), (128, 32), (8, 3), (16, 5)):
        c = oracle.encode(w, K=K, G=G)
        assert c.size == oracle.container_bytes(w.size, K, G, int(c[16:24].view(np.uint64)[0]))
        assert np.array_equal(oracle.decode(c), w)


def test_deterministic_and_size_rule():
    w = inputs.small_gaussian()
    a = oracle.encode(w)
    b = oracle.encode(w.copy())
    assert np.array_equal(a, b)
    total_bits = int(a[16:24].view(np.uint64)[0])
    counts = oracle.histogram(w)
    assert total_bits == cost_of(counts, oracle.code_lengths(counts))
    assert a.size <= oracle.max_container_bytes(w.size, 64, 32)


def test_uniform_exponents_cost_about_eight_bits():
    w = inputs.uniform_patterns(1 << 20, 24)
    c = oracle.encode(w)
    total_bits = int(c[16:24].view(np.uint64)[0])
    assert 7.99 * w.size <= total_bits <= 8.0 * w.size


def test_compression_is_plausible_against_the_pages():
    """Plausibility, not parity: ~1.5:1 (Liguori, abstract) and ~70 % of the
    BF16 size (DFloat11 blog, title and section 02)."""
    w = inputs.small_gaussian()
    c = oracle.encode(w, K=128)
    bits_per_weight = 8.0 * c.size / w.size
    assert 10.0 < bits_per_weight < 11.0
    assert 1.4 < 16.0 / bits_per_weight < 1.6


# ---------------------------------------------------------------- malformed input

def _corrupt_variants(c):
    n = int(c[8:16].view(np.uint64)[0])
    out = {}
    v = c.copy(); v[0] ^= 1; out["magic"] = v
    v = c.copy(); v[4] = 2; out["version"] = v
    v = c.copy(); v[8] ^= 1; out["n"] = v
    v = c.copy(); v[24] ^= 0x10; out["total_bytes"] = v
    out["truncated"] = c[:-1].copy()
    used = int(np.flatnonzero(c[64:320])[0])
    v = c.copy(); v[64 + used] = 0; out["kraft"] = v
    v = c.copy(); v[64 + used] = 30; out["len_over_limit"] = v
    v = c.copy(); v[64 + used] += 1; out["kraft_below_one"] = v
    v = c.copy(); v[320 + 8] ^= 1; out["gbase"] = v
    nc = int(c[40:44].view(np.uint32)[0]); ng = int(c[44:48].view(np.uint32)[0])
    off_clen = (320 + 8 * (ng + 1) + 15) // 16 * 16
    v = c.copy(); v[off_clen] ^= 1; out["clen"] = v
    off_m = int(c[48:56].view(np.uint64)[0])
    off_stream = (off_m + n + 15) // 16 * 16
    pads = [b for b in range(320 + 8 * (ng + 1), off_clen)] + [b for b in range(off_clen + 2 * nc, off_m)] + \
           [b for b in range(off_m + n, off_stream)]
    assert pads, "test input must leave a padding byte"
    v = c.copy(); v[pads[0]] = 1; out["padding"] = v
    v = c.copy(); v[-1] = 1; out["slack"] = v
    assert n > 0
    return out


def test_malformed_containers_are_rejected():
    w = inputs.gaussian(10_003, 0.02, seed=7)
    c = oracle.encode(w)
    assert np.array_equal(oracle.decode(c), w)
    for name, bad in _corrupt_variants(c).items():
        with pytest.raises(oracle.OracleError) as ei:
            oracle.decode(bad)
        assert ei.value.code == oracle.ERR_CORRUPT, name


# ---------------------------------------------------------------- tANS exponent coder

def load_tans_frequencies():
    rows = []
    with open(os.path.join(GOLDEN, "tans_frequencies.txt")) as fh:
        for raw in fh:
            line = raw.split("#", 1)[0].strip()
            if not line:
                continue
            R, cnt, exp = (p.strip() for p in line.split("|"))
            counts = np.zeros(256, dtype=np.uint64)
            for t in cnt.split():
                sym, c = t.split(":")
                counts[int(sym)] = int(c)
            if exp == "refused":
                expected = None
            else:
                expected = np.zeros(256, dtype=np.uint32)
                for t in exp.split():
                    sym, f = t.split(":")
                    expected[int(sym)] = int(f)
            rows.append((int(R), counts, expected))
    return rows


@pytest.mark.parametrize("row", load_tans_frequencies(), ids=lambda r: f"R{r[0]}-{int((r[1] > 0).sum())}sym")
def test_tans_frequency_golden(row):
    R, counts, expected = row
    if expected is None:
        with pytest.raises(oracle.OracleError) as ei:
            oracle.tans_normalize(counts, R)
        assert ei.value.code == oracle.ERR_ARG
    else:
        assert np.array_equal(oracle.tans_normalize(counts, R), expected)


@pytest.mark.parametrize("case", load_golden_containers("tans_containers.txt"), ids=lambda c: c["name"])
def test_tans_golden_containers(case):
    got = oracle.encode_tans(case["input"], K=case["K"], G=case["G"], table_log=case["R"])
    assert got.size == case["bytes"].size
    assert np.array_equal(got, case["bytes"])
    assert np.array_equal(oracle.decode(case["bytes"]), case["input"])


def test_tans_table_golden():
    """The M = 16 table worked by hand in tans_containers.txt."""
    f = np.zeros(256, dtype=np.uint32)
    f[127], f[128] = 13, 3
    sym, k = oracle.tans_tables(f, 4)
    slots_128 = [3, 6, 9]
    assert [j for j in range(16) if sym[j] == 128] == slots_128
    assert all(sym[j] == 127 for j in range(16) if j not in slots_128)
    assert [int(k[j]) for j in slots_128] == [3, 4, 5]
    assert [int(k[j]) for j in range(16) if j not in slots_128] == list(range(13, 26))


def decode_entries(sym, k, R):
    """(symbol, nb, base) of every slot, from the state numbers alone."""
    M = 1 << R
    out = []
    for j in range(M):
        kk = int(k[j])
        nb = R - (kk.bit_length() - 1)
        out.append((int(sym[j]), nb, (kk << nb) - M))
    return out


def random_frequencies(rng, R, used):
    M = 1 << R
    syms = rng.choice(256, size=used, replace=False)
    cuts = np.sort(rng.choice(np.arange(1, M), size=used - 1, replace=False))
    f = np.zeros(256, dtype=np.uint32)
    f[syms] = np.diff(np.concatenate([[0], cuts, [M]]))
    return f


@pytest.mark.parametrize("R", [4, 5, 8, 11, 12])
def test_tans_tables_number_and_tile(R):
    """Each symbol holds exactly f[s] slots numbered f[s] .. 2 f[s] - 1 in ascending slot
    order, and for every symbol the decoder's next-state ranges [base, base + 2^nb) of its
    slots tile [0, M) exactly: from any state, every symbol has exactly one encoding."""
    rng = np.random.default_rng(100 + R)
    M = 1 << R
    for used in sorted({1, 2, 3, min(16, M), min(200, M), min(256, M)}):
        f = random_frequencies(rng, R, used)
        sym, k = oracle.tans_tables(f, R)
        ent = decode_entries(sym, k, R)
        for s in np.flatnonzero(f):
            slots = [j for j in range(M) if sym[j] == s]
            assert len(slots) == f[s]
            assert [int(k[j]) for j in slots] == list(range(int(f[s]), 2 * int(f[s])))
            cover = np.zeros(M, dtype=np.int64)
            for j in slots:
                _, nb, base = ent[j]
                assert 0 <= base and base + (1 << nb) <= M
                cover[base: base + (1 << nb)] += 1
            assert np.all(cover == 1)


def test_tans_normalize_properties():
    rng = np.random.default_rng(7)
    for R in (4, 8, 12):
        M = 1 << R
        for trial in range(40):
            used = int(rng.integers(1, min(M, 256) + 1))
            counts = np.zeros(256, dtype=np.uint64)
            syms = rng.choice(256, size=used, replace=False)
            counts[syms] = rng.integers(1, 10 ** int(rng.integers(1, 7)), size=used)
            f = oracle.tans_normalize(counts, R)
            assert int(f.sum()) == M
            assert np.array_equal(f > 0, counts > 0)
        # counts proportional to a frequency vector come back unchanged
        f0 = random_frequencies(rng, R, min(10, M))
        assert np.array_equal(oracle.tans_normalize(f0.astype(np.uint64) * 37, R), f0)
    assert not oracle.tans_normalize(np.zeros(256, dtype=np.uint64), 12).any()


def dyadic_tensor(n, seed):
    """Exponents 127, 126, 125, 128 with probabilities exactly 1/2, 1/4, 1/8, 1/8."""
    rng = np.random.default_rng(seed)
    e = np.array([127] * (n // 2) + [126] * (n // 4) + [125] * (n // 8) + [128] * (n // 8), dtype=np.uint16)
    rng.shuffle(e)
    low = rng.integers(0, 128, size=n, dtype=np.uint16)
    sign = rng.integers(0, 2, size=n, dtype=np.uint16) << 15
    return (sign | (e << 7) | low).astype(np.uint16)


@pytest.mark.parametrize("K,G,R", [(128, 32, 12), (8, 3, 4), (64, 5, 8)])
def test_tans_dyadic_fields_equal_the_huffman_lengths(K, G, R):
    """With f[s] = M 2^-l exactly, a tANS step for s emits exactly l bits (f <= X >> l <
    2f for every state X in [M, 2M)), so each chunk is R bits longer than its
    package-merge code: checked chunk by chunk against the Huffman oracle."""
    n = 8 * 1000 + 8 * (K // 8) * 3
    w = dyadic_tensor(n, seed=K + R)
    t = oracle.encode_tans(w, K=K, G=G, table_log=R)
    h = oracle.encode(w, K=K, G=G)
    counts = oracle.histogram(w)
    assert list(oracle.code_lengths(counts)[[127, 126, 125, 128]]) == [1, 2, 3, 3]
    ng = int(t[44:48].view(np.uint32)[0])
    nc = ng * G
    off_t = (576 + 8 * (ng + 1) + 15) // 16 * 16
    off_h = (320 + 8 * (ng + 1) + 15) // 16 * 16
    clen_t = t[off_t: off_t + 2 * nc].view(np.uint16).astype(np.int64)
    clen_h = h[off_h: off_h + 2 * nc].view(np.uint16).astype(np.int64)
    assert np.array_equal(clen_t, np.where(clen_h > 0, clen_h + R, 0))
    assert np.array_equal(oracle.decode(t), w)


def test_tans_rate_is_near_the_entropy():
    """On N(0, 0.02^2) exponents the fields cost within 0.003 bits of the empirical
    entropy H (a coder that numbers the states in spread order instead of ascending
    order costs ~0.05 bits more, as much as the Huffman code's excess), and below the
    package-merge code's mean length."""
    w = inputs.gaussian(1 << 20, 0.02, seed=11)
    K, R = 4096, 12
    t = oracle.encode_tans(w, K=K, table_log=R)
    counts = oracle.histogram(w).astype(np.float64)
    p = counts[counts > 0] / counts.sum()
    H = float(-(p * np.log2(p)).sum())
    chunks = -(-w.size // K)
    fields = (int(t[16:24].view(np.uint64)[0]) - R * chunks) / w.size
    huff = cost_of(oracle.histogram(w), oracle.code_lengths(oracle.histogram(w))) / w.size
    assert H - 0.003 <= fields <= H + 0.003, (H, fields)
    assert fields < huff - 0.02


def test_tans_round_trip_every_bit_pattern():
    w = inputs.all_patterns_shuffled(26)
    for R in (8, 12):  # 256 used exponents: at R = 8 every frequency is 1
        c = oracle.encode_tans(w, K=128, table_log=R)
        assert np.array_equal(oracle.decode(c), w)


@pytest.mark.parametrize("name", list(inputs.edge_cases().keys()))
def test_tans_round_trip_edge_cases(name):
    w = inputs.edge_cases()[name]
    used = int((oracle.histogram(w) > 0).sum())
    for K, G, R in ((128, 32, 12), (64, 32, 8), (8, 3, 4), (16, 5, 10)):
        if used > (1 << R):
            with pytest.raises(oracle.OracleError) as ei:
                oracle.encode_tans(w, K=K, G=G, table_log=R)
            assert ei.value.code == oracle.ERR_ARG
            continue
        c = oracle.encode_tans(w, K=K, G=G, table_log=R)
        assert c.size == oracle.tans_container_bytes(w.size, K, G, int(c[16:24].view(np.uint64)[0]))
        assert c.size <= oracle.tans_max_container_bytes(w.size, K, G, R)
        assert np.array_equal(oracle.decode(c), w)


def test_tans_parameters_are_checked():
    w = inputs.gaussian(1000, 0.02, seed=3)
    for K, G, R in ((128, 32, 3), (128, 32, 13), (12, 32, 12), (5464, 32, 12), (128, 0, 12)):
        with pytest.raises(oracle.OracleError) as ei:
            oracle.encode_tans(w, K=K, G=G, table_log=R)
        assert ei.value.code == oracle.ERR_ARG, (K, G, R)
    oracle.encode_tans(w, K=5456, G=1, table_log=12)  # the largest K with (K + 1) R <= 65535


def test_tans_malformed_containers_are_rejected():
    w = inputs.gaussian(10_003, 0.02, seed=8)
    c = oracle.encode_tans(w, K=64)
    assert np.array_equal(oracle.decode(c), w)
    ng = int(c[44:48].view(np.uint32)[0])
    off_clen = (576 + 8 * (ng + 1) + 15) // 16 * 16
    off_m = int(c[48:56].view(np.uint64)[0])
    n = w.size
    off_stream = (off_m + n + 15) // 16 * 16
    bad = {}
    v = c.copy(); v[60] = 0; bad["coder"] = v  # read as a Huffman container: no valid code lengths
    v = c.copy(); v[56] = 13; bad["table_log"] = v
    used = int(np.flatnonzero(c[64:576:2])[0])
    v = c.copy(); v[64 + 2 * used] += 1; bad["freq_sum"] = v
    v = c.copy(); v[576 + 8] ^= 1; bad["gbase"] = v
    v = c.copy(); v[off_clen] ^= 1; bad["clen"] = v
    v = c.copy(); v[off_stream] ^= 0x80; bad["stream_bit"] = v  # the first chunk's state
    v = c.copy(); v[-1] = 1; bad["slack"] = v
    bad["truncated"] = c[:-1].copy()
    for name, b in bad.items():
        with pytest.raises(oracle.OracleError) as ei:
            oracle.decode(b)
        assert ei.value.code == oracle.ERR_CORRUPT, name


def test_tans_chunk_codes_brute_force():
    """For a fixed 16-state table, the chunk codes of every sequence of a given length
    (3 symbols, lengths 1..5: up to 243 sequences) are distinct and prefix-free, as any
    decodable code must be; each code's length is R plus, per symbol s, between
    R - floor(log2(2f-1)) and R - floor(log2 f) bits (the state number k lies in
    [f, 2f) and a step emits R - floor(log2 k) bits); with the dyadic table f = (8, 4, 4)
    every symbol costs exactly its -log2(f / M) bits."""
    R = 4
    for freqs in ({1: 8, 2: 5, 3: 3}, {1: 8, 2: 4, 3: 4}, {1: 14, 2: 1, 3: 1}):
        f = np.zeros(256, dtype=np.uint32)
        for s_, v in freqs.items():
            f[s_] = v
        lo = {s_: R - int(math.floor(math.log2(2 * v - 1))) for s_, v in freqs.items()}
        hi = {s_: R - int(math.floor(math.log2(v))) for s_, v in freqs.items()}
        for L in range(1, 6):
            codes = {}
            for seq in itertools.product(sorted(freqs), repeat=L):
                c = oracle.tans_encode_chunk(f, np.array(seq, dtype=np.uint8), R)
                assert R + sum(lo[x] for x in seq) <= len(c) <= R + sum(hi[x] for x in seq), (freqs, seq, c)
                codes[seq] = c
            vals = sorted(codes.values())
            assert len(set(vals)) == len(vals)
            assert all(not b.startswith(a) for a, b in zip(vals, vals[1:])), (freqs, L)
            if freqs == {1: 8, 2: 4, 3: 4}:
                assert all(len(c) == R + sum(1 if x == 1 else 2 for x in seq) for seq, c in codes.items())
