"""Pins for the CPU oracle: each test checks the oracle against something
other than itself -- hand-derived golden streams, closed forms, brute force,
an independent dynamic program, float semantics, textbook bounds, and the
identity the method guarantees (lossless: decode(encode(x)) == x, "70% Size,
100% Accuracy ... (DFloat11)", Abstract)."""
import itertools
import math

import numpy as np
import pytest
import torch

from conftest import read_golden
from entropy_decoding_b200 import synth


def _hexbytes(s):
    return np.array([int(t, 16) for t in s.split()], np.uint8)


def _symmap(s):
    out = {}
    for t in s.split():
        k, v = t.split(":")
        out[int(k)] = int(v)
    return out


# ----------------------------------------------------------------- golden

@pytest.mark.parametrize("name,nsym", [("bf16_tiny.txt", 256), ("e4m3_tiny.txt", 16)])
def test_golden_hand_example(oracle_mod, name, nsym):
    g = read_golden(name)
    dt = g["dtype"]
    vals = np.array([float(v) for v in g["values"].split()], np.float32)
    if dt == "bf16":
        bits = np.array([int(t, 16) for t in g["bits"].split()], np.uint16)
        assert np.array_equal(synth.to_bf16_bits(vals), bits)  # values <-> stored patterns
    else:
        bits = _hexbytes(g["bits"])
        assert np.array_equal(synth.to_e4m3_bits(vals), bits)
    exps, plane = oracle_mod.split(bits, dt)
    assert exps.tolist() == [int(v) for v in g["exponents"].split()]
    assert np.array_equal(plane, _hexbytes(g["plane"]))

    c = oracle_mod.compress(bits, dt, chunk_bits=int(g["chunk_bits"]),
                            tile_threads=int(g["tile_threads"]))
    want_len = _symmap(g["lengths"])
    for s in range(nsym):
        assert c.lengths[s] == want_len.get(s, 0), s
    want_code = _symmap(g["codes"])
    for s, code in want_code.items():
        assert c.codes[s] == code
    assert c.total_bits == int(g["total_bits"])
    assert np.array_equal(c.stream, _hexbytes(g["stream"]))
    assert np.array_equal(c.gaps, _hexbytes(g["gaps"]))
    assert c.out_off.tolist() == [int(v) for v in g["out_off"].split()]
    assert c.max_span == int(g["max_span"])
    assert np.array_equal(oracle_mod.decompress(c), bits)


# ----------------------------------------------------------------- fields

def test_bf16_fields_match_float_semantics(oracle_mod):
    """For normal BF16 values, the exponent symbol e satisfies
    2^(e-127) <= |x| < 2^(e-126) and the raw field is sign*128 + fraction*128."""
    g = np.random.default_rng(1)
    x = (g.standard_normal(5000) * 10.0 ** g.uniform(-6, 6, 5000)).astype(np.float32)
    bits = synth.to_bf16_bits(x)
    xb = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy().astype(np.float64)
    exps, plane = oracle_mod.split(bits, "bf16")
    m, e = np.frexp(np.abs(xb))  # |x| = m * 2^e, m in [0.5, 1)
    assert np.array_equal(exps.astype(np.int64), e.astype(np.int64) - 1 + 127)
    frac = np.rint((2 * m - 1.0) * 128).astype(np.int64)
    sign = (xb < 0).astype(np.int64)
    assert np.array_equal(plane.astype(np.int64), sign * 128 + frac)


def test_e4m3_fields_match_float_semantics(oracle_mod):
    bits = synth.all_e4m3_patterns()
    xv = torch.from_numpy(bits.copy()).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    exps, plane = oracle_mod.split(bits, "e4m3")
    for i in range(256):
        v = xv[i]
        if not np.isfinite(v) or v == 0:
            continue
        a = abs(v)
        if a >= 2.0 ** -6:  # normal: |x| = (1 + m/8) 2^(e-7)
            e = math.floor(math.log2(a))
            assert exps[i] == e + 7
            mant = round((a / 2.0 ** e - 1.0) * 8)
        else:  # subnormal: |x| = m/8 * 2^-6, exponent field 0
            assert exps[i] == 0
            mant = round(a / 2.0 ** -6 * 8)
        nib = (plane[i // 2] >> (4 * (i % 2))) & 0xF
        assert nib == ((8 if v < 0 else 0) | mant)


# ----------------------------------------------------------------- code lengths

def _cost(counts, lengths):
    return sum(int(c) * int(l) for c, l in zip(counts, lengths))


def _kraft_is_one(lengths):
    return sum(1 << (32 - int(l)) for l in lengths if l > 0) == 1 << 32


def _brute_force_min_cost(counts):
    """Minimum sum f*l over all length vectors with Kraft sum <= 1."""
    m = len(counts)
    best = None
    for ls in itertools.product(range(1, m), repeat=m):
        if sum(2.0 ** -l for l in ls) <= 1.0 + 1e-12:
            c = _cost(counts, ls)
            best = c if best is None or c < best else best
    return best


def test_lengths_optimal_brute_force(oracle_mod):
    g = np.random.default_rng(7)
    for trial in range(120):
        m = int(g.integers(2, 7))
        counts = g.integers(1, 9, m).astype(np.uint64)
        full = np.zeros(256, np.uint64)
        syms = g.choice(256, m, replace=False)
        full[syms] = counts
        lengths = oracle_mod.code_lengths(full, 256, 32)
        assert _cost(counts, lengths[syms]) == _brute_force_min_cost(counts.tolist()), (counts, syms)
        assert _kraft_is_one(lengths[syms])
        assert np.all(lengths[np.setdiff1d(np.arange(256), syms)] == 0)


def _entropy(counts):
    p = counts[counts > 0].astype(np.float64)
    p /= p.sum()
    return float(-(p * np.log2(p)).sum())


def test_lengths_within_entropy_bound(oracle_mod):
    """H <= mean length < H + 1 for an unlimited Huffman code (textbook)."""
    for seed, make in [(0, lambda s: synth.single_matrix(s)[0].tensors[0].bits),
                       (1, lambda s: synth.powers_of_two_bf16([3, 9, 27, 81, 243, 729, 2187], seed=s)),
                       (2, lambda s: synth.random_bits(50000, "bf16", s))]:
        x = make(seed)
        exps, _ = oracle_mod.split(x, "bf16")
        counts = oracle_mod.histogram(exps)
        d, _ = oracle_mod.huffman_depth(counts, 256)
        assert d <= 32
        lengths = oracle_mod.code_lengths(counts, 256, 32)
        mean = _cost(counts, lengths) / counts.sum()
        h = _entropy(counts)
        assert h - 1e-12 <= mean < h + 1.0
        assert _kraft_is_one(lengths[counts > 0])


def test_closed_form_dyadic(oracle_mod):
    """Counts proportional to 2^-k give lengths -log2 p and mean length = H."""
    counts = np.zeros(256, np.uint64)
    probs = [1, 2, 3, 4, 5, 6, 6]  # 2^-1 .. 2^-6, 2^-6
    syms = [120, 7, 200, 33, 64, 250, 1]
    for s, k in zip(syms, probs):
        counts[s] = 2 ** (6 - k) * 10
    lengths = oracle_mod.code_lengths(counts, 256, 32)
    assert [int(lengths[s]) for s in syms] == probs
    assert math.isclose(_cost(counts, lengths) / counts.sum(), _entropy(counts), rel_tol=0, abs_tol=1e-12)


def test_closed_form_two_symbols_and_single(oracle_mod):
    c = np.zeros(256, np.uint64)
    c[[3, 200]] = [1000, 1]
    l = oracle_mod.code_lengths(c, 256, 32)
    assert l[3] == 1 and l[200] == 1 and l.sum() == 2
    c = np.zeros(256, np.uint64)
    c[77] = 5
    l = oracle_mod.code_lengths(c, 256, 32)
    assert l[77] == 1 and l.sum() == 1
    assert oracle_mod.code_lengths(np.zeros(256, np.uint64), 256, 32).sum() == 0


def test_closed_form_geometric(oracle_mod):
    """Counts 2^(k-1), ..., 2, 1, 1: lengths 1, 2, ..., k-1, k-1."""
    k = 12
    counts = np.zeros(256, np.uint64)
    vals = [2 ** (k - 1 - i) for i in range(k - 1)] + [1]
    for i, v in enumerate(vals):
        counts[10 + i] = v
    l = oracle_mod.code_lengths(counts, 256, 32)
    assert [int(l[10 + i]) for i in range(k)] == list(range(1, k)) + [k - 1]


def test_closed_form_uniform_is_identity(oracle_mod):
    """All 65 536 BF16 patterns: every exponent has the same count, so every
    length is 8, the canonical code is the identity and the stream equals the
    exponent bytes.  Same for all 256 E4M3 patterns with 4-bit codes."""
    x = synth.all_bf16_patterns()
    c = oracle_mod.compress(x, "bf16")
    assert np.all(c.lengths == 8)
    assert np.array_equal(c.codes, np.arange(256))
    exps, _ = oracle_mod.split(x, "bf16")
    assert np.array_equal(c.stream, exps)
    y = synth.all_e4m3_patterns()
    c = oracle_mod.compress(y, "e4m3")
    assert np.all(c.lengths == 4)
    assert np.array_equal(c.codes, np.arange(16))
    e, _ = oracle_mod.split(y, "e4m3")
    packed = (e[0::2] << 4) | e[1::2]  # two 4-bit codes per byte, first in the high half
    assert np.array_equal(c.stream, packed)


def _dp_length_limited_cost(counts, max_len):
    """Optimal cost of a prefix code with lengths <= max_len, by a dynamic
    program over depths (heavier symbols never get longer codes): state =
    (symbols placed, free nodes at this depth)."""
    w = sorted((int(c) for c in counts if c > 0), reverse=True)
    m = len(w)
    pre = [0]
    for v in w:
        pre.append(pre[-1] + v)
    INF = float("inf")
    from functools import lru_cache

    @lru_cache(maxsize=None)
    def best(d, i, a):
        if i == m:
            return 0
        if d > max_len or a == 0:
            return INF
        r = INF
        for k in range(0, min(a, m - i) + 1):
            nxt = min(2 * (a - k), m - i - k)
            if nxt == 0 and i + k < m:
                continue
            sub = best(d + 1, i + k, nxt) if i + k < m else 0
            r = min(r, d * (pre[i + k] - pre[i]) + sub)
        return r

    return best(1, 0, 2)


def test_fibonacci_forces_length_limit(oracle_mod):
    """Fibonacci counts F1..F34 give an unlimited Huffman depth of 33; the
    limited code must reach exactly 32, be complete, and cost what the
    independent dynamic program says is optimal."""
    fib = synth.fibonacci_counts(34)
    counts = np.zeros(256, np.uint64)
    counts[100:134] = fib
    d, _ = oracle_mod.huffman_depth(counts, 256)
    assert d == 33
    l = oracle_mod.code_lengths(counts, 256, 32)
    assert int(l.max()) == 32
    assert _kraft_is_one(l[counts > 0])
    assert _cost(counts, l) == _dp_length_limited_cost(counts, 32)
    # tighter limits too (still pinned by the same dynamic program)
    for lim in (12, 16, 20):
        l = oracle_mod.code_lengths(counts, 256, lim)
        assert int(l.max()) <= lim and _kraft_is_one(l[counts > 0])
        assert _cost(counts, l) == _dp_length_limited_cost(counts, lim)


def test_dp_agrees_with_brute_force_on_tiny():
    g = np.random.default_rng(3)
    for _ in range(40):
        m = int(g.integers(2, 6))
        counts = g.integers(1, 9, m).tolist()
        assert _dp_length_limited_cost(counts, 32) == _brute_force_min_cost(counts)


# ----------------------------------------------------------------- canonical codes

def test_canonical_codes_are_kraft_partial_sums(oracle_mod):
    """In (length, symbol) order, each left-justified code equals the Kraft
    sum of all earlier codes -- the defining property of a canonical code --
    and no code is a prefix of another."""
    g = np.random.default_rng(5)
    for _ in range(30):
        m = int(g.integers(2, 200))
        counts = np.zeros(256, np.uint64)
        syms = g.choice(256, m, replace=False)
        counts[syms] = (g.pareto(1.2, m) * 10 + 1).astype(np.uint64)
        l = oracle_mod.code_lengths(counts, 256, 32)
        codes = oracle_mod.canonical_codes(l)
        order = sorted(syms.tolist(), key=lambda s: (int(l[s]), s))
        acc = 0
        for s in order:
            assert int(codes[s]) << (32 - int(l[s])) == acc
            acc += 1 << (32 - int(l[s]))
        assert acc == 1 << 32
        for a, b in itertools.combinations(order[:40], 2):
            la, lb = int(l[a]), int(l[b])
            short, long_, ls, ll = (a, b, la, lb) if la <= lb else (b, a, lb, la)
            assert (int(codes[long_]) >> (ll - ls)) != int(codes[short])


# ----------------------------------------------------------------- aux variables

@pytest.mark.parametrize("chunk_bits,tile_threads", [(128, 256), (64, 128), (32, 8), (256, 4)])
def test_aux_matches_independent_walk(oracle_mod, chunk_bits, tile_threads):
    x = synth.heavy_tail_matrix(0)[0].tensors[0].bits[:300000]
    c = oracle_mod.compress(x, "bf16", chunk_bits=chunk_bits, tile_threads=tile_threads)
    exps, _ = oracle_mod.split(x, "bf16")
    lens = c.lengths[exps].astype(np.int64)
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]])
    total = int(lens.sum())
    assert total == c.total_bits
    n_chunks = -(-total // chunk_bits)
    n_tiles = -(-n_chunks // tile_threads)
    assert c.n_tiles == n_tiles and len(c.gaps) == n_tiles * tile_threads
    c0 = np.arange(n_chunks, dtype=np.int64) * chunk_bits
    idx = np.searchsorted(starts, c0, side="left")
    first = np.where(idx < len(starts), starts[np.minimum(idx, len(starts) - 1)], total)
    assert np.array_equal(c.gaps[:n_chunks].astype(np.int64), first - c0)
    assert np.all(c.gaps[n_chunks:] == 0)
    assert int(c.gaps.max()) <= int(c.lengths.max()) - 1
    b0 = np.arange(n_tiles + 1, dtype=np.int64) * chunk_bits * tile_threads
    assert np.array_equal(c.out_off.astype(np.int64), np.searchsorted(starts, b0, side="left"))
    assert int(c.out_off[-1]) == x.size
    assert c.max_span == int(np.diff(c.out_off.astype(np.int64)).max())


@pytest.mark.parametrize("chunk_bits,tile_threads", [(128, 32), (64, 128), (32, 8), (128, 256)])
def test_chunk_counts_match_independent_tally(oracle_mod, chunk_bits, tile_threads):
    """Codes per chunk against a tally of the code start positions by chunk
    (np.bincount over start // chunk_bits), and each tile's sum against
    out_off's difference (a second walk of the oracle, over tile bounds)."""
    x = synth.heavy_tail_matrix(0)[0].tensors[0].bits[:300000]
    c = oracle_mod.compress(x, "bf16", chunk_bits=chunk_bits, tile_threads=tile_threads)
    exps, _ = oracle_mod.split(x, "bf16")
    got = oracle_mod.chunk_counts(exps, c.lengths, chunk_bits, tile_threads)
    assert len(got) == c.n_tiles * tile_threads
    lens = c.lengths[exps].astype(np.int64)
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]])
    want = np.bincount(starts // chunk_bits, minlength=len(got))
    assert np.array_equal(got.astype(np.int64), want)
    sums = got.astype(np.int64).reshape(-1, tile_threads).sum(axis=1)
    assert np.array_equal(sums, np.diff(c.out_off.astype(np.int64)))
    n_chunks = -(-c.total_bits // chunk_bits)
    assert np.all(got[n_chunks:] == 0) and np.all(got[: n_chunks - 1] > 0)


def test_chunk_counts_closed_form_one_bit_codes(oracle_mod):
    """A constant tensor has one symbol, coded with 1 bit: chunk c holds
    min(chunk_bits, n - c * chunk_bits) codes.  At 256-bit chunks a full chunk
    holds 256 codes, more than a byte: the oracle refuses."""
    n = 1000
    x = synth.constant_bf16(n, 1.0)
    exps, _ = oracle_mod.split(x, "bf16")
    lengths = oracle_mod.build_lengths([x], "bf16")
    assert int(lengths.max()) == 1
    for cb_bits, tt in [(64, 4), (128, 32), (32, 8)]:
        got = oracle_mod.chunk_counts(exps, lengths, cb_bits, tt).astype(np.int64)
        n_chunks = -(-n // cb_bits)
        want = np.zeros(len(got), np.int64)
        want[:n_chunks] = cb_bits
        want[n_chunks - 1] = n - (n_chunks - 1) * cb_bits
        assert np.array_equal(got, want)
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.chunk_counts(exps, lengths, 256, 4)


def test_decode_at_sampled_positions(oracle_mod):
    x = synth.single_matrix(3)[0].tensors[0].bits[:100000]
    c = oracle_mod.compress(x, "bf16")
    exps, _ = oracle_mod.split(x, "bf16")
    lens = c.lengths[exps].astype(np.int64)
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]])
    for j in [0, 1, 777, 50000, 99990]:
        got = oracle_mod.decode_at(c, int(starts[j]), min(10, x.size - j))
        assert np.array_equal(got, exps[j:j + 10])


# ----------------------------------------------------------------- round trips

@pytest.mark.parametrize("case", ["all_bf16", "normal", "heavy", "single", "fib", "random",
                                  "empty", "one", "seven", "eight", "e4m3_all", "e4m3_normal"])
def test_roundtrip_identity(oracle_mod, case):
    dt = "bf16"
    if case == "all_bf16":
        x = synth.all_bf16_patterns()
    elif case == "normal":
        x = synth.single_matrix(0)[0].tensors[0].bits
    elif case == "heavy":
        x = synth.heavy_tail_matrix(0)[0].tensors[0].bits[:1 << 20]
    elif case == "single":
        x = synth.constant_bf16(10000, 0.0)
    elif case == "fib":
        x = synth.powers_of_two_bf16(synth.fibonacci_counts(26), first_exponent=-20)
    elif case == "random":
        x = synth.random_bits(70001, "bf16", 1)
    elif case == "empty":
        x = np.zeros(0, np.uint16)
    elif case == "one":
        x = synth.constant_bf16(1, -3.5)
    elif case == "seven":
        x = synth.random_bits(7, "bf16", 2)
    elif case == "eight":
        x = synth.random_bits(8, "bf16", 3)
    elif case == "e4m3_all":
        dt, x = "e4m3", synth.all_e4m3_patterns()
    else:
        dt = "e4m3"
        ss = np.random.SeedSequence(0).spawn(1)[0]
        x = synth.normal_e4m3(ss, 100003)
    c = oracle_mod.compress(x, dt)
    assert c.max_span <= 128 * 256  # at most one code per stream bit of a tile
    assert np.array_equal(oracle_mod.decompress(c), x)


def test_compressed_size_and_entropy_near_pages(oracle_mod):
    """Gaussian BF16 weights: exponent entropy about 2.5-3 bits ("about
    three" informative exponent bits, "Compressing LLMs without Compromise",
    "Where the redundancy lives") and a container near 70% of BF16 ("70% Size",
    DFloat11 title and Abstract)."""
    x = synth.single_matrix(0)[0].tensors[0].bits
    c = oracle_mod.compress(x, "bf16")
    exps, _ = oracle_mod.split(x, "bf16")
    h = _entropy(oracle_mod.histogram(exps))
    assert 2.3 < h < 3.0
    size = c.stream.size + c.plane.size + c.gaps.size + 8 * c.out_off.size + 256
    assert 0.62 < size / (2 * x.size) < 0.75
