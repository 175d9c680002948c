"""Pins of the oracle's rANS coder (the ANS variant of the exponent code,
"Approaching Shannon Bound with Lossless LLM Weight Compression", Abstract).
Hand-derived states and words, closed forms, the information content of the
output and the page's distance to the Shannon limit; round trips on
adversarial inputs.  CPU only."""
import numpy as np
import pytest

from entropy_decoding_b200 import synth

M, L = 4096, 65536


def test_freqs_hand_examples(oracle_mod):
    q = oracle_mod.rans_freqs
    assert list(q(np.array([3, 1]), 2)) == [3072, 1024]                # exact quarters
    assert list(q(np.array([1, 1, 1]), 3)) == [1366, 1365, 1365]       # floor 1365 each, +1 to symbol 0
    assert list(q(np.array([0, 5, 0, 0]), 4)) == [0, 4096, 0, 0]       # one symbol takes the whole range
    assert list(q(np.array([1, 2, 0]), 3)) == [1365, 2731, 0]          # floor 1365/2730, +1 to the larger count
    # one dominant symbol and 255 rare ones: 4095 + 255 forced ones = 4350,
    # the excess 254 comes off the only symbol above 1
    counts = np.array([10 ** 9] + [1] * 255)
    f = q(counts, 256)
    assert f[0] == 3841 and (f[1:] == 1).all()


def test_freqs_sum_and_support(oracle_mod):
    rng = np.random.default_rng(3)
    for nsym in (16, 256):
        for _ in range(50):
            c = rng.integers(0, 10 ** rng.integers(1, 9), nsym).astype(np.uint64)
            c[rng.random(nsym) < 0.3] = 0
            if c.sum() == 0:
                continue
            f = oracle_mod.rans_freqs(c, nsym)
            assert int(f.sum()) == M
            assert ((f > 0) == (c > 0)).all()


def test_one_symbol_per_coder_hand_derived(oracle_mod):
    """Three symbols in a 32-symbol tile, freqs [3072, 1024]: coders 0-2 code
    one symbol each from 2^16 without moving a word:
    s=0: floor(65536/3072)*4096 + 65536 mod 3072 + 0 = 86016 + 1024 = 87040;
    s=1: 64*4096 + 0 + 3072 = 265216.  The other coders keep 2^16."""
    words, states, tw = oracle_mod.rans_encode(np.array([0, 1, 0], np.uint8), np.array([3072, 1024]), 32)
    assert words.size == 0 and list(tw) == [0, 0]
    assert list(states[:3]) == [87040, 265216, 87040] and (states[3:] == L).all()


def test_word_emission_and_order_hand_derived(oracle_mod):
    """Uniform frequencies (16 each over 256 symbols): coding b from 2^16 gives
    2^24 + 16 b; coding a next moves the low word 16 b out (the state has
    reached 16 << 20) and gives 2^16 + 16 a.  With 34 symbols, coders 0 and 1
    each code two; the words come out in decode order: step 0, coder 0 then
    coder 1, padded to 8."""
    f = np.full(256, 16)
    e = (np.arange(34) * 37 + 11) % 256
    words, states, tw = oracle_mod.rans_encode(e.astype(np.uint8), f, 64)
    assert list(words) == [16 * e[32], 16 * e[33], 0, 0, 0, 0, 0, 0]
    assert list(tw) == [0, 8]
    assert states[0] == L + 16 * e[0] and states[1] == L + 16 * e[1]
    assert all(states[j] == (1 << 24) + 16 * e[j] for j in range(2, 32))


def test_closed_form_single_symbol(oracle_mod):
    x = synth.constant_bf16(100001, -0.75)
    c = oracle_mod.rans_compress(x, "bf16", tile_symbols=4096)
    assert c.words.size == 0 and (c.states == L).all()
    assert np.array_equal(oracle_mod.rans_decompress(c), x)


def test_closed_form_uniform_code(oracle_mod):
    """All 65,536 BF16 patterns: every exponent 256 times, frequency 16 each,
    8 bits a symbol, so each coder moves one word per two symbols."""
    x = synth.all_bf16_patterns()
    c = oracle_mod.rans_compress(x, "bf16", tile_symbols=4096)
    assert (c.freqs == 16).all()
    tiles = len(c.tile_words) - 1
    for t in range(tiles):
        n_t = min(4096, x.size - 4096 * t)
        per_lane = [len(range(j, n_t, 32)) for j in range(32)]
        want = sum(k // 2 for k in per_lane)
        got = int(c.tile_words[t + 1] - c.tile_words[t])
        assert want <= got < want + 8
    assert np.array_equal(oracle_mod.rans_decompress(c), x)


@pytest.mark.parametrize("tile", [4096, 16384])
def test_information_content_and_shannon_gap(oracle_mod, tile):
    """The words and final states hold the symbols' information: 16 bits per
    word plus log2(state) - 16 per coder equals the sum of log2(M / f_s) to
    within 0.01 bit per symbol (the coder's rounding).  Against the empirical
    entropy, words + states + tile offsets stay within 0.1 bit per symbol at
    16384-symbol tiles (the page's 0.01-0.1 bits of the Shannon limit)."""
    x = synth.single_matrix(1)[0].tensors[0].bits
    c = oracle_mod.rans_compress(x, "bf16", tile_symbols=tile)
    exps, _ = oracle_mod.split(x, "bf16")
    cost = np.log2(M / c.freqs[exps].astype(np.float64)).sum()
    real_words = 0
    for t in range(len(c.tile_words) - 1):
        seg = c.words[int(c.tile_words[t]):int(c.tile_words[t + 1])]
        real_words += int(c.tile_words[t + 1] - c.tile_words[t])
    held = 16.0 * real_words + (np.log2(c.states.astype(np.float64)) - 16.0).sum()
    assert abs(held - cost) / x.size < 0.01 + 16.0 * 8 * (len(c.tile_words) - 1) / x.size
    h = np.bincount(exps, minlength=256).astype(np.float64)
    p = h[h > 0] / x.size
    entropy = -(p * np.log2(p)).sum()
    total = 16 * c.words.size + 32 * c.states.size + 64 * len(c.tile_words)
    if tile == 16384:
        assert total / x.size - entropy < 0.1
    assert np.array_equal(oracle_mod.rans_decompress(c), x)


RT = {
    "all_bf16": ("bf16", synth.all_bf16_patterns),
    "all_e4m3": ("e4m3", synth.all_e4m3_patterns),
    "heavy": ("bf16", lambda: synth.heavy_tail_matrix(0)[0].tensors[0].bits[:300007]),
    "fib": ("bf16", lambda: synth.powers_of_two_bf16(synth.fibonacci_counts(26), first_exponent=-20)),
    "random": ("bf16", lambda: synth.random_bits(70001, "bf16", 7)),
    "e4m3_normal": ("e4m3", lambda: synth.normal_e4m3(np.random.SeedSequence(5), 100003)),
    "one": ("bf16", lambda: synth.random_bits(1, "bf16", 8)),
    "thirty_three": ("bf16", lambda: synth.random_bits(33, "bf16", 9)),
    "empty": ("bf16", lambda: np.zeros(0, np.uint16)),
}


@pytest.mark.parametrize("case", list(RT))
@pytest.mark.parametrize("tile", [64, 2048])
def test_roundtrip(oracle_mod, case, tile):
    dt, make = RT[case]
    x = make()
    c = oracle_mod.rans_compress(x, dt, tile_symbols=tile)
    assert np.array_equal(oracle_mod.rans_decompress(c), x)
    assert (c.tile_words % 8 == 0).all() and len(c.tile_words) == -(-x.size // tile) + 1


def test_decoder_refuses_damaged_data(oracle_mod):
    x = synth.single_matrix(2)[0].tensors[0].bits[:50000]
    c = oracle_mod.rans_compress(x, "bf16", tile_symbols=4096)
    bad = c.states.copy()
    bad[5] ^= 1 << 20
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.rans_decode(c.words, bad, c.tile_words, c.n, c.freqs, c.tile_symbols)
