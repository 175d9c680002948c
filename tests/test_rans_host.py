"""The library's rANS encoder against the oracle's: frequencies and every
section byte-equal, groups sharing one table, argument checks.  No GPU."""
import numpy as np
import pytest

from entropy_decoding_b200 import synth


@pytest.fixture(scope="module")
def df11():
    from entropy_decoding_b200 import build
    build.build()
    from entropy_decoding_b200 import df11 as mod
    return mod


CASES = {
    "normal": ("bf16", lambda: synth.single_matrix(0)[0].tensors[0].bits[:300001]),
    "heavy": ("bf16", lambda: synth.heavy_tail_matrix(0)[0].tensors[0].bits[:250003]),
    "all_bf16": ("bf16", synth.all_bf16_patterns),
    "single": ("bf16", lambda: synth.constant_bf16(40000, 3.0)),
    "fib": ("bf16", lambda: synth.powers_of_two_bf16(synth.fibonacci_counts(26), first_exponent=-20)),
    "e4m3": ("e4m3", lambda: synth.normal_e4m3(np.random.SeedSequence(2), 200001)),
    "e4m3_all": ("e4m3", synth.all_e4m3_patterns),
    "tiny": ("bf16", lambda: synth.random_bits(5, "bf16", 1)),
}


@pytest.mark.parametrize("case", list(CASES))
@pytest.mark.parametrize("tile", [0, 64, 4096])
def test_sections_match_oracle(df11, oracle_mod, case, tile):
    dt, make = CASES[case]
    x = make()
    g = df11.df11_rans_encode_group(dt, [x], tile)
    ts = tile or df11.RANS_TILE_DEFAULT
    o = oracle_mod.rans_compress(x, dt, tile_symbols=ts)
    assert np.array_equal(g.freqs(), o.freqs)
    s = g.sections(0)
    assert np.array_equal(s["words"], o.words)
    assert np.array_equal(s["states"], o.states)
    assert np.array_equal(s["tile_words"], o.tile_words)
    assert np.array_equal(s["plane"], o.plane)
    inf = g.info(0)
    assert inf.coded_bytes == 2 * o.words.size + 4 * o.states.size + 8 * o.tile_words.size
    assert inf.n_tiles == len(o.tile_words) - 1


def test_group_shares_one_table(df11, oracle_mod):
    g0 = synth.transformer_block(1)[0]
    xs = [t.bits[: 120000 + 7 * i] for i, t in enumerate(g0.tensors)]
    g = df11.df11_rans_encode_group("bf16", xs, 2048)
    counts = sum(oracle_mod.histogram(oracle_mod.split(x, "bf16")[0]) for x in xs)
    freqs = oracle_mod.rans_freqs(counts[:256], 256)
    assert np.array_equal(g.freqs(), freqs)
    for i, x in enumerate(xs):
        o = oracle_mod.rans_compress(x, "bf16", freqs=freqs, tile_symbols=2048)
        s = g.sections(i)
        assert np.array_equal(s["words"], o.words) and np.array_equal(s["states"], o.states)


def test_rans_beats_huffman_size(df11):
    """On Gaussian weights the rANS payload is smaller than the Huffman
    container's stream and aux (its tiles carry 32 states, but no per-chunk
    gaps or counts and no rounding of code lengths to whole bits)."""
    x = synth.transformer_block(0)[0].tensors[0].bits
    cb = df11.df11_build_codebook("bf16", [x])
    h = df11.df11_encode(cb, x).info()
    huff = h.stream_bytes + h.gaps_bytes + h.counts_bytes + h.out_off_bytes
    r = df11.df11_rans_encode_group("bf16", [x]).info(0)
    assert r.coded_bytes < huff
    assert r.plane_bytes == h.plane_bytes


def test_invalid_arguments(df11):
    x = synth.random_bits(1000, "bf16", 2)
    with pytest.raises(df11.Df11Error):
        df11.df11_rans_encode_group("bf16", [x], 48)   # not a multiple of 32
    with pytest.raises(df11.Df11Error):
        df11.df11_rans_encode_group("bf16", [x], 16)   # below 32
    with pytest.raises(df11.Df11Error):
        df11.df11_rans_encode_group("bf16", [])
