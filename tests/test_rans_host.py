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


def _group_for_container(df11):
    g0 = synth.transformer_block(4)[0]
    xs = [g0.tensors[0].bits[:70001], np.zeros(0, np.uint16), g0.tensors[4].bits[:50003]]
    return xs, df11.df11_rans_encode_group("bf16", xs, 4096)


def test_container_roundtrip(df11):
    xs, g = _group_for_container(df11)
    data = df11.df11_rans_group_serialize(g)
    g2 = df11.df11_rans_group_deserialize(data)
    assert g2.n_tensors == 3 and g2.dtype == "bf16"
    assert np.array_equal(g2.freqs(), g.freqs())
    for i in range(3):
        a, b = g.sections(i), g2.sections(i)
        for k in a:
            assert np.array_equal(a[k], b[k]), (i, k)
    assert df11.df11_rans_group_serialize(g2) == data
    # header, frequencies, and per tensor a record plus its 16-byte aligned sections
    up = lambda v: (v + 15) // 16 * 16
    want = 64 + up(2 * 256)
    for i in range(3):
        inf = g.info(i)
        want += 32 + up(inf.n_tiles * 128) + up((inf.n_tiles + 1) * 8) + up(2 * inf.words) + up(inf.plane_bytes)
    assert len(data) == want


def test_container_e4m3_and_one_symbol(df11):
    for dt, x in [("e4m3", synth.normal_e4m3(np.random.SeedSequence(8), 30001)),
                  ("bf16", synth.constant_bf16(9000, 2.0))]:
        g = df11.df11_rans_encode_group(dt, [x], 1024)
        data = df11.df11_rans_group_serialize(g)
        g2 = df11.df11_rans_group_deserialize(data)
        assert np.array_equal(g2.freqs(), g.freqs())
        assert df11.df11_rans_group_serialize(g2) == data


def test_container_rejects_damage(df11):
    import struct
    xs, g = _group_for_container(df11)
    good = bytearray(df11.df11_rans_group_serialize(g))
    inf0 = g.info(0)
    rec0 = 64 + 512                         # first tensor's record
    states0 = rec0 + 32
    tw0 = states0 + (inf0.n_tiles * 128 + 15) // 16 * 16

    def rejected(buf):
        with pytest.raises(df11.Df11Error) as e:
            df11.df11_rans_group_deserialize(bytes(buf))
        assert e.value.status == df11.DF11_ECORRUPT

    rejected(good[:-16])                                                      # truncated
    rejected(good + b"\0" * 16)                                               # trailing bytes
    bad = bytearray(good); bad[0] ^= 1; rejected(bad)                         # magic
    bad = bytearray(good); struct.pack_into("<I", bad, 8, 2); rejected(bad)   # version
    f = g.freqs()
    s = int(np.flatnonzero(f)[0])
    bad = bytearray(good); struct.pack_into("<H", bad, 64 + 2 * s, int(f[s]) + 1); rejected(bad)  # sum 4097
    bad = bytearray(good); struct.pack_into("<I", bad, states0 + 4 * 3, 1000); rejected(bad)      # state < 2^16
    bad = bytearray(good); struct.pack_into("<Q", bad, tw0 + 8, 3); rejected(bad)                 # offset not a multiple of 8
    bad = bytearray(good); struct.pack_into("<Q", bad, rec0, inf0.n_elems + 5000); rejected(bad)  # tile count mismatch
