"""Host side of the library (code construction, encoder, container, device
image) against the CPU oracle and against independent recomputation.  No GPU
needed: nothing here launches a kernel."""
import ctypes
import struct

import numpy as np
import pytest

from entropy_decoding_b200 import synth


@pytest.fixture(scope="module")
def df11():
    from entropy_decoding_b200 import build
    build.build()
    from entropy_decoding_b200 import df11 as mod
    return mod


def test_library_exports_every_declared_symbol(df11):
    names = df11.exported_names()
    assert len(names) >= 20
    lib = ctypes.CDLL(df11.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert df11.df11_version() == 10000


def test_check_library_exports_the_same_symbols(df11):
    """The bounds-checked build (kernels compiled with -DDF11_CHECK=1) is a
    drop-in twin of libdf11.so: same C-ABI, same version."""
    from entropy_decoding_b200 import build
    path = build.build(check=True)
    lib = ctypes.CDLL(path)
    for n in df11.exported_names():
        assert hasattr(lib, n), n
    lib.df11_version.restype = ctypes.c_int
    assert lib.df11_version() == 10000


def test_library_choice_from_the_environment(df11):
    """DF11_LIBRARY picks the library at import: 'check' loads the
    bounds-checked twin, anything unknown is refused."""
    import os
    import subprocess
    import sys
    from entropy_decoding_b200 import build
    build.build(check=True)
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = "from entropy_decoding_b200 import df11; print(df11.CHECKED, os.path.basename(df11.LIB_PATH))"
    for var, want in (("check", "True libdf11_check.so"), ("normal", "False libdf11.so"), ("", "False libdf11.so")):
        env = dict(os.environ, DF11_LIBRARY=var)
        r = subprocess.run([sys.executable, "-c", "import os; " + code], cwd=root, env=env, capture_output=True,
                           text=True, timeout=300)
        assert r.returncode == 0 and r.stdout.strip() == want, (var, r.stdout, r.stderr[-500:])
    r = subprocess.run([sys.executable, "-c", "import entropy_decoding_b200.df11"], cwd=root,
                       env=dict(os.environ, DF11_LIBRARY="bogus"), capture_output=True, text=True, timeout=300)
    assert r.returncode != 0 and "DF11_LIBRARY" in r.stderr


def _cases():
    return {
        "normal": ("bf16", lambda: synth.single_matrix(0)[0].tensors[0].bits[:400000]),
        "heavy": ("bf16", lambda: synth.heavy_tail_matrix(0)[0].tensors[0].bits[:600000]),
        "all_bf16": ("bf16", synth.all_bf16_patterns),
        "single": ("bf16", lambda: synth.constant_bf16(50000, 1.0)),
        "fib": ("bf16", lambda: synth.powers_of_two_bf16(synth.fibonacci_counts(28), first_exponent=-24)),
        "random": ("bf16", lambda: synth.random_bits(123457, "bf16", 4)),
        "tiny": ("bf16", lambda: synth.random_bits(9, "bf16", 5)),
        "e4m3": ("e4m3", lambda: synth.normal_e4m3(np.random.SeedSequence(1), 300001)),
        "e4m3_all": ("e4m3", synth.all_e4m3_patterns),
    }


@pytest.mark.parametrize("case", list(_cases()))
def test_lengths_and_sections_match_oracle(df11, oracle_mod, case):
    dt, make = _cases()[case]
    x = make()
    cb = df11.df11_build_codebook(dt, [x])
    want = oracle_mod.build_lengths([x], dt)
    assert np.array_equal(cb.lengths(), want)
    for chunk_bits, tile_threads in [(128, 32), (128, 256), (64, 512), (256, 128)]:
        blob = df11.df11_encode(cb, x, chunk_bits, tile_threads)
        o = oracle_mod.compress(x, dt, lengths=want, chunk_bits=chunk_bits, tile_threads=tile_threads)
        info = blob.info()
        s = blob.sections()
        assert info.total_bits == o.total_bits
        assert info.n_tiles == o.n_tiles
        assert info.max_span == o.max_span
        assert np.array_equal(s["stream"], o.stream)
        assert np.array_equal(s["plane"], o.plane)
        assert np.array_equal(s["gaps"], o.gaps)
        assert np.array_equal(s["out_off"], o.out_off)
        exps, _ = oracle_mod.split(x, dt)
        if chunk_bits <= 128:  # counts are stored up to 128-bit chunks
            assert np.array_equal(s["counts"], oracle_mod.chunk_counts(exps, want, chunk_bits, tile_threads))
        else:
            assert s["counts"] is None
        assert df11.df11_encode(cb, x, chunk_bits, tile_threads, chunk_counts=False).sections()["counts"] is None


def test_shared_codebook_over_a_group(df11, oracle_mod):
    g = synth.transformer_block(0)[0]
    xs = [t.bits[: 100000 + 1000 * i] for i, t in enumerate(g.tensors)]
    cb = df11.df11_build_codebook("bf16", xs)
    assert np.array_equal(cb.lengths(), oracle_mod.build_lengths(xs, "bf16"))


def test_length_limit_matches_oracle(df11, oracle_mod):
    x = synth.powers_of_two_bf16(synth.fibonacci_counts(30), first_exponent=-25)
    for lim in (32, 20, 12, 9):
        cb = df11.df11_build_codebook("bf16", [x], lim)
        want = oracle_mod.build_lengths([x], "bf16", lim)
        assert np.array_equal(cb.lengths(), want), lim
        assert cb.lengths().max() <= lim


def test_fibonacci_34_reaches_32_bit_codes(df11, oracle_mod):
    """The 34-symbol Fibonacci histogram (unlimited depth 33) through the
    library: package-merge lengths equal the oracle's, longest code 32."""
    counts = np.zeros(256, np.uint64)
    counts[100:134] = synth.fibonacci_counts(34)
    want = oracle_mod.code_lengths(counts, 256, 32)
    assert want.max() == 32
    cb = df11.df11_codebook_from_lengths("bf16", want)
    assert np.array_equal(cb.lengths(), want)


def _image_layout(img: bytes):
    magic = img[:8]
    assert magic == b"DF11IMG1"
    dtype, chunk, tile, n_luts, fsm_rows, flags = struct.unpack_from("<6I", img, 8)
    n, total, n_tiles, max_span = struct.unpack_from("<4Q", img, 32)
    keys = ["meta", "syms", "lut", "fsm", "gaps", "counts", "out_off", "stream", "plane", "total"]
    lay = dict(zip(keys, struct.unpack_from("<10Q", img, 64)))
    return dict(dtype=dtype, chunk=chunk, tile=tile, n_luts=n_luts, fsm_rows=fsm_rows, flags=flags, n=n,
                total_bits=total, n_tiles=n_tiles, max_span=max_span, **lay)


def _image(df11, blob):
    n = blob.info().device_bytes
    buf = np.zeros(n, np.uint8)
    df11.df11_blob_device_image(blob, buf.ctypes.data, n)
    return buf


def _prefix_decoder(lengths, codes):
    table = {}
    for s, l in enumerate(lengths):
        if l:
            table[(int(l), int(codes[s]))] = s
    return table


def _first_code(table, bits, nbits):
    """(symbol, length) of the code at the top of a `nbits`-bit value, or None."""
    for l in range(1, nbits + 1):
        v = bits >> (nbits - l)
        if (l, v) in table:
            return table[(l, v)], l
    return None


@pytest.mark.parametrize("case", ["normal", "heavy", "fib", "single", "e4m3"])
def test_decode_tables_match_independent_prefix_decode(df11, oracle_mod, case):
    """The device image's 12-bit multi-symbol table and hierarchical 256-entry
    tables, checked entry by entry against a dictionary prefix decode over the
    oracle's canonical codes."""
    dt, make = _cases()[case]
    x = make()
    cb = df11.df11_build_codebook(dt, [x])
    blob = df11.df11_encode(cb, x)
    img = _image(df11, blob)
    lay = _image_layout(img.tobytes()[:256])
    lengths = oracle_mod.build_lengths([x], dt)
    codes = oracle_mod.canonical_codes(lengths)
    table = _prefix_decoder(lengths, codes)
    meta = img[lay["meta"]:lay["meta"] + 16384].view(np.uint32)
    syms = img[lay["syms"]:lay["syms"] + 16384].view(np.uint32)
    for v in range(4096):
        pos, got, starts = 0, [], 0
        while len(got) < 4:
            r = _first_code(table, v & ((1 << (12 - pos)) - 1), 12 - pos) if pos < 12 else None
            if r is None:
                break
            starts |= 1 << pos
            got.append(r[0])
            pos += r[1]
        if not got:
            assert meta[v] == 0x400, v
        else:
            assert meta[v] == pos | (len(got) << 11) | (starts << 20), v
            assert [(int(syms[v]) >> (8 * i)) & 0xFF for i in range(len(got))] == got
    lut = img[lay["lut"]:lay["lut"] + lay["n_luts"] * 512].view(np.uint16)
    rng = np.random.default_rng(0)
    wins = list(rng.integers(0, 2 ** 32, 3000, dtype=np.uint64))
    for s, l in enumerate(lengths):  # every codeword at least once, random tail
        if l:
            wins.append((int(codes[s]) << (32 - int(l))) | int(rng.integers(0, 2 ** (32 - int(l)))))
    for win in wins:
        win = int(win)
        e = int(lut[win >> 24])
        lvl = 1
        while e & 0x8000 and lvl < 4:
            e = int(lut[(e & 0x7FFF) * 256 + ((win >> (24 - 8 * lvl)) & 0xFF)])
            lvl += 1
        r = _first_code(table, win, 32)
        if r is None:
            assert e & 0x4000
        else:
            assert not e & 0xC000
            assert (e & 0xFF, (e >> 8) & 0x3F) == r


def _tree_rows(lengths, codes, max_rows=64):
    """Internal nodes of the code tree as (depth, prefix) in the row order the
    transition tables use: the root first, then decreasing probability mass
    below the node (a code of length l weighs 2^-l), then depth, then prefix.
    The last row is the dead row; returns (nodes of the live rows, rows)."""
    mass = {}
    for s, l in enumerate(lengths):
        l = int(l)
        for d in range(l):
            key = (d, int(codes[s]) >> (l - d))
            mass[key] = mass.get(key, 0.0) + 2.0 ** -l
    nodes = sorted(mass, key=lambda k: (k != (0, 0), -mass[k], k[0], k[1]))
    live = nodes[:max_rows - 1]
    return live, len(live) + 1


@pytest.mark.parametrize("case", ["normal", "heavy", "fib", "single", "e4m3", "random"])
def test_transition_tables_match_independent_prefix_decode(df11, oracle_mod, case):
    """Every entry of the byte-step transition tables in the device image:
    starting from the row's tree node, the 8 bits of the byte are decoded with
    a dictionary prefix decoder over the oracle's canonical codes; the entry
    must list the codes that end in the byte (end mask, count, first four
    symbols) and lead to the row of the node the byte stops on, or to the dead
    row when that node has no row, more than four codes end or a prefix is no
    codeword."""
    dt, make = _cases()[case]
    x = make()
    cb = df11.df11_build_codebook(dt, [x])
    img = _image(df11, df11.df11_encode(cb, x))
    lay = _image_layout(img.tobytes()[:256])
    lengths = oracle_mod.build_lengths([x], dt)
    codes = oracle_mod.canonical_codes(lengths)
    table = _prefix_decoder(lengths, codes)
    live, rows = _tree_rows(lengths, codes)
    assert lay["fsm_rows"] == rows
    row_of = {node: r for r, node in enumerate(live)}
    dead = rows - 1
    fsm = img[lay["fsm"]:lay["fsm"] + rows * 2048].view(np.uint32).reshape(rows, 256, 2)
    assert np.all(fsm[dead, :, 0] == dead << 11) and np.all(fsm[dead, :, 1] == 0)
    for r, (depth, prefix) in enumerate(live):
        for b in range(256):
            bits, nbits = (prefix << 8) | b, depth + 8
            pos, ends, got = 0, 0, []
            while pos < nbits:
                hit = None
                for l in range(1, nbits - pos + 1):
                    if (l, (bits >> (nbits - pos - l)) & ((1 << l) - 1)) in table:
                        hit = l
                        break
                if hit is None:
                    break
                got.append(table[(hit, (bits >> (nbits - pos - hit)) & ((1 << hit) - 1))])
                pos += hit
                ends |= 1 << (pos - depth - 1)
            # the leftover bits: a node with a row, a node without one, or a
            # prefix of no codeword (the last two lead to the dead row)
            rest = nbits - pos
            node = (rest, bits & ((1 << rest) - 1))
            nxt = dead if (len(got) > 4 or node not in row_of) else row_of[node]
            ctl, sy = int(fsm[r, b, 0]), int(fsm[r, b, 1])
            assert ctl & 0xFF == ends, (r, b)
            assert (ctl >> 11) & 0x3F == nxt, (r, b)
            assert ctl >> 29 == min(len(got), 7), (r, b)
            assert ctl & 0x1FFE0700 == 0, (r, b)
            assert sy == sum(s << (8 * i) for i, s in enumerate(got[:4])), (r, b)


def test_serialize_roundtrip_and_size(df11, oracle_mod):
    x = synth.single_matrix(2)[0].tensors[0].bits
    cb = df11.df11_build_codebook("bf16", [x])
    blob = df11.df11_encode(cb, x)
    data = df11.df11_serialize(blob)
    info = blob.info()
    assert len(data) == info.serialized_bytes == blob.compressed_bytes()
    # near the pages' ~70% of BF16 ("70% Size", DFloat11 title / Abstract)
    assert 0.62 < info.serialized_bytes / info.uncompressed_bytes < 0.72
    b2 = df11.df11_deserialize(data)
    s1, s2 = blob.sections(), b2.sections()
    for k in s1:
        assert np.array_equal(s1[k], s2[k])
    assert np.array_equal(b2.lengths(), blob.lengths())
    assert df11.df11_serialize(b2) == data
    assert struct.unpack_from("<I", data, 8)[0] == 2  # version 2: with chunk counts
    # without counts: version 1, the pages' sections only, smaller by the counts
    bare = df11.df11_encode(cb, x, chunk_counts=False)
    d1 = df11.df11_serialize(bare)
    assert struct.unpack_from("<II", d1, 8)[0] == 1 and struct.unpack_from("<I", d1, 60)[0] == 0
    assert 0 < len(data) - len(d1) <= info.counts_bytes + 16
    b1 = df11.df11_deserialize(d1)
    assert b1.sections()["counts"] is None and b1.info().counts_bytes == 0
    assert df11.df11_serialize(b1) == d1
    assert b1.compressed_bytes() == len(d1)


def _container_offsets(info, counts: bool):
    """Section offsets of a serialized blob: 64-byte header, 256 code lengths,
    then gaps, counts (version 2), out_off, each 16-byte aligned."""
    up = lambda v: (v + 15) // 16 * 16
    gaps = up(64 + 256)
    cnt = up(gaps + info.gaps_bytes)
    oo = up(cnt + (info.gaps_bytes if counts else 0))
    return gaps, cnt, oo


def test_deserialize_rejects_corruption(df11):
    x = synth.heavy_tail_matrix(0)[0].tensors[0].bits[:200000]
    cb = df11.df11_build_codebook("bf16", [x])
    blob = df11.df11_encode(cb, x)
    good = bytearray(df11.df11_serialize(blob))
    info = blob.info()

    def rejected(buf):
        with pytest.raises(df11.Df11Error) as e:
            df11.df11_deserialize(bytes(buf))
        assert e.value.status == df11.DF11_ECORRUPT

    rejected(good[:-16])                       # truncated
    bad = bytearray(good); bad[0] ^= 1; rejected(bad)          # magic
    bad = bytearray(good); bad[8] = 9; rejected(bad)           # version
    bad = bytearray(good); bad[16] ^= 1; rejected(bad)         # element count
    lengths_off = 64
    bad = bytearray(good); bad[lengths_off + 120] = 1; rejected(bad)  # Kraft sum > 1
    gaps_off, cnt_off, oo = _container_offsets(info, True)
    bad = bytearray(good); bad[gaps_off + 3] = 200; rejected(bad)     # gap out of range
    bad = bytearray(good); struct.pack_into("<Q", bad, oo + 8 * 2, 0); rejected(bad)  # out_off not monotone
    bad = bytearray(good); struct.pack_into("<Q", bad, oo, 5); rejected(bad)          # out_off[0] != 0
    # chunk counts: a tile whose counts no longer add up to its span, a count
    # above the chunk's bits, a count in a padding chunk
    bad = bytearray(good); bad[cnt_off + 5] += 1; rejected(bad)
    bad = bytearray(good)
    excess = 200 - bad[cnt_off + 5]
    bad[cnt_off + 5] = 200  # keep the tile's sum: take the excess from the chunks after it
    for j in range(6, 32):
        take = min(excess, bad[cnt_off + j])
        bad[cnt_off + j] -= take
        excess -= take
    assert excess == 0
    rejected(bad)
    n_chunks = -(-info.total_bits // info.chunk_bits)
    if n_chunks < info.gaps_bytes:
        bad = bytearray(good); bad[cnt_off + info.gaps_bytes - 1] = 1; rejected(bad)
    # flags: none allowed in version 1, no unknown ones in version 2
    bad = bytearray(good); struct.pack_into("<I", bad, 60, 3); rejected(bad)
    bare = bytearray(df11.df11_serialize(df11.df11_encode(cb, x, chunk_counts=False)))
    bad = bytearray(bare); struct.pack_into("<I", bad, 60, 1); rejected(bad)
    _, _, oo1 = _container_offsets(info, False)
    bad = bytearray(bare); struct.pack_into("<Q", bad, oo1, 5); rejected(bad)
    with pytest.raises(df11.Df11Error):
        df11.df11_deserialize(b"")


def test_encode_rejects_uncovered_symbol(df11):
    x = synth.single_matrix(0)[0].tensors[0].bits[:1000]
    cb = df11.df11_build_codebook("bf16", [x])
    y = x.copy()
    y[5] = 0x7F80  # +inf: exponent 255, absent from the code
    with pytest.raises(df11.Df11Error) as e:
        df11.df11_encode(cb, y)
    assert e.value.status == df11.DF11_EINVAL


def test_invalid_arguments(df11):
    with pytest.raises(df11.Df11Error):
        df11.df11_build_codebook("bf16", [np.zeros(4, np.uint16)], 40)
    with pytest.raises(df11.Df11Error):
        df11.df11_codebook_from_lengths("bf16", np.full(256, 1, np.uint8))  # Kraft sum 128
    cb = df11.df11_build_codebook("bf16", [synth.random_bits(100, "bf16")])
    with pytest.raises(df11.Df11Error):
        df11.df11_encode(cb, synth.random_bits(100, "bf16"), chunk_bits=96)
    assert df11.df11_layout_supported("bf16", 128, 256)
    assert df11.df11_layout_supported("e4m3", 128, 256)
    assert not df11.df11_layout_supported("bf16", 96, 256)


def test_decode_argument_checks_need_no_gpu(df11):
    """Bad launch options and bad streamed-decode arguments are refused
    before any CUDA call (these run without a GPU)."""
    x = synth.random_bits(5000, "bf16", 3)
    cb = df11.df11_build_codebook("bf16", [x])
    blob = df11.df11_encode(cb, x)
    for kw in ({"walker": 3}, {"walker": -1}, {"overlap": 2}, {"max_ctas": -1}, {"warps_per_cta": -4},
               {"chunks_per_thread": -1}, {"diag_expire_waits": 2}):
        with pytest.raises(df11.Df11Error) as e:
            df11.df11_decode_ex([blob], [0x1000], None, 0, **kw)
        assert e.value.status == df11.DF11_EINVAL, kw
    need = (blob.info().device_bytes + 255) // 256 * 256
    fake = 0x10000  # never dereferenced: every check below fails first
    with pytest.raises(df11.Df11Error) as e:  # a group's images do not fit the slot
        df11.df11_decode_streamed([[blob]], [fake], [fake], need - 256, [fake])
    assert e.value.status == df11.DF11_ENOMEM
    with pytest.raises(df11.Df11Error) as e:  # more than 8 slots
        df11.df11_decode_streamed([[blob]], [fake], [fake] * 9, need, [fake])
    assert e.value.status == df11.DF11_EINVAL
    with pytest.raises(df11.Df11Error) as e:  # misaligned slot
        df11.df11_decode_streamed([[blob]], [fake], [fake + 16], need, [fake])
    assert e.value.status == df11.DF11_EINVAL
    other = df11.df11_encode(df11.df11_build_codebook("bf16", [synth.random_bits(5000, "bf16", 4)]),
                             synth.random_bits(5000, "bf16", 4))
    with pytest.raises(df11.Df11Error) as e:  # two codes in one group
        df11.df11_decode_streamed([[blob, other]], [fake, fake], [fake], 4 * need, [fake, fake])
    assert e.value.status == df11.DF11_EINVAL
    with pytest.raises(df11.Df11Error) as e:  # more than 64 blobs in a group
        df11.df11_decode_streamed([[blob] * 65], [fake] * 65, [fake], need * 65, [fake] * 65)
    assert e.value.status == df11.DF11_EINVAL


def test_device_image_layout(df11):
    x = synth.random_bits(300000, "bf16", 9)
    cb = df11.df11_build_codebook("bf16", [x])
    blob = df11.df11_encode(cb, x)
    img = _image(df11, blob)
    lay = _image_layout(img.tobytes()[:256])
    info = blob.info()
    assert lay["total"] == info.device_bytes == img.size
    for k in ("meta", "syms", "lut", "fsm", "gaps", "counts", "out_off", "stream", "plane"):
        assert lay[k] % 256 == 0
    assert lay["gaps"] - lay["fsm"] >= lay["fsm_rows"] * 2048
    # the gaps section keeps 16 zero bytes after the last tile's gaps
    ng = info.n_tiles * info.tile_threads
    assert lay["counts"] - lay["gaps"] >= ng + 16
    assert not img[lay["gaps"] + ng: lay["gaps"] + ng + 16].any()
    # chunk counts (default layout): one byte per chunk, as the blob holds them
    s = blob.sections()
    assert lay["flags"] == 1 and info.counts_bytes == ng
    assert lay["out_off"] - lay["counts"] >= ng
    assert np.array_equal(img[lay["counts"]:lay["counts"] + ng], s["counts"])
    # without them the section is empty and the flag clear
    bare = df11.df11_encode(cb, x, chunk_counts=False)
    lay0 = _image_layout(_image(df11, bare).tobytes()[:256])
    assert lay0["flags"] == 0 and lay0["counts"] == lay0["out_off"] and bare.info().counts_bytes == 0
    assert bare.sections()["counts"] is None
    assert bare.info().device_bytes < info.device_bytes
    tile_bytes = info.chunk_bits // 8 * info.tile_threads
    stream = img[lay["stream"]:lay["plane"]]
    words = stream[: (stream.size // 4) * 4].reshape(-1, 4)[:, ::-1].reshape(-1)  # back to MSB-first bytes
    assert np.array_equal(words[: s["stream"].size], s["stream"])
    assert stream.size >= info.n_tiles * tile_bytes + 16
    assert not words[s["stream"].size:].any()
    assert np.array_equal(img[lay["plane"]:lay["plane"] + info.plane_bytes], s["plane"])
    assert lay["total"] - lay["plane"] >= info.plane_bytes + 32


@pytest.mark.parametrize("k,n", [(64, 128), (192, 384), (4096, 1024)])
def test_gemm_tile_order_matches_oracle(df11, oracle_mod, k, n):
    """The library's operand-tile permutation (host) against the oracle's."""
    w = np.random.default_rng(k * n).integers(0, 1 << 16, k * n, dtype=np.uint16)
    assert np.array_equal(df11.df11_gemm_tile_weights(w, k, n), oracle_mod.gemm_tile(w, k, n))
    with pytest.raises(df11.Df11Error):
        df11.df11_gemm_tile_weights(w[: (k - 1) * n], k - 1, n)
