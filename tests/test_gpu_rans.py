"""GPU decode of the rANS exponent coder: element by element against the
oracle's decoder and the source, ragged sizes, groups in one launch, the
full-size block, damaged data (flagged, guards intact)."""
import struct

import numpy as np
import pytest
import torch

from entropy_decoding_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def df11():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from entropy_decoding_b200 import build
    build.build()
    from entropy_decoding_b200 import df11 as mod
    return mod


def _decode(df11, g, xs, guard=64):
    """Uploads the group, decodes it in one launch into guarded buffers:
    (outputs as numpy bit arrays, error word, guards intact)."""
    df11.rans_upload(g)
    bufs, views = [], []
    for x in xs:
        nbytes = x.size * x.itemsize
        buf = torch.full((nbytes + 2 * guard,), 0xA5, dtype=torch.uint8, device="cuda")
        bufs.append(buf)
        views.append(buf[guard:guard + nbytes])
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.df11_rans_decode(g, [v.data_ptr() for v in views], err.data_ptr(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    outs, ok = [], True
    for x, buf, v in zip(xs, bufs, views):
        outs.append(v.cpu().numpy().view(x.dtype))
        h = buf.cpu().numpy()
        ok &= bool((h[:guard] == 0xA5).all() and (h[guard + v.numel():] == 0xA5).all())
    return outs, int(err.item()), ok


CASES = {
    "normal": ("bf16", lambda: synth.single_matrix(0)[0].tensors[0].bits),
    "heavy": ("bf16", lambda: synth.heavy_tail_matrix(0)[0].tensors[0].bits[: 2 * 10 ** 6 + 3]),
    "all_bf16": ("bf16", synth.all_bf16_patterns),
    "single": ("bf16", lambda: synth.constant_bf16(100003, 0.0)),
    "fib": ("bf16", lambda: synth.powers_of_two_bf16(synth.fibonacci_counts(26), first_exponent=-20)),
    "random": ("bf16", lambda: synth.random_bits(700001, "bf16", 1)),
    "e4m3": ("e4m3", lambda: synth.normal_e4m3(np.random.SeedSequence(0), 1000003)),
    "e4m3_all": ("e4m3", synth.all_e4m3_patterns),
}


@pytest.mark.parametrize("tile", [0, 64, 4096])
@pytest.mark.parametrize("case", list(CASES))
def test_parity(df11, oracle_mod, case, tile):
    dt, make = CASES[case]
    x = make()
    g = df11.df11_rans_encode_group(dt, [x], tile)
    (out,), err, ok = _decode(df11, g, [x])
    assert err == 0 and ok
    assert np.array_equal(out, x)
    o = oracle_mod.rans_compress(x, dt, tile_symbols=tile or df11.RANS_TILE_DEFAULT)
    assert np.array_equal(out, oracle_mod.rans_decompress(o))


@pytest.mark.parametrize("n", [1, 2, 31, 32, 33, 255, 256, 257, 511, 513, 4095, 16383, 16385, 40000])
@pytest.mark.parametrize("dt", ["bf16", "e4m3"])
def test_ragged_sizes(df11, oracle_mod, dt, n):
    x = synth.random_bits(n, dt, n) if n < 40 else (
        synth.single_matrix(n)[0].tensors[0].bits[:n] if dt == "bf16" else synth.normal_e4m3(np.random.SeedSequence(n), n))
    g = df11.df11_rans_encode_group(dt, [x])
    (out,), err, ok = _decode(df11, g, [x])
    assert err == 0 and ok and np.array_equal(out, x)


def test_group_in_one_launch(df11):
    """The matrices of a block (ragged lengths, an empty one) in one launch
    with one table; runs of tiles cross tensor boundaries."""
    g0 = synth.transformer_block(2)[0]
    xs = [t.bits[: t.bits.size // 16 + 17 * i] for i, t in enumerate(g0.tensors)]
    xs.insert(3, np.zeros(0, np.uint16))
    g = df11.df11_rans_encode_group("bf16", xs, 2048)
    outs, err, ok = _decode(df11, g, xs)
    assert err == 0 and ok
    for x, o in zip(xs, outs):
        assert np.array_equal(o, x)


def test_full_size_block(df11, oracle_mod):
    g0 = synth.transformer_block(0)[0]
    xs = [t.bits for t in g0.tensors]
    g = df11.df11_rans_encode_group("bf16", xs)
    outs, err, ok = _decode(df11, g, xs)
    assert err == 0 and ok
    for x, o in zip(xs, outs):
        assert np.array_equal(o, x)
    o = oracle_mod.rans_compress(xs[0], "bf16", freqs=g.freqs())
    assert np.array_equal(outs[0], oracle_mod.rans_decompress(o))


def test_damaged_data_flagged(df11):
    x = synth.single_matrix(7)[0].tensors[0].bits
    g = df11.df11_rans_encode_group("bf16", [x], 4096)
    n_tiles = g.info(0).n_tiles
    states_at = 16384
    tw_at = (states_at + n_tiles * 128 + 255) // 256 * 256
    for what in ("state", "offset"):
        dev = df11.rans_upload(g)
        base = (-dev.data_ptr()) % 256
        if what == "state":
            dev[base + states_at + 4 * 37 + 2] ^= 0x10
        else:
            dev[base + tw_at + 8 * 2: base + tw_at + 8 * 3] = torch.tensor(
                np.frombuffer(struct.pack("<Q", 10 ** 12), np.uint8), device="cuda")
        guard = 64
        nbytes = 2 * x.size
        buf = torch.full((nbytes + 2 * guard,), 0xA5, dtype=torch.uint8, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        df11.df11_rans_decode(g, [buf.data_ptr() + guard], err.data_ptr(), torch.cuda.current_stream().cuda_stream)
        torch.cuda.synchronize()
        e = int(err.item())
        h = buf.cpu().numpy()
        assert (h[:guard] == 0xA5).all() and (h[guard + nbytes:] == 0xA5).all()
        assert e & (df11.DEV_ERR_SPAN if what == "state" else df11.DEV_ERR_AUX)
        # damaged data never sends an access outside its buffer or section
        # (checked access by access in the bounds-checked library)
        assert not e & df11.DEV_ERR_BOUNDS
    # the same group uploaded again decodes exactly
    (out,), err, ok = _decode(df11, g, [x])
    assert err == 0 and ok and np.array_equal(out, x)


def test_launch_shape(df11):
    x = synth.heavy_tail_matrix(0)[0].tensors[0].bits
    g = df11.df11_rans_encode_group("bf16", [x])
    df11.rans_upload(g)
    grid, block, smem = df11.df11_rans_decode_launch_shape(g)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert block == 1024 and 0 < smem <= 227 * 1024
    assert grid == min(sms, -(-g.info(0).n_tiles // 32))


def test_group_from_its_container_decodes(df11):
    """Serialize, read back, upload, decode: the container is enough."""
    g0 = synth.transformer_block(5)[0]
    xs = [g0.tensors[1].bits[:300001], g0.tensors[5].bits[:200003]]
    g = df11.df11_rans_encode_group("bf16", xs, 4096)
    g2 = df11.df11_rans_group_deserialize(df11.df11_rans_group_serialize(g))
    outs, err, ok = _decode(df11, g2, xs)
    assert err == 0 and ok
    for x, o in zip(xs, outs):
        assert np.array_equal(o, x)
