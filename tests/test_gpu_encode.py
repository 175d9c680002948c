"""GPU encoder (histogram, bit packing, auxiliary variables on the device)
against the host encoder and the CPU oracle: the device image it writes must
be byte-identical to the one built from the host encoder's sections, its
histogram equal to the oracle's, and it must decode to the source."""
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


CASES = {
    "normal_1m": ("bf16", lambda: synth.single_matrix(0)[0].tensors[0].bits),
    "heavy": ("bf16", lambda: synth.heavy_tail_matrix(0)[0].tensors[0].bits[: 2 * 10 ** 6 + 3]),
    "all_bf16": ("bf16", synth.all_bf16_patterns),
    "single_symbol": ("bf16", lambda: synth.constant_bf16(100003, 0.0)),
    "fib26": ("bf16", lambda: synth.powers_of_two_bf16(synth.fibonacci_counts(26), first_exponent=-20)),
    "uniform": ("bf16", lambda: synth.random_bits(700001, "bf16", 1)),
    "tiny": ("bf16", lambda: synth.random_bits(17, "bf16", 2)),
    "e4m3_normal": ("e4m3", lambda: synth.normal_e4m3(np.random.SeedSequence(0), 1000003)),
    "e4m3_all": ("e4m3", synth.all_e4m3_patterns),
    "e4m3_tiny": ("e4m3", lambda: synth.random_bits(33, "e4m3", 3)),
}


def _dev(x):
    t = torch.from_numpy(x.view(np.int16) if x.dtype == np.uint16 else x.copy()).cuda()
    return t


def _image_of(df11, blob, nbytes):
    """Host copy of a GPU-encoded blob's device image."""
    keep = blob._keep
    off = (-keep.data_ptr()) % 256
    return keep[off:off + nbytes].cpu().numpy()


@pytest.mark.parametrize("case", list(CASES))
def test_histogram_matches_oracle(df11, oracle_mod, case):
    dt, make = CASES[case]
    x = make()
    counts = torch.zeros(256, dtype=torch.int64, device="cuda")
    xd = _dev(x)
    df11.df11_histogram_device(dt, xd.data_ptr(), x.size, counts.data_ptr())
    torch.cuda.synchronize()
    exps, _ = oracle_mod.split(x, dt)
    want = oracle_mod.histogram(exps)
    assert np.array_equal(counts.cpu().numpy().view(np.uint64), want)
    nsym = 256 if dt == "bf16" else 16
    cb = df11.df11_codebook_from_counts(dt, counts.cpu().numpy().view(np.uint64)[:nsym])
    assert np.array_equal(cb.lengths(), oracle_mod.build_lengths([x], dt))


@pytest.mark.parametrize("counts", [True, False])
@pytest.mark.parametrize("layout", [(128, 32), (128, 256), (64, 512), (256, 128)])
@pytest.mark.parametrize("case", list(CASES))
def test_device_image_equals_host_image(df11, case, layout, counts):
    """Byte-identical images from the GPU and host encoders, with and without
    the chunk-counts section (the GPU adds each thread's run of code starts
    per chunk into the section with atomics)."""
    dt, make = CASES[case]
    x = make()
    cb = df11.df11_build_codebook(dt, [x])
    host = df11.df11_encode(cb, x, *layout, chunk_counts=counts)
    n = host.info().device_bytes
    want = np.zeros(n, np.uint8)
    df11.df11_blob_device_image(host, want.ctypes.data, n)
    dev = df11.encode_on_device(cb, _dev(x), *layout, chunk_counts=counts)
    torch.cuda.synchronize()
    assert dev.info().device_bytes == n
    assert dev.info().max_span == host.info().max_span
    got = _image_of(df11, dev, n)
    diff = np.flatnonzero(got != want)
    assert diff.size == 0, f"{diff.size} bytes differ, first at {diff[:8]}"


@pytest.mark.parametrize("case", list(CASES))
def test_device_encoded_blob_decodes_and_fetches(df11, oracle_mod, case):
    dt, make = CASES[case]
    x = make()
    cb = df11.df11_build_codebook(dt, [x])
    blob = df11.encode_on_device(cb, _dev(x))
    out = df11.empty_output(blob)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.df11_decode([blob], [out.data_ptr()], err.data_ptr())
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(out.cpu().numpy()[: x.size * x.itemsize].view(x.dtype), x)
    with pytest.raises(df11.Df11Error):
        df11.df11_serialize(blob)  # host sections are not there before the fetch
    df11.df11_blob_fetch(blob)
    lengths = oracle_mod.build_lengths([x], dt)
    assert np.array_equal(cb.lengths(), lengths)
    o = oracle_mod.compress(x, dt, lengths=lengths, chunk_bits=128, tile_threads=32)
    sec = blob.sections()
    assert np.array_equal(sec["stream"], o.stream)
    assert np.array_equal(sec["plane"], o.plane)
    assert np.array_equal(sec["gaps"], o.gaps)
    assert np.array_equal(sec["out_off"], o.out_off)
    exps, _ = oracle_mod.split(x, dt)
    assert np.array_equal(sec["counts"], oracle_mod.chunk_counts(exps, lengths, 128, 32))
    assert df11.df11_serialize(blob) == df11.df11_serialize(df11.df11_encode(cb, x))


def test_device_encode_transformer_block_full_size(df11):
    """The block workload encoded on the GPU equals the host encoding and
    decodes in one launch."""
    g = synth.transformer_block(0)[0]
    xs = [t.bits for t in g.tensors]
    cb = df11.df11_build_codebook("bf16", xs)
    blobs = []
    for x in xs:
        b = df11.encode_on_device(cb, _dev(x))
        blobs.append(b)
    outs = [df11.empty_output(b) for b in blobs]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.df11_decode(blobs, [o.data_ptr() for o in outs], err.data_ptr())
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for x, o, b in zip(xs, outs, blobs):
        assert torch.equal(o[: 2 * x.size].view(torch.int16), _dev(x))
    host = df11.df11_encode(cb, xs[4])
    assert blobs[4].info().total_bits == host.info().total_bits
    assert blobs[4].info().max_span == host.info().max_span


def test_uncovered_symbol_rejected(df11):
    x = synth.single_matrix(0)[0].tensors[0].bits[:10000]
    cb = df11.df11_build_codebook("bf16", [x])
    y = x.copy()
    y[777] = 0x7F80  # +inf: exponent 255 has no code here
    with pytest.raises(df11.Df11Error) as e:
        df11.encode_on_device(cb, _dev(y))
    assert e.value.status == df11.DF11_EINVAL


def test_empty_tensor(df11):
    cb = df11.df11_build_codebook("bf16", [synth.random_bits(100, "bf16")])
    blob = df11.encode_on_device(cb, torch.zeros(8, dtype=torch.int16, device="cuda")[:0])
    assert blob.info().n_elems == 0 and blob.info().n_tiles == 0
