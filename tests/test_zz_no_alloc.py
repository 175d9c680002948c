"""df11_encode_device_noalloc (the GPU encoder whose scratch is a static
device array of the library) against the allocating GPU encoder
(df11_encode_device_begin/_end): byte-identical device images and result
fields on consecutive calls, decodes back to the source, and the documented
error cases.  The file name sorts last so that it also runs after every other
GPU test in the same process; it must pass alone as well."""
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


def _dev(x):
    return torch.from_numpy(x.view(np.int16) if x.dtype == np.uint16 else x.copy()).cuda()


def _aligned(nbytes):
    """A 256-byte aligned device buffer of nbytes (torch owns the memory)."""
    buf = torch.empty(nbytes + 256, dtype=torch.uint8, device="cuda")
    off = (-buf.data_ptr()) % 256
    return buf, buf.data_ptr() + off, off


def _reference_image(df11, cb, xd, chunk_bits, tile_threads, counts=True):
    """Image and info from the allocating GPU encoder."""
    blob = df11.encode_on_device(cb, xd, chunk_bits, tile_threads, chunk_counts=counts)
    torch.cuda.synchronize()
    info = blob.info()
    keep = blob._keep
    off = (-keep.data_ptr()) % 256
    return blob, info, keep[off:off + info.device_bytes].cpu().numpy()


def _noalloc_image(df11, cb, xd, chunk_bits, tile_threads, cap, counts=True):
    buf, ptr, off = _aligned(cap)
    r = df11.df11_encode_device_noalloc(cb, xd.data_ptr(), xd.numel(), chunk_bits, tile_threads, ptr, cap,
                                        chunk_counts=counts)
    return buf, ptr, r, buf[off:off + r.image_bytes].cpu().numpy()


def _check_against_reference(df11, dt, x, chunk_bits=128, tile_threads=32, counts=True):
    cb = df11.df11_build_codebook(dt, [x])
    xd = _dev(x)
    blob, info, want = _reference_image(df11, cb, xd, chunk_bits, tile_threads, counts)
    buf, ptr, r, got = _noalloc_image(df11, cb, xd, chunk_bits, tile_threads, info.device_bytes + 4096, counts)
    assert r.image_bytes == info.device_bytes
    assert r.total_bits == info.total_bits
    assert r.n_tiles == info.n_tiles
    assert r.max_span == info.max_span
    diff = np.flatnonzero(got != want)
    assert diff.size == 0, f"{diff.size} bytes differ, first at {diff[:8]}"
    return cb, buf, ptr, r


CALLS = [
    ("bf16", lambda: synth.single_matrix(0)[0].tensors[0].bits, 128, 32),
    ("bf16", lambda: synth.heavy_tail_matrix(1)[0].tensors[0].bits[: 3 * 10 ** 6 + 5], 128, 256),
    ("e4m3", lambda: synth.normal_e4m3(np.random.SeedSequence(4), 2 * 10 ** 6 + 7), 128, 32),
    ("bf16", lambda: synth.random_bits(4099, "bf16", 5), 64, 512),
]


def test_two_calls_in_a_row_match_allocating_encoder(df11):
    """Consecutive calls, a large input then a small one, each byte-equal to
    the allocating encoder: nothing left in the static scratch by the first
    call leaks into the second."""
    for dt, make, cbits, tt in CALLS[:2]:
        _check_against_reference(df11, dt, make(), cbits, tt)


def test_every_call_in_sequence_matches(df11):
    for dt, make, cbits, tt in CALLS + CALLS[::-1]:
        _check_against_reference(df11, dt, make(), cbits, tt)


def test_without_chunk_counts_matches(df11):
    """The layout without the chunk-counts section, after a call with it."""
    x = synth.heavy_tail_matrix(3)[0].tensors[0].bits[: 2 * 10 ** 6 + 9]
    _check_against_reference(df11, "bf16", x)
    _check_against_reference(df11, "bf16", x, counts=False)


def test_same_input_twice_gives_same_image(df11):
    x = synth.single_matrix(2)[0].tensors[0].bits[: 10 ** 6 + 1]
    cb = df11.df11_build_codebook("bf16", [x])
    xd = _dev(x)
    info = df11.df11_encode(cb, x).info()
    imgs = []
    for _ in range(2):
        _, _, r, img = _noalloc_image(df11, cb, xd, 128, 32, info.device_bytes)
        assert r.image_bytes == info.device_bytes and r.max_span == info.max_span
        imgs.append(img)
    assert np.array_equal(imgs[0], imgs[1])


def test_noalloc_image_decodes(df11):
    """A host-encoded blob (same codebook and layout) bound to the no-alloc
    image decodes to the source: the image is what the decoder expects."""
    x = synth.transformer_block(0)[0].tensors[0].bits
    cb, buf, ptr, r = _check_against_reference(df11, "bf16", x)
    host = df11.df11_encode(cb, x)
    df11.df11_blob_bind(host, ptr, r.image_bytes, keep=buf)
    out = df11.empty_output(host)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.df11_decode([host], [out.data_ptr()], err.data_ptr())
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(out[: 2 * x.size].view(torch.int16), _dev(x))


def test_size_limit_rejected_before_any_work(df11):
    cb = df11.df11_build_codebook("bf16", [synth.random_bits(1000, "bf16")])
    src = torch.zeros(16, dtype=torch.int16, device="cuda")
    buf, ptr, _ = _aligned(4096)
    with pytest.raises(df11.Df11Error) as e:
        df11.df11_encode_device_noalloc(cb, src.data_ptr(), df11.NOALLOC_MAX_ELEMS + 1, 128, 32, ptr, 4096)
    assert e.value.status == df11.DF11_EINVAL


def test_image_too_small_reports_size(df11):
    x = synth.random_bits(50000, "bf16", 6)
    cb = df11.df11_build_codebook("bf16", [x])
    need = df11.df11_encode(cb, x).info().device_bytes
    xd = _dev(x)
    buf, ptr, _ = _aligned(need)
    with pytest.raises(df11.Df11Error) as e:
        df11.df11_encode_device_noalloc(cb, xd.data_ptr(), x.size, 128, 32, ptr, need - 1)
    assert e.value.status == df11.DF11_ENOMEM
    assert e.value.result.image_bytes == need
    _check_against_reference(df11, "bf16", x)


def test_uncovered_symbol_then_clean_call(df11):
    """An input with an exponent the code does not cover is rejected, and the
    flag it raised in the scratch does not fail the next, valid call."""
    x = synth.single_matrix(0)[0].tensors[0].bits[:20000]
    cb = df11.df11_build_codebook("bf16", [x])
    y = x.copy()
    y[1234] = 0x7F80  # +inf: exponent 255 has no code here
    yd = _dev(y)
    buf, ptr, _ = _aligned(1 << 20)
    with pytest.raises(df11.Df11Error) as e:
        df11.df11_encode_device_noalloc(cb, yd.data_ptr(), y.size, 128, 32, ptr, 1 << 20)
    assert e.value.status == df11.DF11_EINVAL
    _check_against_reference(df11, "bf16", x)


def test_empty_input(df11):
    cb = df11.df11_build_codebook("bf16", [synth.random_bits(100, "bf16")])
    src = torch.zeros(8, dtype=torch.int16, device="cuda")
    need = df11.df11_encode(cb, np.zeros(0, np.uint16)).info().device_bytes  # header and decode tables
    buf, ptr, _ = _aligned(need)
    r = df11.df11_encode_device_noalloc(cb, src.data_ptr(), 0, 128, 32, ptr, need)
    assert r.n_tiles == 0 and r.total_bits == 0 and r.max_span == 0
    assert r.image_bytes == need


def test_call_takes_no_device_memory(df11):
    """The defining property: once the first call on the device has looked up
    the static scratch, a further call of several MB changes neither the
    device's free memory nor torch's allocation counters (every buffer it
    uses is allocated, and counted, before the measurement)."""
    x = synth.heavy_tail_matrix(5)[0].tensors[0].bits[: 6 * 10 ** 6 + 3]
    cb = df11.df11_build_codebook("bf16", [x])
    xd = _dev(x)
    need = df11.df11_encode(cb, x).info().device_bytes
    buf, ptr, _ = _aligned(need)
    r0 = df11.df11_encode_device_noalloc(cb, xd.data_ptr(), x.size, 128, 32, ptr, need)  # warm-up
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    stats0 = torch.cuda.memory_stats()
    r1 = df11.df11_encode_device_noalloc(cb, xd.data_ptr(), x.size, 128, 32, ptr, need)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    stats1 = torch.cuda.memory_stats()
    assert free1 == free0
    for k in ("allocation.all.allocated", "segment.all.allocated", "reserved_bytes.all.current"):
        assert stats1.get(k) == stats0.get(k), k
    assert (r1.image_bytes, r1.total_bits, r1.max_span) == (r0.image_bytes, r0.total_bits, r0.max_span)
