"""GPU parity: the sm_100a decode kernel, called through the C-ABI, against the
CPU oracle, element by element (bit-exact: the method is lossless, "70% Size,
100% Accuracy ... (DFloat11)", Abstract: bit-for-bit identical outputs)."""
import numpy as np
import pytest
import torch

from entropy_decoding_b200 import synth
from gpu_util import decode_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def df11():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from entropy_decoding_b200 import build
    build.build()
    from entropy_decoding_b200 import df11 as mod
    return mod


def _roundtrip(df11, oracle_mod, x, dt, chunk_bits=128, tile_threads=32, max_len=0, check_oracle=True, cpt=0,
               ctas=0, wpc=0, walker=0, counts="stored"):
    """counts: "stored" (default encoding and decode), "walk" (counts stored,
    the decode told to count with a walk) or "absent" (encoded without)."""
    cb = df11.df11_build_codebook(dt, [x], max_len)
    blob = df11.df11_encode(cb, x, chunk_bits, tile_threads, chunk_counts=counts != "absent")
    cw = 1 if counts == "walk" else 0
    (out,), err, guards = decode_gpu(df11, [blob], chunks_per_thread=cpt, ctas_per_sm=ctas, warps_per_cta=wpc,
                                     walker=walker, count_walk=cw)
    assert err == 0
    assert guards
    if x.size:
        # the byte-step walk reads the stored counts exactly when they are there and not declined
        shape = df11.df11_decode_launch_shape([blob], cpt, ctas, wpc, walker, with_walk=True, count_walk=cw)
        stored = counts == "stored" and chunk_bits <= 128 and shape[3] == df11.WALKER_BYTE_STEP
        assert shape[4] == int(stored)
    assert out.shape == x.shape
    assert np.array_equal(out, x)
    if check_oracle:
        # the oracle builds its own code (lossless either way; equal lengths are pinned on the CPU)
        o = oracle_mod.compress(x, dt, max_len=max_len or 32, chunk_bits=chunk_bits, tile_threads=tile_threads)
        assert np.array_equal(out, oracle_mod.decompress(o))
    return blob


SMALL = {
    "normal_1m": ("bf16", lambda: synth.single_matrix(0)[0].tensors[0].bits),
    "heavy_2m": ("bf16", lambda: synth.heavy_tail_matrix(0)[0].tensors[0].bits[: 2 * 10 ** 6 + 3]),
    "all_bf16": ("bf16", synth.all_bf16_patterns),
    "single_symbol": ("bf16", lambda: synth.constant_bf16(100003, 0.0)),
    "fib26": ("bf16", lambda: synth.powers_of_two_bf16(synth.fibonacci_counts(26), first_exponent=-20)),
    "uniform_random": ("bf16", lambda: synth.random_bits(700001, "bf16", 1)),
    "e4m3_normal": ("e4m3", lambda: synth.normal_e4m3(np.random.SeedSequence(0), 1000003)),
    "e4m3_all": ("e4m3", synth.all_e4m3_patterns),
    "e4m3_random": ("e4m3", lambda: synth.random_bits(500001, "e4m3", 2)),
}


@pytest.mark.parametrize("case", list(SMALL))
def test_parity_small(df11, oracle_mod, case):
    dt, make = SMALL[case]
    _roundtrip(df11, oracle_mod, make(), dt)


@pytest.mark.parametrize("n", [1, 2, 7, 8, 15, 16, 17, 31, 32, 33, 47, 1000, 4095, 4096, 4097])
@pytest.mark.parametrize("dt", ["bf16", "e4m3"])
def test_parity_ragged_sizes(df11, oracle_mod, dt, n):
    x = synth.random_bits(n, dt, n) if n < 40 else (
        synth.single_matrix(n)[0].tensors[0].bits[:n] if dt == "bf16"
        else synth.normal_e4m3(np.random.SeedSequence(n), n))
    _roundtrip(df11, oracle_mod, x, dt)


CTA_LAYOUTS = [(128, 256), (256, 128), (64, 512), (128, 128), (128, 512), (256, 256)]
WARP_LAYOUTS = [(128, 32), (256, 32), (64, 32)]


@pytest.mark.parametrize("cpt", [1, 2])
@pytest.mark.parametrize("layout", CTA_LAYOUTS)
@pytest.mark.parametrize("case", ["heavy_2m", "e4m3_normal", "single_symbol", "uniform_random"])
def test_parity_cta_layouts(df11, oracle_mod, layout, case, cpt):
    """CTA-tile layouts (one out_off per tile of 128-512 chunks, block-wide
    scan), with one and with two chunks per decoding thread."""
    dt, make = SMALL[case]
    _roundtrip(df11, oracle_mod, make(), dt, *layout, cpt=cpt)


# (walker, warps per CTA, chunk counts): the byte-step walk with stored
# counts, with the count walk asked for, and on images without counts
WALKS = [(1, 8, "stored"), (1, 16, "stored"), (2, 16, "stored"), (2, 24, "stored"), (2, 32, "stored"),
         (2, 32, "walk"), (2, 16, "walk"), (2, 32, "absent")]


@pytest.mark.parametrize("walk", WALKS)
@pytest.mark.parametrize("layout", WARP_LAYOUTS)
@pytest.mark.parametrize("case", ["heavy_2m", "e4m3_normal", "single_symbol", "uniform_random", "fib26",
                                  "normal_1m", "all_bf16"])
def test_parity_warp_layouts(df11, oracle_mod, layout, case, walk):
    """Warp-tile layouts (one out_off per 32 chunks, warp-shuffle scan), with
    the 12-bit window walk (8 and 16 warps per CTA) and the byte-step walk (16,
    24 and 32 warps in one CTA per SM), placing the threads' output with the
    stored chunk counts or with the count walk.  A 1-bit code (single_symbol)
    sends every thread of the byte-step walk to the window fallback, random
    bits send many; both must still be exact."""
    dt, make = SMALL[case]
    walker, wpc, counts = walk
    x = make()
    try:
        _roundtrip(df11, oracle_mod, x, dt, *layout, wpc=wpc, walker=walker, counts=counts)
    except df11.Df11Error as e:
        # the byte-step walk asked for with a warp count whose buffers do not
        # fit beside the tables (64-row tables of codes over all 256
        # exponents, long tiles of short codes, 256-bit chunks): refused, and
        # then the library's own warp count, or the automatic walk, must work
        if not (walker == 2 and e.status == df11.DF11_EUNSUPPORTED):
            raise
        try:
            _roundtrip(df11, oracle_mod, x, dt, *layout, walker=walker, counts=counts)
        except df11.Df11Error as e2:
            if e2.status != df11.DF11_EUNSUPPORTED:
                raise
            _roundtrip(df11, oracle_mod, x, dt, *layout, counts=counts)


@pytest.mark.parametrize("ctas", [1, 2])
@pytest.mark.parametrize("layout_cpt", [((128, 256), 1), ((128, 256), 2), ((128, 32), 1)])
def test_parity_launch_options(df11, oracle_mod, layout_cpt, ctas):
    (cb, tt), cpt = layout_cpt
    dt, make = SMALL["heavy_2m"]
    _roundtrip(df11, oracle_mod, make(), dt, cb, tt, cpt=cpt, ctas=ctas)


# (chunk bits, tile threads, walker, chunk counts): the CTA-tile kernel, the
# warp-tile window walk, the byte-step walk with stored counts and with the
# count walk
KERNELS = [(128, 256, 0, "stored"), (128, 32, 1, "stored"), (128, 32, 2, "stored"), (128, 32, 2, "walk")]


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("dt", ["bf16", "e4m3"])
def test_bounds_checks_are_live(df11, kernel, dt):
    """diag_check_bounds: in the bounds-checked library every exponent-buffer
    access of the merge is checked against a bound of 0 bytes, so each one is
    refused: no output byte is written and DF11_DEV_ERR_BOUNDS is set.  The
    normal library ignores the option and decodes exactly, with no flag."""
    chunk_bits, tile_threads, walker, counts = kernel
    x = synth.random_bits(50001, dt, 3) if dt == "bf16" else synth.normal_e4m3(np.random.SeedSequence(3), 50001)
    blob = df11.df11_encode(df11.df11_build_codebook(dt, [x]), x, chunk_bits, tile_threads)
    (out,), err, guards = decode_gpu(df11, [blob], walker=walker, count_walk=int(counts == "walk"),
                                     diag_check_bounds=1)
    assert guards
    if df11.CHECKED:
        assert err & df11.DEV_ERR_BOUNDS
        fill = 0xA5A5 if dt == "bf16" else 0xA5
        assert (out == fill).all()
    else:
        assert err == 0 and np.array_equal(out, x)


def test_parity_32_bit_codes(df11, oracle_mod):
    """Fibonacci counts F1..F34: package-merge limits the code to 32 bits, so
    the decoder walks all four hierarchical levels."""
    x = synth.powers_of_two_bf16(synth.fibonacci_counts(34), first_exponent=-40)
    blob = _roundtrip(df11, oracle_mod, x, "bf16")
    assert blob.info().max_code_len == 32


@pytest.mark.parametrize("limit", [9, 12, 16])
def test_parity_length_limited(df11, oracle_mod, limit):
    x = synth.heavy_tail_matrix(1)[0].tensors[0].bits[:500000]
    blob = _roundtrip(df11, oracle_mod, x, "bf16", max_len=limit)
    assert blob.info().max_code_len <= limit


def test_empty_tensor(df11):
    x = np.zeros(0, np.uint16)
    cb = df11.df11_build_codebook("bf16", [synth.random_bits(100, "bf16")])
    blob = df11.df11_encode(cb, x)
    assert blob.info().n_tiles == 0
    outs, err, _ = decode_gpu(df11, [blob])
    assert err == 0 and outs[0].size == 0


def test_batched_block_launch_scaled(df11, oracle_mod):
    """Seven Llama-3-8B-shaped matrices (scaled by 1/32) sharing one code,
    decoded in ONE launch (DFloat11 Abstract, item (iii))."""
    g = synth.transformer_block(0)[0]
    xs = [t.bits[: t.bits.size // 32 + 77 * i] for i, t in enumerate(g.tensors)]
    cb = df11.df11_build_codebook("bf16", xs)
    blobs = [df11.df11_encode(cb, x) for x in xs]
    outs, err, guards = decode_gpu(df11, blobs)
    assert err == 0 and guards
    lengths = oracle_mod.build_lengths(xs, "bf16")
    for x, out in zip(xs, outs):
        assert np.array_equal(out, x)
        assert np.array_equal(out, oracle_mod.decompress(oracle_mod.compress(x, "bf16", lengths=lengths)))


@pytest.mark.parametrize("max_ctas", [1, 3])
@pytest.mark.parametrize("chunk_bits", [64, 128, 256])
@pytest.mark.parametrize("walker", [1, 2, "2_walk"])
def test_long_runs_across_tensors(df11, oracle_mod, walker, chunk_bits, max_ctas):
    """A capped grid: every warp of the byte-step kernel decodes a long run of
    consecutive tiles that crosses tensor boundaries, so unfinished output
    groups are carried from tile to tile and stored at the ends of runs and
    tensors.  Tensor sizes are ragged on purpose."""
    g = synth.transformer_block(1)[0]
    xs = [t.bits[: t.bits.size // 64 + 13 * i + 5] for i, t in enumerate(g.tensors)]
    xs.append(synth.random_bits(1, "bf16", 3) & 0x3FFF)  # one weight: a run that ends at once
    xs.insert(2, g.tensors[0].bits[:31])
    cb = df11.df11_build_codebook("bf16", xs)
    blobs = [df11.df11_encode(cb, x, chunk_bits, 32) for x in xs]
    count_walk = 1 if walker == "2_walk" else 0
    walker = 2 if walker == "2_walk" else walker
    outs, err, guards = decode_gpu(df11, blobs, walker=walker, warps_per_cta=16, max_ctas=max_ctas,
                                   count_walk=count_walk)
    assert err == 0 and guards
    lengths = oracle_mod.build_lengths(xs, "bf16")
    for x, out in zip(xs, outs):
        assert np.array_equal(out, x)
    assert np.array_equal(outs[0], oracle_mod.decompress(oracle_mod.compress(xs[0], "bf16", lengths=lengths,
                                                                             chunk_bits=chunk_bits, tile_threads=32)))


def test_overlapped_launches(df11, oracle_mod):
    """Independent decodes launched back to back with overlap = 1 (each may
    start while the previous one finishes, programmatic dependent launch) on
    one stream, both walks and a capped grid among them: every output exact,
    no error."""
    s = torch.cuda.Stream()
    jobs = []
    for seed, (walker, max_ctas) in enumerate([(0, 0), (1, 0), (2, 5), (0, 2), (2, 0)]):
        xs = [synth.single_matrix(seed)[0].tensors[0].bits[: 300000 + 7 * seed],
              synth.heavy_tail_matrix(seed)[0].tensors[0].bits[: 200001]]
        cb = df11.df11_build_codebook("bf16", xs)
        blobs = [df11.df11_encode(cb, x) for x in xs]
        with torch.cuda.stream(s):
            for b in blobs:
                df11.upload(b, s)
        outs = [torch.empty(2 * x.size, dtype=torch.uint8, device="cuda") for x in xs]
        jobs.append((xs, blobs, outs, walker, max_ctas))
    s.synchronize()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for xs, blobs, outs, walker, max_ctas in jobs:
        df11.df11_decode_ex(blobs, [o.data_ptr() for o in outs], err.data_ptr(), s.cuda_stream, walker=walker,
                            max_ctas=max_ctas, overlap=1)
    s.synchronize()
    assert int(err.item()) == 0
    for xs, blobs, outs, walker, max_ctas in jobs:
        for x, o in zip(xs, outs):
            assert np.array_equal(o.cpu().numpy().view(np.uint16), x)


@pytest.mark.parametrize("layout_walker", [((128, 32), 2), ((128, 32), 1), ((128, 256), 0)])
def test_bounded_wait_runs_out_and_reports(df11, layout_walker):
    """With diag_expire_waits the kernel issues no copy and each bounded
    wait gets 10 ms: the first one runs out, the launch writes nothing and
    reports DF11_DEV_ERR_TIMEOUT, and the context stays usable (the next,
    normal decode is exact).  Byte-step, window and CTA-tile kernels."""
    import time
    (chunk_bits, tile_threads), walker = layout_walker
    x = synth.single_matrix(3)[0].tensors[0].bits
    blob = df11.df11_encode(df11.df11_build_codebook("bf16", [x]), x, chunk_bits, tile_threads)
    df11.upload(blob)
    torch.cuda.synchronize()
    out = torch.full((2 * x.size,), 0xA5, dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.time()
    df11.df11_decode_ex([blob], [out.data_ptr()], err.data_ptr(), walker=walker, diag_expire_waits=1)
    torch.cuda.synchronize()
    assert time.time() - t0 < 5.0
    assert int(err.item()) & df11.DEV_ERR_TIMEOUT
    assert (out.cpu().numpy() == 0xA5).all()
    err.zero_()
    df11.df11_decode_ex([blob], [out.data_ptr()], err.data_ptr(), walker=walker)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(out.cpu().numpy().view(np.uint16), x)


def test_decode_captured_in_a_cuda_graph(df11):
    """df11_decode_ex launched inside CUDA stream capture (plain and
    overlapped launch) and replayed: every replay exact, no error.  The call
    allocates and synchronises nothing, so it can be captured."""
    g = synth.transformer_block(3)[0]
    xs = [t.bits[: 150000 + 11 * i] for i, t in enumerate(g.tensors[:3])]
    cb = df11.df11_build_codebook("bf16", xs)
    blobs = [df11.df11_encode(cb, x) for x in xs]
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for b in blobs:
            df11.upload(b, s)
    s.synchronize()
    outs = [torch.zeros(2 * x.size, dtype=torch.uint8, device="cuda") for x in xs]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    # one plain launch first: the library's one-time set-up per kernel and
    # device (shared-memory attribute) happens outside the capture
    df11.df11_decode_ex(blobs, [o.data_ptr() for o in outs], err.data_ptr(), s.cuda_stream)
    s.synchronize()
    for overlap in (0, 1):
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            df11.df11_decode_ex(blobs, [o.data_ptr() for o in outs], err.data_ptr(), s.cuda_stream, overlap=overlap)
        for _ in range(3):
            for o in outs:
                o.zero_()
            graph.replay()
            torch.cuda.synchronize()
            assert int(err.item()) == 0
            for x, o in zip(xs, outs):
                assert np.array_equal(o.cpu().numpy().view(np.uint16), x)
        del graph


def test_mixed_codes_rejected(df11):
    a = synth.single_matrix(0)[0].tensors[0].bits[:5000]
    b = synth.heavy_tail_matrix(0)[0].tensors[0].bits[:5000]
    ba = df11.df11_encode(df11.df11_build_codebook("bf16", [a]), a)
    bb = df11.df11_encode(df11.df11_build_codebook("bf16", [b]), b)
    df11.upload(ba)
    df11.upload(bb)
    outs = [df11.empty_output(ba), df11.empty_output(bb)]
    with pytest.raises(df11.Df11Error) as e:
        df11.df11_decode([ba, bb], [o.data_ptr() for o in outs])
    assert e.value.status == df11.DF11_EINVAL


def test_unbound_and_misaligned_rejected(df11):
    x = synth.single_matrix(0)[0].tensors[0].bits[:5000]
    blob = df11.df11_encode(df11.df11_build_codebook("bf16", [x]), x)
    out = df11.empty_output(blob)
    with pytest.raises(df11.Df11Error):
        df11.df11_decode([blob], [out.data_ptr()])  # not bound yet
    df11.upload(blob)
    with pytest.raises(df11.Df11Error):
        df11.df11_decode([blob], [out.data_ptr() + 2])  # 2-byte aligned destination


def test_deterministic_and_stream(df11):
    x = synth.heavy_tail_matrix(2)[0].tensors[0].bits[:3000001]
    blob = df11.df11_encode(df11.df11_build_codebook("bf16", [x]), x)
    s = torch.cuda.Stream()
    a, ea, _ = decode_gpu(df11, [blob], stream=s)
    b, eb, _ = decode_gpu(df11, [blob])
    assert ea == eb == 0
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[0], x)


def test_corrupted_device_data_sets_error_flag(df11):
    """Damaged auxiliary data on the device: the kernel flags it and writes
    nothing outside the destination (guard bytes intact)."""
    x = synth.single_matrix(4)[0].tensors[0].bits
    blob = df11.df11_encode(df11.df11_build_codebook("bf16", [x]), x)
    import struct
    n = blob.info().device_bytes
    img = np.zeros(n, np.uint8)
    df11.df11_blob_device_image(blob, img.ctypes.data, n)
    # layout offsets in the header: meta, syms, lut, fsm, gaps, counts, out_off, ...
    fsm_at = struct.unpack_from("<Q", img.tobytes(), 64 + 8 * 3)[0]
    gaps_at = struct.unpack_from("<Q", img.tobytes(), 64 + 8 * 4)[0]
    counts_at = struct.unpack_from("<Q", img.tobytes(), 64 + 8 * 5)[0]
    out_off_at = struct.unpack_from("<Q", img.tobytes(), 64 + 8 * 6)[0]
    rng = np.random.default_rng(7)
    for what in ("out_off", "gap", "fsm", "count_sum", "count_big"):
        bad = img.copy()
        if what == "out_off":
            bad[out_off_at + 8 * 3: out_off_at + 8 * 4] = np.frombuffer(struct.pack("<Q", 10 ** 12), np.uint8)
        elif what == "gap":
            bad[gaps_at + 5] = (int(bad[gaps_at + 5]) + 3) % 32
        elif what == "count_sum":  # a tile's counts no longer add up to its span
            bad[counts_at + 40] += 1
        elif what == "count_big":  # far more codes than the chunk holds, and a wrong sum
            bad[counts_at + 70] = 255
        else:  # random counts, masks, symbols and rows in the first two transition rows
            bad[fsm_at: fsm_at + 4096] = rng.integers(0, 256, 4096, dtype=np.uint8)
        dev = torch.from_numpy(bad).cuda()
        df11.df11_blob_bind(blob, dev.data_ptr(), n, keep=dev)
        guard = 64
        nbytes = 2 * x.size
        buf = torch.full((nbytes + 2 * guard,), 0xA5, dtype=torch.uint8, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        df11.df11_decode([blob], [buf.data_ptr() + guard], err.data_ptr())
        torch.cuda.synchronize()
        e = int(err.item())
        g = buf.cpu().numpy()
        assert (g[:guard] == 0xA5).all() and (g[guard + nbytes:] == 0xA5).all()
        # damaged data never sends an access outside its buffer or section
        # (checked access by access in the bounds-checked library)
        assert not e & df11.DEV_ERR_BOUNDS
        if what == "out_off":
            assert e & df11.DEV_ERR_AUX
        if what.startswith("count"):
            assert e & df11.DEV_ERR_SPAN
        if what == "fsm":
            # a walk that meets a damaged row either falls back to the window
            # walk (exact output) or miscounts (flagged): never silent
            assert e & df11.DEV_ERR_SPAN or np.array_equal(g[guard:guard + nbytes].view(np.uint16), x)
        # a shifted gap is caught when it changes the tile's code count; when
        # the parse resynchronises to the same count the output is wrong but
        # still inside the destination, which is what is checked above


def _decode_bound_image(df11, blob, img, guard=64, **opts):
    """Binds the blob to a device copy of img (no re-upload) and decodes it
    into a buffer with guard bytes: (output bits, error word, guards intact)."""
    dev = torch.from_numpy(img).cuda()
    df11.df11_blob_bind(blob, dev.data_ptr(), img.size, keep=dev)
    nbytes = 2 * blob.info().n_elems
    buf = torch.full((nbytes + 2 * guard,), 0xA5, dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.df11_decode_ex([blob], [buf.data_ptr() + guard], err.data_ptr(), **opts)
    torch.cuda.synchronize()
    g = buf.cpu().numpy()
    ok = bool((g[:guard] == 0xA5).all() and (g[guard + nbytes:] == 0xA5).all())
    return g[guard:guard + nbytes].view(np.uint16), int(err.item()), ok


@pytest.mark.parametrize("count_walk", [0, 1])
def test_moved_chunk_count_is_caught_and_contained(df11, oracle_mod, count_walk):
    """One code moved between two chunk counts of tile 3 (the tile's sum, and
    so every other thread's position, unchanged): with stored counts the two
    threads' walks disagree with their counts, the launch flags
    DF11_DEV_ERR_SPAN, and every weight outside tile 3's range is still exact
    (the damaged tile's buffer is cleared, nothing carries over).  With the
    count walk the stored counts are not read: exact, no flag."""
    import struct
    x = synth.single_matrix(6)[0].tensors[0].bits
    blob = df11.df11_encode(df11.df11_build_codebook("bf16", [x]), x)
    n = blob.info().device_bytes
    img = np.zeros(n, np.uint8)
    df11.df11_blob_device_image(blob, img.ctypes.data, n)
    counts_at = struct.unpack_from("<Q", img.tobytes(), 64 + 8 * 5)[0]
    t, j = 3, 5
    c = counts_at + 32 * t + j
    assert img[c] > 0
    img[c] -= 1
    img[c + 1] += 1
    out, err, guards = _decode_bound_image(df11, blob, img, count_walk=count_walk)
    assert guards and not err & df11.DEV_ERR_BOUNDS
    if count_walk:
        assert err == 0 and np.array_equal(out, x)
        return
    assert err & df11.DEV_ERR_SPAN
    oo = blob.sections()["out_off"].astype(np.int64)
    assert np.array_equal(out[: oo[t]], x[: oo[t]])
    assert np.array_equal(out[oo[t + 1]:], x[oo[t + 1]:])


def test_launch_mixing_images_with_and_without_counts(df11, oracle_mod):
    """One launch over images with and without chunk counts: the byte-step
    kernel counts with a walk for all of them; exact output."""
    g = synth.transformer_block(2)[0]
    xs = [t.bits[: 200000 + 17 * i] for i, t in enumerate(g.tensors[:4])]
    cb = df11.df11_build_codebook("bf16", xs)
    blobs = [df11.df11_encode(cb, x, chunk_counts=i % 2 == 0) for i, x in enumerate(xs)]
    outs, err, guards = decode_gpu(df11, blobs)
    assert err == 0 and guards
    for x, o in zip(xs, outs):
        assert np.array_equal(o, x)
    assert df11.df11_decode_launch_shape(blobs, with_walk=True)[3:] == (df11.WALKER_BYTE_STEP, 0)
    assert df11.df11_decode_launch_shape(blobs[::2], with_walk=True)[3:] == (df11.WALKER_BYTE_STEP, 1)


def test_transition_rows_past_the_table_are_dead(df11):
    """An E4M3 code has at most 16 transition rows; root entries whose next
    row lies past the last one are sent to the dead row when the table is
    staged, so every thread falls back to the window walk and the output is
    still exact."""
    import struct
    x = synth.normal_e4m3(np.random.SeedSequence(9), 400003)
    blob = df11.df11_encode(df11.df11_build_codebook("e4m3", [x]), x)
    n = blob.info().device_bytes
    img = np.zeros(n, np.uint8)
    df11.df11_blob_device_image(blob, img.ctypes.data, n)
    rows = struct.unpack_from("<I", img.tobytes(), 24)[0]
    assert 2 <= rows <= 16
    fsm_at = struct.unpack_from("<Q", img.tobytes(), 64 + 8 * 3)[0]
    ent = img[fsm_at: fsm_at + 2048].view(np.uint32)
    ent[0::2] |= np.uint32(63 << 11)
    dev = torch.from_numpy(img).cuda()
    df11.df11_blob_bind(blob, dev.data_ptr(), n, keep=dev)
    out = torch.empty(x.size, dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.df11_decode_ex([blob], [out.data_ptr()], err.data_ptr(), walker=df11.WALKER_BYTE_STEP)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(out.cpu().numpy(), x)


def test_decode_host_end_to_end(df11):
    """Host image in pinned memory -> device -> decode -> host output, one call."""
    x = synth.single_matrix(5)[0].tensors[0].bits
    blob = df11.df11_encode(df11.df11_build_codebook("bf16", [x]), x)
    n = blob.info().device_bytes
    himg = torch.empty(n, dtype=torch.uint8, pin_memory=True)
    df11.df11_blob_device_image(blob, himg.data_ptr(), n)
    dimg = torch.empty(n + 256, dtype=torch.uint8, device="cuda")
    dptr = dimg.data_ptr() + (-dimg.data_ptr()) % 256
    dout = torch.empty(2 * x.size, dtype=torch.uint8, device="cuda")
    hout = torch.empty(2 * x.size, dtype=torch.uint8, pin_memory=True)
    s = torch.cuda.current_stream()
    df11.df11_decode_host([blob], [himg.data_ptr()], [dptr], [dout.data_ptr()], [hout.data_ptr()],
                          None, s.cuda_stream)
    s.synchronize()
    assert np.array_equal(hout.numpy().view(np.uint16), x)


def test_launch_shape_is_persistent(df11):
    x = synth.heavy_tail_matrix(0)[0].tensors[0].bits
    blob = df11.df11_encode(df11.df11_build_codebook("bf16", [x]), x)
    df11.upload(blob)
    grid, block, smem = df11.df11_decode_launch_shape([blob])
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    # default layout: warp tiles, byte-step walk, one CTA per SM of as many warps as fit
    assert block in (16 * 32, 24 * 32, 32 * 32)
    assert grid == sms or grid * (block // 32) >= blob.info().n_tiles
    gw, bw, _ = df11.df11_decode_launch_shape([blob], walker=df11.WALKER_WINDOW)
    assert bw == 16 * 32 and (gw % sms == 0 or gw * 16 >= blob.info().n_tiles)
    g8, b8, _ = df11.df11_decode_launch_shape([blob], warps_per_cta=8, ctas_per_sm=1, walker=df11.WALKER_WINDOW)
    assert b8 == 8 * 32 and g8 == sms
    g24, b24, s24 = df11.df11_decode_launch_shape([blob], warps_per_cta=24, walker=df11.WALKER_BYTE_STEP)
    assert b24 == 24 * 32 and g24 == sms and s24 >= 2 * 2048  # at least the root and the dead row
    assert df11.df11_decode_launch_shape([blob], with_walk=True)[3:] == (df11.WALKER_BYTE_STEP, 1)
    assert df11.df11_decode_launch_shape([blob], with_walk=True, count_walk=1)[3:] == (df11.WALKER_BYTE_STEP, 0)
    # stored counts leave out the control-word copy of the tables: less shared memory
    assert df11.df11_decode_launch_shape([blob], count_walk=1)[2] > smem
    # a 1-bit codeword: automatic choice is the window walk
    one = synth.constant_bf16(5000, 0.5)
    b1bit = df11.df11_encode(df11.df11_build_codebook("bf16", [one]), one)
    df11.upload(b1bit)
    assert df11.df11_decode_launch_shape([b1bit], with_walk=True)[3:] == (df11.WALKER_WINDOW, 0)
    cta = df11.df11_encode(df11.df11_build_codebook("bf16", [x]), x, 128, 256)
    df11.upload(cta)
    g1, b1, _ = df11.df11_decode_launch_shape([cta])
    assert b1 == 256 + 32  # CTA tiles: one chunk per decoding thread plus the producer warp
    g2, b2, _ = df11.df11_decode_launch_shape([cta], chunks_per_thread=2, ctas_per_sm=1)
    assert b2 == 256 // 2 + 32 and g2 == min(sms, cta.info().n_tiles)
    assert df11.df11_decode_launch_shape([cta], with_walk=True)[3:] == (df11.WALKER_WINDOW, 0)
    with pytest.raises(df11.Df11Error):
        df11.df11_decode_launch_shape([cta], walker=df11.WALKER_BYTE_STEP)
    assert 0 < smem <= 227 * 1024
