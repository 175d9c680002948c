"""df11_decode_gemm: the decode fused into the GEMM that consumes the weights
(y += x W, weights decoded tile by tile into the tensor cores' shared-memory
operands).  Every output is compared with the oracle's product of the
exactly decoded weights (float64) within the float32 accumulation bound
(K + 16) * 2^-24 * sum_k |x_mk w_kn|, and with decode-then-torch.matmul at
the same bound.  The library's operand-tile order must equal the oracle's."""
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


@pytest.fixture(scope="module")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


def _bf16(a: np.ndarray) -> np.ndarray:
    return synth.to_bf16_bits(np.asarray(a, np.float32))


def _weights(k, n, seed, std=None):
    g = np.random.default_rng(seed)
    return _bf16(g.standard_normal(k * n) * (std if std is not None else 1 / np.sqrt(k)))


def _acts(m, k, seed):
    return _bf16(np.random.default_rng(seed + 1000).standard_normal(m * k))


def _encode(df11, oracle_mod, ws, shapes):
    """Tiles every matrix (checked against the oracle's tiling), one code for all."""
    tiled = []
    for w, (k, n) in zip(ws, shapes):
        t = df11.df11_gemm_tile_weights(w, k, n)
        assert np.array_equal(t, oracle_mod.gemm_tile(w, k, n))
        tiled.append(t)
    cb = df11.df11_build_codebook("bf16", tiled)
    blobs = [df11.df11_encode(cb, t) for t in tiled]
    for b in blobs:
        df11.upload(b)
    return tiled, blobs


def _run(df11, blobs, shapes, xs, m):
    xd = [torch.from_numpy(x.view(np.int16)).cuda() for x in xs]
    yd = [torch.zeros(m * n, dtype=torch.float32, device="cuda") for _, n in shapes]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.df11_decode_gemm([(b, k, n, x.data_ptr(), y.data_ptr()) for b, (k, n), x, y in zip(blobs, shapes, xd, yd)],
                          m, err.data_ptr())
    torch.cuda.synchronize()
    return [y.cpu().numpy().astype(np.float64).reshape(m, -1) for y in yd], int(err.item())


def _check(oracle_mod, y, x, w, m, k, n, what=""):
    want = oracle_mod.gemm(x, w, m, k, n)
    bound = (k + 16) * 2.0 ** -24 * oracle_mod.gemm_abs(x, w, m, k, n)
    bad = np.abs(y - want) > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} of {bad.size} outside the bound, first at {np.argwhere(bad)[:4]}"


@pytest.mark.parametrize("k,n,m", [(64, 128, 1), (128, 128, 2), (256, 256, 16), (512, 384, 5), (1024, 512, 33),
                                   (4096, 256, 64), (192, 640, 17), (64, 1152, 16)])
def test_single_matrix(df11, oracle_mod, k, n, m):
    w, x = _weights(k, n, k + n + m), _acts(m, k, k + n + m)
    tiled, (blob,) = _encode(df11, oracle_mod, [w], [(k, n)])
    (y,), err = _run(df11, [blob], [(k, n)], [x], m)
    assert err == 0
    _check(oracle_mod, y, x, w, m, k, n)
    # the oracle's own container of the tiled weights gives the same product
    c = oracle_mod.compress(tiled[0], "bf16", tile_threads=32)
    assert np.array_equal(oracle_mod.decode_gemm(c, x, m, k, n), oracle_mod.gemm(x, w, m, k, n))


def test_operand_tiles_split_between_ctas(df11, oracle_mod):
    """512 operand tiles over the SMs: CTA ranges start and end inside blocks
    of 128 output rows (their y rows are summed by several CTAs) and inside
    warp tiles of the container."""
    k, n, m = 4096, 1024, 16
    w, x = _weights(k, n, 5), _acts(m, k, 5)
    _, (blob,) = _encode(df11, oracle_mod, [w], [(k, n)])
    grid, block, smem = df11.df11_decode_gemm_launch_shape([(blob, k, n, 0, 0)], m)
    assert block % 128 == 0 and 1 < grid <= 148 and (k // 64) * (n // 128) % grid != 0
    (y,), err = _run(df11, [blob], [(k, n)], [x], m)
    assert err == 0
    _check(oracle_mod, y, x, w, m, k, n)


def test_block_shaped_launch(df11, oracle_mod):
    """Seven matrices shaped like a transformer block's (scaled by 1/8), one
    code, one launch: CTA ranges cross matrix boundaries."""
    shapes = [(512, 512), (512, 128), (512, 128), (512, 512), (512, 1792), (512, 1792), (1792, 512)]
    m = 16
    ws = [_weights(k, n, 40 + i) for i, (k, n) in enumerate(shapes)]
    xs = [_acts(m, k, 40 + i) for i, (k, n) in enumerate(shapes)]
    _, blobs = _encode(df11, oracle_mod, ws, shapes)
    ys, err = _run(df11, blobs, shapes, xs, m)
    assert err == 0
    for i, ((k, n), y, x, w) in enumerate(zip(shapes, ys, xs, ws)):
        _check(oracle_mod, y, x, w, m, k, n, f"matrix {i}")


def test_against_decode_then_matmul(df11, oracle_mod):
    """The same product by the unfused path: df11_decode of the tiled blob,
    the tile order undone on the device, torch.matmul in float32."""
    k, n, m = 2048, 768, 8
    w, x = _weights(k, n, 9), _acts(m, k, 9)
    tiled, (blob,) = _encode(df11, oracle_mod, [w], [(k, n)])
    out = df11.empty_output(blob)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.df11_decode([blob], [out.data_ptr()], err.data_ptr())
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    dec = out[: 2 * k * n].view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(dec, tiled[0])  # the tiled order, bit for bit
    wd = out[: 2 * k * n].view(torch.bfloat16).reshape(n // 128, k // 64, 128, 64).permute(1, 3, 0, 2).reshape(k, n)
    xd = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16).reshape(m, k)
    ref = (xd.float() @ wd.float()).double().cpu().numpy()
    (y,), err = _run(df11, [blob], [(k, n)], [x], m)
    assert err == 0
    bound = (k + 16) * 2.0 ** -24 * oracle_mod.gemm_abs(x, w, m, k, n)
    assert (np.abs(y - ref) <= 2 * bound).all()
    _check(oracle_mod, y, x, w, m, k, n)


def test_accumulates_into_y(df11, oracle_mod):
    """y += x W: a second launch adds the product again."""
    k, n, m = 256, 256, 4
    w, x = _weights(k, n, 12), _acts(m, k, 12)
    _, (blob,) = _encode(df11, oracle_mod, [w], [(k, n)])
    xd = torch.from_numpy(x.view(np.int16)).cuda()
    y = torch.full((m * n,), 0.5, dtype=torch.float32, device="cuda")
    for _ in range(2):
        df11.df11_decode_gemm([(blob, k, n, xd.data_ptr(), y.data_ptr())], m)
    torch.cuda.synchronize()
    want = 0.5 + 2 * oracle_mod.gemm(x, w, m, k, n)
    bound = 2 * (k + 16) * 2.0 ** -24 * oracle_mod.gemm_abs(x, w, m, k, n) + 2.0 ** -22
    assert (np.abs(y.cpu().numpy().astype(np.float64).reshape(m, n) - want) <= bound).all()


def test_long_codes(df11, oracle_mod):
    """Heavy-tailed weights: codes of 20+ bits, walks that leave the
    transition tables and fall back to the window walk."""
    k, n, m = 1024, 1024, 16
    w = synth.heavy_tail_matrix(2)[0].tensors[0].bits[: k * n].copy()
    x = _acts(m, k, 77)
    _, (blob,) = _encode(df11, oracle_mod, [w], [(k, n)])
    assert blob.info().max_code_len >= 18
    (y,), err = _run(df11, [blob], [(k, n)], [x], m)
    assert err == 0
    _check(oracle_mod, y, x, w, m, k, n)


def test_refused_shapes_and_layouts(df11, oracle_mod):
    k, n, m = 128, 128, 4
    w = _weights(k, n, 1)
    _, (blob,) = _encode(df11, oracle_mod, [w], [(k, n)])
    x = torch.zeros(m * k, dtype=torch.int16, device="cuda")
    y = torch.zeros(m * n, dtype=torch.float32, device="cuda")
    for mats, mm, status in [([(blob, k, n, x.data_ptr(), y.data_ptr())], 65, df11.DF11_EINVAL),
                             ([(blob, k, n, x.data_ptr(), y.data_ptr())], 0, df11.DF11_EINVAL),
                             ([(blob, k, n + 128, x.data_ptr(), y.data_ptr())], m, df11.DF11_EINVAL),
                             ([(blob, k + 8, n, x.data_ptr(), y.data_ptr())], m, df11.DF11_EINVAL),
                             ([(blob, k, n, x.data_ptr() + 2, y.data_ptr())], m, df11.DF11_EINVAL)]:
        with pytest.raises(df11.Df11Error) as e:
            df11.df11_decode_gemm(mats, mm)
        assert e.value.status == status
    bare = df11.df11_encode(df11.df11_build_codebook("bf16", [w]), df11.df11_gemm_tile_weights(w, k, n),
                            chunk_counts=False)
    df11.upload(bare)
    with pytest.raises(df11.Df11Error) as e:
        df11.df11_decode_gemm([(bare, k, n, x.data_ptr(), y.data_ptr())], m)
    assert e.value.status == df11.DF11_EUNSUPPORTED


def test_corrupted_counts_are_flagged(df11, oracle_mod):
    """Chunk counts moved between two chunks of a tile in the device image:
    the launch ends (no wait runs out) and flags DF11_DEV_ERR_SPAN."""
    import struct
    k, n, m = 512, 512, 16
    w, x = _weights(k, n, 21), _acts(m, k, 21)
    _, (blob,) = _encode(df11, oracle_mod, [w], [(k, n)])
    nbytes = blob.info().device_bytes
    img = np.zeros(nbytes, np.uint8)
    df11.df11_blob_device_image(blob, img.ctypes.data, nbytes)
    counts_at = struct.unpack_from("<Q", img.tobytes(), 64 + 8 * 5)[0]  # image header: layout.counts
    c = counts_at + 32 * 2 + 3  # tile 2, chunk 3
    assert img[c] > 0
    img[c] -= 1
    img[c + 1] += 1
    dev = torch.from_numpy(img).cuda()  # torch's device blocks are 512-byte aligned
    df11.df11_blob_bind(blob, dev.data_ptr(), nbytes, keep=dev)
    (y,), err = _run(df11, [blob], [(k, n)], [x], m)
    assert err & df11.DEV_ERR_SPAN
    assert not err & df11.DEV_ERR_TIMEOUT
    assert not err & df11.DEV_ERR_BOUNDS


@pytest.mark.slow
def test_full_size_transformer_block(df11, oracle_mod):
    """The Llama-3-8B-shaped block (218M weights, shapes [in, out]) in one
    launch at M = 16, against decode-then-matmul on the device (every output)
    and the oracle's float64 product on sampled output columns."""
    g = synth.transformer_block(0)[0]
    shapes = [tuple(t.shape) for t in g.tensors]
    m = 16
    ws = [t.bits for t in g.tensors]
    xs = [_acts(m, k, 300 + i) for i, (k, n) in enumerate(shapes)]
    tiled = [df11.df11_gemm_tile_weights(w, k, n) for w, (k, n) in zip(ws, shapes)]
    cb = df11.df11_build_codebook("bf16", tiled)
    blobs = [df11.df11_encode(cb, t) for t in tiled]
    for b in blobs:
        df11.upload(b)
    del tiled
    ys, err = _run(df11, blobs, shapes, xs, m)
    assert err == 0
    rng = np.random.default_rng(0)
    for (k, n), y, x, w in zip(shapes, ys, xs, ws):
        wd = torch.from_numpy(w.view(np.int16)).cuda().view(torch.bfloat16).reshape(k, n).float()
        xd = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16).reshape(m, k).float()
        ref = (xd @ wd).double().cpu().numpy()
        scale = (xd.abs() @ wd.abs()).double().cpu().numpy()
        assert (np.abs(y - ref) <= 2 * (k + 16) * 2.0 ** -24 * scale).all()
        cols = rng.choice(n, 64, replace=False)
        W = oracle_mod.bf16_to_float(w).reshape(k, n)[:, cols]
        X = oracle_mod.bf16_to_float(x).reshape(m, k)
        want = X @ W
        bound = (k + 16) * 2.0 ** -24 * (np.abs(X) @ np.abs(W))
        assert (np.abs(y[:, cols] - want) <= bound).all()
