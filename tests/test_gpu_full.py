"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times (default layout: 128-bit chunks, 32-chunk tiles; default launch:
the byte-step walk, one CTA of 32 warps per SM; one df11_decode launch per
codebook group).

Small enough for the oracle (1M and 16.7M weights): every element is
compared with the oracle's decompression.  Larger workloads: every element is
compared with the source weights on the device (the method is lossless, so
decode(encode(x)) == x holds at any size), and sampled runs of weights are
decoded one symbol at a time by the oracle from its own bitstream, starting at
code positions it computes itself."""
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


def _decode_group(df11, blobs, count_walk=0):
    """One launch over the blobs with the benchmark's options (default walk,
    overlapped launch); count_walk = 1 counts with the first-phase walk."""
    imgs = [df11.upload(b) for b in blobs]
    outs = [df11.empty_output(b) for b in blobs]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.df11_decode_ex(blobs, [o.data_ptr() for o in outs], err.data_ptr(), torch.cuda.current_stream().cuda_stream,
                        overlap=1, count_walk=count_walk)
    torch.cuda.synchronize()
    del imgs
    return outs, int(err.item())


def _device_equal(out, x):
    src = torch.from_numpy(x.view(np.int16) if x.dtype == np.uint16 else x).cuda()
    got = out[: x.size * x.itemsize].view(torch.int16 if x.dtype == np.uint16 else torch.uint8)
    return bool(torch.equal(got, src))


def _sampled_oracle(oracle_mod, df11, x, dt, lengths, out, n_samples=200, run=16, seed=0):
    """Oracle-decodes `run` symbols at random positions of its own stream and
    checks the GPU output's exponent field there."""
    c = oracle_mod.compress(x, dt, lengths=lengths)
    exps, _ = oracle_mod.split(x, dt)
    starts = np.concatenate([[0], np.cumsum(c.lengths[exps].astype(np.int64))[:-1]])
    g = np.random.default_rng(seed)
    pos = g.integers(0, max(1, x.size - run), n_samples)
    host = out[: x.size * x.itemsize].cpu().numpy().view(x.dtype)
    got_exps, _ = oracle_mod.split(host, dt)
    for p in pos:
        want = oracle_mod.decode_at(c, int(starts[p]), int(min(run, x.size - p)))
        assert np.array_equal(got_exps[p:p + len(want)], want), int(p)


@pytest.mark.parametrize("cfg", ["single_1024x1024", "heavy_tail_4096x4096"])
def test_full_size_small_configs(df11, oracle_mod, cfg):
    g = (synth.single_matrix(0) if cfg.startswith("single") else synth.heavy_tail_matrix(0))[0]
    x = g.tensors[0].bits
    cb = df11.df11_build_codebook("bf16", [x])
    assert np.array_equal(cb.lengths(), oracle_mod.build_lengths([x], "bf16"))
    blob = df11.df11_encode(cb, x)
    (out,), err = _decode_group(df11, [blob])
    assert err == 0
    host = out[: 2 * x.size].cpu().numpy().view(np.uint16)
    want = oracle_mod.decompress(oracle_mod.compress(x, "bf16"))
    assert np.array_equal(host, want)
    assert np.array_equal(host, x)
    if cfg.startswith("heavy"):
        assert blob.info().max_code_len >= 20  # the long tail reaches the deep table levels


@pytest.mark.parametrize("count_walk", [0, 1])
def test_full_size_transformer_block_one_launch(df11, oracle_mod, count_walk):
    """The block in one launch, placing each thread's output with the stored
    chunk counts (the benchmark's default) and with the first-phase count walk."""
    g = synth.transformer_block(0)[0]
    xs = [t.bits for t in g.tensors]
    cb = df11.df11_build_codebook("bf16", xs)
    lengths = oracle_mod.build_lengths(xs, "bf16")
    assert np.array_equal(cb.lengths(), lengths)
    blobs = [df11.df11_encode(cb, x) for x in xs]
    assert sum(b.info().n_elems for b in blobs) == 218103808
    outs, err = _decode_group(df11, blobs, count_walk)
    assert err == 0
    for x, out in zip(xs, outs):
        assert _device_equal(out, x)
    for x, out, seed in [(xs[0], outs[0], 1), (xs[6], outs[6], 2)]:
        _sampled_oracle(oracle_mod, df11, x, "bf16", lengths, out, seed=seed)


def test_full_size_e4m3(df11, oracle_mod):
    x = synth.e4m3_matrix(0)[0].tensors[0].bits
    cb = df11.df11_build_codebook("e4m3", [x])
    assert np.array_equal(cb.lengths(), oracle_mod.build_lengths([x], "e4m3"))
    blob = df11.df11_encode(cb, x)
    (out,), err = _decode_group(df11, [blob])
    assert err == 0
    assert _device_equal(out, x)
    _sampled_oracle(oracle_mod, df11, x, "e4m3", oracle_mod.build_lengths([x], "e4m3"), out, seed=3)


@pytest.mark.slow
def test_full_size_whole_model(df11, oracle_mod):
    """All 34 codebook groups of the whole-model workload (8,029,995,008
    weights), one launch per group as in the benchmark."""
    total = 0
    n_groups = len(synth.whole_model_specs())
    for gi in range(n_groups):
        g = synth.whole_model_group(0, gi)
        xs = [t.bits for t in g.tensors]
        cb = df11.df11_build_codebook("bf16", xs)
        blobs = [df11.df11_encode(cb, x) for x in xs]
        outs, err = _decode_group(df11, blobs)
        assert err == 0, g.name
        for x, out in zip(xs, outs):
            assert _device_equal(out, x), g.name
            total += x.size
        if gi in (0, 1, n_groups - 1):
            _sampled_oracle(oracle_mod, df11, xs[-1][: 50_000_000], "bf16", oracle_mod.build_lengths(xs, "bf16"),
                            _decode_group(df11, [df11.df11_encode(cb, xs[-1][: 50_000_000])])[0][0],
                            n_samples=64, seed=gi)
        del outs, blobs, xs, g
        torch.cuda.empty_cache()
    assert total == 8029995008
