"""df11_decode_streamed: groups of blobs whose device images stay in pinned
host memory, copied into device staging slots on one stream while earlier
groups decode on another.  Outputs must be bit-exact for every slot count,
and a slot too small for a group is refused before anything is enqueued."""
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


def _groups(df11):
    """Five groups, each with its own code: ragged BF16 tensors and one E4M3 group."""
    out = []
    for gi in range(5):
        if gi == 3:
            xs = [synth.normal_e4m3(np.random.SeedSequence(40 + i), 70001 + 13 * i) for i in range(3)]
            dt = "e4m3"
        else:
            base = synth.heavy_tail_matrix(gi)[0].tensors[0].bits if gi % 2 else synth.single_matrix(gi)[0].tensors[0].bits
            xs = [base[: 90000 + 4097 * i + gi] for i in range(2 + gi % 3)]
            dt = "bf16"
        cb = df11.df11_build_codebook(dt, xs)
        out.append((dt, xs, [df11.df11_encode(cb, x) for x in xs]))
    return out


def _host_images(df11, blobs):
    imgs = []
    for b in blobs:
        n = b.info().device_bytes
        h = torch.empty(n, dtype=torch.uint8, pin_memory=True)
        df11.df11_blob_device_image(b, h.data_ptr(), n)
        imgs.append(h)
    return imgs


def _slot_bytes(groups):
    return max(sum((b.info().device_bytes + 255) // 256 * 256 for b in g[2]) for g in groups)


@pytest.mark.parametrize("n_slots", [1, 2, 3])
def test_streamed_decode_matches_source(df11, n_slots):
    groups = _groups(df11)
    blobs = [b for g in groups for b in g[2]]
    xs = [x for g in groups for x in g[1]]
    imgs = _host_images(df11, blobs)
    cap = _slot_bytes(groups)
    slots = [torch.empty(cap + 256, dtype=torch.uint8, device="cuda") for _ in range(n_slots)]
    slot_ptrs = [s.data_ptr() + (-s.data_ptr()) % 256 for s in slots]
    outs = [torch.full((x.size * x.itemsize + 64,), 0xA5, dtype=torch.uint8, device="cuda") for x in xs]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    cs, ds = torch.cuda.Stream(), torch.cuda.Stream()
    for rep in range(2):  # twice in a row: slots reused across calls
        df11.df11_decode_streamed([g[2] for g in groups], [h.data_ptr() for h in imgs], slot_ptrs, cap,
                                  [o.data_ptr() for o in outs], err.data_ptr(), cs.cuda_stream, ds.cuda_stream)
    ds.synchronize()
    cs.synchronize()
    assert int(err.item()) == 0
    for x, o in zip(xs, outs):
        got = o.cpu().numpy()
        assert np.array_equal(got[: x.size * x.itemsize].view(x.dtype), x)
        assert (got[x.size * x.itemsize:] == 0xA5).all()


def test_streamed_decode_rejects_small_slot(df11):
    groups = _groups(df11)
    blobs = [b for g in groups for b in g[2]]
    imgs = _host_images(df11, blobs)
    cap = _slot_bytes(groups)
    slot = torch.empty(cap, dtype=torch.uint8, device="cuda")
    ptr = slot.data_ptr() + (-slot.data_ptr()) % 256
    outs = [torch.empty(b.info().n_elems * 2, dtype=torch.uint8, device="cuda") for b in blobs]
    with pytest.raises(df11.Df11Error) as e:
        df11.df11_decode_streamed([g[2] for g in groups], [h.data_ptr() for h in imgs], [ptr], cap - 256 * 3,
                                  [o.data_ptr() for o in outs])
    assert e.value.status == df11.DF11_ENOMEM
    with pytest.raises(df11.Df11Error) as e:
        df11.df11_decode_streamed([g[2] for g in groups], [h.data_ptr() for h in imgs], [ptr] * 9, cap,
                                  [o.data_ptr() for o in outs])
    assert e.value.status == df11.DF11_EINVAL


def test_streamed_decode_from_two_host_threads(df11):
    """Two host threads call df11_decode_streamed at the same time, each with
    its own blobs, staging slots and stream pair, four times in a row.  The
    library shares one set of events per device between calls, so it must
    enqueue one call at a time; every output is compared with the oracle's
    decompression of the same tensor."""
    import threading

    import oracle
    oracle.build()
    work = []
    for t in range(2):
        groups = _groups(df11)  # fresh blob objects: each call rebinds its own
        blobs = [b for g in groups for b in g[2]]
        xs = [x for g in groups for x in g[1]]
        dts = [g[0] for g in groups for _ in g[1]]
        imgs = _host_images(df11, blobs)
        cap = _slot_bytes(groups)
        slots = [torch.empty(cap + 256, dtype=torch.uint8, device="cuda") for _ in range(2)]
        outs = [torch.full((x.size * x.itemsize + 64,), 0xA5, dtype=torch.uint8, device="cuda") for x in xs]
        work.append(dict(groups=groups, xs=xs, dts=dts, imgs=imgs, cap=cap, slots=slots, outs=outs,
                         err=torch.zeros(1, dtype=torch.int32, device="cuda"),
                         cs=torch.cuda.Stream(), ds=torch.cuda.Stream()))
    torch.cuda.synchronize()
    start = threading.Barrier(2)
    failures = []

    def run(w):
        try:
            start.wait()
            for _ in range(4):
                df11.df11_decode_streamed([g[2] for g in w["groups"]], [h.data_ptr() for h in w["imgs"]],
                                          [s.data_ptr() + (-s.data_ptr()) % 256 for s in w["slots"]], w["cap"],
                                          [o.data_ptr() for o in w["outs"]], w["err"].data_ptr(),
                                          w["cs"].cuda_stream, w["ds"].cuda_stream)
        except Exception as e:  # reported below, on the main thread
            failures.append(e)

    threads = [threading.Thread(target=run, args=(w,)) for w in work]
    for th in threads:
        th.start()
    for th in threads:
        th.join()
    assert not failures, failures
    torch.cuda.synchronize()
    for w in work:
        assert int(w["err"].item()) == 0
        for x, dt, o in zip(w["xs"], w["dts"], w["outs"]):
            got = o.cpu().numpy()
            want = oracle.decompress(oracle.compress(x, dt))
            assert np.array_equal(got[: x.size * x.itemsize].view(x.dtype), want)
            assert (got[x.size * x.itemsize:] == 0xA5).all()
