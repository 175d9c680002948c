"""Helpers for the GPU tests: decode through the C-ABI with torch-owned device
memory (device memory and streams only; every decode step runs in libdf11)."""
import numpy as np
import torch


def decode_gpu(df11, blobs, stream=None, guard: int = 64, chunks_per_thread: int = 0, ctas_per_sm: int = 0,
               warps_per_cta: int = 0, walker: int = 0, max_ctas: int = 0, count_walk: int = 0,
               diag_check_bounds: int = 0):
    """Uploads the blobs, decodes them in ONE df11_decode launch and returns
    (outputs as numpy bit arrays, device error word, guards intact)."""
    s = stream or torch.cuda.current_stream()
    with torch.cuda.stream(s):
        for b in blobs:
            df11.upload(b, s)
        bufs, views = [], []
        for b in blobs:
            i = b.info()
            nbytes = i.n_elems * (2 if i.dtype == df11.DF11_BF16 else 1)
            buf = torch.full((nbytes + 2 * guard,), 0xA5, dtype=torch.uint8, device="cuda")
            bufs.append(buf)
            views.append(buf[guard:guard + nbytes])
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        df11.df11_decode_ex(blobs, [v.data_ptr() for v in views], err.data_ptr(), s.cuda_stream,
                            chunks_per_thread, ctas_per_sm, warps_per_cta, walker, max_ctas, count_walk=count_walk,
                            diag_check_bounds=diag_check_bounds)
    s.synchronize()
    outs, guards_ok = [], True
    for b, buf, v in zip(blobs, bufs, views):
        i = b.info()
        host = v.cpu().numpy()
        outs.append(host.view(np.uint16) if i.dtype == df11.DF11_BF16 else host)
        g = buf.cpu().numpy()
        guards_ok &= bool((g[:guard] == 0xA5).all() and (g[guard + v.numel():] == 0xA5).all())
    return outs, int(err.item()), guards_ok
