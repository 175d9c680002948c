"""Thin ctypes binding of libdf11 (C-ABI declared in include/df11.h).

Every function here only marshals arguments into the library call of the same
name; encoding runs in the library's host code, decoding in its sm_100a
kernel.  There is no Python or CPU fallback: importing this module raises
when libdf11.so has not been built (``python -m entropy_decoding_b200.build``).

PyTorch is used only as a source of device memory and streams: device
pointers are plain integers (``tensor.data_ptr()``), streams are
``torch.cuda.Stream.cuda_stream`` integers (0 = default stream).

The environment variable DF11_LIBRARY=check loads libdf11_check.so instead:
the same C-ABI with every decode access bounds-checked (an access outside
its buffer or section is skipped and DEV_ERR_BOUNDS set in the launch's
error word).  It is read once, at import.
"""
from __future__ import annotations

import ctypes
import struct
import os
import re

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_VARIANTS = {"": "libdf11.so", "normal": "libdf11.so", "check": "libdf11_check.so"}
_variant = os.environ.get("DF11_LIBRARY", "")
if _variant not in _VARIANTS:
    raise ImportError(f"DF11_LIBRARY={_variant!r}: expected one of 'normal', 'check'")
CHECKED = _variant == "check"
LIB_PATH = os.path.join(_HERE, _VARIANTS[_variant])
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "df11.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{os.path.basename(LIB_PATH)} not built at {LIB_PATH}; "
                      f"run `python -m entropy_decoding_b200.build{' --check' if CHECKED else ''}`")

_lib = ctypes.CDLL(LIB_PATH)

DF11_OK, DF11_EINVAL, DF11_ENOMEM, DF11_ECUDA, DF11_ECORRUPT, DF11_EUNSUPPORTED = range(6)
DF11_BF16, DF11_FP8_E4M3 = 0, 1
DTYPES = {"bf16": DF11_BF16, "e4m3": DF11_FP8_E4M3}
DEV_ERR_SPAN, DEV_ERR_CODE, DEV_ERR_AUX, DEV_ERR_TIMEOUT, DEV_ERR_BOUNDS = 1, 2, 4, 8, 16


class Df11Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {_lib.df11_status_string(status).decode()} ({status})")


class BlobInfo(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int32), ("chunk_bits", ctypes.c_int32), ("tile_threads", ctypes.c_int32),
                ("max_code_len", ctypes.c_int32), ("n_elems", ctypes.c_uint64), ("total_bits", ctypes.c_uint64),
                ("n_tiles", ctypes.c_uint64), ("max_span", ctypes.c_uint64), ("stream_bytes", ctypes.c_uint64),
                ("plane_bytes", ctypes.c_uint64), ("gaps_bytes", ctypes.c_uint64),
                ("out_off_bytes", ctypes.c_uint64), ("serialized_bytes", ctypes.c_uint64),
                ("device_bytes", ctypes.c_uint64), ("uncompressed_bytes", ctypes.c_uint64),
                ("counts_bytes", ctypes.c_uint64)]

    def as_dict(self) -> dict:
        return {k: getattr(self, k) for k, _ in self._fields_}


class EncodeResult(ctypes.Structure):
    _fields_ = [("image_bytes", ctypes.c_uint64), ("total_bits", ctypes.c_uint64), ("n_tiles", ctypes.c_uint64),
                ("max_span", ctypes.c_uint64)]


class RansTensorInfo(ctypes.Structure):
    _fields_ = [("n_elems", ctypes.c_uint64), ("n_tiles", ctypes.c_uint64), ("words", ctypes.c_uint64),
                ("coded_bytes", ctypes.c_uint64), ("plane_bytes", ctypes.c_uint64),
                ("uncompressed_bytes", ctypes.c_uint64)]


class DecodeOpts(ctypes.Structure):
    _fields_ = [("chunks_per_thread", ctypes.c_int32), ("ctas_per_sm", ctypes.c_int32),
                ("warps_per_cta", ctypes.c_int32), ("walker", ctypes.c_int32), ("max_ctas", ctypes.c_int32),
                ("overlap", ctypes.c_int32), ("diag_expire_waits", ctypes.c_int32), ("count_walk", ctypes.c_int32),
                ("diag_check_bounds", ctypes.c_int32)]


class GemmMatrix(ctypes.Structure):
    _fields_ = [("weights", ctypes.c_void_p), ("k", ctypes.c_uint64), ("n", ctypes.c_uint64), ("x", ctypes.c_void_p),
                ("y", ctypes.c_void_p)]


GEMM_TILE_N, GEMM_TILE_K, GEMM_MAX_MATS, GEMM_MAX_BATCH = 128, 64, 8, 64

WALKER_AUTO, WALKER_WINDOW, WALKER_BYTE_STEP = 0, 1, 2
ENCODE_NO_CHUNK_COUNTS = 1  # encoder flag: leave out the chunk-counts section


_P = ctypes.c_void_p
_PP = ctypes.POINTER(ctypes.c_void_p)
_U64 = ctypes.c_uint64
_I = ctypes.c_int
_S = ctypes.c_int  # df11_status

_SIGS = {
    "df11_version": ([], _I),
    "df11_status_string": ([_I], ctypes.c_char_p),
    "df11_build_codebook": ([_I, _PP, ctypes.POINTER(_U64), _I, _I, _PP], _S),
    "df11_codebook_from_lengths": ([_I, _P, _I, _PP], _S),
    "df11_codebook_lengths": ([_P, _P], _S),
    "df11_codebook_free": ([_P], None),
    "df11_encode": ([_P, _P, _U64, _PP], _S),
    "df11_encode_ex": ([_P, _P, _U64, _I, _I, _I, _I, _PP], _S),
    "df11_layout_supported": ([_I, _I, _I], _I),
    "df11_blob_free": ([_P], None),
    "df11_blob_get_info": ([_P, ctypes.POINTER(BlobInfo)], _S),
    "df11_blob_compressed_bytes": ([_P], _U64),
    "df11_blob_sections": ([_P, _PP, _PP, _PP, _PP], _S),
    "df11_blob_chunk_counts": ([_P, _PP], _S),
    "df11_blob_lengths": ([_P, _P], _S),
    "df11_serialize": ([_P, _P, _U64, ctypes.POINTER(_U64)], _S),
    "df11_deserialize": ([_P, _U64, _PP], _S),
    "df11_blob_device_image": ([_P, _P, _U64], _S),
    "df11_blob_bind": ([_P, _P, _U64], _S),
    "df11_blob_upload": ([_P, _P, _U64, _P], _S),
    "df11_decode": ([_PP, _PP, _I, _P, _P], _S),
    "df11_decode_ex": ([_PP, _PP, _I, _P, _P, ctypes.POINTER(DecodeOpts)], _S),
    "df11_decode_launch_shape_ex": ([_PP, _I, ctypes.POINTER(DecodeOpts), ctypes.POINTER(_I), ctypes.POINTER(_I),
                                     ctypes.POINTER(_I), ctypes.POINTER(_I), ctypes.POINTER(_I)], _S),
    "df11_histogram_device": ([_I, _P, _U64, _P, _P], _S),
    "df11_decode_streamed": ([_PP, _P, _I, _PP, _PP, _I, _U64, _PP, _P, _P, _P], _S),
    "df11_codebook_from_counts": ([_I, _P, _I, _I, _PP], _S),
    "df11_encode_device_scratch_bytes": ([_U64], _U64),
    "df11_encode_device_begin": ([_P, _P, _U64, _I, _I, _I, _P, _U64, _P, ctypes.POINTER(_U64), _PP], _S),
    "df11_encode_device_end": ([_P, _P, _U64, _PP], _S),
    "df11_encoding_free": ([_P], None),
    "df11_blob_fetch": ([_P, _P], _S),
    "df11_encode_device_noalloc": ([_P, _P, _U64, _I, _I, _I, _P, _U64, _P, ctypes.POINTER(EncodeResult)], _S),
    "df11_decode_host": ([_PP, _PP, _PP, _PP, _PP, _I, _P, _P], _S),
    "df11_decode_launch_shape": ([_PP, _I, ctypes.POINTER(_I), ctypes.POINTER(_I), ctypes.POINTER(_I)], _S),
    "df11_gemm_tile_weights": ([_P, _U64, _U64, _P], _S),
    "df11_decode_gemm": ([ctypes.POINTER(GemmMatrix), _I, _I, _P, _P], _S),
    "df11_decode_gemm_launch_shape": ([ctypes.POINTER(GemmMatrix), _I, _I, ctypes.POINTER(_I), ctypes.POINTER(_I),
                                       ctypes.POINTER(_I)], _S),
    "df11_rans_encode_group": ([_I, _PP, ctypes.POINTER(_U64), _I, _I, _I, _PP], _S),
    "df11_rans_group_free": ([_P], None),
    "df11_rans_group_freqs": ([_P, _P], _S),
    "df11_rans_group_info": ([_P, _I, ctypes.POINTER(RansTensorInfo)], _S),
    "df11_rans_group_sections": ([_P, _I, _PP, _PP, _PP, _PP], _S),
    "df11_rans_group_device_bytes": ([_P], _U64),
    "df11_rans_group_serialize": ([_P, _P, _U64, ctypes.POINTER(_U64)], _S),
    "df11_rans_group_deserialize": ([_P, _U64, _PP], _S),
    "df11_rans_group_upload": ([_P, _P, _U64, _P], _S),
    "df11_rans_decode": ([_P, _PP, _P, _P], _S),
    "df11_rans_decode_launch_shape": ([_P, ctypes.POINTER(_I), ctypes.POINTER(_I), ctypes.POINTER(_I)], _S),
}
for _name, (_args, _res) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _res


def exported_names() -> list[str]:
    """Function names declared in include/df11.h (for the symbol check)."""
    with open(HEADER_PATH) as f:
        src = f.read()
    return sorted(set(re.findall(r"\b(df11_[a-z_0-9]+)\s*\(", src)))


def _check(status: int, what: str):
    if status != DF11_OK:
        raise Df11Error(status, what)


def _ptr_array(ptrs) -> ctypes.Array:
    return (ctypes.c_void_p * len(ptrs))(*[int(p) if p is not None else None for p in ptrs])


# ----------------------------------------------------------------- objects

class Codebook:
    def __init__(self, handle: int, dtype: str):
        self._h = ctypes.c_void_p(handle)
        self.dtype = dtype

    @property
    def handle(self):
        return self._h

    def lengths(self) -> np.ndarray:
        out = np.zeros(256, np.uint8)
        _check(_lib.df11_codebook_lengths(self._h, out.ctypes.data), "df11_codebook_lengths")
        return out[: 256 if self.dtype == "bf16" else 16]

    def __del__(self, _free=_lib.df11_codebook_free):
        if getattr(self, "_h", None) and self._h.value:
            _free(self._h)
            self._h = None


class Blob:
    def __init__(self, handle: int):
        self._h = ctypes.c_void_p(handle)
        self._keep = None  # device image owner (e.g. a torch tensor)

    @property
    def handle(self):
        return self._h

    def info(self) -> BlobInfo:
        i = BlobInfo()
        _check(_lib.df11_blob_get_info(self._h, ctypes.byref(i)), "df11_blob_get_info")
        return i

    def compressed_bytes(self) -> int:
        return int(_lib.df11_blob_compressed_bytes(self._h))

    @property
    def dtype(self) -> str:
        return "bf16" if self.info().dtype == DF11_BF16 else "e4m3"

    def sections(self) -> dict:
        """Copies of the host sections: stream, plane, gaps, out_off, and counts
        (None when the blob has no chunk counts)."""
        i = self.info()
        ptrs = [ctypes.c_void_p() for _ in range(4)]
        _check(_lib.df11_blob_sections(self._h, *[ctypes.byref(p) for p in ptrs]), "df11_blob_sections")

        def grab(p, n, dt):
            if n == 0:
                return np.zeros(0, dt)
            return np.ctypeslib.as_array(ctypes.cast(p, ctypes.POINTER(ctypes.c_uint8)), (n,)).view(dt).copy()

        return {"stream": grab(ptrs[0], i.stream_bytes, np.uint8),
                "plane": grab(ptrs[1], i.plane_bytes, np.uint8),
                "gaps": grab(ptrs[2], i.gaps_bytes, np.uint8),
                "out_off": grab(ptrs[3], i.out_off_bytes, np.uint64),
                "counts": self.chunk_counts()}

    def chunk_counts(self):
        """Copy of the chunk counts, or None when the blob has none."""
        p = ctypes.c_void_p()
        _check(_lib.df11_blob_chunk_counts(self._h, ctypes.byref(p)), "df11_blob_chunk_counts")
        if not p.value:
            return None
        n = self.info().counts_bytes
        if n == 0:
            return np.zeros(0, np.uint8)
        return np.ctypeslib.as_array(ctypes.cast(p, ctypes.POINTER(ctypes.c_uint8)), (n,)).copy()

    def lengths(self) -> np.ndarray:
        out = np.zeros(256, np.uint8)
        _check(_lib.df11_blob_lengths(self._h, out.ctypes.data), "df11_blob_lengths")
        return out

    def __del__(self, _free=_lib.df11_blob_free):
        if getattr(self, "_h", None) and self._h.value:
            _free(self._h)
            self._h = None


# ----------------------------------------------------------------- functions (same names as the C-ABI)

def df11_version() -> int:
    return _lib.df11_version()


def df11_build_codebook(dtype: str, tensors, max_code_len: int = 0) -> Codebook:
    arrs = [np.ascontiguousarray(t).reshape(-1) for t in tensors]
    ptrs = _ptr_array([a.ctypes.data if a.size else None for a in arrs])
    ns = (_U64 * len(arrs))(*[a.size for a in arrs])
    out = ctypes.c_void_p()
    _check(_lib.df11_build_codebook(DTYPES[dtype], ptrs, ns, len(arrs), max_code_len, ctypes.byref(out)),
           "df11_build_codebook")
    return Codebook(out.value, dtype)


def df11_codebook_from_lengths(dtype: str, lengths) -> Codebook:
    ln = np.ascontiguousarray(lengths, np.uint8)
    out = ctypes.c_void_p()
    _check(_lib.df11_codebook_from_lengths(DTYPES[dtype], ln.ctypes.data, ln.size, ctypes.byref(out)),
           "df11_codebook_from_lengths")
    return Codebook(out.value, dtype)


def _encode_flags(chunk_counts: bool) -> int:
    return 0 if chunk_counts else ENCODE_NO_CHUNK_COUNTS


def df11_encode(cb: Codebook, x: np.ndarray, chunk_bits: int = 128, tile_threads: int = 32,
                n_threads: int = 0, chunk_counts: bool = True) -> Blob:
    a = np.ascontiguousarray(x).reshape(-1)
    out = ctypes.c_void_p()
    _check(_lib.df11_encode_ex(cb.handle, a.ctypes.data if a.size else None, a.size, chunk_bits, tile_threads,
                               _encode_flags(chunk_counts), n_threads, ctypes.byref(out)), "df11_encode")
    return Blob(out.value)


def df11_layout_supported(dtype: str, chunk_bits: int, tile_threads: int) -> bool:
    return bool(_lib.df11_layout_supported(DTYPES[dtype], chunk_bits, tile_threads))


def df11_serialize(blob: Blob) -> bytes:
    used = _U64()
    _lib.df11_serialize(blob.handle, None, 0, ctypes.byref(used))
    buf = np.zeros(used.value, np.uint8)
    _check(_lib.df11_serialize(blob.handle, buf.ctypes.data, buf.size, ctypes.byref(used)), "df11_serialize")
    return buf.tobytes()


def df11_deserialize(data) -> Blob:
    buf = np.frombuffer(data, np.uint8)
    if buf.size == 0:
        buf = np.zeros(1, np.uint8)
        n = 0
    else:
        n = buf.size
    out = ctypes.c_void_p()
    _check(_lib.df11_deserialize(buf.ctypes.data, n, ctypes.byref(out)), "df11_deserialize")
    return Blob(out.value)


def df11_blob_device_image(blob: Blob, host_dst_ptr: int, cap: int):
    _check(_lib.df11_blob_device_image(blob.handle, host_dst_ptr, cap), "df11_blob_device_image")


def df11_blob_bind(blob: Blob, dev_image_ptr: int, cap: int, keep=None):
    _check(_lib.df11_blob_bind(blob.handle, dev_image_ptr, cap), "df11_blob_bind")
    blob._keep = keep


def df11_blob_upload(blob: Blob, dev_dst_ptr: int, cap: int, stream: int = 0, keep=None):
    _check(_lib.df11_blob_upload(blob.handle, dev_dst_ptr, cap, stream or None), "df11_blob_upload")
    blob._keep = keep


def df11_decode(blobs, dst_ptrs, err_ptr: int | None = None, stream: int = 0):
    hs = _ptr_array([b.handle.value for b in blobs])
    ds = _ptr_array(dst_ptrs)
    _check(_lib.df11_decode(hs, ds, len(blobs), err_ptr or None, stream or None), "df11_decode")


def df11_decode_ex(blobs, dst_ptrs, err_ptr: int | None = None, stream: int = 0, chunks_per_thread: int = 0,
                   ctas_per_sm: int = 0, warps_per_cta: int = 0, walker: int = 0, max_ctas: int = 0,
                   overlap: int = 0, diag_expire_waits: int = 0, count_walk: int = 0, diag_check_bounds: int = 0):
    o = DecodeOpts(chunks_per_thread, ctas_per_sm, warps_per_cta, walker, max_ctas, overlap, diag_expire_waits,
                   count_walk, diag_check_bounds)
    _check(_lib.df11_decode_ex(_ptr_array([b.handle.value for b in blobs]), _ptr_array(dst_ptrs), len(blobs),
                               err_ptr or None, stream or None, ctypes.byref(o)), "df11_decode_ex")


def df11_decode_host(blobs, host_image_ptrs, dev_image_ptrs, dst_dev_ptrs, dst_host_ptrs,
                     err_ptr: int | None = None, stream: int = 0):
    _check(_lib.df11_decode_host(_ptr_array([b.handle.value for b in blobs]), _ptr_array(host_image_ptrs),
                                 _ptr_array(dev_image_ptrs), _ptr_array(dst_dev_ptrs), _ptr_array(dst_host_ptrs),
                                 len(blobs), err_ptr or None, stream or None), "df11_decode_host")


def df11_decode_launch_shape(blobs, chunks_per_thread: int = 0, ctas_per_sm: int = 0,
                             warps_per_cta: int = 0, walker: int = 0, with_walk: bool = False,
                             max_ctas: int = 0, count_walk: int = 0):
    """(grid, block, shared-memory bytes) of the launch df11_decode_ex would
    make with these options; with_walk adds the walk it would use and whether
    it reads the stored chunk counts (0 / 1)."""
    g, b, s, w, c = _I(), _I(), _I(), _I(), _I()
    o = DecodeOpts(chunks_per_thread, ctas_per_sm, warps_per_cta, walker, max_ctas, 0, 0, count_walk)
    _check(_lib.df11_decode_launch_shape_ex(_ptr_array([x.handle.value for x in blobs]), len(blobs), ctypes.byref(o),
                                            ctypes.byref(g), ctypes.byref(b), ctypes.byref(s), ctypes.byref(w),
                                            ctypes.byref(c)),
           "df11_decode_launch_shape")
    return (g.value, b.value, s.value, w.value, c.value) if with_walk else (g.value, b.value, s.value)


def df11_decode_streamed(groups, host_image_ptrs, slot_ptrs, slot_bytes: int, dst_ptrs,
                         err_ptr: int | None = None, copy_stream: int = 0, decode_stream: int = 0):
    """groups: list of lists of blobs (one code per group); host_image_ptrs and
    dst_ptrs flat, in the same order as the blobs."""
    blobs = [b for g in groups for b in g]
    sizes = (ctypes.c_int32 * len(groups))(*[len(g) for g in groups])
    _check(_lib.df11_decode_streamed(_ptr_array([b.handle.value for b in blobs]), ctypes.cast(sizes, _P), len(groups),
                                     _ptr_array(host_image_ptrs), _ptr_array(slot_ptrs), len(slot_ptrs), slot_bytes,
                                     _ptr_array(dst_ptrs), err_ptr or None, copy_stream or None, decode_stream or None),
           "df11_decode_streamed")


def df11_histogram_device(dtype: str, src_ptr: int, n: int, counts_ptr: int, stream: int = 0):
    _check(_lib.df11_histogram_device(DTYPES[dtype], src_ptr or None, n, counts_ptr, stream or None),
           "df11_histogram_device")


def df11_codebook_from_counts(dtype: str, counts, max_code_len: int = 0) -> Codebook:
    c = np.ascontiguousarray(counts, np.uint64)
    out = ctypes.c_void_p()
    _check(_lib.df11_codebook_from_counts(DTYPES[dtype], c.ctypes.data, c.size, max_code_len, ctypes.byref(out)),
           "df11_codebook_from_counts")
    return Codebook(out.value, dtype)


def df11_encode_device_scratch_bytes(n: int) -> int:
    return int(_lib.df11_encode_device_scratch_bytes(n))


class Encoding:
    def __init__(self, handle: int, image_bytes: int):
        self._h = ctypes.c_void_p(handle)
        self.image_bytes = image_bytes

    def __del__(self, _free=_lib.df11_encoding_free):
        if getattr(self, "_h", None) and self._h.value:
            _free(self._h)
            self._h = None


def df11_encode_device_begin(cb: Codebook, src_ptr: int, n: int, chunk_bits: int = 128, tile_threads: int = 32,
                             scratch_ptr: int = 0, scratch_cap: int = 0, stream: int = 0,
                             chunk_counts: bool = True) -> Encoding:
    nbytes = _U64()
    out = ctypes.c_void_p()
    _check(_lib.df11_encode_device_begin(cb.handle, src_ptr or None, n, chunk_bits, tile_threads,
                                         _encode_flags(chunk_counts), scratch_ptr or None, scratch_cap,
                                         stream or None, ctypes.byref(nbytes), ctypes.byref(out)),
           "df11_encode_device_begin")
    return Encoding(out.value, nbytes.value)


def df11_encode_device_end(enc: Encoding, image_ptr: int, image_cap: int, keep=None) -> Blob:
    out = ctypes.c_void_p()
    _check(_lib.df11_encode_device_end(enc._h, image_ptr, image_cap, ctypes.byref(out)), "df11_encode_device_end")
    b = Blob(out.value)
    b._keep = keep
    return b


def df11_blob_fetch(blob: Blob, stream: int = 0):
    _check(_lib.df11_blob_fetch(blob.handle, stream or None), "df11_blob_fetch")


NOALLOC_SCRATCH_BYTES = 65536 * 8
NOALLOC_MAX_ELEMS = (65536 - 163) * 4096


def df11_encode_device_noalloc(cb: Codebook, src_ptr: int, n: int, chunk_bits: int, tile_threads: int,
                               image_ptr: int, image_cap: int, stream: int = 0,
                               chunk_counts: bool = True) -> EncodeResult:
    """GPU encode for callers that cannot allocate device memory: scratch is a
    static device array of the library, so n is limited to NOALLOC_MAX_ELEMS.
    Raises Df11Error (status DF11_ENOMEM with .result.image_bytes set when
    the image buffer is too small)."""
    r = EncodeResult()
    st = _lib.df11_encode_device_noalloc(cb.handle, src_ptr or None, n, chunk_bits, tile_threads,
                                         _encode_flags(chunk_counts), image_ptr or None, image_cap, stream or None,
                                         ctypes.byref(r))
    if st != DF11_OK:
        e = Df11Error(st, "df11_encode_device_noalloc")
        e.result = r
        raise e
    return r


# ----------------------------------------------------------------- decode fused into the consuming GEMM

def df11_gemm_tile_weights(w: np.ndarray, k: int, n: int) -> np.ndarray:
    """The operand-tile order of a K x N BF16 matrix (uint16 bits, row-major)."""
    w = np.ascontiguousarray(w, dtype=np.uint16).reshape(-1)
    if w.size != k * n:
        raise ValueError("w must hold k * n weights")
    out = np.empty(k * n, np.uint16)
    _check(_lib.df11_gemm_tile_weights(w.ctypes.data, k, n, out.ctypes.data), "df11_gemm_tile_weights")
    return out


def _gemm_array(mats):
    arr = (GemmMatrix * len(mats))()
    for i, (blob, k, n, x_ptr, y_ptr) in enumerate(mats):
        arr[i] = GemmMatrix(blob.handle.value, k, n, x_ptr or None, y_ptr or None)
    return arr


def df11_decode_gemm(mats, m: int, err_ptr: int | None = None, stream: int = 0):
    """mats: (blob, K, N, x device pointer, y device pointer) per matrix; y += x W."""
    _check(_lib.df11_decode_gemm(_gemm_array(mats), len(mats), m, err_ptr or None, stream or None), "df11_decode_gemm")


def df11_decode_gemm_launch_shape(mats, m: int):
    """(grid, threads per CTA, dynamic shared memory bytes); pointers may be 0."""
    g, b, s = _I(), _I(), _I()
    _check(_lib.df11_decode_gemm_launch_shape(_gemm_array(mats), len(mats), m, ctypes.byref(g), ctypes.byref(b),
                                              ctypes.byref(s)), "df11_decode_gemm_launch_shape")
    return g.value, b.value, s.value


# ----------------------------------------------------------------- torch-side helpers (device memory only)

def upload(blob: Blob, stream=None):
    """Allocates the device image with torch, copies it there and binds it.
    Returns the torch tensor that owns the image (also kept on the blob)."""
    import torch
    n = blob.info().device_bytes
    dev = torch.empty(n + 256, dtype=torch.uint8, device="cuda")
    base = dev.data_ptr()
    off = (-base) % 256
    s = stream.cuda_stream if stream is not None else torch.cuda.current_stream().cuda_stream
    df11_blob_upload(blob, base + off, n, s, keep=dev)
    return dev


def encode_on_device(cb: Codebook, x_dev, chunk_bits: int = 128, tile_threads: int = 32, stream=None,
                     chunk_counts: bool = True) -> Blob:
    """GPU encode of a torch device tensor (raw uint16 / uint8 bits); scratch
    and the image are allocated with torch.  Returns a blob bound to its image."""
    import torch
    s = stream.cuda_stream if stream is not None else torch.cuda.current_stream().cuda_stream
    n = x_dev.numel()
    scratch = torch.empty(df11_encode_device_scratch_bytes(n), dtype=torch.uint8, device=x_dev.device)
    enc = df11_encode_device_begin(cb, x_dev.data_ptr(), n, chunk_bits, tile_threads, scratch.data_ptr(),
                                   scratch.numel(), s, chunk_counts)
    img = torch.empty(enc.image_bytes + 256, dtype=torch.uint8, device=x_dev.device)
    base = img.data_ptr() + (-img.data_ptr()) % 256
    return df11_encode_device_end(enc, base, enc.image_bytes, keep=img)


def elem_bytes(dtype: str) -> int:
    return 2 if dtype == "bf16" else 1


def empty_output(blob: Blob):
    """A device buffer (torch uint8, 16-byte aligned) for the decoded tensor."""
    import torch
    i = blob.info()
    nbytes = i.n_elems * (2 if i.dtype == DF11_BF16 else 1)
    return torch.empty(max(nbytes, 16), dtype=torch.uint8, device="cuda")


# ----------------------------------------------------------------- rANS coder (same names as the C-ABI)

RANS_TILE_DEFAULT = 16384


class RansGroup:
    """Tensors coded with one rANS frequency table (df11_rans_group)."""

    def __init__(self, handle: int, dtype: str, n_tensors: int):
        self._h = ctypes.c_void_p(handle)
        self.dtype = dtype
        self.n_tensors = n_tensors
        self._keep = None

    @property
    def handle(self):
        return self._h

    def freqs(self) -> np.ndarray:
        f = np.zeros(256, np.uint32)
        _check(_lib.df11_rans_group_freqs(self._h, f.ctypes.data), "df11_rans_group_freqs")
        return f[: 256 if self.dtype == "bf16" else 16]

    def info(self, i: int) -> RansTensorInfo:
        r = RansTensorInfo()
        _check(_lib.df11_rans_group_info(self._h, i, ctypes.byref(r)), "df11_rans_group_info")
        return r

    def sections(self, i: int) -> dict:
        """Copies of tensor i's words, states, tile_words and plane."""
        inf = self.info(i)
        ptrs = [ctypes.c_void_p() for _ in range(4)]
        _check(_lib.df11_rans_group_sections(self._h, i, *[ctypes.byref(p) for p in ptrs]), "df11_rans_group_sections")

        def grab(p, n, dt):
            if n == 0:
                return np.zeros(0, dt)
            nb = n * np.dtype(dt).itemsize
            return np.ctypeslib.as_array(ctypes.cast(p, ctypes.POINTER(ctypes.c_uint8)), (nb,)).view(dt).copy()

        return {"words": grab(ptrs[0], inf.words, np.uint16), "states": grab(ptrs[1], inf.n_tiles * 32, np.uint32),
                "tile_words": grab(ptrs[2], inf.n_tiles + 1, np.uint64),
                "plane": grab(ptrs[3], inf.plane_bytes, np.uint8)}

    def device_bytes(self) -> int:
        return int(_lib.df11_rans_group_device_bytes(self._h))

    def __del__(self, _free=_lib.df11_rans_group_free):
        if getattr(self, "_h", None) and self._h.value:
            _free(self._h)
            self._h = None


def df11_rans_encode_group(dtype: str, tensors, tile_symbols: int = 0, n_threads: int = 0) -> RansGroup:
    arrs = [np.ascontiguousarray(t).reshape(-1) for t in tensors]
    ptrs = _ptr_array([a.ctypes.data if a.size else None for a in arrs])
    ns = (_U64 * len(arrs))(*[a.size for a in arrs])
    out = ctypes.c_void_p()
    _check(_lib.df11_rans_encode_group(DTYPES[dtype], ptrs, ns, len(arrs), tile_symbols, n_threads,
                                       ctypes.byref(out)), "df11_rans_encode_group")
    return RansGroup(out.value, dtype, len(arrs))


def df11_rans_group_serialize(g: RansGroup) -> bytes:
    need = _U64()
    _lib.df11_rans_group_serialize(g.handle, None, 0, ctypes.byref(need))
    buf = ctypes.create_string_buffer(need.value)
    _check(_lib.df11_rans_group_serialize(g.handle, buf, need.value, ctypes.byref(need)), "df11_rans_group_serialize")
    return buf.raw[: need.value]


def df11_rans_group_deserialize(data) -> RansGroup:
    b = bytes(data)
    out = ctypes.c_void_p()
    _check(_lib.df11_rans_group_deserialize(b, len(b), ctypes.byref(out)), "df11_rans_group_deserialize")
    dt = "bf16" if struct.unpack_from("<I", b, 12)[0] == DF11_BF16 else "e4m3"
    return RansGroup(out.value, dt, struct.unpack_from("<I", b, 24)[0])


def df11_rans_group_upload(g: RansGroup, dev_ptr: int, cap: int, stream: int = 0, keep=None):
    _check(_lib.df11_rans_group_upload(g.handle, dev_ptr, cap, stream or None), "df11_rans_group_upload")
    g._keep = keep


def df11_rans_decode(g: RansGroup, dst_ptrs, err_ptr: int | None = None, stream: int = 0):
    _check(_lib.df11_rans_decode(g.handle, _ptr_array(dst_ptrs), err_ptr or None, stream or None), "df11_rans_decode")


def df11_rans_decode_launch_shape(g: RansGroup):
    a, b, c = _I(), _I(), _I()
    _check(_lib.df11_rans_decode_launch_shape(g.handle, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)),
           "df11_rans_decode_launch_shape")
    return a.value, b.value, c.value


def rans_upload(g: RansGroup, stream=None):
    """Allocates the group's device image with torch, copies it and binds it."""
    import torch
    n = g.device_bytes()
    dev = torch.empty(n + 256, dtype=torch.uint8, device="cuda")
    base = dev.data_ptr()
    off = (-base) % 256
    s = stream.cuda_stream if stream is not None else torch.cuda.current_stream().cuda_stream
    df11_rans_group_upload(g, base + off, n, s, keep=dev)
    return dev
