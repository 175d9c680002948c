"""CPU oracle for the DFloat11 exponent code -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product (``entropy_decoding_b200``)
never imports it and shares no code with it.

The arithmetic lives in ``df11_oracle.c`` (plain single-threaded C, one
function per step of the method, each citing the passage it follows); this
module only marshals numpy arrays into it and strings the steps together in
the order the method states them:

  split fields -> histogram -> code lengths -> canonical codes -> pack
  -> auxiliary variables          (compression, done offline)
  bit-by-bit tree walk -> merge fields                           (decompression)
  decompression -> operand-tile order undone -> y = x W          (the fused GEMM)

Sources: "70% Size, 100% Accuracy: Lossless LLM Compression for Efficient GPU
Inference via Dynamic-Length Float (DFloat11)", Abstract; "Compressing LLMs
without Compromise" summary page, sections "Where the redundancy lives" and
"Three ways to spend the savings"; "To Compress or Not? ... Exponent
Concentration", Abstract (FP8 variant).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "df11_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "liboracle.so")

NSYM = {"bf16": 256, "e4m3": 16}


def build(force: bool = False) -> str:
    """Compile df11_oracle.c with gcc into oracle/_build/liboracle.so."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    os.makedirs(_LIB_DIR, exist_ok=True)
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-Wall", "-Wextra", "-shared", "-fPIC",
                           "-o", tmp, _SRC])
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        U64 = ctypes.c_uint64
        I = ctypes.c_int
        lib.oracle_split_bf16.argtypes = [P, U64, P, P]
        lib.oracle_split_e4m3.argtypes = [P, U64, P, P]
        lib.oracle_merge_bf16.argtypes = [P, P, U64, P]
        lib.oracle_merge_e4m3.argtypes = [P, P, U64, P]
        lib.oracle_histogram.argtypes = [P, U64, P]
        lib.oracle_code_lengths.argtypes = [P, I, I, P]
        lib.oracle_code_lengths.restype = I
        lib.oracle_huffman_depth.argtypes = [P, I, P]
        lib.oracle_huffman_depth.restype = I
        lib.oracle_canonical_codes.argtypes = [P, I, P]
        lib.oracle_total_bits.argtypes = [P, U64, P]
        lib.oracle_total_bits.restype = U64
        lib.oracle_pack.argtypes = [P, U64, P, P, P, U64]
        lib.oracle_pack.restype = I
        lib.oracle_layout.argtypes = [U64, I, I, P, P]
        lib.oracle_aux.argtypes = [P, U64, P, I, I, P, P, P]
        lib.oracle_aux.restype = I
        lib.oracle_chunk_counts.argtypes = [P, U64, P, I, I, P]
        lib.oracle_chunk_counts.restype = I
        lib.oracle_rans_freqs.argtypes = [P, I, P]
        lib.oracle_rans_freqs.restype = I
        lib.oracle_rans_encode.argtypes = [P, U64, P, I, ctypes.c_uint32, P, U64, P, P]
        lib.oracle_rans_encode.restype = I
        lib.oracle_rans_words_bound.argtypes = [U64, ctypes.c_uint32]
        lib.oracle_rans_words_bound.restype = U64
        lib.oracle_rans_decode.argtypes = [P, P, P, U64, P, I, ctypes.c_uint32, P]
        lib.oracle_rans_decode.restype = I
        lib.oracle_decode.argtypes = [P, U64, P, I, U64, U64, P]
        lib.oracle_decode.restype = I
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


class OracleError(RuntimeError):
    pass


def _check(rc: int, what: str):
    if rc != 0:
        raise OracleError(f"{what} failed with code {rc}")


# ---------------------------------------------------------------- steps

def split(x: np.ndarray, dtype: str):
    """Weights -> (exponent symbols, raw sign+mantissa plane)."""
    lib = _load()
    n = x.size
    exps = np.empty(n, np.uint8)
    if dtype == "bf16":
        x = np.ascontiguousarray(x, dtype=np.uint16)
        plane = np.empty(n, np.uint8)
        lib.oracle_split_bf16(_p(x), n, _p(exps), _p(plane))
    elif dtype == "e4m3":
        x = np.ascontiguousarray(x, dtype=np.uint8)
        plane = np.empty((n + 1) // 2, np.uint8)
        lib.oracle_split_e4m3(_p(x), n, _p(exps), _p(plane))
    else:
        raise ValueError(dtype)
    return exps, plane


def merge(exps: np.ndarray, plane: np.ndarray, n: int, dtype: str) -> np.ndarray:
    lib = _load()
    exps = np.ascontiguousarray(exps, np.uint8)
    plane = np.ascontiguousarray(plane, np.uint8)
    if dtype == "bf16":
        out = np.empty(n, np.uint16)
        lib.oracle_merge_bf16(_p(exps), _p(plane), n, _p(out))
    else:
        out = np.empty(n, np.uint8)
        lib.oracle_merge_e4m3(_p(exps), _p(plane), n, _p(out))
    return out


def histogram(exps: np.ndarray, counts: np.ndarray | None = None) -> np.ndarray:
    lib = _load()
    if counts is None:
        counts = np.zeros(256, np.uint64)
    exps = np.ascontiguousarray(exps, np.uint8)
    lib.oracle_histogram(_p(exps), exps.size, _p(counts))
    return counts


def code_lengths(counts: np.ndarray, nsym: int, max_len: int = 32) -> np.ndarray:
    lib = _load()
    c = np.zeros(256, np.uint64)
    c[: len(counts)] = counts
    lengths = np.zeros(256, np.uint8)
    _check(lib.oracle_code_lengths(_p(c), nsym, max_len, _p(lengths)), "code_lengths")
    return lengths[:nsym].copy()


def huffman_depth(counts: np.ndarray, nsym: int):
    """Unconstrained Huffman lengths and their maximum."""
    lib = _load()
    c = np.zeros(256, np.uint64)
    c[: len(counts)] = counts
    lengths = np.zeros(256, np.uint8)
    d = lib.oracle_huffman_depth(_p(c), nsym, _p(lengths))
    return d, lengths[:nsym].copy()


def canonical_codes(lengths: np.ndarray) -> np.ndarray:
    lib = _load()
    nsym = len(lengths)
    ln = np.ascontiguousarray(lengths, np.uint8)
    codes = np.zeros(nsym, np.uint32)
    lib.oracle_canonical_codes(_p(ln), nsym, _p(codes))
    return codes


def total_bits(exps: np.ndarray, lengths: np.ndarray) -> int:
    lib = _load()
    ln = np.zeros(256, np.uint8)
    ln[: len(lengths)] = lengths
    exps = np.ascontiguousarray(exps, np.uint8)
    return int(lib.oracle_total_bits(_p(exps), exps.size, _p(ln)))


def pack(exps: np.ndarray, lengths: np.ndarray, codes: np.ndarray) -> tuple[np.ndarray, int]:
    lib = _load()
    ln = np.zeros(256, np.uint8)
    ln[: len(lengths)] = lengths
    cd = np.zeros(256, np.uint32)
    cd[: len(codes)] = codes
    exps = np.ascontiguousarray(exps, np.uint8)
    tb = total_bits(exps, ln)
    stream = np.zeros((tb + 7) // 8, np.uint8)
    _check(lib.oracle_pack(_p(exps), exps.size, _p(ln), _p(cd), _p(stream), stream.size), "pack")
    return stream, tb


def layout(total: int, chunk_bits: int, tile_threads: int) -> tuple[int, int]:
    lib = _load()
    nc = ctypes.c_uint64()
    nt = ctypes.c_uint64()
    lib.oracle_layout(total, chunk_bits, tile_threads, ctypes.byref(nc), ctypes.byref(nt))
    return int(nc.value), int(nt.value)


def aux(exps: np.ndarray, lengths: np.ndarray, chunk_bits: int, tile_threads: int):
    lib = _load()
    ln = np.zeros(256, np.uint8)
    ln[: len(lengths)] = lengths
    exps = np.ascontiguousarray(exps, np.uint8)
    tb = total_bits(exps, ln)
    _, nt = layout(tb, chunk_bits, tile_threads)
    gaps = np.zeros(max(nt * tile_threads, 1), np.uint8)
    out_off = np.zeros(nt + 1, np.uint64)
    ms = ctypes.c_uint64()
    _check(lib.oracle_aux(_p(exps), exps.size, _p(ln), chunk_bits, tile_threads,
                          _p(gaps), _p(out_off), ctypes.byref(ms)), "aux")
    return gaps[: nt * tile_threads].copy(), out_off, int(ms.value)


def chunk_counts(exps: np.ndarray, lengths: np.ndarray, chunk_bits: int, tile_threads: int) -> np.ndarray:
    """Codes starting in each chunk (n_tiles * tile_threads bytes, 0 past the
    last chunk): what the first phase of the two-phase kernel counts."""
    lib = _load()
    ln = np.zeros(256, np.uint8)
    ln[: len(lengths)] = lengths
    exps = np.ascontiguousarray(exps, np.uint8)
    _, nt = layout(total_bits(exps, ln), chunk_bits, tile_threads)
    out = np.zeros(max(nt * tile_threads, 1), np.uint8)
    _check(lib.oracle_chunk_counts(_p(exps), exps.size, _p(ln), chunk_bits, tile_threads, _p(out)), "chunk_counts")
    return out[: nt * tile_threads].copy()


def decode(stream: np.ndarray, total: int, lengths: np.ndarray, start_bit: int, count: int) -> np.ndarray:
    lib = _load()
    nsym = len(lengths)
    ln = np.ascontiguousarray(lengths, np.uint8)
    stream = np.ascontiguousarray(stream, np.uint8)
    if stream.size == 0:
        stream = np.zeros(1, np.uint8)
    out = np.empty(max(count, 1), np.uint8)
    _check(lib.oracle_decode(_p(stream), total, _p(ln), nsym, start_bit, count, _p(out)), "decode")
    return out[:count]


# ---------------------------------------------------------------- whole method

@dataclass
class Compressed:
    dtype: str
    n: int
    lengths: np.ndarray      # code length per symbol (0 = unused)
    codes: np.ndarray        # canonical code per symbol
    stream: np.ndarray       # ceil(total_bits / 8) bytes, MSB-first
    total_bits: int
    plane: np.ndarray        # raw sign+mantissa field
    gaps: np.ndarray         # one byte per chunk, padded to whole tiles
    out_off: np.ndarray      # n_tiles + 1 entries
    max_span: int
    chunk_bits: int
    tile_threads: int

    @property
    def n_tiles(self) -> int:
        return len(self.out_off) - 1


def build_lengths(tensors, dtype: str, max_len: int = 32) -> np.ndarray:
    """One code for a group of tensors: histogram summed over all of them."""
    counts = np.zeros(256, np.uint64)
    for x in tensors:
        exps, _ = split(x, dtype)
        histogram(exps, counts)
    return code_lengths(counts[: NSYM[dtype]], NSYM[dtype], max_len)


def compress(x: np.ndarray, dtype: str, lengths: np.ndarray | None = None, max_len: int = 32,
             chunk_bits: int = 128, tile_threads: int = 256) -> Compressed:
    x = np.ascontiguousarray(x).reshape(-1)
    exps, plane = split(x, dtype)
    if lengths is None:
        counts = histogram(exps)
        lengths = code_lengths(counts[: NSYM[dtype]], NSYM[dtype], max_len)
    codes = canonical_codes(lengths)
    stream, tb = pack(exps, lengths, codes)
    gaps, out_off, ms = aux(exps, lengths, chunk_bits, tile_threads)
    return Compressed(dtype, x.size, lengths, codes, stream, tb, plane, gaps, out_off, ms,
                      chunk_bits, tile_threads)


def decompress(c: Compressed) -> np.ndarray:
    exps = decode(c.stream, c.total_bits, c.lengths, 0, c.n)
    return merge(exps, c.plane, c.n, c.dtype)


def decode_at(c: Compressed, start_bit: int, count: int) -> np.ndarray:
    """Exponent symbols of `count` consecutive weights whose first code starts
    at `start_bit` (a sampled slice, decoded one symbol at a time)."""
    return decode(c.stream, c.total_bits, c.lengths, start_bit, count)


# ---------------------------------------------------------------- rANS variant
# ("Approaching Shannon Bound with Lossless LLM Weight Compression", Abstract:
# ANS decoding by tiles; coder details are the readings of df11_oracle.c
# section 9)

RANS_BITS = 12
RANS_M = 1 << RANS_BITS
RANS_L = 1 << 16
RANS_LANES = 32


def rans_freqs(counts: np.ndarray, nsym: int) -> np.ndarray:
    """Quantized frequencies (sum 2^12) from exponent counts."""
    lib = _load()
    c = np.zeros(256, np.uint64)
    c[:nsym] = np.asarray(counts, np.uint64)[:nsym]
    f = np.zeros(256, np.uint32)
    _check(lib.oracle_rans_freqs(_p(c), nsym, _p(f)), "rans_freqs")
    return f[:nsym].copy()


def rans_encode(exps: np.ndarray, freqs: np.ndarray, tile_symbols: int):
    """(words u16, states u32 [n_tiles * 32], tile_words u64 [n_tiles + 1])."""
    lib = _load()
    exps = np.ascontiguousarray(exps, np.uint8)
    fr = np.ascontiguousarray(freqs, np.uint32)
    n = exps.size
    n_tiles = -(-n // tile_symbols)
    cap = int(lib.oracle_rans_words_bound(n, tile_symbols))
    words = np.zeros(max(cap, 1), np.uint16)
    states = np.zeros(max(n_tiles * RANS_LANES, 1), np.uint32)
    tile_words = np.zeros(n_tiles + 1, np.uint64)
    src = exps if n else np.zeros(1, np.uint8)
    _check(lib.oracle_rans_encode(_p(src), n, _p(fr), fr.size, tile_symbols, _p(words), cap, _p(states),
                                  _p(tile_words)), "rans_encode")
    return words[: int(tile_words[-1])].copy(), states[: n_tiles * RANS_LANES].copy(), tile_words


def rans_decode(words: np.ndarray, states: np.ndarray, tile_words: np.ndarray, n: int, freqs: np.ndarray,
                tile_symbols: int) -> np.ndarray:
    lib = _load()
    w = np.ascontiguousarray(words, np.uint16) if words.size else np.zeros(1, np.uint16)
    st = np.ascontiguousarray(states, np.uint32) if states.size else np.zeros(1, np.uint32)
    tw = np.ascontiguousarray(tile_words, np.uint64)
    fr = np.ascontiguousarray(freqs, np.uint32)
    out = np.zeros(max(n, 1), np.uint8)
    _check(lib.oracle_rans_decode(_p(w), _p(st), _p(tw), n, _p(fr), fr.size, tile_symbols, _p(out)),
           "rans_decode")
    return out[:n]


@dataclass
class RansCompressed:
    dtype: str
    n: int
    freqs: np.ndarray       # quantized frequencies, sum 2^12
    words: np.ndarray       # u16 words, tiles 8-word aligned
    states: np.ndarray      # u32, 32 per tile
    tile_words: np.ndarray  # u64, n_tiles + 1
    plane: np.ndarray       # raw sign+mantissa field, as the Huffman container's
    tile_symbols: int


def rans_compress(x: np.ndarray, dtype: str, freqs: np.ndarray | None = None,
                  tile_symbols: int = 16384) -> RansCompressed:
    x = np.ascontiguousarray(x).reshape(-1)
    exps, plane = split(x, dtype)
    if freqs is None:
        freqs = rans_freqs(histogram(exps)[: NSYM[dtype]], NSYM[dtype])
    words, states, tile_words = rans_encode(exps, freqs, tile_symbols)
    return RansCompressed(dtype, x.size, freqs, words, states, tile_words, plane, tile_symbols)


def rans_decompress(c: RansCompressed) -> np.ndarray:
    exps = rans_decode(c.words, c.states, c.tile_words, c.n, c.freqs, c.tile_symbols)
    return merge(exps, c.plane, c.n, c.dtype)


# ---------------------------------------------------------------- decode fused into the consuming GEMM
# ("Compressing LLMs without Compromise" summary page, ZipServ paragraph:
# decompression fused into the matrix multiply; "Approaching Shannon Bound
# with Lossless LLM Weight Compression", Abstract: decoding aligned with the
# GEMM's tiling).  Fusing changes where the decoded weights go, not what is
# computed: the result is the plain product y = x W of the exactly decoded
# weights.  The pages give no tile shape; the reading here is a tcgen05
# operand tile of 128 output rows x 64 reduction columns (one 128-byte
# swizzle row of BF16 per output row), each tile a contiguous run of the
# encoded weights.

GEMM_TILE_N, GEMM_TILE_K = 128, 64


def gemm_tile(w: np.ndarray, k: int, n: int) -> np.ndarray:
    """Operand-tile order of a K x N matrix (row-major, element (k, n) at
    k * N + n): tile t = nb * (K / 64) + kb holds W[64 kb + c][128 nb + r] at
    position 8192 t + 64 r + c."""
    w = np.asarray(w).reshape(k, n)
    return w.reshape(k // GEMM_TILE_K, GEMM_TILE_K, n // GEMM_TILE_N, GEMM_TILE_N).transpose(2, 0, 3, 1).reshape(-1)


def gemm_untile(t: np.ndarray, k: int, n: int) -> np.ndarray:
    """Inverse of gemm_tile: the K x N row-major matrix."""
    t = np.asarray(t).reshape(n // GEMM_TILE_N, k // GEMM_TILE_K, GEMM_TILE_N, GEMM_TILE_K)
    return t.transpose(1, 3, 0, 2).reshape(k, n)


def bf16_to_float(bits: np.ndarray) -> np.ndarray:
    """BF16 bit patterns -> float64 values (BF16 is the high half of FP32)."""
    return (np.asarray(bits, np.uint32) << 16).view(np.float32).astype(np.float64)


def gemm(x_bits: np.ndarray, w_bits: np.ndarray, m: int, k: int, n: int) -> np.ndarray:
    """y = x W in float64 from BF16 bit patterns: x is m x k, W is k x n."""
    return bf16_to_float(x_bits).reshape(m, k) @ bf16_to_float(w_bits).reshape(k, n)


def gemm_abs(x_bits: np.ndarray, w_bits: np.ndarray, m: int, k: int, n: int) -> np.ndarray:
    """sum_k |x_mk w_kn|, the scale of a float32 accumulation's rounding error."""
    return np.abs(bf16_to_float(x_bits).reshape(m, k)) @ np.abs(bf16_to_float(w_bits).reshape(k, n))


def decode_gemm(c: Compressed, x_bits: np.ndarray, m: int, k: int, n: int) -> np.ndarray:
    """What the fused path computes from a tiled container: decompress,
    restore the K x N order, multiply (float64)."""
    return gemm(x_bits, gemm_untile(decompress(c), k, n), m, k, n)
