// encode.cu -- GPU encoder: the offline half of the method run on the device.
//
// "70% Size, 100% Accuracy ... (DFloat11)", Abstract: frequency-based
// dynamic-length codes over the exponent field, plus the auxiliary variables
// (per-chunk gap, per-tile output offset) that coordinate the decoder's
// threads.  "Compressing LLMs without Compromise" summary page, section
// "Three ways to spend the savings": the exponents are Huffman-coded offline;
// here the histogram, the bit packing and the auxiliary variables run on the
// GPU, the code construction (256 or 16 counts) stays on the host.
//
// Output is a device image in the layout the decoder reads (see
// codec.cpp image_layout): stream as 32-bit words with the earliest bit in
// bit 31, byte plane, gaps, out_off, and the decode tables.
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "df11.h"
#include "encode.h"

namespace df11 {
namespace {

constexpr int kEncThreads = 256;
constexpr int kElemsPerThread = 16;
constexpr uint32_t kSegElems = kEncThreads * kElemsPerThread;  // 4096 elements per segment
// chunks a segment's codes can start in: its bits (at most 32 per element)
// over the smallest chunk that stores counts (64 bits), plus both ends
constexpr uint32_t kSegChunks = kSegElems * kMaxCodeLen / 64 + 2;

template <int DT>
__device__ __forceinline__ uint32_t exponent_at(const void *src, uint64_t i) {
    if constexpr (DT == 0) return (static_cast<const uint16_t *>(src)[i] >> 7) & 0xFFu;
    return (static_cast<const uint8_t *>(src)[i] >> 3) & 0xFu;
}

// Loads a thread's 16 elements (fewer at the tensor end) as exponent symbols
// and raw fields.
template <int DT>
__device__ __forceinline__ int load16(const void *src, uint64_t n, uint64_t i0, uint32_t (&e)[16], uint32_t (&f)[16]) {
    int cnt = 0;
    if (i0 + 16 <= n) {
        cnt = 16;
        if constexpr (DT == 0) {
            const uint4 *p = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(src) + i0);
            const uint4 a = __ldg(p), b = __ldg(p + 1);
            const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const uint32_t v = (w[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
                e[j] = (v >> 7) & 0xFFu;
                f[j] = ((v >> 8) & 0x80u) | (v & 0x7Fu);
            }
        } else {
            const uint4 a = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(src) + i0));
            const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const uint32_t v = (w[j >> 2] >> (8 * (j & 3))) & 0xFFu;
                e[j] = (v >> 3) & 0xFu;
                f[j] = ((v >> 4) & 0x8u) | (v & 0x7u);
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            e[j] = 0;
            f[j] = 0;
            if (i0 + j < n) {
                if constexpr (DT == 0) {
                    const uint32_t v = static_cast<const uint16_t *>(src)[i0 + j];
                    e[j] = (v >> 7) & 0xFFu;
                    f[j] = ((v >> 8) & 0x80u) | (v & 0x7Fu);
                } else {
                    const uint32_t v = static_cast<const uint8_t *>(src)[i0 + j];
                    e[j] = (v >> 3) & 0xFu;
                    f[j] = ((v >> 4) & 0x8u) | (v & 0x7u);
                }
                ++cnt;
            }
        }
    }
    return cnt;
}

// Inclusive block scan of one value per thread (kEncThreads threads).
__device__ __forceinline__ uint32_t block_inclusive_scan(uint32_t v, uint32_t *s_warp, uint32_t &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, v, o);
        if (lane >= o) v += t;
    }
    if (lane == 31) s_warp[warp] = v;
    __syncthreads();
    uint32_t before = 0;
    total = 0;
#pragma unroll
    for (int w = 0; w < kEncThreads / 32; ++w) {
        const uint32_t t = s_warp[w];
        before += w < warp ? t : 0u;
        total += t;
    }
    __syncthreads();
    return v + before;
}

// ---------------------------------------------------------------- histogram

// Exponent histogram: per-warp sub-histograms in shared memory, then one
// atomic add per bin and CTA into the 64-bit counts.
template <int DT>
__global__ void __launch_bounds__(kEncThreads) hist_kernel(const void *src, uint64_t n, unsigned long long *counts) {
    constexpr int NB = DT == 0 ? 256 : 16;
    __shared__ uint32_t h[kEncThreads / 32][256];
    const int warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < (kEncThreads / 32) * 256; i += kEncThreads) (&h[0][0])[i] = 0;
    __syncthreads();
    const uint64_t stride = static_cast<uint64_t>(gridDim.x) * kSegElems;
    for (uint64_t base = static_cast<uint64_t>(blockIdx.x) * kSegElems; base < n; base += stride) {
        uint32_t e[16], f[16];
        const int c = load16<DT>(src, n, base + threadIdx.x * 16u, e, f);
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (j < c) atomicAdd(&h[warp][e[j]], 1u);
    }
    __syncthreads();
    for (int b = threadIdx.x; b < NB; b += kEncThreads) {
        uint64_t s = 0;
        for (int w = 0; w < kEncThreads / 32; ++w) s += h[w][b];
        if (s) atomicAdd(counts + b, static_cast<unsigned long long>(s));
    }
}

// ---------------------------------------------------------------- pass 1: bits per segment

template <int DT>
__global__ void __launch_bounds__(kEncThreads)
    seg_bits_kernel(const void *src, uint64_t n, const uint8_t *lengths, uint64_t n_seg, uint64_t *seg_bits,
                    unsigned long long *uncovered) {
    __shared__ uint8_t s_len[256];
    __shared__ uint32_t s_warp[kEncThreads / 32];
    s_len[threadIdx.x] = lengths[threadIdx.x];
    __syncthreads();
    for (uint64_t seg = blockIdx.x; seg < n_seg; seg += gridDim.x) {
        uint32_t e[16], f[16];
        const int c = load16<DT>(src, n, seg * kSegElems + threadIdx.x * 16u, e, f);
        uint32_t bits = 0;
        bool missing = false;
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (j < c) {
                bits += s_len[e[j]];
                missing |= s_len[e[j]] == 0;
            }
        if (missing) atomicOr(uncovered, 1ull);
        uint32_t total;
        block_inclusive_scan(bits, s_warp, total);
        if (threadIdx.x == 0) seg_bits[seg] = total;
    }
}

// Exclusive scan of the segment bit counts in place (one CTA); the total goes
// to *total_bits.
__global__ void __launch_bounds__(1024) seg_scan_kernel(uint64_t *seg, uint64_t n_seg, uint64_t *total_bits) {
    __shared__ uint64_t s_part[1024];
    const uint64_t per = (n_seg + 1023) / 1024;
    const uint64_t b = threadIdx.x * per, e = b + per < n_seg ? b + per : n_seg;
    uint64_t sum = 0;
    for (uint64_t i = b; i < e; ++i) sum += seg[i];
    s_part[threadIdx.x] = sum;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {  // Hillis-Steele over 1024 partial sums
        const uint64_t t = threadIdx.x >= o ? s_part[threadIdx.x - o] : 0;
        __syncthreads();
        s_part[threadIdx.x] += t;
        __syncthreads();
    }
    uint64_t run = s_part[threadIdx.x] - sum;
    for (uint64_t i = b; i < e; ++i) {
        const uint64_t v = seg[i];
        seg[i] = run;
        run += v;
    }
    if (threadIdx.x == 1023) *total_bits = s_part[1023];
}

// ---------------------------------------------------------------- pass 2: pack

struct PackArgs {
    const void *src;
    uint64_t n;
    const uint8_t *lengths;
    const uint32_t *codes;
    const uint64_t *seg_off;
    uint64_t n_seg;
    uint32_t *stream;  // words, earliest bit in bit 31; zeroed
    uint8_t *plane;
    uint8_t *gaps;      // zeroed
    uint32_t *counts;   // chunk counts as words (byte c at bits 8 * (c % 4) of word c / 4), zeroed; or nullptr
    uint64_t *out_off;  // filled with n
    uint32_t chunk_bits;
    uint64_t tile_bits;
};

__device__ __forceinline__ void or_code(uint32_t *stream, uint64_t o, uint32_t code, uint32_t len) {
    const uint64_t w = o >> 5;
    const uint32_t r = static_cast<uint32_t>(o & 31u);
    if (r + len <= 32) {
        atomicOr(stream + w, code << (32 - r - len));
    } else {
        const uint32_t spill = r + len - 32;  // bits that go to the next word
        atomicOr(stream + w, code >> spill);
        atomicOr(stream + w + 1, code << (32 - spill));
    }
}

// Chunk counts are tallied per segment in shared memory (s_cnt[c - c_lo] for
// the segment's chunks [c_lo, c_hi]) and written out by words of 4 chunks: a
// word whose chunks all lie strictly inside the range belongs to this segment
// alone (a neighbouring segment's codes start at or before c_lo, or at or
// after c_hi) and is stored; the words at the ends are added atomically.
template <int DT>
__global__ void __launch_bounds__(kEncThreads) pack_kernel(const PackArgs A) {
    __shared__ uint8_t s_len[256];
    __shared__ uint32_t s_code[256];
    __shared__ uint32_t s_warp[kEncThreads / 32];
    __shared__ uint32_t s_cnt[kSegChunks];
    s_len[threadIdx.x] = A.lengths[threadIdx.x];
    s_code[threadIdx.x] = A.codes[threadIdx.x];
    for (uint32_t i = threadIdx.x; i < kSegChunks; i += kEncThreads) s_cnt[i] = 0;
    __syncthreads();
    const uint64_t cb = A.chunk_bits;
    for (uint64_t seg = blockIdx.x; seg < A.n_seg; seg += gridDim.x) {
        const uint64_t i0 = seg * kSegElems + threadIdx.x * 16u;
        uint32_t e[16], f[16];
        const int c = load16<DT>(A.src, A.n, i0, e, f);
        uint32_t bits = 0;
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (j < c) bits += s_len[e[j]];
        uint32_t total;
        const uint32_t incl = block_inclusive_scan(bits, s_warp, total);
        uint64_t start = A.seg_off[seg] + (incl - bits);
        // the segment's chunks (its codes start in [seg_off, seg_off + total))
        const uint64_t c_lo = A.seg_off[seg] / cb, c_hi = (A.seg_off[seg] + total - 1) / cb;
        // previous element's start: from its code length
        uint64_t prev = ~uint64_t{0};
        if (i0 > 0 && c > 0) prev = start - s_len[exponent_at<DT>(A.src, i0 - 1)];
        // chunk counts: this thread's codes fall in one or two chunks mostly;
        // one shared-memory add per run of codes in the same chunk
        uint64_t run_c = ~uint64_t{0};
        uint32_t run_n = 0;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            if (j >= c) break;
            const uint32_t len = s_len[e[j]];
            or_code(A.stream, start, s_code[e[j]], len);
            const uint64_t ck = start / cb, pk = prev == ~uint64_t{0} ? ~uint64_t{0} : prev / cb;
            if (A.counts) {
                if (ck != run_c) {
                    if (run_n) atomicAdd(&s_cnt[run_c - c_lo], run_n);
                    run_c = ck;
                    run_n = 0;
                }
                ++run_n;
            }
            for (uint64_t q = pk + 1; q <= ck; ++q) A.gaps[q] = static_cast<uint8_t>(start - q * cb);
            const uint64_t tk = start / A.tile_bits, ptk = prev == ~uint64_t{0} ? ~uint64_t{0} : prev / A.tile_bits;
            for (uint64_t q = ptk + 1; q <= tk; ++q) A.out_off[q] = i0 + j;
            prev = start;
            start += len;
        }
        if (A.counts) {
            if (run_n) atomicAdd(&s_cnt[run_c - c_lo], run_n);
            __syncthreads();
            // a chunk of at most 128 bits holds at most 128 starts: bytes never carry
            for (uint64_t wd = c_lo / 4 + threadIdx.x; wd <= c_hi / 4; wd += kEncThreads) {
                uint32_t packed = 0;
#pragma unroll
                for (uint32_t k = 0; k < 4; ++k) {
                    const uint64_t ch = 4 * wd + k;
                    if (ch >= c_lo && ch <= c_hi) {
                        packed |= s_cnt[ch - c_lo] << (8u * k);
                        s_cnt[ch - c_lo] = 0;  // zero again for the next segment
                    }
                }
                if (4 * wd > c_lo && 4 * wd + 3 < c_hi) A.counts[wd] = packed;
                else if (packed) atomicAdd(A.counts + wd, packed);
            }
            // the next segment's adds come after the block scan's barriers
        }
        // raw fields
        if constexpr (DT == 0) {
            if (c == 16) {
                uint4 v;
                v.x = f[0] | f[1] << 8 | f[2] << 16 | f[3] << 24;
                v.y = f[4] | f[5] << 8 | f[6] << 16 | f[7] << 24;
                v.z = f[8] | f[9] << 8 | f[10] << 16 | f[11] << 24;
                v.w = f[12] | f[13] << 8 | f[14] << 16 | f[15] << 24;
                *reinterpret_cast<uint4 *>(A.plane + i0) = v;
            } else {
                for (int j = 0; j < c; ++j) A.plane[i0 + j] = static_cast<uint8_t>(f[j]);
            }
        } else {
            uint32_t lo = 0, hi = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) lo |= f[j] << (4 * j);
#pragma unroll
            for (int j = 0; j < 8; ++j) hi |= f[8 + j] << (4 * j);
            if (c == 16) {
                *reinterpret_cast<uint2 *>(A.plane + i0 / 2) = make_uint2(lo, hi);
            } else {
                const uint64_t both = (static_cast<uint64_t>(hi) << 32) | lo;
                for (int j = 0; j < (c + 1) / 2; ++j) A.plane[i0 / 2 + j] = static_cast<uint8_t>(both >> (8 * j));
            }
        }
    }
}

// Chunks after the last code start hold no start: their gap reaches the end
// of the stream (one CTA; the last code's length comes from the last element).
template <int DT>
__global__ void tail_gaps_kernel(const void *src, uint64_t n, const uint8_t *lengths, uint8_t *gaps, uint64_t n_chunks,
                                 uint64_t total_bits, uint32_t chunk_bits) {
    const uint64_t last_start = total_bits - lengths[exponent_at<DT>(src, n - 1)];
    for (uint64_t c = last_start / chunk_bits + 1 + threadIdx.x; c < n_chunks; c += blockDim.x)
        gaps[c] = static_cast<uint8_t>(total_bits - c * chunk_bits);
}

__global__ void fill_u64_kernel(uint64_t *p, uint64_t count, uint64_t v) {
    for (uint64_t i = blockIdx.x * static_cast<uint64_t>(blockDim.x) + threadIdx.x; i < count;
         i += static_cast<uint64_t>(gridDim.x) * blockDim.x)
        p[i] = v;
}

__global__ void max_span_kernel(const uint64_t *out_off, uint64_t n_tiles, unsigned long long *result) {
    uint64_t m = 0;
    for (uint64_t t = blockIdx.x * static_cast<uint64_t>(blockDim.x) + threadIdx.x; t < n_tiles;
         t += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
        const uint64_t s = out_off[t + 1] - out_off[t];
        m = s > m ? s : m;
    }
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t t = __shfl_down_sync(0xFFFFFFFFu, m, o);
        m = t > m ? t : m;
    }
    if ((threadIdx.x & 31) == 0 && m) atomicMax(result, static_cast<unsigned long long>(m));
}

int grid_for(uint64_t work_units) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const uint64_t g = static_cast<uint64_t>(sms) * 8;
    return static_cast<int>(work_units < g ? (work_units ? work_units : 1) : g);
}

}  // namespace

// scratch: [0, n_seg) segment sums / offsets, [n_seg] total bits, [n_seg + 1]
// largest span, then 256 code lengths (32 words), 256 codes (128 words) and
// a flag set when an element's exponent has no code
uint64_t encode_scratch_bytes(uint64_t n) { return 8 * (segments_of(n) + 2 + 32 + 128 + 1); }

uint64_t segments_of(uint64_t n) { return (n + kSegElems - 1) / kSegElems; }

bool launch_histogram(int dtype, const void *src, uint64_t n, uint64_t *counts, cudaStream_t s) {
    if (!n) return true;
    const int grid = grid_for(segments_of(n));
    if (dtype == kBF16)
        hist_kernel<0><<<grid, kEncThreads, 0, s>>>(src, n, reinterpret_cast<unsigned long long *>(counts));
    else
        hist_kernel<1><<<grid, kEncThreads, 0, s>>>(src, n, reinterpret_cast<unsigned long long *>(counts));
    return cudaGetLastError() == cudaSuccess;
}

EncodeError encode_device_bits(const EncodeJob &J, uint64_t *scratch, cudaStream_t s, uint64_t *total_bits) {
    const uint64_t n_seg = segments_of(J.n);
    *total_bits = 0;
    if (!J.n) return EncodeError::kOk;
    uint8_t *dev_len = reinterpret_cast<uint8_t *>(scratch + n_seg + 2);  // 256 bytes after the sums
    unsigned long long *uncovered = reinterpret_cast<unsigned long long *>(scratch + n_seg + 2 + 32 + 128);
    if (cudaMemcpyAsync(dev_len, J.cb->lengths, 256, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemsetAsync(uncovered, 0, 8, s) != cudaSuccess)
        return EncodeError::kCuda;
    const int grid = grid_for(n_seg);
    if (J.cb->dtype == kBF16)
        seg_bits_kernel<0><<<grid, kEncThreads, 0, s>>>(J.src, J.n, dev_len, n_seg, scratch, uncovered);
    else
        seg_bits_kernel<1><<<grid, kEncThreads, 0, s>>>(J.src, J.n, dev_len, n_seg, scratch, uncovered);
    seg_scan_kernel<<<1, 1024, 0, s>>>(scratch, n_seg, scratch + n_seg);
    uint64_t tb = 0, miss = 0;
    if (cudaMemcpyAsync(&tb, scratch + n_seg, 8, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaMemcpyAsync(&miss, uncovered, 8, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return EncodeError::kCuda;
    if (cudaGetLastError() != cudaSuccess) return EncodeError::kCuda;
    if (miss) return EncodeError::kUncovered;
    *total_bits = tb;
    return EncodeError::kOk;
}

EncodeError encode_device_pack(const EncodeJob &J, uint64_t *scratch, uint64_t total_bits, const ImageLayout &L,
                               uint8_t *image, cudaStream_t s, uint64_t *max_span) {
    const uint64_t n_seg = segments_of(J.n);
    const uint64_t cbits = static_cast<uint64_t>(J.chunk_bits);
    const uint64_t tbits = cbits * static_cast<uint64_t>(J.tile_threads);
    const uint64_t n_chunks = (total_bits + cbits - 1) / cbits;
    const uint64_t n_tiles = (n_chunks + J.tile_threads - 1) / J.tile_threads;
    *max_span = 0;
    // header, decode tables, zeroed stream / gaps, out_off = n
    std::vector<uint8_t> head(L.gaps);
    Blob meta_only;
    meta_only.dtype = J.cb->dtype;
    meta_only.chunk_bits = J.chunk_bits;
    meta_only.tile_threads = J.tile_threads;
    meta_only.n = J.n;
    meta_only.total_bits = total_bits;
    meta_only.n_tiles = n_tiles;
    meta_only.cb = J.cb;
    meta_only.chunk_counts = J.chunk_counts && counts_fit(J.chunk_bits);
    write_image_head(meta_only, L, head.data());
    if (cudaMemcpyAsync(image, head.data(), head.size(), cudaMemcpyHostToDevice, s) != cudaSuccess)
        return EncodeError::kCuda;
    if (cudaMemsetAsync(image + L.gaps, 0, L.total - L.gaps, s) != cudaSuccess) return EncodeError::kCuda;
    uint64_t *out_off = reinterpret_cast<uint64_t *>(image + L.out_off);
    fill_u64_kernel<<<grid_for((n_tiles + 1 + 255) / 256), 256, 0, s>>>(out_off, n_tiles + 1, J.n);
    uint8_t *dev_len = reinterpret_cast<uint8_t *>(scratch + n_seg + 2);
    uint32_t *dev_codes = reinterpret_cast<uint32_t *>(scratch + n_seg + 2 + 32);  // 1 KB after the lengths
    if (cudaMemcpyAsync(dev_codes, J.cb->codes, 1024, cudaMemcpyHostToDevice, s) != cudaSuccess)
        return EncodeError::kCuda;
    PackArgs A;
    A.src = J.src;
    A.n = J.n;
    A.lengths = dev_len;
    A.codes = dev_codes;
    A.seg_off = scratch;
    A.n_seg = n_seg;
    A.stream = reinterpret_cast<uint32_t *>(image + L.stream);
    A.plane = image + L.plane;
    A.gaps = image + L.gaps;
    A.counts = meta_only.chunk_counts ? reinterpret_cast<uint32_t *>(image + L.counts) : nullptr;
    A.out_off = out_off;
    A.chunk_bits = static_cast<uint32_t>(J.chunk_bits);
    A.tile_bits = tbits;
    if (J.cb->dtype == kBF16)
        pack_kernel<0><<<grid_for(n_seg), kEncThreads, 0, s>>>(A);
    else
        pack_kernel<1><<<grid_for(n_seg), kEncThreads, 0, s>>>(A);
    // chunks after the last code start
    if (J.cb->dtype == kBF16)
        tail_gaps_kernel<0><<<1, 128, 0, s>>>(J.src, J.n, dev_len, A.gaps, n_chunks, total_bits, A.chunk_bits);
    else
        tail_gaps_kernel<1><<<1, 128, 0, s>>>(J.src, J.n, dev_len, A.gaps, n_chunks, total_bits, A.chunk_bits);
    unsigned long long *dev_max = reinterpret_cast<unsigned long long *>(scratch + n_seg + 1);
    if (cudaMemsetAsync(dev_max, 0, 8, s) != cudaSuccess) return EncodeError::kCuda;
    max_span_kernel<<<grid_for((n_tiles + 255) / 256), 256, 0, s>>>(out_off, n_tiles, dev_max);
    uint64_t ms = 0;
    if (cudaMemcpyAsync(&ms, dev_max, 8, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return EncodeError::kCuda;
    if (cudaGetLastError() != cudaSuccess) return EncodeError::kCuda;
    // the header was written before the span was known
    if (cudaMemcpyAsync(image + offsetof(ImageHeader, max_span), &ms, 8, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return EncodeError::kCuda;
    *max_span = ms;
    return EncodeError::kOk;
}

// ---------------------------------------------------------------- encoding without allocation
//
// For callers that cannot allocate device memory when they encode (see
// df11_encode_device_noalloc in df11.h): the encoder's scratch lives in one
// static device array per GPU instead of a caller buffer.

namespace {

constexpr uint64_t kNoallocScratchWords = 65536;  // 512 KB on every GPU that loads the library
__device__ __align__(256) uint64_t g_noalloc_scratch[kNoallocScratchWords];

std::mutex g_noalloc_mu;
constexpr int kNoallocDevices = 64;
uint64_t *g_noalloc_addr[kNoallocDevices] = {};

}  // namespace

uint64_t noalloc_max_elems() { return (kNoallocScratchWords - (2 + 32 + 128 + 1)) * kSegElems; }

EncodeError encode_device_noalloc(const EncodeJob &J, uint8_t *image, uint64_t image_cap, cudaStream_t s,
                                  NoallocResult *r) {
    // device address of the static scratch on the current device, looked up
    // once per device (host code cannot use the symbol itself)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoallocDevices) return EncodeError::kCuda;
    uint64_t *scratch = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_noalloc_mu);
        if (!g_noalloc_addr[dev]) {
            void *p = nullptr;
            if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return EncodeError::kCuda;
            g_noalloc_addr[dev] = static_cast<uint64_t *>(p);
        }
        scratch = g_noalloc_addr[dev];
    }
    // pass 1: every slot it reads is written first (sums, total, flag)
    uint64_t total = 0;
    const EncodeError err = encode_device_bits(J, scratch, s, &total);
    if (err != EncodeError::kOk) return err;
    Blob meta;  // metadata only: its sections stay empty
    meta.dtype = J.cb->dtype;
    meta.chunk_bits = J.chunk_bits;
    meta.tile_threads = J.tile_threads;
    meta.n = J.n;
    meta.total_bits = total;
    const uint64_t cbits = static_cast<uint64_t>(J.chunk_bits);
    const uint64_t n_chunks = (total + cbits - 1) / cbits;
    meta.n_tiles = (n_chunks + J.tile_threads - 1) / J.tile_threads;
    meta.cb = J.cb;
    meta.chunk_counts = J.chunk_counts && counts_fit(J.chunk_bits);
    const ImageLayout L = image_layout(meta);
    r->image_bytes = L.total;
    r->total_bits = total;
    r->n_tiles = meta.n_tiles;
    r->max_span = 0;
    if (image_cap < L.total) return EncodeError::kTooSmall;
    // header and decode tables, copied from the codebook without a staging buffer
    ImageHeader h{};
    std::memcpy(h.magic, "DF11IMG1", 8);
    h.dtype = static_cast<uint32_t>(meta.dtype);
    h.chunk_bits = static_cast<uint32_t>(meta.chunk_bits);
    h.tile_threads = static_cast<uint32_t>(meta.tile_threads);
    h.n_luts = static_cast<uint32_t>(J.cb->n_luts());
    h.fsm_rows = static_cast<uint32_t>(J.cb->fsm_rows);
    h.flags = meta.chunk_counts ? kImageFlagCounts : 0u;
    h.n_elems = meta.n;
    h.total_bits = total;
    h.n_tiles = meta.n_tiles;
    h.layout = L;
    if (cudaMemsetAsync(image, 0, L.total, s) != cudaSuccess ||
        cudaMemcpyAsync(image, &h, sizeof h, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(image + L.meta, J.cb->meta.data(), kMultiEntries * 4, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(image + L.syms, J.cb->syms.data(), kMultiEntries * 4, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(image + L.lut, J.cb->lut.data(), J.cb->lut.size() * 2, cudaMemcpyHostToDevice, s) !=
            cudaSuccess ||
        cudaMemcpyAsync(image + L.fsm, J.cb->fsm.data(), J.cb->fsm.size() * 4, cudaMemcpyHostToDevice, s) !=
            cudaSuccess)
        return EncodeError::kCuda;
    if (!J.n) return cudaStreamSynchronize(s) == cudaSuccess ? EncodeError::kOk : EncodeError::kCuda;
    // pass 2, as in encode_device_pack
    const uint64_t n_seg = segments_of(J.n);
    uint64_t *out_off = reinterpret_cast<uint64_t *>(image + L.out_off);
    fill_u64_kernel<<<grid_for((meta.n_tiles + 1 + 255) / 256), 256, 0, s>>>(out_off, meta.n_tiles + 1, J.n);
    uint8_t *dev_len = reinterpret_cast<uint8_t *>(scratch + n_seg + 2);
    uint32_t *dev_codes = reinterpret_cast<uint32_t *>(scratch + n_seg + 2 + 32);
    if (cudaMemcpyAsync(dev_codes, J.cb->codes, 1024, cudaMemcpyHostToDevice, s) != cudaSuccess)
        return EncodeError::kCuda;
    PackArgs A;
    A.src = J.src;
    A.n = J.n;
    A.lengths = dev_len;
    A.codes = dev_codes;
    A.seg_off = scratch;
    A.n_seg = n_seg;
    A.stream = reinterpret_cast<uint32_t *>(image + L.stream);
    A.plane = image + L.plane;
    A.gaps = image + L.gaps;
    A.counts = meta.chunk_counts ? reinterpret_cast<uint32_t *>(image + L.counts) : nullptr;
    A.out_off = out_off;
    A.chunk_bits = static_cast<uint32_t>(J.chunk_bits);
    A.tile_bits = cbits * static_cast<uint64_t>(J.tile_threads);
    if (J.cb->dtype == kBF16) {
        pack_kernel<0><<<grid_for(n_seg), kEncThreads, 0, s>>>(A);
        tail_gaps_kernel<0><<<1, 128, 0, s>>>(J.src, J.n, dev_len, A.gaps, n_chunks, total, A.chunk_bits);
    } else {
        pack_kernel<1><<<grid_for(n_seg), kEncThreads, 0, s>>>(A);
        tail_gaps_kernel<1><<<1, 128, 0, s>>>(J.src, J.n, dev_len, A.gaps, n_chunks, total, A.chunk_bits);
    }
    // the span accumulator keeps the previous call's value: clear it
    unsigned long long *dev_max = reinterpret_cast<unsigned long long *>(scratch + n_seg + 1);
    if (cudaMemsetAsync(dev_max, 0, 8, s) != cudaSuccess) return EncodeError::kCuda;
    max_span_kernel<<<grid_for((meta.n_tiles + 255) / 256), 256, 0, s>>>(out_off, meta.n_tiles, dev_max);
    uint64_t ms = 0;
    if (cudaMemcpyAsync(&ms, dev_max, 8, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return EncodeError::kCuda;
    if (cudaGetLastError() != cudaSuccess) return EncodeError::kCuda;
    if (cudaMemcpyAsync(image + offsetof(ImageHeader, max_span), &ms, 8, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return EncodeError::kCuda;
    r->max_span = ms;
    return EncodeError::kOk;
}

}  // namespace df11
