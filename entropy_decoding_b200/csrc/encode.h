// encode.h -- host entry points of the GPU encoder (encode.cu).
#pragma once

#include <cuda_runtime_api.h>

#include <memory>
#include <string>

#include "codec.h"

namespace df11 {

struct EncodeJob {
    std::shared_ptr<const Codebook> cb;
    const void *src = nullptr;  // device
    uint64_t n = 0;
    int chunk_bits = 128;
    int tile_threads = 32;
    bool chunk_counts = true;  // write the chunk-counts section (chunk_bits <= 128 only)
};

uint64_t segments_of(uint64_t n);
// Scratch the encoder needs: per-segment bit sums, two scalars, the code
// lengths and codes.
uint64_t encode_scratch_bytes(uint64_t n);

bool launch_histogram(int dtype, const void *src, uint64_t n, uint64_t *counts, cudaStream_t s);

// Outcome of a device encode step (no strings: the allocation-free path
// touches no host heap either).
enum class EncodeError { kOk, kUncovered, kTooSmall, kCuda };

// Pass 1: bits per segment, their exclusive scan (left in scratch) and the
// total, read back to the host (synchronises s).
EncodeError encode_device_bits(const EncodeJob &J, uint64_t *scratch, cudaStream_t s, uint64_t *total_bits);

// Pass 2: the device image at `image` (layout L), from the scan in scratch;
// reads back the largest tile span (synchronises s).
EncodeError encode_device_pack(const EncodeJob &J, uint64_t *scratch, uint64_t total_bits, const ImageLayout &L,
                               uint8_t *image, cudaStream_t s, uint64_t *max_span);

// Encoding without any allocation: the scratch is a static device array of
// 512 KB per GPU, so n must not exceed noalloc_max_elems().  Calls that
// overlap on the GPU share that array and race.
struct NoallocResult {
    uint64_t image_bytes, total_bits, n_tiles, max_span;
};
uint64_t noalloc_max_elems();
EncodeError encode_device_noalloc(const EncodeJob &J, uint8_t *image, uint64_t image_cap, cudaStream_t s,
                                  NoallocResult *r);

}  // namespace df11
