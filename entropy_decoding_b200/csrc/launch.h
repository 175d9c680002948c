// launch.h -- host entry points of the decode kernels (decode.cu).
#pragma once

#include <cuda_runtime_api.h>

#include "codec.h"

namespace df11 {

enum class LaunchStatus { kOk, kInvalid, kUnsupported, kCuda };

struct DecodeOptions {
    int chunks_per_thread = 0;  // 0 = kDefaultChunksPerThread
    int ctas_per_sm = 0;        // 0 = as many as fit
    int warps_per_cta = 0;      // warp-tile layouts: 0 = kDefaultWarpsPerCta (window) / most that fit (byte step)
    int walker = 0;             // DF11_WALKER_*: 0 = auto
    int max_ctas = 0;           // grid cap, 0 = none
    int overlap = 0;            // 1: programmatic dependent launch (no dependency on earlier stream work)
    int diag_expire_waits = 0;  // diagnostics: no copies, every wait runs out after 10 ms
    int count_walk = 0;         // 1: byte-step walker counts with a walk even when chunk counts are stored
    int diag_check_bounds = 0;  // diagnostics (bounds-checked build only): the exponent buffer's checked bound is 0
};

constexpr int kDefaultChunksPerThread = 1;
constexpr int kDefaultWarpsPerCta = 16;

struct LaunchShape {
    int grid = 0;
    int block = 0;
    int smem = 0;
    int walker = 0;         // DF11_WALKER_WINDOW or DF11_WALKER_BYTE_STEP
    int stored_counts = 0;  // 1: output positions from the stored chunk counts
};

bool kernel_available(int dtype, int chunk_bits, int tile_threads);

LaunchStatus decode_launch_shape(const Blob *const *blobs, int n, const DecodeOptions &opt, LaunchShape *out);

// One launch decoding every blob into dst[i] on stream s.
LaunchStatus launch_decode(const Blob *const *blobs, void *const *dst, int n, int *err, const DecodeOptions &opt,
                           cudaStream_t s);

}  // namespace df11
