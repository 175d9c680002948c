// launch.h -- host entry points of the decode kernels (decode.cu).
#pragma once

#include <cuda_runtime_api.h>

#include "codec.h"

namespace df11 {

enum class LaunchStatus { kOk, kInvalid, kUnsupported, kCuda };

struct LaunchShape {
    int grid = 0;
    int block = 0;
    int smem = 0;
};

bool kernel_available(int dtype, int chunk_bits, int tile_threads);

LaunchStatus decode_launch_shape(const Blob *const *blobs, int n, LaunchShape *out);

// One launch decoding every blob into dst[i] on stream s.
LaunchStatus launch_decode(const Blob *const *blobs, void *const *dst, int n, int *err, cudaStream_t s);

}  // namespace df11
