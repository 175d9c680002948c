// gemm.h -- host entry of the decode fused into the GEMM that consumes the
// weights (gemm.cu): y += x W with W held Huffman-coded in HBM and decoded
// tile by tile straight into the tensor cores' shared-memory operands.
#pragma once

#include <cuda_runtime_api.h>

#include "codec.h"
#include "launch.h"

namespace df11 {

// Operand tile of the weights: 128 output rows x 64 reduction columns (one
// 128-byte swizzle row of BF16 per output row, four MMAs' K), 8192 weights.
constexpr int kGemmTileN = 128;
constexpr int kGemmTileK = 64;
constexpr int kGemmMaxMats = 8;    // matrices per launch (sharing one code)
constexpr int kGemmMaxBatch = 64;  // rows of x (the MMA's N, padded to 16)
constexpr int kGemmMaxCtas = 256;

struct GemmJob {
    const Blob *w;  // the K x N matrix in operand-tile order (gemm_tile_weights), bound to its image
    uint64_t k, n;
    const void *x;  // device, M x K BF16 row-major
    float *y;       // device, M x N FP32 row-major; the product is added
};

struct GemmShape {
    int grid = 0, block = 0, smem = 0, a_slots = 0, b_slots = 0;
};

// The operand-tile order of a K x N row-major matrix w (element (k, n) at
// k * N + n): tile t = nb * (K / 64) + kb holds rows n = 128 nb .. 128 nb +
// 127 and columns k = 64 kb .. 64 kb + 63, element (r, c) at position
// 8192 t + 64 r + c.  K % 64 == 0 and N % 128 == 0.
void gemm_tile_weights(const uint16_t *w, uint64_t k, uint64_t n, uint16_t *tiled, int n_threads);

LaunchStatus gemm_launch_shape(const GemmJob *jobs, int n, int m, GemmShape *out);
LaunchStatus launch_decode_gemm(const GemmJob *jobs, int n, int m, int *err, cudaStream_t s);

}  // namespace df11
