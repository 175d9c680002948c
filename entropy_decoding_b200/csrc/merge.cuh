// merge.cuh -- the merge of decoded exponents with the raw sign+mantissa
// plane into the original weights, shared by the Huffman decode kernels
// (walk.cuh, decode.cu, gemm.cu) and the rANS decode kernel.
//
// Field layout: "Compressing LLMs without Compromise" summary page, "Where
// the redundancy lives" (BF16 = sign, 8 exponent bits, 7 mantissa bits); the
// plane keeps sign << 7 | mantissa per BF16 weight and sign << 3 | mantissa
// per E4M3 nibble (element 2i in the low nibble).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace df11 {
namespace {

// 4 plane bytes + 4 exponents -> 4 BF16 words (two 32-bit outputs).
__device__ __forceinline__ void merge_bf16x4(uint32_t P, uint32_t X, uint32_t &o0, uint32_t &o1) {
    const uint32_t hi = (P & 0x80808080u) | ((X >> 1) & 0x7F7F7F7Fu);  // sign | exponent[7:1]
    const uint32_t lo = ((X << 7) & 0x80808080u) | (P & 0x7F7F7F7Fu);  // exponent[0] | mantissa
    o0 = __byte_perm(lo, hi, 0x5140);
    o1 = __byte_perm(lo, hi, 0x7362);
}

// 4 plane bytes (8 nibbles) + 8 exponents -> 8 E4M3 bytes.
__device__ __forceinline__ void merge_e4m3x8(uint32_t P, uint32_t X0, uint32_t X1, uint32_t &o0, uint32_t &o1) {
    const uint32_t nl = P & 0x0F0F0F0Fu;         // elements 0, 2, 4, 6
    const uint32_t nh = (P >> 4) & 0x0F0F0F0Fu;  // elements 1, 3, 5, 7
    const uint32_t n0 = __byte_perm(nl, nh, 0x5140);
    const uint32_t n1 = __byte_perm(nl, nh, 0x7362);
    o0 = ((n0 & 0x08080808u) << 4) | ((X0 << 3) & 0x78787878u) | (n0 & 0x07070707u);
    o1 = ((n1 & 0x08080808u) << 4) | ((X1 << 3) & 0x78787878u) | (n1 & 0x07070707u);
}

}  // namespace
}  // namespace df11
