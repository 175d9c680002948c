// rans.h -- the rANS variant of the exponent coder: frequency quantization,
// the multi-threaded encoder and the group's device image (host side), and the
// decode launch (rans_decode.cu).
//
// The coder ("Approaching Shannon Bound with Lossless LLM Weight Compression",
// Abstract: ANS decoding by tiles, within 0.01-0.1 bits of the Shannon limit)
// codes the same exponent symbols as the Huffman container and keeps the same
// raw sign+mantissa plane.  State x in [2^16, 2^32), symbol s with quantized
// frequency f_s and cumulative c_s over M = 2^12:
//     encode  x' = floor(x / f_s) * M + (x mod f_s) + c_s   (after moving the
//             low 16 bits out while x >= f_s << 20)
//     decode  slot = x mod M, s = sym(slot),
//             x = f_s * floor(x / M) + slot - c_s, then x = x << 16 | word
//             while x < 2^16.
// A tile of tile_symbols symbols is coded by 32 interleaved coders (lane j:
// symbols j, j + 32, ...); decoding takes steps k = 0, 1, ... and in a step
// lanes 0..31 in order, each reading at most one word after its symbol.  The
// encoder runs that order backwards from states 2^16 and reverses the words.
// Each tile's words start at a multiple of 8 words (16 bytes).
#pragma once

#include <cstdint>
#include <memory>
#include <string>
#include <vector>

#include <cuda_runtime_api.h>

namespace df11 {

constexpr int kRansBits = 12;
constexpr uint32_t kRansM = 1u << kRansBits;
constexpr uint32_t kRansL = 1u << 16;
constexpr int kRansLanes = 32;
constexpr uint32_t kRansChunkWords = 256;  // words the decoder moves into its ring at a time
constexpr uint64_t kRansWordsTail = 1024;  // zero words after a tensor's words: chunks read ahead
constexpr uint64_t kRansPlaneTail = 512;   // readable bytes after a tensor's plane: whole groups read

struct RansTensor {
    uint64_t n = 0;
    uint64_t n_tiles = 0;
    std::vector<uint16_t> words;       // tile_words.back() words
    std::vector<uint32_t> states;      // n_tiles * 32
    std::vector<uint64_t> tile_words;  // n_tiles + 1, multiples of 8
    std::vector<uint8_t> plane;        // as the Huffman container's
};

struct RansGroup {
    int dtype = 0;
    int nsym = 256;
    uint32_t tile_symbols = 16384;
    uint32_t freqs[256] = {};
    uint32_t table[kRansM] = {};  // decode entry per slot: symbol | (f - 1) << 8 | (slot - c) << 20
    std::vector<RansTensor> tensors;
    const uint8_t *dev_image = nullptr;
    uint64_t dev_cap = 0;
    std::vector<uint8_t> host_image;  // staging copy kept alive for the upload
};

// Offsets of one tensor's sections in the group's device image (each 256-byte
// aligned); the decode table comes first, at offset 0.
struct RansTensorLayout {
    uint64_t states, tile_words, words, plane, end;
};

bool rans_freqs(const uint64_t *counts, int nsym, uint32_t *freqs);
void rans_build_table(const uint32_t *freqs, int nsym, uint32_t *table);
std::string rans_encode_group(int dtype, const void *const *src, const uint64_t *n, int n_tensors,
                              uint32_t tile_symbols, int n_threads, RansGroup *out);
std::vector<RansTensorLayout> rans_layout(const RansGroup &g, uint64_t *total);
void rans_write_image(const RansGroup &g, uint8_t *dst);

// The group's container (the offline form) and its reader, which checks the
// header, the frequencies, every size and tile offset and the states' range.
uint64_t rans_serialized_bytes(const RansGroup &g);
void rans_serialize(const RansGroup &g, uint8_t *dst);
std::string rans_deserialize(const uint8_t *src, uint64_t len, RansGroup *out);

enum class RansLaunch { kOk, kInvalid, kCuda };
// One launch decoding every tensor of the bound group into dst[i].
RansLaunch rans_launch_decode(const RansGroup &g, void *const *dst, int *err, cudaStream_t s, int *grid_out,
                              int *block_out, int *smem_out);

}  // namespace df11
