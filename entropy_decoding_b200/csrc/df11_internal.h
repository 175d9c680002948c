// df11_internal.h -- layout constants and structures shared by the host codec
// (codec.cpp), the C-ABI (capi.cpp) and the decode kernels (decode.cu).
//
// Decode tables (the "compact, hierarchical lookup tables that fit within GPU
// SRAM" of the DFloat11 Abstract, item (i)):
//   * hierarchical LUT: levels of 256 u16 entries indexed by the next 8 stream
//     bits.  Table 0 is the root.  Entry forms:
//       leaf     bit15 = 0: bits 0..7 symbol, bits 8..13 full code length
//       pointer  bit15 = 1: bits 0..14 index of the next-level table
//       invalid  bit14 = 1 (leaf form, length 1): no codeword has this prefix
//     A 32-bit code needs at most 4 levels.
//   * multi-symbol table (an addition for sm_100a's instruction budget): 4096
//     entries indexed by the next 12 stream bits, for the longest run of up
//     to 4 whole codes inside the 12-bit window.  meta[v] (u32) = consumed
//     bits (bits 0..3) | symbols decoded (bits 11..13) | start mask (bit 20+j
//     set when one of those codes starts at window offset j).  Bits 0..10
//     and 11..19 line up with a walker's accumulator (bit position | count
//     << 11), so one add advances both.  meta[v] = kMetaLong (consumed 1024,
//     no symbol) when the first code is longer than 12 bits.  syms[v] holds
//     the symbols, first in the low byte, unused bytes zero.
//   * byte-step transition tables ("fsm"): one row of 256 entries per node of
//     the code tree that a byte boundary can fall on (the root, then the
//     other internal nodes in decreasing order of the probability mass below
//     them, up to kFsmMaxRows - 1 rows), plus a dead row.  Entry (row v,
//     byte b) is what walking the 8 bits of b from node v produces: ctl (u32)
//     = end mask (bit i set when a code ends at bit i of b, bit 0 = the first
//     bit) | next row << kFsmRowShift | codes ended << kFsmCountShift, and
//     syms (u32) = the first up to 4 symbols ended, first in the low byte.
//     A byte that ends more than 4 codes, leads to a node without a row or
//     meets a prefix that is no codeword leads to the dead row, whose
//     entries lead back to it and end no code.  The walk of a byte is thus
//     one lookup that does not depend on where the codes start: the
//     hierarchical tables generalised to every node at a byte boundary.
//     Row v occupies bytes [v * kFsmRowBytes, (v + 1) * kFsmRowBytes), entry
//     b the 8 bytes {ctl, syms} at b * 8 within it.
//   * chunk counts (optional, chunk_bits <= 128): one byte per chunk, the
//     number of codes that start in its chunk_bits stream bits.  With them a
//     decoding thread's output position is a warp scan of stored bytes, and
//     the count walk of the first phase (the two-phase kernel of the DFloat11
//     Abstract, item (ii)) is not needed.  A chunk of at most 128 bits holds
//     at most 128 code starts, so the byte never overflows.
//   * in the device image the stream is stored as 32-bit words whose bit 31
//     is the earliest stream bit (each 4-byte group of the MSB-first byte
//     stream reversed), so a word load needs no byte swap.
#pragma once

#include <cstdint>

namespace df11 {

constexpr int kMultiBits = 12;
constexpr int kMultiEntries = 1 << kMultiBits;
constexpr int kMultiMaxSyms = 4;
constexpr uint32_t kMetaLong = 0x0400;
constexpr int kMetaCountShift = 11;
constexpr int kMetaMaskShift = 20;

constexpr int kLutEntries = 256;
constexpr uint16_t kLutPointer = 0x8000;
constexpr uint16_t kLutInvalid = 0x4000 | (1u << 8);
constexpr int kMaxLutTables = 0x7FFF;
constexpr int kSmemLutTables = 16;  // hierarchical tables staged in shared memory; the rest stay in global

constexpr int kFsmMaxRows = 64;  // including the dead row
constexpr int kFsmRowBytes = kLutEntries * 8;
constexpr int kFsmRowShift = 11;  // row index << 11 = the row's byte offset
constexpr uint32_t kFsmRowMask = static_cast<uint32_t>(kFsmMaxRows - 1) << kFsmRowShift;
constexpr int kFsmCountShift = 29;

constexpr int kMaxCodeLen = 32;
constexpr int kMaxTensorsPerLaunch = 64;
constexpr uint64_t kImageAlign = 256;
constexpr uint64_t kStreamTail = 16;  // zero bytes after the last tile: look-ahead of the last thread
constexpr uint64_t kPlaneTail = 32;
constexpr uint64_t kGapsTail = 16;  // readable bytes after the last tile's gaps: the next chunk's gap
constexpr int kCountsMaxChunkBits = 128;  // chunk counts are stored for chunk_bits up to this
constexpr uint32_t kImageFlagCounts = 1;  // ImageHeader::flags: the chunk-counts section is present

inline uint64_t align_up(uint64_t x, uint64_t a) { return (x + a - 1) / a * a; }

// Offsets of the sections inside one blob's device image.
// counts == out_off when the image has no chunk counts.
struct ImageLayout {
    uint64_t meta, syms, lut, fsm, gaps, counts, out_off, stream, plane, total;
};

// Header at offset 0 of every device image (kept for inspection; the kernel
// takes everything it needs from its launch parameters).
struct ImageHeader {
    char magic[8];  // "DF11IMG1"
    uint32_t dtype, chunk_bits, tile_threads, n_luts, fsm_rows, flags;  // flags: kImageFlagCounts
    uint64_t n_elems, total_bits, n_tiles, max_span;
    ImageLayout layout;
};

// One tensor of a batched launch.  Tiles of all tensors are numbered
// consecutively: tensor i owns global tiles [tile_begin, tile_begin + n_tiles).
struct TensorDesc {
    const uint8_t *stream;
    const uint8_t *plane;
    const uint8_t *gaps;
    const uint8_t *counts;  // nullptr: the image has no chunk counts
    const uint64_t *out_off;
    void *dst;
    uint64_t n;
    uint64_t total_bits;
    uint32_t n_tiles;
    uint32_t tile_begin;
};

struct DecodeParams {
    const uint32_t *meta;
    const uint32_t *syms;
    const uint16_t *lut;
    const uint32_t *fsm;  // fsm_rows * kFsmRowBytes bytes
    int32_t fsm_rows;
    int32_t expire;    // diagnostics: issue no copies, so every wait runs out after wait_ns
    uint64_t wait_ns;  // limit of every mbarrier wait
    int *err;
    int32_t n_luts;
    int32_t n_tensors;
    uint32_t total_tiles;
    uint32_t max_span;  // largest per-tile span over the launch's tensors
    int32_t diag_bounds;  // bounds-checked build: check exponent-buffer accesses against 0 bytes
    int32_t pad;
    TensorDesc t[kMaxTensorsPerLaunch];
};

}  // namespace df11
