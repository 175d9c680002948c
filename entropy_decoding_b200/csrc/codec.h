// codec.h -- host side of libdf11: code construction, decode-table building,
// the multi-threaded encoder, the container and the device image.
#pragma once

#include <cstdint>
#include <memory>
#include <string>
#include <thread>
#include <vector>

#include "df11_internal.h"

namespace df11 {

enum Dtype : int { kBF16 = 0, kE4M3 = 1 };

inline int nsym_of(int dtype) { return dtype == kBF16 ? 256 : 16; }

struct Codebook {
    int dtype = kBF16;
    int nsym = 256;
    uint8_t lengths[256] = {};
    uint32_t codes[256] = {};
    int max_len_used = 0;
    int min_len_used = 0;
    std::vector<uint32_t> meta;  // kMultiEntries
    std::vector<uint32_t> syms;  // kMultiEntries
    std::vector<uint16_t> lut;   // n_luts * kLutEntries
    std::vector<uint32_t> fsm;   // fsm_rows * kLutEntries * 2: {ctl, syms} per entry
    int fsm_rows = 0;            // including the dead row (the last one)
    int n_luts() const { return static_cast<int>(lut.size() / kLutEntries); }
};

struct Blob {
    int dtype = kBF16;
    int chunk_bits = 128;
    int tile_threads = 256;
    uint64_t n = 0;
    uint64_t total_bits = 0;
    uint64_t n_tiles = 0;
    uint64_t max_span = 0;
    std::shared_ptr<const Codebook> cb;
    std::vector<uint8_t> stream;    // ceil(total_bits / 8)
    std::vector<uint8_t> plane;     // n (BF16) or ceil(n / 2) (E4M3)
    std::vector<uint8_t> gaps;      // n_tiles * tile_threads
    bool chunk_counts = false;      // the counts section is part of the container
    std::vector<uint8_t> counts;    // n_tiles * tile_threads when chunk_counts (codes starting per chunk)
    std::vector<uint64_t> out_off;  // n_tiles + 1
    bool device_only = false;  // encoded on the GPU: host sections empty until fetched
    const uint8_t *dev_image = nullptr;
    uint64_t dev_cap = 0;
    std::vector<uint8_t> host_image;  // staging copy kept alive for df11_blob_upload
};

// Runs fn(begin, end) over [0, n_items) split evenly across n_threads host
// threads (0 = all cores).
template <class F>
void parallel_for(uint64_t n_items, int n_threads, F fn) {
    if (n_items == 0) return;
    unsigned hw = std::thread::hardware_concurrency();
    int t = n_threads > 0 ? n_threads : static_cast<int>(hw ? hw : 1);
    if (static_cast<uint64_t>(t) > n_items) t = static_cast<int>(n_items);
    if (t <= 1) {
        fn(uint64_t{0}, n_items);
        return;
    }
    std::vector<std::thread> pool;
    pool.reserve(t);
    for (int k = 0; k < t; ++k) {
        uint64_t b = n_items * k / t, e = n_items * (k + 1) / t;
        pool.emplace_back([=, &fn] { fn(b, e); });
    }
    for (auto &th : pool) th.join();
}

// Code construction.  Returns false when the arguments admit no code.
bool code_lengths(const uint64_t *counts, int nsym, int max_len, uint8_t *lengths);
bool canonical_codes(const uint8_t *lengths, int nsym, uint32_t *codes);  // false: not a prefix code
std::shared_ptr<Codebook> make_codebook(int dtype, const uint8_t *lengths);  // nullptr if invalid

// Histogram of the exponent field, added into counts[256].
void histogram(int dtype, const void *src, uint64_t n, uint64_t *counts, int n_threads);

// Encoder: returns an empty string on success, else the reason.  chunk_counts
// asks for the chunk-counts section (stored only when chunk_bits <= 128).
std::string encode(std::shared_ptr<const Codebook> cb, const void *src, uint64_t n, int chunk_bits,
                   int tile_threads, int n_threads, bool chunk_counts, Blob *out);

// Whether a layout stores chunk counts when they are asked for.
inline bool counts_fit(int chunk_bits) { return chunk_bits <= kCountsMaxChunkBits; }

uint64_t plane_bytes(int dtype, uint64_t n);
uint64_t serialized_bytes(const Blob &b);
void serialize(const Blob &b, uint8_t *dst);
std::string deserialize(const uint8_t *src, uint64_t len, Blob *out);

ImageLayout image_layout(const Blob &b);
void write_image(const Blob &b, uint8_t *dst);
// The image's header and decode tables: bytes [0, L.gaps).
void write_image_head(const Blob &b, const ImageLayout &L, uint8_t *dst);
// Host sections of a blob back from its device image (inverse of write_image).
void read_image_sections(Blob &b, const uint8_t *img);

bool valid_layout(int chunk_bits, int tile_threads);

}  // namespace df11
