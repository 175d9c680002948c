// rans.cpp -- host side of the rANS exponent coder (format in rans.h).
#include "rans.h"

#include <algorithm>
#include <cstring>

#include "codec.h"

namespace df11 {

// Quantized frequencies summing to 2^12: each present symbol gets
// max(1, floor(count * 2^12 / total)); a shortfall is handed out one unit at
// a time over the present symbols by decreasing count (smaller symbol first
// on ties), round after round; an excess is taken back the same way from
// symbols above 1.
bool rans_freqs(const uint64_t *counts, int nsym, uint32_t *freqs) {
    uint64_t total = 0;
    std::vector<int> order;
    for (int s = 0; s < nsym; ++s) {
        freqs[s] = 0;
        total += counts[s];
        if (counts[s]) order.push_back(s);
    }
    if (order.empty()) return true;
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return counts[a] > counts[b]; });
    int64_t sum = 0;
    for (int s : order) {
        const unsigned __int128 q = static_cast<unsigned __int128>(counts[s]) * kRansM / total;
        freqs[s] = std::max<uint32_t>(1u, static_cast<uint32_t>(q));
        sum += freqs[s];
    }
    int64_t d = static_cast<int64_t>(kRansM) - sum;
    const size_t np = order.size();
    for (size_t i = 0; d > 0; ++i, --d) freqs[order[i % np]]++;
    for (size_t i = 0; d < 0; ++i) {
        const int s = order[i % np];
        if (freqs[s] > 1) {
            freqs[s]--;
            ++d;
        }
    }
    return true;
}

void rans_build_table(const uint32_t *freqs, int nsym, uint32_t *table) {
    uint32_t c = 0;
    for (int s = 0; s < nsym; ++s) {
        for (uint32_t v = 0; v < freqs[s]; ++v) table[c + v] = static_cast<uint32_t>(s) | (freqs[s] - 1) << 8 | v << 20;
        c += freqs[s];
    }
}

namespace {

// The words of one tile (in decode order, unpadded) and its 32 final states.
void encode_tile(const uint8_t *e, uint64_t m, const uint32_t *freqs, const uint32_t *cum, std::vector<uint16_t> &out,
                 uint32_t *states) {
    uint32_t x[kRansLanes];
    for (int j = 0; j < kRansLanes; ++j) x[j] = kRansL;
    out.clear();
    const uint64_t steps = (m + kRansLanes - 1) / kRansLanes;
    for (uint64_t k = steps; k-- > 0;) {
        for (int j = kRansLanes - 1; j >= 0; --j) {
            const uint64_t p = k * kRansLanes + static_cast<uint64_t>(j);
            if (p >= m) continue;
            const uint32_t s = e[p], f = freqs[s];
            if (static_cast<uint64_t>(x[j]) >= static_cast<uint64_t>(f) << (32 - kRansBits)) {
                out.push_back(static_cast<uint16_t>(x[j]));
                x[j] >>= 16;
            }
            x[j] = (x[j] / f) * kRansM + x[j] % f + cum[s];
        }
    }
    std::reverse(out.begin(), out.end());
    std::memcpy(states, x, sizeof x);
}

}  // namespace

std::string rans_encode_group(int dtype, const void *const *src, const uint64_t *n, int n_tensors,
                              uint32_t tile_symbols, int n_threads, RansGroup *out) {
    if (dtype != kBF16 && dtype != kE4M3) return "bad dtype";
    if (n_tensors < 1 || tile_symbols < kRansLanes || tile_symbols % kRansLanes || tile_symbols > (1u << 20))
        return "bad arguments";
    RansGroup &g = *out;
    g = RansGroup();
    g.dtype = dtype;
    g.nsym = nsym_of(dtype);
    g.tile_symbols = tile_symbols;
    uint64_t counts[256] = {};
    for (int i = 0; i < n_tensors; ++i) {
        if (n[i] && !src[i]) return "null source";
        histogram(dtype, src[i], n[i], counts, n_threads);
    }
    rans_freqs(counts, g.nsym, g.freqs);
    bool any = false;
    for (int s = 0; s < g.nsym; ++s) any |= g.freqs[s] != 0;
    if (any) rans_build_table(g.freqs, g.nsym, g.table);
    uint32_t cum[257] = {};
    for (int s = 0; s < g.nsym; ++s) cum[s + 1] = cum[s] + g.freqs[s];
    g.tensors.resize(n_tensors);
    for (int i = 0; i < n_tensors; ++i) {
        RansTensor &t = g.tensors[i];
        t.n = n[i];
        t.n_tiles = (n[i] + tile_symbols - 1) / tile_symbols;
        t.plane.assign(plane_bytes(dtype, n[i]), 0);
        std::vector<uint8_t> exps(n[i]);
        // fields, as the Huffman encoder splits them
        parallel_for((n[i] + 4095) / 4096, n_threads, [&](uint64_t b0, uint64_t b1) {
            for (uint64_t b = b0; b < b1; ++b) {
                const uint64_t lo = b * 4096, hi = std::min(n[i], lo + 4096);
                if (dtype == kBF16) {
                    const uint16_t *w = static_cast<const uint16_t *>(src[i]);
                    for (uint64_t k = lo; k < hi; ++k) {
                        exps[k] = static_cast<uint8_t>((w[k] >> 7) & 0xFF);
                        t.plane[k] = static_cast<uint8_t>(((w[k] >> 8) & 0x80) | (w[k] & 0x7F));
                    }
                } else {  // element pairs share a plane byte; blocks of 4096 keep pairs together
                    const uint8_t *w = static_cast<const uint8_t *>(src[i]);
                    for (uint64_t k = lo; k < hi; ++k) {
                        exps[k] = static_cast<uint8_t>((w[k] >> 3) & 0xF);
                        const uint8_t nib = static_cast<uint8_t>(((w[k] >> 4) & 0x8) | (w[k] & 0x7));
                        t.plane[k >> 1] = static_cast<uint8_t>(t.plane[k >> 1] | (nib << ((k & 1) * 4)));
                    }
                }
            }
        });
        // tiles in parallel, then concatenated with 8-word alignment
        std::vector<std::vector<uint16_t>> tw(t.n_tiles);
        t.states.assign(t.n_tiles * kRansLanes, 0);
        parallel_for(t.n_tiles, n_threads, [&](uint64_t a, uint64_t b) {
            for (uint64_t k = a; k < b; ++k) {
                const uint64_t base = k * tile_symbols, m = std::min<uint64_t>(tile_symbols, n[i] - base);
                encode_tile(exps.data() + base, m, g.freqs, cum, tw[k], t.states.data() + k * kRansLanes);
            }
        });
        t.tile_words.assign(t.n_tiles + 1, 0);
        uint64_t pos = 0;
        for (uint64_t k = 0; k < t.n_tiles; ++k) {
            t.tile_words[k] = pos;
            pos += (tw[k].size() + 7) / 8 * 8;
        }
        t.tile_words[t.n_tiles] = pos;
        t.words.assign(pos, 0);
        for (uint64_t k = 0; k < t.n_tiles; ++k)
            if (!tw[k].empty()) std::memcpy(t.words.data() + t.tile_words[k], tw[k].data(), tw[k].size() * 2);
    }
    return "";
}

std::vector<RansTensorLayout> rans_layout(const RansGroup &g, uint64_t *total) {
    std::vector<RansTensorLayout> L(g.tensors.size());
    uint64_t o = align_up(kRansM * 4, kImageAlign);
    for (size_t i = 0; i < g.tensors.size(); ++i) {
        const RansTensor &t = g.tensors[i];
        L[i].states = o;
        o = align_up(o + t.n_tiles * kRansLanes * 4, kImageAlign);
        L[i].tile_words = o;
        o = align_up(o + (t.n_tiles + 1) * 8, kImageAlign);
        L[i].words = o;
        o = align_up(o + (t.words.size() + kRansWordsTail) * 2, kImageAlign);
        L[i].plane = o;
        o = align_up(o + plane_bytes(g.dtype, t.n) + kRansPlaneTail, kImageAlign);
        L[i].end = o;
    }
    *total = o;
    return L;
}

void rans_write_image(const RansGroup &g, uint8_t *dst) {
    uint64_t total = 0;
    const auto L = rans_layout(g, &total);
    std::memset(dst, 0, total);
    std::memcpy(dst, g.table, sizeof g.table);
    for (size_t i = 0; i < g.tensors.size(); ++i) {
        const RansTensor &t = g.tensors[i];
        if (!t.states.empty()) std::memcpy(dst + L[i].states, t.states.data(), t.states.size() * 4);
        std::memcpy(dst + L[i].tile_words, t.tile_words.data(), t.tile_words.size() * 8);
        if (!t.words.empty()) std::memcpy(dst + L[i].words, t.words.data(), t.words.size() * 2);
        if (!t.plane.empty()) std::memcpy(dst + L[i].plane, t.plane.data(), t.plane.size());
    }
}

}  // namespace df11

// ---------------------------------------------------------------- container
//
// One file per group: a 64-byte header, the frequencies (u16 per symbol),
// then per tensor a 32-byte record (n, n_tiles, words, reserved) followed by
// its states, tile word offsets, words and plane, every section 16-byte
// aligned.  The decode table is derived from the frequencies.

namespace df11 {
namespace {

struct RansFileHeader {
    char magic[8];  // "DF11RANS"
    uint32_t version;
    uint32_t dtype;
    uint32_t nsym;
    uint32_t tile_symbols;
    uint32_t n_tensors;
    uint32_t reserved[9];
};
static_assert(sizeof(RansFileHeader) == 64, "header layout");

struct RansFileTensor {
    uint64_t n, n_tiles, words, reserved;
};

const char kRansMagic[8] = {'D', 'F', '1', '1', 'R', 'A', 'N', 'S'};

inline uint64_t up16(uint64_t x) { return (x + 15) / 16 * 16; }

// Bytes of a tensor's sections after its record.
uint64_t tensor_bytes(int dtype, uint64_t n, uint64_t n_tiles, uint64_t words) {
    uint64_t o = up16(n_tiles * kRansLanes * 4);
    o += up16((n_tiles + 1) * 8);
    o += up16(words * 2);
    o += up16(plane_bytes(dtype, n));
    return o;
}

}  // namespace

uint64_t rans_serialized_bytes(const RansGroup &g) {
    uint64_t o = sizeof(RansFileHeader) + up16(static_cast<uint64_t>(g.nsym) * 2);
    for (const RansTensor &t : g.tensors)
        o += sizeof(RansFileTensor) + tensor_bytes(g.dtype, t.n, t.n_tiles, t.words.size());
    return o;
}

void rans_serialize(const RansGroup &g, uint8_t *dst) {
    const uint64_t total = rans_serialized_bytes(g);
    std::memset(dst, 0, total);
    RansFileHeader h{};
    std::memcpy(h.magic, kRansMagic, 8);
    h.version = 1;
    h.dtype = static_cast<uint32_t>(g.dtype);
    h.nsym = static_cast<uint32_t>(g.nsym);
    h.tile_symbols = g.tile_symbols;
    h.n_tensors = static_cast<uint32_t>(g.tensors.size());
    std::memcpy(dst, &h, sizeof h);
    uint64_t o = sizeof h;
    for (int s = 0; s < g.nsym; ++s) {
        const uint16_t f = static_cast<uint16_t>(g.freqs[s]);
        std::memcpy(dst + o + 2 * s, &f, 2);
    }
    o += up16(static_cast<uint64_t>(g.nsym) * 2);
    for (const RansTensor &t : g.tensors) {
        const RansFileTensor r{t.n, t.n_tiles, t.words.size(), 0};
        std::memcpy(dst + o, &r, sizeof r);
        o += sizeof r;
        if (!t.states.empty()) std::memcpy(dst + o, t.states.data(), t.states.size() * 4);
        o += up16(t.states.size() * 4);
        std::memcpy(dst + o, t.tile_words.data(), t.tile_words.size() * 8);
        o += up16(t.tile_words.size() * 8);
        if (!t.words.empty()) std::memcpy(dst + o, t.words.data(), t.words.size() * 2);
        o += up16(t.words.size() * 2);
        if (!t.plane.empty()) std::memcpy(dst + o, t.plane.data(), t.plane.size());
        o += up16(t.plane.size());
    }
}

std::string rans_deserialize(const uint8_t *src, uint64_t len, RansGroup *out) {
    if (len < sizeof(RansFileHeader)) return "truncated header";
    RansFileHeader h;
    std::memcpy(&h, src, sizeof h);
    if (std::memcmp(h.magic, kRansMagic, 8) != 0) return "bad magic";
    if (h.version != 1) return "unknown version";
    if (h.dtype != kBF16 && h.dtype != kE4M3) return "bad dtype";
    const int dtype = static_cast<int>(h.dtype);
    if (h.nsym != static_cast<uint32_t>(nsym_of(dtype))) return "bad symbol count";
    if (h.tile_symbols < kRansLanes || h.tile_symbols % kRansLanes || h.tile_symbols > (1u << 20))
        return "bad tile size";
    if (h.n_tensors < 1 || h.n_tensors > 64) return "bad tensor count";
    RansGroup &g = *out;
    g = RansGroup();
    g.dtype = dtype;
    g.nsym = static_cast<int>(h.nsym);
    g.tile_symbols = h.tile_symbols;
    uint64_t o = sizeof h;
    if (len < o + up16(static_cast<uint64_t>(g.nsym) * 2)) return "truncated frequencies";
    uint32_t sum = 0;
    for (int s = 0; s < g.nsym; ++s) {
        uint16_t f;
        std::memcpy(&f, src + o + 2 * s, 2);
        if (f > kRansM) return "frequency out of range";
        g.freqs[s] = f;
        sum += f;
    }
    o += up16(static_cast<uint64_t>(g.nsym) * 2);
    bool any_symbols = false;
    g.tensors.resize(h.n_tensors);
    for (uint32_t i = 0; i < h.n_tensors; ++i) {
        if (len < o + sizeof(RansFileTensor)) return "truncated tensor record";
        RansFileTensor r;
        std::memcpy(&r, src + o, sizeof r);
        o += sizeof r;
        if (r.n > (uint64_t{1} << 40) || r.reserved) return "bad tensor record";
        if (r.n_tiles != (r.n + h.tile_symbols - 1) / h.tile_symbols) return "tile count mismatch";
        if (r.words > r.n + 8 * r.n_tiles) return "word count out of range";
        const uint64_t need = tensor_bytes(dtype, r.n, r.n_tiles, r.words);
        if (len < o + need) return "truncated tensor sections";
        RansTensor &t = g.tensors[i];
        t.n = r.n;
        t.n_tiles = r.n_tiles;
        any_symbols |= r.n != 0;
        t.states.resize(r.n_tiles * kRansLanes);
        if (!t.states.empty()) std::memcpy(t.states.data(), src + o, t.states.size() * 4);
        o += up16(t.states.size() * 4);
        t.tile_words.resize(r.n_tiles + 1);
        std::memcpy(t.tile_words.data(), src + o, t.tile_words.size() * 8);
        o += up16(t.tile_words.size() * 8);
        t.words.resize(r.words);
        if (r.words) std::memcpy(t.words.data(), src + o, r.words * 2);
        o += up16(r.words * 2);
        t.plane.assign(src + o, src + o + plane_bytes(dtype, r.n));
        o += up16(t.plane.size());
        if (t.tile_words[0] != 0 || t.tile_words[r.n_tiles] != r.words) return "tile offsets endpoints";
        for (uint64_t k = 0; k < r.n_tiles; ++k) {
            if (t.tile_words[k + 1] < t.tile_words[k] || t.tile_words[k + 1] % 8) return "tile offsets";
            // a tile of m symbols takes at most one word per symbol, plus padding
            const uint64_t m = std::min<uint64_t>(h.tile_symbols, r.n - k * h.tile_symbols);
            if (t.tile_words[k + 1] - t.tile_words[k] > m + 7) return "tile word count out of range";
        }
        for (uint32_t x : t.states)
            if (x < kRansL) return "state below 2^16";
        if (dtype == kE4M3 && (r.n & 1) && (t.plane.back() & 0xF0)) return "nonzero plane padding";
    }
    if (o != len) return "container size mismatch";
    // the table: frequencies summing to 2^12 (all zero only for a group without symbols)
    if (sum != kRansM && (any_symbols || sum != 0)) return "frequencies do not sum to 4096";
    if (sum == kRansM) rans_build_table(g.freqs, g.nsym, g.table);
    return "";
}

}  // namespace df11
