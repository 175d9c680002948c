// codec.cpp -- host side of libdf11.
//
// Offline half of "70% Size, 100% Accuracy ... (DFloat11)", Abstract: an
// entropy code over the exponent field ("dynamic-length encodings ... based
// on frequency"), the compressed layout with its auxiliary variables, and the
// hierarchical lookup tables the decoder keeps in shared memory.  Field
// layout from the "Compressing LLMs without Compromise" summary page, section
// "Where the redundancy lives"; FP8 from "To Compress or Not? ... Exponent
// Concentration", Abstract.
#include "codec.h"

#include <algorithm>
#include <cmath>
#include <atomic>
#include <cstring>
#include <thread>

namespace df11 {

namespace {

inline uint8_t exponent_of(int dtype, const void *src, uint64_t i) {
    if (dtype == kBF16) return static_cast<uint8_t>((static_cast<const uint16_t *>(src)[i] >> 7) & 0xFF);
    return static_cast<uint8_t>((static_cast<const uint8_t *>(src)[i] >> 3) & 0xF);
}

// ---------------------------------------------------------------- Huffman

// Two-queue Huffman construction over leaves sorted by (count, symbol).
// Merged nodes are created with non-decreasing counts, so the queue of merged
// nodes stays ordered; on equal counts a leaf is taken before a merged node
// and older merged nodes before newer ones.  Returns the deepest leaf.
int huffman(const uint64_t *counts, int nsym, uint8_t *lengths) {
    std::vector<int> leaves;
    for (int s = 0; s < nsym; ++s) {
        lengths[s] = 0;
        if (counts[s]) leaves.push_back(s);
    }
    const int m = static_cast<int>(leaves.size());
    if (m == 0) return 0;
    if (m == 1) {
        lengths[leaves[0]] = 1;
        return 1;
    }
    std::stable_sort(leaves.begin(), leaves.end(),
                     [&](int a, int b) { return counts[a] < counts[b]; });
    // node ids: 0..m-1 leaves (in sorted order), m.. merged nodes
    std::vector<uint64_t> w(2 * m);
    std::vector<int> parent(2 * m, -1);
    for (int i = 0; i < m; ++i) w[i] = counts[leaves[i]];
    int li = 0, qi = m, next = m;
    auto take = [&]() {
        if (li < m && (qi >= next || w[li] <= w[qi])) return li++;
        return qi++;
    };
    while (next < 2 * m - 1) {
        int a = take();
        int b = take();
        w[next] = w[a] + w[b];
        parent[a] = parent[b] = next;
        ++next;
    }
    // depth by walking merged nodes from the root down (root = 2m-2)
    std::vector<int> depth(2 * m, 0);
    for (int v = 2 * m - 3; v >= 0; --v) depth[v] = depth[parent[v]] + 1;
    int maxd = 0;
    for (int i = 0; i < m; ++i) {
        lengths[leaves[i]] = static_cast<uint8_t>(depth[i]);
        maxd = std::max(maxd, depth[i]);
    }
    return maxd;
}

// Package-merge: optimal lengths under a length limit.  Each level's list
// merges the sorted leaves with the pairs of the next-deeper list; equal
// weights keep leaves first.  Lengths = occurrences of each leaf among the
// first 2(m-1) items of the top list.
bool package_merge(const uint64_t *counts, int nsym, int max_len, uint8_t *lengths) {
    std::vector<int> leaves;
    for (int s = 0; s < nsym; ++s) {
        lengths[s] = 0;
        if (counts[s]) leaves.push_back(s);
    }
    const int m = static_cast<int>(leaves.size());
    if (m <= 1) {
        if (m == 1) lengths[leaves[0]] = 1;
        return true;
    }
    if (max_len < 32 && (uint64_t{1} << max_len) < static_cast<uint64_t>(m)) return false;
    std::stable_sort(leaves.begin(), leaves.end(),
                     [&](int a, int b) { return counts[a] < counts[b]; });
    // An item carries the per-leaf occurrence counts it covers; m <= 256 and
    // max_len <= 32, so dense count vectors stay small.
    struct Item {
        uint64_t w;
        std::vector<uint16_t> occ;  // per leaf index
    };
    std::vector<Item> prev;
    for (int level = max_len; level >= 1; --level) {
        std::vector<Item> packs;
        for (size_t i = 0; i + 1 < prev.size(); i += 2) {
            Item p;
            p.w = prev[i].w + prev[i + 1].w;
            p.occ = prev[i].occ;
            for (int k = 0; k < m; ++k) p.occ[k] = static_cast<uint16_t>(p.occ[k] + prev[i + 1].occ[k]);
            packs.push_back(std::move(p));
        }
        std::vector<Item> cur;
        cur.reserve(m + packs.size());
        size_t pi = 0;
        for (int i = 0; i < m || pi < packs.size();) {
            if (pi >= packs.size() || (i < m && counts[leaves[i]] <= packs[pi].w)) {
                Item leaf;
                leaf.w = counts[leaves[i]];
                leaf.occ.assign(m, 0);
                leaf.occ[i] = 1;
                cur.push_back(std::move(leaf));
                ++i;
            } else {
                cur.push_back(std::move(packs[pi++]));
            }
        }
        prev.swap(cur);
    }
    std::vector<int> len(m, 0);
    for (int i = 0; i < 2 * (m - 1); ++i)
        for (int k = 0; k < m; ++k) len[k] += prev[i].occ[k];
    for (int k = 0; k < m; ++k) lengths[leaves[k]] = static_cast<uint8_t>(len[k]);
    return true;
}

}  // namespace

bool code_lengths(const uint64_t *counts, int nsym, int max_len, uint8_t *lengths) {
    if (nsym < 1 || nsym > 256 || max_len < 1 || max_len > kMaxCodeLen) return false;
    int d = huffman(counts, nsym, lengths);
    if (d <= max_len) return true;
    return package_merge(counts, nsym, max_len, lengths);
}

bool canonical_codes(const uint8_t *lengths, int nsym, uint32_t *codes) {
    // Count codes per length, then hand out consecutive values per length in
    // symbol order; the first code of each length continues from the last
    // code of the shorter lengths, shifted left.
    uint32_t per_len[kMaxCodeLen + 2] = {};
    for (int s = 0; s < nsym; ++s) {
        if (lengths[s] > kMaxCodeLen) return false;
        if (lengths[s]) per_len[lengths[s]]++;
    }
    uint64_t next[kMaxCodeLen + 2] = {};
    uint64_t code = 0;
    for (int l = 1; l <= kMaxCodeLen; ++l) {
        code = (code + per_len[l - 1]) << 1;
        next[l] = code;
        if (per_len[l] && next[l] + per_len[l] > (uint64_t{1} << l)) return false;  // Kraft sum > 1
    }
    for (int s = 0; s < nsym; ++s) {
        codes[s] = 0;
        if (lengths[s]) codes[s] = static_cast<uint32_t>(next[lengths[s]]++);
    }
    return true;
}

namespace {

// Hierarchical 256-entry tables.  A code of length L is walked 8 bits per
// level; levels above its last one hold pointers, its last level holds the
// leaf replicated over the unused low bits.
bool build_lut(const uint8_t *lengths, const uint32_t *codes, int nsym, std::vector<uint16_t> &lut) {
    lut.assign(kLutEntries, kLutInvalid);
    for (int s = 0; s < nsym; ++s) {
        int L = lengths[s];
        if (!L) continue;
        uint32_t c = codes[s];
        int table = 0, rem = L;
        while (rem > 8) {
            uint32_t idx = (c >> (rem - 8)) & 0xFF;
            uint16_t &e = lut[static_cast<size_t>(table) * kLutEntries + idx];
            if (e & kLutPointer) {
                table = e & 0x7FFF;
            } else {
                if (e != kLutInvalid) return false;  // a shorter code is a prefix
                int nt = static_cast<int>(lut.size() / kLutEntries);
                if (nt > kMaxLutTables) return false;
                e = static_cast<uint16_t>(kLutPointer | nt);
                lut.resize(lut.size() + kLutEntries, kLutInvalid);
                table = nt;
            }
            rem -= 8;
        }
        uint32_t low = c & ((1u << rem) - 1);
        uint32_t first = low << (8 - rem), span = 1u << (8 - rem);
        for (uint32_t j = 0; j < span; ++j) {
            uint16_t &e = lut[static_cast<size_t>(table) * kLutEntries + first + j];
            if (e != kLutInvalid) return false;
            e = static_cast<uint16_t>(s | (L << 8));
        }
    }
    return true;
}

// Multi-symbol table over 12-bit windows, from a length-indexed canonical
// decoder: a code of length l matches when the next l bits fall in the range
// of length-l codes.
void build_multi(const uint8_t *lengths, const uint32_t *codes, int nsym, std::vector<uint32_t> &meta,
                 std::vector<uint32_t> &syms) {
    int lo_sym[kMaxCodeLen + 1];
    uint32_t first[kMaxCodeLen + 1], cnt[kMaxCodeLen + 1] = {};
    int by_code[kMaxCodeLen + 1][256];
    for (int l = 0; l <= kMaxCodeLen; ++l) {
        first[l] = 0xFFFFFFFFu;
        lo_sym[l] = -1;
    }
    for (int s = 0; s < nsym; ++s) {
        int l = lengths[s];
        if (!l) continue;
        if (codes[s] < first[l]) first[l] = codes[s];
    }
    for (int s = 0; s < nsym; ++s) {
        int l = lengths[s];
        if (!l) continue;
        by_code[l][codes[s] - first[l]] = s;
        cnt[l]++;
        lo_sym[l] = 0;
    }
    meta.assign(kMultiEntries, kMetaLong);
    syms.assign(kMultiEntries, 0);
    for (uint32_t v = 0; v < static_cast<uint32_t>(kMultiEntries); ++v) {
        int pos = 0, k = 0;
        uint32_t packed = 0, starts = 0;
        while (k < kMultiMaxSyms) {
            int found = -1, flen = 0;
            for (int l = 1; l <= kMultiBits - pos; ++l) {
                if (lo_sym[l] < 0) continue;
                uint32_t bits = (v >> (kMultiBits - pos - l)) & ((1u << l) - 1);
                if (bits >= first[l] && bits - first[l] < cnt[l]) {
                    found = by_code[l][bits - first[l]];
                    flen = l;
                    break;
                }
            }
            if (found < 0) break;
            starts |= 1u << pos;
            packed |= static_cast<uint32_t>(found) << (8 * k);
            pos += flen;
            ++k;
        }
        if (k) {
            meta[v] = static_cast<uint32_t>(pos) | (static_cast<uint32_t>(k) << kMetaCountShift) |
                      (starts << kMetaMaskShift);
            syms[v] = packed;
        }
    }
}

// Byte-step transition tables over the code tree (layout in df11_internal.h).
// The tree is built from the canonical codes; the rows go to the internal
// nodes with the most probability mass below them, taking 2^-length as a
// code's probability (a byte boundary falls on node v with a probability
// proportional to that mass), so the dead row is rarely reached.
void build_fsm(const uint8_t *lengths, const uint32_t *codes, int nsym, std::vector<uint32_t> &fsm,
               int &rows) {
    struct Node {
        int child[2] = {-1, -1};
        int sym = -1;
        int depth = 0;
        uint64_t prefix = 0;
        double mass = 0.0;
    };
    std::vector<Node> nodes(1);
    for (int s = 0; s < nsym; ++s) {
        const int L = lengths[s];
        if (!L) continue;
        int v = 0;
        for (int i = L - 1; i >= 0; --i) {
            const int bit = static_cast<int>((codes[s] >> i) & 1u);
            if (nodes[v].child[bit] < 0) {
                Node n;
                n.depth = nodes[v].depth + 1;
                n.prefix = (nodes[v].prefix << 1) | static_cast<uint64_t>(bit);
                nodes.push_back(n);
                nodes[v].child[bit] = static_cast<int>(nodes.size()) - 1;
            }
            v = nodes[v].child[bit];
        }
        nodes[v].sym = s;
        nodes[v].mass = std::ldexp(1.0, -L);
    }
    // children are created after their parent: one backward pass sums the masses
    for (int v = static_cast<int>(nodes.size()) - 1; v > 0; --v) {
        for (int c : nodes[v].child)
            if (c >= 0) nodes[v].mass += nodes[c].mass;
    }
    for (int c : nodes[0].child)
        if (c >= 0) nodes[0].mass += nodes[c].mass;
    std::vector<int> internal;
    for (int v = 0; v < static_cast<int>(nodes.size()); ++v)
        if (nodes[v].sym < 0) internal.push_back(v);
    std::stable_sort(internal.begin() + 1, internal.end(), [&](int a, int b) {
        if (nodes[a].mass != nodes[b].mass) return nodes[a].mass > nodes[b].mass;
        if (nodes[a].depth != nodes[b].depth) return nodes[a].depth < nodes[b].depth;
        return nodes[a].prefix < nodes[b].prefix;
    });
    const int live = std::min<int>(static_cast<int>(internal.size()), kFsmMaxRows - 1);
    rows = live + 1;
    const uint32_t dead = static_cast<uint32_t>(live);
    std::vector<int> row_of(nodes.size(), -1);
    for (int r = 0; r < live; ++r) row_of[internal[r]] = r;
    fsm.assign(static_cast<size_t>(rows) * kLutEntries * 2, 0);
    for (int r = 0; r < rows; ++r) {
        for (uint32_t b = 0; b < static_cast<uint32_t>(kLutEntries); ++b) {
            uint32_t ctl = dead << kFsmRowShift, packed = 0;
            if (r < live) {
                int v = internal[r], k = 0;
                uint32_t ends = 0;
                bool bad = false;
                for (int i = 0; i < 8; ++i) {
                    const int c = nodes[v].child[(b >> (7 - i)) & 1u];
                    if (c < 0) {
                        bad = true;
                        break;
                    }
                    if (nodes[c].sym >= 0) {
                        if (k < 4) packed |= static_cast<uint32_t>(nodes[c].sym) << (8 * k);
                        ++k;
                        ends |= 1u << i;
                        v = 0;
                    } else {
                        v = c;
                    }
                }
                const uint32_t next = (bad || k > 4 || row_of[v] < 0) ? dead : static_cast<uint32_t>(row_of[v]);
                ctl = ends | (next << kFsmRowShift) | (static_cast<uint32_t>(std::min(k, 7)) << kFsmCountShift);
            }
            const size_t e = (static_cast<size_t>(r) * kLutEntries + b) * 2;
            fsm[e] = ctl;
            fsm[e + 1] = packed;
        }
    }
}

}  // namespace

std::shared_ptr<Codebook> make_codebook(int dtype, const uint8_t *lengths) {
    auto cb = std::make_shared<Codebook>();
    cb->dtype = dtype;
    cb->nsym = nsym_of(dtype);
    int maxl = 0, minl = 0;
    for (int s = 0; s < cb->nsym; ++s) {
        cb->lengths[s] = lengths[s];
        if (lengths[s]) {
            maxl = std::max<int>(maxl, lengths[s]);
            minl = minl ? std::min<int>(minl, lengths[s]) : lengths[s];
        }
    }
    cb->max_len_used = maxl;
    cb->min_len_used = minl;
    if (!canonical_codes(cb->lengths, cb->nsym, cb->codes)) return nullptr;
    if (!build_lut(cb->lengths, cb->codes, cb->nsym, cb->lut)) return nullptr;
    build_multi(cb->lengths, cb->codes, cb->nsym, cb->meta, cb->syms);
    build_fsm(cb->lengths, cb->codes, cb->nsym, cb->fsm, cb->fsm_rows);
    return cb;
}

void histogram(int dtype, const void *src, uint64_t n, uint64_t *counts, int n_threads) {
    const int nsym = nsym_of(dtype);
    std::vector<std::vector<uint64_t>> parts;
    std::atomic<int> slot{0};
    unsigned hw = std::thread::hardware_concurrency();
    int t = n_threads > 0 ? n_threads : static_cast<int>(hw ? hw : 1);
    parts.assign(t + 1, std::vector<uint64_t>(256, 0));
    parallel_for(n, t, [&](uint64_t b, uint64_t e) {
        auto &h = parts[slot.fetch_add(1)];
        for (uint64_t i = b; i < e; ++i) h[exponent_of(dtype, src, i)]++;
    });
    for (auto &h : parts)
        for (int s = 0; s < nsym; ++s) counts[s] += h[s];
}

bool valid_layout(int chunk_bits, int tile_threads) {
    return (chunk_bits == 64 || chunk_bits == 128 || chunk_bits == 256) &&
           (tile_threads == 32 || tile_threads == 128 || tile_threads == 256 || tile_threads == 512);
}

uint64_t plane_bytes(int dtype, uint64_t n) { return dtype == kBF16 ? n : (n + 1) / 2; }

namespace {

inline void or_byte(uint8_t *p, uint8_t v) { __atomic_fetch_or(p, v, __ATOMIC_RELAXED); }

}  // namespace

std::string encode(std::shared_ptr<const Codebook> cb, const void *src, uint64_t n, int chunk_bits,
                   int tile_threads, int n_threads, bool chunk_counts, Blob *out) {
    if (!valid_layout(chunk_bits, tile_threads)) return "unsupported layout";
    if (n && !src) return "null source";
    const int dtype = cb->dtype;
    Blob &b = *out;
    b = Blob();
    b.dtype = dtype;
    b.chunk_bits = chunk_bits;
    b.tile_threads = tile_threads;
    b.n = n;
    b.cb = cb;
    b.chunk_counts = chunk_counts && counts_fit(chunk_bits);
    b.plane.assign(plane_bytes(dtype, n), 0);

    // segments of an even number of elements (E4M3 packs pairs into a byte)
    const uint64_t seg_elems = std::max<uint64_t>(1 << 16, ((n / 256) + 1) & ~uint64_t{1});
    const uint64_t n_seg = n ? (n + seg_elems - 1) / seg_elems : 0;
    std::vector<uint64_t> seg_bits(n_seg + 1, 0);
    std::vector<uint8_t> exps(n);
    std::atomic<bool> uncovered{false};
    const uint8_t *len = cb->lengths;

    // pass 1: split fields, count code bits per segment
    parallel_for(n_seg, n_threads, [&](uint64_t s0, uint64_t s1) {
        for (uint64_t s = s0; s < s1; ++s) {
            uint64_t i0 = s * seg_elems, i1 = std::min(n, i0 + seg_elems), bits = 0;
            if (dtype == kBF16) {
                const uint16_t *w = static_cast<const uint16_t *>(src);
                for (uint64_t i = i0; i < i1; ++i) {
                    uint16_t v = w[i];
                    uint8_t e = static_cast<uint8_t>((v >> 7) & 0xFF);
                    exps[i] = e;
                    b.plane[i] = static_cast<uint8_t>(((v >> 8) & 0x80) | (v & 0x7F));
                    bits += len[e];
                    if (!len[e]) uncovered = true;
                }
            } else {
                const uint8_t *w = static_cast<const uint8_t *>(src);
                for (uint64_t i = i0; i < i1; ++i) {
                    uint8_t v = w[i];
                    uint8_t e = static_cast<uint8_t>((v >> 3) & 0xF);
                    uint8_t nib = static_cast<uint8_t>(((v >> 4) & 0x8) | (v & 0x7));
                    exps[i] = e;
                    b.plane[i >> 1] = static_cast<uint8_t>(b.plane[i >> 1] | (nib << ((i & 1) * 4)));
                    bits += len[e];
                    if (!len[e]) uncovered = true;
                }
            }
            seg_bits[s + 1] = bits;
        }
    });
    if (uncovered) return "tensor holds an exponent the code does not cover";
    for (uint64_t s = 0; s < n_seg; ++s) seg_bits[s + 1] += seg_bits[s];
    const uint64_t total = seg_bits[n_seg];
    b.total_bits = total;
    const uint64_t cbits = static_cast<uint64_t>(chunk_bits);
    const uint64_t tbits = cbits * static_cast<uint64_t>(tile_threads);
    const uint64_t n_chunks = (total + cbits - 1) / cbits;
    b.n_tiles = (n_chunks + tile_threads - 1) / tile_threads;
    b.stream.assign((total + 7) / 8, 0);
    b.gaps.assign(b.n_tiles * tile_threads, 0);
    b.out_off.assign(b.n_tiles + 1, n);
    if (!b.out_off.empty()) b.out_off[0] = 0;
    const uint32_t *code = cb->codes;

    // pass 2: pack codes MSB-first; record the first code start of every
    // chunk (gap) and of every tile (out_off)
    parallel_for(n_seg, n_threads, [&](uint64_t s0, uint64_t s1) {
        for (uint64_t s = s0; s < s1; ++s) {
            uint64_t i0 = s * seg_elems, i1 = std::min(n, i0 + seg_elems);
            uint64_t start = seg_bits[s];
            uint64_t prev_chunk = i0 ? (start - len[exps[i0 - 1]]) / cbits : ~uint64_t{0};
            uint64_t prev_tile = i0 ? (start - len[exps[i0 - 1]]) / tbits : ~uint64_t{0};
            uint8_t *outp = b.stream.data();
            uint64_t byte = start >> 3;
            int nacc = static_cast<int>(start & 7);
            bool shared_first = nacc != 0;
            uint64_t acc = 0;
            for (uint64_t i = i0; i < i1; ++i) {
                const uint8_t e = exps[i];
                const int l = len[e];
                uint64_t c_idx = start / cbits;
                if (c_idx != prev_chunk) {
                    for (uint64_t c = prev_chunk + 1; c <= c_idx; ++c) b.gaps[c] = static_cast<uint8_t>(start - c * cbits);
                    prev_chunk = c_idx;
                }
                uint64_t t_idx = start / tbits;
                if (t_idx != prev_tile) {
                    for (uint64_t t = prev_tile + 1; t <= t_idx; ++t) b.out_off[t] = i;
                    prev_tile = t_idx;
                }
                start += l;
                acc |= static_cast<uint64_t>(code[e]) << (64 - nacc - l);
                nacc += l;
                if (nacc >= 32) {
                    uint8_t v0 = static_cast<uint8_t>(acc >> 56);
                    if (shared_first) {
                        or_byte(outp + byte, v0);
                        shared_first = false;
                    } else {
                        outp[byte] = v0;
                    }
                    outp[byte + 1] = static_cast<uint8_t>(acc >> 48);
                    outp[byte + 2] = static_cast<uint8_t>(acc >> 40);
                    outp[byte + 3] = static_cast<uint8_t>(acc >> 32);
                    byte += 4;
                    acc <<= 32;
                    nacc -= 32;
                }
            }
            while (nacc >= 8) {
                uint8_t v0 = static_cast<uint8_t>(acc >> 56);
                if (shared_first) {
                    or_byte(outp + byte, v0);
                    shared_first = false;
                } else {
                    outp[byte] = v0;
                }
                ++byte;
                acc <<= 8;
                nacc -= 8;
            }
            if (nacc > 0) or_byte(outp + byte, static_cast<uint8_t>(acc >> 56));
        }
    });
    // chunks after the last code start (at most the final one): no start, so
    // the gap reaches the end of the stream
    if (n) {
        uint64_t last_start = total - len[exps[n - 1]];
        for (uint64_t c = last_start / cbits + 1; c < n_chunks; ++c) b.gaps[c] = static_cast<uint8_t>(total - c * cbits);
    }
    uint64_t ms = 0;
    for (uint64_t t = 0; t < b.n_tiles; ++t) ms = std::max(ms, b.out_off[t + 1] - b.out_off[t]);
    b.max_span = ms;

    // pass 3 (chunk counts): codes starting in each chunk.  A segment counts
    // the chunk its first code starts in locally (an earlier segment may
    // count codes of that chunk too) and every later chunk in place, which
    // no other segment touches; the local counts are added afterwards.
    if (b.chunk_counts) {
        b.counts.assign(b.n_tiles * tile_threads, 0);
        std::vector<uint32_t> first_count(n_seg, 0);
        parallel_for(n_seg, n_threads, [&](uint64_t s0, uint64_t s1) {
            for (uint64_t s = s0; s < s1; ++s) {
                const uint64_t i0 = s * seg_elems, i1 = std::min(n, i0 + seg_elems);
                uint64_t start = seg_bits[s];
                const uint64_t c_first = start / cbits;
                uint32_t local = 0;
                for (uint64_t i = i0; i < i1; ++i) {
                    const uint64_t c = start / cbits;
                    if (c == c_first) ++local;
                    else ++b.counts[c];
                    start += len[exps[i]];
                }
                first_count[s] = local;
            }
        });
        for (uint64_t s = 0; s < n_seg; ++s)
            b.counts[seg_bits[s] / cbits] = static_cast<uint8_t>(b.counts[seg_bits[s] / cbits] + first_count[s]);
    }
    return "";
}

// ---------------------------------------------------------------- container

namespace {

struct FileHeader {
    char magic[8];
    uint32_t version;
    uint32_t dtype;
    uint64_t n_elems;
    uint64_t total_bits;
    uint32_t chunk_bits;
    uint32_t tile_threads;
    uint64_t n_tiles;
    uint64_t max_span;
    uint32_t nsym;
    uint32_t flags;  // version 2: bit 0 = the chunk-counts section follows the gaps
};
static_assert(sizeof(FileHeader) == 64, "header layout");
constexpr uint32_t kFileFlagCounts = 1;

const char kMagic[8] = {'D', 'F', '1', '1', 'B', '2', '0', '0'};

struct FileLayout {
    uint64_t lengths, gaps, counts, out_off, stream, plane, total;
};

FileLayout file_layout(int dtype, uint64_t n, uint64_t total_bits, uint64_t n_tiles, int tile_threads,
                       bool counts) {
    FileLayout f;
    f.lengths = sizeof(FileHeader);
    f.gaps = align_up(f.lengths + 256, 16);
    f.counts = align_up(f.gaps + n_tiles * tile_threads, 16);
    f.out_off = align_up(f.counts + (counts ? n_tiles * tile_threads : 0), 16);
    f.stream = align_up(f.out_off + (n_tiles + 1) * 8, 16);
    f.plane = align_up(f.stream + (total_bits + 7) / 8, 16);
    f.total = align_up(f.plane + plane_bytes(dtype, n), 16);
    return f;
}

}  // namespace

uint64_t serialized_bytes(const Blob &b) {
    return file_layout(b.dtype, b.n, b.total_bits, b.n_tiles, b.tile_threads, b.chunk_counts).total;
}

void serialize(const Blob &b, uint8_t *dst) {
    FileLayout f = file_layout(b.dtype, b.n, b.total_bits, b.n_tiles, b.tile_threads, b.chunk_counts);
    std::memset(dst, 0, f.total);
    FileHeader h{};
    std::memcpy(h.magic, kMagic, 8);
    // version 1 (no flags) unless the counts section is present
    h.version = b.chunk_counts ? 2 : 1;
    h.flags = b.chunk_counts ? kFileFlagCounts : 0;
    h.dtype = static_cast<uint32_t>(b.dtype);
    h.n_elems = b.n;
    h.total_bits = b.total_bits;
    h.chunk_bits = static_cast<uint32_t>(b.chunk_bits);
    h.tile_threads = static_cast<uint32_t>(b.tile_threads);
    h.n_tiles = b.n_tiles;
    h.max_span = b.max_span;
    h.nsym = static_cast<uint32_t>(nsym_of(b.dtype));
    std::memcpy(dst, &h, sizeof h);
    std::memcpy(dst + f.lengths, b.cb->lengths, 256);
    if (!b.gaps.empty()) std::memcpy(dst + f.gaps, b.gaps.data(), b.gaps.size());
    if (b.chunk_counts && !b.counts.empty()) std::memcpy(dst + f.counts, b.counts.data(), b.counts.size());
    std::memcpy(dst + f.out_off, b.out_off.data(), b.out_off.size() * 8);
    if (!b.stream.empty()) std::memcpy(dst + f.stream, b.stream.data(), b.stream.size());
    if (!b.plane.empty()) std::memcpy(dst + f.plane, b.plane.data(), b.plane.size());
}

std::string deserialize(const uint8_t *src, uint64_t len, Blob *out) {
    if (len < sizeof(FileHeader) + 256) return "truncated header";
    FileHeader h;
    std::memcpy(&h, src, sizeof h);
    if (std::memcmp(h.magic, kMagic, 8) != 0) return "bad magic";
    if (h.version != 1 && h.version != 2) return "unknown version";
    if (h.version == 1 && h.flags) return "flags in a version 1 container";
    if (h.flags & ~kFileFlagCounts) return "unknown flags";
    const bool has_counts = (h.flags & kFileFlagCounts) != 0;
    if (h.dtype != kBF16 && h.dtype != kE4M3) return "bad dtype";
    const int dtype = static_cast<int>(h.dtype);
    if (h.nsym != static_cast<uint32_t>(nsym_of(dtype))) return "bad symbol count";
    if (!valid_layout(static_cast<int>(h.chunk_bits), static_cast<int>(h.tile_threads))) return "bad layout";
    if (has_counts && !counts_fit(static_cast<int>(h.chunk_bits))) return "chunk counts with chunks over 128 bits";
    if (h.n_elems > (uint64_t{1} << 48)) return "element count out of range";
    const uint64_t cbits = h.chunk_bits, tbits = cbits * h.tile_threads;
    const uint64_t n_chunks = (h.total_bits + cbits - 1) / cbits;
    if (h.n_tiles != (n_chunks + h.tile_threads - 1) / h.tile_threads) return "tile count mismatch";
    if (h.total_bits > h.n_elems * kMaxCodeLen || h.total_bits < h.n_elems) return "stream length out of range";
    FileLayout f = file_layout(dtype, h.n_elems, h.total_bits, h.n_tiles, static_cast<int>(h.tile_threads),
                               has_counts);
    if (f.total != len) return "container size mismatch";
    uint8_t lengths[256];
    std::memcpy(lengths, src + f.lengths, 256);
    for (int s = nsym_of(dtype); s < 256; ++s)
        if (lengths[s]) return "length for a symbol outside the alphabet";
    auto cb = make_codebook(dtype, lengths);
    if (!cb) return "code lengths do not form a prefix code";
    if (h.n_elems && !cb->max_len_used) return "empty code for a non-empty tensor";
    Blob &b = *out;
    b = Blob();
    b.dtype = dtype;
    b.chunk_bits = static_cast<int>(h.chunk_bits);
    b.tile_threads = static_cast<int>(h.tile_threads);
    b.n = h.n_elems;
    b.total_bits = h.total_bits;
    b.n_tiles = h.n_tiles;
    b.max_span = h.max_span;
    b.cb = cb;
    b.gaps.assign(src + f.gaps, src + f.gaps + h.n_tiles * h.tile_threads);
    b.chunk_counts = has_counts;
    if (has_counts) b.counts.assign(src + f.counts, src + f.counts + h.n_tiles * h.tile_threads);
    b.out_off.resize(h.n_tiles + 1);
    std::memcpy(b.out_off.data(), src + f.out_off, (h.n_tiles + 1) * 8);
    b.stream.assign(src + f.stream, src + f.stream + (h.total_bits + 7) / 8);
    b.plane.assign(src + f.plane, src + f.plane + plane_bytes(dtype, h.n_elems));
    // auxiliary values
    if (b.out_off[0] != 0 || b.out_off[h.n_tiles] != h.n_elems) return "out_off endpoints";
    uint64_t ms = 0;
    for (uint64_t t = 0; t < h.n_tiles; ++t) {
        if (b.out_off[t + 1] < b.out_off[t]) return "out_off not monotone";
        uint64_t span = b.out_off[t + 1] - b.out_off[t];
        if (span > tbits) return "tile span exceeds its bits";
        ms = std::max(ms, span);
    }
    if (ms != h.max_span) return "max_span mismatch";
    for (uint64_t c = 0; c < b.gaps.size(); ++c) {
        if (c < n_chunks) {
            if (b.gaps[c] >= cb->max_len_used && c + 1 < n_chunks) return "gap beyond the longest code";
            if (c * cbits + b.gaps[c] > h.total_bits) return "gap beyond the stream";
        } else if (b.gaps[c]) {
            return "nonzero padding gap";
        }
    }
    if (has_counts) {
        // each tile's counts add up to its span; padding chunks start no code
        for (uint64_t t = 0; t < h.n_tiles; ++t) {
            uint64_t sum = 0;
            for (uint64_t j = 0; j < h.tile_threads; ++j) {
                const uint64_t c = t * h.tile_threads + j;
                if (c >= n_chunks && b.counts[c]) return "nonzero padding count";
                if (b.counts[c] > cbits) return "chunk count above its bits";
                sum += b.counts[c];
            }
            if (sum != b.out_off[t + 1] - b.out_off[t]) return "chunk counts do not add up to the tile span";
        }
    }
    if (h.total_bits & 7) {
        uint8_t pad_mask = static_cast<uint8_t>(0xFFu >> (h.total_bits & 7));
        if (b.stream.back() & pad_mask) return "nonzero stream padding";
    }
    if (dtype == kE4M3 && (h.n_elems & 1) && (b.plane.back() & 0xF0)) return "nonzero plane padding";
    return "";
}

// ---------------------------------------------------------------- device image

ImageLayout image_layout(const Blob &b) {
    ImageLayout L;
    uint64_t o = align_up(sizeof(ImageHeader), kImageAlign);
    L.meta = o;
    o = align_up(o + kMultiEntries * 4, kImageAlign);
    L.syms = o;
    o = align_up(o + kMultiEntries * 4, kImageAlign);
    L.lut = o;
    o = align_up(o + b.cb->lut.size() * 2, kImageAlign);
    L.fsm = o;
    o = align_up(o + b.cb->fsm.size() * 4, kImageAlign);
    L.gaps = o;
    o = align_up(o + b.n_tiles * static_cast<uint64_t>(b.tile_threads) + kGapsTail, kImageAlign);
    L.counts = o;
    if (b.chunk_counts) o = align_up(o + b.n_tiles * static_cast<uint64_t>(b.tile_threads), kImageAlign);
    L.out_off = o;
    o = align_up(o + (b.n_tiles + 1) * 8, kImageAlign);
    L.stream = o;
    o = align_up(o + b.n_tiles * (static_cast<uint64_t>(b.chunk_bits) / 8) * b.tile_threads + kStreamTail, kImageAlign);
    L.plane = o;
    o = align_up(o + align_up(plane_bytes(b.dtype, b.n), 16) + kPlaneTail, kImageAlign);
    L.total = o;
    return L;
}

void write_image_head(const Blob &b, const ImageLayout &L, uint8_t *dst) {
    std::memset(dst, 0, L.gaps);
    ImageHeader h{};
    std::memcpy(h.magic, "DF11IMG1", 8);
    h.dtype = static_cast<uint32_t>(b.dtype);
    h.chunk_bits = static_cast<uint32_t>(b.chunk_bits);
    h.tile_threads = static_cast<uint32_t>(b.tile_threads);
    h.n_luts = static_cast<uint32_t>(b.cb->n_luts());
    h.fsm_rows = static_cast<uint32_t>(b.cb->fsm_rows);
    h.flags = b.chunk_counts ? kImageFlagCounts : 0u;
    h.n_elems = b.n;
    h.total_bits = b.total_bits;
    h.n_tiles = b.n_tiles;
    h.max_span = b.max_span;
    h.layout = L;
    std::memcpy(dst, &h, sizeof h);
    std::memcpy(dst + L.meta, b.cb->meta.data(), kMultiEntries * 4);
    std::memcpy(dst + L.syms, b.cb->syms.data(), kMultiEntries * 4);
    std::memcpy(dst + L.lut, b.cb->lut.data(), b.cb->lut.size() * 2);
    std::memcpy(dst + L.fsm, b.cb->fsm.data(), b.cb->fsm.size() * 4);
}

void write_image(const Blob &b, uint8_t *dst) {
    ImageLayout L = image_layout(b);
    std::memset(dst, 0, L.total);
    write_image_head(b, L, dst);
    if (!b.gaps.empty()) std::memcpy(dst + L.gaps, b.gaps.data(), b.gaps.size());
    if (b.chunk_counts && !b.counts.empty()) std::memcpy(dst + L.counts, b.counts.data(), b.counts.size());
    std::memcpy(dst + L.out_off, b.out_off.data(), b.out_off.size() * 8);
    // stream as 32-bit words, earliest bit in bit 31 (little-endian storage)
    for (uint64_t i = 0; i < b.stream.size(); ++i) dst[L.stream + (i ^ 3)] = b.stream[i];
    if (!b.plane.empty()) std::memcpy(dst + L.plane, b.plane.data(), b.plane.size());
}

void read_image_sections(Blob &b, const uint8_t *img) {
    const ImageLayout L = image_layout(b);
    b.gaps.assign(img + L.gaps, img + L.gaps + b.n_tiles * b.tile_threads);
    if (b.chunk_counts) b.counts.assign(img + L.counts, img + L.counts + b.n_tiles * b.tile_threads);
    else b.counts.clear();
    b.out_off.resize(b.n_tiles + 1);
    std::memcpy(b.out_off.data(), img + L.out_off, (b.n_tiles + 1) * 8);
    b.stream.resize((b.total_bits + 7) / 8);
    for (uint64_t i = 0; i < b.stream.size(); ++i) b.stream[i] = img[L.stream + (i ^ 3)];
    b.plane.assign(img + L.plane, img + L.plane + plane_bytes(b.dtype, b.n));
    b.device_only = false;
}

}  // namespace df11
