// decode.cu -- sm_100a decode of Huffman-coded exponents back into the exact
// BF16 / FP8-E4M3 bit patterns.
//
// Method: "70% Size, 100% Accuracy ... (DFloat11)", Abstract, items (i)-(iii):
//   (i)   lookup tables in on-chip SRAM: the hierarchical 256-entry tables and
//         a 12-bit multi-symbol table are staged in shared memory once per CTA;
//   (ii)  a two-phase kernel: every thread owns chunk_bits stream bits and a
//         `gap` (offset of the first code starting in its chunk); phase 1
//         counts the codes that start in the chunk, a warp-shuffle + block
//         scan plus the tile's `out_off` gives every thread its output index,
//         phase 2 decodes again and writes the exponents;
//   (iii) block-level batching: one launch covers every tensor of a
//         transformer block through a table of tensor descriptors.
// Field layout ("Compressing LLMs without Compromise" summary page, "Where the
// redundancy lives"): BF16 = sign | 8-bit exponent | 7-bit mantissa, the raw
// byte plane holds sign << 7 | mantissa.  FP8 ("To Compress or Not? ...",
// Abstract): E4M3 = sign | 4-bit exponent | 3-bit mantissa, the plane holds
// one nibble sign << 3 | mantissa per weight.
//
// B200 structure (not in the sources, which predate this GPU):
//   * persistent CTAs, grid = SMs x resident CTAs, tiles strided over CTAs;
//   * one producer warp per CTA stages each tile's stream slice, gaps and
//     plane span into shared memory with 1-D TMA bulk copies (local global
//     memory, never multicast) on an mbarrier pipeline of STAGES buffers,
//     so the next tiles' loads overlap the current tile's decode;
//   * 8 (or 4 / 16) consumer warps decode; all waits are bounded (2 s of
//     %globaltimer) and report DF11_DEV_ERR_TIMEOUT instead of hanging;
//   * the merge reads 16 plane bytes and 16 (32 for E4M3) exponents from
//     shared memory per thread and writes 32 output bytes with two 16-byte
//     stores; tile edges that share a 32-byte group with the neighbouring
//     tile are written element by element.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <utility>

#include "df11.h"
#include "launch.h"
#include "walk.cuh"

namespace df11 {
namespace {

// ------------------------------------------------------------------ shared memory plan

struct StageMeta {
    uint64_t S;         // global index of the tile's first code
    uint32_t span;      // codes starting in the tile
    uint32_t tensor;    // descriptor index
    uint32_t local_tile;
    uint32_t bad;       // auxiliary data out of range: skip the tile
    uint32_t pad[2];
};
static_assert(sizeof(StageMeta) == 32, "stage meta");

constexpr uint32_t kCtrlBytes = 1024;
constexpr uint32_t kSmemBudget = 227u * 1024u;  // opt-in dynamic shared memory per CTA on sm_100
constexpr int kStreamStages = 2;
constexpr int kPrefetchGroups = 4;  // plane groups per thread loaded at tile start

// Shared memory of one CTA:
//   control (barriers, per-stage tile metadata, warp totals)
//   decode tables: 12-bit multi-symbol meta (u32) and symbols (u32), the
//   first hierarchical 256-entry tables (u16)
//   kStreamStages x (tile stream slice + 16 look-ahead bytes), x (gaps)
//   the tile's exponents in output order (all zero between tiles)
struct Plan {
    uint32_t stream_bytes, gaps_bytes, exps_bytes;
    uint32_t off_meta, off_syms, off_lut, off_stream, off_gaps, off_exps, total;
};

__host__ __device__ inline uint32_t up128(uint32_t x) { return (x + 127u) & ~127u; }

__host__ __device__ inline Plan make_plan(int chunk_bits, int chunks, uint32_t max_span, int n_lut_smem) {
    Plan p;
    p.stream_bytes = static_cast<uint32_t>(chunks * chunk_bits / 8) + 16u;
    p.gaps_bytes = static_cast<uint32_t>(chunks);
    p.exps_bytes = up128(max_span + 2u * 32u + 16u);
    p.off_meta = kCtrlBytes;
    p.off_syms = p.off_meta + kMultiEntries * 4;
    p.off_lut = p.off_syms + kMultiEntries * 4;
    p.off_stream = up128(p.off_lut + static_cast<uint32_t>(n_lut_smem) * kLutEntries * 2);
    p.off_gaps = p.off_stream + kStreamStages * up128(p.stream_bytes);
    p.off_exps = p.off_gaps + kStreamStages * up128(p.gaps_bytes);
    p.total = p.off_exps + p.exps_bytes;
    return p;
}

__device__ __forceinline__ void st_global_v4(void *p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ uint4 ld_global_stream_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// One group's plane bytes, checked in the bounds-checked build (zeros outside).
__device__ __forceinline__ uint4 plane_v4(const uint8_t *p, Guard &G) {
    return G.pl(p, 16) ? ld_global_stream_v4(p) : make_uint4(0u, 0u, 0u, 0u);
}

__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Stores the elements of a 32-byte output group that fall in [lo, hi) (tile-local
// element indices); the rest of the group belongs to a neighbouring tile or
// lies past the end of the tensor.  Rare: at most two groups per tile.
template <int DT>
__device__ __noinline__ void store_partial(uint8_t *out, uint4 a, uint4 b, uint32_t e0, uint32_t lo, uint32_t hi) {
    const uint32_t wv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    if constexpr (DT == 0) {
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (e0 + j >= lo && e0 + j < hi)
                reinterpret_cast<uint16_t *>(out)[j] = static_cast<uint16_t>(wv[j >> 1] >> (16 * (j & 1)));
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (e0 + j >= lo && e0 + j < hi) out[j] = static_cast<uint8_t>(wv[j >> 2] >> (8 * (j & 3)));
    }
}

// Merges group i of a tile: 16 plane bytes p4 with its exponents from shared
// memory (which are then cleared for the next tile) into 32 output bytes.
// [lo, hi) are the tile's elements relative to the first group's first element.
template <int DT, bool PARTIAL = true>
__device__ __forceinline__ void merge_group(uint4 p4, uint32_t i, uint8_t *s_exps, uint8_t *dst_tile, uint32_t lo,
                                            uint32_t hi, Guard &G) {
    constexpr uint32_t GROUP = DT == 0 ? 16u : 32u;
    if constexpr (!PARTIAL) {
        if (i * GROUP < lo || i * GROUP + GROUP > hi) return;  // edge group: stored by edge_groups()
    }
    if (!G.ex(s_exps + (DT == 0 ? 16u : 32u) * i, DT == 0 ? 16u : 32u)) return;
    uint4 a, b;
    if constexpr (DT == 0) {
        uint4 *xp = reinterpret_cast<uint4 *>(s_exps + 16 * i);
        const uint4 x4 = *xp;
        *xp = make_uint4(0, 0, 0, 0);
        merge_bf16x4(p4.x, x4.x, a.x, a.y);
        merge_bf16x4(p4.y, x4.y, a.z, a.w);
        merge_bf16x4(p4.z, x4.z, b.x, b.y);
        merge_bf16x4(p4.w, x4.w, b.z, b.w);
    } else {
        uint4 *xp = reinterpret_cast<uint4 *>(s_exps + 32 * i);
        const uint4 x0 = xp[0];
        const uint4 x1 = xp[1];
        xp[0] = make_uint4(0, 0, 0, 0);
        xp[1] = make_uint4(0, 0, 0, 0);
        merge_e4m3x8(p4.x, x0.x, x0.y, a.x, a.y);
        merge_e4m3x8(p4.y, x0.z, x0.w, a.z, a.w);
        merge_e4m3x8(p4.z, x1.x, x1.y, b.x, b.y);
        merge_e4m3x8(p4.w, x1.z, x1.w, b.z, b.w);
    }
    const uint32_t e0 = i * GROUP;
    uint8_t *out = dst_tile + 32u * i;
    if (!PARTIAL || (e0 >= lo && e0 + GROUP <= hi)) {
        if (G.out(out, 32)) {
            st_global_v4(out, a);
            st_global_v4(out + 16, b);
        }
    } else if (G.out_elems(out, e0, GROUP, lo, hi, DT == 0 ? 2u : 1u)) {
        store_partial<DT>(out, a, b, e0, lo, hi);
    }
}

// The first and last group of a warp tile can be shared with the neighbouring
// tile.  The whole warp stores them element by element, one element per lane
// per pass: the group's 16 plane bytes come from the lane that loaded them
// (shuffled), its exponents from shared memory, which are then cleared.
template <int DT>
__device__ __forceinline__ void edge_groups(const uint4 (&pre)[kPrefetchGroups], const uint8_t *plane, uint32_t ng,
                                            uint8_t *s_exps, uint8_t *dst_tile, uint32_t lo, uint32_t hi, int lane,
                                            Guard &G) {
    constexpr uint32_t GROUP = DT == 0 ? 16u : 32u;
    const uint32_t last = ng - 1;
    const bool head = lo != 0, tail = (hi % GROUP) != 0 && !(head && last == 0);
#pragma unroll
    for (int which = 0; which < 2; ++which) {
        const bool on = which == 0 ? head : tail;
        if (!on) continue;  // warp-uniform
        const uint32_t g = which == 0 ? 0u : last;
        // plane bytes of group g: held by lane g % 32 in pre[g / 32] when g < 32 * kPrefetchGroups
        uint4 v;
        const uint32_t u = g / 32u;
        if (u < kPrefetchGroups) {
            uint4 mine = pre[0];
#pragma unroll
            for (int k = 1; k < kPrefetchGroups; ++k)
                if (u == static_cast<uint32_t>(k)) mine = pre[k];
            const int src = static_cast<int>(g % 32u);
            v.x = __shfl_sync(0xFFFFFFFFu, mine.x, src);
            v.y = __shfl_sync(0xFFFFFFFFu, mine.y, src);
            v.z = __shfl_sync(0xFFFFFFFFu, mine.z, src);
            v.w = __shfl_sync(0xFFFFFFFFu, mine.w, src);
        } else {
            v = plane_v4(plane + 16u * g, G);
        }
#pragma unroll
        for (uint32_t j0 = 0; j0 < GROUP; j0 += 32) {
            const uint32_t j = j0 + static_cast<uint32_t>(lane);
            if (j < GROUP) {
                const uint32_t e = g * GROUP + j;
                if (!G.ex(s_exps + e, 1)) continue;
                const uint32_t x = s_exps[e];
                s_exps[e] = 0;
                if (e >= lo && e < hi && G.out(dst_tile + e * (DT == 0 ? 2u : 1u), DT == 0 ? 2u : 1u)) {
                    const uint32_t wi = DT == 0 ? (j >> 2) : (j >> 3);
                    const uint32_t word = wi == 0 ? v.x : (wi == 1 ? v.y : (wi == 2 ? v.z : v.w));
                    if constexpr (DT == 0) {
                        const uint32_t pb = (word >> (8 * (j & 3))) & 0xFFu;
                        const uint32_t val = ((pb & 0x80u) << 8) | (x << 7) | (pb & 0x7Fu);
                        reinterpret_cast<uint16_t *>(dst_tile)[e] = static_cast<uint16_t>(val);
                    } else {
                        const uint32_t nib = (word >> (4 * (j & 7))) & 0xFu;
                        dst_tile[e] = static_cast<uint8_t>(((nib & 8u) << 4) | (x << 3) | (nib & 7u));
                    }
                }
            }
        }
    }
}

// Output half-groups: half j of a tile covers output bytes [16j, 16j + 16),
// plane bytes [8j, 8j + 8) and 8 (BF16) or 16 (E4M3) exponents.  Lane L of
// store round r takes half 32r + L, so each 16-byte store instruction of the
// warp writes 512 contiguous bytes.
// The 16-byte store at a constant offset OFF from p (the offset is part of
// the instruction: one address register serves every round).
template <int OFF>
__device__ __forceinline__ void st_global_v4_at(void *p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0+%1], {%2, %3, %4, %5};" ::"l"(p), "n"(OFF), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

template <int DT>
__device__ __noinline__ void store_partial_half(uint8_t *out, uint4 a, uint32_t e0, uint32_t lo, uint32_t hi) {
    const uint32_t wv[4] = {a.x, a.y, a.z, a.w};
    if constexpr (DT == 0) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (e0 + j >= lo && e0 + j < hi)
                reinterpret_cast<uint16_t *>(out)[j] = static_cast<uint16_t>(wv[j >> 1] >> (16 * (j & 1)));
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (e0 + j >= lo && e0 + j < hi) out[j] = static_cast<uint8_t>(wv[j >> 2] >> (8 * (j & 3)));
    }
}

template <int DT, bool PARTIAL>
__device__ __forceinline__ void merge_half(uint2 p2, uint32_t j, uint8_t *s_exps, uint8_t *dst_tile, uint32_t lo,
                                           uint32_t hi, Guard &G) {
    uint4 a;
    uint32_t e0;
    if (!G.ex(s_exps + (DT == 0 ? 8u : 16u) * j, DT == 0 ? 8u : 16u)) return;
    if constexpr (DT == 0) {
        uint2 *xp = reinterpret_cast<uint2 *>(s_exps + 8 * j);
        const uint2 x2 = *xp;
        *xp = make_uint2(0, 0);
        merge_bf16x4(p2.x, x2.x, a.x, a.y);
        merge_bf16x4(p2.y, x2.y, a.z, a.w);
        e0 = 8u * j;
    } else {
        uint4 *xp = reinterpret_cast<uint4 *>(s_exps + 16 * j);
        const uint4 x4 = *xp;
        *xp = make_uint4(0, 0, 0, 0);
        merge_e4m3x8(p2.x, x4.x, x4.y, a.x, a.y);
        merge_e4m3x8(p2.y, x4.z, x4.w, a.z, a.w);
        e0 = 16u * j;
    }
    uint8_t *out = dst_tile + 16u * j;
    constexpr uint32_t HALF = DT == 0 ? 8u : 16u;
    if (!PARTIAL || (e0 >= lo && e0 + HALF <= hi)) {
        if (G.out(out, 16)) st_global_v4(out, a);
    } else if (G.out_elems(out, e0, HALF, lo, hi, DT == 0 ? 2u : 1u)) {
        store_partial_half<DT>(out, a, e0, lo, hi);
    }
}

// Round U (>= 1) of the merge for a lane: half j = lane + 32 U, whole (no
// piecewise store).  x_l and out_l are the lane's round-0 addresses in the
// exponent buffer and the tile's output.
template <int DT, int U>
__device__ __forceinline__ void merge_half_round(uint2 p2, uint8_t *x_l, uint8_t *out_l, Guard &G) {
    uint4 a;
    if (!G.ex(x_l + (DT == 0 ? 256 : 512) * U, DT == 0 ? 8u : 16u)) return;
    if constexpr (DT == 0) {
        uint2 *xp = reinterpret_cast<uint2 *>(x_l + 256 * U);
        const uint2 x2 = *xp;
        *xp = make_uint2(0, 0);
        merge_bf16x4(p2.x, x2.x, a.x, a.y);
        merge_bf16x4(p2.y, x2.y, a.z, a.w);
    } else {
        uint4 *xp = reinterpret_cast<uint4 *>(x_l + 512 * U);
        const uint4 x4 = *xp;
        *xp = make_uint4(0, 0, 0, 0);
        merge_e4m3x8(p2.x, x4.x, x4.y, a.x, a.y);
        merge_e4m3x8(p2.y, x4.z, x4.w, a.z, a.w);
    }
    if (G.out(out_l + 512 * U, 16)) st_global_v4_at<512 * U>(out_l, a);
}

template <int DT, int... U>
__device__ __forceinline__ void merge_rounds(const uint2 *pre, uint32_t lane, uint32_t nh, uint8_t *x_l, uint8_t *out_l,
                                             Guard &G, std::integer_sequence<int, U...>) {
    ((lane + 32u * (U + 1) < nh ? merge_half_round<DT, U + 1>(pre[U + 1], x_l, out_l, G) : (void)0), ...);
}


// ------------------------------------------------------------------ kernel

// DT: 0 = BF16, 1 = E4M3.  CB: stream bits per chunk.  CPT: chunks per
// decoding thread.  NTH: decoding threads per CTA; a tile has NTH * CPT chunks.
// The CTA has NTH / 32 consumer warps and one producer warp.
template <int DT, int CB, int CPT, int NTH>
__global__ void __launch_bounds__(NTH + 32, (NTH + 32) * 3 <= 1024 ? 3 : 1)
    decode_kernel(const __grid_constant__ DecodeParams P, const uint32_t max_span, const int n_lut_smem) {
    constexpr int CW = CB / 32;
    constexpr int NW = NTH / 32;
    constexpr int CHUNKS = NTH * CPT;
    constexpr uint32_t TILE_BYTES = CHUNKS * CB / 8;
    constexpr uint32_t GROUP = DT == 0 ? 16u : 32u;  // elements per 16 plane bytes
    extern __shared__ __align__(128) uint8_t smem[];
    const Plan plan = make_plan(CB, CHUNKS, max_span, n_lut_smem);

    uint64_t *full_s = reinterpret_cast<uint64_t *>(smem);  // stream + gaps landed
    uint64_t *empty_s = full_s + kStreamStages;             // stream slot free again
    StageMeta *smeta = reinterpret_cast<StageMeta *>(smem + 128);
    uint32_t *warp_tot = reinterpret_cast<uint32_t *>(smem + 384);
    uint32_t *s_meta = reinterpret_cast<uint32_t *>(smem + plan.off_meta);
    uint32_t *s_syms = reinterpret_cast<uint32_t *>(smem + plan.off_syms);
    uint16_t *s_lut = reinterpret_cast<uint16_t *>(smem + plan.off_lut);
    uint8_t *s_exps = smem + plan.off_exps;

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;

    // stage the decode tables (all warps), zero the exponent buffer,
    // initialise the pipeline barriers
    {
        const uint4 *g = reinterpret_cast<const uint4 *>(P.meta);
        uint4 *s = reinterpret_cast<uint4 *>(s_meta);
        for (int i = tid; i < kMultiEntries * 4 / 16; i += NTH + 32) {
            uint4 v = __ldg(g + i);
            v.x = sane_meta(v.x);
            v.y = sane_meta(v.y);
            v.z = sane_meta(v.z);
            v.w = sane_meta(v.w);
            s[i] = v;
        }
        g = reinterpret_cast<const uint4 *>(P.syms);
        s = reinterpret_cast<uint4 *>(s_syms);
        for (int i = tid; i < kMultiEntries * 4 / 16; i += NTH + 32) s[i] = __ldg(g + i);
        g = reinterpret_cast<const uint4 *>(P.lut);
        s = reinterpret_cast<uint4 *>(s_lut);
        for (int i = tid; i < lut_stage_count(n_lut_smem, P.n_luts) * kLutEntries * 2 / 16; i += NTH + 32)
            s[i] = __ldg(g + i);
        s = reinterpret_cast<uint4 *>(s_exps);
        for (uint32_t i = tid; i < plan.exps_bytes / 16; i += NTH + 32) s[i] = make_uint4(0, 0, 0, 0);
    }
    if (tid == 0) {
        for (int s = 0; s < kStreamStages; ++s) {
            mbar_init(&full_s[s], 1);
            mbar_init(&empty_s[s], NW);
        }
        warp_tot[NW] = 0;  // abort marker
        fence_mbar_init();
    }
    __syncthreads();
    allow_dependent_launch();

    uint8_t *const s_stream0 = smem + plan.off_stream;
    uint8_t *const s_gaps0 = smem + plan.off_gaps;
    const uint32_t stream_stride = up128(plan.stream_bytes);
    const uint32_t gaps_stride = up128(plan.gaps_bytes);

    if (warp == NW) {
        // ---------------- producer warp: one lane issues every copy
        if (lane != 0 || P.expire) return;
        uint32_t k = 0, armed = 0, last_parity = 0;
        for (uint32_t t = blockIdx.x; t < P.total_tiles; t += gridDim.x, ++k) {
            const int s = static_cast<int>(k % kStreamStages);
            const uint32_t ph = (k / kStreamStages) & 1u;
            if (!mbar_wait(&empty_s[s], ph ^ 1u, P.wait_ns)) {
                report(P.err, DF11_DEV_ERR_TIMEOUT);
                break;
            }
            int ti = 0;
            while (ti + 1 < P.n_tensors && t >= P.t[ti + 1].tile_begin) ++ti;
            const TensorDesc &d = P.t[ti];
            const uint32_t lt = t - d.tile_begin;
            uint32_t cerr = 0;
            const bool src_ok =
                in_bounds(lt, 2, static_cast<uint64_t>(d.n_tiles) + 1u, cerr) &&
                in_bounds(static_cast<uint64_t>(lt) * TILE_BYTES, plan.stream_bytes,
                          static_cast<uint64_t>(d.n_tiles) * TILE_BYTES + kStreamTail, cerr) &&
                in_bounds(static_cast<uint64_t>(lt) * CHUNKS, plan.gaps_bytes,
                          static_cast<uint64_t>(d.n_tiles) * CHUNKS + kGapsTail, cerr);
            uint64_t S = src_ok ? __ldg(d.out_off + lt) : 0u;
            const uint64_t E = src_ok ? __ldg(d.out_off + lt + 1) : 0u;
            uint32_t bad = 0;
            if (E < S || E > d.n || E - S > max_span) {
                report(P.err, DF11_DEV_ERR_AUX);
                bad = 1;
                S = 0;
            }
            if (!src_ok) {
                report(P.err, cerr);
                bad = 1;
            }
            const uint32_t span = bad ? 0u : static_cast<uint32_t>(E - S);
            StageMeta &m = smeta[s];
            m.S = S;
            m.span = span;
            m.tensor = static_cast<uint32_t>(ti);
            m.local_tile = lt;
            m.bad = bad;
            if (src_ok) {
                mbar_arrive_expect_tx(&full_s[s], plan.stream_bytes + plan.gaps_bytes);
                bulk_load(s_stream0 + s * stream_stride, d.stream + static_cast<uint64_t>(lt) * TILE_BYTES,
                          plan.stream_bytes, &full_s[s]);
                bulk_load(s_gaps0 + s * gaps_stride, d.gaps + static_cast<uint64_t>(lt) * CHUNKS, plan.gaps_bytes,
                          &full_s[s]);
            } else {
                mbar_arrive(&full_s[s]);  // nothing copied: the tile is marked bad
            }
            // the merge reads this tile's plane span from global memory: pull it into L2 now
            if (span) {
                const uint64_t a0 = (S / GROUP) * 16u, a1 = ((S + span + GROUP - 1) / GROUP) * 16u;
                Guard Gp;
                Gp.tensor<DT>(d);
                if (Gp.pl(d.plane + a0, a1 - a0)) prefetch_l2(d.plane + a0, static_cast<uint32_t>(a1 - a0));
                if (Gp.flags()) report(P.err, Gp.flags());
            }
            armed |= 1u << s;
            last_parity = (last_parity & ~(1u << s)) | (ph << s);
        }
        // keep the CTA alive until every copy it issued has landed
        for (int s = 0; s < kStreamStages; ++s)
            if (armed & (1u << s))
                if (!mbar_wait(&full_s[s], (last_parity >> s) & 1u, P.wait_ns)) report(P.err, DF11_DEV_ERR_TIMEOUT);
        return;
    }

    // ---------------- consumer warps
    const Tables T{s_meta, s_syms, s_lut, P.lut, n_lut_smem, P.n_luts, smem_addr(s_exps),
                   smem_addr(s_exps) + plan.exps_bytes};
    uint32_t err = 0;
    in_bounds(0, static_cast<uint64_t>(max(n_lut_smem, 0)), static_cast<uint64_t>(max(P.n_luts, 0)), err);
    Guard G;
    G.buffer(s_exps, P.diag_bounds ? 0u : plan.exps_bytes);
    uint32_t k = 0;
    for (uint32_t t = blockIdx.x; t < P.total_tiles; t += gridDim.x, ++k) {
        const int s = static_cast<int>(k % kStreamStages);
        const uint32_t ph = (k / kStreamStages) & 1u;
        const bool landed = mbar_wait(&full_s[s], ph, P.wait_ns);
        const StageMeta m = smeta[s];
        const int ti = landed && m.tensor < static_cast<uint32_t>(P.n_tensors) ? static_cast<int>(m.tensor) : 0;
        const TensorDesc &d = P.t[ti];
        G.tensor<DT>(d);

        // ---- the tile's plane span (16 bytes per group of GROUP elements): the
        // first kPrefetchGroups groups of this thread are loaded now, so they
        // arrive while the chunk is decoded; the merge loads any others itself
        const uint64_t g0 = m.S / GROUP;
        const uint32_t ng =
            landed && !m.bad && m.span ? static_cast<uint32_t>((m.S + m.span + GROUP - 1) / GROUP - g0) : 0u;
        const uint8_t *plane = d.plane + g0 * 16u;
        uint4 pre[kPrefetchGroups];
#pragma unroll
        for (int u = 0; u < kPrefetchGroups; ++u) {
            const uint32_t i = tid + u * NTH;
            if (i < ng) pre[u] = plane_v4(plane + 16u * i, G);
        }

        // ---- this thread's CPT consecutive chunks + one look-ahead word
        const uint8_t *sst = s_stream0 + s * stream_stride + tid * (CPT * CB / 8);
        uint32_t w[CPT * CW + 1] = {};
        const bool st_ok = in_bounds(static_cast<uint64_t>(tid) * (CPT * CB / 8), CPT * CB / 8 + 4, plan.stream_bytes, err);
        if (!st_ok) {
        } else if constexpr ((CPT * CW) % 4 == 0) {
#pragma unroll
            for (int j = 0; j < CPT * CW / 4; ++j) {
                const uint4 v = *reinterpret_cast<const uint4 *>(sst + 16 * j);
                w[4 * j + 0] = v.x;
                w[4 * j + 1] = v.y;
                w[4 * j + 2] = v.z;
                w[4 * j + 3] = v.w;
            }
        } else {
            const uint2 v = *reinterpret_cast<const uint2 *>(sst);
            w[0] = v.x;
            w[1] = v.y;
        }
        {
            const uint32_t nxt = __shfl_down_sync(0xFFFFFFFFu, w[0], 1);
            w[CPT * CW] =
                lane == 31 ? (st_ok ? *reinterpret_cast<const uint32_t *>(sst + CPT * CB / 8) : 0u) : nxt;
        }
        int gap[CPT], E[CPT];
        const uint8_t *sg = s_gaps0 + s * gaps_stride + tid * CPT;
        const bool sg_ok = in_bounds(static_cast<uint64_t>(tid) * CPT, CPT, plan.gaps_bytes, err);
        // stream bits of this tile from this thread's first chunk on (clamped)
        const int64_t rem64 = static_cast<int64_t>(d.total_bits) -
                              static_cast<int64_t>(m.local_tile) * (static_cast<int64_t>(CHUNKS) * CB) -
                              static_cast<int64_t>(tid * CPT * CB);
        const int rem = rem64 > CPT * CB ? CPT * CB : (rem64 < 0 ? 0 : static_cast<int>(rem64));
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
            const int g = sg_ok ? sg[c] : 0;
            if (g >= 32) err |= DF11_DEV_ERR_AUX;
            gap[c] = min(g, 63);
            E[c] = min(max(rem - c * CB, 0), CB);
        }

        // ---- phase 1: count
        uint32_t cnt[CPT];
        count_codes<CW, CPT>(w, gap, E, T, cnt, err);
        uint32_t mine = 0;
#pragma unroll
        for (int c = 0; c < CPT; ++c) mine += cnt[c];

        // ---- scan: warp shuffles, then the warp totals
        uint32_t incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) warp_tot[warp] = incl;
        if (!landed) warp_tot[NW] = 1;
        consumer_sync(NTH);
        if (warp_tot[NW]) {
            err |= DF11_DEV_ERR_TIMEOUT;
            break;
        }
        uint32_t prefix = 0, total = 0;
#pragma unroll
        for (int i = 0; i < NW; i += 4) {
            const uint4 v = *reinterpret_cast<const uint4 *>(warp_tot + i);
            const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4 && i + j < NW; ++j) {
                total += vv[j];
                prefix += i + j < warp ? vv[j] : 0u;
            }
        }
        const bool good = !m.bad && total == m.span;
        if (!good && !m.bad && tid == 0) err |= DF11_DEV_ERR_SPAN;

        // ---- phase 2: decode again, exponents into shared memory in output order
        if (good && m.span) {
            const uint32_t q = smem_addr(s_exps) + static_cast<uint32_t>(m.S % GROUP) + prefix + incl - mine;
            emit_codes<CW, CPT, 0>(w, gap[0], E[0], T, q, err);
            if constexpr (CPT > 1) emit_codes<CW, CPT, 1>(w, gap[1], E[1], T, q + cnt[0], err);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_s[s]);
        consumer_sync(NTH);

        // ---- merge with the raw plane (read from global/L2), 16-byte stores;
        // each group's exponents are cleared for the next tile once read
        if (good && m.span) {
            uint8_t *dst_tile = static_cast<uint8_t *>(d.dst) + g0 * 32u;
            const uint32_t lo = static_cast<uint32_t>(m.S % GROUP), hi = lo + m.span;
#pragma unroll
            for (int u = 0; u < kPrefetchGroups; ++u) {
                const uint32_t i = tid + u * NTH;
                if (i < ng) merge_group<DT>(pre[u], i, s_exps, dst_tile, lo, hi, G);
            }
            for (uint32_t i = tid + kPrefetchGroups * NTH; i < ng; i += NTH)
                merge_group<DT>(plane_v4(plane + 16u * i, G), i, s_exps, dst_tile, lo, hi, G);
        }
    }
    report(P.err, err | G.flags());
}

// ------------------------------------------------------------------ warp-tile kernel

// Shared memory of the warp-tile kernel: the decode tables once per CTA, then
// per warp two stream stages (the tile's 32 chunks + 16 look-ahead bytes,
// then its 32 gaps), two mbarriers and the warp's exponent buffer.
struct WarpPlan {
    uint32_t stage_bytes, exps_bytes, warp_bytes;
    uint32_t off_meta, off_syms, off_lut, off_warps, total;
};

__host__ __device__ inline WarpPlan make_warp_plan(int chunk_bits, int nwarp, uint32_t max_span, int n_lut_smem) {
    WarpPlan p;
    p.stage_bytes = static_cast<uint32_t>(32 * chunk_bits / 8) + 16u + 32u;  // stream + look-ahead, gaps
    p.exps_bytes = (max_span + 2u * 32u + 16u + 15u) & ~15u;
    p.warp_bytes = (16u + 2u * p.stage_bytes + p.exps_bytes + 127u) & ~127u;
    p.off_meta = 0;
    p.off_syms = p.off_meta + kMultiEntries * 4;
    p.off_lut = p.off_syms + kMultiEntries * 4;
    p.off_warps = up128(p.off_lut + static_cast<uint32_t>(n_lut_smem) * kLutEntries * 2);
    p.total = p.off_warps + static_cast<uint32_t>(nwarp) * p.warp_bytes;
    return p;
}

// Descriptor index of tile t (tiles of all tensors are numbered consecutively),
// searching forward from `from`: a warp's tiles only increase.
__device__ __forceinline__ int tensor_of(const DecodeParams &P, uint32_t t, int from = 0) {
    int ti = from;
    while (ti + 1 < P.n_tensors && t >= P.t[ti + 1].tile_begin) ++ti;
    return ti;
}

// One tile = 32 chunks = one warp.  The per-tile output offsets of the
// container (out_off) are per warp here, so a warp's tiles are decoded with a
// warp-shuffle scan only and the warps of a CTA never wait for each other:
// each warp streams its own tiles through two shared-memory stages with 1-D
// TMA bulk copies (issued by its lane 0 two tiles ahead, completing on the
// warp's own mbarriers), runs phase 1, the scan, phase 2 and the merge.  The
// decode tables are staged once per CTA.
template <int DT, int CB, int NWARP>
__global__ void __launch_bounds__(NWARP * 32, NWARP <= 8 ? 4 : 2)
    decode_warp_kernel(const __grid_constant__ DecodeParams P, const uint32_t max_span, const int n_lut_smem) {
    constexpr int CW = CB / 32;
    constexpr uint32_t TILE_BYTES = 32 * CB / 8;
    constexpr uint32_t GROUP = DT == 0 ? 16u : 32u;
    extern __shared__ __align__(128) uint8_t smem[];
    const WarpPlan plan = make_warp_plan(CB, NWARP, max_span, n_lut_smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    uint32_t *s_meta = reinterpret_cast<uint32_t *>(smem + plan.off_meta);
    uint32_t *s_syms = reinterpret_cast<uint32_t *>(smem + plan.off_syms);
    uint16_t *s_lut = reinterpret_cast<uint16_t *>(smem + plan.off_lut);
    uint8_t *wbase = smem + plan.off_warps + warp * plan.warp_bytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(wbase);  // [2]
    uint8_t *stage0 = wbase + 16;
    uint8_t *s_exps = wbase + 16 + 2 * plan.stage_bytes;

    {
        const uint4 *g = reinterpret_cast<const uint4 *>(P.meta);
        uint4 *s = reinterpret_cast<uint4 *>(s_meta);
        for (int i = tid; i < kMultiEntries * 4 / 16; i += NWARP * 32) {
            uint4 v = __ldg(g + i);
            v.x = sane_meta(v.x);
            v.y = sane_meta(v.y);
            v.z = sane_meta(v.z);
            v.w = sane_meta(v.w);
            s[i] = v;
        }
        g = reinterpret_cast<const uint4 *>(P.syms);
        s = reinterpret_cast<uint4 *>(s_syms);
        for (int i = tid; i < kMultiEntries * 4 / 16; i += NWARP * 32) s[i] = __ldg(g + i);
        g = reinterpret_cast<const uint4 *>(P.lut);
        s = reinterpret_cast<uint4 *>(s_lut);
        for (int i = tid; i < lut_stage_count(n_lut_smem, P.n_luts) * kLutEntries * 2 / 16; i += NWARP * 32)
            s[i] = __ldg(g + i);
        s = reinterpret_cast<uint4 *>(s_exps);
        for (uint32_t i = lane; i < plan.exps_bytes / 16; i += 32) s[i] = make_uint4(0, 0, 0, 0);
    }
    if (lane == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        fence_mbar_init();
    }
    __syncthreads();
    allow_dependent_launch();

    const uint32_t stride = gridDim.x * NWARP;
    const uint32_t first = blockIdx.x * NWARP + warp;
    uint32_t issued = 0;  // bit s: stage s holds a copy not yet waited for
    uint32_t par = 0;     // bit s: phase parity of that copy
    // lane 0: copy tile t's stream slice and gaps into stage s
    int ti_issue = 0, ti_cur = 0;
    auto issue = [&](uint32_t t, int s) {
        ti_issue = tensor_of(P, t, ti_issue);
        const TensorDesc &d = P.t[ti_issue];
        const uint32_t lt = t - d.tile_begin;
        uint8_t *st = stage0 + s * plan.stage_bytes;
        uint32_t cerr = 0;
        if (in_bounds(static_cast<uint64_t>(lt) * TILE_BYTES, TILE_BYTES + 16u,
                      static_cast<uint64_t>(d.n_tiles) * TILE_BYTES + kStreamTail, cerr) &&
            in_bounds(static_cast<uint64_t>(lt) * 32u, 32u, static_cast<uint64_t>(d.n_tiles) * 32u + kGapsTail, cerr)) {
            mbar_arrive_expect_tx(&full[s], TILE_BYTES + 16u + 32u);
            bulk_load(st, d.stream + static_cast<uint64_t>(lt) * TILE_BYTES, TILE_BYTES + 16u, &full[s]);
            bulk_load(st + TILE_BYTES + 16u, d.gaps + static_cast<uint64_t>(lt) * 32u, 32u, &full[s]);
        } else {
            mbar_arrive(&full[s]);  // nothing copied: the stage keeps stale bytes, the error is reported
            report(P.err, cerr);
        }
    };
    if (!P.expire) {
        if (lane == 0) {
            if (first < P.total_tiles) issue(first, 0);
            if (first + stride < P.total_tiles) issue(first + stride, 1);
        }
        if (first < P.total_tiles) issued |= 1u;
        if (first + stride < P.total_tiles) issued |= 2u;
    }

    const Tables T{s_meta, s_syms, s_lut, P.lut, n_lut_smem, P.n_luts, smem_addr(s_exps),
                   smem_addr(s_exps) + plan.exps_bytes};
    uint32_t err = 0;
    in_bounds(0, static_cast<uint64_t>(max(n_lut_smem, 0)), static_cast<uint64_t>(max(P.n_luts, 0)), err);
    Guard G;
    G.buffer(s_exps, P.diag_bounds ? 0u : plan.exps_bytes);
    uint32_t k = 0;
    for (uint32_t t = first; t < P.total_tiles; t += stride, ++k) {
        const int s = static_cast<int>(k & 1u);
        const uint32_t ph = (k >> 1) & 1u;
        ti_cur = tensor_of(P, t, ti_cur);
        const TensorDesc &d = P.t[ti_cur];
        G.tensor<DT>(d);
        const uint32_t lt = t - d.tile_begin;
        const bool oo = in_bounds(lt, 2, static_cast<uint64_t>(d.n_tiles) + 1u, err);
        uint64_t S = oo ? __ldg(d.out_off + lt) : 1u;
        const uint64_t Eo = oo ? __ldg(d.out_off + lt + 1) : 0u;
        const bool bad = Eo < S || Eo > d.n || Eo - S > max_span;
        if (bad) S = 0;
        const uint32_t span = bad ? 0u : static_cast<uint32_t>(Eo - S);

        // the tile's plane span: the first kPrefetchGroups groups of each lane now
        const uint64_t g0 = S / GROUP;
        const uint32_t ng = span ? static_cast<uint32_t>((S + span + GROUP - 1) / GROUP - g0) : 0u;
        const uint8_t *plane = d.plane + g0 * 16u;
        uint4 pre[kPrefetchGroups];
#pragma unroll
        for (int u = 0; u < kPrefetchGroups; ++u) {
            const uint32_t i = lane + 32u * u;
            if (i < ng) pre[u] = plane_v4(plane + 16u * i, G);
        }

        const bool landed = __all_sync(0xFFFFFFFFu, mbar_wait(&full[s], ph, P.wait_ns));
        if (!landed) {
            err |= DF11_DEV_ERR_TIMEOUT;
            break;
        }
        issued &= ~(1u << s);
        // every stage read below stays inside the stage: 32 chunks, the look-ahead word, 32 gaps
        in_bounds(TILE_BYTES + 16u, 32u, plan.stage_bytes, err);
        const uint8_t *st = stage0 + s * plan.stage_bytes;
        uint32_t w[CW + 1];
        if constexpr (CW % 4 == 0) {
#pragma unroll
            for (int j = 0; j < CW / 4; ++j) {
                const uint4 v = *reinterpret_cast<const uint4 *>(st + lane * (CB / 8) + 16 * j);
                w[4 * j + 0] = v.x;
                w[4 * j + 1] = v.y;
                w[4 * j + 2] = v.z;
                w[4 * j + 3] = v.w;
            }
        } else {
            const uint2 v = *reinterpret_cast<const uint2 *>(st + lane * (CB / 8));
            w[0] = v.x;
            w[1] = v.y;
        }
        {
            const uint32_t nxt = __shfl_down_sync(0xFFFFFFFFu, w[0], 1);
            w[CW] = lane == 31 ? *reinterpret_cast<const uint32_t *>(st + TILE_BYTES) : nxt;
        }
        int gap[1], E[1];
        {
            const int g = st[TILE_BYTES + 16u + lane];
            if (g >= 32) err |= DF11_DEV_ERR_AUX;
            gap[0] = min(g, 63);
            const int64_t rem64 = static_cast<int64_t>(d.total_bits) -
                                  static_cast<int64_t>(lt) * (32 * CB) - static_cast<int64_t>(lane * CB);
            E[0] = rem64 >= CB ? CB : (rem64 <= 0 ? 0 : static_cast<int>(rem64));
        }
        // the stage's words are in registers: refill it with tile t + 2 * stride
        __syncwarp();
        if (t + 2 * stride < P.total_tiles) {
            if (lane == 0) {
                fence_proxy_async_smem();
                issue(t + 2 * stride, s);
            }
            issued |= 1u << s;
            par = (par & ~(1u << s)) | ((((k + 2) >> 1) & 1u) << s);
        }

        // ---- phase 1, warp scan
        uint32_t cnt[1];
        count_codes<CW, 1>(w, gap, E, T, cnt, err);
        uint32_t incl = cnt[0];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += v;
        }
        const uint32_t total = __shfl_sync(0xFFFFFFFFu, incl, 31);
        const bool good = !bad && total == span;
        if (bad) err |= DF11_DEV_ERR_AUX;
        else if (!good) err |= DF11_DEV_ERR_SPAN;

        // ---- phase 2, then the merge
        if (good && span) {
            emit_codes<CW, 1, 0>(w, gap[0], E[0], T, smem_addr(s_exps) + static_cast<uint32_t>(S % GROUP) + incl - cnt[0],
                                 err);
            __syncwarp();
            uint8_t *dst_tile = static_cast<uint8_t *>(d.dst) + g0 * 32u;
            const uint32_t lo = static_cast<uint32_t>(S % GROUP), hi = lo + span;
#pragma unroll
            for (int u = 0; u < kPrefetchGroups; ++u) {
                const uint32_t i = lane + 32u * u;
                if (i < ng) merge_group<DT, false>(pre[u], i, s_exps, dst_tile, lo, hi, G);
            }
            for (uint32_t i = lane + 32u * kPrefetchGroups; i < ng; i += 32)
                merge_group<DT, false>(plane_v4(plane + 16u * i, G), i, s_exps, dst_tile, lo, hi, G);
            edge_groups<DT>(pre, plane, ng, s_exps, dst_tile, lo, hi, lane, G);
            __syncwarp();
        }
    }
    err |= G.flags();
    // after an abort: wait (bounded) for copies that were issued but never consumed
    for (int s = 0; s < 2; ++s)
        if (issued & (1u << s))
            if (!mbar_wait(&full[s], (par >> s) & 1u, P.wait_ns)) err |= DF11_DEV_ERR_TIMEOUT;
    err = __reduce_or_sync(0xFFFFFFFFu, err);
    if (lane == 0) report(P.err, err);
}

// Shared memory of the byte-step kernel: the transition table (fsm_rows rows
// of kFsmRowBytes) at offset 0, its control words alone (rows of 1 KB: end
// mask, row << 10, count << 24; only when the kernel counts with a walk),
// the root hierarchical table, then per warp its mbarrier, one stage (the
// tile's 32 chunks + 16 look-ahead bytes, then 48 gap bytes: its own 32 and
// the next tile's first 16, then with stored counts the tile's 32 chunk
// counts) and its exponent buffer.
struct FsmPlan {
    uint32_t stage_bytes, exps_bytes, warp_bytes, off_ctl, off_lut, off_warps, total;
};

__host__ __device__ inline FsmPlan make_fsm_plan(int chunk_bits, int nwarp, uint32_t max_span, int fsm_rows,
                                                 bool counts) {
    FsmPlan p;
    p.stage_bytes = static_cast<uint32_t>(32 * chunk_bits / 8) + 16u + 48u + (counts ? 32u : 0u);
    // the tile's span after its offset in the first group (< 32), plus room for
    // the last group's rounding; with stored counts, plus what one thread's
    // walk can write past the range its stored count gives it (4 symbols a
    // step, chunk_bits / 8 + 4 steps at most, and the word it ends in) when
    // the stream disagrees with the count
    const uint32_t slack = counts ? 32u + 4u * static_cast<uint32_t>(chunk_bits / 8 + 6) : 2u * 32u + 16u;
    p.exps_bytes = (max_span + slack + 15u) & ~15u;
    p.warp_bytes = (16u + p.stage_bytes + p.exps_bytes + 127u) & ~127u;
    p.off_ctl = static_cast<uint32_t>(fsm_rows) * kFsmRowBytes;
    p.off_lut = p.off_ctl + (counts ? 0u : static_cast<uint32_t>(fsm_rows) * (kFsmRowBytes / 2));
    p.off_warps = up128(p.off_lut + kLutEntries * 2);
    p.total = p.off_warps + static_cast<uint32_t>(nwarp) * p.warp_bytes;
    return p;
}

// Warp tiles (32 chunks) decoded with the byte-step walk, one CTA of NWARP
// warps per SM sharing the transition table.  Each warp decodes a contiguous
// run of tiles, streaming them through one shared-memory stage (lane 0
// refills it with the next tile as soon as the current one is in registers,
// so the copy has a whole tile's decode to land), and runs phase 1, the warp
// scan, phase 2 and the merge per tile.  Threads whose walk reaches the dead
// row, or whose range is cut short by the end of the stream, take the window
// walk instead (12-bit table read from global memory through L1).
//
// A tile's last output group usually continues in the next tile.  Its
// exponents stay at the start of the buffer ("carried") and the next tile of
// the run, which decodes the rest of the group right after them, merges it
// as a whole group; a group is stored piecewise only where a run or a tensor
// begins or ends.
//
// CNT: the images store chunk counts, copied with the tile, and the scan of
// those bytes places each thread's output: no count walk (phase 1).  Each
// thread's walk is then checked against its stored count; a walk that ends a
// different number of codes flags DF11_DEV_ERR_SPAN, its tile's exponent
// buffer is cleared afterwards, and the carried group is dropped.
template <int DT, int CB, int NWARP, bool CNT>
__global__ void __launch_bounds__(NWARP * 32, 1)
    decode_fsm_kernel(const __grid_constant__ DecodeParams P, const uint32_t max_span, const int) {
    constexpr int CW = CB / 32;
    constexpr int NFIX = kFixedSteps<CB>;
    constexpr uint32_t TILE_BYTES = 32 * CB / 8;
    constexpr uint32_t GROUP = DT == 0 ? 16u : 32u;
    constexpr uint32_t STAGE_TX = TILE_BYTES + 16u + 48u + (CNT ? 32u : 0u);
    static_assert(!CNT || CB <= kCountsMaxChunkBits, "chunk counts need chunks of at most 128 bits");
    extern __shared__ __align__(128) uint8_t smem[];
    const int rows = P.fsm_rows;
    const FsmPlan plan = make_fsm_plan(CB, NWARP, max_span, rows, CNT);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint16_t *s_lut = reinterpret_cast<uint16_t *>(smem + plan.off_lut);
    uint8_t *wbase = smem + plan.off_warps + warp * plan.warp_bytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(wbase);
    uint8_t *stage = wbase + 16;
    uint8_t *s_exps = wbase + 16 + plan.stage_bytes;
    const uint32_t dead = static_cast<uint32_t>(rows - 1) << kFsmRowShift;

    {
        // the transition table and its control words; a row index past the
        // last row (damaged tables) is redirected to the dead row so every
        // lookup stays inside
        const uint4 *g = reinterpret_cast<const uint4 *>(P.fsm);
        uint4 *s = reinterpret_cast<uint4 *>(smem);
        uint2 *sc = reinterpret_cast<uint2 *>(smem + plan.off_ctl);
        const uint32_t lim = static_cast<uint32_t>(rows) << kFsmRowShift;
        for (int i = tid; i < rows * kFsmRowBytes / 16; i += NWARP * 32) {
            uint4 v = __ldg(g + i);
            if ((v.x & kFsmRowMask) >= lim) v.x = (v.x & ~kFsmRowMask) | dead;
            if ((v.z & kFsmRowMask) >= lim) v.z = (v.z & ~kFsmRowMask) | dead;
            s[i] = v;
            if constexpr (!CNT)
                sc[i] = make_uint2((v.x & 0xFFu) | ((v.x & kFsmRowMask) >> 1) | ((v.x >> kFsmCountShift) << 24),
                                   (v.z & 0xFFu) | ((v.z & kFsmRowMask) >> 1) | ((v.z >> kFsmCountShift) << 24));
        }
        const uint4 *gl = reinterpret_cast<const uint4 *>(P.lut);
        uint4 *sl = reinterpret_cast<uint4 *>(s_lut);
        for (int i = tid; i < kLutEntries * 2 / 16; i += NWARP * 32) sl[i] = __ldg(gl + i);
        uint4 *se = reinterpret_cast<uint4 *>(s_exps);
        for (uint32_t i = lane; i < plan.exps_bytes / 16; i += 32) se[i] = make_uint4(0, 0, 0, 0);
    }
    if (lane == 0) {
        mbar_init(&full[0], 1);
        fence_mbar_init();
    }
    __syncthreads();
    allow_dependent_launch();

    // this warp's run of tiles
    const uint32_t nwt = gridDim.x * NWARP;
    const uint32_t per = (P.total_tiles + nwt - 1) / nwt;
    const uint32_t t_begin = min((blockIdx.x * NWARP + warp) * per, P.total_tiles);
    const uint32_t t_end = min(t_begin + per, P.total_tiles);
    int ti_issue = tensor_of(P, t_begin), ti_cur = ti_issue;
    // the first tile of the tensor after ti: a warp's run stays in one tensor
    // for most tiles, so the descriptor search runs only when it crosses one
    auto next_begin = [&](int ti) -> uint32_t { return ti + 1 < P.n_tensors ? P.t[ti + 1].tile_begin : 0xFFFFFFFFu; };
    uint32_t nb_issue = next_begin(ti_issue), nb_cur = nb_issue;
    // lane 0: copy tile t's stream slice and gaps into the stage
    auto issue = [&](uint32_t t) {
        if (t >= nb_issue) {
            ti_issue = tensor_of(P, t, ti_issue);
            nb_issue = next_begin(ti_issue);
        }
        const TensorDesc &d = P.t[ti_issue];
        const uint32_t lt = t - d.tile_begin;
        uint32_t cerr = 0;
        if (in_bounds(static_cast<uint64_t>(lt) * TILE_BYTES, TILE_BYTES + 16u,
                      static_cast<uint64_t>(d.n_tiles) * TILE_BYTES + kStreamTail, cerr) &&
            in_bounds(static_cast<uint64_t>(lt) * 32u, 48u, static_cast<uint64_t>(d.n_tiles) * 32u + kGapsTail, cerr) &&
            (!CNT || in_bounds(static_cast<uint64_t>(lt) * 32u, 32u, static_cast<uint64_t>(d.n_tiles) * 32u, cerr))) {
            mbar_arrive_expect_tx(&full[0], STAGE_TX);
            bulk_load(stage, d.stream + static_cast<uint64_t>(lt) * TILE_BYTES, TILE_BYTES + 16u, &full[0]);
            bulk_load(stage + TILE_BYTES + 16u, d.gaps + static_cast<uint64_t>(lt) * 32u, 48u, &full[0]);
            if constexpr (CNT)
                bulk_load(stage + TILE_BYTES + 64u, d.counts + static_cast<uint64_t>(lt) * 32u, 32u, &full[0]);
        } else {
            mbar_arrive(&full[0]);  // nothing copied: the stage keeps stale bytes, the error is reported
            report(P.err, cerr);
        }
    };
    if (lane == 0 && t_begin < t_end && !P.expire) issue(t_begin);
    bool pending = t_begin < t_end && !P.expire;

    // the window walk of the fallback: 12-bit table in global memory, root
    // hierarchical table in shared memory
    const Tables T{P.meta, P.syms, s_lut, P.lut, 1, P.n_luts, smem_addr(s_exps), smem_addr(s_exps) + plan.exps_bytes};
    uint32_t err = 0;
    // every stage read stays inside the stage: 32 chunks, the look-ahead
    // words, 48 gaps, with stored counts 32 counts
    in_bounds(0, STAGE_TX, plan.stage_bytes, err);
    Guard G;
    G.buffer(s_exps, P.diag_bounds ? 0u : plan.exps_bytes);
    const uint32_t exps_lo = smem_addr(s_exps), exps_hi = exps_lo + plan.exps_bytes;
    const uint32_t ctl_bytes = static_cast<uint32_t>(rows) * (kFsmRowBytes / 2);
    const uint32_t fsm_bytes = static_cast<uint32_t>(rows) * kFsmRowBytes;
    uint32_t k = 0;
    // carried group: exponents of its elements [0, carry_n) at the buffer start
    uint32_t carry_n = 0;
    uint64_t carry_g = 0;
    int carry_ti = 0;
    // stores the carried elements alone (lane 0) and clears their exponents
    auto flush_carry = [&]() {
        if (lane == 0) {
            const TensorDesc &dc = P.t[carry_ti];
            Guard Gc = G;
            Gc.tensor<DT>(dc);
            merge_group<DT, true>(plane_v4(dc.plane + carry_g * 16u, Gc), 0u, s_exps,
                                  static_cast<uint8_t *>(dc.dst) + carry_g * 32u, 0u, carry_n, Gc);
            err |= Gc.flags();
        }
        carry_n = 0;
        __syncwarp();
    };

    for (uint32_t t = t_begin; t < t_end; ++t, ++k) {
        if (t >= nb_cur) {
            ti_cur = tensor_of(P, t, ti_cur);
            nb_cur = next_begin(ti_cur);
        }
        const TensorDesc &d = P.t[ti_cur];
        G.tensor<DT>(d);
        const uint32_t lt = t - d.tile_begin;
        const bool oo = in_bounds(lt, 2, static_cast<uint64_t>(d.n_tiles) + 1u, err);
        uint64_t S = oo ? __ldg(d.out_off + lt) : 1u;
        const uint64_t Eo = oo ? __ldg(d.out_off + lt + 1) : 0u;
        const bool bad = Eo - S > max_span || Eo > d.n;  // Eo < S wraps above max_span
        if (bad) S = 0;
        const uint32_t span = bad ? 0u : static_cast<uint32_t>(Eo - S);
        const uint64_t g0 = S / GROUP;
        const uint32_t s0 = static_cast<uint32_t>(S % GROUP);
        const uint32_t ng = span ? static_cast<uint32_t>((S + span + GROUP - 1) / GROUP - g0) : 0u;
        // the carried group goes on in this tile only if the tile starts right after it
        if (carry_n && !(span && ti_cur == carry_ti && g0 == carry_g && s0 == carry_n)) flush_carry();
        const bool joined = carry_n != 0;

        // the tile's plane span: the first kPrefetchGroups groups of each lane now
        const uint8_t *plane = d.plane + g0 * 16u;
        uint2 pre[2 * kPrefetchGroups];
        prefetch_halves(pre, plane + 8u * lane, lane, 2 * ng, G, std::make_integer_sequence<int, 2 * kPrefetchGroups>{});

        const bool landed = __all_sync(0xFFFFFFFFu, mbar_wait(&full[0], k & 1u, P.wait_ns));
        if (!landed) {
            err |= DF11_DEV_ERR_TIMEOUT;
            break;
        }
        pending = false;
        uint32_t w[CW + 1], w2;
        if constexpr (CW % 4 == 0) {
#pragma unroll
            for (int j = 0; j < CW / 4; ++j) {
                const uint4 v = *reinterpret_cast<const uint4 *>(stage + lane * (CB / 8) + 16 * j);
                w[4 * j + 0] = v.x;
                w[4 * j + 1] = v.y;
                w[4 * j + 2] = v.z;
                w[4 * j + 3] = v.w;
            }
        } else {
            const uint2 v = *reinterpret_cast<const uint2 *>(stage + lane * (CB / 8));
            w[0] = v.x;
            w[1] = v.y;
        }
        {
            const uint32_t n0 = __shfl_down_sync(0xFFFFFFFFu, w[0], 1);
            const uint32_t n1 = __shfl_down_sync(0xFFFFFFFFu, w[1], 1);
            const uint32_t *la = reinterpret_cast<const uint32_t *>(stage + TILE_BYTES);
            w[CW] = lane == 31 ? la[0] : n0;
            w2 = lane == 31 ? la[1] : n1;
        }
        const int graw = stage[TILE_BYTES + 16u + lane];
        const int gnext = stage[TILE_BYTES + 16u + lane + 1];
        uint32_t cnt = CNT ? static_cast<uint32_t>(stage[TILE_BYTES + 64u + lane]) : 0u;
        // the stage is in registers: refill it with the run's next tile
        __syncwarp();
        if (t + 1 < t_end) {
            if (lane == 0) {
                fence_proxy_async_smem();
                issue(t + 1);
            }
            pending = true;
        }

        // ---- this thread's range of codes
        // stream bits from this thread's chunk on: the tile's remainder (64-bit,
        // warp-uniform) clamped to [-1, 32 CB + 256], then 32-bit per thread
        // (no range reaches past CB + 255 bits of its chunk).  Only a tensor's
        // last tile can hold fewer: every other tile is followed by one whose
        // first gap is at most the bits left after this tile, so its lanes'
        // ranges come out the same with the clamp's upper value
        int rem0 = 32 * CB + 256;
        if (lt + 1u >= d.n_tiles) {
            const int64_t trem = static_cast<int64_t>(d.total_bits) - static_cast<int64_t>(lt) * (32 * CB);
            rem0 = static_cast<int>(max(min(trem, static_cast<int64_t>(32 * CB + 256)), static_cast<int64_t>(-1)));
        }
        const int rem = rem0 - lane * CB;
        const int E = min(max(rem, 0), CB);
        if (graw >= 32) err |= DF11_DEV_ERR_AUX;
        const int g = min(graw, 63);
        const int nbits = max(min(rem, CB + gnext) - g, -1);
        const bool whole = graw < 32 && gnext < 32 && nbits >= 8 * NFIX;
        const int nfull = nbits >> 3, r = nbits & 7;
        const int jmax = static_cast<int>(__reduce_max_sync(0xFFFFFFFFu, whole ? nfull + (r != 0) : 0));

        // ---- the thread's number of codes: stored, or counted by phase 1
        // (threads without a whole range count with the window walk; with
        // stored counts that count checks the stored one)
        bool slow, mism = false;
        if constexpr (CNT) {
            slow = !whole;
        } else {
            uint32_t ctl;
            const uint32_t dead_c = dead >> 1;
            cnt = byte_step_count<CB>(w, w2, g & 31, nfull, r, jmax, smem + plan.off_ctl, dead_c, ctl, ctl_bytes, err);
            slow = !whole || (ctl & kCtlRowMask) == dead_c;
        }
        if (__any_sync(0xFFFFFFFFu, slow)) {
            if (slow) {
                const int gg[1] = {g}, ee[1] = {E};
                uint32_t c1[1];
                count_codes<CW, 1, true>(w, gg, ee, T, c1, err);
                if (CNT) mism = c1[0] != cnt;
                else cnt = c1[0];
            }
        }
        uint32_t incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += v;
        }
        const uint32_t total = __shfl_sync(0xFFFFFFFFu, incl, 31);
        const bool good = !bad && total == span;
        if (bad) err |= DF11_DEV_ERR_AUX;
        else if (!good) err |= DF11_DEV_ERR_SPAN;

        // ---- phase 2, then the merge
        if (good && span) {
            const uint32_t qrel = s0 + incl - cnt;
            const uint32_t q = smem_addr(s_exps) + qrel;
            // the word a range starts in may hold carried exponents: start from it
            const uint32_t acc0 =
                joined && G.ex(s_exps + (qrel & ~3u), 4) ? *reinterpret_cast<const uint32_t *>(s_exps + (qrel & ~3u)) : 0u;
            __syncwarp();
            uint32_t acc = 0, wp = 0, f8 = 0, last = 0;
            if (!slow)
                byte_step_emit<CB>(w, w2, g, nfull, r, jmax, smem, q, acc0, dead, acc, wp, f8, last, fsm_bytes, exps_lo,
                                   exps_hi, err);
            // with stored counts: a walk that left the tables is redone with the
            // window walk below; a whole walk must end the stored number of codes
            // (8 bits of f8 per code: wp * 8 + f8 advanced by 8 per symbol from q * 8)
            bool redo = false;
            if constexpr (CNT) {
                redo = !slow && (last & kFsmRowMask) == dead;
                if (!slow && !redo && (wp - q) * 8u + f8 != 8u * cnt) mism = true;
            }
            __syncwarp();  // every plain store of phase 2 before the OR-ed words
            if (!slow && !redo && f8 && in_bounds(wp - exps_lo, 4, exps_hi - exps_lo, err))
                asm volatile("red.shared.or.b32 [%0], %1;" ::"r"(wp), "r"(acc) : "memory");
            if constexpr (CNT) {
                if (__any_sync(0xFFFFFFFFu, redo)) {
                    if (redo) {
                        const int gg[1] = {g}, ee[1] = {E};
                        uint32_t c1[1];
                        count_codes<CW, 1, true>(w, gg, ee, T, c1, err);
                        if (c1[0] != cnt) mism = true;
                    }
                }
                slow = (slow || redo) && !mism;  // a thread whose count disagrees writes nothing more
            }
            if (__any_sync(0xFFFFFFFFu, slow)) {
                if (slow) emit_codes<CW, 1, 0, true>(w, g, E, T, q, err);
            }
            __syncwarp();
            // groups [0, nmerge): group 0 is whole when it continues the carry
            // or starts on a group boundary; an unfinished last group becomes
            // the next carry (unless it is also the unfinished first group,
            // the one group that may be stored piecewise)
            uint8_t *dst_tile = static_cast<uint8_t *>(d.dst) + g0 * 32u;
            const uint32_t lo = joined ? 0u : s0, hi = s0 + span;
            const bool keep = (hi % GROUP) != 0 && !(ng == 1 && lo != 0);
            const uint32_t nmerge = keep ? ng - 1 : ng;
            const uint32_t nh = 2u * nmerge;
            if (static_cast<uint32_t>(lane) < nh) merge_half<DT, true>(pre[0], lane, s_exps, dst_tile, lo, hi, G);
            merge_rounds<DT>(pre, lane, nh, s_exps + (DT == 0 ? 8u : 16u) * lane, dst_tile + 16u * lane, G,
                             std::make_integer_sequence<int, 2 * kPrefetchGroups - 1>{});
            for (uint32_t j = lane + 64u * kPrefetchGroups; j < nh; j += 32)
                merge_half<DT, false>(plane_v2(plane + 8u * j, G), j, s_exps, dst_tile, lo, hi, G);
            __syncwarp();
            if (keep) {
                if (ng > 1 && lane < static_cast<int>(GROUP / 16u)) {  // move the group's exponents to the start
                    uint4 *src = reinterpret_cast<uint4 *>(s_exps + GROUP * (ng - 1)) + lane;
                    if (G.ex(src, 16) && G.ex(s_exps + 16 * lane, 16)) {
                        reinterpret_cast<uint4 *>(s_exps)[lane] = *src;
                        *src = make_uint4(0, 0, 0, 0);
                    }
                }
                carry_n = hi % GROUP;
                carry_g = g0 + ng - 1;
                carry_ti = ti_cur;
                __syncwarp();
            } else {
                carry_n = 0;  // a carried group was merged above
            }
            if (CNT && __any_sync(0xFFFFFFFFu, mism)) {
                // a walk wrote past its stored range: clear the whole buffer
                // (the tile's output is flagged) and drop the carried group
                uint4 *se = reinterpret_cast<uint4 *>(s_exps);
                for (uint32_t i = lane; i < plan.exps_bytes / 16; i += 32) se[i] = make_uint4(0, 0, 0, 0);
                carry_n = 0;
                __syncwarp();
            }
        }
        if (mism) err |= DF11_DEV_ERR_SPAN;
    }
    if (carry_n) flush_carry();
    // after an abort: wait (bounded) for a copy that was issued but never consumed
    if (pending)
        if (!mbar_wait(&full[0], k & 1u, P.wait_ns)) err |= DF11_DEV_ERR_TIMEOUT;
    err = __reduce_or_sync(0xFFFFFFFFu, err | G.flags());
    if (lane == 0) report(P.err, err);
}

// ------------------------------------------------------------------ host side

using KernelFn = void (*)(DecodeParams, uint32_t, int);

// chunks = chunks per tile (the container's tile_threads).  chunks == 32: a
// warp-tile kernel with nwarp warps per CTA, walking with the 12-bit window
// (walker DF11_WALKER_WINDOW) or the byte-step tables (DF11_WALKER_BYTE_STEP);
// otherwise the CTA-tile kernel with chunks / cpt decoding threads and a
// producer warp.  counts: the byte-step kernel that reads stored chunk
// counts instead of counting with a walk.
struct KernelEntry {
    int dtype, chunk_bits, chunks, cpt, nwarp, walker, counts;
    KernelFn fn;
};

#define DF11_KERNEL(DT, CB, CH)                                             \
    {DT, CB, CH, 1, 0, DF11_WALKER_WINDOW, 0, &decode_kernel<DT, CB, 1, CH>}, \
    {                                                                       \
        DT, CB, CH, 2, 0, DF11_WALKER_WINDOW, 0, &decode_kernel<DT, CB, 2, CH / 2> \
    }
#define DF11_WARP_KERNEL(DT, CB)                                                      \
    {DT, CB, 32, 1, 8, DF11_WALKER_WINDOW, 0, &decode_warp_kernel<DT, CB, 8>},         \
        {DT, CB, 32, 1, 16, DF11_WALKER_WINDOW, 0, &decode_warp_kernel<DT, CB, 16>},   \
        {DT, CB, 32, 1, 16, DF11_WALKER_BYTE_STEP, 0, &decode_fsm_kernel<DT, CB, 16, false>}, \
        {DT, CB, 32, 1, 24, DF11_WALKER_BYTE_STEP, 0, &decode_fsm_kernel<DT, CB, 24, false>}, \
    {                                                                                 \
        DT, CB, 32, 1, 32, DF11_WALKER_BYTE_STEP, 0, &decode_fsm_kernel<DT, CB, 32, false>  \
    }
#define DF11_COUNTS_KERNEL(DT, CB)                                                   \
    {DT, CB, 32, 1, 16, DF11_WALKER_BYTE_STEP, 1, &decode_fsm_kernel<DT, CB, 16, true>}, \
        {DT, CB, 32, 1, 24, DF11_WALKER_BYTE_STEP, 1, &decode_fsm_kernel<DT, CB, 24, true>}, \
    {                                                                                \
        DT, CB, 32, 1, 32, DF11_WALKER_BYTE_STEP, 1, &decode_fsm_kernel<DT, CB, 32, true>  \
    }

const KernelEntry kKernels[] = {
    DF11_COUNTS_KERNEL(0, 128), DF11_COUNTS_KERNEL(1, 128), DF11_COUNTS_KERNEL(0, 64), DF11_COUNTS_KERNEL(1, 64),
    DF11_WARP_KERNEL(0, 128), DF11_WARP_KERNEL(1, 128), DF11_WARP_KERNEL(0, 256), DF11_WARP_KERNEL(1, 256),
    DF11_WARP_KERNEL(0, 64),  DF11_WARP_KERNEL(1, 64),
    DF11_KERNEL(0, 128, 256), DF11_KERNEL(1, 128, 256), DF11_KERNEL(0, 256, 128), DF11_KERNEL(1, 256, 128),
    DF11_KERNEL(0, 64, 512),  DF11_KERNEL(1, 64, 512),  DF11_KERNEL(0, 128, 128), DF11_KERNEL(1, 128, 128),
    DF11_KERNEL(0, 128, 512), DF11_KERNEL(1, 128, 512), DF11_KERNEL(0, 256, 256), DF11_KERNEL(1, 256, 256),
};

const KernelEntry *find_kernel(int dtype, int chunk_bits, int chunks, int cpt, int nwarp, int walker,
                               int counts = 0) {
    for (const auto &e : kKernels)
        if (e.dtype == dtype && e.chunk_bits == chunk_bits && e.chunks == chunks && e.cpt == cpt &&
            e.nwarp == nwarp && e.walker == walker && e.counts == counts)
            return &e;
    return nullptr;
}

std::mutex g_attr_mu;
constexpr int kMaxDevices = 64;
bool g_attr_set[kMaxDevices][sizeof(kKernels) / sizeof(kKernels[0])] = {};
int g_sm_count[kMaxDevices] = {};
int g_smem_optin[kMaxDevices] = {};

// Per-device one-time set-up: opt the kernel in to large dynamic shared
// memory and read the SM count.
bool prepare(const KernelEntry *ke, int dev) {
    if (dev < 0 || dev >= kMaxDevices) return false;
    const size_t idx = static_cast<size_t>(ke - kKernels);
    std::lock_guard<std::mutex> lk(g_attr_mu);
    if (!g_sm_count[dev]) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
        g_sm_count[dev] = v;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return false;
        g_smem_optin[dev] = v;
    }
    if (!g_attr_set[dev][idx]) {
        if (cudaFuncSetAttribute(reinterpret_cast<const void *>(ke->fn), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 g_smem_optin[dev]) != cudaSuccess)
            return false;
        g_attr_set[dev][idx] = true;
    }
    return true;
}

struct Prepared {
    DecodeParams params;
    const KernelEntry *ke = nullptr;
    uint32_t max_span = 0;
    int n_lut_smem = 0;
    int ctas_per_sm = 0;
    int max_ctas = 0;
    uint32_t smem = 0;
};

LaunchStatus build_params(const Blob *const *blobs, void *const *dst, int n, int *err, const DecodeOptions &opt,
                          Prepared *out) {
    if (n < 1 || n > kMaxTensorsPerLaunch || !blobs[0]) return LaunchStatus::kInvalid;
    const Blob &b0 = *blobs[0];
    const bool warp_tiles = b0.tile_threads == 32;
    const int cpt = opt.chunks_per_thread ? opt.chunks_per_thread : kDefaultChunksPerThread;
    if (cpt != 1 && cpt != 2) return LaunchStatus::kInvalid;
    if (warp_tiles && cpt != 1) return LaunchStatus::kInvalid;
    if (opt.walker < DF11_WALKER_AUTO || opt.walker > DF11_WALKER_BYTE_STEP) return LaunchStatus::kInvalid;
    if (!warp_tiles && opt.walker == DF11_WALKER_BYTE_STEP) return LaunchStatus::kUnsupported;
    DecodeParams &P = out->params;
    P = DecodeParams{};
    uint64_t tiles = 0, max_span = 0;
    int nt = 0;
    bool all_counts = true;  // every non-empty image of the launch stores chunk counts
    for (int i = 0; i < n; ++i) {
        if (!blobs[i]) return LaunchStatus::kInvalid;
        const Blob &b = *blobs[i];
        if (!b.dev_image || b.dtype != b0.dtype || b.chunk_bits != b0.chunk_bits ||
            b.tile_threads != b0.tile_threads)
            return LaunchStatus::kInvalid;
        for (int s = 0; s < 256; ++s)
            if (b.cb->lengths[s] != b0.cb->lengths[s]) return LaunchStatus::kInvalid;
        if (b.dev_cap < image_layout(b).total) return LaunchStatus::kInvalid;
        if (!b.n) continue;
        if (!dst || !dst[i] || reinterpret_cast<uintptr_t>(dst[i]) % 16) return LaunchStatus::kInvalid;
        const ImageLayout L = image_layout(b);
        TensorDesc &d = P.t[nt++];
        d.stream = b.dev_image + L.stream;
        d.plane = b.dev_image + L.plane;
        d.gaps = b.dev_image + L.gaps;
        d.counts = b.chunk_counts ? b.dev_image + L.counts : nullptr;
        all_counts = all_counts && b.chunk_counts;
        d.out_off = reinterpret_cast<const uint64_t *>(b.dev_image + L.out_off);
        d.dst = dst[i];
        d.n = b.n;
        d.total_bits = b.total_bits;
        d.n_tiles = static_cast<uint32_t>(b.n_tiles);
        d.tile_begin = static_cast<uint32_t>(tiles);
        tiles += b.n_tiles;
        if (b.max_span > max_span) max_span = b.max_span;
    }
    if (tiles >= (uint64_t{1} << 31)) return LaunchStatus::kInvalid;
    // kernel: the byte-step walk for warp tiles unless the window walk is asked
    // for, the code has a 1-bit codeword (a byte would end up to 8 codes) or
    // its tables and the warps' buffers do not fit in shared memory; it reads
    // the stored chunk counts when every image has them and no count walk is
    // asked for
    const int rows = b0.cb->fsm_rows;
    const int use_counts = all_counts && nt > 0 && !opt.count_walk && counts_fit(b0.chunk_bits) ? 1 : 0;
    const KernelEntry *ke = nullptr;
    if (warp_tiles && opt.walker != DF11_WALKER_WINDOW && rows >= 2 && rows <= kFsmMaxRows &&
        (opt.walker == DF11_WALKER_BYTE_STEP || b0.cb->min_len_used >= 2)) {
        const int tries[3] = {32, 24, 16};
        for (int nw : tries) {
            if (opt.warps_per_cta && opt.warps_per_cta != nw) continue;
            if (make_fsm_plan(b0.chunk_bits, nw, static_cast<uint32_t>(max_span), rows, use_counts).total >
                kSmemBudget)
                continue;
            ke = find_kernel(b0.dtype, b0.chunk_bits, 32, 1, nw, DF11_WALKER_BYTE_STEP, use_counts);
            if (ke) break;
        }
        if (!ke && opt.walker == DF11_WALKER_BYTE_STEP) return LaunchStatus::kUnsupported;
    }
    if (!ke) {
        const int nwarp = warp_tiles ? (opt.warps_per_cta ? opt.warps_per_cta : kDefaultWarpsPerCta) : 0;
        ke = find_kernel(b0.dtype, b0.chunk_bits, b0.tile_threads, cpt, nwarp, DF11_WALKER_WINDOW);
        if (!ke) return LaunchStatus::kUnsupported;
    }
    const ImageLayout L0 = image_layout(b0);
    P.meta = reinterpret_cast<const uint32_t *>(b0.dev_image + L0.meta);
    P.syms = reinterpret_cast<const uint32_t *>(b0.dev_image + L0.syms);
    P.lut = reinterpret_cast<const uint16_t *>(b0.dev_image + L0.lut);
    P.fsm = reinterpret_cast<const uint32_t *>(b0.dev_image + L0.fsm);
    P.fsm_rows = rows;
    P.expire = opt.diag_expire_waits ? 1 : 0;
    P.diag_bounds = opt.diag_check_bounds ? 1 : 0;
    P.pad = 0;
    P.wait_ns = opt.diag_expire_waits ? 10000000ull : 2000000000ull;
    P.err = err;
    P.n_luts = b0.cb->n_luts();
    P.n_tensors = nt;
    P.total_tiles = static_cast<uint32_t>(tiles);
    P.max_span = static_cast<uint32_t>(max_span);
    out->ke = ke;
    out->max_span = static_cast<uint32_t>(max_span);
    out->n_lut_smem = P.n_luts < kSmemLutTables ? P.n_luts : kSmemLutTables;
    out->ctas_per_sm = opt.ctas_per_sm;
    out->max_ctas = opt.max_ctas;
    if (ke->walker == DF11_WALKER_BYTE_STEP)
        out->smem = make_fsm_plan(b0.chunk_bits, ke->nwarp, out->max_span, rows, ke->counts != 0).total;
    else if (warp_tiles)
        out->smem = make_warp_plan(b0.chunk_bits, ke->nwarp, out->max_span, out->n_lut_smem).total;
    else
        out->smem = make_plan(b0.chunk_bits, b0.tile_threads, out->max_span, out->n_lut_smem).total;
    if (out->smem > kSmemBudget) return LaunchStatus::kUnsupported;
    return LaunchStatus::kOk;
}

LaunchStatus shape_for(const Prepared &pp, LaunchShape *sh) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LaunchStatus::kCuda;
    if (!prepare(pp.ke, dev)) return LaunchStatus::kCuda;
    if (static_cast<int>(pp.smem) > g_smem_optin[dev]) return LaunchStatus::kUnsupported;
    const int block = pp.ke->nwarp ? pp.ke->nwarp * 32 : pp.ke->chunks / pp.ke->cpt + 32;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, pp.ke->fn, block, pp.smem) != cudaSuccess)
        return LaunchStatus::kCuda;
    if (per_sm < 1) return LaunchStatus::kUnsupported;
    if (pp.ctas_per_sm > 0 && pp.ctas_per_sm < per_sm) per_sm = pp.ctas_per_sm;
    const uint64_t want = static_cast<uint64_t>(per_sm) * static_cast<uint64_t>(g_sm_count[dev]);
    // one CTA per tile (CTA kernel) or per nwarp tiles (warp kernel) at most
    const uint64_t tiles_per_cta = pp.ke->nwarp ? static_cast<uint64_t>(pp.ke->nwarp) : 1u;
    const uint64_t need = (pp.params.total_tiles + tiles_per_cta - 1) / tiles_per_cta;
    uint64_t grid = want < need ? want : need;
    if (pp.max_ctas > 0 && grid > static_cast<uint64_t>(pp.max_ctas)) grid = static_cast<uint64_t>(pp.max_ctas);
    sh->grid = static_cast<int>(grid);
    sh->block = block;
    sh->smem = static_cast<int>(pp.smem);
    sh->walker = pp.ke->walker;
    sh->stored_counts = pp.ke->counts;
    return LaunchStatus::kOk;
}

}  // namespace

bool kernel_available(int dtype, int chunk_bits, int tile_threads) {
    return find_kernel(dtype, chunk_bits, tile_threads, 1, tile_threads == 32 ? kDefaultWarpsPerCta : 0,
                       DF11_WALKER_WINDOW) != nullptr;
}

LaunchStatus decode_launch_shape(const Blob *const *blobs, int n, const DecodeOptions &opt, LaunchShape *out) {
    Prepared pp;
    // the shape does not depend on the destinations: use 16-byte aligned stand-ins
    void *fake[kMaxTensorsPerLaunch];
    for (int i = 0; i < n && i < kMaxTensorsPerLaunch; ++i) fake[i] = reinterpret_cast<void *>(uintptr_t{256});
    LaunchStatus st = build_params(blobs, fake, n, nullptr, opt, &pp);
    if (st != LaunchStatus::kOk) return st;
    if (!pp.params.total_tiles) {
        *out = LaunchShape{};
        return LaunchStatus::kOk;
    }
    return shape_for(pp, out);
}

LaunchStatus launch_decode(const Blob *const *blobs, void *const *dst, int n, int *err, const DecodeOptions &opt,
                           cudaStream_t s) {
    Prepared pp;
    LaunchStatus st = build_params(blobs, dst, n, err, opt, &pp);
    if (st != LaunchStatus::kOk) return st;
    if (!pp.params.total_tiles) return LaunchStatus::kOk;
    LaunchShape sh;
    st = shape_for(pp, &sh);
    if (st != LaunchStatus::kOk) return st;
    if (opt.overlap) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(sh.grid));
        cfg.blockDim = dim3(static_cast<unsigned>(sh.block));
        cfg.dynamicSmemBytes = static_cast<size_t>(sh.smem);
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, pp.ke->fn, pp.params, pp.max_span, pp.n_lut_smem) != cudaSuccess)
            return LaunchStatus::kCuda;
    } else {
        pp.ke->fn<<<sh.grid, sh.block, sh.smem, s>>>(pp.params, pp.max_span, pp.n_lut_smem);
    }
    if (cudaGetLastError() != cudaSuccess) return LaunchStatus::kCuda;
    return LaunchStatus::kOk;
}

}  // namespace df11
