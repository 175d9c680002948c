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

#include "../../include/df11.h"
#include "launch.h"

namespace df11 {
namespace {

// ------------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t tx) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(tx)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Waits for the phase of `parity` to complete; false after kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_ns() - t0 > kWaitLimitNs) return false;
    }
    return true;
}

// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`.
// Both addresses 16-byte aligned, bytes a positive multiple of 16.
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *gmem_src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(smem_dst)),
        "l"(gmem_src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void consumer_sync(int nthreads) {
    asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

__device__ __forceinline__ uint32_t bswap32(uint32_t x) { return __byte_perm(x, 0, 0x0123); }

__device__ __forceinline__ void report(int *err, uint32_t bits) {
    if (err && bits) atomicOr(err, static_cast<int>(bits));
}

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

struct Plan {
    uint32_t stream_bytes;  // per stage: tile stream + 16 look-ahead bytes
    uint32_t gaps_bytes;    // per stage
    uint32_t plane_bytes;   // per stage
    uint32_t stage_bytes;
    uint32_t off_meta, off_syms, off_lut, off_stage, off_exps, exps_bytes, total;
};

__host__ __device__ inline uint32_t up128(uint32_t x) { return (x + 127u) & ~127u; }

__host__ __device__ inline Plan make_plan(int dtype, int chunk_bits, int nt, int stages, uint32_t max_span,
                                          int n_lut_smem) {
    Plan p;
    p.stream_bytes = static_cast<uint32_t>(nt * chunk_bits / 8) + 16u;
    p.gaps_bytes = static_cast<uint32_t>(nt);
    // plane span of a tile: BF16 16-element groups (16 plane bytes), E4M3
    // 32-element groups (16 plane bytes)
    p.plane_bytes = dtype == 0 ? ((max_span + 32u + 15u) & ~15u) : (((max_span + 1u) / 2u + 48u + 15u) & ~15u);
    p.stage_bytes = up128(p.stream_bytes) + up128(p.gaps_bytes) + up128(p.plane_bytes);
    p.off_meta = kCtrlBytes;
    p.off_syms = p.off_meta + kMultiEntries * 2;
    p.off_lut = p.off_syms + kMultiEntries * 4;
    p.off_stage = up128(p.off_lut + static_cast<uint32_t>(n_lut_smem) * kLutEntries * 2);
    p.off_exps = p.off_stage + static_cast<uint32_t>(stages) * p.stage_bytes;
    p.exps_bytes = up128(max_span + 2u * 32u + 16u);
    p.total = p.off_exps + p.exps_bytes;
    return p;
}

// ------------------------------------------------------------------ the two walks

// Walks the codes that start in one thread's chunk.  w[0..CW] hold the chunk
// (CW 32-bit words, most significant bit first) plus one look-ahead word;
// decoding starts at bit p = gap and stops before bit E (chunk_bits, or the
// stream end inside the last chunk).  EMIT = false counts (phase 1); EMIT =
// true also writes each symbol to out[0..count) (phase 2).  Both passes take
// the identical path through the same tables, so they visit the same codes.
template <bool EMIT, int CW>
__device__ __forceinline__ uint32_t walk(const uint32_t (&w)[CW + 1], int p, const int E,
                                         const uint16_t *__restrict__ meta, const uint32_t *__restrict__ syms,
                                         const uint16_t *__restrict__ lut_s, const uint16_t *__restrict__ lut_g,
                                         const int n_lut_smem, uint8_t *__restrict__ out, uint32_t &err) {
    uint32_t cnt = 0;
#pragma unroll
    for (int k = 0; k < CW; ++k) {
        const int base = 32 * k;
        const int ls = min(32, E - base);                     // a code may start here
        const int lm = min(32, E - base - (kMultiBits - 1));  // a whole 12-bit window lies before E
        const uint32_t hi = w[k], lo = w[k + 1];
        while (p < ls) {
            const uint32_t win = __funnelshift_l(lo, hi, p);  // stream bits [p, p + 32) of this word pair
            if (p < lm) {
                const uint32_t idx = win >> (32 - kMultiBits);
                const uint32_t mm = meta[idx];
                if (!(mm & kMetaLong)) {
                    const uint32_t c = mm >> 8;
                    if (EMIT) {
                        const uint32_t sy = syms[idx];
                        out[cnt] = static_cast<uint8_t>(sy);
                        if (c > 1) out[cnt + 1] = static_cast<uint8_t>(sy >> 8);
                        if (c > 2) out[cnt + 2] = static_cast<uint8_t>(sy >> 16);
                        if (c > 3) out[cnt + 3] = static_cast<uint8_t>(sy >> 24);
                    }
                    p += static_cast<int>(mm & 0x3Fu);
                    cnt += c;
                    continue;
                }
            }
            // one code through the hierarchical 256-entry tables
            uint32_t e = lut_s[win >> 24];
#pragma unroll 1
            for (int lvl = 1; (e & kLutPointer) && lvl < 4; ++lvl) {
                const uint32_t tbl = e & 0x7FFFu;
                const uint32_t ix = tbl * kLutEntries + ((win >> (24 - 8 * lvl)) & 0xFFu);
                e = static_cast<int>(tbl) < n_lut_smem ? lut_s[ix] : __ldg(lut_g + ix);
            }
            if (e & (kLutPointer | 0x4000u)) {  // no codeword: count one bit so the walk still ends
                err |= DF11_DEV_ERR_CODE;
                e = 1u << 8;
            }
            if (EMIT) out[cnt] = static_cast<uint8_t>(e);
            p += static_cast<int>((e >> 8) & 0x3Fu);
            cnt += 1;
        }
        p -= 32;
    }
    return cnt;
}

// ------------------------------------------------------------------ field merges

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

__device__ __forceinline__ void st_global_v4(void *p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// ------------------------------------------------------------------ kernel

template <int DT, int CB, int NT, int STAGES>
__global__ void __launch_bounds__(NT + 32, 1)
    decode_kernel(const __grid_constant__ DecodeParams P, const uint32_t max_span, const int n_lut_smem) {
    constexpr int CW = CB / 32;
    constexpr int NW = NT / 32;
    constexpr uint32_t GROUP = DT == 0 ? 16u : 32u;  // elements per 16 plane bytes
    extern __shared__ __align__(128) uint8_t smem[];
    const Plan plan = make_plan(DT, CB, NT, STAGES, max_span, n_lut_smem);

    uint64_t *full = reinterpret_cast<uint64_t *>(smem);
    uint64_t *empty = full + STAGES;
    StageMeta *smeta = reinterpret_cast<StageMeta *>(smem + 128);
    uint32_t *warp_tot = reinterpret_cast<uint32_t *>(smem + 128 + 32 * 8);
    uint16_t *s_meta = reinterpret_cast<uint16_t *>(smem + plan.off_meta);
    uint32_t *s_syms = reinterpret_cast<uint32_t *>(smem + plan.off_syms);
    uint16_t *s_lut = reinterpret_cast<uint16_t *>(smem + plan.off_lut);
    uint8_t *s_exps = smem + plan.off_exps;

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;

    // stage the decode tables (all warps), initialise the pipeline barriers
    {
        const uint4 *g = reinterpret_cast<const uint4 *>(P.meta);
        uint4 *s = reinterpret_cast<uint4 *>(s_meta);
        for (int i = tid; i < kMultiEntries * 2 / 16; i += NT + 32) s[i] = __ldg(g + i);
        g = reinterpret_cast<const uint4 *>(P.syms);
        s = reinterpret_cast<uint4 *>(s_syms);
        for (int i = tid; i < kMultiEntries * 4 / 16; i += NT + 32) s[i] = __ldg(g + i);
        g = reinterpret_cast<const uint4 *>(P.lut);
        s = reinterpret_cast<uint4 *>(s_lut);
        for (int i = tid; i < n_lut_smem * kLutEntries * 2 / 16; i += NT + 32) s[i] = __ldg(g + i);
    }
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NW);
        }
        warp_tot[NW] = 0;  // abort marker
        fence_mbar_init();
    }
    __syncthreads();

    auto stage_stream = [&](int s) { return smem + plan.off_stage + s * plan.stage_bytes; };
    auto stage_gaps = [&](int s) { return stage_stream(s) + up128(plan.stream_bytes); };
    auto stage_plane = [&](int s) { return stage_gaps(s) + up128(plan.gaps_bytes); };

    if (warp == NW) {
        // ---------------- producer warp: one lane issues every copy
        if (lane != 0) return;
        uint32_t k = 0;
        uint32_t armed = 0;          // bit s: stage s has been armed at least once
        uint32_t last_parity = 0;    // bit s: parity of its last armed phase
        for (uint32_t t = blockIdx.x; t < P.total_tiles; t += gridDim.x, ++k) {
            const int s = static_cast<int>(k % STAGES);
            const uint32_t ph = (k / STAGES) & 1u;
            if (!mbar_wait(&empty[s], ph ^ 1u)) {
                report(P.err, DF11_DEV_ERR_TIMEOUT);
                break;
            }
            int ti = 0;
            while (ti + 1 < P.n_tensors && t >= P.t[ti + 1].tile_begin) ++ti;
            const TensorDesc &d = P.t[ti];
            const uint32_t lt = t - d.tile_begin;
            uint64_t S = __ldg(d.out_off + lt);
            const uint64_t E = __ldg(d.out_off + lt + 1);
            uint32_t bad = 0;
            if (E < S || E > d.n || E - S > max_span) {
                report(P.err, DF11_DEV_ERR_AUX);
                bad = 1;
                S = 0;
            }
            const uint32_t span = bad ? 0u : static_cast<uint32_t>(E - S);
            StageMeta &m = smeta[s];
            m.S = S;
            m.span = span;
            m.tensor = static_cast<uint32_t>(ti);
            m.local_tile = lt;
            m.bad = bad;
            uint64_t a0 = 0, a1 = 0;
            if (span) {
                a0 = (S / GROUP) * 16u;
                a1 = ((S + span + GROUP - 1) / GROUP) * 16u;
            }
            const uint32_t pbytes = static_cast<uint32_t>(a1 - a0);
            mbar_arrive_expect_tx(&full[s], plan.stream_bytes + plan.gaps_bytes + pbytes);
            bulk_load(stage_stream(s), d.stream + static_cast<uint64_t>(lt) * (NT * CB / 8), plan.stream_bytes,
                      &full[s]);
            bulk_load(stage_gaps(s), d.gaps + static_cast<uint64_t>(lt) * NT, plan.gaps_bytes, &full[s]);
            if (pbytes) bulk_load(stage_plane(s), d.plane + a0, pbytes, &full[s]);
            armed |= 1u << s;
            last_parity = (last_parity & ~(1u << s)) | (ph << s);
        }
        // keep the CTA alive until every copy it issued has landed
        for (int s = 0; s < STAGES; ++s)
            if (armed & (1u << s))
                if (!mbar_wait(&full[s], (last_parity >> s) & 1u)) report(P.err, DF11_DEV_ERR_TIMEOUT);
        return;
    }

    // ---------------- consumer warps
    uint32_t err = 0;
    uint32_t k = 0;
    for (uint32_t t = blockIdx.x; t < P.total_tiles; t += gridDim.x, ++k) {
        const int s = static_cast<int>(k % STAGES);
        const uint32_t ph = (k / STAGES) & 1u;
        const bool landed = mbar_wait(&full[s], ph);
        const StageMeta m = smeta[s];
        const int ti = landed && m.tensor < static_cast<uint32_t>(P.n_tensors) ? static_cast<int>(m.tensor) : 0;
        const TensorDesc &d = P.t[ti];

        // ---- phase 1: load this thread's chunk, count the codes starting in it
        const uint8_t *sst = stage_stream(s);
        uint32_t w[CW + 1];
        if constexpr (CW % 4 == 0) {
#pragma unroll
            for (int j = 0; j < CW / 4; ++j) {
                const uint4 v = *reinterpret_cast<const uint4 *>(sst + tid * (CB / 8) + 16 * j);
                w[4 * j + 0] = bswap32(v.x);
                w[4 * j + 1] = bswap32(v.y);
                w[4 * j + 2] = bswap32(v.z);
                w[4 * j + 3] = bswap32(v.w);
            }
        } else {
            const uint2 v = *reinterpret_cast<const uint2 *>(sst + tid * (CB / 8));
            w[0] = bswap32(v.x);
            w[1] = bswap32(v.y);
        }
        {
            // look-ahead word: the next thread's first word (lane 31 reads it)
            const uint32_t nxt = __shfl_down_sync(0xFFFFFFFFu, w[0], 1);
            w[CW] = lane == 31 ? bswap32(*reinterpret_cast<const uint32_t *>(sst + (tid + 1) * (CB / 8))) : nxt;
        }
        const int gap = stage_gaps(s)[tid];
        const int64_t chunk_start = (static_cast<int64_t>(m.local_tile) * NT + tid) * CB;
        const int64_t rem = static_cast<int64_t>(d.total_bits) - chunk_start;
        const int E = rem >= CB ? CB : (rem <= 0 ? 0 : static_cast<int>(rem));
        const uint32_t cnt =
            walk<false, CW>(w, gap, E, s_meta, s_syms, s_lut, P.lut, n_lut_smem, nullptr, err);

        // ---- scan: warp shuffles, then the warp totals
        uint32_t incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) warp_tot[warp] = incl;
        if (!landed) warp_tot[NW] = 1;  // abort marker, read after the barrier
        consumer_sync(NT);
        if (warp_tot[NW]) {
            err |= DF11_DEV_ERR_TIMEOUT;
            break;
        }
        uint32_t prefix = 0, total = 0;
#pragma unroll
        for (int i = 0; i < NW; ++i) {
            const uint32_t v = warp_tot[i];
            total += v;
            prefix += i < warp ? v : 0u;
        }
        const uint32_t q0 = prefix + incl - cnt;
        const bool good = !m.bad && total == m.span;
        if (!good && !m.bad && tid == 0) err |= DF11_DEV_ERR_SPAN;

        // ---- phase 2: decode again, exponents into shared memory
        if (good && m.span)
            walk<true, CW>(w, gap, E, s_meta, s_syms, s_lut, P.lut, n_lut_smem,
                           s_exps + (m.S % GROUP) + q0, err);
        consumer_sync(NT);

        // ---- merge with the raw plane, 16-byte stores
        if (good && m.span) {
            const uint64_t g0 = m.S / GROUP;
            const uint32_t ng = static_cast<uint32_t>((m.S + m.span + GROUP - 1) / GROUP - g0);
            const uint8_t *spl = stage_plane(s);
            uint8_t *dst = static_cast<uint8_t *>(d.dst);
            const uint64_t lo = m.S, hi = m.S + m.span;
            for (uint32_t i = tid; i < ng; i += NT) {
                const uint4 p4 = *reinterpret_cast<const uint4 *>(spl + 16 * i);
                uint4 a, b;
                if constexpr (DT == 0) {
                    const uint4 x4 = *reinterpret_cast<const uint4 *>(s_exps + 16 * i);
                    merge_bf16x4(p4.x, x4.x, a.x, a.y);
                    merge_bf16x4(p4.y, x4.y, a.z, a.w);
                    merge_bf16x4(p4.z, x4.z, b.x, b.y);
                    merge_bf16x4(p4.w, x4.w, b.z, b.w);
                } else {
                    const uint4 x0 = *reinterpret_cast<const uint4 *>(s_exps + 32 * i);
                    const uint4 x1 = *reinterpret_cast<const uint4 *>(s_exps + 32 * i + 16);
                    merge_e4m3x8(p4.x, x0.x, x0.y, a.x, a.y);
                    merge_e4m3x8(p4.y, x0.z, x0.w, a.z, a.w);
                    merge_e4m3x8(p4.z, x1.x, x1.y, b.x, b.y);
                    merge_e4m3x8(p4.w, x1.z, x1.w, b.z, b.w);
                }
                const uint64_t e0 = (g0 + i) * GROUP;
                uint8_t *out = dst + e0 * (DT == 0 ? 2 : 1);
                if (e0 >= lo && e0 + GROUP <= hi) {
                    st_global_v4(out, a);
                    st_global_v4(out + 16, b);
                } else {
                    // group shared with a neighbouring tile or past the tensor end
                    const uint32_t wv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
                    if constexpr (DT == 0) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const uint64_t pos = e0 + j;
                            if (pos >= lo && pos < hi)
                                reinterpret_cast<uint16_t *>(out)[j] =
                                    static_cast<uint16_t>(wv[j >> 1] >> (16 * (j & 1)));
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const uint64_t pos = e0 + j;
                            if (pos >= lo && pos < hi) out[j] = static_cast<uint8_t>(wv[j >> 2] >> (8 * (j & 3)));
                        }
                    }
                }
            }
        }
        // ---- release the stage (every warp is done reading it)
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }
    report(P.err, err);
}

// ------------------------------------------------------------------ host side

constexpr int kStages = 2;

using KernelFn = void (*)(DecodeParams, uint32_t, int);

struct KernelEntry {
    int dtype, chunk_bits, nt;
    KernelFn fn;
};

#define DF11_KERNEL(DT, CB, NT) {DT, CB, NT, &decode_kernel<DT, CB, NT, kStages>}

const KernelEntry kKernels[] = {
    DF11_KERNEL(0, 128, 256), DF11_KERNEL(1, 128, 256), DF11_KERNEL(0, 256, 128), DF11_KERNEL(1, 256, 128),
    DF11_KERNEL(0, 64, 512),  DF11_KERNEL(1, 64, 512),  DF11_KERNEL(0, 128, 128), DF11_KERNEL(1, 128, 128),
    DF11_KERNEL(0, 128, 512), DF11_KERNEL(1, 128, 512), DF11_KERNEL(0, 256, 256), DF11_KERNEL(1, 256, 256),
};

const KernelEntry *find_kernel(int dtype, int chunk_bits, int nt) {
    for (const auto &e : kKernels)
        if (e.dtype == dtype && e.chunk_bits == chunk_bits && e.nt == nt) return &e;
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
    Plan plan;
};

LaunchStatus build_params(const Blob *const *blobs, void *const *dst, int n, int *err, Prepared *out) {
    if (n < 1 || n > kMaxTensorsPerLaunch || !blobs[0]) return LaunchStatus::kInvalid;
    const Blob &b0 = *blobs[0];
    const KernelEntry *ke = find_kernel(b0.dtype, b0.chunk_bits, b0.tile_threads);
    if (!ke) return LaunchStatus::kUnsupported;
    DecodeParams &P = out->params;
    P = DecodeParams{};
    uint64_t tiles = 0, max_span = 0;
    int nt = 0;
    for (int i = 0; i < n; ++i) {
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
    const ImageLayout L0 = image_layout(b0);
    P.meta = reinterpret_cast<const uint16_t *>(b0.dev_image + L0.meta);
    P.syms = reinterpret_cast<const uint32_t *>(b0.dev_image + L0.syms);
    P.lut = reinterpret_cast<const uint16_t *>(b0.dev_image + L0.lut);
    P.err = err;
    P.n_luts = b0.cb->n_luts();
    P.n_tensors = nt;
    P.total_tiles = static_cast<uint32_t>(tiles);
    P.max_span = static_cast<uint32_t>(max_span);
    out->ke = ke;
    out->max_span = static_cast<uint32_t>(max_span);
    out->n_lut_smem = P.n_luts < kSmemLutTables ? P.n_luts : kSmemLutTables;
    out->plan = make_plan(b0.dtype, b0.chunk_bits, b0.tile_threads, kStages, out->max_span, out->n_lut_smem);
    return LaunchStatus::kOk;
}

LaunchStatus shape_for(const Prepared &pp, LaunchShape *sh) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LaunchStatus::kCuda;
    if (!prepare(pp.ke, dev)) return LaunchStatus::kCuda;
    if (static_cast<int>(pp.plan.total) > g_smem_optin[dev]) return LaunchStatus::kUnsupported;
    const int block = pp.ke->nt + 32;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, pp.ke->fn, block, pp.plan.total) != cudaSuccess)
        return LaunchStatus::kCuda;
    if (per_sm < 1) return LaunchStatus::kUnsupported;
    const uint64_t want = static_cast<uint64_t>(per_sm) * static_cast<uint64_t>(g_sm_count[dev]);
    sh->grid = static_cast<int>(want < pp.params.total_tiles ? want : pp.params.total_tiles);
    sh->block = block;
    sh->smem = static_cast<int>(pp.plan.total);
    return LaunchStatus::kOk;
}

}  // namespace

bool kernel_available(int dtype, int chunk_bits, int tile_threads) {
    return find_kernel(dtype, chunk_bits, tile_threads) != nullptr;
}

LaunchStatus decode_launch_shape(const Blob *const *blobs, int n, LaunchShape *out) {
    Prepared pp;
    // shape does not depend on the destinations: use 16-byte aligned stand-ins
    void *fake[kMaxTensorsPerLaunch];
    for (int i = 0; i < n && i < kMaxTensorsPerLaunch; ++i) fake[i] = reinterpret_cast<void *>(uintptr_t{256});
    LaunchStatus st = build_params(blobs, fake, n, nullptr, &pp);
    if (st != LaunchStatus::kOk) return st;
    if (!pp.params.total_tiles) {
        *out = LaunchShape{};
        return LaunchStatus::kOk;
    }
    return shape_for(pp, out);
}

LaunchStatus launch_decode(const Blob *const *blobs, void *const *dst, int n, int *err, cudaStream_t s) {
    Prepared pp;
    LaunchStatus st = build_params(blobs, dst, n, err, &pp);
    if (st != LaunchStatus::kOk) return st;
    if (!pp.params.total_tiles) return LaunchStatus::kOk;
    LaunchShape sh;
    st = shape_for(pp, &sh);
    if (st != LaunchStatus::kOk) return st;
    pp.ke->fn<<<sh.grid, sh.block, sh.smem, s>>>(pp.params, pp.max_span, pp.n_lut_smem);
    if (cudaGetLastError() != cudaSuccess) return LaunchStatus::kCuda;
    return LaunchStatus::kOk;
}

}  // namespace df11
