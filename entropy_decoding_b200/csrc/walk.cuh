// walk.cuh -- device code shared by the decode kernels (decode.cu) and the
// decode fused into the consuming GEMM (gemm.cu): PTX helpers (mbarriers,
// 1-D bulk copies, bounded waits), the walks of a thread's chunk through the
// decode tables, and the merge of exponents with the raw sign+mantissa plane.
//
// Method: "70% Size, 100% Accuracy ... (DFloat11)", Abstract, items (i)
// (lookup tables in on-chip SRAM) and (ii) (a two-phase kernel: count the
// codes of each thread's chunk, scan for output positions, decode and write).
// Field layout: "Compressing LLMs without Compromise" summary page, "Where the
// redundancy lives".  Table formats: df11_internal.h.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>
#include <utility>

#include "check.cuh"
#include "df11.h"
#include "df11_internal.h"
#include "merge.cuh"

namespace df11 {
namespace {

// The buffers a thread's merge touches: one tensor's output (n elements of 2
// or 1 bytes) and readable plane (n or ceil(n / 2) bytes, padded to 16 bytes
// plus the image's tail), and the shared-memory exponent buffer it decodes
// into.  In the bounds-checked build every access is checked against them
// (an access outside is skipped and recorded in err); in the normal build
// the struct is empty and every check is true.
struct Guard {
#if DF11_CHECK
    uintptr_t dst = 0, plane = 0, exps = 0;
    uint64_t dst_bytes = 0, plane_bytes = 0;
    uint32_t exps_bytes = 0, err = 0;

    __device__ __forceinline__ bool span(const void *p, uint64_t len, uintptr_t base, uint64_t cap) {
        return in_bounds(static_cast<uint64_t>(reinterpret_cast<uintptr_t>(p) - base), len, cap, err);
    }
#endif
    // the plane of n elements
    template <int DT>
    __device__ __forceinline__ void plane_of(const uint8_t *p, uint64_t n) {
#if DF11_CHECK
        plane = reinterpret_cast<uintptr_t>(p);
        plane_bytes = ((DT == 0 ? n : (n + 1) / 2) + 15u) / 16u * 16u + kPlaneTail;
#else
        (void)p;
        (void)n;
#endif
    }
    // a tensor's plane and output
    template <int DT>
    __device__ __forceinline__ void tensor(const TensorDesc &d) {
        plane_of<DT>(d.plane, d.n);
#if DF11_CHECK
        dst = reinterpret_cast<uintptr_t>(d.dst);
        dst_bytes = d.n * (DT == 0 ? 2u : 1u);
#endif
    }
    __device__ __forceinline__ void buffer(const uint8_t *e, uint32_t bytes) {
#if DF11_CHECK
        exps = reinterpret_cast<uintptr_t>(e);
        exps_bytes = bytes;
#else
        (void)e;
        (void)bytes;
#endif
    }
    // output bytes [p, p + len)
    __device__ __forceinline__ bool out(const void *p, uint64_t len) {
#if DF11_CHECK
        return span(p, len, dst, dst_bytes);
#else
        (void)p;
        (void)len;
        return true;
#endif
    }
    // the elements [lo, hi) of the ne elements (esz bytes each) of a unit
    // starting at element e0, stored at p
    __device__ __forceinline__ bool out_elems(const void *p, uint32_t e0, uint32_t ne, uint32_t lo, uint32_t hi,
                                              uint32_t esz) {
#if DF11_CHECK
        const uint32_t a = max(e0, lo), b = min(e0 + ne, hi);
        return a >= b || out(static_cast<const uint8_t *>(p) + (a - e0) * esz, static_cast<uint64_t>(b - a) * esz);
#else
        (void)p;
        (void)e0;
        (void)ne;
        (void)lo;
        (void)hi;
        (void)esz;
        return true;
#endif
    }
    // plane bytes [p, p + len)
    __device__ __forceinline__ bool pl(const void *p, uint64_t len) {
#if DF11_CHECK
        return span(p, len, plane, plane_bytes);
#else
        (void)p;
        (void)len;
        return true;
#endif
    }
    // exponent-buffer bytes [p, p + len) (a generic pointer into shared memory)
    __device__ __forceinline__ bool ex(const void *p, uint64_t len) {
#if DF11_CHECK
        return span(p, len, exps, exps_bytes);
#else
        (void)p;
        (void)len;
        return true;
#endif
    }
    __device__ __forceinline__ uint32_t flags() const {
#if DF11_CHECK
        return err;
#else
        return 0u;
#endif
    }
};

// Hierarchical tables a kernel stages in shared memory: n_lut_smem, in the
// bounds-checked build no more than the launch's n_luts.
__device__ __forceinline__ int lut_stage_count(int n_lut_smem, int n_luts) {
#if DF11_CHECK
    return min(n_lut_smem, n_luts);
#else
    (void)n_luts;
    return n_lut_smem;
#endif
}

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

// Waits for the phase of `parity` to complete; false after limit_ns (the
// launch's DecodeParams::wait_ns: 2 s, or 10 ms when its waits are made to
// run out on purpose).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_ns() - t0 > limit_ns) return false;
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

// Lets a kernel launched after this one with programmatic stream
// serialization start as soon as SMs free up (no effect otherwise).  Decode
// launches never consume a previous decode's output, so they trigger at once.
__device__ __forceinline__ void allow_dependent_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void report(int *err, uint32_t bits) {
    if (err && bits) atomicOr(err, static_cast<int>(bits));
}


// ------------------------------------------------------------------ decoding a chunk

struct Tables {
    const uint32_t *meta;   // shared
    const uint32_t *syms;   // shared
    const uint16_t *lut_s;  // shared: hierarchical tables [0, n_lut_smem)
    const uint16_t *lut_g;  // global: all hierarchical tables
    int n_lut_smem;
    int n_luts;
    // shared-memory byte addresses [out_lo, out_hi) the window walk may write
    // symbols to (checked in the bounds-checked build only)
    uint32_t out_lo = 0, out_hi = 0xFFFFFFFFu;
};

// One code through the hierarchical 256-entry tables; `win` holds the next 32
// stream bits, most significant first.  Returns symbol | length << 8.  A bit
// pattern that is no codeword (possible only for a one-symbol code or a
// damaged stream), a pointer past the last table or a zero length (damaged
// tables) is flagged and consumed as one 1-bit code, so every step advances.
__device__ __forceinline__ uint32_t lut_decode(uint32_t win, const Tables &T, uint32_t &err) {
    uint32_t e = T.lut_s[win >> 24];
#pragma unroll 1
    for (int lvl = 1; (e & kLutPointer) && lvl < 4; ++lvl) {
        const int tbl = static_cast<int>(e & 0x7FFFu);
        if (tbl >= T.n_luts) break;
        const uint32_t ix = static_cast<uint32_t>(tbl) * kLutEntries + ((win >> (24 - 8 * lvl)) & 0xFFu);
        if (tbl < T.n_lut_smem) {
            e = in_bounds(ix, 1, static_cast<uint64_t>(T.n_lut_smem) * kLutEntries, err) ? T.lut_s[ix] : 0u;
        } else {
            e = in_bounds(ix, 1, static_cast<uint64_t>(T.n_luts) * kLutEntries, err) ? __ldg(T.lut_g + ix) : 0u;
        }
    }
    if ((e & (kLutPointer | 0x4000u)) || !(e & 0x3F00u)) {
        err |= DF11_DEV_ERR_CODE;
        e = 1u << 8;
    }
    return e;
}

// A multi-symbol entry is used only when it consumes 1..12 bits, yields 1..4
// symbols and its start mask has one bit per symbol starting at offset 0;
// anything else (a damaged table) becomes the long-code sentinel, whose codes
// the hierarchical tables then decode one at a time.
__device__ __forceinline__ uint32_t sane_meta(uint32_t e) {
    const uint32_t used = e & 0x7FFu, n = (e >> kMetaCountShift) & 0x1FFu, mask = e >> kMetaMaskShift;
    const bool ok = used >= 1 && used <= kMultiBits && n >= 1 && n <= kMultiMaxSyms && (mask & 1u) &&
                    static_cast<uint32_t>(__popc(mask)) == n && mask < (1u << used);
    return ok ? e : kMetaLong;
}

// Multi-symbol table reads: shared-memory copies were checked when staged;
// GM = true reads the image in global memory and checks each entry.
template <bool GM>
__device__ __forceinline__ uint32_t meta_at(const Tables &T, uint32_t idx, uint32_t &err) {
    if (!in_bounds(idx, 1, kMultiEntries, err)) return kMetaLong;
    if constexpr (GM) return sane_meta(__ldg(T.meta + idx));
    else return T.meta[idx];
}

template <bool GM>
__device__ __forceinline__ uint32_t syms_at(const Tables &T, uint32_t idx, uint32_t &err) {
    if (!in_bounds(idx, 1, kMultiEntries, err)) return 0u;
    if constexpr (GM) return __ldg(T.syms + idx);
    else return T.syms[idx];
}

// Number of an entry's codes that start before bit `room` of its window.
__device__ __forceinline__ uint32_t starts_before(uint32_t mm, int room) {
    return static_cast<uint32_t>(__popc((mm >> kMetaMaskShift) & ((1u << room) - 1u)));
}

// Field masks of a walker's accumulator acc = p | count << kMetaCountShift.
constexpr uint32_t kPosMask = (1u << kMetaCountShift) - 1u;
constexpr uint32_t kCountOne = 1u << kMetaCountShift;

// Phase 1 (CTA-tile kernel): count the codes that start in each of this
// thread's CPT chunks, with the chunk in registers.  Chunk c occupies
// w[c*CW .. c*CW+CW-1] (earliest bit first) and w[c*CW+CW] is its look-ahead
// word (the next chunk's first word).  Its walk starts at bit gap[c] and
// counts codes that start before bit E[c].  The walk moves through the chunk
// 32 bits at a time ("stage" k reads the word pair w[k], w[k+1]).  While a
// whole 12-bit window lies before E, one lookup in the multi-symbol table
// consumes up to 4 codes; in the last 11 bits before E the entry's start mask
// counts only the codes that start before E; codes longer than 12 bits (the
// sentinel entry) go through the hierarchical tables.  acc = p | count << 11
// and an entry is consumed | count << 11 | mask << 20, so one add advances
// both (the mask lands above the count field); the sentinel adds 1024 to p,
// which ends the loop.  The CPT chunks advance in lockstep.
template <int CW, int CPT, bool GM = false>
__device__ __forceinline__ void count_codes(const uint32_t (&w)[CPT * CW + 1], const int (&gap)[CPT],
                                            const int (&E)[CPT], const Tables &T, uint32_t (&cnt)[CPT],
                                            uint32_t &err) {
    uint32_t acc[CPT];
#pragma unroll
    for (int c = 0; c < CPT; ++c) acc[c] = static_cast<uint32_t>(gap[c]);
#pragma unroll
    for (int k = 0; k < CW; ++k) {
        int lm[CPT], ls[CPT], er[CPT];
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
            er[c] = E[c] - 32 * k;
            lm[c] = min(32, er[c] - (kMultiBits - 1));
            ls[c] = min(32, er[c]);
        }
        for (;;) {
            for (;;) {
                bool act[CPT], any = false;
#pragma unroll
                for (int c = 0; c < CPT; ++c) {
                    act[c] = static_cast<int>(acc[c] & kPosMask) < lm[c];
                    any |= act[c];
                }
                if (!any) break;
#pragma unroll
                for (int c = 0; c < CPT; ++c) {
                    if (act[c]) {
                        const uint32_t win = __funnelshift_l(w[c * CW + k + 1], w[c * CW + k], acc[c]);
                        acc[c] += meta_at<GM>(T, win >> (32 - kMultiBits), err);
                    }
                }
            }
            bool more = false;
#pragma unroll
            for (int c = 0; c < CPT; ++c) {
                int p = static_cast<int>(acc[c] & kPosMask);
                bool single = false;
                if (p >= static_cast<int>(kMetaLong)) {  // sentinel: the first code is longer than 12 bits
                    acc[c] -= kMetaLong;
                    p -= kMetaLong;
                    single = true;
                } else if (p >= ls[c]) {
                    continue;
                }
                const uint32_t win = __funnelshift_l(w[c * CW + k + 1], w[c * CW + k], p);
                const uint32_t mm = single ? kMetaLong : meta_at<GM>(T, win >> (32 - kMultiBits), err);
                if (mm & kMetaLong) {
                    const uint32_t e = lut_decode(win, T, err);
                    acc[c] += ((e >> 8) & 0x3Fu) + kCountOne;
                } else {  // last bits before E: count only the codes that start before it
                    acc[c] += (mm & 0xFu) + (starts_before(mm, er[c] - p) << kMetaCountShift);
                }
                more = true;
            }
            if (!more) break;
        }
#pragma unroll
        for (int c = 0; c < CPT; ++c) acc[c] -= min(acc[c] & kPosMask, 32u);
    }
#pragma unroll
    for (int c = 0; c < CPT; ++c) cnt[c] = (acc[c] >> kMetaCountShift) & 0x1FFu;
}

// ORs up to 4 symbol bytes `sy` (unused high bytes zero) into shared memory at
// byte address out: the one or two 32-bit words they touch.  The exponent
// buffer is zero before phase 2, so neighbouring chunks can OR into a word
// they share and the zero high bytes leave other symbols intact.
__device__ __forceinline__ void put_symbols(uint32_t sy, uint32_t out, const Tables &T, uint32_t &err) {
    const uint32_t a = out & ~3u, sh = (out & 3u) << 3;
    if (!in_bounds(a - T.out_lo, sh ? 8u : 4u, T.out_hi - T.out_lo, err)) return;
    asm volatile("red.shared.or.b32 [%0], %1;" ::"r"(a), "r"(sy << sh) : "memory");
    if (sh) asm volatile("red.shared.or.b32 [%0+4], %1;" ::"r"(a), "r"(__funnelshift_l(sy, 0u, sh)) : "memory");
}

// Phase 2 (CTA-tile kernel): decode chunk C again along the same path as
// phase 1 and write its symbols from shared-memory byte address q on.
template <int CW, int CPT, int C, bool GM = false>
__device__ __forceinline__ void emit_codes(const uint32_t (&w)[CPT * CW + 1], int p, const int E, const Tables &T,
                                           uint32_t q, uint32_t &err) {
    uint32_t out = q;
#pragma unroll
    for (int k = 0; k < CW; ++k) {
        const int er = E - 32 * k;
        const int lm = min(32, er - (kMultiBits - 1));
        const int ls = min(32, er);
        const uint32_t hi = w[C * CW + k], lw = w[C * CW + k + 1];
        for (;;) {
            while (p < lm) {
                const uint32_t win = __funnelshift_l(lw, hi, p);
                const uint32_t idx = win >> (32 - kMultiBits);
                const uint32_t mm = meta_at<GM>(T, idx, err);
                p += static_cast<int>(mm & kPosMask);
                put_symbols(syms_at<GM>(T, idx, err), out, T, err);
                out += (mm >> kMetaCountShift) & 7u;
            }
            bool single = false;
            if (p >= static_cast<int>(kMetaLong)) {
                p -= kMetaLong;
                single = true;
            } else if (p >= ls) {
                break;
            }
            const uint32_t win = __funnelshift_l(lw, hi, p);
            const uint32_t idx = win >> (32 - kMultiBits);
            const uint32_t mm = single ? kMetaLong : meta_at<GM>(T, idx, err);
            if (mm & kMetaLong) {
                const uint32_t e = lut_decode(win, T, err);
                p += static_cast<int>((e >> 8) & 0x3Fu);
                put_symbols(e & 0xFFu, out, T, err);
                out += 1;
            } else {
                const uint32_t nv = starts_before(mm, er - p);
                const uint32_t nb = 8u * nv;
                const uint32_t sy = nb >= 32 ? syms_at<GM>(T, idx, err) : (syms_at<GM>(T, idx, err) & ((1u << nb) - 1u));
                p += static_cast<int>(mm & 0xFu);
                if (nv) put_symbols(sy, out, T, err);
                out += nv;
            }
        }
        p -= min(p, 32);
    }
}

// ------------------------------------------------------------------ async-proxy fence

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ byte-step kernel

// Steps of the byte-step walk taken unconditionally by a chunk: its range is
// CB + (next gap) - (gap) bits, at least CB - 31 (a gap is below 32), so every
// chunk with a whole range takes its first (CB - 32) / 8 steps without
// per-step checks.
template <int CB>
constexpr int kFixedSteps = (CB - 32) / 8;

// Row base + byte k of x times the entry size, as a byte permute and a
// multiply-add (the multiply-add issues on the FMA pipe).
template <uint32_t ENTRY>
__device__ __forceinline__ uint32_t step_addr(uint32_t x, int k, uint32_t base) {
    const uint32_t b = __byte_perm(x, 0u, 0x4440u + static_cast<uint32_t>(3 - k));
    uint32_t a;
    asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(a) : "r"(b), "n"(ENTRY), "r"(base));
    return a;
}

// Row field of the compact control words (row << 10: rows of 1 KB).
constexpr uint32_t kCtlRowMask = kFsmRowMask >> 1;

// The byte-step walk of one chunk.  The thread's codes occupy bits [g, g +
// 8 * nfull + r) of the words w[0..CW] followed by w2 (earliest bit first):
// from the first code start in the chunk to the first code start in the next
// chunk (or the end of the stream).  Step j looks up byte j of that range in
// the row of the tree node the previous step stopped on (the root first): the
// entry lists the codes that end in the byte and the next row.  Steps below
// NFIX are taken by every thread on the byte-step walk (kFixedSteps); the
// others are predicated on nfull, and the warp stops after its longest range
// (jmax steps).  A last partial byte (r bits) counts only
// the codes whose end mask bit falls in its first r bits; those end exactly
// at the range's end, so the codes of the next chunk are never counted.
//
// Phase 1 (byte_step_count) walks the compact control words (4 bytes per
// entry, so a warp's random lookups spread over all 32 banks: end mask in
// bits 0..7, row << 10, codes ended << 24, so adding whole words counts the
// codes while the lower fields of at most 20 steps stay below bit 24) and
// returns the number of codes; ctl_out receives the last control word, whose row is the
// dead row (`dead`, in control-word form) when the walk left the tables or the
// partial byte ends more than the 4 codes an entry holds (possible only with
// a 1-bit codeword).
template <int CB>
__device__ __forceinline__ uint32_t byte_step_count(const uint32_t (&w)[CB / 32 + 1], uint32_t w2, int g, int nfull,
                                                    int r, int jmax, const uint8_t *ctl_tab, uint32_t dead,
                                                    uint32_t &ctl_out, uint32_t tab_bytes, uint32_t &err) {
    constexpr int CW = CB / 32, NFIX = kFixedSteps<CB>;
    uint32_t ctl = 0, cnt = 0;
#pragma unroll
    for (int m = 0; m <= CW; ++m) {
        if (4 * m >= NFIX && 4 * m >= jmax) break;  // warp-uniform
        const uint32_t x = __funnelshift_l(m < CW ? w[m + 1] : w2, w[m], static_cast<uint32_t>(g));
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int j = 4 * m + k;
            if (j >= NFIX && j >= jmax) break;
            const uint32_t ea = step_addr<4>(x, k, ctl & kCtlRowMask);
            const uint32_t e = in_bounds(ea, 4, tab_bytes, err) ? *reinterpret_cast<const uint32_t *>(ctl_tab + ea) : dead;
            if (j < NFIX || j < nfull) {
                ctl = e;
                cnt += e;  // the count field at bit 24 gathers the codes; the fields below it never carry into it
            } else if (j == nfull) {
                const uint32_t c = static_cast<uint32_t>(__popc(e & ((1u << r) - 1u)));
                cnt += c << 24;
                if (c > 4) ctl = dead;
            }
        }
    }
    ctl_out = ctl;
    return cnt >> 24;
}

// Puts symbol bytes sy (c8 / 8 of them, unused bytes zero) after the f8 / 8
// pending bytes of acc; a completed word goes to byte address wp (inside
// [lo_a, hi_a), checked in the bounds-checked build).
__device__ __forceinline__ void emit_word(uint32_t sy, uint32_t c8, uint32_t &acc, uint32_t &wp, uint32_t &f8,
                                          uint32_t lo_a, uint32_t hi_a, uint32_t &err) {
    const uint32_t lo = acc | (sy << f8);
    const uint32_t hi = __funnelshift_l(sy, 0u, f8);  // bytes pushed past the word
    f8 += c8;
    if (f8 >= 32u) {
        if (in_bounds(wp - lo_a, 4, hi_a - lo_a, err))
            asm volatile("st.shared.u32 [%0], %1;" ::"r"(wp), "r"(lo) : "memory");
        wp += 4u;
        f8 -= 32u;
        acc = hi;
    } else {
        acc = lo;
    }
}

// Phase 2: the same walk on the full entries {ctl, syms}, writing the symbols
// in order from shared-memory byte address `out` on.  Symbols are assembled
// in a register (acc holds f8 / 8 pending bytes, starting from acc0, the
// current content of the word `out` falls in; unused bytes zero) and every
// completed 32-bit word is stored with one plain store.  The word the range
// starts in may hold earlier threads' bytes (stored as zeros here) and the
// word it ends in later threads' bytes: that last, partial word is returned
// in acc / wp / f8 and OR-ed in by the caller after a __syncwarp, so it
// lands after every plain store of the warp and no store clears another
// thread's bytes.  The buffer is zero outside the words written.  The
// steps after the whole bytes only keep the entry of the last, partial byte
// (j == nfull), whose codes are emitted once after the loop.  ctl_out
// receives the last control word, whose row is the dead row (`dead`) when
// the walk left the tables or the partial byte ends more than 4 codes.
template <int CB>
__device__ __forceinline__ void byte_step_emit(const uint32_t (&w)[CB / 32 + 1], uint32_t w2, int g, int nfull,
                                               int r, int jmax, const uint8_t *tab, uint32_t out, uint32_t acc0,
                                               uint32_t dead, uint32_t &acc, uint32_t &wp, uint32_t &f8,
                                               uint32_t &ctl_out, uint32_t tab_bytes, uint32_t lo_a, uint32_t hi_a,
                                               uint32_t &err) {
    constexpr int CW = CB / 32, NFIX = kFixedSteps<CB>;
    uint32_t ctl = 0;
    acc = acc0;
    wp = out & ~3u;
    f8 = (out & 3u) << 3;
    uint2 ep = make_uint2(0u, 0u);
#pragma unroll
    for (int m = 0; m <= CW; ++m) {
        if (4 * m >= NFIX && 4 * m >= jmax) break;  // warp-uniform
        const uint32_t x = __funnelshift_l(m < CW ? w[m + 1] : w2, w[m], static_cast<uint32_t>(g));
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int j = 4 * m + k;
            if (j >= NFIX && j >= jmax) break;
            const uint32_t ea = step_addr<8>(x, k, ctl & kFsmRowMask);
            const uint2 e =
                in_bounds(ea, 8, tab_bytes, err) ? *reinterpret_cast<const uint2 *>(tab + ea) : make_uint2(dead, 0u);
            if (j < NFIX || j < nfull) {
                ctl = e.x;
                emit_word(e.y, e.x >> (kFsmCountShift - 3), acc, wp, f8, lo_a, hi_a, err);
            } else if (j == nfull) {
                ep = e;  // the partial byte: emitted once after the loop
            }
        }
    }
    if (r) {
        const uint32_t ce = static_cast<uint32_t>(__popc(ep.x & ((1u << r) - 1u)));
        const uint32_t c = min(ce, 4u);
        emit_word(c ? ep.y & (0xFFFFFFFFu >> (32u - 8u * c)) : 0u, 8u * c, acc, wp, f8, lo_a, hi_a, err);
        if (ce > 4) ctl = dead;
    }
    ctl_out = ctl;
}

// ------------------------------------------------------------------ plane loads

// 8 plane bytes (one output half: 8 BF16 or 16 E4M3 weights), streamed past L1.
__device__ __forceinline__ uint2 ld_global_stream_v2(const void *p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

// The same load at a constant offset OFF from p (the offset is part of the
// instruction: one address register serves every round).
template <int OFF>
__device__ __forceinline__ uint2 ld_global_stream_v2_at(const void *p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2+%3];" : "=r"(v.x), "=r"(v.y) : "l"(p), "n"(OFF));
    return v;
}

// pre[U] = the plane bytes of half lane + 32 U (pl = the lane's first half)
// for the halves below nhalf: a tile's first halves, loaded at tile start so
// they arrive while the tile decodes.
template <int... U>
__device__ __forceinline__ void prefetch_halves(uint2 *pre, const uint8_t *pl, uint32_t lane, uint32_t nhalf,
                                                Guard &G, std::integer_sequence<int, U...>) {
    ((lane + 32u * U < nhalf && G.pl(pl + 256 * U, 8) ? (void)(pre[U] = ld_global_stream_v2_at<256 * U>(pl))
                                                       : (void)0),
     ...);
}

// One half's plane bytes, checked in the bounds-checked build (zeros outside).
__device__ __forceinline__ uint2 plane_v2(const uint8_t *p, Guard &G) {
    return G.pl(p, 8) ? ld_global_stream_v2(p) : make_uint2(0u, 0u);
}

}  // namespace
}  // namespace df11
