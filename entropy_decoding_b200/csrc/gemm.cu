// gemm.cu -- the decode of Huffman-coded BF16 weights fused into the GEMM that
// consumes them, y += x W, on the fifth-generation tensor cores of sm_100a.
//
// Method: "Compressing LLMs without Compromise" summary page, ZipServ
// paragraph (decompression fused into the matrix multiply, so the decoded
// weights go straight to the tensor cores instead of through HBM), and
// "Approaching Shannon Bound with Lossless LLM Weight Compression", Abstract
// (decoding aligned with the GEMM's tiling).  The decode itself is the
// DFloat11 one ("70% Size, 100% Accuracy ... (DFloat11)", Abstract, items
// (i)-(iii)): tables in shared memory, each thread's output place from its
// chunk's code count (stored counts + warp scan), then the decoding walk; one
// launch for all matrices that share a code.
//
// Layout.  The weights are encoded in operand-tile order (gemm.h): every
// operand tile of 128 output rows x 64 reduction columns is a contiguous run
// of 8192 weights of the ordinary container (stream, gaps, chunk counts,
// out_off per warp tile, plane).  So the decode's output positions map to
// operand tiles by a shift, and nothing else of the container changes.
//
// One CTA per SM owns a contiguous range of operand tiles ("k-tiles"):
//   * warps 0..19 decode the container's warp tiles that cover the range,
//     round robin, with the byte-step walk (phase 2 into the warp's own
//     exponent buffer, as in the decode kernel), and merge them with the raw
//     sign+mantissa plane (prefetched into registers at tile start) straight
//     into BF16 operand tiles in the swizzled K-major layout that
//     tcgen05.mma reads (a ring of operand slots, rows of kGemmTileK weights,
//     the swizzle as wide as a row); a counter per operand slot hands a
//     completed k-tile (128 x kGemmTileK weights placed) to the MMA warp;
//   * warp 20 (lane 0) issues the copies of the activation tiles
//     (cp.async.bulk.tensor with the same swizzle, no multicast; rows past
//     M read as zeros) and the MMAs of each k-tile (M = 128 output rows, N =
//     M padded to 16, K = 16 each; one TMEM accumulator per MMA of a tile,
//     so they do not wait for each other), and
//     frees each k-tile's slot once its MMAs completed (checked without
//     blocking, so several k-tiles' MMAs are in flight);
//   * warps 20..23 drain the accumulators (tcgen05.ld) into y with
//     floating-point adds whenever the range leaves a block of 128 output
//     rows: y's rows are split over CTAs along K, so y accumulates.
// Every wait is bounded (%globaltimer); a timeout sets DF11_DEV_ERR_TIMEOUT
// and a CTA-wide abort flag that ends every other wait at once.  No copy is
// in flight and no TMEM is held when a CTA exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <thread>
#include <vector>

#include "df11.h"
#include "gemm.h"
#include "walk.cuh"

namespace df11 {
namespace {

constexpr int kDecodeWarps = 20;  // warps 0..19 decode; 20..23 copy, multiply and drain
constexpr int kMmaWarp = kDecodeWarps;  // a multiple of 4: warps kMmaWarp + q reach TMEM lanes 32 q .. 32 q + 31
constexpr int kGemmThreads = 32 * (kDecodeWarps + 4);
constexpr uint32_t kKTile = kGemmTileN * kGemmTileK;  // weights of one operand tile
constexpr int kKTileShift = kGemmTileK == 16 ? 11 : (kGemmTileK == 32 ? 12 : 13);
static_assert(kKTile == 1u << kKTileShift, "operand tile of 16, 32 or 64 columns");
constexpr uint32_t kRowBytes = 2 * kGemmTileK;     // one operand row: the swizzle's width
constexpr uint32_t kATileBytes = 2 * kKTile;       // BF16 operand tile: 128 rows
constexpr uint32_t kSwzMask = kRowBytes / 16 - 1;  // 16-byte chunks of a row, less one
// descriptor layout type of that swizzle (128 B: 2, 64 B: 4, 32 B: 6)
constexpr uint64_t kSwzLayout = kRowBytes == 128 ? 2 : (kRowBytes == 64 ? 4 : 6);
constexpr int kMaxASlots = 32, kMaxBSlots = 32;
constexpr int kCB = 128;  // chunk bits of the containers the kernel reads
constexpr uint32_t kTileBytes = 32 * kCB / 8;
constexpr uint32_t kStageTx = kTileBytes + 16u + 48u + 32u;  // stream + look-ahead, gaps, counts
constexpr uint32_t kStageBytes = (kStageTx + 15u) & ~15u;
constexpr uint32_t kCtrlBytes = 2048;
constexpr int kPrefetchHalves = 8;  // plane halves per thread loaded at tile start

struct GemmMat {
    const uint8_t *stream, *plane, *gaps, *counts;
    const uint64_t *out_off;
    float *y;
    uint64_t n;           // weights: K * N
    uint64_t total_bits;  // stream length
    uint32_t n_tiles;     // warp tiles of the container
    uint32_t tile_begin;  // launch-wide index of its first warp tile
    uint32_t kt_begin;    // launch-wide index of its first operand tile
    uint32_t k_tiles;     // K / kGemmTileK: operand tiles per block of 128 output rows
    uint32_t n_out;       // N
    uint32_t pad;
};

struct GemmParams {
    CUtensorMap xmap[kGemmMaxMats];  // x of each matrix: 2-D, box kGemmTileK x mpad, row-wide swizzle
    const uint32_t *meta, *syms;     // 12-bit multi-symbol table (window-walk fallback)
    const uint16_t *lut;             // hierarchical tables
    const uint32_t *fsm;             // byte-step transition tables
    int *err;
    uint64_t wait_ns;
    int32_t fsm_rows, n_luts, n_mats, m;
    int32_t mpad, a_slots, b_slots;
    uint32_t a_magic, b_magic;  // ceil(2^32 / a_slots), ceil(2^32 / b_slots): division by a multiply-high
    uint32_t exps_bytes;        // a decode warp's exponent buffer
    uint32_t max_span, total_kt;
    GemmMat mt[kGemmMaxMats];
    uint32_t cta_kt[kGemmMaxCtas + 1];  // CTA c owns operand tiles [cta_kt[c], cta_kt[c + 1])
    uint32_t cta_vt[kGemmMaxCtas][2];   // and decodes warp tiles [cta_vt[c][0], cta_vt[c][1])
};

// Shared memory, from a 1024-byte aligned base: the transition table, the
// root hierarchical table, the control block, per decode warp its stage and
// exponent buffer, the operand slots and the activation slots (1024-byte
// aligned, as the swizzle needs).
struct GemmPlan {
    uint32_t off_lut, off_ctrl, off_warps, warp_bytes, off_a, off_b, b_bytes, total;
};

__host__ __device__ inline uint32_t up1024(uint32_t x) { return (x + 1023u) & ~1023u; }

__host__ __device__ inline GemmPlan make_gemm_plan(int rows, int mpad, int a_slots, int b_slots, uint32_t exps_bytes) {
    GemmPlan p;
    p.off_lut = static_cast<uint32_t>(rows) * kFsmRowBytes;
    p.off_ctrl = (p.off_lut + kLutEntries * 2 + 127u) & ~127u;
    p.off_warps = p.off_ctrl + kCtrlBytes;
    p.warp_bytes = kStageBytes + exps_bytes;
    p.off_a = up1024(p.off_warps + kDecodeWarps * p.warp_bytes);
    p.b_bytes = static_cast<uint32_t>(mpad) * kRowBytes;
    p.off_b = p.off_a + static_cast<uint32_t>(a_slots) * kATileBytes;
    p.total = p.off_b + static_cast<uint32_t>(b_slots) * p.b_bytes;
    return p;
}

// Exponent buffer of a decode warp: the tile's span after its offset in the
// first half (< 8), what one thread's walk can write past the range its
// stored count gives it when the stream disagrees with the count (4 symbols
// a step, chunk_bits / 8 + 4 steps, the word it ends in), rounded to 16.
__host__ __device__ inline uint32_t gemm_exps_bytes(uint32_t max_span) {
    return (max_span + 8u + 32u + 4u * (kCB / 8 + 6) + 15u) & ~15u;
}

struct GemmCtrl {
    uint64_t stage_full[kDecodeWarps];  // a decode warp's stage landed
    uint64_t b_full[kMaxBSlots];        // an activation tile landed
    uint64_t mma_done[kMaxASlots];      // the MMAs of the k-tile in an operand slot completed
    uint32_t acount[kMaxASlots];        // weights placed into each operand slot
    uint32_t a_ready[kMaxASlots];       // k-tiles completed in each operand slot
    uint32_t a_free[kMaxASlots];        // k-tiles multiplied out of each operand slot
    uint32_t abort;                     // a wait gave up: every other wait ends
    uint32_t tmem;                      // accumulator address
};
static_assert(sizeof(GemmCtrl) <= kCtrlBytes, "control block");

// ------------------------------------------------------------------ tcgen05 / TMA helpers

__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Arrives on `bar` once every tcgen05 operation this thread issued before has completed.
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

// D (TMEM) = A x B^T (+ D when acc != 0); A and B K-major in shared memory.
__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

// 16 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tc_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor of a K-major operand in the row-wide
// swizzle: rows of kRowBytes, 8-row groups 8 kRowBytes apart (stride byte
// offset), the leading byte offset unused (1), descriptor version 1.  The
// k-th MMA of a tile (K = 16) starts 32 k bytes into the rows.
__device__ __forceinline__ uint64_t swz_desc(uint32_t saddr) {
    return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (uint64_t{1} << 16) |
           (static_cast<uint64_t>(8u * kRowBytes >> 4) << 32) | (uint64_t{1} << 46) | (kSwzLayout << 61);
}

// Byte offset o (from a 1024-byte aligned base) in the row-wide swizzle: the
// 16-byte chunks of a row are permuted by the row's low bits (address bits
// 4.. XOR bits 7..).
__device__ __forceinline__ uint32_t swz(uint32_t o) { return o ^ (((o >> 7) & kSwzMask) << 4); }

// Elements [lo, hi) of an 8-weight half (the others belong to a neighbouring
// tile or lie outside the CTA's range), one 2-byte store each.
__device__ __noinline__ void store_half_part(uint8_t *a, uint4 o, uint32_t e, uint32_t lo, uint32_t hi) {
    const uint32_t ov[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
    for (uint32_t i = 0; i < 8; ++i)
        if (e + i >= lo && e + i < hi)
            reinterpret_cast<uint16_t *>(a)[i] = static_cast<uint16_t>(ov[i >> 1] >> (16 * (i & 1)));
}

// 2-D tile copy global -> shared through a tensor map (no multicast).
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(smem_addr(dst)),
        "l"(map), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

// Non-blocking test of an mbarrier phase (try_wait may suspend the thread for
// a while; the MMA warp's polling loop must not).
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ void named_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ uint32_t ld_vol(const uint32_t *p) { return *reinterpret_cast<const volatile uint32_t *>(p); }

__device__ __forceinline__ void set_abort(GemmCtrl &C) { atomicExch(&C.abort, 1u); }

// x / d and x % d for a slot count d in 2..8 by a multiply-high with
// m = ceil(2^32 / d), exact for every x < 2^32 / d.
struct SlotDiv {
    uint32_t d, m;
    __device__ __forceinline__ uint32_t q(uint32_t x) const { return __umulhi(x, m); }
    __device__ __forceinline__ uint32_t r(uint32_t x) const { return x - q(x) * d; }
};

// Acquire load, release add (shared memory, CTA scope): a release orders
// every write the thread saw before it (the warp's, after a __syncwarp).
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_addr(p)) : "memory");
    return v;
}

__device__ __forceinline__ uint32_t atom_add_release(uint32_t *p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.release.cta.shared::cta.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(smem_addr(p)), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ void red_add_release(uint32_t *p, uint32_t v) {
    asm volatile("red.release.cta.shared::cta.add.u32 [%0], %1;" ::"r"(smem_addr(p)), "r"(v) : "memory");
}

// Waits until *ctr >= target (an acquire); false when the CTA aborted or the
// wait ran past limit_ns (which aborts the CTA).
__device__ __noinline__ bool wait_gen_slow(uint32_t *ctr, uint32_t target, GemmCtrl &C, uint64_t limit_ns) {
    const uint64_t t0 = global_ns();
    for (;;) {
        __nanosleep(64);
        if (ld_acquire(ctr) >= target) return true;
        if (ld_vol(&C.abort)) return false;
        if (global_ns() - t0 > limit_ns) {
            set_abort(C);
            return false;
        }
    }
}

__device__ __forceinline__ bool wait_gen(uint32_t *ctr, uint32_t target, GemmCtrl &C, uint64_t limit_ns) {
    return ld_acquire(ctr) >= target || wait_gen_slow(ctr, target, C, limit_ns);
}

__device__ __forceinline__ int mat_of_tile(const GemmParams &P, uint32_t v, int from) {
    int i = from;
    while (i + 1 < P.n_mats && v >= P.mt[i + 1].tile_begin) ++i;
    return i;
}

__device__ __forceinline__ int mat_of_kt(const GemmParams &P, uint32_t kt) {
    int i = 0;
    while (i + 1 < P.n_mats && kt >= P.mt[i + 1].kt_begin) ++i;
    return i;
}

// ------------------------------------------------------------------ kernel

__global__ void __launch_bounds__(kGemmThreads, 1) decode_gemm_kernel(const __grid_constant__ GemmParams P) {
    constexpr int CB = kCB, CW = CB / 32, NFIX = kFixedSteps<CB>;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const GemmPlan plan = make_gemm_plan(P.fsm_rows, P.mpad, P.a_slots, P.b_slots, P.exps_bytes);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    GemmCtrl &C = *reinterpret_cast<GemmCtrl *>(smem + plan.off_ctrl);
    uint16_t *s_lut = reinterpret_cast<uint16_t *>(smem + plan.off_lut);
    uint8_t *abase = smem + plan.off_a;
    const uint32_t SA = static_cast<uint32_t>(P.a_slots), SB = static_cast<uint32_t>(P.b_slots);
    const SlotDiv dA{SA, P.a_magic}, dB{SB, P.b_magic};
    const uint32_t ring_w = SA * kKTile;  // weights the operand ring holds
    const int rows = P.fsm_rows;
    const uint32_t dead = static_cast<uint32_t>(rows - 1) << kFsmRowShift;
    const uint32_t cta = blockIdx.x;
    const uint32_t kt_lo = P.cta_kt[cta], kt_hi = P.cta_kt[cta + 1], n_kt = kt_hi - kt_lo;
    const uint64_t lo = static_cast<uint64_t>(kt_lo) * kKTile, hi = static_cast<uint64_t>(kt_hi) * kKTile;
    // TMEM: one FP32 accumulator of mpad columns per MMA of a tile (K = 16
    // each, kGemmTileK / 16 of them), so a tile's MMAs do not wait for each
    // other's results; the drain adds them up.  A power of two >= 32 columns.
    constexpr uint32_t kAccs = kGemmTileK / 16;
    const uint32_t acc_cols = kAccs * static_cast<uint32_t>(P.mpad);
    const uint32_t ncols = acc_cols <= 32 ? 32u : acc_cols <= 64 ? 64u : acc_cols <= 128 ? 128u : 256u;

    // ---- set-up: tables (a row index past the last row is redirected to the
    // dead row), zeroed control block, stages and exponent buffers
    {
        const uint4 *g = reinterpret_cast<const uint4 *>(P.fsm);
        uint4 *s = reinterpret_cast<uint4 *>(smem);
        const uint32_t lim = static_cast<uint32_t>(rows) << kFsmRowShift;
        for (int i = tid; i < rows * kFsmRowBytes / 16; i += kGemmThreads) {
            uint4 v = __ldg(g + i);
            if ((v.x & kFsmRowMask) >= lim) v.x = (v.x & ~kFsmRowMask) | dead;
            if ((v.z & kFsmRowMask) >= lim) v.z = (v.z & ~kFsmRowMask) | dead;
            s[i] = v;
        }
        const uint4 *gl = reinterpret_cast<const uint4 *>(P.lut);
        uint4 *sl = reinterpret_cast<uint4 *>(s_lut);
        for (int i = tid; i < kLutEntries * 2 / 16; i += kGemmThreads) sl[i] = __ldg(gl + i);
        uint4 *z = reinterpret_cast<uint4 *>(smem + plan.off_ctrl);
        for (uint32_t i = tid; i < (plan.off_a - plan.off_ctrl) / 16; i += kGemmThreads) z[i] = make_uint4(0, 0, 0, 0);
    }
    __syncthreads();
    if (tid == 0) {
        for (int w = 0; w < kDecodeWarps; ++w) mbar_init(&C.stage_full[w], 1);
        for (uint32_t s = 0; s < SB; ++s) mbar_init(&C.b_full[s], 1);
        for (uint32_t s = 0; s < SA; ++s) mbar_init(&C.mma_done[s], 1);
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&C.tmem, ncols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    uint32_t err = 0;
    if (warp < kDecodeWarps) {
        // =============================== decode warps
        uint8_t *stage = smem + plan.off_warps + warp * plan.warp_bytes;
        uint8_t *s_exps = stage + kStageBytes;
        uint64_t *full = &C.stage_full[warp];
        const uint32_t v_lo = P.cta_vt[cta][0], v_hi = P.cta_vt[cta][1];
        const uint32_t v0 = v_lo + static_cast<uint32_t>(warp);
        int mi_issue = mat_of_tile(P, v0 < v_hi ? v0 : v_lo, 0), mi_cur = mi_issue;
        // lane 0: copy warp tile v's stream slice, gaps and chunk counts into the stage
        auto issue = [&](uint32_t v) {
            mi_issue = mat_of_tile(P, v, mi_issue);
            const GemmMat &d = P.mt[mi_issue];
            const uint32_t lt = v - d.tile_begin;
            uint32_t cerr = 0;
            if (in_bounds(static_cast<uint64_t>(lt) * kTileBytes, kTileBytes + 16u,
                          static_cast<uint64_t>(d.n_tiles) * kTileBytes + kStreamTail, cerr) &&
                in_bounds(static_cast<uint64_t>(lt) * 32u, 48u, static_cast<uint64_t>(d.n_tiles) * 32u + kGapsTail,
                          cerr) &&
                in_bounds(static_cast<uint64_t>(lt) * 32u, 32u, static_cast<uint64_t>(d.n_tiles) * 32u, cerr)) {
                mbar_arrive_expect_tx(full, kStageTx);
                bulk_load(stage, d.stream + static_cast<uint64_t>(lt) * kTileBytes, kTileBytes + 16u, full);
                bulk_load(stage + kTileBytes + 16u, d.gaps + static_cast<uint64_t>(lt) * 32u, 48u, full);
                bulk_load(stage + kTileBytes + 64u, d.counts + static_cast<uint64_t>(lt) * 32u, 32u, full);
            } else {
                mbar_arrive(full);  // nothing copied: the stage keeps stale bytes, the error is reported
                report(P.err, cerr);
            }
        };
        if (lane == 0 && v0 < v_hi) issue(v0);
        bool pending = v0 < v_hi;
        const Tables T{P.meta, P.syms, s_lut, P.lut, 1, P.n_luts, smem_addr(s_exps), smem_addr(s_exps) + P.exps_bytes};
        // every stage read stays inside the stage: 32 chunks, the look-ahead
        // words, 48 gaps, 32 counts
        in_bounds(0, kStageTx, kStageBytes, err);
        Guard G;
        G.buffer(s_exps, P.exps_bytes);
        const uint32_t exps_lo = smem_addr(s_exps), exps_hi = exps_lo + P.exps_bytes;
        const uint32_t fsm_bytes = static_cast<uint32_t>(rows) * kFsmRowBytes, ring_bytes = SA * kATileBytes;
        // a k-tile slot receives n more weights; the warp that completes it hands it to the MMA warp
        auto placed = [&](uint32_t kr, uint32_t n) {
            const uint32_t sa = dA.r(kr);
            if (atom_add_release(&C.acount[sa], n) + n == kKTile) {
                C.acount[sa] = 0;
                red_add_release(&C.a_ready[sa], 1u);
            }
        };

        uint32_t k = 0;
        for (uint32_t v = v0; v < v_hi; v += kDecodeWarps, ++k) {
            mi_cur = mat_of_tile(P, v, mi_cur);
            const GemmMat &d = P.mt[mi_cur];
            G.plane_of<0>(d.plane, d.n);
            const uint32_t lt = v - d.tile_begin;
            const bool oo = in_bounds(lt, 2, static_cast<uint64_t>(d.n_tiles) + 1u, err);
            uint64_t S = oo ? __ldg(d.out_off + lt) : 1u;
            const uint64_t Eo = oo ? __ldg(d.out_off + lt + 1) : 0u;
            const bool bad = Eo - S > P.max_span || Eo > d.n;  // Eo < S wraps above max_span
            if (bad) S = 0;
            const uint32_t span = bad ? 0u : static_cast<uint32_t>(Eo - S);
            // output halves (8 weights) of the tile; the first kPrefetchHalves of each lane now
            const uint64_t h0 = S >> 3;
            const uint32_t s0 = static_cast<uint32_t>(S & 7u);
            const uint32_t nh = span ? static_cast<uint32_t>(((S + span + 7u) >> 3) - h0) : 0u;
            const uint8_t *plane = d.plane + h0 * 8u;
            uint2 pre[kPrefetchHalves];
            prefetch_halves(pre, plane + 8u * lane, lane, nh, G, std::make_integer_sequence<int, kPrefetchHalves>{});

            const bool landed = __all_sync(0xFFFFFFFFu, mbar_wait(full, k & 1u, P.wait_ns));
            if (!landed) {
                err |= DF11_DEV_ERR_TIMEOUT;
                if (lane == 0) set_abort(C);
                break;
            }
            pending = false;
            uint32_t w[CW + 1], w2;
#pragma unroll
            for (int j = 0; j < CW / 4; ++j) {
                const uint4 q4 = *reinterpret_cast<const uint4 *>(stage + lane * (CB / 8) + 16 * j);
                w[4 * j + 0] = q4.x;
                w[4 * j + 1] = q4.y;
                w[4 * j + 2] = q4.z;
                w[4 * j + 3] = q4.w;
            }
            {
                const uint32_t n0 = __shfl_down_sync(0xFFFFFFFFu, w[0], 1);
                const uint32_t n1 = __shfl_down_sync(0xFFFFFFFFu, w[1], 1);
                const uint32_t *la = reinterpret_cast<const uint32_t *>(stage + kTileBytes);
                w[CW] = lane == 31 ? la[0] : n0;
                w2 = lane == 31 ? la[1] : n1;
            }
            const int graw = stage[kTileBytes + 16u + lane];
            const int gnext = stage[kTileBytes + 16u + lane + 1];
            const uint32_t cnt = stage[kTileBytes + 64u + lane];
            __syncwarp();
            if (v + kDecodeWarps < v_hi) {
                if (lane == 0) {
                    fence_proxy_async_smem();
                    issue(v + kDecodeWarps);
                }
                pending = true;
            }

            // ---- this thread's range of codes (as in the decode kernel)
            const int64_t trem = static_cast<int64_t>(d.total_bits) - static_cast<int64_t>(lt) * (32 * CB);
            const int rem =
                static_cast<int>(max(min(trem, static_cast<int64_t>(32 * CB + 256)), static_cast<int64_t>(-1))) -
                lane * CB;
            const int E = min(max(rem, 0), CB);
            if (graw >= 32) err |= DF11_DEV_ERR_AUX;
            const int g = min(graw, 63);
            const int nbits = max(min(rem, CB + gnext) - g, -1);
            const bool whole = graw < 32 && gnext < 32 && nbits >= 8 * NFIX;
            const int nfull = nbits >> 3, r = nbits & 7;
            const int jmax = static_cast<int>(__reduce_max_sync(0xFFFFFFFFu, whole ? nfull + (r != 0) : 0));
            bool slow = !whole, mism = false;
            if (__any_sync(0xFFFFFFFFu, slow)) {
                if (slow) {
                    const int gg[1] = {g}, ee[1] = {E};
                    uint32_t c1[1];
                    count_codes<CW, 1, true>(w, gg, ee, T, c1, err);
                    mism = c1[0] != cnt;
                }
            }
            uint32_t incl = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += t;
            }
            const uint32_t total = __shfl_sync(0xFFFFFFFFu, incl, 31);
            const bool good = !bad && total == span;
            if (bad) err |= DF11_DEV_ERR_AUX;
            else if (!good) err |= DF11_DEV_ERR_SPAN;

            if (good && span) {
                // ---- phase 2 into the warp's exponent buffer (element h0 * 8 at offset 0)
                const uint32_t q = smem_addr(s_exps) + s0 + incl - cnt;
                __syncwarp();
                uint32_t acc = 0, wp = 0, f8 = 0, last = 0;
                if (!slow)
                    byte_step_emit<CB>(w, w2, g, nfull, r, jmax, smem, q, 0u, dead, acc, wp, f8, last, fsm_bytes, exps_lo,
                                       exps_hi, err);
                bool redo = false;
                if (!slow) {
                    redo = (last & kFsmRowMask) == dead;
                    if (!redo && (wp - q) * 8u + f8 != 8u * cnt) mism = true;
                }
                __syncwarp();  // every plain store before the OR-ed last words
                if (!slow && !redo && f8 && in_bounds(wp - exps_lo, 4, exps_hi - exps_lo, err))
                    asm volatile("red.shared.or.b32 [%0], %1;" ::"r"(wp), "r"(acc) : "memory");
                if (__any_sync(0xFFFFFFFFu, redo)) {
                    if (redo) {
                        const int gg[1] = {g}, ee[1] = {E};
                        uint32_t c1[1];
                        count_codes<CW, 1, true>(w, gg, ee, T, c1, err);
                        if (c1[0] != cnt) mism = true;
                    }
                }
                slow = (slow || redo) && !mism;
                if (__any_sync(0xFFFFFFFFu, slow)) {
                    if (slow) emit_codes<CW, 1, 0, true>(w, g, E, T, q, err);
                }
                __syncwarp();

                // ---- the part of the tile inside this CTA's range, launch-wide
                const uint64_t base = static_cast<uint64_t>(d.kt_begin) * kKTile;
                const uint64_t in_lo = max(base + S, lo), in_hi = min(base + S + span, hi);
                uint32_t kr0 = 0, kr1 = 0;
                if (in_lo < in_hi) {
                    // its k-tiles' operand slots are free once the k-tiles SA before were multiplied
                    kr0 = static_cast<uint32_t>((in_lo - lo) >> kKTileShift);
                    kr1 = static_cast<uint32_t>((in_hi - 1u - lo) >> kKTileShift);  // kr0 + 1 at most
                    bool ok = true;
                    if (lane == 0)
                        ok = wait_gen(&C.a_free[dA.r(kr0)], dA.q(kr0), C, P.wait_ns) &&
                             (kr1 == kr0 || wait_gen(&C.a_free[dA.r(kr1)], dA.q(kr1), C, P.wait_ns));
                    if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) {
                        err |= DF11_DEV_ERR_TIMEOUT;
                        break;
                    }
                    __syncwarp();
                }
                // ---- merge: half j (8 weights: 8 plane bytes, 8 exponents) -> 16
                // bytes of an operand row.  The operand slots form a ring of
                // ring_w weights, 2 bytes each in order (a k-tile's 128 rows of
                // kGemmTileK weights), swizzled; the exponents are cleared
                // for the next tile.  Positions relative to the tile's first half
                // (32-bit: a tile spans < 2^16 weights).
                const uint64_t e_first = base + (h0 << 3);
                const uint32_t lo_rel = in_lo < in_hi ? static_cast<uint32_t>(max(in_lo, e_first) - e_first) : 0u;
                const uint32_t hi_rel = in_lo < in_hi ? static_cast<uint32_t>(in_hi - e_first) : 0u;
                // ring place of half 0 (a tile starting before the range starts at the ring's end)
                const int32_t rel0 = static_cast<int32_t>(static_cast<int64_t>(e_first) - static_cast<int64_t>(lo));
                const uint32_t rbase = rel0 < 0 ? static_cast<uint32_t>(rel0 + static_cast<int32_t>(ring_w))
                                                : static_cast<uint32_t>(rel0) -
                                                      dA.q(static_cast<uint32_t>(rel0) >> kKTileShift) * ring_w;
                const bool wraps = rbase + 8u * nh > ring_w;
                // no wrap: round rr of a lane is 512 bytes after round 0 (512 / kRowBytes rows on);
                // its swizzle chunk flips by (4 & kSwzMask) between even and odd rounds
                const uint32_t a_even = swz(2u * rbase + 16u * static_cast<uint32_t>(lane));
                const uint32_t a_odd = a_even ^ ((4u & kSwzMask) << 4);
                auto ring_off = [&](uint32_t jj) -> uint32_t {
                    uint32_t rp = rbase + 8u * jj;
                    if (rp >= ring_w) rp -= ring_w;
                    return swz(2u * rp);
                };
                auto merge_one = [&](uint32_t jj, uint2 p2, uint32_t aoff) {
                    if (!G.ex(s_exps + 8u * jj, 8) || !in_bounds(aoff, 16, ring_bytes, err)) return;
                    uint2 *xp = reinterpret_cast<uint2 *>(s_exps + 8u * jj);
                    const uint2 x2 = *xp;
                    *xp = make_uint2(0u, 0u);
                    const uint32_t e = 8u * jj;
                    if (e + 8u <= lo_rel || e >= hi_rel) return;
                    uint4 o;
                    merge_bf16x4(p2.x, x2.x, o.x, o.y);
                    merge_bf16x4(p2.y, x2.y, o.z, o.w);
                    if (e >= lo_rel && e + 8u <= hi_rel) *reinterpret_cast<uint4 *>(abase + aoff) = o;
                    else store_half_part(abase + aoff, o, e, lo_rel, hi_rel);
                };
#pragma unroll
                for (int rr = 0; rr < kPrefetchHalves; ++rr) {
                    const uint32_t jj = static_cast<uint32_t>(lane) + 32u * rr;
                    if (jj < nh) merge_one(jj, pre[rr], wraps ? ring_off(jj) : ((rr & 1) ? a_odd : a_even) + 512u * rr);
                }
                for (uint32_t jj = static_cast<uint32_t>(lane) + 32u * kPrefetchHalves; jj < nh; jj += 32)
                    merge_one(jj, plane_v2(plane + 8u * jj, G), ring_off(jj));
                fence_proxy_async_smem();  // the operand tiles are read by the tensor core (async proxy)
                if (__any_sync(0xFFFFFFFFu, mism)) {
                    // a walk wrote past its stored range: clear the whole buffer (flagged below)
                    uint4 *se = reinterpret_cast<uint4 *>(s_exps);
                    for (uint32_t i = lane; i < P.exps_bytes / 16; i += 32) se[i] = make_uint4(0, 0, 0, 0);
                }
                __syncwarp();
                if (in_lo < in_hi && lane == 0) {
                    const uint64_t e0 = lo + (static_cast<uint64_t>(kr0) + 1u) * kKTile;
                    placed(kr0, static_cast<uint32_t>(min(in_hi, e0) - in_lo));
                    if (kr1 != kr0) placed(kr1, static_cast<uint32_t>(in_hi - e0));
                }
            }
            if (mism) err |= DF11_DEV_ERR_SPAN;
        }
        // after an abort: wait (bounded) for a copy that was issued but never consumed
        if (pending)
            if (!mbar_wait(full, k & 1u, P.wait_ns)) err |= DF11_DEV_ERR_TIMEOUT;
        err |= G.flags();
    } else {
        // =============================== warps 20..23: copies, MMAs, drain
        const int quarter = warp - kDecodeWarps;  // TMEM lanes 32 quarter .. 32 quarter + 31
        const uint32_t tmem = C.tmem;
        const bool issuer = warp == kMmaWarp;
        // instruction descriptor: FP32 accumulate, BF16 A and B, both K-major,
        // N = mpad, M = 128
        const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((static_cast<uint32_t>(P.mpad) >> 3) << 17) |
                               ((128u >> 4) << 24);
        uint32_t n_x = 0;
        auto issue_x = [&](uint32_t kr) {
            const uint32_t kt = kt_lo + kr;
            const int mi = mat_of_kt(P, kt);
            const GemmMat &d = P.mt[mi];
            const uint32_t kb = (kt - d.kt_begin) % d.k_tiles;
            const uint32_t sb = dB.r(kr);
            uint64_t *bar = &C.b_full[sb];
            mbar_arrive_expect_tx(bar, plan.b_bytes);
            tma_load_2d(smem + plan.off_b + sb * plan.b_bytes, &P.xmap[mi], static_cast<int>(kb * kGemmTileK),
                        0, bar);
        };
        if (issuer && lane == 0)
            for (; n_x < n_kt && n_x < SB; ++n_x) issue_x(n_x);
        n_x = __shfl_sync(0xFFFFFFFFu, n_x, 0);
        bool aborted = false;
        uint32_t kr = 0;
        while (kr < n_kt) {  // one block of 128 output rows of one matrix at a time
            const uint32_t kt = kt_lo + kr;
            const GemmMat &d = P.mt[mat_of_kt(P, kt)];
            const uint32_t nb = (kt - d.kt_begin) / d.k_tiles;
            const uint32_t seg_end = min(n_kt, d.kt_begin + (nb + 1u) * d.k_tiles - kt_lo);
            if (issuer && !aborted) {
                // lane 0 alone: issue every k-tile's MMA whose operand and
                // activation tiles are there, retire completed ones in order
                // (slot freed, next activation tile copied), never blocking; the
                // clock is read only in idle stretches
                if (lane == 0) {
                    uint32_t issued = kr, retired = kr, idle = 0;
                    uint64_t t0 = 0;
                    while (retired < seg_end) {
                        bool prog = false;
                        while (retired < issued && mbar_test_wait(&C.mma_done[dA.r(retired)], dA.q(retired) & 1u)) {
                            red_add_release(&C.a_free[dA.r(retired)], 1u);
                            if (n_x < n_kt) issue_x(n_x++);  // n_x == retired + SB: into the slot just freed
                            ++retired;
                            prog = true;
                        }
                        while (issued < seg_end && ld_acquire(&C.a_ready[dA.r(issued)]) >= dA.q(issued) + 1u &&
                               mbar_test_wait(&C.b_full[dB.r(issued)], dB.q(issued) & 1u)) {
                            tc_fence_after();
                            const uint32_t a0 = smem_addr(abase + dA.r(issued) * kATileBytes);
                            const uint32_t b0 = smem_addr(smem + plan.off_b + dB.r(issued) * plan.b_bytes);
#pragma unroll
                            for (int k16 = 0; k16 < kGemmTileK / 16; ++k16)
                                tc_mma(tmem + static_cast<uint32_t>(k16) * static_cast<uint32_t>(P.mpad),
                                       swz_desc(a0 + 32u * k16), swz_desc(b0 + 32u * k16), idesc,
                                       issued > kr ? 1u : 0u);
                            tc_commit(&C.mma_done[dA.r(issued)]);
                            ++issued;
                            prog = true;
                        }
                        if (prog) {
                            idle = 0;
                            continue;
                        }
                        if (idle++ == 0) {
                            t0 = global_ns();
                        } else if ((idle & 31u) == 0 && (ld_vol(&C.abort) || global_ns() - t0 > P.wait_ns)) {
                            set_abort(C);
                            aborted = true;
                            err |= DF11_DEV_ERR_TIMEOUT;
                            // MMAs still in flight must complete before the CTA exits
                            while (retired < issued) {
                                if (!mbar_wait(&C.mma_done[dA.r(retired)], dA.q(retired) & 1u, P.wait_ns)) break;
                                ++retired;
                            }
                            break;
                        }
                        __nanosleep(32);
                    }
                }
                __syncwarp();
                aborted = __shfl_sync(0xFFFFFFFFu, aborted, 0);
                n_x = __shfl_sync(0xFFFFFFFFu, n_x, 0);
            }
            // drain the accumulators of this block of rows into y
            named_sync(1, 128);  // warps kMmaWarp .. kMmaWarp + 3
            const bool skip = __shfl_sync(0xFFFFFFFFu, ld_vol(&C.abort), 0) != 0;
            if (!skip) {
                tc_fence_after();
                float *yc = d.y + static_cast<uint64_t>(nb) * kGemmTileN + 32u * quarter + lane;
                for (int c0 = 0; c0 < P.mpad; c0 += 16) {
                    uint32_t vv[16];
                    float sum[16];
                    tc_ld16(tmem + (static_cast<uint32_t>(32 * quarter) << 16) + static_cast<uint32_t>(c0), vv);
                    tc_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) sum[j] = __uint_as_float(vv[j]);
                    for (uint32_t a = 1; a < kAccs; ++a) {
                        tc_ld16(tmem + (static_cast<uint32_t>(32 * quarter) << 16) + a * static_cast<uint32_t>(P.mpad) +
                                    static_cast<uint32_t>(c0), vv);
                        tc_wait_ld();
#pragma unroll
                        for (int j = 0; j < 16; ++j) sum[j] += __uint_as_float(vv[j]);
                    }
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (c0 + j < P.m) atomicAdd(yc + static_cast<uint64_t>(c0 + j) * d.n_out, sum[j]);
                }
            }
            tc_fence_before();
            named_sync(1, 128);  // warps kMmaWarp .. kMmaWarp + 3
            kr = seg_end;
        }
        if (issuer) {
            // no copy may be in flight when the CTA exits: wait (bounded) for the
            // last copy issued into every activation slot
            if (lane == 0) {
                for (uint32_t s = 0; s < SB; ++s) {
                    const uint32_t issued = n_x > s ? dB.q(n_x - 1u - s) + 1u : 0u;
                    if (issued && !mbar_wait(&C.b_full[s], (issued - 1u) & 1u, P.wait_ns)) err |= DF11_DEV_ERR_TIMEOUT;
                }
            }
            __syncwarp();
            tmem_dealloc(tmem, ncols);
        }
    }
    err = __reduce_or_sync(0xFFFFFFFFu, err);
    if (lane == 0) report(P.err, err);
}

// ------------------------------------------------------------------ host side

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::mutex g_gemm_mu;
EncodeTiledFn g_encode_tiled = nullptr;
constexpr int kGemmDevices = 64;
bool g_gemm_attr[kGemmDevices] = {};
int g_gemm_sms[kGemmDevices] = {};

EncodeTiledFn encode_tiled() {
    std::lock_guard<std::mutex> lk(g_gemm_mu);
    if (!g_encode_tiled) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return nullptr;
        g_encode_tiled = reinterpret_cast<EncodeTiledFn>(fn);
    }
    return g_encode_tiled;
}

bool gemm_prepare(int dev, int *sms) {
    if (dev < 0 || dev >= kGemmDevices) return false;
    std::lock_guard<std::mutex> lk(g_gemm_mu);
    if (!g_gemm_attr[dev]) {
        int v = 0, optin = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
        if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return false;
        if (cudaFuncSetAttribute(reinterpret_cast<const void *>(&decode_gemm_kernel),
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, optin) != cudaSuccess)
            return false;
        g_gemm_sms[dev] = v;
        g_gemm_attr[dev] = true;
    }
    *sms = g_gemm_sms[dev];
    return true;
}

// Warp tile holding launch-wide position `pos` (first tile whose codes reach
// it); `end`: the first warp tile that lies wholly at or after `pos`.
uint32_t tile_at(const GemmJob *jobs, const GemmMat *mt, int n, uint64_t pos, bool end) {
    int i = 0;
    if (end) {
        while (i + 1 < n && pos > static_cast<uint64_t>(mt[i + 1].kt_begin) * kKTile) ++i;
    } else {
        while (i + 1 < n && pos >= static_cast<uint64_t>(mt[i + 1].kt_begin) * kKTile) ++i;
    }
    const uint64_t p = pos - static_cast<uint64_t>(mt[i].kt_begin) * kKTile;
    const std::vector<uint64_t> &oo = jobs[i].w->out_off;
    const size_t nt = oo.size() - 1;
    size_t t;
    if (end) {
        t = static_cast<size_t>(std::lower_bound(oo.begin(), oo.begin() + nt, p) - oo.begin());
    } else {
        t = static_cast<size_t>(std::upper_bound(oo.begin(), oo.begin() + nt, p) - oo.begin());
        t = t ? t - 1 : 0;
    }
    return mt[i].tile_begin + static_cast<uint32_t>(t);
}

struct GemmPrepared {
    GemmParams params;
    GemmShape shape;
};

LaunchStatus build_gemm(const GemmJob *jobs, int n, int m, int *err, bool with_maps, GemmPrepared *out) {
    if (!jobs || n < 1 || n > kGemmMaxMats || m < 1 || m > kGemmMaxBatch) return LaunchStatus::kInvalid;
    GemmParams &P = out->params;
    std::memset(&P, 0, sizeof P);
    const Blob *b0 = jobs[0].w;
    if (!b0 || !b0->cb) return LaunchStatus::kInvalid;
    uint64_t tiles = 0, kts = 0, weights = 0, max_span = 0;
    for (int i = 0; i < n; ++i) {
        const GemmJob &J = jobs[i];
        const Blob *b = J.w;
        if (!b || !b->dev_image || !b->cb || b->device_only) return LaunchStatus::kInvalid;
        if (b->dtype != kBF16 || b->chunk_bits != kCB || b->tile_threads != 32 || !b->chunk_counts)
            return LaunchStatus::kUnsupported;
        for (int s = 0; s < 256; ++s)
            if (b->cb->lengths[s] != b0->cb->lengths[s]) return LaunchStatus::kInvalid;
        if (J.k == 0 || J.n == 0 || J.k % kGemmTileK || J.n % kGemmTileN || b->n != J.k * J.n)
            return LaunchStatus::kInvalid;
        if (!J.x || !J.y || reinterpret_cast<uintptr_t>(J.x) % 16 || reinterpret_cast<uintptr_t>(J.y) % 4)
            return LaunchStatus::kInvalid;
        if (b->dev_cap < image_layout(*b).total || b->out_off.size() != b->n_tiles + 1) return LaunchStatus::kInvalid;
        const ImageLayout L = image_layout(*b);
        GemmMat &d = P.mt[i];
        d.stream = b->dev_image + L.stream;
        d.plane = b->dev_image + L.plane;
        d.gaps = b->dev_image + L.gaps;
        d.counts = b->dev_image + L.counts;
        d.out_off = reinterpret_cast<const uint64_t *>(b->dev_image + L.out_off);
        d.y = J.y;
        d.n = b->n;
        d.total_bits = b->total_bits;
        d.n_tiles = static_cast<uint32_t>(b->n_tiles);
        d.tile_begin = static_cast<uint32_t>(tiles);
        d.kt_begin = static_cast<uint32_t>(kts);
        d.k_tiles = static_cast<uint32_t>(J.k / kGemmTileK);
        d.n_out = static_cast<uint32_t>(J.n);
        tiles += b->n_tiles;
        kts += b->n / kKTile;
        weights += b->n;
        max_span = std::max(max_span, b->max_span);
    }
    if (tiles >= (uint64_t{1} << 31) || weights >= (uint64_t{1} << 40)) return LaunchStatus::kInvalid;
    const int rows = b0->cb->fsm_rows;
    if (rows < 2 || rows > kFsmMaxRows || b0->cb->min_len_used < 2) return LaunchStatus::kUnsupported;
    const ImageLayout L0 = image_layout(*b0);
    P.meta = reinterpret_cast<const uint32_t *>(b0->dev_image + L0.meta);
    P.syms = reinterpret_cast<const uint32_t *>(b0->dev_image + L0.syms);
    P.lut = reinterpret_cast<const uint16_t *>(b0->dev_image + L0.lut);
    P.fsm = reinterpret_cast<const uint32_t *>(b0->dev_image + L0.fsm);
    P.err = err;
    P.wait_ns = 2000000000ull;
    P.fsm_rows = rows;
    P.n_luts = b0->cb->n_luts();
    P.n_mats = n;
    P.m = m;
    P.mpad = (m + 15) / 16 * 16;
    if (max_span > kKTile) return LaunchStatus::kUnsupported;  // a tile's codes must touch <= 2 operand tiles
    P.max_span = static_cast<uint32_t>(max_span);
    P.total_kt = static_cast<uint32_t>(kts);
    // slots: 3 activation tiles (8 when an operand tile holds fewer than 64
    // columns), operand tiles as many as fit, 4..32 (3 activation slots
    // instead of 4 leave room for a seventh operand slot on the block at
    // M = 16: 0.305 vs 0.311 ms)
    P.exps_bytes = gemm_exps_bytes(P.max_span);
    P.b_slots = kGemmTileK >= 64 ? 3 : 8;
    const uint32_t budget = 227u * 1024u - 1024u;  // opt-in shared memory less the alignment slack
    P.a_slots = kMaxASlots;
    while (P.a_slots > 4 && make_gemm_plan(rows, P.mpad, P.a_slots, P.b_slots, P.exps_bytes).total > budget)
        --P.a_slots;
    if (make_gemm_plan(rows, P.mpad, P.a_slots, P.b_slots, P.exps_bytes).total > budget)
        return LaunchStatus::kUnsupported;
    P.a_magic = static_cast<uint32_t>(((uint64_t{1} << 32) + P.a_slots - 1) / P.a_slots);
    P.b_magic = static_cast<uint32_t>(((uint64_t{1} << 32) + P.b_slots - 1) / P.b_slots);
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || !gemm_prepare(dev, &sms)) return LaunchStatus::kCuda;
    const uint32_t grid = static_cast<uint32_t>(std::min<uint64_t>({static_cast<uint64_t>(sms), kts,
                                                                     static_cast<uint64_t>(kGemmMaxCtas)}));
    for (uint32_t c = 0; c <= grid; ++c) P.cta_kt[c] = static_cast<uint32_t>(kts * c / grid);
    for (uint32_t c = 0; c < grid; ++c) {
        P.cta_vt[c][0] = tile_at(jobs, P.mt, n, static_cast<uint64_t>(P.cta_kt[c]) * kKTile, false);
        P.cta_vt[c][1] = tile_at(jobs, P.mt, n, static_cast<uint64_t>(P.cta_kt[c + 1]) * kKTile, true);
    }
    if (with_maps) {
        EncodeTiledFn enc = encode_tiled();
        if (!enc) return LaunchStatus::kCuda;
        for (int i = 0; i < n; ++i) {
            const cuuint64_t dims[2] = {jobs[i].k, static_cast<cuuint64_t>(m)};
            const cuuint64_t strides[1] = {jobs[i].k * 2};
            const cuuint32_t box[2] = {static_cast<cuuint32_t>(kGemmTileK), static_cast<cuuint32_t>(P.mpad)};
            const cuuint32_t estr[2] = {1, 1};
            if (enc(&P.xmap[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(jobs[i].x), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    kRowBytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                     : (kRowBytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B),
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return LaunchStatus::kInvalid;
        }
    }
    out->shape.grid = static_cast<int>(grid);
    out->shape.block = kGemmThreads;
    out->shape.smem =
        static_cast<int>(make_gemm_plan(rows, P.mpad, P.a_slots, P.b_slots, P.exps_bytes).total + 1024u);
    out->shape.a_slots = P.a_slots;
    out->shape.b_slots = P.b_slots;
    return LaunchStatus::kOk;
}

}  // namespace

void gemm_tile_weights(const uint16_t *w, uint64_t k, uint64_t n, uint16_t *tiled, int n_threads) {
    const uint64_t kt = k / kGemmTileK, nt = n / kGemmTileN;
    parallel_for(nt * kt, n_threads, [&](uint64_t b, uint64_t e) {
        for (uint64_t t = b; t < e; ++t) {
            const uint64_t nb = t / kt, kb = t % kt;
            uint16_t *dst = tiled + t * kKTile;
            for (uint64_t r = 0; r < kGemmTileN; ++r)
                for (uint64_t c = 0; c < kGemmTileK; ++c)
                    dst[r * kGemmTileK + c] = w[(kb * kGemmTileK + c) * n + nb * kGemmTileN + r];
        }
    });
}

LaunchStatus gemm_launch_shape(const GemmJob *jobs, int n, int m, GemmShape *out) {
    GemmPrepared pp;
    const LaunchStatus st = build_gemm(jobs, n, m, nullptr, false, &pp);
    if (st == LaunchStatus::kOk) *out = pp.shape;
    return st;
}

LaunchStatus launch_decode_gemm(const GemmJob *jobs, int n, int m, int *err, cudaStream_t s) {
    GemmPrepared pp;
    const LaunchStatus st = build_gemm(jobs, n, m, err, true, &pp);
    if (st != LaunchStatus::kOk) return st;
    decode_gemm_kernel<<<pp.shape.grid, pp.shape.block, pp.shape.smem, s>>>(pp.params);
    if (cudaGetLastError() != cudaSuccess) return LaunchStatus::kCuda;
    return LaunchStatus::kOk;
}

}  // namespace df11
