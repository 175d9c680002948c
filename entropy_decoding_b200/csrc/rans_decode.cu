// rans_decode.cu -- GPU decode of the rANS exponent coder (format in rans.h).
//
// One warp decodes one tile at a time (a contiguous run of tiles per warp):
// its 32 lanes are the tile's 32 interleaved coders.  A step decodes 32
// consecutive symbols, one per lane, through the 4096-entry slot table in
// shared memory (entry: symbol, f - 1 and slot - c, so the state update is
// one multiply-add and one add); the lanes whose state fell below 2^16 take
// the next words of the tile's stream in lane order (a ballot and a
// population count give each its word).  The words reach shared memory
// through a per-warp ring of 1024 words filled 256 words at a time, each
// chunk loaded into registers one refill ahead; the ring's first words are
// mirrored after its end, so a group of steps reads it without wrapping.
// Every 16 steps the warp merges the decoded exponents with the raw plane
// (loaded one group ahead) and writes 32 (BF16) or 16 (E4M3) bytes per lane.
// Groups whose steps all have 32 symbols take a path without per-lane checks.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "check.cuh"
#include "df11.h"
#include "df11_internal.h"
#include "merge.cuh"
#include "rans.h"

namespace df11 {
namespace {

constexpr int kRansMaxTensors = 64;
constexpr uint32_t kRing = 1024;  // words in a warp's ring: 4 chunks
constexpr int kRansWarps = 32;

struct RansTensorDesc {
    const uint32_t *states;
    const uint64_t *tile_words;
    const uint16_t *words;  // followed by kRansWordsTail readable zero words
    const uint8_t *plane;   // followed by kRansPlaneTail readable bytes
    void *dst;
    uint64_t n;
    uint64_t words_len;
    uint32_t n_tiles;
    uint32_t tile_begin;
};

struct RansParams {
    const uint32_t *table;
    int *err;
    uint32_t tile_symbols;
    uint32_t total_tiles;
    int32_t n_tensors;
    RansTensorDesc t[kRansMaxTensors];
};

__device__ __forceinline__ uint4 ld_nc_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint2 ld_nc_v2(const void *p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// A ring word (written by this warp before the __syncwarp that precedes
// the group; the address depends on the step's ballot, so the load cannot
// move above it).
__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
    uint16_t v;
    asm("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ void st_v4(void *p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// G steps of the tile's 32 coders from step k0 on.  FULL: every step has 32
// symbols (no per-lane check); else lane j decodes in step k only when
// 32 k + j < m.  x: the lane's state; ra: the shared-memory address of the
// next word in the ring (below the ring's end at the group's start; the
// mirror covers the group's reads); the exponents go to s_ex[32 s + lane].
// Ring reads are checked against [ring_lo, ring_lo + ring_bytes) in the
// bounds-checked build.
template <uint32_t G, bool FULL>
__device__ __forceinline__ void decode_group(uint32_t &x, uint32_t &ra, uint32_t k0, uint32_t m, int lane,
                                             uint32_t below, const uint32_t *s_tab, uint8_t *s_ex, uint32_t ring_lo,
                                             uint32_t ring_bytes, uint32_t &err) {
#pragma unroll
    for (uint32_t s = 0; s < G; ++s) {
        const uint32_t e = s_tab[x & (kRansM - 1u)];
        const uint32_t q = x >> kRansBits;
        uint32_t xn = q * ((e >> 8) & 0xFFFu) + q + (e >> 20);  // f floor(x / M) + slot - c
        bool need;
        if constexpr (FULL) {
            need = xn < kRansL;
        } else {
            const bool act = (k0 + s) * 32u + static_cast<uint32_t>(lane) < m;
            if (!act) xn = x;
            need = act && xn < kRansL;
        }
        const uint32_t mask = __ballot_sync(0xFFFFFFFFu, need);
        const uint32_t wa = ra + 2u * __popc(mask & below);
        if (need && in_bounds(wa - ring_lo, 2, ring_bytes, err))
            xn = __byte_perm(lds_u16(wa), xn, 0x5410);  // xn << 16 | word
        ra += 2u * __popc(mask);
        x = xn;
        s_ex[s * 32u + lane] = static_cast<uint8_t>(e);
    }
}

template <int DT, int NWARP>
__global__ void __launch_bounds__(NWARP * 32, 1) rans_decode_kernel(const __grid_constant__ RansParams P) {
    constexpr uint32_t G = 16u;                 // steps per merge group
    constexpr uint32_t GW = G * 32u;             // symbols per group, and the most words it can take
    constexpr uint32_t WARP_BYTES = (kRing + GW) * 2u + GW;
    extern __shared__ __align__(16) uint8_t smem[];
    uint32_t *s_tab = reinterpret_cast<uint32_t *>(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint16_t *ring = reinterpret_cast<uint16_t *>(smem + kRansM * 4u + warp * WARP_BYTES);
    uint8_t *s_ex = smem + kRansM * 4u + warp * WARP_BYTES + (kRing + GW) * 2u;
    for (int i = tid; i < static_cast<int>(kRansM / 4); i += NWARP * 32)
        reinterpret_cast<uint4 *>(s_tab)[i] = __ldg(reinterpret_cast<const uint4 *>(P.table) + i);
    __syncthreads();
    const uint32_t ring_addr = smem_u32(ring);

    const uint32_t nwt = gridDim.x * NWARP;
    const uint32_t per = (P.total_tiles + nwt - 1) / nwt;
    const uint32_t t_begin = min((blockIdx.x * NWARP + warp) * per, P.total_tiles);
    const uint32_t t_end = min(t_begin + per, P.total_tiles);
    const uint32_t below = (1u << lane) - 1u;
    uint32_t err = 0;
    int ti = 0;
    for (uint32_t t = t_begin; t < t_end; ++t) {
        while (ti + 1 < P.n_tensors && t >= P.t[ti + 1].tile_begin) ++ti;
        const RansTensorDesc &d = P.t[ti];
        const uint32_t lt = t - d.tile_begin;
        const uint64_t e0 = static_cast<uint64_t>(lt) * P.tile_symbols;
        const uint32_t m = static_cast<uint32_t>(min(static_cast<uint64_t>(P.tile_symbols), d.n - e0));
        if (!in_bounds(lt, 2, static_cast<uint64_t>(d.n_tiles) + 1u, err)) continue;
        const uint64_t wb = d.tile_words[lt], we = d.tile_words[lt + 1];
        if (wb > we || we > d.words_len || (wb & 7u)) {
            err |= DF11_DEV_ERR_AUX;
            continue;
        }
        uint32_t x = in_bounds(static_cast<uint64_t>(lt) * 32u + lane, 1, static_cast<uint64_t>(d.n_tiles) * 32u, err)
                         ? d.states[static_cast<uint64_t>(lt) * 32u + lane]
                         : kRansL;
        // readable plane bytes (the section plus its tail) and output bytes,
        // for the bounds-checked build
        const uint64_t plane_cap = (DT == 0 ? d.n : (d.n + 1) / 2) + kRansPlaneTail;
        const uint64_t out_cap = d.n * (DT == 0 ? 2u : 1u);
        const uint16_t *ws = d.words + wb;  // 16-byte aligned: wb is a multiple of 8 words
        const uint64_t avail = d.words_len + kRansWordsTail - wb;
        // chunk c = words [256 c, 256 c + 256) of the tile, lane's 8 of them;
        // nothing is read past the section's tail
        auto load_chunk = [&](uint32_t c) -> uint4 {
            const uint64_t w0 = static_cast<uint64_t>(c) * kRansChunkWords + 8u * lane;
            return w0 + 8u <= avail ? ld_nc_v4(ws + w0) : make_uint4(0, 0, 0, 0);
        };
        // chunk c into its ring slot (c % 4), and into the mirror after the
        // ring when the slot holds the ring's first GW words
        auto put_chunk = [&](uint32_t c, uint4 v) {
            const uint32_t slot = c & 3u;
            reinterpret_cast<uint4 *>(ring + slot * kRansChunkWords)[lane] = v;
            if (slot * kRansChunkWords < GW) reinterpret_cast<uint4 *>(ring + kRing + slot * kRansChunkWords)[lane] = v;
        };
        // the lane's plane bytes of the group starting at step k: 16 (BF16:
        // weights 16 lane .. 16 lane + 15 of the group) or 8 (E4M3: 16 nibbles)
        const uint8_t *pl_lane = d.plane + (DT == 0 ? e0 + 16u * lane : e0 / 2u + 8u * lane);
        auto plane_of = [&](uint32_t k) -> uint4 {
            const uint64_t off = static_cast<uint64_t>(pl_lane - d.plane) + (DT == 0 ? 32u : 16u) * k;
            if (!in_bounds(off, DT == 0 ? 16u : 8u, plane_cap, err)) return make_uint4(0u, 0u, 0u, 0u);
            if constexpr (DT == 0) {
                return ld_nc_v4(pl_lane + 32u * k);
            } else {
                const uint2 v = ld_nc_v2(pl_lane + 16u * k);
                return make_uint4(v.x, v.y, 0u, 0u);
            }
        };
        put_chunk(0, load_chunk(0));
        uint4 pf = load_chunk(1);
        uint32_t loaded = 1;  // chunks [0, loaded) have entered the ring (the last 4 are in it)
        uint32_t ptr = 0;     // words taken
        const uint32_t steps = (m + 31u) / 32u, full_steps = m / 32u;
        uint8_t *out = static_cast<uint8_t *>(d.dst);
        uint4 pl = plane_of(0);
        for (uint32_t k0 = 0; k0 < steps; k0 += G) {
            // the ring must hold words [ptr, ptr + GW): refill by chunks; a
            // chunk's slot is reused only once every word of it was taken
            while (loaded * kRansChunkWords < ptr + GW) {
                put_chunk(loaded, pf);
                ++loaded;
                pf = load_chunk(loaded);
            }
            __syncwarp();
            // the next group's plane bytes now: they arrive while this group decodes
            const uint4 pl_next = k0 + G < steps ? plane_of(k0 + G) : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t ra0 = ring_addr + 2u * (ptr & (kRing - 1u));
            uint32_t ra = ra0;
            if (k0 + G <= full_steps)
                decode_group<G, true>(x, ra, k0, m, lane, below, s_tab, s_ex, ring_addr, (kRing + GW) * 2u, err);
            else
                decode_group<G, false>(x, ra, k0, m, lane, below, s_tab, s_ex, ring_addr, (kRing + GW) * 2u, err);
            ptr += (ra - ra0) >> 1;
            __syncwarp();
            // merge: weights [g0, g0 + cnt) of the tile's output
            const uint64_t g0 = e0 + static_cast<uint64_t>(k0) * 32u;
            const uint32_t cnt = min(GW, m - k0 * 32u);
            if constexpr (DT == 0) {
                const uint4 ex = *reinterpret_cast<const uint4 *>(s_ex + 16u * lane);
                uint4 o, o2;
                merge_bf16x4(pl.x, ex.x, o.x, o.y);
                merge_bf16x4(pl.y, ex.y, o.z, o.w);
                merge_bf16x4(pl.z, ex.z, o2.x, o2.y);
                merge_bf16x4(pl.w, ex.w, o2.z, o2.w);
                uint8_t *dp = out + 2u * (g0 + 16u * lane);
                const uint32_t nw = 16u * lane < cnt ? min(16u, cnt - 16u * lane) : 0u;  // weights this lane stores
                if (!in_bounds_or_empty(2u * (g0 + 16u * lane), 2u * nw, out_cap, err)) {
                } else if (16u * lane + 16u <= cnt) {
                    st_v4(dp, o);
                    st_v4(dp + 16, o2);
                } else {
                    const uint32_t v[8] = {o.x, o.y, o.z, o.w, o2.x, o2.y, o2.z, o2.w};
#pragma unroll
                    for (uint32_t j = 0; j < 16; ++j)
                        if (16u * lane + j < cnt)
                            reinterpret_cast<uint16_t *>(dp)[j] = static_cast<uint16_t>(v[j >> 1] >> (16 * (j & 1)));
                }
            } else {
                const uint4 ex = *reinterpret_cast<const uint4 *>(s_ex + 16u * lane);
                uint4 o;
                merge_e4m3x8(pl.x, ex.x, ex.y, o.x, o.y);
                merge_e4m3x8(pl.y, ex.z, ex.w, o.z, o.w);
                uint8_t *dp = out + g0 + 16u * lane;
                const uint32_t nw = 16u * lane < cnt ? min(16u, cnt - 16u * lane) : 0u;  // weights this lane stores
                if (!in_bounds_or_empty(g0 + 16u * lane, nw, out_cap, err)) {
                } else if (16u * lane + 16u <= cnt) {
                    st_v4(dp, o);
                } else {
                    const uint32_t v[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
                    for (uint32_t j = 0; j < 16; ++j)
                        if (16u * lane + j < cnt) dp[j] = static_cast<uint8_t>(v[j >> 2] >> (8 * (j & 3)));
                }
            }
            pl = pl_next;
            __syncwarp();
        }
        // every coder back at 2^16, and the tile's words taken up to its padding
        if (!__all_sync(0xFFFFFFFFu, x == kRansL) || ptr > we - wb || we - wb - ptr >= 8u)
            err |= DF11_DEV_ERR_SPAN;
    }
    err = __reduce_or_sync(0xFFFFFFFFu, err);
    if (lane == 0 && err && P.err) atomicOr(P.err, static_cast<int>(err));
}

using RansFn = void (*)(RansParams);

std::mutex g_rans_mu;
constexpr int kMaxDev = 64;
bool g_rans_attr[kMaxDev][2] = {};
int g_rans_sms[kMaxDev] = {};

uint32_t rans_smem_bytes(int) {
    const uint32_t gw = 16u * 32u;
    return kRansM * 4u + kRansWarps * ((kRing + gw) * 2u + gw);
}

}  // namespace

RansLaunch rans_launch_decode(const RansGroup &g, void *const *dst, int *err, cudaStream_t s, int *grid_out,
                              int *block_out, int *smem_out) {
    const int nt = static_cast<int>(g.tensors.size());
    if (!g.dev_image || nt < 1 || nt > kRansMaxTensors) return RansLaunch::kInvalid;
    uint64_t total = 0;
    const auto L = rans_layout(g, &total);
    if (g.dev_cap < total) return RansLaunch::kInvalid;
    RansParams P{};
    P.table = reinterpret_cast<const uint32_t *>(g.dev_image);
    P.err = err;
    P.tile_symbols = g.tile_symbols;
    uint64_t tiles = 0;
    int k = 0;
    for (int i = 0; i < nt; ++i) {
        const RansTensor &t = g.tensors[i];
        if (!t.n) continue;
        if (dst && (!dst[i] || reinterpret_cast<uintptr_t>(dst[i]) % 16)) return RansLaunch::kInvalid;
        RansTensorDesc &d = P.t[k++];
        d.states = reinterpret_cast<const uint32_t *>(g.dev_image + L[i].states);
        d.tile_words = reinterpret_cast<const uint64_t *>(g.dev_image + L[i].tile_words);
        d.words = reinterpret_cast<const uint16_t *>(g.dev_image + L[i].words);
        d.plane = g.dev_image + L[i].plane;
        d.dst = dst ? dst[i] : nullptr;
        d.n = t.n;
        d.words_len = t.words.size();
        d.n_tiles = static_cast<uint32_t>(t.n_tiles);
        d.tile_begin = static_cast<uint32_t>(tiles);
        tiles += t.n_tiles;
    }
    if (tiles >= (uint64_t{1} << 31)) return RansLaunch::kInvalid;
    P.n_tensors = k;
    P.total_tiles = static_cast<uint32_t>(tiles);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return RansLaunch::kCuda;
    const RansFn fn = g.dtype == DF11_BF16 ? &rans_decode_kernel<0, kRansWarps> : &rans_decode_kernel<1, kRansWarps>;
    const uint32_t smem = rans_smem_bytes(g.dtype);
    {
        std::lock_guard<std::mutex> lk(g_rans_mu);
        if (!g_rans_sms[dev] &&
            cudaDeviceGetAttribute(&g_rans_sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return RansLaunch::kCuda;
        bool &set = g_rans_attr[dev][g.dtype == DF11_BF16 ? 0 : 1];
        if (!set) {
            if (cudaFuncSetAttribute(reinterpret_cast<const void *>(fn), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem)) != cudaSuccess)
                return RansLaunch::kCuda;
            set = true;
        }
    }
    const uint64_t need = (tiles + kRansWarps - 1) / kRansWarps;
    const int grid = static_cast<int>(need < static_cast<uint64_t>(g_rans_sms[dev]) ? need : g_rans_sms[dev]);
    if (grid_out) *grid_out = grid;
    if (block_out) *block_out = kRansWarps * 32;
    if (smem_out) *smem_out = static_cast<int>(smem);
    if (!dst || tiles == 0) return RansLaunch::kOk;
    fn<<<grid, kRansWarps * 32, smem, s>>>(P);
    return cudaGetLastError() == cudaSuccess ? RansLaunch::kOk : RansLaunch::kCuda;
}

}  // namespace df11
