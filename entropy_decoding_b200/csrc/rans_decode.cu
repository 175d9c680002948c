// rans_decode.cu -- GPU decode of the rANS exponent coder (format in rans.h).
//
// One warp decodes one tile at a time (a contiguous run of tiles per warp):
// its 32 lanes are the tile's 32 interleaved coders.  A step decodes 32
// consecutive symbols, one per lane, through the 4096-entry slot table in
// shared memory; the lanes whose state fell below 2^16 take the next words
// of the tile's stream in lane order (a ballot and a population count give
// each its word).  The words reach shared memory through a per-warp ring of
// 1024 words filled 256 words at a time, each chunk loaded into registers one
// refill ahead.  Every 8 steps (16 for E4M3) the warp merges the decoded
// exponents with the raw plane and writes 16 bytes per lane.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "df11.h"
#include "df11_internal.h"
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

__device__ __forceinline__ void st_v4(void *p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// 4 plane bytes (sign << 7 | mantissa) and 4 exponents -> 4 BF16 (two words).
__device__ __forceinline__ void bf16x4(uint32_t p, uint32_t e, uint32_t &w0, uint32_t &w1) {
    const uint32_t hi = (p & 0x80808080u) | ((e >> 1) & 0x7F7F7F7Fu);  // sign | exponent bits 7..1
    const uint32_t lo = ((e << 7) & 0x80808080u) | (p & 0x7F7F7F7Fu);  // exponent bit 0 | mantissa
    w0 = __byte_perm(lo, hi, 0x5140);
    w1 = __byte_perm(lo, hi, 0x7362);
}

// 4 plane nibbles (sign << 3 | mantissa, element i in bits 4i..4i+3) and 4
// exponents -> 4 E4M3 bytes.
__device__ __forceinline__ uint32_t e4m3x4(uint32_t nib, uint32_t e) {
    uint32_t w = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t q = (nib >> (4 * i)) & 0xFu, x = (e >> (8 * i)) & 0xFu;
        w |= (((q & 8u) << 4) | (x << 3) | (q & 7u)) << (8 * i);
    }
    return w;
}

template <int DT, int NWARP>
__global__ void __launch_bounds__(NWARP * 32, 1) rans_decode_kernel(const __grid_constant__ RansParams P) {
    constexpr uint32_t G = DT == 0 ? 8u : 16u;  // steps per merge group
    constexpr uint32_t GW = G * 32u;             // symbols per group, and the most words it can take
    constexpr uint32_t WARP_BYTES = kRing * 2u + GW;
    extern __shared__ __align__(16) uint8_t smem[];
    uint32_t *s_tab = reinterpret_cast<uint32_t *>(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint16_t *ring = reinterpret_cast<uint16_t *>(smem + kRansM * 4u + warp * WARP_BYTES);
    uint8_t *s_ex = smem + kRansM * 4u + warp * WARP_BYTES + kRing * 2u;
    for (int i = tid; i < static_cast<int>(kRansM / 4); i += NWARP * 32)
        reinterpret_cast<uint4 *>(s_tab)[i] = __ldg(reinterpret_cast<const uint4 *>(P.table) + i);
    __syncthreads();

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
        const uint64_t wb = d.tile_words[lt], we = d.tile_words[lt + 1];
        if (wb > we || we > d.words_len || (wb & 7u)) {
            err |= DF11_DEV_ERR_AUX;
            continue;
        }
        uint32_t x = d.states[static_cast<uint64_t>(lt) * 32u + lane];
        const uint16_t *ws = d.words + wb;  // 16-byte aligned: wb is a multiple of 8 words
        const uint64_t avail = d.words_len + kRansWordsTail - wb;
        // chunk c = words [256 c, 256 c + 256) of the tile, lane's 8 of them;
        // nothing is read past the section's tail
        auto load_chunk = [&](uint32_t c) -> uint4 {
            const uint64_t w0 = static_cast<uint64_t>(c) * kRansChunkWords + 8u * lane;
            return w0 + 8u <= avail ? ld_nc_v4(ws + w0) : make_uint4(0, 0, 0, 0);
        };
        reinterpret_cast<uint4 *>(ring)[lane] = load_chunk(0);
        uint4 pf = load_chunk(1);
        uint32_t loaded = 1;  // chunks [0, loaded) have entered the ring (the last 4 are in it)
        uint32_t ptr = 0;     // words taken
        const uint32_t steps = (m + 31u) / 32u;
        uint8_t *out = static_cast<uint8_t *>(d.dst);
        for (uint32_t k0 = 0; k0 < steps; k0 += G) {
            // the ring must hold words [ptr, ptr + GW): refill by chunks; a
            // chunk's slot is reused only once every word of it was taken
            while (loaded * kRansChunkWords < ptr + GW) {
                reinterpret_cast<uint4 *>(ring + (loaded & 3u) * kRansChunkWords)[lane] = pf;
                ++loaded;
                pf = load_chunk(loaded);
            }
            __syncwarp();
            const uint64_t g0 = e0 + static_cast<uint64_t>(k0) * 32u;  // first weight of the group
            const uint2 pl = ld_nc_v2(d.plane + (DT == 0 ? g0 : g0 / 2u) + 8u * lane);
#pragma unroll
            for (uint32_t s = 0; s < G; ++s) {
                const bool act = (k0 + s) * 32u + lane < m;
                const uint32_t slot = x & (kRansM - 1u);
                const uint32_t e = s_tab[slot];
                uint32_t xn = (((e >> 8) & 0xFFFu) + 1u) * (x >> kRansBits) + slot - (e >> 20);
                if (!act) xn = x;
                const bool need = act && xn < kRansL;
                const uint32_t mask = __ballot_sync(0xFFFFFFFFu, need);
                if (need) xn = (xn << 16) | ring[(ptr + __popc(mask & below)) & (kRing - 1u)];
                ptr += __popc(mask);
                x = xn;
                s_ex[s * 32u + lane] = static_cast<uint8_t>(e);
            }
            __syncwarp();
            // merge: weights [g0, g0 + cnt) of the tile's output
            const uint32_t cnt = min(GW, m - k0 * 32u);
            if constexpr (DT == 0) {
                const uint2 ex = *reinterpret_cast<const uint2 *>(s_ex + 8u * lane);
                uint4 o;
                bf16x4(pl.x, ex.x, o.x, o.y);
                bf16x4(pl.y, ex.y, o.z, o.w);
                uint8_t *dp = out + 2u * (g0 + 8u * lane);
                if (8u * lane + 8u <= cnt) {
                    st_v4(dp, o);
                } else {
                    const uint32_t v[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
                    for (uint32_t j = 0; j < 8; ++j)
                        if (8u * lane + j < cnt)
                            reinterpret_cast<uint16_t *>(dp)[j] = static_cast<uint16_t>(v[j >> 1] >> (16 * (j & 1)));
                }
            } else {
                const uint4 ex = *reinterpret_cast<const uint4 *>(s_ex + 16u * lane);
                uint4 o;
                o.x = e4m3x4(pl.x, ex.x);
                o.y = e4m3x4(pl.x >> 16, ex.y);
                o.z = e4m3x4(pl.y, ex.z);
                o.w = e4m3x4(pl.y >> 16, ex.w);
                uint8_t *dp = out + g0 + 16u * lane;
                if (16u * lane + 16u <= cnt) {
                    st_v4(dp, o);
                } else {
                    const uint32_t v[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
                    for (uint32_t j = 0; j < 16; ++j)
                        if (16u * lane + j < cnt) dp[j] = static_cast<uint8_t>(v[j >> 2] >> (8 * (j & 3)));
                }
            }
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

uint32_t rans_smem_bytes(int dtype) {
    const uint32_t gw = (dtype == DF11_BF16 ? 8u : 16u) * 32u;
    return kRansM * 4u + kRansWarps * (kRing * 2u + gw);
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
