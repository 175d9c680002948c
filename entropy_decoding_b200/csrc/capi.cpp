// capi.cpp -- the extern "C" boundary of libdf11 (declared in include/df11.h).
// Argument checking and object lifetimes live here; the arithmetic lives in
// codec.cpp (host) and decode.cu (device).
#include <cuda_runtime_api.h>

#include <cstring>
#include <mutex>
#include <new>

#include "df11.h"
#include "codec.h"
#include "encode.h"
#include "gemm.h"
#include "launch.h"
#include "rans.h"

struct df11_codebook {
    std::shared_ptr<df11::Codebook> cb;
};

struct df11_blob {
    df11::Blob b;
};

struct df11_encoding {
    df11::EncodeJob job;
    uint64_t *scratch = nullptr;
    cudaStream_t stream = nullptr;
    uint64_t total_bits = 0;
    uint64_t image_bytes = 0;
    bool packed = false;
};

namespace {

bool valid_dtype(df11_dtype d) { return d == DF11_BF16 || d == DF11_FP8_E4M3; }
bool valid_encode_flags(int flags) { return (flags & ~DF11_ENCODE_NO_CHUNK_COUNTS) == 0; }

df11_status from_launch(df11::LaunchStatus s) {
    switch (s) {
        case df11::LaunchStatus::kOk: return DF11_OK;
        case df11::LaunchStatus::kInvalid: return DF11_EINVAL;
        case df11::LaunchStatus::kUnsupported: return DF11_EUNSUPPORTED;
        default: return DF11_ECUDA;
    }
}

// Events of df11_decode_streamed, created once per device: per slot, "copy
// done" (recorded on the copy stream) and "slot free" (recorded on the decode
// stream after the decode that read the slot).  Every call re-records them,
// so one call's enqueue loop runs under its device's g_enqueue_mu: a wait
// then always refers to a record made earlier by the same call (or by a call
// that finished enqueueing before it started, which only adds an ordering),
// never to a record another thread makes between this call's record and wait.
constexpr int kStreamSlots = 8;
constexpr int kEventDevices = 64;
std::mutex g_event_mu;
cudaEvent_t g_events[kEventDevices][2 * kStreamSlots] = {};
std::mutex g_enqueue_mu[kEventDevices];

cudaEvent_t *stream_events() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kEventDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_event_mu);
    if (!g_events[dev][0]) {
        for (int i = 0; i < 2 * kStreamSlots; ++i)
            if (cudaEventCreateWithFlags(&g_events[dev][i], cudaEventDisableTiming) != cudaSuccess) return nullptr;
    }
    return g_events[dev];
}

df11_status gemm_jobs(const df11_gemm_matrix *mats, int n_mats, bool stand_ins, df11::GemmJob *jobs) {
    if (!mats || n_mats < 1 || n_mats > DF11_GEMM_MAX_MATS) return DF11_EINVAL;
    for (int i = 0; i < n_mats; ++i) {
        if (!mats[i].weights) return DF11_EINVAL;
        jobs[i].w = &mats[i].weights->b;
        jobs[i].k = mats[i].k;
        jobs[i].n = mats[i].n;
        // the shape does not depend on x and y: 16-byte aligned stand-ins when absent
        jobs[i].x = stand_ins && !mats[i].x ? reinterpret_cast<const void *>(uintptr_t{256}) : mats[i].x;
        jobs[i].y = stand_ins && !mats[i].y ? reinterpret_cast<float *>(uintptr_t{256}) : mats[i].y;
    }
    return DF11_OK;
}

}  // namespace

extern "C" {

int df11_version(void) { return 10000; }

const char *df11_status_string(df11_status s) {
    switch (s) {
        case DF11_OK: return "ok";
        case DF11_EINVAL: return "invalid argument";
        case DF11_ENOMEM: return "out of memory or buffer too small";
        case DF11_ECUDA: return "CUDA error";
        case DF11_ECORRUPT: return "corrupt container";
        case DF11_EUNSUPPORTED: return "unsupported";
    }
    return "unknown status";
}

df11_status df11_build_codebook(df11_dtype dtype, const void *const *host_tensors, const uint64_t *n_elems,
                                int n_tensors, int max_code_len, df11_codebook **out) {
    if (!out || !valid_dtype(dtype) || n_tensors < 0 || (n_tensors > 0 && (!host_tensors || !n_elems)))
        return DF11_EINVAL;
    if (max_code_len == 0) max_code_len = df11::kMaxCodeLen;
    if (max_code_len < 1 || max_code_len > df11::kMaxCodeLen) return DF11_EINVAL;
    *out = nullptr;
    try {
        uint64_t counts[256] = {};
        for (int i = 0; i < n_tensors; ++i) {
            if (n_elems[i] && !host_tensors[i]) return DF11_EINVAL;
            df11::histogram(dtype, host_tensors[i], n_elems[i], counts, 0);
        }
        uint8_t lengths[256] = {};
        if (!df11::code_lengths(counts, df11::nsym_of(dtype), max_code_len, lengths)) return DF11_EINVAL;
        auto cb = df11::make_codebook(dtype, lengths);
        if (!cb) return DF11_EINVAL;
        *out = new df11_codebook{cb};
        return DF11_OK;
    } catch (const std::bad_alloc &) {
        return DF11_ENOMEM;
    }
}

df11_status df11_codebook_from_lengths(df11_dtype dtype, const uint8_t *lengths, int n_lengths,
                                       df11_codebook **out) {
    if (!out || !lengths || !valid_dtype(dtype) || n_lengths != df11::nsym_of(dtype)) return DF11_EINVAL;
    *out = nullptr;
    try {
        uint8_t l[256] = {};
        std::memcpy(l, lengths, static_cast<size_t>(n_lengths));
        auto cb = df11::make_codebook(dtype, l);
        if (!cb) return DF11_EINVAL;
        *out = new df11_codebook{cb};
        return DF11_OK;
    } catch (const std::bad_alloc &) {
        return DF11_ENOMEM;
    }
}

df11_status df11_codebook_lengths(const df11_codebook *cb, uint8_t *lengths) {
    if (!cb || !lengths) return DF11_EINVAL;
    std::memcpy(lengths, cb->cb->lengths, 256);
    return DF11_OK;
}

void df11_codebook_free(df11_codebook *cb) { delete cb; }

df11_status df11_encode_ex(const df11_codebook *cb, const void *host_src, uint64_t n_elems, int chunk_bits,
                           int tile_threads, int flags, int n_threads, df11_blob **out) {
    if (!cb || !out || (n_elems && !host_src) || n_threads < 0) return DF11_EINVAL;
    if (!df11::valid_layout(chunk_bits, tile_threads) || !valid_encode_flags(flags)) return DF11_EINVAL;
    *out = nullptr;
    try {
        auto *blob = new df11_blob;
        std::string err = df11::encode(cb->cb, host_src, n_elems, chunk_bits, tile_threads, n_threads,
                                       !(flags & DF11_ENCODE_NO_CHUNK_COUNTS), &blob->b);
        if (!err.empty()) {
            delete blob;
            return DF11_EINVAL;
        }
        *out = blob;
        return DF11_OK;
    } catch (const std::bad_alloc &) {
        return DF11_ENOMEM;
    }
}

df11_status df11_encode(const df11_codebook *cb, const void *host_src, uint64_t n_elems, df11_blob **out) {
    return df11_encode_ex(cb, host_src, n_elems, 128, 32, 0, 0, out);
}

int df11_layout_supported(df11_dtype dtype, int chunk_bits, int tile_threads) {
    if (!valid_dtype(dtype)) return 0;
    return df11::kernel_available(dtype, chunk_bits, tile_threads) ? 1 : 0;
}

void df11_blob_free(df11_blob *blob) { delete blob; }

df11_status df11_blob_get_info(const df11_blob *blob, df11_blob_info *info) {
    if (!blob || !info) return DF11_EINVAL;
    const df11::Blob &b = blob->b;
    std::memset(info, 0, sizeof *info);
    info->dtype = b.dtype;
    info->chunk_bits = b.chunk_bits;
    info->tile_threads = b.tile_threads;
    info->max_code_len = b.cb->max_len_used;
    info->n_elems = b.n;
    info->total_bits = b.total_bits;
    info->n_tiles = b.n_tiles;
    info->max_span = b.max_span;
    info->stream_bytes = (b.total_bits + 7) / 8;
    info->plane_bytes = df11::plane_bytes(b.dtype, b.n);
    info->gaps_bytes = b.n_tiles * static_cast<uint64_t>(b.tile_threads);
    info->out_off_bytes = (b.n_tiles + 1) * 8;
    info->serialized_bytes = df11::serialized_bytes(b);
    info->device_bytes = df11::image_layout(b).total;
    info->uncompressed_bytes = b.dtype == df11::kBF16 ? 2 * b.n : b.n;
    info->counts_bytes = b.chunk_counts ? b.n_tiles * static_cast<uint64_t>(b.tile_threads) : 0;
    return DF11_OK;
}

uint64_t df11_blob_compressed_bytes(const df11_blob *blob) { return blob ? df11::serialized_bytes(blob->b) : 0; }

df11_status df11_blob_sections(const df11_blob *blob, const uint8_t **stream, const uint8_t **plane,
                               const uint8_t **gaps, const uint64_t **out_off) {
    if (!blob || blob->b.device_only) return DF11_EINVAL;
    if (stream) *stream = blob->b.stream.data();
    if (plane) *plane = blob->b.plane.data();
    if (gaps) *gaps = blob->b.gaps.data();
    if (out_off) *out_off = blob->b.out_off.data();
    return DF11_OK;
}

df11_status df11_blob_chunk_counts(const df11_blob *blob, const uint8_t **counts) {
    if (!blob || !counts || blob->b.device_only) return DF11_EINVAL;
    *counts = blob->b.chunk_counts ? blob->b.counts.data() : nullptr;
    return DF11_OK;
}

df11_status df11_blob_lengths(const df11_blob *blob, uint8_t *lengths) {
    if (!blob || !lengths) return DF11_EINVAL;
    std::memcpy(lengths, blob->b.cb->lengths, 256);
    return DF11_OK;
}

df11_status df11_serialize(const df11_blob *blob, void *buf, uint64_t cap, uint64_t *used) {
    if (!blob || blob->b.device_only) return DF11_EINVAL;
    uint64_t need = df11::serialized_bytes(blob->b);
    if (used) *used = need;
    if (!buf || cap < need) return DF11_ENOMEM;
    df11::serialize(blob->b, static_cast<uint8_t *>(buf));
    return DF11_OK;
}

df11_status df11_deserialize(const void *buf, uint64_t len, df11_blob **out) {
    if (!buf || !out) return DF11_EINVAL;
    *out = nullptr;
    try {
        auto *blob = new df11_blob;
        std::string err = df11::deserialize(static_cast<const uint8_t *>(buf), len, &blob->b);
        if (!err.empty()) {
            delete blob;
            return DF11_ECORRUPT;
        }
        *out = blob;
        return DF11_OK;
    } catch (const std::bad_alloc &) {
        return DF11_ENOMEM;
    }
}

df11_status df11_blob_device_image(const df11_blob *blob, void *host_dst, uint64_t cap) {
    if (!blob || !host_dst || blob->b.device_only) return DF11_EINVAL;
    if (cap < df11::image_layout(blob->b).total) return DF11_ENOMEM;
    df11::write_image(blob->b, static_cast<uint8_t *>(host_dst));
    return DF11_OK;
}

df11_status df11_blob_bind(df11_blob *blob, const void *dev_image, uint64_t cap) {
    if (!blob || !dev_image) return DF11_EINVAL;
    if (reinterpret_cast<uintptr_t>(dev_image) % df11::kImageAlign) return DF11_EINVAL;
    if (cap < df11::image_layout(blob->b).total) return DF11_ENOMEM;
    blob->b.dev_image = static_cast<const uint8_t *>(dev_image);
    blob->b.dev_cap = cap;
    return DF11_OK;
}

df11_status df11_blob_upload(df11_blob *blob, void *dev_dst, uint64_t cap, df11_stream stream) {
    if (!blob || !dev_dst || blob->b.device_only) return DF11_EINVAL;
    if (reinterpret_cast<uintptr_t>(dev_dst) % df11::kImageAlign) return DF11_EINVAL;
    const uint64_t need = df11::image_layout(blob->b).total;
    if (cap < need) return DF11_ENOMEM;
    try {
        blob->b.host_image.resize(need);
    } catch (const std::bad_alloc &) {
        return DF11_ENOMEM;
    }
    df11::write_image(blob->b, blob->b.host_image.data());
    if (cudaMemcpyAsync(dev_dst, blob->b.host_image.data(), need, cudaMemcpyHostToDevice,
                        reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return DF11_ECUDA;
    blob->b.dev_image = static_cast<const uint8_t *>(dev_dst);
    blob->b.dev_cap = cap;
    return DF11_OK;
}

df11_status df11_decode_ex(const df11_blob *const *blobs, void *const *dst_dev, int n_blobs, int *dev_err_flag,
                           df11_stream stream, const df11_decode_opts *opts) {
    if (!blobs || !dst_dev || n_blobs < 1 || n_blobs > df11::kMaxTensorsPerLaunch) return DF11_EINVAL;
    const df11::Blob *bs[df11::kMaxTensorsPerLaunch];
    for (int i = 0; i < n_blobs; ++i) {
        if (!blobs[i]) return DF11_EINVAL;
        bs[i] = &blobs[i]->b;
    }
    df11::DecodeOptions o;
    if (opts) {
        o.chunks_per_thread = opts->chunks_per_thread;
        o.ctas_per_sm = opts->ctas_per_sm;
        o.warps_per_cta = opts->warps_per_cta;
        o.walker = opts->walker;
        o.max_ctas = opts->max_ctas;
        o.overlap = opts->overlap;
        o.diag_expire_waits = opts->diag_expire_waits;
        o.count_walk = opts->count_walk;
        o.diag_check_bounds = opts->diag_check_bounds;
        if (o.chunks_per_thread < 0 || o.ctas_per_sm < 0 || o.warps_per_cta < 0 || o.walker < 0 ||
            o.walker > DF11_WALKER_BYTE_STEP || o.max_ctas < 0 || o.overlap < 0 || o.overlap > 1 ||
            o.diag_expire_waits < 0 || o.diag_expire_waits > 1 || o.count_walk < 0 || o.count_walk > 1 ||
            o.diag_check_bounds < 0 || o.diag_check_bounds > 1)
            return DF11_EINVAL;
    }
    return from_launch(df11::launch_decode(bs, dst_dev, n_blobs, dev_err_flag, o,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

df11_status df11_decode(const df11_blob *const *blobs, void *const *dst_dev, int n_blobs, int *dev_err_flag,
                        df11_stream stream) {
    return df11_decode_ex(blobs, dst_dev, n_blobs, dev_err_flag, stream, nullptr);
}

df11_status df11_decode_host(df11_blob *const *blobs, const void *const *host_images, void *const *dev_images,
                             void *const *dst_dev, void *const *dst_host, int n_blobs, int *dev_err_flag,
                             df11_stream stream) {
    if (!blobs || !host_images || !dev_images || !dst_dev || !dst_host || n_blobs < 1 ||
        n_blobs > df11::kMaxTensorsPerLaunch)
        return DF11_EINVAL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    for (int i = 0; i < n_blobs; ++i) {
        if (!blobs[i] || !host_images[i] || !dev_images[i] || !dst_host[i]) return DF11_EINVAL;
        const uint64_t need = df11::image_layout(blobs[i]->b).total;
        if (reinterpret_cast<uintptr_t>(dev_images[i]) % df11::kImageAlign) return DF11_EINVAL;
        if (cudaMemcpyAsync(dev_images[i], host_images[i], need, cudaMemcpyHostToDevice, s) != cudaSuccess)
            return DF11_ECUDA;
        blobs[i]->b.dev_image = static_cast<const uint8_t *>(dev_images[i]);
        blobs[i]->b.dev_cap = need;
    }
    df11_status st = df11_decode(reinterpret_cast<const df11_blob *const *>(blobs), dst_dev, n_blobs,
                                 dev_err_flag, stream);
    if (st != DF11_OK) return st;
    for (int i = 0; i < n_blobs; ++i) {
        const df11::Blob &b = blobs[i]->b;
        const uint64_t bytes = b.dtype == df11::kBF16 ? 2 * b.n : b.n;
        if (bytes && cudaMemcpyAsync(dst_host[i], dst_dev[i], bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
            return DF11_ECUDA;
    }
    return DF11_OK;
}

df11_status df11_decode_streamed(df11_blob *const *blobs, const int32_t *group_sizes, int n_groups,
                                 const void *const *host_images, void *const *slots, int n_slots,
                                 uint64_t slot_bytes, void *const *dst_dev, int *dev_err_flag,
                                 df11_stream copy_stream, df11_stream decode_stream) {
    if (!blobs || !group_sizes || n_groups < 1 || !host_images || !slots || n_slots < 1 ||
        n_slots > kStreamSlots || !dst_dev)
        return DF11_EINVAL;
    // check every group before enqueueing anything
    int at = 0;
    for (int g = 0; g < n_groups; ++g) {
        const int k = group_sizes[g];
        if (k < 1 || k > df11::kMaxTensorsPerLaunch) return DF11_EINVAL;
        uint64_t need = 0;
        for (int i = at; i < at + k; ++i) {
            if (!blobs[i] || !host_images[i]) return DF11_EINVAL;
            // one launch per group: one code and one layout in it
            const df11::Blob &b = blobs[i]->b, &f = blobs[at]->b;
            if (b.dtype != f.dtype || b.chunk_bits != f.chunk_bits || b.tile_threads != f.tile_threads ||
                std::memcmp(b.cb->lengths, f.cb->lengths, sizeof b.cb->lengths) != 0)
                return DF11_EINVAL;
            need += df11::align_up(df11::image_layout(b).total, df11::kImageAlign);
        }
        if (need > slot_bytes) return DF11_ENOMEM;
        at += k;
    }
    for (int s = 0; s < n_slots; ++s)
        if (!slots[s] || reinterpret_cast<uintptr_t>(slots[s]) % df11::kImageAlign) return DF11_EINVAL;
    cudaEvent_t *ev = stream_events();
    if (!ev) return DF11_ECUDA;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DF11_ECUDA;
    std::lock_guard<std::mutex> enqueue_lock(g_enqueue_mu[dev]);  // dev < kEventDevices: stream_events checked
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(copy_stream);
    cudaStream_t ds = reinterpret_cast<cudaStream_t>(decode_stream);
    at = 0;
    for (int g = 0; g < n_groups; ++g) {
        const int s = g % n_slots, k = group_sizes[g];
        cudaEvent_t copied = ev[2 * s], freed = ev[2 * s + 1];
        // the slot's previous group has been decoded
        if (cudaStreamWaitEvent(cs, freed, 0) != cudaSuccess) return DF11_ECUDA;
        uint8_t *dst = static_cast<uint8_t *>(slots[s]);
        for (int i = at; i < at + k; ++i) {
            df11::Blob &b = blobs[i]->b;
            const uint64_t bytes = df11::image_layout(b).total;
            if (cudaMemcpyAsync(dst, host_images[i], bytes, cudaMemcpyHostToDevice, cs) != cudaSuccess)
                return DF11_ECUDA;
            b.dev_image = dst;
            b.dev_cap = bytes;
            dst += df11::align_up(bytes, df11::kImageAlign);
        }
        if (cudaEventRecord(copied, cs) != cudaSuccess || cudaStreamWaitEvent(ds, copied, 0) != cudaSuccess)
            return DF11_ECUDA;
        const df11_status st = df11_decode(reinterpret_cast<const df11_blob *const *>(blobs + at), dst_dev + at, k,
                                           dev_err_flag, decode_stream);
        if (st != DF11_OK) return st;
        if (cudaEventRecord(freed, ds) != cudaSuccess) return DF11_ECUDA;
        at += k;
    }
    return DF11_OK;
}

df11_status df11_gemm_tile_weights(const uint16_t *host_w, uint64_t k, uint64_t n, uint16_t *host_tiled) {
    if (!host_w || !host_tiled || k == 0 || n == 0 || k % DF11_GEMM_TILE_K || n % DF11_GEMM_TILE_N) return DF11_EINVAL;
    if (k > (uint64_t{1} << 40) / n) return DF11_EINVAL;
    const uint8_t *a = reinterpret_cast<const uint8_t *>(host_w), *b = reinterpret_cast<const uint8_t *>(host_tiled);
    if (a < b + 2 * k * n && b < a + 2 * k * n) return DF11_EINVAL;  // the buffers overlap
    df11::gemm_tile_weights(host_w, k, n, host_tiled, 0);
    return DF11_OK;
}

df11_status df11_decode_gemm(const df11_gemm_matrix *mats, int n_mats, int m, int *dev_err_flag,
                             df11_stream stream) {
    df11::GemmJob jobs[df11::kGemmMaxMats];
    const df11_status st = gemm_jobs(mats, n_mats, false, jobs);
    if (st != DF11_OK) return st;
    return from_launch(df11::launch_decode_gemm(jobs, n_mats, m, dev_err_flag, reinterpret_cast<cudaStream_t>(stream)));
}

df11_status df11_decode_gemm_launch_shape(const df11_gemm_matrix *mats, int n_mats, int m, int *grid, int *block,
                                          int *smem_bytes) {
    df11::GemmJob jobs[df11::kGemmMaxMats];
    const df11_status st = gemm_jobs(mats, n_mats, true, jobs);
    if (st != DF11_OK) return st;
    df11::GemmShape sh;
    const df11::LaunchStatus ls = df11::gemm_launch_shape(jobs, n_mats, m, &sh);
    if (ls != df11::LaunchStatus::kOk) return from_launch(ls);
    if (grid) *grid = sh.grid;
    if (block) *block = sh.block;
    if (smem_bytes) *smem_bytes = sh.smem;
    return DF11_OK;
}

df11_status df11_decode_launch_shape(const df11_blob *const *blobs, int n_blobs, int *grid, int *block,
                                     int *smem_bytes) {
    return df11_decode_launch_shape_ex(blobs, n_blobs, nullptr, grid, block, smem_bytes, nullptr, nullptr);
}

df11_status df11_decode_launch_shape_ex(const df11_blob *const *blobs, int n_blobs, const df11_decode_opts *opts,
                                        int *grid, int *block, int *smem_bytes, int *walker,
                                        int *stored_counts) {
    if (!blobs || n_blobs < 1 || n_blobs > df11::kMaxTensorsPerLaunch) return DF11_EINVAL;
    const df11::Blob *bs[df11::kMaxTensorsPerLaunch];
    for (int i = 0; i < n_blobs; ++i) {
        if (!blobs[i]) return DF11_EINVAL;
        bs[i] = &blobs[i]->b;
    }
    df11::LaunchShape sh;
    df11::DecodeOptions o;
    if (opts) {
        o.chunks_per_thread = opts->chunks_per_thread;
        o.ctas_per_sm = opts->ctas_per_sm;
        o.warps_per_cta = opts->warps_per_cta;
        o.walker = opts->walker;
        o.max_ctas = opts->max_ctas;
        o.count_walk = opts->count_walk;
        if (o.chunks_per_thread < 0 || o.ctas_per_sm < 0 || o.warps_per_cta < 0 || o.walker < 0 ||
            o.walker > DF11_WALKER_BYTE_STEP || o.max_ctas < 0 || o.count_walk < 0 || o.count_walk > 1)
            return DF11_EINVAL;
    }
    df11::LaunchStatus st = df11::decode_launch_shape(bs, n_blobs, o, &sh);
    if (st != df11::LaunchStatus::kOk) return from_launch(st);
    if (grid) *grid = sh.grid;
    if (block) *block = sh.block;
    if (smem_bytes) *smem_bytes = sh.smem;
    if (walker) *walker = sh.walker;
    if (stored_counts) *stored_counts = sh.stored_counts;
    return DF11_OK;
}

// ---------------------------------------------------------------- GPU encoder

df11_status df11_histogram_device(df11_dtype dtype, const void *src_dev, uint64_t n_elems, uint64_t *counts_dev,
                                  df11_stream stream) {
    if (!valid_dtype(dtype) || !counts_dev || (n_elems && !src_dev)) return DF11_EINVAL;
    if (reinterpret_cast<uintptr_t>(src_dev) % 16) return DF11_EINVAL;
    return df11::launch_histogram(dtype, src_dev, n_elems, counts_dev, reinterpret_cast<cudaStream_t>(stream))
               ? DF11_OK
               : DF11_ECUDA;
}

df11_status df11_codebook_from_counts(df11_dtype dtype, const uint64_t *counts, int n_counts, int max_code_len,
                                      df11_codebook **out) {
    if (!out || !counts || !valid_dtype(dtype) || n_counts != df11::nsym_of(dtype)) return DF11_EINVAL;
    if (max_code_len == 0) max_code_len = df11::kMaxCodeLen;
    if (max_code_len < 1 || max_code_len > df11::kMaxCodeLen) return DF11_EINVAL;
    *out = nullptr;
    try {
        uint64_t c[256] = {};
        std::memcpy(c, counts, static_cast<size_t>(n_counts) * 8);
        uint8_t lengths[256] = {};
        if (!df11::code_lengths(c, n_counts, max_code_len, lengths)) return DF11_EINVAL;
        auto cb = df11::make_codebook(dtype, lengths);
        if (!cb) return DF11_EINVAL;
        *out = new df11_codebook{cb};
        return DF11_OK;
    } catch (const std::bad_alloc &) {
        return DF11_ENOMEM;
    }
}

uint64_t df11_encode_device_scratch_bytes(uint64_t n_elems) { return df11::encode_scratch_bytes(n_elems); }

df11_status df11_encode_device_begin(const df11_codebook *cb, const void *src_dev, uint64_t n_elems, int chunk_bits,
                                     int tile_threads, int flags, void *scratch_dev, uint64_t scratch_cap,
                                     df11_stream stream, uint64_t *image_bytes, df11_encoding **out) {
    if (!cb || !out || !image_bytes || !scratch_dev || (n_elems && !src_dev)) return DF11_EINVAL;
    if (!df11::valid_layout(chunk_bits, tile_threads) || !valid_encode_flags(flags)) return DF11_EINVAL;
    if (reinterpret_cast<uintptr_t>(src_dev) % 16 || reinterpret_cast<uintptr_t>(scratch_dev) % 16) return DF11_EINVAL;
    if (scratch_cap < df11::encode_scratch_bytes(n_elems)) return DF11_ENOMEM;
    *out = nullptr;
    try {
        auto *enc = new df11_encoding;
        enc->job.cb = cb->cb;
        enc->job.src = src_dev;
        enc->job.n = n_elems;
        enc->job.chunk_bits = chunk_bits;
        enc->job.tile_threads = tile_threads;
        enc->job.chunk_counts = !(flags & DF11_ENCODE_NO_CHUNK_COUNTS) && df11::counts_fit(chunk_bits);
        enc->scratch = static_cast<uint64_t *>(scratch_dev);
        enc->stream = reinterpret_cast<cudaStream_t>(stream);
        const df11::EncodeError err = df11::encode_device_bits(enc->job, enc->scratch, enc->stream, &enc->total_bits);
        if (err != df11::EncodeError::kOk) {
            delete enc;
            return err == df11::EncodeError::kUncovered ? DF11_EINVAL : DF11_ECUDA;
        }
        df11::Blob meta;
        meta.dtype = cb->cb->dtype;
        meta.chunk_bits = chunk_bits;
        meta.tile_threads = tile_threads;
        meta.n = n_elems;
        meta.total_bits = enc->total_bits;
        const uint64_t cbits = static_cast<uint64_t>(chunk_bits);
        meta.n_tiles = ((enc->total_bits + cbits - 1) / cbits + tile_threads - 1) / tile_threads;
        meta.cb = cb->cb;
        meta.chunk_counts = enc->job.chunk_counts;
        enc->image_bytes = df11::image_layout(meta).total;
        *image_bytes = enc->image_bytes;
        *out = enc;
        return DF11_OK;
    } catch (const std::bad_alloc &) {
        return DF11_ENOMEM;
    }
}

df11_status df11_encode_device_end(df11_encoding *enc, void *image_dev, uint64_t image_cap, df11_blob **out) {
    if (!enc || !image_dev || !out || enc->packed) return DF11_EINVAL;
    if (reinterpret_cast<uintptr_t>(image_dev) % df11::kImageAlign) return DF11_EINVAL;
    if (image_cap < enc->image_bytes) return DF11_ENOMEM;
    *out = nullptr;
    try {
        auto *blob = new df11_blob;
        df11::Blob &b = blob->b;
        b.dtype = enc->job.cb->dtype;
        b.chunk_bits = enc->job.chunk_bits;
        b.tile_threads = enc->job.tile_threads;
        b.n = enc->job.n;
        b.total_bits = enc->total_bits;
        const uint64_t cbits = static_cast<uint64_t>(b.chunk_bits);
        b.n_tiles = ((b.total_bits + cbits - 1) / cbits + b.tile_threads - 1) / b.tile_threads;
        b.cb = enc->job.cb;
        b.chunk_counts = enc->job.chunk_counts;
        b.device_only = true;
        const df11::ImageLayout L = df11::image_layout(b);
        if (b.n) {
            const df11::EncodeError err = df11::encode_device_pack(enc->job, enc->scratch, b.total_bits, L,
                                                                   static_cast<uint8_t *>(image_dev), enc->stream,
                                                                   &b.max_span);
            if (err != df11::EncodeError::kOk) {
                delete blob;
                return DF11_ECUDA;
            }
        } else {
            std::vector<uint8_t> img(L.total, 0);
            df11::write_image_head(b, L, img.data());
            if (cudaMemcpyAsync(image_dev, img.data(), img.size(), cudaMemcpyHostToDevice, enc->stream) !=
                    cudaSuccess ||
                cudaStreamSynchronize(enc->stream) != cudaSuccess) {
                delete blob;
                return DF11_ECUDA;
            }
        }
        b.dev_image = static_cast<const uint8_t *>(image_dev);
        b.dev_cap = image_cap;
        enc->packed = true;
        *out = blob;
        return DF11_OK;
    } catch (const std::bad_alloc &) {
        return DF11_ENOMEM;
    }
}

void df11_encoding_free(df11_encoding *enc) { delete enc; }

df11_status df11_blob_fetch(df11_blob *blob, df11_stream stream) {
    if (!blob || !blob->b.dev_image) return DF11_EINVAL;
    if (!blob->b.device_only) return DF11_OK;
    try {
        const df11::ImageLayout L = df11::image_layout(blob->b);
        std::vector<uint8_t> img(L.total);
        cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
        if (cudaMemcpyAsync(img.data(), blob->b.dev_image, L.total, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return DF11_ECUDA;
        df11::read_image_sections(blob->b, img.data());
        return DF11_OK;
    } catch (const std::bad_alloc &) {
        return DF11_ENOMEM;
    }
}

df11_status df11_encode_device_noalloc(const df11_codebook *cb, const void *src_dev, uint64_t n_elems,
                                       int chunk_bits, int tile_threads, int flags, void *image_dev,
                                       uint64_t image_cap, df11_stream stream, df11_encode_result *result) {
    if (!cb || !result || !image_dev || (n_elems && !src_dev)) return DF11_EINVAL;
    if (!df11::valid_layout(chunk_bits, tile_threads) || !valid_encode_flags(flags)) return DF11_EINVAL;
    if (n_elems > df11::noalloc_max_elems()) return DF11_EINVAL;
    if (reinterpret_cast<uintptr_t>(src_dev) % 16 || reinterpret_cast<uintptr_t>(image_dev) % df11::kImageAlign)
        return DF11_EINVAL;
    df11::EncodeJob job;
    job.cb = cb->cb;
    job.src = src_dev;
    job.n = n_elems;
    job.chunk_bits = chunk_bits;
    job.tile_threads = tile_threads;
    job.chunk_counts = !(flags & DF11_ENCODE_NO_CHUNK_COUNTS) && df11::counts_fit(chunk_bits);
    df11::NoallocResult r{};
    const df11::EncodeError err = df11::encode_device_noalloc(job, static_cast<uint8_t *>(image_dev), image_cap,
                                                              reinterpret_cast<cudaStream_t>(stream), &r);
    result->image_bytes = r.image_bytes;
    result->total_bits = r.total_bits;
    result->n_tiles = r.n_tiles;
    result->max_span = r.max_span;
    switch (err) {
        case df11::EncodeError::kOk: return DF11_OK;
        case df11::EncodeError::kTooSmall: return DF11_ENOMEM;
        case df11::EncodeError::kUncovered: return DF11_EINVAL;
        default: return DF11_ECUDA;
    }
}

// ---------------------------------------------------------------- rANS coder

struct df11_rans_group {
    df11::RansGroup g;
};

df11_status df11_rans_encode_group(df11_dtype dtype, const void *const *host_tensors, const uint64_t *n_elems,
                                   int n_tensors, int tile_symbols, int n_threads, df11_rans_group **out) {
    if (!out || !valid_dtype(dtype) || n_tensors < 1 || n_tensors > 64 || !host_tensors || !n_elems ||
        n_threads < 0 || tile_symbols < 0)
        return DF11_EINVAL;
    *out = nullptr;
    try {
        auto *g = new df11_rans_group;
        const uint32_t ts = tile_symbols ? static_cast<uint32_t>(tile_symbols) : DF11_RANS_TILE_DEFAULT;
        const std::string err = df11::rans_encode_group(dtype, host_tensors, n_elems, n_tensors, ts, n_threads, &g->g);
        if (!err.empty()) {
            delete g;
            return DF11_EINVAL;
        }
        *out = g;
        return DF11_OK;
    } catch (const std::bad_alloc &) {
        return DF11_ENOMEM;
    }
}

void df11_rans_group_free(df11_rans_group *g) { delete g; }

df11_status df11_rans_group_freqs(const df11_rans_group *g, uint32_t *freqs) {
    if (!g || !freqs) return DF11_EINVAL;
    std::memcpy(freqs, g->g.freqs, sizeof g->g.freqs);
    return DF11_OK;
}

df11_status df11_rans_group_info(const df11_rans_group *g, int tensor, df11_rans_tensor_info *info) {
    if (!g || !info || tensor < 0 || tensor >= static_cast<int>(g->g.tensors.size())) return DF11_EINVAL;
    const df11::RansTensor &t = g->g.tensors[tensor];
    info->n_elems = t.n;
    info->n_tiles = t.n_tiles;
    info->words = t.words.size();
    info->coded_bytes = t.words.size() * 2 + t.states.size() * 4 + t.tile_words.size() * 8;
    info->plane_bytes = t.plane.size();
    info->uncompressed_bytes = g->g.dtype == df11::kBF16 ? 2 * t.n : t.n;
    return DF11_OK;
}

df11_status df11_rans_group_sections(const df11_rans_group *g, int tensor, const uint16_t **words,
                                     const uint32_t **states, const uint64_t **tile_words, const uint8_t **plane) {
    if (!g || tensor < 0 || tensor >= static_cast<int>(g->g.tensors.size())) return DF11_EINVAL;
    const df11::RansTensor &t = g->g.tensors[tensor];
    if (words) *words = t.words.data();
    if (states) *states = t.states.data();
    if (tile_words) *tile_words = t.tile_words.data();
    if (plane) *plane = t.plane.data();
    return DF11_OK;
}

df11_status df11_rans_group_serialize(const df11_rans_group *g, void *buf, uint64_t cap, uint64_t *used) {
    if (!g) return DF11_EINVAL;
    const uint64_t need = df11::rans_serialized_bytes(g->g);
    if (used) *used = need;
    if (!buf || cap < need) return DF11_ENOMEM;
    df11::rans_serialize(g->g, static_cast<uint8_t *>(buf));
    return DF11_OK;
}

df11_status df11_rans_group_deserialize(const void *buf, uint64_t len, df11_rans_group **out) {
    if (!buf || !out) return DF11_EINVAL;
    *out = nullptr;
    try {
        auto *g = new df11_rans_group;
        if (!df11::rans_deserialize(static_cast<const uint8_t *>(buf), len, &g->g).empty()) {
            delete g;
            return DF11_ECORRUPT;
        }
        *out = g;
        return DF11_OK;
    } catch (const std::bad_alloc &) {
        return DF11_ENOMEM;
    }
}

uint64_t df11_rans_group_device_bytes(const df11_rans_group *g) {
    if (!g) return 0;
    uint64_t total = 0;
    df11::rans_layout(g->g, &total);
    return total;
}

df11_status df11_rans_group_upload(df11_rans_group *g, void *dev_dst, uint64_t cap, df11_stream stream) {
    if (!g || !dev_dst || reinterpret_cast<uintptr_t>(dev_dst) % df11::kImageAlign) return DF11_EINVAL;
    const uint64_t need = df11_rans_group_device_bytes(g);
    if (cap < need) return DF11_ENOMEM;
    try {
        g->g.host_image.resize(need);
    } catch (const std::bad_alloc &) {
        return DF11_ENOMEM;
    }
    df11::rans_write_image(g->g, g->g.host_image.data());
    if (cudaMemcpyAsync(dev_dst, g->g.host_image.data(), need, cudaMemcpyHostToDevice,
                        reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return DF11_ECUDA;
    g->g.dev_image = static_cast<const uint8_t *>(dev_dst);
    g->g.dev_cap = cap;
    return DF11_OK;
}

df11_status df11_rans_decode(const df11_rans_group *g, void *const *dst_dev, int *dev_err_flag, df11_stream stream) {
    if (!g || !dst_dev) return DF11_EINVAL;
    switch (df11::rans_launch_decode(g->g, dst_dev, dev_err_flag, reinterpret_cast<cudaStream_t>(stream), nullptr,
                                     nullptr, nullptr)) {
    case df11::RansLaunch::kOk: return DF11_OK;
    case df11::RansLaunch::kInvalid: return DF11_EINVAL;
    default: return DF11_ECUDA;
    }
}

df11_status df11_rans_decode_launch_shape(const df11_rans_group *g, int *grid, int *block, int *smem_bytes) {
    if (!g) return DF11_EINVAL;
    switch (df11::rans_launch_decode(g->g, nullptr, nullptr, nullptr, grid, block, smem_bytes)) {
    case df11::RansLaunch::kOk: return DF11_OK;
    case df11::RansLaunch::kInvalid: return DF11_EINVAL;
    default: return DF11_ECUDA;
    }
}

}  // extern "C"
