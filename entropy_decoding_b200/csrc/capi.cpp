// capi.cpp -- the extern "C" boundary of libdf11 (declared in include/df11.h).
// Argument checking and object lifetimes live here; the arithmetic lives in
// codec.cpp (host) and decode.cu (device).
#include <cuda_runtime_api.h>

#include <cstring>
#include <new>

#include "df11.h"
#include "codec.h"
#include "launch.h"

struct df11_codebook {
    std::shared_ptr<df11::Codebook> cb;
};

struct df11_blob {
    df11::Blob b;
};

namespace {

bool valid_dtype(df11_dtype d) { return d == DF11_BF16 || d == DF11_FP8_E4M3; }

df11_status from_launch(df11::LaunchStatus s) {
    switch (s) {
        case df11::LaunchStatus::kOk: return DF11_OK;
        case df11::LaunchStatus::kInvalid: return DF11_EINVAL;
        case df11::LaunchStatus::kUnsupported: return DF11_EUNSUPPORTED;
        default: return DF11_ECUDA;
    }
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
                           int tile_threads, int n_threads, df11_blob **out) {
    if (!cb || !out || (n_elems && !host_src) || n_threads < 0) return DF11_EINVAL;
    if (!df11::valid_layout(chunk_bits, tile_threads)) return DF11_EINVAL;
    *out = nullptr;
    try {
        auto *blob = new df11_blob;
        std::string err = df11::encode(cb->cb, host_src, n_elems, chunk_bits, tile_threads, n_threads, &blob->b);
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
    return df11_encode_ex(cb, host_src, n_elems, 128, 32, 0, out);
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
    info->stream_bytes = b.stream.size();
    info->plane_bytes = b.plane.size();
    info->gaps_bytes = b.gaps.size();
    info->out_off_bytes = b.out_off.size() * 8;
    info->serialized_bytes = df11::serialized_bytes(b);
    info->device_bytes = df11::image_layout(b).total;
    info->uncompressed_bytes = b.dtype == df11::kBF16 ? 2 * b.n : b.n;
    return DF11_OK;
}

df11_status df11_blob_sections(const df11_blob *blob, const uint8_t **stream, const uint8_t **plane,
                               const uint8_t **gaps, const uint64_t **out_off) {
    if (!blob) return DF11_EINVAL;
    if (stream) *stream = blob->b.stream.data();
    if (plane) *plane = blob->b.plane.data();
    if (gaps) *gaps = blob->b.gaps.data();
    if (out_off) *out_off = blob->b.out_off.data();
    return DF11_OK;
}

df11_status df11_blob_lengths(const df11_blob *blob, uint8_t *lengths) {
    if (!blob || !lengths) return DF11_EINVAL;
    std::memcpy(lengths, blob->b.cb->lengths, 256);
    return DF11_OK;
}

df11_status df11_serialize(const df11_blob *blob, void *buf, uint64_t cap, uint64_t *used) {
    if (!blob) return DF11_EINVAL;
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
    if (!blob || !host_dst) return DF11_EINVAL;
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
    if (!blob || !dev_dst) return DF11_EINVAL;
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
        if (o.chunks_per_thread < 0 || o.ctas_per_sm < 0 || o.warps_per_cta < 0) return DF11_EINVAL;
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

df11_status df11_decode_launch_shape(const df11_blob *const *blobs, int n_blobs, int *grid, int *block,
                                     int *smem_bytes) {
    return df11_decode_launch_shape_ex(blobs, n_blobs, nullptr, grid, block, smem_bytes);
}

df11_status df11_decode_launch_shape_ex(const df11_blob *const *blobs, int n_blobs, const df11_decode_opts *opts,
                                        int *grid, int *block, int *smem_bytes) {
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
    }
    df11::LaunchStatus st = df11::decode_launch_shape(bs, n_blobs, o, &sh);
    if (st != df11::LaunchStatus::kOk) return from_launch(st);
    if (grid) *grid = sh.grid;
    if (block) *block = sh.block;
    if (smem_bytes) *smem_bytes = sh.smem;
    return DF11_OK;
}

}  // extern "C"
