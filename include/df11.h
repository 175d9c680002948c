/*
 * df11.h -- C-ABI of libdf11: lossless BF16 / FP8-E4M3 weight compression by
 * Huffman-coding the exponent field, with a B200 (sm_100a) decode kernel.
 *
 * The operations follow "70% Size, 100% Accuracy: Lossless LLM Compression
 * for Efficient GPU Inference via Dynamic-Length Float (DFloat11)", Abstract:
 *   - frequency-based dynamic-length (Huffman) codes for the low-entropy part
 *     of each weight, built offline ............. df11_build_codebook
 *   - the compressed tensor: raw sign+mantissa plane, packed code stream and
 *     lightweight auxiliary variables that coordinate thread read/write
 *     positions ................................. df11_encode
 *   - online GPU decompression with lookup tables in on-chip SRAM and a
 *     two-phase kernel, one launch per transformer block (all matrices of the
 *     block in one launch) ...................... df11_decode
 * and "Compressing LLMs without Compromise" summary page, section "Where the
 * redundancy lives" (BF16 = 1 sign + 8 exponent + 7 mantissa bits; only the
 * exponent is low-entropy) and section "Three ways to spend the savings"
 * (exponents Huffman-coded offline, lookup tables in GPU shared memory);
 * "To Compress or Not? ... Exponent Concentration", Abstract (FP8 variant).
 *
 * Conventions for every function:
 *   - Host pointers are ordinary CPU memory; "device" pointers are CUDA
 *     global-memory addresses of the current device.  No function takes or
 *     returns framework (torch) objects.
 *   - Objects (df11_codebook, df11_blob) are created by the library and owned
 *     by the caller, who frees them with the matching *_free function.  Input
 *     buffers are only read during the call unless stated otherwise.
 *   - Errors are returned synchronously as df11_status; nothing aborts or
 *     prints.  Calls are thread-safe for distinct objects.
 *   - Decoding never allocates memory and never synchronises: the caller
 *     provides every device buffer and owns the stream.
 */
#ifndef DF11_H
#define DF11_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DF11_OK = 0,
    DF11_EINVAL = 1,       /* bad argument (null pointer, size, alignment, mixed codes) */
    DF11_ENOMEM = 2,       /* host allocation failed, or a caller buffer is too small */
    DF11_ECUDA = 3,        /* a CUDA runtime call or kernel launch failed */
    DF11_ECORRUPT = 4,     /* a serialized container failed validation */
    DF11_EUNSUPPORTED = 5  /* a valid request this build has no kernel for */
} df11_status;

typedef enum {
    DF11_BF16 = 0,      /* 16-bit words: sign | 8-bit exponent | 7-bit mantissa */
    DF11_FP8_E4M3 = 1   /* bytes: sign | 4-bit exponent | 3-bit mantissa */
} df11_dtype;

/* Bits the decode kernel ORs into the caller's device error word.  Any
 * non-zero value means some output of that call is not valid; the kernel
 * still never writes outside the destination buffers it was given. */
#define DF11_DEV_ERR_SPAN 1u     /* a tile decoded a different number of codes than its out_off span,
                                    or a chunk a different number than its stored count */
#define DF11_DEV_ERR_CODE 2u     /* the stream held a bit pattern that is no codeword */
#define DF11_DEV_ERR_AUX 4u      /* an auxiliary value (gap, out_off) out of its valid range */
#define DF11_DEV_ERR_TIMEOUT 8u  /* a bounded wait on an on-chip barrier gave up */
#define DF11_DEV_ERR_BOUNDS 16u  /* bounds-checked debug build only (libdf11_check.so, built with
                                    -DDF11_CHECK=1): a shared- or global-memory access fell outside
                                    its buffer or section and was skipped; never set by libdf11.so */

/* Same type as cudaStream_t; pass 0 for the legacy default stream. */
typedef struct CUstream_st *df11_stream;

typedef struct df11_codebook df11_codebook; /* host object: code lengths + decode tables */
typedef struct df11_blob df11_blob;         /* host object: one compressed tensor */
typedef struct df11_encoding df11_encoding; /* host object: a GPU encode between its two steps */

/* Library version: major * 10000 + minor * 100 + patch. */
int df11_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char *df11_status_string(df11_status status);

/* ---------------------------------------------------------------------
 * Codebook  (DFloat11 Abstract: "dynamic-length encodings ... based on
 * frequency"; summary page: "Huffman-codes the exponents offline")
 * ------------------------------------------------------------------ */

/* Builds one code for a group of tensors (e.g. every matrix of one transformer
 * block): the exponent histogram is summed over all n_tensors tensors, Huffman
 * code lengths are computed (ties broken by (count, symbol) with merged nodes
 * after leaves in creation order) and limited to max_code_len bits by
 * package-merge when needed; codes are canonical.
 *   dtype          DF11_BF16 (exponent = 8 bits, 256 symbols) or
 *                  DF11_FP8_E4M3 (4 bits, 16 symbols).
 *   host_tensors   n_tensors host pointers to the raw weights (uint16 words
 *                  for BF16, bytes for E4M3); a pointer may be NULL only when
 *                  its n_elems is 0.
 *   n_elems        n_tensors element counts.
 *   max_code_len   1..32, or 0 for 32; must allow a complete code
 *                  (2^max_code_len >= number of distinct symbols).
 *   out            receives the new codebook (caller frees).
 * Errors: DF11_EINVAL for bad arguments, DF11_ENOMEM. */
df11_status df11_build_codebook(df11_dtype dtype, const void *const *host_tensors,
                                const uint64_t *n_elems, int n_tensors, int max_code_len,
                                df11_codebook **out);

/* Builds a codebook from explicit code lengths (n_lengths = 256 for BF16, 16
 * for E4M3; 0 = symbol unused).  The lengths must form a prefix code (Kraft
 * sum <= 1) with every length <= 32.  Errors: DF11_EINVAL. */
df11_status df11_codebook_from_lengths(df11_dtype dtype, const uint8_t *lengths, int n_lengths,
                                       df11_codebook **out);

/* Copies the code length of every symbol into lengths[0..255] (E4M3 uses the
 * first 16; the rest are 0). */
df11_status df11_codebook_lengths(const df11_codebook *cb, uint8_t *lengths);

void df11_codebook_free(df11_codebook *cb);

/* ---------------------------------------------------------------------
 * Encoding  (DFloat11 Abstract: "lightweight auxiliary variables")
 * ------------------------------------------------------------------ */

/* Compresses one tensor with a codebook (whose code must cover every exponent
 * the tensor holds).  Default layout: chunk_bits = 128 stream bits per decode
 * thread, tile_threads = 32 chunks per tile (one warp: out_off is kept per
 * warp-sized block of threads); all host cores are used.
 * The blob holds, in host memory:
 *   plane    n bytes (BF16: sign << 7 | mantissa) or ceil(n/2) bytes (E4M3:
 *            nibble sign << 3 | mantissa, element 2i in the low nibble)
 *   stream   the canonical codes of the exponents in element order, most
 *            significant bit first (stream bit k = bit 7 - k%8 of byte k/8)
 *   gaps     one byte per chunk: offset of the first code that starts in the
 *            chunk (padded with 0 to whole tiles)
 *   counts   one byte per chunk: the number of codes that start in the chunk
 *            (padded with 0 to whole tiles).  Not in the pages' format: it
 *            lets the decoder place each thread's output with a scan of
 *            stored bytes instead of a first walk over the codes that only
 *            counts them (the first of the two phases of the DFloat11
 *            Abstract, item (ii)).  Costs chunk_bits / 8 : 1 of the stream
 *            (about 0.17 bits per weight at 128-bit chunks); left out with
 *            DF11_ENCODE_NO_CHUNK_COUNTS and for 256-bit chunks.
 *   out_off  n_tiles + 1 uint64 values: codes starting before each tile
 * Errors: DF11_EINVAL (bad layout, or a symbol the code does not cover),
 * DF11_ENOMEM. */
df11_status df11_encode(const df11_codebook *cb, const void *host_src, uint64_t n_elems,
                        df11_blob **out);

/* Flags of df11_encode_ex, df11_encode_device_begin and
 * df11_encode_device_noalloc (0 = the default layout's sections). */
#define DF11_ENCODE_NO_CHUNK_COUNTS 1 /* leave out the counts section: the pages' format, smallest size */

/* df11_encode with an explicit layout: chunk_bits in {64, 128, 256},
 * tile_threads (chunks per tile, one out_off entry each) in {32, 128, 256,
 * 512}; flags from DF11_ENCODE_*; n_threads host threads (0 = all cores).
 * df11_decode supports the layouts listed by df11_layout_supported.  Errors
 * as df11_encode, and DF11_EINVAL for an unknown flag. */
df11_status df11_encode_ex(const df11_codebook *cb, const void *host_src, uint64_t n_elems,
                           int chunk_bits, int tile_threads, int flags, int n_threads, df11_blob **out);

/* 1 when df11_decode has a kernel for this (dtype, chunk_bits, tile_threads). */
int df11_layout_supported(df11_dtype dtype, int chunk_bits, int tile_threads);

void df11_blob_free(df11_blob *blob);

typedef struct {
    int32_t dtype;            /* df11_dtype */
    int32_t chunk_bits;
    int32_t tile_threads;
    int32_t max_code_len;     /* longest code actually used */
    uint64_t n_elems;
    uint64_t total_bits;      /* stream length in bits */
    uint64_t n_tiles;
    uint64_t max_span;        /* most codes that start in one tile */
    uint64_t stream_bytes;    /* ceil(total_bits / 8) */
    uint64_t plane_bytes;
    uint64_t gaps_bytes;
    uint64_t out_off_bytes;
    uint64_t serialized_bytes;/* size of df11_serialize's output: the container */
    uint64_t device_bytes;    /* size of the device image (df11_blob_device_image) */
    uint64_t uncompressed_bytes;
    uint64_t counts_bytes;    /* chunk counts: n_tiles * tile_threads, 0 when the blob has none */
} df11_blob_info;

df11_status df11_blob_get_info(const df11_blob *blob, df11_blob_info *info);

/* Size in bytes of the blob's container (df11_serialize's output: header,
 * code lengths, gaps, chunk counts when present, out_off, stream and plane),
 * the numerator of the compression ratio; equal to info.serialized_bytes.
 * 0 for a NULL blob. */
uint64_t df11_blob_compressed_bytes(const df11_blob *blob);

/* Read-only host views of the blob's sections (valid until the blob is freed);
 * any output pointer may be NULL.  DF11_EINVAL for a GPU-encoded blob that
 * was not fetched (df11_blob_fetch). */
df11_status df11_blob_sections(const df11_blob *blob, const uint8_t **stream, const uint8_t **plane,
                               const uint8_t **gaps, const uint64_t **out_off);

/* *counts receives a read-only host view of the chunk counts
 * (info.counts_bytes bytes), or NULL when the blob has none.  DF11_EINVAL as
 * df11_blob_sections. */
df11_status df11_blob_chunk_counts(const df11_blob *blob, const uint8_t **counts);

/* Copies the code lengths the blob was encoded with into lengths[0..255]. */
df11_status df11_blob_lengths(const df11_blob *blob, uint8_t *lengths);

/* ---------------------------------------------------------------------
 * Container (the offline, on-disk form)
 * ------------------------------------------------------------------ */

/* Writes the container (header with code lengths, gaps, chunk counts when
 * the blob has them, out_off, stream, plane; sections 16-byte aligned) into
 * buf[0..cap): format version 2 with counts, else version 1.  *used receives
 * info.serialized_bytes.  Errors: DF11_ENOMEM when cap is too small. */
df11_status df11_serialize(const df11_blob *blob, void *buf, uint64_t cap, uint64_t *used);

/* Reads a container; validates the header, the code (Kraft sum, lengths),
 * the section sizes and every auxiliary value against the layout rules.
 * Errors: DF11_ECORRUPT for any inconsistency, DF11_ENOMEM. */
df11_status df11_deserialize(const void *buf, uint64_t len, df11_blob **out);

/* ---------------------------------------------------------------------
 * Device image and decoding  (DFloat11 Abstract: hierarchical lookup tables
 * in SRAM, two-phase kernel, transformer-block-level decompression)
 * ------------------------------------------------------------------ */

/* Writes the blob's device image into host memory host_dst[0..cap) (cap >=
 * info.device_bytes; pinned memory makes the later copy asynchronous).  The
 * image is one buffer with 256-byte aligned sections: the decode tables
 * built from the code lengths, gaps, chunk counts (when the blob has them),
 * out_off, the stream padded with zeros to whole tiles plus 16 bytes, and the
 * plane padded to 16 bytes plus 32. */
df11_status df11_blob_device_image(const df11_blob *blob, void *host_dst, uint64_t cap);

/* Records that the blob's device image is at device address dev_image
 * (256-byte aligned, cap >= info.device_bytes), placed there by the caller.
 * The memory stays owned by the caller and must outlive the decodes. */
df11_status df11_blob_bind(df11_blob *blob, const void *dev_image, uint64_t cap);

/* Convenience: builds the image in a host buffer held by the blob, copies it
 * to dev_dst with cudaMemcpyAsync on `stream`, and binds it.  The caller owns
 * dev_dst.  Errors: DF11_EINVAL, DF11_ENOMEM, DF11_ECUDA. */
df11_status df11_blob_upload(df11_blob *blob, void *dev_dst, uint64_t cap, df11_stream stream);

/* Decodes n_blobs bound blobs in ONE kernel launch on `stream`, asynchronously.
 *   blobs        all encoded with the same code lengths, dtype and layout (a
 *                transformer block shares one codebook); otherwise DF11_EINVAL.
 *   dst_dev      n_blobs device pointers, 16-byte aligned, each holding
 *                n_elems * 2 bytes (BF16) or n_elems bytes (E4M3); written
 *                with the exact original bit patterns.  Buffers must not
 *                overlap each other or the images.
 *   n_blobs      1..64 per launch (more: DF11_EINVAL; split the call).
 *   dev_err_flag device int, or NULL.  The kernel ORs DF11_DEV_ERR_* bits into
 *                it when the data is inconsistent; the caller zeroes it.
 * Never allocates, never synchronises.  Errors: DF11_EINVAL (unbound blob,
 * misaligned or NULL pointer, mixed codes), DF11_EUNSUPPORTED (layout without
 * a kernel), DF11_ECUDA (launch failure). */
df11_status df11_decode(const df11_blob *const *blobs, void *const *dst_dev, int n_blobs,
                        int *dev_err_flag, df11_stream stream);

/* Tuning knobs of the decode launch; zero-initialise for the defaults. */
typedef struct {
    int32_t chunks_per_thread; /* CTA-tile layouts: chunks each decoding thread walks, 1 or 2 (0 = 1) */
    int32_t ctas_per_sm;       /* persistent CTAs per SM, capped by occupancy (0 = as many as fit) */
    int32_t warps_per_cta;     /* warp-tile layout (tile_threads 32): warps per CTA; window walker 8 or
                                  16 (0 = 16), byte-step walker 16, 24 or 32 (0 = the most that fit) */
    int32_t walker;            /* warp-tile layout: DF11_WALKER_AUTO (0), DF11_WALKER_WINDOW or
                                  DF11_WALKER_BYTE_STEP; CTA-tile layouts take 0 or WINDOW only.
                                  The window walk always counts with a first walk */
    int32_t max_ctas;          /* upper bound on the grid (0 = none): fewer persistent CTAs leave
                                  SMs free for work running beside the decode */
    int32_t overlap;           /* 1: the launch reads nothing that the work before it on the
                                  stream writes, so it may start while the previous kernel is
                                  still finishing (programmatic dependent launch); 0: ordinary
                                  stream order */
    int32_t diag_expire_waits; /* diagnostics, 0 in normal use.  1: the kernel issues no copies
                                  and gives each of its bounded waits 10 ms instead of 2 s, so
                                  the first wait runs out: the launch decodes nothing, sets
                                  DF11_DEV_ERR_TIMEOUT in dev_err_flag and ends (how a stalled
                                  copy is reported, exercised without a fault) */
    int32_t count_walk;        /* byte-step walker: 0 = place each thread's output with the chunk
                                  counts when every image of the launch stores them, else walk;
                                  1 = always walk each chunk once to count its codes first (the
                                  first phase of the two-phase kernel), ignoring stored counts */
    int32_t diag_check_bounds; /* diagnostics, 0 in normal use; acts in libdf11_check.so only
                                  (libdf11.so ignores it).  1: every exponent-buffer access of
                                  the merge is checked against a bound of 0 bytes, so each is
                                  refused and skipped: the launch writes no output and sets
                                  DF11_DEV_ERR_BOUNDS (shows the checks are live, without a
                                  fault) */
} df11_decode_opts;

/* How a decoding thread walks its chunk (both give the same output).
 * WINDOW: lookups in the 12-bit multi-symbol table, each consuming the
 * whole codes in the next 12 bits (a variable number of bits).
 * BYTE_STEP: lookups in the byte-step transition tables, one per 8 stream
 * bits whatever the code boundaries, so every thread of a warp takes the
 * same number of steps; a thread whose walk reaches the dead row falls back
 * to the window walk.  One CTA per SM holds the tables (up to 128 KB of
 * shared memory).  AUTO picks BYTE_STEP for warp tiles when the code has no
 * 1-bit codeword and the tables fit, else WINDOW. */
#define DF11_WALKER_AUTO 0
#define DF11_WALKER_WINDOW 1
#define DF11_WALKER_BYTE_STEP 2

/* df11_decode with explicit launch options (opts may be NULL).  The result is
 * identical for every option value; only the speed changes. */
df11_status df11_decode_ex(const df11_blob *const *blobs, void *const *dst_dev, int n_blobs,
                           int *dev_err_flag, df11_stream stream, const df11_decode_opts *opts);

/* End-to-end decode from host memory to host memory, all on `stream` and
 * asynchronous (the caller synchronises the stream before reading dst_host):
 * for each blob, cudaMemcpyAsync host_images[i] (its device image, e.g. from
 * df11_blob_device_image into pinned memory) to dev_images[i] and bind it;
 * one df11_decode launch into dst_dev; then cudaMemcpyAsync dst_dev[i] to
 * dst_host[i].  All buffers are the caller's.  Errors as df11_decode. */
df11_status df11_decode_host(df11_blob *const *blobs, const void *const *host_images,
                             void *const *dev_images, void *const *dst_dev, void *const *dst_host,
                             int n_blobs, int *dev_err_flag, df11_stream stream);

/* Decode of weights kept in host memory, streamed group by group: the
 * offloaded-weights case of "70% Size, 100% Accuracy ... (DFloat11)",
 * Abstract (decompression on the GPU of compressed weights), with the
 * transfer of the next group overlapping the decode of the current one.
 *   blobs        n_blobs = sum(group_sizes) blobs, group after group; the
 *                blobs of one group share one code (as in one df11_decode)
 *   group_sizes  n_groups counts, each 1..64
 *   host_images  per blob, its device image (df11_blob_device_image) in
 *                pinned host memory, unchanged until decode_stream completes
 *   slots        n_slots (1..8) device staging buffers of slot_bytes each,
 *                256-byte aligned; group g is copied into slot g % n_slots,
 *                its images packed at 256-byte boundaries
 *   dst_dev      per blob, output as in df11_decode
 *   copy_stream  the host-to-device copies; decode_stream the launches.
 * Group g's copy waits for the decode that last used its slot; its decode
 * waits for its copy, so with 2 slots the copy of group g + 1 overlaps the
 * decode of group g.  Asynchronous; the caller synchronises decode_stream.
 * On return every blob is bound to its place in its slot (rebind before
 * decoding it again: the slot is reused).  Allocates no device memory; the
 * first call on a device creates 2 x 8 CUDA events that live until exit.
 * Calls from several host threads (each with its own streams, slots and
 * blobs) are safe: the library enqueues one call at a time per device, so
 * each copy waits for the right decode.  A call may then also wait for the
 * decodes of a call enqueued before it on other streams (the events are
 * shared); that orders the two calls but never changes an output.
 * Errors: DF11_EINVAL (arguments, group size, mixed codes in a group),
 * DF11_ENOMEM (a group's images exceed slot_bytes), both found before
 * anything is enqueued; DF11_EUNSUPPORTED and DF11_ECUDA (copy, event or
 * launch failure) stop at the failing group, the groups before it staying
 * enqueued (synchronise both streams before reusing the slots). */
df11_status df11_decode_streamed(df11_blob *const *blobs, const int32_t *group_sizes, int n_groups,
                                 const void *const *host_images, void *const *slots, int n_slots,
                                 uint64_t slot_bytes, void *const *dst_dev, int *dev_err_flag,
                                 df11_stream copy_stream, df11_stream decode_stream);

/* Launch shape df11_decode would use for these blobs on the current device:
 * grid (persistent CTAs), threads per CTA and dynamic shared memory bytes.
 * Any output pointer may be NULL. */
df11_status df11_decode_launch_shape(const df11_blob *const *blobs, int n_blobs, int *grid,
                                     int *block, int *smem_bytes);

/* As df11_decode_launch_shape, for the given options (opts may be NULL);
 * *walker (nullable) receives the walk the launch would use,
 * DF11_WALKER_WINDOW or DF11_WALKER_BYTE_STEP, and *stored_counts (nullable)
 * 1 when it places the threads' output with the stored chunk counts, 0 when
 * it walks to count. */
df11_status df11_decode_launch_shape_ex(const df11_blob *const *blobs, int n_blobs,
                                        const df11_decode_opts *opts, int *grid, int *block,
                                        int *smem_bytes, int *walker, int *stored_counts);

/* ---------------------------------------------------------------------
 * GPU encoder (the offline half, run on the device)
 * ------------------------------------------------------------------ */

/* Adds the exponent histogram of a device tensor into counts_dev (device
 * array of 256 uint64 for BF16, 16 for E4M3; the caller zeroes it), on
 * `stream`, asynchronously.  src_dev must be 16-byte aligned.  Errors:
 * DF11_EINVAL, DF11_ECUDA. */
df11_status df11_histogram_device(df11_dtype dtype, const void *src_dev, uint64_t n_elems,
                                  uint64_t *counts_dev, df11_stream stream);

/* Builds a codebook from exponent counts (host array of 256 / 16 uint64, e.g.
 * copied back from df11_histogram_device): the same code construction as
 * df11_build_codebook.  Errors: DF11_EINVAL, DF11_ENOMEM. */
df11_status df11_codebook_from_counts(df11_dtype dtype, const uint64_t *counts, int n_counts,
                                      int max_code_len, df11_codebook **out);

/* Device scratch bytes df11_encode_device_begin needs for n_elems weights
 * (8 bytes per 4096 weights plus 1.3 KB). */
uint64_t df11_encode_device_scratch_bytes(uint64_t n_elems);

/* GPU encode, step 1: computes every code length on the device, scans them
 * and returns the exact device-image size in *image_bytes.  Synchronises
 * `stream` once (to read the stream length back).  src_dev (the raw weights,
 * 16-byte aligned) and scratch_dev (>= df11_encode_device_scratch_bytes,
 * 16-byte aligned) must stay valid until df11_encode_device_end.  flags as
 * df11_encode_ex.  Errors: DF11_EINVAL (bad arguments, or an exponent the
 * code does not cover), DF11_ENOMEM (scratch too small), DF11_ECUDA. */
df11_status df11_encode_device_begin(const df11_codebook *cb, const void *src_dev, uint64_t n_elems,
                                     int chunk_bits, int tile_threads, int flags, void *scratch_dev,
                                     uint64_t scratch_cap, df11_stream stream, uint64_t *image_bytes,
                                     df11_encoding **out);

/* GPU encode, step 2: writes the device image (byte-identical to the one
 * df11_blob_device_image produces for the same tensor and codebook) into
 * image_dev (256-byte aligned, >= *image_bytes of step 1) and returns a blob
 * bound to it, ready for df11_decode.  Synchronises the stream once (to read
 * the largest tile span).  The blob's host sections are empty until
 * df11_blob_fetch.  Errors: DF11_EINVAL, DF11_ENOMEM, DF11_ECUDA. */
df11_status df11_encode_device_end(df11_encoding *enc, void *image_dev, uint64_t image_cap,
                                   df11_blob **out);

void df11_encoding_free(df11_encoding *enc);

/* Copies a GPU-encoded blob's sections back from its device image into host
 * memory (synchronises `stream`), after which df11_serialize,
 * df11_blob_sections and df11_blob_device_image work on it.  A no-op for
 * host-encoded blobs.  Errors: DF11_EINVAL (unbound), DF11_ENOMEM,
 * DF11_ECUDA. */
df11_status df11_blob_fetch(df11_blob *blob, df11_stream stream);

/* ---------------------------------------------------------------------
 * GPU encoding that allocates nothing
 * ------------------------------------------------------------------ */

/* The paper has no counterpart to this call: it exists for programs that
 * cannot allocate device memory at the moment they encode.  Examples are
 * inference servers that reserve nearly all HBM for weights and KV cache at
 * start-up (a cudaMalloc would fail or fragment that pool), and loops that
 * must not pay cudaMalloc/cudaFree's implicit device synchronisation.
 *
 * df11_encode_device_noalloc does what df11_encode_device_begin + _end do and
 * writes the same device image, byte for byte, into the caller's image_dev.
 * It calls no cudaMalloc, cudaFree or other allocating routine, on the device
 * or the host.  The caller passes the raw weights (src_dev, 16-byte aligned)
 * and the image buffer (image_dev, 256-byte aligned, image_cap bytes); flags
 * as df11_encode_ex.
 *
 * Scratch.  Its scratch is one static device array of
 * DF11_NOALLOC_SCRATCH_BYTES, which every GPU that loads the library holds
 * until the process exits.  That bounds n_elems at DF11_NOALLOC_MAX_ELEMS;
 * larger tensors are rejected with DF11_EINVAL before any GPU work.
 *
 * First call per device.  It looks up the array's device address with
 * cudaGetSymbolAddress, with that device current.  Make this first call
 * before any stream capture.  With lazy module loading (the CUDA 12
 * default) that lookup is also when the driver loads the encoder's code and
 * places the array in device memory, so a program that later reserves
 * nearly all HBM should make the first call at start-up, before reserving
 * it (a call with n_elems = 0 and an image buffer of the empty tensor's
 * size is enough).
 *
 * Overlapping calls.  Every call shares the array, and the array keeps the
 * last call's contents (each call clears what must start at zero). Calls
 * that overlap on the GPU, from other threads or on other streams of the
 * same device, race and must be serialised by the caller.
 *
 * Synchronisation.  The call synchronises `stream` (it reads the stream
 * length and the largest tile span back).
 *
 * Result.  *result receives image_bytes, total_bits, n_tiles and max_span.
 * When image_cap < image_bytes the call returns DF11_ENOMEM with
 * result->image_bytes set and the image untouched.
 *
 * Errors: DF11_EINVAL (arguments, size limit, or an exponent the code does
 * not cover), DF11_ENOMEM, DF11_ECUDA. */
#define DF11_NOALLOC_SCRATCH_BYTES (65536ull * 8ull)
#define DF11_NOALLOC_MAX_ELEMS ((65536ull - 163ull) * 4096ull)

typedef struct {
    uint64_t image_bytes; /* device image size this tensor needs */
    uint64_t total_bits;  /* stream length in bits */
    uint64_t n_tiles;
    uint64_t max_span;    /* most codes that start in one tile */
} df11_encode_result;

df11_status df11_encode_device_noalloc(const df11_codebook *cb, const void *src_dev, uint64_t n_elems,
                                       int chunk_bits, int tile_threads, int flags, void *image_dev,
                                       uint64_t image_cap, df11_stream stream,
                                       df11_encode_result *result);

/* ---------------------------------------------------------------------
 * Decode fused into the consuming GEMM  ("Compressing LLMs without
 * Compromise" summary page, ZipServ paragraph: decompression fused into the
 * matrix multiply so the decoded weights go straight to the tensor cores;
 * "Approaching Shannon Bound with Lossless LLM Weight Compression",
 * Abstract: decoding aligned with the GEMM's tiling)
 * ------------------------------------------------------------------ */

/* Operand tile of the fused GEMM: 128 output rows x 64 reduction columns. */
#define DF11_GEMM_TILE_N 128
#define DF11_GEMM_TILE_K 64
#define DF11_GEMM_MAX_MATS 8   /* matrices per df11_decode_gemm launch */
#define DF11_GEMM_MAX_BATCH 64 /* rows of x */

/* Writes the operand-tile order of a K x N BF16 weight matrix (host_w,
 * row-major: element (k, n) at k * N + n, the layer mapping K inputs to N
 * outputs) into host_tiled (K * N words, caller's buffer, not overlapping
 * host_w): tile t = nb * (K / 64) + kb holds outputs n = 128 nb ..
 * 128 nb + 127 and inputs k = 64 kb .. 64 kb + 63, element (r, c) at
 * 8192 t + 64 r + c, i.e. host_w[(64 kb + c) * N + 128 nb + r].  Encoding the
 * result with df11_encode gives the blob df11_decode_gemm consumes; decoding
 * it with df11_decode gives back the tiled order.  K % 64 == 0 and
 * N % 128 == 0, else DF11_EINVAL. */
df11_status df11_gemm_tile_weights(const uint16_t *host_w, uint64_t k, uint64_t n, uint16_t *host_tiled);

typedef struct {
    const df11_blob *weights; /* bound blob of the tiled K x N matrix: BF16, the default layout
                                 (128-bit chunks, 32-chunk tiles, chunk counts), host sections present */
    uint64_t k, n;            /* K inputs (multiple of 64), N outputs (multiple of 128) */
    const void *x;            /* device, M x K BF16 row-major, 16-byte aligned, rows K * 2 bytes apart */
    float *y;                 /* device, M x N FP32 row-major, 4-byte aligned: y += x W */
} df11_gemm_matrix;

/* y_i += x_i W_i for every matrix of the launch, in ONE kernel launch on
 * `stream`, asynchronously: the weights are decoded tile by tile into shared
 * memory and multiplied there by the tensor cores (FP32 accumulation); the
 * decoded weights never reach HBM.  y is accumulated with floating-point
 * adds (the reduction over K is split between CTAs), so the caller zeroes y
 * for a plain product, and the rounding order of y varies from run to run
 * (every y element is within (K + 16) * 2^-24 * sum_k |x_mk w_kn| of the
 * exact product plus what y held: K products added in FP32, plus the adds of
 * a tile's four accumulators and of the CTAs that share the reduction).  The matrices share one code (one codebook),
 * as in df11_decode.  M = m in 1..DF11_GEMM_MAX_BATCH; n_mats in
 * 1..DF11_GEMM_MAX_MATS.  dev_err_flag as in df11_decode (its bits mean the
 * y of that launch is not valid).  Never allocates, never synchronises.
 * Errors: DF11_EINVAL (arguments, shapes, alignment, an unbound or
 * GPU-encoded blob without host sections, mixed codes), DF11_EUNSUPPORTED
 * (another dtype or layout, a code with a 1-bit codeword, tables too large
 * for shared memory), DF11_ECUDA. */
df11_status df11_decode_gemm(const df11_gemm_matrix *mats, int n_mats, int m, int *dev_err_flag,
                             df11_stream stream);

/* Grid, threads per CTA and dynamic shared memory of that launch on the
 * current device (any output may be NULL); x and y are not read. */
df11_status df11_decode_gemm_launch_shape(const df11_gemm_matrix *mats, int n_mats, int m, int *grid, int *block,
                                          int *smem_bytes);

/* ---------------------------------------------------------------------
 * rANS variant of the exponent coder
 * ------------------------------------------------------------------ */

/* The same exponent symbols and raw plane as the Huffman container, coded
 * with range asymmetric numeral systems instead of a prefix code: the
 * tile-level ANS decoding of "Approaching Shannon Bound with Lossless LLM
 * Weight Compression", Abstract (which gives no coder details; the format
 * below is this library's).
 *   frequencies  quantized to a total of 2^12 over the group's exponent
 *                histogram (every present symbol at least 1)
 *   state        32 bits in [2^16, 2^32); 16-bit words move in and out
 *   tiles        tile_symbols symbols (a multiple of 32), coded by 32
 *                interleaved coders: coder j takes symbols j, j+32, ...
 *                Decoding runs steps, and in each step coders 0..31 in
 *                order; a coder whose state fell below 2^16 after its symbol
 *                reads the tile's next word.
 *   per tile     32 initial states (u32) and its words' offset (u64, a
 *                multiple of 8 words)
 * One group = the tensors of one launch, sharing one frequency table (a
 * transformer block).  Decoding is exact: the output equals the source bits. */
typedef struct df11_rans_group df11_rans_group;

#define DF11_RANS_TILE_DEFAULT 16384

typedef struct {
    uint64_t n_elems;
    uint64_t n_tiles;
    uint64_t words;        /* 16-bit words, with the padding between tiles */
    uint64_t coded_bytes;  /* words * 2 + states (n_tiles * 128) + offsets ((n_tiles + 1) * 8) */
    uint64_t plane_bytes;
    uint64_t uncompressed_bytes;
} df11_rans_tensor_info;

/* Encodes n_tensors host tensors (dtype's raw bits) with one frequency table
 * built from all of them; tile_symbols a multiple of 32 in [32, 2^20] (0 =
 * DF11_RANS_TILE_DEFAULT); n_threads host threads (0 = all cores).
 * Errors: DF11_EINVAL, DF11_ENOMEM. */
df11_status df11_rans_encode_group(df11_dtype dtype, const void *const *host_tensors, const uint64_t *n_elems,
                                   int n_tensors, int tile_symbols, int n_threads, df11_rans_group **out);

void df11_rans_group_free(df11_rans_group *g);

/* The quantized frequencies (freqs[0..255]; E4M3 uses 16). */
df11_status df11_rans_group_freqs(const df11_rans_group *g, uint32_t *freqs);

df11_status df11_rans_group_info(const df11_rans_group *g, int tensor, df11_rans_tensor_info *info);

/* Read-only host views of one tensor's sections (valid until the group is
 * freed); any output may be NULL. */
df11_status df11_rans_group_sections(const df11_rans_group *g, int tensor, const uint16_t **words,
                                     const uint32_t **states, const uint64_t **tile_words,
                                     const uint8_t **plane);

/* The group's container (offline form): a 64-byte header ("DF11RANS",
 * version 1, dtype, symbols, tile size, tensor count), the frequencies (u16
 * per symbol), then per tensor a 32-byte record (n, n_tiles, words) and its
 * states, tile offsets, words and plane, each section 16-byte aligned.
 * *used receives the size; DF11_ENOMEM when cap is too small. */
df11_status df11_rans_group_serialize(const df11_rans_group *g, void *buf, uint64_t cap, uint64_t *used);

/* Reads a container; checks the header, that the frequencies sum to 2^12,
 * every size, the tile offsets (monotone, multiples of 8, at most one word
 * per symbol plus padding) and that every state is at least 2^16.  Errors:
 * DF11_ECORRUPT, DF11_ENOMEM. */
df11_status df11_rans_group_deserialize(const void *buf, uint64_t len, df11_rans_group **out);

/* Bytes of the group's device image: the 4096-entry decode table, then per
 * tensor its states, offsets, words (plus 1024 zero words) and plane (plus
 * 512 bytes), each section 256-byte aligned. */
uint64_t df11_rans_group_device_bytes(const df11_rans_group *g);

/* Builds the image in host memory held by the group, copies it to dev_dst
 * (256-byte aligned, cap >= device bytes) on `stream` and binds it.  The
 * caller owns dev_dst.  Errors: DF11_EINVAL, DF11_ENOMEM, DF11_ECUDA. */
df11_status df11_rans_group_upload(df11_rans_group *g, void *dev_dst, uint64_t cap, df11_stream stream);

/* Decodes every tensor of the bound group in one launch on `stream`,
 * asynchronously; dst_dev[i] as in df11_decode (16-byte aligned).  Damaged
 * data ORs DF11_DEV_ERR_SPAN (a tile's coders do not end in their initial
 * state, or took other than its words) or DF11_DEV_ERR_AUX (offsets out of
 * range) into dev_err_flag; nothing is written outside the destinations.
 * Errors: DF11_EINVAL (unbound group, bad pointer), DF11_ECUDA. */
df11_status df11_rans_decode(const df11_rans_group *g, void *const *dst_dev, int *dev_err_flag,
                             df11_stream stream);

/* Grid, threads per CTA and dynamic shared memory of that launch (any output
 * may be NULL; the group must be bound). */
df11_status df11_rans_decode_launch_shape(const df11_rans_group *g, int *grid, int *block, int *smem_bytes);

#ifdef __cplusplus
}
#endif

#endif /* DF11_H */
