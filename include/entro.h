/*
 * entro.h -- C ABI of libentro: lossless Huffman coding of tensor-level
 * quantized LLM weights, and sm_100a kernels that decode them on demand.
 *
 * The method: "EntroLLM: Entropy Encoded Weight Compression for Efficient
 * Large Language Model Inference on Edge Devices" (arXiv 2505.02380v4) --
 * abstract and method details: mixed tensor-level quantization (unsigned or
 * asymmetric per tensor), Huffman coding of the integer codes, a chunked
 * stream that decodes in parallel.  "LazyWeights: Decode-on-Demand Edge LLMs"
 * (arXiv 2611.17108v1), abstract: codes stored in interleaved lanes and
 * decoded on demand so that memory moves only coded bytes.
 *
 * Conventions for every call:
 *  - Return value: ENTRO_OK (0) or a negative ENTRO_E_* code; nothing is
 *    launched when a call returns an error.  entro_strerror() names a code.
 *  - Device calls are asynchronous on the caller's stream (a cudaStream_t
 *    passed as void*; NULL = the legacy default stream).  Argument and
 *    launch errors come back as the return value.  Errors found while
 *    decoding (an invalid code, a lane stream that runs past its chunk, a
 *    bounded wait that gave up) are written to the optional device word
 *    *d_status: the first error wins (atomic compare-and-swap from 0), later
 *    ones are dropped.  The caller zeroes *d_status before the call and reads
 *    it after synchronising.  Kernels never trap or assert.
 *  - All device buffers passed in belong to the caller (allocate them with
 *    any CUDA allocator, e.g. torch); the library never frees them.
 *    Host objects created by the library (entro_blob, entro_tensor) are freed
 *    with their own _free call.
 *  - There is no CPU fallback: every decode runs on the GPU.
 */
#ifndef ENTRO_H
#define ENTRO_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ENTRO_API __attribute__((visibility("default")))
#else
#define ENTRO_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define ENTRO_OK 0
#define ENTRO_E_INVAL -1    /* bad argument (null pointer, bad option, misaligned buffer) */
#define ENTRO_E_LIMIT -2    /* outside a documented limit (alphabet vs max_len, zero point, sizes) */
#define ENTRO_E_FORMAT -3   /* blob bytes are not a valid version-1 blob */
#define ENTRO_E_CORRUPT -4  /* device: a bit pattern that is no code of the table */
#define ENTRO_E_OVERRUN -5  /* device: a lane or chunk stream read past its end */
#define ENTRO_E_NOMEM -6    /* host allocation failed */
#define ENTRO_E_CUDA -7     /* a CUDA runtime call failed */
#define ENTRO_E_TIMEOUT -8  /* device: a bounded wait on a copy gave up */

/* Quantization choice per tensor (EntroLLM abstract: "a combination of
 * unsigned and asymmetric quantization"; method details, mixed quantization). */
#define ENTRO_QUANT_AUTO 0     /* the scheme whose codes have lower entropy; ties -> unsigned */
#define ENTRO_QUANT_UNSIGNED 1 /* zero = 0, scale = max/(2^b-1); only for min >= 0 */
#define ENTRO_QUANT_ASYM 2     /* scale = (max-min)/(2^b-1), zero = round(-min/scale) */

#define ENTRO_SCHEME_UNSIGNED 0
#define ENTRO_SCHEME_ASYM 1

/* Chunk formats (EntroLLM technical summary, parallel decoding over chunks;
 * LazyWeights abstract, interleaved lanes). */
#define ENTRO_FORMAT_SINGLE 1 /* one bitstream per chunk, chunks bit-contiguous */
#define ENTRO_FORMAT_LANES 2  /* 32 (or 64) word-interleaved lane bitstreams per chunk */
#define ENTRO_FORMAT_ROWS 3   /* row tiles: a chunk is L = 32 (or 64) rows by chunk_symbols / L columns,
                                 lane l holding row l of the tile; word-interleaved like LANES.  Made for
                                 the fused GEMV; cols must be a multiple of 8 */
#define ENTRO_FORMAT_ROWS_CO 4 /* row tiles in consumption order: the tiles and lane bitstreams of ROWS,
                                  each lane keeping only its own words (a per-lane word count leads the
                                  chunk), stored in the order a lock-step decoder takes them instead of
                                  padded to the tile's longest lane.  Decodes through every call ROWS
                                  does (32-lane tiles) */

typedef struct entro_encode_opts {
    int32_t bits;          /* 4 or 8 */
    int32_t quant_mode;    /* ENTRO_QUANT_* */
    int32_t max_len;       /* code length limit, 1..24; 0 = 16 for 8-bit, 12 for 4-bit */
    int32_t format;        /* ENTRO_FORMAT_* */
    int64_t chunk_symbols; /* 0 = 4096 (single) / 8192 (lanes, rows).  Lanes and rows: a multiple of
                              8 * lanes in [8 * lanes, 16384].  Single: 1 .. 2^20. */
    int32_t threads;       /* host threads for encoding; 0 = all hardware threads */
    int32_t lanes;         /* lanes / rows formats: 32 (also 0) or 64 interleaved lanes per chunk; a
                              chunk must then hold a multiple of 8 * lanes symbols */
} entro_encode_opts;

typedef struct entro_blob entro_blob;     /* host copy of one encoded tensor (serialized bytes) */
typedef struct entro_tensor entro_tensor; /* host handle to a tensor uploaded to device memory */

typedef struct entro_info {
    int32_t bits, scheme, max_len, format;
    int64_t rows, cols, n, chunk_symbols, n_chunks;
    float scale;
    int32_t zero;
    uint64_t payload_bytes;   /* coded words, including lane padding */
    uint64_t index_bytes;     /* 16 bytes per chunk + 16 */
    uint64_t blob_bytes;      /* whole serialized blob */
    uint64_t coded_bits;      /* sum of the code lengths of all symbols (0 if unknown: a lanes
                                 blob read back with entro_blob_from_bytes) */
    uint32_t max_chunk_words; /* lanes: longest lane of any chunk in 32-bit words */
    uint32_t lanes;           /* interleaved lanes per chunk (1 for the single-stream format) */
    uint8_t lengths[256];     /* code length per symbol, 0 = symbol absent */
} entro_info;

/* Quantize a row-major fp32 [rows, cols] tensor on the host, build its
 * length-limited canonical Huffman code (package-merge, RFC 1951 canonical
 * order) and encode it in chunks (LazyWeights abstract: "interleaved lanes"; the
 * lane count is a format parameter).  *out receives a library-owned blob; free it
 * with entro_blob_free.  rows*cols may be 0 (an empty blob).  Errors:
 * E_INVAL (NaN/Inf weight, bad option, null pointer, UNSIGNED with a negative
 * weight), E_LIMIT (more distinct codes than 2^max_len allows, zero point
 * beyond 2^24, scale underflow), E_NOMEM. */
ENTRO_API int entro_encode(const float *host_w, int64_t rows, int64_t cols, const entro_encode_opts *opts,
                 entro_blob **out);

/* Copy and validate serialized blob bytes (e.g. read from a file).  Errors:
 * E_FORMAT for anything that is not a consistent version-1 blob. */
ENTRO_API int entro_blob_from_bytes(const void *data, uint64_t size, entro_blob **out);

/* Borrow the serialized bytes of a blob (valid until entro_blob_free). */
ENTRO_API int entro_blob_bytes(const entro_blob *blob, const void **data, uint64_t *size);

ENTRO_API int entro_blob_info(const entro_blob *blob, entro_info *out);

ENTRO_API void entro_blob_free(entro_blob *blob);

/* Bytes of device memory entro_upload needs for this blob (decode tables,
 * chunk index, payload and a small read-ahead pad). */
ENTRO_API int entro_device_bytes(const entro_blob *blob, uint64_t *bytes);

/* Copy a blob's decode image into caller-owned device memory d_mem (at least
 * entro_device_bytes, 256-byte aligned) on `stream`.  d_mem must outlive the
 * returned handle.  The blob may be freed once this call returns.  Errors:
 * E_INVAL (null/misaligned/too small), E_LIMIT (a chunk too large for the
 * decoder's shared-memory staging), E_CUDA. */
ENTRO_API int entro_upload(const entro_blob *blob, void *d_mem, uint64_t d_bytes, void *stream,
                 entro_tensor **out);

ENTRO_API void entro_tensor_free(entro_tensor *t);

/* Decode to the integer codes.  8-bit: d_out is uint8[n].  4-bit: d_out is
 * ceil(n/2) bytes, byte i holding code 2i in its low nibble and code 2i+1 in
 * its high nibble (a missing last code is 0).  d_out must be 16-byte aligned.
 * (EntroLLM technical summary: lossless Huffman coding of the quantized
 * weights; parallel decoding of the chunks.) */
ENTRO_API int entro_decode_codes(const entro_tensor *t, void *d_out, int32_t *d_status, void *stream);

/* Decode and dequantize: d_out[i] = bf16_rne(float(q_i - zero) * scale), the
 * product taken in fp32 and rounded to nearest-even; bf16[n], row-major
 * [rows, cols], 16-byte aligned. */
ENTRO_API int entro_decode_dequant_bf16(const entro_tensor *t, void *d_out, int32_t *d_status, void *stream);

/* Fused decode -> dequantize -> GEMV for token generation: for b < batch and
 * r < rows, d_y[b*rows + r] = sum_k w[r,k] * x[b*cols + k], w the bf16
 * weights of entro_decode_dequant_bf16 (never written to memory), x bf16
 * [batch, cols], accumulation in fp32; batch in 1..16; d_x 16-byte aligned.
 * Row-tile format (any shape of it): a warp decodes a tile's 32 (64) rows and
 * multiplies them on the tensor cores (mma.sync m16n8k16, bf16 operands,
 * fp32 accumulation) for every batch size.  Lanes format: cols a multiple of
 * 8 * lanes (256 or 512) and chunk_symbols a multiple of cols (chunks of
 * whole rows); batch 1-2 use fp32 FMAs of the bf16 products in the decoding
 * warp, batch 3-16 the tensor cores with the warps of a block decoding
 * consecutive rows.  Every sum is taken in a fixed order, so results are
 * bit-reproducible. */
ENTRO_API int entro_decode_gemv(const entro_tensor *t, const void *d_x, int32_t batch, float *d_y,
                      int32_t *d_status, void *stream);

/* Grouped launches: several tensors decoded by ONE kernel launch -- every
 * projection of a decoder step through the fused GEMV, or a whole model to
 * bf16.  entro_group_prepare writes the launch's work table (one entry per
 * tensor, with the x / y / output pointers baked in) into caller-owned device
 * memory d_table of at least entro_group_table_bytes(count) bytes (256-byte
 * aligned) and returns a host handle; it synchronises `stream` once.
 * entro_group_launch then launches without any host-device traffic, as often
 * as wanted (for instance once per generated token).  d_table, the tensors'
 * device images and the x / y / output buffers must stay valid while the
 * handle is used; all tensors must share the device, the bit width, the
 * format (lanes or row tiles) and the lane count (E_INVAL from
 * entro_group_prepare otherwise).
 * kind:
 *   ENTRO_GROUP_GEMV  xs[i] bf16 [batch, cols_i], ys[i] fp32 [batch, rows_i]
 *                     (the per-tensor rules of entro_decode_gemv apply)
 *   ENTRO_GROUP_BF16  outs[i] bf16 [rows_i, cols_i] (lanes or row-tile format) */
#define ENTRO_GROUP_GEMV 1
#define ENTRO_GROUP_BF16 2
typedef struct entro_group entro_group;
ENTRO_API uint64_t entro_group_table_bytes(int32_t count);
ENTRO_API int entro_group_prepare(const entro_tensor *const *tensors, int32_t count, int32_t kind, const void *const *xs,
                        float *const *ys, void *const *outs, int32_t batch, void *d_table, uint64_t table_bytes,
                        void *stream, entro_group **out);
ENTRO_API int entro_group_launch(const entro_group *group, int32_t *d_status, void *stream);
ENTRO_API void entro_group_free(entro_group *group);

ENTRO_API const char *entro_strerror(int code);

/* The grouped fused GEMV (ENTRO_GROUP_GEMV) for callers that cannot allocate
 * device memory -- code running inside an allocator's hooks, or a runtime
 * that reserves the whole device up front and allows no cudaMalloc later.  No
 * counterpart on the EntroLLM or LazyWeights pages: it only changes where the
 * launch's work table lives.  The table is a fixed array inside the library
 * (ENTRO_STATIC_GROUP_MAX entries of 184 bytes, about 92 KB, held on every
 * GPU that loads the library until the process exits); the caller still
 * passes the uploaded tensors, the activations xs[i] (bf16 [batch, cols_i])
 * and the outputs ys[i] (fp32 [batch, rows_i]), with the rules of
 * entro_decode_gemv for each.  Each call rewrites the table from host memory
 * on `stream` and launches; nothing is allocated or freed, on the host heap
 * or on the device.  The tensors' device must be the current device.  The
 * first call on a device looks up the table's device address
 * (cudaGetSymbolAddress).  All calls share the one table, so calls whose launches may overlap on the
 * GPU (other streams, other host threads) race: serialise them.  Errors:
 * ENTRO_E_LIMIT when count > ENTRO_STATIC_GROUP_MAX, otherwise as
 * entro_decode_gemv. */
#define ENTRO_STATIC_GROUP_MAX 512
ENTRO_API int entro_decode_gemv_group_static(const entro_tensor *const *tensors, const void *const *xs,
                                             float *const *ys, int32_t count, int32_t batch, int32_t *d_status,
                                             void *stream);

/* Launch overlap (not in the pages: a B200 launch option).  When enabled,
 * decode launches that fill each SM with one or two large CTAs (the lanes-
 * format kernels on tensors large enough for it) are made with programmatic
 * dependent launch:
 * such a launch may start while the kernel launched just
 * before it on the same stream is still finishing, and overlaps that kernel's
 * tail with its own start-up (chunk index, tables and first coded words
 * fetched from device memory).  Before the previous kernel has completed, a
 * decode kernel reads only the tensor's device image (tables, index, coded
 * words); activations, outputs and the status word are touched only after it
 * has completed, as without overlap.  Enable it only if no kernel launched
 * right before a decode call on the same stream writes that tensor's device
 * image (copies, such as entro_upload's, are always waited for).  Process-
 * wide; off by default.  Returns the previous setting. */
ENTRO_API int entro_set_overlap(int enable);

/* Test hook for the bounded waits (no counterpart on the pages).  With
 * extra_bytes > 0, every later launch declares extra_bytes more on the
 * barrier of its decode-table copy than the copy delivers, so that barrier
 * never completes: the kernel's bounded wait gives up after about a second,
 * writes ENTRO_E_TIMEOUT to the status word, lets its copies in flight land
 * (again a bounded wait) and returns; outputs are then incomplete.  0 (the
 * default) turns it off.  Process-wide; returns the previous value. */
ENTRO_API uint32_t entro_test_stall_tables(uint32_t extra_bytes);

/* Text of the last CUDA runtime error behind an ENTRO_E_CUDA return on the
 * calling host thread ("" if none). */
ENTRO_API const char *entro_last_cuda_error(void);

/* Library version: 100 * major + minor. */
ENTRO_API int entro_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ENTRO_H */
