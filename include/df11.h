/*
 * df11.h -- C ABI of a B200-native DFloat11 (DF11) decompressor.
 *
 * DF11 ("DFloat11: Kompresi inferensi GPU lossless yang mengecilkan LLM
 * menjadi 70% ukurannya", id.news.hada.io/topic?id=20542) stores a BFloat16
 * matrix as two byte arrays: EncodedExponent, the 8-bit exponents Huffman
 * coded and bit-packed, and PackedSignMantissa, sign and mantissa verbatim
 * (section "Format DFloat11").  The GPU rebuilds the exact BF16 values right
 * before they are used (section "Dekompresi yang disesuaikan untuk inferensi
 * GPU"), helped by hierarchical 256-entry LUTs ("Decoding berbasis LUT
 * hierarkis") and per-thread / per-block metadata ("Kernel GPU 2 tahap dan
 * metadata bantu").
 *
 * Entry points, by the side they run on:
 *   - host: df11_build_format compresses BF16 matrices into the format
 *     (df11_format_arrays / df11_format_info read it back, df11_free drops
 *     it); df11_plan_from_histogram builds only the code and the sizes from
 *     256 exponent counts;
 *   - device decode: df11_decompress rebuilds the BF16 matrix on a CUDA
 *     stream (df11_decompress_sms on at most a given number of SMs);
 *     df11_decompress_gemv decodes and multiplies by vectors without storing
 *     the weights (CUDA cores); df11_decompress_gemm does the same for a
 *     batch of vectors on the tensor cores (tile-major streams, see
 *     df11_tile_major; df11_gemm_scratch_bytes sizes its scratch);
 *     df11_decompress_host takes the arrays in host memory and
 *     overlaps the copies with the decode; df11_read_status reads the
 *     kernels' error word;
 *   - device encode: df11_device_histogram counts exponents of a device
 *     array; df11_device_encode (caller scratch) and
 *     df11_device_encode_static (library scratch) write the compressed
 *     arrays of a plan into device buffers;
 *   - rANS variant of the exponent coder (the page's discussion proposes
 *     rANS instead of Huffman coding): df11_rans_build compresses on the
 *     host (df11_rans_format_arrays, df11_rans_free), df11_rans_decompress
 *     rebuilds the BF16 matrix on the device.
 * No entry point takes or returns framework types; all pointers are plain
 * host or device addresses as stated per argument.
 *
 * Byte layout of the format (every reader of the arrays relies on it):
 *   - element = BF16 bits w; exponent = (w >> 7) & 0xFF, which must be < 240
 *     (240..255 are LUT pointers); PackedSignMantissa byte = (w >> 8 & 0x80)
 *     | (w & 0x7F).
 *   - code lengths: Huffman over the exponent histogram, ties merged by
 *     smallest (weight, smallest symbol in subtree); if the longest code
 *     exceeds 32 bits, optimal 32-bit-limited lengths by package-merge.  A
 *     single distinct exponent gets length 1.
 *   - codes: canonical (symbols sorted by (length, symbol) get increasing
 *     values).  CodeLengths[256] therefore fixes the whole code.
 *   - EncodedExponent: codes concatenated MSB-first; bit i of the stream is
 *     bit (7 - i % 8) of byte i / 8.  Zero padded.
 *   - segment s = stream bits [64 s, 64 s + 64) (8 bytes per GPU thread).
 *     Gap[s] = (first code start >= 64 s, or total_bits if none) - 64 s, in
 *     [0, 31]; stored as 5-bit fields LSB-first in uint64 words (field s at
 *     bits 5 s .. 5 s + 4 of the little-endian word sequence).
 *   - block b = segments [T b, T b + T).  BlockOffset[b] = number of codes
 *     that start before bit 64 T b; BlockOffset[num_blocks] = n.
 *   - LUTs: k tables of 256 bytes.  Table 0 is indexed by the first 8 bits
 *     of the 32-bit window, a child table by the next 8 bits.  An entry is a
 *     symbol (< 240) or a pointer 256 - j to table j (j = 1 .. 16); children
 *     are numbered level by level in increasing order of their bit prefix.
 *
 * Threading: the host functions are thread-safe for distinct handles.  The
 * device functions are stream-ordered and never synchronise except where
 * stated (df11_read_status).
 */
#ifndef DF11_H
#define DF11_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DF11_ABI_VERSION 1
#define DF11_MAX_CODE_LEN 32     /* longest code: Gaps are 5 bits wide */
#define DF11_SEGMENT_BYTES 8     /* encoded bytes per GPU thread */
#define DF11_MAX_LUTS 17         /* root + 16 children (pointers 240..255) */
#define DF11_DEFAULT_THREADS 64  /* default segments (threads) per block */

typedef enum df11_status {
    DF11_OK = 0,
    DF11_ERR_INVALID_ARG = 1,          /* bad pointer, size, alignment or T */
    DF11_ERR_UNSUPPORTED_EXPONENT = 2, /* an input exponent is in 240..255 */
    DF11_ERR_TOO_LARGE = 3,            /* n >= 2^32 elements in one stream */
    DF11_ERR_TOO_MANY_LUTS = 4,        /* the code needs > 16 child LUTs */
    DF11_ERR_CUDA = 5,                 /* a CUDA runtime call failed */
    DF11_ERR_CORRUPT = 6,              /* the kernel found inconsistent data */
    DF11_ERR_NO_MEMORY = 7             /* host allocation failed */
} df11_status;

/* Opaque handle: a host-resident compressed stream (owns its arrays). */
typedef struct df11_format df11_format;

/*
 * The arrays of one compressed stream.  The same struct describes host
 * copies (df11_format_arrays) or device copies (filled in by the caller after
 * uploading each array).  Sizes include the padding the kernel relies on.
 */
typedef struct df11_arrays {
    uint64_t n;                 /* BF16 elements in the stream */
    uint64_t total_bits;        /* valid bits of encoded_exponent */
    uint64_t num_segments;      /* ceil(total_bits / 64) */
    uint32_t threads_per_block; /* T: segments per block (multiple of 32, 32..1024;
                                   the decoder takes T = 32 or 64: one warp) */
    uint32_t num_blocks;        /* ceil(num_segments / T) */
    uint32_t num_luts;          /* k, 1 .. 17 */
    uint32_t max_code_len;      /* longest code length, <= 32 */
    uint32_t max_block_elems;   /* max_b BlockOffset[b+1] - BlockOffset[b] */
    uint32_t min_code_len;      /* shortest code length, 1..32; 0 = not known
                                   (the decoder then assumes 1).  The decoder
                                   sizes its per-segment staging buffers by it
                                   and reports DF11_ERR_CORRUPT if a code is
                                   shorter than stated */
    const uint8_t *encoded_exponent;     /* num_blocks*T*8 + 16 bytes, zero padded, 16-B aligned */
    uint64_t encoded_exponent_bytes;
    const uint8_t *packed_sign_mantissa; /* round_up(n, 16) + 16 bytes, 16-B aligned */
    uint64_t packed_sign_mantissa_bytes;
    const uint64_t *gaps;                /* ceil(5*num_blocks*T / 64) + 2 words */
    uint64_t gaps_words;
    const uint32_t *block_offset;        /* num_blocks + 1 entries */
    const uint8_t *luts;                 /* num_luts * 256 bytes */
    const uint8_t *code_lengths;         /* 256 bytes, indexed by exponent */
    const uint32_t *symbol_table;        /* optional, 16-B aligned: the decoders' derived table,
                                            4096 entries (df11_build_format fills it; see
                                            df11_symbol_table); NULL: each CTA derives it from
                                            luts and code_lengths.  Exponent bytes past an
                                            entry's count are ignored; an entry of more than
                                            3 codes or 12 bits, of fewer bits than codes (or
                                            than 2 per code when min_code_len >= 2), or a 0
                                            entry where the LUTs hold a code of <= 12 bits,
                                            is reported as DF11_ERR_CORRUPT */
} df11_arrays;

/* Statistics of a built stream ("Ruang kompresi": exponent entropy and the
 * number of exponent values in use; "Decoding berbasis LUT hierarkis": L, k). */
typedef struct df11_info {
    uint64_t n;
    uint64_t total_bits;
    uint64_t compressed_bytes; /* ceil(total_bits/8) + n + gaps + offsets + LUTs + 256 */
    double entropy_bits;       /* Shannon entropy of the exponent histogram */
    double avg_code_len;       /* total_bits / n */
    uint32_t distinct_exponents;
    uint32_t max_code_len;
    uint32_t num_luts;
    uint32_t threads_per_block;
    uint64_t histogram[256];
} df11_info;

/*
 * df11_build_format -- compress BF16 matrices into one DF11 stream
 * ("Format DFloat11"; metadata per "Kernel GPU 2 tahap dan metadata bantu").
 *   mats[i]   host pointer to counts[i] BF16 bit patterns (uint16), row-major;
 *             matrix i occupies elements [sum_{j<i} counts[j], ...) of the
 *             stream.  One Huffman code covers all matrices (a transformer
 *             block is compressed as one stream, "Dekompresi per transformer
 *             block").  NULL allowed when counts[i] == 0.
 *   threads_per_block  T, a multiple of 32 in [32, 1024] (0 = default 64).
 *             df11_decompress requires T = 32 or 64 (a block is one warp).
 *   out       receives a new handle, owned by the caller (df11_free).
 * Inputs are only read.  Errors: DF11_ERR_INVALID_ARG, _UNSUPPORTED_EXPONENT,
 * _TOO_LARGE (total n >= 2^32), _TOO_MANY_LUTS, _NO_MEMORY; *out is NULL then.
 * Runs on the host with up to hardware_concurrency threads; needs no GPU.
 */
df11_status df11_build_format(const uint16_t *const *mats, const uint64_t *counts,
                              int num_mats, uint32_t threads_per_block,
                              df11_format **out);

/* Borrowed host views of a handle's arrays (valid until df11_free). */
df11_status df11_format_arrays(const df11_format *f, df11_arrays *out);

/* Statistics of a handle. */
df11_status df11_format_info(const df11_format *f, df11_info *out);

/* Frees a handle; NULL is allowed. */
void df11_free(df11_format *f);

/* Static English text for a status code. */
const char *df11_strerror(df11_status s);

/*
 * df11_decompress -- rebuild the BF16 stream on the GPU
 * ("Dekompresi yang disesuaikan untuk inferensi GPU", "Decoding berbasis LUT
 * hierarkis", "Kernel GPU 2 tahap dan metadata bantu").
 *   dev        arrays whose pointers are DEVICE addresses (sizes as in the
 *              host view); only read.
 *   dst        device pointer to dev->n uint16 BF16 outputs, 16-byte aligned;
 *              written in full, nothing else is written.
 *   status_dev device pointer to one uint32, OR-accumulated with
 *              DF11_ERR_CORRUPT when the kernel meets inconsistent data (the
 *              affected block's outputs are then left unwritten); zero it
 *              before the first call.
 *   stream     a cudaStream_t (NULL = legacy default stream).
 * Asynchronous; returns DF11_ERR_INVALID_ARG for bad arguments (checked on
 * the host, nothing launched) or DF11_ERR_CUDA when the launch fails.
 * n == 0 launches nothing.  The kernel never traps and every loop is bounded.
 */
df11_status df11_decompress(const df11_arrays *dev, uint16_t *dst,
                            uint32_t *status_dev, void *stream);

/*
 * df11_decompress_sms -- df11_decompress on at most `max_sms` SMs
 * ("Dekompresi per transformer block": decompressing the next block while
 * the current one is used).  The decoder otherwise runs one persistent CTA
 * on every SM, which leaves no SM to kernels on other streams until it ends;
 * a cap leaves the remaining SMs to them.  max_sms = 0 means every SM (the
 * same as df11_decompress); arguments, outputs and errors as there.
 */
df11_status df11_decompress_sms(const df11_arrays *dev, uint16_t *dst,
                                uint32_t *status_dev, void *stream, uint32_t max_sms);

/* One matrix of df11_decompress_gemv: `rows` x `cols` BF16 weights, row-major,
 * the next rows*cols elements of the stream (matrices in stream order). */
typedef struct df11_gemv_matrix {
    uint32_t rows;
    uint32_t cols;       /* a multiple of 16 */
    const uint16_t *x;   /* device: cols BF16 activations, 16-byte aligned */
    float *y;            /* device: rows float32 outputs, 4-byte aligned */
} df11_gemv_matrix;

/*
 * df11_decompress_gemv -- decode and use in one pass: y_m += W_m x_m for
 * every matrix m of the stream, the BF16 weights W_m decoded on chip and
 * never written to memory ("Dekompresi yang disesuaikan untuk inferensi
 * GPU": weights are decompressed only to be multiplied, then discarded).
 * The same decode as df11_decompress; each decoded weight is multiplied by
 * its activation in float32 and the products of a row are summed per warp
 * and added to y by atomic adds (so the summation order, and the last bits
 * of y, vary between runs; the error is that of a float32 sum of the row's
 * cols products).
 *   dev       the stream's arrays (device pointers), as df11_decompress.
 *   mats      host array of num_mats (1..16) matrices whose rows*cols add
 *             up to dev->n; y is accumulated, not overwritten: zero it for
 *             y = W x.
 *   status_dev, stream: as df11_decompress.
 * Asynchronous; DF11_ERR_INVALID_ARG for bad arguments (nothing launched),
 * DF11_ERR_CUDA if the launch fails.
 */
df11_status df11_decompress_gemv(const df11_arrays *dev, const df11_gemv_matrix *mats, uint32_t num_mats,
                                 uint32_t *status_dev, void *stream);

/* One matrix of df11_decompress_gemm: `rows` x `cols` BF16 weights W, the
 * next rows*cols elements of the stream (matrices in stream order), stored
 * in TILE-MAJOR order (df11_tile_major): 128 x 64 tiles, row tiles in order,
 * within a row tile the column tiles in order, within a tile 128 rows of 64
 * elements. */
typedef struct df11_gemm_matrix {
    uint32_t rows;       /* a multiple of 128 */
    uint32_t cols;       /* a multiple of 64 */
    const uint16_t *x;   /* device: batch x cols BF16 activations, row-major, 16-byte aligned */
    float *y;            /* device: batch x rows float32 outputs, row-major, 4-byte aligned */
} df11_gemm_matrix;

/*
 * df11_decompress_gemm -- decode and multiply for a batch of activation
 * vectors: Y_m += X_m W_m^T for every matrix m of the stream, on the tensor
 * cores (tcgen05.mma, BF16 inputs, float32 accumulation), W_m decoded tile by
 * tile into shared memory and never written to global memory ("Dekompresi
 * yang disesuaikan untuk inferensi GPU": decompress right before the matrix
 * multiplication; the page's discussion proposes a GEMM that decompresses
 * each tile before its arithmetic).  Every output is a float32 sum of cols
 * exact BF16 products, accumulated by the tensor core over K chunks of 64 and
 * by atomic adds over groups of 16 chunks (so the last bits of Y vary between
 * runs).
 *   dev        the stream's arrays (device pointers), as df11_decompress;
 *              the matrices' elements in tile-major order.
 *   mats       host array of num_mats (1..16) matrices whose rows*cols add
 *              up to dev->n; Y is accumulated, not overwritten.
 *   batch      number of activation vectors: a multiple of 16, 16..256.
 *   scratch    device buffer of at least df11_gemm_scratch_bytes(mats,
 *              num_mats, batch) bytes, 16-byte aligned, owned by the caller
 *              and not in use by other work until this call's kernels end
 *              (it receives X repacked for the tensor core and each work
 *              unit's format blocks).
 *   status_dev, stream: as df11_decompress.  Bit 31 of *status_dev set means
 *              a bounded wait inside the kernel ran out (Y incomplete).
 * Asynchronous (two launches on `stream`); DF11_ERR_INVALID_ARG for bad
 * arguments (nothing launched), DF11_ERR_CUDA if a launch fails.
 */
df11_status df11_decompress_gemm(const df11_arrays *dev, const df11_gemm_matrix *mats, uint32_t num_mats,
                                 uint32_t batch, void *scratch, uint64_t scratch_bytes,
                                 uint32_t *status_dev, void *stream);

/* Scratch bytes df11_decompress_gemm needs for these matrices and batch;
 * 0 if the arguments are invalid (see df11_decompress_gemm). */
uint64_t df11_gemm_scratch_bytes(const df11_gemm_matrix *mats, uint32_t num_mats, uint32_t batch);

/*
 * df11_tile_major -- host: writes the rows x cols row-major BF16 matrix src
 * (host memory) to dst (host, rows*cols elements, not overlapping src) in the
 * tile-major order df11_decompress_gemm reads: for each row tile of 128 rows,
 * for each column tile of 64 columns, its 128 rows of 64 elements.  Compress
 * the result with df11_build_format.  DF11_ERR_INVALID_ARG unless rows is a
 * multiple of 128 and cols of 64.
 */
df11_status df11_tile_major(const uint16_t *src, uint32_t rows, uint32_t cols, uint16_t *dst);

/*
 * df11_symbol_table -- host: the decoders' derived 12-bit table of a code
 * ("Decoding berbasis LUT hierarkis": the page's LUTs answer one code per
 * lookup chain; the table answers, for each 12-bit window, the first up to
 * three whole codes inside it: exponents rotated right by one bit in bytes
 * 0..2, their total length in bits 24..28, their count in bits 29..30).
 * luts: num_luts * 256 bytes; code_lengths: 256 bytes; out: 4096 entries.
 * df11_build_format and df11_plan_from_histogram store it with a stream
 * (df11_arrays.symbol_table); a caller that uploads it spares every CTA of
 * every launch its derivation.  DF11_ERR_INVALID_ARG for null pointers or
 * num_luts outside 1..17.
 */
df11_status df11_symbol_table(const uint8_t *luts, const uint8_t *code_lengths, uint32_t num_luts, uint32_t *out);

/*
 * df11_decompress_host -- the same decode, starting and ending in host
 * memory: copies every array of *host (host pointers, ideally pinned) into
 * the device buffers named by *dev_buffers (device pointers with at least the
 * host sizes; they are overwritten although the struct's pointers are const),
 * runs df11_decompress into dst_dev, then copies the n outputs to dst_host.
 * The work goes in pieces of whole format blocks (about 8 Mi outputs each):
 * a piece's arrays are copied up on one internal stream, it is decoded on
 * `stream`, its outputs are copied down on a second internal stream, so that
 * with pinned host memory the two copy directions and the decode overlap.
 * The internal streams first wait for the work already queued on `stream`,
 * and `stream` waits for the last copy: the call is stream-ordered on
 * `stream` and does not synchronise.  BlockOffset is read on the host.
 */
df11_status df11_decompress_host(const df11_arrays *host, const df11_arrays *dev_buffers,
                                 uint16_t *dst_dev, uint16_t *dst_host,
                                 uint32_t *status_dev, void *stream);

/*
 * df11_read_status -- synchronises `stream`, reads *status_dev (device
 * pointer) and returns DF11_OK if it is 0, else DF11_ERR_CORRUPT
 * (DF11_ERR_CUDA if the copy fails).  The kernels only OR bits into the word:
 * DF11_ERR_CORRUPT's value for inconsistent data, bit 31 for a bounded wait
 * of df11_decompress_gemm that ran out.  Zero it before the calls it covers.
 */
df11_status df11_read_status(const uint32_t *status_dev, void *stream);

/* ------------------------------------------------------------------------
 * Compression of weights already in device memory.  The page compresses
 * offline ("Format DFloat11"); these entry points run the same steps on the
 * GPU and produce exactly the arrays df11_build_format builds on the host
 * (the same code, the same bytes).  Three calls:
 *   1. df11_device_histogram   exponent counts, on the device;
 *   2. df11_plan_from_histogram the code, LUTs and array sizes, on the host;
 *   3. df11_device_encode       every array, on the device, into buffers
 *                               the caller allocated with the plan's sizes.
 * ---------------------------------------------------------------------- */

/*
 * df11_device_histogram -- exponent histogram of n BF16 patterns.
 *   w_dev     device pointer, 16-byte aligned, n uint16 (only read).
 *   hist_dev  device pointer to 256 uint64, overwritten with the counts of
 *             exponents 0..255 ("Ruang kompresi": the exponent is bits 7..14).
 * Asynchronous on `stream`.  DF11_ERR_INVALID_ARG for NULL / misaligned
 * pointers, DF11_ERR_CUDA if a launch fails.
 */
df11_status df11_device_histogram(const uint16_t *w_dev, uint64_t n, uint64_t *hist_dev, void *stream);

/*
 * df11_plan_from_histogram -- the code of a stream from its exponent counts
 * ("Format DFloat11"; LUTs per "Decoding berbasis LUT hierarkis"): Huffman
 * lengths (package-merge when deeper than 32), canonical codes, LUTs and
 * CodeLengths, and the sizes of every array (total_bits = sum hist * length).
 *   hist      host pointer to 256 counts (only read).
 *   out       receives a handle owned by the caller (df11_free).  Its
 *             df11_format_arrays view has the sizes, host pointers for luts
 *             and code_lengths, NULL for the other arrays, and
 *             max_block_elems = 0 (known once the elements are encoded).
 * Errors as df11_build_format (exponents 240..255, n >= 2^32, > 16 child
 * LUTs).
 */
df11_status df11_plan_from_histogram(const uint64_t *hist, uint32_t threads_per_block, df11_format **out);

/* Scratch words df11_device_encode needs for n elements (one per chunk of
 * 8192 elements, plus one). */
uint64_t df11_device_encode_scratch_words(uint64_t n);

/*
 * df11_device_encode -- every array of the stream, on the device
 * ("Format DFloat11"; Gaps and BlockOffset per "Kernel GPU 2 tahap dan
 * metadata bantu").
 *   plan      from df11_plan_from_histogram of these elements' histogram.
 *   w_dev     device pointer, 16-byte aligned, plan's n uint16 (only read).
 *   dst_dev   device pointers with at least the plan's sizes (alignment as
 *             df11_decompress requires); all six arrays are written, the
 *             LUTs and CodeLengths copied from the plan.  Its scalar fields
 *             are not read.
 *   scratch_dev  device pointer to scratch_words uint64 (at least
 *             df11_device_encode_scratch_words(n)); contents need not start
 *             at zero and are meaningless afterwards.
 *   max_block_elems_dev  device pointer to one uint32: the largest block's
 *             element count (the df11_arrays field of the same name).
 *   status_dev  device pointer to one uint32, OR-accumulated with
 *             DF11_ERR_CORRUPT when the elements do not match the plan (an
 *             exponent without a code, or another total bit count); the
 *             arrays are then not a valid stream.  Zero it first.
 * Asynchronous on `stream`; every write stays inside the given sizes.
 * DF11_ERR_INVALID_ARG for bad pointers, sizes or alignment, DF11_ERR_CUDA
 * if a CUDA call fails.
 */
df11_status df11_device_encode(const df11_format *plan, const uint16_t *w_dev, const df11_arrays *dst_dev,
                               uint64_t *scratch_dev, uint64_t scratch_words, uint32_t *max_block_elems_dev,
                               uint32_t *status_dev, void *stream);

/*
 * df11_device_encode_static -- df11_device_encode with its scratch in a
 * fixed device array inside the library instead of a caller's buffer: the
 * call allocates nothing.  The DFloat11 page has no counterpart (it
 * compresses offline on the host); this variant is for callers that may not
 * allocate device memory at the point of the call.
 *   Limit: streams of at most 2^29 elements (65,536 chunks of 8192; the
 *   array is 512 KiB per device).  Larger plans return DF11_ERR_TOO_LARGE
 *   and nothing is launched.
 *   plan, w_dev, dst_dev, max_block_elems_dev, status_dev, stream: as
 *   df11_device_encode (status_dev must be zeroed by the caller).
 * The array is shared by every call on a device: calls that overlap in time
 * (on other streams or from other threads) race on it and must be
 * serialised by the caller.  No entry of it has to start at zero (a call
 * writes every entry it reads before reading it), so it is never cleared.
 * Each call made while `stream` is not being captured looks up the array's
 * address on the current device (cudaGetSymbolAddress), so a device reset
 * between calls, which may move the array, is picked up.  A call made while
 * `stream` is being captured reuses the last address looked up on that
 * device; make the first call on a device before any stream capture.
 * DF11_ERR_CUDA if the lookup fails or no address has been looked up yet.
 */
df11_status df11_device_encode_static(const df11_format *plan, const uint16_t *w_dev, const df11_arrays *dst_dev,
                                      uint32_t *max_block_elems_dev, uint32_t *status_dev, void *stream);

/*
 * rANS variant of the exponent coder.  The page's discussion proposes rANS
 * (range asymmetric numeral systems) as an entropy coder better suited to
 * SIMD-style hardware than Huffman coding; this variant codes the same 8-bit
 * exponents with it and keeps sign and mantissa verbatim, so the same BF16
 * matrix comes back bit for bit.  Layout (the pages fix none of it):
 *   - model: exponent counts quantised to frequencies freq[256] summing to
 *     2^prob_bits (12): every present exponent gets max(1, floor(h M / n)),
 *     then the largest frequency (ties: smallest exponent) loses one while
 *     the sum exceeds M, the largest count (ties: smallest exponent) gains
 *     one while it falls short.  Every exponent 0..255 is allowed.
 *   - state: 32 bits in [2^16, 2^32); a decode step takes slot = x mod M,
 *     the exponent s whose range [cum[s], cum[s] + freq[s]) holds it, and
 *     x = freq[s] (x >> prob_bits) + slot - cum[s]; below 2^16 the state
 *     takes the next 16-bit word: x = (x << 16) | word.
 *   - blocks of 512 * chunks elements (chunks <= 15); lane l (0..31) of
 *     block b owns elements b 512 chunks + 512 j + 16 l + i (j < chunks,
 *     i < 16), decoded in the order (j, i), all lanes stepping together;
 *     each lane has its own stream of words, and a lane whose state fell
 *     below 2^16 after a step takes the next word of it; a lane skips steps
 *     whose element lies at or past n.  Every lane ends the block at
 *     x = 2^16 with its stream used up.
 *   - states[32 b + l] is lane l's start state in block b; the words of
 *     block b are words[block_word[b] .. block_word[b + 1]): lane 0's stream,
 *     then lane 1's, ..., lane 31's, lane_words[32 b + l] words each (at most
 *     one per step: 16 chunks <= 240).
 */
typedef struct df11_rans_format df11_rans_format;

typedef struct df11_rans_arrays {
    uint64_t n;                          /* BF16 elements */
    uint64_t num_words;                  /* 16-bit words of all blocks */
    uint32_t prob_bits;                  /* 12 */
    uint32_t chunks;                     /* 16-element chunks per lane and block, 1..15 */
    uint32_t num_blocks;                 /* ceil(n / (512 chunks)) */
    uint32_t max_block_words;            /* largest block_word[b + 1] - block_word[b] */
    const uint16_t *words;               /* num_words + 8 (zero padding) */
    const uint32_t *states;              /* 32 * num_blocks */
    const uint32_t *block_word;          /* num_blocks + 1 */
    const uint8_t *lane_words;           /* 32 * num_blocks: words of each lane's stream */
    const uint16_t *freq;                /* 256, summing to 2^prob_bits (0 when n = 0) */
    const uint8_t *packed_sign_mantissa; /* round_up(n, 16) + 16 bytes, 16-B aligned */
    uint64_t packed_sign_mantissa_bytes;
} df11_rans_arrays;

/*
 * df11_rans_build -- host: compress num_mats BF16 matrices (as
 * df11_build_format; matrices concatenated) with the rANS exponent coder.
 *   chunks: 16-element chunks per lane and block (0 = 10: 5120-element blocks).
 * On success *out owns every array (host memory); DF11_ERR_TOO_LARGE for
 * n >= 2^32, DF11_ERR_INVALID_ARG for bad pointers or chunks > 15.
 */
df11_status df11_rans_build(const uint16_t *const *mats, const uint64_t *counts, int num_mats, uint32_t chunks,
                            df11_rans_format **out);

/* df11_rans_format_arrays -- borrowed host pointers and sizes of a built
 * stream (valid until df11_rans_free). */
df11_status df11_rans_format_arrays(const df11_rans_format *f, df11_rans_arrays *out);

/* df11_rans_free -- releases a stream (NULL-safe). */
void df11_rans_free(df11_rans_format *f);

/*
 * df11_rans_decompress -- device: rebuild the n BF16 values of a stream whose
 * arrays the caller has uploaded (dev: the same struct with device pointers)
 * into dst_dev (16-byte aligned, n elements), asynchronously on `stream`.
 * One warp decodes one block; the exponents of a lane's 16 elements are
 * merged with their sign/mantissa bytes and stored with one 32-byte store.
 * Inconsistent words, states, offsets or lane counts set DF11_ERR_CORRUPT
 * in *status_dev (caller-zeroed) and leave that block's outputs
 * unspecified; nothing traps or reads out of bounds.  Argument errors
 * (including words not 16-byte aligned) return DF11_ERR_INVALID_ARG
 * synchronously.
 */
df11_status df11_rans_decompress(const df11_rans_arrays *dev, uint16_t *dst_dev, uint32_t *status_dev,
                                 void *stream);

#ifdef __cplusplus
}
#endif

#endif /* DF11_H */
