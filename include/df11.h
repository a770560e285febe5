/*
 * df11.h -- C ABI of the DFloat11 (DF11) exponent-stream codec for B200.
 *
 * DF11 stores a BF16 weight as a canonical Huffman code of its 8-bit exponent
 * plus one raw byte (sign << 7 | 7-bit mantissa); decoding on the GPU rebuilds
 * the bit-exact BF16 matrices of one transformer block in one launch.
 * Method: "DFloat11: lossless BFloat16 compression" (ai-infrastructure.net),
 * sections "What it is" (field split), "Architecture" (hierarchical lookup
 * tables, the two-phase kernel with Gaps and BlockOutputPos, block-level
 * batching) and "How it works: the core algorithm" (Huffman lengths,
 * canonical codes, MSB-first encoding).
 *
 * Conventions for every call:
 *   - Plain C, no exceptions cross the ABI; each call returns df11_status.
 *   - The caller owns every buffer.  The library allocates no device memory,
 *     keeps no pointer after a call returns and never synchronises a stream.
 *   - Host buffers are host pointers; fields documented as "device" are CUDA
 *     device pointers on the current device.
 *
 * Artifact format (one block = every matrix that shares one codebook):
 *   exponent code  canonical Huffman code, length 1..max_code_len (<= 16),
 *                  codes assigned in ascending (length, symbol) order.
 *   exp_stream     codes of all elements, in element order, MSB-first: stream
 *                  bit i is bit 7 - i%8 of byte i/8.  Zero padded to
 *                  n_threads * bytes_per_thread + DF11_STREAM_PAD bytes.
 *   thread slice   with B = 8 * bytes_per_thread, thread g owns stream bits
 *                  [B*g, B*g + B) and decodes every code that STARTS in that
 *                  slice and before total_bits; a code may run up to 15 bits
 *                  past it.
 *   gaps           4-bit offset, per thread, of the first code start in its
 *                  slice (the end of the stream counts as a start; slices at
 *                  or past the end hold 0).  Two per byte, thread 2j in the
 *                  low nibble of byte j.
 *   counts         uint8 per thread: the number of codes that start in its
 *                  slice (0 past the end of the stream; at most
 *                  ceil(8 * bytes_per_thread / min_code_len), so at most 128).  The
 *                  pages store no per-thread count: their decoder's first
 *                  phase decodes every slice once only to count its codes.
 *                  Stored, the counts give each thread its output offset
 *                  from one warp prefix sum before it decodes, so the slice
 *                  is decoded once, straight into place; they cost one byte
 *                  per slice (about 1.5% of a compressed LLM block).
 *   chunk_pos      uint32[n_chunks+1]: chunk c (threads_per_chunk = 32
 *                  threads, one warp) writes elements [chunk_pos[c],
 *                  chunk_pos[c+1]); the last entry is n_elements.  (The pages
 *                  keep one such 32-bit position per thread block,
 *                  "BlockOutputPos"; here it is one per warp, so warps never
 *                  wait for each other.)
 *   signmant       uint8[n_elements] (padded to a multiple of 16): byte k is
 *                  (sign << 7) | mantissa of element k.
 *   lut            n_tables * 256 uint16 entries; table 0 is indexed by the
 *                  next 8 stream bits.  Entry bits:
 *                    bit 15 = 1       pointer: bits 0..7 name the sub-table
 *                                     (1..n_tables-1) indexed by the 8 bits
 *                                     after the first 8;
 *                    bit 15 = 0       leaf: bits 0..7 the exponent, bits 8..12
 *                                     the total code length (1..16);
 *                    bit 14 = 1       no code has this prefix (only in a
 *                                     single-symbol codebook); bits 8..12 hold
 *                                     1; a decoder that reads it reports a
 *                                     corrupt stream.
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
    DF11_ERR_INVALID_ARGUMENT = 1, /* bad pointer, size, layout or parameter    */
    DF11_ERR_BUFFER_TOO_SMALL = 2, /* a caller buffer is shorter than required  */
    DF11_ERR_OVERFLOW = 3,         /* element count >= 2^32                     */
    DF11_ERR_CORRUPT = 4,          /* artifact fails a structural check         */
    DF11_ERR_CUDA = 5,             /* a CUDA runtime call failed                */
    DF11_ERR_TIMEOUT = 6           /* reserved (device waits report DF11_DEVERR_TIMEOUT) */
} df11_status;

/* Bits the decoder ORs into the caller's device error word. */
#define DF11_DEVERR_COUNT 0x1u    /* a chunk's counts disagree with chunk_pos, a
                                     count is impossible, or a thread's codes
                                     do not end where the next thread's first
                                     code starts (corrupt stream, gaps or
                                     counts); a chunk whose counts disagree
                                     with chunk_pos writes nothing */
#define DF11_DEVERR_BAD_CODE 0x2u /* a window hit a "no code" or bad pointer
                                     entry (corrupt stream or table)           */
#define DF11_DEVERR_BAD_POS 0x4u  /* chunk_pos not monotone or beyond
                                     out_capacity; that chunk writes nothing   */
#define DF11_DEVERR_TIMEOUT 0x8u  /* a bounded wait for a staged copy ran out;
                                     that chunk's output is not trustworthy    */
#define DF11_DEVERR_MISMATCH 0x10u /* GPU compressor: an exponent without a code,
                                     or a bit total other than the codebook's  */
#define DF11_DEVERR_CHECKSUM 0x20u /* df11_verify_device_async: a segment's
                                     CRC-32C differs from the expected value;
                                     df11_decompress_verified_async: a chunk's
                                     sum differs                              */
#define DF11_DEVERR_BOUNDS 0x40u   /* checked build (libdf11_checked.so) only: an
                                     invariant that keeps an access in bounds
                                     failed; the access was skipped            */

#define DF11_MAX_CODE_LEN 16u     /* longest code the format allows           */
#define DF11_MIN_CODE_LEN_CAP 8u  /* smallest cap accepted by build_codebook  */
#define DF11_STREAM_PAD 16u       /* zero bytes after the last thread slice   */
#define DF11_THREADS_PER_CHUNK 32u /* one warp per chunk                       */

/* Codebook of one block.  Caller-allocated plain data (about 134 KB). */
typedef struct {
    uint64_t histogram[256];   /* exponent counts over the block's matrices   */
    uint32_t code[256];        /* canonical code, right-aligned in code_len   */
    uint8_t code_len[256];     /* 0 = exponent absent                          */
    uint32_t max_code_len;     /* the cap the lengths were built under         */
    uint32_t n_symbols;        /* exponents that occur                         */
    uint32_t n_tables;         /* lookup tables used in lut (1..256)           */
    uint32_t longest_code;     /* max code_len                                 */
    uint64_t n_elements;       /* total elements histogrammed                  */
    uint64_t total_bits;       /* sum histogram[s] * code_len[s]              */
    uint16_t lut[256 * 256];   /* first n_tables * 256 entries used            */
} df11_codebook;

/* Compress-time layout: threads per chunk and bytes of stream per thread.
 * The library decodes threads_per_chunk == 32 (one warp) and bytes_per_thread in
 * {8, 16} (64- or 128-bit slices; the pages use 8). */
typedef struct {
    uint32_t threads_per_chunk;
    uint32_t bytes_per_thread;
} df11_layout;

/* Exact sizes of the arrays df11_compress fills. */
typedef struct {
    uint64_t n_chunks;
    uint64_t n_threads;         /* n_chunks * threads_per_chunk                */
    uint64_t exp_stream_bytes;  /* n_threads * bytes_per_thread + STREAM_PAD   */
    uint64_t gaps_bytes;        /* n_threads / 2                               */
    uint64_t counts_bytes;      /* n_threads                                   */
    uint64_t chunk_pos_count;   /* n_chunks + 1 (uint32 entries)               */
    uint64_t signmant_bytes;    /* n_elements rounded up to a multiple of 16   */
    uint64_t lut_entries;       /* n_tables * 256 (uint16 entries)             */
} df11_sizes;

/* Header fields shared by the host and device views of a block.
 * min_code_len is the shortest code in the codebook; the decoder treats any
 * table entry shorter than it as corrupt, which bounds the codes per slice
 * and so the decoder's per-warp buffers. */
typedef struct {
    uint32_t max_code_len;
    uint32_t threads_per_chunk;
    uint32_t bytes_per_thread;
    uint32_t n_tables;
    uint32_t min_code_len;
    uint32_t reserved;          /* 0 */
    uint64_t total_bits;
    uint64_t n_elements;
    uint64_t n_chunks;
} df11_header;

/* A compressed block in host memory; every array is caller-owned and sized by
 * df11_compress_sizes.  `*_bytes` / `*_count` fields give the buffer lengths. */
typedef struct {
    df11_header hdr;
    uint8_t *exp_stream;  uint64_t exp_stream_bytes;
    uint8_t *gaps;        uint64_t gaps_bytes;
    uint8_t *counts;      uint64_t counts_bytes;
    uint32_t *chunk_pos;  uint64_t chunk_pos_count;
    uint8_t *signmant;    uint64_t signmant_bytes;
    uint16_t *lut;        uint64_t lut_entries;
} df11_host_block;

/* The same block after the caller copied each array to the GPU (device
 * pointers).  Every array must be 16-byte aligned (any cudaMalloc / torch
 * allocation is).  decode_table is optional: NULL, or the
 * DF11_DECODE_TABLE_ENTRIES entries df11_build_decode_table made from this
 * block's tables, copied to the GPU (see there). */
typedef struct {
    df11_header hdr;
    const uint8_t *exp_stream;  uint64_t exp_stream_bytes;
    const uint8_t *gaps;        uint64_t gaps_bytes;
    const uint8_t *counts;      uint64_t counts_bytes;
    const uint32_t *chunk_pos;  uint64_t chunk_pos_count;
    const uint8_t *signmant;    uint64_t signmant_bytes;
    const uint16_t *lut;        uint64_t lut_entries;
    const uint64_t *decode_table;
} df11_device_block;

/* Host.  Histograms the exponents of n_mats BF16 matrices (bit patterns,
 * host memory, mats[i] holds numel[i] elements), builds optimal code lengths
 * under max_code_len (in [8, 16]; exactly optimal, not a heuristic), the
 * canonical codes and the two-level 256-entry lookup tables.
 * ("What it is"; "Architecture", hierarchical lookup tables; "How it works",
 * huffman_lengths / canonical_codes.)
 * Errors: INVALID_ARGUMENT for null pointers, n_mats == 0, zero elements or a
 * cap outside [8, 16]; OVERFLOW when the element count reaches 2^32. */
df11_status df11_build_codebook(const uint16_t *const *mats, const uint64_t *numel,
                                uint32_t n_mats, uint32_t max_code_len,
                                df11_codebook *out);

/* Host.  The codebook for a given 256-bin exponent histogram (for example
 * one df11_histogram_device computed): the same lengths, codes and tables
 * df11_build_codebook would build from the data.  Errors as for
 * df11_build_codebook. */
df11_status df11_build_codebook_from_histogram(const uint64_t histogram[256], uint32_t max_code_len,
                                               df11_codebook *out);

/* Host.  Sizes of every array df11_compress fills for this codebook and
 * layout, from the histogram alone (no pass over the data).
 * Errors: INVALID_ARGUMENT for an unsupported layout or an empty codebook. */
df11_status df11_compress_sizes(const df11_codebook *cb, const df11_layout *layout,
                                df11_sizes *out);

/* Host.  The slice width this library decodes a block fastest with: 8 bytes
 * per thread (the pages' layout, "Architecture") when the block's shortest
 * code is 1 bit -- 16-byte slices of 1-bit codes need twice the decoder's
 * per-warp buffers, so half the warps fit -- or when the block has fewer
 * 16-byte-slice chunks than the decoder keeps warps resident on sm_count
 * SMs (DF11_DECODE_WARPS_PER_SM each): shorter chunks then finish sooner and
 * spread over more warps; otherwise 16.  Returns 0 for a null or empty
 * codebook or sm_count == 0. */
#define DF11_DECODE_WARPS_PER_SM 46u
uint32_t df11_preferred_bytes_per_thread(const df11_codebook *cb, uint32_t sm_count);

/* Host.  Encodes one block ("Architecture": Gaps, BlockOutputPos; "How it
 * works": encode).  `out` carries caller buffers of at least the sizes
 * df11_compress_sizes reports; the call fills them and out->hdr.  The
 * matrices must be the ones the codebook was built from (same histogram).
 * Errors: INVALID_ARGUMENT (bad pointers/layout, histogram mismatch),
 * BUFFER_TOO_SMALL, OVERFLOW. */
df11_status df11_compress(const df11_codebook *cb, const df11_layout *layout,
                          const uint16_t *const *mats, const uint64_t *numel,
                          uint32_t n_mats, df11_host_block *out);

/* Host.  Structural checks of a block without decoding it: header against
 * array sizes, chunk_pos monotone from 0 to n_elements, every gap below the
 * code-length cap, every table entry well formed.  Returns CORRUPT on the
 * first failure, INVALID_ARGUMENT for null pointers. */
df11_status df11_validate(const df11_host_block *blk);

/* Host.  The decoder's multi-code table for a block's lookup tables
 * (lut: n_tables * 256 entries, as df11_compress writes them; min_code_len
 * from the block header).  The decode kernel indexes it with the next
 * DF11_DECODE_TABLE_WINDOW_BITS stream bits and takes up to four whole
 * codes per lookup; it is a function of the tables alone, so it is built
 * once per block (like the tables, at compress or load time) and kept on
 * the GPU beside the block (df11_device_block.decode_table).  Without it,
 * every decode CTA builds the same table in its prologue.  Entry k (a
 * uint64) serves the window whose first stream bit is bit 0 of k: bits
 * 0..31 hold the whole codes the window starts with (at most four), as
 * exponents rotated right by one bit (bit 0 moved to bit 7), one per byte,
 * unused bytes zero; bits 32..63 hold their total length | (8 x count) << 16,
 * or 0x80000000 when the first code is longer than the window.  Entries are
 * read as malformed tables are: the decoder treats bad entries of `lut`
 * (and shorter than min_code_len) as "no code" before building.  A table
 * that is not this block's gives wrong output, never an access out of
 * bounds: the kernel replaces entries whose length and count are impossible
 * by the long-code marker, and masks unused symbol bytes.
 * ("Architecture", hierarchical lookup tables kept in SRAM.)
 * Errors: INVALID_ARGUMENT for null pointers, n_tables outside 1..256 or
 * min_code_len outside 1..16. */
#define DF11_DECODE_TABLE_WINDOW_BITS 11u
#define DF11_DECODE_TABLE_ENTRIES 2048u   /* 16 KB */
df11_status df11_build_decode_table(const uint16_t *lut, uint32_t n_tables, uint32_t min_code_len,
                                    uint64_t *table);

/* GPU.  Enqueues ONE kernel launch on `stream` (a cudaStream_t; NULL = the
 * legacy default stream) that decodes every element of the block into
 * out_bf16[0 .. n_elements) (device, 16-byte aligned, BF16 bit patterns);
 * matrix i of the block starts at the sum of the previous matrices' sizes.
 * ("Architecture": one batched decode per transformer block.)
 * Host-side checks only: INVALID_ARGUMENT for null or misaligned pointers,
 * an unsupported layout, array sizes that disagree with the header, or
 * out_capacity < n_elements; CUDA when the launch fails.  Problems found on
 * the device (a corrupt artifact) OR DF11_DEVERR_* bits into *d_error
 * (device uint32, may be NULL; the caller zeroes it); the kernel never writes
 * outside [0, out_capacity) and never traps.  Safe to call concurrently on
 * different streams. */
df11_status df11_decompress_async(const df11_device_block *blk, uint16_t *out_bf16,
                                  uint64_t out_capacity, uint32_t *d_error,
                                  void *stream);

/* GPU.  df11_decompress_async launching max_ctas CTAs (at most one per 16
 * chunks; 0 = one wave of resident CTAs on every SM).  Decode CTAs loop over
 * the block's chunks, so any count decodes the whole block: fewer than a
 * wave leave SMs to work on other streams, more than a wave run as waves of
 * short-lived CTAs that each free their SM when done, which lets kernels of
 * a higher-priority stream (such as the matrix products consuming the
 * previous block) take SMs between them ("Architecture": decode runs before
 * each block's forward pass; overlapping it with the previous block's
 * compute is this library's addition).  Same checks and errors as
 * df11_decompress_async. */
df11_status df11_decompress_async_ctas(const df11_device_block *blk, uint16_t *out_bf16,
                                       uint64_t out_capacity, uint32_t *d_error,
                                       uint32_t max_ctas, void *stream);

/* Bytes of a scheduling workspace. */
#define DF11_SCHED_WORKSPACE_BYTES 2048u

/* GPU.  df11_decompress_async_ctas with a scheduling workspace: device
 * memory of DF11_SCHED_WORKSPACE_BYTES, 16-byte aligned, all zero before
 * its first use (cudaMemset once); the kernel leaves it zero when it
 * completes.  Without one (NULL) warp k of the grid's W warps decodes
 * chunks k, k + W, k + 2W, ...; with one, in a block of at least five such
 * rounds the chunks of the last three are instead claimed one at a time by
 * whichever warps get there first, so warps and SMs that ran faster take
 * more of them and the launch ends within about one chunk time of its last
 * claim.  Output is identical either way.
 * (The pages leave the split of chunks over thread blocks open,
 * "Architecture"; this is the library's choice.)  A workspace serves one
 * launch at a time: launches that may run concurrently (different streams,
 * or graphs replayed on different streams) need different workspaces, as
 * with a cuBLAS workspace.  Same checks and errors as df11_decompress_async,
 * plus INVALID_ARGUMENT for a misaligned workspace. */
df11_status df11_decompress_async_ws(const df11_device_block *blk, uint16_t *out_bf16,
                                     uint64_t out_capacity, uint32_t *d_error,
                                     uint32_t max_ctas, void *workspace, void *stream);

/* GPU.  Decodes only chunks [chunk_begin, chunk_end) of the block (chunk c =
 * threads 32c .. 32c + 31, DF11_THREADS_PER_CHUNK * bytes_per_thread bytes of
 * exp_stream): out_bf16[chunk_pos[chunk_begin] .. chunk_pos[chunk_end]) and
 * nothing else.  Chunks are independent given their gaps and output
 * positions ("Architecture": each thread block decodes its chunk alone), so
 * a block can be decoded piece by piece as it arrives, for instance while
 * the next piece is copied in and the last one copied out.  One launch reads
 * only:
 *   - exp_stream bytes [32 W chunk_begin, 32 W chunk_end + DF11_STREAM_PAD)
 *     (W = bytes_per_thread);
 *   - gaps bytes [16 chunk_begin, 16 chunk_end + 1) (the low nibble of the
 *     last one, the gap of the thread after the range, when chunk_end <
 *     n_chunks);
 *   - counts bytes [32 chunk_begin, 32 chunk_end);
 *   - chunk_pos[chunk_begin .. chunk_end];
 *   - signmant bytes [p0 & ~15, (p1 + 15) & ~15), with p0 and p1 the
 *     positions of chunk_begin and chunk_end;
 *   - the tables.
 * `workspace` as for df11_decompress_async_ws (may be NULL).  Errors: those
 * of df11_decompress_async, and INVALID_ARGUMENT for an empty range or one
 * past n_chunks, or a misaligned workspace. */
df11_status df11_decompress_range_async(const df11_device_block *blk, uint64_t chunk_begin,
                                        uint64_t chunk_end, uint16_t *out_bf16, uint64_t out_capacity,
                                        uint32_t *d_error, void *workspace, void *stream);

/* GPU, diagnostic.  Runs the decode kernel's bounded barrier wait on a
 * barrier that nothing arrives on: one warp polls it `polls` times (1..4096),
 * gives up and writes DF11_DEVERR_TIMEOUT to *d_status (device uint32) --
 * what a decode whose staged copy never lands ORs into its error word.
 * Shows that a wait that runs out returns a status instead of hanging, with
 * no fault and the context still usable.  (No counterpart on the pages,
 * whose kernel neither stages copies nor reports errors; "Failure modes"
 * only warns that corruption is silent.)  Errors: INVALID_ARGUMENT, CUDA. */
df11_status df11_selftest_bounded_wait(uint32_t polls, uint32_t *d_status, void *stream);

/* ---- Decode fused with its consumer: matrix-vector products --------------
 * The pages decode a block into a BF16 buffer and then run its matrix
 * products ("DFloat11: lossless BFloat16 compression", "Architecture":
 * decode, block matmuls, discard).  For a few tokens the products are
 * matrix-vector work bound by reading the weights, so this call multiplies
 * each weight as it is decoded and never writes the BF16 block to HBM
 * (this library's addition).  Matrix i of the block (mats[i], in block
 * order, rows x cols row-major, cols a multiple of 8) gets
 *     y[t][r] += sum_c W[r][c] * x[t][c],   t < n_tokens (1..8),
 * with x device BF16 (n_tokens x cols, token-major, 16-byte aligned) and y
 * device FP32 (n_tokens x rows, 4-byte aligned, zeroed by the caller: the
 * kernel accumulates into it with atomic adds, so the summation order and
 * the last bits of y vary between runs).  Products and sums are FP32.  The
 * activations should be finite: a chunk's end groups multiply the
 * neighbouring chunk's columns by +0, so an infinite x entry can turn an
 * infinite y into NaN. */
typedef struct {
    uint64_t rows;
    uint64_t cols;
    const uint16_t *x;
    float *y;
} df11_gemv_matrix;

/* GPU.  One launch on `stream`.  `workspace` is a scheduling workspace as
 * for df11_decompress_async_ws, or NULL.  Errors: INVALID_ARGUMENT (the
 * block checks of df11_decompress_async, n_mats outside 1..128, n_tokens
 * outside 1..8, a matrix with cols not a multiple of 8 or misaligned
 * pointers, matrices that do not add up to the block's elements, a
 * misaligned workspace), CUDA.  Device errors go to *d_error as for
 * df11_decompress_async. */
df11_status df11_decode_gemv_async(const df11_device_block *blk, const df11_gemv_matrix *mats,
                                   uint32_t n_mats, uint32_t n_tokens, uint32_t *d_error,
                                   void *workspace, void *stream);

/* ---- GPU-side compressor --------------------------------------------------
 * The pages compress on the CPU only ("DFloat11: lossless BFloat16
 * compression", "How to develop with it": minutes per block on one thread).
 * These calls do the same on the GPU for a block already in device memory,
 * producing exactly the arrays df11_compress produces for the same codebook.
 */

/* GPU.  Adds the exponent histogram of d_in[0 .. n) (device, BF16 bit
 * patterns, 16-byte aligned) into d_hist (device uint64[256], 8-byte
 * aligned; the caller zeroes it).  One launch on `stream`.  Errors:
 * INVALID_ARGUMENT for null/misaligned pointers or n == 0, CUDA. */
df11_status df11_histogram_device(const uint16_t *d_in, uint64_t n, uint64_t *d_hist, void *stream);

/* Scratch bytes df11_compress_device needs for n elements: 12 bytes per
 * 8192 elements (rounded up) for the segment bit counts and starts, and 2
 * bytes per 32 elements for the bit counts the encode pass reuses. */
uint64_t df11_compress_device_scratch_bytes(uint64_t n_elements);

/* GPU.  Encodes d_in[0 .. n) (device, the block's matrices concatenated,
 * 16-byte aligned) with the codebook cb (host) into the device arrays of
 * `out` (exp_stream, gaps, counts, chunk_pos, signmant; sized by
 * df11_compress_sizes, 16-byte aligned) and fills out->hdr.  out->lut is not
 * touched: the caller copies cb->lut (n_tables * 256 entries) into it.
 * d_scratch (device, 16-byte aligned, >= df11_compress_device_scratch_bytes)
 * is caller-owned work space.  Four kernel launches on `stream`; nothing is
 * allocated and nothing synchronises.  Data that disagree with the codebook
 * (an exponent without a code, another bit total) OR DF11_DEVERR_MISMATCH
 * into *d_error (device, may be NULL).  Errors: INVALID_ARGUMENT (pointers,
 * alignment, n != cb->n_elements, layout), BUFFER_TOO_SMALL, OVERFLOW, CUDA. */
df11_status df11_compress_device(const df11_codebook *cb, const df11_layout *layout,
                                 const uint16_t *d_in, uint64_t n, df11_device_block *out,
                                 void *d_scratch, uint64_t scratch_bytes, uint32_t *d_error,
                                 void *stream);

/* ---- allocation-free compressor (no counterpart on the pages) -------------
 * The same GPU compression as df11_compress_device, for callers that cannot
 * let a library allocate device memory -- a serving runtime or framework that
 * reserves the whole GPU for its own pool (cudaMalloc would fail or escape
 * its accounting), or code that must not call cudaFree, which synchronises
 * the device.  Instead of caller scratch it uses one fixed device array of
 * DF11_NOALLOC_SCRATCH_BYTES that the library holds on every GPU that loads
 * it, until the process exits.
 *   - Blocks of more than DF11_NOALLOC_MAX_ELEMENTS elements are rejected
 *     with DF11_ERR_BUFFER_TOO_SMALL; nothing is launched.
 *   - The first call on a device looks up the array's device address with
 *     cudaGetSymbolAddress (with that device current); make that first call
 *     before any stream capture.  Later calls in the same CUDA context reuse
 *     the address; a call in another context (a new primary context after
 *     cudaDeviceReset, or a driver context of the caller's) looks it up
 *     again, so make the first call in each context before capturing too.
 *   - Every call shares the one array, which keeps the last call's contents;
 *     each call writes all it reads, so nothing needs clearing.  Calls whose
 *     work overlaps on the GPU (another stream, another host thread) race on
 *     the array: order them on one stream or synchronise between them.
 *   - Nothing is allocated or freed.  Arguments, outputs, error behaviour and
 *     results are those of df11_compress_device. */
#define DF11_NOALLOC_SCRATCH_BYTES (1u << 20)
#define DF11_NOALLOC_MAX_ELEMENTS 715816960ull   /* 87380 segments of 8192 */
df11_status df11_compress_device_noalloc(const df11_codebook *cb, const df11_layout *layout,
                                         const uint16_t *d_in, uint64_t n, df11_device_block *out,
                                         uint32_t *d_error, void *stream);

/* Human-readable name of a status code (static string). */
/* ---- Integrity: CRC-32C per 4096-byte segment -----------------------------
 * One flipped bit in the exponent stream desyncs the Huffman decoder and
 * silently rewrites most of a tensor; the pages tell users to checksum DF11
 * artifacts on download and after every copy ("DFloat11: lossless BFloat16
 * compression", "How to run it in production" and "Failure modes").  The
 * checksum of a block is a list of CRC-32C values (Castagnoli: reflected
 * polynomial 0x82F63B78, initial value and final XOR 0xFFFFFFFF; the
 * iSCSI / SSE4.2 CRC), one per DF11_CRC_SEGMENT_BYTES-byte segment of each
 * array, arrays in the order exp_stream, gaps, counts, chunk_pos
 * (little-endian bytes), signmant, lut (little-endian bytes), each over the
 * array sizes in
 * the block struct; an array's last segment may be shorter.  Segments let
 * the GPU check run in parallel and point at the damaged region.  The
 * decoder itself flags desynchronised chunks (DF11_DEVERR_COUNT), but not a
 * flipped sign or mantissa bit: only the checksum covers those. */
#define DF11_CRC_SEGMENT_BYTES 4096u

/* Host.  Number of checksum values of a block (0 for NULL). */
uint64_t df11_checksum_count(const df11_host_block *blk);

/* Host.  The CRC-32C of data[0 .. n) (the standard check value of the
 * nine bytes "123456789" is 0xE3069283). */
uint32_t df11_crc32c(const void *data, uint64_t n);

/* Host.  Writes the block's checksum list into crc[0 .. n_crc);
 * n_crc must equal df11_checksum_count(blk).  INVALID_ARGUMENT otherwise or
 * for null pointers. */
df11_status df11_checksum(const df11_host_block *blk, uint32_t *crc, uint64_t n_crc);

/* GPU.  Computes the same list for a block in device memory into d_crc
 * (device, 4-byte aligned, n_crc values = the count of the matching host
 * block).  One launch on `stream`.  INVALID_ARGUMENT for null or
 * misaligned pointers (arrays must be 16-byte aligned) or a wrong n_crc;
 * CUDA when the launch fails. */
df11_status df11_checksum_device_async(const df11_device_block *blk, uint32_t *d_crc, uint64_t n_crc,
                                       void *stream);

/* GPU.  Recomputes the list and compares it with d_expected (device): each
 * mismatching segment ORs DF11_DEVERR_CHECKSUM into *d_error and, when
 * d_first_bad (device uint64, 8-byte aligned, set to UINT64_MAX by the
 * caller) is given, lowers it to the segment's index.  Same argument errors
 * as df11_checksum_device_async; d_error must not be NULL. */
df11_status df11_verify_device_async(const df11_device_block *blk, const uint32_t *d_expected,
                                     uint64_t n_crc, uint32_t *d_error, uint64_t *d_first_bad,
                                     void *stream);

/* ---- Integrity inside the decode: per-chunk sums -------------------------
 * A checksum the decode kernel can check as it decodes, from the bytes it
 * reads anyway (this library's addition; the pages ask only to checksum
 * artifacts, "How to run it in production").  One 32-bit sum per chunk c
 * (threads 32c .. 32c + 31, B = 8 * bytes_per_thread bits per slice): the
 * sum mod 2^32 of mix(v, tag) over
 *   - the chunk's 32 B stream bits as B words: bit i of word k is chunk
 *     stream bit 32k + i (MSB-first within bytes); tag k;
 *   - each thread t = 0..31: v = gap | count << 8; tag 0x10000 + t;
 *   - v = chunk_pos[c] (tag 0x20000) and chunk_pos[c + 1] (tag 0x20001);
 *   - the sign|mantissa bytes of elements [p0, p1) = [chunk_pos[c],
 *     chunk_pos[c + 1]), b = p0 rounded down to a multiple of 8: each group
 *     [8q, 8q + 8) inside [p0, p1) as two little-endian words, tags 0x100000
 *     + 2r and 0x100000 + 2r + 1 (r = q - b / 8); every other element e as its
 *     byte, tag 0x200000 + e - b;
 *   - chunk 0 only: the tables as little-endian words (entries 2i, 2i + 1),
 *     tag 0x400000 + i;
 * mix(v, tag) = y ^ (y >> 16) with y = (v ^ tag * 0x9E3779B1) * 0x85EBCA6B,
 * all mod 2^32 -- for a fixed tag a bijection of v, so a change in any one
 * item changes the sum.  Unlike the CRC-32C list it can be checked by the
 * decode itself at a small cost (about five instructions per 4 bytes), and
 * it points at the damaged chunk.  The decoder's multi-code table is not
 * covered (it is derived from the tables). */

/* Host.  Writes the n_chunks per-chunk sums of blk into sums[0 .. n).
 * INVALID_ARGUMENT for null pointers, n != blk->hdr.n_chunks, a layout the
 * library does not decode, arrays shorter than the header implies, or
 * positions that decrease or pass the sign|mantissa bytes. */
df11_status df11_chunk_sums(const df11_host_block *blk, uint32_t *sums, uint64_t n);

/* GPU.  df11_decompress_range_async over the whole block (chunk_begin = 0,
 * chunk_end = n_chunks) that also computes every chunk's sum as it decodes
 * and compares it with d_sums[c] (device, n_chunks values of
 * df11_chunk_sums): a mismatch ORs DF11_DEVERR_CHECKSUM into *d_error.  A
 * chunk is bad when its sum differs or its decode reports an error (its
 * flag); when d_first_bad (device uint64, 8-byte aligned, set to UINT64_MAX
 * by the caller) is given, it is lowered to the lowest bad chunk.  A damaged
 * byte is reported at its own chunk or at the chunk before it, which also
 * reads the next chunk's first stream word (codes that cross into it) and
 * its first thread's gap.  workspace: as for df11_decompress_async_ws.  Chunks of
 * a CTA whose tables never arrived are neither decoded nor summed (that
 * sets DF11_DEVERR_TIMEOUT).  The output is written as by
 * df11_decompress_async.  Errors: those of df11_decompress_async_ws, and
 * INVALID_ARGUMENT for null or misaligned d_sums, d_error or d_first_bad. */
df11_status df11_decompress_verified_async(const df11_device_block *blk, uint16_t *out_bf16,
                                           uint64_t out_capacity, uint32_t *d_error, const uint32_t *d_sums,
                                           uint64_t *d_first_bad, void *workspace, void *stream);

/* ---- Streamed decoding: upload -> decode -> consume ----------------------
 * The pages decode each transformer block right before its matrix products
 * and discard the BF16 copy afterwards ("DFloat11: lossless BFloat16
 * compression", "Architecture": block-level batching); the upstream README
 * adds CPU offloading with one block on the GPU at a time ("DFloat11:
 * Lossless Compression of LLMs and Diffusion Models for Efficient GPU
 * Inference", news "Efficient CPU Offloading Now Supported!").  A pipeline
 * orders those stages on the caller's streams so that uploading block i+1,
 * decoding it and consuming block i overlap.
 *
 * A pipeline has n_slots slots; slot s pairs a caller-owned device staging
 * block (for uploaded compressed arrays) with a caller-owned output buffer.
 * It owns only CUDA events (three per slot), never device memory, and never
 * blocks the host.  Ordering per slot:
 *   upload  (copy stream)     waits until the slot's previous decode ran;
 *   decode  (decode stream)   waits for the slot's last upload and for the
 *                             consumer's release of the slot's output;
 *   acquire (consumer stream) waits for the slot's last decode;
 *   release (consumer stream) marks the slot's output free.
 * A slot used without upload (block already in HBM) skips the first wait.
 * Each wait refers to the event's most recent record when the call is made,
 * so enqueue the stages in block order: a slot's next upload after its
 * previous decode, its next decode after the consumer's release.  Calls
 * must come from one host thread per pipeline, on the device that was
 * current at creation (else INVALID_ARGUMENT). */
typedef struct df11_pipeline df11_pipeline;

/* Host.  Creates a pipeline of n_slots (1..64) slots.  Errors:
 * INVALID_ARGUMENT, CUDA (no device or event creation failed). */
df11_status df11_pipeline_create(uint32_t n_slots, df11_pipeline **out);

/* Host.  Destroys the pipeline's events (work already enqueued still runs). */
df11_status df11_pipeline_destroy(df11_pipeline *p);

/* Copy stage.  Enqueues on copy_stream the host -> device copies of src's
 * six arrays into dst's arrays (sizes from src; src should be pinned host
 * memory for the copies to overlap with kernels).  dst->hdr is not written:
 * the caller decodes with src->hdr.  Errors: INVALID_ARGUMENT (null
 * pointers, slot out of range, wrong device), BUFFER_TOO_SMALL (a dst array
 * smaller than its src, checked before anything is enqueued), CUDA. */
df11_status df11_pipeline_upload(df11_pipeline *p, uint32_t slot, const df11_host_block *src,
                                 const df11_device_block *dst, void *copy_stream);

/* Decode stage.  Enqueues on decode_stream the slot's waits and
 * df11_decompress_async_ws(blk, out_bf16, out_capacity, d_error, max_ctas,
 * workspace), then marks the slot decoded.  Decodes of one slot are ordered
 * by its events, so a slot can keep one workspace; slots whose decodes may
 * overlap (other decode streams) need different ones.  NULL = the static
 * chunk schedule.  Errors: those of the decode call, and
 * INVALID_ARGUMENT for a bad pipeline, slot or device. */
df11_status df11_pipeline_decode(df11_pipeline *p, uint32_t slot, const df11_device_block *blk,
                                 uint16_t *out_bf16, uint64_t out_capacity, uint32_t *d_error,
                                 uint32_t max_ctas, void *workspace, void *decode_stream);

/* Verify stage (optional, "after every copy").  Enqueues on `stream`,
 * after the slot's last upload, df11_verify_device_async(blk, d_expected,
 * n_crc, d_error, d_first_bad); enqueue it on the decode stream before
 * df11_pipeline_decode so the decode follows it.  Errors: those of the
 * verify call, INVALID_ARGUMENT for a bad pipeline, slot or device. */
df11_status df11_pipeline_verify(df11_pipeline *p, uint32_t slot, const df11_device_block *blk,
                                 const uint32_t *d_expected, uint64_t n_crc, uint32_t *d_error,
                                 uint64_t *d_first_bad, void *stream);

/* Consume stage.  acquire: consumer_stream waits for the slot's last
 * decode.  release: records that the consumer is done with the slot's
 * output (enqueue it after the last kernel that reads it). */
df11_status df11_pipeline_acquire(df11_pipeline *p, uint32_t slot, void *consumer_stream);
df11_status df11_pipeline_release(df11_pipeline *p, uint32_t slot, void *consumer_stream);

/* ---- One block as a flat byte buffer (files) -------------------------------
 * The pages keep DF11 models in safetensors files and tell users to checksum
 * artifacts on download and after every copy ("DFloat11: lossless BFloat16
 * compression", "How to run it in production", "Failure modes").  The
 * library's own container for one block: a 128-byte header (magic
 * "DF11BLK\0", version 2, the block header, the six array lengths, the
 * checksum count, the CRC-32C of those header bytes), the six arrays in
 * the order exp_stream, gaps, counts, chunk_pos, signmant, lut, each at a
 * 16-byte aligned offset, then the checksum list of df11_checksum.
 * Little-endian.
 */

/* Host.  Bytes df11_serialize writes for blk (0 for NULL or absurd sizes). */
uint64_t df11_serialized_bytes(const df11_host_block *blk);

/* Host.  Writes blk into buf[0 .. df11_serialized_bytes(blk)).  Errors:
 * INVALID_ARGUMENT (null pointers), BUFFER_TOO_SMALL. */
df11_status df11_serialize(const df11_host_block *blk, void *buf, uint64_t buf_bytes);

/* Host.  Reads a buffer written by df11_serialize (buf_bytes must be its
 * exact length): checks the magic, version and header CRC, the sizes,
 * that all padding is zero, every segment checksum and the block's
 * structure (df11_validate), so that every byte is checked, then
 * fills *blk with pointers INTO buf (no copy; buf must outlive blk).
 * *first_bad (may be NULL) receives the index of the first segment whose
 * checksum differs, else UINT64_MAX.  Errors: INVALID_ARGUMENT (null
 * pointers), CORRUPT (anything that does not check out; *blk untouched). */
df11_status df11_deserialize(const void *buf, uint64_t buf_bytes, df11_host_block *blk,
                             uint64_t *first_bad);

const char *df11_status_string(df11_status s);

#ifdef __cplusplus
}
#endif

#endif /* DF11_H */
