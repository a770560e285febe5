/*
 * df11_oracle.h -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, single-threaded C restatement of the DFloat11 (DF11) codec:
 * split a BF16 word into exponent and sign|mantissa bytes, Huffman-code the
 * exponent with a canonical, length-limited code, write the bitstream, derive
 * the per-thread gap / per-chunk output-position metadata, and decode the
 * stream one bit at a time.  It exists to check the product library and its
 * GPU kernel; nothing in the product path may call it.  It shares no code,
 * header, table or constant with the library under huffman_decode_b200/.
 *
 * Sources (the web pages this method is described on):
 *   [DF11-page] "DFloat11: lossless BFloat16 compression" (ai-infrastructure.net),
 *               sections "What it is", "Architecture" and
 *               "How it works: the core algorithm" (executed numpy sketch and
 *               its printed output); "How to run it in production" and
 *               "Failure modes" (checksum every artifact).
 *
 * Every function below names the passage it follows.  All functions return 0
 * on success and a negative value on a detected error.
 */
#ifndef DF11_ORACLE_H
#define DF11_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* [DF11-page] "What it is" / split_bf16: the exponent is bits 14..7 of the
 * BF16 word; the raw byte keeps the sign in bit 7 and the 7 mantissa bits. */
void orc_split(const uint16_t *w, uint64_t n, uint8_t *exp_out, uint8_t *sm_out);

/* [DF11-page] join_bf16: the inverse of orc_split. */
void orc_join(const uint8_t *exp_in, const uint8_t *sm_in, uint64_t n, uint16_t *w_out);

/* Adds the 256-bin exponent histogram of exp[0..n) into counts (not cleared). */
void orc_histogram_add(const uint8_t *exp, uint64_t n, uint64_t counts[256]);

/* Shannon entropy in bits of the distribution given by counts (fp64). */
double orc_entropy(const uint64_t counts[256]);

/* [DF11-page] huffman_lengths: plain Huffman with the page's tie rule --
 * a min-queue keyed by (count, insertion index); live symbols enter in
 * ascending symbol order, each merged node takes the next index; every merge
 * deepens every symbol under both children by one.  One live symbol gets
 * length 1.  len[s] = 0 for absent symbols.  Returns the number of live
 * symbols, or -1 if there are none. */
int orc_huffman_lengths(const uint64_t counts[256], uint8_t len[256]);

/* Optimal code lengths under a maximum length `cap` by package-merge
 * (Larmore & Hirschberg, "A fast algorithm for optimal length-limited Huffman
 * codes", J. ACM 37(3), 1990), written out with explicit per-item symbol
 * multiplicities.  Needs 2 <= live symbols <= 2^cap.  Returns the number of
 * live symbols or -1. */
int orc_package_merge_lengths(const uint64_t counts[256], int cap, uint8_t len[256]);

/* The code lengths DF11 uses under a length cap ([DF11-page] "Architecture",
 * hierarchical lookup tables: real exponent trees reach 24-32 bits and the
 * format must bound them): the page's Huffman lengths when their maximum is
 * within the cap, else package-merge.  Both are optimal. */
int orc_code_lengths(const uint64_t counts[256], int cap, uint8_t len[256]);

/* [DF11-page] canonical_codes: symbols in ascending (length, symbol) order;
 * the first gets code 0; each next code is the previous plus one, shifted
 * left by the growth in length.  code[s] is right-aligned in len[s] bits. */
int orc_canonical_codes(const uint8_t len[256], uint32_t code[256]);

/* Sum over symbols of count * length. */
uint64_t orc_total_bits(const uint64_t counts[256], const uint8_t len[256]);

/* [DF11-page] encode: codes concatenated in element order, most significant
 * bit first.  Stream bit i is bit (7 - i%8) of byte i/8.  The caller zeroes
 * `stream` (stream_bytes long).  Returns the bit count through *total_bits. */
int orc_encode(const uint8_t *exp, uint64_t n, const uint8_t len[256],
               const uint32_t code[256], uint8_t *stream, uint64_t stream_bytes,
               uint64_t *total_bits);

/* Bit-by-bit canonical decode (no lookup tables) of n symbols starting at
 * stream bit `start_bit`.  Reading past stream_bytes or meeting a bit pattern
 * that is no code returns -1.  *end_bit receives the bit after the last code. */
int orc_decode(const uint8_t *stream, uint64_t stream_bytes, uint64_t start_bit,
               uint64_t n, const uint8_t len[256], uint8_t *exp_out, uint64_t *end_bit);

/* First code in the 16-bit MSB-first window v: the symbol and its length, or
 * -1 when no code is a prefix of v (only possible with a single live symbol). */
int orc_first_code(uint32_t v16, const uint8_t len[256], int *sym, int *clen);

/* orc_first_code for every 16-bit window: sym_out/len_out[v] (len 0 = none). */
int orc_first_code_table(const uint8_t len[256], int16_t *sym_out, uint8_t *len_out);

/* [DF11-page] "Architecture", two-phase kernel: each thread owns a fixed
 * slice of bytes_per_thread bytes of the stream; Gaps holds the bit offset of
 * the first code that starts inside the slice; one output position is kept
 * per group of threads_per_chunk threads.  Code k starts at
 * s_k = sum_{j<k} len(exp_j); s_n = total_bits is counted as a start so a
 * slice whose codes all began earlier still points at the end.
 *   gap[g]   = min{ s_k >= B*g } - B*g for slices with B*g < total_bits, else 0
 *   count[g] = #{ k < n : B*g <= s_k < B*(g+1) }   (codes starting in slice g)
 *   pos[c]   = #{ k < n : s_k < c*T*B },  c = 0..n_chunks  (B = 8*bytes_per_thread)
 * gap and count are unpacked (one byte per thread, n_threads = n_chunks*T
 * entries).  count is what the page's first decode phase computes for each
 * thread ("Architecture", the two-phase kernel); the library's format stores
 * it. */
int orc_metadata(const uint8_t *exp, uint64_t n, const uint8_t len[256],
                 uint32_t threads_per_chunk, uint32_t bytes_per_thread,
                 uint64_t n_chunks, uint8_t *gap, uint8_t *count, uint32_t *pos);

/* [DF11-page] "How to run it in production": checksum every artifact.  The
 * checksum is CRC-32C (Castagnoli), written here bit by bit from its
 * definition: the generator x^32 + x^28 + x^27 + x^26 + x^25 + x^23 + x^22 +
 * x^20 + x^19 + x^18 + x^14 + x^13 + x^11 + x^10 + x^9 + x^8 + x^6 + 1,
 * message bits taken least-significant first in every byte (a reflected
 * register, so the generator appears as 0x82F63B78), register preset to all
 * ones, result complemented.  No tables. */
uint32_t orc_crc32c(const uint8_t *data, uint64_t n);

/* The checksum list of one array: the CRC-32C of every `seg`-byte segment
 * of data[0 .. n) in order (the last one may be shorter); returns the
 * number of values written to out (ceil(n / seg)). */
uint64_t orc_segment_crcs(const uint8_t *data, uint64_t n, uint64_t seg, uint32_t *out);

/* Per-chunk sum: the integrity check the library's decoder can run as it
 * decodes (the pages ask only to checksum artifacts, "How to run it in
 * production"; this is the library's own check, computed by the decode
 * kernel from the bytes it already holds).  For chunk c (threads 32c..32c+31,
 * B = 8 * bytes_per_thread bits per slice), the sum mod 2^32 of mix(v, tag)
 * over these items:
 *   - stream words k = 0 .. B - 1 (the chunk's 32 B stream bits, words of 32):
 *     bit i of v is chunk stream bit 32k + i (MSB-first within bytes); tag k;
 *   - threads t = 0..31: v = gap | count << 8 of thread 32c + t;
 *     tag 0x10000 + t;
 *   - v = chunk_pos[c], tag 0x20000; v = chunk_pos[c + 1], tag 0x20001;
 *   - sign|mantissa bytes of elements [p0, p1) = [chunk_pos[c],
 *     chunk_pos[c + 1]), with b = p0 rounded down to a multiple of 8: each
 *     8-element group [8q, 8q + 8) inside [p0, p1) gives two little-endian
 *     words of its bytes, tags 0x100000 + 2r and 0x100000 + 2r + 1 (r = q -
 *     b / 8); every other element e gives its byte alone, tag 0x200000 + e - b;
 *   - chunk 0 only: the tables as little-endian words (entries 2i and 2i + 1,
 *     i < 128 n_tables), tag 0x400000 + i.
 * mix(v, tag) = y ^ (y >> 16), y = (v ^ tag * 0x9E3779B1) * 0x85EBCA6B (mod
 * 2^32): for each tag a bijection of v, so any change of one item changes
 * the sum.  gaps are packed (two per byte), counts one byte per thread.
 * Returns 0, or -1 for bad arguments (positions that decrease or pass
 * signmant_bytes among them). */
int orc_chunk_sums(const uint8_t *stream, const uint8_t *gaps, const uint8_t *counts, const uint32_t *pos,
                   const uint8_t *signmant, uint64_t signmant_bytes, const uint16_t *lut, uint32_t n_tables,
                   uint32_t bytes_per_thread, uint64_t n_chunks, uint32_t *out);

#ifdef __cplusplus
}
#endif

#endif /* DF11_ORACLE_H */
