/*
 * df11_oracle.c -- TEST INFRASTRUCTURE ONLY (see df11_oracle.h).
 *
 * Plain, slow and single-threaded on purpose: every step is written the
 * obvious way so it can be checked against the page by eye.  Only the tests,
 * the smoke check and the benchmark's CPU-baseline leg may call it.
 *
 * [DF11-page] = "DFloat11: lossless BFloat16 compression" (ai-infrastructure.net).
 */
#include "df11_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ fields */

/* [DF11-page] "What it is": BF16 = 1 sign | 8 exponent | 7 mantissa bits;
 * split_bf16 keeps the exponent byte and packs (sign << 7) | mantissa. */
void orc_split(const uint16_t *w, uint64_t n, uint8_t *exp_out, uint8_t *sm_out)
{
    for (uint64_t i = 0; i < n; ++i) {
        uint16_t x = w[i];
        uint8_t sign = (uint8_t)((x >> 15) & 1u);
        uint8_t exponent = (uint8_t)((x >> 7) & 0xFFu);
        uint8_t mantissa = (uint8_t)(x & 0x7Fu);
        exp_out[i] = exponent;
        sm_out[i] = (uint8_t)((sign << 7) | mantissa);
    }
}

/* [DF11-page] join_bf16. */
void orc_join(const uint8_t *exp_in, const uint8_t *sm_in, uint64_t n, uint16_t *w_out)
{
    for (uint64_t i = 0; i < n; ++i) {
        uint16_t sign = (uint16_t)(sm_in[i] >> 7);
        uint16_t mantissa = (uint16_t)(sm_in[i] & 0x7Fu);
        uint16_t exponent = (uint16_t)exp_in[i];
        w_out[i] = (uint16_t)((sign << 15) | (exponent << 7) | mantissa);
    }
}

/* ------------------------------------------------------------- statistics */

void orc_histogram_add(const uint8_t *exp, uint64_t n, uint64_t counts[256])
{
    for (uint64_t i = 0; i < n; ++i)
        counts[exp[i]] += 1;
}

/* [DF11-page] entropy_bits: H = -sum p log2 p over symbols that occur. */
double orc_entropy(const uint64_t counts[256])
{
    double total = 0.0;
    for (int s = 0; s < 256; ++s)
        total += (double)counts[s];
    if (total == 0.0)
        return 0.0;
    double h = 0.0;
    for (int s = 0; s < 256; ++s) {
        if (counts[s] == 0)
            continue;
        double p = (double)counts[s] / total;
        h -= p * log2(p);
    }
    return h;
}

uint64_t orc_total_bits(const uint64_t counts[256], const uint8_t len[256])
{
    uint64_t t = 0;
    for (int s = 0; s < 256; ++s)
        t += counts[s] * (uint64_t)len[s];
    return t;
}

/* --------------------------------------------------------- code lengths */

/* [DF11-page] huffman_lengths.  The queue is small (<= 511 nodes), so the two
 * smallest entries are found by a linear scan instead of a heap; the order
 * (count, insertion index) is total, so the merges are the page's merges. */
int orc_huffman_lengths(const uint64_t counts[256], uint8_t len[256])
{
    uint64_t node_count[512];
    int node_index[512];
    int node_alive[512];
    int group[256];      /* node that currently holds symbol s, or -1 */
    int depth[256];
    int n_nodes = 0;

    memset(len, 0, 256);
    for (int s = 0; s < 256; ++s) {
        group[s] = -1;
        depth[s] = 0;
        if (counts[s] > 0) {
            node_count[n_nodes] = counts[s];
            node_index[n_nodes] = n_nodes;     /* insertion order = symbol order */
            node_alive[n_nodes] = 1;
            group[s] = n_nodes;
            n_nodes += 1;
        }
    }
    int live = n_nodes;
    if (live == 0)
        return -1;
    if (live == 1) {
        for (int s = 0; s < 256; ++s)
            if (counts[s] > 0)
                len[s] = 1;
        return 1;
    }
    int next_index = n_nodes;
    int queue_size = n_nodes;
    while (queue_size > 1) {
        int pick[2];
        for (int k = 0; k < 2; ++k) {
            int best = -1;
            for (int i = 0; i < n_nodes; ++i) {
                if (!node_alive[i])
                    continue;
                if (best < 0 || node_count[i] < node_count[best] ||
                    (node_count[i] == node_count[best] && node_index[i] < node_index[best]))
                    best = i;
            }
            pick[k] = best;
            node_alive[best] = 0;
        }
        int z = n_nodes++;
        node_count[z] = node_count[pick[0]] + node_count[pick[1]];
        node_index[z] = next_index++;
        node_alive[z] = 1;
        for (int s = 0; s < 256; ++s) {
            if (group[s] == pick[0] || group[s] == pick[1]) {
                depth[s] += 1;
                group[s] = z;
            }
        }
        queue_size -= 1;
    }
    for (int s = 0; s < 256; ++s)
        len[s] = (uint8_t)depth[s];
    return live;
}

/* One package-merge item: its weight and how many times each symbol occurs
 * in it (a package of packages can hold a symbol more than once). */
typedef struct {
    uint64_t weight;
    uint8_t mult[256];
} pm_item;

/* Package-merge (Larmore & Hirschberg 1990).  The list for the deepest level
 * is the leaves sorted by weight.  Each step pairs adjacent items of the list
 * into packages and merges the packages with the leaves, by weight.  After
 * cap-1 steps the first 2n-2 items of the list are selected; a symbol's code
 * length is the number of times it occurs among them. */
int orc_package_merge_lengths(const uint64_t counts[256], int cap, uint8_t len[256])
{
    int n = 0;
    int order[256];
    memset(len, 0, 256);
    for (int s = 0; s < 256; ++s)
        if (counts[s] > 0)
            order[n++] = s;
    if (n < 2 || cap < 1 || cap > 32)
        return -1;
    if (cap < 9 && n > (1 << cap))
        return -1;
    /* leaves by (count, symbol), insertion sort */
    for (int i = 1; i < n; ++i) {
        int s = order[i];
        int j = i - 1;
        while (j >= 0 && (counts[order[j]] > counts[s] ||
                          (counts[order[j]] == counts[s] && order[j] > s))) {
            order[j + 1] = order[j];
            --j;
        }
        order[j + 1] = s;
    }
    int max_items = 2 * n;
    pm_item *leaves = (pm_item *)calloc((size_t)n, sizeof(pm_item));
    pm_item *list = (pm_item *)calloc((size_t)max_items, sizeof(pm_item));
    pm_item *packages = (pm_item *)calloc((size_t)max_items, sizeof(pm_item));
    pm_item *merged = (pm_item *)calloc((size_t)max_items, sizeof(pm_item));
    if (!leaves || !list || !packages || !merged) {
        free(leaves); free(list); free(packages); free(merged);
        return -1;
    }
    for (int i = 0; i < n; ++i) {
        leaves[i].weight = counts[order[i]];
        leaves[i].mult[order[i]] = 1;
        list[i] = leaves[i];
    }
    int list_len = n;
    for (int step = 1; step < cap; ++step) {
        int n_pk = list_len / 2;
        for (int i = 0; i < n_pk; ++i) {
            pm_item *a = &list[2 * i];
            pm_item *b = &list[2 * i + 1];
            packages[i].weight = a->weight + b->weight;
            for (int s = 0; s < 256; ++s)
                packages[i].mult[s] = (uint8_t)(a->mult[s] + b->mult[s]);
        }
        /* merge leaves and packages by weight; a leaf goes first on a tie */
        int i = 0, j = 0, m = 0;
        while (i < n || j < n_pk) {
            if (j >= n_pk || (i < n && leaves[i].weight <= packages[j].weight))
                merged[m++] = leaves[i++];
            else
                merged[m++] = packages[j++];
        }
        memcpy(list, merged, (size_t)m * sizeof(pm_item));
        list_len = m;
    }
    int take = 2 * n - 2;
    int depth[256];
    memset(depth, 0, sizeof(depth));
    for (int i = 0; i < take && i < list_len; ++i)
        for (int s = 0; s < 256; ++s)
            depth[s] += list[i].mult[s];
    for (int s = 0; s < 256; ++s)
        len[s] = (uint8_t)depth[s];
    free(leaves); free(list); free(packages); free(merged);
    return n;
}

int orc_code_lengths(const uint64_t counts[256], int cap, uint8_t len[256])
{
    int live = orc_huffman_lengths(counts, len);
    if (live <= 1)
        return live;
    int max_len = 0;
    for (int s = 0; s < 256; ++s)
        if (len[s] > max_len)
            max_len = len[s];
    if (max_len <= cap)
        return live;
    return orc_package_merge_lengths(counts, cap, len);
}

/* ---------------------------------------------------------------- codes */

/* [DF11-page] canonical_codes. */
int orc_canonical_codes(const uint8_t len[256], uint32_t code[256])
{
    int order[256];
    int n = 0;
    memset(code, 0, 256 * sizeof(uint32_t));
    for (int s = 0; s < 256; ++s)
        if (len[s] > 0)
            order[n++] = s;
    /* ascending (length, symbol); symbols are already ascending, so a stable
     * insertion sort on length is enough */
    for (int i = 1; i < n; ++i) {
        int s = order[i];
        int j = i - 1;
        while (j >= 0 && len[order[j]] > len[s]) {
            order[j + 1] = order[j];
            --j;
        }
        order[j + 1] = s;
    }
    uint64_t c = 0;
    int prev_len = 0;
    for (int i = 0; i < n; ++i) {
        int s = order[i];
        if (len[s] > 32)
            return -1;
        c <<= (len[s] - prev_len);
        if (c >= ((uint64_t)1 << len[s]))
            return -1; /* lengths violate Kraft's inequality */
        code[s] = (uint32_t)c;
        c += 1;
        prev_len = len[s];
    }
    return 0;
}

/* ------------------------------------------------------------ bitstream */

/* [DF11-page] encode, one bit at a time. */
int orc_encode(const uint8_t *exp, uint64_t n, const uint8_t len[256],
               const uint32_t code[256], uint8_t *stream, uint64_t stream_bytes,
               uint64_t *total_bits)
{
    uint64_t bit = 0;
    for (uint64_t k = 0; k < n; ++k) {
        int l = len[exp[k]];
        uint32_t c = code[exp[k]];
        if (l == 0)
            return -1; /* symbol has no code */
        for (int i = 0; i < l; ++i) {
            uint32_t b = (c >> (l - 1 - i)) & 1u;
            uint64_t byte = bit >> 3;
            if (byte >= stream_bytes)
                return -1;
            if (b)
                stream[byte] |= (uint8_t)(0x80u >> (bit & 7));
            bit += 1;
        }
    }
    *total_bits = bit;
    return 0;
}

/* Per-length tables of the canonical code: how many codes have length l,
 * the first (smallest) code of length l, and the symbols by (length, symbol). */
typedef struct {
    int max_len;
    uint32_t count[33];
    uint32_t first[33];
    uint32_t offset[33];
    int sorted[256];
} canon_table;

static int canon_build(const uint8_t len[256], canon_table *t)
{
    memset(t, 0, sizeof(*t));
    for (int s = 0; s < 256; ++s) {
        if (len[s] > 32)
            return -1;
        if (len[s] > 0) {
            t->count[len[s]] += 1;
            if (len[s] > t->max_len)
                t->max_len = len[s];
        }
    }
    if (t->max_len == 0)
        return -1;
    /* the first code of each length, by the same rule as the assignment:
     * after the last code of length l comes (that code + 1) << 1 */
    uint64_t first = 0;
    uint32_t off = 0;
    for (int l = 1; l <= 32; ++l) {
        t->first[l] = (uint32_t)first;
        t->offset[l] = off;
        off += t->count[l];
        first = (first + t->count[l]) << 1;
    }
    uint32_t fill[33];
    memcpy(fill, t->offset, sizeof(fill));
    for (int l = 1; l <= 32; ++l)
        for (int s = 0; s < 256; ++s)
            if (len[s] == l)
                t->sorted[fill[l]++] = s;
    return 0;
}

static int stream_bit(const uint8_t *stream, uint64_t stream_bytes, uint64_t i, int *b)
{
    uint64_t byte = i >> 3;
    if (byte >= stream_bytes)
        return -1;
    *b = (stream[byte] >> (7 - (i & 7))) & 1;
    return 0;
}

int orc_decode(const uint8_t *stream, uint64_t stream_bytes, uint64_t start_bit,
               uint64_t n, const uint8_t len[256], uint8_t *exp_out, uint64_t *end_bit)
{
    canon_table t;
    if (canon_build(len, &t) != 0)
        return -1;
    uint64_t pos = start_bit;
    for (uint64_t k = 0; k < n; ++k) {
        uint32_t c = 0;
        int found = 0;
        for (int l = 1; l <= t.max_len; ++l) {
            int b;
            if (stream_bit(stream, stream_bytes, pos, &b) != 0)
                return -1;
            pos += 1;
            c = (c << 1) | (uint32_t)b;
            if (t.count[l] > 0 && c - t.first[l] < t.count[l]) {
                exp_out[k] = (uint8_t)t.sorted[t.offset[l] + (c - t.first[l])];
                found = 1;
                break;
            }
        }
        if (!found)
            return -1;
    }
    if (end_bit)
        *end_bit = pos;
    return 0;
}

int orc_first_code(uint32_t v16, const uint8_t len[256], int *sym, int *clen)
{
    canon_table t;
    if (canon_build(len, &t) != 0)
        return -1;
    uint32_t c = 0;
    for (int l = 1; l <= t.max_len && l <= 16; ++l) {
        c = (c << 1) | ((v16 >> (16 - l)) & 1u);
        if (t.count[l] > 0 && c - t.first[l] < t.count[l]) {
            *sym = t.sorted[t.offset[l] + (c - t.first[l])];
            *clen = l;
            return 0;
        }
    }
    return -1;
}

int orc_first_code_table(const uint8_t len[256], int16_t *sym_out, uint8_t *len_out)
{
    for (uint32_t v = 0; v < 65536u; ++v) {
        int sym = -1, clen = 0;
        if (orc_first_code(v, len, &sym, &clen) != 0) {
            sym = -1;
            clen = 0;
        }
        sym_out[v] = (int16_t)sym;
        len_out[v] = (uint8_t)clen;
    }
    return 0;
}

/* ------------------------------------------------------------- metadata */

int orc_metadata(const uint8_t *exp, uint64_t n, const uint8_t len[256],
                 uint32_t threads_per_chunk, uint32_t bytes_per_thread,
                 uint64_t n_chunks, uint8_t *gap, uint8_t *count, uint32_t *pos)
{
    if (n >= ((uint64_t)1 << 32) || threads_per_chunk == 0 || bytes_per_thread == 0)
        return -1;
    uint64_t slice_bits = 8ull * bytes_per_thread;
    uint64_t n_threads = n_chunks * threads_per_chunk;
    uint64_t total = 0;
    for (uint64_t k = 0; k < n; ++k)
        total += len[exp[k]];

    /* gaps: s walks the code starts s_0, s_1, ..., s_n = total */
    uint64_t k = 0, s = 0;
    for (uint64_t g = 0; g < n_threads; ++g) {
        uint64_t base = slice_bits * g;
        if (base >= total) {
            gap[g] = 0;
            continue;
        }
        while (k < n && s < base) {
            s += len[exp[k]];
            k += 1;
        }
        uint64_t d = s - base;
        if (d > 255)
            return -1;
        gap[g] = (uint8_t)d;
    }

    /* per-thread counts: every code start s_k < total lands in slice s_k / B */
    for (uint64_t g = 0; g < n_threads; ++g)
        count[g] = 0;
    s = 0;
    for (k = 0; k < n; ++k) {
        uint64_t g = s / slice_bits;
        if (g >= n_threads || count[g] == 255)
            return -1;
        count[g] += 1;
        s += len[exp[k]];
    }

    /* chunk output positions */
    k = 0;
    s = 0;
    for (uint64_t c = 0; c <= n_chunks; ++c) {
        uint64_t limit = c * threads_per_chunk * slice_bits;
        while (k < n && s < limit) {
            s += len[exp[k]];
            k += 1;
        }
        pos[c] = (uint32_t)k;
    }
    return 0;
}


/* ---- checksum ----------------------------------------------------------- */

uint32_t orc_crc32c(const uint8_t *data, uint64_t n)
{
    const uint32_t poly = 0x82F63B78u;   /* the generator, bit-reversed */
    uint32_t reg = 0xFFFFFFFFu;
    for (uint64_t i = 0; i < n; ++i) {
        reg ^= data[i];
        for (int b = 0; b < 8; ++b) {
            if (reg & 1u)
                reg = (reg >> 1) ^ poly;
            else
                reg >>= 1;
        }
    }
    return ~reg;
}

uint64_t orc_segment_crcs(const uint8_t *data, uint64_t n, uint64_t seg, uint32_t *out)
{
    uint64_t k = 0;
    for (uint64_t off = 0; off < n; off += seg, ++k)
        out[k] = orc_crc32c(data + off, n - off < seg ? n - off : seg);
    return k;
}

/* ----------------------------------------------------------- chunk sums */

static uint32_t orc_mix(uint32_t v, uint32_t tag)
{
    uint32_t x = v ^ (uint32_t)(tag * 0x9E3779B1u);
    uint32_t y = x * 0x85EBCA6Bu;
    return y ^ (y >> 16);
}

int orc_chunk_sums(const uint8_t *stream, const uint8_t *gaps, const uint8_t *counts, const uint32_t *pos,
                   const uint8_t *signmant, uint64_t signmant_bytes, const uint16_t *lut, uint32_t n_tables,
                   uint32_t bytes_per_thread, uint64_t n_chunks, uint32_t *out)
{
    if (bytes_per_thread == 0 || n_tables == 0)
        return -1;
    for (uint64_t c = 0; c < n_chunks; ++c)
        if (pos[c] > pos[c + 1] || pos[c + 1] > signmant_bytes)
            return -1;
    const uint64_t slice_bits = 8ull * bytes_per_thread;
    const uint64_t chunk_bytes = 32ull * bytes_per_thread;
    for (uint64_t c = 0; c < n_chunks; ++c) {
        uint32_t sum = 0;
        /* stream words, bit by bit */
        for (uint64_t k = 0; k < slice_bits; ++k) {
            uint32_t v = 0;
            for (uint32_t i = 0; i < 32; ++i) {
                uint64_t j = 32 * k + i;
                uint8_t byte = stream[chunk_bytes * c + j / 8];
                uint32_t bit = (byte >> (7 - j % 8)) & 1u;
                v |= bit << i;
            }
            sum += orc_mix(v, (uint32_t)k);
        }
        /* thread words */
        for (uint32_t t = 0; t < 32; ++t) {
            uint64_t g = 32 * c + t;
            uint32_t gap = (gaps[g / 2] >> (4 * (g % 2))) & 15u;
            sum += orc_mix(gap | ((uint32_t)counts[g] << 8), 0x10000u + t);
        }
        /* positions */
        uint64_t p0 = pos[c], p1 = pos[c + 1];
        sum += orc_mix((uint32_t)p0, 0x20000u);
        sum += orc_mix((uint32_t)p1, 0x20001u);
        /* sign|mantissa bytes */
        uint64_t b = p0 - p0 % 8;
        for (uint64_t e = p0; e < p1; ++e) {
            uint64_t q = e / 8;
            int whole = 8 * q >= p0 && 8 * q + 8 <= p1;
            if (!whole)
                sum += orc_mix(signmant[e], (uint32_t)(0x200000u + (e - b)));
        }
        for (uint64_t q = (p0 + 7) / 8; 8 * q + 8 <= p1; ++q) {
            const uint8_t *g8 = signmant + 8 * q;
            uint32_t v0 = g8[0] | ((uint32_t)g8[1] << 8) | ((uint32_t)g8[2] << 16) | ((uint32_t)g8[3] << 24);
            uint32_t v1 = g8[4] | ((uint32_t)g8[5] << 8) | ((uint32_t)g8[6] << 16) | ((uint32_t)g8[7] << 24);
            uint64_t r = q - b / 8;
            sum += orc_mix(v0, (uint32_t)(0x100000u + 2 * r));
            sum += orc_mix(v1, (uint32_t)(0x100000u + 2 * r + 1));
        }
        /* the tables, in chunk 0 */
        if (c == 0)
            for (uint64_t i = 0; i < 128ull * n_tables; ++i)
                sum += orc_mix(lut[2 * i] | ((uint32_t)lut[2 * i + 1] << 16), (uint32_t)(0x400000u + i));
        out[c] = sum;
    }
    return 0;
}
