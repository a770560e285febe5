// df11_host.cpp -- host half of the DF11 codec: codebook builder, block
// compressor and structural validator behind the C ABI in include/df11.h.
//
// Method: "DFloat11: lossless BFloat16 compression" (ai-infrastructure.net):
//   "What it is"           -- exponent byte Huffman coded, sign|mantissa raw;
//   "Architecture"         -- hierarchical 8-bit lookup tables, per-thread
//                             Gaps, per-block output positions;
//   "How it works: ..."    -- canonical code assignment, MSB-first stream.
// Code lengths here come from an exact dynamic program over the levels of a
// full binary tree (not the page's heap): same optimum, bounded depth.
#include "df11.h"

#include <algorithm>
#include <atomic>
#include <cstring>
#include <thread>
#include <vector>

namespace {


// ------------------------------------------------------------ threading

unsigned worker_count(uint64_t work_items)
{
    unsigned hw = std::thread::hardware_concurrency();
    if (hw == 0)
        hw = 1;
    hw = std::min(hw, 32u);
    uint64_t by_size = work_items / (1u << 20) + 1;  // >= 1M items per worker
    return (unsigned)std::min<uint64_t>(hw, by_size);
}

template <class F>
void parallel_for(unsigned n, F &&fn)
{
    if (n <= 1) {
        if (n == 1)
            fn(0u);
        return;
    }
    std::vector<std::thread> th;
    th.reserve(n);
    for (unsigned i = 0; i < n; ++i)
        th.emplace_back([&fn, i] { fn(i); });
    for (auto &t : th)
        t.join();
}

// A block's elements as one virtual sequence across its matrices.
struct ElementView {
    const uint16_t *const *mats;
    const uint64_t *numel;
    uint32_t n_mats;
    std::vector<uint64_t> start;  // first global index of each matrix
    uint64_t total = 0;

    ElementView(const uint16_t *const *m, const uint64_t *ne, uint32_t nm)
        : mats(m), numel(ne), n_mats(nm), start(nm + 1, 0)
    {
        for (uint32_t i = 0; i < nm; ++i)
            start[i + 1] = start[i] + ne[i];
        total = start[nm];
    }

    // Calls fn(global_index, value) for elements [lo, hi) in order.
    template <class F>
    void for_range(uint64_t lo, uint64_t hi, F &&fn) const
    {
        if (lo >= hi)
            return;
        uint32_t m = (uint32_t)(std::upper_bound(start.begin(), start.end(), lo) - start.begin()) - 1;
        uint64_t k = lo;
        while (k < hi && m < n_mats) {
            uint64_t mend = std::min(hi, start[m + 1]);
            const uint16_t *p = mats[m] + (k - start[m]);
            for (; k < mend; ++k, ++p)
                fn(k, *p);
            ++m;
        }
    }
};

bool check_mats(const uint16_t *const *mats, const uint64_t *numel, uint32_t n_mats)
{
    if (!mats || !numel || n_mats == 0)
        return false;
    for (uint32_t i = 0; i < n_mats; ++i)
        if (numel[i] > 0 && !mats[i])
            return false;
    return true;
}

void histogram(const ElementView &v, uint64_t out[256])
{
    unsigned nw = worker_count(v.total);
    std::vector<uint64_t> part((size_t)nw * 256, 0);
    parallel_for(nw, [&](unsigned w) {
        uint64_t lo = v.total * w / nw, hi = v.total * (w + 1) / nw;
        uint64_t *h = part.data() + (size_t)w * 256;
        v.for_range(lo, hi, [h](uint64_t, uint16_t x) { h[(x >> 7) & 0xFF] += 1; });
    });
    for (int s = 0; s < 256; ++s) {
        uint64_t t = 0;
        for (unsigned w = 0; w < nw; ++w)
            t += part[(size_t)w * 256 + s];
        out[s] = t;
    }
}

// ------------------------------------------------------- code lengths
//
// Optimal code lengths with every length <= cap.  An optimal prefix code
// with n >= 2 symbols is a full binary tree and heavier symbols sit no
// deeper than lighter ones, so with the weights sorted heaviest first the
// tree is described level by level: after level d, `c` symbols are leaves at
// depth <= d and `a` nodes of depth d are internal.  Level d+1 offers 2a
// nodes, m of which become the next m leaves.  The cost sum_i w_i*depth_i
// equals the sum over levels of the weight still unplaced when that level is
// entered, so each step adds suffix_weight[c].  The table is exact.
bool optimal_lengths(const uint64_t hist[256], uint32_t cap, uint8_t len[256])
{
    std::memset(len, 0, 256);
    std::vector<int> sym;
    for (int s = 0; s < 256; ++s)
        if (hist[s] > 0)
            sym.push_back(s);
    const int n = (int)sym.size();
    if (n == 0)
        return false;
    if (n == 1) {
        len[sym[0]] = 1;
        return true;
    }
    if (cap < 32 && (uint64_t)n > (1ull << cap))
        return false;
    std::stable_sort(sym.begin(), sym.end(), [&](int a, int b) { return hist[a] > hist[b]; });
    std::vector<uint64_t> suffix(n + 1, 0);
    for (int i = n - 1; i >= 0; --i)
        suffix[i] = suffix[i + 1] + hist[sym[i]];

    const int A = n / 2 + 2;  // internal nodes at one level never exceed n/2
    const uint64_t INF = ~0ull;
    auto idx = [A](int c, int a) { return (size_t)c * A + a; };
    std::vector<uint64_t> cur((size_t)(n + 1) * A, INF), nxt((size_t)(n + 1) * A, INF);
    // choice[d][c][a] = leaves placed at level d to reach state (c, a)
    std::vector<uint16_t> choice((size_t)(cap + 1) * (n + 1) * A, 0xFFFF);
    cur[idx(0, 1)] = 0;  // level 0: the root is internal
    for (uint32_t d = 0; d < cap; ++d) {
        std::fill(nxt.begin(), nxt.end(), INF);
        const uint32_t levels_left = cap - d - 1;  // levels below d+1
        for (int c = 0; c <= n; ++c) {
            for (int a = 0; a < A; ++a) {
                uint64_t f = cur[idx(c, a)];
                if (f == INF)
                    continue;
                uint64_t cost = f + suffix[c];
                int nodes = 2 * a;
                int mmax = std::min(nodes, n - c);
                for (int m = 0; m <= mmax; ++m) {
                    int c2 = c + m, a2 = nodes - m;
                    int rest = n - c2;
                    if (a2 == 0 ? rest != 0 : (rest < 2 * a2))
                        continue;
                    if (a2 >= A)
                        continue;
                    if (a2 > 0 && levels_left < 63 &&
                        (uint64_t)a2 << levels_left < (uint64_t)rest)
                        continue;
                    size_t j = idx(c2, a2);
                    if (cost < nxt[j]) {
                        nxt[j] = cost;
                        choice[(size_t)(d + 1) * (n + 1) * A + j] = (uint16_t)m;
                    }
                }
            }
        }
        std::swap(cur, nxt);
    }
    if (cur[idx(n, 0)] == INF)
        return false;
    // walk back from (n, 0) at level cap
    int c = n, a = 0;
    for (int d = (int)cap; d >= 1; --d) {
        uint16_t m = choice[(size_t)d * (n + 1) * A + idx(c, a)];
        if (m == 0xFFFF)
            return false;
        for (int i = c - m; i < c; ++i)
            len[sym[i]] = (uint8_t)d;
        int prev_c = c - m;
        int prev_a = (a + m) / 2;
        c = prev_c;
        a = prev_a;
    }
    return c == 0 && a == 1;
}

// Canonical codes: symbols in ascending (length, symbol) order take
// consecutive values; moving to a longer length appends zero bits.
void canonical_codes(const uint8_t len[256], uint32_t code[256])
{
    uint32_t count[DF11_MAX_CODE_LEN + 2] = {0};
    for (int s = 0; s < 256; ++s)
        if (len[s])
            count[len[s]] += 1;
    uint32_t next[DF11_MAX_CODE_LEN + 2] = {0};
    uint32_t c = 0;
    for (uint32_t l = 1; l <= DF11_MAX_CODE_LEN; ++l) {
        c = (c + count[l - 1]) << 1;
        next[l] = c;
    }
    // count[0] is 0, so next[1] = 0
    for (int s = 0; s < 256; ++s)
        code[s] = len[s] ? next[len[s]]++ : 0;
}

constexpr uint16_t kLutPointer = 0x8000;
constexpr uint16_t kLutNoCode = 0x4000 | (1u << 8);

// Two-level 256-entry tables: codes of <= 8 bits fill their range of the
// root; longer codes share one sub-table per distinct first byte.
uint32_t build_lut(const uint8_t len[256], const uint32_t code[256], uint16_t *lut)
{
    std::memset(lut, 0, sizeof(uint16_t) * 256 * 256);
    for (int i = 0; i < 256; ++i)
        lut[i] = kLutNoCode;
    // sub-tables are numbered in ascending order of their first byte
    int table_of_prefix[256];
    std::fill(table_of_prefix, table_of_prefix + 256, -1);
    bool long_prefix[256] = {false};
    for (int s = 0; s < 256; ++s)
        if (len[s] > 8)
            long_prefix[code[s] >> (len[s] - 8)] = true;
    uint32_t n_tables = 1;
    for (int pfx = 0; pfx < 256; ++pfx)
        if (long_prefix[pfx]) {
            table_of_prefix[pfx] = (int)n_tables;
            lut[pfx] = (uint16_t)(kLutPointer | n_tables);
            ++n_tables;
        }
    for (int s = 0; s < 256; ++s) {
        uint32_t l = len[s];
        if (l == 0)
            continue;
        uint16_t leaf = (uint16_t)((l << 8) | (uint32_t)s);
        if (l <= 8) {
            uint32_t base = code[s] << (8 - l);
            for (uint32_t i = 0; i < (1u << (8 - l)); ++i)
                lut[base + i] = leaf;
        } else {
            int t = table_of_prefix[code[s] >> (l - 8)];
            uint32_t suffix = code[s] & ((1u << (l - 8)) - 1);
            uint32_t base = suffix << (16 - l);
            for (uint32_t i = 0; i < (1u << (16 - l)); ++i)
                lut[(uint32_t)t * 256 + base + i] = leaf;
        }
    }
    return n_tables;
}

bool layout_ok(const df11_layout *ly)
{
    if (!ly)
        return false;
    return ly->threads_per_chunk == DF11_THREADS_PER_CHUNK &&
           (ly->bytes_per_thread == 8 || ly->bytes_per_thread == 16);
}

df11_sizes sizes_for(uint64_t total_bits, uint64_t n_elements, uint32_t n_tables,
                     const df11_layout *ly)
{
    df11_sizes z;
    uint64_t chunk_bits = (uint64_t)ly->threads_per_chunk * ly->bytes_per_thread * 8;
    z.n_chunks = (total_bits + chunk_bits - 1) / chunk_bits;
    z.n_threads = z.n_chunks * ly->threads_per_chunk;
    z.exp_stream_bytes = z.n_threads * ly->bytes_per_thread + DF11_STREAM_PAD;
    z.gaps_bytes = z.n_threads / 2;
    z.counts_bytes = z.n_threads;
    z.chunk_pos_count = z.n_chunks + 1;
    z.signmant_bytes = (n_elements + 15) / 16 * 16;
    z.lut_entries = (uint64_t)n_tables * 256;
    return z;
}

}  // namespace

// ================================================================== C ABI

extern "C" {

const char *df11_status_string(df11_status s)
{
    switch (s) {
    case DF11_OK: return "ok";
    case DF11_ERR_INVALID_ARGUMENT: return "invalid argument";
    case DF11_ERR_BUFFER_TOO_SMALL: return "buffer too small";
    case DF11_ERR_OVERFLOW: return "element count overflow (>= 2^32)";
    case DF11_ERR_CORRUPT: return "corrupt artifact";
    case DF11_ERR_CUDA: return "CUDA error";
    case DF11_ERR_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

df11_status df11_build_codebook(const uint16_t *const *mats, const uint64_t *numel,
                                uint32_t n_mats, uint32_t max_code_len, df11_codebook *out)
{
    if (!out || !check_mats(mats, numel, n_mats))
        return DF11_ERR_INVALID_ARGUMENT;
    if (max_code_len < DF11_MIN_CODE_LEN_CAP || max_code_len > DF11_MAX_CODE_LEN)
        return DF11_ERR_INVALID_ARGUMENT;
    ElementView v(mats, numel, n_mats);
    if (v.total == 0)
        return DF11_ERR_INVALID_ARGUMENT;
    if (v.total >= (1ull << 32))
        return DF11_ERR_OVERFLOW;
    uint64_t h[256];
    histogram(v, h);
    return df11_build_codebook_from_histogram(h, max_code_len, out);
}

df11_status df11_build_codebook_from_histogram(const uint64_t hist[256], uint32_t max_code_len,
                                               df11_codebook *out)
{
    if (!hist || !out)
        return DF11_ERR_INVALID_ARGUMENT;
    if (max_code_len < DF11_MIN_CODE_LEN_CAP || max_code_len > DF11_MAX_CODE_LEN)
        return DF11_ERR_INVALID_ARGUMENT;
    uint64_t total = 0;
    for (int s = 0; s < 256; ++s)
        total += hist[s];
    if (total == 0)
        return DF11_ERR_INVALID_ARGUMENT;
    if (total >= (1ull << 32))
        return DF11_ERR_OVERFLOW;
    std::memset(out, 0, sizeof(*out));
    std::memcpy(out->histogram, hist, sizeof(out->histogram));
    if (!optimal_lengths(out->histogram, max_code_len, out->code_len))
        return DF11_ERR_INVALID_ARGUMENT;
    canonical_codes(out->code_len, out->code);
    out->n_tables = build_lut(out->code_len, out->code, out->lut);
    out->max_code_len = max_code_len;
    out->n_elements = total;
    for (int s = 0; s < 256; ++s) {
        if (out->code_len[s]) {
            out->n_symbols += 1;
            out->longest_code = std::max<uint32_t>(out->longest_code, out->code_len[s]);
            out->total_bits += out->histogram[s] * out->code_len[s];
        }
    }
    return DF11_OK;
}

extern "C" uint32_t df11_preferred_bytes_per_thread(const df11_codebook *cb, uint32_t sm_count)
{
    if (!cb || cb->total_bits == 0 || sm_count == 0)
        return 0;
    uint32_t shortest = DF11_MAX_CODE_LEN;
    for (int s = 0; s < 256; ++s)
        if (cb->code_len[s] && cb->code_len[s] < shortest)
            shortest = cb->code_len[s];
    if (shortest == 1)
        return 8;
    const uint64_t chunk_bits = (uint64_t)DF11_THREADS_PER_CHUNK * 8 * 16;
    const uint64_t chunks = (cb->total_bits + chunk_bits - 1) / chunk_bits;
    return chunks < (uint64_t)sm_count * DF11_DECODE_WARPS_PER_SM ? 8u : 16u;
}

df11_status df11_compress_sizes(const df11_codebook *cb, const df11_layout *layout,
                                df11_sizes *out)
{
    if (!cb || !out || !layout_ok(layout) || cb->n_elements == 0 || cb->total_bits == 0 ||
        cb->n_tables == 0 || cb->n_tables > 256)
        return DF11_ERR_INVALID_ARGUMENT;
    *out = sizes_for(cb->total_bits, cb->n_elements, cb->n_tables, layout);
    return DF11_OK;
}

df11_status df11_compress(const df11_codebook *cb, const df11_layout *layout,
                          const uint16_t *const *mats, const uint64_t *numel,
                          uint32_t n_mats, df11_host_block *out)
{
    if (!cb || !out || !layout_ok(layout) || !check_mats(mats, numel, n_mats))
        return DF11_ERR_INVALID_ARGUMENT;
    if (!out->exp_stream || !out->gaps || !out->counts || !out->chunk_pos || !out->signmant || !out->lut)
        return DF11_ERR_INVALID_ARGUMENT;
    ElementView v(mats, numel, n_mats);
    if (v.total == 0 || v.total != cb->n_elements)
        return DF11_ERR_INVALID_ARGUMENT;
    if (v.total >= (1ull << 32))
        return DF11_ERR_OVERFLOW;
    df11_sizes z;
    df11_status st = df11_compress_sizes(cb, layout, &z);
    if (st != DF11_OK)
        return st;
    if (out->exp_stream_bytes < z.exp_stream_bytes || out->gaps_bytes < z.gaps_bytes ||
        out->counts_bytes < z.counts_bytes || out->chunk_pos_count < z.chunk_pos_count ||
        out->signmant_bytes < z.signmant_bytes || out->lut_entries < z.lut_entries)
        return DF11_ERR_BUFFER_TOO_SMALL;

    uint64_t h[256];
    histogram(v, h);
    if (std::memcmp(h, cb->histogram, sizeof(h)) != 0)
        return DF11_ERR_INVALID_ARGUMENT;

    const uint8_t *len = cb->code_len;
    const uint32_t *code = cb->code;
    const uint32_t T = layout->threads_per_chunk;
    const uint64_t kSliceBits = 8ull * layout->bytes_per_thread;
    const uint64_t N = v.total;
    const uint64_t total_bits = cb->total_bits;

    // Segments of the element sequence, encoded in parallel at known offsets.
    const unsigned nw = worker_count(N);
    const unsigned nseg = nw;
    std::vector<uint64_t> seg_lo(nseg + 1), seg_bits(nseg + 1, 0);
    for (unsigned i = 0; i <= nseg; ++i)
        seg_lo[i] = N * i / nseg;
    parallel_for(nseg, [&](unsigned i) {
        uint64_t b = 0;
        v.for_range(seg_lo[i], seg_lo[i + 1], [&](uint64_t, uint16_t x) { b += len[(x >> 7) & 0xFF]; });
        seg_bits[i] = b;
    });
    std::vector<uint64_t> seg_start(nseg + 1, 0);
    for (unsigned i = 0; i < nseg; ++i)
        seg_start[i + 1] = seg_start[i] + seg_bits[i];
    if (seg_start[nseg] != total_bits)
        return DF11_ERR_INVALID_ARGUMENT;

    uint8_t *stream = out->exp_stream;
    const uint64_t used_bytes = (total_bits + 7) / 8;
    std::memset(stream + used_bytes, 0, z.exp_stream_bytes - used_bytes);
    std::vector<uint8_t> gap_tmp(z.n_threads, 0);
    // element index of the first code starting in each slice (N for slices
    // no code starts in); a slice's count is the difference to the next one
    std::vector<uint32_t> first_elem(z.n_threads + 1, (uint32_t)N);
    std::vector<uint8_t> first_byte(nseg, 0);
    uint32_t *pos = out->chunk_pos;
    std::memset(pos, 0, sizeof(uint32_t) * z.chunk_pos_count);

    parallel_for(nseg, [&](unsigned i) {
        uint64_t lo = seg_lo[i], hi = seg_lo[i + 1];
        uint64_t bit = seg_start[i];
        uint64_t byte_at = bit >> 3;
        const bool shared_first = (bit & 7) != 0;
        bool first_pending = shared_first;
        uint64_t acc = 0;
        uint32_t nacc = (uint32_t)(bit & 7);  // leading bits owned by the previous segment
        // slice of the previous code start, to spot the first start in a slice
        uint64_t prev_slice = ~0ull;
        if (lo > 0) {
            uint64_t prev_len = 0;
            v.for_range(lo - 1, lo, [&](uint64_t, uint16_t x) { prev_len = len[(x >> 7) & 0xFF]; });
            prev_slice = (bit - prev_len) / kSliceBits;
        }
        auto emit = [&](uint8_t b) {
            if (first_pending) {
                first_byte[i] = b;
                first_pending = false;
            } else {
                stream[byte_at] = b;
            }
            ++byte_at;
        };
        v.for_range(lo, hi, [&](uint64_t k, uint16_t x) {
            uint32_t s = (x >> 7) & 0xFF;
            uint64_t g = bit / kSliceBits;
            if (g != prev_slice) {
                gap_tmp[g] = (uint8_t)(bit - g * kSliceBits);
                first_elem[g] = (uint32_t)k;
                if (g % T == 0)
                    pos[g / T] = (uint32_t)k;
                prev_slice = g;
            }
            uint32_t l = len[s];
            acc = (acc << l) | code[s];
            nacc += l;
            bit += l;
            while (nacc >= 8) {
                emit((uint8_t)(acc >> (nacc - 8)));
                nacc -= 8;
            }
        });
        if (nacc > 0)
            emit((uint8_t)(acc << (8 - nacc)));
        if (first_pending)  // the segment never finished its first byte
            first_byte[i] = 0;
    });
    // merge the bytes shared between neighbouring segments
    for (unsigned i = 0; i < nseg; ++i)
        if (seg_start[i] & 7)
            stream[seg_start[i] >> 3] |= first_byte[i];
    // the end of the stream counts as a code start
    {
        uint64_t g = total_bits / kSliceBits;
        uint64_t last_len = 0;
        v.for_range(N - 1, N, [&](uint64_t, uint16_t x) { last_len = len[(x >> 7) & 0xFF]; });
        uint64_t last_slice = (total_bits - last_len) / kSliceBits;
        if (g < z.n_threads && g != last_slice) {
            gap_tmp[g] = (uint8_t)(total_bits - g * kSliceBits);
            if (g % T == 0)
                pos[g / T] = (uint32_t)N;
        }
        pos[z.n_chunks] = (uint32_t)N;
    }
    for (uint64_t j = 0; j < z.gaps_bytes; ++j)
        out->gaps[j] = (uint8_t)((gap_tmp[2 * j] & 0xF) | ((gap_tmp[2 * j + 1] & 0xF) << 4));
    for (uint64_t g = 0; g < z.n_threads; ++g)
        out->counts[g] = (uint8_t)(first_elem[g + 1] - first_elem[g]);

    parallel_for(nw, [&](unsigned w) {
        uint64_t lo = N * w / nw, hi = N * (w + 1) / nw;
        uint8_t *sm = out->signmant;
        v.for_range(lo, hi, [sm](uint64_t k, uint16_t x) {
            sm[k] = (uint8_t)(((x >> 8) & 0x80) | (x & 0x7F));
        });
    });
    std::memset(out->signmant + N, 0, z.signmant_bytes - N);
    std::memcpy(out->lut, cb->lut, sizeof(uint16_t) * z.lut_entries);

    out->hdr.max_code_len = cb->max_code_len;
    out->hdr.threads_per_chunk = T;
    out->hdr.bytes_per_thread = layout->bytes_per_thread;
    out->hdr.n_tables = cb->n_tables;
    out->hdr.min_code_len = DF11_MAX_CODE_LEN;
    for (int s = 0; s < 256; ++s)
        if (cb->code_len[s] && cb->code_len[s] < out->hdr.min_code_len)
            out->hdr.min_code_len = cb->code_len[s];
    out->hdr.reserved = 0;
    out->hdr.total_bits = total_bits;
    out->hdr.n_elements = N;
    out->hdr.n_chunks = z.n_chunks;
    return DF11_OK;
}

df11_status df11_validate(const df11_host_block *b)
{
    if (!b || !b->exp_stream || !b->gaps || !b->counts || !b->chunk_pos || !b->signmant || !b->lut)
        return DF11_ERR_INVALID_ARGUMENT;
    const df11_header &h = b->hdr;
    df11_layout ly{h.threads_per_chunk, h.bytes_per_thread};
    if (!layout_ok(&ly) || h.max_code_len < 1 || h.max_code_len > DF11_MAX_CODE_LEN ||
        h.n_tables < 1 || h.n_tables > 256 || h.n_elements == 0 ||
        h.min_code_len < 1 || h.min_code_len > h.max_code_len ||
        h.n_elements >= (1ull << 32) || h.total_bits < h.n_elements ||
        h.total_bits > h.n_elements * h.max_code_len)
        return DF11_ERR_CORRUPT;
    df11_sizes z = sizes_for(h.total_bits, h.n_elements, h.n_tables, &ly);
    if (h.n_chunks != z.n_chunks || b->exp_stream_bytes < z.exp_stream_bytes ||
        b->gaps_bytes < z.gaps_bytes || b->counts_bytes < z.counts_bytes ||
        b->chunk_pos_count < z.chunk_pos_count ||
        b->signmant_bytes < h.n_elements || b->lut_entries < z.lut_entries)
        return DF11_ERR_CORRUPT;
    // output positions: 0 .. n_elements, monotone, at most one code per bit
    const uint64_t kSliceBits = 8ull * h.bytes_per_thread;
    const uint64_t chunk_bits = (uint64_t)h.threads_per_chunk * kSliceBits;
    if (b->chunk_pos[0] != 0 || b->chunk_pos[h.n_chunks] != h.n_elements)
        return DF11_ERR_CORRUPT;
    for (uint64_t c = 0; c < h.n_chunks; ++c) {
        uint32_t a = b->chunk_pos[c], e = b->chunk_pos[c + 1];
        if (e < a || e - a > chunk_bits)
            return DF11_ERR_CORRUPT;
    }
    // gaps: below the cap inside the stream, zero past its end, zero for thread 0
    for (uint64_t g = 0; g < z.n_threads; ++g) {
        uint32_t gap = (b->gaps[g >> 1] >> ((g & 1) * 4)) & 0xF;
        uint64_t base = g * kSliceBits;
        if (base >= h.total_bits ? gap != 0 : (gap >= h.max_code_len || base + gap > h.total_bits))
            return DF11_ERR_CORRUPT;
    }
    if ((b->gaps[0] & 0xF) != 0)
        return DF11_ERR_CORRUPT;
    // counts: a chunk's add up to its output range; none above what the
    // shortest code allows in a slice, none past the end of the stream
    for (uint64_t c = 0; c < h.n_chunks; ++c) {
        uint64_t sum = 0;
        for (uint64_t t = 0; t < h.threads_per_chunk; ++t) {
            const uint64_t g = c * h.threads_per_chunk + t;
            const uint32_t n = b->counts[g];
            if (n > (kSliceBits + h.min_code_len - 1) / h.min_code_len ||
                (g * kSliceBits >= h.total_bits && n != 0))
                return DF11_ERR_CORRUPT;
            sum += n;
        }
        if (sum != (uint64_t)b->chunk_pos[c + 1] - b->chunk_pos[c])
            return DF11_ERR_CORRUPT;
    }
    // tables: root leaves <= 8 bits, pointers to existing sub-tables, each
    // sub-table entry a leaf of 9..cap bits
    for (uint32_t t = 0; t < h.n_tables; ++t) {
        for (uint32_t i = 0; i < 256; ++i) {
            uint16_t e = b->lut[t * 256 + i];
            uint32_t l = (e >> 8) & 0x1F;
            if (e & kLutPointer) {
                uint32_t to = e & 0xFF;
                if (t != 0 || to == 0 || to >= h.n_tables || (e & 0x7F00))
                    return DF11_ERR_CORRUPT;
            } else if (e & 0x4000) {
                if (e != kLutNoCode || t != 0 || h.min_code_len != 1)
                    return DF11_ERR_CORRUPT;
            } else if (t == 0 ? (l < 1 || l > 8) : (l < 9 || l > h.max_code_len)) {
                return DF11_ERR_CORRUPT;
            } else if (l < h.min_code_len) {
                return DF11_ERR_CORRUPT;
            }
        }
    }
    return DF11_OK;
}

df11_status df11_build_decode_table(const uint16_t *lut, uint32_t n_tables, uint32_t min_code_len,
                                    uint64_t *table)
{
    if (!lut || !table || n_tables < 1 || n_tables > 256 || min_code_len < 1 ||
        min_code_len > DF11_MAX_CODE_LEN)
        return DF11_ERR_INVALID_ARGUMENT;
    // the tables as the decoder sanitises them: a malformed entry, or one
    // shorter than the shortest code, reads as "no code"
    const uint16_t no_code = (uint16_t)(0x4000u | (min_code_len << 8));
    std::vector<uint16_t> t((size_t)n_tables * 256);
    for (uint32_t i = 0; i < n_tables * 256u; ++i) {
        uint32_t e = lut[i];
        if (e & kLutPointer) {
            const uint32_t to = e & 0xFFu;
            if (i >= 256u || to == 0 || to >= n_tables || (e & 0x7F00u))
                e = no_code;
        } else {
            const uint32_t l = (e >> 8) & 0x1Fu;
            if ((e & 0x4000u) || l < min_code_len || l > DF11_MAX_CODE_LEN)
                e = no_code;
        }
        t[i] = (uint16_t)e;
    }
    // entry k serves the window whose first stream bit is bit 0 of k:
    // the whole codes the window starts with, at most four, as rotated
    // exponents (bit 0 moved to bit 7) in bytes 0..3, and their total
    // length | 8 x count << 16; a first code longer than the window (or
    // none) gives the marker 0x80000000 << 32
    for (uint32_t k = 0; k < DF11_DECODE_TABLE_ENTRIES; ++k) {
        uint32_t win = 0;   // MSB-first: first stream bit at bit 31
        for (uint32_t b = 0; b < DF11_DECODE_TABLE_WINDOW_BITS; ++b)
            win |= ((k >> b) & 1u) << (31 - b);
        uint32_t used = 0, n = 0, syms = 0;
        while (n < 4) {
            const uint32_t v = win << used;
            uint32_t e = t[v >> 24];
            if (e & kLutPointer)
                e = t[((e & 0xFFu) << 8) | ((v >> 16) & 0xFFu)];
            if (e & 0x4000u)
                break;
            const uint32_t l = (e >> 8) & 0x1Fu;
            if (used + l > DF11_DECODE_TABLE_WINDOW_BITS)
                break;
            const uint32_t x = e & 0xFFu;
            syms |= (((x >> 1) | ((x & 1u) << 7)) & 0xFFu) << (8 * n);
            ++n;
            used += l;
        }
        const uint32_t y = n ? used | (8u * n << 16) : 0x80000000u;
        table[k] = (uint64_t)syms | ((uint64_t)y << 32);
    }
    return DF11_OK;
}

}  // extern "C"
