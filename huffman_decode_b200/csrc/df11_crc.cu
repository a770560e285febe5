// df11_crc.cu -- CRC-32C checksums of a DF11 artifact, on the host and on
// the GPU.
//
// The pages warn that one flipped bit in the exponent stream silently
// rewrites most of a tensor and tell users to checksum DF11 artifacts on
// download and after every copy ("DFloat11: lossless BFloat16 compression",
// sections "How to run it in production" and "Failure modes"; the
// corruption test in "How it works: the core algorithm").  Here the checksum
// is a list: the CRC-32C (Castagnoli; reflected polynomial 0x82F63B78,
// initial value and final XOR 0xFFFFFFFF) of every 4096-byte segment of the
// block's six arrays, in the order exp_stream, gaps, counts, chunk_pos,
// signmant, lut (the last segment of an array is shorter).  Segments make the GPU
// check embarrassingly parallel and locate damage.
//
// GPU method: one warp per segment, lane l covers bytes [128 l, 128 l + 128)
// of it.  A lane folds its bytes four at a time (x = crc ^ word; crc = x
// advanced over four zero bytes, which is linear in x: four 256-entry table
// lookups in a copy of the tables private to the lane, so the 32 lanes of a
// warp never meet on a shared-memory bank).  The 32 partial CRCs are joined
// in a five-level tree: CRC is linear, and crc(A || B) = crc(A) advanced
// over |B| zero bytes, XOR crc(B).  "Advance over 2^j zero bytes"
// is a table operator S_j (4 x 256 words) built in shared memory by
// squaring S_{j-1}.  The initial value enters the same way: the standard CRC
// of n bytes is the zero-initialised one XOR (0xFFFFFFFF advanced over n
// bytes) XOR 0xFFFFFFFF.
#include "df11.h"

#include <cuda_runtime.h>

#include <atomic>
#include <cstring>

namespace {

constexpr uint32_t kPolyReflected = 0x82F63B78u;
constexpr uint64_t kSeg = DF11_CRC_SEGMENT_BYTES;
constexpr int kLaneBytes = (int)(kSeg / 32);     // 128
constexpr int kShiftOps = 13;                    // advance by 2^0 .. 2^12 bytes
constexpr int kCrcThreads = 1024;
// shared: byte table | S_0..S_12 | a lane-private copy of S_2 (the four-byte
// fold), entry e of lane l at word 32 e + l, so every lane reads its own bank
constexpr size_t kPrivWords = 1024 * 32;
constexpr size_t kCrcSmem = (256 + (size_t)kShiftOps * 1024 + kPrivWords) * 4;

static_assert(kSeg == 4096, "one warp of 32 lanes x 128 bytes per segment");

constexpr int kArrays = 6;

struct ArrayView {
    const uint8_t *ptr[kArrays];
    uint64_t len[kArrays];
    uint64_t first[kArrays + 1];   // first segment index of each array; first[kArrays] = total
};

template <class Block>
ArrayView view_of(const Block *b)
{
    ArrayView v;
    const uint8_t *ps[kArrays] = {b->exp_stream, b->gaps, b->counts,
                                  reinterpret_cast<const uint8_t *>(b->chunk_pos), b->signmant,
                                  reinterpret_cast<const uint8_t *>(b->lut)};
    const uint64_t ls[kArrays] = {b->exp_stream_bytes, b->gaps_bytes, b->counts_bytes, b->chunk_pos_count * 4,
                                  b->signmant_bytes, b->lut_entries * 2};
    v.first[0] = 0;
    for (int a = 0; a < kArrays; ++a) {
        v.ptr[a] = ps[a];
        v.len[a] = ls[a];
        v.first[a + 1] = v.first[a] + (ls[a] + kSeg - 1) / kSeg;
    }
    return v;
}


// ---- host ------------------------------------------------------------------

struct ByteTable {
    uint32_t v[256];
    ByteTable()
    {
        for (uint32_t i = 0; i < 256; ++i) {
            uint32_t c = i;
            for (int k = 0; k < 8; ++k)
                c = (c >> 1) ^ (kPolyReflected & (0u - (c & 1u)));
            v[i] = c;
        }
    }
};

uint32_t crc_bytes_table(uint32_t c, const uint8_t *p, uint64_t n)
{
    static const ByteTable t;   // built once, thread-safe
    for (uint64_t i = 0; i < n; ++i)
        c = (c >> 8) ^ t.v[(c ^ p[i]) & 0xFFu];
    return c;
}

#if defined(__x86_64__)
// The SSE4.2 crc32 instruction computes exactly this CRC (Castagnoli,
// reflected) without the initial value and final XOR.
__attribute__((target("sse4.2"))) uint32_t crc_bytes_sse42(uint32_t c, const uint8_t *p, uint64_t n)
{
    uint64_t c64 = c;
    while (n >= 8) {
        uint64_t w;
        std::memcpy(&w, p, 8);
        c64 = __builtin_ia32_crc32di(c64, w);
        p += 8;
        n -= 8;
    }
    c = (uint32_t)c64;
    while (n--)
        c = __builtin_ia32_crc32qi(c, *p++);
    return c;
}

bool have_sse42()
{
    static const bool ok = __builtin_cpu_supports("sse4.2");
    return ok;
}
#endif

uint32_t crc32c_host(const uint8_t *p, uint64_t n)
{
#if defined(__x86_64__)
    if (have_sse42())
        return ~crc_bytes_sse42(0xFFFFFFFFu, p, n);
#endif
    return ~crc_bytes_table(0xFFFFFFFFu, p, n);
}

// ---- device ----------------------------------------------------------------

__device__ __forceinline__ uint32_t advance(const uint32_t *op, uint32_t c)
{
    return op[c & 0xFFu] ^ op[256 + ((c >> 8) & 0xFFu)] ^ op[512 + ((c >> 16) & 0xFFu)] ^ op[768 + (c >> 24)];
}

// Advance c over m zero bytes (m < 2^kShiftOps) with the squaring operators.
__device__ __forceinline__ uint32_t advance_by(const uint32_t *ops, uint32_t c, uint32_t m)
{
#pragma unroll
    for (int j = 0; j < kShiftOps; ++j)
        if ((m >> j) & 1u)
            c = advance(ops + j * 1024, c);
    return c;
}

// c advanced over the four bytes of w (operator S_2), from the lane's
// private copy: lane_priv points at word `lane` of it.
__device__ __forceinline__ uint32_t fold_word(const uint32_t *lane_priv, uint32_t c, uint32_t w)
{
    const uint32_t x = c ^ w;
    return lane_priv[32 * (x & 0xFFu)] ^ lane_priv[32 * (256 + ((x >> 8) & 0xFFu))] ^
           lane_priv[32 * (512 + ((x >> 16) & 0xFFu))] ^ lane_priv[32 * (768 + (x >> 24))];
}

__global__ void __launch_bounds__(kCrcThreads) crc_kernel(ArrayView av, uint32_t *out, const uint32_t *expected,
                                                          uint32_t *err, unsigned long long *first_bad)
{
    extern __shared__ uint32_t tab[];
    uint32_t *t0 = tab;          // one-byte step table
    uint32_t *ops = tab + 256;   // S_j[k][v] = (v << 8k) advanced over 2^j zero bytes
    const int tid = threadIdx.x;
    for (int i = tid; i < 256; i += blockDim.x) {
        uint32_t c = (uint32_t)i;
        for (int k = 0; k < 8; ++k)
            c = (c >> 1) ^ (kPolyReflected & (0u - (c & 1u)));
        t0[i] = c;
    }
    __syncthreads();
    for (int i = tid; i < 1024; i += blockDim.x) {
        const uint32_t c = (uint32_t)(i & 255) << (8 * (i >> 8));
        ops[i] = (c >> 8) ^ t0[c & 0xFFu];
    }
    __syncthreads();
    for (int j = 1; j < kShiftOps; ++j) {
        for (int i = tid; i < 1024; i += blockDim.x)
            ops[j * 1024 + i] = advance(ops + (j - 1) * 1024, ops[(j - 1) * 1024 + i]);
        __syncthreads();
    }
    uint32_t *priv = ops + kShiftOps * 1024;
    for (int i = tid; i < (int)kPrivWords; i += blockDim.x)
        priv[i] = ops[2 * 1024 + (i >> 5)];
    __syncthreads();

    const int lane = tid & 31;
    const uint32_t *lane_priv = priv + lane;
    // the initial value's part of a full segment's CRC
    const uint32_t init_full = advance(ops + 12 * 1024, 0xFFFFFFFFu);
    const uint64_t warps = blockDim.x >> 5;
    const uint64_t total = av.first[kArrays];
    for (uint64_t seg = blockIdx.x * warps + (tid >> 5); seg < total; seg += gridDim.x * warps) {
        // the array holding the segment: the last one whose first segment is
        // <= seg (empty arrays share their first index with the next one)
        const uint8_t *aptr = av.ptr[0];
        uint64_t alen = av.len[0], afirst = 0;
#pragma unroll
        for (int k = 1; k < kArrays; ++k)
            if (seg >= av.first[k]) {
                aptr = av.ptr[k];
                alen = av.len[k];
                afirst = av.first[k];
            }
        const uint64_t local = seg - afirst;
        const uint8_t *base = aptr + local * kSeg;
        const uint64_t rem = alen - local * kSeg;
        const uint32_t n = (uint32_t)(rem < kSeg ? rem : kSeg);
        uint32_t c = 0;
        if (n == (uint32_t)kSeg) {
            // a full segment: lane l folds the four 32-byte runs l, l + 32,
            // l + 64 and l + 96 (bytes 32 l + 1024 k), so each load
            // instruction reads 1 KB of contiguous bytes, as four independent
            // chains; joins them (advancing over the 1 KB between runs);
            // then a five-level tree in which lanes 2^(j+1) i join the value
            // of the lane 2^j on, advanced over 32 * 2^j bytes (lane 0 ends
            // with the segment's)
            uint32_t v[kLaneBytes / 4];
            const uint8_t *src = base + 32 * lane;
            if ((reinterpret_cast<uintptr_t>(aptr) & 31u) == 0) {
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    asm volatile("ld.global.nc.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                                 : "=r"(v[8 * k]), "=r"(v[8 * k + 1]), "=r"(v[8 * k + 2]), "=r"(v[8 * k + 3]),
                                   "=r"(v[8 * k + 4]), "=r"(v[8 * k + 5]), "=r"(v[8 * k + 6]), "=r"(v[8 * k + 7])
                                 : "l"(src + 1024 * k));
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint4 q = __ldg(reinterpret_cast<const uint4 *>(src + 1024 * (k >> 1)) + (k & 1));
                    v[4 * k] = q.x;
                    v[4 * k + 1] = q.y;
                    v[4 * k + 2] = q.z;
                    v[4 * k + 3] = q.w;
                }
            }
            uint32_t r[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int w = 0; w < 8; ++w) {
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    r[k] = fold_word(lane_priv, r[k], v[8 * k + w]);
            }
            c = r[0];
#pragma unroll
            for (int k = 1; k < 4; ++k)
                c = advance(ops + 10 * 1024, c) ^ r[k];         // S_10: over 1024 zero bytes
#pragma unroll
            for (int j = 0; j < 5; ++j) {
                const uint32_t right = __shfl_down_sync(0xFFFFFFFFu, c, 1 << j);
                c = advance(ops + (5 + j) * 1024, c) ^ right;   // S_{5+j}: over 32 * 2^j zero bytes
            }
        } else {
            // the short last segment of an array: lanes fold what they have,
            // advance over the bytes after their run, and the warp XORs
            const uint32_t beg = (uint32_t)(kLaneBytes * lane);
            const uint32_t end = beg < n ? min(n, beg + (uint32_t)kLaneBytes) : beg;
            uint32_t q = beg;
            for (; q + 16 <= end; q += 16) {
                const uint4 v = __ldg(reinterpret_cast<const uint4 *>(base + q));
                c = fold_word(lane_priv, c, v.x);
                c = fold_word(lane_priv, c, v.y);
                c = fold_word(lane_priv, c, v.z);
                c = fold_word(lane_priv, c, v.w);
            }
            for (; q < end; ++q)
                c = (c >> 8) ^ t0[(c ^ base[q]) & 0xFFu];
            c = advance_by(ops, c, end > beg ? n - end : 0u);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                c ^= __shfl_xor_sync(0xFFFFFFFFu, c, o);
        }
        if (lane == 0) {
            const uint32_t crc = c ^ (n == (uint32_t)kSeg ? init_full : advance_by(ops, 0xFFFFFFFFu, n)) ^ 0xFFFFFFFFu;
            if (out)
                out[seg] = crc;
            if (expected && expected[seg] != crc) {
                atomicOr(err, DF11_DEVERR_CHECKSUM);
                if (first_bad)
                    atomicMin(first_bad, (unsigned long long)seg);
            }
        }
    }
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

df11_status launch_crc(const df11_device_block *blk, uint32_t *d_out, const uint32_t *d_expected,
                       uint64_t n_crc, uint32_t *d_error, uint64_t *d_first_bad, void *stream)
{
    if (!blk || !blk->exp_stream || !blk->gaps || !blk->counts || !blk->chunk_pos || !blk->signmant || !blk->lut)
        return DF11_ERR_INVALID_ARGUMENT;
    if (!aligned16(blk->exp_stream) || !aligned16(blk->gaps) || !aligned16(blk->counts) || !aligned16(blk->chunk_pos) ||
        !aligned16(blk->signmant) || !aligned16(blk->lut))
        return DF11_ERR_INVALID_ARGUMENT;
    const ArrayView av = view_of(blk);
    if (n_crc != av.first[kArrays] || av.first[kArrays] == 0)
        return DF11_ERR_INVALID_ARGUMENT;
    if ((reinterpret_cast<uintptr_t>(d_out) & 3u) || (reinterpret_cast<uintptr_t>(d_expected) & 3u) ||
        (reinterpret_cast<uintptr_t>(d_error) & 3u) || (reinterpret_cast<uintptr_t>(d_first_bad) & 7u))
        return DF11_ERR_INVALID_ARGUMENT;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return DF11_ERR_CUDA;
    static std::atomic<int> attr_done[64];
    if (dev < 0 || dev >= 64)
        return DF11_ERR_CUDA;
    if (!attr_done[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(crc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kCrcSmem) !=
            cudaSuccess)
            return DF11_ERR_CUDA;
        attr_done[dev].store(1, std::memory_order_release);
    }
    const uint64_t warps = kCrcThreads / 32;
    const uint64_t need = (av.first[kArrays] + warps - 1) / warps;
    const uint64_t cap = (uint64_t)sms;   // one 32-warp CTA per SM (the private table fills shared memory)
    const unsigned grid = (unsigned)(need < cap ? need : cap);
    crc_kernel<<<grid, kCrcThreads, kCrcSmem, reinterpret_cast<cudaStream_t>(stream)>>>(
        av, d_out, d_expected, d_error, reinterpret_cast<unsigned long long *>(d_first_bad));
    return cudaGetLastError() == cudaSuccess ? DF11_OK : DF11_ERR_CUDA;
}

}  // namespace

extern "C" uint64_t df11_checksum_count(const df11_host_block *blk)
{
    if (!blk)
        return 0;
    return view_of(blk).first[kArrays];
}

extern "C" df11_status df11_checksum(const df11_host_block *blk, uint32_t *crc, uint64_t n_crc)
{
    if (!blk || !crc || !blk->exp_stream || !blk->gaps || !blk->counts || !blk->chunk_pos || !blk->signmant || !blk->lut)
        return DF11_ERR_INVALID_ARGUMENT;
    const ArrayView av = view_of(blk);
    if (n_crc != av.first[kArrays])
        return DF11_ERR_INVALID_ARGUMENT;
    for (int a = 0; a < kArrays; ++a)
        for (uint64_t s = 0; s < av.first[a + 1] - av.first[a]; ++s) {
            const uint64_t off = s * kSeg;
            const uint64_t n = av.len[a] - off < kSeg ? av.len[a] - off : kSeg;
            crc[av.first[a] + s] = crc32c_host(av.ptr[a] + off, n);
        }
    return DF11_OK;
}

extern "C" uint32_t df11_crc32c(const void *data, uint64_t n)
{
    if (!data && n)
        return 0;
    return crc32c_host(static_cast<const uint8_t *>(data), n);
}

extern "C" df11_status df11_checksum_device_async(const df11_device_block *blk, uint32_t *d_crc, uint64_t n_crc,
                                                  void *stream)
{
    if (!d_crc)
        return DF11_ERR_INVALID_ARGUMENT;
    return launch_crc(blk, d_crc, nullptr, n_crc, nullptr, nullptr, stream);
}

extern "C" df11_status df11_verify_device_async(const df11_device_block *blk, const uint32_t *d_expected,
                                                uint64_t n_crc, uint32_t *d_error, uint64_t *d_first_bad,
                                                void *stream)
{
    if (!d_expected || !d_error)
        return DF11_ERR_INVALID_ARGUMENT;
    return launch_crc(blk, nullptr, d_expected, n_crc, d_error, d_first_bad, stream);
}

// ---- per-chunk sums (host) ---------------------------------------------------
// The same sums the decode kernel's verifying path computes (include/df11.h):
// the chunk's stream words (bit-reversed big-endian words), the threads'
// gap and count, the two positions, the sign|mantissa bytes (whole 8-element
// groups as two words, the rest byte by byte), and in chunk 0 the tables.

namespace {

inline uint32_t chunk_mix(uint32_t v, uint32_t tag)
{
    const uint32_t y = (v ^ (tag * 0x9E3779B1u)) * 0x85EBCA6Bu;
    return y ^ (y >> 16);
}

inline uint32_t brev32(uint32_t x)
{
    x = ((x >> 1) & 0x55555555u) | ((x & 0x55555555u) << 1);
    x = ((x >> 2) & 0x33333333u) | ((x & 0x33333333u) << 2);
    x = ((x >> 4) & 0x0F0F0F0Fu) | ((x & 0x0F0F0F0Fu) << 4);
    return __builtin_bswap32(x);   // bytes reversed too: the whole word bit-reversed
}

inline uint32_t le32(const uint8_t *p)
{
    uint32_t v;
    std::memcpy(&v, p, 4);
    return v;
}

}  // namespace

extern "C" df11_status df11_chunk_sums(const df11_host_block *blk, uint32_t *sums, uint64_t n)
{
    if (!blk || !sums || !blk->exp_stream || !blk->gaps || !blk->counts || !blk->chunk_pos ||
        !blk->signmant || !blk->lut || n != blk->hdr.n_chunks || blk->hdr.threads_per_chunk != 32 ||
        (blk->hdr.bytes_per_thread != 8 && blk->hdr.bytes_per_thread != 16))
        return DF11_ERR_INVALID_ARGUMENT;
    const uint64_t W = blk->hdr.bytes_per_thread;
    if (blk->exp_stream_bytes < 32 * W * n || blk->gaps_bytes < 16 * n || blk->counts_bytes < 32 * n ||
        blk->chunk_pos_count < n + 1 || blk->lut_entries < 256ull * blk->hdr.n_tables)
        return DF11_ERR_INVALID_ARGUMENT;
    for (uint64_t c = 0; c < n; ++c) {
        uint32_t sum = 0;
        const uint8_t *st = blk->exp_stream + 32 * W * c;
        for (uint32_t k = 0; k < 8 * W; ++k)   // stream bit 32k + i at bit i: bit-reversed big-endian word
            sum += chunk_mix(brev32(__builtin_bswap32(le32(st + 4 * k))), k);
        for (uint32_t t = 0; t < 32; ++t) {
            const uint64_t g = 32 * c + t;
            const uint32_t gap = (blk->gaps[g >> 1] >> ((g & 1) * 4)) & 0xFu;
            sum += chunk_mix(gap | ((uint32_t)blk->counts[g] << 8), 0x10000u + t);
        }
        const uint64_t p0 = blk->chunk_pos[c], p1 = blk->chunk_pos[c + 1];
        if (p1 < p0 || p1 > blk->signmant_bytes)
            return DF11_ERR_INVALID_ARGUMENT;
        sum += chunk_mix((uint32_t)p0, 0x20000u) + chunk_mix((uint32_t)p1, 0x20001u);
        const uint64_t b = p0 & ~7ull;
        const uint64_t g_first = (p0 + 7) >> 3, g_end = p1 >> 3;   // whole groups [g_first, g_end)
        for (uint64_t q = g_first; q < g_end; ++q) {
            const uint32_t r = (uint32_t)(q - (b >> 3));
            sum += chunk_mix(le32(blk->signmant + 8 * q), 0x100000u + 2 * r) +
                   chunk_mix(le32(blk->signmant + 8 * q + 4), 0x100000u + 2 * r + 1);
        }
        const uint64_t whole_lo = g_first < g_end ? 8 * g_first : p1, whole_hi = g_first < g_end ? 8 * g_end : p1;
        for (uint64_t e = p0; e < p1; ++e)
            if (e < whole_lo || e >= whole_hi)
                sum += chunk_mix(blk->signmant[e], (uint32_t)(0x200000u + (e - b)));
        if (c == 0)
            for (uint32_t i = 0; i < 128u * blk->hdr.n_tables; ++i)
                sum += chunk_mix(blk->lut[2 * i] | ((uint32_t)blk->lut[2 * i + 1] << 16), 0x400000u + i);
        sums[c] = sum;
    }
    return DF11_OK;
}
