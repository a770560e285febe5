// df11_decode.cu -- GPU decode of one DF11 block into BF16 (sm_100a).
//
// Method: "DFloat11: lossless BFloat16 compression" (ai-infrastructure.net),
// section "Architecture": each thread owns a fixed 8-byte slice of the
// exponent stream and starts at its Gaps offset; a block-wide prefix sum of
// per-thread counts places the outputs; exponents are joined with the raw
// sign|mantissa bytes and written with coalesced stores; one launch covers
// every matrix of a block.
//
// B200 design (differs from the page's two-phase kernel):
//   * single decode pass: each thread decodes its slice once, packing four
//     exponents per 32-bit word into a shared-memory slot column (conflict
//     free: at any loop step all active lanes write the same slot row);
//   * warp-shuffle + block scan of the counts; the words are then compacted
//     into a contiguous exponent buffer placed at the chunk's 8-element
//     alignment, so the merge reads 8 exponents and 8 sign|mantissa bytes
//     per thread and writes one 16-byte BF16 vector per thread;
//   * 16-bit table entries carrying (symbol, total length) or a sub-table
//     pointer, sanitised once per CTA when copied to shared memory, so the
//     hot loop needs no bounds checks;
//   * persistent CTAs, grid = resident CTAs per SM x SM count.
// No tensor cores: this is integer decode, bounded by HBM and issue rate.
#include "df11.h"

#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

namespace {

constexpr int kSlotRows = 16;          // 64 codes max per 64-bit slice, 4 per word
constexpr int kSliceBits = 64;
constexpr uint32_t kLutPointer = 0x8000u;
constexpr uint32_t kLutNoCode = 0x4000u | (1u << 8);

struct DecodeParams {
    const uint8_t *stream;
    const uint8_t *gaps;
    const uint32_t *chunk_pos;
    const uint8_t *signmant;
    const uint16_t *lut;
    uint16_t *out;
    uint32_t *err;
    uint64_t total_bits;
    uint64_t n_chunks;
    uint64_t out_limit;   // min(n_elements, out_capacity)
    uint32_t n_tables;
};

template <int T>
constexpr size_t smem_bytes_for(uint32_t n_tables)
{
    return (size_t)kSlotRows * T * 4 + (size_t)kSliceBits * T + 16 + (size_t)n_tables * 512;
}

__device__ __forceinline__ uint32_t bswap32(uint32_t x) { return __byte_perm(x, 0, 0x0123); }

// Two BF16 words from two exponent bytes (low 16 bits of e, s) and two
// sign|mantissa bytes: v = [s0 e0 s1 e1] as bytes; per 16-bit half,
// exponent -> bits 14..7, sign -> bit 15, mantissa -> bits 6..0.
__device__ __forceinline__ uint32_t join2(uint32_t v)
{
    return ((v >> 1) & 0x7F807F80u) | ((v & 0x00800080u) << 8) | (v & 0x007F007Fu);
}

__device__ __forceinline__ uint16_t join1(uint32_t e, uint32_t s)
{
    return (uint16_t)(((s & 0x80u) << 8) | (e << 7) | (s & 0x7Fu));
}

template <int T>
__global__ void __launch_bounds__(T) df11_decode_kernel(DecodeParams p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    uint32_t *slots = reinterpret_cast<uint32_t *>(smem);               // [kSlotRows][T]
    uint8_t *ebuf = smem + (size_t)kSlotRows * T * 4;                   // 64*T + 16
    uint16_t *lut = reinterpret_cast<uint16_t *>(ebuf + kSliceBits * T + 16);
    __shared__ uint32_t warp_excl[T / 32];
    __shared__ uint32_t chunk_info[3];

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const uint32_t n_tables = p.n_tables;

    // Tables -> shared memory.  Anything malformed becomes a "no code" entry
    // (length 1), so the decode loop below always advances and never indexes
    // outside the tables.
    for (uint32_t i = tid; i < n_tables * 256u; i += T) {
        uint32_t e = p.lut[i];
        if (e & kLutPointer) {
            uint32_t to = e & 0xFFu;
            if (i >= 256u || to == 0 || to >= n_tables || (e & 0x7F00u))
                e = kLutNoCode;
        } else {
            uint32_t l = (e >> 8) & 0x1Fu;
            if ((e & 0x4000u) || l == 0 || l > 16)
                e = kLutNoCode;
        }
        lut[i] = (uint16_t)e;
    }
    __syncthreads();

    uint32_t err = 0;
    for (uint64_t chunk = blockIdx.x; chunk < p.n_chunks; chunk += gridDim.x) {
        // ---- decode this thread's slice -------------------------------
        const uint64_t g = chunk * T + tid;
        const uint64_t bit0 = g * kSliceBits;
        const uint2 v01 = *reinterpret_cast<const uint2 *>(p.stream + 8 * g);
        const uint32_t v2 = *reinterpret_cast<const uint32_t *>(p.stream + 8 * g + 8);
        const uint32_t gap = (p.gaps[g >> 1] >> ((g & 1) * 4)) & 0xFu;
        const int end = bit0 >= p.total_bits ? 0
                        : (int)min((uint64_t)kSliceBits, p.total_bits - bit0);
        uint32_t hi = bswap32(v01.x), lo = bswap32(v01.y);
        const uint32_t w2 = bswap32(v2);
        int bitpos = (int)gap;
        uint32_t count = 0, acc = 0, seen = 0;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int lim = min(end, 32 * (half + 1));
            while (bitpos < lim) {
                const uint32_t win = __funnelshift_l(lo, hi, (uint32_t)bitpos);
                uint32_t e = lut[win >> 24];
                if (e & kLutPointer)
                    e = lut[((e & 0xFFu) << 8) | ((win >> 16) & 0xFFu)];
                seen |= e;
                acc = (acc >> 8) | (e << 24);
                bitpos += (int)((e >> 8) & 0x1Fu);
                ++count;
                if ((count & 3u) == 0)
                    slots[((count >> 2) - 1) * T + tid] = acc;
            }
            hi = lo;
            lo = w2;
        }
        if (count & 3u)
            slots[(count >> 2) * T + tid] = acc >> (8 * (4 - (count & 3u)));
        if (seen & 0x4000u)
            err |= DF11_DEVERR_BAD_CODE;

        // ---- block scan of the counts ----------------------------------
        uint32_t incl = count;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (lane >= d)
                incl += y;
        }
        if (lane == 31)
            warp_excl[warp] = incl;
        if (tid == 0) {
            chunk_info[0] = p.chunk_pos[chunk];
            chunk_info[1] = p.chunk_pos[chunk + 1];
        }
        __syncthreads();
        if (warp == 0) {
            const uint32_t ws = lane < T / 32 ? warp_excl[lane] : 0u;
            uint32_t wi = ws;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, wi, d);
                if (lane >= d)
                    wi += y;
            }
            if (lane < T / 32)
                warp_excl[lane] = wi - ws;
            if (lane == 31)
                chunk_info[2] = wi;
        }
        __syncthreads();

        const uint32_t pos0 = chunk_info[0];
        const uint32_t pos1 = chunk_info[1];
        const uint32_t total = chunk_info[2];
        // uniform across the CTA: every thread takes the same branch
        if (pos1 < pos0 || (uint64_t)pos1 > p.out_limit || pos1 - pos0 > (uint32_t)(kSliceBits * T)) {
            err |= DF11_DEVERR_BAD_POS;
            __syncthreads();  // chunk_info is rewritten by the next chunk
            continue;
        }
        if (total != pos1 - pos0)
            err |= DF11_DEVERR_COUNT;
        const uint32_t n_write = min(total, pos1 - pos0);

        // ---- compaction into the chunk's exponent buffer ----------------
        const uint32_t head = pos0 & 7u;
        const uint32_t off = warp_excl[warp] + incl - count;
        uint8_t *dst = ebuf + head + off;
        for (uint32_t q = 0; q * 4 < count; ++q) {
            const uint32_t w = slots[q * T + tid];
#pragma unroll
            for (uint32_t b = 0; b < 4; ++b) {
                const uint32_t k = q * 4 + b;
                if (k < count && off + k < n_write)
                    dst[k] = (uint8_t)(w >> (8 * b));
            }
        }
        __syncthreads();

        // ---- merge with sign|mantissa and store -------------------------
        const uint64_t base = (uint64_t)pos0 - head;       // 8-element aligned
        const uint32_t span = head + n_write;
        const uint32_t groups = (span + 7) / 8;
        for (uint32_t i = tid; i < groups; i += T) {
            const uint32_t l0 = 8 * i;
            const uint64_t g0 = base + l0;
            if (l0 >= head && l0 + 8 <= span) {
                const uint2 e8 = *reinterpret_cast<const uint2 *>(ebuf + l0);
                const uint2 s8 = __ldg(reinterpret_cast<const uint2 *>(p.signmant + g0));
                uint4 o;
                o.x = join2(__byte_perm(s8.x, e8.x, 0x5140));
                o.y = join2(__byte_perm(s8.x, e8.x, 0x7362));
                o.z = join2(__byte_perm(s8.y, e8.y, 0x5140));
                o.w = join2(__byte_perm(s8.y, e8.y, 0x7362));
                *reinterpret_cast<uint4 *>(p.out + g0) = o;
            } else {
                for (uint32_t j = 0; j < 8; ++j) {
                    const uint32_t l = l0 + j;
                    if (l >= head && l < span)
                        p.out[base + l] = join1(ebuf[l], p.signmant[base + l]);
                }
            }
        }
        __syncthreads();
    }
    if (err && p.err)
        atomicOr(p.err, err);
}

// ------------------------------------------------------------ launch

constexpr int kMaxDevices = 64;
// resident CTAs per SM, by device, threads-per-chunk variant and table count
std::atomic<int> g_occupancy[kMaxDevices][3][257];
std::atomic<int> g_sm_count[kMaxDevices];
std::atomic<int> g_attr_done[kMaxDevices][3];

template <int T>
df11_status launch(const DecodeParams &prm, int dev, int variant, cudaStream_t stream)
{
    const size_t smem = smem_bytes_for<T>(prm.n_tables);
    if (!g_attr_done[dev][variant].load(std::memory_order_acquire)) {
        cudaError_t e = cudaFuncSetAttribute(df11_decode_kernel<T>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem_bytes_for<T>(256));
        if (e != cudaSuccess)
            return DF11_ERR_CUDA;
        g_attr_done[dev][variant].store(1, std::memory_order_release);
    }
    int sms = g_sm_count[dev].load(std::memory_order_relaxed);
    if (sms == 0) {
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return DF11_ERR_CUDA;
        g_sm_count[dev].store(sms, std::memory_order_relaxed);
    }
    int occ = g_occupancy[dev][variant][prm.n_tables].load(std::memory_order_relaxed);
    if (occ == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, df11_decode_kernel<T>, T, smem) !=
            cudaSuccess)
            return DF11_ERR_CUDA;
        if (occ < 1)
            return DF11_ERR_CUDA;
        g_occupancy[dev][variant][prm.n_tables].store(occ, std::memory_order_relaxed);
    }
    const uint64_t resident = (uint64_t)occ * (uint64_t)sms;
    const unsigned grid = (unsigned)(prm.n_chunks < resident ? prm.n_chunks : resident);
    df11_decode_kernel<T><<<grid, T, smem, stream>>>(prm);
    return cudaGetLastError() == cudaSuccess ? DF11_OK : DF11_ERR_CUDA;
}

bool aligned(const void *ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

}  // namespace

extern "C" df11_status df11_decompress_async(const df11_device_block *blk, uint16_t *out_bf16,
                                             uint64_t out_capacity, uint32_t *d_error,
                                             void *stream)
{
    if (!blk || !out_bf16)
        return DF11_ERR_INVALID_ARGUMENT;
    const df11_header &h = blk->hdr;
    const uint32_t T = h.threads_per_chunk;
    if ((T != 128 && T != 256 && T != 512) || h.bytes_per_thread != DF11_BYTES_PER_THREAD)
        return DF11_ERR_INVALID_ARGUMENT;
    if (h.n_elements == 0 || h.n_elements >= (1ull << 32) || h.n_tables < 1 || h.n_tables > 256 ||
        h.total_bits == 0 || out_capacity < h.n_elements)
        return DF11_ERR_INVALID_ARGUMENT;
    const uint64_t chunk_bits = (uint64_t)T * kSliceBits;
    if (h.n_chunks != (h.total_bits + chunk_bits - 1) / chunk_bits)
        return DF11_ERR_INVALID_ARGUMENT;
    const uint64_t n_threads = h.n_chunks * T;
    if (!blk->exp_stream || !blk->gaps || !blk->chunk_pos || !blk->signmant || !blk->lut)
        return DF11_ERR_INVALID_ARGUMENT;
    if (blk->exp_stream_bytes < n_threads * 8 + DF11_STREAM_PAD || blk->gaps_bytes < n_threads / 2 ||
        blk->chunk_pos_count < h.n_chunks + 1 || blk->signmant_bytes < h.n_elements ||
        blk->lut_entries < (uint64_t)h.n_tables * 256)
        return DF11_ERR_INVALID_ARGUMENT;
    if (!aligned(blk->exp_stream, 16) || !aligned(blk->chunk_pos, 16) || !aligned(blk->lut, 16) ||
        !aligned(blk->signmant, 8) || !aligned(out_bf16, 16) || !aligned(d_error, 4))
        return DF11_ERR_INVALID_ARGUMENT;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return DF11_ERR_CUDA;

    DecodeParams prm;
    prm.stream = blk->exp_stream;
    prm.gaps = blk->gaps;
    prm.chunk_pos = blk->chunk_pos;
    prm.signmant = blk->signmant;
    prm.lut = blk->lut;
    prm.out = out_bf16;
    prm.err = d_error;
    prm.total_bits = h.total_bits;
    prm.n_chunks = h.n_chunks;
    prm.out_limit = h.n_elements < out_capacity ? h.n_elements : out_capacity;
    prm.n_tables = h.n_tables;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (T) {
    case 128: return launch<128>(prm, dev, 0, s);
    case 256: return launch<256>(prm, dev, 1, s);
    default: return launch<512>(prm, dev, 2, s);
    }
}
