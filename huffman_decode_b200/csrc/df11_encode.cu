// df11_encode.cu -- GPU-side DF11 compressor (sm_100a).
//
// The pages compress on the CPU only ("DFloat11: lossless BFloat16
// compression", section "How to develop with it": single-thread compression
// per transformer block, minutes per block).  This file does the same work
// on the GPU for one block already in device memory:
//   1. df11_histogram_device   -- 256-bin exponent histogram (per-CTA shared
//                                 histograms, one global add per bin and CTA);
//   2. (host) df11_build_codebook_from_histogram -- code lengths, canonical
//                                 codes and tables from that histogram;
//   3. df11_compress_device    -- bit count per segment of 8192 elements
//      (one warp per segment; also summed per run of 256 segments), then one
//      encode pass, a CTA per segment, in which every thread knows its first
//      bit (the run totals and segment counts before its segment, and a CTA
//      scan): it appends its codes MSB-first to a bit accumulator and stores
//      each stream word it completes into the segment's staging in shared
//      memory, ORs its part-filled last word into the next thread's, records
//      the gap of every slice whose first code it owns and the output
//      position of every chunk that starts in such a slice, counts its codes
//      per slice, and writes its sign|mantissa bytes; the staged words then
//      go to global memory with plain stores, ORing only the two words a
//      segment may share with its neighbours, and the staged counts are
//      added into the (zeroed) counts array, four per word.
// The result is byte-identical to df11_compress (host) for the same
// codebook and layout ("How it works": canonical codes, MSB-first encode;
// "Architecture": Gaps and per-chunk output positions).
#include "df11.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>

namespace {

constexpr int kEncThreads = 256;
constexpr int kElemsPerThread = 32;
constexpr int kSegElems = kEncThreads * kElemsPerThread;   // 8192 elements per segment
constexpr int kRunSegs = 256;   // segments per run: an encode CTA sums <= kRunSegs - 1 counts and the run totals

// Code table passed by value: entry s = code | (length << 24); length 0 = absent.
struct CodeTable {
    uint32_t e[256];
};

struct EncodeParams {
    const uint16_t *in;
    uint8_t *stream;
    uint8_t *gaps;
    uint8_t *counts;
    uint32_t *chunk_pos;
    uint8_t *signmant;
    uint32_t *seg_bits;     // scratch: bits per segment
    uint64_t *run_bits;     // scratch: bits per run of kRunSegs segments
    uint32_t *code_table;   // scratch: the code table (code | length << 24), as in CodeTable
    uint16_t *grp_bits;     // scratch: bits per 32 elements of full segments, or null
    uint32_t *err;          // optional device error word
    uint64_t n;
    uint64_t n_seg;
    uint64_t total_bits;    // what the codebook promises
    uint64_t n_threads;     // decoding threads (slices)
    uint32_t slice_shift;   // log2(bits per slice)
    uint32_t threads_per_chunk;
};

__device__ __forceinline__ uint32_t bswap32(uint32_t x) { return __byte_perm(x, 0, 0x0123); }

// ---- histogram ---------------------------------------------------------------

__global__ void __launch_bounds__(256) histogram_kernel(const uint16_t *in, uint64_t n, uint64_t *hist)
{
    __shared__ uint32_t h[256];
    h[threadIdx.x] = 0;
    __syncthreads();
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x * 8;
    const uint64_t n8 = n & ~7ull;
    for (uint64_t i = ((uint64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8; i < n8; i += stride) {
        const uint4 v = *reinterpret_cast<const uint4 *>(in + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            atomicAdd(&h[(w[k] >> 7) & 0xFFu], 1u);
            atomicAdd(&h[(w[k] >> 23) & 0xFFu], 1u);
        }
    }
    if (blockIdx.x == 0)
        for (uint64_t i = n8 + threadIdx.x; i < n; i += blockDim.x)
            atomicAdd(&h[(in[i] >> 7) & 0xFFu], 1u);
    __syncthreads();
    if (h[threadIdx.x])
        atomicAdd(reinterpret_cast<unsigned long long *>(&hist[threadIdx.x]),
                  (unsigned long long)h[threadIdx.x]);
}

// ---- encode: per-thread code lengths -----------------------------------------

// Loads this thread's up to 32 elements, two to a word, element 2i in the
// low half of w[i] (zero past n).
__device__ __forceinline__ void load_words(const EncodeParams &p, uint64_t e0, uint32_t (&w)[16])
{
    if (e0 + kElemsPerThread <= p.n) {
        const uint4 *src = reinterpret_cast<const uint4 *>(p.in + e0);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 v = src[q];
            w[4 * q] = v.x;
            w[4 * q + 1] = v.y;
            w[4 * q + 2] = v.z;
            w[4 * q + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const uint64_t i = e0 + 2 * k;
            const uint32_t a = i < p.n ? p.in[i] : 0u;
            const uint32_t b = i + 1 < p.n ? p.in[i + 1] : 0u;
            w[k] = a | (b << 16);
        }
    }
}

// Bits of this thread's elements, counted here (when the bit-count pass kept
// no group counts, or in the last segment); *bad is set when an element's
// exponent has no code.
__device__ __forceinline__ uint32_t count_bits(const EncodeParams &p, const uint2 *code_tab, uint64_t e0,
                                               const uint32_t (&w)[16], bool &bad)
{
    uint32_t bits = 0;
#pragma unroll
    for (int k = 0; k < kElemsPerThread; ++k) {
        if (e0 + k < p.n) {
            const uint32_t x = (w[k >> 1] >> (16 * (k & 1))) & 0xFFFFu;
            const uint32_t l = code_tab[(x >> 7) & 0xFFu].y;
            bad |= l == 0;
            bits += l;
        }
    }
    return bits;
}

// Block-wide exclusive scan of one value per thread (256 threads).
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t *warp_tot, uint32_t &total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d)
            incl += y;
    }
    if (lane == 31)
        warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const uint32_t t = lane < kEncThreads / 32 ? warp_tot[lane] : 0u;
        uint32_t ti = t;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, ti, d);
            if (lane >= d)
                ti += y;
        }
        if (lane < kEncThreads / 32)
            warp_tot[lane] = ti - t;
        if (lane == 31)
            warp_tot[kEncThreads / 32] = ti;
    }
    __syncthreads();
    total = warp_tot[kEncThreads / 32];
    return warp_tot[warp] + incl - v;
}

// Bits of every segment: one warp per segment, whose lanes read it 512
// contiguous bytes at a time (lane l takes bytes [16 l, 16 l + 16) of each),
// then a warp sum, also added to the total of the segment's run of
// kRunSegs segments.  Built for 8 resident CTAs per SM (32 registers, no
// spills), so the launch's 8 CTAs per SM all start at once: at 40 registers
// only 6 fit and the last quarter of the CTAs ran as a second wave.
__global__ void __launch_bounds__(256, 8) segment_bits_kernel(EncodeParams p)
{
    __shared__ uint32_t len_tab[256];
    len_tab[threadIdx.x] = p.code_table[threadIdx.x] >> 24;
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const uint64_t warps = (uint64_t)gridDim.x * (blockDim.x >> 5);
    bool bad = false;
    for (uint64_t seg = (uint64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); seg < p.n_seg;
         seg += warps) {
        const uint64_t s0 = seg * kSegElems;
        uint32_t bits = 0;
        if (s0 + kSegElems <= p.n) {
            const uint4 *src = reinterpret_cast<const uint4 *>(p.in + s0) + lane;
#pragma unroll 8
            for (int q = 0; q < kSegElems / 32 / 8; ++q) {
                const uint4 v = src[32 * q];
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
                uint32_t part = 0;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t a = len_tab[(w4[k] >> 7) & 0xFFu];
                    const uint32_t b = len_tab[(w4[k] >> 23) & 0xFFu];
                    bad |= (a == 0) | (b == 0);
                    part += a + b;
                }
                bits += part;
                if (p.grp_bits) {
                    // lanes 4m .. 4m + 3 hold the 32 elements of group 8q + m
                    part += __shfl_xor_sync(0xFFFFFFFFu, part, 1);
                    part += __shfl_xor_sync(0xFFFFFFFFu, part, 2);
                    if ((lane & 3) == 0)
                        p.grp_bits[seg * (kSegElems / kElemsPerThread) + 8 * q + (lane >> 2)] = (uint16_t)part;
                }
            }
        } else {
            for (uint64_t i = s0 + lane; i < s0 + kSegElems && i < p.n; i += 32) {
                const uint32_t l = len_tab[(p.in[i] >> 7) & 0xFFu];
                bad |= l == 0;
                bits += l;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            bits += __shfl_xor_sync(0xFFFFFFFFu, bits, o);
        if (lane == 0) {
            p.seg_bits[seg] = bits;
            atomicAdd(reinterpret_cast<unsigned long long *>(p.run_bits + seg / kRunSegs),
                      (unsigned long long)bits);
        }
    }
    if (bad && p.err)
        atomicOr(p.err, DF11_DEVERR_MISMATCH);
}

// Zeroes the stream, gaps, counts, run totals and sign|mantissa tail; fills
// chunk positions with n; copies the code table into global memory (read
// there with per-thread indices, which a kernel parameter would serialise).
__global__ void prepare_kernel(EncodeParams p, CodeTable ct, uint64_t stream_words, uint64_t gap_words,
                               uint64_t n_chunks, uint64_t sm_bytes)
{
    const uint64_t tid = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (tid < 256)
        p.code_table[tid] = ct.e[tid];
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    uint4 *s128 = reinterpret_cast<uint4 *>(p.stream);
    for (uint64_t i = tid; i < stream_words / 4; i += stride)
        s128[i] = make_uint4(0u, 0u, 0u, 0u);
    uint32_t *s32 = reinterpret_cast<uint32_t *>(p.stream);
    for (uint64_t i = stream_words / 4 * 4 + tid; i < stream_words; i += stride)
        s32[i] = 0;
    uint32_t *g32 = reinterpret_cast<uint32_t *>(p.gaps);
    for (uint64_t i = tid; i < gap_words; i += stride)
        g32[i] = 0;
    uint32_t *c32 = reinterpret_cast<uint32_t *>(p.counts);
    for (uint64_t i = tid; i < p.n_threads / 4; i += stride)
        c32[i] = 0;
    for (uint64_t i = tid; i <= n_chunks; i += stride)
        p.chunk_pos[i] = (uint32_t)p.n;
    for (uint64_t i = p.n + tid; i < sm_bytes; i += stride)
        p.signmant[i] = 0;
    for (uint64_t i = tid; i < (p.n_seg + kRunSegs - 1) / kRunSegs; i += stride)
        p.run_bits[i] = 0;
}

// Shared staging of one segment's output: stream words in bit order (bit 31
// = first bit), and one word per slice that a code of the segment opens:
// the opening element's index in the segment | gap << 16 | kOpened.
constexpr int kStageWords = kSegElems * 16 / 32 + 4;            // 16-bit codes at most
constexpr int kSliceStage = (kSegElems * 16 / 64 / 8 + 2) * 8;  // 64-bit slices at the finest
constexpr uint32_t kOpened = 0x80000000u;

// Bits of one segment's encode, per thread: the codes of its elements are
// appended to a right-aligned bit accumulator (hi:lo, nb bits) that starts
// with the thread's offset into its first stream word as zero bits, so each
// 32 bits it completes are one whole stream word.
struct BitSink {
    uint32_t lo, hi, nb;
    uint32_t sp;   // shared address of the next stream word
    __device__ __forceinline__ void put(uint32_t c, uint32_t l)   // l <= 32, nb < 32
    {
        asm volatile(
            "{\n\t"
            ".reg .pred p;\n\t"
            ".reg .b32 t, s;\n\t"
            "shf.l.clamp.b32 %1, %0, %1, %4;\n\t"   // hi:lo <<= l
            "shl.b32 t, %0, %4;\n\t"
            "or.b32 %0, t, %5;\n\t"
            "add.u32 %2, %2, %4;\n\t"
            "setp.ge.u32 p, %2, 32;\n\t"
            "sub.u32 s, %2, 32;\n\t"
            "shf.r.clamp.b32 t, %0, %1, s;\n\t"     // the completed word: bits [nb - 32, nb)
            "@p st.shared.u32 [%3], t;\n\t"
            "@p add.u32 %3, %3, 4;\n\t"
            "@p mov.u32 %2, s;\n\t"
            "}"
            : "+r"(lo), "+r"(hi), "+r"(nb), "+r"(sp)
            : "r"(l), "r"(c)
            : "memory");
    }
};

// One segment of 8192 elements per CTA, 32 per thread.  Every thread knows
// its first bit (the segment's start, from the run totals and the segment
// counts before it, plus a CTA scan of the kept group counts) and encodes its
// codes MSB-first.  A completed stream word is stored by the thread that
// completes it (its first bits may be the previous thread's: zeros here);
// after a barrier each thread ORs its part-filled last word into the word
// the next thread completed.  A slice that one of the thread's codes opens
// gets its gap, and a chunk that starts there its output position (rare: a
// branch, tested once per four codes); the codes of each slice are counted
// into its staged byte.  Then the staged words go to global memory.
__global__ void __launch_bounds__(kEncThreads, 4) encode_kernel(EncodeParams p)
{
    __shared__ uint2 code_tab[256];   // code (right-aligned), length; length 0 = absent
    __shared__ uint32_t warp_tot[kEncThreads / 32 + 1];
    __shared__ unsigned long long seg_first;
    __shared__ uint32_t last_elem[kEncThreads / 32];   // each warp's last element
    __shared__ __align__(16) uint32_t sw[kStageWords];
    __shared__ __align__(16) uint32_t so[kSliceStage];
    const uint32_t tid = threadIdx.x;
    const uint64_t seg = blockIdx.x;
    const bool tail = (seg + 1) * kSegElems > p.n;
    // Global loads first, all independent: this thread's elements (and its
    // group's kept bit count), and in warp 0 the run totals and segment
    // counts before this segment in its run, spread over the 32 lanes.
    const uint64_t e0 = seg * kSegElems + (uint64_t)tid * kElemsPerThread;
    uint32_t w[16];
    const bool counted = p.grp_bits != nullptr && !tail;
    const uint32_t counted_bits = counted ? p.grp_bits[e0 / kElemsPerThread] : 0u;
    load_words(p, e0, w);
    unsigned long long acc = 0;
    if (tid < 32) {
        const uint64_t run = seg / kRunSegs;
        const uint64_t first = run * kRunSegs;
        uint32_t sb[kRunSegs / 32];
#pragma unroll
        for (int i = 0; i < kRunSegs / 32; ++i) {
            const uint64_t j = first + (uint64_t)(32 * i) + tid;
            sb[i] = j < seg ? p.seg_bits[j] : 0u;
        }
        for (uint64_t r = tid; r < run; r += 32)
            acc += p.run_bits[r];
#pragma unroll
        for (int i = 0; i < kRunSegs / 32; ++i)
            acc += sb[i];
    }
    // the element before this thread's first: the previous thread's last
    // (thread 0: loaded)
    uint32_t prev = __shfl_up_sync(0xFFFFFFFFu, w[15] >> 16, 1);
    if ((tid & 31) == 0)
        prev = tid == 0 ? (e0 > 0 ? (uint32_t)p.in[e0 - 1] : 0u) : 0xFFFFFFFFu;
    {
        const uint32_t e = p.code_table[tid];
        code_tab[tid] = make_uint2(e & 0xFFFFFFu, e >> 24);
    }
    static_assert(kSliceStage % 4 == 0 && kStageWords % 4 == 0, "vector zeroing");
    for (uint32_t i = tid; i < kSliceStage / 4; i += kEncThreads)
        reinterpret_cast<uint4 *>(so)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (tail)   // words nobody completes in the last segment
        for (uint32_t i = tid; i < kStageWords / 4; i += kEncThreads)
            reinterpret_cast<uint4 *>(sw)[i] = make_uint4(0u, 0u, 0u, 0u);
    if ((tid & 31) == 31)
        last_elem[tid >> 5] = w[15] >> 16;
    if (tid < 32) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
        if (tid == 0)
            seg_first = acc;
    }
    __syncthreads();
    if (prev == 0xFFFFFFFFu)
        prev = last_elem[(tid >> 5) - 1];

    bool bad = false;
    uint32_t bits = counted_bits;
    if (!counted)
        bits = count_bits(p, code_tab, e0, w, bad);
    uint32_t seg_total;
    const uint32_t off = block_exclusive_scan(bits, warp_tot, seg_total);
    const uint64_t S = seg_first;                         // first bit of the segment
    const uint64_t wbase = S >> 5;                        // stream word of sw[0]
    const uint32_t sh = p.slice_shift;
    const uint64_t gS = S >> sh;                          // slice of the segment's first bit
    const uint64_t gbase = gS >> 3;                       // gap word of staged slice 0
    // Positions below are local: lb = bit - (gS << sh), so the slice of a
    // local bit is gS + (lb >> sh) and its staged byte (lb >> sh) + (gS & 7).
    const uint32_t lb0 = (uint32_t)(S - (gS << sh));
    const uint32_t sw_a = (uint32_t)__cvta_generic_to_shared(sw);

    BitSink out;
    out.lo = out.hi = 0;
    out.nb = (uint32_t)((S + off) & 31);
    out.sp = sw_a + 4u * (uint32_t)(((S + off) >> 5) - wbase);
    uint32_t cnt = 0;
    if (e0 < p.n) {
        uint32_t lb = lb0 + off;                          // local bit of the next code
        // First local bit of the slice after the one holding the previous
        // code start (0 for element 0, or when that start lies before the
        // segment's first slice): a code starting at or past it opens a slice.
        uint32_t next_open = 0;
        if (e0 > 0) {
            const uint32_t lp = code_tab[(prev >> 7) & 0xFFu].y;
            if (lb >= lp)
                next_open = (((lb - lp) >> sh) + 1) << sh;
        }
        const uint32_t goff = (uint32_t)(gS & 7u);
        const uint32_t so_a = (uint32_t)__cvta_generic_to_shared(so) + 4u * goff;
        const uint32_t k0 = tid * kElemsPerThread;         // first element, in the segment
        cnt = (uint32_t)min((uint64_t)kElemsPerThread, p.n - e0);
        // The code of element k, starting at local bit s, opens a slice (its
        // gap s - slice start is below 16, so s & 15).
        auto open = [&](uint32_t k, uint32_t s) {
            const uint32_t gl = s >> sh;
            asm volatile("st.shared.u32 [%0], %1;" ::"r"(so_a + 4u * gl), "r"((k0 + k) | (s & 15u) << 16 | kOpened)
                         : "memory");
            next_open = (gl + 1) << sh;
        };
        if (cnt == kElemsPerThread) {
            // Four codes at a time.  At most one of them opens a slice: an
            // opening code starts within 15 bits of its slice's start, and
            // the next three start within 48 bits after it, short of the
            // next slice (at least 64 bits on).
#pragma unroll
            for (uint32_t q = 0; q < kElemsPerThread / 4; ++q) {
                const uint32_t x0 = w[2 * q], x1 = w[2 * q + 1];
                const uint2 c0 = code_tab[(x0 >> 7) & 0xFFu];
                const uint2 c1 = code_tab[(x0 >> 23) & 0xFFu];
                const uint2 c2 = code_tab[(x1 >> 7) & 0xFFu];
                const uint2 c3 = code_tab[(x1 >> 23) & 0xFFu];
                const uint32_t l01 = c0.y + c1.y;
                const uint32_t l012 = l01 + c2.y;
                if (lb + l012 >= next_open) {
                    const uint32_t k = lb >= next_open ? 0u : lb + c0.y >= next_open ? 1u
                                                          : lb + l01 >= next_open ? 2u : 3u;
                    const uint32_t s = lb + (k == 0 ? 0u : k == 1 ? c0.y : k == 2 ? l01 : l012);
                    open(4 * q + k, s);
                }
                lb += l012 + c3.y;
                out.put((c0.x << c1.y) | c1.x, l01);
                out.put((c2.x << c3.y) | c3.x, c2.y + c3.y);
            }
        } else {
#pragma unroll
            for (uint32_t k = 0; k < kElemsPerThread; ++k) {
                if (k >= cnt)
                    break;
                const uint2 c = code_tab[(w[k >> 1] >> (16 * (k & 1) + 7)) & 0xFFu];
                if (lb >= next_open)
                    open(k, lb);
                lb += c.y;
                out.put(c.x, c.y);
            }
        }
        // the end of the stream counts as a code start for the gap of its slice
        if (e0 + cnt == p.n && gS + (uint64_t)(lb >> sh) < p.n_threads && lb >= next_open)
            open(cnt, lb);
        // sign|mantissa bytes
        if (cnt == kElemsPerThread) {
            uint32_t sm[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint32_t a = w[2 * q], b = w[2 * q + 1];
                // element bytes: (x >> 8) & 0x80 | x & 0x7F for 4 elements
                const uint32_t lo = __byte_perm(a, b, 0x6420);   // low bytes of the 4 elements
                const uint32_t hi = __byte_perm(a, b, 0x7531);   // high bytes
                sm[q] = (lo & 0x7F7F7F7Fu) | (hi & 0x80808080u);
            }
            uint4 *dst = reinterpret_cast<uint4 *>(p.signmant + e0);
            dst[0] = make_uint4(sm[0], sm[1], sm[2], sm[3]);
            dst[1] = make_uint4(sm[4], sm[5], sm[6], sm[7]);
        } else {
#pragma unroll
            for (uint32_t k = 0; k < kElemsPerThread; ++k) {
                if (k < cnt) {
                    const uint32_t x = (w[k >> 1] >> (16 * (k & 1))) & 0xFFFFu;
                    p.signmant[e0 + k] = (uint8_t)(((x >> 8) & 0x80u) | (x & 0x7Fu));
                }
            }
        }
    }
    if (bad && p.err)
        atomicOr(p.err, DF11_DEVERR_MISMATCH);
    // The part-filled last word: the next thread of a full segment completes
    // it, so ORed after the barrier; the last thread's is the segment's own
    // last word, stored.  (The last segment's words start zeroed: its last
    // threads may complete none.)
    const uint32_t part = out.nb ? out.lo << (32u - out.nb) : 0u;
    if (out.nb && !tail && tid == kEncThreads - 1)
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(out.sp), "r"(part) : "memory");
    __syncthreads();
    if (out.nb && (tail || tid != kEncThreads - 1))
        asm volatile("red.shared.or.b32 [%0], %1;" ::"r"(out.sp), "r"(part) : "memory");
    __syncthreads();

    // ---- staged words -> global: words that may be shared with the
    // neighbouring segments (the first and the last) are ORed in
    const uint64_t end_bit = S + seg_total;
    if (seg == p.n_seg - 1 && tid == 0 && end_bit != p.total_bits && p.err)
        atomicOr(p.err, DF11_DEVERR_MISMATCH);
    if (seg_total) {
        const uint32_t nw = (uint32_t)(((end_bit + 31) >> 5) - wbase);
        uint32_t *g32 = reinterpret_cast<uint32_t *>(p.stream) + wbase;
        for (uint32_t i = tid; i < nw; i += kEncThreads) {
            const uint32_t v = bswap32(sw[i]);
            if (i == 0 || i == nw - 1)
                atomicOr(g32 + i, v);
            else
                g32[i] = v;
        }
    }
    // ---- slices: gaps, counts, chunk positions.  Staged slice gi is slice
    // gbase * 8 + gi.  This segment's bits lie in staged slices [goff,
    // gend), and its end bit in slice glend (gend - 1, or gend when the end
    // bit starts a slice).  Its codes starting in slice gi are a(gi + 1) -
    // a(gi), a(gi) = the element that opens slice gi if one of this
    // segment's does, else 0 for the first slice (opened before the segment)
    // and ne for slices past the segment's last code start (a(gend) = ne).
    // The previous segment's end bit lies in slice goff and the next one's
    // first bit in slice glend: words holding those two slices are ORed
    // (gaps) or added (counts) into the zeroed arrays, the others stored.
    {
        const uint32_t goff = (uint32_t)(gS & 7u);
        const uint32_t ne = (uint32_t)min((uint64_t)kSegElems, p.n - seg * kSegElems);
        const uint32_t glend = (uint32_t)((end_bit >> sh) - gS) + goff;
        const uint32_t gend = seg_total ? (uint32_t)(((end_bit - 1) >> sh) - gS) + 1 + goff : goff;
        auto a_of = [&](uint32_t gi) -> uint32_t {
            const uint32_t v = so[gi];
            return (v & kOpened) ? (v & 0xFFFFu) : gi == goff ? 0u : ne;
        };
        const uint64_t gwords = p.n_threads / 8;                  // gaps array length in words
        uint32_t *gg = reinterpret_cast<uint32_t *>(p.gaps) + gbase;
        for (uint32_t i = tid; i <= glend / 8 && gbase + i < gwords; i += kEncThreads) {
            // eight gap nibbles, slice 8i + k at bits 4k
            uint32_t v = 0;
#pragma unroll
            for (int k = 0; k < 8; ++k)
                v |= ((so[8 * i + k] >> 16) & 0xFu) << (4 * k);
            if (i == 0 || i == glend / 8)
                atomicOr(gg + i, v);
            else
                gg[i] = v;
        }
        // counts: slice 4i + k at byte k of word i (a count is at most 128,
        // so bytes never carry)
        uint32_t *cc = reinterpret_cast<uint32_t *>(p.counts) + 2 * gbase;
        const uint64_t cwords = p.n_threads / 4;
        for (uint32_t i = goff / 4 + tid; gend > goff && i <= (gend - 1) / 4 && 2 * gbase + i < cwords;
             i += kEncThreads) {
            uint32_t v = 0;
#pragma unroll
            for (uint32_t k = 0; k < 4; ++k) {
                const uint32_t gi = 4 * i + k;
                if (gi >= goff && gi < gend) {
                    const uint32_t a_next = gi + 1 < gend ? a_of(gi + 1) : ne;
                    v |= (a_next - a_of(gi)) << (8 * k);
                }
            }
            if (i == goff / 4 || i == glend / 4) {
                if (v)
                    atomicAdd(cc + i, v);
            } else {
                cc[i] = v;
            }
        }
        // output position of every chunk whose first slice a code of this
        // segment (or the end of the stream) opens
        const uint32_t c0 = (uint32_t)((gbase * 8 + 31) / 32 * 32 - gbase * 8);   // first staged chunk start
        for (uint32_t gi = c0 + 32 * tid; gi <= glend; gi += 32 * kEncThreads) {
            const uint32_t v = so[gi];
            if (v & kOpened)
                p.chunk_pos[(gbase * 8 + gi) / DF11_THREADS_PER_CHUNK] = (uint32_t)(seg * kSegElems + (v & 0xFFFFu));
        }
    }
}

bool aligned(const void *ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

uint64_t n_segments(uint64_t n) { return (n + kSegElems - 1) / kSegElems; }

// Scratch: code table (1 KB) | segment bits (4 bytes per segment, rounded to 16) | run totals
// (8 bytes per run of kRunSegs segments, rounded to 16) | group bits (2 bytes
// per 32 elements of every segment).  The allocation-free path goes without
// the group bits.
constexpr uint64_t kTableBytes = 256 * 4;
uint64_t run_bits_offset(uint64_t n) { return kTableBytes + ((n_segments(n) * 4 + 15) & ~15ull); }

uint64_t segment_scratch_bytes(uint64_t n)
{
    const uint64_t runs = (n_segments(n) + kRunSegs - 1) / kRunSegs;
    return run_bits_offset(n) + ((runs * 8 + 15) & ~15ull);
}

df11_status compress_device_impl(const df11_codebook *cb, const df11_layout *layout, const uint16_t *d_in,
                                 uint64_t n, df11_device_block *out, void *d_scratch, uint64_t scratch_bytes,
                                 bool group_bits, uint32_t *d_error, void *stream);

}  // namespace

extern "C" {

df11_status df11_histogram_device(const uint16_t *d_in, uint64_t n, uint64_t *d_hist, void *stream)
{
    if (!d_in || !d_hist || n == 0 || !aligned(d_in, 16) || !aligned(d_hist, 8))
        return DF11_ERR_INVALID_ARGUMENT;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return DF11_ERR_CUDA;
    const uint64_t want = (n + 256 * 8 - 1) / (256 * 8);
    const uint64_t cap = (uint64_t)sms * 8;
    const unsigned grid = (unsigned)(want < cap ? (want ? want : 1) : cap);
    histogram_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(d_in, n, d_hist);
    return cudaGetLastError() == cudaSuccess ? DF11_OK : DF11_ERR_CUDA;
}

uint64_t df11_compress_device_scratch_bytes(uint64_t n_elements)
{
    return segment_scratch_bytes(n_elements) + n_segments(n_elements) * (kSegElems / kElemsPerThread) * 2;
}

df11_status df11_compress_device(const df11_codebook *cb, const df11_layout *layout,
                                 const uint16_t *d_in, uint64_t n, df11_device_block *out,
                                 void *d_scratch, uint64_t scratch_bytes, uint32_t *d_error,
                                 void *stream)
{
    return compress_device_impl(cb, layout, d_in, n, out, d_scratch, scratch_bytes, true, d_error, stream);
}

}  // extern "C"

namespace {

df11_status compress_device_impl(const df11_codebook *cb, const df11_layout *layout, const uint16_t *d_in,
                                 uint64_t n, df11_device_block *out, void *d_scratch, uint64_t scratch_bytes,
                                 bool group_bits, uint32_t *d_error, void *stream)
{
    if (!cb || !layout || !d_in || !out || !d_scratch)
        return DF11_ERR_INVALID_ARGUMENT;
    if (n == 0 || n != cb->n_elements)
        return DF11_ERR_INVALID_ARGUMENT;
    if (n >= (1ull << 32))
        return DF11_ERR_OVERFLOW;
    df11_sizes z;
    df11_status st = df11_compress_sizes(cb, layout, &z);
    if (st != DF11_OK)
        return st;
    if (scratch_bytes < (group_bits ? df11_compress_device_scratch_bytes(n) : segment_scratch_bytes(n)))
        return DF11_ERR_BUFFER_TOO_SMALL;
    if (!out->exp_stream || !out->gaps || !out->counts || !out->chunk_pos || !out->signmant)
        return DF11_ERR_INVALID_ARGUMENT;
    if (out->exp_stream_bytes < z.exp_stream_bytes || out->gaps_bytes < z.gaps_bytes ||
        out->counts_bytes < z.counts_bytes || out->chunk_pos_count < z.chunk_pos_count ||
        out->signmant_bytes < z.signmant_bytes)
        return DF11_ERR_BUFFER_TOO_SMALL;
    if (!aligned(d_in, 16) || !aligned(out->exp_stream, 16) || !aligned(out->gaps, 16) ||
        !aligned(out->counts, 16) ||
        !aligned(out->chunk_pos, 16) || !aligned(out->signmant, 16) || !aligned(d_scratch, 16) ||
        !aligned(d_error, 4))
        return DF11_ERR_INVALID_ARGUMENT;

    EncodeParams p;
    p.in = d_in;
    // the arrays are written through the const-qualified device view
    p.stream = const_cast<uint8_t *>(out->exp_stream);
    p.gaps = const_cast<uint8_t *>(out->gaps);
    p.counts = const_cast<uint8_t *>(out->counts);
    p.chunk_pos = const_cast<uint32_t *>(out->chunk_pos);
    p.signmant = const_cast<uint8_t *>(out->signmant);
    p.n_seg = n_segments(n);
    p.code_table = reinterpret_cast<uint32_t *>(d_scratch);
    p.seg_bits = reinterpret_cast<uint32_t *>(reinterpret_cast<uint8_t *>(d_scratch) + kTableBytes);
    p.run_bits = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(d_scratch) + run_bits_offset(n));
    p.grp_bits = group_bits ? reinterpret_cast<uint16_t *>(reinterpret_cast<uint8_t *>(d_scratch) +
                                                           segment_scratch_bytes(n))
                            : nullptr;
    p.err = d_error;
    p.n = n;
    p.total_bits = cb->total_bits;
    p.n_threads = z.n_threads;
    p.slice_shift = layout->bytes_per_thread == 16 ? 7u : 6u;
    p.threads_per_chunk = layout->threads_per_chunk;
    CodeTable ct;
    for (int s = 0; s < 256; ++s)
        ct.e[s] = cb->code_len[s] ? (cb->code[s] | ((uint32_t)cb->code_len[s] << 24)) : 0u;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return DF11_ERR_CUDA;
    prepare_kernel<<<sms * 8, 256, 0, s>>>(p, ct, z.exp_stream_bytes / 4, (z.gaps_bytes + 3) / 4,
                                                z.n_chunks, z.signmant_bytes);
    segment_bits_kernel<<<(unsigned)((p.n_seg + 7) / 8 < (uint64_t)sms * 8 ? (p.n_seg + 7) / 8 : (uint64_t)sms * 8),
                          256, 0, s>>>(p);
    encode_kernel<<<(unsigned)p.n_seg, kEncThreads, 0, s>>>(p);
    if (cudaGetLastError() != cudaSuccess)
        return DF11_ERR_CUDA;
    out->hdr.max_code_len = cb->max_code_len;
    out->hdr.threads_per_chunk = layout->threads_per_chunk;
    out->hdr.bytes_per_thread = layout->bytes_per_thread;
    out->hdr.n_tables = cb->n_tables;
    out->hdr.min_code_len = DF11_MAX_CODE_LEN;
    for (int k = 0; k < 256; ++k)
        if (cb->code_len[k] && cb->code_len[k] < out->hdr.min_code_len)
            out->hdr.min_code_len = cb->code_len[k];
    out->hdr.reserved = 0;
    out->hdr.total_bits = cb->total_bits;
    out->hdr.n_elements = n;
    out->hdr.n_chunks = z.n_chunks;
    return DF11_OK;
}

}  // namespace

// ---- allocation-free variant -------------------------------------------------
// Some callers cannot let a library allocate device memory: a serving runtime
// or framework that reserves the whole GPU for its own memory pool up front
// (cudaMalloc then fails, or bypasses the pool's accounting), or code that
// must not call cudaFree, which synchronises the device.  For them,
// df11_compress_device_noalloc takes its work space from the fixed array
// below instead of from the caller.

namespace {

constexpr uint64_t kNoAllocScratchBytes = DF11_NOALLOC_SCRATCH_BYTES;
constexpr int kNoAllocMaxDevices = 64;

// Segment bit counts and starts of the last call.  Every call writes all the
// entries it reads before reading them, so nothing needs clearing.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// The array's device address belongs to the module as loaded into one CUDA
// context: a context made after cudaDeviceReset, or another driver context
// on the same device, loads the module again at another address.  So the
// address is cached per device together with the identity of the context it
// was looked up in (the driver's context ID, reached through the runtime's
// entry-point query so the library needs no link to the driver library),
// and looked up again whenever the current context differs.
struct NoAllocSlot {
    unsigned long long ctx_id = 0;   // 0 = nothing cached
    uintptr_t addr = 0;
};
NoAllocSlot g_noalloc_slot[kNoAllocMaxDevices];
std::mutex g_noalloc_mutex;

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// ID of the context current on this thread, or 0 when it cannot be had.
unsigned long long current_context_id()
{
    static const auto fns = [] {
        std::pair<CtxGetCurrentFn, CtxGetIdFn> f{nullptr, nullptr};
        void *a = nullptr, *b = nullptr;
        cudaDriverEntryPointQueryResult qa, qb;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
            qa == cudaDriverEntryPointSuccess &&
            cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
            qb == cudaDriverEntryPointSuccess) {
            f.first = reinterpret_cast<CtxGetCurrentFn>(a);
            f.second = reinterpret_cast<CtxGetIdFn>(b);
        }
        return f;
    }();
    if (!fns.first || !fns.second)
        return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (fns.first(&ctx) != CUDA_SUCCESS || ctx == nullptr || fns.second(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

}  // namespace

extern "C" df11_status df11_compress_device_noalloc(const df11_codebook *cb,
                                                    const df11_layout *layout,
                                                    const uint16_t *d_in, uint64_t n,
                                                    df11_device_block *out, uint32_t *d_error,
                                                    void *stream)
{
    if (!cb || !layout || !d_in || !out)
        return DF11_ERR_INVALID_ARGUMENT;
    if (n > DF11_NOALLOC_MAX_ELEMENTS)
        return DF11_ERR_BUFFER_TOO_SMALL;       // the fixed work space is too small
    if (segment_scratch_bytes(n) > kNoAllocScratchBytes)
        return DF11_ERR_BUFFER_TOO_SMALL;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices)
        return DF11_ERR_CUDA;
    unsigned long long ctx = current_context_id();   // 0 before the runtime made one current
    uintptr_t addr = 0;
    {
        std::lock_guard<std::mutex> lock(g_noalloc_mutex);
        NoAllocSlot &slot = g_noalloc_slot[dev];
        if (ctx != 0 && slot.ctx_id == ctx) {
            addr = slot.addr;
        } else {
            // host code only knows a stand-in for the array: ask the runtime
            // for its address in the current context
            void *ptr = nullptr;
            if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
                return DF11_ERR_CUDA;
            addr = reinterpret_cast<uintptr_t>(ptr);
            slot.ctx_id = current_context_id();   // the lookup made a context current
            slot.addr = addr;
        }
    }
    return compress_device_impl(cb, layout, d_in, n, out, reinterpret_cast<void *>(addr), kNoAllocScratchBytes,
                                false, d_error, stream);
}
