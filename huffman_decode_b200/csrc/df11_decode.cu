// df11_decode.cu -- GPU decode of one DF11 block into BF16 (sm_100a).
//
// Method: "DFloat11: lossless BFloat16 compression" (ai-infrastructure.net),
// section "Architecture": each thread owns a fixed slice of the exponent
// stream and starts at its Gaps offset; a prefix sum of per-thread code
// counts places the outputs; exponents are joined with the raw sign|mantissa
// bytes and written with coalesced stores; one launch covers every matrix of
// a block (block-level batching).
//
// B200 design (differs from the page's kernel):
//   * one warp = one chunk: output positions are stored per 32 threads, so
//     every warp scans, decodes and stores on its own, with no block-wide
//     barrier after the prologue (the claimed schedule below adds one at
//     the very end, to count the CTA out);
//   * one decode pass instead of the page's two: the format stores each
//     thread's code count, so a warp scan of the stored counts (shuffles)
//     gives each lane its output offset before it decodes, and the lane
//     decodes its slice once, writing its exponents four per 32-bit word
//     straight into place in a contiguous, 8-element-aligned per-warp
//     exponent buffer.  Full chunks of 128-bit slices store plain words
//     (every lane's first word lands before any lane's third segment, and
//     each lane's part-filled last word is ORed over its neighbour's first
//     at the end); 64-bit slices and the block's last chunk OR into a zeroed
//     buffer.  A tail check confirms that each lane decoded exactly its
//     stored count and ended where the next code starts;
//   * up to four codes per lookup: an 11-bit window indexes a 2048-entry
//     table (built once on the host, or in shared memory from the format's
//     two-level 16-bit tables); longer codes fall back to the two-level
//     tables.  The lane state packs the bit position and the fill of the
//     word being built, so one add steps both;
//   * exponents travel rotated right by one bit (bit 0 on top), which is
//     where the BF16 halves want them: the merge is two bit-selects and two
//     byte permutes per four weights, with no shifts, and one 16-byte store
//     per lane and group;
//   * the chunk's sign|mantissa bytes are staged into shared memory by one
//     TMA bulk copy (cp.async.bulk + mbarrier) issued before decoding, and
//     the tables by bulk copies in the prologue; the next chunk's stream
//     words, counts and positions are loaded into registers a chunk ahead;
//   * per-warp buffers are sized by the codebook's shortest code (the kernel
//     rejects table entries shorter than it), so blocks whose codes are at
//     least 2 bits long fit twice as many warps per SM;
//   * persistent CTAs, grid = resident CTAs per SM x SM count: two CTAs of
//     23 warps per SM (a 40-register build, 46 warps) or one of up to 32,
//     whichever keeps more warps resident; a block smaller than one full CTA
//     per SM gets one CTA per SM of just enough warps;
//   * with a scheduling workspace, the last few rounds of chunks are not
//     dealt out but claimed one at a time from four global counters (each
//     warp claims a chunk ahead, so the atomic's latency hides behind a
//     decode): warps and SMs that ran slower take fewer of them and all
//     finish within about one chunk of each other.  Claiming only the tail
//     keeps the atomics off the memory system for most of the launch.  The
//     last CTA out resets the counters;
//   * optionally (the verifying build) every chunk's bytes are summed as
//     they are read and checked against a per-chunk list.
// Also here: decoding a chunk range alone (df11_decompress_range_async), the
// verifying decode (df11_decompress_verified_async), the fused matrix-vector
// products (df11_decode_gemv_async), the bounded-wait self-test, and the
// run-time bound checks of the checked build.
// No tensor cores: this is integer decode, bounded by HBM traffic and issue.
#include "df11.h"

#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

namespace {

constexpr uint32_t kLutPointer = 0x8000u;
constexpr int kWindowBits = 11;                    // multi-code table index width
constexpr int kMultiEntries = 1 << kWindowBits;
constexpr int kMaxCodesPerEntry = 4;
static_assert(kWindowBits == DF11_DECODE_TABLE_WINDOW_BITS && kMultiEntries == DF11_DECODE_TABLE_ENTRIES,
              "the host-built decode table has the kernel's shape");
constexpr int kEntryBytes = 8;                     // multi-code entry: symbols | step
constexpr uint32_t kLongStep = 0x4000u;            // step of an entry whose first code is long
constexpr int kMaxWarpsPerCta = 32;
// A checked build (-DDF11_CHECKED, libdf11_checked.so) verifies at run time
// the invariants that keep every access in bounds, ORs DF11_DEVERR_BOUNDS
// and skips the access when one fails.  The normal build compiles the checks
// away.
#ifdef DF11_CHECKED
#define DF11_CHECK(err, cond) ((cond) ? true : ((err) |= DF11_DEVERR_BOUNDS, false))
#else
#define DF11_CHECK(err, cond) true
#endif
constexpr uint32_t kWaitLimit = 1u << 22;          // bounded mbarrier polls
constexpr uint32_t kWaitHintNs = 2000;              // longest suspension of one poll (so <= 8.4 s in all)

struct DecodeParams {
    const uint8_t *stream;
    const uint8_t *gaps;
    const uint8_t *counts;
    const uint32_t *chunk_pos;
    const uint8_t *signmant;
    const uint16_t *lut;
    uint16_t *out;
    uint32_t *err;
    uint64_t total_bits;
    uint64_t n_chunks;
    uint64_t out_limit;   // min(n_elements, out_capacity)
    uint32_t n_tables;
    uint32_t min_len;     // shortest legal code; shorter table entries are corrupt
    uint32_t full_chunks; // chunks lying wholly below total_bits (every slice full)
    uint64_t gaps_limit;  // gap bytes readable from `gaps` (the next thread's gap after the last chunk)
    uint32_t *sched;      // scheduling workspace, zero between launches; or null
    const uint2 *multi_src;   // the multi-code table built on the host, or null
    const uint32_t *sums;     // verifying decode: the expected per-chunk sums
    uint64_t *first_bad;      // verifying decode: lowest chunk found bad, or null
};
// Scheduling workspace: claim counter q at word q * kSchedStride (pools on
// separate 256-byte stretches, so on different L2 lines), CTAs done at word
// kSchedDoneWord.
constexpr int kSchedPools = 4;
constexpr int kSchedStride = 64;
constexpr int kSchedDoneWord = kSchedPools * kSchedStride;
constexpr int kSchedTailRounds = 3;   // rounds of chunks left to claiming
static_assert((kSchedDoneWord + 1) * 4 <= DF11_SCHED_WORKSPACE_BYTES, "workspace too small");

// Decode fused with a matrix-vector product: every matrix of the block is
// multiplied by n_tokens activation rows as it is decoded, and the BF16
// weights never reach HBM.
constexpr int kGemvMaxMats = 128;

struct GemvMat {
    uint32_t start;    // first element of the matrix in the block
    uint32_t cols;     // row length, a multiple of 8
    uint32_t rows;
    uint32_t pad;
    const uint16_t *x; // n_tokens x cols BF16, token-major
    float *y;          // n_tokens x rows FP32, accumulated into
};

struct GemvParams {
    uint32_t n_mats;
    uint32_t n_tokens;
    GemvMat m[kGemvMaxMats];
};

// Per-warp buffers for W stream bytes per lane and codes of at least MINLEN
// bits: the contiguous exponent buffer and the staged sign|mantissa bytes.
// A lane writes its codes to the exponent buffer at its output offset head
// (< 8) + off, off + count <= 32 kMaxCodes.  A corrupt stream can make the
// lane's main loop write up to kMaxCodes + 1 codes whatever its count (every
// code that starts below end - 10 + 11), so the buffer has that much slack.
template <int W, int MINLEN>
struct Geometry {
    static constexpr int kSliceBits = 8 * W;                         // 64 or 128
    static constexpr int kMaxCodes = (kSliceBits + MINLEN - 1) / MINLEN;  // per lane
    static constexpr int kEbufBytes = 33 * kMaxCodes + 16;           // multiple of 16
    static constexpr int kSbufBytes = 32 * kMaxCodes + 32;           // 16-aligned copy range
    static constexpr int kWarpBytes = kEbufBytes + kSbufBytes;
    static constexpr int kWords = W / 4 + 1;                         // stream words incl. halo
    static_assert(kWarpBytes % 16 == 0, "per-warp area must keep 16-byte alignment");
    static_assert(kMaxCodes % 16 == 0, "buffer sizes keep 16-byte alignment");
    static_assert(7 + (32 * kMaxCodes - 1) + (kMaxCodes + 1) + 3 <= kEbufBytes, "exponent buffer too small");
};

// Shared memory: mbarriers | multi-code table | code lengths | per-warp areas
// | two-level tables.
// one mbarrier per warp, and one for the prologue's table copies
constexpr size_t kBarBytes = ((kMaxWarpsPerCta + 1) * 8 + 15) / 16 * 16;
constexpr size_t kHeadBytes = kBarBytes + kMultiEntries * kEntryBytes + 256;
// per-warp areas and the tables after them keep 16-byte alignment (TMA
// destinations, 8- and 16-byte shared accesses)
static_assert(kHeadBytes % 16 == 0, "shared-memory head must keep 16-byte alignment");

template <int W, int MINLEN>
constexpr size_t smem_bytes_for(int warps, uint32_t n_tables)
{
    return kHeadBytes + (size_t)warps * Geometry<W, MINLEN>::kWarpBytes + (size_t)n_tables * 512;
}

__device__ __forceinline__ uint32_t bswap32(uint32_t x) { return __byte_perm(x, 0, 0x0123); }

// A compile-time int that converts like a runtime one (lets one code path be
// instantiated with a constant slice end).
template <int V>
struct ConstInt {
    __device__ constexpr operator int() const { return V; }
};

// Exponent byte rotated right by one bit: bit 0 moves to bit 7.
__host__ __device__ __forceinline__ uint32_t rot_exp(uint32_t e) { return (e >> 1) | ((e & 1u) << 7); }

// Four BF16 values from four rotated exponent bytes (r) and four
// sign|mantissa bytes (s), element k in byte k.  BF16 = sign (bit 15) |
// exponent (14..7) | mantissa (6..0), so its low byte is (exponent bit 0) << 7
// | mantissa and its high byte is sign << 7 | exponent >> 1: each is one
// bit-select of r and s under the mask 0x80, then the halves interleave.
__device__ __forceinline__ uint2 join4(uint32_t r, uint32_t s)
{
    uint32_t lo, hi;
    // lo = r where mask 0x80808080, else s
    asm("lop3.b32 %0, %1, %2, %3, 0xE4;" : "=r"(lo) : "r"(r), "r"(s), "r"(0x80808080u));
    // hi = s where mask 0x80808080, else r
    asm("lop3.b32 %0, %1, %2, %3, 0xE4;" : "=r"(hi) : "r"(s), "r"(r), "r"(0x80808080u));
    return make_uint2(__byte_perm(lo, hi, 0x5140), __byte_perm(lo, hi, 0x7362));
}

__device__ __forceinline__ uint16_t join1(uint32_t r, uint32_t s)
{
    return (uint16_t)((((s & 0x80u) | (r & 0x7Fu)) << 8) | (r & 0x80u) | (s & 0x7Fu));
}

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

// One item of a chunk's integrity sum (the definition is in df11.h):
// mix(v, tag) with tag_mul = tag * 0x9E3779B1 precomputed.
__device__ __forceinline__ uint32_t chunk_mix(uint32_t v, uint32_t tag_mul)
{
    const uint32_t y = (v ^ tag_mul) * 0x85EBCA6Bu;
    return y ^ (y >> 16);
}
constexpr uint32_t kTagMul = 0x9E3779B1u;

// ---- 32-bit shared-window accesses -----------------------------------------
// The hot loops address shared memory with 32-bit shared-window offsets.
// Table reads (read-only after the prologue) may be scheduled freely; reads
// of data written during a chunk are ordered with "memory".

__device__ __forceinline__ uint32_t lds_u16(uint32_t a)
{
    unsigned short v;
    asm("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds_u8(uint32_t a)
{
    uint32_t v;
    asm("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint2 lds_v2(uint32_t a)
{
    uint2 v;
    asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds_u8_m(uint32_t a)
{
    uint32_t v;
    asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ void red_or_u32(uint32_t a, uint32_t v)
{
    asm volatile("red.shared.or.b32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ void sts_u32(uint32_t a, uint32_t v)
{
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}

static_assert(kEntryBytes == 8, "lookup_step scales the table index by 8");

// Lane decode state X: bit position in bits 0..13; kLongStep (bit 14) is
// added by an entry whose first code is longer than the window (it ends the
// lookup loop); fill of the word being filled (in bits, 0..24 between
// lookups) in bits 26..31, so a full word (fill >= 32) is X >= 2^31.  A table
// entry's step y = total length | 8 x count << 26 advances both fields with
// one add.
constexpr int kFillShift = 26;
constexpr uint32_t kFillOne = 1u << kFillShift;   // X units of one fill bit
constexpr uint32_t kWordFull = 32u * kFillOne;    // fill >= 32
constexpr uint32_t kPosMask = 0xFFFFu;            // bit position and the long marker

// y of a table entry holding n codes of total length t
__host__ __device__ constexpr uint32_t entry_step(uint32_t t, uint32_t n) { return t | (8u * n << kFillShift); }
// codes of a table entry's y
__device__ __forceinline__ uint32_t entry_codes(uint32_t y) { return y >> (kFillShift + 3); }

// One multi-code lookup for window `win` (the upcoming stream bits, first
// lowest): appends the entry's symbols to the word being filled at the
// fill, steps X, computes the next window from the stream words lo:hi, and
// when the word is full stores it to the exponent buffer (OR: ORs it into a
// zeroed buffer) and starts the next word with the symbols past it.  One
// predicated block, so the store is not a branch; the next window is formed
// before the store so it waits only on the step.
template <bool OR>
__device__ __forceinline__ void lookup_step(uint32_t &X, uint32_t &win, uint32_t &accl, uint32_t &sp,
                                            uint2 &r, uint32_t lo, uint32_t hi, uint32_t multi_a)
{
    if constexpr (OR)
        asm volatile(
            "{\n\t"
            ".reg .b32 a, f, t;\n\t"
            ".reg .pred p;\n\t"
            "and.b32 a, %1, %9;\n\t"
            "mad.lo.u32 a, a, 8, %8;\n\t"
            "ld.shared.v2.u32 {%4, %5}, [a];\n\t"
            "shr.b32 f, %0, 26;\n\t"
            "shf.l.wrap.b32 t, %10, %4, f;\n\t"
            "or.b32 %2, %2, t;\n\t"
            "add.u32 %0, %0, %5;\n\t"
            "shf.r.wrap.b32 %1, %6, %7, %0;\n\t"
            "setp.ge.u32 p, %0, %11;\n\t"
            "@p red.shared.or.b32 [%3], %2;\n\t"
            "@p shf.l.wrap.b32 %2, %4, %10, f;\n\t"
            "@p add.u32 %3, %3, 4;\n\t"
            "@p sub.u32 %0, %0, %11;\n\t"
            "}"
            : "+r"(X), "+r"(win), "+r"(accl), "+r"(sp), "=r"(r.x), "=r"(r.y)
            : "r"(lo), "r"(hi), "r"(multi_a), "n"(kMultiEntries - 1), "r"(0u), "n"(kWordFull)
            : "memory");
    else
        asm volatile(
            "{\n\t"
            ".reg .b32 a, f, t;\n\t"
            ".reg .pred p;\n\t"
            "and.b32 a, %1, %9;\n\t"
            "mad.lo.u32 a, a, 8, %8;\n\t"
            "ld.shared.v2.u32 {%4, %5}, [a];\n\t"
            "shr.b32 f, %0, 26;\n\t"                // fill
            "shf.l.wrap.b32 t, %10, %4, f;\n\t"     // symbols << fill
            "or.b32 %2, %2, t;\n\t"
            "add.u32 %0, %0, %5;\n\t"
            "shf.r.wrap.b32 %1, %6, %7, %0;\n\t"    // next window: (hi:lo) >> bit position
            "setp.ge.u32 p, %0, %11;\n\t"           // the word is full
            "@p st.shared.u32 [%3], %2;\n\t"
            "@p shf.l.wrap.b32 %2, %4, %10, f;\n\t" // the next word: symbols past this one
            "@p add.u32 %3, %3, 4;\n\t"
            "@p sub.u32 %0, %0, %11;\n\t"
            "}"
            : "+r"(X), "+r"(win), "+r"(accl), "+r"(sp), "=r"(r.x), "=r"(r.y)
            : "r"(lo), "r"(hi), "r"(multi_a), "n"(kMultiEntries - 1), "r"(0u), "n"(kWordFull)
            : "memory");
}

// ---- mbarrier + bulk copy (TMA) helpers ------------------------------------

__device__ __forceinline__ void mbar_init(uint32_t bar)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
}

// Copies `bytes` (multiple of 16, 16-byte aligned ends) from global to shared
// memory; completion is signalled on `bar` (one arrival carrying the bytes).
__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                              uint32_t bar)
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// Copies `bytes` (multiple of 16, 16-byte aligned ends) from global to shared
// memory, completing on `bar`, whose expected byte count the caller set.
__device__ __forceinline__ void bulk_copy_g2s_tx(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// Waits until the barrier completes the phase with the given parity; gives up
// after `limit` polls (each suspends the thread for at most kWaitHintNs)
// and returns false.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint32_t limit = kWaitLimit)
{
    for (uint32_t i = 0; i < limit; ++i) {
        uint32_t done;
        asm volatile(
            "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.b32 %0, 1, 0, p; }"
            : "=r"(done)
            : "r"(bar), "r"(parity), "n"(kWaitHintNs)
            : "memory");
        if (done)
            return true;
    }
    return false;
}

// Loads the lane's stream words and its thread metadata: meta = gap |
// next thread's gap << 4 (lane 31 only; the other lanes take it from their
// neighbour) | count << 8.  Words are bit-reversed: stream bit 32k + i
// (MSB-first in the bytes) is bit i of word k, so a right funnel shift by the
// bit position leaves the upcoming bits, first bit lowest.
template <int W>
__device__ __forceinline__ void load_slice(const DecodeParams &p, uint64_t chunk, int lane,
                                           uint32_t (&w)[W / 4 + 1], uint32_t &meta)
{
    const uint64_t g = chunk * 32 + lane;
    const uint8_t *src = p.stream + (uint64_t)W * g;
    if constexpr (W == 8) {
        const uint2 a = *reinterpret_cast<const uint2 *>(src);
        w[0] = __brev(bswap32(a.x));
        w[1] = __brev(bswap32(a.y));
        w[2] = __brev(bswap32(*reinterpret_cast<const uint32_t *>(src + 8)));
    } else {
        const uint4 a = *reinterpret_cast<const uint4 *>(src);
        w[0] = __brev(bswap32(a.x));
        w[1] = __brev(bswap32(a.y));
        w[2] = __brev(bswap32(a.z));
        w[3] = __brev(bswap32(a.w));
        w[4] = __brev(bswap32(*reinterpret_cast<const uint32_t *>(src + 16)));
    }
    meta = ((p.gaps[g >> 1] >> ((g & 1) * 4)) & 0xFu) | ((uint32_t)p.counts[g] << 8);
    if (lane == 31 && 16 * (chunk + 1) < p.gaps_limit)
        meta |= (p.gaps[16 * (chunk + 1)] & 0xFu) << 4;
}

// Matrix of block element e: the last one whose start is <= e.
__device__ __forceinline__ int gemv_matrix_of(const GemvParams *gp, uint32_t e)
{
    int lo = 0, hi = (int)gp->n_mats - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (gp->m[mid].start <= e)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

// acc + w * x for BF16 w and x (each the low or high half of a 32-bit
// word) in one FP32 fused multiply-add.  A product of two BF16 values is
// exact in FP32, so this equals fmaf(float(w), float(x), acc), bit for bit;
// the halves are read in place, with no conversion instructions.
__device__ __forceinline__ float fma_bf16_lo(uint32_t w, uint32_t x, float acc)
{
    asm("{ .reg .b16 wl, wh, xl, xh;\n\t"
        "mov.b32 {wl, wh}, %1;\n\t"
        "mov.b32 {xl, xh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, wl, xl, %0;\n\t"
        "}"
        : "+f"(acc) : "r"(w), "r"(x));
    return acc;
}
__device__ __forceinline__ float fma_bf16_hi(uint32_t w, uint32_t x, float acc)
{
    asm("{ .reg .b16 wl, wh, xl, xh;\n\t"
        "mov.b32 {wl, wh}, %1;\n\t"
        "mov.b32 {xl, xh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, wh, xh, %0;\n\t"
        "}"
        : "+f"(acc) : "r"(w), "r"(x));
    return acc;
}

// Adds the chunk's products to y.  The groups of 8 elements that touch
// the chunk's range [head, head + n_write) (relative to base, 8-aligned)
// are taken one row segment at a time: a segment is the groups of one row
// of one matrix (groups never straddle rows because rows and matrices
// start at multiples of 8).  The lanes share a segment's groups, keep one
// partial sum per token, and a warp sum adds each token's total to y with
// one atomic add.  Matrix and row are located once per chunk and then
// stepped.  In the first and last groups only the chunk's own elements
// count: their other bytes are zeroed first, in both buffers, which makes
// those weights +0 (exactly what masking them would give), so the product
// loop has no end cases.  ebuf holds the chunk's rotated exponents, sgrp
// its sign|mantissa bytes (group 0 of the chunk at offset 0 of both); the
// staged copy has landed, and both are this warp's own.
template <int TT>
__device__ __forceinline__ void gemv_chunk(const GemvParams *gp, uint32_t head, uint32_t n_write, uint64_t base,
                                           int lane, uint32_t ebuf_a, uint32_t sgrp_a)
{
    const uint32_t nt = gp->n_tokens;
    const uint32_t span = head + n_write;
    const uint32_t ngroups = (span + 7) >> 3;
    if (ngroups == 0)
        return;
    {
        // lanes 0..7: bytes [0, head) of group 0; lanes 8..15: bytes
        // [span, 8 ngroups) of the last group
        const uint32_t j = lane < 8 ? (uint32_t)lane : span + (uint32_t)lane - 8u;
        const uint32_t lim = lane < 8 ? head : 8u * ngroups;
        if (lane < 16 && j < lim) {
            asm volatile("st.shared.u8 [%0], %1;" ::"r"(ebuf_a + j), "r"(0u) : "memory");
            asm volatile("st.shared.u8 [%0], %1;" ::"r"(sgrp_a + j), "r"(0u) : "memory");
        }
        __syncwarp();
        // the product loop's shared loads are plain (schedulable) asm: route
        // their base addresses through ordered asm so no load can be placed
        // above these stores
        asm volatile("mov.b32 %0, %0;" : "+r"(ebuf_a)::"memory");
        asm volatile("mov.b32 %0, %0;" : "+r"(sgrp_a)::"memory");
    }
    // matrix, row and column of group 0
    int m = gemv_matrix_of(gp, (uint32_t)base);
    uint32_t cols = gp->m[m].cols, rows = gp->m[m].rows;
    uint32_t r, c;
    {
        const uint32_t o = (uint32_t)base - gp->m[m].start;
        r = o / cols;
        c = o - r * cols;
    }
    const uint16_t *xm = gp->m[m].x;
    float *ym = gp->m[m].y;
    uint32_t g = 0;
    for (;;) {
        const uint32_t gend = min(ngroups, g + ((cols - c) >> 3));
        const uint16_t *xr = xm + c;                        // activations at the segment's first column
        float acc[TT];
#pragma unroll
        for (int t = 0; t < TT; ++t)
            acc[t] = 0.f;
        // The buffers were written before the warp's last __syncwarp, which
        // orders these plain shared loads; the activation loads go first so
        // their latency overlaps the weight assembly.
#pragma unroll(TT <= 2 ? 2 : 1)
        for (uint32_t i = g + lane; i < gend; i += 32) {
            const uint32_t dc = 8u * (i - g);               // column offset within the segment
            constexpr int TP = TT < 2 ? TT : 2;             // tokens whose rows are loaded together
            uint4 xv[TP];
#pragma unroll
            for (int t = 0; t < TP; ++t)
                xv[t] = t < (int)nt ? __ldg(reinterpret_cast<const uint4 *>(xr + (size_t)t * cols + dc))
                                    : make_uint4(0u, 0u, 0u, 0u);
            const uint2 e8 = lds_v2(ebuf_a + 8u * i);
            const uint2 s8 = lds_v2(sgrp_a + 8u * i);
            const uint2 wa = join4(e8.x, s8.x);   // weights 0, 1 | 2, 3 of the group
            const uint2 wb = join4(e8.y, s8.y);   // weights 4, 5 | 6, 7
#pragma unroll
            for (int t0 = 0; t0 < TT; t0 += TP) {
#pragma unroll
                for (int u = 0; u < TP; ++u) {
                    const int t = t0 + u;
                    if (t0 > 0 && t < (int)nt)                 // later token blocks load here
                        xv[u] = __ldg(reinterpret_cast<const uint4 *>(xr + (size_t)t * cols + dc));
                }
#pragma unroll
                for (int u = 0; u < TP; ++u) {
                    const int t = t0 + u;
                    if (t < (int)nt) {
                        const uint4 xv_t = xv[u];
                        float a = acc[t];
                        a = fma_bf16_lo(wa.x, xv_t.x, a);
                        a = fma_bf16_hi(wa.x, xv_t.x, a);
                        a = fma_bf16_lo(wa.y, xv_t.y, a);
                        a = fma_bf16_hi(wa.y, xv_t.y, a);
                        a = fma_bf16_lo(wb.x, xv_t.z, a);
                        a = fma_bf16_hi(wb.x, xv_t.z, a);
                        a = fma_bf16_lo(wb.y, xv_t.w, a);
                        a = fma_bf16_hi(wb.y, xv_t.w, a);
                        acc[t] = a;
                    }
                }
            }
        }
#pragma unroll
        for (int t = 0; t < TT; ++t) {
            float a = acc[t];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                a += __shfl_xor_sync(0xFFFFFFFFu, a, off);
            if (lane == 0 && t < (int)nt)
                atomicAdd(ym + (size_t)t * rows + r, a);
        }
        if (gend >= ngroups)
            break;
        // the next row, or the first row of the next matrix
        g = gend;
        c = 0;
        if (++r == rows) {
            ++m;
            cols = gp->m[m].cols;
            rows = gp->m[m].rows;
            xm = gp->m[m].x;
            ym = gp->m[m].y;
            r = 0;
        }
    }
}

// Two-level table lookup of the code at the front of window `win` (first
// stream bit lowest): the entry as the multi-code table would hold it for
// that one code (rotated exponent; length | 8 << 16).
__device__ __forceinline__ uint2 long_code(uint32_t win, uint32_t lut_a, uint32_t &seen)
{
    const uint32_t wm = __brev(win);
    uint32_t e = lds_u16(lut_a + ((wm >> 24) << 1));
    if (e & kLutPointer)
        e = lds_u16(lut_a + ((((e & 0xFFu) << 8) | ((wm >> 16) & 0xFFu)) << 1));
    seen |= e;
    return make_uint2(rot_exp(e & 0xFFu), entry_step((e >> 8) & 0x1Fu, 1));
}

// Decodes the codes of a full slice (every lane of the chunk has one) into
// the exponent buffer: this lane's codes go to bytes a, a + 1, ... (a =
// offset within the buffer at shared-window address ebuf_a), four per word,
// and each word is stored as it fills (the fill starts at byte a's place in
// its word).  Its last lookup may also decode the first codes of the next
// lane: they come from the same bit position, so they are the next lane's
// own bytes.  A word two lanes share (the word a lane's run ends in, when
// the next lane's run starts inside it) is stored by both: by the next lane
// when it fills its first word (zeros below its first byte), and by this
// lane when the next lane's first codes, decoded at its end, complete the
// word.  The next lane fills its first word within its first 64 bits (at
// most three codes from bit 15); this lane completes the word only in the
// lookup that crosses the slice end, so a warp barrier after the first two
// stream words puts the complete word last.  A last word still part-filled
// at the end is left in accl at address sp (fill in X) for the caller to OR
// in.  Returns X: bit position after the last lookup (bits 0..15), fill
// (bits 16..21); r holds the last table entry.
//
// kOr: the words are ORed into a zeroed buffer instead, which needs no
// order: for 64-bit slices (too short for the order above), and in the
// block's last chunk, whose slices end at the end of the stream (`end`
// below the slice width) or lie past it.
template <int W, bool kOr>
__device__ __forceinline__ uint32_t decode_slice(const uint32_t (&w)[W / 4 + 1], uint32_t gap, uint32_t a, int end,
                                                 uint32_t ebuf_a, uint32_t multi_a, uint32_t lut_a, uint32_t &seen,
                                                 uint32_t &sp, uint32_t &accl, uint2 &r)
{
    constexpr int kWords = W / 4 + 1;
    static_assert(kOr || 8 * W - (kWindowBits - 1) > 64, "the ordered stores need slices over 74 bits");
    uint32_t X = gap | ((a & 3u) * 8u * kFillOne);
    sp = ebuf_a + (a & ~3u);
    accl = 0;
    r = make_uint2(0u, 0u);
#pragma unroll
    for (int h = 0; h < kWords - 1; ++h) {
        if (!kOr && h == 2)
            __syncwarp();   // every lane's first word is stored by now
        const uint32_t lo = w[h], hi = w[h + 1];
        const uint32_t lim = (uint32_t)max(0, min(end, 32 * (h + 1)));
        uint32_t win = __funnelshift_r(lo, hi, X);
        for (;;) {
            while ((X & kPosMask) < lim)
                lookup_step<kOr>(X, win, accl, sp, r, lo, hi, multi_a);
            if (!(X & kLongStep))
                break;
            // the first code is longer than the window: take it from the
            // two-level tables
            X -= kLongStep;
            r = long_code(win, lut_a, seen);
            const uint32_t f = X >> kFillShift;
            accl |= __funnelshift_l(0u, r.x, f);
            const uint32_t acch = __funnelshift_l(r.x, 0u, f);
            X += r.y;
            if (X >= kWordFull) {
                if constexpr (kOr)
                    red_or_u32(sp, accl);
                else
                    sts_u32(sp, accl);
                sp += 4;
                accl = acch;
                X -= kWordFull;
            }
            win = __funnelshift_r(lo, hi, X);
        }
    }
    return X;
}

// The chunk body.  TT = 0: BF16 output; TT > 0: fused matrix-vector product
// for up to TT tokens (gp != nullptr).  VER: also sum every chunk's bytes as
// they are read and compare with p.sums (BF16 output only).
template <int W, int MINLEN, int TT, bool VER = false>
__device__ __forceinline__ void decode_body(const DecodeParams &p, const GemvParams *gp)
{
    static_assert(!VER || TT == 0, "the verifying decode writes BF16");
    using G = Geometry<W, MINLEN>;
    extern __shared__ __align__(16) uint8_t smem[];
    const int warps = blockDim.x >> 5;
    uint64_t *mbar = reinterpret_cast<uint64_t *>(smem);
    uint2 *multi = reinterpret_cast<uint2 *>(smem + kBarBytes);
    uint8_t *len_of = smem + kBarBytes + kMultiEntries * kEntryBytes;   // by rotated exponent
    uint8_t *warp_area = smem + kHeadBytes;
    uint16_t *lut = reinterpret_cast<uint16_t *>(warp_area + (size_t)warps * G::kWarpBytes);

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const uint32_t n_tables = p.n_tables;
    const uint32_t min_len = p.min_len;
    // "no code" in shared memory: flagged, and as long as the shortest code,
    // so every decode step advances by at least min_len bits
    const uint32_t no_code = 0x4000u | (min_len << 8);

    // ---- this warp's first chunk: its loads overlap the table build ---------
    // (chunk indices fit in 32 bits: a block has fewer than 2^32 elements,
    // and a chunk holds at least 32 slices of 64 bits)
    const uint32_t n_chunks = (uint32_t)p.n_chunks;
    const uint32_t n_warps = gridDim.x * (uint32_t)warps;
    const uint32_t gw = blockIdx.x * (uint32_t)warps + (uint32_t)warp;
    uint32_t chunk = gw;
    // Rounds below r_static are dealt out: chunk gw + k n_warps is this
    // warp's k-th.  With a workspace, chunks from d0 on are claimed: pool q
    // holds d0 + q, d0 + q + 4, ..., and warp gw claims from pool gw % 4.
    // Blocks of fewer rounds keep the plain deal: their imbalance is the
    // rounding of chunks to warps, which claiming cannot remove.
    const uint32_t rounds = n_chunks / n_warps;
    const uint32_t r_static = rounds - kSchedTailRounds;
    const uint32_t d0 = r_static * n_warps;
    const bool dyn = p.sched != nullptr && rounds >= (uint32_t)kSchedTailRounds + 2;
    const uint32_t q = gw % kSchedPools;
    uint32_t *const pool = p.sched + q * kSchedStride;
    uint32_t claim = 0;   // lane 0: the last claim's result
    uint32_t w[G::kWords];
    uint32_t meta = 0, pos0 = 0, pos1 = 0;
#pragma unroll
    for (int k = 0; k < G::kWords; ++k)
        w[k] = 0;
    if (chunk < n_chunks) {
        load_slice<W>(p, chunk, lane, w, meta);
        pos0 = p.chunk_pos[chunk];
        pos1 = p.chunk_pos[chunk + 1];
    }

    // ---- prologue: the tables into shared memory -----------------------------
    // One thread copies the format's two-level tables, and the multi-code
    // table when it was built on the host, with bulk copies (TMA) that
    // complete on the prologue barrier; the first chunk's loads are in flight
    // meanwhile.  Then every thread checks its share of the entries in place.
    const uint32_t pbar = smem_addr(&mbar[kMaxWarpsPerCta]);
    const uint32_t multi_a = smem_addr(multi);
    const uint32_t lut_bytes = n_tables * 512u;
    if (tid == 0) {
        mbar_init(pbar);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        const uint32_t bytes = lut_bytes + (p.multi_src ? (uint32_t)(kMultiEntries * kEntryBytes) : 0u);
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(pbar), "r"(bytes) : "memory");
        bulk_copy_g2s_tx(smem_addr(lut), p.lut, lut_bytes, pbar);
        if (p.multi_src)
            bulk_copy_g2s_tx(multi_a, p.multi_src, kMultiEntries * kEntryBytes, pbar);
    }
    if (lane == 0)
        mbar_init(smem_addr(&mbar[warp]));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    __syncthreads();
    // (a copy that never lands leaves the tables unchecked: the CTA decodes
    // nothing and reports a timeout)
    const bool tables_late = __syncthreads_or(!mbar_wait(pbar, 0u)) != 0;
    // Two-level tables, sanitised: anything malformed (bad pointer, bad
    // length, shorter than the shortest code) becomes "no code", so decoding
    // never indexes outside the tables and a lane never produces more codes
    // than its buffers hold.
    for (uint32_t i = tid; !tables_late && i < n_tables * 256u; i += blockDim.x) {
        uint32_t e = lut[i];
        if (e & kLutPointer) {
            const uint32_t to = e & 0xFFu;
            if (i >= 256u || to == 0 || to >= n_tables || (e & 0x7F00u))
                e = no_code;
        } else {
            const uint32_t l = (e >> 8) & 0x1Fu;
            if ((e & 0x4000u) || l < min_len || l > 16)
                e = no_code;
            else
                len_of[rot_exp(e & 0xFFu)] = (uint8_t)l;   // every leaf of a symbol holds its length
        }
        lut[i] = (uint16_t)e;
    }
    // ---- prologue: multi-code table -----------------------------------------
    // Entry for an 11-bit window, stored at the window's bit-reversed value
    // (first stream bit lowest, as the decoder reads it): x = the whole codes
    // the window starts with (at most 4), as rotated exponents in bytes 0..3
    // (unused bytes 0); y = entry_step(total length, count).  When the first
    // code is longer than the window (or is no code) the entry is x = 0, y =
    // kLongStep: adding it ends the lookup loop, and the decoder takes the
    // two-level path.
    if (p.multi_src) {
        // built once on the host (df11_build_decode_table): any entry whose
        // count and length no table of this block could hold becomes the
        // long-code marker, so a lane still advances at least min_len bits
        // per code and never writes more codes than its buffer holds (the
        // host table's y is length | 8 x count << 16; its long-code marker
        // 2^31)
        for (int slot = tid; !tables_late && slot < kMultiEntries; slot += blockDim.x) {
            uint2 v = multi[slot];
            const uint32_t n = v.y >> 19, t = v.y & 0xFFFFu;
            if (v.y != (t | (n << 19)) || n < 1 || n > (uint32_t)kMaxCodesPerEntry ||
                t > (uint32_t)kWindowBits || t < n * min_len) {
                v = make_uint2(0u, kLongStep);
            } else {
                if (n < 4)
                    v.x &= (1u << (8 * n)) - 1u;
                v.y = entry_step(t, n);
            }
            multi[slot] = v;
        }
    }
    __syncthreads();
    if (!p.multi_src && !tables_late) {
        for (int slot = tid; slot < kMultiEntries; slot += blockDim.x) {
            // consecutive threads fill consecutive entries (conflict-free stores)
            const uint32_t idx = __brev((uint32_t)slot) >> (32 - kWindowBits);
            const uint32_t win = idx << (32 - kWindowBits);   // MSB-first window
            uint32_t t = 0, n = 0, syms = 0;
            while (n < kMaxCodesPerEntry) {
                const uint32_t v = win << t;
                uint32_t e = lut[v >> 24];
                if (e & kLutPointer)
                    e = lut[((e & 0xFFu) << 8) | ((v >> 16) & 0xFFu)];
                if (e & 0x4000u)
                    break;
                const uint32_t l = (e >> 8) & 0x1Fu;
                if (t + l > (uint32_t)kWindowBits)
                    break;
                syms |= rot_exp(e & 0xFFu) << (8 * n);
                ++n;
                t += l;
            }
            multi[slot] = make_uint2(syms, n ? entry_step(t, n) : kLongStep);
        }
        __syncthreads();
    }

    // shared-window addresses (bytes)
    const uint32_t smem_base = smem_addr(smem);
    const uint32_t len_a = multi_a + kMultiEntries * kEntryBytes;
    const uint32_t lut_a = smem_base + (uint32_t)kHeadBytes + (uint32_t)(warps * G::kWarpBytes);
    const uint32_t ebuf_a = smem_base + (uint32_t)kHeadBytes + (uint32_t)(warp * G::kWarpBytes);
    const uint32_t sbuf_a = ebuf_a + G::kEbufBytes;
    const uint32_t bar = smem_addr(&mbar[warp]);
    uint32_t parity = 0;

    if (tables_late) {
        // let a late copy land before the CTA's shared memory is released
        mbar_wait(pbar, 0u);
        if (tid == 0 && p.err)
            atomicOr(p.err, DF11_DEVERR_TIMEOUT);
    }
    // (the dynamic schedule gives every warp a chunk, and its CTAs count
    // themselves out at the end even when they decode nothing)
    if (chunk >= n_chunks || (tables_late && !dyn))
        return;

    uint32_t err = 0;
    bool stalled = false;      // a staged copy did not arrive in time
    uint32_t n_done = 0;       // chunks this warp has finished
    // (verifying) kReported in err: this warp has reported a bad chunk
    constexpr uint32_t kReported = 0x80000000u;

    while (!tables_late) {
        // ---- positions (warp-uniform) and the staged sign|mantissa copy -----
        const bool pos_ok = pos0 <= pos1 && (uint64_t)pos1 <= p.out_limit &&
                            pos1 - pos0 <= (uint32_t)(32 * G::kMaxCodes);
        const uint32_t head = pos0 & 7u;
        const uint64_t base = (uint64_t)pos0 - head;           // 8-element aligned
        const uint32_t gfirst = head ? 1u : 0u;
        // copy [pos0 & ~15, ceil16(pos1)) -> sbuf; group i is at sbuf + (pos0 & 8) + 8i
        const uint64_t cp_lo = (uint64_t)pos0 & ~15ull;
        uint32_t cp_bytes = pos_ok ? (uint32_t)((((uint64_t)pos1 + 15) & ~15ull) - cp_lo) : 0u;
        // (warp-uniform) the copy stays inside the block's sign|mantissa
        // bytes and the warp's buffer
        if (cp_bytes && !DF11_CHECK(err, cp_bytes <= (uint32_t)G::kSbufBytes &&
                                             cp_lo + cp_bytes <= ((p.out_limit + 15) & ~15ull)))
            cp_bytes = 0;
        if (cp_bytes && lane == 0)
            bulk_copy_g2s(sbuf_a, p.signmant + cp_lo, cp_bytes, bar);

        // ---- the next chunk's slice and positions, loaded ahead -------------
        uint32_t next;
        if (!dyn || n_done + 1 < r_static) {
            next = chunk + n_warps;
            if (dyn && n_done + 2 == r_static && lane == 0)
                claim = atomicAdd(pool, 1u);      // the first claimed chunk, a chunk ahead
        } else {
            next = d0 + q + kSchedPools * __shfl_sync(0xFFFFFFFFu, claim, 0);
            if (lane == 0 && next < n_chunks)
                claim = atomicAdd(pool, 1u);      // the chunk after next
        }
        const bool has_next = next < n_chunks;
        uint32_t nw[G::kWords];
        uint32_t nmeta = 0, npos0 = 0, npos1 = 0;
        if (has_next) {
            load_slice<W>(p, next, lane, nw, nmeta);
            npos0 = p.chunk_pos[next];
            npos1 = p.chunk_pos[next + 1];
        }

        // thread metadata: gap, count and the next thread's gap
        const uint32_t gap = meta & 0xFu;
        const uint32_t cnt = meta >> 8;
        // (verifying) the lane's items of the chunk sum: its stream words,
        // its gap and count, and on lane 0 the two positions
        // The lanes' sums add up to zero for an intact chunk: lane 0 starts
        // from minus the expected sum.
        uint32_t vsum = 0;
        if constexpr (VER) {
#pragma unroll
            for (int j = 0; j < W / 4; ++j)
                vsum += chunk_mix(w[j], (uint32_t)((W / 4) * lane + j) * kTagMul);
            vsum += chunk_mix(gap | (cnt << 8), (0x10000u + (uint32_t)lane) * kTagMul);
            if (lane == 0)
                vsum += chunk_mix(pos0, 0x20000u * kTagMul) + chunk_mix(pos1, 0x20001u * kTagMul) -
                        p.sums[chunk];

        }
        const uint32_t gap_up = __shfl_down_sync(0xFFFFFFFFu, gap, 1);
        const uint32_t gnext = lane == 31 ? (meta >> 4) & 0xFu : gap_up;
        // ---- warp scan of the stored counts: each lane's output offset -----
        uint32_t incl = cnt;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (lane >= d)
                incl += y;
        }
        const uint32_t total = __shfl_sync(0xFFFFFFFFu, incl, 31);
        const uint32_t off = incl - cnt;
        const bool counts_ok = !__any_sync(0xFFFFFFFFu, cnt > (uint32_t)G::kMaxCodes) && total == pos1 - pos0;
        if (!pos_ok) {
            err |= DF11_DEVERR_BAD_POS;
        } else if (!counts_ok) {
            err |= DF11_DEVERR_COUNT;
        } else {
            const uint32_t n_write = total;

            // ---- decode this lane's codes straight into place ---------------
            // Lane bytes go to ebuf[head + off, head + off + cnt).
            const uint32_t a = head + off;
            // (checked build) every word the lane may store lies in the
            // buffer: at most kMaxCodes + 3 codes from a
            const bool write_ok =
                __all_sync(0xFFFFFFFFu, DF11_CHECK(err, a + G::kMaxCodes + 8 <= (uint32_t)G::kEbufBytes));
            uint32_t seen = 0;
            bool lane_bad = false;
            // The lane's codes start in [gap, end): end is the slice width,
            // or the end of the stream in the block's last chunk; the next
            // code (the next thread's first, or the end of the stream) must
            // start where they end.
            const bool full = chunk < p.full_chunks;
            int end = G::kSliceBits;
            int expect = G::kSliceBits + (int)gnext;
            if (!full) {
                const uint64_t bit0 = ((uint64_t)chunk * 32 + lane) * (uint64_t)G::kSliceBits;
                if (bit0 + G::kSliceBits >= p.total_bits) {
                    end = bit0 >= p.total_bits ? 0 : (int)(p.total_bits - bit0);
                    expect = end;
                }
            }
            // 128-bit slices of a full chunk: ordered plain stores; else ORs
            // into a zeroed buffer
            constexpr bool kOrAlways = G::kSliceBits - (kWindowBits - 1) <= 64;
            const bool use_or = kOrAlways || !full;
            if (use_or) {
                // zero the words the lanes OR into (up to the next lane's
                // first codes after the last lane's run)
                const uint32_t zend = min((uint32_t)G::kEbufBytes, (head + total + 6u + 15u) & ~15u);
                for (uint32_t i = 16u * lane; i < zend; i += 512u)
                    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(ebuf_a + i), "r"(0u)
                                 : "memory");
                __syncwarp();
            }
            uint32_t sp = 0, accl = 0, X = 0;
            uint2 r = make_uint2(0u, 0u);
            if (write_ok && cnt) {
                if (use_or)
                    X = decode_slice<W, true>(w, gap, a, end, ebuf_a, multi_a, lut_a, seen, sp, accl, r);
                else
                    X = decode_slice<W, kOrAlways>(w, gap, a, G::kSliceBits, ebuf_a, multi_a, lut_a, seen, sp,
                                                   accl, r);
            }
            if (cnt) {
                // Codes of the last entry that start at or past `end` are the
                // next lane's; the first of them (or the end of the entry) is
                // where the next code starts.  The entry's code starts c0 <=
                // c1 <= c2 <= c3 never fall (lengths are unsigned), so the
                // codes that pass `end` are a suffix and the next start is the
                // lowest start at or past it.
                const uint32_t emitted = sp - ebuf_a + (X >> (kFillShift + 3)) - a;
                const uint32_t n = entry_codes(r.y);
                const int pos = (int)(X & 0xFFFFu);
                const int c0 = pos - (int)(r.y & 0xFFFFu);   // start of the entry's first code
                const int c1 = c0 + (int)lds_u8(len_a + (r.x & 0xFFu));
                const int c2 = c1 + (int)lds_u8(len_a + ((r.x >> 8) & 0xFFu));
                const int c3 = c2 + (int)lds_u8(len_a + ((r.x >> 16) & 0xFFu));
                const bool p1 = n > 1u && c1 >= end, p2 = n > 2u && c2 >= end, p3 = n > 3u && c3 >= end;
                const uint32_t passed = (uint32_t)p1 + (uint32_t)p2 + (uint32_t)p3;
                const int next_start = p1 ? c1 : p2 ? c2 : p3 ? c3 : pos;
                lane_bad = emitted - passed != cnt || next_start != expect;
            }
            __syncwarp();
            // the part-filled last word: ORed over the next lane's first word
            // (zeros below its first byte) or the zeroed buffer; a full
            // chunk's last lane's is its own
            if (write_ok && cnt && (X >> kFillShift)) {
                if (use_or || lane < 31)
                    red_or_u32(sp, accl);
                else
                    sts_u32(sp, accl);
            }
            if (lane_bad)
                err |= DF11_DEVERR_COUNT;
            if (seen & 0x4000u)
                err |= DF11_DEVERR_BAD_CODE;
            __syncwarp();

            // ---- wait for the staged sign|mantissa bytes --------------------
            if (cp_bytes) {
                if (!mbar_wait(bar, parity)) {
                    err |= DF11_DEVERR_TIMEOUT;
                    stalled = true;
                }
                parity ^= 1u;
            }

            // ---- merge with sign|mantissa and store -------------------------
            // Whole groups: 8 exponents + 8 sign|mantissa bytes -> one 16-byte
            // store per lane.  The partial groups at both ends (<= 7 elements
            // each) take one element per lane on lanes 0..15.
            // the merge's groups lie inside the output range and the staged bytes
            const bool merge_ok =
                DF11_CHECK(err, (uint64_t)pos0 + n_write <= p.out_limit &&
                                    (pos0 & 8u) + 8u * ((head + n_write + 7) >> 3) <= (uint32_t)G::kSbufBytes);
            if (!stalled && TT == 0 && merge_ok) {
                const uint32_t span = head + n_write;
                const uint32_t mend = span >> 3;                   // whole groups end
                const uint32_t sgrp_a = sbuf_a + (pos0 & 8u);     // group 0 of the chunk
                uint4 *const out16 = reinterpret_cast<uint4 *>(p.out + base);
                // The group loads are plain asm, so the two groups of an
                // unrolled pair load together; their bases pass through
                // ordered asm after the staged copy's wait, which keeps every
                // load below it.
                uint32_t eb = ebuf_a, sg = sgrp_a;
                asm volatile("mov.b32 %0, %0;" : "+r"(eb)::"memory");
                asm volatile("mov.b32 %0, %0;" : "+r"(sg)::"memory");
#pragma unroll 2
                for (uint32_t i = gfirst + lane; i < mend; i += 32) {
                    const uint2 e8 = lds_v2(eb + 8u * i);
                    const uint2 s8 = lds_v2(sg + 8u * i);
                    const uint2 x = join4(e8.x, s8.x);
                    const uint2 y = join4(e8.y, s8.y);
                    out16[i] = make_uint4(x.x, x.y, y.x, y.y);
                    if constexpr (VER) {
                        const uint32_t t = (0x100000u + 2u * i) * kTagMul;
                        vsum += chunk_mix(s8.x, t) + chunk_mix(s8.y, t + kTagMul);
                    }
                }
                const uint32_t fs = gfirst * 8;                    // first whole-group element
                const uint32_t hend = min(fs, span);               // head part: [head, hend)
                const uint32_t tbeg = max(mend * 8, fs);           // tail part: [tbeg, span)
                // lanes 0..7 take the head part's elements, lanes 8..15 the tail's
                const uint32_t l = lane < 8 ? head + (uint32_t)lane : tbeg + (uint32_t)lane - 8u;
                const uint32_t lim = lane < 8 ? hend : span;
                if (lane < 16 && l < lim) {
                    const uint32_t sm = lds_u8_m(sgrp_a + l);
                    p.out[base + l] = join1(lds_u8_m(ebuf_a + l), sm);
                    if constexpr (VER)
                        vsum += chunk_mix(sm, (0x200000u + l) * kTagMul);
                }
            }
            if constexpr (VER) {
                if (chunk == 0) {
                    // chunk 0 also covers the tables, read as they are stored
                    const uint32_t *lw = reinterpret_cast<const uint32_t *>(p.lut);
                    for (uint32_t i = (uint32_t)lane; i < 128u * n_tables; i += 32u)
                        vsum += chunk_mix(lw[i], (0x400000u + i) * kTagMul);
                }
                // (all lanes: a merge that did not run leaves the sum short)
                if (__reduce_add_sync(0xFFFFFFFFu, vsum) != 0u)
                    err |= DF11_DEVERR_CHECKSUM;
            }
            if constexpr (TT > 0) {
                if (!stalled && merge_ok)
                    gemv_chunk<TT>(gp, head, n_write, base, lane, ebuf_a, sbuf_a + (pos0 & 8u));
            }
            __syncwarp();
        }
        if constexpr (VER) {
            // a chunk is bad when its sum differs or its decode failed (the
            // warp's flags only grow and its chunks come in increasing order,
            // so reporting its first bad chunk gives the minimum)
            if (!(err & kReported) && __any_sync(0xFFFFFFFFu, err != 0)) {
                err |= kReported;
                if (lane == 0 && p.first_bad)
                    atomicMin(reinterpret_cast<unsigned long long *>(p.first_bad), (unsigned long long)chunk);
            }
        }

        ++n_done;
        if (!has_next || stalled)
            break;
        chunk = next;
#pragma unroll
        for (int k = 0; k < G::kWords; ++k)
            w[k] = nw[k];
        meta = nmeta;
        pos0 = npos0;
        pos1 = npos1;
    }
    if (stalled)   // let the late copy land before this CTA's shared memory is released
        mbar_wait(bar, parity ^ 1u);
    if constexpr (VER)
        err &= ~kReported;
    if (err && p.err)
        atomicOr(p.err, err);
    if (dyn) {
        // a claim still in flight (after a stall) must land before the CTA
        // counts itself out: the and waits for its result
        uint32_t z = 0;
        if (lane == 0)
            asm volatile("and.b32 %0, %1, 0;" : "=r"(z) : "r"(claim));
        __threadfence();
        __syncthreads();
        if (tid == 0 && atomicAdd(p.sched + kSchedDoneWord, 1u + z) == gridDim.x - 1) {
            // every other CTA is out: ready for the next launch
#pragma unroll
            for (int i = 0; i < kSchedPools; ++i)
                p.sched[i * kSchedStride] = 0;
            p.sched[kSchedDoneWord] = 0;
            __threadfence();
        }
    }
}

// The bounded wait's give-up path, on its own: one warp waits on a barrier
// that nothing arrives on, and reports what the decode would report.
__global__ void bounded_wait_kernel(uint32_t polls, uint32_t *status)
{
    __shared__ __align__(8) uint64_t bar;
    const uint32_t a = smem_addr(&bar);
    if (threadIdx.x == 0)
        mbar_init(a);   // one arrival expected; none comes
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    __syncwarp();
    const bool done = mbar_wait(a, 0u, polls);
    if (threadIdx.x == 0)
        *status = done ? 0u : DF11_DEVERR_TIMEOUT;
}

// A decode kernel is compiled for one resident CTA per SM (up to 32 warps)
// or two (up to 23 warps each): with two, the register cap is 40 per thread
// (11.5 warps per SM sub-partition), and two 23-warp CTAs fill the SM's
// shared memory with 46 warps instead of 32.  Each CTA holds its own copy
// of the tables.
// (The verifying decode keeps two more values per lane: 20 warps, 48
// registers.)
template <int CPS, bool VER = false>
constexpr int kCtaWarps = CPS == 1 ? kMaxWarpsPerCta : VER ? 23 : 23;

template <int W, int MINLEN, int CPS, bool VER = false>
__global__ void __launch_bounds__(kCtaWarps<CPS, VER> * 32, CPS) df11_decode_kernel(DecodeParams p)
{
    decode_body<W, MINLEN, 0, VER>(p, nullptr);
}

// The fused products at one token also come as two CTAs of up to 20 warps
// per SM (48 registers, no spills; 40 warps per SM against 32).
constexpr int kGemv2Warps = 20;

template <int W, int MINLEN, int TT, int CPS>
__global__ void __launch_bounds__(CPS == 1 ? kMaxWarpsPerCta * 32 : kGemv2Warps * 32, CPS)
    df11_gemv_kernel(DecodeParams p, const __grid_constant__ GemvParams gp)
{
    decode_body<W, MINLEN, TT>(p, &gp);
}

// ------------------------------------------------------------ launch

constexpr int kMaxDevices = 64;
// kernel variants: (slice width, shortest code) x (store with one CTA per
// SM, products for 1, 2, 4, 8 tokens, store with two CTAs per SM, the
// verifying store with one and with two CTAs per SM, products for 1 token
// with two CTAs per SM)
constexpr int kVariantsPerLayout = 9;
constexpr int kVariants = 4 * kVariantsPerLayout;
// resident CTAs per SM, by device, kernel variant and table count
std::atomic<int> g_occupancy[kMaxDevices][kVariants][257];
std::atomic<int> g_attr_done[kMaxDevices][kVariants];

// Per-device properties the launch shapes need (read once).
struct DeviceProps {
    int sms;
    int smem_per_sm;      // shared memory of one SM
    int smem_reserved;    // shared memory the system reserves per CTA
    int smem_optin;       // largest dynamic shared memory of one CTA
};
std::atomic<int> g_props_done[kMaxDevices];
DeviceProps g_props[kMaxDevices];

df11_status device_props(int dev, DeviceProps &out)
{
    if (!g_props_done[dev].load(std::memory_order_acquire)) {
        DeviceProps d;
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) !=
                cudaSuccess ||
            cudaDeviceGetAttribute(&d.smem_reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) !=
                cudaSuccess ||
            cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
            return DF11_ERR_CUDA;
        g_props[dev] = d;   // identical values if two threads race here
        g_props_done[dev].store(1, std::memory_order_release);
    }
    out = g_props[dev];
    return DF11_OK;
}

struct LaunchShape {
    int warps;
    size_t smem;
    unsigned grid;
    int resident_warps;   // warps resident per SM
};

// Warps per CTA (as many as shared memory holds for `cps` CTAs per SM, at
// most max_warps), shared memory, and the grid (one wave of resident CTAs
// by default; max_ctas overrides it) for one kernel variant; sets the
// shared-memory attribute once per device.  The resident CTAs per SM are
// queried (and cached per variant and table count) only for the variant's
// own CTA size, `cached`; other sizes give a grid of max_ctas.
template <int W, int MINLEN, typename Kernel>
df11_status shape_launch(Kernel kernel, int v, const DecodeParams &prm, int dev, uint32_t max_ctas,
                         int max_warps, int cps, LaunchShape &ls, bool cached = true,
                         int carveout = (int)cudaSharedmemCarveoutMaxShared)
{
    DeviceProps d;
    if (device_props(dev, d) != DF11_OK)
        return DF11_ERR_CUDA;
    const size_t limit = (size_t)min(d.smem_optin, d.smem_per_sm / cps - d.smem_reserved);
    int warps = max_warps;
    while (warps > 1 && smem_bytes_for<W, MINLEN>(warps, prm.n_tables) > limit)
        --warps;
    const size_t smem = smem_bytes_for<W, MINLEN>(warps, prm.n_tables);
    if (smem > limit)
        return DF11_ERR_INVALID_ARGUMENT;
    if (!g_attr_done[dev][v].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, d.smem_optin) !=
                cudaSuccess ||
            cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, carveout) !=
                cudaSuccess)
            return DF11_ERR_CUDA;
        g_attr_done[dev][v].store(1, std::memory_order_release);
    }
    int occ = cached ? g_occupancy[dev][v][prm.n_tables].load(std::memory_order_relaxed) : 1;
    if (occ == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, warps * 32, smem) != cudaSuccess)
            return DF11_ERR_CUDA;
        if (occ < 1)
            return DF11_ERR_CUDA;
        g_occupancy[dev][v][prm.n_tables].store(occ, std::memory_order_relaxed);
    }
    const uint64_t ctas_needed = (prm.n_chunks + warps - 1) / warps;
    const uint64_t resident = (uint64_t)occ * (uint64_t)d.sms;
    // default: one wave of resident CTAs, each looping over chunks; a given
    // count may be smaller (SMs left to other streams) or larger (waves of
    // short-lived CTAs that free their SM as each one finishes)
    const uint64_t want = max_ctas ? (uint64_t)max_ctas : resident;
    ls.warps = warps;
    ls.smem = smem;
    ls.grid = (unsigned)(ctas_needed < want ? ctas_needed : want);
    ls.resident_warps = occ * warps;
    return DF11_OK;
}

template <int W, int MINLEN>
constexpr int variant_base()
{
    return ((W == 8 ? 0 : 2) + (MINLEN == 1 ? 0 : 1)) * kVariantsPerLayout;
}

// Launches the store kernel shaped for one or two CTAs per SM, whichever
// keeps more warps resident (one on a tie: fewer table copies to build).  A
// block of fewer chunks than one full CTA per SM holds gets one CTA per SM
// of just enough warps for one chunk each, so every SM shares the work
// instead of a few full CTAs.
template <int W, int MINLEN, bool VER = false>
df11_status launch(const DecodeParams &prm, int dev, cudaStream_t stream, uint32_t max_ctas)
{
    auto k1 = df11_decode_kernel<W, MINLEN, 1, VER>;
    auto k2 = df11_decode_kernel<W, MINLEN, 2, VER>;
    const int v1 = variant_base<W, MINLEN>() + (VER ? 6 : 0), v2 = variant_base<W, MINLEN>() + (VER ? 7 : 5);
    if (!max_ctas) {
        DeviceProps d;
        if (device_props(dev, d) != DF11_OK)
            return DF11_ERR_CUDA;
        const uint64_t sms = (uint64_t)d.sms;
        if (prm.n_chunks < sms * (uint64_t)kCtaWarps<2, VER>) {
            const int warps = (int)((prm.n_chunks + sms - 1) / sms);
            LaunchShape s1;
            const df11_status st =
                shape_launch<W, MINLEN>(k1, v1, prm, dev, (uint32_t)sms, warps, 1, s1, false);
            if (st == DF11_OK) {
                k1<<<s1.grid, s1.warps * 32, s1.smem, stream>>>(prm);
                return cudaGetLastError() == cudaSuccess ? DF11_OK : DF11_ERR_CUDA;
            }
        }
    }
    LaunchShape s1, s2;
    const df11_status st1 = shape_launch<W, MINLEN>(k1, v1, prm, dev, max_ctas, kCtaWarps<1, VER>, 1, s1);
    const df11_status st2 = shape_launch<W, MINLEN>(k2, v2, prm, dev, max_ctas, kCtaWarps<2, VER>, 2, s2);
    if (st1 != DF11_OK && st2 != DF11_OK)
        return st1;
    if (st2 == DF11_OK && (st1 != DF11_OK || s2.resident_warps > s1.resident_warps))
        k2<<<s2.grid, s2.warps * 32, s2.smem, stream>>>(prm);
    else
        k1<<<s1.grid, s1.warps * 32, s1.smem, stream>>>(prm);
    return cudaGetLastError() == cudaSuccess ? DF11_OK : DF11_ERR_CUDA;
}

// The fused products' one CTA per SM needs about two thirds of the shared
// memory; asking for no more leaves the rest to L1, which then holds the
// activation rows the warps read over and over (2-4% faster than the
// largest shared-memory split).
constexpr int kGemvCarveout = 70;   // percent of the SM's shared memory

template <int W, int MINLEN, int TT>
df11_status launch_gemv(const DecodeParams &prm, const GemvParams &gp, int dev, cudaStream_t stream)
{
    auto kernel = df11_gemv_kernel<W, MINLEN, TT, 1>;
    constexpr int v = variant_base<W, MINLEN>() + (TT == 1 ? 1 : TT == 2 ? 2 : TT == 4 ? 3 : 4);
    LaunchShape ls;
    const df11_status st =
        shape_launch<W, MINLEN>(kernel, v, prm, dev, 0, kMaxWarpsPerCta, 1, ls, true, kGemvCarveout);
    if constexpr (TT == 1) {
        // the two-CTA shape when it keeps more warps resident
        auto k2 = df11_gemv_kernel<W, MINLEN, TT, 2>;
        LaunchShape l2;
        if (shape_launch<W, MINLEN>(k2, variant_base<W, MINLEN>() + 8, prm, dev, 0, kGemv2Warps, 2, l2) == DF11_OK &&
            (st != DF11_OK || l2.resident_warps > ls.resident_warps)) {
            k2<<<l2.grid, l2.warps * 32, l2.smem, stream>>>(prm, gp);
            return cudaGetLastError() == cudaSuccess ? DF11_OK : DF11_ERR_CUDA;
        }
    }
    if (st != DF11_OK)
        return st;
    kernel<<<ls.grid, ls.warps * 32, ls.smem, stream>>>(prm, gp);
    return cudaGetLastError() == cudaSuccess ? DF11_OK : DF11_ERR_CUDA;
}

template <int W, int MINLEN>
df11_status launch_gemv_tokens(const DecodeParams &prm, const GemvParams &gp, int dev, cudaStream_t stream)
{
    if (gp.n_tokens <= 1)
        return launch_gemv<W, MINLEN, 1>(prm, gp, dev, stream);
    if (gp.n_tokens <= 2)
        return launch_gemv<W, MINLEN, 2>(prm, gp, dev, stream);
    if (gp.n_tokens <= 4)
        return launch_gemv<W, MINLEN, 4>(prm, gp, dev, stream);
    return launch_gemv<W, MINLEN, 8>(prm, gp, dev, stream);
}

bool aligned(const void *ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

}  // namespace

extern "C" df11_status df11_decompress_async(const df11_device_block *blk, uint16_t *out_bf16,
                                             uint64_t out_capacity, uint32_t *d_error,
                                             void *stream)
{
    return df11_decompress_async_ctas(blk, out_bf16, out_capacity, d_error, 0, stream);
}

namespace {

// Host-side checks of a device block and the decode parameters for it.
df11_status block_params(const df11_device_block *blk, uint16_t *out_bf16, uint64_t out_limit, uint32_t *d_error,
                         DecodeParams &prm, int &dev)
{
    if (!blk)
        return DF11_ERR_INVALID_ARGUMENT;
    const df11_header &h = blk->hdr;
    const uint32_t W = h.bytes_per_thread;
    if (h.threads_per_chunk != DF11_THREADS_PER_CHUNK || (W != 8 && W != 16))
        return DF11_ERR_INVALID_ARGUMENT;
    if (h.n_elements == 0 || h.n_elements >= (1ull << 32) || h.n_tables < 1 || h.n_tables > 256 ||
        h.total_bits == 0 || out_limit < h.n_elements || h.min_code_len < 1 ||
        h.min_code_len > DF11_MAX_CODE_LEN)
        return DF11_ERR_INVALID_ARGUMENT;
    const uint64_t chunk_bits = (uint64_t)DF11_THREADS_PER_CHUNK * 8 * W;
    if (h.n_chunks != (h.total_bits + chunk_bits - 1) / chunk_bits)
        return DF11_ERR_INVALID_ARGUMENT;
    const uint64_t n_threads = h.n_chunks * DF11_THREADS_PER_CHUNK;
    if (!blk->exp_stream || !blk->gaps || !blk->counts || !blk->chunk_pos || !blk->signmant || !blk->lut)
        return DF11_ERR_INVALID_ARGUMENT;
    if (blk->exp_stream_bytes < n_threads * W + DF11_STREAM_PAD || blk->gaps_bytes < n_threads / 2 ||
        blk->counts_bytes < n_threads ||
        blk->chunk_pos_count < h.n_chunks + 1 ||
        blk->signmant_bytes < (h.n_elements + 15) / 16 * 16 ||
        blk->lut_entries < (uint64_t)h.n_tables * 256)
        return DF11_ERR_INVALID_ARGUMENT;
    if (!aligned(blk->exp_stream, 16) || !aligned(blk->chunk_pos, 16) || !aligned(blk->lut, 16) ||
        !aligned(blk->signmant, 16) || !aligned(blk->gaps, 16) || !aligned(blk->counts, 16) ||
        !aligned(out_bf16, 16) ||
        !aligned(d_error, 4) || !aligned(blk->decode_table, 16))
        return DF11_ERR_INVALID_ARGUMENT;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return DF11_ERR_CUDA;
    prm.stream = blk->exp_stream;
    prm.gaps = blk->gaps;
    prm.counts = blk->counts;
    prm.gaps_limit = n_threads / 2;
    prm.chunk_pos = blk->chunk_pos;
    prm.signmant = blk->signmant;
    prm.lut = blk->lut;
    prm.out = out_bf16;
    prm.err = d_error;
    prm.total_bits = h.total_bits;
    prm.n_chunks = h.n_chunks;
    prm.out_limit = h.n_elements < out_limit ? h.n_elements : out_limit;
    prm.n_tables = h.n_tables;
    prm.min_len = h.min_code_len;
    prm.full_chunks = (uint32_t)(h.total_bits / chunk_bits);
    prm.sched = nullptr;
    prm.multi_src = reinterpret_cast<const uint2 *>(blk->decode_table);
    prm.sums = nullptr;
    prm.first_bad = nullptr;
    return DF11_OK;
}

}  // namespace

extern "C" df11_status df11_decompress_async_ctas(const df11_device_block *blk, uint16_t *out_bf16,
                                                  uint64_t out_capacity, uint32_t *d_error,
                                                  uint32_t max_ctas, void *stream)
{
    return df11_decompress_async_ws(blk, out_bf16, out_capacity, d_error, max_ctas, nullptr, stream);
}

extern "C" df11_status df11_decompress_async_ws(const df11_device_block *blk, uint16_t *out_bf16,
                                                uint64_t out_capacity, uint32_t *d_error,
                                                uint32_t max_ctas, void *workspace, void *stream)
{
    if (!out_bf16 || !aligned(workspace, 16))
        return DF11_ERR_INVALID_ARGUMENT;
    DecodeParams prm;
    int dev = 0;
    const df11_status st = block_params(blk, out_bf16, out_capacity, d_error, prm, dev);
    if (st != DF11_OK)
        return st;
    prm.sched = static_cast<uint32_t *>(workspace);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (blk->hdr.bytes_per_thread == 8)
        return prm.min_len >= 2 ? launch<8, 2>(prm, dev, s, max_ctas) : launch<8, 1>(prm, dev, s, max_ctas);
    return prm.min_len >= 2 ? launch<16, 2>(prm, dev, s, max_ctas) : launch<16, 1>(prm, dev, s, max_ctas);
}

extern "C" df11_status df11_selftest_bounded_wait(uint32_t polls, uint32_t *d_status, void *stream)
{
    if (!d_status || !aligned(d_status, 4) || polls == 0 || polls > 4096)
        return DF11_ERR_INVALID_ARGUMENT;
    bounded_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(polls, d_status);
    return cudaGetLastError() == cudaSuccess ? DF11_OK : DF11_ERR_CUDA;
}

extern "C" df11_status df11_decompress_range_async(const df11_device_block *blk, uint64_t chunk_begin,
                                                   uint64_t chunk_end, uint16_t *out_bf16, uint64_t out_capacity,
                                                   uint32_t *d_error, void *workspace, void *stream)
{
    if (!blk || !out_bf16 || !aligned(workspace, 16) || chunk_begin >= chunk_end ||
        chunk_end > blk->hdr.n_chunks)
        return DF11_ERR_INVALID_ARGUMENT;
    DecodeParams prm;
    int dev = 0;
    const df11_status st = block_params(blk, out_bf16, out_capacity, d_error, prm, dev);
    if (st != DF11_OK)
        return st;
    // The same launch over a block that starts at chunk_begin: chunks are
    // independent given their gaps and positions, and positions (hence the
    // sign|mantissa and output offsets) stay absolute.
    const uint32_t W = blk->hdr.bytes_per_thread;
    const uint64_t chunk_bits = (uint64_t)DF11_THREADS_PER_CHUNK * 8 * W;
    prm.stream += chunk_begin * DF11_THREADS_PER_CHUNK * W;
    prm.gaps += chunk_begin * (DF11_THREADS_PER_CHUNK / 2);
    prm.gaps_limit -= chunk_begin * (DF11_THREADS_PER_CHUNK / 2);   // the thread after the range included
    prm.counts += chunk_begin * DF11_THREADS_PER_CHUNK;
    prm.chunk_pos += chunk_begin;
    prm.total_bits -= chunk_begin * chunk_bits;
    prm.n_chunks = chunk_end - chunk_begin;
    const uint64_t full = prm.total_bits / chunk_bits;
    prm.full_chunks = (uint32_t)(full < prm.n_chunks ? full : prm.n_chunks);
    prm.sched = static_cast<uint32_t *>(workspace);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (W == 8)
        return prm.min_len >= 2 ? launch<8, 2>(prm, dev, s, 0) : launch<8, 1>(prm, dev, s, 0);
    return prm.min_len >= 2 ? launch<16, 2>(prm, dev, s, 0) : launch<16, 1>(prm, dev, s, 0);
}

extern "C" df11_status df11_decode_gemv_async(const df11_device_block *blk, const df11_gemv_matrix *mats,
                                              uint32_t n_mats, uint32_t n_tokens, uint32_t *d_error,
                                              void *workspace, void *stream)
{
    if (!blk || !mats || n_mats == 0 || n_mats > (uint32_t)kGemvMaxMats || n_tokens == 0 || n_tokens > 8 ||
        !aligned(workspace, 16))
        return DF11_ERR_INVALID_ARGUMENT;
    GemvParams gp;
    gp.n_mats = n_mats;
    gp.n_tokens = n_tokens;
    uint64_t start = 0;
    for (uint32_t i = 0; i < n_mats; ++i) {
        const df11_gemv_matrix &m = mats[i];
        if (m.rows == 0 || m.cols == 0 || (m.cols & 7u) || !m.x || !m.y || !aligned(m.x, 16) ||
            !aligned(m.y, 4))
            return DF11_ERR_INVALID_ARGUMENT;
        if (m.rows >= (1ull << 32) || m.cols >= (1ull << 32))
            return DF11_ERR_INVALID_ARGUMENT;
        gp.m[i].start = (uint32_t)start;
        gp.m[i].cols = (uint32_t)m.cols;
        gp.m[i].rows = (uint32_t)m.rows;
        gp.m[i].pad = 0;
        gp.m[i].x = m.x;
        gp.m[i].y = m.y;
        start += m.rows * m.cols;
        if (start >= (1ull << 32))
            return DF11_ERR_INVALID_ARGUMENT;
    }
    if (start != blk->hdr.n_elements)
        return DF11_ERR_INVALID_ARGUMENT;
    DecodeParams prm;
    int dev = 0;
    // no BF16 output: a dummy aligned pointer satisfies the checks and is never written
    const df11_status st =
        block_params(blk, reinterpret_cast<uint16_t *>(16), blk->hdr.n_elements, d_error, prm, dev);
    if (st != DF11_OK)
        return st;
    prm.out = nullptr;
    prm.sched = static_cast<uint32_t *>(workspace);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (blk->hdr.bytes_per_thread == 8)
        return prm.min_len >= 2 ? launch_gemv_tokens<8, 2>(prm, gp, dev, s) : launch_gemv_tokens<8, 1>(prm, gp, dev, s);
    return prm.min_len >= 2 ? launch_gemv_tokens<16, 2>(prm, gp, dev, s) : launch_gemv_tokens<16, 1>(prm, gp, dev, s);
}

extern "C" df11_status df11_decompress_verified_async(const df11_device_block *blk, uint16_t *out_bf16,
                                                      uint64_t out_capacity, uint32_t *d_error,
                                                      const uint32_t *d_sums, uint64_t *d_first_bad,
                                                      void *workspace, void *stream)
{
    if (!out_bf16 || !d_error || !d_sums || !aligned(d_sums, 4) || !aligned(d_first_bad, 8) ||
        !aligned(workspace, 16))
        return DF11_ERR_INVALID_ARGUMENT;
    DecodeParams prm;
    int dev = 0;
    const df11_status st = block_params(blk, out_bf16, out_capacity, d_error, prm, dev);
    if (st != DF11_OK)
        return st;
    prm.sched = static_cast<uint32_t *>(workspace);
    prm.sums = d_sums;
    prm.first_bad = d_first_bad;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (blk->hdr.bytes_per_thread == 8)
        return prm.min_len >= 2 ? launch<8, 2, true>(prm, dev, s, 0) : launch<8, 1, true>(prm, dev, s, 0);
    return prm.min_len >= 2 ? launch<16, 2, true>(prm, dev, s, 0) : launch<16, 1, true>(prm, dev, s, 0);
}
