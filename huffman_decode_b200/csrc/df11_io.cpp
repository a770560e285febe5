// df11_io.cpp -- a DF11 block as one flat byte buffer (for files), with the
// checksum list inside.
//
// The pages store DF11 models as safetensors files and tell users to
// checksum artifacts on download and after every copy ("DFloat11: lossless
// BFloat16 compression", "How to run it in production" and "Failure
// modes").  This is the library's own container for one block:
//
//   offset 0     header (128 bytes): magic "DF11BLK\0", version, header
//                size, the block header, the six array lengths, the number
//                of checksums, the CRC-32C of all of the above;
//   then         exp_stream, gaps, counts, chunk_pos, signmant, lut, each
//                starting on a 16-byte boundary (zero padding between them);
//   then         the checksum list: CRC-32C of every 4096-byte segment of
//                the six arrays (df11_checksum), little-endian uint32.
//
// Reading verifies the header CRC, the sizes, that all padding is zero,
// every segment checksum and the block's structure (df11_validate) before
// handing out pointers into the buffer, so every byte is checked.  Host only; little-endian hosts only (x86-64, aarch64).
#include "df11.h"

#include <cstddef>
#include <cstring>
#include <vector>

namespace {

constexpr char kMagic[8] = {'D', 'F', '1', '1', 'B', 'L', 'K', '\0'};
constexpr uint32_t kVersion = 2;   // 2: the per-thread counts array
constexpr uint64_t kHeaderBytes = 128;

struct FileHeader {
    char magic[8];
    uint32_t version;
    uint32_t header_bytes;
    df11_header hdr;
    uint64_t exp_stream_bytes;
    uint64_t gaps_bytes;
    uint64_t counts_bytes;
    uint64_t chunk_pos_count;
    uint64_t signmant_bytes;
    uint64_t lut_entries;
    uint64_t n_crc;
    uint32_t header_crc;   // CRC-32C of every byte before this field
};
static_assert(sizeof(FileHeader) <= kHeaderBytes, "file header must fit its 128 bytes");
static_assert(sizeof(df11_header) == 48, "block header layout");

uint64_t up16(uint64_t x) { return (x + 15) & ~15ull; }

constexpr int kArrays = 6;

struct Layout {
    uint64_t off[kArrays];   // array offsets
    uint64_t len[kArrays];   // array byte lengths
    uint64_t crc_off;
    uint64_t total;
};

bool layout_of(uint64_t es, uint64_t gb, uint64_t cb, uint64_t cp, uint64_t sm, uint64_t lt, uint64_t n_crc,
               Layout &l)
{
    // reject lengths whose byte counts would overflow
    if (cp > (1ull << 60) || lt > (1ull << 60) || n_crc > (1ull << 60))
        return false;
    const uint64_t len[kArrays] = {es, gb, cb, cp * 4, sm, lt * 2};
    uint64_t at = kHeaderBytes;
    for (int a = 0; a < kArrays; ++a) {
        if (len[a] > (1ull << 61) || at > (1ull << 61))
            return false;
        l.off[a] = at;
        l.len[a] = len[a];
        at = up16(at + len[a]);
    }
    l.crc_off = at;
    l.total = at + n_crc * 4;
    return true;
}

}  // namespace

extern "C" uint64_t df11_serialized_bytes(const df11_host_block *blk)
{
    if (!blk)
        return 0;
    Layout l;
    if (!layout_of(blk->exp_stream_bytes, blk->gaps_bytes, blk->counts_bytes, blk->chunk_pos_count,
                   blk->signmant_bytes, blk->lut_entries, df11_checksum_count(blk), l))
        return 0;
    return l.total;
}

extern "C" df11_status df11_serialize(const df11_host_block *blk, void *buf, uint64_t buf_bytes)
{
    if (!blk || !buf || !blk->exp_stream || !blk->gaps || !blk->counts || !blk->chunk_pos || !blk->signmant ||
        !blk->lut)
        return DF11_ERR_INVALID_ARGUMENT;
    const uint64_t n_crc = df11_checksum_count(blk);
    Layout l;
    if (!layout_of(blk->exp_stream_bytes, blk->gaps_bytes, blk->counts_bytes, blk->chunk_pos_count,
                   blk->signmant_bytes, blk->lut_entries, n_crc, l))
        return DF11_ERR_INVALID_ARGUMENT;
    if (buf_bytes < l.total)
        return DF11_ERR_BUFFER_TOO_SMALL;
    uint8_t *out = static_cast<uint8_t *>(buf);
    std::memset(out, 0, l.total);
    FileHeader fh;
    std::memset(&fh, 0, sizeof(fh));
    std::memcpy(fh.magic, kMagic, sizeof(kMagic));
    fh.version = kVersion;
    fh.header_bytes = (uint32_t)kHeaderBytes;
    fh.hdr = blk->hdr;
    fh.exp_stream_bytes = blk->exp_stream_bytes;
    fh.gaps_bytes = blk->gaps_bytes;
    fh.counts_bytes = blk->counts_bytes;
    fh.chunk_pos_count = blk->chunk_pos_count;
    fh.signmant_bytes = blk->signmant_bytes;
    fh.lut_entries = blk->lut_entries;
    fh.n_crc = n_crc;
    fh.header_crc = df11_crc32c(&fh, offsetof(FileHeader, header_crc));
    std::memcpy(out, &fh, sizeof(fh));
    const void *src[kArrays] = {blk->exp_stream, blk->gaps, blk->counts, blk->chunk_pos, blk->signmant, blk->lut};
    for (int a = 0; a < kArrays; ++a)
        if (l.len[a])
            std::memcpy(out + l.off[a], src[a], l.len[a]);
    std::vector<uint32_t> crc(n_crc);
    const df11_status st = df11_checksum(blk, crc.data(), n_crc);
    if (st != DF11_OK)
        return st;
    if (n_crc)
        std::memcpy(out + l.crc_off, crc.data(), n_crc * 4);
    return DF11_OK;
}

extern "C" df11_status df11_deserialize(const void *buf, uint64_t buf_bytes, df11_host_block *blk,
                                        uint64_t *first_bad)
{
    if (!buf || !blk)
        return DF11_ERR_INVALID_ARGUMENT;
    if (first_bad)
        *first_bad = UINT64_MAX;
    const uint8_t *in = static_cast<const uint8_t *>(buf);
    if (buf_bytes < kHeaderBytes)
        return DF11_ERR_CORRUPT;
    FileHeader fh;
    std::memcpy(&fh, in, sizeof(fh));
    if (std::memcmp(fh.magic, kMagic, sizeof(kMagic)) != 0 || fh.version != kVersion ||
        fh.header_bytes != kHeaderBytes || fh.header_crc != df11_crc32c(&fh, offsetof(FileHeader, header_crc)))
        return DF11_ERR_CORRUPT;
    Layout l;
    if (!layout_of(fh.exp_stream_bytes, fh.gaps_bytes, fh.counts_bytes, fh.chunk_pos_count, fh.signmant_bytes,
                   fh.lut_entries, fh.n_crc, l) ||
        l.total != buf_bytes)
        return DF11_ERR_CORRUPT;
    // every byte is checked: the padding after the header and after each
    // array must be zero (the checksums cover the arrays)
    for (uint64_t i = offsetof(FileHeader, header_crc) + 4; i < kHeaderBytes; ++i)
        if (in[i])
            return DF11_ERR_CORRUPT;
    for (int a = 0; a < kArrays; ++a) {
        const uint64_t end = l.off[a] + l.len[a];
        const uint64_t next = a < kArrays - 1 ? l.off[a + 1] : l.crc_off;
        for (uint64_t i = end; i < next; ++i)
            if (in[i])
                return DF11_ERR_CORRUPT;
    }
    // pointers into the buffer (the library only reads through them)
    df11_host_block b;
    b.hdr = fh.hdr;
    b.exp_stream = const_cast<uint8_t *>(in + l.off[0]);
    b.exp_stream_bytes = fh.exp_stream_bytes;
    b.gaps = const_cast<uint8_t *>(in + l.off[1]);
    b.gaps_bytes = fh.gaps_bytes;
    b.counts = const_cast<uint8_t *>(in + l.off[2]);
    b.counts_bytes = fh.counts_bytes;
    b.chunk_pos = reinterpret_cast<uint32_t *>(const_cast<uint8_t *>(in + l.off[3]));
    b.chunk_pos_count = fh.chunk_pos_count;
    b.signmant = const_cast<uint8_t *>(in + l.off[4]);
    b.signmant_bytes = fh.signmant_bytes;
    b.lut = reinterpret_cast<uint16_t *>(const_cast<uint8_t *>(in + l.off[5]));
    b.lut_entries = fh.lut_entries;
    if (df11_checksum_count(&b) != fh.n_crc)
        return DF11_ERR_CORRUPT;
    std::vector<uint32_t> crc(fh.n_crc);
    df11_status st = df11_checksum(&b, crc.data(), fh.n_crc);
    if (st != DF11_OK)
        return DF11_ERR_CORRUPT;
    for (uint64_t k = 0; k < fh.n_crc; ++k) {
        uint32_t want;
        std::memcpy(&want, in + l.crc_off + 4 * k, 4);
        if (want != crc[k]) {
            if (first_bad)
                *first_bad = k;
            return DF11_ERR_CORRUPT;
        }
    }
    st = df11_validate(&b);
    if (st != DF11_OK)
        return DF11_ERR_CORRUPT;
    *blk = b;
    return DF11_OK;
}
