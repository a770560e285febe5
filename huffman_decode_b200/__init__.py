"""DFloat11 exponent-stream codec for NVIDIA B200 (sm_100a).

Lossless BF16 weight compression: the exponent byte of every weight is
canonical-Huffman coded (length cap 16), the sign|mantissa byte is kept raw,
and one GPU launch per block rebuilds the bit-exact BF16 matrices.  The work
happens in libdf11.so (C ABI in include/df11.h); this package only binds it.
"""
from .df11 import (  # noqa: F401
    CRC_SEGMENT_BYTES, DEVERR_BOUNDS, DEVERR_BAD_CODE, DEVERR_BAD_POS, DEVERR_CHECKSUM, DEVERR_COUNT, DEVERR_MISMATCH,
    DEVERR_TIMEOUT, DF11Error, checksum, checksum_count, checksum_device, crc32c, verify_device,
    DeviceBlock, EXPORTED_SYMBOLS, LAYOUTS, HostBlock, PinnedHostBlock, Pipeline, build_codebook,
    decode_gemv_async, SCHED_WORKSPACE_BYTES, sched_workspace, decompress_range_async,
    selftest_bounded_wait,
    build_codebook_from_histogram, build_decode_table, chunk_sums, decompress_verified_async, compress, compress_device, compress_device_noalloc,
    compress_device_scratch_bytes,
    compress_sizes, decompress_async, histogram_device, library_path, load_library, preferred_bytes_per_thread,
    validate,
)
