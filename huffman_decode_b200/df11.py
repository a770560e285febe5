"""Python binding of the DF11 C ABI (include/df11.h): argument marshalling only.

Every step of the codec runs in libdf11.so -- the host compressor in C++,
the decode in the sm_100a kernel.  torch is used for device memory and
streams; numpy for host buffers.  Names follow the C calls:

    cb  = build_codebook(mats, max_code_len=16)
    hb  = compress(cb, mats)               # 32 threads x 16 bytes per chunk
    validate(hb)
    db  = hb.to_device("cuda")
    decompress_async(db, out, error=None, stream=None)
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field

import numpy as np

from . import build as _build

# ------------------------------------------------------------ constants

DF11_OK = 0
DF11_ERR_INVALID_ARGUMENT = 1
DF11_ERR_BUFFER_TOO_SMALL = 2
DF11_ERR_CORRUPT = 4
STATUS_NAMES = {
    0: "DF11_OK", 1: "DF11_ERR_INVALID_ARGUMENT", 2: "DF11_ERR_BUFFER_TOO_SMALL",
    3: "DF11_ERR_OVERFLOW", 4: "DF11_ERR_CORRUPT", 5: "DF11_ERR_CUDA", 6: "DF11_ERR_TIMEOUT",
}
DEVERR_COUNT = 0x1
DEVERR_BAD_CODE = 0x2
DEVERR_BAD_POS = 0x4
DEVERR_TIMEOUT = 0x8
DEVERR_MISMATCH = 0x10
DEVERR_CHECKSUM = 0x20
DEVERR_BOUNDS = 0x40
MAX_CODE_LEN = 16
STREAM_PAD = 16
THREADS_PER_CHUNK = 32
BYTES_PER_THREAD = 16           # 128-bit slices: fastest layout on B200
LAYOUTS = ((32, 8), (32, 16))   # (threads_per_chunk, bytes_per_thread) the library decodes
ARRAYS = ("exp_stream", "gaps", "counts", "chunk_pos", "signmant", "lut")   # artifact order

EXPORTED_SYMBOLS = (
    "df11_build_codebook", "df11_build_codebook_from_histogram", "df11_compress_sizes",
    "df11_compress", "df11_validate", "df11_decompress_async", "df11_status_string",
    "df11_histogram_device", "df11_compress_device_scratch_bytes", "df11_compress_device",
    "df11_compress_device_noalloc", "df11_decompress_async_ctas", "df11_pipeline_create",
    "df11_pipeline_destroy", "df11_pipeline_upload", "df11_pipeline_decode", "df11_pipeline_acquire",
    "df11_pipeline_release", "df11_checksum_count", "df11_crc32c", "df11_checksum",
    "df11_checksum_device_async", "df11_verify_device_async", "df11_pipeline_verify",
    "df11_decode_gemv_async", "df11_decompress_async_ws", "df11_decompress_range_async",
    "df11_selftest_bounded_wait", "df11_serialized_bytes", "df11_serialize", "df11_deserialize",
    "df11_build_decode_table", "df11_chunk_sums", "df11_decompress_verified_async",
    "df11_preferred_bytes_per_thread",
)
SCHED_WORKSPACE_BYTES = 2048
CRC_SEGMENT_BYTES = 4096
NOALLOC_SCRATCH_BYTES = 1 << 20
NOALLOC_MAX_ELEMENTS = 715816960
DECODE_TABLE_ENTRIES = 2048
DECODE_TABLE_WINDOW_BITS = 11


class DF11Error(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = status
        super().__init__(f"{call} returned {STATUS_NAMES.get(status, status)}")


# ------------------------------------------------------- C structures

class Codebook(ctypes.Structure):
    _fields_ = [
        ("histogram", ctypes.c_uint64 * 256),
        ("code", ctypes.c_uint32 * 256),
        ("code_len", ctypes.c_uint8 * 256),
        ("max_code_len", ctypes.c_uint32),
        ("n_symbols", ctypes.c_uint32),
        ("n_tables", ctypes.c_uint32),
        ("longest_code", ctypes.c_uint32),
        ("n_elements", ctypes.c_uint64),
        ("total_bits", ctypes.c_uint64),
        ("lut", ctypes.c_uint16 * (256 * 256)),
    ]

    def lengths(self) -> np.ndarray:
        return np.ctypeslib.as_array(self.code_len).copy()

    def codes(self) -> np.ndarray:
        return np.ctypeslib.as_array(self.code).copy()

    def counts(self) -> np.ndarray:
        return np.ctypeslib.as_array(self.histogram).copy()

    def tables(self) -> np.ndarray:
        return np.ctypeslib.as_array(self.lut)[: self.n_tables * 256].copy()


class Layout(ctypes.Structure):
    _fields_ = [("threads_per_chunk", ctypes.c_uint32), ("bytes_per_thread", ctypes.c_uint32)]


class Sizes(ctypes.Structure):
    _fields_ = [
        ("n_chunks", ctypes.c_uint64), ("n_threads", ctypes.c_uint64),
        ("exp_stream_bytes", ctypes.c_uint64), ("gaps_bytes", ctypes.c_uint64),
        ("counts_bytes", ctypes.c_uint64),
        ("chunk_pos_count", ctypes.c_uint64), ("signmant_bytes", ctypes.c_uint64),
        ("lut_entries", ctypes.c_uint64),
    ]


class Header(ctypes.Structure):
    _fields_ = [
        ("max_code_len", ctypes.c_uint32), ("threads_per_chunk", ctypes.c_uint32),
        ("bytes_per_thread", ctypes.c_uint32), ("n_tables", ctypes.c_uint32),
        ("min_code_len", ctypes.c_uint32), ("reserved", ctypes.c_uint32),
        ("total_bits", ctypes.c_uint64), ("n_elements", ctypes.c_uint64),
        ("n_chunks", ctypes.c_uint64),
    ]


class _Block(ctypes.Structure):
    _fields_ = [
        ("hdr", Header),
        ("exp_stream", ctypes.c_void_p), ("exp_stream_bytes", ctypes.c_uint64),
        ("gaps", ctypes.c_void_p), ("gaps_bytes", ctypes.c_uint64),
        ("counts", ctypes.c_void_p), ("counts_bytes", ctypes.c_uint64),
        ("chunk_pos", ctypes.c_void_p), ("chunk_pos_count", ctypes.c_uint64),
        ("signmant", ctypes.c_void_p), ("signmant_bytes", ctypes.c_uint64),
        ("lut", ctypes.c_void_p), ("lut_entries", ctypes.c_uint64),
        ("decode_table", ctypes.c_void_p),   # df11_device_block only (host calls ignore it)
    ]


# ------------------------------------------------------------ loading

_lib = None


def load_library(path: str | None = None):
    """Loads libdf11.so -- or libdf11_checked.so, the build whose decode
    kernel checks its bounds at run time, when the environment has
    DF11_CHECKED=1 -- building it first if a source is newer.  Raises if the
    library cannot be built or loaded: there is no fallback path."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    if path is None:
        path = _build.build(checked=os.environ.get("DF11_CHECKED") == "1")
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    U32 = ctypes.c_uint32
    U64 = ctypes.c_uint64
    S = ctypes.c_int
    for name, res, args in (
        ("df11_build_codebook", S, [P, P, U32, U32, P]),
        ("df11_compress_sizes", S, [P, P, P]),
        ("df11_compress", S, [P, P, P, P, U32, P]),
        ("df11_validate", S, [P]),
        ("df11_decompress_async", S, [P, P, U64, P, P]),
        ("df11_status_string", ctypes.c_char_p, [S]),
        ("df11_build_codebook_from_histogram", S, [P, U32, P]),
        ("df11_histogram_device", S, [P, U64, P, P]),
        ("df11_compress_device_scratch_bytes", U64, [U64]),
        ("df11_compress_device", S, [P, P, P, U64, P, P, U64, P, P]),
        ("df11_compress_device_noalloc", S, [P, P, P, U64, P, P, P]),
        ("df11_decompress_async_ctas", S, [P, P, U64, P, U32, P]),
        ("df11_pipeline_create", S, [U32, P]),
        ("df11_pipeline_destroy", S, [P]),
        ("df11_pipeline_upload", S, [P, U32, P, P, P]),
        ("df11_pipeline_decode", S, [P, U32, P, P, U64, P, U32, P, P]),
        ("df11_pipeline_acquire", S, [P, U32, P]),
        ("df11_pipeline_release", S, [P, U32, P]),
        ("df11_checksum_count", U64, [P]),
        ("df11_crc32c", U32, [P, U64]),
        ("df11_checksum", S, [P, P, U64]),
        ("df11_checksum_device_async", S, [P, P, U64, P]),
        ("df11_verify_device_async", S, [P, P, U64, P, P, P]),
        ("df11_pipeline_verify", S, [P, U32, P, P, U64, P, P, P]),
        ("df11_decode_gemv_async", S, [P, P, U32, U32, P, P, P]),
        ("df11_decompress_async_ws", S, [P, P, U64, P, U32, P, P]),
        ("df11_decompress_range_async", S, [P, U64, U64, P, U64, P, P, P]),
        ("df11_selftest_bounded_wait", S, [U32, P, P]),
        ("df11_serialized_bytes", U64, [P]),
        ("df11_serialize", S, [P, P, U64]),
        ("df11_deserialize", S, [P, U64, P, P]),
        ("df11_build_decode_table", S, [P, U32, U32, P]),
        ("df11_chunk_sums", S, [P, P, U64]),
        ("df11_decompress_verified_async", S, [P, P, U64, P, P, P, P, P]),
        ("df11_preferred_bytes_per_thread", U32, [P, U32]),
    ):
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path == _build.LIB_PATH:
        _lib = lib
    return lib


def library_path() -> str:
    """Path of the library this process uses (the checked one when
    DF11_CHECKED=1)."""
    return _build.CHECKED_LIB_PATH if os.environ.get("DF11_CHECKED") == "1" else _build.LIB_PATH


def _check(status: int, call: str):
    if status != DF11_OK:
        raise DF11Error(status, call)


def _mats_args(mats):
    arrs = [np.ascontiguousarray(m, dtype=np.uint16).reshape(-1) for m in mats]
    ptrs = (ctypes.c_void_p * len(arrs))(*[a.ctypes.data for a in arrs])
    numel = (ctypes.c_uint64 * len(arrs))(*[a.size for a in arrs])
    return arrs, ptrs, numel


# ------------------------------------------------------------ host calls

def build_codebook(mats, max_code_len: int = MAX_CODE_LEN) -> Codebook:
    """df11_build_codebook over a list of BF16 bit-pattern arrays (uint16)."""
    arrs, ptrs, numel = _mats_args(mats)
    cb = Codebook()
    _check(load_library().df11_build_codebook(ptrs, numel, len(arrs), max_code_len,
                                               ctypes.byref(cb)), "df11_build_codebook")
    return cb


def preferred_bytes_per_thread(cb: Codebook, sm_count: int | None = None) -> int:
    """df11_preferred_bytes_per_thread: the slice width (8 or 16 bytes per
    thread) this library decodes the block fastest with on a GPU of sm_count
    SMs (default: the current CUDA device's)."""
    if sm_count is None:
        import torch
        sm_count = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    v = int(load_library().df11_preferred_bytes_per_thread(ctypes.byref(cb), int(sm_count)))
    if v == 0:
        raise ValueError("empty codebook or sm_count == 0")
    return v


def compress_sizes(cb: Codebook, threads_per_chunk: int = THREADS_PER_CHUNK,
                   bytes_per_thread: int = BYTES_PER_THREAD) -> Sizes:
    z = Sizes()
    ly = Layout(threads_per_chunk, bytes_per_thread)
    _check(load_library().df11_compress_sizes(ctypes.byref(cb), ctypes.byref(ly),
                                              ctypes.byref(z)), "df11_compress_sizes")
    return z


@dataclass
class HostBlock:
    """A compressed block in host memory (numpy arrays owned by Python)."""
    header: Header
    exp_stream: np.ndarray
    gaps: np.ndarray
    counts: np.ndarray
    chunk_pos: np.ndarray
    signmant: np.ndarray
    lut: np.ndarray
    matrix_numel: list = field(default_factory=list)

    def c_struct(self) -> _Block:
        b = _Block()
        b.hdr = self.header
        for name in ARRAYS:
            a = getattr(self, name)
            setattr(b, name, a.ctypes.data)
        b.exp_stream_bytes = self.exp_stream.nbytes
        b.gaps_bytes = self.gaps.nbytes
        b.counts_bytes = self.counts.nbytes
        b.chunk_pos_count = self.chunk_pos.size
        b.signmant_bytes = self.signmant.nbytes
        b.lut_entries = self.lut.size
        return b

    @property
    def n_elements(self) -> int:
        return int(self.header.n_elements)

    def compressed_bytes(self) -> int:
        """Bytes a decode reads: stream, gaps, counts, positions,
        sign|mantissa, tables."""
        return int(sum(getattr(self, n).nbytes for n in ARRAYS))

    def arrays(self):
        return {n: getattr(self, n) for n in ARRAYS}

    def to_bytes(self) -> bytes:
        """df11_serialize: the block as one flat buffer (header, the six
        arrays, the CRC-32C checksum list).  matrix_numel is not stored."""
        lib = load_library()
        b = self.c_struct()
        n = int(lib.df11_serialized_bytes(ctypes.byref(b)))
        if n == 0:
            raise DF11Error(DF11_ERR_INVALID_ARGUMENT, "df11_serialized_bytes")
        buf = np.empty(n, dtype=np.uint8)
        _check(lib.df11_serialize(ctypes.byref(b), buf.ctypes.data, n), "df11_serialize")
        return buf.tobytes()

    @staticmethod
    def from_bytes(data) -> "HostBlock":
        """df11_deserialize: checks the header, sizes, every segment checksum
        and the block's structure, then copies the arrays out.  Raises
        DF11Error (with .first_bad_segment, or None) when anything is off."""
        src = np.frombuffer(data, dtype=np.uint8)
        store = np.zeros(max(1, src.size), dtype=np.uint8)   # a real pointer even when empty
        store[: src.size] = src
        buf = store[: src.size]
        blk = _Block()
        first = ctypes.c_uint64(0)
        st = load_library().df11_deserialize(store.ctypes.data, src.size, ctypes.byref(blk),
                                             ctypes.byref(first))
        if st != DF11_OK:
            e = DF11Error(st, "df11_deserialize")
            e.first_bad_segment = None if first.value == (1 << 64) - 1 else int(first.value)
            raise e
        base = store.ctypes.data

        def take(ptr, nbytes, dtype):
            off = int(ptr) - base
            return buf[off:off + nbytes].view(dtype).copy()

        return HostBlock(header=Header.from_buffer_copy(blk.hdr),
                         exp_stream=take(blk.exp_stream, blk.exp_stream_bytes, np.uint8),
                         gaps=take(blk.gaps, blk.gaps_bytes, np.uint8),
                         counts=take(blk.counts, blk.counts_bytes, np.uint8),
                         chunk_pos=take(blk.chunk_pos, 4 * blk.chunk_pos_count, np.uint32),
                         signmant=take(blk.signmant, blk.signmant_bytes, np.uint8),
                         lut=take(blk.lut, 2 * blk.lut_entries, np.uint16))

    def save(self, path) -> None:
        with open(path, "wb") as f:
            f.write(self.to_bytes())

    @staticmethod
    def load(path) -> "HostBlock":
        with open(path, "rb") as f:
            return HostBlock.from_bytes(f.read())

    def pinned(self) -> "PinnedHostBlock":
        """A copy of the block in page-locked host memory (torch pinned
        tensors), so host -> device copies of it run asynchronously."""
        import torch
        t = {n: torch.from_numpy(a.view(np.uint8).reshape(-1)).pin_memory()
             for n, a in self.arrays().items()}
        return PinnedHostBlock(header=self.header, tensors=t,
                               sizes={n: a.nbytes for n, a in self.arrays().items()},
                               matrix_numel=list(self.matrix_numel))

    def to_device(self, device="cuda", pin: bool = False, decode_table: bool = True) -> "DeviceBlock":
        """The block's arrays copied to the GPU, plus (decode_table=True) the
        decoder's multi-code table built from its lookup tables
        (df11_build_decode_table), so decode launches copy it instead of
        building it in every CTA."""
        import torch
        t = {}
        for name, a in self.arrays().items():
            src = torch.from_numpy(a.view(np.uint8))
            if pin:
                src = src.pin_memory()
            t[name] = src.to(device, non_blocking=pin)
        db = DeviceBlock(header=self.header, tensors=t,
                         sizes={n: a.nbytes for n, a in self.arrays().items()},
                         matrix_numel=list(self.matrix_numel))
        if decode_table:
            db.attach_decode_table(self.lut)
        return db


def build_decode_table(lut, n_tables: int, min_code_len: int) -> np.ndarray:
    """df11_build_decode_table: the decoder's 2048-entry multi-code table
    (uint64 entries) for a block's lookup tables."""
    lut = np.ascontiguousarray(lut, dtype=np.uint16)
    if lut.size < int(n_tables) * 256:
        raise ValueError("lut holds fewer than n_tables * 256 entries")
    out = np.empty(DECODE_TABLE_ENTRIES, np.uint64)
    _check(load_library().df11_build_decode_table(lut.ctypes.data, int(n_tables), int(min_code_len),
                                                  out.ctypes.data), "df11_build_decode_table")
    return out


def _struct_from_tensors(header, tensors, sizes, decode_table=None) -> _Block:
    b = _Block()
    b.hdr = header
    b.decode_table = decode_table.data_ptr() if decode_table is not None else None
    for name, t in tensors.items():
        setattr(b, name, t.data_ptr())
    b.exp_stream_bytes = sizes["exp_stream"]
    b.gaps_bytes = sizes["gaps"]
    b.counts_bytes = sizes["counts"]
    b.chunk_pos_count = sizes["chunk_pos"] // 4
    b.signmant_bytes = sizes["signmant"]
    b.lut_entries = sizes["lut"] // 2
    return b


@dataclass
class PinnedHostBlock:
    """A compressed block whose arrays are pinned host (uint8) tensors."""
    header: Header
    tensors: dict
    sizes: dict
    matrix_numel: list = field(default_factory=list)

    def c_struct(self) -> _Block:
        return _struct_from_tensors(self.header, self.tensors, self.sizes)

    @property
    def n_elements(self) -> int:
        return int(self.header.n_elements)

    def compressed_bytes(self) -> int:
        return int(sum(self.sizes.values()))


def compress(cb: Codebook, mats, threads_per_chunk: int = THREADS_PER_CHUNK,
             bytes_per_thread: int = BYTES_PER_THREAD) -> HostBlock:
    """df11_compress into freshly allocated numpy buffers of the exact sizes."""
    arrs, ptrs, numel = _mats_args(mats)
    z = compress_sizes(cb, threads_per_chunk, bytes_per_thread)
    hb = HostBlock(
        header=Header(),
        exp_stream=np.empty(z.exp_stream_bytes, np.uint8),
        gaps=np.empty(z.gaps_bytes, np.uint8),
        counts=np.empty(z.counts_bytes, np.uint8),
        chunk_pos=np.empty(z.chunk_pos_count, np.uint32),
        signmant=np.empty(z.signmant_bytes, np.uint8),
        lut=np.empty(z.lut_entries, np.uint16),
        matrix_numel=[a.size for a in arrs],
    )
    blk = hb.c_struct()
    ly = Layout(threads_per_chunk, bytes_per_thread)
    _check(load_library().df11_compress(ctypes.byref(cb), ctypes.byref(ly), ptrs, numel,
                                        len(arrs), ctypes.byref(blk)), "df11_compress")
    hb.header = blk.hdr
    return hb


def validate(hb: HostBlock) -> int:
    """df11_validate; returns the status code (0 = structurally sound)."""
    blk = hb.c_struct()
    return int(load_library().df11_validate(ctypes.byref(blk)))


# ------------------------------------------------------------ device call

@dataclass
class DeviceBlock:
    """The block's arrays as uint8 torch tensors on one GPU, and optionally
    the decoder's multi-code table (a uint8 tensor of 16 KB; not part of the
    artifact, built from its tables)."""
    header: Header
    tensors: dict
    sizes: dict
    matrix_numel: list = field(default_factory=list)
    decode_table: object = None

    def c_struct(self) -> _Block:
        return _struct_from_tensors(self.header, self.tensors, self.sizes, self.decode_table)

    def attach_decode_table(self, lut) -> None:
        """Builds the multi-code table for this block's header and host
        copy of its tables, and keeps it on the block's device."""
        import torch
        tab = build_decode_table(lut, self.header.n_tables, self.header.min_code_len)
        dev = self.tensors["lut"].device
        self.decode_table = torch.from_numpy(tab.view(np.uint8)).to(dev)

    @property
    def n_elements(self) -> int:
        return int(self.header.n_elements)

    def compressed_bytes(self) -> int:
        return int(sum(self.sizes.values()))

    @staticmethod
    def staging(sizes: dict, device="cuda") -> "DeviceBlock":
        """Empty device arrays of the given byte sizes (a pipeline slot's
        staging area); the header is filled by the upload that uses it."""
        import torch
        t = {n: torch.empty(max(int(b), 16), dtype=torch.uint8, device=device)
             for n, b in sizes.items()}
        return DeviceBlock(header=Header(), tensors=t, sizes={n: int(b) for n, b in sizes.items()})


_WORKSPACES: dict = {}


def sched_workspace(device, stream_handle: int):
    """The scheduling workspace this module uses for launches on one stream
    (DF11_SCHED_WORKSPACE_BYTES of zeroed device memory, created on first
    use).  Launches on one stream run one after another, so they can share
    it; launches on different streams get different workspaces.  Creation
    waits for the zero fill (it runs on torch's current stream, the launches
    on theirs), so make the first launch on a stream outside graph capture."""
    import torch
    dev = torch.device(device)
    key = (dev.index if dev.index is not None else torch.cuda.current_device(), int(stream_handle))
    ws = _WORKSPACES.get(key)
    if ws is None:
        ws = _zeroed_workspace(torch.device("cuda", key[0]))
        _WORKSPACES[key] = ws
    return ws


def _zeroed_workspace(device):
    import torch
    ws = torch.zeros(SCHED_WORKSPACE_BYTES, dtype=torch.uint8, device=device)
    torch.cuda.synchronize(device)
    return ws


def _workspace_ptr(workspace, device, handle):
    """True: this stream's workspace; False/None: static chunk schedule; a
    tensor: that workspace."""
    if workspace is True:
        return sched_workspace(device, handle).data_ptr()
    if workspace is None or workspace is False:
        return None
    if workspace.numel() * workspace.element_size() < SCHED_WORKSPACE_BYTES or not workspace.is_cuda:
        raise ValueError(f"workspace must be >= {SCHED_WORKSPACE_BYTES} bytes of CUDA memory")
    return workspace.data_ptr()


def decompress_async(db: DeviceBlock, out, error=None, stream=None, c_block=None,
                     capacity: int | None = None, max_ctas: int = 0, workspace=True) -> None:
    """df11_decompress_async_ws: one kernel launch decoding the whole block
    into `out` (a CUDA tensor of >= n_elements 16-bit elements, e.g. bfloat16
    or int16) on `stream` (torch.cuda.Stream, raw handle, or the current
    stream).  `error` is an optional int32 CUDA tensor the kernel ORs error
    bits into; `capacity` (default out.numel()) is the element count the
    kernel may write; `max_ctas` > 0 caps the launch; `workspace` (default:
    one per stream) selects the dynamic chunk schedule, False the static
    one."""
    if out.element_size() != 2 or not out.is_cuda or not out.is_contiguous():
        raise ValueError("out must be a contiguous CUDA tensor of 16-bit elements")
    handle = _raw_stream(stream, out.device)
    blk = c_block if c_block is not None else db.c_struct()
    err_ptr = error.data_ptr() if error is not None else None
    cap = out.numel() if capacity is None else min(int(capacity), out.numel())
    _check(load_library().df11_decompress_async_ws(ctypes.byref(blk), out.data_ptr(), cap, err_ptr,
                                                   int(max_ctas), _workspace_ptr(workspace, out.device, handle),
                                                   handle), "df11_decompress_async_ws")


def selftest_bounded_wait(polls: int, status, stream=None) -> None:
    """df11_selftest_bounded_wait: one warp polls a barrier nothing arrives
    on `polls` times and writes the timeout status into `status` (int32 CUDA
    tensor)."""
    _check(load_library().df11_selftest_bounded_wait(int(polls), status.data_ptr(),
                                                     _raw_stream(stream, status.device)),
           "df11_selftest_bounded_wait")


def decompress_range_async(db: DeviceBlock, chunk_begin: int, chunk_end: int, out, error=None,
                           stream=None, c_block=None, workspace=True) -> None:
    """df11_decompress_range_async: decodes chunks [chunk_begin, chunk_end) of
    the block into their part of `out` (the whole block's output buffer,
    16-bit CUDA tensor); `workspace` as for decompress_async."""
    if out.element_size() != 2 or not out.is_cuda or not out.is_contiguous():
        raise ValueError("out must be a contiguous CUDA tensor of 16-bit elements")
    handle = _raw_stream(stream, out.device)
    blk = c_block if c_block is not None else db.c_struct()
    err_ptr = error.data_ptr() if error is not None else None
    _check(load_library().df11_decompress_range_async(ctypes.byref(blk), int(chunk_begin), int(chunk_end),
                                                      out.data_ptr(), out.numel(), err_ptr,
                                                      _workspace_ptr(workspace, out.device, handle), handle),
           "df11_decompress_range_async")


# ------------------------------------------------------- GPU-side compressor

def _stream_handle(stream, device):
    import torch
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def build_codebook_from_histogram(hist, max_code_len: int = MAX_CODE_LEN) -> Codebook:
    """df11_build_codebook_from_histogram (host) from 256 exponent counts."""
    h = np.ascontiguousarray(np.asarray(hist).reshape(-1)[:256], dtype=np.uint64)
    if h.size != 256:
        raise ValueError("histogram needs 256 bins")
    cb = Codebook()
    _check(load_library().df11_build_codebook_from_histogram(h.ctypes.data, max_code_len,
                                                              ctypes.byref(cb)),
           "df11_build_codebook_from_histogram")
    return cb


def histogram_device(d_in, stream=None):
    """df11_histogram_device: exponent histogram of a contiguous CUDA tensor of
    16-bit elements; returns an int64 CUDA tensor of 256 counts."""
    import torch
    if d_in.element_size() != 2 or not d_in.is_cuda or not d_in.is_contiguous():
        raise ValueError("d_in must be a contiguous CUDA tensor of 16-bit elements")
    hist = torch.zeros(256, dtype=torch.int64, device=d_in.device)
    _check(load_library().df11_histogram_device(d_in.data_ptr(), d_in.numel(), hist.data_ptr(),
                                                _stream_handle(stream, d_in.device)),
           "df11_histogram_device")
    return hist


def compress_device_scratch_bytes(n_elements: int) -> int:
    return int(load_library().df11_compress_device_scratch_bytes(n_elements))


def compress_device(cb: Codebook, d_in, threads_per_chunk: int = THREADS_PER_CHUNK,
                    bytes_per_thread: int = BYTES_PER_THREAD, stream=None, error=None,
                    scratch=None) -> DeviceBlock:
    """df11_compress_device: encodes a contiguous CUDA tensor of BF16 bit
    patterns (the block's matrices concatenated) into freshly allocated device
    arrays; the codebook's tables are copied into the block's lut array."""
    import torch
    if d_in.element_size() != 2 or not d_in.is_cuda or not d_in.is_contiguous():
        raise ValueError("d_in must be a contiguous CUDA tensor of 16-bit elements")
    dev = d_in.device
    z = compress_sizes(cb, threads_per_chunk, bytes_per_thread)
    sizes = {"exp_stream": z.exp_stream_bytes, "gaps": z.gaps_bytes, "counts": z.counts_bytes,
             "chunk_pos": z.chunk_pos_count * 4, "signmant": z.signmant_bytes,
             "lut": z.lut_entries * 2}
    t = {name: torch.empty(nbytes, dtype=torch.uint8, device=dev) for name, nbytes in sizes.items()}
    t["lut"].copy_(torch.from_numpy(cb.tables().view(np.uint8)))
    if scratch is None:
        scratch = torch.empty(max(compress_device_scratch_bytes(d_in.numel()), 16),
                              dtype=torch.uint8, device=dev)
    db = DeviceBlock(header=Header(), tensors=t, sizes=sizes, matrix_numel=[d_in.numel()])
    blk = db.c_struct()
    ly = Layout(threads_per_chunk, bytes_per_thread)
    _check(load_library().df11_compress_device(
        ctypes.byref(cb), ctypes.byref(ly), d_in.data_ptr(), d_in.numel(), ctypes.byref(blk),
        scratch.data_ptr(), scratch.numel(), error.data_ptr() if error is not None else None,
        _stream_handle(stream, dev)), "df11_compress_device")
    db.header = blk.hdr
    db.attach_decode_table(cb.tables())
    return db


def compress_device_noalloc(cb: Codebook, d_in, threads_per_chunk: int = THREADS_PER_CHUNK,
                            bytes_per_thread: int = BYTES_PER_THREAD, stream=None,
                            error=None) -> DeviceBlock:
    """df11_compress_device_noalloc: the GPU compressor for callers that cannot
    let a library allocate device memory (a runtime that reserves the GPU for
    its own pool, code that must not call cudaFree).  Its work space is one
    fixed device array inside the library, shared by every call, so calls
    must not overlap on the GPU.  The output arrays here are still allocated
    by this Python wrapper through torch; a C caller passes its own."""
    import torch
    if d_in.element_size() != 2 or not d_in.is_cuda or not d_in.is_contiguous():
        raise ValueError("d_in must be a contiguous CUDA tensor of 16-bit elements")
    dev = d_in.device
    z = compress_sizes(cb, threads_per_chunk, bytes_per_thread)
    sizes = {"exp_stream": z.exp_stream_bytes, "gaps": z.gaps_bytes, "counts": z.counts_bytes,
             "chunk_pos": z.chunk_pos_count * 4, "signmant": z.signmant_bytes,
             "lut": z.lut_entries * 2}
    t = {name: torch.empty(nbytes, dtype=torch.uint8, device=dev) for name, nbytes in sizes.items()}
    t["lut"].copy_(torch.from_numpy(cb.tables().view(np.uint8)))
    db = DeviceBlock(header=Header(), tensors=t, sizes=sizes, matrix_numel=[d_in.numel()])
    blk = db.c_struct()
    ly = Layout(threads_per_chunk, bytes_per_thread)
    _check(load_library().df11_compress_device_noalloc(
        ctypes.byref(cb), ctypes.byref(ly), d_in.data_ptr(), d_in.numel(), ctypes.byref(blk),
        error.data_ptr() if error is not None else None, _stream_handle(stream, dev)),
        "df11_compress_device_noalloc")
    db.header = blk.hdr
    db.attach_decode_table(cb.tables())
    return db


# ------------------------------------------------------- streamed decoding

class Pipeline:
    """df11_pipeline_*: event ordering of upload -> decode -> consume over
    caller streams and `n_slots` slots (see include/df11.h).  The C pipeline
    owns CUDA events only; this object also keeps one decode scheduling
    workspace per slot (device memory, allocated on the first decode of the
    slot); staging blocks and outputs belong to the caller."""

    def __init__(self, n_slots: int = 2):
        self._lib = load_library()
        h = ctypes.c_void_p()
        _check(self._lib.df11_pipeline_create(int(n_slots), ctypes.byref(h)), "df11_pipeline_create")
        self._h = h
        self.n_slots = int(n_slots)
        self._ws = {}

    def close(self):
        if self._h is not None and self._h.value:
            _check(self._lib.df11_pipeline_destroy(self._h), "df11_pipeline_destroy")
        self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def upload(self, slot: int, src, dst: "DeviceBlock", stream) -> None:
        """Host -> device copies of `src` (HostBlock or PinnedHostBlock) into
        the staging block `dst`; dst takes src's header."""
        s = src.c_struct()
        # the destination offers its whole capacity; afterwards it describes
        # the uploaded block (its header and array sizes)
        d = _struct_from_tensors(dst.header, dst.tensors, {n: t.numel() for n, t in dst.tensors.items()})
        _check(self._lib.df11_pipeline_upload(self._h, int(slot), ctypes.byref(s), ctypes.byref(d),
                                              _raw_stream(stream)), "df11_pipeline_upload")
        dst.header = src.header
        dst.sizes = dict(src.sizes)
        dst.matrix_numel = list(src.matrix_numel)
        dst._keep = src   # the copy reads src after this call returns

    def decode(self, slot: int, blk: "DeviceBlock", out, error=None, stream=None,
               max_ctas: int = 0, workspace=True) -> None:
        """Decode stage of `slot`; `workspace` True = the slot's own
        scheduling workspace (claimed tail), False = the static schedule."""
        if out.element_size() != 2 or not out.is_cuda or not out.is_contiguous():
            raise ValueError("out must be a contiguous CUDA tensor of 16-bit elements")
        b = blk.c_struct()
        err_ptr = error.data_ptr() if error is not None else None
        ws_ptr = None
        if workspace:
            ws = self._ws.get(int(slot))
            if ws is None:
                ws = _zeroed_workspace(out.device)
                self._ws[int(slot)] = ws
            ws_ptr = ws.data_ptr()
        _check(self._lib.df11_pipeline_decode(self._h, int(slot), ctypes.byref(b), out.data_ptr(),
                                              out.numel(), err_ptr, int(max_ctas), ws_ptr,
                                              _raw_stream(stream, out.device)),
               "df11_pipeline_decode")

    def acquire(self, slot: int, stream) -> None:
        _check(self._lib.df11_pipeline_acquire(self._h, int(slot), _raw_stream(stream)),
               "df11_pipeline_acquire")

    def verify(self, slot: int, blk: "DeviceBlock", expected, error, first_bad=None,
               stream=None) -> None:
        """Checksum check of the slot's staging block after its upload, on
        `stream` (put it on the decode stream before decode)."""
        b = blk.c_struct()
        fb = first_bad.data_ptr() if first_bad is not None else None
        _check(self._lib.df11_pipeline_verify(self._h, int(slot), ctypes.byref(b), expected.data_ptr(),
                                              expected.numel(), error.data_ptr(), fb,
                                              _raw_stream(stream)), "df11_pipeline_verify")

    def release(self, slot: int, stream) -> None:
        _check(self._lib.df11_pipeline_release(self._h, int(slot), _raw_stream(stream)),
               "df11_pipeline_release")


def _raw_stream(stream, device=None):
    if stream is None:
        import torch
        return torch.cuda.current_stream(device).cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


# ------------------------------------------------------------- integrity

def crc32c(data) -> int:
    """df11_crc32c of a bytes-like object or numpy array (its raw bytes)."""
    a = np.ascontiguousarray(np.frombuffer(data, np.uint8) if isinstance(data, (bytes, bytearray))
                             else np.asarray(data)).view(np.uint8).reshape(-1)
    return int(load_library().df11_crc32c(a.ctypes.data if a.size else None, a.size))


def checksum_count(blk) -> int:
    """Checksum values of a block (HostBlock, PinnedHostBlock or DeviceBlock):
    one per 4096-byte segment of each array."""
    b = blk.c_struct()
    return int(load_library().df11_checksum_count(ctypes.byref(b)))


def checksum(hb: HostBlock) -> np.ndarray:
    """df11_checksum: the block's CRC-32C list, computed on the host."""
    n = checksum_count(hb)
    out = np.empty(n, np.uint32)
    b = hb.c_struct()
    _check(load_library().df11_checksum(ctypes.byref(b), out.ctypes.data, n), "df11_checksum")
    return out


def checksum_device(db: "DeviceBlock", stream=None):
    """df11_checksum_device_async into a new int32 CUDA tensor (the uint32
    values' bit patterns)."""
    import torch
    dev = next(iter(db.tensors.values())).device
    n = checksum_count(db)
    out = torch.empty(n, dtype=torch.int32, device=dev)
    b = db.c_struct()
    _check(load_library().df11_checksum_device_async(ctypes.byref(b), out.data_ptr(), n,
                                                     _raw_stream(stream, dev)),
           "df11_checksum_device_async")
    return out


def verify_device(db: "DeviceBlock", expected, error, first_bad=None, stream=None) -> None:
    """df11_verify_device_async: ORs DEVERR_CHECKSUM into `error` (int32
    CUDA tensor) if any segment differs from `expected` (int32 CUDA tensor of
    the checksum list); `first_bad` (int64 CUDA tensor, preset to -1, i.e.
    UINT64_MAX) receives the lowest bad segment index."""
    b = db.c_struct()
    fb = first_bad.data_ptr() if first_bad is not None else None
    _check(load_library().df11_verify_device_async(ctypes.byref(b), expected.data_ptr(),
                                                   expected.numel(), error.data_ptr(), fb,
                                                   _raw_stream(stream, error.device)),
           "df11_verify_device_async")


def chunk_sums(hb: HostBlock) -> np.ndarray:
    """df11_chunk_sums: the block's per-chunk integrity sums (uint32, one per
    chunk), computed on the host."""
    n = int(hb.header.n_chunks)
    out = np.empty(n, np.uint32)
    b = hb.c_struct()
    _check(load_library().df11_chunk_sums(ctypes.byref(b), out.ctypes.data, n), "df11_chunk_sums")
    return out


def decompress_verified_async(db: "DeviceBlock", out, sums, error, first_bad=None, stream=None,
                              c_block=None, workspace=True) -> None:
    """df11_decompress_verified_async: decodes the whole block into `out` as
    decompress_async does and checks every chunk's sum against `sums` (int32
    CUDA tensor of the chunk_sums values' bit patterns); a mismatch ORs
    DEVERR_CHECKSUM into `error` (int32 CUDA tensor), and `first_bad` (int64
    CUDA tensor preset to -1, i.e. UINT64_MAX) receives the lowest chunk whose
    sum differs or whose decode failed."""
    if out.element_size() != 2 or not out.is_cuda or not out.is_contiguous():
        raise ValueError("out must be a contiguous CUDA tensor of 16-bit elements")
    if sums.element_size() != 4 or not sums.is_cuda or sums.numel() < db.header.n_chunks:
        raise ValueError("sums must be a CUDA tensor of n_chunks 32-bit values")
    handle = _raw_stream(stream, out.device)
    blk = c_block if c_block is not None else db.c_struct()
    fb = first_bad.data_ptr() if first_bad is not None else None
    _check(load_library().df11_decompress_verified_async(ctypes.byref(blk), out.data_ptr(), out.numel(),
                                                         error.data_ptr(), sums.data_ptr(), fb,
                                                         _workspace_ptr(workspace, out.device, handle),
                                                         handle),
           "df11_decompress_verified_async")


# ------------------------------------------------ decode fused with products

class GemvMatrix(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_uint64), ("cols", ctypes.c_uint64),
                ("x", ctypes.c_void_p), ("y", ctypes.c_void_p)]


def decode_gemv_async(db: "DeviceBlock", shapes, xs, ys, error=None, stream=None, workspace=True) -> None:
    """df11_decode_gemv_async: for matrix i of the block, shapes[i] = (rows,
    cols), adds xs[i] (n_tokens x cols, 16-bit CUDA tensor of BF16 bits)
    times W_i^T into ys[i] (n_tokens x rows, float32 CUDA tensor, zeroed by
    the caller), decoding the block once and never writing it in BF16.
    `workspace` as for decompress_async."""
    n = len(shapes)
    if len(xs) != n or len(ys) != n or n == 0:
        raise ValueError("one x and one y per matrix")
    n_tokens = int(xs[0].shape[0])
    arr = (GemvMatrix * n)()
    for i, ((r, c), x, y) in enumerate(zip(shapes, xs, ys)):
        if x.element_size() != 2 or not x.is_contiguous() or tuple(x.shape) != (n_tokens, c):
            raise ValueError(f"x[{i}] must be a contiguous {n_tokens} x {c} 16-bit tensor")
        if y.dtype.itemsize != 4 or not y.is_contiguous() or tuple(y.shape) != (n_tokens, r):
            raise ValueError(f"y[{i}] must be a contiguous {n_tokens} x {r} float32 tensor")
        arr[i] = GemvMatrix(int(r), int(c), x.data_ptr(), y.data_ptr())
    b = db.c_struct()
    err_ptr = error.data_ptr() if error is not None else None
    handle = _raw_stream(stream, xs[0].device)
    _check(load_library().df11_decode_gemv_async(ctypes.byref(b), arr, n, n_tokens, err_ptr,
                                                 _workspace_ptr(workspace, xs[0].device, handle), handle),
           "df11_decode_gemv_async")
