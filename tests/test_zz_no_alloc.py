"""The allocation-free GPU compressor, df11_compress_device_noalloc.

It exists for callers that cannot let a library allocate device memory: a
serving runtime or framework that reserves the whole GPU for its own pool
(cudaMalloc would fail or escape its accounting), or code that must not call
cudaFree because it synchronises the device.  Its work space is one fixed
device array inside the library that every call shares and that keeps the
last call's contents, so these tests call it twice in a row, on different
blocks, and compare each result byte for byte with df11_compress_device,
which takes caller scratch.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

import workloads
import huffman_decode_b200 as df11
from huffman_decode_b200 import df11 as binding

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _flat(mats):
    return np.concatenate([np.ascontiguousarray(m, dtype=np.uint16).reshape(-1) for m in mats])


def _same_block(a, b):
    for name in ("total_bits", "n_elements", "n_chunks", "n_tables", "min_code_len"):
        assert getattr(a.header, name) == getattr(b.header, name), name
    for name in a.tensors:
        assert torch.equal(a.tensors[name], b.tensors[name]), name


@pytest.mark.parametrize("bpt", [16, 8])
def test_noalloc_matches_caller_scratch_on_two_calls_in_a_row(bpt):
    # a larger block first, then a smaller one: the second call runs over
    # work space still holding the first call's values
    blocks = [[m for _, m in workloads.llama_block(1007, scale_div=16)],
              [m for _, m in workloads.heavy_tail(4009, (512, 1024))]]
    for mats in blocks:
        w = _flat(mats)
        d_in = torch.from_numpy(w.view(np.int16)).cuda()
        cb = df11.build_codebook([w])
        err_a = torch.zeros(1, dtype=torch.int32, device="cuda")
        err_b = torch.zeros(1, dtype=torch.int32, device="cuda")
        want = df11.compress_device(cb, d_in, 32, bpt, error=err_a)
        got = df11.compress_device_noalloc(cb, d_in, 32, bpt, error=err_b)
        torch.cuda.synchronize()
        assert int(err_a.item()) == 0 and int(err_b.item()) == 0
        _same_block(got, want)
        out = torch.empty(w.size, dtype=torch.int16, device="cuda")
        df11.decompress_async(got, out)
        torch.cuda.synchronize()
        assert np.array_equal(out.cpu().numpy().view(np.uint16), w)


def test_noalloc_rejects_blocks_beyond_its_fixed_work_space():
    """More elements than the fixed array covers: a clear error, nothing
    launched (the size is checked before any pointer is used)."""
    lib = df11.load_library()
    cb = binding.Codebook()
    cb.n_elements = df11.df11.NOALLOC_MAX_ELEMENTS + 1
    ly = binding.Layout(32, 16)
    blk = binding._Block()
    fake = 1 << 20
    st = lib.df11_compress_device_noalloc(ctypes.byref(cb), ctypes.byref(ly), fake,
                                          df11.df11.NOALLOC_MAX_ELEMENTS + 1, ctypes.byref(blk),
                                          None, None)
    assert st == 2   # DF11_ERR_BUFFER_TOO_SMALL
