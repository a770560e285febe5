"""GPU-side compressor (histogram + encode kernels, through the C ABI)
against the oracle's artifact and the host compressor.

The artifact a block compresses to on the GPU must equal, array by array and
byte by byte, the oracle's own (oracle.compress_block with the codebook's
code lengths) and the one the host library writes for the same codebook;
the GPU decode of it must give back the input.  Page: "DFloat11: lossless BFloat16
compression" ("How to develop with it": compression; "Architecture": the
format's Gaps and output positions).
"""
import numpy as np
import pytest

import oracle
import workloads
import huffman_decode_b200 as df11

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _flat(mats):
    return np.concatenate([np.ascontiguousarray(m, dtype=np.uint16).reshape(-1) for m in mats])


def _dev(w):
    return torch.from_numpy(w.view(np.int16)).cuda()


def check_against_oracle(mats, cb, db, bpt):
    """The GPU arrays against the oracle's own artifact for the same code
    lengths: the MSB-first stream, every thread's gap (the offset of the
    first code starting in its slice), every chunk's output position and the
    sign|mantissa bytes, byte for byte ("Architecture": Gaps and
    BlockOutputPos; "How it works": encode)."""
    ob = oracle.compress_block(mats, lengths=cb.lengths(), threads_per_chunk=32, bytes_per_thread=bpt)
    assert db.header.total_bits == ob.total_bits and db.header.n_chunks == ob.n_chunks
    stream = db.tensors["exp_stream"].cpu().numpy()
    assert stream.size == ob.stream.size
    bad = np.nonzero(stream != ob.stream)[0]
    assert bad.size == 0, f"stream: {bad.size} bytes differ from the oracle, first at {bad[:8]}"
    packed = db.tensors["gaps"].cpu().numpy()
    gaps = np.empty(packed.size * 2, np.uint8)
    gaps[0::2], gaps[1::2] = packed & 15, packed >> 4
    assert gaps.size == ob.gap.size
    bad = np.nonzero(gaps != ob.gap)[0]
    assert bad.size == 0, f"gaps: {bad.size} threads differ from the oracle, first at {bad[:8]}"
    pos = db.tensors["chunk_pos"].cpu().numpy().view(np.uint32)
    assert np.array_equal(pos, ob.pos)
    sm = db.tensors["signmant"].cpu().numpy()
    assert np.array_equal(sm[: ob.signmant.size], ob.signmant)
    assert not sm[ob.signmant.size:].any()


def check_gpu_compress(mats, bpt=16):
    w = _flat(mats)
    d_in = _dev(w)
    hist = df11.histogram_device(d_in).cpu().numpy().astype(np.uint64)
    assert np.array_equal(hist, oracle.histogram(oracle.split(w)[0]))
    cb = df11.build_codebook_from_histogram(hist)
    hb = df11.compress(cb, [w], 32, bpt)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    db = df11.compress_device(cb, d_in, 32, bpt, error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for name in ("total_bits", "n_elements", "n_chunks", "n_tables", "min_code_len",
                 "max_code_len", "threads_per_chunk", "bytes_per_thread"):
        assert getattr(db.header, name) == getattr(hb.header, name), name
    for name, a in hb.arrays().items():
        got = db.tensors[name].cpu().numpy()
        want = a.view(np.uint8)
        bad = np.nonzero(got != want)[0]
        assert bad.size == 0, f"{name}: {bad.size} bytes differ, first at {bad[:8]}"
    check_against_oracle(mats, cb, db, bpt)
    out = torch.empty(w.size, dtype=torch.int16, device="cuda")
    derr = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.decompress_async(db, out, derr)
    torch.cuda.synchronize()
    assert int(derr.item()) == 0
    assert np.array_equal(out.cpu().numpy().view(np.uint16), w)
    return cb, db


SMALL = {
    "single_1024x1024": lambda: workloads.single_matrix(0),
    "llama_block_div64": lambda: workloads.llama_block(1000, scale_div=64),
    "flux_block_div64": lambda: workloads.flux_block(5000, scale_div=64),
    "heavy_tail_1024": lambda: workloads.heavy_tail(4001, (1024, 1024)),
    "single_exponent_1024": lambda: workloads.single_exponent(4002, (1024, 1024)),
    "uniform_bits_1024": lambda: workloads.uniform_bits(4003, (1024, 1024)),
}


@pytest.mark.parametrize("name", sorted(SMALL))
@pytest.mark.parametrize("bpt", [8, 16])
def test_gpu_compress_matches_host(name, bpt):
    check_gpu_compress([m for _, m in SMALL[name]()], bpt)


@pytest.mark.parametrize("n", [1, 2, 7, 8, 9, 31, 32, 33, 8191, 8192, 8193, 16385, 100003])
def test_gpu_compress_sizes_and_segment_edges(n):
    rng = np.random.default_rng(n)
    w = workloads.to_bf16((rng.standard_normal(n) * 0.02).astype(np.float32))
    check_gpu_compress([w], 16)
    check_gpu_compress([w], 8)


def test_gpu_compress_all_bf16_patterns():
    allw = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    check_gpu_compress([allw, allw[::-1].copy()], 16)


@pytest.mark.parametrize("name", ["llama8b_block", "flux_dit_block"])
def test_gpu_compress_full_size(name):
    check_gpu_compress([m for _, m in workloads.WORKLOADS[name]()], 16)


def test_gpu_compress_flags_data_the_codebook_does_not_cover():
    rng = np.random.default_rng(3)
    w = workloads.to_bf16((rng.standard_normal(50000) * 0.02).astype(np.float32))
    cb = df11.build_codebook([w])
    other = w.copy()
    other[123] = (other[123] & np.uint16(0x807F)) | np.uint16(0xFE << 7)   # exponent with no code
    assert cb.lengths()[0xFE] == 0
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.compress_device(cb, _dev(other), error=err)
    torch.cuda.synchronize()
    assert int(err.item()) & df11.DEVERR_MISMATCH
