"""GPU checksums of DF11 artifacts (df11_checksum_device_async,
df11_verify_device_async, df11_pipeline_verify) against the oracle.

The checksum list is the CRC-32C of every 4096-byte segment of the block's
five arrays.  The GPU list must equal the oracle's bit-by-bit CRCs exactly
(integer work, zero tolerance); a flipped bit anywhere must be reported with
the index of its segment.  Page: "DFloat11: lossless BFloat16 compression",
"How to run it in production" and "Failure modes" (checksum artifacts on
download and after every copy).
"""
import numpy as np
import pytest

import oracle
import workloads
import huffman_decode_b200 as df11

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

ARRAYS = ("exp_stream", "gaps", "counts", "chunk_pos", "signmant", "lut")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _oracle_list(hb):
    return oracle.block_checksums(hb.exp_stream, hb.gaps, hb.counts, hb.chunk_pos, hb.signmant, hb.lut)


def _block(name):
    mats = {
        "llama_div256": lambda: workloads.llama_block(1003, scale_div=256),
        "heavy_tail_512": lambda: workloads.heavy_tail(4001, (512, 512)),
        "single_exponent_64": lambda: workloads.single_exponent(4002, (64, 64)),
        "uniform_bits_256": lambda: workloads.uniform_bits(4003, (256, 256)),
        "tiny_3x8": lambda: workloads.single_matrix(5, shape=(3, 8)),
    }[name]()
    mats = [m for _, m in mats]
    cb = df11.build_codebook(mats)
    return df11.compress(cb, mats)


NAMES = ["llama_div256", "heavy_tail_512", "single_exponent_64", "uniform_bits_256", "tiny_3x8"]


@pytest.mark.parametrize("name", NAMES)
def test_device_checksum_list_equals_oracle(name):
    hb = _block(name)
    db = hb.to_device("cuda")
    got = df11.checksum_device(db)
    torch.cuda.synchronize()
    ref = _oracle_list(hb)
    assert np.array_equal(got.cpu().numpy().view(np.uint32), ref)


def _segment_of(hb, array, byte):
    """Index in the checksum list of the segment holding `byte` of `array`."""
    k = 0
    for a in ARRAYS:
        n = getattr(hb, a).nbytes
        if a == array:
            return k + byte // df11.CRC_SEGMENT_BYTES
        k += (n + df11.CRC_SEGMENT_BYTES - 1) // df11.CRC_SEGMENT_BYTES
    raise KeyError(array)


@pytest.mark.parametrize("name", ["llama_div256", "single_exponent_64"])
def test_verify_reports_the_flipped_segment(name):
    hb = _block(name)
    expected = torch.from_numpy(_oracle_list(hb).view(np.int32)).cuda()
    rng = np.random.default_rng(5)
    db = hb.to_device("cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    first = torch.full((1,), -1, dtype=torch.int64, device="cuda")
    df11.verify_device(db, expected, err, first)
    torch.cuda.synchronize()
    assert int(err.item()) == 0 and int(first.item()) == -1
    for a in ARRAYS:
        t = db.tensors[a]
        nbytes = getattr(hb, a).nbytes
        for byte in sorted({0, nbytes - 1, int(rng.integers(0, nbytes))}):
            bit = int(rng.integers(0, 8))
            t[byte] ^= (1 << bit)
            err.zero_()
            first.fill_(-1)
            df11.verify_device(db, expected, err, first)
            torch.cuda.synchronize()
            t[byte] ^= (1 << bit)
            assert int(err.item()) == df11.DEVERR_CHECKSUM, (a, byte)
            assert int(first.item()) == _segment_of(hb, a, byte), (a, byte)


@pytest.mark.slow
def test_full_block_device_checksum():
    """Llama-3.1-8B-shaped block, drawn and compressed on the GPU: the GPU
    list equals the library's host list everywhere and the oracle's CRC on
    sampled segments of every array (the oracle is bit-serial)."""
    d_in = workloads.llama_block_device(1000, "cuda")
    hist = df11.histogram_device(d_in)
    cb = df11.build_codebook_from_histogram(hist.cpu().numpy().astype(np.uint64))
    db = df11.compress_device(cb, d_in)
    got = df11.checksum_device(db).cpu().numpy().view(np.uint32)
    host = {a: db.tensors[a][: db.sizes[a]].cpu().numpy() for a in ARRAYS}
    hb = df11.HostBlock(header=db.header, exp_stream=host["exp_stream"], gaps=host["gaps"],
                        counts=host["counts"], chunk_pos=host["chunk_pos"].view(np.uint32), signmant=host["signmant"],
                        lut=host["lut"].view(np.uint16))
    assert np.array_equal(got, df11.checksum(hb))
    rng = np.random.default_rng(9)
    k0 = 0
    for a in ARRAYS:
        raw = host[a]
        nseg = (raw.size + 4095) // 4096
        for s in sorted(set(rng.integers(0, nseg, 8).tolist()) | {0, nseg - 1}):
            assert got[k0 + s] == oracle.crc32c(raw[4096 * s: 4096 * (s + 1)]), (a, s)
        k0 += nseg
    assert k0 == got.size


def test_pipeline_verify_stage():
    """Offload pipeline with the verify stage after every upload: clean
    blocks pass; a block whose expected list is wrong is flagged."""
    blocks = [_block("llama_div256"), _block("heavy_tail_512"), _block("uniform_bits_256")]
    srcs = [hb.pinned() for hb in blocks]
    sizes = {n: max(s.sizes[n] for s in srcs) for n in srcs[0].sizes}
    staging = [df11.DeviceBlock.staging(sizes) for _ in range(2)]
    exp = [torch.from_numpy(_oracle_list(hb).view(np.int32)).cuda() for hb in blocks]
    bad = exp[1].clone()
    bad[-1] ^= 1
    n_max = max(hb.n_elements for hb in blocks)
    outs = [torch.empty(n_max, dtype=torch.int16, device="cuda") for _ in range(2)]
    s_copy, s_dec = torch.cuda.Stream(), torch.cuda.Stream()
    for lists, want in ((exp, [0, 0, 0]), ([exp[0], bad, exp[2]], [0, df11.DEVERR_CHECKSUM, 0])):
        errs = [torch.zeros(1, dtype=torch.int32, device="cuda") for _ in blocks]
        firsts = [torch.full((1,), -1, dtype=torch.int64, device="cuda") for _ in blocks]
        torch.cuda.synchronize()
        with df11.Pipeline(2) as pipe:
            for i in range(len(blocks)):
                slot = i % 2
                pipe.upload(slot, srcs[i], staging[slot], s_copy)
                pipe.verify(slot, staging[slot], lists[i], errs[i], firsts[i], s_dec)
                pipe.decode(slot, staging[slot], outs[slot], errs[i], s_dec)
                pipe.acquire(slot, s_dec)
                pipe.release(slot, s_dec)
            torch.cuda.synchronize()
        assert [int(e.item()) for e in errs] == want
        if want[1]:
            assert int(firsts[1].item()) == lists[1].numel() - 1
