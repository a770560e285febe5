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


# ------------------------------------------------ decode with chunk sums
# df11_decompress_verified_async: the decode kernel sums every chunk's bytes
# as it reads them and compares with the sums of df11_chunk_sums; the
# expected sums here are the oracle's.

def _oracle_chunk_sums(hb):
    h = hb.header
    return oracle.chunk_sums(hb.exp_stream, hb.gaps, hb.counts, hb.chunk_pos, hb.signmant, hb.lut,
                             h.n_tables, h.bytes_per_thread, h.n_chunks)


def _block_input(name):
    mats = {
        "llama_div256": lambda: workloads.llama_block(1003, scale_div=256),
        "heavy_tail_512": lambda: workloads.heavy_tail(4001, (512, 512)),
        "single_exponent_64": lambda: workloads.single_exponent(4002, (64, 64)),
        "uniform_bits_256": lambda: workloads.uniform_bits(4003, (256, 256)),
        "tiny_3x8": lambda: workloads.single_matrix(5, shape=(3, 8)),
    }[name]()
    return np.concatenate([m.reshape(-1) for _, m in mats])


def _verified(db, sums, n):
    out = torch.empty(n, dtype=torch.int16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    first = torch.full((1,), -1, dtype=torch.int64, device="cuda")
    df11.decompress_verified_async(db, out, sums, err, first)
    torch.cuda.synchronize()
    return out, int(err.item()), int(first.item())


@pytest.mark.parametrize("name", NAMES)
@pytest.mark.parametrize("bpt", [8, 16])
def test_verified_decode_of_clean_blocks(name, bpt):
    w = _block_input(name)
    cb = df11.build_codebook([w])
    hb = df11.compress(cb, [w], 32, bpt)
    sums = _oracle_chunk_sums(hb)
    assert np.array_equal(df11.chunk_sums(hb), sums)
    db = hb.to_device("cuda")
    out, err, first = _verified(db, torch.from_numpy(sums.view(np.int32)).cuda(), w.size)
    assert err == 0 and first == -1
    assert np.array_equal(out.cpu().numpy().view(np.uint16), w)
    # a wrong expected sum is reported at its chunk, and the output is still written
    for c in sorted({0, hb.header.n_chunks - 1, hb.header.n_chunks // 2}):
        bad = sums.copy()
        bad[c] ^= np.uint32(1 << (c % 32))
        out, err, first = _verified(db, torch.from_numpy(bad.view(np.int32)).cuda(), w.size)
        assert err == df11.DEVERR_CHECKSUM and first == c
        assert np.array_equal(out.cpu().numpy().view(np.uint16), w)


def _allowed_first_bad(hb, array, byte, bit):
    """Chunks a flipped bit may be reported at: the lowest chunk whose sum
    covers it, or the chunk before, which also reads the next chunk's first
    stream word (codes that cross into it) and its first thread's gap (where
    its last code must end); None for bytes no chunk covers."""
    h = hb.header
    cb = 32 * h.bytes_per_thread
    n = h.n_chunks
    pos = hb.chunk_pos
    if array == "exp_stream":
        if byte >= n * cb:
            return None
        c = byte // cb
        return {c, c - 1} - {-1} if byte % cb < 4 else {c}
    if array == "gaps":
        if 2 * byte >= 32 * n:
            return None
        c = (2 * byte) // 32
        return {c, c - 1} - {-1} if byte % 16 == 0 and bit < 4 else {c}
    if array == "counts":
        return {byte // 32} if byte < 32 * n else None
    if array == "chunk_pos":
        k = byte // 4
        return {max(k - 1, 0)} if k <= n else None
    if array == "signmant":
        owners = [c for c in range(n) if pos[c] <= byte < pos[c + 1]]
        return {owners[0]} if owners else None
    if array == "lut":
        return {0}
    raise KeyError(array)


@pytest.mark.parametrize("name", ["llama_div256", "heavy_tail_512", "single_exponent_64"])
@pytest.mark.parametrize("bpt", [8, 16])
def test_verified_decode_reports_a_flipped_bit_at_its_chunk(name, bpt):
    """One bit flipped in each array at several places (ends, chunk edges,
    random): the launch reports an error and the lowest bad chunk the flip
    can spoil; a bit outside every chunk changes nothing."""
    w = _block_input(name)
    cb = df11.build_codebook([w])
    hb = df11.compress(cb, [w], 32, bpt)
    sums = torch.from_numpy(_oracle_chunk_sums(hb).view(np.int32)).cuda()
    db = hb.to_device("cuda")
    rng = np.random.default_rng(17)
    n = hb.header.n_chunks
    cbytes = 32 * hb.header.bytes_per_thread
    for a in ARRAYS:
        t = db.tensors[a]
        nbytes = getattr(hb, a).nbytes
        places = {0, nbytes - 1, int(rng.integers(0, nbytes)), int(rng.integers(0, nbytes))}
        if a == "exp_stream":
            places |= {cbytes * min(1, n - 1), cbytes * min(1, n - 1) + 5, n * cbytes}
        if a == "gaps":
            places |= {16 * min(1, n - 1)}
        if a == "chunk_pos":
            places |= {4 * n, 4 * min(1, n), 4 * n + 3}
        if a == "signmant":
            places |= {int(hb.chunk_pos[min(1, n)]), hb.n_elements - 1}
        for byte in sorted(p for p in places if p < nbytes):
            for bit in sorted({int(rng.integers(0, 8)), 0, 7}):
                allowed = _allowed_first_bad(hb, a, byte, bit)
                t[byte] ^= (1 << bit)
                out, err, first = _verified(db, sums, w.size)
                t[byte] ^= (1 << bit)
                if allowed is None:
                    assert err == 0 and first == -1, (a, byte, bit)
                    assert np.array_equal(out.cpu().numpy().view(np.uint16), w), (a, byte, bit)
                else:
                    assert err != 0 and first in allowed, (a, byte, bit, err, first, allowed)
    out, err, first = _verified(db, sums, w.size)
    assert err == 0 and first == -1


@pytest.mark.slow
def test_verified_decode_full_block():
    """Llama-3.1-8B-shaped block compressed on the GPU: the oracle's chunk
    sums equal the library's; the verified decode of the clean block is
    exact and silent; one flipped bit in each array is reported at its
    chunk."""
    d_in = workloads.llama_block_device(1000, "cuda")
    hist = df11.histogram_device(d_in)
    cb = df11.build_codebook_from_histogram(hist.cpu().numpy().astype(np.uint64))
    db = df11.compress_device(cb, d_in)
    host = {a: db.tensors[a][: db.sizes[a]].cpu().numpy() for a in ARRAYS}
    hb = df11.HostBlock(header=db.header, exp_stream=host["exp_stream"], gaps=host["gaps"],
                        counts=host["counts"], chunk_pos=host["chunk_pos"].view(np.uint32),
                        signmant=host["signmant"], lut=host["lut"].view(np.uint16))
    ref = _oracle_chunk_sums(hb)
    assert np.array_equal(df11.chunk_sums(hb), ref)
    sums = torch.from_numpy(ref.view(np.int32)).cuda()
    n = d_in.numel()
    out, err, first = _verified(db, sums, n)
    assert err == 0 and first == -1
    assert torch.equal(out, d_in)
    rng = np.random.default_rng(23)
    for a in ARRAYS:
        t = db.tensors[a]
        nbytes = db.sizes[a]
        byte = int(rng.integers(0, nbytes))
        bit = int(rng.integers(0, 8))
        allowed = _allowed_first_bad(hb, a, byte, bit)
        t[byte] ^= (1 << bit)
        out, err, first = _verified(db, sums, n)
        t[byte] ^= (1 << bit)
        if allowed is None:
            assert err == 0 and first == -1, (a, byte)
        else:
            assert err != 0 and first in allowed, (a, byte, err, first, allowed)


def test_checksum_of_arrays_only_16_byte_aligned():
    """The GPU checksum list of a block whose every array starts 16 bytes
    past a 32-byte boundary (the kernel's 16-byte load path) equals the
    oracle's, and verification and decode work on it."""
    hb = _block("llama_div256")
    aligned = hb.to_device("cuda")
    t = {}
    for a in ARRAYS:
        raw = aligned.tensors[a]
        buf = torch.zeros(raw.numel() + 64, dtype=torch.uint8, device="cuda")
        off = (16 - buf.data_ptr() % 32) % 32
        view = buf[off: off + raw.numel()]
        assert view.data_ptr() % 32 == 16
        view.copy_(raw)
        t[a] = view
    db = df11.DeviceBlock(header=aligned.header, tensors=t, sizes=aligned.sizes,
                          matrix_numel=aligned.matrix_numel)
    got = df11.checksum_device(db)
    torch.cuda.synchronize()
    ref = _oracle_list(hb)
    assert np.array_equal(got.cpu().numpy().view(np.uint32), ref)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    first = torch.full((1,), -1, dtype=torch.int64, device="cuda")
    df11.verify_device(db, torch.from_numpy(ref.view(np.int32)).cuda(), err, first)
    torch.cuda.synchronize()
    assert int(err.item()) == 0 and int(first.item()) == -1
