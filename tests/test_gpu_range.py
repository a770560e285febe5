"""Decoding a block piece by piece (df11_decompress_range_async) against the
oracle.

Chunks are independent given their gaps and output positions ("DFloat11:
lossless BFloat16 compression", "Architecture": each thread block decodes
its own chunk), so decoding any partition of the chunks, in any order, must
give the oracle's decode of the whole block bit for bit (integer work, zero
tolerance).  A range launch must also read only its own chunks' bytes and
write only its own output range: the tests poison everything else.
"""
import numpy as np
import pytest

import oracle
import workloads
import huffman_decode_b200 as df11

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

STREAM_PAD = 16
SENTINEL = 0x5A5A


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _block(bpt, scale_div=64, seed=1000):
    mats = [m for _, m in workloads.llama_block(seed, scale_div=scale_div)]
    cb = df11.build_codebook(mats)
    hb = df11.compress(cb, mats, 32, bpt)
    ref = oracle.decode_block(hb.exp_stream, hb.n_elements, cb.lengths(), hb.signmant)
    assert np.array_equal(ref, np.concatenate([m.reshape(-1) for m in mats]))
    return hb, ref


def _cuts(n_chunks, rng, pieces):
    inner = sorted(set(rng.integers(1, n_chunks, pieces - 1).tolist())) if n_chunks > 1 else []
    return [0] + inner + [n_chunks]


@pytest.mark.parametrize("bpt", [8, 16])
@pytest.mark.parametrize("workspace", [True, False])
def test_any_partition_in_any_order_equals_the_oracle(bpt, workspace):
    hb, ref = _block(bpt)
    n_chunks = int(hb.header.n_chunks)
    db = hb.to_device("cuda")
    rng = np.random.default_rng(bpt)
    for pieces in (1, 2, 7, 33):
        cuts = _cuts(n_chunks, rng, pieces)
        # single-chunk pieces at both ends too
        cuts = sorted(set(cuts) | {1, n_chunks - 1})
        spans = list(zip(cuts[:-1], cuts[1:]))
        rng.shuffle(spans)
        out = torch.full((hb.n_elements,), SENTINEL, dtype=torch.int16, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        for c0, c1 in spans:
            df11.decompress_range_async(db, c0, c1, out, err, workspace=workspace)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        got = out.cpu().numpy().view(np.uint16)
        bad = np.nonzero(got != ref)[0]
        assert bad.size == 0, f"{pieces} pieces: {bad.size} mismatches, first at {bad[:8]}"


@pytest.mark.parametrize("bpt", [8, 16])
def test_a_range_reads_and_writes_only_its_own_bytes(bpt):
    """Device arrays hold garbage except the bytes the header lists for the
    range; the range's output must be exact and nothing else written."""
    hb, ref = _block(bpt, scale_div=32, seed=1001)
    n_chunks = int(hb.header.n_chunks)
    W = 32 * bpt
    pos = hb.chunk_pos.astype(np.int64)
    db = hb.to_device("cuda")
    rng = np.random.default_rng(7 + bpt)
    spans = [(0, 1), (n_chunks - 1, n_chunks), (0, n_chunks)]
    for _ in range(4):
        a, b = sorted(rng.choice(np.arange(n_chunks + 1), 2, replace=False).tolist())
        spans.append((a, b))
    for c0, c1 in spans:
        # poison every array, then restore only what the range may read
        for name in ("exp_stream", "gaps", "counts", "chunk_pos", "signmant"):
            db.tensors[name].fill_(0xA5)
        src = {n: torch.from_numpy(getattr(hb, n).view(np.uint8)).cuda()
               for n in ("exp_stream", "gaps", "counts", "chunk_pos", "signmant")}
        s0, s1 = W * c0, min(W * c1 + STREAM_PAD, hb.exp_stream.nbytes)
        db.tensors["exp_stream"][s0:s1] = src["exp_stream"][s0:s1]
        g1 = min(16 * c1 + 1, hb.gaps.nbytes)       # and the gap of the thread after the range
        db.tensors["gaps"][16 * c0:g1] = src["gaps"][16 * c0:g1]
        db.tensors["counts"][32 * c0:32 * c1] = src["counts"][32 * c0:32 * c1]
        db.tensors["chunk_pos"][4 * c0:4 * (c1 + 1)] = src["chunk_pos"][4 * c0:4 * (c1 + 1)]
        p0, p1 = int(pos[c0]), int(pos[c1])
        m0, m1 = p0 & ~15, min((p1 + 15) & ~15, hb.signmant.nbytes)
        db.tensors["signmant"][m0:m1] = src["signmant"][m0:m1]
        out = torch.full((hb.n_elements,), SENTINEL, dtype=torch.int16, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        df11.decompress_range_async(db, c0, c1, out, err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0, (c0, c1)
        got = out.cpu().numpy().view(np.uint16)
        assert np.array_equal(got[p0:p1], ref[p0:p1]), (c0, c1)
        assert np.all(got[:p0] == SENTINEL) and np.all(got[p1:] == SENTINEL), (c0, c1)


def test_full_size_block_in_two_claimed_pieces():
    """Two halves of the Llama-3.1-8B-shaped block: each has over five
    rounds of chunks for a full wave of warps, so each range launch claims
    its last rounds from the (per-stream) scheduling workspace."""
    mats = [m for _, m in workloads.llama_block(1001)]
    w = np.concatenate([m.reshape(-1) for m in mats])
    hb = df11.compress(df11.build_codebook(mats), mats)
    db = hb.to_device("cuda")
    n_chunks = int(hb.header.n_chunks)
    out = torch.full((hb.n_elements,), SENTINEL, dtype=torch.int16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.zeros(df11.SCHED_WORKSPACE_BYTES, dtype=torch.uint8, device="cuda")
    for c0, c1 in ((n_chunks // 2, n_chunks), (0, n_chunks // 2)):
        df11.decompress_range_async(db, c0, c1, out, err, workspace=ws)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert int(ws.count_nonzero().item()) == 0
    assert np.array_equal(out.cpu().numpy().view(np.uint16), w)


def test_full_size_block_in_pieces():
    """The Llama-3.1-8B-shaped block in 8 pieces on two streams, against the
    input bits (the oracle's whole-block parity at this size is in
    test_gpu_parity)."""
    mats = [m for _, m in workloads.llama_block(1000)]
    w = np.concatenate([m.reshape(-1) for m in mats])
    hb = df11.compress(df11.build_codebook(mats), mats)
    db = hb.to_device("cuda")
    n_chunks = int(hb.header.n_chunks)
    cuts = [n_chunks * k // 8 for k in range(9)]
    out = torch.empty(hb.n_elements, dtype=torch.int16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    torch.cuda.synchronize()
    for k in range(8):
        df11.decompress_range_async(db, cuts[k], cuts[k + 1], out, err, stream=streams[k % 2])
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(out.cpu().numpy().view(np.uint16), w)
