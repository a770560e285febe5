"""GPU decode (sm_100a kernel, called through the C ABI) against the oracle.

Every output element must equal the oracle's serial bit-by-bit decode of the
same artifact, which must equal the input BF16 bits: zero tolerance, this is
integer work.  Workloads: the five configurations at full size plus small and
degenerate cases.  Page: "DFloat11: lossless BFloat16 compression".
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


def gpu_decode(hb, capacity=None, guard=0, stream=None, workspace=True, decode_table=True):
    """Decode on cuda:0 into a buffer with `guard` extra elements set to a
    sentinel; returns (output incl. guard as uint16, error word).
    decode_table: the multi-code table built on the host (else every CTA
    builds it)."""
    db = hb.to_device("cuda", decode_table=decode_table)
    n = hb.n_elements
    out = torch.full((n + guard,), 0x5A5A, dtype=torch.int16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.decompress_async(db, out, err, stream=stream, capacity=capacity, workspace=workspace)
    torch.cuda.synchronize()
    return out.cpu().numpy().view(np.uint16), int(err.item())


def check_block(mats, bytes_per_thread=8, oracle_decode=True, workspace=True, decode_table=True):
    w = _flat(mats)
    cb = df11.build_codebook(mats)
    hb = df11.compress(cb, mats, 32, bytes_per_thread)
    got, err = gpu_decode(hb, guard=8, workspace=workspace, decode_table=decode_table)
    assert err == 0
    assert np.all(got[w.size:] == 0x5A5A), "wrote past the block"
    got = got[: w.size]
    if oracle_decode:
        ref = oracle.decode_block(hb.exp_stream, hb.n_elements, cb.lengths(), hb.signmant)
        assert np.array_equal(ref, w)
        bad = np.nonzero(got != ref)[0]
    else:
        bad = np.nonzero(got != w)[0]
    assert bad.size == 0, f"{bad.size} mismatches, first at {bad[:8]}"
    return cb, hb


# ------------------------------------------------------------- small cases

SMALL = {
    "single_1024x1024": lambda: workloads.single_matrix(0),
    "llama_block_div64": lambda: workloads.llama_block(1000, scale_div=64),
    "flux_block_div64": lambda: workloads.flux_block(5000, scale_div=64),
    "heavy_tail_1024": lambda: workloads.heavy_tail(4001, (1024, 1024)),
    "single_exponent_1024": lambda: workloads.single_exponent(4002, (1024, 1024)),
    "uniform_bits_1024": lambda: workloads.uniform_bits(4003, (1024, 1024)),
}


BPT = [8, 16]


@pytest.mark.parametrize("name", sorted(SMALL))
@pytest.mark.parametrize("bpt", BPT)
@pytest.mark.parametrize("schedule", ["dynamic", "static"])
@pytest.mark.parametrize("table", ["prebuilt", "per_cta"])
def test_small_workloads(name, bpt, schedule, table):
    check_block([m for _, m in SMALL[name]()], bytes_per_thread=bpt, workspace=schedule == "dynamic",
                decode_table=table == "prebuilt")


def test_garbage_decode_table_stays_in_bounds():
    """A decode table that is not the block's (random words, and one with
    impossible lengths and counts) gives wrong output or error bits, but
    every write stays inside the output buffer: the kernel turns entries no
    table could hold into the long-code marker and masks unused symbol
    bytes."""
    mats = [m for _, m in workloads.llama_block(1000, scale_div=64)]
    hb = df11.compress(df11.build_codebook(mats), mats)
    n = hb.n_elements
    rng = np.random.default_rng(7)
    good = df11.build_decode_table(hb.lut, hb.header.n_tables, hb.header.min_code_len)
    tables = [rng.integers(0, 1 << 63, good.size, dtype=np.uint64),
              good ^ np.uint64(0x0000_0001_0000_0000),                 # lengths one off
              (good & np.uint64(0xFFFFFFFF)) | np.uint64((1 | 4 << 19) << 32),   # 4 codes in 1 bit
              good.copy()]
    tables[3][::3] = np.uint64(0)                                       # zero entries
    for tab in tables:
        db = hb.to_device("cuda", decode_table=False)
        db.decode_table = torch.from_numpy(tab.view(np.uint8).copy()).cuda()
        out = torch.full((n + 64,), 0x5A5A, dtype=torch.int16, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        df11.decompress_async(db, out, err, capacity=n)
        torch.cuda.synchronize()
        got = out.cpu().numpy().view(np.uint16)
        assert np.all(got[n:] == 0x5A5A), "wrote past the output"
    # the block's own table again: exact
    got, err = gpu_decode(hb, guard=8)
    assert err == 0 and np.array_equal(got[:n], _flat(mats))


# ------------------------------------------------------- chunk schedules

@pytest.mark.parametrize("max_ctas", [0, 1, 7, 148, 200, 1 << 20])
def test_dynamic_schedule_leaves_workspace_zero(max_ctas):
    """With a workspace, warps past their first rounds claim chunks from
    counters; every launch must decode every chunk exactly right and leave
    the workspace zero for the next launch (any grid: one CTA, a partial
    wave, two waves of CTAs, one short-lived CTA per 32 chunks).  The block
    has over five rounds of chunks for every grid but the largest, so all
    the others claim chunks."""
    mats = [m for _, m in workloads.llama_block(1000, scale_div=4)]
    w = _flat(mats)
    hb = df11.compress(df11.build_codebook(mats), mats)
    db = hb.to_device("cuda")
    ws = torch.zeros(df11.SCHED_WORKSPACE_BYTES, dtype=torch.uint8, device="cuda")
    out = torch.empty(hb.n_elements, dtype=torch.int16, device="cuda")
    for rep in range(3):
        out.fill_(0x5A5A)
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        df11.decompress_async(db, out, err, max_ctas=max_ctas, workspace=ws)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        assert np.array_equal(out.cpu().numpy().view(np.uint16), w), rep
        assert int(ws.count_nonzero().item()) == 0, rep


def test_schedules_agree_on_the_full_block():
    mats = [m for _, m in workloads.llama_block(1000)]
    w = _flat(mats)
    hb = df11.compress(df11.build_codebook(mats), mats)
    for workspace in (True, False):
        got, err = gpu_decode(hb, workspace=workspace)
        assert err == 0 and np.array_equal(got, w), workspace


def test_dynamic_schedule_with_a_corrupt_block_still_resets():
    """A block with a wrong chunk position: the error bit is set and the
    workspace still ends zero, so the next (clean) launch is exact."""
    mats = [m for _, m in workloads.llama_block(22, scale_div=4)]
    hb = df11.compress(df11.build_codebook(mats), mats)
    ws = torch.zeros(df11.SCHED_WORKSPACE_BYTES, dtype=torch.uint8, device="cuda")
    bad = df11.compress(df11.build_codebook(mats), mats)
    bad.chunk_pos[bad.chunk_pos.size // 2] += 3
    _, err = gpu_decode(bad, workspace=ws)
    assert err & df11.DEVERR_COUNT
    assert int(ws.count_nonzero().item()) == 0
    got, err = gpu_decode(hb, workspace=ws)
    assert err == 0 and np.array_equal(got, _flat(mats))


@pytest.mark.parametrize("bpt", BPT)
def test_all_bf16_patterns(bpt):
    allw = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    check_block([allw], bytes_per_thread=bpt)
    rng = np.random.default_rng(11)
    check_block([allw, rng.permutation(allw), allw[::-1].copy()], bytes_per_thread=bpt)


@pytest.mark.parametrize("n", [1, 2, 3, 7, 8, 9, 15, 16, 17, 31, 33, 255, 257, 4097])
@pytest.mark.parametrize("bpt", BPT)
def test_tiny_sizes(n, bpt):
    rng = np.random.default_rng(n)
    w = workloads.to_bf16((rng.standard_normal(n) * 0.02).astype(np.float32))
    check_block([w], bytes_per_thread=bpt)


@pytest.mark.parametrize("delta", [-1, 0, 1])
@pytest.mark.parametrize("bpt", BPT)
def test_chunk_boundary(delta, bpt):
    n = 32 * 8 * bpt + delta            # 1-bit codes: total bits == elements
    rng = np.random.default_rng(77)
    e = np.where(rng.random(n) < 0.5, 0x7A, 0x7B).astype(np.uint16)
    w = (e << np.uint16(7)) | rng.integers(0, 256, n).astype(np.uint16) & np.uint16(0x807F)
    cb, hb = check_block([w], bytes_per_thread=bpt)
    assert hb.header.n_chunks == (1 if delta <= 0 else 2)


@pytest.mark.parametrize("bpt", BPT)
def test_codes_crossing_slice_ends(bpt):
    """Short codes packed so that many slices end inside a multi-code table
    window: codes past a slice end belong to the next lane."""
    rng = np.random.default_rng(123)
    syms = np.array([0x70, 0x71, 0x72, 0x73, 0x74, 0x75, 0x76, 0x77], np.uint16)
    p = np.array([0.4, 0.2, 0.15, 0.1, 0.07, 0.05, 0.02, 0.01])
    e = rng.choice(syms, 300000, p=p)
    w = (e << np.uint16(7)) | rng.integers(0, 256, e.size).astype(np.uint16) & np.uint16(0x807F)
    check_block([w], bytes_per_thread=bpt)


@pytest.mark.parametrize("bpt", BPT)
def test_many_tables_fewer_warps_per_cta(bpt):
    """128 decode tables (64 KB in shared memory): the launch fits fewer warps
    per CTA and every element must still match the oracle; one code is a
    single bit (shortest code 1)."""
    mats = [m for _, m in workloads.many_tables()]
    cb, hb = check_block(mats, bytes_per_thread=bpt)
    assert cb.n_tables >= 100
    assert hb.header.min_code_len == 1


def test_many_matrices_keep_caller_order():
    rng = np.random.default_rng(5)
    mats = [workloads.to_bf16((rng.standard_normal(int(k)) * s).astype(np.float32))
            for k, s in zip(rng.integers(1, 5000, 40), rng.uniform(0.001, 0.1, 40))]
    check_block(mats)
    check_block(mats, bytes_per_thread=16)


def test_two_streams_concurrently():
    a = [m for _, m in workloads.llama_block(1003, scale_div=32)]
    b = [m for _, m in workloads.heavy_tail(4005, (1024, 2048))]
    ha = df11.compress(df11.build_codebook(a), a)
    hbk = df11.compress(df11.build_codebook(b), b)
    da, dbk = ha.to_device("cuda"), hbk.to_device("cuda")
    oa = torch.empty(ha.n_elements, dtype=torch.int16, device="cuda")
    ob = torch.empty(hbk.n_elements, dtype=torch.int16, device="cuda")
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    for _ in range(3):
        df11.decompress_async(da, oa, stream=s1)
        df11.decompress_async(dbk, ob, stream=s2)
    torch.cuda.synchronize()
    assert np.array_equal(oa.cpu().numpy().view(np.uint16), _flat(a))
    assert np.array_equal(ob.cpu().numpy().view(np.uint16), _flat(b))


# ------------------------------------------------- corrupt input, no trap

def _small_block(seed=21):
    mats = [m for _, m in workloads.llama_block(seed, scale_div=512)]
    cb = df11.build_codebook(mats)
    return mats, cb, df11.compress(cb, mats)


def test_wrong_chunk_position_sets_count_bit():
    """A position that disagrees with its chunks' counts: both chunks it
    bounds report it and write nothing; the other chunks stay exact."""
    mats, cb, hb = _small_block()
    assert hb.header.n_chunks >= 3
    hb.chunk_pos[1] += 1
    got, err = gpu_decode(hb, guard=64)
    assert err & df11.DEVERR_COUNT
    n = hb.n_elements
    assert np.all(got[n:] == 0x5A5A)
    w = _flat(mats)
    p2 = int(hb.chunk_pos[2])
    assert np.all(got[:p2] == 0x5A5A)
    assert np.array_equal(got[p2:n], w[p2:])


def test_non_monotone_and_out_of_range_positions_write_nothing_outside():
    mats, cb, hb = _small_block()
    hb.chunk_pos[2] = hb.chunk_pos[1] - 1
    got, err = gpu_decode(hb, guard=64)
    assert err & df11.DEVERR_BAD_POS
    assert np.all(got[hb.n_elements:] == 0x5A5A)
    mats, cb, hb = _small_block()
    n = hb.n_elements
    hb.chunk_pos[-1] = n + 40          # past the caller's capacity
    got, err = gpu_decode(hb, capacity=n, guard=64)
    assert err & df11.DEVERR_BAD_POS
    assert np.all(got[n:] == 0x5A5A)


def test_no_code_window_sets_bad_code_bit():
    mats = [m for _, m in workloads.single_exponent(4002, (64, 64))]
    cb = df11.build_codebook(mats)
    hb = df11.compress(cb, mats)
    assert cb.n_symbols == 1 and not hb.exp_stream.any()
    hb.exp_stream[100] = 0x80          # a '1' bit: no code starts with it
    got, err = gpu_decode(hb, guard=16)
    assert err & df11.DEVERR_BAD_CODE
    assert np.all(got[hb.n_elements:] == 0x5A5A)


@pytest.mark.parametrize("bpt", BPT)
def test_header_claiming_longer_shortest_code_is_caught(bpt):
    """A header whose min_code_len is larger than the codes in the tables
    makes the kernel treat the short codes as corrupt: it reports it and
    still writes nothing outside the block."""
    mats = [m for _, m in workloads.llama_block(31, scale_div=512)]
    cb = df11.build_codebook(mats)
    hb = df11.compress(cb, mats, 32, bpt)
    assert hb.header.min_code_len == 2
    hb.header.min_code_len = 3
    got, err = gpu_decode(hb, guard=64)
    assert err & (df11.DEVERR_BAD_CODE | df11.DEVERR_COUNT)
    assert np.all(got[hb.n_elements:] == 0x5A5A)


@pytest.mark.parametrize("bpt", BPT)
def test_header_claiming_shorter_shortest_code_still_decodes(bpt):
    """min_code_len smaller than the real shortest code only enlarges the
    kernel's buffers; the output stays exact."""
    mats = [m for _, m in workloads.llama_block(32, scale_div=512)]
    cb = df11.build_codebook(mats)
    hb = df11.compress(cb, mats, 32, bpt)
    hb.header.min_code_len = 1
    got, err = gpu_decode(hb, guard=8)
    assert err == 0
    assert np.array_equal(got[: hb.n_elements], _flat(mats))


def _chunk_breaks_contract(stream, lengths, gap, count, total_bits, chunk, tpc, slice_bits):
    """The per-thread contract the kernel checks, by the oracle's bit-by-bit
    decode: thread g decodes the codes that start in [gap, end) of its
    slice (end = the slice end, or the end of the stream); there must be
    count[g] of them, and the next code must start where they end (the next
    thread's first code, B (g + 1) + gap[g + 1], or the end of the stream).
    True when some thread of `chunk` breaks it."""
    for t in range(tpc):
        g = chunk * tpc + t
        b0 = slice_bits * g
        if b0 >= total_bits:
            continue
        p = b0 + int(gap[g])
        end = min(b0 + slice_bits, total_bits)
        n = 0
        while p < end:
            _, p = oracle.decode(stream, 1, lengths, start_bit=p)
            n += 1
        nb = b0 + slice_bits
        expect = nb + int(gap[g + 1]) if nb < total_bits else total_bits
        if n != int(count[g]) or (n and p != expect):
            return True
    return False


@pytest.mark.parametrize("bpt", BPT)
def test_flipped_bit_detected_exactly_when_a_thread_breaks_its_contract(bpt):
    """A flipped stream bit desyncs only the thread(s) that read it; the
    kernel sets the count bit exactly when the oracle says a thread of the
    chunk no longer decodes its stored count of codes ending where the next
    thread's first code starts."""
    mats = [m for _, m in workloads.single_matrix(0, shape=(64, 512))]
    cb = df11.build_codebook(mats)
    L = cb.lengths()
    rng = np.random.default_rng(99)
    flagged = 0
    for trial in range(24):
        hb = df11.compress(cb, mats, 32, bpt)
        gaps = np.empty(hb.gaps.size * 2, np.uint8)
        gaps[0::2], gaps[1::2] = hb.gaps & 15, hb.gaps >> 4
        bit = int(rng.integers(0, hb.header.total_bits))
        hb.exp_stream[bit // 8] ^= np.uint8(0x80 >> (bit % 8))
        chunk = bit // (32 * 8 * bpt)
        broken = False
        for c in {max(chunk - 1, 0), chunk}:
            broken |= _chunk_breaks_contract(hb.exp_stream, L, gaps, hb.counts, hb.header.total_bits, c, 32,
                                             8 * bpt)
        _, err = gpu_decode(hb)
        assert bool(err & df11.DEVERR_COUNT) == broken, (trial, bit)
        flagged += broken
    assert flagged > 0


def test_corrupt_counts_are_caught_and_stay_in_bounds():
    """Counts that disagree with the positions, exceed what a slice can hold,
    or move codes between threads: the count bit is set and nothing is
    written outside the output."""
    mats = [m for _, m in workloads.llama_block(1000, scale_div=64)]
    hb0 = df11.compress(df11.build_codebook(mats), mats)
    n = hb0.n_elements
    rng = np.random.default_rng(5)
    for kind in ("plus_one", "max", "swap", "zero"):
        hb = df11.compress(df11.build_codebook(mats), mats)
        g = int(rng.integers(0, hb.counts.size - 40))
        g -= g % 32
        if kind == "plus_one":
            hb.counts[g + 3] += 1
        elif kind == "max":
            hb.counts[g + 5] = 255
        elif kind == "swap":            # same chunk total, codes moved between threads
            hb.counts[g + 7] += 2
            hb.counts[g + 8] -= 2
        else:
            hb.counts[g + 9] = 0
            hb.counts[g + 10] += hb0.counts[g + 9]
        got, err = gpu_decode(hb, guard=64)
        assert err & df11.DEVERR_COUNT, kind
        assert np.all(got[n:] == 0x5A5A), kind


# --------------------------------------------------------- full workloads

@pytest.mark.parametrize("name", ["single_1024x1024", "llama8b_block", "adversarial_heavy_tail",
                                  "adversarial_single_exponent", "adversarial_uniform_bits",
                                  "flux_dit_block"])
@pytest.mark.parametrize("bpt", BPT)
def test_full_size_workload(name, bpt):
    """The configurations at full size, in both layouts (the benchmark times
    the default one), every element compared with the oracle."""
    mats = [m for _, m in workloads.WORKLOADS[name]()]
    check_block(mats, bytes_per_thread=bpt)


def test_model_stream_all_32_blocks_into_one_reused_buffer():
    """The 8B-scale stream as specified: 32 Llama-3.1-8B-shaped blocks drawn
    by numpy with seeds 1000..1031, each with its own codebook, decoded one
    after another on one stream into one reused BF16 buffer ("Architecture":
    block-level batching, decode then discard).  Every block is compared
    element by element with its input; on blocks 0, 1, 16 and 31 the input is
    first checked to equal the oracle's serial decode of the same artifact."""
    seeds = workloads.llama_model_seeds(32)
    oracle_checked = {seeds[0], seeds[1], seeds[16], seeds[-1]}
    stream = torch.cuda.current_stream()
    out = None
    seen = []
    for sd, w in workloads.llama_model_blocks(seeds):
        cb = df11.build_codebook([w])
        hb = df11.compress(cb, [w])
        if sd in oracle_checked:
            ref = oracle.decode_block(hb.exp_stream, hb.n_elements, cb.lengths(), hb.signmant)
            assert np.array_equal(ref, w), sd
        db = hb.to_device("cuda")
        if out is None:
            out = torch.empty(hb.n_elements, dtype=torch.int16, device="cuda")
        assert out.numel() == hb.n_elements
        out.fill_(0x5A5A)
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        df11.decompress_async(db, out, err, stream=stream)
        want = torch.from_numpy(w.view(np.int16)).cuda()
        assert int(err.item()) == 0, sd
        assert torch.equal(out, want), sd
        seen.append(sd)
        del db, want
    assert seen == seeds


def test_a_block_read_back_from_its_file_decodes_exactly(tmp_path):
    """The flat container (df11_serialize) written to a file, read back and
    checked (df11_deserialize), then decoded on the GPU."""
    mats = [m for _, m in workloads.llama_block(1006, scale_div=32)]
    hb = df11.compress(df11.build_codebook(mats), mats)
    path = tmp_path / "block.df11"
    hb.save(path)
    got, err = gpu_decode(df11.HostBlock.load(path), guard=8)
    assert err == 0
    w = _flat(mats)
    assert np.array_equal(got[: w.size], w) and np.all(got[w.size:] == 0x5A5A)
