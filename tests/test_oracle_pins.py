"""Pins for the CPU oracle: values the page prints, closed forms, invariants
and brute force on tiny inputs.  None of these re-types the oracle's own
formulas; each compares it with something fixed outside it.

Page: "DFloat11: lossless BFloat16 compression" (ai-infrastructure.net).
"""
import itertools
import math

import numpy as np
import pytest

import oracle
import workloads


# ------------------------------------------------------------ BF16 fields

def test_split_join_exhaustive_and_float_semantics():
    """Every one of the 65536 BF16 patterns: join(split(w)) == w; the
    exponent byte brackets the magnitude of the float the pattern encodes; the
    top bit of the raw byte is the float's sign ("What it is": 1 sign,
    8 exponent, 7 mantissa bits)."""
    w = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    e, s = oracle.split(w)
    assert np.array_equal(oracle.join(e, s), w)
    f = (w.astype(np.uint32) << 16).view(np.float32)
    finite = np.isfinite(f)
    # sign bit of the raw byte == the float's sign bit (+-0 and NaN included)
    assert np.array_equal((s >> 7).astype(bool), np.signbit(f))
    # normal numbers: 2^(e-127) <= |x| < 2^(e-126)
    normal = finite & (e > 0)
    a = np.abs(f[normal]).astype(np.float64)
    ee = e[normal].astype(np.float64)
    assert np.all(a >= np.exp2(ee - 127)) and np.all(a < np.exp2(ee - 126))
    # exponent 0: zero or subnormal; exponent 255: Inf or NaN
    assert np.all(np.abs(f[e == 0]) < np.finfo(np.float32).tiny)
    assert not np.any(np.isfinite(f[e == 255]))
    # the mantissa bits are the low 7 bits of the raw byte: among patterns with
    # the same sign and exponent, ordering by the raw byte orders |x|
    sel = (e == 127) & ((s >> 7) == 0)
    order = np.argsort(s[sel])
    assert np.all(np.diff(f[sel][order]) > 0)


# ----------------------------------------------------- the worked example

def _worked_example_inputs():
    rng = np.random.default_rng(0)
    w = workloads.to_bf16(rng.normal(0.0, 0.02, 200_000).astype(np.float32))
    u = rng.integers(0, 256, 200_000).astype(np.uint8)
    q = workloads.to_bf16((rng.integers(-127, 128, 200_000) * (0.02 / 127)).astype(np.float32))
    return w, u, q


def test_worked_example_statistics(golden_worked_example):
    g = golden_worked_example
    w, _, _ = _worked_example_inputs()
    e, s = oracle.split(w)
    c = oracle.histogram(e)
    assert int((c > 0).sum()) == int(g["distinct_exponents"])
    H = oracle.entropy(c)
    assert f"{H:.3f}" == g["exponent_entropy_bits"]
    L = oracle.huffman_lengths(c)
    avg = oracle.total_bits(c, L) / e.size
    assert f"{avg:.3f}" == g["avg_code_bits"]
    assert int(L.max()) == int(g["max_code_len"])
    assert f"{8.0 + avg:.3f}" == g["bits_per_weight"]
    assert f"{(8.0 + avg) / 16 * 100:.1f}" == g["percent_of_bf16"]
    assert f"{oracle.entropy(oracle.histogram(s)):.3f}" == g["signmant_entropy_bits"]
    # Huffman within one bit of the Shannon limit
    assert H <= avg < H + 1.0
    # under the 16-bit cap the page's code is already optimal: same lengths
    assert np.array_equal(oracle.code_lengths(c, 16), L)
    assert oracle.total_bits(c, oracle.package_merge_lengths(c, 16)) == oracle.total_bits(c, L)


def test_worked_example_roundtrip_chunks_and_tables(golden_worked_example):
    g = golden_worked_example
    w, _, _ = _worked_example_inputs()
    e, s = oracle.split(w)
    c = oracle.histogram(e)
    L = oracle.huffman_lengths(c)
    codes = oracle.canonical_codes(L)
    stream, tb = oracle.encode(e, L, codes)
    assert tb == oracle.total_bits(c, L)
    d, end = oracle.decode(stream, e.size, L)
    assert end == tb
    assert np.array_equal(oracle.join(d, s), w)
    # chunks of 4096 symbols decoded from their start bits == serial decode
    chunk = int(g["chunk_symbols"])
    starts = np.concatenate([[0], np.cumsum(L[e].astype(np.int64))])[::chunk]
    starts = starts[starts < tb] if e.size % chunk else starts[:-1]
    assert len(starts) == int(g["n_chunks"])
    assert len(starts) * 4 == int(g["offset_array_bytes"])
    parts = []
    for i, st in enumerate(starts.tolist()):
        n = min(chunk, e.size - i * chunk)
        parts.append(oracle.decode(stream, n, L, start_bit=st)[0])
    assert np.array_equal(np.concatenate(parts), e)
    # the page's hierarchy of 8-bit tables: one root plus one table per
    # distinct leading byte among codes longer than 8 bits
    prefixes = {int(codes[k]) >> (int(L[k]) - 8) for k in range(256) if L[k] > 8}
    assert 1 + len(prefixes) == int(g["hier_tables"])


def test_worked_example_corruption(golden_worked_example):
    """One flipped bit desyncs the stream: the page counts the weights that
    decode wrong from bit 0 with that bit flipped."""
    g = golden_worked_example
    w, _, _ = _worked_example_inputs()
    e, _ = oracle.split(w)
    L = oracle.huffman_lengths(oracle.histogram(e))
    stream, _ = oracle.encode(e, L, oracle.canonical_codes(L))
    bad = np.concatenate([stream, np.zeros(64, np.uint8)])
    i = int(g["flipped_bit_index"])
    bad[i // 8] ^= np.uint8(0x80 >> (i % 8))
    d, _ = oracle.decode(bad, e.size, L)
    assert int((d != e).sum()) == int(g["flipped_bit_wrong"])


def test_worked_example_adversarial(golden_worked_example):
    g = golden_worked_example
    _, u, q = _worked_example_inputs()
    uc = oracle.histogram(u)
    ubits = 8.0 + oracle.total_bits(uc, oracle.huffman_lengths(uc)) / u.size
    assert f"{ubits:.3f}" == g["uniform_bits_per_weight"]
    assert f"{ubits + 32.0 / int(g['chunk_symbols']):.3f}" == g["uniform_bits_with_offsets"]
    d = np.full(1000, 0x3E, np.uint8)
    dc = oracle.histogram(d)
    dbits = 8.0 + oracle.total_bits(dc, oracle.huffman_lengths(dc)) / d.size
    assert f"{dbits:.3f}" == g["single_exponent_bits_per_weight"]
    qe, _ = oracle.split(q)
    qc = oracle.histogram(qe)
    qbits = 8.0 + oracle.total_bits(qc, oracle.huffman_lengths(qc)) / q.size
    assert f"{qbits:.3f}" == g["int8_bits_per_weight"]
    _, wc = np.unique(q, return_counts=True)
    word_h = oracle.entropy(np.pad(wc, (0, 256 - wc.size)).astype(np.uint64)) if wc.size <= 256 else None
    assert word_h is not None and f"{word_h:.3f}" == g["int8_word_entropy_bits"]


# ------------------------------------------------------------ closed forms

def _counts(d):
    c = np.zeros(256, np.uint64)
    for s, v in d.items():
        c[s] = v
    return c


@pytest.mark.parametrize("fn", ["huffman", "package_merge", "code_lengths"])
def test_uniform_256_gives_8_bits(fn):
    c = np.full(256, 7, np.uint64)
    L = {"huffman": oracle.huffman_lengths,
         "package_merge": lambda c: oracle.package_merge_lengths(c, 16),
         "code_lengths": lambda c: oracle.code_lengths(c, 16)}[fn](c)
    assert np.all(L == 8)


@pytest.mark.parametrize("fn", ["huffman", "package_merge", "code_lengths"])
def test_dyadic_lengths_are_minus_log2_p(fn):
    # p = 1/2, 1/4, ..., 1/2^9, 1/2^9 over 10 symbols spread over the alphabet
    syms = [3, 17, 40, 41, 99, 128, 200, 201, 254, 255]
    cnt = [2 ** (8 - i) for i in range(9)] + [1]
    c = _counts(dict(zip(syms, cnt)))
    L = {"huffman": oracle.huffman_lengths,
         "package_merge": lambda c: oracle.package_merge_lengths(c, 16),
         "code_lengths": lambda c: oracle.code_lengths(c, 16)}[fn](c)
    total = sum(cnt)
    for s, k in zip(syms, cnt):
        assert L[s] == round(-math.log2(k / total))
    assert oracle.total_bits(c, L) / total == pytest.approx(oracle.entropy(c), abs=1e-12)


def test_two_and_one_symbols():
    c2 = _counts({5: 1000, 250: 1})
    for L in (oracle.huffman_lengths(c2), oracle.package_merge_lengths(c2, 16),
              oracle.code_lengths(c2, 16)):
        assert L[5] == 1 and L[250] == 1 and int(L.sum()) == 2
    c1 = _counts({0x79: 12345})
    L = oracle.code_lengths(c1, 16)
    assert L[0x79] == 1 and int(L.sum()) == 1
    assert oracle.canonical_codes(L)[0x79] == 0
    with pytest.raises(ValueError):
        oracle.code_lengths(np.zeros(256, np.uint64), 16)


def test_rfc1951_canonical_example():
    """RFC 1951 section 3.2.2 gives lengths (3,3,3,3,3,2,4,4) for symbols A..H
    and the canonical codes 010 011 100 101 110 00 1110 1111 -- the same
    (length, symbol) ordered assignment the page uses."""
    lens = np.zeros(256, np.uint8)
    lens[[65, 66, 67, 68, 69, 70, 71, 72]] = [3, 3, 3, 3, 3, 2, 4, 4]
    codes = oracle.canonical_codes(lens)
    want = ["010", "011", "100", "101", "110", "00", "1110", "1111"]
    for s, wcode in zip(range(65, 73), want):
        assert format(int(codes[s]), f"0{lens[s]}b") == wcode


# ---------------------------------------------------------------- invariants

def _random_counts(rng, n_sym, skew):
    c = np.zeros(256, np.uint64)
    syms = rng.choice(256, n_sym, replace=False)
    c[syms] = np.maximum(1, (rng.pareto(skew, n_sym) * 1000).astype(np.uint64))
    return c


@pytest.mark.parametrize("seed", range(12))
def test_kraft_cap_and_entropy_bounds(seed):
    rng = np.random.default_rng(seed)
    c = _random_counts(rng, int(rng.integers(2, 257)), float(rng.uniform(0.3, 3.0)))
    H = oracle.entropy(c)
    Lh = oracle.huffman_lengths(c)
    live = c > 0
    assert np.all((Lh > 0) == live)
    assert sum(2.0 ** -int(x) for x in Lh[live]) == 1.0           # Kraft equality
    avg = oracle.total_bits(c, Lh) / float(c.sum())
    assert H <= avg + 1e-12 and avg < H + 1.0
    for cap in (8, 9, 12, 16):
        L = oracle.code_lengths(c, cap)
        assert np.all((L > 0) == live) and int(L.max()) <= cap
        assert sum(2.0 ** -int(x) for x in L[live]) == 1.0
        assert oracle.total_bits(c, L) >= oracle.total_bits(c, Lh)
        # the capped optimum cannot beat a looser cap
        if cap < 16:
            assert oracle.total_bits(c, L) >= oracle.total_bits(c, oracle.code_lengths(c, 16))


def test_fibonacci_counts_exceed_and_respect_the_cap():
    """Fibonacci counts give the deepest Huffman tree (depth n-1); the cap
    must then come from package-merge."""
    fib = [1, 1]
    while len(fib) < 24:
        fib.append(fib[-1] + fib[-2])
    c = _counts(dict(zip(range(10, 34), fib)))
    Lh = oracle.huffman_lengths(c)
    assert int(Lh.max()) == 23
    L = oracle.code_lengths(c, 16)
    assert int(L.max()) == 16
    assert sum(2.0 ** -int(x) for x in L[c > 0]) == 1.0


def _brute_min_cost(counts_list, cap):
    best = None
    n = len(counts_list)
    for lens in itertools.product(range(1, cap + 1), repeat=n):
        if sum(2.0 ** -l for l in lens) <= 1.0:
            cost = sum(k * l for k, l in zip(counts_list, lens))
            best = cost if best is None else min(best, cost)
    return best


@pytest.mark.parametrize("seed", range(40))
def test_length_limited_optimal_vs_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(2, 7))
    cap_lo = max(1, math.ceil(math.log2(n)))
    cap = int(rng.integers(cap_lo, 7))
    if seed % 3 == 0:
        cnt = [int(x) for x in (np.cumprod(rng.integers(1, 4, n)) + rng.integers(0, 3, n))]
    else:
        cnt = [int(x) for x in rng.integers(1, 50, n)]
    syms = sorted(rng.choice(256, n, replace=False).tolist())
    c = _counts(dict(zip(syms, cnt)))
    best = _brute_min_cost(cnt, cap)
    assert oracle.total_bits(c, oracle.package_merge_lengths(c, cap)) == best
    L = oracle.code_lengths(c, cap)
    assert int(L.max()) <= cap and oracle.total_bits(c, L) == best
    # unlimited Huffman is the optimum with cap n-1
    assert oracle.total_bits(c, oracle.huffman_lengths(c)) == _brute_min_cost(cnt, max(1, n - 1))


# --------------------------------------------------- bitstream, brute force

def _codebook(lengths_by_sym):
    lens = np.zeros(256, np.uint8)
    for s, l in lengths_by_sym.items():
        lens[s] = l
    return lens, oracle.canonical_codes(lens)


@pytest.mark.parametrize("book", [{7: 1, 9: 2, 200: 2},
                                  {0: 2, 1: 2, 2: 2, 255: 2},
                                  {10: 1, 11: 2, 12: 3, 13: 3}])
def test_encode_decode_all_short_sequences(book):
    lens, codes = _codebook(book)
    syms = sorted(book)
    strings = {s: format(int(codes[s]), f"0{lens[s]}b") for s in syms}
    # canonical codes are prefix free
    for a in syms:
        for b in syms:
            if a != b:
                assert not strings[b].startswith(strings[a])
    for n in range(0, 7):
        for seq in itertools.product(syms, repeat=n):
            e = np.array(seq, np.uint8)
            stream, tb = oracle.encode(e, lens, codes)
            bits = "".join(strings[s] for s in seq)
            assert tb == len(bits)
            got = "".join(format(int(b), "08b") for b in stream)[:tb]
            assert got == bits
            assert "".join(format(int(b), "08b") for b in stream)[tb:].strip("0") == ""
            if n:
                d, end = oracle.decode(stream, n, lens)
                assert end == tb and d.tolist() == list(seq)


def test_decode_rejects_non_code_and_overrun():
    lens, codes = _codebook({42: 1})               # single code "0"
    with pytest.raises(ValueError):
        oracle.decode(np.array([0x80], np.uint8), 1, lens)   # bit "1" is no code
    lens, codes = _codebook({1: 1, 2: 2, 3: 2})
    with pytest.raises(ValueError):
        oracle.decode(np.array([0x00], np.uint8), 9, lens)   # runs off the end


def test_first_code_table_brute_force():
    lens, codes = _codebook({1: 1, 2: 3, 3: 3, 4: 3, 5: 4, 6: 5, 7: 5})
    sym, ln = oracle.first_code_table(lens)
    strings = {s: format(int(codes[s]), f"0{lens[s]}b") for s in range(1, 8)}
    for v in range(0, 65536, 97):
        bits = format(v, "016b")
        hits = [s for s, st in strings.items() if bits.startswith(st)]
        assert len(hits) == 1
        assert sym[v] == hits[0] and ln[v] == len(strings[hits[0]])
    lens1, _ = _codebook({9: 1})
    sym1, ln1 = oracle.first_code_table(lens1)
    assert np.all(sym1[:32768] == 9) and np.all(ln1[:32768] == 1)
    assert np.all(sym1[32768:] == -1) and np.all(ln1[32768:] == 0)


# ------------------------------------------------------ metadata, brute force

def _brute_metadata(lens_per_symbol, T, W, n_chunks):
    starts = [0]
    for l in lens_per_symbol:
        starts.append(starts[-1] + l)
    total = starts[-1]
    B = 8 * W
    gap = []
    for g in range(n_chunks * T):
        if B * g >= total:
            gap.append(0)
        else:
            gap.append(min(s for s in starts if s >= B * g) - B * g)
    pos = [sum(1 for s in starts[:-1] if s < c * T * B) for c in range(n_chunks + 1)]
    count = [sum(1 for s in starts[:-1] if B * g <= s < B * (g + 1)) for g in range(n_chunks * T)]
    return gap, count, pos


@pytest.mark.parametrize("seed", range(8))
@pytest.mark.parametrize("T,W", [(2, 1), (4, 2), (8, 8), (4, 8)])
def test_metadata_brute_force_and_thread_decode(seed, T, W):
    """Gaps, per-thread counts and chunk positions against their
    definitions, and the properties the decoder rests on: every thread
    decoding the codes that start in its slice, from its gap, reproduces the
    serial decode; it decodes exactly count[g] codes, and they end where the
    next thread's first code starts (or at the end of the stream); each
    chunk yields exactly pos[c+1]-pos[c] symbols, the sum of its counts."""
    rng = np.random.default_rng(seed)
    n_sym = int(rng.integers(1, 9))
    syms = rng.choice(256, n_sym, replace=False)
    c = np.zeros(256, np.uint64)
    c[syms] = rng.integers(1, 40, n_sym).astype(np.uint64)
    L = oracle.code_lengths(c, 16)
    p = c[syms].astype(np.float64) / float(c[syms].sum())
    n = int(rng.integers(1, 400))
    e = rng.choice(syms, n, p=p).astype(np.uint8)
    codes = oracle.canonical_codes(L)
    lens_seq = [int(L[x]) for x in e]
    tb = sum(lens_seq)
    B = 8 * W
    n_chunks = (tb + T * B - 1) // (T * B)
    gap, count, pos = oracle.metadata(e, L, T, W, n_chunks)
    bg, bc, bp = _brute_metadata(lens_seq, T, W, n_chunks)
    assert gap.tolist() == bg and pos.tolist() == bp and count.tolist() == bc
    assert int(gap.max()) < max(int(L.max()), 1) or tb == 0
    stream, _ = oracle.encode(e, L, codes, n_chunks * T * W + 16)
    out = []
    for ch in range(n_chunks):
        got = 0
        for t in range(T):
            g = ch * T + t
            p0 = B * g + int(gap[g])
            end = min(B * (g + 1), tb)
            mine = 0
            while p0 < end:
                d, nxt = oracle.decode(stream, 1, L, start_bit=p0)
                out.append(int(d[0]))
                p0 = nxt
                got += 1
                mine += 1
            assert mine == int(count[g])
            nxt_start = B * (g + 1) + int(gap[g + 1]) if g + 1 < gap.size and B * (g + 1) < tb else tb
            if mine:
                assert p0 == nxt_start
        assert got == int(pos[ch + 1] - pos[ch]) == int(count[ch * T:(ch + 1) * T].sum())
    assert out == e.tolist()


# ------------------------------------------------------------- checksum
# "DFloat11: lossless BFloat16 compression", "How to run it in production":
# checksum every artifact.  The oracle's CRC-32C is pinned to published check
# values and to the definition as a polynomial remainder, computed here with
# Python integers (no register loop, no reflection trick in the arithmetic).

def _crc32c_by_division(data: bytes) -> int:
    """CRC-32C as the remainder of (M(x) x^32 + (x^31 + ... + 1) x^n) by the
    Castagnoli generator, where M's coefficients are the n message bits in
    order, least significant bit of each byte first; the remainder's
    coefficients are then read lowest degree first and complemented."""
    bits = [(b >> i) & 1 for b in data for i in range(8)]
    n = len(bits)
    m = 0
    for bit in bits:
        m = (m << 1) | bit
    v = (m << 32) ^ (0xFFFFFFFF << n)
    g = 0x11EDC6F41
    for sh in range(v.bit_length() - 33, -1, -1):
        if (v >> (sh + 32)) & 1:
            v ^= g << sh
    return int(f"{v:032b}"[::-1], 2) ^ 0xFFFFFFFF


def test_crc32c_published_vectors():
    from conftest import read_golden
    g = read_golden("crc32c_vectors.txt")
    msgs = {
        "check_123456789": b"123456789",
        "zeros_32": bytes(32),
        "ones_32": bytes([0xFF] * 32),
        "incrementing_32": bytes(range(32)),
        "decrementing_32": bytes(range(31, -1, -1)),
    }
    for k, m in msgs.items():
        assert oracle.crc32c(m) == int(g[k], 16), k
        assert _crc32c_by_division(m) == int(g[k], 16), k


@pytest.mark.parametrize("seed", range(4))
def test_crc32c_equals_polynomial_remainder(seed):
    rng = np.random.default_rng(seed)
    for n in (0, 1, 2, 3, 4, 5, 15, 16, 17, 63, 64, 65, 300):
        d = rng.integers(0, 256, n, dtype=np.uint8).tobytes()
        assert oracle.crc32c(d) == _crc32c_by_division(d), n


def test_crc32c_detects_every_single_bit_flip():
    """A CRC with a generator of more than one term catches every one-bit
    error: the flip's error polynomial x^k is not a multiple of g."""
    d = bytearray(np.random.default_rng(7).integers(0, 256, 64, dtype=np.uint8).tobytes())
    base = oracle.crc32c(bytes(d))
    for i in range(len(d) * 8):
        d[i // 8] ^= 1 << (i % 8)
        assert oracle.crc32c(bytes(d)) != base
        d[i // 8] ^= 1 << (i % 8)


def test_segment_crcs_split_and_ragged_tail():
    rng = np.random.default_rng(3)
    a = rng.integers(0, 256, 3 * 4096 + 123, dtype=np.uint8)
    s = oracle.segment_crcs(a)
    assert s.size == 4
    for k in range(4):
        assert s[k] == _crc32c_by_division(a[4096 * k: 4096 * (k + 1)].tobytes())
    assert oracle.segment_crcs(np.zeros(0, np.uint8)).size == 0
    assert oracle.segment_crcs(np.zeros(4096, np.uint8)).size == 1


# ------------------------------------------------------------ chunk sums
# The per-chunk sum is this library's own check (the page asks only that
# artifacts be checksummed, "How to run it in production"), so no page
# prints a value of it.  It is pinned to what it is for: every one-bit
# change of any array it covers changes exactly the sums of the chunks that
# read that bit, bytes outside every chunk change nothing, and the sum
# depends on where each item sits, not only on the multiset of items.

def _tiny_artifact(seed, W):
    """A small oracle artifact with 32 threads per chunk: (stream, packed
    gaps, counts, pos, signmant, lut, n_tables, n_chunks)."""
    rng = np.random.default_rng(seed)
    mats = [workloads.to_bf16((rng.standard_normal(5000 + 97 * seed) * 0.02).astype(np.float32))]
    ob = oracle.compress_block(mats, threads_per_chunk=32, bytes_per_thread=W)
    gap = np.zeros(ob.gap.size + (ob.gap.size & 1), np.uint8)
    gap[: ob.gap.size] = ob.gap
    packed = (gap[0::2] | (gap[1::2] << 4)).astype(np.uint8)
    sm = np.concatenate([ob.signmant, rng.integers(0, 256, 5, dtype=np.uint8)])   # bytes past the end
    n_tables = 2
    lut = rng.integers(0, 65536, 256 * n_tables, dtype=np.uint16)
    return [ob.stream.copy(), packed, ob.thread_count.copy(), ob.pos.copy(), sm, lut, n_tables, ob.n_chunks]


def _sums(a, W):
    stream, gaps, counts, pos, sm, lut, n_tables, n_chunks = a
    return oracle.chunk_sums(stream, gaps, counts, pos, sm, lut, n_tables, W, n_chunks)


@pytest.mark.parametrize("W", [8, 16])
def test_chunk_sums_every_bit_flip_changes_exactly_its_chunks(W):
    a = _tiny_artifact(1, W)
    stream, gaps, counts, pos, sm, lut, n_tables, n_chunks = a
    assert n_chunks >= 3
    base = _sums(a, W)
    chunk_bytes = 32 * W

    def owners(name, i):
        if name == "stream":
            return {i // chunk_bytes} if i < n_chunks * chunk_bytes else set()
        if name == "gaps":
            return {(2 * i) // 32} if 2 * i < 32 * n_chunks else set()
        if name == "counts":
            return {i // 32} if i < 32 * n_chunks else set()
        if name == "signmant":
            return {c for c in range(n_chunks) if pos[c] <= i < pos[c + 1]}
        if name == "lut":
            return {0}
        raise AssertionError(name)

    for idx, name in ((0, "stream"), (1, "gaps"), (2, "counts"), (4, "signmant"), (5, "lut")):
        arr = a[idx].view(np.uint8)
        for i in range(arr.size):
            want = owners(name, i // a[idx].itemsize if name == "lut" else i)
            for bit in range(8):
                arr[i] ^= 1 << bit
                changed = set(np.nonzero(_sums(a, W) != base)[0].tolist())
                arr[i] ^= 1 << bit
                assert changed == want, (name, i, bit)
    # positions: a flip that keeps them ordered and in range changes the two
    # chunks that share the position; any other is rejected
    for c in range(n_chunks + 1):
        for bit in range(32):
            pos[c] ^= np.uint32(1 << bit)
            ok = all(pos[k] <= pos[k + 1] for k in range(n_chunks)) and pos[n_chunks] <= sm.size
            if ok:
                changed = set(np.nonzero(_sums(a, W) != base)[0].tolist())
                assert changed == {k for k in (c - 1, c) if 0 <= k < n_chunks}, (c, bit)
            else:
                with pytest.raises(ValueError):
                    _sums(a, W)
            pos[c] ^= np.uint32(1 << bit)
    assert np.array_equal(_sums(a, W), base)


def test_chunk_sums_depend_on_item_places():
    """Swapping two unequal items of one chunk (stream words, threads'
    metadata, 8-byte groups, single bytes) changes its sum: every item
    carries its place."""
    W = 16
    a = _tiny_artifact(2, W)
    stream, gaps, counts, pos, sm, lut, n_tables, n_chunks = a
    base = _sums(a, W)
    s32 = stream[: 32 * W * n_chunks].view(np.uint32)
    k = next(k for k in range(1, 32) if s32[k] != s32[0])
    s32[[0, k]] = s32[[k, 0]]
    assert _sums(a, W)[0] != base[0]
    s32[[0, k]] = s32[[k, 0]]
    t = next(t for t in range(1, 32) if counts[t] != counts[0])
    counts[[0, t]] = counts[[t, 0]]
    assert _sums(a, W)[0] != base[0]
    counts[[0, t]] = counts[[t, 0]]
    c = 1
    p0, p1 = int(pos[c]), int(pos[c + 1])
    q0 = (p0 + 7) // 8
    assert 8 * q0 + 16 <= p1
    g = sm[8 * q0: 8 * q0 + 16].copy()
    sm[8 * q0: 8 * q0 + 16] = np.concatenate([g[8:], g[:8]])
    assert _sums(a, W)[c] != base[c] or np.array_equal(g[8:], g[:8])
    sm[8 * q0: 8 * q0 + 16] = g
    e = next(e for e in range(p0 + 1, p1) if sm[e] != sm[p0])
    sm[[p0, e]] = sm[[e, p0]]
    assert _sums(a, W)[c] != base[c]
    sm[[p0, e]] = sm[[e, p0]]
    assert np.array_equal(_sums(a, W), base)
