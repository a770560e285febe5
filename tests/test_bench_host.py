"""Host logic of bench.py that needs no GPU: the piece plan of the
pipelined end-to-end step and the CPU-baseline helpers."""
import os

import pytest

import bench


@pytest.mark.parametrize("pieces", [1, 3, 8, 10**6])
@pytest.mark.parametrize("bpt", [8, 16])
def test_e2e_plan_covers_every_byte_a_range_reads(pieces, bpt):
    """The pieces partition the chunks; each piece's copy spans hold every
    byte its range decode reads (the header's list for
    df11_decompress_range_async) and stay inside the arrays; together the
    spans cover the arrays, and the output ranges tile the block."""
    import numpy as np
    import huffman_decode_b200 as df11
    import workloads
    mats = [m for _, m in workloads.llama_block(1005, scale_div=256)]
    hb = df11.compress(df11.build_codebook(mats), mats, 32, bpt)
    plan = bench.e2e_plan(hb, pieces)
    n_chunks = int(hb.header.n_chunks)
    assert plan[0][0] == 0 and plan[-1][1] == n_chunks
    assert all(a[1] == b[0] for a, b in zip(plan[:-1], plan[1:]))
    assert all(c0 < c1 for c0, c1, *_ in plan)
    W = 32 * bpt
    pos = hb.chunk_pos.astype(np.int64)
    covered = {n: np.zeros(getattr(hb, n).nbytes, bool)
               for n in ("exp_stream", "gaps", "counts", "chunk_pos", "signmant")}
    out_prev = 0
    for c0, c1, p0, p1, spans in plan:
        assert (p0, p1) == (pos[c0], pos[c1]) and p0 == out_prev
        out_prev = p1
        got = {n: (a, b) for n, a, b in spans}
        need = {"exp_stream": (W * c0, min(W * c1 + 16, hb.exp_stream.nbytes)),
                "gaps": (16 * c0, min(16 * c1 + 1, hb.gaps.nbytes)),
                "counts": (32 * c0, 32 * c1),
                "chunk_pos": (4 * c0, 4 * (c1 + 1)),
                "signmant": (p0 & ~15, min((p1 + 15) & ~15, hb.signmant.nbytes))}
        for n, (a, b) in need.items():
            ga, gb = got[n]
            assert ga <= a and gb >= b and 0 <= ga <= gb <= getattr(hb, n).nbytes, (n, c0, c1)
            covered[n][ga:gb] = True
    assert out_prev == hb.n_elements
    # together the pieces move every byte of the stream words, gaps, positions
    # and sign|mantissa bytes a whole-block decode reads
    assert covered["gaps"][: 16 * n_chunks].all()
    assert covered["counts"][: 32 * n_chunks].all()
    assert covered["chunk_pos"][: 4 * (n_chunks + 1)].all()
    assert covered["exp_stream"][: W * n_chunks].all()
    assert covered["signmant"][: hb.n_elements].all()


def test_one_core_pinning_restores_the_affinity():
    if not hasattr(os, "sched_getaffinity"):
        pytest.skip("no affinity control on this platform")
    before = os.sched_getaffinity(0)
    inside, core = bench.pinned_to_one_core(lambda: os.sched_getaffinity(0))
    assert os.sched_getaffinity(0) == before
    if core is not None:
        assert inside == {core} and core in before


def test_host_cpu_fields():
    h = bench.host_cpu()
    assert set(h) == {"cpu_model", "host_logical_cpus"}
    assert h["host_logical_cpus"] == os.cpu_count()
