"""Streamed decoding on the GPU: the CTA-capped decode call and the
upload -> decode -> consume pipeline (df11_pipeline_*), called through the C
ABI.

The pipeline's product is ordering: every block a consumer reads must be the
bit-exact block it asked for, although uploads, decodes and the consumer run
on three streams and two slots are reused.  The consumer and the decoder are
delayed on purpose (a GPU sleep before they touch a slot), so a missing wait
shows up as a stale or overwritten block.  Decoded blocks are compared with
the input bits, which the oracle's decode of the same artifact equals (checked
here for one block per case).  Pages: "DFloat11: lossless BFloat16
compression" ("Architecture": a block is decoded before its matrix products
and dropped after), and the upstream README ("DFloat11: Lossless Compression
of LLMs and Diffusion Models for Efficient GPU Inference", news "Efficient CPU
Offloading Now Supported!").
"""
import numpy as np
import pytest

import oracle
import workloads
import huffman_decode_b200 as df11

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

SLEEP = 200_000   # GPU cycles (about 0.1 ms) of delay before touching a slot


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _flat(mats):
    return np.concatenate([np.ascontiguousarray(m, dtype=np.uint16).reshape(-1) for m in mats])


@pytest.fixture(scope="module")
def blocks():
    """Six small Llama-shaped blocks of different sizes, one codebook each."""
    out = []
    for i, div in enumerate((256, 192, 256, 320, 256, 224)):
        mats = [m for _, m in workloads.llama_block(2000 + i, scale_div=div)]
        cb = df11.build_codebook(mats)
        hb = df11.compress(cb, mats)
        out.append((_flat(mats), cb, hb))
    # the oracle pins the artifact of the first block
    w, cb, hb = out[0]
    ref = oracle.decode_block(hb.exp_stream, hb.n_elements, cb.lengths(), hb.signmant)
    assert np.array_equal(ref, w)
    return out


@pytest.mark.parametrize("max_ctas", [1, 2, 7, 148, 1 << 20])
def test_ctas_cap_is_bit_exact(blocks, max_ctas):
    w, cb, hb = blocks[0]
    db = hb.to_device("cuda")
    out = torch.full((w.size + 8,), 0x5A5A, dtype=torch.int16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.decompress_async(db, out, err, max_ctas=max_ctas, capacity=w.size)
    torch.cuda.synchronize()
    got = out.cpu().numpy().view(np.uint16)
    assert int(err.item()) == 0
    assert np.array_equal(got[: w.size], w)
    assert np.all(got[w.size:] == 0x5A5A)


def _run(blocks, upload: bool, n_slots: int = 2, max_ctas: int = 0, delay_consumer=True,
         delay_decoder=True):
    n_max = max(w.size for w, _, _ in blocks)
    outs = [torch.empty(n_max, dtype=torch.int16, device="cuda") for _ in range(n_slots)]
    results = [torch.empty(w.size, dtype=torch.int16, device="cuda") for w, _, _ in blocks]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    s_copy, s_dec, s_use = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    if upload:
        srcs = [hb.pinned() for _, _, hb in blocks]
        sizes = {n: max(s.sizes[n] for s in srcs) for n in srcs[0].sizes}
        staging = [df11.DeviceBlock.staging(sizes) for _ in range(n_slots)]
    else:
        resident = [hb.to_device("cuda") for _, _, hb in blocks]
    torch.cuda.synchronize()
    with df11.Pipeline(n_slots) as pipe:
        for i, (w, _, _) in enumerate(blocks):
            slot = i % n_slots
            if upload:
                pipe.upload(slot, srcs[i], staging[slot], s_copy)
                blk = staging[slot]
            else:
                blk = resident[i]
            if delay_decoder and i % 2:
                with torch.cuda.stream(s_dec):
                    torch.cuda._sleep(SLEEP)
            pipe.decode(slot, blk, outs[slot], err, s_dec, max_ctas=max_ctas)
            pipe.acquire(slot, s_use)
            with torch.cuda.stream(s_use):
                if delay_consumer:
                    torch.cuda._sleep(SLEEP)
                results[i].copy_(outs[slot][: w.size])
            pipe.release(slot, s_use)
        torch.cuda.synchronize()
    assert int(err.item()) == 0
    for i, (w, _, _) in enumerate(blocks):
        got = results[i].cpu().numpy().view(np.uint16)
        bad = np.nonzero(got != w)[0]
        assert bad.size == 0, f"block {i}: {bad.size} mismatches, first at {bad[:8]}"


def test_pipeline_resident_two_slots(blocks):
    _run(blocks, upload=False)


def test_pipeline_resident_one_slot_capped(blocks):
    _run(blocks, upload=False, n_slots=1, max_ctas=16)


def test_pipeline_offload_two_slots(blocks):
    _run(blocks, upload=True)


def test_pipeline_offload_three_slots_capped(blocks):
    _run(blocks, upload=True, n_slots=3, max_ctas=40, delay_decoder=False)


def test_pipeline_staging_too_small(blocks):
    _, _, hb = blocks[0]
    src = hb.pinned()
    small = {n: b - 16 if n == "signmant" else b for n, b in src.sizes.items()}
    staging = df11.DeviceBlock.staging(small)
    with df11.Pipeline(2) as pipe:
        with pytest.raises(df11.DF11Error) as e:
            pipe.upload(0, src, staging, torch.cuda.current_stream())
        assert e.value.status == 2   # DF11_ERR_BUFFER_TOO_SMALL
    torch.cuda.synchronize()
