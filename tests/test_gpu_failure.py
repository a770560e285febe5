"""Failure detection on the GPU without a fault.

The decode kernel's only wait is on the barrier of its staged sign|mantissa
copy, and it is bounded: after its poll limit it gives up, ORs
DEVERR_TIMEOUT into the caller's error word and finishes.  A copy that never
lands cannot be produced safely, so df11_selftest_bounded_wait runs that
same wait on a barrier nothing arrives on.  The test checks that the status
comes back, quickly, and that the context still decodes correctly after.
Corrupt-input detection (count, code and position errors) is in
test_gpu_parity.
"""
import numpy as np
import pytest

import workloads
import huffman_decode_b200 as df11

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


@pytest.mark.parametrize("polls", [1, 64, 4096])
def test_a_wait_that_runs_out_reports_a_timeout(polls):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    df11.selftest_bounded_wait(polls, status)
    b.record()
    torch.cuda.synchronize()
    assert int(status.item()) == df11.DEVERR_TIMEOUT
    assert a.elapsed_time(b) < 2000.0     # milliseconds: it gave up, it did not hang


def test_the_context_decodes_after_a_timeout():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.selftest_bounded_wait(64, status)
    mats = [m for _, m in workloads.llama_block(1004, scale_div=64)]
    hb = df11.compress(df11.build_codebook(mats), mats)
    db = hb.to_device("cuda")
    out = torch.empty(hb.n_elements, dtype=torch.int16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.decompress_async(db, out, err)
    torch.cuda.synchronize()
    assert int(status.item()) == df11.DEVERR_TIMEOUT
    assert int(err.item()) == 0
    assert np.array_equal(out.cpu().numpy().view(np.uint16), np.concatenate([m.reshape(-1) for m in mats]))
