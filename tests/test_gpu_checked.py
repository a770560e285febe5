"""The bound-checked build (libdf11_checked.so, DF11_CHECKED=1).

It is the same library compiled with -DDF11_CHECKED: the decode kernel
verifies at run time the invariants that keep its staged copy, its slot
columns, its exponent buffer and its merge inside their buffers, and ORs
DF11_DEVERR_BOUNDS instead of making an access that would break one.  A child
process loads it and decodes clean and corrupt blocks through every entry
(whole block under both chunk schedules, chunk ranges, fused products): the
output must be the input bit for bit on clean blocks, and no launch may
report DEVERR_BOUNDS, corrupt ones included.  This stands in for a memory
sanitizer, which is not available on this hardware.
"""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import json, sys
import numpy as np, torch
import huffman_decode_b200 as df11, workloads
torch.cuda.set_device(0)
out = {"lib": df11.load_library()._name, "cases": []}

def run(name, hb, mats, fn):
    db = hb.to_device("cuda")
    o = torch.full((hb.n_elements + 8,), 0x5A5A, dtype=torch.int16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    fn(db, o, err)
    torch.cuda.synchronize()
    got = o.cpu().numpy().view(np.uint16)
    exact = mats is not None and np.array_equal(got[:hb.n_elements], np.concatenate([m.reshape(-1) for m in mats]))
    out["cases"].append({"name": name, "err": int(err.item()), "exact": bool(exact),
                         "guard": bool(np.all(got[hb.n_elements:] == 0x5A5A))})

blocks = {
    "llama_div64": lambda: workloads.llama_block(1000, scale_div=64),
    "llama_div4": lambda: workloads.llama_block(1000, scale_div=4),
    "heavy_tail_1024": lambda: workloads.heavy_tail(4001, (1024, 1024)),
    "single_exponent_1024": lambda: workloads.single_exponent(4002, (1024, 1024)),
    "uniform_bits_1024": lambda: workloads.uniform_bits(4003, (1024, 1024)),
    "tiny_3x8": lambda: workloads.single_matrix(5, shape=(3, 8)),
}
for name, make in blocks.items():
    mats = [m for _, m in make()]
    cb = df11.build_codebook(mats)
    for bpt in (8, 16):
        hb = df11.compress(cb, mats, 32, bpt)
        n = hb.n_elements
        for ws in (True, False):
            run(f"{name}/bpt{bpt}/ws{ws}", hb, mats,
                lambda db, o, e, ws=ws: df11.decompress_async(db, o, e, capacity=n, workspace=ws))
        nch = int(hb.header.n_chunks)
        cuts = sorted({0, nch // 3, nch // 2, nch})
        def ranges(db, o, e, cuts=cuts):
            for c0, c1 in zip(cuts[:-1], cuts[1:]):
                if c1 > c0:
                    df11.decompress_range_async(db, c0, c1, o, e)
        run(f"{name}/bpt{bpt}/ranges", hb, mats, ranges)
    # corrupt positions: the decoder reports them, the checks stay quiet
    hb = df11.compress(cb, mats)
    if hb.header.n_chunks >= 3:
        bad = df11.compress(cb, mats)
        bad.chunk_pos[1] += 1
        run(f"{name}/corrupt_pos", bad, None, lambda db, o, e: df11.decompress_async(db, o, e, capacity=hb.n_elements))
# fused products
mats = [m for _, m in workloads.llama_block(3000, scale_div=64)]
hb = df11.compress(df11.build_codebook(mats), mats)
db = hb.to_device("cuda")
shapes = [m.shape for m in mats]
xs = [torch.from_numpy(workloads.activations(7 + i, 3, c).view(np.int16)).cuda() for i, (_, c) in enumerate(shapes)]
ys = [torch.zeros(3, r, dtype=torch.float32, device="cuda") for r, _ in shapes]
err = torch.zeros(1, dtype=torch.int32, device="cuda")
df11.decode_gemv_async(db, shapes, xs, ys, err)
torch.cuda.synchronize()
out["cases"].append({"name": "gemv", "err": int(err.item()), "exact": True, "guard": True})
print(json.dumps(out))
'''


@pytest.fixture(scope="module")
def child_report():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    env = dict(os.environ, DF11_CHECKED="1", PYTHONPATH=ROOT + os.pathsep + os.environ.get("PYTHONPATH", ""))
    res = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True, text=True,
                         timeout=900)
    assert res.returncode == 0, res.stderr[-3000:]
    return json.loads(res.stdout.strip().splitlines()[-1])


def test_the_checked_library_is_the_one_loaded(child_report):
    assert child_report["lib"].endswith("libdf11_checked.so")


def test_no_bounds_error_and_exact_output(child_report):
    import huffman_decode_b200 as df11
    cases = child_report["cases"]
    assert len(cases) > 40
    for c in cases:
        assert not (c["err"] & df11.DEVERR_BOUNDS), c
        assert c["guard"], c
        if "corrupt" in c["name"]:
            assert c["err"] & (df11.DEVERR_COUNT | df11.DEVERR_BAD_POS), c
        else:
            assert c["err"] == 0 and c["exact"], c
