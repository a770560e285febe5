"""Decode fused with matrix-vector products (df11_decode_gemv_async) against
an FP64 reference.

For matrix i of the block the kernel adds x_i W_i^T into y_i (FP32) while it
decodes W_i.  The weights are the block's input BF16 values, which the
oracle's serial decode of the artifact reproduces bit for bit (checked here),
so the reference is the plain FP64 product of those weights and the BF16
activations.  Tolerance, from the arithmetic: every y entry is a sum of
n = cols products of BF16 numbers (exact in FP32) formed with FP32 fused
multiply-adds and FP32 atomic adds, at most n + 1 roundings on any path of
the summation tree, so |y - y_ref| <= gamma(n + 1) * sum |w x| with
gamma(k) = k u / (1 - k u), u = 2^-24 (the standard bound for summation in
any order).  Page: "DFloat11: lossless BFloat16 compression", "Architecture"
(a block's weights are decoded and then consumed by its matrix products).
"""
import numpy as np
import pytest

import oracle
import workloads
import huffman_decode_b200 as df11

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

U = 2.0 ** -24


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def run_and_check(mats, n_tokens, bytes_per_thread=16, seed=77, workspace=True):
    cb = df11.build_codebook(mats)
    hb = df11.compress(cb, mats, 32, bytes_per_thread)
    flat = np.concatenate([m.reshape(-1) for m in mats])
    # the weights the kernel sees are the oracle's decode of the artifact
    ref_bits = oracle.decode_block(hb.exp_stream, hb.n_elements, cb.lengths(), hb.signmant)
    assert np.array_equal(ref_bits, flat)
    db = hb.to_device("cuda")
    shapes = [m.shape for m in mats]
    xs_host = [workloads.activations(seed + i, n_tokens, c) for i, (_, c) in enumerate(shapes)]
    xs = [torch.from_numpy(x.view(np.int16)).cuda() for x in xs_host]
    ys = [torch.zeros(n_tokens, r, dtype=torch.float32, device="cuda") for r, _ in shapes]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.decode_gemv_async(db, shapes, xs, ys, err, workspace=workspace)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for i, (m, x) in enumerate(zip(mats, xs_host)):
        w = _f64(m)
        xf = _f64(x)
        y_ref = xf @ w.T
        mag = np.abs(xf) @ np.abs(w).T
        k = m.shape[1] + 1
        tol = k * U / (1 - k * U) * mag + 1e-30
        got = ys[i].cpu().numpy().astype(np.float64)
        bad = np.nonzero(np.abs(got - y_ref) > tol)
        assert bad[0].size == 0, (f"matrix {i} {m.shape}: {bad[0].size} entries off, first "
                                  f"{got[bad][:3]} vs {y_ref[bad][:3]} (tol {tol[bad][:3]})")
    return ys


@pytest.mark.parametrize("n_tokens", [1, 3, 8])
@pytest.mark.parametrize("bpt", [8, 16])
def test_llama_block_products(n_tokens, bpt):
    mats = [m for _, m in workloads.llama_block(3000, scale_div=64)]
    run_and_check(mats, n_tokens, bpt)


@pytest.mark.parametrize("workspace", [True, False])
def test_products_under_both_chunk_schedules(workspace):
    """A block of over five rounds of chunks for a full wave of warps, so
    with a workspace the last rounds really are claimed."""
    mats = [m for _, m in workloads.llama_block(3002, scale_div=4)]
    run_and_check(mats, 2, workspace=workspace)


def test_flux_block_69_matrices():
    """69 matrices; 64 of them have rows of exactly 256 elements."""
    mats = [m for _, m in workloads.flux_block(5100, scale_div=64)]
    run_and_check(mats, 2)


@pytest.mark.parametrize("n_tokens", [1, 4])
def test_rows_shorter_than_a_step(n_tokens):
    mats = [m for _, m in workloads.small_cols_block()]
    run_and_check(mats, n_tokens)


def test_one_bit_codes_and_many_tables():
    """A 1-bit code and many second-level tables; the rare exponents stay in
    a range whose products and sums are finite in FP32."""
    mats = [m for _, m in workloads.many_tables(rare_exponents=range(0x20, 0xC0))]
    cb = df11.build_codebook(mats)
    assert cb.n_tables >= 20
    run_and_check(mats, 5)


def test_products_match_decode_then_matmul():
    """The fused result against decoding to BF16 and multiplying on the GPU
    (cuBLAS, FP32 accumulation): both are within the summation bound of the
    FP64 product, so they agree to twice that bound."""
    mats = [m for _, m in workloads.llama_block(3001, scale_div=128)]
    n_tokens = 4
    ys = run_and_check(mats, n_tokens, seed=91)
    cb = df11.build_codebook(mats)
    hb = df11.compress(cb, mats)
    db = hb.to_device("cuda")
    out = torch.empty(hb.n_elements, dtype=torch.bfloat16, device="cuda")
    df11.decompress_async(db, out)
    off = 0
    for i, m in enumerate(mats):
        r, c = m.shape
        w = out[off:off + r * c].view(r, c).float()
        x = torch.from_numpy(workloads.activations(91 + i, n_tokens, c).view(np.int16)).cuda()
        x = (x.to(torch.int32) << 16).view(torch.float32)
        y2 = x @ w.t()
        mag = (x.abs() @ w.abs().t()).double()
        k = c + 1
        tol = 2 * k * U / (1 - k * U) * mag + 1e-30
        assert bool(((ys[i].double() - y2.double()).abs() <= tol).all()), i
        off += r * c
