"""GPU parity of dfx_decode_gemm: Y = X W^T with W decoded from its container inside
the GEMM kernel (tcgen05 tensor cores, FP32 accumulation in tensor memory).

* the decoded W the kernel multiplies (written to d_w_out on request) equals the input
  bit for bit, i.e. the oracle's decode of the same container;
* on an integer grid (W = k * 2^-6 with |k| <= 256, X integers in [-8, 8]) every
  product and every partial sum is a multiple of 2^-6 below 2^18 in magnitude, exact in
  FP32, so Y must equal the exact product bit for bit whatever the accumulation order;
* on Gaussian weights Y agrees with the exact product (float64 from the same BF16
  values) within the bound of FP32 summation in any order,
  |Y - Y_exact| <= K * 2^-23 * sum_k |x_k w_k| (each BF16 x BF16 product is exact in
  FP32, each of the K - 1 additions rounds with a relative error of at most 2^-24, and
  2^-23 covers an accumulator that truncates);
* argument checks, a corrupt container, and the full-size gate projection of the
  Llama-3-8B-shaped layer.
"""
import numpy as np
import pytest
import torch

import oracle
import lossless_entropy_coded_exponent_b200 as dfx
from lossless_entropy_coded_exponent_b200 import build as dfx_build
from lossless_entropy_coded_exponent_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    dfx_build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dfx.lib()


def bf16_to_f64(u16: np.ndarray) -> np.ndarray:
    return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def make_x(tokens: int, cols: int, seed: int) -> np.ndarray:
    """tokens x cols BF16 activations (as u16): N(0, 0.5^2) rounded to nearest even."""
    return inputs.gaussian(tokens * cols, 0.5, seed=seed).reshape(tokens, cols)


def grid_w(n: int, seed: int) -> np.ndarray:
    """BF16 weights k * 2^-6, k = a rounded N(0, 40^2) draw clipped to [-256, 256]."""
    k = np.clip(np.rint(np.random.default_rng(seed).standard_normal(n) * 40.0), -256, 256)
    return inputs.bf16_from_f32((k * 2.0 ** -6).astype(np.float32))


def grid_x(tokens: int, cols: int, seed: int) -> np.ndarray:
    """BF16 activations: integers uniform in [-8, 8]."""
    v = np.random.default_rng(seed).integers(-8, 9, size=(tokens, cols)).astype(np.float32)
    return inputs.bf16_from_f32(v)


def check_y_exact(y: np.ndarray, x16: np.ndarray, w16: np.ndarray) -> None:
    exact = bf16_to_f64(x16) @ bf16_to_f64(w16).T
    assert np.all(np.abs(exact) < 2.0 ** 18) and np.array_equal(exact, exact.astype(np.float32))
    assert np.array_equal(y, exact.astype(np.float32))


def check_y(y: np.ndarray, x16: np.ndarray, w16: np.ndarray) -> float:
    xf, wf = bf16_to_f64(x16), bf16_to_f64(w16)
    exact = xf @ wf.T
    bound = x16.shape[1] * 2.0 ** -23 * (np.abs(xf) @ np.abs(wf).T)
    err = np.abs(y.astype(np.float64) - exact)
    assert np.all(err <= bound + 1e-30), f"max excess {float(np.max(err - bound))}"
    return float(np.max(err / np.maximum(bound, 1e-30)))


def run_gemm(comp: np.ndarray, rows: int, cols: int, x16: np.ndarray, K: int, want_w: bool = True,
             expect_status: int = 0):
    tokens = x16.shape[0]
    with dfx.dfx_plan(rows * cols, chunk_symbols=K) as plan:
        d_comp = torch.from_numpy(comp).cuda()
        d_x = torch.from_numpy(np.ascontiguousarray(x16).view(np.int16)).cuda()
        d_y = torch.full((tokens, rows), float("nan"), dtype=torch.float32, device="cuda")
        d_w = torch.full((rows * cols,), -1, dtype=torch.int16, device="cuda") if want_w else None
        dfx.dfx_decode_gemm(plan, d_comp, d_comp.numel(), rows, cols, d_x, tokens, d_y, d_w)
        st = dfx.dfx_device_status(plan)
        if expect_status == 0:
            assert st == 0, f"device status 0x{st:x}"
        y = d_y.cpu().numpy()
        w = d_w.cpu().numpy().view(np.uint16) if want_w else None
    return y, w, st


CASES = [
    # rows, cols, K, tokens
    (256, 4096, 128, 16),   # one group per row, two CTAs' worth of rows per SM at most
    (300, 4096, 128, 1),    # ragged tiles, one token
    (7, 4096, 128, 5),      # fewer rows than SMs
    (130, 8192, 128, 17),   # two groups per row, 32 accumulator columns
    (96, 4096, 64, 32),     # K = 64: two groups per row, the largest token count
    (40, 2048, 32, 3),      # K = 32: two groups per row
]


@pytest.mark.parametrize("rows,cols,K,tokens", CASES)
def test_decode_gemm_exact_on_integer_grid(rows, cols, K, tokens):
    w16 = grid_w(rows * cols, seed=rows + cols + K)
    x16 = grid_x(tokens, cols, seed=tokens + 500)
    comp = oracle.encode(w16, K=K)
    y, w, _ = run_gemm(comp, rows, cols, x16, K)
    assert np.array_equal(w, w16), "the decoded W inside the GEMM differs from the input"
    assert np.array_equal(w, oracle.decode(comp))
    check_y_exact(y, x16, w16.reshape(rows, cols))


@pytest.mark.parametrize("rows,cols,K,tokens", CASES[:3])
def test_decode_gemm_gaussian_within_fp32_bound(rows, cols, K, tokens):
    w16 = inputs.gaussian(rows * cols, 0.02, seed=rows + cols + K)
    x16 = make_x(tokens, cols, seed=tokens + 500)
    comp = oracle.encode(w16, K=K)
    y, w, _ = run_gemm(comp, rows, cols, x16, K)
    assert np.array_equal(w, w16)
    check_y(y, x16, w16.reshape(rows, cols))


def test_decode_gemm_one_hot_columns():
    """Token t of X is 2^(t mod 5) at column k_t and zero elsewhere, so Y[t] is column
    k_t of W times that power of two, exactly; the k_t cover every 16-byte chunk
    position of every K atom of a step, both halves of a pair and several steps."""
    rows, cols = 160, 4096
    w16 = inputs.gaussian(rows * cols, 0.02, seed=31)
    ks = [0, 1, 7, 8, 63, 64, 130, 255, 256, 1000, 2047, 2048, 3071, 3333, 4094, 4095] + list(range(9, 4096, 257))[:16]
    x = np.zeros((len(ks), cols), dtype=np.float32)
    for t, k in enumerate(ks):
        x[t, k] = 2.0 ** (t % 5)
    x16 = inputs.bf16_from_f32(x)
    comp = oracle.encode(w16, K=128)
    y, w, _ = run_gemm(comp, rows, cols, x16, 128)
    wf = bf16_to_f64(w16.reshape(rows, cols))
    for t, k in enumerate(ks):
        assert np.array_equal(y[t], (wf[:, k] * 2.0 ** (t % 5)).astype(np.float32)), (t, k)


def test_decode_gemm_long_codes():
    """A code book that reaches the 24-bit length limit: the Fibonacci-count tensor
    (exponents 100..127, counts F1..F28) padded to 204 whole rows of 4096 with more
    values of its most frequent exponent, so codes longer than the 14-bit pair table
    take the canonical path inside the GEMM."""
    rows, cols = 204, 4096
    fib = inputs.fibonacci_clamp_tensor(3)
    pad = (np.uint16(127) << np.uint16(7)) | (np.arange(rows * cols - fib.size, dtype=np.uint16) & np.uint16(0x807F))
    w16 = np.concatenate([fib, pad.astype(np.uint16)])
    assert oracle.code_lengths(oracle.histogram(w16)).max() == 24
    x16 = make_x(16, cols, seed=77)
    comp = oracle.encode(w16, K=128)
    y, w, _ = run_gemm(comp, rows, cols, x16, 128)
    assert np.array_equal(w, w16)
    check_y(y, x16, w16.reshape(rows, cols))


def test_decode_gemm_without_w_out_equals_with_it():
    rows, cols = 200, 4096
    w16 = inputs.gaussian(rows * cols, 0.02, seed=3)
    x16 = make_x(16, cols, seed=4)
    comp = oracle.encode(w16, K=128)
    y1, _, _ = run_gemm(comp, rows, cols, x16, 128, want_w=True)
    y2, _, _ = run_gemm(comp, rows, cols, x16, 128, want_w=False)
    assert np.array_equal(y1, y2)


def test_gate_projection_full_size():
    """The gate projection of the Llama-3-8B-shaped layer (14336 x 4096, N(0, 1/4096)),
    X 16 x 4096: the configuration the benchmark times."""
    rows, cols = 14336, 4096
    w16 = inputs.llama3_8b_layer_tensor(4)
    assert w16.size == rows * cols
    x16 = make_x(16, cols, seed=7)
    comp = oracle.encode(w16, K=128)
    y, w, _ = run_gemm(comp, rows, cols, x16, 128)
    assert np.array_equal(w, w16)
    check_y(y, x16, w16.reshape(rows, cols))


def test_decode_gemm_argument_checks():
    rows, cols = 64, 4096
    w16 = inputs.gaussian(rows * cols, 0.02, seed=9)
    comp = torch.from_numpy(oracle.encode(w16, K=128)).cuda()
    x = torch.zeros(33, cols, dtype=torch.int16, device="cuda")
    y = torch.zeros(33, rows, dtype=torch.float32, device="cuda")

    def code(**kw):
        args = dict(rows=rows, cols=cols, tokens=16)
        args.update(kw)
        with dfx.dfx_plan(rows * cols) as plan:
            with pytest.raises(dfx.DfxError) as e:
                dfx.dfx_decode_gemm(plan, comp, comp.numel(), args["rows"], args["cols"], x, args["tokens"], y)
            return e.value.code

    assert code(tokens=0) == dfx.DFX_ERR_ARG
    assert code(tokens=33) == dfx.DFX_ERR_ARG
    assert code(rows=128, cols=2048) == dfx.DFX_ERR_UNSUPPORTED  # a group would span two rows
    assert code(rows=65) == dfx.DFX_ERR_ARG                      # rows * cols != n
    with dfx.dfx_plan(rows * cols, coder=dfx.DFX_CODER_TANS) as plan:
        with pytest.raises(dfx.DfxError) as e:
            dfx.dfx_decode_gemm(plan, comp, comp.numel(), rows, cols, x, 16, y)
        assert e.value.code == dfx.DFX_ERR_UNSUPPORTED


def test_decode_gemm_same_n_other_shape():
    """The plan fixes n only: the same container read as 32 x 8192 (two groups per row)
    gives that shape's product."""
    w16 = grid_w(64 * 4096, seed=12)
    x16 = grid_x(4, 8192, seed=13)
    comp = oracle.encode(w16, K=128)
    y, w, _ = run_gemm(comp, 32, 8192, x16, 128)
    assert np.array_equal(w, w16)
    check_y_exact(y, x16, w16.reshape(32, 8192))


def test_decode_gemm_corrupt_container_sets_status():
    rows, cols = 64, 4096
    w16 = inputs.gaussian(rows * cols, 0.02, seed=14)
    c = oracle.encode(w16, K=128)
    ng = int(c[44:48].view(np.uint32)[0])
    off_clen = (320 + 8 * (ng + 1) + 15) // 16 * 16
    bad = c.copy()
    bad[off_clen + 2 * 100] ^= 0x1  # one chunk length
    x16 = make_x(16, cols, seed=15)
    _, _, st = run_gemm(bad, rows, cols, x16, 128, expect_status=dfx.DFX_STATUS_INDEX)
    assert st & dfx.DFX_STATUS_INDEX
    bad = c.copy()
    bad[0] ^= 1  # magic
    _, _, st = run_gemm(bad, rows, cols, x16, 128, expect_status=dfx.DFX_STATUS_HEADER)
    assert st & dfx.DFX_STATUS_HEADER
    # the context is healthy afterwards
    y, w, _ = run_gemm(c, rows, cols, x16, 128)
    assert np.array_equal(w, w16)
    check_y(y, x16, w16.reshape(rows, cols))
