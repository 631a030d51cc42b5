"""GPU parity of the tANS coder with two interleaved states per chunk (coder 2) against the
CPU oracle (rule T6), through the C ABI:

* encode bytes == oracle bytes (integer work: exact), edge cases to a full-size 70B-layer
  tensor, ragged last chunks whose odd length ends on state A;
* decode of oracle-written containers == the input, bit for bit, every chunk size and
  several table sizes; range and batch decodes;
* a coder-1 container given to a coder-2 plan (and the reverse) is a header error.
"""
import numpy as np
import pytest
import torch

import oracle
import lossless_entropy_coded_exponent_b200 as dfx
from lossless_entropy_coded_exponent_b200 import build as dfx_build
from lossless_entropy_coded_exponent_b200 import inputs

pytestmark = pytest.mark.gpu
TANS2 = dfx.DFX_CODER_TANS2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    dfx_build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dfx.lib()


def to_dev(w: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(w).view(np.int16)).cuda()


def to_host_u16(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def plan_for(n: int, K: int, R: int = 12, coder: int = TANS2):
    return dfx.dfx_plan(n, chunk_symbols=K, coder=coder, table_log=R)


def gpu_encode(w: np.ndarray, K: int, R: int = 12) -> np.ndarray:
    x = to_dev(w)
    with plan_for(w.size, K, R) as plan:
        out = torch.full((plan.max_compressed_bytes,), 0xAB, dtype=torch.uint8, device="cuda")
        ws = torch.full((plan.workspace_bytes,), 0xCD, dtype=torch.uint8, device="cuda")
        size = dfx.dfx_encode(plan, x, out, out.numel(), ws, ws.numel(), want_size=True)
        assert dfx.dfx_device_status(plan) == 0
        host = out.cpu().numpy()
    assert np.all(host[size:] == 0), "bytes past the container must be zeroed"
    return host[:size].copy()


def gpu_decode(c: np.ndarray, n: int, K: int, R: int = 12, coder: int = TANS2):
    comp = torch.from_numpy(c).cuda()
    with plan_for(n, K, R, coder) as plan:
        out = torch.full((max(n, 1),), -1, dtype=torch.int16, device="cuda")
        dfx.dfx_decode(plan, comp, comp.numel(), out)
        st = dfx.dfx_device_status(plan)
    return to_host_u16(out)[:n], st


SMALL_CASES = {"small_gaussian": inputs.small_gaussian,
               **{k: (lambda k=k: inputs.edge_cases()[k]) for k in inputs.edge_cases()}}


@pytest.mark.parametrize("K", [128, 64, 32])
@pytest.mark.parametrize("name", list(SMALL_CASES))
def test_encode_bytes_match_oracle(name, K):
    w = SMALL_CASES[name]()
    ref = oracle.encode_tans(w, K=K, states=2)
    got = gpu_encode(w, K)
    assert got.size == ref.size and np.array_equal(got, ref)


@pytest.mark.parametrize("K", [128, 64, 32])
@pytest.mark.parametrize("name", list(SMALL_CASES))
def test_decode_oracle_container(name, K):
    w = SMALL_CASES[name]()
    got, st = gpu_decode(oracle.encode_tans(w, K=K, states=2), w.size, K)
    assert st == 0 and np.array_equal(got, w)


@pytest.mark.parametrize("n", [1, 7, 9, 4096 * 3 + 13, 4096 * 5 + 8 * 7 + 5])
def test_ragged_chunks(n):
    """The last chunk holds an odd number of elements (its last symbol on state A) or a
    partial block: encode equals the oracle, decode restores the input."""
    w = inputs.gaussian(n, 0.02, seed=n)
    ref = oracle.encode_tans(w, K=128, states=2)
    got = gpu_encode(w, 128)
    assert np.array_equal(got, ref)
    dec, st = gpu_decode(got, w.size, 128)
    assert st == 0 and np.array_equal(dec, w)


@pytest.mark.parametrize("R", [8, 10, 12])
def test_table_sizes(R):
    w = inputs.projection_with_outliers()
    ref = oracle.encode_tans(w, K=64, table_log=R, states=2)
    got = gpu_encode(w, 64, R)
    assert np.array_equal(got, ref)
    dec, st = gpu_decode(ref, w.size, 64, R)
    assert st == 0 and np.array_equal(dec, w)


def test_layer70b_tensor_full_size():
    """One 8192 x 28672 tensor of the 70B layer stream: encode bytes equal the oracle's,
    decoded twice into a reused buffer as in the benchmark."""
    w = inputs.layer70b_tensor(0)
    ref = oracle.encode_tans(w, K=128, states=2)
    got = gpu_encode(w, 128)
    assert got.size == ref.size and np.array_equal(got, ref)
    comp = torch.from_numpy(got).cuda()
    x = to_dev(w)
    with plan_for(w.size, 128) as plan:
        out = torch.empty_like(x)
        for _ in range(2):
            dfx.dfx_decode(plan, comp, comp.numel(), out)
        assert dfx.dfx_device_status(plan) == 0
    assert torch.equal(out, x)


def test_ranges_and_batch():
    ge = 32 * 128
    w0 = inputs.projection_with_outliers()[: ge * 40 + 1001].copy()
    w1 = inputs.gaussian(ge * 7 + 8, 0.03, seed=12)
    c0, c1 = oracle.encode_tans(w0, K=128, states=2), oracle.encode_tans(w1, K=128, states=2)
    d0, d1 = torch.from_numpy(c0).cuda(), torch.from_numpy(c1).cuda()
    ng = -(-w0.size // ge)
    with plan_for(w0.size, 128) as p0, plan_for(w1.size, 128) as p1:
        for first, count in [(0, ng), (3, 5), (ng - 1, 1)]:
            m = min(w0.size, (first + count) * ge) - first * ge
            out = torch.full((m,), -1, dtype=torch.int16, device="cuda")
            dfx.dfx_decode_range(p0, d0, d0.numel(), first, count, out)
            assert dfx.dfx_device_status(p0) == 0
            assert np.array_equal(to_host_u16(out), w0[first * ge: first * ge + m]), (first, count)
        o0 = torch.empty(w0.size, dtype=torch.int16, device="cuda")
        o1 = torch.empty(w1.size, dtype=torch.int16, device="cuda")
        dfx.dfx_decode_batch([p0, p1], [d0, d1], [d0.numel(), d1.numel()], [o0, o1])
        assert dfx.dfx_device_status(p0) == 0 and dfx.dfx_device_status(p1) == 0
        assert np.array_equal(to_host_u16(o0), w0) and np.array_equal(to_host_u16(o1), w1)


def test_coder_mismatch_is_a_header_error():
    w = inputs.gaussian(5000, 0.02, seed=4)
    one = oracle.encode_tans(w, K=64)
    two = oracle.encode_tans(w, K=64, states=2)
    _, st = gpu_decode(one, w.size, 64, coder=TANS2)
    assert st & dfx.DFX_STATUS_HEADER
    _, st = gpu_decode(two, w.size, 64, coder=dfx.DFX_CODER_TANS)
    assert st & dfx.DFX_STATUS_HEADER


def test_corrupt_containers_set_status_and_do_not_fault():
    w = inputs.gaussian(20000, 0.02, seed=6)
    c = oracle.encode_tans(w, K=64, states=2)
    rng = np.random.default_rng(2)
    flagged = 0
    for _ in range(12):
        bad = c.copy()
        pos = int(rng.integers(c.size - 400, c.size - 16))
        bad[pos] ^= np.uint8(1 << int(rng.integers(0, 8)))
        dec, st = gpu_decode(bad, w.size, 64)
        flagged += st != 0
    assert flagged >= 8
