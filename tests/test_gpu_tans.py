"""GPU parity of the tANS exponent coder (coder 1) against the CPU oracle, through the C ABI.

* encode bytes == oracle bytes (integer work: exact), edge cases to full-size tensors;
* decode of oracle-written containers == the input, bit for bit, every table size;
* range, batch and host-streamed decodes of tANS containers;
* corrupt containers and coder mismatches set the device status word and never fault.
"""
import numpy as np
import pytest
import torch

import oracle
import lossless_entropy_coded_exponent_b200 as dfx
from lossless_entropy_coded_exponent_b200 import build as dfx_build
from lossless_entropy_coded_exponent_b200 import inputs

pytestmark = pytest.mark.gpu
TANS = dfx.DFX_CODER_TANS


@pytest.fixture(scope="module", autouse=True)
def _lib():
    dfx_build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dfx.lib()


def to_dev(w: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(w).view(np.int16)).cuda()


def to_host_u16(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def plan_for(n: int, K: int, R: int = 12):
    return dfx.dfx_plan(n, chunk_symbols=K, coder=TANS, table_log=R)


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


def gpu_decode(c: np.ndarray, n: int, K: int, R: int = 12):
    comp = torch.from_numpy(c).cuda()
    with plan_for(n, K, R) as plan:
        out = torch.full((max(n, 1),), -1, dtype=torch.int16, device="cuda")
        dfx.dfx_decode(plan, comp, comp.numel(), out)
        st = dfx.dfx_device_status(plan)
    return to_host_u16(out)[:n], st


SMALL_CASES = {"small_gaussian": inputs.small_gaussian, **{k: (lambda k=k: inputs.edge_cases()[k]) for k in inputs.edge_cases()}}


@pytest.mark.parametrize("K", [128, 64, 32])
@pytest.mark.parametrize("name", list(SMALL_CASES))
def test_encode_bytes_match_oracle(name, K):
    w = SMALL_CASES[name]()
    ref = oracle.encode_tans(w, K=K)
    got = gpu_encode(w, K)
    assert got.size == ref.size
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("K", [128, 64, 32])
@pytest.mark.parametrize("name", list(SMALL_CASES))
def test_decode_oracle_container(name, K):
    w = SMALL_CASES[name]()
    got, st = gpu_decode(oracle.encode_tans(w, K=K), w.size, K)
    assert st == 0, hex(st)
    assert np.array_equal(got, w)


@pytest.mark.parametrize("R", [8, 9, 10, 11])
def test_encode_every_table_size(R):
    w = inputs.projection_with_outliers()[: 4096 * 50 + 77].copy()
    ref = oracle.encode_tans(w, K=128, table_log=R)
    got = gpu_encode(w, 128, R)
    assert np.array_equal(got, ref)
    dec, st = gpu_decode(got, w.size, 128, R)
    assert st == 0 and np.array_equal(dec, w)


def few_exponents(n: int, values: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    e = (120 + rng.integers(0, values, size=n)).astype(np.uint16)
    return ((rng.integers(0, 2, size=n, dtype=np.uint16) << 15) | (e << 7) |
            rng.integers(0, 128, size=n, dtype=np.uint16)).astype(np.uint16)


@pytest.mark.parametrize("R", [4, 5, 6, 7])
def test_decode_small_tables(R):
    """Tables of 16..128 states (the encoder needs room for 256 values, the decoder not)."""
    w = few_exponents(4096 * 40 + 5, min(1 << R, 12), seed=R)
    c = oracle.encode_tans(w, K=64, table_log=R)
    got, st = gpu_decode(c, w.size, 64, R)
    assert st == 0, hex(st)
    assert np.array_equal(got, w)


def test_projection_with_outliers_round_trip():
    w = inputs.projection_with_outliers()
    for K in (128, 64):
        got = gpu_encode(w, K)
        assert np.array_equal(got, oracle.encode_tans(w, K=K))
        dec, st = gpu_decode(got, w.size, K)
        assert st == 0 and np.array_equal(dec, w)


def test_layer_tensor_full_size():
    """A 14336 x 4096 projection: encode bytes equal the oracle's, decode restores it."""
    w = inputs.llama3_8b_layer_tensor(4)
    ref = oracle.encode_tans(w, K=128)
    got = gpu_encode(w, 128)
    assert got.size == ref.size and np.array_equal(got, ref)
    dec, st = gpu_decode(got, w.size, 128)
    assert st == 0 and np.array_equal(dec, w)


def test_layer70b_tensor_full_size():
    """One 8192 x 28672 tensor of the 70B layer stream, decoded twice into a reused
    buffer as in the benchmark; encode bytes equal the oracle's."""
    w = inputs.layer70b_tensor(0)
    ref = oracle.encode_tans(w, K=128)
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


def test_ranges_batch_and_host_stream():
    ge = 32 * 128
    w0 = inputs.projection_with_outliers()[: ge * 40 + 1001].copy()
    w1 = inputs.gaussian(ge * 7 + 8, 0.03, seed=12)
    c0, c1 = oracle.encode_tans(w0, K=128), oracle.encode_tans(w1, K=128)
    d0, d1 = torch.from_numpy(c0).cuda(), torch.from_numpy(c1).cuda()
    ng = -(-w0.size // ge)
    with plan_for(w0.size, 128) as p0, plan_for(w1.size, 128) as p1:
        for first, count in [(0, ng), (3, 5), (ng - 1, 1), (ng // 2, ng - ng // 2)]:
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
        host = torch.from_numpy(c0).pin_memory()
        staging = torch.empty(c0.size, dtype=torch.uint8, device="cuda")
        o0.fill_(-1)
        s_copy, s_dec = torch.cuda.Stream(), torch.cuda.Stream()
        dfx.dfx_decode_host(p0, host, c0.size, staging, c0.size, o0, slices=5, copy_stream=s_copy, decode_stream=s_dec)
        s_dec.synchronize()
        assert dfx.dfx_device_status(p0, stream=s_dec) == 0
        assert np.array_equal(to_host_u16(o0), w0)
    with plan_for(w1.size, 128) as pt, dfx.dfx_plan(w1.size, chunk_symbols=128) as ph:
        with pytest.raises(dfx.DfxError) as e:  # one launch decodes one coder
            dfx.dfx_decode_batch([pt, ph], [d1, d1], [d1.numel(), d1.numel()], [o1, o1])
        assert e.value.code == dfx.DFX_ERR_UNSUPPORTED


def corrupt_variants(c: np.ndarray) -> dict:
    ng = int(c[44:48].view(np.uint32)[0])
    nc = int(c[40:44].view(np.uint32)[0])
    off_clen = (576 + 8 * (ng + 1) + 15) // 16 * 16
    off_stream = (int(c[48:56].view(np.uint64)[0]) + int(c[8:16].view(np.uint64)[0]) + 15) // 16 * 16
    used = int(np.flatnonzero(c[64:576:2])[0])
    v = {}
    x = c.copy(); x[0] ^= 1; v["magic"] = (x, dfx.DFX_STATUS_HEADER)
    x = c.copy(); x[60] = 0; v["coder"] = (x, dfx.DFX_STATUS_HEADER)
    x = c.copy(); x[56] = 13; v["table_log"] = (x, dfx.DFX_STATUS_HEADER)
    x = c.copy(); x[24] ^= 0x10; v["total_bytes"] = (x, dfx.DFX_STATUS_HEADER)
    x = c.copy(); x[64 + 2 * used] += 1; v["freq_sum"] = (x, dfx.DFX_STATUS_TABLE)
    x = c.copy(); x[576 + 8 * (ng // 2)] ^= 0x3; v["gbase"] = (x, dfx.DFX_STATUS_INDEX)
    x = c.copy(); x[off_clen + 2 * (nc // 3)] ^= 0x1; v["clen"] = (x, dfx.DFX_STATUS_INDEX)
    x = c.copy(); x[off_stream: off_stream + 4096] = 0xFF; v["stream_ones"] = (x, dfx.DFX_STATUS_STREAM)
    x = c.copy(); x[off_stream + 3] ^= 0x80; v["first_state"] = (x, dfx.DFX_STATUS_STREAM)
    return v


def test_corrupt_containers_set_status_and_do_not_fault():
    w = inputs.gaussian(1 << 20, 0.02, seed=7)
    c = oracle.encode_tans(w, K=64)
    for name, (bad, flag) in corrupt_variants(c).items():
        with pytest.raises(oracle.OracleError):  # the oracle rejects each of them too
            oracle.decode(bad)
        _, st = gpu_decode(bad, w.size, 64)
        assert st & flag, (name, hex(st))
    got, st = gpu_decode(c, w.size, 64)  # the context is still healthy afterwards
    assert st == 0 and np.array_equal(got, w)


def test_coder_mismatch_is_a_header_error():
    w = inputs.gaussian(4096 * 9, 0.02, seed=9)
    _, st = gpu_decode(oracle.encode(w, K=64), w.size, 64)  # a Huffman container, tANS plan
    assert st & dfx.DFX_STATUS_HEADER
    comp = torch.from_numpy(oracle.encode_tans(w, K=64)).cuda()
    with dfx.dfx_plan(w.size, chunk_symbols=64) as plan:  # a tANS container, Huffman plan
        out = torch.empty(w.size, dtype=torch.int16, device="cuda")
        dfx.dfx_decode(plan, comp, comp.numel(), out)
        assert dfx.dfx_device_status(plan) & dfx.DFX_STATUS_HEADER


def test_encode_refuses_tables_too_small_for_all_exponents():
    x = to_dev(inputs.gaussian(1000, 0.02, seed=3))
    with plan_for(1000, 128, 7) as plan:
        out = torch.empty(plan.max_compressed_bytes, dtype=torch.uint8, device="cuda")
        ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
        with pytest.raises(dfx.DfxError) as e:
            dfx.dfx_encode(plan, x, out, out.numel(), ws, ws.numel())
        assert e.value.code == dfx.DFX_ERR_UNSUPPORTED


def test_bounded_wait_runs_out_and_reports_timeout():
    w = inputs.gaussian(4096 * 32 * 4, 0.02, seed=5)
    c = oracle.encode_tans(w, K=128)
    dfx.dfx_debug_inject(dfx.DFX_INJECT_SKIP_SLICE_COPY)
    try:
        _, st = gpu_decode(c, w.size, 128)
    finally:
        dfx.dfx_debug_inject(0)
    assert st & dfx.DFX_STATUS_TIMEOUT
    got, st = gpu_decode(c, w.size, 128)
    assert st == 0 and np.array_equal(got, w)
