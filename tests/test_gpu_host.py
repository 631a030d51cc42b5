"""GPU parity of the host-streamed decode (dfx_decode_host: a container in pinned host
memory copied slice by slice while the slices decode) against the input, bit for bit."""
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


def decode_from_host(c: np.ndarray, n: int, K: int, slices: int, staging_bytes=None):
    host = torch.from_numpy(c).pin_memory()
    cap = c.size if staging_bytes is None else staging_bytes
    staging = torch.full((max(cap, 16),), 0xEE, dtype=torch.uint8, device="cuda")
    out = torch.full((max(n, 1),), -1, dtype=torch.int16, device="cuda")
    s_copy, s_dec = torch.cuda.Stream(), torch.cuda.Stream()
    with dfx.dfx_plan(n, chunk_symbols=K) as plan:
        dfx.dfx_decode_host(plan, host, c.size, staging, cap, out, slices=slices, copy_stream=s_copy,
                            decode_stream=s_dec)
        s_dec.synchronize()
        st = dfx.dfx_device_status(plan, stream=s_dec)
    return out.cpu().numpy().view(np.uint16)[:n], st


@pytest.mark.parametrize("K", [128, 64])
@pytest.mark.parametrize("slices", [1, 3, 8, 0, 64])
def test_host_stream_round_trip(K, slices):
    w = inputs.projection_with_outliers()[: 4096 * 100 + 333].copy()
    got, st = decode_from_host(oracle.encode(w, K=K), w.size, K, slices)
    assert st == 0
    assert np.array_equal(got, w)


def test_host_stream_full_size_layer_tensor():
    w = inputs.llama3_8b_layer_tensor(6)  # down_proj, 4096 x 14336
    got, st = decode_from_host(oracle.encode(w, K=128), w.size, 128, 16)
    assert st == 0 and np.array_equal(got, w)


def test_host_stream_errors():
    w = inputs.gaussian(4096 * 10, 0.02, seed=41)
    c = oracle.encode(w, K=128)
    with pytest.raises(dfx.DfxError) as e:
        decode_from_host(c, w.size, 128, 4, staging_bytes=c.size - 16)
    assert e.value.code == dfx.DFX_ERR_CAPACITY
    bad = c.copy()
    bad[0] ^= 1  # magic: the kernel flags it
    _, st = decode_from_host(bad, w.size, 128, 4)
    assert st & dfx.DFX_STATUS_HEADER
    big = c.copy()
    big[24:32] = np.frombuffer(np.uint64(c.size + 4096).tobytes(), dtype=np.uint8)  # larger than the buffer
    with pytest.raises(dfx.DfxError) as e:
        decode_from_host(big, w.size, 128, 4)
    assert e.value.code == dfx.DFX_ERR_CORRUPT
