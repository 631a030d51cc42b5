"""dfx_encode_static: the encoder entry point that allocates no device memory.

It serves callers that may not call cudaMalloc/cudaFree (their HBM belongs to
their own pool allocator, or they must avoid cudaFree's implicit device
synchronisation).  Its scratch is a fixed array inside the library that every
call reuses, so this checks it against dfx_encode, and against the CPU oracle's
container, on two calls in a row: the second call starts from the first call's
leftovers in that array.  The file is named to run last in a full test run.
"""
import numpy as np
import pytest
import torch

import oracle
import lossless_entropy_coded_exponent_b200 as dfx
from lossless_entropy_coded_exponent_b200 import build as dfx_build
from lossless_entropy_coded_exponent_b200 import inputs

pytestmark = pytest.mark.gpu


def encode_with_plan(x: torch.Tensor, n: int, K: int) -> np.ndarray:
    with dfx.dfx_plan(n, chunk_symbols=K) as plan:
        out = torch.empty(plan.max_compressed_bytes, dtype=torch.uint8, device="cuda")
        ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
        size = dfx.dfx_encode(plan, x, out, out.numel(), ws, ws.numel(), want_size=True)
        return out[:size].cpu().numpy()


def test_static_encoder_matches_dfx_encode_on_two_calls_in_a_row():
    dfx_build.build()
    assert torch.cuda.is_available(), "GPU test needs a CUDA device"
    cases = [
        (inputs.projection_with_outliers(), 64),   # 16.7 M weights: fills much of the scratch
        (inputs.gaussian(1_000_003, 0.02, seed=21), 64),  # smaller, ragged: runs on the leftovers
    ]
    for w, K in cases:
        x = torch.from_numpy(w.view(np.int16)).cuda()
        ref = encode_with_plan(x, w.size, K)
        cap = dfx.dfx_container_layout(w.size, 8 * w.size, chunk_symbols=K)["total_bytes"]
        out = torch.full((cap,), 0x5A, dtype=torch.uint8, device="cuda")
        size = dfx.dfx_encode_static(x, w.size, out, cap, want_size=True, chunk_symbols=K)
        got = out.cpu().numpy()
        assert size == ref.size
        assert np.array_equal(got[:size], ref)
        assert np.all(got[size:] == 0x5A)  # bytes past the container are left as they were
        assert np.array_equal(got[:size], oracle.encode(w, K=K))


def test_static_encoder_rejects_sizes_beyond_its_scratch():
    dfx_build.build()
    # 262144 groups of 32 chunks of 32 codes is the limit; one more element is over it
    n = 262144 * 32 * 32 + 1
    x = torch.zeros(16, dtype=torch.int16, device="cuda")
    out = torch.zeros(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(dfx.DfxError) as e:
        dfx.dfx_encode_static(x, n, out, 1 << 40, chunk_symbols=32)
    assert e.value.code == dfx.DFX_ERR_CAPACITY
