"""GPU parity of the range decode (dfx_decode_range: the elements of a run of groups
into a buffer that holds just that slice) against the input, bit for bit; a tensor
restored slice by slice through one small buffer equals the whole."""
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


def decode_range(plan, comp, first, count, n, K):
    ge = 32 * K
    m = max(0, min(n, (first + count) * ge) - first * ge)
    out = torch.full((max(m, 1),), -1, dtype=torch.int16, device="cuda")
    dfx.dfx_decode_range(plan, comp, comp.numel(), first, count, out)
    st = dfx.dfx_device_status(plan)
    return out.cpu().numpy().view(np.uint16)[:m], st


@pytest.mark.parametrize("K", [128, 64])
@pytest.mark.parametrize("n", [40 * 4096 * 2 + 1001, 4096 * 64])
def test_ranges_match_the_input(K, n):
    w = inputs.projection_with_outliers()[:n].copy()
    comp = torch.from_numpy(oracle.encode(w, K=K)).cuda()
    ge = 32 * K
    ng = -(-n // ge)
    with dfx.dfx_plan(n, chunk_symbols=K) as plan:
        for first, count in [(0, ng), (0, 1), (3, 5), (ng - 2, 2), (ng - 1, 1), (ng // 2, ng - ng // 2), (7, 0)]:
            got, st = decode_range(plan, comp, first, count, n, K)
            assert st == 0, (first, count, hex(st))
            assert np.array_equal(got, w[first * ge: min(n, (first + count) * ge)]), (first, count)


def test_slice_by_slice_through_one_buffer():
    """A weight matrix restored 512 rows (groups) at a time through one reused buffer."""
    w = inputs.llama3_8b_layer_tensor(4)  # gate_proj, 14336 x 4096
    rows, cols = 14336, 4096
    comp = torch.from_numpy(oracle.encode(w, K=128)).cuda()
    with dfx.dfx_plan(w.size, chunk_symbols=128) as plan:
        assert dfx.group_elements(plan) == cols  # one group per row at K = 128
        buf = torch.empty(512 * cols, dtype=torch.int16, device="cuda")
        parts = []
        for r in range(0, rows, 512):
            dfx.dfx_decode_range(plan, comp, comp.numel(), r, 512, buf)
            parts.append(buf.cpu().numpy().view(np.uint16).copy())
        assert dfx.dfx_device_status(plan) == 0
    assert np.array_equal(np.concatenate(parts), w)


def test_range_past_the_end_is_refused():
    w = inputs.gaussian(4096 * 3, 0.02, seed=31)
    comp = torch.from_numpy(oracle.encode(w, K=128)).cuda()
    out = torch.empty(w.size, dtype=torch.int16, device="cuda")
    with dfx.dfx_plan(w.size) as plan:
        with pytest.raises(dfx.DfxError) as e:
            dfx.dfx_decode_range(plan, comp, comp.numel(), 2, 2, out)
        assert e.value.code == dfx.DFX_ERR_ARG


def test_corrupt_range_sets_status():
    w = inputs.gaussian(4096 * 40, 0.02, seed=32)
    c = oracle.encode(w, K=128)
    c[0] ^= 1  # magic
    comp = torch.from_numpy(c).cuda()
    with dfx.dfx_plan(w.size) as plan:
        out = torch.empty(4096 * 4, dtype=torch.int16, device="cuda")
        dfx.dfx_decode_range(plan, comp, comp.numel(), 10, 4, out)
        assert dfx.dfx_device_status(plan) & dfx.DFX_STATUS_HEADER
