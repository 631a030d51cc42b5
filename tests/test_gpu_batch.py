"""GPU parity of the multi-tensor decode (dfx_decode_batch, one launch for several
containers) against the CPU oracle: every tensor of the batch decodes bit for bit to
its input, corruption stays confined to its own tensor's status word, and the
batch rules (shared chunk size, at most 32 tensors) are enforced."""
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


def to_dev(w: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(w).view(np.int16)).cuda()


def decode_batch(containers, sizes, K=64):
    """Batch-decode host containers; returns the decoded words and status words."""
    plans = [dfx.dfx_plan(n, chunk_symbols=K) for n in sizes]
    try:
        comps = [torch.from_numpy(c).cuda() for c in containers]
        outs = [torch.full((max(n, 1),), -1, dtype=torch.int16, device="cuda") for n in sizes]
        dfx.dfx_decode_batch(plans, comps, [c.numel() for c in comps], outs)
        status = [dfx.dfx_device_status(p) for p in plans]
        got = [o.cpu().numpy().view(np.uint16)[:n] for o, n in zip(outs, sizes)]
        return got, status
    finally:
        for p in plans:
            p.free()


MIXED = [("empty", 0), ("one", 1), ("seven", 7), ("ragged", 4097), ("groups+1", 3 * 2048 + 1),
         ("million", 1_000_003), ("full_groups", 2048 * 40)]


@pytest.mark.parametrize("K", [64, 32, 128])
def test_mixed_sizes_from_oracle_containers(K):
    ws = [inputs.gaussian(n, 0.02, seed=70 + i) for i, (_, n) in enumerate(MIXED)]
    containers = [oracle.encode(w, K=K) for w in ws]
    got, status = decode_batch(containers, [w.size for w in ws], K)
    for (name, _), w, g, st in zip(MIXED, ws, got, status):
        assert st == 0, (name, hex(st))
        assert np.array_equal(g, w), name


def test_special_values_and_long_codes_in_one_batch():
    ec = inputs.edge_cases()
    ws = [ec[k] for k in sorted(ec)] + [inputs.fibonacci_clamp_tensor(3), inputs.projection_with_outliers()]
    containers = [oracle.encode(w, K=64) for w in ws]
    got, status = decode_batch(containers, [w.size for w in ws])
    for w, g, st in zip(ws, got, status):
        assert st == 0
        assert np.array_equal(g, w)


def test_llama3_8b_layer_in_one_launch():
    """The seven projections of a Llama-3-8B-shaped layer (218 M weights) in one launch.
    Each container is written by the GPU encoder at the default chunk size K = 128 and
    is first checked byte for byte against the oracle's container of the same tensor."""
    ws = [inputs.llama3_8b_layer_tensor(i) for i in range(len(inputs.LLAMA3_8B_LAYER))]
    plans = [dfx.dfx_plan(w.size) for w in ws]
    try:
        comps, sizes = [], []
        for w, p in zip(ws, plans):
            out = torch.empty(p.max_compressed_bytes, dtype=torch.uint8, device="cuda")
            ws_ = torch.empty(p.workspace_bytes, dtype=torch.uint8, device="cuda")
            size = dfx.dfx_encode(p, to_dev(w), out, out.numel(), ws_, ws_.numel(), want_size=True)
            assert np.array_equal(out[:size].cpu().numpy(), oracle.encode(w, K=128))
            comps.append(out[:size].clone())
            sizes.append(size)
        outs = [torch.empty(w.size, dtype=torch.int16, device="cuda") for w in ws]
        dfx.dfx_decode_batch(plans, comps, sizes, outs)
        for w, o, p in zip(ws, outs, plans):
            assert dfx.dfx_device_status(p) == 0
            assert torch.equal(o, to_dev(w))
    finally:
        for p in plans:
            p.free()


def test_corruption_stays_in_its_tensor():
    ws = [inputs.gaussian(n, 0.02, seed=90 + i) for i, n in enumerate([2048 * 50, 2048 * 20 + 5, 2048 * 7])]
    containers = [oracle.encode(w, K=64) for w in ws]
    bad = containers[1].copy()
    ng = int(bad[44:48].view(np.uint32)[0])
    bad[320 + 8 * (ng // 2)] ^= 0x3  # a group start bit
    got, status = decode_batch([containers[0], bad, containers[2]], [w.size for w in ws])
    assert status[0] == 0 and status[2] == 0
    assert status[1] & dfx.DFX_STATUS_INDEX
    assert np.array_equal(got[0], ws[0]) and np.array_equal(got[2], ws[2])


def test_batch_of_one_equals_dfx_decode():
    w = inputs.small_gaussian()
    c = oracle.encode(w, K=64)
    got, status = decode_batch([c], [w.size])
    assert status == [0] and np.array_equal(got[0], w)


def test_mixed_chunk_sizes_are_refused():
    a, b = dfx.dfx_plan(4096, chunk_symbols=64), dfx.dfx_plan(4096, chunk_symbols=128)
    try:
        comp = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
        out = torch.empty(4096, dtype=torch.int16, device="cuda")
        out2 = torch.empty(4096, dtype=torch.int16, device="cuda")
        with pytest.raises(dfx.DfxError) as e:
            dfx.dfx_decode_batch([a, b], [comp, comp], [comp.numel()] * 2, [out, out2])
        assert e.value.code == dfx.DFX_ERR_UNSUPPORTED
    finally:
        a.free()
        b.free()


def test_back_to_back_launches_of_one_plan():
    """Decodes of one plan, ranges and whole tensors, one after another on a stream, into
    reused buffers."""
    w = inputs.gaussian(4096 * 333 + 17, 0.02, seed=95)
    c = torch.from_numpy(oracle.encode(w, K=128)).cuda()
    x = to_dev(w)
    with dfx.dfx_plan(w.size) as plan:
        out = torch.full_like(x, -1)
        for rep in range(3):
            out.fill_(-1)
            dfx.dfx_decode(plan, c, c.numel(), out)
            assert torch.equal(out, x), rep
            part = torch.full((4096 * 100,), -1, dtype=torch.int16, device="cuda")
            dfx.dfx_decode_range(plan, c, c.numel(), 200, 100, part)
            assert torch.equal(part, x[4096 * 200: 4096 * 300]), rep
        assert dfx.dfx_device_status(plan) == 0


@pytest.mark.parametrize("K", [128, 64])
def test_early_read_back_to_back_decodes(K):
    """DFX_DECODE_EARLY_READ: containers written once, then decoded one after another into
    one reused buffer and into separate buffers, launches back to back (each CTA reads its
    container while the previous decode finishes and writes only after it)."""
    ws = [inputs.llama3_8b_layer_tensor(i) for i in (0, 2, 3, 1)]  # 4096^2, 1024x4096, 1024x4096, 4096^2
    comps = [torch.from_numpy(oracle.encode(w, K=K)).cuda() for w in ws]
    xs = [to_dev(w) for w in ws]
    plans = [dfx.dfx_plan(w.size, chunk_symbols=K, decode_flags=dfx.DFX_DECODE_EARLY_READ) for w in ws]
    try:
        big = torch.full((max(w.size for w in ws),), -1, dtype=torch.int16, device="cuda")
        outs = [torch.full_like(x, -1) for x in xs]
        for _ in range(3):
            for p, c, o in zip(plans, comps, outs):
                dfx.dfx_decode(p, c, c.numel(), o)
            for p, c, x in zip(plans, comps, xs):
                dfx.dfx_decode(p, c, c.numel(), big)
        torch.cuda.synchronize()
        assert all(dfx.dfx_device_status(p) == 0 for p in plans)
        assert all(torch.equal(o, x) for o, x in zip(outs, xs))
        assert torch.equal(big[: xs[-1].numel()], xs[-1])
    finally:
        for p in plans:
            p.free()
