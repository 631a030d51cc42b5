"""Host-side checks of libdfx that need no GPU: the shared library loads, exports
every symbol include/dfx.h declares, its layout arithmetic agrees with the
oracle's, and argument errors come back before any CUDA call."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import lossless_entropy_coded_exponent_b200 as dfx
from lossless_entropy_coded_exponent_b200 import build as dfx_build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "dfx.h")


@pytest.fixture(scope="module")
def lib():
    dfx_build.build()
    return dfx.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(dfx_\w+)\s*\(", src, flags=re.M)


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert set(names) == set(dfx.EXPORTS)
    for name in names:
        assert hasattr(lib, name), name


def test_version_and_strerror(lib):
    assert dfx.dfx_version() >> 16 == 1
    for code in range(0, 8):
        assert isinstance(dfx.dfx_strerror(code), str) and dfx.dfx_strerror(code)
    assert dfx.dfx_strerror(dfx.DFX_OK) == "ok"


@pytest.mark.parametrize("n", [0, 1, 7, 4097, 1_000_003, 1 << 20, 234_881_024])
@pytest.mark.parametrize("K", [32, 64, 128])
def test_layout_agrees_with_oracle(lib, n, K):
    for total_bits in (0, 1, 31, 32, 33, 8 * n):
        lay = dfx.dfx_container_layout(n, total_bits, chunk_symbols=K)
        assert lay["total_bytes"] == oracle.container_bytes(n, K, 32, total_bits)
        assert lay["n_group"] == -(-n // (32 * K)) and lay["n_chunk"] == 32 * lay["n_group"]
        for key in ("off_clen", "off_m", "off_stream"):
            assert lay[key] % 16 == 0
    assert dfx.dfx_container_layout(n, 8 * n, chunk_symbols=K)["total_bytes"] == oracle.max_container_bytes(n, K, 32)


def test_layout_matches_an_oracle_container(lib):
    w = np.arange(5000, dtype=np.uint16)
    c = oracle.encode(w, K=64)
    total_bits = int(c[16:24].view(np.uint64)[0])
    lay = dfx.dfx_container_layout(w.size, total_bits, chunk_symbols=64)
    assert lay["total_bytes"] == c.size
    assert lay["off_m"] == int(c[48:56].view(np.uint64)[0])


def test_host_argument_errors_precede_cuda(lib):
    with pytest.raises(dfx.DfxError) as e:
        dfx.dfx_plan(1 << 32)
    assert e.value.code == dfx.DFX_ERR_TOO_LARGE
    with pytest.raises(dfx.DfxError) as e:
        dfx.dfx_plan(1000, max_len=7)
    assert e.value.code == dfx.DFX_ERR_ARG
    with pytest.raises(dfx.DfxError) as e:
        dfx.dfx_plan(1000, chunk_symbols=96)
    assert e.value.code == dfx.DFX_ERR_UNSUPPORTED
    with pytest.raises(dfx.DfxError) as e:
        dfx.dfx_plan(1000, group_chunks=16)
    assert e.value.code == dfx.DFX_ERR_UNSUPPORTED
    with pytest.raises(dfx.DfxError) as e:
        dfx.dfx_container_layout(10, 0, chunk_symbols=4000)
    assert e.value.code == dfx.DFX_ERR_ARG
    with pytest.raises(dfx.DfxError) as e:
        dfx.dfx_container_layout(10, 0, chunk_symbols=60)  # not a multiple of 8
    assert e.value.code == dfx.DFX_ERR_ARG
    with pytest.raises(dfx.DfxError) as e:
        dfx.dfx_plan(1000, decode_flags=0x2)  # an unknown decode flag
    assert e.value.code == dfx.DFX_ERR_ARG


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(dfx, "_lib_handle", None)
    monkeypatch.setattr(dfx, "LIB_PATH", str(tmp_path / "libdfx.so"))
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        dfx.dfx_version()


def test_batch_argument_errors_precede_cuda(lib):
    vp = ctypes.c_void_p
    assert lib.dfx_decode_batch(None, None, None, None, 0, None) == dfx.DFX_OK  # nothing to do
    assert lib.dfx_decode_batch(None, None, None, None, 1, None) == dfx.DFX_ERR_ARG
    arr = (vp * 33)()
    sizes = (ctypes.c_size_t * 33)()
    assert lib.dfx_decode_batch(arr, arr, sizes, arr, 33, None) == dfx.DFX_ERR_ARG  # at most 32 tensors
    assert lib.dfx_decode_batch(arr, arr, sizes, arr, 2, None) == dfx.DFX_ERR_ARG  # null plans
    with pytest.raises(ValueError):
        dfx.dfx_decode_batch([None], [], [], [])


def test_range_argument_errors_precede_cuda(lib):
    assert lib.dfx_decode_range(None, None, 0, 0, 1, None, None) == dfx.DFX_ERR_ARG


def test_host_decode_argument_errors_precede_cuda(lib):
    assert lib.dfx_decode_host(None, None, 0, None, 0, None, 0, None, None) == dfx.DFX_ERR_ARG


def test_debug_inject_flags(lib):
    assert lib.dfx_debug_inject(0x2) == dfx.DFX_ERR_ARG
    assert lib.dfx_debug_inject(0) == dfx.DFX_OK


@pytest.mark.parametrize("n", [0, 5, 4097, 1_000_003, 234_881_024])
@pytest.mark.parametrize("K,R", [(32, 12), (128, 12), (64, 8), (128, 4)])
def test_tans_layout_agrees_with_oracle(lib, n, K, R):
    nc = 32 * -(-n // (32 * K))
    for total_bits in (0, 1, 33, R * (n + nc)):
        lay = dfx.dfx_container_layout(n, total_bits, chunk_symbols=K, coder=dfx.DFX_CODER_TANS, table_log=R)
        assert lay["total_bytes"] == oracle.tans_container_bytes(n, K, 32, total_bits)
        assert lay["off_len"] == 64 and lay["off_gbase"] == 576
    lay = dfx.dfx_container_layout(n, R * (n + nc), chunk_symbols=K, coder=dfx.DFX_CODER_TANS, table_log=R)
    assert lay["total_bytes"] == oracle.tans_max_container_bytes(n, K, 32, R)


def test_tans_layout_matches_an_oracle_container(lib):
    w = np.arange(5000, dtype=np.uint16) % 1024
    c = oracle.encode_tans(w, K=64)
    total_bits = int(c[16:24].view(np.uint64)[0])
    lay = dfx.dfx_container_layout(w.size, total_bits, chunk_symbols=64, coder=dfx.DFX_CODER_TANS)
    assert lay["total_bytes"] == c.size
    assert lay["off_m"] == int(c[48:56].view(np.uint64)[0])


def test_tans_argument_errors_precede_cuda(lib):
    for kw in ({"table_log": 3}, {"table_log": 13}, {"chunk_symbols": 5464}):
        with pytest.raises(dfx.DfxError) as e:
            dfx.dfx_plan(1000, coder=dfx.DFX_CODER_TANS, **kw)
        assert e.value.code == dfx.DFX_ERR_ARG, kw
    with pytest.raises(dfx.DfxError) as e:
        dfx.dfx_plan(1000, coder=3)
    assert e.value.code == dfx.DFX_ERR_ARG
    # a chunk's length (fields and states) must fit u16: one state more with coder 2
    dfx.dfx_container_layout(10, 0, chunk_symbols=6552, coder=dfx.DFX_CODER_TANS, table_log=10)  # 6553 x 10
    with pytest.raises(dfx.DfxError) as e:
        dfx.dfx_container_layout(10, 0, chunk_symbols=6552, coder=dfx.DFX_CODER_TANS2, table_log=10)  # 6554 x 10
    assert e.value.code == dfx.DFX_ERR_ARG
    # the tANS coder ignores max_len, the Huffman coder table_log
    with pytest.raises(dfx.DfxError) as e:
        dfx.dfx_container_layout(10, 0, chunk_symbols=5464, coder=dfx.DFX_CODER_TANS)  # 5465 x 12 > 65535
    assert e.value.code == dfx.DFX_ERR_ARG
    dfx.dfx_container_layout(10, 0, chunk_symbols=4000, max_len=99, coder=dfx.DFX_CODER_TANS)
    dfx.dfx_container_layout(10, 0, table_log=99)
    for coder in (dfx.DFX_CODER_TANS, dfx.DFX_CODER_TANS2):
        with pytest.raises(dfx.DfxError) as e:
            dfx.dfx_encode_static(None, 10, None, 0, coder=coder)
        assert e.value.code == dfx.DFX_ERR_UNSUPPORTED


def header_struct_fields(name):
    """(type, field) pairs of `typedef struct { ... } name;` in include/dfx.h, in order."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    body = re.search(r"typedef struct \{([^{}]*)\}\s*" + name + r"\s*;", src).group(1)
    out = []
    for decl in body.split(";"):
        decl = decl.strip()
        if not decl:
            continue
        ctype, names = decl.split(None, 1)
        out += [(ctype, n.strip()) for n in names.split(",")]
    return out


@pytest.mark.parametrize("name", ["dfx_params", "dfx_layout"])
def test_ctypes_structs_mirror_the_header(name):
    """The binding's ctypes structures have the header's fields, in order, with the same
    widths: a field added on one side only would shift every later one."""
    widths = {"uint32_t": ctypes.c_uint32, "uint64_t": ctypes.c_uint64}
    declared = header_struct_fields(name)
    mirror = getattr(dfx, name)._fields_
    assert [n for _, n in declared] == [n for n, _ in mirror]
    assert all(widths[t] is c for (t, _), (_, c) in zip(declared, mirror))


def test_binding_constants_match_the_header():
    """Every DFX_* constant of the binding has the value include/dfx.h defines."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    defined = {name: int(val.rstrip("uU"), 0)
               for name, val in re.findall(r"^#define\s+(DFX_\w+)\s+(0x[0-9a-fA-F]+u?|\d+u?)\s*$", src, flags=re.M)}
    mirrored = {k: v for k, v in vars(dfx).items() if k.startswith("DFX_") and isinstance(v, int)}
    assert mirrored, "the binding defines no DFX_ constants"
    for name, value in mirrored.items():
        assert name in defined, f"{name} is not defined in include/dfx.h"
        assert defined[name] == value, (name, value, defined[name])
