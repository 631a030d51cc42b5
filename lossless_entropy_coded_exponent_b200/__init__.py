"""Lossless BF16 weight codec for B200: Python binding of libdfx (include/dfx.h).

The calls keep the C names and only marshal arguments: pointers are taken from
torch tensors (or passed as integers), streams from ``torch.cuda.Stream``
objects.  Every step of encoding and decoding runs in the CUDA kernels of
``libdfx.so``; there is no CPU fallback, and every call raises
``DfxError`` if the library has not been built (``python -m
lossless_entropy_coded_exponent_b200.build``) or a call fails.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdfx.so")

DFX_OK = 0
DFX_ERR_ARG = 1
DFX_ERR_CAPACITY = 2
DFX_ERR_CORRUPT = 3
DFX_ERR_TOO_LARGE = 4
DFX_ERR_CUDA = 5
DFX_ERR_UNSUPPORTED = 6

DFX_STATUS_HEADER = 0x1
DFX_STATUS_TABLE = 0x2
DFX_STATUS_INDEX = 0x4
DFX_STATUS_STREAM = 0x8
DFX_STATUS_TIMEOUT = 0x10
DFX_INJECT_SKIP_SLICE_COPY = 0x1
DFX_CODER_HUFFMAN = 0
DFX_CODER_TANS = 1
DFX_CODER_TANS2 = 2  # tANS with two interleaved states per chunk
DFX_DECODE_EARLY_READ = 0x1

# The exported C symbols, in include/dfx.h order.
EXPORTS = (
    "dfx_version",
    "dfx_strerror",
    "dfx_container_layout",
    "dfx_plan",
    "dfx_encode",
    "dfx_decode",
    "dfx_decode_range",
    "dfx_decode_host",
    "dfx_decode_gemm",
    "dfx_decode_batch",
    "dfx_device_status",
    "dfx_free",
    "dfx_encode_static",
    "dfx_debug_inject",
)


class DfxError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {dfx_strerror(code) if _lib_handle else code} (code {code})")
        self.code = code


class dfx_params(ctypes.Structure):
    _fields_ = [("chunk_symbols", ctypes.c_uint32), ("group_chunks", ctypes.c_uint32), ("max_len", ctypes.c_uint32),
                ("coder", ctypes.c_uint32), ("table_log", ctypes.c_uint32), ("decode_flags", ctypes.c_uint32)]


class dfx_layout(ctypes.Structure):
    _fields_ = [(name, ctypes.c_uint64) for name in
                ("n", "n_chunk", "n_group", "off_len", "off_gbase", "off_clen", "off_m", "off_stream",
                 "stream_bytes", "total_bytes")]


_lib_handle = None


def lib() -> ctypes.CDLL:
    """The loaded libdfx.so; raises if it has not been built."""
    global _lib_handle
    if _lib_handle is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libdfx.so is missing at {LIB_PATH}: build it with "
                "`python -m lossless_entropy_coded_exponent_b200.build` (there is no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        vp = ctypes.c_void_p
        L.dfx_version.argtypes = []
        L.dfx_version.restype = ctypes.c_uint32
        L.dfx_strerror.argtypes = [ctypes.c_int]
        L.dfx_strerror.restype = ctypes.c_char_p
        L.dfx_container_layout.argtypes = [ctypes.c_uint64, ctypes.POINTER(dfx_params), ctypes.c_uint64,
                                           ctypes.POINTER(dfx_layout)]
        L.dfx_plan.argtypes = [ctypes.POINTER(vp), ctypes.c_uint64, ctypes.POINTER(dfx_params),
                               ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_size_t)]
        L.dfx_encode.argtypes = [vp, vp, vp, ctypes.c_size_t, vp, ctypes.c_size_t, ctypes.POINTER(ctypes.c_size_t), vp]
        L.dfx_decode.argtypes = [vp, vp, ctypes.c_size_t, vp, vp]
        L.dfx_decode_range.argtypes = [vp, vp, ctypes.c_size_t, ctypes.c_uint64, ctypes.c_uint64, vp, vp]
        L.dfx_decode_host.argtypes = [vp, vp, ctypes.c_size_t, vp, ctypes.c_size_t, vp, ctypes.c_uint32, vp, vp]
        L.dfx_decode_gemm.argtypes = [vp, vp, ctypes.c_size_t, ctypes.c_uint64, ctypes.c_uint64, vp, ctypes.c_uint32, vp,
                                      vp, vp]
        L.dfx_decode_batch.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(ctypes.c_size_t),
                                       ctypes.POINTER(vp), ctypes.c_uint32, vp]
        L.dfx_device_status.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint32)]
        L.dfx_free.argtypes = [vp]
        L.dfx_debug_inject.argtypes = [ctypes.c_uint32]
        L.dfx_encode_static.argtypes = [vp, ctypes.c_uint64, ctypes.POINTER(dfx_params), vp, ctypes.c_size_t,
                                        ctypes.POINTER(ctypes.c_size_t), vp]
        for f in ("dfx_container_layout", "dfx_plan", "dfx_encode", "dfx_decode", "dfx_decode_range", "dfx_decode_host",
                  "dfx_decode_gemm", "dfx_decode_batch",
                  "dfx_device_status", "dfx_free", "dfx_encode_static", "dfx_debug_inject"):
            getattr(L, f).restype = ctypes.c_int
        _lib_handle = L
    return _lib_handle


def _check(rc: int, what: str) -> None:
    if rc != DFX_OK:
        raise DfxError(rc, what)


def _ptr(x) -> int | None:
    """Device pointer of a tensor, or an integer address as is."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s) -> int | None:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _params(chunk_symbols=0, group_chunks=0, max_len=0, coder=DFX_CODER_HUFFMAN, table_log=0, decode_flags=0):
    return dfx_params(chunk_symbols, group_chunks, max_len, coder, table_log, decode_flags)


def dfx_version() -> int:
    return int(lib().dfx_version())


def dfx_strerror(code: int) -> str:
    return lib().dfx_strerror(code).decode()


def dfx_container_layout(n: int, total_bits: int, chunk_symbols=0, group_chunks=0, max_len=0,
                         coder=DFX_CODER_HUFFMAN, table_log=0) -> dict:
    out = dfx_layout()
    p = _params(chunk_symbols, group_chunks, max_len, coder, table_log)
    _check(lib().dfx_container_layout(n, ctypes.byref(p), total_bits, ctypes.byref(out)), "dfx_container_layout")
    return {name: int(getattr(out, name)) for name, _ in dfx_layout._fields_}


class Plan:
    """An open dfx plan (the C ``dfx_plan_t``) plus the sizes dfx_plan reported."""

    def __init__(self, handle: int, n: int, max_compressed_bytes: int, workspace_bytes: int, params: tuple):
        self.handle = handle
        self.n = n
        self.max_compressed_bytes = max_compressed_bytes
        self.workspace_bytes = workspace_bytes
        self.params = params

    def free(self) -> None:
        if self.handle:
            _check(lib().dfx_free(self.handle), "dfx_free")
            self.handle = None

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.free()

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def dfx_plan(n: int, chunk_symbols: int = 0, group_chunks: int = 0, max_len: int = 0,
             coder: int = DFX_CODER_HUFFMAN, table_log: int = 0, decode_flags: int = 0) -> Plan:
    h = ctypes.c_void_p()
    mx = ctypes.c_size_t()
    ws = ctypes.c_size_t()
    p = _params(chunk_symbols, group_chunks, max_len, coder, table_log, decode_flags)
    _check(lib().dfx_plan(ctypes.byref(h), n, ctypes.byref(p), ctypes.byref(mx), ctypes.byref(ws)), "dfx_plan")
    return Plan(h.value, n, mx.value, ws.value, (chunk_symbols, group_chunks, max_len, coder, table_log))


def dfx_encode(plan: Plan, d_bf16, d_out, out_capacity: int, d_workspace, workspace_bytes: int,
               want_size: bool = False, stream=None) -> int | None:
    size = ctypes.c_size_t()
    rc = lib().dfx_encode(plan.handle, _ptr(d_bf16), _ptr(d_out), out_capacity, _ptr(d_workspace), workspace_bytes,
                          ctypes.byref(size) if want_size else None, _stream(stream))
    _check(rc, "dfx_encode")
    return size.value if want_size else None


def dfx_decode(plan: Plan, d_comp, comp_bytes: int, d_bf16, stream=None) -> None:
    _check(lib().dfx_decode(plan.handle, _ptr(d_comp), comp_bytes, _ptr(d_bf16), _stream(stream)), "dfx_decode")


DEFAULT_CHUNK_SYMBOLS = 128  # dfx_params.chunk_symbols = 0 means this (include/dfx.h)


def group_elements(plan: Plan) -> int:
    """Elements per group of the plan's containers (32 chunks of chunk_symbols)."""
    return 32 * (plan.params[0] or DEFAULT_CHUNK_SYMBOLS)


def dfx_decode_range(plan: Plan, d_comp, comp_bytes: int, first_group: int, group_count: int, d_bf16,
                     stream=None) -> None:
    """Decode groups [first_group, first_group + group_count) into d_bf16 (which holds
    element first_group * 32 * chunk_symbols at index 0)."""
    _check(lib().dfx_decode_range(plan.handle, _ptr(d_comp), comp_bytes, first_group, group_count, _ptr(d_bf16),
                                  _stream(stream)), "dfx_decode_range")


def dfx_decode_host(plan: Plan, h_comp, comp_bytes: int, d_staging, staging_bytes: int, d_bf16, slices: int = 0,
                    copy_stream=None, decode_stream=None) -> None:
    """Stream a container in (pinned) host memory to d_staging slice by slice while
    decoding the slices into d_bf16 (copies on copy_stream, decoding on decode_stream)."""
    _check(lib().dfx_decode_host(plan.handle, _ptr(h_comp), comp_bytes, _ptr(d_staging), staging_bytes,
                                 _ptr(d_bf16), slices, _stream(copy_stream), _stream(decode_stream)),
           "dfx_decode_host")


def dfx_decode_gemm(plan: Plan, d_comp, comp_bytes: int, rows: int, cols: int, d_x, tokens: int, d_y,
                    d_w_out=None, stream=None) -> None:
    """Y = X W^T with W (rows x cols BF16) decoded from its container inside the GEMM
    kernel; X tokens x cols BF16, Y tokens x rows FP32; d_w_out (optional) also
    receives the decoded W."""
    _check(lib().dfx_decode_gemm(plan.handle, _ptr(d_comp), comp_bytes, rows, cols, _ptr(d_x), tokens, _ptr(d_y),
                                 _ptr(d_w_out), _stream(stream)), "dfx_decode_gemm")


def dfx_decode_batch(plans, d_comps, comp_bytes, d_bf16s, stream=None) -> None:
    """Decode several containers with one kernel launch (sequences of equal length)."""
    n = len(plans)
    if not (len(d_comps) == len(comp_bytes) == len(d_bf16s) == n):
        raise ValueError("dfx_decode_batch: plans, containers, sizes and outputs differ in length")
    vp = ctypes.c_void_p
    hp = (vp * max(n, 1))(*[p.handle if p is not None else None for p in plans])
    cp = (vp * max(n, 1))(*[_ptr(c) for c in d_comps])
    sz = (ctypes.c_size_t * max(n, 1))(*[int(b) for b in comp_bytes])
    op = (vp * max(n, 1))(*[_ptr(o) for o in d_bf16s])
    _check(lib().dfx_decode_batch(hp, cp, sz, op, n, _stream(stream)), "dfx_decode_batch")


def dfx_debug_inject(flags: int) -> None:
    """Test hook: DFX_INJECT_SKIP_SLICE_COPY makes later decodes leave one stream-slice
    copy out so that a bounded wait runs out (status DFX_STATUS_TIMEOUT); 0 restores."""
    _check(lib().dfx_debug_inject(flags), "dfx_debug_inject")


def dfx_device_status(plan: Plan, stream=None) -> int:
    v = ctypes.c_uint32()
    _check(lib().dfx_device_status(plan.handle, _stream(stream), ctypes.byref(v)), "dfx_device_status")
    return int(v.value)


def dfx_free(plan: Plan) -> None:
    plan.free()


def dfx_encode_static(d_bf16, n: int, d_out, out_capacity: int, want_size: bool = False, stream=None,
                      chunk_symbols: int = 0, group_chunks: int = 0, max_len: int = 0,
                      coder: int = DFX_CODER_HUFFMAN) -> int | None:
    """Encode without any device allocation by the library (no plan, no workspace);
    for callers whose device memory is owned by another allocator (coder 0 only)."""
    size = ctypes.c_size_t()
    p = _params(chunk_symbols, group_chunks, max_len, coder)
    rc = lib().dfx_encode_static(_ptr(d_bf16), n, ctypes.byref(p), _ptr(d_out), out_capacity,
                                 ctypes.byref(size) if want_size else None, _stream(stream))
    _check(rc, "dfx_encode_static")
    return size.value if want_size else None


# ---------------------------------------------------------------- tensor helpers
# Allocation goes through torch; the work is the C calls above.

def encode(x, plan: Plan | None = None, stream=None, **params):
    """Compress a CUDA tensor of BF16 (or int16/uint16 bit patterns); returns the
    container as a uint8 CUDA tensor trimmed to its size (synchronises `stream`)."""
    import torch

    flat = x.reshape(-1)
    own = plan is None
    plan = plan or dfx_plan(flat.numel(), **params)
    try:
        out = torch.empty(plan.max_compressed_bytes, dtype=torch.uint8, device=flat.device)
        ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=flat.device)
        size = dfx_encode(plan, flat, out, out.numel(), ws, ws.numel(), want_size=True, stream=stream)
        return out[:size].clone()
    finally:
        if own:
            plan.free()


def decode(comp, n: int, plan: Plan | None = None, out=None, stream=None, check: bool = True, **params):
    """Decode a container (uint8 CUDA tensor) into a BF16 CUDA tensor of n elements.
    With check=True the stream is synchronised and a corrupt container raises."""
    import torch

    own = plan is None
    plan = plan or dfx_plan(n, **params)
    try:
        if out is None:
            out = torch.empty(n, dtype=torch.bfloat16, device=comp.device)
        dfx_decode(plan, comp, comp.numel(), out, stream=stream)
        if check:
            st = dfx_device_status(plan, stream=stream)
            if st:
                raise DfxError(DFX_ERR_CORRUPT, f"dfx_decode (device status 0x{st:x})")
        return out
    finally:
        if own:
            plan.free()
