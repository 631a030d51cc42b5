"""ctypes marshalling for the CPU oracle in ``oracle/dfx_oracle.c``.

TEST INFRASTRUCTURE ONLY.  The oracle is the plain single-threaded CPU
statement of the DFX1 codec (both exponent coders: canonical Huffman and
tANS) that the CUDA library is checked against.  Only
the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this module; the product path (``lossless_entropy_coded_exponent_b200``)
never does, and the two share no code.  Every function here only moves
arguments across the C boundary: the arithmetic lives in the C file.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dfx_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

OK, ERR_ARG, ERR_CAPACITY, ERR_CORRUPT = 0, 1, 2, 3


class OracleError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"oracle {what} failed with code {code}")
        self.code = code


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboracle.so`` (gcc, -O2, plain C11)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-shared", "-fPIC", "-o", tmp, _SRC]
        )
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        u8p = ctypes.POINTER(ctypes.c_uint8)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        u32p = ctypes.POINTER(ctypes.c_uint32)
        u64p = ctypes.POINTER(ctypes.c_uint64)
        L.dfxo_exponent.argtypes = [ctypes.c_uint16]
        L.dfxo_exponent.restype = ctypes.c_uint8
        L.dfxo_partner.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        L.dfxo_partner.restype = ctypes.c_uint64
        L.dfxo_sign_mantissa.argtypes = [ctypes.c_uint16, ctypes.c_uint16]
        L.dfxo_sign_mantissa.restype = ctypes.c_uint8
        L.dfxo_merge.argtypes = [ctypes.c_uint8, ctypes.c_uint8, ctypes.c_uint8]
        L.dfxo_merge.restype = ctypes.c_uint16
        L.dfxo_histogram.argtypes = [u16p, ctypes.c_uint64, u64p]
        L.dfxo_code_lengths.argtypes = [u64p, ctypes.c_uint32, u8p]
        L.dfxo_canonical_codes.argtypes = [u8p, u32p]
        L.dfxo_container_bytes.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint64]
        L.dfxo_container_bytes.restype = ctypes.c_uint64
        L.dfxo_max_container_bytes.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32]
        L.dfxo_max_container_bytes.restype = ctypes.c_uint64
        L.dfxo_encode.argtypes = [u16p, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32,
                                  u8p, ctypes.c_uint64, u64p]
        L.dfxo_decode.argtypes = [u8p, ctypes.c_uint64, u16p, ctypes.c_uint64, u64p]
        L.dfxo_tans_normalize.argtypes = [u64p, ctypes.c_uint32, u32p]
        L.dfxo_tans_tables.argtypes = [u32p, ctypes.c_uint32, u8p, u32p]
        L.dfxo_encode_tans.argtypes = [u16p, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32,
                                       u8p, ctypes.c_uint64, u64p]
        L.dfxo_tans_encode_chunk.argtypes = [u32p, ctypes.c_uint32, u8p, ctypes.c_uint32, u8p, u64p]
        L.dfxo_tans_encode_chunk.restype = ctypes.c_int
        L.dfxo_tans_encode_chunk_ways.argtypes = [u32p, ctypes.c_uint32, ctypes.c_uint32, u8p, ctypes.c_uint32, u8p,
                                                  u64p]
        L.dfxo_tans_encode_chunk_ways.restype = ctypes.c_int
        L.dfxo_encode_tans2.argtypes = [u16p, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32,
                                        u8p, ctypes.c_uint64, u64p]
        L.dfxo_encode_tans2.restype = ctypes.c_int
        L.dfxo_tans2_max_container_bytes.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32,
                                                     ctypes.c_uint32]
        L.dfxo_tans2_max_container_bytes.restype = ctypes.c_uint64
        L.dfxo_tans_container_bytes.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint64]
        L.dfxo_tans_container_bytes.restype = ctypes.c_uint64
        L.dfxo_tans_max_container_bytes.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32,
                                                    ctypes.c_uint32]
        L.dfxo_tans_max_container_bytes.restype = ctypes.c_uint64
        for f in ("dfxo_histogram", "dfxo_code_lengths", "dfxo_canonical_codes", "dfxo_encode", "dfxo_decode",
                  "dfxo_tans_normalize", "dfxo_tans_tables", "dfxo_encode_tans"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def exponent(w: int) -> int:
    return int(lib().dfxo_exponent(w))


def partner(x: int, n: int) -> int:
    return int(lib().dfxo_partner(x, n))


def sign_mantissa(w: int, partner_w: int) -> int:
    return int(lib().dfxo_sign_mantissa(w, partner_w))


def merge(e: int, m: int, m_partner: int) -> int:
    return int(lib().dfxo_merge(e, m, m_partner))


def histogram(w: np.ndarray) -> np.ndarray:
    w = np.ascontiguousarray(w, dtype=np.uint16)
    counts = np.zeros(256, dtype=np.uint64)
    rc = lib().dfxo_histogram(_ptr(w, ctypes.c_uint16), w.size, _ptr(counts, ctypes.c_uint64))
    if rc:
        raise OracleError(rc, "histogram")
    return counts


def code_lengths(counts, max_len: int = 24) -> np.ndarray:
    c = np.zeros(256, dtype=np.uint64)
    src = np.asarray(counts, dtype=np.uint64)
    c[: src.size] = src
    out = np.zeros(256, dtype=np.uint8)
    rc = lib().dfxo_code_lengths(_ptr(c, ctypes.c_uint64), max_len, _ptr(out, ctypes.c_uint8))
    if rc:
        raise OracleError(rc, "code_lengths")
    return out


def canonical_codes(lengths) -> np.ndarray:
    ln = np.zeros(256, dtype=np.uint8)
    src = np.asarray(lengths, dtype=np.uint8)
    ln[: src.size] = src
    code = np.zeros(256, dtype=np.uint32)
    rc = lib().dfxo_canonical_codes(_ptr(ln, ctypes.c_uint8), _ptr(code, ctypes.c_uint32))
    if rc:
        raise OracleError(rc, "canonical_codes")
    return code


def container_bytes(n: int, K: int, G: int, total_bits: int) -> int:
    return int(lib().dfxo_container_bytes(n, K, G, total_bits))


def max_container_bytes(n: int, K: int, G: int) -> int:
    return int(lib().dfxo_max_container_bytes(n, K, G))


def encode(w: np.ndarray, K: int = 64, G: int = 32, max_len: int = 24) -> np.ndarray:
    """Whole-tensor encode into a fresh uint8 array holding exactly the container."""
    w = np.ascontiguousarray(w, dtype=np.uint16).reshape(-1)
    cap = max_container_bytes(w.size, K, G)
    out = np.empty(cap, dtype=np.uint8)
    used = np.zeros(1, dtype=np.uint64)
    rc = lib().dfxo_encode(_ptr(w, ctypes.c_uint16), w.size, K, G, max_len,
                           _ptr(out, ctypes.c_uint8), cap, _ptr(used, ctypes.c_uint64))
    if rc:
        raise OracleError(rc, "encode")
    return out[: int(used[0])].copy()


def tans_normalize(counts, table_log: int = 12) -> np.ndarray:
    """Rule T1: the frequencies (summing to 2**table_log) of a count vector."""
    c = np.zeros(256, dtype=np.uint64)
    src = np.asarray(counts, dtype=np.uint64)
    c[: src.size] = src
    f = np.zeros(256, dtype=np.uint32)
    rc = lib().dfxo_tans_normalize(_ptr(c, ctypes.c_uint64), table_log, _ptr(f, ctypes.c_uint32))
    if rc:
        raise OracleError(rc, "tans_normalize")
    return f


def tans_tables(freq, table_log: int = 12):
    """Rules T2 and T3: (symbol, state number k) of every table slot."""
    f = np.zeros(256, dtype=np.uint32)
    src = np.asarray(freq, dtype=np.uint32)
    f[: src.size] = src
    m = 1 << table_log
    sym = np.zeros(m, dtype=np.uint8)
    k = np.zeros(m, dtype=np.uint32)
    rc = lib().dfxo_tans_tables(_ptr(f, ctypes.c_uint32), table_log, _ptr(sym, ctypes.c_uint8),
                                _ptr(k, ctypes.c_uint32))
    if rc:
        raise OracleError(rc, "tans_tables")
    return sym, k


def tans_encode_chunk(freq, symbols, table_log: int = 12, states: int = 1) -> str:
    """Rule T4 (states = 1) or T6 (states = 2) for one chunk with a given frequency
    table: its bits as a '0'/'1' string."""
    f = np.zeros(256, dtype=np.uint32)
    src = np.asarray(freq, dtype=np.uint32)
    f[: src.size] = src
    syms = np.ascontiguousarray(symbols, dtype=np.uint8)
    out = np.zeros((table_log * (syms.size + states) + 7) // 8 + 8, dtype=np.uint8)
    bits = np.zeros(1, dtype=np.uint64)
    rc = lib().dfxo_tans_encode_chunk_ways(_ptr(f, ctypes.c_uint32), table_log, states, _ptr(syms, ctypes.c_uint8),
                                           syms.size, _ptr(out, ctypes.c_uint8), _ptr(bits, ctypes.c_uint64))
    if rc:
        raise OracleError(rc, "tans_encode_chunk")
    nbits = int(bits[0])
    # the stream layout: bit k is bit 31 - k % 32 of little-endian 32-bit word k / 32
    words = np.frombuffer(out[: (out.size // 4) * 4].tobytes(), dtype="<u4")
    return "".join(str((int(words[k // 32]) >> (31 - k % 32)) & 1) for k in range(nbits))


def tans_container_bytes(n: int, K: int, G: int, total_bits: int) -> int:
    return int(lib().dfxo_tans_container_bytes(n, K, G, total_bits))


def tans_max_container_bytes(n: int, K: int, G: int, table_log: int = 12) -> int:
    return int(lib().dfxo_tans_max_container_bytes(n, K, G, table_log))


def tans2_max_container_bytes(n: int, K: int, G: int, table_log: int = 12) -> int:
    return int(lib().dfxo_tans2_max_container_bytes(n, K, G, table_log))


def encode_tans(w: np.ndarray, K: int = 128, G: int = 32, table_log: int = 12, states: int = 1) -> np.ndarray:
    """Whole-tensor encode with the tANS exponent coder: coder 1 (one state per
    chunk, rules T1-T5) or, with states = 2, coder 2 (rule T6 added)."""
    if states not in (1, 2):
        raise ValueError("states must be 1 or 2")
    w = np.ascontiguousarray(w, dtype=np.uint16).reshape(-1)
    cap = (tans_max_container_bytes if states == 1 else tans2_max_container_bytes)(w.size, K, G, table_log)
    out = np.empty(cap, dtype=np.uint8)
    used = np.zeros(1, dtype=np.uint64)
    fn = lib().dfxo_encode_tans if states == 1 else lib().dfxo_encode_tans2
    rc = fn(_ptr(w, ctypes.c_uint16), w.size, K, G, table_log, _ptr(out, ctypes.c_uint8), cap,
            _ptr(used, ctypes.c_uint64))
    if rc:
        raise OracleError(rc, "encode_tans")
    return out[: int(used[0])].copy()


def decode(c: np.ndarray, n_cap: int | None = None) -> np.ndarray:
    """Decode a container; raises OracleError(ERR_CORRUPT) on any malformed byte."""
    c = np.ascontiguousarray(c, dtype=np.uint8).reshape(-1)
    if n_cap is None:
        n_cap = int(c[8:16].view(np.uint64)[0]) if c.size >= 16 else 0
        n_cap = min(n_cap, 1 << 32)
    out = np.empty(max(n_cap, 1), dtype=np.uint16)
    n_out = np.zeros(1, dtype=np.uint64)
    rc = lib().dfxo_decode(_ptr(c, ctypes.c_uint8), c.size, _ptr(out, ctypes.c_uint16), n_cap,
                           _ptr(n_out, ctypes.c_uint64))
    if rc:
        raise OracleError(rc, "decode")
    return out[: int(n_out[0])]
