"""CPU oracle for paged decode attention (test infrastructure).

Only the test suite, the smoke check and the benchmark's CPU-baseline leg may
import this package.  It shares no code with the CUDA path: the arithmetic is
the plain fp64 C in attention.c (built with gcc into liboracle.so) and the
block manager model in pagepool.py.

Functions take and return numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from .pagepool import (  # noqa: F401
    PAGE_SIZE,
    PagePool,
    PagedRequest,
    PoolExhausted,
    kv_bytes_per_token,
    naive_utilisation,
    paged_utilisation,
    pages_needed,
    slot_of,
)

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attention.c")
_LIB = os.path.join(_HERE, "liboracle.so")

DTYPE_CODE = {np.dtype(np.float32): 0, np.dtype(np.float16): 1}
BF16 = "bf16"  # bf16 arrays travel as uint16 bit patterns with dtype tag "bf16"


def build(force: bool = False) -> str:
    """Compile attention.c into liboracle.so with gcc (OpenMP over (seq, head))."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i32, i64, vp, dbl = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_double
        lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_half_to_double.restype = dbl
        lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_double.restype = dbl
        lib.oracle_decode_attention.argtypes = [
            ctypes.c_int, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, i32, dbl, vp]
        lib.oracle_decode_attention.restype = None
        lib.oracle_reshape_and_cache.argtypes = [vp, vp, vp, i32, vp, vp, i32, i32, i32, i32]
        lib.oracle_reshape_and_cache.restype = None
        lib.oracle_copy_blocks.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32]
        lib.oracle_copy_blocks.restype = None
        lib.oracle_slot_of.argtypes = [vp, i64, i32]
        lib.oracle_slot_of.restype = i64
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _contig(a, dtype=None):
    return np.ascontiguousarray(a if dtype is None else np.asarray(a, dtype=dtype))


def half_to_double(bits: int) -> float:
    return _load().oracle_half_to_double(bits)


def bf16_to_double(bits: int) -> float:
    return _load().oracle_bf16_to_double(bits)


def decode_attention(q, k_pool, v_pool, block_tables, context_lens, scale, dtype=None,
                     num_threads: int | None = None):
    """fp64 decode attention through the block tables.

    q: [S, Hq, D]; k_pool, v_pool: [NB, Hkv, block_size, D] (float32, float16,
    or uint16 bf16 bit patterns with dtype="bf16"); block_tables: [S, max_blocks]
    int32; context_lens: [S] int32.  Returns float64 [S, Hq, D].
    """
    lib = _load()
    q = _contig(q)
    k_pool = _contig(k_pool)
    v_pool = _contig(v_pool)
    bt = _contig(block_tables, np.int32)
    cl = _contig(context_lens, np.int32)
    if dtype == BF16:
        code = 2
    else:
        code = DTYPE_CODE[q.dtype]
    assert k_pool.dtype == q.dtype and v_pool.dtype == q.dtype
    S, Hq, D = q.shape
    NB, Hkv, bs, D2 = k_pool.shape
    assert D2 == D and v_pool.shape == k_pool.shape and Hq % Hkv == 0
    assert bt.ndim == 2 and bt.shape[0] == S and cl.shape == (S,)
    out = np.zeros((S, Hq, D), dtype=np.float64)
    if num_threads is not None:
        os.environ["OMP_NUM_THREADS"] = str(num_threads)
    lib.oracle_decode_attention(code, _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(bt), bt.shape[1],
                                _ptr(cl), S, Hq, Hkv, D, bs, float(scale), _ptr(out))
    return out


def reshape_and_cache(k_new, v_new, slot_mapping, k_pool, v_pool):
    """Scatter new tokens' K/V rows into their slots, in place on k_pool/v_pool."""
    lib = _load()
    k_new = _contig(k_new)
    v_new = _contig(v_new)
    sm = _contig(slot_mapping, np.int32)
    assert k_pool.flags.c_contiguous and v_pool.flags.c_contiguous
    NB, H, bs, D = k_pool.shape
    T = sm.shape[0]
    assert k_new.shape == (T, H, D) and v_new.shape == (T, H, D)
    lib.oracle_reshape_and_cache(_ptr(k_new), _ptr(v_new), _ptr(sm), T, _ptr(k_pool), _ptr(v_pool),
                                 H, D, bs, k_pool.dtype.itemsize)


def copy_blocks(k_pool, v_pool, pairs):
    """Copy whole blocks src -> dst for each (src, dst) row of pairs, in place."""
    lib = _load()
    pr = _contig(pairs, np.int32).reshape(-1, 2)
    assert k_pool.flags.c_contiguous and v_pool.flags.c_contiguous
    NB, H, bs, D = k_pool.shape
    lib.oracle_copy_blocks(_ptr(k_pool), _ptr(v_pool), _ptr(pr), pr.shape[0], H, D, bs,
                           k_pool.dtype.itemsize)


def slot_of_c(block_table_row, pos: int, block_size: int = PAGE_SIZE) -> int:
    row = _contig(block_table_row, np.int32)
    return int(_load().oracle_slot_of(_ptr(row), pos, block_size))


def within_tolerance(gpu, ref, atol=2e-3, rtol=1e-2):
    """Elementwise |gpu - ref| <= atol + rtol * |ref| (the parity gate)."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return np.abs(gpu - ref) <= atol + rtol * np.abs(ref)
