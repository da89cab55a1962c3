"""CPU oracle for the FP8 paged KV-cache decode path (ctypes wrapper of oracle.c).

TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check in __graft_entry__ and
the CPU-baseline leg of bench.py may import this package.  The product path
(fp8_kv_paged_kvq_b200) never imports it and shares no code with it.

All arrays are numpy arrays on the host.  BF16 tensors travel as uint16 bit
patterns.  Every function is a thin marshalling layer over oracle.c; the
arithmetic, and the passages of the source pages it follows, are documented
there.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

FP8, BF16 = 0, 1
SCALE_TENSOR, SCALE_HEAD, SCALE_TOKEN = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, strict IEEE: no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", _SRC, "-o", _LIB_PATH, "-lm"]
        subprocess.check_call(cmd)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        _lib = ctypes.CDLL(_LIB_PATH)
        _lib.oracle_e4m3_decode.restype = ctypes.c_double
        _lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        _lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        _lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        _lib.oracle_scale_from_amax.restype = ctypes.c_float
        _lib.oracle_scale_from_amax.argtypes = [ctypes.c_float]
        _lib.oracle_bf16_to_f32.restype = ctypes.c_float
        _lib.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
    return _lib


def set_threads(n: int = 0) -> int:
    """Threads the oracle's parallel loops use (n <= 0: leave as is); returns the setting."""
    return int(lib().oracle_set_threads(ctypes.c_int(n)))


def _p(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(codes.shape, dtype=np.float64)
    lib().oracle_e4m3_decode_array(_p(codes), _p(out), ctypes.c_int64(codes.size))
    return out


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    lib().oracle_e4m3_encode_array(_p(x), _p(out), ctypes.c_int64(x.size))
    return out


def e4m3_encode_bits_range(start: int, count: int) -> np.ndarray:
    out = np.empty(count, dtype=np.uint8)
    lib().oracle_e4m3_encode_bits_range(ctypes.c_uint32(start), ctypes.c_uint32(count), _p(out))
    return out


def e4m3_quantize_bits_range(start: int, count: int, scale: float) -> np.ndarray:
    """Codes of (float bits start + i) / scale with IEEE binary32 division."""
    out = np.empty(count, dtype=np.uint8)
    lib().oracle_e4m3_quantize_bits_range(ctypes.c_uint32(start), ctypes.c_uint32(count),
                                          ctypes.c_float(scale), _p(out))
    return out


def scale_from_amax(amax: float) -> float:
    return float(lib().oracle_scale_from_amax(ctypes.c_float(amax)))


def scales(x_bf16_bits: np.ndarray, per_head: bool) -> np.ndarray:
    """Scales of a BF16 tensor [T][H][D]: [1] (per tensor) or [H] (per head)."""
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    T, H, D = x.shape
    out = np.empty(H if per_head else 1, dtype=np.float32)
    lib().oracle_scales(_p(x), ctypes.c_int64(T), ctypes.c_int32(H), ctypes.c_int32(D),
                        ctypes.c_int32(1 if per_head else 0), _p(out))
    return out


def amax(x_bf16_bits: np.ndarray, per_head: bool, out: np.ndarray) -> np.ndarray:
    """Fold max|x| of a BF16 tensor [T][H][D] into out ([1] or [H] float32), in place."""
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    T, H, D = x.shape
    assert out.dtype == np.float32 and out.flags["C_CONTIGUOUS"]
    lib().oracle_amax(_p(x), ctypes.c_int64(T), ctypes.c_int32(H), ctypes.c_int32(D),
                      ctypes.c_int32(1 if per_head else 0), _p(out))
    return out


class Cache:
    """Host copy of a paged cache: the same fields the CUDA library's cache descriptor holds."""

    def __init__(self, dtype, scale_mode, num_pages, page_size, num_kv_heads, head_dim_k,
                 head_dim_v, k_pages, v_pages, k_scale, v_scale, page_tags):
        self.dtype = dtype
        self.scale_mode = scale_mode
        self.num_pages = num_pages
        self.page_size = page_size
        self.num_kv_heads = num_kv_heads
        self.head_dim_k = head_dim_k
        self.head_dim_v = head_dim_v
        self.k_pages = k_pages
        self.v_pages = v_pages
        self.k_scale = k_scale
        self.v_scale = v_scale
        self.page_tags = page_tags

    def _args(self):
        return [ctypes.c_int32(self.dtype), ctypes.c_int32(self.scale_mode),
                ctypes.c_int32(self.num_pages), ctypes.c_int32(self.page_size),
                ctypes.c_int32(self.num_kv_heads), ctypes.c_int32(self.head_dim_k),
                ctypes.c_int32(self.head_dim_v), _p(self.k_pages), _p(self.v_pages),
                _p(self.k_scale), _p(self.v_scale)]


def append(cache: Cache, k_new, v_new, slot_mapping, realloc_pages=None) -> None:
    """Bump tags of realloc_pages, then quantize/write the new tokens (in place on cache)."""
    k_new = np.ascontiguousarray(k_new, dtype=np.uint16)
    v_new = None if v_new is None else np.ascontiguousarray(v_new, dtype=np.uint16)
    slot_mapping = np.ascontiguousarray(slot_mapping, dtype=np.int32)
    rp = None if realloc_pages is None else np.ascontiguousarray(realloc_pages, dtype=np.int32)
    lib().oracle_append(*cache._args(), _p(cache.page_tags), _p(k_new), _p(v_new),
                        _p(slot_mapping), ctypes.c_int32(slot_mapping.size), _p(rp),
                        ctypes.c_int32(0 if rp is None else rp.size))


def validate(page_tags, block_table, expected_tags, seq_lens, page_size, first_bad=False):
    """Abort mask u8 [B]; with first_bad=True also each request's first failing
    block-table index (int32 [B], -1 if none)."""
    page_tags = np.ascontiguousarray(page_tags, dtype=np.uint32)
    block_table = np.ascontiguousarray(block_table, dtype=np.int32)
    expected_tags = np.ascontiguousarray(expected_tags, dtype=np.uint32)
    seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B, max_pages = block_table.shape
    out = np.empty(B, dtype=np.uint8)
    fb = np.empty(B, dtype=np.int32) if first_bad else None
    lib().oracle_validate(_p(page_tags), ctypes.c_int32(page_tags.size), _p(block_table),
                          _p(expected_tags), _p(seq_lens), ctypes.c_int32(page_size),
                          ctypes.c_int32(B), ctypes.c_int32(max_pages), _p(out), _p(fb))
    return (out, fb) if first_bad else out


def decode(cache: Cache, q_bf16_bits, block_table, seq_lens, abort_mask, sm_scale, rows=None):
    """fp64 decode attention.  Returns (out [n_rows][Dv] float64, lse [n_rows] float64)."""
    q = np.ascontiguousarray(q_bf16_bits, dtype=np.uint16)
    B, Hq, _ = q.shape
    block_table = np.ascontiguousarray(block_table, dtype=np.int32)
    seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    am = None if abort_mask is None else np.ascontiguousarray(abort_mask, dtype=np.uint8)
    rws = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    n = B * Hq if rws is None else rws.size
    out = np.empty((n, cache.head_dim_v), dtype=np.float64)
    lse = np.empty(n, dtype=np.float64)
    lib().oracle_decode(*cache._args(), _p(q), ctypes.c_int32(Hq), _p(block_table),
                        ctypes.c_int32(block_table.shape[1]), _p(seq_lens), ctypes.c_int32(B),
                        _p(am), ctypes.c_float(sm_scale), _p(rws), ctypes.c_int32(n), _p(out),
                        _p(lse))
    return out, lse
