"""Python binding of libkvq.so: the FP8 (E4M3) paged KV-cache decode path for B200.

Argument marshalling only: every step of the path runs in the CUDA kernels of
libkvq.so (csrc/).  Tensors are torch CUDA tensors; the library receives raw
device pointers and the current CUDA stream.  There is no CPU fallback: if the
shared library is missing or fails to load, every call raises.

Entry points mirror include/kvq.h:
    amax, scale_from_amax    per-tensor / per-head scale = amax / 448
    append                   tag bump on reallocation + quantize-on-append
    validate                 batched page-tag check -> abort mask
    decode, decode_bf16      split-KV paged decode attention (+ LSE combine)
    decode_noalloc           FP8 decode using the library's fixed scratch array
    e4m3_encode_bits         the device E4M3 conversion, for exhaustive checks
    device_error             read/clear the device-side error word
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvq.so")

KVQ_OK, KVQ_ERR_INVALID_ARG, KVQ_ERR_UNSUPPORTED, KVQ_ERR_WORKSPACE, KVQ_ERR_CUDA = range(5)
# bits of the device-side error word (kvq_device_error)
DEVICE_ERR_WAIT_TIMEOUT = 1    # a bounded wait gave up: that launch's outputs are invalid
DEVICE_ERR_TMEM_BASE = 2       # a wide-kernel pair's tensor memory was not at column 0
FP8_E4M3, BF16 = 0, 1
SCALE_TENSOR, SCALE_HEAD, SCALE_TOKEN = 0, 1, 2

_VP = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_U32 = ctypes.c_uint32


class KvqError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {_status_string(status)}")


class KvqCacheDesc(ctypes.Structure):
    """Mirror of the C struct kvq_cache."""
    _fields_ = [("dtype", _I32), ("scale_mode", _I32), ("num_pages", _I32),
                ("page_size", _I32), ("num_kv_heads", _I32), ("head_dim_k", _I32),
                ("head_dim_v", _I32), ("k_pages", _VP), ("v_pages", _VP),
                ("k_scale", _VP), ("v_scale", _VP), ("page_tags", _VP)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libkvq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m fp8_kv_paged_kvq_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.kvq_status_string.restype = ctypes.c_char_p
        L.kvq_status_string.argtypes = [_I32]
        L.kvq_amax.argtypes = [_VP, _I64, _I32, _I32, _I32, _VP, _VP]
        L.kvq_scale_from_amax.argtypes = [_VP, _VP, _I32, _VP]
        L.kvq_append.argtypes = [ctypes.POINTER(KvqCacheDesc), _VP, _VP, _VP, _I32, _VP, _I32, _VP]
        L.kvq_validate.argtypes = [_VP, _I32, _VP, _VP, _VP, _I32, _I32, _I32, _VP, _VP, _VP, _VP]
        L.kvq_decode_workspace_size.restype = ctypes.c_size_t
        L.kvq_decode_workspace_size.argtypes = [ctypes.POINTER(KvqCacheDesc), _I32, _I32, _I32]
        dec = [ctypes.POINTER(KvqCacheDesc), _VP, _I32, _VP, _I32, _VP, _I32, _VP, ctypes.c_float,
               _VP, _VP, _VP, ctypes.c_size_t, _I32, _VP]
        L.kvq_decode.argtypes = dec
        L.kvq_decode_bf16.argtypes = dec
        L.kvq_decode_noalloc.argtypes = [ctypes.POINTER(KvqCacheDesc), _VP, _I32, _VP, _I32, _VP,
                                         _I32, _VP, ctypes.c_float, _VP, _VP, _I32, _VP]
        L.kvq_e4m3_encode_bits.argtypes = [_U32, _U32, _VP, _VP]
        L.kvq_e4m3_quantize_bits.argtypes = [_U32, _U32, ctypes.c_float, _VP, _VP]
        L.kvq_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32)]
        L.kvq_wait_timeout_check.argtypes = [_VP, _VP]
        for f in ("kvq_amax", "kvq_scale_from_amax", "kvq_append", "kvq_validate", "kvq_decode",
                  "kvq_decode_bf16", "kvq_decode_noalloc", "kvq_e4m3_encode_bits",
                  "kvq_e4m3_quantize_bits",
                  "kvq_device_error", "kvq_wait_timeout_check"):
            getattr(L, f).restype = _I32
        _lib = L
    return _lib


def _status_string(s: int) -> str:
    return lib().kvq_status_string(s).decode()


def _check(fn: str, status: int) -> None:
    if status != KVQ_OK:
        raise KvqError(fn, status)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("kvq expects CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("kvq expects contiguous tensors")
    return _VP(t.data_ptr())


def _stream(stream) -> _VP:
    s = torch.cuda.current_stream() if stream is None else stream
    return _VP(s.cuda_stream)


# ---------------------------------------------------------------------------
# Cache
# ---------------------------------------------------------------------------
class PagedCache:
    """A paged KV cache in device memory (allocated by torch) plus its C descriptor.

    k_pages [P][Hkv][ps][Dk] (uint8 codes or bf16), v_pages [P][Hkv][ps][Dv] or None
    (V is the first Dv dims of K), scales per scale_mode, page_tags uint32 [P]
    (stored as int32 storage; the library treats them as uint32).
    """

    def __init__(self, dtype: int, scale_mode: int, num_pages: int, page_size: int,
                 num_kv_heads: int, head_dim_k: int, head_dim_v: int, v_alias: bool = False,
                 device="cuda", tags: Optional[torch.Tensor] = None):
        self.dtype, self.scale_mode = dtype, scale_mode
        self.num_pages, self.page_size = num_pages, page_size
        self.num_kv_heads, self.head_dim_k, self.head_dim_v = num_kv_heads, head_dim_k, head_dim_v
        self.v_alias = v_alias
        P, ps, H = num_pages, page_size, num_kv_heads
        el = torch.uint8 if dtype == FP8_E4M3 else torch.bfloat16
        self.k_pages = torch.zeros((P, H, ps, head_dim_k), dtype=el, device=device)
        self.v_pages = None if v_alias else torch.zeros((P, H, ps, head_dim_v), dtype=el,
                                                        device=device)
        self.k_scale = self.v_scale = None
        if dtype == FP8_E4M3:
            shape = {SCALE_TENSOR: (1,), SCALE_HEAD: (H,), SCALE_TOKEN: (P, H, ps)}[scale_mode]
            self.k_scale = torch.ones(shape, dtype=torch.float32, device=device)
            if not v_alias:
                self.v_scale = torch.ones(shape, dtype=torch.float32, device=device)
        if tags is None:
            self.page_tags = torch.zeros(P, dtype=torch.int32, device=device)
        else:
            self.page_tags = tags.to(device=device, dtype=torch.int32).contiguous()
        self.desc = KvqCacheDesc(dtype, scale_mode, P, ps, H, head_dim_k, head_dim_v,
                                 self.k_pages.data_ptr(),
                                 None if self.v_pages is None else self.v_pages.data_ptr(),
                                 None if self.k_scale is None else self.k_scale.data_ptr(),
                                 None if self.v_scale is None else self.v_scale.data_ptr(),
                                 self.page_tags.data_ptr())

    @property
    def fp8(self) -> bool:
        return self.dtype == FP8_E4M3

    def nbytes(self) -> int:
        n = self.k_pages.numel() * self.k_pages.element_size()
        if self.v_pages is not None:
            n += self.v_pages.numel() * self.v_pages.element_size()
        return n


# ---------------------------------------------------------------------------
# Calls
# ---------------------------------------------------------------------------
def amax(x: torch.Tensor, per_head: bool, out: Optional[torch.Tensor] = None,
         stream=None) -> torch.Tensor:
    """Fold max|x| of bf16 x[T][H][D] into out (float32 [1] or [H], zeroed if created here)."""
    T, H, D = x.shape
    if out is None:
        out = torch.zeros(H if per_head else 1, dtype=torch.float32, device=x.device)
    _check("kvq_amax", lib().kvq_amax(_ptr(x), T, H, D, int(per_head), _ptr(out), _stream(stream)))
    return out


def scale_from_amax(a: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None):
    out = torch.empty_like(a) if out is None else out
    _check("kvq_scale_from_amax",
           lib().kvq_scale_from_amax(_ptr(a), _ptr(out), a.numel(), _stream(stream)))
    return out


def append(cache: PagedCache, k_new: torch.Tensor, v_new: Optional[torch.Tensor],
           slot_mapping: torch.Tensor, realloc_pages: Optional[torch.Tensor] = None,
           stream=None) -> None:
    T = slot_mapping.numel()
    nr = 0 if realloc_pages is None else realloc_pages.numel()
    _check("kvq_append", lib().kvq_append(
        ctypes.byref(cache.desc), _ptr(k_new), _ptr(v_new), _ptr(slot_mapping), T,
        _ptr(realloc_pages) if nr else None, nr, _stream(stream)))


def validate(page_tags: torch.Tensor, block_table: torch.Tensor, expected_tags: torch.Tensor,
             seq_lens: torch.Tensor, page_size: int, abort_mask: Optional[torch.Tensor] = None,
             stream=None, n_aborted: Optional[torch.Tensor] = None,
             first_bad: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Abort mask u8 [B].  Optional telemetry, filled on the device: n_aborted
    (int32 [1]) = aborted requests; first_bad (int32 [B]) = each request's
    first failing block-table index, or -1."""
    B, max_pages = block_table.shape
    if abort_mask is None:
        abort_mask = torch.empty(B, dtype=torch.uint8, device=block_table.device)
    _check("kvq_validate", lib().kvq_validate(
        _ptr(page_tags), page_tags.numel(), _ptr(block_table), _ptr(expected_tags),
        _ptr(seq_lens), page_size, B, max_pages, _ptr(abort_mask), _ptr(n_aborted),
        _ptr(first_bad), _stream(stream)))
    return abort_mask


def decode_workspace_size(cache: PagedCache, B: int, num_q_heads: int, num_ctas: int = 0) -> int:
    return int(lib().kvq_decode_workspace_size(ctypes.byref(cache.desc), B, num_q_heads, num_ctas))


def alloc_workspace(cache: PagedCache, B: int, num_q_heads: int, num_ctas: int = 0,
                    device="cuda") -> torch.Tensor:
    n = decode_workspace_size(cache, B, num_q_heads, num_ctas)
    if n == 0:
        raise KvqError("kvq_decode_workspace_size", KVQ_ERR_UNSUPPORTED)
    return torch.empty(n, dtype=torch.uint8, device=device)


def decode(cache: PagedCache, q: torch.Tensor, block_table: torch.Tensor, seq_lens: torch.Tensor,
           abort_mask: Optional[torch.Tensor], sm_scale: float, out=None, lse=None,
           workspace: Optional[torch.Tensor] = None, num_ctas: int = 0, stream=None):
    """Decode attention; dispatches to kvq_decode (FP8 cache) or kvq_decode_bf16."""
    B, Hq, _ = q.shape
    if out is None:
        out = torch.empty((B, Hq, cache.head_dim_v), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(cache, B, Hq, num_ctas, q.device)
    fn = lib().kvq_decode if cache.fp8 else lib().kvq_decode_bf16
    _check("kvq_decode" if cache.fp8 else "kvq_decode_bf16", fn(
        ctypes.byref(cache.desc), _ptr(q), Hq, _ptr(block_table), block_table.shape[1],
        _ptr(seq_lens), B, _ptr(abort_mask), ctypes.c_float(sm_scale), _ptr(out), _ptr(lse),
        _ptr(workspace), workspace.numel(), num_ctas, _stream(stream)))
    return out, lse


decode_bf16 = decode


def decode_noalloc(cache: PagedCache, q: torch.Tensor, block_table: torch.Tensor,
                   seq_lens: torch.Tensor, abort_mask: Optional[torch.Tensor], sm_scale: float,
                   out: torch.Tensor, lse: Optional[torch.Tensor], num_ctas: int = 0, stream=None):
    """FP8 decode whose scratch is the library's fixed device array (no workspace argument).

    For callers that cannot allocate device memory; out / lse must be given.  Calls on one
    device share the array, so order them on one stream."""
    B, Hq, _ = q.shape
    _check("kvq_decode_noalloc", lib().kvq_decode_noalloc(
        ctypes.byref(cache.desc), _ptr(q), Hq, _ptr(block_table), block_table.shape[1],
        _ptr(seq_lens), B, _ptr(abort_mask), ctypes.c_float(sm_scale), _ptr(out), _ptr(lse),
        num_ctas, _stream(stream)))
    return out, lse


def e4m3_encode_bits(start: int, count: int, out: Optional[torch.Tensor] = None, stream=None):
    if out is None:
        out = torch.empty(count, dtype=torch.uint8, device="cuda")
    _check("kvq_e4m3_encode_bits",
           lib().kvq_e4m3_encode_bits(start, count, _ptr(out), _stream(stream)))
    return out


def e4m3_quantize_bits(start: int, count: int, scale: float,
                       out: Optional[torch.Tensor] = None, stream=None):
    """E4M3 codes of (float with bit pattern start + i) / scale, as kvq_append divides."""
    if out is None:
        out = torch.empty(count, dtype=torch.uint8, device="cuda")
    _check("kvq_e4m3_quantize_bits",
           lib().kvq_e4m3_quantize_bits(start, count, ctypes.c_float(scale), _ptr(out),
                                        _stream(stream)))
    return out


def wait_timeout_check(timed_out: torch.Tensor, stream=None) -> None:
    """Run the bounded-wait check kernel (about one second); see kvq_wait_timeout_check."""
    _check("kvq_wait_timeout_check", lib().kvq_wait_timeout_check(_ptr(timed_out), _stream(stream)))


def device_error() -> int:
    """Read and clear the device-side error word (DEVICE_ERR_* bits)."""
    v = ctypes.c_uint32(0)
    _check("kvq_device_error", lib().kvq_device_error(ctypes.byref(v)))
    return int(v.value)
