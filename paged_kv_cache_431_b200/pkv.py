"""Python binding of libpkv.so -- argument marshalling only.

Every function forwards to the C-ABI entry point of the same name (declared in
``include/pkv.h``) with raw device pointers taken from torch tensors and the current
torch CUDA stream.  All computation runs in the library's CUDA kernels; there is no
fallback.  If the library cannot be loaded the import fails with an error.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

BLOCK_SIZE = 16
F16, BF16, INT8, INT4, FP8E4M3 = 0, 1, 2, 3, 4
QUANTIZED = (INT8, INT4, FP8E4M3)
DEV_BAD_BLOCK, DEV_BAD_SLOT, DEV_BAD_LENGTH, DEV_TIMEOUT = 0x1, 0x2, 0x4, 0x8
ENGINE_AUTO, ENGINE_MMA, ENGINE_FMA2, ENGINE_FMA = 0, 1, 2, 3

_TORCH16 = {F16: torch.float16, BF16: torch.bfloat16}


class PkvError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {strerror(status)} (status {status})")
        self.status = status


class _PoolDesc(ctypes.Structure):
    _fields_ = [("num_layers", ctypes.c_int32), ("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("kv_dtype", ctypes.c_int32),
                ("k_data", ctypes.c_void_p), ("v_data", ctypes.c_void_p), ("k_scale", ctypes.c_void_p),
                ("v_scale", ctypes.c_void_p), ("device_status", ctypes.c_void_p)]


class _DecodeOpts(ctypes.Structure):
    _fields_ = [("engine", ctypes.c_int32), ("partition_tokens", ctypes.c_int32)]


_lib = None


def library_path() -> str:
    return _build.LIB


def lib() -> ctypes.CDLL:
    """Load libpkv.so (building it with nvcc first if it is missing or stale)."""
    global _lib
    if _lib is not None:
        return _lib
    path = _build.LIB
    try:
        path = _build.build()
    except Exception as e:  # no nvcc here: a prebuilt library must exist
        if not os.path.exists(path):
            raise RuntimeError(f"libpkv.so is missing and could not be built: {e}") from e
    L = ctypes.CDLL(path)
    P, i32, sz, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    L.pkv_version.restype = i32
    L.pkv_strerror.restype = ctypes.c_char_p
    L.pkv_strerror.argtypes = [i32]
    L.pkv_pool_bytes.restype = sz
    L.pkv_pool_bytes.argtypes = [P, P]
    L.kv_pool_create.restype = i32
    L.kv_pool_create.argtypes = [P, P]
    L.kv_pool_destroy.restype = i32
    L.kv_pool_destroy.argtypes = [P]
    L.kv_append_workspace_bytes.restype = sz
    L.kv_append_workspace_bytes.argtypes = [P, i32]
    L.kv_append.restype = i32
    L.kv_append.argtypes = [P, i32, P, P, i32, P, i32, P, sz, P]
    L.paged_decode_workspace_bytes.restype = sz
    L.paged_decode_workspace_bytes.argtypes = [P, i32, i32, i32, P]
    L.paged_decode_attn.restype = i32
    L.paged_decode_attn.argtypes = [P, i32, P, i32, P, i32, P, i32, i32, i32, f32, P, P, sz, P, P]
    L.paged_prefill_workspace_bytes.restype = sz
    L.paged_prefill_workspace_bytes.argtypes = [P, i32, i32, i32]
    L.paged_prefill_chunk_attn.restype = i32
    L.paged_prefill_chunk_attn.argtypes = [P, i32, P, i32, P, i32, i32, i32, i32, f32, P, P, sz, P]
    L.pkv_read_device_status.restype = i32
    L.pkv_read_device_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_int32)]
    _lib = L
    return L


def strerror(status: int) -> str:
    return lib().pkv_strerror(status).decode()


def _check(rc: int, what: str):
    if rc != 0:
        raise PkvError(rc, what)


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def row_bytes(kv_dtype: int, head_dim: int) -> int:
    return {F16: 2 * head_dim, BF16: 2 * head_dim, INT8: head_dim, FP8E4M3: head_dim, INT4: head_dim // 2}[kv_dtype]


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float16:
        return F16
    if t.dtype == torch.bfloat16:
        return BF16
    raise ValueError(f"unsupported tensor dtype {t.dtype}")


class KVPool:
    """A handle on caller-owned K/V pool memory (torch tensors).

    k_data / v_data: [L, N, H_kv, 16, head_dim] f16/bf16 tensors, or [L, N, H_kv, 16,
    row_bytes] uint8 for quantized dtypes; k_scale / v_scale: fp32 [L, N, H_kv].
    """

    def __init__(self, k_data, v_data, kv_dtype: int, head_dim: int, k_scale=None, v_scale=None,
                 device_status=None):
        if k_data.dim() != 5 or k_data.shape != v_data.shape:
            raise ValueError("k_data / v_data must be [L, N, H_kv, 16, row]")
        L, N, H, bs, _ = k_data.shape
        self.k_data, self.v_data, self.k_scale, self.v_scale = k_data, v_data, k_scale, v_scale
        self.device_status = device_status
        self.num_layers, self.num_blocks, self.num_kv_heads, self.head_dim = L, N, H, head_dim
        self.kv_dtype = kv_dtype
        self._desc = _PoolDesc(L, N, bs, H, head_dim, kv_dtype, _ptr(k_data), _ptr(v_data), _ptr(k_scale),
                               _ptr(v_scale), _ptr(device_status))
        h = ctypes.c_void_p()
        _check(lib().kv_pool_create(ctypes.byref(self._desc), ctypes.byref(h)), "kv_pool_create")
        self.handle = h

    @classmethod
    def allocate(cls, num_layers: int, num_blocks: int, num_kv_heads: int, head_dim: int, kv_dtype: int,
                 device="cuda", with_status: bool = True) -> "KVPool":
        shape = (num_layers, num_blocks, num_kv_heads, BLOCK_SIZE)
        if kv_dtype in _TORCH16:
            k = torch.zeros(*shape, head_dim, dtype=_TORCH16[kv_dtype], device=device)
            v = torch.zeros_like(k)
            ks = vs = None
        else:
            k = torch.zeros(*shape, row_bytes(kv_dtype, head_dim), dtype=torch.uint8, device=device)
            v = torch.zeros_like(k)
            ks = torch.zeros(num_layers, num_blocks, num_kv_heads, dtype=torch.float32, device=device)
            vs = torch.zeros_like(ks)
        st = torch.zeros(1, dtype=torch.int32, device=device) if with_status else None
        return cls(k, v, kv_dtype, head_dim, ks, vs, st)

    def close(self):
        if getattr(self, "handle", None) is not None and _lib is not None:
            _lib.kv_pool_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def kv_pool_create(k_data, v_data, kv_dtype: int, head_dim: int, k_scale=None, v_scale=None,
                   device_status=None) -> KVPool:
    return KVPool(k_data, v_data, kv_dtype, head_dim, k_scale, v_scale, device_status)


def pkv_pool_bytes(num_layers: int, num_blocks: int, num_kv_heads: int, head_dim: int, kv_dtype: int):
    """(pool bytes of K (== V), scale bytes of K (== V)) from the library's sizing helper."""
    d = _PoolDesc(num_layers, num_blocks, BLOCK_SIZE, num_kv_heads, head_dim, kv_dtype, None, None, None, None, None)
    sb = ctypes.c_size_t(0)
    n = lib().pkv_pool_bytes(ctypes.byref(d), ctypes.byref(sb))
    return int(n), int(sb.value)


def kv_append_workspace_bytes(pool: KVPool, num_tokens: int) -> int:
    return int(lib().kv_append_workspace_bytes(pool.handle, num_tokens))


def kv_append(pool: KVPool, layer: int, k: torch.Tensor, v: torch.Tensor, slot_mapping: torch.Tensor,
              workspace: torch.Tensor | None = None, stream=None) -> None:
    """Write tokens k, v [T, H_kv, head_dim] into slots slot_mapping [T] (int32)."""
    T = slot_mapping.shape[0]
    need = kv_append_workspace_bytes(pool, T)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=k.device)
    _check(lib().kv_append(pool.handle, layer, _ptr(k), _ptr(v), _dtype_code(k), _ptr(slot_mapping), T,
                           _ptr(workspace), workspace.numel() * workspace.element_size() if workspace is not None
                           else 0, _stream(stream)), "kv_append")


def _opts(engine: int, partition_tokens: int):
    if engine == 0 and partition_tokens == 0:
        return None
    return ctypes.byref(_DecodeOpts(engine, partition_tokens))


def paged_decode_workspace_bytes(pool: KVPool, num_seqs: int, num_q_heads: int, max_context_len: int,
                                 engine: int = 0, partition_tokens: int = 0) -> int:
    return int(lib().paged_decode_workspace_bytes(pool.handle, num_seqs, num_q_heads, max_context_len,
                                                  _opts(engine, partition_tokens)))


def paged_decode_attn(pool: KVPool, layer: int, q: torch.Tensor, block_tables: torch.Tensor,
                      context_lens: torch.Tensor, scale: float, max_context_len: int,
                      out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                      engine: int = 0, partition_tokens: int = 0, stream=None) -> torch.Tensor:
    """Decode attention for q [B, H_q, head_dim]; returns fp32 out [B, H_q, head_dim]."""
    B, H_q, d = q.shape
    if out is None:
        out = torch.empty(B, H_q, d, dtype=torch.float32, device=q.device)
    need = paged_decode_workspace_bytes(pool, B, H_q, max_context_len, engine, partition_tokens)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().paged_decode_attn(pool.handle, layer, _ptr(q), _dtype_code(q), _ptr(block_tables),
                                   block_tables.shape[1], _ptr(context_lens), B, H_q, max_context_len,
                                   float(scale), _ptr(out), _ptr(workspace), ws_bytes,
                                   _opts(engine, partition_tokens), _stream(stream)), "paged_decode_attn")
    return out


NOALLOC_SCRATCH_BYTES = 32 << 20


def paged_decode_attn_noalloc(pool: KVPool, layer: int, q: torch.Tensor, block_tables: torch.Tensor,
                              context_lens: torch.Tensor, scale: float, max_context_len: int,
                              out: torch.Tensor | None = None, engine: int = 0, partition_tokens: int = 0,
                              stream=None) -> torch.Tensor:
    """paged_decode_attn without a workspace argument, for callers that cannot allocate device
    memory for one: the split-K partials use the library's fixed 32 MiB device buffer.  Only
    the output is the caller's.  Calls that may overlap on the GPU share that buffer and race;
    issue them in order on one stream."""
    L = lib()
    fn = L.paged_decode_attn_noalloc
    P, i32 = ctypes.c_void_p, ctypes.c_int
    fn.restype = i32
    fn.argtypes = [P, i32, P, i32, P, i32, P, i32, i32, i32, ctypes.c_float, P, P, P]
    B, H_q, d = q.shape
    if out is None:
        out = torch.empty(B, H_q, d, dtype=torch.float32, device=q.device)
    _check(fn(pool.handle, layer, _ptr(q), _dtype_code(q), _ptr(block_tables), block_tables.shape[1],
              _ptr(context_lens), B, H_q, max_context_len, float(scale), _ptr(out),
              _opts(engine, partition_tokens), _stream(stream)), "paged_decode_attn_noalloc")
    return out


def paged_prefill_chunk_attn(pool: KVPool, layer: int, q: torch.Tensor, block_table: torch.Tensor,
                             ctx_before: int, scale: float, out: torch.Tensor | None = None,
                             stream=None) -> torch.Tensor:
    """Chunked-prefill attention for q [C, H_q, head_dim] at positions ctx_before + i."""
    C, H_q, d = q.shape
    if out is None:
        out = torch.empty(C, H_q, d, dtype=torch.float32, device=q.device)
    _check(lib().paged_prefill_chunk_attn(pool.handle, layer, _ptr(q), _dtype_code(q), _ptr(block_table),
                                          block_table.shape[-1], ctx_before, C, H_q, float(scale), _ptr(out),
                                          None, 0, _stream(stream)), "paged_prefill_chunk_attn")
    return out


def read_device_status(pool: KVPool, stream=None) -> int:
    """Synchronize the stream and return (and clear) the pool's device status bits."""
    st = ctypes.c_int32(0)
    rc = lib().pkv_read_device_status(pool.handle, _stream(stream), ctypes.byref(st))
    if rc not in (0, -7, -8):
        _check(rc, "pkv_read_device_status")
    return int(st.value)
