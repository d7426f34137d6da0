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
MAX_LAYERS = 256          # PKV_MAX_LAYERS
F16, BF16, INT8, INT4, FP8E4M3 = 0, 1, 2, 3, 4
QUANTIZED = (INT8, INT4, FP8E4M3)
DEV_BAD_BLOCK, DEV_BAD_SLOT, DEV_BAD_LENGTH, DEV_TIMEOUT, DEV_BAD_PREFIX = 0x1, 0x2, 0x4, 0x8, 0x10
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
    _fields_ = [("engine", ctypes.c_int32), ("partition_tokens", ctypes.c_int32), ("sliding_window", ctypes.c_int32)]


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
    L.kv_pool_create_layers.restype = i32
    L.kv_pool_create_layers.argtypes = [P, P, P, P, P, P]
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
    L.kv_copy_blocks.restype = i32
    L.kv_copy_blocks.argtypes = [P, P, P, i32, P]
    L.kv_swap_bytes_per_block.restype = sz
    L.kv_swap_bytes_per_block.argtypes = [P]
    L.kv_swap_out.restype = i32
    L.kv_swap_out.argtypes = [P, P, i32, P, P]
    L.kv_swap_in.restype = i32
    L.kv_swap_in.argtypes = [P, P, i32, P, P]
    L.paged_decode_attn_noalloc.restype = i32
    L.paged_decode_attn_noalloc.argtypes = [P, i32, P, i32, P, i32, P, i32, i32, i32, f32, P, P, P]
    L.paged_decode_cascade_workspace_bytes.restype = sz
    L.paged_decode_cascade_workspace_bytes.argtypes = [P, i32, i32, i32, i32, P]
    L.paged_decode_attn_cascade.restype = i32
    L.paged_decode_attn_cascade.argtypes = [P, i32, P, i32, P, i32, P, i32, i32, i32, i32, f32, P, P, sz, P, P]
    L.paged_prefill_chunk_attn_window.restype = i32
    L.paged_prefill_chunk_attn_window.argtypes = [P, i32, P, i32, P, i32, i32, i32, i32, f32, i32, P, P]
    L.pkv_read_device_status.restype = i32
    L.pkv_read_device_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_int32)]
    L.pkv_get_device_status.restype = i32
    L.pkv_get_device_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_int32)]
    L.pkv_test_withhold_copy.restype = i32
    L.pkv_test_withhold_copy.argtypes = [i32, ctypes.c_longlong]
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
    def from_layers(cls, k_layers, v_layers, kv_dtype: int, head_dim: int, k_scales=None, v_scales=None,
                    device_status=None) -> "KVPool":
        """A handle over per-layer allocations (kv_pool_create_layers): k_layers[l] / v_layers[l]
        [N, H_kv, 16, row] tensors, k_scales[l] / v_scales[l] fp32 [N, H_kv] (quantized)."""
        L = len(k_layers)
        if L == 0 or len(v_layers) != L or any(t.dim() != 4 or t.shape != k_layers[0].shape
                                                 for t in list(k_layers) + list(v_layers)):
            raise ValueError("k_layers / v_layers must be equal-shaped [N, H_kv, 16, row] tensors")
        self = cls.__new__(cls)
        N, H, bs, _ = k_layers[0].shape
        self.k_data, self.v_data = list(k_layers), list(v_layers)
        self.k_scale = None if k_scales is None else list(k_scales)
        self.v_scale = None if v_scales is None else list(v_scales)
        self.device_status = device_status
        self.num_layers, self.num_blocks, self.num_kv_heads, self.head_dim = L, N, H, head_dim
        self.kv_dtype = kv_dtype
        self._desc = _PoolDesc(L, N, bs, H, head_dim, kv_dtype, None, None, None, None, _ptr(device_status))
        arr = lambda ts: None if ts is None else (ctypes.c_void_p * L)(*[_ptr(t) for t in ts])  # noqa: E731
        self._arrays = (arr(self.k_data), arr(self.v_data), arr(self.k_scale), arr(self.v_scale))
        h = ctypes.c_void_p()
        _check(lib().kv_pool_create_layers(ctypes.byref(self._desc), *self._arrays, ctypes.byref(h)),
               "kv_pool_create_layers")
        self.handle = h
        return self

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


def _opts(engine: int, partition_tokens: int, sliding_window: int = 0):
    if engine == 0 and partition_tokens == 0 and sliding_window == 0:
        return None
    return ctypes.byref(_DecodeOpts(engine, partition_tokens, sliding_window))


def paged_decode_workspace_bytes(pool: KVPool, num_seqs: int, num_q_heads: int, max_context_len: int,
                                 engine: int = 0, partition_tokens: int = 0, sliding_window: int = 0) -> int:
    return int(lib().paged_decode_workspace_bytes(pool.handle, num_seqs, num_q_heads, max_context_len,
                                                  _opts(engine, partition_tokens, sliding_window)))


def paged_decode_attn(pool: KVPool, layer: int, q: torch.Tensor, block_tables: torch.Tensor,
                      context_lens: torch.Tensor, scale: float, max_context_len: int,
                      out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                      engine: int = 0, partition_tokens: int = 0, sliding_window: int = 0,
                      stream=None) -> torch.Tensor:
    """Decode attention for q [B, H_q, head_dim]; returns fp32 out [B, H_q, head_dim].
    sliding_window > 0: the query sees only the last sliding_window positions."""
    B, H_q, d = q.shape
    if out is None:
        out = torch.empty(B, H_q, d, dtype=torch.float32, device=q.device)
    need = paged_decode_workspace_bytes(pool, B, H_q, max_context_len, engine, partition_tokens, sliding_window)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().paged_decode_attn(pool.handle, layer, _ptr(q), _dtype_code(q), _ptr(block_tables),
                                   block_tables.shape[1], _ptr(context_lens), B, H_q, max_context_len,
                                   float(scale), _ptr(out), _ptr(workspace), ws_bytes,
                                   _opts(engine, partition_tokens, sliding_window), _stream(stream)),
           "paged_decode_attn")
    return out


def paged_decode_cascade_workspace_bytes(pool: KVPool, num_seqs: int, num_q_heads: int, max_context_len: int,
                                        shared_prefix_len: int, engine: int = 0, partition_tokens: int = 0) -> int:
    return int(lib().paged_decode_cascade_workspace_bytes(pool.handle, num_seqs, num_q_heads, max_context_len,
                                                          shared_prefix_len, _opts(engine, partition_tokens)))


def paged_decode_attn_cascade(pool: KVPool, layer: int, q: torch.Tensor, block_tables: torch.Tensor,
                              context_lens: torch.Tensor, scale: float, max_context_len: int,
                              shared_prefix_len: int, out: torch.Tensor | None = None,
                              workspace: torch.Tensor | None = None, engine: int = 0, partition_tokens: int = 0,
                              sliding_window: int = 0, stream=None) -> torch.Tensor:
    """Decode attention for a batch whose tables all start with the same shared_prefix_len
    tokens (row 0's blocks): the prefix is attended once per KV group on the tensor cores."""
    fn = lib().paged_decode_attn_cascade
    B, H_q, d = q.shape
    if out is None:
        out = torch.empty(B, H_q, d, dtype=torch.float32, device=q.device)
    need = paged_decode_cascade_workspace_bytes(pool, B, H_q, max_context_len, shared_prefix_len, engine,
                                                partition_tokens)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(fn(pool.handle, layer, _ptr(q), _dtype_code(q), _ptr(block_tables), block_tables.shape[1],
              _ptr(context_lens), B, H_q, max_context_len, shared_prefix_len, float(scale), _ptr(out),
              _ptr(workspace), ws_bytes, _opts(engine, partition_tokens, sliding_window), _stream(stream)),
           "paged_decode_attn_cascade")
    return out


NOALLOC_SCRATCH_BYTES = 32 << 20


def paged_decode_attn_noalloc(pool: KVPool, layer: int, q: torch.Tensor, block_tables: torch.Tensor,
                              context_lens: torch.Tensor, scale: float, max_context_len: int,
                              out: torch.Tensor | None = None, engine: int = 0, partition_tokens: int = 0,
                              sliding_window: int = 0, stream=None) -> torch.Tensor:
    """paged_decode_attn without a workspace argument, for callers that cannot allocate device
    memory for one: the split-K partials use the library's fixed 32 MiB device buffer.  Only
    the output is the caller's.  Calls that may overlap on the GPU share that buffer and race;
    issue them in order on one stream."""
    fn = lib().paged_decode_attn_noalloc
    B, H_q, d = q.shape
    if out is None:
        out = torch.empty(B, H_q, d, dtype=torch.float32, device=q.device)
    _check(fn(pool.handle, layer, _ptr(q), _dtype_code(q), _ptr(block_tables), block_tables.shape[1],
              _ptr(context_lens), B, H_q, max_context_len, float(scale), _ptr(out),
              _opts(engine, partition_tokens, sliding_window), _stream(stream)), "paged_decode_attn_noalloc")
    return out


def paged_prefill_chunk_attn(pool: KVPool, layer: int, q: torch.Tensor, block_table: torch.Tensor,
                             ctx_before: int, scale: float, out: torch.Tensor | None = None,
                             sliding_window: int = 0, stream=None) -> torch.Tensor:
    """Chunked-prefill attention for q [C, H_q, head_dim] at positions ctx_before + i
    (sliding_window > 0: each row sees only the last sliding_window positions up to itself)."""
    C, H_q, d = q.shape
    if out is None:
        out = torch.empty(C, H_q, d, dtype=torch.float32, device=q.device)
    if sliding_window == 0:
        _check(lib().paged_prefill_chunk_attn(pool.handle, layer, _ptr(q), _dtype_code(q), _ptr(block_table),
                                              block_table.shape[-1], ctx_before, C, H_q, float(scale), _ptr(out),
                                              None, 0, _stream(stream)), "paged_prefill_chunk_attn")
        return out
    fn = lib().paged_prefill_chunk_attn_window
    _check(fn(pool.handle, layer, _ptr(q), _dtype_code(q), _ptr(block_table), block_table.shape[-1], ctx_before, C,
              H_q, float(scale), int(sliding_window), _ptr(out), _stream(stream)), "paged_prefill_chunk_attn_window")
    return out


def kv_copy_blocks(pool: KVPool, src: torch.Tensor, dst: torch.Tensor, stream=None) -> None:
    """Copy physical block src[j] onto block dst[j] (all layers, K, V and scales); int32 tensors."""
    if src.shape != dst.shape or src.dim() != 1:
        raise ValueError("src and dst must be int32 vectors of one length")
    _check(lib().kv_copy_blocks(pool.handle, _ptr(src), _ptr(dst), src.shape[0], _stream(stream)),
           "kv_copy_blocks")


def kv_swap_bytes_per_block(pool: KVPool) -> int:
    return int(lib().kv_swap_bytes_per_block(pool.handle))


def _host_ptr(t: torch.Tensor):
    if t.is_cuda or not t.is_pinned() or not t.is_contiguous():
        raise ValueError("expected a contiguous pinned host tensor")
    return ctypes.c_void_p(t.data_ptr())


def _check_swap_buffer(pool: KVPool, blocks: torch.Tensor, host: torch.Tensor):
    if host.numel() * host.element_size() < blocks.shape[0] * kv_swap_bytes_per_block(pool):
        raise ValueError("host swap buffer too small")


def kv_swap_out(pool: KVPool, blocks: torch.Tensor, host: torch.Tensor, stream=None) -> None:
    """Copy blocks [int32, device] to consecutive slots of the pinned host buffer `host`."""
    _check_swap_buffer(pool, blocks, host)
    _check(lib().kv_swap_out(pool.handle, _ptr(blocks), blocks.shape[0], _host_ptr(host), _stream(stream)),
           "kv_swap_out")


def kv_swap_in(pool: KVPool, blocks: torch.Tensor, host: torch.Tensor, stream=None) -> None:
    """Copy consecutive slots of the pinned host buffer `host` into blocks [int32, device]."""
    _check_swap_buffer(pool, blocks, host)
    _check(lib().kv_swap_in(pool.handle, _ptr(blocks), blocks.shape[0], _host_ptr(host), _stream(stream)),
           "kv_swap_in")


def read_device_status(pool: KVPool, stream=None) -> int:
    """Synchronize the stream and return (and clear) the pool's device status bits."""
    st = ctypes.c_int32(0)
    rc = lib().pkv_read_device_status(pool.handle, _stream(stream), ctypes.byref(st))
    if rc not in (0, -7, -8):
        _check(rc, "pkv_read_device_status")
    return int(st.value)


def get_device_status(pool: KVPool, stream=None) -> tuple[int, int]:
    """pkv_get_device_status: (its return code, the status bits it read and cleared)."""
    st = ctypes.c_int32(0)
    rc = lib().pkv_get_device_status(pool.handle, _stream(stream), ctypes.byref(st))
    if rc not in (0, -7, -8):
        _check(rc, "pkv_get_device_status")
    return int(rc), int(st.value)


def test_withhold_copy(tile: int, wait_cycles: int = 0) -> None:
    """pkv_test_withhold_copy: from now on every attention kernel withholds the copy of its
    `tile`-th K/V tile and bounds its waits at `wait_cycles` SM cycles (tile < 0: off)."""
    _check(lib().pkv_test_withhold_copy(int(tile), int(wait_cycles)), "pkv_test_withhold_copy")


# ------------------------------------------------------------ block manager --

ERR_NO_BLOCKS, ERR_STATE = -10, -11


class _BMStats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("num_blocks", "free_blocks", "cached_blocks", "used_blocks",
                                              "shared_blocks", "num_sequences", "prefix_queries", "prefix_hits",
                                              "cow_copies", "evictions")]


def _bm_lib():
    L = lib()
    if getattr(L, "_bm_ready", False):
        return L
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    pi = ctypes.POINTER(ctypes.c_int32)
    sig = {
        "pkv_bm_create": (ctypes.c_int, [i32, ctypes.c_int, P]),
        "pkv_bm_destroy": (ctypes.c_int, [P]),
        "pkv_bm_free_blocks": (i64, [P]),
        "pkv_bm_refcount": (ctypes.c_int, [P, i32]),
        "pkv_bm_add_sequence": (ctypes.c_int, [P, i64, pi, i32, pi]),
        "pkv_bm_blocks_needed": (ctypes.c_int, [P, i64, i32]),
        "pkv_bm_append_slots": (ctypes.c_int, [P, i64, pi, i32, pi, pi, pi, pi]),
        "pkv_bm_fork": (ctypes.c_int, [P, i64, i64]),
        "pkv_bm_free_sequence": (ctypes.c_int, [P, i64]),
        "pkv_bm_block_table": (ctypes.c_int, [P, i64, pi, i32, pi, pi]),
        "pkv_bm_swap_out": (ctypes.c_int, [P, i64, pi, i32, pi]),
        "pkv_bm_swap_in": (ctypes.c_int, [P, i64, pi, i32, pi]),
        "pkv_bm_get_stats": (ctypes.c_int, [P, ctypes.POINTER(_BMStats)]),
        "pkv_bm_check": (ctypes.c_int, [P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype, fn.argtypes = res, args
    L._bm_ready = True
    return L


def _i32_array(values):
    values = list(values)
    return (ctypes.c_int32 * max(1, len(values)))(*values)


class BlockManager:
    """Host-side block manager of a paged KV cache (free list, reference counts,
    copy-on-write, prefix cache, swap bookkeeping); a thin wrapper of pkv_bm_* in libpkv.

    Methods raise PkvError on a non-zero status; ``append_slots`` returns
    ``(slot_mapping list, cow pair or None)``."""

    def __init__(self, num_blocks: int, enable_prefix_cache: bool = True):
        self._L = _bm_lib()
        h = ctypes.c_void_p()
        _check(self._L.pkv_bm_create(num_blocks, 1 if enable_prefix_cache else 0, ctypes.byref(h)), "pkv_bm_create")
        self.handle = h
        self.num_blocks = num_blocks

    def close(self):
        if getattr(self, "handle", None) is not None:
            self._L.pkv_bm_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def free_blocks(self) -> int:
        n = int(self._L.pkv_bm_free_blocks(self.handle))
        _check(min(n, 0), "pkv_bm_free_blocks")
        return n

    def refcount(self, block: int) -> int:
        n = self._L.pkv_bm_refcount(self.handle, block)
        _check(min(n, 0), "pkv_bm_refcount")
        return n

    def add_sequence(self, seq_id: int, prompt=None, n_prompt: int | None = None) -> int:
        """Register a sequence; returns the number of prompt tokens found in the prefix cache."""
        toks = None if prompt is None else _i32_array(prompt)
        n = len(prompt) if prompt is not None else int(n_prompt or 0)
        cached = ctypes.c_int32(0)
        _check(self._L.pkv_bm_add_sequence(self.handle, seq_id, toks, n, ctypes.byref(cached)),
               "pkv_bm_add_sequence")
        return int(cached.value)

    def blocks_needed(self, seq_id: int, n: int) -> int:
        r = self._L.pkv_bm_blocks_needed(self.handle, seq_id, n)
        _check(min(r, 0), "pkv_bm_blocks_needed")
        return r

    def append_slots(self, seq_id: int, n: int, tokens=None):
        slots = (ctypes.c_int32 * max(1, n))()
        src, dst, ncow = ctypes.c_int32(-1), ctypes.c_int32(-1), ctypes.c_int32(0)
        toks = None if tokens is None else _i32_array(tokens)
        if tokens is not None and len(tokens) != n:
            raise ValueError("len(tokens) != n")
        _check(self._L.pkv_bm_append_slots(self.handle, seq_id, toks, n, slots, ctypes.byref(src), ctypes.byref(dst),
                                           ctypes.byref(ncow)), "pkv_bm_append_slots")
        return list(slots)[:n], ((int(src.value), int(dst.value)) if ncow.value else None)

    def fork(self, parent_id: int, child_id: int) -> None:
        _check(self._L.pkv_bm_fork(self.handle, parent_id, child_id), "pkv_bm_fork")

    def free_sequence(self, seq_id: int) -> None:
        _check(self._L.pkv_bm_free_sequence(self.handle, seq_id), "pkv_bm_free_sequence")

    def block_table(self, seq_id: int):
        """(list of physical blocks, number of tokens)."""
        nb, nt = ctypes.c_int32(0), ctypes.c_int32(0)
        rc = self._L.pkv_bm_block_table(self.handle, seq_id, None, 0, ctypes.byref(nb), ctypes.byref(nt))
        if rc not in (0, -2):
            _check(rc, "pkv_bm_block_table")
        buf = (ctypes.c_int32 * max(1, nb.value))()
        _check(self._L.pkv_bm_block_table(self.handle, seq_id, buf, nb.value, None, None), "pkv_bm_block_table")
        return list(buf)[:nb.value], int(nt.value)

    def swap_out(self, seq_id: int):
        """Release the sequence's blocks; returns them (to be copied out with kv_swap_out)."""
        table, _ = self.block_table(seq_id)
        buf = (ctypes.c_int32 * max(1, len(table)))()
        n = ctypes.c_int32(0)
        _check(self._L.pkv_bm_swap_out(self.handle, seq_id, buf, len(table), ctypes.byref(n)), "pkv_bm_swap_out")
        return list(buf)[:n.value]

    def swap_in(self, seq_id: int, num_blocks: int):
        """Give a swapped-out sequence fresh blocks; returns them (to be filled with kv_swap_in)."""
        buf = (ctypes.c_int32 * max(1, num_blocks))()
        n = ctypes.c_int32(0)
        _check(self._L.pkv_bm_swap_in(self.handle, seq_id, buf, num_blocks, ctypes.byref(n)), "pkv_bm_swap_in")
        return list(buf)[:n.value]

    def stats(self) -> dict:
        s = _BMStats()
        _check(self._L.pkv_bm_get_stats(self.handle, ctypes.byref(s)), "pkv_bm_get_stats")
        return {n: int(getattr(s, n)) for n, _ in _BMStats._fields_}

    def check(self) -> None:
        _check(self._L.pkv_bm_check(self.handle), "pkv_bm_check")
