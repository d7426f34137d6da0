"""CPU oracle for attention over a paged KV cache -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package.  The product path (``paged_kv_cache_431_b200``) never
imports it, and the two share no code: the oracle is plain C (``pkv_oracle.c``),
compiled with gcc, computing attention in fp64 from its definition and the
quantization codes in IEEE fp32.

This module is argument marshalling for that C library (numpy arrays in, numpy
arrays out) plus a small ``Pool`` holder for the oracle's own copy of a KV pool.

Sources (web pages on paged KV caches), cited in the C file:
  "KV cache, continuous batching and paged attention"  (KV size, paged attention)
  "KV cache, GQA, paging and continuous batching"      (memory equation, block table)
  inference guide "a2-inf-2"                           (quantization, chunked prefill)
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pkv_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libpkv_oracle.so")

BLOCK = 16
F16, BF16, INT8, INT4, FP8 = 0, 1, 2, 3, 4
QUANTIZED = (INT8, INT4, FP8)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


class use_library:
    """Temporarily run the oracle functions on another build of the C source (the
    mutation tests use this to check that the pins catch planted mistakes)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        self.saved = _lib
        _lib = None
        lib(self.path)

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved


def compile_source(src_text: str, out_path: str) -> str:
    """Compile C source text with the oracle's flags into ``out_path``."""
    c_path = out_path + ".c"
    with open(c_path, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                           "-fno-fast-math", "-w", "-o", out_path, c_path, "-lm"])
    return out_path


def lib(path: str | None = None):
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(path or build())
        P = ctypes.c_void_p
        i32, i64, f32 = ctypes.c_int, ctypes.c_int64, ctypes.c_float
        _lib.orc_kv_bytes_per_token.restype = i64
        _lib.orc_kv_bytes_per_token.argtypes = [i32, i32, i32, i32]
        _lib.orc_kv_cache_bytes.restype = i64
        _lib.orc_kv_cache_bytes.argtypes = [i32, i32, i32, i32, i64, i64]
        _lib.orc_blocks_for_tokens.restype = i64
        _lib.orc_blocks_for_tokens.argtypes = [i64]
        _lib.orc_waste_slots.restype = i64
        _lib.orc_waste_slots.argtypes = [i64]
        _lib.orc_e4m3_from_f32.restype = ctypes.c_uint8
        _lib.orc_e4m3_from_f32.argtypes = [f32]
        _lib.orc_e4m3_to_f64.restype = ctypes.c_double
        _lib.orc_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        for name in ("orc_e4m3_encode_array", "orc_e4m3_decode_array",
                     "orc_f16_decode_array", "orc_bf16_decode_array"):
            getattr(_lib, name).restype = None
            getattr(_lib, name).argtypes = [P, P, i64]
        _lib.orc_pool_dequant.restype = i32
        _lib.orc_pool_dequant.argtypes = [i32, i32, i32, i32, P, P, P]
        _lib.orc_kv_append.restype = i32
        _lib.orc_kv_append.argtypes = [i32, i32, i32, i32, P, P, P, P, P, P, i32, P, i32]
        _lib.orc_paged_decode.restype = i32
        _lib.orc_paged_decode.argtypes = [i32, i32, i32, i32, P, P, P, P, P, i32, i32, P, i32, P, i32, f32, P]
        _lib.orc_paged_prefill_chunk.restype = i32
        _lib.orc_paged_prefill_chunk.argtypes = [i32, i32, i32, i32, P, P, P, P, P, i32, i32, P, i32, i32,
                                                 i32, f32, P]
        _lib.orc_paged_decode_window.restype = i32
        _lib.orc_paged_decode_window.argtypes = [i32, i32, i32, i32, P, P, P, P, P, i32, i32, P, i32, P, i32, f32,
                                                 i32, P]
        _lib.orc_paged_prefill_chunk_window.restype = i32
        _lib.orc_paged_prefill_chunk_window.argtypes = [i32, i32, i32, i32, P, P, P, P, P, i32, i32, P, i32, i32,
                                                        i32, f32, i32, P]
    return _lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with status {rc}")


def row_bytes(dtype: int, d: int) -> int:
    return {F16: 2 * d, BF16: 2 * d, INT8: d, FP8: d, INT4: d // 2}[dtype]


def as_u16(a) -> np.ndarray:
    """A 16-bit float array (numpy float16, or a torch f16/bf16 tensor) as raw uint16 bits."""
    if isinstance(a, np.ndarray):
        return np.ascontiguousarray(a).view(np.uint16)
    import torch  # only for reading a tensor's bytes
    t = a.detach().contiguous().cpu()
    assert t.dtype in (torch.float16, torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


# ----------------------------------------------------------------- sizes --

def kv_bytes_per_token(layers: int, kv_heads: int, head_dim: int, bytes_per_elem: int) -> int:
    return int(lib().orc_kv_bytes_per_token(layers, kv_heads, head_dim, bytes_per_elem))


def kv_cache_bytes(layers, kv_heads, head_dim, bytes_per_elem, seq_len, batch) -> int:
    return int(lib().orc_kv_cache_bytes(layers, kv_heads, head_dim, bytes_per_elem, seq_len, batch))


def blocks_for_tokens(n: int) -> int:
    return int(lib().orc_blocks_for_tokens(n))


def waste_slots(n: int) -> int:
    return int(lib().orc_waste_slots(n))


# ---------------------------------------------------------------- codecs --

def e4m3_encode(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().orc_e4m3_encode_array(_ptr(x), _ptr(out), x.size)
    return out


def e4m3_decode(c) -> np.ndarray:
    c = np.ascontiguousarray(c, dtype=np.uint8)
    out = np.empty(c.shape, np.float64)
    lib().orc_e4m3_decode_array(_ptr(c), _ptr(out), c.size)
    return out


def f16_decode(h) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(h.shape, np.float64)
    lib().orc_f16_decode_array(_ptr(h), _ptr(out), h.size)
    return out


def bf16_decode(h) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(h.shape, np.float64)
    lib().orc_bf16_decode_array(_ptr(h), _ptr(out), h.size)
    return out


# ------------------------------------------------------------------ pool --

class Pool:
    """The oracle's own copy of one layer's K/V pool.

    ``k``/``v`` hold raw bytes [N, H_kv, 16, row_bytes]; ``k_scale``/``v_scale`` are
    fp32 [N, H_kv] (used by quantized dtypes only).
    """

    def __init__(self, num_blocks: int, num_kv_heads: int, head_dim: int, dtype: int,
                 k: np.ndarray | None = None, v: np.ndarray | None = None,
                 k_scale: np.ndarray | None = None, v_scale: np.ndarray | None = None):
        self.N, self.H_kv, self.d, self.dtype = num_blocks, num_kv_heads, head_dim, dtype
        shape = (num_blocks, num_kv_heads, BLOCK, row_bytes(dtype, head_dim))
        self.k = np.zeros(shape, np.uint8) if k is None else np.ascontiguousarray(k).view(np.uint8).reshape(shape)
        self.v = np.zeros(shape, np.uint8) if v is None else np.ascontiguousarray(v).view(np.uint8).reshape(shape)
        sshape = (num_blocks, num_kv_heads)
        self.k_scale = (np.zeros(sshape, np.float32) if k_scale is None
                        else np.ascontiguousarray(k_scale, dtype=np.float32).reshape(sshape))
        self.v_scale = (np.zeros(sshape, np.float32) if v_scale is None
                        else np.ascontiguousarray(v_scale, dtype=np.float32).reshape(sshape))

    def copy(self) -> "Pool":
        return Pool(self.N, self.H_kv, self.d, self.dtype, self.k.copy(), self.v.copy(),
                    self.k_scale.copy(), self.v_scale.copy())

    def dequant(self, which: str = "k") -> np.ndarray:
        """Every element's value in fp64, [N, H_kv, 16, d]."""
        out = np.empty((self.N, self.H_kv, BLOCK, self.d), np.float64)
        pool, sc = (self.k, self.k_scale) if which == "k" else (self.v, self.v_scale)
        _check(lib().orc_pool_dequant(self.N, self.H_kv, self.d, self.dtype, _ptr(pool), _ptr(sc), _ptr(out)),
               "pool_dequant")
        return out


def kv_append(pool: Pool, k_src, v_src, src_dtype: int, slots) -> None:
    """Write tokens [T, H_kv, d] (16-bit source bits) into their slots (in place)."""
    k_src, v_src = as_u16(k_src), as_u16(v_src)
    slots = np.ascontiguousarray(slots, dtype=np.int32)
    T = slots.shape[0]
    assert k_src.shape == (T, pool.H_kv, pool.d) and v_src.shape == k_src.shape
    _check(lib().orc_kv_append(pool.N, pool.H_kv, pool.d, pool.dtype, _ptr(pool.k), _ptr(pool.v),
                               _ptr(pool.k_scale), _ptr(pool.v_scale), _ptr(k_src), _ptr(v_src),
                               src_dtype, _ptr(slots), T), "kv_append")


def paged_decode(pool: Pool, q, q_dtype: int, block_tables, ctx_lens, scale: float, window: int = 0) -> np.ndarray:
    """Decode attention, fp64 [B, H_q, d]; window > 0: only the `window` most recent positions."""
    q = as_u16(q)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(ctx_lens, dtype=np.int32)
    B, H_q, d = q.shape
    assert d == pool.d and bt.shape[0] == B and cl.shape == (B,)
    out = np.empty((B, H_q, d), np.float64)
    _check(lib().orc_paged_decode_window(pool.N, pool.H_kv, pool.d, pool.dtype, _ptr(pool.k), _ptr(pool.v),
                                         _ptr(pool.k_scale), _ptr(pool.v_scale), _ptr(q), q_dtype, H_q,
                                         _ptr(bt), bt.shape[1], _ptr(cl), B, float(scale), int(window), _ptr(out)),
           "paged_decode")
    return out


def paged_prefill_chunk(pool: Pool, q, q_dtype: int, block_table, ctx_before: int, scale: float,
                        window: int = 0) -> np.ndarray:
    """Chunked-prefill attention of C query positions after ctx_before cached ones, fp64 [C, H_q, d];
    window > 0: each row sees only the `window` most recent positions up to itself."""
    q = as_u16(q)
    bt = np.ascontiguousarray(block_table, dtype=np.int32).reshape(-1)
    C, H_q, d = q.shape
    out = np.empty((C, H_q, d), np.float64)
    _check(lib().orc_paged_prefill_chunk_window(pool.N, pool.H_kv, pool.d, pool.dtype, _ptr(pool.k),
                                                _ptr(pool.v), _ptr(pool.k_scale), _ptr(pool.v_scale), _ptr(q),
                                                q_dtype, H_q, _ptr(bt), bt.shape[0], ctx_before, C, float(scale),
                                                int(window), _ptr(out)),
           "paged_prefill_chunk")
    return out


# ------------------------------------------------------- whole-block moves --

def copy_blocks(pools: list, src, dst) -> None:
    """Copy-on-write at divergence ("KV cache, continuous batching and paged attention",
    section "Paged attention"): in every layer's pool, block dst[j] takes the K and V
    tiles of all heads and the scales of block src[j].  Pairs are applied in order."""
    for s, t in zip(np.asarray(src).tolist(), np.asarray(dst).tolist()):
        for p in pools:
            p.k[t] = p.k[s]
            p.v[t] = p.v[s]
            p.k_scale[t] = p.k_scale[s]
            p.v_scale[t] = p.v_scale[s]


def swap_image(pools: list, blocks) -> np.ndarray:
    """Host image of swapped-out blocks ("KV cache, GQA, paging and continuous batching",
    section "The scheduler, and preemption": a preempted sequence's blocks go to host
    memory).  One row of bytes per block: for each layer its K then V tiles of all heads,
    then (quantized pools) for each layer its K then V scales as fp32."""
    quant = pools[0].dtype in (INT8, INT4, FP8)
    rows = []
    for b in np.asarray(blocks).tolist():
        parts = []
        for p in pools:
            parts += [p.k[b].reshape(-1), p.v[b].reshape(-1)]
        if quant:
            for p in pools:
                parts += [p.k_scale[b].view(np.uint8), p.v_scale[b].view(np.uint8)]
        rows.append(np.concatenate(parts))
    width = sum(2 * p.k[0].size for p in pools) + (sum(2 * p.H_kv * 4 for p in pools) if quant else 0)
    return np.stack(rows) if rows else np.zeros((0, width), np.uint8)


def swap_restore(pools: list, blocks, image: np.ndarray) -> None:
    """Inverse of swap_image: block blocks[j] takes row j of the image, in place."""
    quant = pools[0].dtype in (INT8, INT4, FP8)
    for j, b in enumerate(np.asarray(blocks).tolist()):
        row, at = image[j], 0
        for p in pools:
            n = p.k[b].size
            p.k[b] = row[at:at + n].reshape(p.k[b].shape)
            p.v[b] = row[at + n:at + 2 * n].reshape(p.v[b].shape)
            at += 2 * n
        if quant:
            for p in pools:
                n = 4 * p.H_kv
                p.k_scale[b] = row[at:at + n].copy().view(np.float32)
                p.v_scale[b] = row[at + n:at + 2 * n].copy().view(np.float32)
                at += 2 * n
        assert at == row.size
