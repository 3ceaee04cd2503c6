"""Python binding of libkvq.so, the B200 (sm_100a) quantized paged KV cache.

Argument marshalling only: every step of the write and read paths runs in the
library's CUDA kernels.  The names mirror include/kvq.h.  Torch is used for
device memory, dtypes and streams.  There is no fallback: if libkvq.so is
missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libkvq.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "kvq.h")

KVQ_OK = 0
KVQ_ERR_INVALID = -1
KVQ_ERR_UNSUPPORTED = -2
KVQ_ERR_CUDA = -3
KVQ_ERR_POOL_EXHAUSTED = -4
KVQ_ERR_OUT_OF_RANGE = -5
KVQ_ERR_DEVICE_TIMEOUT = -6
KVQ_ERR_WORKSPACE = -7

KVQ_F16, KVQ_BF16, KVQ_F32 = 0, 1, 2

HEAD_DIM = 128
BLOCK_SIZE = 16
SEGMENT_BYTES = 1664

_lock = threading.Lock()
_lib = None


class KvqError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {kvq_error_string(status)} ({status})")


class CacheDesc(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("k_bits", ctypes.c_int32), ("v_bits", ctypes.c_int32), ("group", ctypes.c_int32),
                ("pool", ctypes.c_void_p)]


class WindowDesc(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("num_seqs", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("sink", ctypes.c_int32), ("recent", ctypes.c_int32)]


def lib():
    """Load libkvq.so (raises if it is absent: there is no other path)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing; build it with python -m bit_kv_cache_18_b200.build")
            L = ctypes.CDLL(LIB_PATH)
            i32, i64, u64, sz, vp, f32 = (ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t,
                                          ctypes.c_void_p, ctypes.c_float)
            dp = ctypes.POINTER(CacheDesc)
            sig = {
                "kvq_parse_dtype": (ctypes.c_int, [ctypes.c_char_p, vp, vp, vp]),
                "kvq_cache_bytes": (sz, [dp]),
                "kvq_block_table": (ctypes.c_int, [i32, i32, vp, i32, i32, u64, vp, vp]),
                "kvq_slot_mapping": (ctypes.c_int, [vp, i32, vp, vp, i32, i32, vp]),
                "kvq_quantize_append": (ctypes.c_int, [dp, vp, vp, ctypes.c_int, i32, i64, vp, vp]),
                "kvq_decode_workspace_bytes": (sz, [dp, i32, i32, i32]),
                "kvq_decode_workspace_bytes_ex": (sz, [dp, i32, i32, i32, i32]),
                "kvq_decode_attention": (ctypes.c_int, [dp, vp, ctypes.c_int, i32, i32, vp, i32, vp, i32, f32, vp,
                                                        ctypes.c_int, vp, sz, vp]),
                "kvq_decode_attention_ex": (ctypes.c_int, [dp, vp, ctypes.c_int, i32, i32, vp, i32, vp, i32, f32,
                                                           vp, ctypes.c_int, vp, sz, i32, vp]),
                "kvq_decode_attention_noalloc": (ctypes.c_int, [dp, vp, ctypes.c_int, i32, i32, vp, i32, vp, i32, f32,
                                                                vp, ctypes.c_int, vp]),
                "kvq_append_decode_attention": (ctypes.c_int, [dp, vp, vp, ctypes.c_int, i64, vp, ctypes.c_int, i32,
                                                               i32, vp, i32, vp, i32, f32, vp, ctypes.c_int, vp, sz,
                                                               vp]),
                "kvq_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_uint32, vp, vp]),
                "kvq_window_bytes": (sz, [ctypes.POINTER(WindowDesc)]),
                "kvq_window_append": (ctypes.c_int, [ctypes.POINTER(WindowDesc), vp, vp, i64, vp, vp, i32, vp]),
                "kvq_decode_window_workspace_bytes": (sz, [dp, i32, i32, i32]),
                "kvq_decode_attention_window": (ctypes.c_int, [dp, ctypes.POINTER(WindowDesc), vp, ctypes.c_int, i32,
                                                               i32, vp, i32, vp, i32, f32, vp, ctypes.c_int, vp, sz,
                                                               vp]),
                "kvq_last_device_status": (ctypes.c_int, [vp]),
                "kvq_error_string": (ctypes.c_char_p, [ctypes.c_int]),
            }
            for name, (res, args) in sig.items():
                f = getattr(L, name)
                f.restype, f.argtypes = res, args
            _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/kvq.h declares."""
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z_]+)\s*\(", text)))


def kvq_error_string(status: int) -> str:
    return lib().kvq_error_string(status).decode()


def _check(rc: int, what: str):
    if rc != KVQ_OK:
        raise KvqError(rc, what)


def _stream_ptr(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t) -> int:
    import torch
    return {torch.float16: KVQ_F16, torch.bfloat16: KVQ_BF16, torch.float32: KVQ_F32}[t.dtype]


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


# ---- host-only helpers -------------------------------------------------------

def kvq_parse_dtype(s: str):
    kb, vb, g = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    rc = lib().kvq_parse_dtype(s.encode(), ctypes.byref(kb), ctypes.byref(vb), ctypes.byref(g))
    return rc, (kb.value, vb.value, g.value)


# The cache presets the library builds, as (key bits, value bits); the first
# is the pages' default, kvarn_k4v2_g128.
PRESETS = ((4, 2), (4, 4), (2, 2), (8, 4))


def make_desc(num_blocks: int, num_kv_heads: int, pool=None, preset=(4, 2)) -> CacheDesc:
    return CacheDesc(num_blocks, BLOCK_SIZE, num_kv_heads, HEAD_DIM, preset[0], preset[1], HEAD_DIM,
                     pool.data_ptr() if pool is not None else None)


def kvq_cache_bytes(desc: CacheDesc) -> int:
    return lib().kvq_cache_bytes(ctypes.byref(desc))


def kvq_block_table(num_blocks, seq_lens, max_blocks_per_seq, shuffle_seed=0, block_size=BLOCK_SIZE):
    """-> (block_table int32 numpy [batch, max_blocks_per_seq], blocks_used)"""
    import numpy as np
    lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    out = np.empty((lens.size, max_blocks_per_seq), dtype=np.int32)
    used = ctypes.c_int32()
    _check(lib().kvq_block_table(num_blocks, block_size, lens.ctypes.data, lens.size, max_blocks_per_seq,
                                 shuffle_seed, out.ctypes.data, ctypes.byref(used)), "kvq_block_table")
    return out, used.value


def kvq_slot_mapping(block_table, positions, seq_ids, block_size=BLOCK_SIZE):
    import numpy as np
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    pos = np.ascontiguousarray(positions, dtype=np.int32)
    sid = np.ascontiguousarray(seq_ids, dtype=np.int32)
    out = np.empty(pos.size, dtype=np.int32)
    _check(lib().kvq_slot_mapping(bt.ctypes.data, bt.shape[1], pos.ctypes.data, sid.ctypes.data, pos.size,
                                  block_size, out.ctypes.data), "kvq_slot_mapping")
    return out


# ---- device calls ------------------------------------------------------------

def new_pool(num_blocks: int, num_kv_heads: int, device="cuda", preset=(4, 2)):
    """A caller-owned pool tensor (uint8) sized by kvq_cache_bytes."""
    import torch
    nbytes = kvq_cache_bytes(make_desc(num_blocks, num_kv_heads, preset=preset))
    return torch.zeros(nbytes, dtype=torch.uint8, device=device)


def kvq_quantize_append(pool, num_blocks, num_kv_heads, k, v, slot_mapping, stream=None, token_stride=None,
                        preset=(4, 2)):
    """k, v: [n_tokens, ..., Hkv*128 elements per row] fp16/bf16 device tensors
    with stride(0) = token_stride; slot_mapping: int32 device [n_tokens]."""
    desc = make_desc(num_blocks, num_kv_heads, pool, preset)
    n = int(slot_mapping.numel())
    ts = k.stride(0) if token_stride is None else token_stride
    rc = lib().kvq_quantize_append(ctypes.byref(desc), _ptr(k), _ptr(v), _dtype_code(k), n, ts, _ptr(slot_mapping),
                                   _stream_ptr(stream))
    _check(rc, "kvq_quantize_append")


def kvq_decode_workspace_bytes(num_blocks, num_kv_heads, batch, num_q_heads, max_seq_len, blocks_per_split=0,
                               preset=(4, 2)):
    desc = make_desc(num_blocks, num_kv_heads, preset=preset)
    return lib().kvq_decode_workspace_bytes_ex(ctypes.byref(desc), batch, num_q_heads, max_seq_len,
                                               blocks_per_split)


def new_workspace(num_blocks, num_kv_heads, batch, num_q_heads, max_seq_len, blocks_per_split=0, device="cuda",
                  preset=(4, 2)):
    import torch
    n = kvq_decode_workspace_bytes(num_blocks, num_kv_heads, batch, num_q_heads, max_seq_len, blocks_per_split,
                                   preset)
    if n == 0:
        raise KvqError(KVQ_ERR_UNSUPPORTED, "kvq_decode_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def kvq_decode_attention(pool, num_blocks, num_kv_heads, q, block_table, seq_lens, max_seq_len, out, workspace,
                         softmax_scale=0.0, blocks_per_split=0, stream=None, preset=(4, 2)):
    """q: [batch, Hq, 128] device; block_table int32 [batch, max_blocks]; seq_lens int32 [batch];
    out: [batch, Hq, 128] device (fp32/bf16/fp16); workspace from new_workspace()."""
    desc = make_desc(num_blocks, num_kv_heads, pool, preset)
    batch, hq, _ = q.shape
    rc = lib().kvq_decode_attention_ex(ctypes.byref(desc), _ptr(q), _dtype_code(q), batch, hq, _ptr(block_table),
                                       block_table.shape[1], _ptr(seq_lens), max_seq_len, softmax_scale, _ptr(out),
                                       _dtype_code(out), _ptr(workspace), workspace.numel(), blocks_per_split,
                                       _stream_ptr(stream))
    _check(rc, "kvq_decode_attention")


def kvq_append_decode_attention(pool, num_blocks, num_kv_heads, k_new, v_new, q, block_table, seq_lens, max_seq_len,
                                out, workspace, softmax_scale=0.0, stream=None, token_stride=None, preset=(4, 2)):
    """One fused decode step: the new token of each sequence (k_new, v_new:
    [batch, ..., Hkv*128] fp16/bf16 rows) is quantized into position
    seq_lens[b] - 1, then decode attention runs over the grown cache."""
    desc = make_desc(num_blocks, num_kv_heads, pool, preset)
    batch, hq, _ = q.shape
    ts = k_new.stride(0) if token_stride is None else token_stride
    rc = lib().kvq_append_decode_attention(ctypes.byref(desc), _ptr(k_new), _ptr(v_new), _dtype_code(k_new), ts,
                                           _ptr(q), _dtype_code(q), batch, hq, _ptr(block_table),
                                           block_table.shape[1], _ptr(seq_lens), max_seq_len, softmax_scale,
                                           _ptr(out), _dtype_code(out), _ptr(workspace), workspace.numel(),
                                           _stream_ptr(stream))
    _check(rc, "kvq_append_decode_attention")


def kvq_decode_attention_noalloc(pool, num_blocks, num_kv_heads, q, block_table, seq_lens, max_seq_len, out,
                                 softmax_scale=0.0, stream=None, preset=(4, 2)):
    """kvq_decode_attention with the library's fixed device scratch instead of
    a caller workspace (for callers that cannot allocate at call time)."""
    desc = make_desc(num_blocks, num_kv_heads, pool, preset)
    batch, hq, _ = q.shape
    rc = lib().kvq_decode_attention_noalloc(ctypes.byref(desc), _ptr(q), _dtype_code(q), batch, hq,
                                            _ptr(block_table), block_table.shape[1], _ptr(seq_lens), max_seq_len,
                                            softmax_scale, _ptr(out), _dtype_code(out), _stream_ptr(stream))
    _check(rc, "kvq_decode_attention_noalloc")


# ---- bf16 window of sink and recent tokens -------------------------------------

def make_window(num_seqs, num_kv_heads, sink, recent, data=None) -> WindowDesc:
    return WindowDesc(data.data_ptr() if data is not None else None, num_seqs, num_kv_heads, sink, recent)


def kvq_window_bytes(num_seqs, num_kv_heads, sink, recent) -> int:
    return lib().kvq_window_bytes(ctypes.byref(make_window(num_seqs, num_kv_heads, sink, recent)))


def new_window(num_seqs, num_kv_heads, sink, recent, device="cuda"):
    """A zeroed window buffer: bf16 [num_seqs, Hkv, sink + recent, 2, 128]."""
    import torch
    if kvq_window_bytes(num_seqs, num_kv_heads, sink, recent) == 0 and num_seqs * (sink + recent) > 0:
        raise KvqError(KVQ_ERR_INVALID, "kvq_window_bytes")
    return torch.zeros((num_seqs, num_kv_heads, sink + recent, 2, HEAD_DIM), dtype=torch.bfloat16, device=device)


def kvq_window_append(window, sink, recent, k, v, seq_ids, positions, stream=None, token_stride=None):
    """k, v: [n, ..., Hkv*128] bf16 rows; seq_ids, positions: int32 [n] device."""
    num_seqs, hkv = window.shape[0], window.shape[1]
    w = make_window(num_seqs, hkv, sink, recent, window)
    ts = k.stride(0) if token_stride is None else token_stride
    rc = lib().kvq_window_append(ctypes.byref(w), _ptr(k), _ptr(v), ts, _ptr(seq_ids), _ptr(positions),
                                 seq_ids.numel(), _stream_ptr(stream))
    _check(rc, "kvq_window_append")


def new_window_workspace(num_blocks, num_kv_heads, batch, num_q_heads, max_seq_len, device="cuda", preset=(4, 2)):
    import torch
    desc = make_desc(num_blocks, num_kv_heads, preset=preset)
    n = lib().kvq_decode_window_workspace_bytes(ctypes.byref(desc), batch, num_q_heads, max_seq_len)
    if n == 0:
        raise KvqError(KVQ_ERR_UNSUPPORTED, "kvq_decode_window_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def kvq_decode_attention_window(pool, num_blocks, num_kv_heads, window, sink, recent, q, block_table, seq_lens,
                                max_seq_len, out, workspace, softmax_scale=0.0, stream=None, preset=(4, 2)):
    """kvq_decode_attention with the window's raw rows at the sink and recent
    positions; workspace from new_window_workspace()."""
    desc = make_desc(num_blocks, num_kv_heads, pool, preset)
    w = make_window(window.shape[0], window.shape[1], sink, recent, window)
    batch, hq, _ = q.shape
    rc = lib().kvq_decode_attention_window(ctypes.byref(desc), ctypes.byref(w), _ptr(q), _dtype_code(q), batch, hq,
                                           _ptr(block_table), block_table.shape[1], _ptr(seq_lens), max_seq_len,
                                           softmax_scale, _ptr(out), _dtype_code(out), _ptr(workspace),
                                           workspace.numel(), _stream_ptr(stream))
    _check(rc, "kvq_decode_attention_window")


def kvq_selftest_wait_timeout(limit_us: int, elapsed_ns=None, stream=None):
    """Launch the bounded-wait self-test (a wait that must give up after
    limit_us microseconds); elapsed_ns: optional int64 device tensor of one
    element."""
    rc = lib().kvq_selftest_wait_timeout(limit_us, _ptr(elapsed_ns), _stream_ptr(stream))
    _check(rc, "kvq_selftest_wait_timeout")


def kvq_last_device_status(stream=None) -> int:
    return lib().kvq_last_device_status(_stream_ptr(stream))
