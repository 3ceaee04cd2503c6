"""Seeded synthetic inputs shared by the CPU oracle and the CUDA library.

This package holds no arithmetic of the quantisation method; it only makes
input bits.  Every value is a pure function of (seed, tensor id, index), so a
sample of a large workload can be regenerated without generating the rest.

The workload recipes (shapes, outlier channels, ragged lengths, shuffled
block tables) follow the synthetic configurations of the KV-cache build:
K/V ~ N(0,1) with a few fixed per-head outlier channels scaled up, queries
~ N(0,1).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_synth.c")
_LIB = os.path.join(_HERE, "libkvq_synth.so")
_lock = threading.Lock()
_lib = None

F16, BF16, F32, F64 = 0, 1, 2, 3

# tensor ids of the streams used by the workloads
TID_K, TID_V, TID_Q, TID_LENS, TID_PERM, TID_NEWK, TID_NEWV = 1, 2, 3, 4, 5, 6, 7


def build(force: bool = False) -> str:
    """Compile libkvq_synth.so next to its source (gcc, a second or two)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            i64, u64, i32, dbl, vp = ctypes.c_int64, ctypes.c_uint64, ctypes.c_int32, ctypes.c_double, ctypes.c_void_p
            lib.synth_normal.argtypes = [u64, u64, i64, i64, ctypes.c_int, vp]
            lib.synth_outliers.argtypes = [u64, u64, i32, i32, i32, dbl, dbl, vp, vp]
            lib.synth_kv.argtypes = [u64, u64, i64, i64, i32, i32, i32, dbl, dbl, ctypes.c_int, vp]
            lib.synth_uniform_int.argtypes = [u64, u64, i64, i32, i32, vp]
            lib.synth_permutation.argtypes = [u64, u64, i64, vp]
            for f in (lib.synth_normal, lib.synth_outliers, lib.synth_kv, lib.synth_uniform_int, lib.synth_permutation):
                f.restype = None
            _lib = lib
    return _lib


def _np_dtype(dtype: int):
    return {F16: np.uint16, BF16: np.uint16, F32: np.float32, F64: np.float64}[dtype]


def normal(seed: int, tensor_id: int, n: int, dtype: int = F64, offset: int = 0) -> np.ndarray:
    lib = _load()
    out = np.empty(n, dtype=_np_dtype(dtype))
    lib.synth_normal(seed, tensor_id, offset, n, dtype, out.ctypes.data)
    return out


def outliers(seed: int, tensor_id: int, num_heads: int, d: int, n_out: int, fmin: float, fmax: float):
    lib = _load()
    ch = np.zeros((num_heads, max(n_out, 1)), dtype=np.int32)
    fa = np.zeros((num_heads, max(n_out, 1)), dtype=np.float64)
    if n_out:
        lib.synth_outliers(seed, tensor_id, num_heads, d, n_out, fmin, fmax, ch.ctypes.data, fa.ctypes.data)
    return ch[:, :n_out], fa[:, :n_out]


def kv(seed: int, tensor_id: int, t0: int, n_tokens: int, num_heads: int, d: int, n_out: int,
       fmin: float, fmax: float, dtype: int = BF16, threads: int | None = None) -> np.ndarray:
    """Rows [t0, t0+n_tokens) of a [T, Hkv, d] K or V tensor (raw bits for f16/bf16)."""
    lib = _load()
    out = np.empty((n_tokens, num_heads, d), dtype=_np_dtype(dtype))
    if n_tokens == 0:
        return out
    threads = threads or min(32, os.cpu_count() or 1)
    chunk = max(1, -(-n_tokens // (threads * 4)))
    row_bytes = num_heads * d * out.itemsize

    def work(s):
        n = min(chunk, n_tokens - s)
        lib.synth_kv(seed, tensor_id, t0 + s, n, num_heads, d, n_out, fmin, fmax, dtype,
                     out.ctypes.data + s * row_bytes)

    if n_tokens <= chunk or threads <= 1:
        for s in range(0, n_tokens, chunk):
            work(s)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(work, range(0, n_tokens, chunk)))
    return out


def uniform_int(seed: int, tensor_id: int, n: int, lo: int, hi: int) -> np.ndarray:
    lib = _load()
    out = np.empty(n, dtype=np.int32)
    lib.synth_uniform_int(seed, tensor_id, n, lo, hi, out.ctypes.data)
    return out


def permutation(seed: int, tensor_id: int, n: int) -> np.ndarray:
    lib = _load()
    out = np.empty(n, dtype=np.int32)
    lib.synth_permutation(seed, tensor_id, n, out.ctypes.data)
    return out


# --------------------------------------------------------------------------
# Workload recipes.  Each returns plain numpy arrays (raw bf16/f16 bits as
# uint16) plus the geometry; nothing here depends on the CUDA library.

class Workload:
    """A decode workload: cached K/V, per-sequence lengths, block table, query."""

    def __init__(self, name, batch, num_q_heads, num_kv_heads, head_dim, seq_lens, block_size,
                 dtype, n_out, fmin, fmax, seed, shuffle=True, extra_blocks=0):
        self.name = name
        self.batch = batch
        self.hq = num_q_heads
        self.hkv = num_kv_heads
        self.d = head_dim
        self.seq_lens = np.asarray(seq_lens, dtype=np.int32)
        self.bs = block_size
        self.dtype = dtype
        self.n_out, self.fmin, self.fmax = n_out, fmin, fmax
        self.seed = seed
        nblk = (self.seq_lens + block_size - 1) // block_size
        self.max_blocks_per_seq = int(max(1, nblk.max() if len(nblk) else 1))
        self.num_blocks = int(nblk.sum()) + extra_blocks
        # physical blocks: a seeded shuffle of the pool (identity when shuffle=False)
        order = permutation(seed, TID_PERM, self.num_blocks) if shuffle else np.arange(self.num_blocks, dtype=np.int32)
        bt = np.full((batch, self.max_blocks_per_seq), -1, dtype=np.int32)
        pos = 0
        for b in range(batch):
            bt[b, : nblk[b]] = order[pos: pos + nblk[b]]
            pos += nblk[b]
        self.block_table = bt
        # token offsets of each sequence inside the flat [sum L, Hkv, d] K/V stream
        self.token_offsets = np.concatenate([[0], np.cumsum(self.seq_lens)[:-1]]).astype(np.int64)

    @property
    def total_tokens(self) -> int:
        return int(self.seq_lens.sum())

    def kv_rows(self, which: int, t0: int, n: int) -> np.ndarray:
        """Rows [t0, t0+n) of the flat K (which=TID_K) or V (TID_V) stream."""
        return kv(self.seed, which, t0, n, self.hkv, self.d, self.n_out, self.fmin, self.fmax, self.dtype)

    def slots(self) -> np.ndarray:
        """Slot of every token of the flat stream: block_table[b][t // bs] * bs + t % bs."""
        out = np.empty(self.total_tokens, dtype=np.int32)
        for b in range(self.batch):
            L = int(self.seq_lens[b])
            t = np.arange(L)
            out[self.token_offsets[b]: self.token_offsets[b] + L] = self.block_table[b, t // self.bs] * self.bs + t % self.bs
        return out

    def query(self, dtype: int | None = None) -> np.ndarray:
        dt = self.dtype if dtype is None else dtype
        return normal(self.seed, TID_Q, self.batch * self.hq * self.d, dt).reshape(self.batch, self.hq, self.d)


def tiny(seed: int = 0) -> Workload:
    """1 sequence, 1 query head, 1 kv head, d=128, 256 tokens, blocks of 16;
    fp16 K/V ~ N(0,1) with 4 fixed outlier channels x20; identity block table."""
    return Workload("tiny", 1, 1, 1, 128, [256], 16, F16, 4, 20.0, 20.0, seed, shuffle=False)


def qwen3_32b_layer(seed: int = 0, context: int = 16384) -> Workload:
    """Batch 1, 64 query / 8 kv heads, d=128, 16K context, blocks of 16, bf16
    K/V ~ N(0,1) with 3 of 128 channels (about 2%) scaled x10..x30, shuffled pool."""
    return Workload("qwen3-32b-layer", 1, 64, 8, 128, [context], 16, BF16, 3, 10.0, 30.0, seed)


def batched(seed: int = 0, batch: int = 32, lo: int = 4096, hi: int = 16384) -> Workload:
    """Batch 32, 64/8 heads, ragged lengths uniform in [4096, 16384]."""
    lens = uniform_int(seed, TID_LENS, batch, lo, hi)
    return Workload("batched-ragged", batch, 64, 8, 128, lens, 16, BF16, 3, 10.0, 30.0, seed)


def long_context(seed: int = 0, batch: int = 8, context: int = 131072) -> Workload:
    """Llama-3.1-70B-shaped: batch 8, 64/8 heads, 128K context per sequence."""
    return Workload("llama-70b-long", batch, 64, 8, 128, [context] * batch, 16, BF16, 3, 10.0, 30.0, seed)


def mixed_decode(seed: int = 0, batch: int = 64, context: int = 8192) -> Workload:
    """64 sequences of 8192 cached tokens, 8 kv heads (query heads 64)."""
    return Workload("mixed-decode", batch, 64, 8, 128, [context] * batch, 16, BF16, 3, 10.0, 30.0, seed,
                    extra_blocks=batch)
