"""ctypes front end of the CPU oracle (kvq_oracle.cpp).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline may use this package; the library under bit_kv_cache_18_b200/ never
imports, links or calls it, and it never calls the library.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.cpp")
_HDR = os.path.join(_HERE, "kvq_oracle.h")
_LIB = os.path.join(_HERE, "libkvq_oracle.so")
_lock = threading.Lock()
_lib = None

F16, BF16, F32 = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile libkvq_oracle.so next to its source with g++ (plain -O2)."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-std=c++17", "-O2", "-fPIC", "-shared", _SRC, "-o", tmp, "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


class Geom(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("k_bits", ctypes.c_int32), ("v_bits", ctypes.c_int32)]


def geom(num_blocks, num_kv_heads, block_size=16, head_dim=128, k_bits=4, v_bits=2) -> Geom:
    return Geom(num_blocks, block_size, num_kv_heads, head_dim, k_bits, v_bits)


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            i32, i64, u16, dbl, vp, sz = (ctypes.c_int32, ctypes.c_int64, ctypes.c_uint16, ctypes.c_double,
                                          ctypes.c_void_p, ctypes.c_size_t)
            gp = ctypes.POINTER(Geom)
            sig = {
                "kvqo_f64_to_f16": (u16, [dbl]),
                "kvqo_f16_to_f64": (dbl, [u16]),
                "kvqo_bf16_to_f64": (dbl, [u16]),
                "kvqo_hadamard": (ctypes.c_int, [i32, vp]),
                "kvqo_rotate": (ctypes.c_int, [i32, vp, vp]),
                "kvqo_quantize_vector": (ctypes.c_int, [i32, vp, i32, i32, vp, vp, vp, vp]),
                "kvqo_codes_given_meta": (ctypes.c_int, [i32, vp, i32, u16, u16, vp]),
                "kvqo_quotients": (ctypes.c_int, [i32, vp, u16, u16, vp]),
                "kvqo_meta_exact": (ctypes.c_int, [i32, vp, i32, i32, vp, vp]),
                "kvqo_dequantize_vector": (ctypes.c_int, [i32, vp, u16, u16, vp, vp]),
                "kvqo_segment_bytes": (sz, [gp]),
                "kvqo_pool_bytes": (sz, [gp]),
                "kvqo_pack_token": (ctypes.c_int, [gp, vp, i32, i32, i32, vp, u16, u16, vp, u16, u16]),
                "kvqo_unpack_token": (ctypes.c_int, [gp, vp, i32, i32, i32, vp, vp, vp, vp, vp, vp]),
                "kvqo_quantize_append": (ctypes.c_int, [gp, vp, vp, vp, i32, i32, i64, vp, i32]),
                "kvqo_decode_one": (ctypes.c_int, [gp, vp, vp, i32, i32, i32, vp, i32, dbl, i32, vp]),
                "kvqo_decode_attention": (ctypes.c_int, [gp, vp, vp, i32, i32, i32, vp, i32, vp, dbl, i32, i32, vp]),
                "kvqo_attention_dense": (ctypes.c_int, [i32, i32, vp, vp, i32, i64, i32, vp, i32, i32, i32, dbl, vp]),
                "kvqo_window_append": (ctypes.c_int, [i32, i32, i32, i32, i32, vp, vp, vp, i64, vp, vp, i32]),
                "kvqo_decode_attention_window": (ctypes.c_int, [gp, vp, vp, i32, i32, vp, i32, i32, i32, vp, i32, vp,
                                                                dbl, i32, vp]),
                "kvqo_packed_bytes_per_token_head": (dbl, [i32, i32, i32]),
                "kvqo_dense_bytes_per_token": (dbl, [i32, i32, i32, i32]),
            }
            for name, (res, args) in sig.items():
                f = getattr(L, name)
                f.restype, f.argtypes = res, args
            _lib = L
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what} returned {rc}")


# ---- thin wrappers ---------------------------------------------------------

def f64_to_f16(x: float) -> int:
    return lib().kvqo_f64_to_f16(float(x))


def f16_to_f64(h: int) -> float:
    return lib().kvqo_f16_to_f64(int(h))


def bf16_to_f64(b: int) -> float:
    return lib().kvqo_bf16_to_f64(int(b))


def hadamard(d: int) -> np.ndarray:
    H = np.zeros((d, d), dtype=np.int8)
    _check(lib().kvqo_hadamard(d, _p(H)), "hadamard")
    return H


def rotate(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    r = np.zeros_like(x)
    _check(lib().kvqo_rotate(x.size, _p(x), _p(r)), "rotate")
    return r


def quantize_vector(x: np.ndarray, bits: int, normalize: bool = True):
    """-> (codes uint8[d], S fp16 bits, Z fp16 bits, r float64[d])"""
    x = np.ascontiguousarray(x, dtype=np.float64)
    d = x.size
    codes = np.zeros(d, dtype=np.uint8)
    S = ctypes.c_uint16()
    Z = ctypes.c_uint16()
    r = np.zeros(d, dtype=np.float64)
    _check(lib().kvqo_quantize_vector(d, _p(x), bits, int(normalize), _p(codes), ctypes.byref(S),
                                      ctypes.byref(Z), _p(r)), "quantize_vector")
    return codes, S.value, Z.value, r


def codes_given_meta(r: np.ndarray, bits: int, S: int, Z: int) -> np.ndarray:
    r = np.ascontiguousarray(r, dtype=np.float64)
    codes = np.zeros(r.size, dtype=np.uint8)
    _check(lib().kvqo_codes_given_meta(r.size, _p(r), bits, S, Z, _p(codes)), "codes_given_meta")
    return codes


def quotients(r: np.ndarray, S: int, Z: int) -> np.ndarray:
    r = np.ascontiguousarray(r, dtype=np.float64)
    q = np.zeros(r.size, dtype=np.float64)
    _check(lib().kvqo_quotients(r.size, _p(r), S, Z, _p(q)), "quotients")
    return q


def meta_exact(x: np.ndarray, bits: int, normalize: bool = True):
    x = np.ascontiguousarray(x, dtype=np.float64)
    s = ctypes.c_double()
    z = ctypes.c_double()
    _check(lib().kvqo_meta_exact(x.size, _p(x), bits, int(normalize), ctypes.byref(s), ctypes.byref(z)),
           "meta_exact")
    return s.value, z.value


def dequantize_vector(codes: np.ndarray, S: int, Z: int):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    xh = np.zeros(codes.size, dtype=np.float64)
    rh = np.zeros(codes.size, dtype=np.float64)
    _check(lib().kvqo_dequantize_vector(codes.size, _p(codes), S, Z, _p(xh), _p(rh)), "dequantize_vector")
    return xh, rh


def segment_bytes(g: Geom) -> int:
    return lib().kvqo_segment_bytes(ctypes.byref(g))


def pool_bytes(g: Geom) -> int:
    return lib().kvqo_pool_bytes(ctypes.byref(g))


def new_pool(g: Geom, fill: int = 0) -> np.ndarray:
    return np.full(pool_bytes(g), fill, dtype=np.uint8)


def pack_token(g, pool, p, o, h, kc, Sk, Zk, vc, Sv, Zv) -> int:
    kc = np.ascontiguousarray(kc, dtype=np.uint8)
    vc = np.ascontiguousarray(vc, dtype=np.uint8)
    return lib().kvqo_pack_token(ctypes.byref(g), _p(pool), p, o, h, _p(kc), Sk, Zk, _p(vc), Sv, Zv)


def unpack_token(g, pool, p, o, h):
    d = g.head_dim
    kc = np.zeros(d, dtype=np.uint8)
    vc = np.zeros(d, dtype=np.uint8)
    m = [ctypes.c_uint16() for _ in range(4)]
    _check(lib().kvqo_unpack_token(ctypes.byref(g), _p(pool), p, o, h, _p(kc), ctypes.byref(m[0]),
                                   ctypes.byref(m[1]), _p(vc), ctypes.byref(m[2]), ctypes.byref(m[3])),
           "unpack_token")
    return kc, m[0].value, m[1].value, vc, m[2].value, m[3].value


def quantize_append(g, pool, k, v, in_dtype, slots, token_stride=None, normalize=True) -> int:
    """k, v: arrays [n_tokens, ...] (raw uint16 bits for f16/bf16, float32 for F32)."""
    n = int(slots.size)
    row = g.num_kv_heads * g.head_dim
    ts = row if token_stride is None else token_stride
    slots = np.ascontiguousarray(slots, dtype=np.int32)
    return lib().kvqo_quantize_append(ctypes.byref(g), _p(pool), _p(k), _p(v), in_dtype, n, ts, _p(slots),
                                      int(normalize))


def decode_one(g, pool, q_row, q_dtype, num_q_heads, j, bt_row, seq_len, scale=0.0, form=0) -> np.ndarray:
    out = np.zeros(g.head_dim, dtype=np.float64)
    bt_row = np.ascontiguousarray(bt_row, dtype=np.int32)
    q_row = np.ascontiguousarray(q_row)
    _check(lib().kvqo_decode_one(ctypes.byref(g), _p(pool), _p(q_row), q_dtype, num_q_heads, j, _p(bt_row),
                                 seq_len, scale, form, _p(out)), "decode_one")
    return out


def decode_attention(g, pool, q, q_dtype, block_table, seq_lens, scale=0.0, form=0, nthreads=1) -> np.ndarray:
    q = np.ascontiguousarray(q)
    batch, hq, d = q.shape
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    out = np.zeros((batch, hq, d), dtype=np.float64)
    _check(lib().kvqo_decode_attention(ctypes.byref(g), _p(pool), _p(q), q_dtype, batch, hq, _p(bt), bt.shape[1],
                                       _p(lens), scale, form, nthreads, _p(out)), "decode_attention")
    return out


def new_window(num_seqs, num_kv_heads, sink, recent, d=128, fill=0) -> np.ndarray:
    """A window buffer of bf16 bits [num_seqs, Hkv, sink + recent, 2, d]."""
    return np.full((num_seqs, num_kv_heads, sink + recent, 2, d), fill, dtype=np.uint16)


def window_append(win, sink, recent, k, v, seq_ids, positions, token_stride=None) -> None:
    """k, v: bf16 bits [n, Hkv, d] (rows as in the write path); sequence
    seq_ids[n] (negative: skipped), position positions[n]."""
    num_seqs, hkv, rows, _, d = win.shape
    assert rows == sink + recent
    n = len(seq_ids)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = np.ascontiguousarray(v, dtype=np.uint16)
    ts = hkv * d if token_stride is None else token_stride
    ids = np.ascontiguousarray(seq_ids, dtype=np.int32)
    pos = np.ascontiguousarray(positions, dtype=np.int32)
    _check(lib().kvqo_window_append(d, hkv, sink, recent, num_seqs, _p(win), _p(k), _p(v), ts, _p(ids), _p(pos), n),
           "window_append")


def decode_attention_window(g, pool, win, sink, recent, q, q_dtype, block_table, seq_lens, scale=0.0,
                            nthreads=1) -> np.ndarray:
    q = np.ascontiguousarray(q)
    batch, hq, d = q.shape
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    out = np.zeros((batch, hq, d), dtype=np.float64)
    w = np.ascontiguousarray(win, dtype=np.uint16)
    _check(lib().kvqo_decode_attention_window(ctypes.byref(g), _p(pool), _p(w), sink, recent, _p(q), q_dtype, batch,
                                              hq, _p(bt), bt.shape[1], _p(lens), scale, nthreads, _p(out)),
           "decode_attention_window")
    return out


def attention_dense(k, v, kv_dtype, q_row, q_dtype, num_q_heads, j, scale=0.0, token_stride=None) -> np.ndarray:
    """k, v: [L, Hkv, d] raw rows."""
    L, hkv, d = k.shape
    ts = hkv * d if token_stride is None else token_stride
    out = np.zeros(d, dtype=np.float64)
    q_row = np.ascontiguousarray(q_row)
    _check(lib().kvqo_attention_dense(d, hkv, _p(np.ascontiguousarray(k)), _p(np.ascontiguousarray(v)), kv_dtype,
                                      ts, L, _p(q_row), q_dtype, num_q_heads, j, scale, _p(out)), "attention_dense")
    return out


def packed_bytes_per_token_head(d=128, k_bits=4, v_bits=2) -> float:
    return lib().kvqo_packed_bytes_per_token_head(d, k_bits, v_bits)


def dense_bytes_per_token(layers, num_kv_heads, d, bytes_per_elem) -> float:
    return lib().kvqo_dense_bytes_per_token(layers, num_kv_heads, d, bytes_per_elem)
