"""Parity checking used by the GPU tests.

The rules for comparing a quantized pool written by the CUDA kernel with the
oracle's (the two compute in different precisions, so exact agreement is
required only away from rounding boundaries):
  - codes must be bit-exact, except at near-ties: an element whose oracle
    quotient (r_i - Z)/S lies within 1e-3 of k + 1/2 may differ by one code;
    such mismatches may make up at most 1e-4 of all elements;
  - S and Z must be bit-exact, except in a group whose exact (unrounded)
    value lies within 1e-3 of an fp16 ulp from a rounding midpoint, where
    they may differ by one ulp; the codes of such a group are then checked
    against the codes the oracle computes from the GPU's S and Z.
"""
from __future__ import annotations

import numpy as np

import oracle

NEAR_TIE = 1e-3
MAX_MISMATCH_FRACTION = 1e-4
ATTN_TOL = 2e-3


def to_f64(bits: np.ndarray, dtype: int) -> np.ndarray:
    if dtype == oracle.F16:
        return bits.view(np.float16).astype(np.float64)
    if dtype == oracle.BF16:
        return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return bits.astype(np.float64)


def _near_midpoint(exact: float, a: int, b: int) -> bool:
    va, vb = oracle.f16_to_f64(a), oracle.f16_to_f64(b)
    ulp = abs(va - vb)
    return abs(int(a) - int(b)) == 1 and abs(exact - (va + vb) / 2) <= NEAR_TIE * ulp


class QuantReport:
    def __init__(self):
        self.vectors = 0
        self.elements = 0
        self.code_mismatches = 0
        self.meta_mismatch_groups = 0
        self.failures: list[str] = []

    def ok(self) -> bool:
        return not self.failures and self.code_mismatches <= MAX_MISMATCH_FRACTION * max(self.elements, 1)

    def __repr__(self):
        return (f"QuantReport(vectors={self.vectors}, code_mismatches={self.code_mismatches}/{self.elements}, "
                f"meta_1ulp_groups={self.meta_mismatch_groups}, failures={self.failures[:5]})")


def check_vector(rep: QuantReport, x: np.ndarray, bits: int, gpu_codes, gpu_S: int, gpu_Z: int, where: str):
    """One group: GPU codes/metadata against the oracle under the rules above."""
    codes, S, Z, r = oracle.quantize_vector(x, bits)
    rep.vectors += 1
    rep.elements += codes.size
    if (gpu_S, gpu_Z) != (S, Z):
        s_ex, z_ex = oracle.meta_exact(x, bits)
        for name, ex, a, b in (("S", s_ex, gpu_S, S), ("Z", z_ex, gpu_Z, Z)):
            if a != b and not _near_midpoint(ex, a, b):
                rep.failures.append(f"{where}: {name} gpu={a:#06x} oracle={b:#06x} exact={ex!r}")
                return
        rep.meta_mismatch_groups += 1
        S, Z = gpu_S, gpu_Z
        codes = oracle.codes_given_meta(r, bits, S, Z)
    diff = np.asarray(gpu_codes, dtype=np.int64) - codes.astype(np.int64)
    bad = np.nonzero(diff)[0]
    if bad.size:
        q = oracle.quotients(r, S, Z)
        frac = np.abs(q[bad] - np.floor(q[bad]) - 0.5)
        if np.any(np.abs(diff[bad]) > 1) or np.any(frac > NEAR_TIE):
            rep.failures.append(f"{where}: codes differ away from ties at {bad[:8].tolist()}")
        rep.code_mismatches += int(bad.size)


def check_pool_tokens(rep: QuantReport, gpu_pool: np.ndarray, num_blocks: int, hkv: int, k_rows, v_rows,
                      in_dtype: int, slots, tokens, heads=None, preset=(4, 2)):
    """Check (token, head) groups: k_rows/v_rows hold [n, Hkv, 128] raw input rows;
    preset = (key bits, value bits) of the pool."""
    g = oracle.geom(num_blocks=num_blocks, num_kv_heads=hkv, k_bits=preset[0], v_bits=preset[1])
    heads = range(hkv) if heads is None else heads
    for t in tokens:
        s = int(slots[t])
        if s < 0:
            continue
        p, o = divmod(s, 16)
        for h in heads:
            kc, Sk, Zk, vc, Sv, Zv = oracle.unpack_token(g, gpu_pool, p, o, h)
            check_vector(rep, to_f64(k_rows[t, h], in_dtype), preset[0], kc, Sk, Zk, f"t{t} h{h} K")
            check_vector(rep, to_f64(v_rows[t, h], in_dtype), preset[1], vc, Sv, Zv, f"t{t} h{h} V")


# ---------------------------------------------------------------- full sizes

def threads() -> int:
    import os
    return max(1, min(64, os.cpu_count() or 1))


def oracle_append_threaded(g, pool: np.ndarray, k, v, in_dtype: int, slots, nthreads: int | None = None):
    """oracle.quantize_append over token ranges on several threads (the
    calls write disjoint slots of the same pool; ctypes releases the GIL)."""
    from concurrent.futures import ThreadPoolExecutor
    n = int(slots.size)
    nt = nthreads or threads()
    step = max(1024, -(-n // (4 * nt)))

    def work(t0):
        t1 = min(n, t0 + step)
        rc = oracle.quantize_append(g, pool, np.ascontiguousarray(k[t0:t1]), np.ascontiguousarray(v[t0:t1]),
                                    in_dtype, np.ascontiguousarray(slots[t0:t1]))
        assert rc == 0, rc

    with ThreadPoolExecutor(nt) as ex:
        list(ex.map(work, range(0, n, step)))


def _token_bytes(pool: np.ndarray, num_blocks: int, hkv: int, slots, preset):
    """[n, hkv, bytes of one token-head] gathered from a pool: K row, V row
    and the four fp16 factors of each (token, head)."""
    kb, vb = preset
    kr, vr = 16 * kb, 16 * vb
    seg = 16 * (kr + vr) + 128
    offk = 16 * kr
    p = (slots // 16).astype(np.int64)
    o = (slots % 16).astype(np.int64)
    cols = [o[:, None] * kr + np.arange(kr)[None, :], offk + o[:, None] * vr + np.arange(vr)[None, :]]
    for f in range(4):  # S_K, Z_K, S_V, Z_V
        base = 16 * (kr + vr) + 32 * f
        cols.append(base + 2 * o[:, None] + np.arange(2)[None, :])
    cols = np.concatenate(cols, axis=1)                             # [n, bytes]
    flat = pool.reshape(num_blocks, hkv, seg)
    return flat[p[:, None, None], np.arange(hkv)[None, :, None], cols[:, None, :]]


def compare_pools(rep: QuantReport, gpu_pool: np.ndarray, oracle_pool: np.ndarray, num_blocks: int, hkv: int,
                  k_rows, v_rows, in_dtype: int, slots, tokens=None, preset=(4, 2), chunk=65536):
    """Every (token, head) group of `tokens` (default: all with a slot): the
    GPU-written bytes against the oracle-written ones; groups whose bytes
    differ go through check_vector (near-tie and midpoint rules)."""
    slots = np.asarray(slots)
    tokens = np.arange(slots.size) if tokens is None else np.asarray(tokens)
    tokens = tokens[slots[tokens] >= 0]
    per = 2 * 128 + 0  # elements per token-head (K and V)
    for c0 in range(0, tokens.size, chunk):
        tk = tokens[c0:c0 + chunk]
        a = _token_bytes(gpu_pool, num_blocks, hkv, slots[tk], preset)
        b = _token_bytes(oracle_pool, num_blocks, hkv, slots[tk], preset)
        diff = np.any(a != b, axis=2)
        rep.vectors += 2 * diff.size
        rep.elements += per * diff.size
        for ti, h in zip(*np.nonzero(diff)):
            t = int(tk[ti])
            sub = QuantReport()
            check_pool_tokens(sub, gpu_pool, num_blocks, hkv, k_rows, v_rows, in_dtype, slots, [t], heads=[int(h)],
                              preset=preset)
            rep.code_mismatches += sub.code_mismatches
            rep.meta_mismatch_groups += sub.meta_mismatch_groups
            rep.failures += sub.failures
