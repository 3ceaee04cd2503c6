"""Decode parity where the lazy running max of the read path works hardest.

The decode kernel keeps a running max m per query head that only moves when
a token's score (plus the exponent bound of its value scale) exceeds it by
a trigger margin, then jumps to the chunk's max plus a headroom; partial
sums run in an integer accumulator on the tensor cores, and a move switches
to a second accumulator whose predecessor is folded one chunk later.  These
tests build inputs whose scores rise steadily along the sequence, so that
(nearly) every chunk of 128 tokens moves the max, and a split longer than
a split of the longest kind.  Expected values come from the oracle's
plain softmax attention on the same packed bytes ("KVarN vs TurboQuant",
dothoosh.com: scale folding at read time).
"""
import numpy as np
import pytest

import helpers
import oracle
import synth

pytestmark = pytest.mark.gpu

from test_gpu_parity import _check_decode, _gpu_decode  # noqa: E402


def _fp16_bits(x):
    return np.asarray(x, dtype=np.float64).astype(np.float16).view(np.uint16)


def _rising_pool(wl, rise_per_chunk):
    """Oracle-written pool whose keys carry a ramp along the mean direction
    of their query heads: scores rise by about rise_per_chunk (base-2 units)
    per 128 tokens."""
    G = wl.hq // wl.hkv
    q = wl.query().view(np.float16).astype(np.float64)  # [B, Hq, 128]
    k = wl.kv_rows(synth.TID_K, 0, wl.total_tokens).view(np.float16).astype(np.float64)  # [T, Hkv, 128]
    v = wl.kv_rows(synth.TID_V, 0, wl.total_tokens)
    tau_log2e = (1.0 / np.sqrt(128.0)) * np.log2(np.e)
    for b in range(wl.batch):
        L = int(wl.seq_lens[b])
        off = int(wl.token_offsets[b])
        ramp = np.arange(L, dtype=np.float64) / 128.0  # chunks
        for h in range(wl.hkv):
            u = q[b, h * G:(h + 1) * G].mean(axis=0)
            uhat = u / np.linalg.norm(u)
            gain = float(np.mean(q[b, h * G:(h + 1) * G] @ uhat))  # score per unit of ramp amplitude
            amp = rise_per_chunk / (tau_log2e * gain)
            k[off:off + L, h] += np.outer(ramp * amp, uhat)
    k16 = _fp16_bits(k)
    g = oracle.geom(num_blocks=wl.num_blocks, num_kv_heads=wl.hkv)
    pool = oracle.new_pool(g)
    assert oracle.quantize_append(g, pool, k16, v, wl.dtype, wl.slots()) == 0
    return g, pool


@pytest.mark.parametrize("bps", [0, 2, 1000])
def test_decode_rising_scores_move_every_chunk(kvq, cuda, bps):
    wl = synth.Workload("rise", 2, 16, 2, 128, [2048, 1500], 16, synth.F16, 2, 4.0, 8.0, seed=91)
    g, pool = _rising_pool(wl, rise_per_chunk=6.0)
    q = wl.query()
    got, _ = _gpu_decode(kvq, wl, pool, q, wl.dtype, bps=bps)
    err = _check_decode(wl, g, pool, q, wl.dtype, got)
    assert kvq.kvq_last_device_status() == 0
    print(f"\nrising scores, blocks per split {bps}: max abs err {err:.2e}")


def test_decode_rising_scores_slowly(kvq, cuda):
    """A rise just above the trigger margin every other chunk."""
    wl = synth.Workload("rise2", 1, 8, 1, 128, [4000], 16, synth.F16, 2, 4.0, 8.0, seed=92)
    g, pool = _rising_pool(wl, rise_per_chunk=1.6)
    q = wl.query()
    got, _ = _gpu_decode(kvq, wl, pool, q, wl.dtype, bps=1000)
    _check_decode(wl, g, pool, q, wl.dtype, got)


def test_decode_single_split_of_the_longest_kind(kvq, cuda):
    """One split of 128 chunks (1024 blocks, the longest a CTA takes, less a
    ragged tail): the integer accumulators run the whole split without a
    restart and stay exact."""
    L = 128 * 128 - 37
    wl = synth.Workload("long1", 1, 8, 1, 128, [L], 16, synth.F16, 2, 4.0, 8.0, seed=93)
    g = oracle.geom(num_blocks=wl.num_blocks, num_kv_heads=wl.hkv)
    pool = oracle.new_pool(g)
    k = wl.kv_rows(synth.TID_K, 0, L)
    v = wl.kv_rows(synth.TID_V, 0, L)
    assert oracle.quantize_append(g, pool, k, v, wl.dtype, wl.slots()) == 0
    q = wl.query()
    got, _ = _gpu_decode(kvq, wl, pool, q, wl.dtype, bps=wl.max_blocks_per_seq)
    _check_decode(wl, g, pool, q, wl.dtype, got)
    assert helpers.ATTN_TOL == 2e-3
