"""GPU parity of the other cache presets (k4v4, k2v2, k8v4: the same write
and read paths at other bit widths) against the CPU oracle on the same seeded
inputs, with the rules of test_gpu_parity.py: codes bit-exact except at
near-ties, S and Z bit-exact except at fp16 rounding midpoints, decode
outputs within 2e-3 of the oracle's double-precision attention read from
oracle-written codes.  k4v2 (the default) is covered there."""
import numpy as np
import pytest

import helpers
import oracle
import synth

pytestmark = pytest.mark.gpu

PRESETS = [(4, 4), (2, 2), (8, 4)]


def _torch():
    import torch
    return torch


def _dev_u16(arr, dtype):
    torch = _torch()
    t = torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).cuda()
    return t.view(torch.float16 if dtype == synth.F16 else torch.bfloat16)


def _geom(wl, preset):
    return oracle.geom(num_blocks=wl.num_blocks, num_kv_heads=wl.hkv, k_bits=preset[0], v_bits=preset[1])


# Small appends take a warp per head vector (at most 1024 per tensor), larger
# ones tensor-core tiles of 128 vectors; both with ragged tails.
@pytest.mark.parametrize("preset", PRESETS)
@pytest.mark.parametrize("make", [lambda: synth.Workload("q", 3, 16, 8, 128, [70, 1, 33], 16, synth.BF16, 3, 10.0,
                                                         30.0, seed=11),
                                  lambda: synth.Workload("qb", 2, 16, 8, 128, [70, 93], 16, synth.F16, 3, 10.0, 30.0,
                                                         seed=14)])
def test_preset_quantize_matches_oracle(kvq, cuda, preset, make):
    torch = _torch()
    wl = make()
    T = wl.total_tokens
    k = wl.kv_rows(synth.TID_K, 0, T)
    v = wl.kv_rows(synth.TID_V, 0, T)
    slots = wl.slots()
    nbytes = kvq.kvq_cache_bytes(kvq.make_desc(wl.num_blocks, wl.hkv, preset=preset))
    assert nbytes == wl.num_blocks * wl.hkv * (16 * 128 * (preset[0] + preset[1]) // 8 + 128)
    pool = torch.full((nbytes,), 0x5A, dtype=torch.uint8, device="cuda")
    kvq.kvq_quantize_append(pool, wl.num_blocks, wl.hkv, _dev_u16(k, wl.dtype).reshape(T, -1),
                            _dev_u16(v, wl.dtype).reshape(T, -1), torch.from_numpy(slots).cuda(), preset=preset)
    assert kvq.kvq_last_device_status() == 0
    gpu = pool.cpu().numpy()
    rep = helpers.QuantReport()
    helpers.check_pool_tokens(rep, gpu, wl.num_blocks, wl.hkv, k, v, wl.dtype, slots, range(T), preset=preset)
    assert rep.ok(), rep


@pytest.mark.parametrize("preset", PRESETS)
@pytest.mark.parametrize("G,bps", [(8, 0), (8, 1), (1, 0), (4, 3)])
def test_preset_decode_matches_oracle(kvq, cuda, preset, G, bps):
    """Ragged lengths (empty, one token, block edges, several chunks), GQA
    groups 1, 4, 8, one or several splits per sequence."""
    torch = _torch()
    wl = synth.Workload("pd", 6, 2 * G, 2, 128, [1, 15, 16, 17, 300, 0], 16, synth.BF16, 3, 10.0, 30.0,
                        seed=60 + G + 7 * preset[0] + preset[1], extra_blocks=3)
    g = _geom(wl, preset)
    pool = oracle.new_pool(g)
    assert oracle.quantize_append(g, pool, wl.kv_rows(synth.TID_K, 0, wl.total_tokens),
                                  wl.kv_rows(synth.TID_V, 0, wl.total_tokens), wl.dtype, wl.slots()) == 0
    q = wl.query()
    msl = int(wl.seq_lens.max())
    out = torch.empty((wl.batch, wl.hq, 128), dtype=torch.float32, device="cuda")
    ws = kvq.new_workspace(wl.num_blocks, wl.hkv, wl.batch, wl.hq, msl, bps, preset=preset)
    kvq.kvq_decode_attention(torch.from_numpy(pool).cuda(), wl.num_blocks, wl.hkv, _dev_u16(q, wl.dtype),
                             torch.from_numpy(wl.block_table).cuda(), torch.from_numpy(wl.seq_lens).cuda(), msl, out,
                             ws, blocks_per_split=bps, preset=preset)
    assert kvq.kvq_last_device_status() == 0
    got = out.cpu().numpy().astype(np.float64)
    want = oracle.decode_attention(g, pool, q, wl.dtype, wl.block_table, wl.seq_lens, nthreads=8)
    assert np.all(np.isfinite(got))
    assert np.max(np.abs(got - want)) <= helpers.ATTN_TOL, np.max(np.abs(got - want))
    assert not got[5].any()  # length 0 -> zeros


@pytest.mark.parametrize("preset", PRESETS)
def test_preset_append_decode(kvq, cuda, preset):
    """The fused one-step call writes the bytes the write path writes and gives
    the outputs the read path gives, and both agree with the oracle."""
    torch = _torch()
    wl = synth.Workload("pa", 4, 16, 2, 128, [70, 1, 300, 0], 16, synth.BF16, 3, 10.0, 30.0, seed=70 + preset[0],
                        extra_blocks=2)
    T = wl.total_tokens
    k = wl.kv_rows(synth.TID_K, 0, T)
    v = wl.kv_rows(synth.TID_V, 0, T)
    slots = wl.slots()
    last = np.array([int(wl.token_offsets[b]) + int(wl.seq_lens[b]) - 1 for b in range(wl.batch)
                     if wl.seq_lens[b] > 0])
    keep = np.setdiff1d(np.arange(T), last)
    g = _geom(wl, preset)
    base = oracle.new_pool(g, fill=0x5A)
    assert oracle.quantize_append(g, base, np.ascontiguousarray(k[keep]), np.ascontiguousarray(v[keep]), wl.dtype,
                                  slots[keep]) == 0
    kn = np.zeros((wl.batch, wl.hkv, 128), np.uint16)
    vn = np.zeros((wl.batch, wl.hkv, 128), np.uint16)
    for b in range(wl.batch):
        if wl.seq_lens[b] > 0:
            t = int(wl.token_offsets[b]) + int(wl.seq_lens[b]) - 1
            kn[b], vn[b] = k[t], v[t]
    q = wl.query()
    qd = _dev_u16(q, wl.dtype)
    bt = torch.from_numpy(wl.block_table).cuda()
    sl = torch.from_numpy(wl.seq_lens).cuda()
    msl = int(wl.seq_lens.max())
    ws = kvq.new_workspace(wl.num_blocks, wl.hkv, wl.batch, wl.hq, msl, preset=preset)
    pool1 = torch.from_numpy(base.copy()).cuda()
    kvq.kvq_quantize_append(pool1, wl.num_blocks, wl.hkv, _dev_u16(k[last], wl.dtype).reshape(len(last), -1),
                            _dev_u16(v[last], wl.dtype).reshape(len(last), -1),
                            torch.from_numpy(slots[last].copy()).cuda(), preset=preset)
    out1 = torch.empty((wl.batch, wl.hq, 128), dtype=torch.float32, device="cuda")
    kvq.kvq_decode_attention(pool1, wl.num_blocks, wl.hkv, qd, bt, sl, msl, out1, ws, preset=preset)
    pool2 = torch.from_numpy(base.copy()).cuda()
    out2 = torch.empty_like(out1)
    kvq.kvq_append_decode_attention(pool2, wl.num_blocks, wl.hkv, _dev_u16(kn, wl.dtype).reshape(wl.batch, -1),
                                    _dev_u16(vn, wl.dtype).reshape(wl.batch, -1), qd, bt, sl, msl, out2, ws,
                                    preset=preset)
    assert kvq.kvq_last_device_status() == 0
    p1, p2 = pool1.cpu().numpy(), pool2.cpu().numpy()
    assert np.array_equal(p1, p2)
    assert torch.equal(out1, out2)
    rep = helpers.QuantReport()
    helpers.check_pool_tokens(rep, p2, wl.num_blocks, wl.hkv, k, v, wl.dtype, slots, last, preset=preset)
    assert rep.ok(), rep
    want = oracle.decode_attention(g, p2, q, wl.dtype, wl.block_table, wl.seq_lens, nthreads=8)
    got = out2.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(got - want)) <= helpers.ATTN_TOL, np.max(np.abs(got - want))
