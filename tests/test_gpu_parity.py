"""GPU parity: the CUDA path through the C-ABI against the CPU oracle on the
same seeded inputs.  Quantized codes must be bit-exact except at near-ties
(tests/helpers.py); decode outputs must be within 2e-3 (max abs, fp32) of the
oracle's double-precision attention read from the same codes, which here are
always written by the oracle and uploaded (no oracle input comes from the
CUDA path)."""
import math

import numpy as np
import pytest

import helpers
import oracle
import synth

pytestmark = pytest.mark.gpu


def _torch():
    import torch
    return torch


def _dev_u16(arr, dtype):
    torch = _torch()
    t = torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).cuda()
    return t.view(torch.float16 if dtype == synth.F16 else torch.bfloat16)


def _oracle_pool(wl):
    g = oracle.geom(num_blocks=wl.num_blocks, num_kv_heads=wl.hkv)
    pool = oracle.new_pool(g)
    k = wl.kv_rows(synth.TID_K, 0, wl.total_tokens)
    v = wl.kv_rows(synth.TID_V, 0, wl.total_tokens)
    assert oracle.quantize_append(g, pool, k, v, wl.dtype, wl.slots()) == 0
    return g, pool, k, v


def _gpu_decode(kvq, wl, pool_np, q_np, q_dtype, out_dtype="f32", bps=0, max_seq_len=None, seq_lens=None,
                block_table=None):
    torch = _torch()
    pool = torch.from_numpy(pool_np).cuda()
    if q_dtype == synth.F32:
        q = torch.from_numpy(q_np.astype(np.float32)).cuda()
    else:
        q = _dev_u16(q_np, q_dtype)
    lens = wl.seq_lens if seq_lens is None else np.asarray(seq_lens, np.int32)
    bt = torch.from_numpy(wl.block_table if block_table is None else block_table).cuda()
    sl = torch.from_numpy(lens).cuda()
    msl = int(lens.max()) if max_seq_len is None else max_seq_len
    out = torch.empty((wl.batch, wl.hq, 128), dtype={"f32": torch.float32, "bf16": torch.bfloat16,
                                                      "f16": torch.float16}[out_dtype], device="cuda")
    ws = kvq.new_workspace(wl.num_blocks, wl.hkv, wl.batch, wl.hq, msl, bps)
    kvq.kvq_decode_attention(pool, wl.num_blocks, wl.hkv, q, bt, sl, msl, out, ws, blocks_per_split=bps)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64), ws


# ------------------------------------------------------------------ write path

def _run_quantize(kvq, wl, slots, k, v, pool_fill=0x5A):
    torch = _torch()
    pool = torch.full((kvq.kvq_cache_bytes(kvq.make_desc(wl.num_blocks, wl.hkv)),), pool_fill, dtype=torch.uint8,
                      device="cuda")
    kd = _dev_u16(k, wl.dtype).reshape(k.shape[0], -1)
    vd = _dev_u16(v, wl.dtype).reshape(v.shape[0], -1)
    sd = torch.from_numpy(np.ascontiguousarray(slots, np.int32)).cuda()
    kvq.kvq_quantize_append(pool, wl.num_blocks, wl.hkv, kd, vd, sd)
    assert kvq.kvq_last_device_status() == 0
    return pool.cpu().numpy()


# The write path takes a warp per head vector for small appends (at most 1024
# head vectors per tensor) and tensor-core tiles of 128 head vectors above
# that; both paths are covered, with ragged tails, and the tile path with
# bf16 and fp16 inputs (the two forms of its MMA).
@pytest.mark.parametrize("make", [lambda: synth.tiny(0),
                                  lambda: synth.Workload("q", 3, 16, 8, 128, [70, 1, 33], 16, synth.BF16, 3, 10.0,
                                                         30.0, seed=11),
                                  lambda: synth.Workload("qb", 2, 16, 8, 128, [70, 93], 16, synth.BF16, 3, 10.0,
                                                         30.0, seed=14),
                                  lambda: synth.Workload("qb16", 2, 16, 8, 128, [70, 93], 16, synth.F16, 3, 10.0,
                                                         30.0, seed=16)])
def test_quantize_matches_oracle(kvq, cuda, make):
    wl = make()
    k = wl.kv_rows(synth.TID_K, 0, wl.total_tokens)
    v = wl.kv_rows(synth.TID_V, 0, wl.total_tokens)
    slots = wl.slots()
    gpu = _run_quantize(kvq, wl, slots, k, v)
    rep = helpers.QuantReport()
    helpers.check_pool_tokens(rep, gpu, wl.num_blocks, wl.hkv, k, v, wl.dtype, slots, range(wl.total_tokens))
    assert rep.ok(), rep
    # bytes of the pool no token maps to are untouched
    written = np.zeros((wl.num_blocks, wl.hkv, 16), bool)
    for s in slots:
        written[s // 16, :, s % 16] = True
    seg = gpu.reshape(wl.num_blocks, wl.hkv, 1664)
    for p in range(wl.num_blocks):
        for o in range(16):
            if not written[p, 0, o]:
                assert np.all(seg[p, :, o * 64:(o + 1) * 64] == 0x5A)
                assert np.all(seg[p, :, 1024 + o * 32:1024 + (o + 1) * 32] == 0x5A)


def test_quantize_bulk_many_tiles(kvq, cuda):
    """More tiles than the persistent grid holds at once (two CTAs per SM):
    every CTA walks several tiles through both operand buffers; a sample of
    tokens (every 17th and the last eight) is checked against the oracle."""
    wl = synth.Workload("qm", 2, 16, 8, 128, [1500, 1491], 16, synth.BF16, 3, 10.0, 30.0, seed=15)
    T = wl.total_tokens
    k = wl.kv_rows(synth.TID_K, 0, T)
    v = wl.kv_rows(synth.TID_V, 0, T)
    slots = wl.slots()
    gpu = _run_quantize(kvq, wl, slots, k, v)
    rep = helpers.QuantReport()
    tokens = sorted(set(range(0, T, 17)) | set(range(T - 8, T)))
    helpers.check_pool_tokens(rep, gpu, wl.num_blocks, wl.hkv, k, v, wl.dtype, slots, tokens)
    assert rep.ok(), rep


@pytest.mark.parametrize("n", [40, 600])
def test_quantize_edge_inputs(kvq, cuda, n):
    """Zero vectors, one-hot vectors (flat after rotation: S = 0), skipped
    slots, a strided (non-dense) token layout and a lone token in a block;
    40 tokens take the small-append path, 600 the bulk path."""
    torch = _torch()
    hkv = 2
    wl = synth.Workload("e", 1, 2, hkv, 128, [n], 16, synth.BF16, 3, 10.0, 30.0, seed=12, extra_blocks=2,
                        shuffle=False)
    k = wl.kv_rows(synth.TID_K, 0, n)
    v = wl.kv_rows(synth.TID_V, 0, n)
    k[0] = 0
    v[1] = 0
    k[2, :, :] = 0
    k[2, :, 0] = np.array([2.5], np.float32).view(np.uint32)[0] >> 16  # bf16 bits of 2.5
    slots = wl.slots().copy()
    slots[5] = -1
    slots[7] = wl.num_blocks * 16 - 1  # last slot of the pool
    # strided rows: each token row padded to 3*128 elements
    stride = 3 * 128
    kp = np.zeros((n, stride), np.uint16)
    vp = np.zeros((n, stride), np.uint16)
    kp[:, :hkv * 128] = k.reshape(n, -1)
    vp[:, :hkv * 128] = v.reshape(n, -1)
    pool = torch.full((wl.num_blocks * hkv * 1664,), 0x33, dtype=torch.uint8, device="cuda")
    kvq.kvq_quantize_append(pool, wl.num_blocks, hkv, _dev_u16(kp, wl.dtype), _dev_u16(vp, wl.dtype),
                            torch.from_numpy(slots).cuda())
    assert kvq.kvq_last_device_status() == 0
    gpu = pool.cpu().numpy()
    rep = helpers.QuantReport()
    helpers.check_pool_tokens(rep, gpu, wl.num_blocks, hkv, k, v, wl.dtype, slots, range(n))
    assert rep.ok(), rep
    g = oracle.geom(num_blocks=wl.num_blocks, num_kv_heads=hkv)
    kc, Sk, Zk, *_ = oracle.unpack_token(g, gpu, slots[0] // 16, slots[0] % 16, 0)
    assert Sk == 0 and Zk == 0 and not kc.any()
    kc, Sk, Zk, *_ = oracle.unpack_token(g, gpu, slots[2] // 16, slots[2] % 16, 0)
    assert Sk == 0 and not kc.any()
    s5 = wl.slots()[5]
    seg = gpu.reshape(wl.num_blocks, hkv, 1664)
    assert np.all(seg[s5 // 16, :, (s5 % 16) * 64:(s5 % 16 + 1) * 64] == 0x33)


def test_quantize_reports_slot_outside_pool(kvq, cuda):
    torch = _torch()
    wl = synth.Workload("e", 1, 1, 1, 128, [3], 16, synth.F16, 0, 1.0, 1.0, seed=13)
    k = wl.kv_rows(synth.TID_K, 0, 3)
    pool = torch.zeros(wl.num_blocks * 1664, dtype=torch.uint8, device="cuda")
    slots = torch.tensor([0, 16 * wl.num_blocks + 3, 1], dtype=torch.int32, device="cuda")
    kvq.kvq_quantize_append(pool, wl.num_blocks, 1, _dev_u16(k, wl.dtype).reshape(3, -1),
                            _dev_u16(k, wl.dtype).reshape(3, -1), slots)
    assert kvq.kvq_last_device_status() == kvq.KVQ_ERR_OUT_OF_RANGE
    assert kvq.kvq_last_device_status() == 0  # read-and-clear


# ------------------------------------------------------------------ read path

def _check_decode(wl, g, pool, q, q_dtype, got, rel=0.0):
    """max |got - want| <= 2e-3 (+ rel*|want| for a bf16/fp16 output)."""
    want = oracle.decode_attention(g, pool, q, q_dtype, wl.block_table, wl.seq_lens, nthreads=8)
    assert np.all(np.isfinite(got))
    excess = np.abs(got - want) - (helpers.ATTN_TOL + rel * np.abs(want))
    assert excess.max() <= 0, (np.max(np.abs(got - want)), excess.max())
    return float(np.max(np.abs(got - want)))


def test_decode_tiny(kvq, cuda):
    wl = synth.tiny(0)
    g, pool, _, _ = _oracle_pool(wl)
    q = wl.query()
    got, _ = _gpu_decode(kvq, wl, pool, q, wl.dtype)
    _check_decode(wl, g, pool, q, wl.dtype, got)


@pytest.mark.parametrize("bps", [0, 1, 3, 1000])
def test_decode_ragged_gqa8(kvq, cuda, bps):
    wl = synth.Workload("r", 6, 16, 2, 128, [1, 15, 16, 17, 100, 0], 16, synth.BF16, 3, 10.0, 30.0, seed=21,
                        extra_blocks=3)
    g, pool, _, _ = _oracle_pool(wl)
    q = wl.query()
    got, _ = _gpu_decode(kvq, wl, pool, q, wl.dtype, bps=bps)
    _check_decode(wl, g, pool, q, wl.dtype, got)
    assert not got[5].any()  # length 0 -> zeros


@pytest.mark.parametrize("bps", [1, 2])
def test_decode_many_splits(kvq, cuda, bps):
    """Many splits per sequence (400 tokens in splits of one or two blocks:
    more records than the merge takes in one batch of 16), empty splits of
    a shorter sequence, and an empty sequence."""
    wl = synth.Workload("m", 3, 16, 2, 128, [400, 33, 0], 16, synth.BF16, 3, 10.0, 30.0, seed=23, extra_blocks=2)
    g, pool, _, _ = _oracle_pool(wl)
    q = wl.query()
    got, _ = _gpu_decode(kvq, wl, pool, q, wl.dtype, bps=bps)
    _check_decode(wl, g, pool, q, wl.dtype, got)
    assert not got[2].any()


@pytest.mark.parametrize("G", [1, 2, 4])
def test_decode_group_sizes(kvq, cuda, G):
    wl = synth.Workload("g", 2, 4 * G, 4, 128, [129, 47], 16, synth.F16, 4, 20.0, 20.0, seed=30 + G)
    g, pool, _, _ = _oracle_pool(wl)
    q = wl.query()
    got, _ = _gpu_decode(kvq, wl, pool, q, wl.dtype)
    _check_decode(wl, g, pool, q, wl.dtype, got)


@pytest.mark.parametrize("q_dtype,out_dtype,rel", [(synth.F32, "f32", 0.0), (synth.F16, "bf16", 2.0 ** -8),
                                                   (synth.BF16, "f16", 2.0 ** -11)])
def test_decode_dtypes(kvq, cuda, q_dtype, out_dtype, rel):
    wl = synth.Workload("d", 2, 16, 2, 128, [90, 200], 16, synth.BF16, 3, 10.0, 30.0, seed=40)
    g, pool, _, _ = _oracle_pool(wl)
    q = synth.normal(wl.seed, synth.TID_Q, wl.batch * wl.hq * 128, q_dtype).reshape(wl.batch, wl.hq, 128)
    got, _ = _gpu_decode(kvq, wl, pool, q, q_dtype, out_dtype=out_dtype)
    # bf16/f16 outputs carry their own rounding on top of the 2e-3 kernel bound
    _check_decode(wl, g, pool, q, q_dtype, got, rel=rel)


# The fused step's appended block lies in the first chunk of a split ("short",
# many splits) or, with one split per sequence ("one_split": 80 x 8 kv heads
# are more CTAs than the SMs hold, so the plan does not split), in chunks
# 0 .. 5 of it: the first three chunks are copied before the append is
# written, except the one holding the new block.
_APPEND_LENS = {
    "short": (4, 16, 2, [70, 1, 33, 0]),
    "one_split": (80, 16, 8, [0, 1, 700, 384, 385, 513] + [(97 * i * i + 31 * i) % 701 for i in range(74)]),
}


@pytest.mark.parametrize("case", sorted(_APPEND_LENS))
def test_append_decode_matches_append_then_decode(kvq, cuda, case):
    """The fused one-step call writes the same pool bytes as the write path
    followed by the read path, gives the same outputs, and both agree with
    the oracle (codes: near-tie rules; outputs: 2e-3 on the same codes)."""
    torch = _torch()
    batch, hq, hkv, lens = _APPEND_LENS[case]
    wl = synth.Workload("ad", batch, hq, hkv, 128, lens, 16, synth.BF16, 3, 10.0, 30.0, seed=25, extra_blocks=2)
    T = wl.total_tokens
    k = wl.kv_rows(synth.TID_K, 0, T)
    v = wl.kv_rows(synth.TID_V, 0, T)
    slots = wl.slots()
    last = np.array([int(wl.token_offsets[b]) + int(wl.seq_lens[b]) - 1 for b in range(wl.batch)
                     if wl.seq_lens[b] > 0])
    keep = np.setdiff1d(np.arange(T), last)
    g = oracle.geom(num_blocks=wl.num_blocks, num_kv_heads=wl.hkv)
    base = oracle.new_pool(g, fill=0x5A)
    assert oracle.quantize_append(g, base, np.ascontiguousarray(k[keep]), np.ascontiguousarray(v[keep]), wl.dtype,
                                  slots[keep]) == 0
    # new rows per sequence (zeros for the empty sequence, which appends nothing)
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
    ws = kvq.new_workspace(wl.num_blocks, wl.hkv, wl.batch, wl.hq, msl)
    # two calls: write path, then read path
    pool1 = torch.from_numpy(base.copy()).cuda()
    kvq.kvq_quantize_append(pool1, wl.num_blocks, wl.hkv, _dev_u16(k[last], wl.dtype).reshape(len(last), -1),
                            _dev_u16(v[last], wl.dtype).reshape(len(last), -1),
                            torch.from_numpy(slots[last].copy()).cuda())
    out1 = torch.empty((wl.batch, wl.hq, 128), dtype=torch.float32, device="cuda")
    kvq.kvq_decode_attention(pool1, wl.num_blocks, wl.hkv, qd, bt, sl, msl, out1, ws)
    # one fused call
    pool2 = torch.from_numpy(base.copy()).cuda()
    out2 = torch.empty_like(out1)
    kvq.kvq_append_decode_attention(pool2, wl.num_blocks, wl.hkv, _dev_u16(kn, wl.dtype).reshape(wl.batch, -1),
                                    _dev_u16(vn, wl.dtype).reshape(wl.batch, -1), qd, bt, sl, msl, out2, ws)
    assert kvq.kvq_last_device_status() == 0
    p1, p2 = pool1.cpu().numpy(), pool2.cpu().numpy()
    assert np.array_equal(p1, p2)
    assert torch.equal(out1, out2)
    rep = helpers.QuantReport()
    helpers.check_pool_tokens(rep, p2, wl.num_blocks, wl.hkv, k, v, wl.dtype, slots, last)
    assert rep.ok(), rep
    _check_decode(wl, g, p2, q, wl.dtype, out2.cpu().numpy().astype(np.float64))
    for b in range(wl.batch):
        if wl.seq_lens[b] == 0:  # an empty sequence appends nothing and reads nothing
            assert not out2[b].any()


def test_append_decode_with_bad_length_writes_nothing(kvq, cuda):
    """A sequence length beyond max_seq_len (or the table row) is recorded as
    out of range, its read is truncated, and the fused step appends nothing:
    the pool bytes stay as they were (the write position would otherwise be
    a clamped one, not seq_lens[b] - 1)."""
    torch = _torch()
    wl = synth.Workload("bl", 2, 16, 2, 128, [48, 40], 16, synth.BF16, 3, 10.0, 30.0, seed=26, extra_blocks=4)
    g, pool, _, _ = _oracle_pool(wl)
    msl = int(wl.seq_lens.max())
    # sequence 0 claims 16 more tokens than max_seq_len (and than its row)
    bad_lens = wl.seq_lens.copy()
    bad_lens[0] = msl + 16
    kn = wl.kv_rows(synth.TID_NEWK, 0, wl.batch)
    vn = wl.kv_rows(synth.TID_NEWV, 0, wl.batch)
    dpool = torch.from_numpy(pool.copy()).cuda()
    out = torch.empty((wl.batch, wl.hq, 128), dtype=torch.float32, device="cuda")
    ws = kvq.new_workspace(wl.num_blocks, wl.hkv, wl.batch, wl.hq, msl)
    kvq.kvq_append_decode_attention(dpool, wl.num_blocks, wl.hkv, _dev_u16(kn, wl.dtype).reshape(wl.batch, -1),
                                    _dev_u16(vn, wl.dtype).reshape(wl.batch, -1), _dev_u16(wl.query(), wl.dtype),
                                    torch.from_numpy(wl.block_table).cuda(), torch.from_numpy(bad_lens).cuda(), msl,
                                    out, ws)
    assert kvq.kvq_last_device_status() == kvq.KVQ_ERR_OUT_OF_RANGE
    after = dpool.cpu().numpy()
    seg = lambda a: a.reshape(wl.num_blocks, wl.hkv, 1664)
    # sequence 0's blocks are untouched; sequence 1 appended its new token at position 39
    rows0 = wl.block_table[0][wl.block_table[0] >= 0]
    assert np.array_equal(seg(after)[rows0], seg(pool)[rows0])
    p1, o1 = divmod(int(wl.block_table[1][39 // 16]) * 16 + 39 % 16, 16)
    changed = np.nonzero(np.any(seg(after) != seg(pool), axis=2))
    assert set(changed[0].tolist()) <= {p1}
    rep = helpers.QuantReport()
    helpers.check_pool_tokens(rep, after, wl.num_blocks, wl.hkv, kn, vn, wl.dtype,
                              np.array([-1, p1 * 16 + o1], np.int32), [1])
    assert rep.ok(), rep
    # the truncated read of sequence 0 (its 48 tokens) and the read of sequence 1 match the oracle
    want = oracle.decode_attention(g, after, wl.query(), wl.dtype, wl.block_table, wl.seq_lens)
    assert np.max(np.abs(out.cpu().numpy().astype(np.float64) - want)) <= helpers.ATTN_TOL


def test_decode_workspace_is_reusable(kvq, cuda):
    """Tickets reset themselves: the same workspace serves repeated calls."""
    torch = _torch()
    wl = synth.Workload("w", 2, 16, 2, 128, [300, 77], 16, synth.BF16, 3, 10.0, 30.0, seed=50)
    g, pool, _, _ = _oracle_pool(wl)
    q = wl.query()
    got1, ws = _gpu_decode(kvq, wl, pool, q, wl.dtype, bps=2)
    tickets = ws[:256].view(torch.int32)[: wl.batch * wl.hkv]
    assert not tickets.any()
    dpool = torch.from_numpy(pool).cuda()
    out = torch.empty((wl.batch, wl.hq, 128), dtype=torch.float32, device="cuda")
    for _ in range(3):
        kvq.kvq_decode_attention(dpool, wl.num_blocks, wl.hkv, _dev_u16(q, wl.dtype),
                                 torch.from_numpy(wl.block_table).cuda(), torch.from_numpy(wl.seq_lens).cuda(),
                                 int(wl.seq_lens.max()), out, ws, blocks_per_split=2)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy().astype(np.float64), got1)


def test_decode_reports_bad_block_id(kvq, cuda):
    wl = synth.Workload("b", 1, 8, 1, 128, [64], 16, synth.BF16, 3, 10.0, 30.0, seed=60, extra_blocks=1)
    g, pool, _, _ = _oracle_pool(wl)
    q = wl.query()
    bt = wl.block_table.copy()
    bt[0, 2] = wl.num_blocks + 5
    got, _ = _gpu_decode(kvq, wl, pool, q, wl.dtype, block_table=bt)
    assert kvq.kvq_last_device_status() == kvq.KVQ_ERR_OUT_OF_RANGE
    assert np.all(np.isfinite(got))
    # the bad block's tokens are skipped: the oracle over the other three blocks agrees
    keep = [0, 1, 3]
    bt3 = np.full((1, 3), -1, np.int32)
    bt3[0] = wl.block_table[0, keep]
    pool2 = pool.copy()
    want = oracle.decode_attention(g, pool2, q, wl.dtype, bt3, np.array([48], np.int32))
    assert np.max(np.abs(got - want)) <= helpers.ATTN_TOL


def test_end_to_end_against_unquantized(kvq, cuda):
    """GPU write then GPU read against oracle write then oracle read; also
    reports (does not gate) the error of the quantised cache against fp16
    attention on the raw inputs."""
    torch = _torch()
    wl = synth.Workload("x", 2, 16, 2, 128, [256, 93], 16, synth.BF16, 3, 10.0, 30.0, seed=70)
    g, opool, k, v = _oracle_pool(wl)
    gpool = _run_quantize(kvq, wl, wl.slots(), k, v)
    q = wl.query()
    got, _ = _gpu_decode(kvq, wl, gpool, q, wl.dtype)
    want = oracle.decode_attention(g, opool, q, wl.dtype, wl.block_table, wl.seq_lens)
    assert np.max(np.abs(got - want)) <= helpers.ATTN_TOL
    dense_err = 0.0
    for b in range(wl.batch):
        L = int(wl.seq_lens[b])
        off = int(wl.token_offsets[b])
        for j in range(wl.hq):
            ref = oracle.attention_dense(k[off:off + L], v[off:off + L], wl.dtype, q[b, j], wl.dtype, wl.hq, j)
            dense_err = max(dense_err, float(np.max(np.abs(got[b, j] - ref))))
    print(f"\nk4v2_g128 decode vs unquantized attention: max abs err {dense_err:.4f}")
    assert math.isfinite(dense_err)


def test_decode_ignores_garbage_in_unused_slots(kvq, cuda):
    """Rows past the end of a sequence hold whatever the pool held before
    (here 0xFF bytes: NaN scales and zero points); they must not leak in."""
    wl = synth.Workload("n", 3, 16, 2, 128, [17, 5, 250], 16, synth.BF16, 3, 10.0, 30.0, seed=80, extra_blocks=2)
    g = oracle.geom(num_blocks=wl.num_blocks, num_kv_heads=wl.hkv)
    pool = oracle.new_pool(g, fill=0xFF)
    k = wl.kv_rows(synth.TID_K, 0, wl.total_tokens)
    v = wl.kv_rows(synth.TID_V, 0, wl.total_tokens)
    assert oracle.quantize_append(g, pool, k, v, wl.dtype, wl.slots()) == 0
    q = wl.query()
    for bps in (0, 1):
        got, _ = _gpu_decode(kvq, wl, pool, q, wl.dtype, bps=bps)
        _check_decode(wl, g, pool, q, wl.dtype, got)
