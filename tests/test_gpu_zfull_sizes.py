"""Full-size parity at the benchmarked sizes, through the C ABI, in the
default (benchmarked) split plan.

Write path: the GPU-written pool against the oracle-written pool, every
(token, head) group compared byte for byte, the differing ones under the
near-tie rules of tests/helpers.py.  Read path: the GPU decodes a pool the
oracle wrote (no oracle input comes from the CUDA path), and its outputs are
compared with the oracle's attention over the same bytes (max abs error
<= 2e-3).  The workloads are the seeded synthetic stand-ins for the pages'
Qwen3-32B (16K context) and Llama-3.1-70B (128K context) decodes ("Трюк
Huawei с KV-кэшем", lede; "Kompresja pamięci podręcznej KV to decyzja
infrastrukturalna..." (encorp.ai), HBM-math section)."""
import numpy as np
import pytest

import helpers
import oracle
import synth

pytestmark = pytest.mark.gpu

from test_gpu_parity import _dev_u16, _torch  # noqa: E402


def _gpu_write(kvq, wl, k, v, slots, fill=0):
    torch = _torch()
    T = slots.size
    pool = torch.full((wl.num_blocks * wl.hkv * 1664,), fill, dtype=torch.uint8, device="cuda")
    kvq.kvq_quantize_append(pool, wl.num_blocks, wl.hkv, _dev_u16(k, wl.dtype).reshape(T, -1),
                            _dev_u16(v, wl.dtype).reshape(T, -1), torch.from_numpy(slots).cuda())
    assert kvq.kvq_last_device_status() == 0
    return pool


def _decode(kvq, wl, pool, q, out_dtype="f32", bps=0, fused=None):
    """GPU decode of `pool` (a device tensor); fused = (k_new, v_new) rows
    [batch, Hkv, 128] to run the one-step append + decode call instead."""
    torch = _torch()
    msl = int(wl.seq_lens.max())
    out = torch.empty((wl.batch, wl.hq, 128), dtype={"f32": torch.float32, "bf16": torch.bfloat16}[out_dtype],
                      device="cuda")
    ws = kvq.new_workspace(wl.num_blocks, wl.hkv, wl.batch, wl.hq, msl, bps)
    bt = torch.from_numpy(wl.block_table).cuda()
    sl = torch.from_numpy(wl.seq_lens).cuda()
    qd = _dev_u16(q, wl.dtype)
    if fused is None:
        kvq.kvq_decode_attention(pool, wl.num_blocks, wl.hkv, qd, bt, sl, msl, out, ws, blocks_per_split=bps)
    else:
        kn, vn = fused
        kvq.kvq_append_decode_attention(pool, wl.num_blocks, wl.hkv, _dev_u16(kn, wl.dtype).reshape(wl.batch, -1),
                                        _dev_u16(vn, wl.dtype).reshape(wl.batch, -1), qd, bt, sl, msl, out, ws)
    assert kvq.kvq_last_device_status() == 0
    return out.float().cpu().numpy().astype(np.float64)


def _head_pool(pool, num_blocks, hkv, h):
    """The segments of kv head h alone, as a one-head pool (same block ids)."""
    return np.ascontiguousarray(pool.reshape(num_blocks, hkv, 1664)[:, h]).reshape(-1)


def _plain_pairs(wl, opool, q, got, pairs):
    """Max abs error of the GPU outputs against the oracle's plain definition
    on the listed (sequence, kv head) pairs, all G query heads of each."""
    from concurrent.futures import ThreadPoolExecutor
    G = wl.hq // wl.hkv
    g1 = oracle.geom(num_blocks=wl.num_blocks, num_kv_heads=1)

    def one(bh):
        b, h = bh
        hp = _head_pool(opool, wl.num_blocks, wl.hkv, h)
        qh = np.ascontiguousarray(q[b:b + 1, h * G:(h + 1) * G])
        want = oracle.decode_attention(g1, hp, qh, wl.dtype, wl.block_table[b:b + 1], wl.seq_lens[b:b + 1],
                                       form=0, nthreads=1)
        return float(np.max(np.abs(got[b, h * G:(h + 1) * G] - want[0])))

    with ThreadPoolExecutor(min(len(pairs), helpers.threads())) as ex:
        return max(ex.map(one, pairs))


def _last_positions(wl):
    return np.array([int(wl.token_offsets[b]) + int(wl.seq_lens[b]) - 1 for b in range(wl.batch)])


def test_full_size_qwen3_32b_layer_all_heads_all_codes(kvq, cuda):
    """Batch 1, 64/8 heads, 16384 tokens: all 131072 token-heads' codes; the
    bench's step (the fused append of the new token at position 16383, then
    decode) on an oracle-written pool, all 64 query heads, fp32 and bf16
    outputs."""
    torch = _torch()
    wl = synth.qwen3_32b_layer(0)
    T = wl.total_tokens
    k = wl.kv_rows(synth.TID_K, 0, T)
    v = wl.kv_rows(synth.TID_V, 0, T)
    slots = wl.slots()
    g = oracle.geom(num_blocks=wl.num_blocks, num_kv_heads=wl.hkv)
    opool = oracle.new_pool(g)
    helpers.oracle_append_threaded(g, opool, k, v, wl.dtype, slots)
    gpool = _gpu_write(kvq, wl, k, v, slots).cpu().numpy()
    rep = helpers.QuantReport()
    helpers.compare_pools(rep, gpool, opool, wl.num_blocks, wl.hkv, k, v, wl.dtype, slots)
    assert rep.vectors == 2 * T * wl.hkv
    assert rep.ok(), rep
    # the fused step: the oracle's pool without the last token, whose rows the
    # call appends; then decode of all 64 query heads
    last = _last_positions(wl)
    base = opool.copy()
    seg = base.reshape(wl.num_blocks, wl.hkv, 1664)
    p, o = divmod(int(slots[last[0]]), 16)
    seg[p, :, o * 64:(o + 1) * 64] = 0x5A
    seg[p, :, 1024 + o * 32:1024 + (o + 1) * 32] = 0x5A
    q = wl.query()
    want = oracle.decode_attention(g, opool, q, wl.dtype, wl.block_table, wl.seq_lens, nthreads=helpers.threads())
    for out_dtype, rel in (("f32", 0.0), ("bf16", 2.0 ** -8)):
        dpool = torch.from_numpy(base.copy()).cuda()
        got = _decode(kvq, wl, dpool, q, out_dtype, fused=(k[last], v[last]))
        after = dpool.cpu().numpy()
        rep = helpers.QuantReport()
        helpers.compare_pools(rep, after, opool, wl.num_blocks, wl.hkv, k, v, wl.dtype, slots, tokens=last)
        assert rep.ok(), rep
        mask = np.ones(base.size, bool)
        mask_seg = mask.reshape(wl.num_blocks, wl.hkv, 1664)
        mask_seg[p, :, o * 64:(o + 1) * 64] = False
        mask_seg[p, :, 1024 + o * 32:1024 + (o + 1) * 32] = False
        mask_seg[p, :, 1536 + 2 * o:1536 + 2 * o + 2] = False
        mask_seg[p, :, 1568 + 2 * o:1568 + 2 * o + 2] = False
        mask_seg[p, :, 1600 + 2 * o:1600 + 2 * o + 2] = False
        mask_seg[p, :, 1632 + 2 * o:1632 + 2 * o + 2] = False
        assert np.array_equal(after[mask], base[mask])  # nothing else written
        err = np.abs(got - want) - (helpers.ATTN_TOL + rel * np.abs(want))
        print(f"\nqwen3-32b layer, fused step, {out_dtype} out: max abs err {np.max(np.abs(got - want)):.2e}")
        assert err.max() <= 0


def test_full_size_batched_ragged(kvq, cuda):
    """Batch 32, ragged lengths U[4096, 16384], 64/8 heads: all codes; decode
    of the oracle-written pool, all 2048 (b, j) pairs against the oracle's
    folded form and 64 seeded pairs (8 sequences x 8 heads of distinct kv
    heads) against its plain definition."""
    torch = _torch()
    wl = synth.batched(0)
    T = wl.total_tokens
    k = wl.kv_rows(synth.TID_K, 0, T)
    v = wl.kv_rows(synth.TID_V, 0, T)
    slots = wl.slots()
    g = oracle.geom(num_blocks=wl.num_blocks, num_kv_heads=wl.hkv)
    opool = oracle.new_pool(g)
    helpers.oracle_append_threaded(g, opool, k, v, wl.dtype, slots)
    gpool = _gpu_write(kvq, wl, k, v, slots).cpu().numpy()
    rep = helpers.QuantReport()
    helpers.compare_pools(rep, gpool, opool, wl.num_blocks, wl.hkv, k, v, wl.dtype, slots)
    assert rep.vectors == 2 * T * wl.hkv
    assert rep.ok(), rep
    del gpool, k, v
    q = wl.query()
    got = _decode(kvq, wl, torch.from_numpy(opool).cuda(), q)
    folded = oracle.decode_attention(g, opool, q, wl.dtype, wl.block_table, wl.seq_lens, form=1,
                                     nthreads=helpers.threads())
    err = float(np.max(np.abs(got - folded)))
    print(f"\nbatched 32 x U[4096,16384]: all pairs vs folded oracle {err:.2e}")
    assert err <= helpers.ATTN_TOL
    # distinct sequences, kv head h for the h-th of them
    bs = np.random.default_rng(7).choice(wl.batch, 8, replace=False)
    worst = _plain_pairs(wl, opool, q, got, [(int(b), h) for h, b in enumerate(bs)])
    print(f"batched: 64 sampled pairs vs plain oracle {worst:.2e}")
    assert worst <= helpers.ATTN_TOL


def _long_pool(kvq, wl, sampled):
    """The long workload's pool: every block holds GPU-written segments of the
    seeded stream's first 16384 tokens (repeated); the (sequence, kv head)
    pairs in `sampled` hold the oracle's bytes for their own 131072 tokens."""
    torch = _torch()
    T0 = 16384
    nb0 = T0 // wl.bs
    k0 = wl.kv_rows(synth.TID_K, 0, T0)
    v0 = wl.kv_rows(synth.TID_V, 0, T0)
    base = kvq.new_pool(nb0, wl.hkv)
    kvq.kvq_quantize_append(base, nb0, wl.hkv, _dev_u16(k0, wl.dtype).reshape(T0, -1),
                            _dev_u16(v0, wl.dtype).reshape(T0, -1), torch.arange(T0, dtype=torch.int32, device="cuda"))
    assert kvq.kvq_last_device_status() == 0
    pool = kvq.new_pool(wl.num_blocks, wl.hkv)
    seg = pool.view(wl.num_blocks, wl.hkv, 1664)
    b0 = base.view(nb0, wl.hkv, 1664)
    for s in range(0, wl.num_blocks, nb0):
        n = min(nb0, wl.num_blocks - s)
        seg[s:s + n].copy_(b0[:n])
    del base, b0
    slots = wl.slots()
    g1 = oracle.geom(num_blocks=wl.num_blocks, num_kv_heads=1)
    opools = {}
    for b, h in sampled:
        L = int(wl.seq_lens[b])
        off = int(wl.token_offsets[b])
        k = wl.kv_rows(synth.TID_K, off, L)
        v = wl.kv_rows(synth.TID_V, off, L)
        ks = np.ascontiguousarray(k[:, h:h + 1])
        vs = np.ascontiguousarray(v[:, h:h + 1])
        del k, v
        op = oracle.new_pool(g1)
        s_slots = np.ascontiguousarray(slots[off:off + L])
        helpers.oracle_append_threaded(g1, op, ks, vs, wl.dtype, s_slots)
        used = torch.from_numpy(np.unique(s_slots // wl.bs)).cuda().long()
        seg[used, h] = torch.from_numpy(op.reshape(wl.num_blocks, 1664)).cuda()[used]
        opools[(b, h)] = op
    return pool, opools


def test_full_size_long_context_sampled_pairs(kvq, cuda):
    """Llama-3.1-70B-shaped: batch 8 x 131072 tokens, 64/8 heads.  One kv head
    per sequence (head b of sequence b: eight distinct heads) holds oracle
    bytes; its 8 query heads (64 (b, j) pairs in all) are checked against the
    oracle's plain attention, in the default split plan and with splits of
    the longest kind (1024 blocks = 128 chunks per CTA, eight per sequence)."""
    torch = _torch()
    wl = synth.long_context(0)
    G = wl.hq // wl.hkv
    sampled = [(b, b % wl.hkv) for b in range(wl.batch)]
    pool, opools = _long_pool(kvq, wl, sampled)
    q = wl.query()
    from concurrent.futures import ThreadPoolExecutor
    g1 = oracle.geom(num_blocks=wl.num_blocks, num_kv_heads=1)

    def want_of(bh):
        b, h = bh
        qh = np.ascontiguousarray(q[b:b + 1, h * G:(h + 1) * G])
        return oracle.decode_attention(g1, opools[bh], qh, wl.dtype, wl.block_table[b:b + 1], wl.seq_lens[b:b + 1],
                                       nthreads=1)[0]

    with ThreadPoolExecutor(min(len(sampled), helpers.threads())) as ex:
        wants = dict(zip(sampled, ex.map(want_of, sampled)))
    for bps in (0, 1024):
        got = _decode(kvq, wl, pool, q, bps=bps)
        assert np.all(np.isfinite(got))
        worst = max(float(np.max(np.abs(got[b, h * G:(h + 1) * G] - w))) for (b, h), w in wants.items())
        print(f"\nlong 8 x 131072, blocks per split {bps}: 64 sampled pairs max abs err {worst:.2e}")
        assert worst <= helpers.ATTN_TOL


def test_full_size_mixed_step(kvq, cuda):
    """The mixed write + read step: 64 sequences of 8192 cached tokens, one
    new token per sequence appended and read in the same fused launch (the
    benchmarked step).  Every appended token-head's codes against the oracle;
    the other cached tokens are the oracle's; all 4096 (b, j) pairs against
    the oracle's folded form and 64 seeded pairs (8 sequences, distinct kv
    heads) against its plain definition.  Then the separate prefill pass
    (16 x 16384 fresh tokens) through the bulk write path: a seeded sample
    of 65536 token-heads against the oracle."""
    torch = _torch()
    wl = synth.mixed_decode(0)
    T = wl.total_tokens
    k = wl.kv_rows(synth.TID_K, 0, T)
    v = wl.kv_rows(synth.TID_V, 0, T)
    slots = wl.slots()
    last = _last_positions(wl)
    keep = np.setdiff1d(np.arange(T), last)
    g = oracle.geom(num_blocks=wl.num_blocks, num_kv_heads=wl.hkv)
    full = oracle.new_pool(g)
    helpers.oracle_append_threaded(g, full, k, v, wl.dtype, slots)
    # the cache before the step: the new tokens' code rows not written yet
    base = full.copy()
    bseg = base.reshape(wl.num_blocks, wl.hkv, 1664)
    for t in last:
        p, o = divmod(int(slots[t]), 16)
        bseg[p, :, o * 64:(o + 1) * 64] = 0x5A
        bseg[p, :, 1024 + o * 32:1024 + (o + 1) * 32] = 0x5A
    assert keep.size == T - wl.batch
    q = wl.query()
    dpool = torch.from_numpy(base).cuda()
    got = _decode(kvq, wl, dpool, q, fused=(k[last], v[last]))
    after = dpool.cpu().numpy()
    rep = helpers.QuantReport()
    helpers.compare_pools(rep, after, full, wl.num_blocks, wl.hkv, k, v, wl.dtype, slots, tokens=last)
    assert rep.vectors == 2 * wl.batch * wl.hkv
    assert rep.ok(), rep
    folded = oracle.decode_attention(g, full, q, wl.dtype, wl.block_table, wl.seq_lens, form=1,
                                     nthreads=helpers.threads())
    err = float(np.max(np.abs(got - folded)))
    print(f"\nmixed 64 x 8192 fused step: all pairs vs folded oracle {err:.2e}")
    assert err <= helpers.ATTN_TOL
    bs = np.random.default_rng(11).choice(wl.batch, 8, replace=False)
    worst = _plain_pairs(wl, full, q, got, [(int(b), h) for h, b in enumerate(bs)])
    print(f"mixed: 64 sampled pairs vs plain oracle {worst:.2e}")
    assert worst <= helpers.ATTN_TOL
    del dpool, base, full, k, v

    # the prefill pass: 16 x 16384 fresh tokens, shuffled slots
    pf = synth.Workload("prefill", 16, 64, 8, 128, [16384] * 16, 16, synth.BF16, 3, 10.0, 30.0, seed=3)
    T = pf.total_tokens
    kp = pf.kv_rows(synth.TID_K, 0, T)
    vp = pf.kv_rows(synth.TID_V, 0, T)
    sp = pf.slots()
    gpool = _gpu_write(kvq, pf, kp, vp, sp).cpu().numpy()
    sample = np.sort(np.random.default_rng(12).choice(T, 8192, replace=False))
    g2 = oracle.geom(num_blocks=pf.num_blocks, num_kv_heads=pf.hkv)
    op = oracle.new_pool(g2)
    helpers.oracle_append_threaded(g2, op, kp[sample], vp[sample], pf.dtype, sp[sample])
    rep = helpers.QuantReport()
    helpers.compare_pools(rep, gpool, op, pf.num_blocks, pf.hkv, kp, vp, pf.dtype, sp, tokens=sample)
    assert rep.vectors == 2 * sample.size * pf.hkv
    assert rep.ok(), rep
