"""Full-size parity of the Llama-3.1-70B-shaped long-context decode
(batch 8 x 131072 tokens, 64/8 heads), on one sampled (sequence, kv head).

The pool holds the full workload's geometry: every block is filled with
GPU-written segments of the seeded stream (the first 16384 tokens, repeated),
and the sampled sequence's blocks of the sampled kv head are replaced by the
oracle's bytes for that sequence's own 131072 tokens.  The GPU decodes the
whole batch in the benchmarked (default) split plan and with four splits per
sequence (one CTA walks 256 chunks, restarting its integer accumulator after
128); the sampled outputs are compared with the oracle's plain softmax
attention over the same bytes ("KVarN vs TurboQuant", dothoosh.com: the
read path folds the group scales into attention).
"""
import numpy as np
import pytest

import helpers
import oracle
import synth

pytestmark = pytest.mark.gpu

from test_gpu_parity import _dev_u16, _torch  # noqa: E402


def test_full_size_long_context_sampled_head(kvq, cuda):
    torch = _torch()
    wl = synth.long_context(0)
    G = wl.hq // wl.hkv
    b_s, h_s = 3, 5
    L = int(wl.seq_lens[b_s])
    off = int(wl.token_offsets[b_s])
    slots = wl.slots()

    # every block: GPU-written segments of the first 16384 tokens, repeated
    T0 = 16384
    nb0 = T0 // wl.bs
    k0 = wl.kv_rows(synth.TID_K, 0, T0)
    v0 = wl.kv_rows(synth.TID_V, 0, T0)
    base = kvq.new_pool(nb0, wl.hkv)
    kvq.kvq_quantize_append(base, nb0, wl.hkv, _dev_u16(k0, wl.dtype).reshape(T0, -1),
                            _dev_u16(v0, wl.dtype).reshape(T0, -1),
                            torch.arange(T0, dtype=torch.int32, device="cuda"))
    assert kvq.kvq_last_device_status() == 0
    del k0, v0
    pool = kvq.new_pool(wl.num_blocks, wl.hkv)
    seg = pool.view(wl.num_blocks, wl.hkv, 1664)
    b0 = base.view(nb0, wl.hkv, 1664)
    for s in range(0, wl.num_blocks, nb0):
        n = min(nb0, wl.num_blocks - s)
        seg[s:s + n].copy_(b0[:n])
    del base, b0

    # the sampled (sequence, kv head): the oracle's bytes for its own tokens
    k = wl.kv_rows(synth.TID_K, off, L)
    v = wl.kv_rows(synth.TID_V, off, L)
    ks = np.ascontiguousarray(k[:, h_s:h_s + 1])
    vs = np.ascontiguousarray(v[:, h_s:h_s + 1])
    del k, v
    g1 = oracle.geom(num_blocks=wl.num_blocks, num_kv_heads=1)
    opool = oracle.new_pool(g1)
    s_slots = np.ascontiguousarray(slots[off:off + L])
    assert oracle.quantize_append(g1, opool, ks, vs, wl.dtype, s_slots) == 0
    used = torch.from_numpy(np.unique(s_slots // wl.bs)).cuda().long()
    seg[used, h_s] = torch.from_numpy(opool.reshape(wl.num_blocks, 1664)).cuda()[used]

    q = wl.query()
    qh = np.ascontiguousarray(q[b_s:b_s + 1, h_s * G:(h_s + 1) * G])
    want = oracle.decode_attention(g1, opool, qh, wl.dtype, wl.block_table[b_s:b_s + 1], wl.seq_lens[b_s:b_s + 1],
                                   nthreads=8)[0]

    bt = torch.from_numpy(wl.block_table).cuda()
    lens = torch.from_numpy(wl.seq_lens).cuda()
    qd = _dev_u16(q, wl.dtype)
    for bps in (0, wl.max_blocks_per_seq // 4):
        out = torch.empty((wl.batch, wl.hq, 128), dtype=torch.float32, device="cuda")
        ws = kvq.new_workspace(wl.num_blocks, wl.hkv, wl.batch, wl.hq, L, bps)
        kvq.kvq_decode_attention(pool, wl.num_blocks, wl.hkv, qd, bt, lens, L, out, ws, blocks_per_split=bps)
        torch.cuda.synchronize()
        assert kvq.kvq_last_device_status() == 0
        got = out[b_s, h_s * G:(h_s + 1) * G].cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(out.cpu().numpy()))
        err = float(np.max(np.abs(got - want)))
        print(f"\nlong context 8 x 131072, blocks per split {bps}: sampled max abs err {err:.2e}")
        assert err <= helpers.ATTN_TOL
