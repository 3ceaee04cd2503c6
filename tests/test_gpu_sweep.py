"""A seeded sweep of decode configurations against the CPU oracle: random
batch sizes, GQA groups, kv head counts, presets, ragged lengths (empty ones
included), split granularities, output dtypes and, in about half the cases, a
bf16 window of sink and recent tokens.  Each case is drawn from a fixed seed,
so a failure names a reproducible configuration; the rules are those of the
other decode parity tests (max abs 2e-3 against the oracle's double-precision
attention over oracle-written pools, plus 2^-8 relative for a bf16 output)."""
import numpy as np
import pytest

import helpers
import oracle
import synth

pytestmark = pytest.mark.gpu

PRESETS = [(4, 2), (4, 4), (2, 2), (8, 4)]
N_CASES = 24


def _case(i):
    r = np.random.default_rng(1000 + i)
    G = int(r.choice([1, 2, 4, 8]))
    hkv = int(r.choice([1, 2, 4]))
    batch = int(r.integers(1, 6))
    lens = [int(x) for x in r.integers(0, 3000, size=batch)]
    if r.random() < 0.3:
        lens[int(r.integers(0, batch))] = 0
    preset = PRESETS[int(r.integers(0, len(PRESETS)))]
    window = None
    if r.random() < 0.5:
        window = (int(r.integers(0, 65)), int(r.choice([0, 1, 7, 64, 200, 1024])))
    bps = 0 if window else int(r.choice([0, 1, 2, 5, 64]))
    out = "bf16" if r.random() < 0.3 else "f32"
    return dict(G=G, hkv=hkv, lens=lens, preset=preset, window=window, bps=bps, out=out, seed=200 + i)


@pytest.mark.parametrize("i", range(N_CASES))
def test_decode_sweep(kvq, cuda, i):
    import torch
    c = _case(i)
    wl = synth.Workload("s", len(c["lens"]), c["G"] * c["hkv"], c["hkv"], 128, c["lens"], 16, synth.BF16, 3, 10.0,
                        30.0, seed=c["seed"], extra_blocks=2)
    g = oracle.geom(num_blocks=wl.num_blocks, num_kv_heads=wl.hkv, k_bits=c["preset"][0], v_bits=c["preset"][1])
    pool_np = oracle.new_pool(g)
    k = wl.kv_rows(synth.TID_K, 0, wl.total_tokens)
    v = wl.kv_rows(synth.TID_V, 0, wl.total_tokens)
    assert oracle.quantize_append(g, pool_np, k, v, wl.dtype, wl.slots()) == 0
    q_np = wl.query()
    pool = torch.from_numpy(pool_np).cuda()
    q = torch.from_numpy(np.ascontiguousarray(q_np).view(np.int16)).cuda().view(torch.bfloat16)
    bt = torch.from_numpy(wl.block_table).cuda()
    sl = torch.from_numpy(wl.seq_lens).cuda()
    msl = max(int(wl.seq_lens.max()), 1)
    out = torch.empty((wl.batch, wl.hq, 128), dtype=torch.float32 if c["out"] == "f32" else torch.bfloat16,
                      device="cuda")
    if c["window"]:
        sink, recent = c["window"]
        win_np = oracle.new_window(wl.batch, wl.hkv, sink, recent)
        for b in range(wl.batch):
            L = int(wl.seq_lens[b])
            rows = wl.token_offsets[b] + np.arange(L)
            oracle.window_append(win_np, sink, recent, k[rows], v[rows], [b] * L, list(range(L)))
        win = torch.from_numpy(win_np.view(np.int16)).cuda().view(torch.bfloat16)
        ws = kvq.new_window_workspace(wl.num_blocks, wl.hkv, wl.batch, wl.hq, msl, preset=c["preset"])
        kvq.kvq_decode_attention_window(pool, wl.num_blocks, wl.hkv, win, sink, recent, q, bt, sl, msl, out, ws,
                                        preset=c["preset"])
        want = oracle.decode_attention_window(g, pool_np, win_np, sink, recent, q_np, wl.dtype, wl.block_table,
                                              wl.seq_lens, nthreads=8)
    else:
        ws = kvq.new_workspace(wl.num_blocks, wl.hkv, wl.batch, wl.hq, msl, c["bps"], preset=c["preset"])
        kvq.kvq_decode_attention(pool, wl.num_blocks, wl.hkv, q, bt, sl, msl, out, ws, blocks_per_split=c["bps"],
                                 preset=c["preset"])
        want = oracle.decode_attention(g, pool_np, q_np, wl.dtype, wl.block_table, wl.seq_lens, nthreads=8)
    torch.cuda.synchronize()
    assert kvq.kvq_last_device_status() == 0, c
    got = out.float().cpu().numpy().astype(np.float64)
    rel = 2.0 ** -8 if c["out"] == "bf16" else 0.0
    assert np.all(np.isfinite(got)), c
    excess = np.abs(got - want) - (helpers.ATTN_TOL + rel * np.abs(want))
    assert excess.max() <= 0, (c, float(np.max(np.abs(got - want))))
    for b in range(wl.batch):
        if wl.seq_lens[b] == 0:
            assert not got[b].any(), c
