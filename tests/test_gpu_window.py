"""GPU parity of the bf16 window of sink and recent tokens ("Kompresja
pamięci podręcznej KV to decyzja infrastrukturalna..." (encorp.ai), OSCAR
section: the first and the most recent tokens stay in BF16, the history is
compressed).  The window append must write the same bytes as the oracle's;
the window decode must be within 2e-3 (max abs, fp32) of the oracle's
double-precision attention over the same pool and window, both written by the
oracle (no oracle input comes from the CUDA path)."""
import numpy as np
import pytest

import helpers
import oracle
import synth

pytestmark = pytest.mark.gpu


def _torch():
    import torch
    return torch


def _oracle_pool(wl, preset=(4, 2)):
    g = oracle.geom(num_blocks=wl.num_blocks, num_kv_heads=wl.hkv, k_bits=preset[0], v_bits=preset[1])
    pool = oracle.new_pool(g)
    k = wl.kv_rows(synth.TID_K, 0, wl.total_tokens)
    v = wl.kv_rows(synth.TID_V, 0, wl.total_tokens)
    assert oracle.quantize_append(g, pool, k, v, wl.dtype, wl.slots()) == 0
    return g, pool, k, v


def _oracle_window(wl, k, v, sink, recent):
    """Every token of every sequence appended in order, as a decode loop would."""
    win = oracle.new_window(wl.batch, wl.hkv, sink, recent)
    for b in range(wl.batch):
        L = int(wl.seq_lens[b])
        rows = wl.token_offsets[b] + np.arange(L)
        oracle.window_append(win, sink, recent, k[rows], v[rows], [b] * L, list(range(L)))
    return win


def _gpu_decode_window(kvq, wl, pool_np, win_np, sink, recent, q_np, out_dtype="f32", preset=(4, 2)):
    torch = _torch()
    pool = torch.from_numpy(pool_np).cuda()
    win = torch.from_numpy(win_np.view(np.int16)).cuda().view(torch.bfloat16)
    q = torch.from_numpy(np.ascontiguousarray(q_np).view(np.int16)).cuda().view(torch.bfloat16)
    bt = torch.from_numpy(wl.block_table).cuda()
    sl = torch.from_numpy(wl.seq_lens).cuda()
    msl = max(int(wl.seq_lens.max()), 1)
    out = torch.empty((wl.batch, wl.hq, 128), dtype={"f32": torch.float32, "bf16": torch.bfloat16}[out_dtype],
                      device="cuda")
    ws = kvq.new_window_workspace(wl.num_blocks, wl.hkv, wl.batch, wl.hq, msl, preset=preset)
    kvq.kvq_decode_attention_window(pool, wl.num_blocks, wl.hkv, win, sink, recent, q, bt, sl, msl, out, ws,
                                    preset=preset)
    torch.cuda.synchronize()
    assert kvq.kvq_last_device_status() == 0
    return out.float().cpu().numpy().astype(np.float64)


def _check(wl, g, pool, win, sink, recent, q, got, rel=0.0):
    want = oracle.decode_attention_window(g, pool, win, sink, recent, q, wl.dtype, wl.block_table, wl.seq_lens,
                                          nthreads=8)
    assert np.all(np.isfinite(got))
    excess = np.abs(got - want) - (helpers.ATTN_TOL + rel * np.abs(want))
    assert excess.max() <= 0, (np.max(np.abs(got - want)), excess.max())
    return want


# lengths across the sink, the recent window and block and chunk boundaries
_RAGGED = [1, 15, 16, 17, 300, 0, 2100]


@pytest.mark.parametrize("sink,recent", [(4, 64), (0, 128), (16, 0), (3, 7), (64, 1024), (0, 0)])
def test_window_decode_ragged(kvq, cuda, sink, recent):
    wl = synth.Workload("w", len(_RAGGED), 16, 2, 128, _RAGGED, 16, synth.BF16, 3, 10.0, 30.0, seed=61,
                        extra_blocks=3)
    g, pool, k, v = _oracle_pool(wl)
    win = _oracle_window(wl, k, v, sink, recent)
    q = wl.query()
    got = _gpu_decode_window(kvq, wl, pool, win, sink, recent, q)
    _check(wl, g, pool, win, sink, recent, q, got)
    assert not got[5].any()  # length 0 -> zeros


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_window_decode_group_sizes(kvq, cuda, G):
    wl = synth.Workload("wg", 2, 2 * G, 2, 128, [777, 130], 16, synth.BF16, 3, 10.0, 30.0, seed=70 + G)
    g, pool, k, v = _oracle_pool(wl)
    win = _oracle_window(wl, k, v, 4, 100)
    q = wl.query()
    got = _gpu_decode_window(kvq, wl, pool, win, 4, 100, q)
    _check(wl, g, pool, win, 4, 100, q, got)


@pytest.mark.parametrize("preset", [(4, 4), (2, 2), (8, 4)])
def test_window_decode_presets(kvq, cuda, preset):
    """The other presets: the same window CTA and masking over pools of other widths."""
    wl = synth.Workload("wp", 3, 16, 2, 128, [900, 40, 2], 16, synth.BF16, 3, 10.0, 30.0, seed=90 + preset[0])
    g, pool, k, v = _oracle_pool(wl, preset)
    win = _oracle_window(wl, k, v, 4, 64)
    q = wl.query()
    got = _gpu_decode_window(kvq, wl, pool, win, 4, 64, q, preset=preset)
    _check(wl, g, pool, win, 4, 64, q, got)


def test_window_decode_f32_query(kvq, cuda):
    """fp32 queries (the window CTA and the split CTAs read q in its own dtype)."""
    torch = _torch()
    wl = synth.Workload("wq", 2, 16, 2, 128, [700, 90], 16, synth.BF16, 3, 10.0, 30.0, seed=95)
    g, pool_np, k, v = _oracle_pool(wl)
    win_np = _oracle_window(wl, k, v, 4, 64)
    q_np = synth.normal(95, synth.TID_Q, wl.batch * wl.hq * 128, synth.F32).reshape(wl.batch, wl.hq, 128)
    pool = torch.from_numpy(pool_np).cuda()
    win = torch.from_numpy(win_np.view(np.int16)).cuda().view(torch.bfloat16)
    q = torch.from_numpy(np.ascontiguousarray(q_np, dtype=np.float32)).cuda()
    bt = torch.from_numpy(wl.block_table).cuda()
    sl = torch.from_numpy(wl.seq_lens).cuda()
    msl = int(wl.seq_lens.max())
    out = torch.empty((wl.batch, wl.hq, 128), dtype=torch.float32, device="cuda")
    ws = kvq.new_window_workspace(wl.num_blocks, wl.hkv, wl.batch, wl.hq, msl)
    kvq.kvq_decode_attention_window(pool, wl.num_blocks, wl.hkv, win, 4, 64, q, bt, sl, msl, out, ws)
    torch.cuda.synchronize()
    assert kvq.kvq_last_device_status() == 0
    want = oracle.decode_attention_window(g, pool_np, win_np, 4, 64, q_np, synth.F32, wl.block_table, wl.seq_lens,
                                          nthreads=8)
    got = out.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(got - want)) <= helpers.ATTN_TOL


def test_window_decode_bf16_output(kvq, cuda):
    wl = synth.Workload("wb", 3, 32, 4, 128, [5000, 64, 129], 16, synth.BF16, 3, 10.0, 30.0, seed=77)
    g, pool, k, v = _oracle_pool(wl)
    win = _oracle_window(wl, k, v, 8, 256)
    q = wl.query()
    got = _gpu_decode_window(kvq, wl, pool, win, 8, 256, q, out_dtype="bf16")
    _check(wl, g, pool, win, 8, 256, q, got, rel=2.0 ** -8)


def test_window_decode_full_size_qwen3_32b_layer(kvq, cuda):
    """The Qwen3-32B-shaped layer (16K tokens, 64/8 heads) with 4 sink and
    128 recent tokens: all 64 query heads against the oracle."""
    wl = synth.qwen3_32b_layer(0)
    g, pool, k, v = _oracle_pool(wl)
    win = _oracle_window(wl, k, v, 4, 128)
    q = wl.query()
    got = _gpu_decode_window(kvq, wl, pool, win, 4, 128, q)
    want = _check(wl, g, pool, win, 4, 128, q, got)
    # the window changes the result: the same call without it reads the quantized rows
    plain = oracle.decode_attention(g, pool, q, wl.dtype, wl.block_table, wl.seq_lens, nthreads=8)
    assert np.max(np.abs(plain - want)) > 1e-4


def test_window_append_matches_oracle(kvq, cuda):
    """Tokens of several sequences in one call, in no particular order, each
    to distinct rows; then a call with a sequence id out of range writes
    nothing and records KVQ_ERR_OUT_OF_RANGE."""
    torch = _torch()
    hkv, sink, recent, nseq = 3, 5, 9, 4
    n = nseq * recent
    rows = synth.kv(81, synth.TID_K, 0, n, hkv, 128, 3, 10.0, 30.0, synth.BF16)
    vrows = synth.kv(81, synth.TID_V, 0, n, hkv, 128, 3, 10.0, 30.0, synth.BF16)
    # (sequence, position) pairs whose sink and ring rows are all distinct
    pairs = [(s, t) for s in range(nseq) for t in range(recent)]
    order = np.random.default_rng(5).permutation(len(pairs))
    ids = np.array([pairs[i][0] for i in order], dtype=np.int32)
    pos = np.array([pairs[i][1] for i in order], dtype=np.int32)
    ids[7] = -1  # skipped
    want = oracle.new_window(nseq, hkv, sink, recent, fill=0x3F80)
    oracle.window_append(want, sink, recent, rows, vrows, ids, pos)
    win = torch.from_numpy(np.full(want.shape, 0x3F80, dtype=np.uint16).view(np.int16)).cuda().view(torch.bfloat16)
    k = torch.from_numpy(rows.reshape(n, -1).view(np.int16)).cuda().view(torch.bfloat16)
    v = torch.from_numpy(vrows.reshape(n, -1).view(np.int16)).cuda().view(torch.bfloat16)
    kvq.kvq_window_append(win, sink, recent, k, v, torch.from_numpy(ids).cuda(), torch.from_numpy(pos).cuda())
    torch.cuda.synchronize()
    assert kvq.kvq_last_device_status() == 0
    got = win.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, want)
    bad = torch.tensor([nseq], dtype=torch.int32, device="cuda")
    kvq.kvq_window_append(win, sink, recent, k[:1], v[:1], bad, torch.tensor([0], dtype=torch.int32, device="cuda"))
    assert kvq.kvq_last_device_status() == kvq.KVQ_ERR_OUT_OF_RANGE
    assert np.array_equal(win.view(torch.int16).cpu().numpy().view(np.uint16), want)
