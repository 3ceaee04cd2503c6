"""The decode entry point that allocates nothing.

Some callers cannot allocate device memory when they call the decode (an
allocator that forbids runtime allocations, a plugin that is handed only its
input and output buffers).  kvq_decode_attention_noalloc serves them from a
fixed scratch array inside the library.  This file runs last (pytest collects
files in name order) so that a failure here never hides the other tests, and
it passes both alone in a fresh process and after the other tests."""
import ctypes

import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu


def _setup(kvq):
    import torch
    wl = synth.Workload("na", 3, 16, 2, 128, [300, 17, 129], 16, synth.BF16, 3, 10.0, 30.0, seed=90, extra_blocks=2)
    g = oracle.geom(num_blocks=wl.num_blocks, num_kv_heads=wl.hkv)
    pool = oracle.new_pool(g)
    k = wl.kv_rows(synth.TID_K, 0, wl.total_tokens)
    v = wl.kv_rows(synth.TID_V, 0, wl.total_tokens)
    assert oracle.quantize_append(g, pool, k, v, wl.dtype, wl.slots()) == 0
    dev = torch.device("cuda:0")
    d = dict(pool=torch.from_numpy(pool).to(dev),
             q=torch.from_numpy(wl.query().view(np.int16)).to(dev).view(torch.bfloat16),
             bt=torch.from_numpy(wl.block_table).to(dev), sl=torch.from_numpy(wl.seq_lens).to(dev),
             msl=int(wl.seq_lens.max()))
    return wl, d


def test_noalloc_matches_workspace_entry_point_twice(kvq, cuda):
    import torch
    wl, d = _setup(kvq)
    ref = torch.empty((wl.batch, wl.hq, 128), dtype=torch.float32, device="cuda")
    ws = kvq.new_workspace(wl.num_blocks, wl.hkv, wl.batch, wl.hq, d["msl"])
    kvq.kvq_decode_attention(d["pool"], wl.num_blocks, wl.hkv, d["q"], d["bt"], d["sl"], d["msl"], ref, ws)
    L = kvq.lib()
    desc = kvq.make_desc(wl.num_blocks, wl.hkv, d["pool"])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):  # the second call sees the scratch the first one left behind
        out = torch.full((wl.batch, wl.hq, 128), float("nan"), dtype=torch.float32, device="cuda")
        rc = L.kvq_decode_attention_noalloc(ctypes.byref(desc), ctypes.c_void_p(d["q"].data_ptr()), kvq.KVQ_BF16,
                                            wl.batch, wl.hq, ctypes.c_void_p(d["bt"].data_ptr()), d["bt"].shape[1],
                                            ctypes.c_void_p(d["sl"].data_ptr()), d["msl"], ctypes.c_float(0.0),
                                            ctypes.c_void_p(out.data_ptr()), kvq.KVQ_F32, stream)
        assert rc == kvq.KVQ_OK
        assert kvq.kvq_last_device_status() == 0
        diff = (out - ref).abs().max().item()
        assert diff <= 2e-3, diff


def test_noalloc_rejects_problems_beyond_its_scratch(kvq, cuda):
    import torch
    wl, d = _setup(kvq)
    big_batch = 4096  # 4096 x 16 query heads x >= 1 split x 528 B > 32 MiB
    L = kvq.lib()
    desc = kvq.make_desc(wl.num_blocks, wl.hkv, d["pool"])
    out = torch.empty(1, dtype=torch.float32, device="cuda")
    rc = L.kvq_decode_attention_noalloc(ctypes.byref(desc), ctypes.c_void_p(d["q"].data_ptr()), kvq.KVQ_BF16,
                                        big_batch, wl.hq, ctypes.c_void_p(d["bt"].data_ptr()), d["bt"].shape[1],
                                        ctypes.c_void_p(d["sl"].data_ptr()), d["msl"], ctypes.c_float(0.0),
                                        ctypes.c_void_p(out.data_ptr()), kvq.KVQ_F32,
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == kvq.KVQ_ERR_WORKSPACE
