"""The C-ABI library loads without a GPU, exports every symbol include/kvq.h
declares, and its host-only entry points and argument checks behave as
documented.  No kernel is launched here."""
import ctypes

import numpy as np
import pytest


def test_every_declared_symbol_is_exported(kvq):
    names = kvq.header_functions()
    assert "kvq_quantize_append" in names and "kvq_decode_attention" in names and "kvq_block_table" in names
    raw = ctypes.CDLL(kvq.LIB_PATH)
    missing = [n for n in names if not hasattr(raw, n)]
    assert not missing, missing


def test_parse_dtype(kvq):
    assert kvq.kvq_parse_dtype("kvarn_k4v2_g128") == (0, (4, 2, 128))
    # the other presets built: the same kernels at other bit widths
    for kb, vb in ((4, 4), (2, 2), (8, 4)):
        assert kvq.kvq_parse_dtype(f"kvarn_k{kb}v{vb}_g128") == (0, (kb, vb, 128))
    # well formed but not built: other widths, other groups
    for s, parsed in (("kvarn_k8v8_g128", (8, 8, 128)), ("kvarn_k4v2_g64", (4, 2, 64)),
                      ("kvarn_k3v2_g128", (3, 2, 128))):
        rc, got = kvq.kvq_parse_dtype(s)
        assert rc == kvq.KVQ_ERR_UNSUPPORTED and got == parsed
    for bad in ("fp8", "kvarn_k4v2_g128x", "kvarn_k4v2", "kvarn_kv2_g128", ""):
        assert kvq.kvq_parse_dtype(bad)[0] == kvq.KVQ_ERR_INVALID


def test_error_strings(kvq):
    for code in range(0, -8, -1):
        assert kvq.kvq_error_string(code)
    assert kvq.kvq_error_string(-99) == "unknown status"


def test_cache_bytes(kvq):
    assert kvq.kvq_cache_bytes(kvq.make_desc(1024, 8)) == 1024 * 8 * 1664
    # segment = 16 rows of K and V codes + 4 x 16 fp16 factors
    for (kb, vb), seg in (((4, 4), 2176), ((2, 2), 1152), ((8, 4), 3200)):
        assert seg == 16 * 128 * (kb + vb) // 8 + 128
        assert kvq.kvq_cache_bytes(kvq.make_desc(10, 3, preset=(kb, vb))) == 10 * 3 * seg
    assert kvq.kvq_cache_bytes(kvq.make_desc(10, 3, preset=(8, 8))) == 0
    d = kvq.make_desc(4, 2)
    d.head_dim = 64
    assert kvq.kvq_cache_bytes(d) == 0
    # 104 bytes per token per kv head: 64 B of 4-bit keys, 32 B of 2-bit values, 4 fp16
    assert 1664 / 16 == 104


def test_block_table_identity_and_shuffle(kvq):
    lens = [40, 0, 16, 17]
    bt, used = kvq.kvq_block_table(10, lens, 4, shuffle_seed=0)
    assert used == 3 + 0 + 1 + 2
    assert bt.tolist() == [[0, 1, 2, -1], [-1] * 4, [3, -1, -1, -1], [4, 5, -1, -1]]
    bt2, used2 = kvq.kvq_block_table(10, lens, 4, shuffle_seed=1234)
    assert used2 == used
    flat = bt2[bt2 >= 0]
    assert len(set(flat.tolist())) == used and flat.min() >= 0 and flat.max() < 10
    assert (bt2 >= 0).tolist() == (bt >= 0).tolist()
    again, _ = kvq.kvq_block_table(10, lens, 4, shuffle_seed=1234)
    assert np.array_equal(bt2, again)


def test_block_table_errors(kvq):
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_block_table(2, [40], 4)
    assert e.value.status == kvq.KVQ_ERR_POOL_EXHAUSTED
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_block_table(100, [80], 4)
    assert e.value.status == kvq.KVQ_ERR_INVALID


def test_slot_mapping(kvq):
    bt = np.array([[7, 3, -1], [5, -1, -1]], dtype=np.int32)
    slots = kvq.kvq_slot_mapping(bt, positions=[0, 15, 16, 31, 2, 16], seq_ids=[0, 0, 0, 0, 1, 1])
    assert slots.tolist() == [112, 127, 48, 63, 82, -1]
    with pytest.raises(kvq.KvqError):
        kvq.kvq_slot_mapping(bt, positions=[48], seq_ids=[0])


def test_argument_checks_need_no_device(kvq):
    L = kvq.lib()
    d = kvq.make_desc(4, 2)
    # null pool / inputs
    assert L.kvq_quantize_append(ctypes.byref(d), None, None, kvq.KVQ_BF16, 1, 256, None, None) == kvq.KVQ_ERR_INVALID
    # zero tokens is a no-op even with null pointers
    assert L.kvq_quantize_append(ctypes.byref(d), None, None, kvq.KVQ_BF16, 0, 256, None, None) == kvq.KVQ_OK
    # fp32 cache input is not a supported write dtype
    assert L.kvq_quantize_append(ctypes.byref(d), None, None, kvq.KVQ_F32, 1, 256, None, None) == kvq.KVQ_ERR_UNSUPPORTED
    # misaligned pointers
    d.pool = 0x1000
    assert L.kvq_quantize_append(ctypes.byref(d), ctypes.c_void_p(0x1008), ctypes.c_void_p(0x2000), kvq.KVQ_BF16, 1,
                                 256, ctypes.c_void_p(0x3000), None) == kvq.KVQ_ERR_INVALID
    # token stride shorter than a row
    assert L.kvq_quantize_append(ctypes.byref(d), ctypes.c_void_p(0x1000), ctypes.c_void_p(0x2000), kvq.KVQ_BF16, 1,
                                 128, ctypes.c_void_p(0x3000), None) == kvq.KVQ_ERR_INVALID
    # unsupported GQA group (24 / 8 = 3) and a non-multiple
    args = (ctypes.c_void_p(0x1000), kvq.KVQ_BF16, 1)
    assert L.kvq_decode_attention(ctypes.byref(d), *args, 6, None, 1, None, 16, 0.0, None, kvq.KVQ_F32, None, 0,
                                  None) == kvq.KVQ_ERR_UNSUPPORTED
    assert L.kvq_decode_attention(ctypes.byref(d), *args, 3, None, 1, None, 16, 0.0, None, kvq.KVQ_F32, None, 0,
                                  None) == kvq.KVQ_ERR_UNSUPPORTED
    # missing workspace
    one = ctypes.c_void_p(0x4000)
    assert L.kvq_decode_attention(ctypes.byref(d), *args, 2, one, 1, one, 16, 0.0, one, kvq.KVQ_F32, None, 0,
                                  None) == kvq.KVQ_ERR_WORKSPACE
    # bad head dim
    d.head_dim = 64
    assert L.kvq_decode_attention(ctypes.byref(d), *args, 2, one, 1, one, 16, 0.0, one, kvq.KVQ_F32, one, 1 << 20,
                                  None) == kvq.KVQ_ERR_UNSUPPORTED


def test_fused_and_noalloc_argument_checks_need_no_device(kvq):
    L = kvq.lib()
    d = kvq.make_desc(4, 2)
    d.pool = 0x1000
    one = ctypes.c_void_p(0x4000)
    k_new, v_new = ctypes.c_void_p(0x5000), ctypes.c_void_p(0x6000)

    def fused(k, v, in_dtype, stride, batch):
        return L.kvq_append_decode_attention(ctypes.byref(d), k, v, in_dtype, stride, one, kvq.KVQ_BF16, batch, 16,
                                             one, 1, one, 16, 0.0, one, kvq.KVQ_F32, None, 0, None)

    # the new rows: fp16/bf16 only, present, 16-byte aligned, a stride that holds a row
    assert fused(k_new, v_new, kvq.KVQ_F32, 256, 1) == kvq.KVQ_ERR_INVALID
    assert fused(None, v_new, kvq.KVQ_BF16, 256, 1) == kvq.KVQ_ERR_INVALID
    assert fused(ctypes.c_void_p(0x5008), v_new, kvq.KVQ_BF16, 256, 1) == kvq.KVQ_ERR_INVALID
    assert fused(k_new, v_new, kvq.KVQ_BF16, 128, 1) == kvq.KVQ_ERR_INVALID
    assert fused(k_new, v_new, kvq.KVQ_BF16, 260, 1) == kvq.KVQ_ERR_INVALID
    # then the decode rules: here the missing workspace
    assert fused(k_new, v_new, kvq.KVQ_BF16, 256, 1) == kvq.KVQ_ERR_WORKSPACE
    # an empty batch launches nothing
    assert fused(None, None, kvq.KVQ_BF16, 256, 0) == kvq.KVQ_OK
    # no-allocation entry point: an empty batch is a no-op; a head count that
    # the kv heads do not divide gets the same code as from kvq_decode_attention
    assert L.kvq_decode_attention_noalloc(ctypes.byref(d), one, kvq.KVQ_BF16, 0, 16, one, 1, one, 16, 0.0, one,
                                          kvq.KVQ_F32, None) == kvq.KVQ_OK
    assert L.kvq_decode_attention_noalloc(ctypes.byref(d), one, kvq.KVQ_BF16, 1, 15, one, 1, one, 16, 0.0, one,
                                          kvq.KVQ_F32, None) == kvq.KVQ_ERR_UNSUPPORTED
    assert L.kvq_decode_attention(ctypes.byref(d), one, kvq.KVQ_BF16, 1, 15, one, 1, one, 16, 0.0, one,
                                  kvq.KVQ_F32, one, 1 << 20, None) == kvq.KVQ_ERR_UNSUPPORTED
    assert L.kvq_decode_attention_noalloc(ctypes.byref(d), one, kvq.KVQ_BF16, -1, 16, one, 1, one, 16, 0.0, one,
                                          kvq.KVQ_F32, None) == kvq.KVQ_ERR_INVALID


@pytest.mark.parametrize("kb,vb", [(8, 8), (3, 2), (4, 1)])
def test_unsupported_presets_are_rejected_before_any_launch(kvq, kb, vb):
    L = kvq.lib()
    d = kvq.make_desc(4, 2)
    d.k_bits, d.v_bits = kb, vb
    d.pool = 0x1000
    one = ctypes.c_void_p(0x4000)
    assert L.kvq_cache_bytes(ctypes.byref(d)) == 0
    assert L.kvq_quantize_append(ctypes.byref(d), one, one, kvq.KVQ_BF16, 1, 256, one, None) == kvq.KVQ_ERR_UNSUPPORTED
    assert L.kvq_decode_attention(ctypes.byref(d), one, kvq.KVQ_BF16, 1, 16, one, 1, one, 16, 0.0, one, kvq.KVQ_F32,
                                  one, 1 << 20, None) == kvq.KVQ_ERR_UNSUPPORTED
    assert L.kvq_decode_workspace_bytes(ctypes.byref(d), 1, 16, 16) == 0


@pytest.mark.parametrize("preset", [(4, 2), (4, 4), (2, 2), (8, 4)])
def test_workspace_bytes_do_not_depend_on_the_preset(kvq, preset):
    """The split-K partials hold fp32 (o~, m, l) per query head and split,
    whatever the code widths."""
    assert kvq.kvq_decode_workspace_bytes(1024, 8, 1, 64, 16384, blocks_per_split=1024, preset=preset) == \
        256 + 64 * 1 * 132 * 4


def test_split_length_is_capped(kvq):
    """A decode CTA stages its split's block ids in shared memory, 1024 of
    them: a requested split longer than 1024 blocks (16384 tokens) is cut
    further; at most 256 splits, so a sequence beyond 256 x 1024 blocks is
    not supported (the workspace query returns 0); the workspace holds one
    partial record per query head and split."""
    rec = 64 * 132 * 4
    assert kvq.kvq_decode_workspace_bytes(8192, 8, 1, 64, 131072, blocks_per_split=8192) == 256 + 8 * rec
    assert kvq.kvq_decode_workspace_bytes(8192, 8, 1, 64, 131072, blocks_per_split=1024) == 256 + 8 * rec
    assert kvq.kvq_decode_workspace_bytes(8192, 8, 1, 64, 131072, blocks_per_split=512) == 256 + 16 * rec
    # 16384 tokens = 1024 blocks still fit in one split; one block more does not
    assert kvq.kvq_decode_workspace_bytes(1024, 8, 1, 64, 16384, blocks_per_split=1024) == 256 + 1 * rec
    assert kvq.kvq_decode_workspace_bytes(1025, 8, 1, 64, 16400, blocks_per_split=1025) == 256 + 2 * rec
    # too few splits requested: raised to what 256 splits of 1024 blocks allow
    longest = 256 * 1024 * 16
    assert kvq.kvq_decode_workspace_bytes(1, 8, 1, 64, longest, blocks_per_split=100000) == 256 + 256 * rec
    assert kvq.kvq_decode_workspace_bytes(1, 8, 1, 64, longest + 16, blocks_per_split=0) == 0
    # the default plan obeys the same bound
    n_default = (kvq.kvq_decode_workspace_bytes(8192, 8, 1, 64, 131072) - 256) // rec
    assert n_default >= 8


def test_workspace_bytes(kvq):
    n = kvq.kvq_decode_workspace_bytes(1024, 8, 1, 64, 16384)
    assert n > 0 and n % 4 == 0
    n1 = kvq.kvq_decode_workspace_bytes(1024, 8, 1, 64, 16384, blocks_per_split=1024)
    assert n1 == 256 + 64 * 1 * 132 * 4
    assert kvq.kvq_decode_workspace_bytes(1024, 8, 1, 60, 16384) == 0


def test_selftest_rejects_limits_out_of_range(kvq):
    """Checked on the host, before anything is launched: 1 us .. 1 s."""
    L = kvq.lib()
    assert L.kvq_selftest_wait_timeout(0, None, None) == kvq.KVQ_ERR_INVALID
    assert L.kvq_selftest_wait_timeout(1000001, None, None) == kvq.KVQ_ERR_INVALID


def test_window_argument_checks_need_no_device(kvq):
    """The bf16 window of sink and recent tokens: buffer size, limits (sink
    <= 64, recent <= 1024), row pointers and strides, the extra record of the
    window decode's workspace, and the descriptor rules of the window decode;
    all checked on the host before anything is launched."""
    L = kvq.lib()
    assert kvq.kvq_window_bytes(2, 8, 4, 128) == 2 * 8 * 132 * 2 * 128 * 2
    assert kvq.kvq_window_bytes(3, 1, 64, 1024) == 3 * 1088 * 512
    for bad in ((2, 8, 65, 0), (2, 8, 0, 1025), (2, 8, -1, 4), (2, 0, 4, 4), (-1, 8, 4, 4)):
        assert kvq.kvq_window_bytes(*bad) == 0, bad
    w = kvq.make_window(2, 2, 4, 16)
    w.data = 0x10000
    one = ctypes.c_void_p(0x4000)
    k, v = ctypes.c_void_p(0x5000), ctypes.c_void_p(0x6000)

    def append(win, kk, vv, stride, n):
        return L.kvq_window_append(ctypes.byref(win), kk, vv, stride, one, one, n, None)

    assert append(w, None, None, 256, 0) == kvq.KVQ_OK  # nothing to copy
    assert append(w, None, v, 256, 1) == kvq.KVQ_ERR_INVALID
    assert append(w, ctypes.c_void_p(0x5008), v, 256, 1) == kvq.KVQ_ERR_INVALID
    assert append(w, k, v, 128, 1) == kvq.KVQ_ERR_INVALID  # a row is 2 heads x 128
    assert append(w, k, v, 260, 1) == kvq.KVQ_ERR_INVALID  # not a multiple of 8
    assert append(w, k, v, 256, -1) == kvq.KVQ_ERR_INVALID
    bad = kvq.make_window(2, 2, 65, 16)
    bad.data = 0x10000
    assert append(bad, k, v, 256, 1) == kvq.KVQ_ERR_INVALID
    nodata = kvq.make_window(2, 2, 4, 16)
    assert append(nodata, k, v, 256, 1) == kvq.KVQ_ERR_INVALID
    misaligned = kvq.make_window(2, 2, 4, 16)
    misaligned.data = 0x10008
    assert append(misaligned, k, v, 256, 1) == kvq.KVQ_ERR_INVALID
    # the window decode's workspace holds one record more per query head
    d = kvq.make_desc(1024, 8)
    base = L.kvq_decode_workspace_bytes(ctypes.byref(d), 3, 64, 16384)
    assert L.kvq_decode_window_workspace_bytes(ctypes.byref(d), 3, 64, 16384) == base + 3 * 64 * 132 * 4
    # descriptor rules: kv heads must match the pool's, the batch must fit the window's sequences
    d = kvq.make_desc(4, 2)
    d.pool = 0x1000

    def decode(win, batch, ws, ws_bytes):
        return L.kvq_decode_attention_window(ctypes.byref(d), ctypes.byref(win), one, kvq.KVQ_BF16, batch, 16, one,
                                             1, one, 16, 0.0, one, kvq.KVQ_F32, ws, ws_bytes, None)

    w3 = kvq.make_window(2, 3, 4, 16)
    w3.data = 0x10000
    assert decode(w3, 1, None, 0) == kvq.KVQ_ERR_INVALID
    assert decode(w, 3, None, 0) == kvq.KVQ_ERR_INVALID
    assert decode(w, 1, None, 0) == kvq.KVQ_ERR_WORKSPACE
    assert decode(bad, 1, None, 0) == kvq.KVQ_ERR_INVALID
