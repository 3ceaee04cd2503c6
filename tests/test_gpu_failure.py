"""Failure detection without a GPU fault.

Every device-side wait of the kernels is bounded: when it runs out, the
kernel records KVQ_ERR_DEVICE_TIMEOUT in the device status word, leaves
nothing of its own in flight and returns, so the context stays usable.  The
self-test entry point makes one such wait on a barrier that nothing ever
arrives at; this test watches the status come back and then runs a normal
decode in the same process against the oracle."""
import numpy as np
import pytest

import helpers
import oracle
import synth

pytestmark = pytest.mark.gpu

from test_gpu_parity import _dev_u16, _oracle_pool, _torch  # noqa: E402


def test_bounded_wait_gives_up_and_the_context_stays_usable(kvq, cuda):
    torch = _torch()
    assert kvq.kvq_last_device_status() in (0, kvq.KVQ_ERR_OUT_OF_RANGE)  # read and clear what came before
    elapsed = torch.zeros(1, dtype=torch.int64, device="cuda")
    for limit_us in (10, 2000):
        kvq.kvq_selftest_wait_timeout(limit_us, elapsed)
        assert kvq.kvq_last_device_status() == kvq.KVQ_ERR_DEVICE_TIMEOUT
        assert kvq.kvq_last_device_status() == 0  # read and clear
        print(f"\nbounded wait of {limit_us} us gave up after {elapsed.item() / 1e3:.1f} us")
        # it gave up no earlier than its limit, and not long after it
        assert limit_us * 1000 <= elapsed.item() <= limit_us * 1000 + 1_000_000
    # a normal decode afterwards, in the same context
    wl = synth.Workload("f", 2, 16, 2, 128, [200, 33], 16, synth.BF16, 3, 10.0, 30.0, seed=95)
    g, pool, _, _ = _oracle_pool(wl)
    q = wl.query()
    out = torch.empty((wl.batch, wl.hq, 128), dtype=torch.float32, device="cuda")
    ws = kvq.new_workspace(wl.num_blocks, wl.hkv, wl.batch, wl.hq, int(wl.seq_lens.max()))
    kvq.kvq_decode_attention(torch.from_numpy(pool).cuda(), wl.num_blocks, wl.hkv, _dev_u16(q, wl.dtype),
                             torch.from_numpy(wl.block_table).cuda(), torch.from_numpy(wl.seq_lens).cuda(),
                             int(wl.seq_lens.max()), out, ws)
    assert kvq.kvq_last_device_status() == 0
    want = oracle.decode_attention(g, pool, q, wl.dtype, wl.block_table, wl.seq_lens)
    assert np.max(np.abs(out.cpu().numpy().astype(np.float64) - want)) <= helpers.ATTN_TOL
