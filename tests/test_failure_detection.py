"""Failure detection on the GPU without a fault (GPU only).

Every mbarrier wait in the kernels is bounded (about 2 s of SM clocks) and watches a per-CTA abort
flag. Here the test hook attn_debug_drop_copy makes one page copy of the decode split kernel never
happen while its bytes are still expected, so that wait runs out: the CTA raises the timeout bit in
the device status word, drains its own copies and returns, and the call ends. The next call on the
same context must work normally.
"""
import pytest
import torch

from exact_attention_161_b200 import synth
from parity import assert_close, f64, oracle_decode

pytestmark = pytest.mark.gpu


def _decode(api, cache):
    o, lse = api.attn_decode_paged(cache.q.cuda(), cache.k_pages.cuda(), cache.v_pages.cuda(),
                                   cache.block_table.cuda(), cache.seq_lens.cuda())
    torch.cuda.synchronize()
    return o, lse


def test_bounded_wait_reports_timeout_and_context_survives(cuda_api):
    cache = synth.paged_decode_inputs(2, 8, 2, 128, 16, seq_lens=[600, 100], seed=40)
    assert cuda_api.device_status() == 0
    cuda_api.debug_drop_copy(True)
    try:
        _decode(cuda_api, cache)
    finally:
        cuda_api.debug_drop_copy(False)
    flags = cuda_api.device_status()
    assert flags & cuda_api.DEVICE_TIMEOUT
    assert cuda_api.device_status() == 0  # reading clears the word
    o, lse = _decode(cuda_api, cache)
    assert cuda_api.device_status() == 0
    o_ref, lse_ref = oracle_decode(cache)
    assert_close(f64(o), f64(lse), o_ref, lse_ref, "decode after a timed-out call")
