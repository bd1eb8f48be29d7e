"""Failure detection on the GPU without a fault (GPU only).

Every mbarrier wait in the kernels is bounded (about 2 s of SM clocks) and watches a per-CTA abort
flag. Here the test hook attn_debug_drop_copy makes one copy of a kernel's first CTA never happen
while its bytes are still expected (a page of the decode split kernel, a key tile of the prefill
kernel, a query/dO tile of the backward kernel), so that wait runs out: the CTA raises the timeout
bit in the device status word, drains its own copies and returns, and the call ends. The next call
on the same context must work normally.
"""
import pytest
import torch

from exact_attention_161_b200 import synth
import oracle
from parity import assert_close, f64, oracle_decode, oracle_prefill
from test_parity_bwd import check_grad

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


def _with_dropped_copy(api, call):
    assert api.device_status() == 0
    api.debug_drop_copy(True)
    try:
        call()
        torch.cuda.synchronize()
    finally:
        api.debug_drop_copy(False)
    flags = api.device_status()
    assert flags & api.DEVICE_TIMEOUT
    assert api.device_status() == 0


def test_prefill_timeout_reported_and_context_survives(cuda_api):
    q, k, v = synth.prefill_inputs(1, 4, 2, 640, 128, seed=41)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    _with_dropped_copy(cuda_api, lambda: cuda_api.attn_fwd(qd, kd, vd, causal=True, rope_base=10000.0))
    o, lse = cuda_api.attn_fwd(qd, kd, vd, causal=True, rope_base=10000.0)
    torch.cuda.synchronize()
    assert cuda_api.device_status() == 0
    o_ref, lse_ref = oracle_prefill(q, k, v, True, 0, 10000.0, 128 ** -0.5)
    assert_close(f64(o), f64(lse), o_ref, lse_ref, "prefill after a timed-out call")


def test_backward_timeout_reported_and_context_survives(cuda_api):
    q, k, v = synth.prefill_inputs(1, 4, 2, 640, 128, seed=42)
    dout = synth.randn_bf16((1, 4, 640, 128), torch.Generator().manual_seed(43))
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    o, lse = cuda_api.attn_fwd(qd, kd, vd, causal=True, rope_base=10000.0)
    _with_dropped_copy(cuda_api, lambda: cuda_api.attn_bwd(qd, kd, vd, o, lse, dod, causal=True, rope_base=10000.0))
    dq, dk, dv = cuda_api.attn_bwd(qd, kd, vd, o, lse, dod, causal=True, rope_base=10000.0)
    torch.cuda.synchronize()
    assert cuda_api.device_status() == 0
    rq, rk, rv = oracle.attention_bwd(synth.bits(q), synth.bits(k), synth.bits(v), synth.bits(dout), causal=True,
                                      rope_base=10000.0, scale=128 ** -0.5)
    check_grad("dq", dq, rq)
    check_grad("dk", dk, rk)
    check_grad("dv", dv, rv)
