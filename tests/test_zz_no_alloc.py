"""attn_decode_paged_noalloc: the decode entry point for callers that cannot allocate device
memory at call time (for example a plugin whose host framework owns the device memory pool, or a
serving loop that cannot afford cudaMalloc's device-wide synchronisation). Its scratch is a
fixed array inside the library.

The test calls it through the C ABI and checks it against attn_decode_paged, which takes a
caller workspace, on calls in a row with different inputs: the two run the same kernels with the
same launch shapes on the same inputs, so their outputs must agree bit for bit (and therefore
within the parity tolerance as well). The second call shows that the scratch left behind by the
first does not leak into the result, and a third call repeats the first input and must reproduce
the first result exactly. It runs alone in a fresh process or after the other tests (the first
call on the device sets the scratch up). This file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from exact_attention_161_b200 import synth
from parity import assert_close, f64

pytestmark = pytest.mark.gpu


def _noalloc_call(api, cache_dev, o, lse):
    q, kp, vp, bt, sl = cache_dev
    S, Hq, D = q.shape
    num_pages, Hkv, page_size, _ = kp.shape
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    return api.lib.attn_decode_paged_noalloc(ptr(q), ptr(kp), ptr(vp), ptr(bt), ptr(sl), S, bt.shape[1], num_pages,
                                             page_size, Hq, Hkv, D, 0.0, ptr(o), ptr(lse),
                                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _to_dev(cache):
    return [cache.q.cuda(), cache.k_pages.cuda(), cache.v_pages.cuda(), cache.block_table.cuda(),
            cache.seq_lens.cuda()]


def _same_bits(a, b):
    if a.dtype == torch.bfloat16:
        return torch.equal(a.view(torch.int16), b.view(torch.int16))
    return torch.equal(a.view(torch.int32), b.view(torch.int32))


def test_noalloc_matches_workspace_entry_point_on_two_calls(cuda_api):
    caches = [
        synth.paged_decode_inputs(9, 32, 8, 128, 16, seq_lens=[1, 15, 16, 17, 511, 512, 513, 4000, 9000],
                                  seed=31),
        synth.paged_decode_inputs(5, 8, 2, 128, 16, seq_lens=[700, 3, 2048, 64, 1500], seed=32),
    ]
    outs = []
    for cache in caches + caches[:1]:  # the third call repeats the first input
        dev = _to_dev(cache)
        o_ref, lse_ref = cuda_api.attn_decode_paged(*dev)
        o = torch.empty_like(o_ref)
        lse = torch.empty_like(lse_ref)
        st = _noalloc_call(cuda_api, dev, o, lse)
        assert st == cuda_api.ATTN_OK, cuda_api.last_error()
        torch.cuda.synchronize()
        assert cuda_api.device_status() == 0
        assert_close(f64(o), f64(lse), f64(o_ref), f64(lse_ref), "no-alloc vs workspace decode")
        assert _same_bits(o, o_ref) and _same_bits(lse, lse_ref), "no-alloc output differs from the workspace call"
        outs.append((o, lse))
    assert _same_bits(outs[2][0], outs[0][0]) and _same_bits(outs[2][1], outs[0][1])


def test_noalloc_rejects_requests_beyond_its_scratch(cuda_api):
    # 2048 sequences x 32 heads x 32 splits x (128 + 2) floats > 40 MiB: rejected before any launch
    fake = ctypes.c_void_p(0x10000)
    st = cuda_api.lib.attn_decode_paged_noalloc(fake, fake, fake, fake, fake, 2048, 1024, 100, 16, 32, 8, 128, 0.0,
                                                fake, None, None)
    assert st == cuda_api.ATTN_ERR_INVALID_ARG
    assert "no-alloc limit" in cuda_api.last_error()
