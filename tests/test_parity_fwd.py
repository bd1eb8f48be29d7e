"""Prefill parity: the CUDA attention forward against the fp64 oracle (GPU only).

Small cases compare every element of O and LSE; they span several 128-row tiles and ragged
tails, GQA/MQA/MHA, causal, sliding-window and full masks, RoPE and no RoPE, D = 64 and 128.
The prefill workloads at full size run through the same call the benchmark times and are compared
on every element of O and every LSE.
"""
import numpy as np
import pytest
import torch

from exact_attention_161_b200 import synth
from parity import assert_close, f64, oracle_prefill, report

pytestmark = pytest.mark.gpu

# B, Hq, Hkv, N, D, causal, window, rope_base
SMALL = [
    (1, 1, 1, 128, 64, 0, 0, 0.0),          # the single-head N=128 d=64 workload's shape
    (1, 1, 1, 1, 64, 0, 0, 0.0),
    (1, 1, 1, 1, 128, 1, 0, 10000.0),
    (1, 2, 1, 17, 64, 1, 0, 10000.0),
    (1, 4, 1, 127, 128, 1, 0, 10000.0),
    (2, 2, 2, 129, 128, 0, 0, 0.0),
    (2, 3, 3, 257, 64, 1, 0, 0.0),
    (1, 8, 2, 300, 128, 1, 7, 10000.0),
    (1, 4, 4, 1000, 128, 1, 128, 500000.0),
    (1, 4, 1, 1000, 64, 1, 200, 10000.0),
    (1, 2, 2, 513, 128, 1, 1, 10000.0),     # window 1: each row sees only itself
    (1, 2, 1, 700, 128, 1, 4096, 10000.0),  # window >= N: plain causal
    (1, 2, 2, 640, 128, 0, 0, 10000.0),     # RoPE without a mask
    (1, 2, 2, 2048, 128, 1, 0, 10000.0),    # a two-head slice of the N=2048 MHA workload
    (1, 32, 8, 1024, 128, 1, 0, 500000.0),  # the GQA workload's heads at N=1024
]


def _ids(c):
    return "B%dHq%dHkv%dN%dD%d_c%d_w%d_r%g" % c


@pytest.mark.parametrize("case", SMALL, ids=_ids)
def test_small_all_rows(cuda_api, case):
    B, Hq, Hkv, N, D, causal, window, rope = case
    q, k, v = synth.prefill_inputs(B, Hq, Hkv, N, D, seed=100 + SMALL.index(case))
    scale = D ** -0.5
    o, lse = cuda_api.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, window=window, rope_base=rope)
    torch.cuda.synchronize()
    assert cuda_api.device_status() == 0
    o_ref, lse_ref = oracle_prefill(q, k, v, causal, window, rope, scale)
    assert_close(f64(o), f64(lse), o_ref, lse_ref, _ids(case))


def test_window_one_returns_values_exactly(cuda_api):
    """Window 1: the only visible key is the row itself, so O = V (bf16 round trip exact)."""
    q, k, v = synth.prefill_inputs(1, 4, 2, 300, 128, seed=5)
    o, _ = cuda_api.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True, window=1, rope_base=10000.0)
    vr = v.repeat_interleave(2, dim=1)
    assert torch.equal(o.cpu().view(torch.int16), vr.view(torch.int16))


def test_gqa_equals_repeated_kv(cuda_api):
    """GQA on Hkv heads gives the same bits as MHA on K/V repeated per group."""
    q, k, v = synth.prefill_inputs(1, 8, 2, 400, 128, seed=6)
    o1, l1 = cuda_api.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True, rope_base=10000.0)
    kr, vr = k.repeat_interleave(4, dim=1), v.repeat_interleave(4, dim=1)
    o2, l2 = cuda_api.attn_fwd(q.cuda(), kr.cuda(), vr.cuda(), causal=True, rope_base=10000.0)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)


def test_no_lse_pointer(cuda_api):
    q, k, v = synth.prefill_inputs(1, 2, 2, 200, 64, seed=7)
    o, lse = cuda_api.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True, want_lse=False)
    o2, _ = cuda_api.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
    assert lse is None and torch.equal(o.view(torch.int16), o2.view(torch.int16))


def test_deterministic_and_stream_independent(cuda_api):
    """Two calls, and a call on a side stream (which has its own rotation scratch), give the same
    bits: the work schedule is static and no result depends on timing."""
    q, k, v = (x.cuda() for x in synth.prefill_inputs(2, 8, 2, 1100, 128, seed=8))
    o1, l1 = cuda_api.attn_fwd(q, k, v, causal=True, rope_base=10000.0)
    o2, l2 = cuda_api.attn_fwd(q, k, v, causal=True, rope_base=10000.0)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        o3, l3 = torch.empty_like(o1), torch.empty_like(l1)
        cuda_api.attn_fwd(q, k, v, causal=True, rope_base=10000.0, o=o3, lse=l3, stream=side)
    side.synchronize()
    torch.cuda.synchronize()
    assert cuda_api.device_status() == 0
    for o, lse in ((o2, l2), (o3, l3)):
        assert torch.equal(o1.view(torch.int16), o.view(torch.int16)) and torch.equal(l1, lse)


def test_cache_growth_leaves_results_unchanged(cuda_api):
    """The RoPE tables and the rotation scratch are cached and grow on demand: a call repeated
    after larger calls (which regrow both) and a call with another base gives the same bits."""
    a = [x.cuda() for x in synth.prefill_inputs(1, 4, 2, 900, 128, seed=10)]
    b = [x.cuda() for x in synth.prefill_inputs(2, 4, 4, 3100, 128, seed=11)]
    o1, l1 = cuda_api.attn_fwd(*a, causal=True, rope_base=10000.0)
    cuda_api.attn_fwd(*b, causal=True, rope_base=10000.0)
    cuda_api.attn_fwd(*b, causal=True, rope_base=500000.0)
    o2, l2 = cuda_api.attn_fwd(*a, causal=True, rope_base=10000.0)
    torch.cuda.synchronize()
    assert cuda_api.device_status() == 0
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)


def test_explicit_scale(cuda_api):
    """A softmax scale other than 1/sqrt(D) (0.2 at D = 64, against the default 0.125)."""
    q, k, v = synth.prefill_inputs(1, 4, 2, 333, 64, seed=9)
    o, lse = cuda_api.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True, rope_base=10000.0, scale=0.2)
    torch.cuda.synchronize()
    assert cuda_api.device_status() == 0
    o_ref, lse_ref = oracle_prefill(q, k, v, 1, 0, 10000.0, 0.2)
    assert_close(f64(o), f64(lse), o_ref, lse_ref, "scale 0.2")


@pytest.mark.parametrize("cfg", synth.PREFILL_CONFIGS, ids=lambda c: c.name)
def test_workload_full_size_all_rows(cuda_api, cfg):
    """The workloads at full size, in the benchmark's launch configuration: every element of O and
    every row's LSE against the oracle, which materialises each full score row ("Why is attention
    O(n^2), how does FlashAttention help, ...", "Deep dive: FlashAttention": the tiled result equals
    the full softmax)."""
    q, k, v = synth.prefill_inputs_for(cfg)
    o, lse = cuda_api.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=cfg.causal, window=cfg.window,
                               rope_base=cfg.rope_base)
    torch.cuda.synchronize()
    assert cuda_api.device_status() == 0
    o_ref, lse_ref = oracle_prefill(q, k, v, cfg.causal, cfg.window, cfg.rope_base, cfg.scale)
    report(cfg.name, *assert_close(f64(o), f64(lse), o_ref, lse_ref, cfg.name))
