"""Decode-step parity (GPU only): append of the new tokens' rotated keys and values into their page
slots, then multi-token attention over the cache, against the fp64 oracle's decode step; bit-exact
reduction to the one-token decode; paged = contiguous; device checks of the append."""
import numpy as np
import pytest
import torch

import oracle
from exact_attention_161_b200 import synth
from parity import assert_close, bits, f64

pytestmark = pytest.mark.gpu

# lengths cross page (16) and chunk (512) boundaries with the new tokens
LENS = [4, 16, 17, 100, 511, 512, 513, 515, 1030]


def _run(api, inp, rope_base, append=True):
    c = inp.cache
    kp, vp = c.k_pages.cuda(), c.v_pages.cuda()
    o, lse = api.attn_decode_step(inp.q.cuda(), kp, vp, c.block_table.cuda(), c.seq_lens.cuda(),
                                  k_new=inp.k_new.cuda() if append else None, v_new=inp.v_new.cuda() if append else None,
                                  rope_base=rope_base)
    torch.cuda.synchronize()
    return o, lse, kp, vp


def _oracle(inp, rope_base, append=True):
    c = inp.cache
    return oracle.decode_step(bits(inp.q), bits(inp.k_new) if append else None, bits(inp.v_new) if append else None,
                              bits(c.k_pages), bits(c.v_pages), c.block_table.numpy(), c.seq_lens.numpy(),
                              rope_base=rope_base)


def _check_pages(kp, vp, kp_ref, vp_ref):
    """Every slot bit-exact: values are copied, and keys are rotated with fp64 cos/sin by unfused
    fp64 products and one rounding to bf16, which is how the oracle rounds them."""
    assert np.array_equal(bits(vp.cpu()), vp_ref)
    assert np.array_equal(bits(kp.cpu()), kp_ref)


@pytest.mark.parametrize("T,Hq,Hkv,D,rope", [
    (1, 8, 2, 128, 10000.0), (2, 8, 2, 128, 10000.0), (4, 32, 8, 128, 500000.0), (3, 8, 2, 64, 10000.0),
    (4, 16, 1, 128, 0.0), (8, 4, 4, 64, 10000.0), (16, 8, 2, 128, 10000.0), (33, 8, 2, 64, 10000.0)])
def test_step_vs_oracle(cuda_api, T, Hq, Hkv, D, rope):
    lens = [max(n, T) for n in LENS]
    inp = synth.decode_step_inputs(len(lens), T, Hq, Hkv, D, 16, seq_lens=lens, spare_frac=0.25, seed=T * 100 + Hq + D)
    o, lse, kp, vp = _run(cuda_api, inp, rope)
    assert cuda_api.device_status() == 0
    o_ref, lse_ref, kp_ref, vp_ref = _oracle(inp, rope)
    _check_pages(kp, vp, kp_ref, vp_ref)
    assert_close(f64(o), f64(lse), o_ref, lse_ref, "decode step T%d Hq%d Hkv%d D%d" % (T, Hq, Hkv, D))


def test_step_without_append(cuda_api):
    """k_new = NULL: the cache already holds the new tokens; nothing is written."""
    inp = synth.decode_step_inputs(len(LENS), 3, 8, 2, 128, 16, seq_lens=LENS, seed=21, poison=False)
    o, lse, kp, vp = _run(cuda_api, inp, 10000.0, append=False)
    assert cuda_api.device_status() == 0
    o_ref, lse_ref, kp_ref, vp_ref = _oracle(inp, 10000.0, append=False)
    assert np.array_equal(bits(kp.cpu()), kp_ref) and np.array_equal(bits(vp.cpu()), vp_ref)
    assert_close(f64(o), f64(lse), o_ref, lse_ref, "decode step without append")


def test_one_token_equals_decode_bitwise(cuda_api):
    """One token, no RoPE, no append: the step runs the one-token decode and gives its bits."""
    inp = synth.decode_step_inputs(len(LENS), 1, 8, 2, 128, 16, seq_lens=LENS, seed=22, poison=False)
    c = inp.cache
    o, lse, _, _ = _run(cuda_api, inp, 0.0, append=False)
    o2, lse2 = cuda_api.attn_decode_paged(inp.q[:, 0].contiguous().cuda(), c.k_pages.cuda(), c.v_pages.cuda(),
                                          c.block_table.cuda(), c.seq_lens.cuda())
    assert torch.equal(o[:, 0].view(torch.int16), o2.view(torch.int16)) and torch.equal(lse[:, 0], lse2)


def test_step_paged_equals_contiguous(cuda_api):
    inp = synth.decode_step_inputs(len(LENS), 4, 8, 2, 128, 16, seq_lens=LENS, spare_frac=0.3, seed=23)
    o1, l1, _, _ = _run(cuda_api, inp, 10000.0)
    inp2 = synth.DecodeStepInputs(synth.contiguous_copy(inp.cache), inp.q, inp.k_new, inp.v_new)
    o2, l2, _, _ = _run(cuda_api, inp2, 10000.0)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)


def test_step_workload_full_size(cuda_api):
    """The 64-sequence paged workload with one new token per sequence, RoPE 1e4, appended: every row,
    and four new tokens per sequence (multi-token decode)."""
    cfg = synth.PAGED_DECODE_64
    for T in (1, 4):
        inp = synth.decode_step_inputs_for(cfg, T)
        o, lse, kp, vp = _run(cuda_api, inp, 10000.0)
        assert cuda_api.device_status() == 0
        o_ref, lse_ref, kp_ref, vp_ref = _oracle(inp, 10000.0)
        _check_pages(kp, vp, kp_ref, vp_ref)
        assert_close(f64(o), f64(lse), o_ref, lse_ref, "%s T=%d" % (cfg.name, T))


def test_append_device_checks(cuda_api):
    """A new token whose block-table entry is out of range is not written and raises the bad-page
    bit; a length shorter than q_len raises the length bit. Both are host-made inputs caught by the
    kernels' own checks before any access."""
    inp = synth.decode_step_inputs(3, 2, 8, 2, 128, 16, seq_lens=[40, 40, 40], seed=24)
    c = inp.cache
    good = c.block_table[1, 2].item()
    c.block_table[1, 2] = c.num_pages + 5  # the page of positions 32..47: both new tokens of seq 1
    kp_before = c.k_pages.clone()
    c.seq_lens[2] = 1
    o, _, kp, _ = _run(cuda_api, inp, 10000.0)
    flags = cuda_api.device_status()
    assert flags & cuda_api.DEVICE_BAD_PAGE and flags & cuda_api.DEVICE_BAD_SEQLEN
    assert torch.equal(kp[good].cpu().view(torch.int16), kp_before[good].view(torch.int16))
    assert bool(torch.isnan(o[2].float()).all())
    assert cuda_api.device_status() == 0
