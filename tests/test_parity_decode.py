"""Paged-decode parity (GPU only): the CUDA split + merge against the fp64 oracle, bit-exact
agreement between a paged cache and its contiguous copy, NaN-poisoned slack, and the device-side
checks of block-table entries and sequence lengths."""
import numpy as np
import pytest
import torch

from exact_attention_161_b200 import synth
from parity import assert_close, f64, oracle_decode

pytestmark = pytest.mark.gpu

LENS = [1, 15, 16, 17, 511, 512, 513, 1000, 2049]


def _run(api, cache, **kw):
    c = [cache.q.cuda(), cache.k_pages.cuda(), cache.v_pages.cuda(), cache.block_table.cuda(),
         cache.seq_lens.cuda()]
    o, lse = api.attn_decode_paged(*c, **kw)
    torch.cuda.synchronize()
    return o, lse


@pytest.mark.parametrize("Hq,Hkv,D", [(8, 2, 128), (8, 2, 64), (32, 8, 128), (16, 1, 128), (4, 4, 64)])
def test_small_vs_oracle(cuda_api, Hq, Hkv, D):
    cache = synth.paged_decode_inputs(len(LENS), Hq, Hkv, D, 16, seq_lens=LENS, spare_frac=0.25, seed=Hq + D)
    o, lse = _run(cuda_api, cache)
    assert cuda_api.device_status() == 0
    o_ref, lse_ref = oracle_decode(cache)
    assert_close(f64(o), f64(lse), o_ref, lse_ref, "decode Hq%d Hkv%d D%d" % (Hq, Hkv, D))


def test_paged_equals_contiguous_bitwise(cuda_api):
    cache = synth.paged_decode_inputs(len(LENS), 8, 2, 128, 16, seq_lens=LENS, spare_frac=0.3, seed=11)
    o1, l1 = _run(cuda_api, cache)
    o2, l2 = _run(cuda_api, synth.contiguous_copy(cache))
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)


def test_shared_pages(cuda_api):
    """Two sequences whose block tables point at the same physical pages (block sharing) and
    carry the same query give identical outputs."""
    cache = synth.paged_decode_inputs(2, 8, 2, 128, 16, seq_lens=[700, 700], seed=12)
    cache.block_table[1] = cache.block_table[0]
    cache.q[1] = cache.q[0]
    o, lse = _run(cuda_api, cache)
    assert torch.equal(o[0].view(torch.int16), o[1].view(torch.int16)) and torch.equal(lse[0], lse[1])


def test_workload_full_size(cuda_api):
    """The 64-sequence paged-decode workload, every output row, and its contiguous copy."""
    cfg = synth.PAGED_DECODE_64
    cache = synth.paged_decode_inputs_for(cfg)
    o, lse = _run(cuda_api, cache)
    assert cuda_api.device_status() == 0
    o_ref, lse_ref = oracle_decode(cache)
    assert_close(f64(o), f64(lse), o_ref, lse_ref, cfg.name)
    o2, l2 = _run(cuda_api, synth.contiguous_copy(cache))
    assert torch.equal(o.view(torch.int16), o2.view(torch.int16)) and torch.equal(lse, l2)


def test_device_checks_flag_bad_entries(cuda_api):
    """Host-made bad inputs: an out-of-range block-table entry and a zero sequence length are
    caught by the kernel's own checks (no access is made) and reported in the status word."""
    cache = synth.paged_decode_inputs(3, 8, 2, 128, 16, seq_lens=[40, 40, 40], seed=13)
    cache.block_table[1, 1] = cache.num_pages + 7
    cache.seq_lens[2] = 0
    o, _ = _run(cuda_api, cache)
    flags = cuda_api.device_status()
    assert flags & cuda_api.DEVICE_BAD_PAGE and flags & cuda_api.DEVICE_BAD_SEQLEN
    assert bool(torch.isnan(o[2].float()).all())
    assert cuda_api.device_status() == 0  # reading clears the word
