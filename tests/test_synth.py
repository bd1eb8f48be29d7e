"""The seeded input generator: determinism, the 1/sqrt(d) variance argument, and the paged
cache's structure (CPU only)."""
import math

import numpy as np
import torch

from exact_attention_161_b200 import synth


def test_seeded_and_deterministic():
    a = synth.prefill_inputs(1, 2, 1, 64, 64, 5)
    b = synth.prefill_inputs(1, 2, 1, 64, 64, 5)
    assert all(torch.equal(x.view(torch.int16), y.view(torch.int16)) for x, y in zip(a, b))
    assert a[0].dtype == torch.bfloat16 and a[1].shape == (1, 1, 64, 64)


def test_scaled_scores_have_unit_variance():
    """q, k with unit-variance entries: q.k has variance d, q.k/sqrt(d) variance 1
    ("attention-transformers", Q "Why is attention scaled by 1/sqrt(dk)?")."""
    g = torch.Generator().manual_seed(123)
    d = 128
    q = synth.randn_bf16((100000, d), g).double()
    k = synth.randn_bf16((100000, d), g).double()
    s = (q * k).sum(dim=1) / d ** 0.5
    assert abs(float(s.var()) - 1.0) < 0.02


def test_paged_cache_structure():
    lens = [1, 15, 16, 17, 511, 512, 513]
    c = synth.paged_decode_inputs(len(lens), 8, 2, 64, 16, seq_lens=lens, spare_frac=0.1, seed=9)
    pages = [(n + 15) // 16 for n in lens]
    assert c.max_blocks == max(pages)
    used = sum(pages)
    assert c.num_pages == used + round(used * 0.1)
    bt = c.block_table.numpy()
    live = np.concatenate([bt[s, :pages[s]] for s in range(len(lens))])
    assert len(set(live.tolist())) == used and live.min() >= 0 and live.max() < c.num_pages
    for s in range(len(lens)):
        assert np.all(bt[s, pages[s]:] == -1)
    kb = c.k_pages.view(torch.int16).numpy().view(np.uint16)
    for s, n in enumerate(lens):
        last = bt[s, pages[s] - 1]
        tail = n - (pages[s] - 1) * 16
        assert np.all(kb[last, :, tail:, :] == synth.BF16_NAN_BITS)
        assert not np.any(kb[last, :, :tail, :] == synth.BF16_NAN_BITS)
    spare = sorted(set(range(c.num_pages)) - set(live.tolist()))
    assert np.all(kb[spare] == synth.BF16_NAN_BITS)


def test_contiguous_copy_and_identity_order_hold_the_same_tokens():
    lens = [3, 40, 17]
    a = synth.paged_decode_inputs(3, 4, 2, 64, 16, seq_lens=lens, seed=4, permute=True)
    b = synth.paged_decode_inputs(3, 4, 2, 64, 16, seq_lens=lens, seed=4, permute=False)
    c = synth.contiguous_copy(a)
    for s, n in enumerate(lens):
        np_ = (n + 15) // 16
        for x in (b, c):
            pa = a.k_pages[a.block_table[s, :np_].long()]
            px = x.k_pages[x.block_table[s, :np_].long()]
            ta = pa.permute(1, 0, 2, 3).reshape(2, -1, 64)[:, :n]
            tx = px.permute(1, 0, 2, 3).reshape(2, -1, 64)[:, :n]
            assert torch.equal(ta.view(torch.int16), tx.view(torch.int16))


def test_decode_step_inputs_poison_only_the_new_slots():
    """The new tokens' slots (positions len-T .. len-1) hold NaN until an append fills them; every
    earlier token is the plain cache's."""
    lens = [3, 16, 17, 40]
    plain = synth.paged_decode_inputs(len(lens), 8, 2, 64, 16, seq_lens=lens, seed=9, spare_frac=0.5)
    st = synth.decode_step_inputs(len(lens), 3, 8, 2, 64, 16, seq_lens=lens, seed=9, spare_frac=0.5)
    assert st.q.shape == (4, 3, 8, 64) and st.k_new.shape == (4, 3, 2, 64) and st.T == 3
    for s, n in enumerate(lens):
        for pos in range(n):
            page, slot = int(st.cache.block_table[s, pos // 16]), pos % 16
            got = st.cache.k_pages[page, :, slot]
            if pos >= n - 3:
                assert bool(torch.isnan(got.float()).all())
            else:
                assert torch.equal(got.view(torch.int16), plain.k_pages[page, :, slot].view(torch.int16))


def test_fp8_inputs_are_exact_scaled_e4m3():
    """Per-tensor descales are powers of two covering max|x| with e4m3's largest value 448, and the
    e4m3 codes decode (through torch) to values within e4m3 rounding of the fp32 draws."""
    f = synth.fp8_inputs(1, 2, 1, 64, 128, seed=3)
    g = torch.Generator().manual_seed(3)
    for x8, d in ((f.q8, f.descale_q), (f.k8, f.descale_k), (f.v8, f.descale_v)):
        assert x8.dtype == torch.uint8
        assert math.log2(d) == int(math.log2(d))
        vals = x8.view(torch.float8_e4m3fn).double()
        assert float(vals.abs().max()) <= 448.0 and not bool(torch.isnan(vals).any())
    x = torch.randn((1, 2, 64, 128), generator=g, dtype=torch.float32).double()
    back = f.q8.view(torch.float8_e4m3fn).double() * f.descale_q
    assert float(((back - x).abs() - 2.0 ** -4 * x.abs() - 2.0 ** -9 * f.descale_q).max()) <= 0.0


def test_alibi_slopes_are_the_geometric_sequence():
    s = synth.alibi_slopes(8)
    assert s.dtype == torch.float32 and s.shape == (8,)
    assert torch.equal(s, torch.tensor([2.0 ** -(h + 1) for h in range(8)], dtype=torch.float32))
