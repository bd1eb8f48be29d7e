"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each ``check_*`` function takes an oracle library handle (``oracle._lib()`` or a deliberately
broken copy built by the mutation tests) and raises AssertionError when the oracle disagrees
with the pin. None of them re-types the oracle's own formula: they use hand-derived values,
closed forms of special cases, library routines (torch's float64 scaled_dot_product_attention,
scipy's logsumexp, torch's bf16 conversion) and invariants.
"""
import json
import math
import os

import numpy as np
import torch

import oracle
from exact_attention_161_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "hand_cases.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _to_bits(values):
    """Exact bf16 values -> bit patterns through torch (values must be bf16-representable)."""
    t = torch.tensor(np.asarray(values, dtype=np.float32)).to(torch.bfloat16)
    assert np.array_equal(t.float().numpy().astype(np.float64), np.asarray(values, np.float64))
    return t.view(torch.int16).numpy().view(np.uint16)


def _f64(bits):
    return oracle.bf16_bits_to_f64(bits)


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return synth.bits(synth.randn_bf16(shape, g))


def _sdpa64(q, k, v, scale, causal=False, mask=None, gqa=False):
    """torch's float64 CPU scaled_dot_product_attention (a library routine)."""
    qt, kt, vt = (torch.from_numpy(_f64(x)) for x in (q, k, v))
    return torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=mask, is_causal=causal, scale=scale, enable_gqa=gqa).numpy()


# ---------------------------------------------------------------------------------- rounding

def check_round_bf16_golden(lib):
    for case in _golden()["bf16_rounding"]["cases"]:
        got = int(oracle.round_bf16(np.array([case["x"]]), lib=lib)[0])
        assert got == case["bits"], (case, got)


def check_round_bf16_matches_torch(lib):
    """On binary32 inputs (no double rounding possible) the result must equal torch's RNE
    float32 -> bfloat16 conversion, ties included."""
    rng = np.random.default_rng(7)
    x = rng.standard_normal(20000).astype(np.float32) * np.float32(3.0)
    u = x.view(np.uint32).copy()
    u[:2000] = (u[:2000] & 0xFFFF0000) | 0x8000       # exact ties
    u[2000:4000] = (u[2000:4000] & 0xFFFF0000) | 0x7FFF
    u[4000:6000] = (u[4000:6000] & 0xFFFF0000) | 0x8001
    x = u.view(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.round_bf16(x.astype(np.float64), lib=lib)
    assert np.array_equal(got, want)


# ---------------------------------------------------------------------------------- RoPE

def check_rope_golden(lib):
    g = _golden()["rope_d4"]
    for case in g["cases"]:
        x = _to_bits(case["x"])[None, :]
        got = _f64(oracle.rope_bf16(x, np.array([case["pos"]]), g["base"], lib=lib))[0]
        assert np.array_equal(got, np.asarray(case["bf16"])), (case, got)


def check_rope_matches_sinusoid(lib):
    """Rotating (1,0) gives (cos, sin) of the angle and rotating (0,1) gives (-sin, cos). With
    base 10000 the angles are those of the sinusoidal encoding PE(pos,2i) = sin(pos/10000^(2i/d))
    ("attention-transformers", Q "Explain sinusoidal positional encoding"), evaluated here with
    numpy and rounded to bf16 by torch."""
    D = 64
    pos = np.array([0, 1, 7, 100, 2047, 30000], dtype=np.int64)
    i = np.arange(D // 2)
    pe_sin = np.sin(pos[:, None] / np.power(10000.0, 2 * i[None, :] / D))
    pe_cos = np.cos(pos[:, None] / np.power(10000.0, 2 * i[None, :] / D))
    for x_pair, want0, want1 in (((1.0, 0.0), pe_cos, pe_sin), ((0.0, 1.0), -pe_sin, pe_cos)):
        x = _to_bits(np.tile(np.array(x_pair), (len(pos), D // 2)))
        got = _f64(oracle.rope_bf16(x, pos, 10000.0, lib=lib))
        want = np.empty((len(pos), D))
        want[:, 0::2], want[:, 1::2] = want0, want1
        want_bf16 = torch.from_numpy(want).to(torch.bfloat16).double().numpy()
        # torch rounds float64 -> bf16 directly; allow one bf16 ulp for the last-bit angle
        # difference between numpy's and libm's sin/cos.
        assert np.allclose(got, want_bf16, rtol=2.0 ** -7, atol=2.0 ** -14), np.abs(got - want_bf16).max()


def check_rope_norm_and_identity(lib):
    x = _rand((64, 128), 11)
    pos0 = np.zeros(64, dtype=np.int64)
    assert np.array_equal(oracle.rope_bf16(x, pos0, 10000.0, lib=lib), x)
    pos = np.arange(64, dtype=np.int64) * 517
    y = _f64(oracle.rope_bf16(x, pos, 500000.0, lib=lib))
    xn = np.linalg.norm(_f64(x).reshape(64, 64, 2), axis=2)
    yn = np.linalg.norm(y.reshape(64, 64, 2), axis=2)
    # each pair keeps its length up to the two bf16 roundings
    assert np.all(np.abs(yn - xn) <= 2.0 ** -7 * xn + 1e-30)


def check_rope_relative(lib):
    """(R_i q).(R_j k) depends only on i - j ("How does Rotary Position Embedding (RoPE) work?");
    up to the bf16 rounding of the rotated values."""
    D = 128
    q = _rand((1, D), 12)
    k = _rand((1, D), 13)
    base = 10000.0
    for i, j, t in ((5, 2, 1000), (100, 0, 7), (40, 90, 3000)):
        a = _f64(oracle.rope_bf16(q, np.array([i]), base, lib=lib)) @ _f64(oracle.rope_bf16(k, np.array([j]), base, lib=lib)).T
        b = _f64(oracle.rope_bf16(q, np.array([i + t]), base, lib=lib)) @ _f64(oracle.rope_bf16(k, np.array([j + t]), base, lib=lib)).T
        bound = 2.0 ** -6 * np.linalg.norm(_f64(q)) * np.linalg.norm(_f64(k))
        assert abs(a - b) <= bound, (i, j, t, a, b)


# ---------------------------------------------------------------------------------- prefill

def check_hand_two_tokens(lib):
    c = _golden()["sdpa_two_tokens"]
    q = _to_bits(c["q"]).reshape(1, 1, 1, 2)
    k = _to_bits(c["k"]).reshape(1, 1, 2, 2)
    v = _to_bits(c["v"]).reshape(1, 1, 2, 2)
    # a 2-token sequence whose two queries are both q
    q2 = np.concatenate([q, q], axis=2)
    o, lse = oracle.attention(q2, k, v, causal=False, scale=c["scale"], lib=lib)
    assert np.allclose(o[0, 0, 0], c["o_full"], atol=1e-8) and abs(lse[0, 0, 0] - c["lse_full"]) < 1e-8
    o, lse = oracle.attention(q2, k, v, causal=True, scale=c["scale"], lib=lib)
    assert np.allclose(o[0, 0, 0], c["o_causal_row0"], atol=0) and abs(lse[0, 0, 0] - c["lse_causal_row0"]) < 1e-8
    assert np.allclose(o[0, 0, 1], c["o_full"], atol=1e-8) and abs(lse[0, 0, 1] - c["lse_full"]) < 1e-8


def check_library_sdpa(lib):
    """Without RoPE the oracle must agree with torch's float64 SDPA: the single-head N=128 d=64
    workload, and a two-batch four-head slice of the N=2048 d=128 causal workload."""
    q, k, v = (synth.bits(t) for t in synth.prefill_inputs(1, 1, 1, 128, 64, 1001))
    for causal in (False, True):
        o, _ = oracle.attention(q, k, v, causal=causal, scale=0.125, lib=lib)
        ref = _sdpa64(q, k, v, 0.125, causal=causal)
        assert np.abs(o - ref).max() < 1e-12
    q, k, v = (synth.bits(t) for t in synth.prefill_inputs(2, 4, 4, 512, 128, 1002))
    o, _ = oracle.attention(q, k, v, causal=True, scale=128 ** -0.5, lib=lib)
    ref = _sdpa64(q, k, v, 128 ** -0.5, causal=True)
    assert np.abs(o - ref).max() < 1e-12


def check_library_window(lib):
    N, w = 200, 37
    q, k, v = (synth.bits(t) for t in synth.prefill_inputs(1, 2, 2, N, 64, 21))
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    mask = torch.from_numpy((j <= i) & (j >= i - w + 1))
    o, _ = oracle.attention(q, k, v, causal=True, window=w, scale=0.125, lib=lib)
    ref = _sdpa64(q, k, v, 0.125, mask=mask)
    assert np.abs(o - ref).max() < 1e-12


def check_library_gqa(lib):
    """Query head h reads K/V head h // (Hq/Hkv): the convention of torch's enable_gqa."""
    q = _rand((2, 8, 96, 64), 31).reshape(2, 8, 96, 64)
    k = _rand((2, 2, 96, 64), 32).reshape(2, 2, 96, 64)
    v = _rand((2, 2, 96, 64), 33).reshape(2, 2, 96, 64)
    o, _ = oracle.attention(q, k, v, causal=True, scale=0.125, lib=lib)
    ref = _sdpa64(q, k, v, 0.125, causal=True, gqa=True)
    assert np.abs(o - ref).max() < 1e-12


def check_gqa_reduces_to_mha(lib):
    """GQA equals MHA on K/V repeated per group; Hkv = Hq is MHA; Hkv = 1 is MQA
    ("Transformer Complexity, Inference Optimization, GQA and FlashAttention", Part 3)."""
    q = _rand((1, 8, 64, 64), 41).reshape(1, 8, 64, 64)
    for hkv in (1, 2, 8):
        k = _rand((1, hkv, 64, 64), 42).reshape(1, hkv, 64, 64)
        v = _rand((1, hkv, 64, 64), 43).reshape(1, hkv, 64, 64)
        o, lse = oracle.attention(q, k, v, causal=True, rope_base=10000.0, scale=0.125, lib=lib)
        kr, vr = np.repeat(k, 8 // hkv, axis=1), np.repeat(v, 8 // hkv, axis=1)
        o2, lse2 = oracle.attention(q, kr, vr, causal=True, rope_base=10000.0, scale=0.125, lib=lib)
        assert np.array_equal(o, o2) and np.array_equal(lse, lse2)


def check_lse_library(lib):
    """LSE = ln sum exp(scaled scores) over the visible keys, via scipy's logsumexp."""
    from scipy.special import logsumexp
    N, D = 150, 64
    q, k, v = (synth.bits(t) for t in synth.prefill_inputs(1, 1, 1, N, D, 51))
    _, lse = oracle.attention(q, k, v, causal=True, window=60, scale=0.125, lib=lib)
    s = (_f64(q[0, 0]) @ _f64(k[0, 0]).T) * 0.125
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    s = np.where((j <= i) & (j >= i - 59), s, -np.inf)
    assert np.abs(lse[0, 0] - logsumexp(s, axis=1)).max() < 1e-12


def check_probability_rows(lib):
    """With V = identity (D = N) row i of O is row i of P. Every row sums to 1 and every masked
    entry is exactly 0 -- the mask acts on the logits before the softmax
    ("Transformer Attention Mechanism Interview Deep Dive", "Causal masking")."""
    N = 32
    q = _rand((1, 1, N, N), 61).reshape(1, 1, N, N)
    k = _rand((1, 1, N, N), 62).reshape(1, 1, N, N)
    v = _to_bits(np.eye(N)).reshape(1, 1, N, N)
    for causal, window in ((False, 0), (True, 0), (True, 5)):
        p, _ = oracle.attention(q, k, v, causal=causal, window=window, scale=1 / math.sqrt(N), lib=lib)
        p = p[0, 0]
        assert np.abs(p.sum(axis=1) - 1.0).max() < 1e-12
        i = np.arange(N)[:, None]
        j = np.arange(N)[None, :]
        visible = np.ones((N, N), bool)
        if causal:
            visible &= j <= i
        if window:
            visible &= j >= i - window + 1
        assert np.all(p[~visible] == 0.0) and np.all(p[visible] > 0.0)
        # number of attended pairs: N^2, N(N+1)/2, or sum_i min(i+1, w) (window cost O(n*w))
        want = N * N if not causal else sum(min(r + 1, window or N) for r in range(N))
        assert int((p > 0).sum()) == want


def check_permutation_equivariance(lib):
    """Without position information and without a mask, permuting the tokens permutes the
    outputs the same way ("attention-transformers", Q "Why does a transformer need positional
    encoding?")."""
    N = 64
    q, k, v = (synth.bits(t) for t in synth.prefill_inputs(1, 2, 2, N, 64, 71))
    perm = np.random.default_rng(3).permutation(N)
    o, lse = oracle.attention(q, k, v, scale=0.125, lib=lib)
    op, lsep = oracle.attention(q[:, :, perm], k[:, :, perm], v[:, :, perm], scale=0.125, lib=lib)
    assert np.abs(op - o[:, :, perm]).max() < 1e-13 and np.abs(lsep - lse[:, :, perm]).max() < 1e-13


def check_causal_row0_and_window1(lib):
    N = 48
    q, k, v = (synth.bits(t) for t in synth.prefill_inputs(1, 3, 3, N, 64, 81))
    o, lse = oracle.attention(q, k, v, causal=True, rope_base=10000.0, scale=0.125, lib=lib)
    assert np.array_equal(o[:, :, 0], _f64(v[:, :, 0]))
    s00 = np.einsum("bhd,bhd->bh", _f64(q[:, :, 0]), _f64(k[:, :, 0])) * 0.125  # pos 0: no rotation
    assert np.abs(lse[:, :, 0] - s00).max() < 1e-13
    o1, _ = oracle.attention(q, k, v, causal=True, window=1, rope_base=10000.0, scale=0.125, lib=lib)
    assert np.array_equal(o1, _f64(v))
    ow, lsew = oracle.attention(q, k, v, causal=True, window=N, rope_base=10000.0, scale=0.125, lib=lib)
    assert np.array_equal(ow, o) and np.array_equal(lsew, lse)


def check_equal_scores(lib):
    """q = 0 gives equal scores: O_i is the mean of the visible values, LSE_i = ln(count)."""
    N = 40
    _, k, v = (synth.bits(t) for t in synth.prefill_inputs(1, 1, 1, N, 64, 91))
    q = np.zeros((1, 1, N, 64), dtype=np.uint16)
    o, lse = oracle.attention(q, k, v, causal=True, scale=0.125, lib=lib)
    vv = _f64(v[0, 0])
    means = np.cumsum(vv, axis=0) / np.arange(1, N + 1)[:, None]
    assert np.abs(o[0, 0] - means).max() < 1e-13
    assert np.abs(lse[0, 0] - np.log(np.arange(1, N + 1))).max() < 1e-13


def check_rows_subset(lib):
    """Row-sampled evaluation returns exactly the rows of the full evaluation."""
    q, k, v = (synth.bits(t) for t in synth.prefill_inputs(2, 4, 2, 100, 64, 95))
    o, lse = oracle.attention(q, k, v, causal=True, window=30, rope_base=10000.0, scale=0.125, lib=lib)
    rows = np.array([0, 99, 100, 357, 799, 401], dtype=np.int64)
    os_, ls_ = oracle.attention(q, k, v, causal=True, window=30, rope_base=10000.0, scale=0.125,
                                rows=rows, lib=lib)
    assert np.array_equal(os_, o.reshape(-1, 64)[rows]) and np.array_equal(ls_, lse.reshape(-1)[rows])


def online_softmax_reference(q, k, v, scale, block, causal):
    """The pages' streaming recurrence ("Why is attention O(n^2), how does FlashAttention help,
    ...", "Deep dive: FlashAttention"), in fp64, one K/V block at a time. Test-only."""
    N = q.shape[0]
    m = np.full(N, -np.inf)
    l = np.zeros(N)
    o = np.zeros_like(q)
    for j0 in range(0, N, block):
        kb, vb = k[j0:j0 + block], v[j0:j0 + block]
        s = q @ kb.T * scale
        if causal:
            s = np.where(np.arange(j0, j0 + kb.shape[0])[None, :] <= np.arange(N)[:, None], s, -np.inf)
        m_new = np.maximum(m, s.max(axis=1))
        p = np.exp(s - m_new[:, None])
        alpha = np.exp(m - m_new)
        l = alpha * l + p.sum(axis=1)
        o = alpha[:, None] * o + p @ vb
        m = m_new
    return o / l[:, None], m + np.log(l)


def check_online_recurrence(lib):
    """The tiled recurrence reaches the materialised result up to rounding, for any block size
    ("Exact: the rescaling makes the result identical to a full softmax")."""
    N, D = 130, 64
    q, k, v = (synth.bits(t) for t in synth.prefill_inputs(1, 1, 1, N, D, 97))
    o, lse = oracle.attention(q, k, v, causal=True, scale=0.125, lib=lib)
    for block in (1, 3, 16, 128, N):
        ob, lseb = online_softmax_reference(_f64(q[0, 0]), _f64(k[0, 0]), _f64(v[0, 0]), 0.125, block, True)
        assert np.abs(ob - o[0, 0]).max() < 1e-12 and np.abs(lseb - lse[0, 0]).max() < 1e-12


# ---------------------------------------------------------------------------------- decode

def _small_cache(seed=5, permute=True, poison=True, lens=(1, 15, 16, 17, 40, 33)):
    return synth.paged_decode_inputs(len(lens), 8, 2, 64, 16, seq_lens=list(lens), spare_frac=0.5,
                                     seed=seed, permute=permute, poison=poison)


def _decode(cache, lib):
    return oracle.decode_paged(synth.bits(cache.q), synth.bits(cache.k_pages), synth.bits(cache.v_pages),
                               cache.block_table.numpy(), cache.seq_lens.numpy(), lib=lib)


def _gather(cache, s):
    n = int(cache.seq_lens[s])
    pages = cache.block_table[s, :(n + cache.page_size - 1) // cache.page_size].long()
    k = cache.k_pages[pages].permute(1, 0, 2, 3).reshape(cache.Hkv, -1, cache.D)[:, :n]
    v = cache.v_pages[pages].permute(1, 0, 2, 3).reshape(cache.Hkv, -1, cache.D)[:, :n]
    return k, v


def check_decode_is_last_prefill_row(lib):
    """One decode step attends to the T cached keys: it equals the last row of causal prefill
    over the same sequence ("Why is attention O(n^2), ...", prefill vs. decode)."""
    cache = _small_cache()
    o, lse = _decode(cache, lib)
    for s in range(cache.num_seqs):
        n = int(cache.seq_lens[s])
        k, v = _gather(cache, s)
        qs = np.zeros((1, cache.Hq, n, cache.D), np.uint16)
        qs[0, :, n - 1] = synth.bits(cache.q[s])
        op, lsep = oracle.attention(qs, synth.bits(k.contiguous())[None], synth.bits(v.contiguous())[None],
                                    causal=True, scale=cache.D ** -0.5, lib=lib)
        assert np.array_equal(o[s], op[0, :, n - 1]) and np.array_equal(lse[s], lsep[0, :, n - 1])


def check_decode_library(lib):
    cache = _small_cache(seed=6)
    o, _ = _decode(cache, lib)
    for s in range(cache.num_seqs):
        k, v = _gather(cache, s)
        ref = _sdpa64(synth.bits(cache.q[s])[:, None, :], synth.bits(k.contiguous()),
                      synth.bits(v.contiguous()), cache.D ** -0.5, gqa=True)
        assert np.abs(o[s] - ref[:, 0]).max() < 1e-12


def check_decode_paging_invariance(lib):
    """Paging is indirection only: the permuted pool and its contiguous copy give the same bits,
    and NaN in spare pages and page tails never reaches the output."""
    cache = _small_cache(seed=8)
    o, lse = _decode(cache, lib)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    o2, lse2 = _decode(synth.contiguous_copy(cache), lib)
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2)
    ident = _small_cache(seed=8, permute=False)
    o3, lse3 = _decode(ident, lib)
    assert np.array_equal(o, o3) and np.array_equal(lse, lse3)


def _step_inputs(T, seed, rope_base, lens=(4, 16, 17, 40, 33, 64)):
    return synth.decode_step_inputs(len(lens), T, 8, 2, 64, 16, seq_lens=list(lens), spare_frac=0.5, seed=seed)


def _step(inp, rope_base, lib, with_new=True):
    c = inp.cache
    return oracle.decode_step(synth.bits(inp.q), synth.bits(inp.k_new) if with_new else None,
                              synth.bits(inp.v_new) if with_new else None, synth.bits(c.k_pages),
                              synth.bits(c.v_pages), c.block_table.numpy(), c.seq_lens.numpy(), rope_base=rope_base,
                              lib=lib)


def _gather_bits(kp, vp, cache, s):
    n = int(cache.seq_lens[s])
    pages = cache.block_table[s, :(n + cache.page_size - 1) // cache.page_size].numpy()
    k = kp[pages].transpose(1, 0, 2, 3).reshape(cache.Hkv, -1, cache.D)[:, :n]
    v = vp[pages].transpose(1, 0, 2, 3).reshape(cache.Hkv, -1, cache.D)[:, :n]
    return np.ascontiguousarray(k), np.ascontiguousarray(v)


def check_decode_step_append_slots(lib):
    """The append writes exactly the new tokens' slots: the key rotated at its position, the value
    as given; every other slot keeps its bits ("Self-Attention Complexity, ...", Part 3)."""
    T, base = 3, 10000.0
    inp = _step_inputs(T, 11, base)
    c = inp.cache
    _, _, kp, vp = _step(inp, base, lib)
    k0, v0 = synth.bits(c.k_pages).copy(), synth.bits(c.v_pages).copy()
    touched = np.zeros(k0.shape[:1] + k0.shape[2:3], bool)  # [page, slot]
    for s in range(c.num_seqs):
        n = int(c.seq_lens[s])
        for t in range(T):
            pos = n - T + t
            page, slot = int(c.block_table[s, pos // 16]), pos % 16
            touched[page, slot] = True
            for g in range(c.Hkv):
                want_k = oracle.rope_bf16(synth.bits(inp.k_new[s, t, g])[None], np.array([pos]), base, lib=lib)[0]
                assert np.array_equal(kp[page, g, slot], want_k)
                assert np.array_equal(vp[page, g, slot], synth.bits(inp.v_new[s, t, g]))
    keep = ~touched[:, None, :, None].repeat(c.Hkv, 1).repeat(c.D, 3)
    assert np.array_equal(kp[keep], k0[keep]) and np.array_equal(vp[keep], v0[keep])


def check_decode_step_is_last_prefill_rows(lib):
    """T new tokens attend like the last T rows of causal prefill over the whole sequence, with q
    rotated at positions len-T .. len-1 (the decode query sits at the end of its sequence)."""
    T, base = 4, 500.0
    inp = _step_inputs(T, 12, base)
    c = inp.cache
    o, lse, kp, vp = _step(inp, base, lib)
    for s in range(c.num_seqs):
        n = int(c.seq_lens[s])
        k, v = _gather_bits(kp, vp, c, s)
        pos = np.arange(n - T, n)
        qs = np.zeros((1, c.Hq, n, c.D), np.uint16)
        for h in range(c.Hq):
            qs[0, h, n - T:] = oracle.rope_bf16(synth.bits(inp.q[s, :, h]), pos, base, lib=lib)
        op, lsep = oracle.attention(qs, k[None], v[None], causal=True, scale=c.D ** -0.5, lib=lib)
        assert np.array_equal(o[s], op[0, :, n - T:].transpose(1, 0, 2))
        assert np.array_equal(lse[s], lsep[0, :, n - T:].T)


def check_decode_step_prefill_with_rope(lib):
    """Against prefill with RoPE applied inside: a cache holding rotated keys of a sequence plus
    the last T tokens appended unrotated gives the last T rows of RoPE prefill on that sequence."""
    T, base = 2, 10000.0
    lens = (5, 17, 32)
    inp = _step_inputs(T, 13, base, lens=lens)
    c = inp.cache
    k_full = [_rand((c.Hkv, n, c.D), 140 + s) for s, n in enumerate(lens)]
    kp = synth.bits(c.k_pages).copy()
    for s, n in enumerate(lens):
        for j in range(n - T):
            page, slot = int(c.block_table[s, j // 16]), j % 16
            kp[page, :, slot] = oracle.rope_bf16(k_full[s][:, j], np.full(c.Hkv, j), base, lib=lib)
    k_new = np.stack([k_full[s][:, n - T:].transpose(1, 0, 2) for s, n in enumerate(lens)])
    o, lse, kp2, vp2 = oracle.decode_step(synth.bits(inp.q), np.ascontiguousarray(k_new), synth.bits(inp.v_new), kp,
                                          synth.bits(c.v_pages), c.block_table.numpy(), c.seq_lens.numpy(),
                                          rope_base=base, lib=lib)
    for s, n in enumerate(lens):
        _, v = _gather_bits(kp2, vp2, c, s)
        qs = np.zeros((1, c.Hq, n, c.D), np.uint16)
        qs[0, :, n - T:] = synth.bits(inp.q[s]).transpose(1, 0, 2)
        op, lsep = oracle.attention(qs, k_full[s][None], v[None], causal=True, rope_base=base, scale=c.D ** -0.5,
                                    lib=lib)
        assert np.array_equal(o[s], op[0, :, n - T:].transpose(1, 0, 2))
        assert np.array_equal(lse[s], lsep[0, :, n - T:].T)


def check_decode_step_library(lib):
    """torch float64 SDPA on the gathered cache, with the rotated queries and a causal mask over
    the last T positions."""
    T, base = 3, 10000.0
    inp = _step_inputs(T, 15, base)
    c = inp.cache
    o, _, kp, vp = _step(inp, base, lib)
    for s in range(c.num_seqs):
        n = int(c.seq_lens[s])
        k, v = _gather_bits(kp, vp, c, s)
        pos = np.arange(n - T, n)
        qr = np.stack([oracle.rope_bf16(synth.bits(inp.q[s, :, h]), pos, base, lib=lib) for h in range(c.Hq)])
        mask = np.arange(n)[None, :] <= pos[:, None]
        ref = _sdpa64(qr, k, v, c.D ** -0.5, mask=torch.tensor(mask), gqa=True)
        assert np.abs(o[s] - ref.transpose(1, 0, 2)).max() < 1e-12


def check_decode_step_reduces_to_decode(lib):
    """One token, no append, no RoPE: the decode step is the one-token paged decode."""
    inp = _step_inputs(1, 16, 0.0)
    c = inp.cache
    o, lse, _, _ = oracle.decode_step(synth.bits(inp.q), None, None, synth.bits(c.k_pages), synth.bits(c.v_pages),
                                      c.block_table.numpy(), c.seq_lens.numpy(), lib=lib)
    c.k_pages.view(torch.int16)[torch.isnan(c.k_pages)] = 0  # the poisoned new slots now hold tokens
    c.v_pages.view(torch.int16)[torch.isnan(c.v_pages)] = 0
    o1, lse1, _, _ = oracle.decode_step(synth.bits(inp.q), None, None, synth.bits(c.k_pages), synth.bits(c.v_pages),
                                        c.block_table.numpy(), c.seq_lens.numpy(), lib=lib)
    c1 = synth.PagedCache(inp.q[:, 0].contiguous(), c.k_pages, c.v_pages, c.block_table, c.seq_lens, c.page_size,
                          c.Hq, c.Hkv, c.D)
    o2, lse2 = _decode(c1, lib)
    assert np.array_equal(o1[:, 0], o2) and np.array_equal(lse1[:, 0], lse2)
    assert not np.all(np.isfinite(o))  # the unfilled NaN slot is read: the step does attend to it


# ---------------------------------------------------------------------------------- position variants

def check_rope_half_split_library(lib):
    """Half-split pairing against the rotate-half formulation written with torch in float64:
    x * [cos, cos] + rotate_half(x) * [sin, sin], rotate_half(x) = [-x2, x1]; then the pinned
    bf16 rounding."""
    D, base = 16, 10000.0
    x = _rand((9, D), 41)
    pos = np.array([0, 1, 2, 5, 17, 100, 999, 4096, 32767])
    got = oracle.rope_bf16_ex(x, pos, base, half_split=True, lib=lib)
    xt = torch.from_numpy(_f64(x))
    theta = base ** (-2.0 * torch.arange(D // 2, dtype=torch.float64) / D)
    ang = torch.from_numpy(pos.astype(np.float64))[:, None] * theta[None, :]
    cos, sin = torch.cat([ang.cos(), ang.cos()], 1), torch.cat([ang.sin(), ang.sin()], 1)
    rot = torch.cat([-xt[:, D // 2:], xt[:, :D // 2]], 1)
    ref = oracle.round_bf16((xt * cos + rot * sin).numpy(), lib=lib)
    assert np.array_equal(got, ref)
    assert not np.array_equal(got, oracle.rope_bf16(x, pos, base, lib=lib))  # the pairing matters


def check_rope_position_interpolation(lib):
    """Position Interpolation divides positions: factor f at position f*k equals plain RoPE at k."""
    x = _rand((6, 32), 42)
    for f in (2.0, 4.0):
        k = np.array([0, 1, 3, 10, 250, 4000])
        got = oracle.rope_bf16_ex(x, (k * f).astype(np.int64), 10000.0, pos_scale=f, lib=lib)
        assert np.array_equal(got, oracle.rope_bf16(x, k, 10000.0, lib=lib))


def check_rope_ntk_frequencies(lib):
    """NTK-aware scaling keeps the highest frequency (pair 0) and divides the lowest (pair D/2-1) by
    the factor: pair 0 matches plain RoPE at any position, and the last pair at position f*p matches
    plain RoPE at p (within one bf16 step: the two angles agree only up to fp64 rounding)."""
    D, f = 32, 4.0
    x = _rand((7, D), 43)
    p = np.array([1, 2, 7, 33, 500, 1000, 3000])
    ntk = oracle.rope_bf16_ex(x, p * 4, 10000.0, ntk_factor=f, lib=lib)
    plain_same_pos = oracle.rope_bf16(x, p * 4, 10000.0, lib=lib)
    assert np.array_equal(ntk[:, :2], plain_same_pos[:, :2])
    plain = oracle.rope_bf16(x, p, 10000.0, lib=lib)
    a, b = _f64(ntk[:, -2:]), _f64(plain[:, -2:])
    assert np.all(np.abs(a - b) <= np.abs(b) * 2.0 ** -7 + 1e-12)
    assert not np.array_equal(ntk[:, 2:-2], plain_same_pos[:, 2:-2])  # middle frequencies move


def check_alibi_closed_form(lib):
    """q = 0 leaves only the bias: row i weighs key j <= i by e^(-m (i - j)), so with V = identity
    O_i[j] is that weight normalised and LSE_i = ln((1 - e^(-m (i+1))) / (1 - e^(-m)))."""
    N, D, m = 12, 16, 0.375
    q = np.zeros((1, 1, N, D), np.uint16)
    k = _rand((1, 1, N, D), 44)
    v = _to_bits(np.eye(N, D)[None, None])
    o, lse = oracle.attention_pos(q, k, v, causal=True, alibi_slopes=[m], lib=lib)
    for i in range(N):
        w = np.exp(-m * (i - np.arange(i + 1)))
        assert np.abs(o[0, 0, i, :i + 1] - w / w.sum()).max() < 1e-14
        assert np.abs(o[0, 0, i, i + 1:]).max() == 0.0
        assert abs(lse[0, 0, i] - math.log((1 - math.exp(-m * (i + 1))) / (1 - math.exp(-m)))) < 1e-13


def check_alibi_library(lib):
    """ALiBi with GQA and RoPE against torch float64 SDPA given the bias -m_h (i - j) as a float mask."""
    B, Hq, Hkv, N, D = 1, 4, 2, 20, 8
    q, k, v = _rand((B, Hq, N, D), 45), _rand((B, Hkv, N, D), 46), _rand((B, Hkv, N, D), 47)
    slopes = np.array([0.5, 0.25, 0.125, 0.0625])
    base = 100.0
    o, _ = oracle.attention_pos(q, k, v, causal=True, rope_base=base, alibi_slopes=slopes, lib=lib)
    pos = np.arange(N)
    qr = np.stack([oracle.rope_bf16(q[0, h], pos, base, lib=lib) for h in range(Hq)])[None]
    kr = np.stack([oracle.rope_bf16(k[0, g], pos, base, lib=lib) for g in range(Hkv)])[None]
    i, j = np.meshgrid(pos, pos, indexing="ij")
    bias = np.where(j <= i, -slopes[:, None, None] * (i - j)[None], -np.inf)[None]
    ref = _sdpa64(qr, kr, v, D ** -0.5, mask=torch.from_numpy(bias), gqa=True)
    assert np.abs(o - ref).max() < 1e-12


def check_position_variants_combined(lib):
    """Half-split pairing, both scalings and ALiBi together reduce to the plain oracle when the
    variants are neutral, and the half-split result equals interleaved RoPE on dimensions
    permuted so that (i, i + D/2) become (2i, 2i+1) -- a score is unchanged by permuting the
    dimensions of q and k alike."""
    B, Hq, Hkv, N, D = 1, 2, 1, 24, 16
    q, k, v = _rand((B, Hq, N, D), 48), _rand((B, Hkv, N, D), 49), _rand((B, Hkv, N, D), 50)
    o1, l1 = oracle.attention_pos(q, k, v, causal=True, rope_base=500.0, lib=lib)
    o2, l2 = oracle.attention(q, k, v, causal=True, rope_base=500.0, lib=lib)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    perm = np.stack([np.arange(D // 2), np.arange(D // 2) + D // 2], 1).reshape(-1)
    oh, lh = oracle.attention_pos(q, k, v, causal=True, rope_base=500.0, rope_half_split=True, rope_pos_scale=2.0,
                                  rope_ntk_factor=3.0, lib=lib)
    op, lp = oracle.attention_pos(np.ascontiguousarray(q[..., perm]), np.ascontiguousarray(k[..., perm]), v,
                                  causal=True, rope_base=500.0, rope_pos_scale=2.0, rope_ntk_factor=3.0, lib=lib)
    assert np.abs(oh - op).max() < 1e-12 and np.abs(lh - lp).max() < 1e-12


# ---------------------------------------------------------------------------------- FP8

def check_e4m3_golden_and_library(lib):
    """e4m3 decoding: values worked by hand from the encoding (bias 7, 3 mantissa bits, subnormals
    m * 2^-9, S.1111.111 = NaN), and torch's float8_e4m3fn conversion on all 256 codes."""
    hand = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0, 0x39: 1.125,
            0x3F: 1.875, 0x40: 2.0, 0x7E: 448.0, 0xFE: -448.0, 0xB8: -1.0, 0x80: -0.0}
    codes = np.array(sorted(hand), np.uint8)
    got = oracle.e4m3_to_f64(codes, lib=lib)
    assert np.array_equal(got, np.array([hand[c] for c in sorted(hand)]))
    assert np.isnan(oracle.e4m3_to_f64(np.array([0x7F, 0xFF], np.uint8), lib=lib)).all()
    allc = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(allc).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = oracle.e4m3_to_f64(allc, lib=lib)
    ok = np.isnan(ref) & np.isnan(mine) | (ref == mine)
    assert ok.all()


def check_fp8_attention_library(lib):
    """FP8 attention = torch float64 SDPA on the dequantised tensors (values times descales)."""
    f = synth.fp8_inputs(1, 4, 2, 40, 16, 60)
    o, lse = oracle.attention_fp8(f.q8.numpy(), f.k8.numpy(), f.v8.numpy(), f.descale_q, f.descale_k, f.descale_v,
                                  causal=True, lib=lib)
    deq = [torch.from_numpy(oracle.e4m3_to_f64(x.numpy(), lib=lib) * d)
           for x, d in ((f.q8, f.descale_q), (f.k8, f.descale_k), (f.v8, f.descale_v))]
    ref = torch.nn.functional.scaled_dot_product_attention(*deq, is_causal=True, scale=16 ** -0.5, enable_gqa=True)
    assert np.abs(o - ref.numpy()).max() < 1e-12
    s = torch.einsum("bhid,bhjd->bhij", deq[0], deq[1].repeat_interleave(2, dim=1)) * 16 ** -0.5
    s = s.masked_fill(torch.ones(40, 40, dtype=torch.bool).triu(1), float("-inf"))
    assert np.abs(lse - torch.logsumexp(s, -1).numpy()).max() < 1e-12


def check_fp8_descales(lib):
    """The value scale of V scales O exactly (powers of two); the scores depend on descale_q *
    descale_k only."""
    f = synth.fp8_inputs(1, 2, 1, 24, 16, 61)
    args = (f.q8.numpy(), f.k8.numpy(), f.v8.numpy())
    o1, l1 = oracle.attention_fp8(*args, 0.5, 0.25, 1.0, causal=True, lib=lib)
    o2, l2 = oracle.attention_fp8(*args, 0.25, 0.5, 4.0, causal=True, lib=lib)
    assert np.array_equal(o1 * 4.0, o2) and np.array_equal(l1, l2)


ALL_CHECKS = [
    check_round_bf16_golden, check_round_bf16_matches_torch, check_rope_golden,
    check_rope_matches_sinusoid, check_rope_norm_and_identity, check_rope_relative,
    check_hand_two_tokens, check_library_sdpa, check_library_window, check_library_gqa,
    check_gqa_reduces_to_mha, check_lse_library, check_probability_rows,
    check_permutation_equivariance, check_causal_row0_and_window1, check_equal_scores,
    check_rows_subset, check_online_recurrence, check_decode_is_last_prefill_row,
    check_decode_library, check_decode_paging_invariance, check_decode_step_append_slots,
    check_decode_step_is_last_prefill_rows, check_decode_step_prefill_with_rope, check_decode_step_library,
    check_decode_step_reduces_to_decode, check_rope_half_split_library, check_rope_position_interpolation,
    check_rope_ntk_frequencies, check_alibi_closed_form, check_alibi_library, check_position_variants_combined,
    check_e4m3_golden_and_library, check_fp8_attention_library, check_fp8_descales,
]


# ---------------------------------------------------------------------------------- backward

def _bwd_case(seed, B=1, Hq=2, Hkv=1, N=9, D=4):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Hq, N, D))
    k = rng.standard_normal((B, Hkv, N, D))
    v = rng.standard_normal((B, Hkv, N, D))
    do = rng.standard_normal((B, Hq, N, D))
    return q, k, v, do


def check_bwd_finite_differences(lib):
    """Every gradient entry against a central difference of L = sum(O * dO) (brute force)."""
    for causal, window, rope in ((0, 0, 0.0), (1, 0, 0.0), (1, 3, 0.0), (1, 0, 50.0)):
        q, k, v, do = _bwd_case(17 + window)
        dq, dk, dv = oracle.attention_bwd_f64(q, k, v, do, causal=causal, window=window, rope_base=rope, lib=lib)

        def loss(qq, kk, vv):
            o, _ = oracle.attention_f64(qq, kk, vv, causal=causal, window=window, rope_base=rope, lib=lib)
            return float((o * do).sum())

        eps = 1e-6
        for which, (arr, grad) in enumerate(((q, dq), (k, dk), (v, dv))):
            for idx in np.ndindex(arr.shape):
                a = arr.copy()
                a[idx] += eps
                args = [q, k, v]
                args[which] = a
                lp = loss(*args)
                a[idx] -= 2 * eps
                args[which] = a
                lm = loss(*args)
                assert abs((lp - lm) / (2 * eps) - grad[idx]) < 1e-7, (causal, window, rope, which, idx)


def _torch_rope(x, base):
    """Pairwise rotation written with torch ops, so autograd supplies the chain rule."""
    if base <= 0:
        return x
    N, D = x.shape[-2], x.shape[-1]
    pos = torch.arange(N, dtype=torch.float64)[:, None]
    theta = base ** (-2.0 * torch.arange(D // 2, dtype=torch.float64) / D)
    ang = pos * theta[None, :]
    c, s = torch.cos(ang), torch.sin(ang)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    y = torch.stack((x0 * c - x1 * s, x0 * s + x1 * c), dim=-1)
    return y.reshape(x.shape)


def check_bwd_torch_autograd(lib):
    """Gradients against torch float64 autograd through SDPA (masks, GQA) and the rotation."""
    for causal, window, rope in ((0, 0, 0.0), (1, 0, 0.0), (1, 5, 0.0), (1, 0, 1000.0)):
        q, k, v, do = _bwd_case(23, B=2, Hq=4, Hkv=2, N=24, D=8)
        dq, dk, dv = oracle.attention_bwd_f64(q, k, v, do, causal=causal, window=window, rope_base=rope, lib=lib)
        qt, kt, vt = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        mask = None
        if window:
            i = torch.arange(24)[:, None]
            j = torch.arange(24)[None, :]
            mask = (j <= i) & (j >= i - window + 1)
        o = torch.nn.functional.scaled_dot_product_attention(
            _torch_rope(qt, rope), _torch_rope(kt, rope), vt, attn_mask=mask, is_causal=bool(causal and not window),
            scale=8 ** -0.5, enable_gqa=True)
        (o * torch.tensor(do)).sum().backward()
        assert np.abs(dq - qt.grad.numpy()).max() < 1e-10
        assert np.abs(dk - kt.grad.numpy()).max() < 1e-10
        assert np.abs(dv - vt.grad.numpy()).max() < 1e-10


def check_bwd_gqa_is_sum_over_group(lib):
    """The K/V gradient of a shared head is the sum of the gradients of its repeated copies."""
    q, k, v, do = _bwd_case(29, Hq=4, Hkv=2, N=12, D=4)
    dq, dk, dv = oracle.attention_bwd_f64(q, k, v, do, causal=1, rope_base=10.0, lib=lib)
    kr, vr = np.repeat(k, 2, axis=1), np.repeat(v, 2, axis=1)
    dq2, dk2, dv2 = oracle.attention_bwd_f64(q, kr, vr, do, causal=1, rope_base=10.0, lib=lib)
    assert np.abs(dq - dq2).max() < 1e-12
    assert np.abs(dk - dk2.reshape(1, 2, 2, 12, 4).sum(axis=2)).max() < 1e-12
    assert np.abs(dv - dv2.reshape(1, 2, 2, 12, 4).sum(axis=2)).max() < 1e-12


def check_bwd_bf16_entry(lib):
    """The bf16 entry point is the fp64 one on the exact input values with bf16-rounded rotation."""
    q, k, v = (synth.bits(t) for t in synth.prefill_inputs(1, 2, 1, 40, 64, 33))
    do = _rand((1, 2, 40, 64), 34).reshape(1, 2, 40, 64)
    g1 = oracle.attention_bwd(q, k, v, do, causal=True, rope_base=10000.0, scale=0.125, lib=lib)
    g2 = oracle.attention_bwd_f64(_f64(q), _f64(k), _f64(v), _f64(do), causal=True, rope_base=10000.0, scale=0.125,
                                  round_rotated=True, lib=lib)
    assert all(np.array_equal(a, b) for a, b in zip(g1, g2))


def check_bwd_dq_rows_match_full(lib):
    """dq of selected rows equals the full backward's dq at those rows (bf16 entry, RoPE, GQA, window)."""
    q, k, v = (synth.bits(t) for t in synth.prefill_inputs(1, 4, 2, 70, 16, 35))
    do = synth.bits(synth.randn_bf16((1, 4, 70, 16), torch.Generator().manual_seed(36)))
    for causal, window in ((1, 0), (1, 9), (0, 0)):
        dq, _, _ = oracle.attention_bwd(q, k, v, do, causal=causal, window=window, rope_base=100.0, scale=0.25, lib=lib)
        rows = np.array([0, 5, 69, 70, 139, 200, 279])
        got = oracle.attention_bwd_dq_rows(q, k, v, do, rows, causal=causal, window=window, rope_base=100.0, scale=0.25,
                                           lib=lib)
        assert np.abs(got - dq.reshape(-1, 16)[rows]).max() < 1e-13


ALL_CHECKS += [check_bwd_finite_differences, check_bwd_torch_autograd, check_bwd_gqa_is_sum_over_group,
               check_bwd_bf16_entry, check_bwd_dq_rows_match_full]
