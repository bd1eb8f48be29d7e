"""Position-variant parity (GPU only): half-split RoPE pairing, Position Interpolation, NTK-aware
base scaling and ALiBi in the prefill kernel, against the fp64 oracle's attention_pos.

Tolerances are those of attn_fwd, except the max-abs bound with ALiBi. Steep slopes concentrate a
row's weight on a few keys, so outputs reach the size of single V entries (up to ~4.5 for N(0,1)
data), where one bf16 step of the stored output is up to 2^-5. There the bound is per element,
max(2e-2, 2^-7 |reference|): two half-steps of bf16 at the reference value.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_attention_161_b200 import synth
from parity import LSE_MAX_ABS, O_MAX_ABS, O_REL_RMS, assert_close, bits, f64, report


def assert_close_alibi(o, lse, o_ref, lse_ref, what):
    o = np.asarray(o, np.float64)
    assert np.all(np.isfinite(o)), what
    d = o - o_ref
    rel_rms = np.sqrt((d ** 2).sum() / (o_ref ** 2).sum())
    worst = (np.abs(d) / np.maximum(O_MAX_ABS, 2.0 ** -7 * np.abs(o_ref))).max()
    assert rel_rms <= O_REL_RMS, "%s rel-RMS %.3e" % (what, rel_rms)
    assert worst <= 1.0, "%s max-abs over its per-element bound by %.2fx" % (what, worst)
    assert np.abs(np.asarray(lse, np.float64) - lse_ref).max() <= LSE_MAX_ABS, what


def _close(case, o, lse, o_ref, lse_ref, what):
    (assert_close_alibi if case[-1] else assert_close)(o, lse, o_ref, lse_ref, what)

pytestmark = pytest.mark.gpu

# B, Hq, Hkv, N, D, causal, window, rope_base, half_split, pos_scale, ntk, alibi
CASES = [
    (1, 4, 2, 300, 128, 1, 0, 10000.0, True, 1.0, 1.0, False),
    (1, 2, 2, 257, 64, 0, 0, 10000.0, True, 1.0, 1.0, False),
    (1, 4, 1, 640, 128, 1, 0, 10000.0, False, 4.0, 1.0, False),
    (1, 4, 1, 640, 128, 1, 0, 10000.0, False, 1.0, 8.0, False),
    (1, 2, 2, 513, 64, 1, 100, 500000.0, True, 2.0, 4.0, False),
    (1, 8, 2, 300, 128, 1, 0, 0.0, False, 1.0, 1.0, True),
    (1, 8, 8, 1000, 128, 1, 0, 10000.0, False, 1.0, 1.0, True),
    (2, 4, 2, 129, 64, 1, 64, 10000.0, True, 4.0, 2.0, True),
    (1, 32, 8, 1024, 128, 1, 0, 500000.0, True, 1.0, 4.0, True),
]


def _ids(c):
    return "B%dHq%dHkv%dN%dD%d_c%d_w%d_r%g_half%d_pi%g_ntk%g_alibi%d" % c


def _gpu(api, q, k, v, case):
    B, Hq, Hkv, N, D, causal, window, rope, half, ps, ntk, alibi = case
    slopes = synth.alibi_slopes(Hq).cuda() if alibi else None
    o, lse = api.attn_fwd_pos(q.cuda(), k.cuda(), v.cuda(), causal=causal, window=window, rope_base=rope,
                              rope_half_split=half, rope_pos_scale=ps, rope_ntk_factor=ntk, alibi_slopes=slopes)
    torch.cuda.synchronize()
    return o, lse


def _oracle(q, k, v, case, rows=None):
    B, Hq, Hkv, N, D, causal, window, rope, half, ps, ntk, alibi = case
    slopes = synth.alibi_slopes(Hq).double().numpy() if alibi else None
    return oracle.attention_pos(bits(q), bits(k), bits(v), causal=causal, window=window, rope_base=rope,
                                rope_half_split=half, rope_pos_scale=ps, rope_ntk_factor=ntk, alibi_slopes=slopes,
                                rows=rows)


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_variant_vs_oracle(cuda_api, case):
    B, Hq, Hkv, N, D = case[:5]
    q, k, v = synth.prefill_inputs(B, Hq, Hkv, N, D, seed=500 + CASES.index(case))
    o, lse = _gpu(cuda_api, q, k, v, case)
    assert cuda_api.device_status() == 0
    o_ref, lse_ref = _oracle(q, k, v, case)
    _close(case, f64(o), f64(lse), o_ref, lse_ref, _ids(case))


def test_neutral_variants_are_attn_fwd(cuda_api):
    """Interleaved pairing, both factors 1 and no ALiBi: the same bits as attn_fwd."""
    q, k, v = synth.prefill_inputs(1, 8, 2, 500, 128, seed=520)
    o1, l1 = cuda_api.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True, rope_base=10000.0)
    o2, l2 = _gpu(cuda_api, q, k, v, (1, 8, 2, 500, 128, 1, 0, 10000.0, False, 1.0, 1.0, False))
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)


@pytest.mark.parametrize("D", [64, 128])
def test_half_split_is_interleaved_on_permuted_dims(cuda_api, D):
    """Half-split RoPE equals interleaved RoPE on q and k whose dimensions are permuted so that
    (i, i + D/2) become (2i, 2i+1): the same bits, since both rotate the same numbers the same way."""
    q, k, v = synth.prefill_inputs(1, 4, 2, 400, D, seed=521)
    perm = torch.stack([torch.arange(D // 2), torch.arange(D // 2) + D // 2], 1).reshape(-1)
    o1, l1 = _gpu(cuda_api, q, k, v, (1, 4, 2, 400, D, 1, 0, 10000.0, True, 1.0, 1.0, False))
    qp, kp = q[..., perm].contiguous(), k[..., perm].contiguous()
    o2, l2 = _gpu(cuda_api, qp, kp, v, (1, 4, 2, 400, D, 1, 0, 10000.0, False, 1.0, 1.0, False))
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)


@pytest.mark.parametrize("D,half,ps,ntk", [(128, False, 1.0, 1.0), (64, False, 1.0, 1.0), (128, True, 2.0, 4.0)])
def test_rope_pass_rotates_exactly(cuda_api, D, half, ps, ntk):
    """With RoPE, the forward equals bit for bit the forward without RoPE on q and k rotated by the
    oracle (for half-split pairing with the dimensions permuted to the interleaved order the
    library uses): the library rotates each element in fp64 and rounds it once to bf16, as the
    oracle does, so the attention kernel sees the oracle's rotated operands."""
    B, Hq, Hkv, N, base = 2, 4, 2, 333, 10000.0
    q, k, v = synth.prefill_inputs(B, Hq, Hkv, N, D, seed=523)
    perm = torch.stack([torch.arange(D // 2), torch.arange(D // 2) + D // 2], 1).reshape(-1)

    def rotated(x):
        rows = bits(x).reshape(-1, D)
        pos = np.tile(np.arange(N, dtype=np.int64), rows.shape[0] // N)
        r = oracle.rope_bf16_ex(rows, pos, base, half_split=half, pos_scale=ps, ntk_factor=ntk)
        t = torch.from_numpy(np.ascontiguousarray(r).view(np.int16)).view(torch.bfloat16).reshape(x.shape)
        return t[..., perm].contiguous() if half else t

    o1, l1 = _gpu(cuda_api, q, k, v, (B, Hq, Hkv, N, D, 1, 0, base, half, ps, ntk, False))
    o2, l2 = cuda_api.attn_fwd(rotated(q).cuda(), rotated(k).cuda(), v.cuda(), causal=True, rope_base=0.0)
    torch.cuda.synchronize()
    assert cuda_api.device_status() == 0
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)


def _with_special_values(x, seed):
    """x with a seeded share of its entries replaced by signed zeros (10%), bf16 subnormals (5%) and
    normals of 2^-126 to 2^-120 (5%), whose rotations round into the bf16 subnormal range."""
    rng = np.random.default_rng(seed)
    b = bits(x).copy()
    u = rng.random(b.shape)
    sign = (rng.integers(0, 2, b.shape) << 15).astype(np.uint16)
    sub = rng.integers(1, 0x80, b.shape).astype(np.uint16)
    tiny = ((rng.integers(1, 8, b.shape) << 7) | rng.integers(0, 0x80, b.shape)).astype(np.uint16)
    b = np.where(u < 0.10, sign, b)
    b = np.where((u >= 0.10) & (u < 0.15), sign | sub, b)
    b = np.where((u >= 0.15) & (u < 0.20), sign | tiny, b)
    return torch.from_numpy(b.view(np.int16)).view(torch.bfloat16)


@pytest.mark.parametrize("half", [False, True])
def test_rope_pass_rotates_special_values_exactly(cuda_api, half):
    """The rotation pass on signed zeros, subnormal inputs and results that round to subnormals
    (the paths that leave the field-moving conversions) still equals the oracle's rotation bit for
    bit, checked as in the test above."""
    B, Hq, Hkv, N, D, base = 1, 2, 1, 200, 128, 10000.0
    q, k, v = synth.prefill_inputs(B, Hq, Hkv, N, D, seed=524)
    q, k = _with_special_values(q, 1), _with_special_values(k, 2)
    perm = torch.stack([torch.arange(D // 2), torch.arange(D // 2) + D // 2], 1).reshape(-1)

    def rotated(x):
        rows = bits(x).reshape(-1, D)
        pos = np.tile(np.arange(N, dtype=np.int64), rows.shape[0] // N)
        r = oracle.rope_bf16_ex(rows, pos, base, half_split=half)
        t = torch.from_numpy(np.ascontiguousarray(r).view(np.int16)).view(torch.bfloat16).reshape(x.shape)
        return t[..., perm].contiguous() if half else t

    qr = bits(rotated(q))
    subnormal = ((qr & 0x7F80) == 0) & ((qr & 0x7F) != 0)
    assert np.count_nonzero(subnormal) > 0.005 * qr.size and np.count_nonzero((qr & 0x7FFF) == 0) > 0
    o1, l1 = _gpu(cuda_api, q, k, v, (B, Hq, Hkv, N, D, 1, 0, base, half, 1.0, 1.0, False))
    o2, l2 = cuda_api.attn_fwd(rotated(q).cuda(), rotated(k).cuda(), v.cuda(), causal=True, rope_base=0.0)
    torch.cuda.synchronize()
    assert cuda_api.device_status() == 0
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)


def test_alibi_full_size_all_rows(cuda_api):
    """ALiBi (with half-split RoPE and NTK scaling) on the GQA causal N=8192 workload, every row."""
    cfg = synth.GQA_CAUSAL_N8192
    q, k, v = synth.prefill_inputs_for(cfg)
    case = (cfg.B, cfg.Hq, cfg.Hkv, cfg.N, cfg.D, 1, 0, cfg.rope_base, True, 1.0, 4.0, True)
    o, lse = _gpu(cuda_api, q, k, v, case)
    assert cuda_api.device_status() == 0
    o_ref, lse_ref = _oracle(q, k, v, case)
    og, lg = f64(o), f64(lse)
    _close(case, og, lg, o_ref, lse_ref, "alibi full size")
    d = og - o_ref
    report("alibi_" + cfg.name, float(np.abs(d).max()), float(np.sqrt((d ** 2).sum() / (o_ref ** 2).sum())),
           float(np.abs(lg - lse_ref).max()))
