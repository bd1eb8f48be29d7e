"""Backward parity (GPU only): gradients from attn_bwd against the fp64 oracle's backward.

The GPU path runs its own forward (O and LSE) and then the backward, as training does; the oracle
computes the exact gradients of sum(O * dO) from the same bf16 inputs. Tolerances (the gradients
are stored in bf16, and P and dS pass through bf16 on the way to the tensor cores): relative RMS
<= 5e-3 over each gradient tensor, and max-abs <= max|gradient| / 128 (four bf16 half-ulps at the
largest gradient). Both scales have a floor (RMS 1e-3, max-abs 1e-4): with one visible key per
row the softmax is constant, so dS = dP - D and hence dq and dk are exactly zero, and what remains is
fp32 cancellation of two equal dot products.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_attention_161_b200 import synth

pytestmark = pytest.mark.gpu

GRAD_REL_RMS = 5e-3
GRAD_MAX_ABS_FRAC = 1.0 / 128
RMS_FLOOR = 1e-3
ABS_FLOOR = 1e-4

# B, Hq, Hkv, N, D, causal, window, rope_base
CASES = [
    (1, 1, 1, 128, 64, 0, 0, 0.0),
    (1, 2, 1, 200, 128, 1, 0, 10000.0),
    (2, 2, 2, 129, 128, 0, 0, 0.0),
    (1, 4, 2, 300, 64, 1, 0, 0.0),
    (1, 4, 4, 500, 128, 1, 100, 10000.0),
    (1, 8, 2, 256, 128, 1, 0, 500000.0),
    (1, 2, 2, 17, 128, 1, 0, 10000.0),
    (1, 2, 1, 1, 64, 1, 0, 10000.0),
    (1, 4, 2, 640, 128, 0, 0, 10000.0),
    (4, 16, 16, 2048, 128, 1, 0, 10000.0),  # the N=2048 MHA workload's shape
    (1, 4, 2, 700, 64, 1, 200, 10000.0),    # D = 64 through the dQ drain's two column groups, window
    (2, 8, 2, 520, 64, 0, 0, 500000.0),     # D = 64, non-causal, 4 query heads per K/V head
]


def _ids(c):
    return "B%dHq%dHkv%dN%dD%d_c%d_w%d_r%g" % c


def check_grad(name, got, ref):
    x = got.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(x)), name
    d = x - ref
    rel_rms = np.sqrt((d ** 2).mean()) / max(np.sqrt((ref ** 2).mean()), RMS_FLOOR)
    max_abs = np.abs(d).max()
    assert rel_rms <= GRAD_REL_RMS, "%s rel-RMS %.3e" % (name, rel_rms)
    assert max_abs <= GRAD_MAX_ABS_FRAC * np.abs(ref).max() + ABS_FLOOR, "%s max-abs %.3e (max ref %.3e)" % (
        name, max_abs, np.abs(ref).max())
    return float(rel_rms), float(max_abs)


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_backward_vs_oracle(cuda_api, case):
    B, Hq, Hkv, N, D, causal, window, rope = case
    ci = CASES.index(case)
    q, k, v = synth.prefill_inputs(B, Hq, Hkv, N, D, seed=300 + ci)
    dout = synth.randn_bf16((B, Hq, N, D), torch.Generator().manual_seed(400 + ci))
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    o, lse = cuda_api.attn_fwd(qd, kd, vd, causal=causal, window=window, rope_base=rope)
    dq, dk, dv = cuda_api.attn_bwd(qd, kd, vd, o, lse, dod, causal=causal, window=window, rope_base=rope)
    torch.cuda.synchronize()
    assert cuda_api.device_status() == 0
    rq, rk, rv = oracle.attention_bwd(synth.bits(q), synth.bits(k), synth.bits(v), synth.bits(dout), causal=causal,
                                      window=window, rope_base=rope, scale=D ** -0.5)
    check_grad("dq", dq, rq)
    check_grad("dk", dk, rk)
    check_grad("dv", dv, rv)


def test_backward_gqa_equals_repeated_heads(cuda_api):
    """dk, dv of a shared K/V head equal the sums over the copies when K/V are repeated per head."""
    q, k, v = synth.prefill_inputs(1, 4, 2, 300, 128, seed=77)
    dout = synth.randn_bf16((1, 4, 300, 128), torch.Generator().manual_seed(78)).cuda()
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o, lse = cuda_api.attn_fwd(qd, kd, vd, causal=True, rope_base=10000.0)
    dq, dk, dv = cuda_api.attn_bwd(qd, kd, vd, o, lse, dout, causal=True, rope_base=10000.0)
    kr, vr = kd.repeat_interleave(2, dim=1), vd.repeat_interleave(2, dim=1)
    o2, lse2 = cuda_api.attn_fwd(qd, kr, vr, causal=True, rope_base=10000.0)
    dq2, dk2, dv2 = cuda_api.attn_bwd(qd, kr, vr, o2, lse2, dout, causal=True, rope_base=10000.0)
    assert_same_up_to_sum_order(dq, dq2)
    for a, b in ((dk, dk2), (dv, dv2)):
        summed = b.float().reshape(1, 2, 2, 300, 128).sum(dim=2)
        assert float((a.float() - summed).abs().max()) <= 2.0 ** -7 * float(summed.abs().max())


def assert_same_up_to_sum_order(a, b):
    """a and b are dq from two calls: fp32 sums of the same partials (one per key tile) in different
    orders, rounded to bf16. Reordering moves an fp32 sum by a few 2^-24 of the partials' size, and
    the chain rule makes each row's dS sum to zero, so partials can cancel to a result far smaller
    than they are: the bound is one bf16 ulp of the element or 2^-16 of the largest |dq|."""
    af, bf = a.float(), b.float()
    tol = torch.maximum(af.abs() * 2.0 ** -7, torch.full_like(af, 2.0 ** -16 * float(af.abs().max())))
    bad = (af - bf).abs() > tol
    if bool(bad.any()):
        i = int(torch.nonzero(bad.flatten())[0])
        raise AssertionError(f"dq repeats differ at flat index {i}: {float(af.flatten()[i])} vs "
                             f"{float(bf.flatten()[i])}, max |dq| {float(af.abs().max())}")


def test_backward_deterministic(cuda_api):
    """Two backward calls: dK and dV are each accumulated by one CTA in a fixed order, so their bits
    repeat. dQ is a sum of fp32 partials, one per key tile, added into device memory in the order
    the CTAs get there; repeats agree up to that summation order."""
    q, k, v = (x.cuda() for x in synth.prefill_inputs(1, 8, 2, 700, 128, seed=79))
    dout = synth.randn_bf16((1, 8, 700, 128), torch.Generator().manual_seed(80)).cuda()
    o, lse = cuda_api.attn_fwd(q, k, v, causal=True, rope_base=10000.0)
    first = cuda_api.attn_bwd(q, k, v, o, lse, dout, causal=True, rope_base=10000.0)
    second = cuda_api.attn_bwd(q, k, v, o, lse, dout, causal=True, rope_base=10000.0)
    torch.cuda.synchronize()
    assert cuda_api.device_status() == 0
    assert_same_up_to_sum_order(first[0], second[0])
    for a, b in zip(first[1:], second[1:]):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_backward_workload_full_size(cuda_api):
    """The backward the benchmark times (GQA causal N=8192, RoPE 5e5), every element of dq, dk and
    dv against the oracle's full backward, and two exact identities:
    - sum_j dV[b, g, j] = sum over the group's heads and rows of dO (each row of P sums to 1);
    - sum_j R_j dK[b, g, j] = 0 with R_j the rotation at position j (each row of dS sums to 0).
    The two sums are compared within 6 standard deviations of independent per-element errors of
    2^-8 relative (the bf16 rounding of P, dS and the stored gradient)."""
    cfg = synth.GQA_CAUSAL_N8192
    q, k, v = synth.prefill_inputs_for(cfg)
    dout = synth.randn_bf16(tuple(q.shape), torch.Generator().manual_seed(cfg.seed + 1))
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    o, lse = cuda_api.attn_fwd(qd, kd, vd, causal=True, rope_base=cfg.rope_base)
    dq, dk, dv = cuda_api.attn_bwd(qd, kd, vd, o, lse, dod, causal=True, rope_base=cfg.rope_base)
    torch.cuda.synchronize()
    assert cuda_api.device_status() == 0
    rq, rk, rv = oracle.attention_bwd(synth.bits(q), synth.bits(k), synth.bits(v), synth.bits(dout), causal=True,
                                      rope_base=cfg.rope_base, scale=cfg.scale)
    for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        rel, mx = check_grad(name, got, ref)
        print("PARITY bwd_%s_%s rel_rms=%.3e max_abs=%.3e max_ref=%.3e" % (name, cfg.name, rel, mx,
                                                                         float(np.abs(ref).max())))
    del rq, rk, rv
    G = cfg.Hq // cfg.Hkv
    dv64 = dv.double().cpu()
    lhs = dv64.sum(dim=2)                                                   # [B, Hkv, D]
    rhs = dout.double().reshape(cfg.B, cfg.Hkv, G, cfg.N, cfg.D).sum(dim=(2, 3))
    bound = 6 * 2.0 ** -8 * dv64.pow(2).sum(dim=2).sqrt() + 1e-6
    assert bool(((lhs - rhs).abs() <= bound).all()), float(((lhs - rhs).abs() / bound).max())
    dk64 = dk.double().cpu().numpy()
    half = cfg.D // 2
    theta = cfg.rope_base ** (-2.0 * np.arange(half) / cfg.D)
    ang = np.arange(cfg.N)[:, None] * theta[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x0, x1 = dk64[..., 0::2], dk64[..., 1::2]
    rot = np.empty_like(dk64)
    rot[..., 0::2] = x0 * c - x1 * s
    rot[..., 1::2] = x0 * s + x1 * c
    total = rot.sum(axis=2)
    bound_k = 6 * 2.0 ** -8 * np.sqrt((dk64 ** 2).sum(axis=2)) + 1e-6
    assert np.all(np.abs(total) <= bound_k), float((np.abs(total) / bound_k).max())
