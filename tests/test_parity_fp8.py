"""FP8 e4m3 prefill parity (GPU only) against exact fp64 attention on the dequantised inputs.

Tolerances, from the arithmetic: the inputs are the same e4m3 values on both sides and the scores
accumulate exact e4m3 products in fp32, so the LSE keeps the bf16 path's bound. P is rounded to
e4m3 (3 mantissa bits, nearest even: relative error <= 2^-4, about 2.6% RMS over the values P
takes) before the P V product; each output is a weighted mean of V rows, so its error is that
relative rounding carried through the same weights: rel-RMS about 2.6% (bound 4e-2) and max-abs
at most 2^-4 max|v| when every rounding error lines up (bound 2^-3 max|v|, leaving room for
probabilities below e4m3's normal range).
"""
import numpy as np
import pytest
import torch

import oracle
from exact_attention_161_b200 import synth
from parity import f64, report

pytestmark = pytest.mark.gpu

FP8_REL_RMS = 4e-2
FP8_LSE_MAX_ABS = 1e-3

# B, Hq, Hkv, N, causal, window
CASES = [
    (1, 4, 2, 300, 1, 0),
    (2, 2, 2, 129, 0, 0),
    (1, 8, 2, 1000, 1, 200),
    (1, 2, 1, 1, 1, 0),
    (1, 4, 4, 640, 0, 0),
    (1, 32, 8, 1024, 1, 0),
]


def _ids(c):
    return "B%dHq%dHkv%dN%d_c%d_w%d" % c


def _check(o, lse, o_ref, lse_ref, vmax, what):
    og, lg = f64(o), f64(lse)
    assert np.all(np.isfinite(og)), what
    d = og - o_ref
    rel = np.sqrt((d ** 2).sum() / max((o_ref ** 2).sum(), 1e-300))
    mx = np.abs(d).max()
    le = np.abs(lg - lse_ref).max()
    assert rel <= FP8_REL_RMS, "%s rel-RMS %.3e" % (what, rel)
    assert mx <= 2.0 ** -3 * vmax, "%s max-abs %.3e (max|v| %.3f)" % (what, mx, vmax)
    assert le <= FP8_LSE_MAX_ABS, "%s LSE max-abs %.3e" % (what, le)
    return rel, mx, le


def _run(api, f, causal, window):
    o, lse = api.attn_fwd_fp8(f.q8.cuda(), f.k8.cuda(), f.v8.cuda(), f.descale_q, f.descale_k, f.descale_v,
                              causal=causal, window=window)
    torch.cuda.synchronize()
    return o, lse


def _vmax(f):
    return float(np.abs(oracle.e4m3_to_f64(f.v8.numpy())).max()) * f.descale_v


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_fp8_vs_oracle(cuda_api, case):
    B, Hq, Hkv, N, causal, window = case
    f = synth.fp8_inputs(B, Hq, Hkv, N, 128, seed=700 + CASES.index(case))
    o, lse = _run(cuda_api, f, causal, window)
    assert cuda_api.device_status() == 0
    o_ref, lse_ref = oracle.attention_fp8(f.q8.numpy(), f.k8.numpy(), f.v8.numpy(), f.descale_q, f.descale_k,
                                          f.descale_v, causal=causal, window=window)
    _check(o, lse, o_ref, lse_ref, _vmax(f), _ids(case))


def test_fp8_value_scale_is_exact(cuda_api):
    """Doubling descale_v doubles every output exactly; the LSE does not move."""
    f = synth.fp8_inputs(1, 4, 2, 300, 128, seed=720)
    o1, l1 = _run(cuda_api, f, 1, 0)
    f.descale_v *= 2.0
    o2, l2 = _run(cuda_api, f, 1, 0)
    assert torch.equal((o1.float() * 2).to(torch.bfloat16).view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1, l2)


def test_fp8_full_size_all_rows(cuda_api):
    """The GQA causal N=8192 workload's shape in e4m3, every row."""
    cfg = synth.GQA_CAUSAL_N8192
    f = synth.fp8_inputs_for(cfg)
    o, lse = _run(cuda_api, f, 1, 0)
    assert cuda_api.device_status() == 0
    o_ref, lse_ref = oracle.attention_fp8(f.q8.numpy(), f.k8.numpy(), f.v8.numpy(), f.descale_q, f.descale_k,
                                          f.descale_v, causal=True)
    rel, mx, le = _check(o, lse, o_ref, lse_ref, _vmax(f), "fp8 full size")
    report("fp8_" + cfg.name, mx, rel, le)
