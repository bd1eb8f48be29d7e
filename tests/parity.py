"""Shared helpers of the GPU parity tests: tolerances, row sampling, comparisons.

Tolerances (bf16 inputs, fp32 accumulation, against the fp64 oracle):
  output O   max-abs error <= 2e-2 and relative RMS error <= 5e-3 over the compared elements;
  LSE        max-abs error <= 1e-3 (natural log).
Paged decode must additionally equal, bit for bit, the same kernel run on a contiguous copy.
"""
import numpy as np
import torch

import oracle
from exact_attention_161_b200 import synth

O_MAX_ABS = 2e-2
O_REL_RMS = 5e-3
LSE_MAX_ABS = 1e-3


def errors(o_gpu, lse_gpu, o_ref, lse_ref):
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    diff = o_gpu - o_ref
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    rel_rms = float(np.sqrt((diff ** 2).sum() / max((o_ref ** 2).sum(), 1e-300)))
    lse_abs = float(np.abs(np.asarray(lse_gpu, np.float64) - lse_ref).max()) if lse_ref is not None else 0.0
    return max_abs, rel_rms, lse_abs


def assert_close(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    assert np.all(np.isfinite(np.asarray(o_gpu, np.float64))), "non-finite output " + what
    max_abs, rel_rms, lse_abs = errors(o_gpu, lse_gpu, o_ref, lse_ref)
    assert max_abs <= O_MAX_ABS, "%s O max-abs %.3e > %.0e" % (what, max_abs, O_MAX_ABS)
    assert rel_rms <= O_REL_RMS, "%s O rel-RMS %.3e > %.0e" % (what, rel_rms, O_REL_RMS)
    assert lse_abs <= LSE_MAX_ABS, "%s LSE max-abs %.3e > %.0e" % (what, lse_abs, LSE_MAX_ABS)
    return max_abs, rel_rms, lse_abs


def report(what, max_abs, rel_rms, lse_abs):
    """Print the measured errors of a parity case (shown with pytest -s)."""
    print("PARITY %s max_abs=%.3e rel_rms=%.3e lse_max_abs=%.3e" % (what, max_abs, rel_rms, lse_abs))


def sample_rows(B, Hq, N, per_head=12, heads=None, seed=0):
    """Flat row ids ((b*Hq + h)*N + i): every head (or the given ones), the first and last
    rows, both sides of every tile boundary near the start and end, and random rows."""
    rng = np.random.default_rng(seed)
    fixed = {0, 1, 2, 127, 128, 129, N // 2, N - 129, N - 128, N - 2, N - 1}
    rows = []
    for b in range(B):
        for h in (heads if heads is not None else range(Hq)):
            picks = {i for i in fixed if 0 <= i < N}
            picks |= set(rng.integers(0, N, size=max(0, per_head - len(picks))).tolist())
            rows += [(b * Hq + h) * N + i for i in sorted(picks)]
    return np.array(rows, dtype=np.int64)


def to_cuda(*ts):
    return [t.cuda() for t in ts]


def f64(t):
    """bf16/fp32 CUDA tensor -> float64 numpy (exact)."""
    return t.detach().float().cpu().numpy().astype(np.float64)


def bits(t):
    return synth.bits(t.cpu())


def oracle_prefill(q, k, v, causal, window, rope_base, scale, rows=None):
    return oracle.attention(bits(q), bits(k), bits(v), causal=causal, window=window, rope_base=rope_base,
                            scale=scale, rows=rows)


def oracle_decode(cache, scale=None):
    return oracle.decode_paged(bits(cache.q), bits(cache.k_pages), bits(cache.v_pages), cache.block_table.numpy(),
                               cache.seq_lens.numpy(), scale=scale)
