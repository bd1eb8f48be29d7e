"""fp64 CPU oracle for exact attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package. It shares no code with the CUDA path: the arithmetic lives in
``oracle.c`` (plain C, fp64, one materialised score row per query); this module only
marshals numpy arrays.

Tensors cross as raw bf16 bit patterns (``numpy.uint16``), so the oracle sees exactly the
bits the GPU sees. Results come back as float64.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None


def _lib(path: str = None):
    global _LIB
    if path is not None:
        lib = ctypes.CDLL(path)
        _declare(lib)
        return lib
    if _LIB is None:
        _LIB = ctypes.CDLL(_build.build())
        _declare(_LIB)
    return _LIB


def _declare(lib):
    p = ctypes.c_void_p
    i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
    lib.oracle_attention.argtypes = [p, p, p, i32, i32, i32, i32, i32, i32, i32, f64, f64, p, i64,
                                     p, p, i32]
    lib.oracle_attention.restype = i32
    lib.oracle_decode_paged.argtypes = [p, p, p, p, p, i32, i32, i32, i32, i32, i32, i32, f64, p, p,
                                        i32]
    lib.oracle_decode_paged.restype = i32
    lib.oracle_decode_step.argtypes = [p, p, p, p, p, p, p, i32, i32, i32, i32, i32, i32, i32, i32, f64, f64, p,
                                       p, i32]
    lib.oracle_decode_step.restype = i32
    lib.oracle_rope_bf16_ex.argtypes = [p, p, i64, i32, f64, i32, f64, f64, p]
    lib.oracle_rope_bf16_ex.restype = i32
    lib.oracle_attention_pos.argtypes = [p, p, p, i32, i32, i32, i32, i32, i32, i32, f64, i32, f64, f64, p, f64, p,
                                         i64, p, p, i32]
    lib.oracle_attention_pos.restype = i32
    lib.oracle_e4m3_to_f64.argtypes = [p, i64, p]
    lib.oracle_e4m3_to_f64.restype = None
    lib.oracle_attention_bwd_dq_rows.argtypes = [p, p, p, p, i32, i32, i32, i32, i32, i32, i32, f64, f64, p, i64, p,
                                                 i32]
    lib.oracle_attention_bwd_dq_rows.restype = i32
    lib.oracle_rope_bf16.argtypes = [p, p, i64, i32, f64, p]
    lib.oracle_rope_bf16.restype = i32
    lib.oracle_round_bf16_array.argtypes = [p, i64, p]
    lib.oracle_round_bf16_array.restype = None
    lib.oracle_max_threads.argtypes = []
    lib.oracle_max_threads.restype = i32
    lib.oracle_attention_f64.argtypes = [p, p, p, i32, i32, i32, i32, i32, i32, i32, f64, f64, i32, p, p]
    lib.oracle_attention_f64.restype = i32
    lib.oracle_attention_bwd_f64.argtypes = [p, p, p, p, i32, i32, i32, i32, i32, i32, i32, f64, f64, i32, p,
                                             p, p, i32]
    lib.oracle_attention_bwd_f64.restype = i32
    lib.oracle_attention_bwd.argtypes = [p, p, p, p, i32, i32, i32, i32, i32, i32, i32, f64, f64, p, p, p, i32]
    lib.oracle_attention_bwd.restype = i32


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def _bits(a):
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("oracle inputs are bf16 bit patterns (numpy.uint16), got %s" % a.dtype)
    return a


class OracleError(RuntimeError):
    pass


def max_threads(lib=None) -> int:
    return int((lib or _lib()).oracle_max_threads())


def attention(q, k, v, causal=False, window=0, rope_base=0.0, scale=None, rows=None,
              nthreads=0, lib=None):
    """Exact attention in fp64.

    q: uint16 [B, Hq, N, D]; k, v: uint16 [B, Hkv, N, D] (bf16 bits).
    rows: None for all rows, else int64 flat row ids ((b*Hq + h)*N + i).
    Returns (o, lse): float64 [B, Hq, N, D] and [B, Hq, N], or [len(rows), D] and [len(rows)].
    """
    lib = lib or _lib()
    q, k, v = _bits(q), _bits(k), _bits(v)
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, D) or v.shape != k.shape:
        raise ValueError("k/v shape mismatch")
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    if rows is None:
        n = B * Hq * N
        rows_arr = None
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        n = rows_arr.size
    o = np.empty((n, D), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    st = lib.oracle_attention(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, N, D, int(causal),
                              int(window), float(rope_base), float(scale), _ptr(rows_arr),
                              n, _ptr(o), _ptr(lse), int(nthreads))
    if st != 0:
        raise OracleError("oracle_attention failed with status %d" % st)
    if rows is None:
        return o.reshape(B, Hq, N, D), lse.reshape(B, Hq, N)
    return o, lse


def attention_f64(q, k, v, causal=False, window=0, rope_base=0.0, scale=None, round_rotated=False, lib=None):
    """Forward on float64 inputs (q [B,Hq,N,D], k/v [B,Hkv,N,D]); round_rotated=False keeps the
    rotation exact. Returns (o, lse) float64."""
    lib = lib or _lib()
    q, k, v = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v))
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    o = np.empty_like(q)
    lse = np.empty((B, Hq, N))
    st = lib.oracle_attention_f64(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, N, D, int(causal), int(window),
                                  float(rope_base), float(scale), int(bool(round_rotated)), _ptr(o), _ptr(lse))
    if st != 0:
        raise OracleError("oracle_attention_f64 failed with status %d" % st)
    return o, lse


def attention_bwd_f64(q, k, v, dout, causal=False, window=0, rope_base=0.0, scale=None, round_rotated=False,
                      nthreads=0, lib=None):
    """Gradients (dq, dk, dv) of sum(O * dout) on float64 inputs."""
    lib = lib or _lib()
    q, k, v, dout = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v, dout))
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    st = lib.oracle_attention_bwd_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), B, Hq, Hkv, N, D, int(causal),
                                      int(window), float(rope_base), float(scale), int(bool(round_rotated)),
                                      _ptr(dq), _ptr(dk), _ptr(dv), int(nthreads))
    if st != 0:
        raise OracleError("oracle_attention_bwd_f64 failed with status %d" % st)
    return dq, dk, dv


def attention_bwd(q, k, v, dout, causal=False, window=0, rope_base=0.0, scale=None, nthreads=0, lib=None):
    """Gradients (dq, dk, dv) of sum(O * dout) for bf16 bit-pattern inputs (uint16), float64 out;
    the rotated q, k are rounded to bf16 as in the forward."""
    lib = lib or _lib()
    q, k, v, dout = _bits(q), _bits(k), _bits(v), _bits(dout)
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    dq = np.empty(q.shape)
    dk = np.empty(k.shape)
    dv = np.empty(v.shape)
    st = lib.oracle_attention_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), B, Hq, Hkv, N, D, int(causal), int(window),
                                  float(rope_base), float(scale), _ptr(dq), _ptr(dk), _ptr(dv), int(nthreads))
    if st != 0:
        raise OracleError("oracle_attention_bwd failed with status %d" % st)
    return dq, dk, dv


def decode_paged(q, k_pages, v_pages, block_table, seq_lens, scale=None, nthreads=0, lib=None):
    """One-token decode over a paged KV cache, in fp64.

    q: uint16 [S, Hq, D]; k_pages, v_pages: uint16 [num_pages, Hkv, page_size, D];
    block_table: int32 [S, max_blocks]; seq_lens: int32 [S].
    Returns (o [S, Hq, D], lse [S, Hq]) as float64.
    """
    lib = lib or _lib()
    q, k_pages, v_pages = _bits(q), _bits(k_pages), _bits(v_pages)
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    S, Hq, D = q.shape
    num_pages, Hkv, page_size, D2 = k_pages.shape
    if D2 != D or v_pages.shape != k_pages.shape or bt.shape[0] != S or sl.shape != (S,):
        raise ValueError("decode shape mismatch")
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    o = np.empty((S, Hq, D), dtype=np.float64)
    lse = np.empty((S, Hq), dtype=np.float64)
    st = lib.oracle_decode_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(bt), _ptr(sl), S,
                                 bt.shape[1], num_pages, page_size, Hq, Hkv, D, float(scale),
                                 _ptr(o), _ptr(lse), int(nthreads))
    if st != 0:
        raise OracleError("oracle_decode_paged failed with status %d" % st)
    return o, lse


def decode_step(q, k_new, v_new, k_pages, v_pages, block_table, seq_lens, rope_base=0.0, scale=None, nthreads=0,
                lib=None):
    """Decode step in fp64: append the new tokens' keys (rotated) and values to the paged cache, then
    attend each new token's rotated query causally to the cache.

    q: uint16 [S, T, Hq, D]; k_new, v_new: uint16 [S, T, Hkv, D] or both None; k_pages, v_pages:
    uint16 [num_pages, Hkv, page_size, D] (not modified: the updated copies are returned);
    block_table: int32 [S, max_blocks]; seq_lens: int32 [S], counting the T new tokens.
    Returns (o [S, T, Hq, D], lse [S, T, Hq], k_pages', v_pages').
    """
    lib = lib or _lib()
    q = _bits(q)
    kp, vp = _bits(k_pages).copy(), _bits(v_pages).copy()
    if (k_new is None) != (v_new is None):
        raise ValueError("k_new and v_new go together")
    kn = _bits(k_new) if k_new is not None else None
    vn = _bits(v_new) if v_new is not None else None
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    S, T, Hq, D = q.shape
    num_pages, Hkv, page_size, D2 = kp.shape
    if D2 != D or vp.shape != kp.shape or bt.shape[0] != S or sl.shape != (S,):
        raise ValueError("decode shape mismatch")
    if kn is not None and (kn.shape != (S, T, Hkv, D) or vn.shape != kn.shape):
        raise ValueError("k_new/v_new shape mismatch")
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    o = np.empty((S, T, Hq, D), dtype=np.float64)
    lse = np.empty((S, T, Hq), dtype=np.float64)
    st = lib.oracle_decode_step(_ptr(q), _ptr(kn), _ptr(vn), _ptr(kp), _ptr(vp), _ptr(bt), _ptr(sl), S, T,
                                bt.shape[1], num_pages, page_size, Hq, Hkv, D, float(rope_base), float(scale),
                                _ptr(o), _ptr(lse), int(nthreads))
    if st != 0:
        raise OracleError("oracle_decode_step failed with status %d" % st)
    return o, lse, kp, vp


def attention_pos(q, k, v, causal=False, window=0, rope_base=0.0, rope_half_split=False, rope_pos_scale=1.0,
                  rope_ntk_factor=1.0, alibi_slopes=None, scale=None, rows=None, nthreads=0, lib=None):
    """Exact attention in fp64 with position variants: half-split RoPE pairing, Position
    Interpolation (positions divided by rope_pos_scale), NTK-aware base scaling (base times
    rope_ntk_factor^(D/(D-2))), and ALiBi (alibi_slopes: per-query-head slopes m_h, logits minus
    m_h (i - j)). Shapes and returns as ``attention``."""
    lib = lib or _lib()
    q, k, v = _bits(q), _bits(k), _bits(v)
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, D) or v.shape != k.shape:
        raise ValueError("k/v shape mismatch")
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    slopes = None if alibi_slopes is None else np.ascontiguousarray(alibi_slopes, dtype=np.float64)
    if slopes is not None and slopes.shape != (Hq,):
        raise ValueError("alibi_slopes must have Hq entries")
    if rows is None:
        n = B * Hq * N
        rws = None
    else:
        rws = np.ascontiguousarray(rows, dtype=np.int64)
        n = rws.shape[0]
    o = np.empty((n, D), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    st = lib.oracle_attention_pos(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, N, D, int(causal), int(window),
                                  float(rope_base), int(bool(rope_half_split)), float(rope_pos_scale),
                                  float(rope_ntk_factor), _ptr(slopes), float(scale), _ptr(rws), n, _ptr(o), _ptr(lse),
                                  int(nthreads))
    if st != 0:
        raise OracleError("oracle_attention_pos failed with status %d" % st)
    if rows is None:
        return o.reshape(B, Hq, N, D), lse.reshape(B, Hq, N)
    return o, lse


def rope_bf16_ex(x, pos, base, half_split=False, pos_scale=1.0, ntk_factor=1.0, lib=None):
    """``rope_bf16`` with a choice of pairing ((2i, 2i+1) or (i, i + D/2)), Position Interpolation
    and NTK-aware base scaling."""
    lib = lib or _lib()
    x = _bits(x)
    n, D = x.shape
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    out = np.empty_like(x)
    st = lib.oracle_rope_bf16_ex(_ptr(x), _ptr(pos), n, D, float(base), int(bool(half_split)), float(pos_scale),
                                 float(ntk_factor), _ptr(out))
    if st != 0:
        raise OracleError("oracle_rope_bf16_ex failed with status %d" % st)
    return out


def e4m3_to_f64(x, lib=None):
    """FP8 e4m3 bit patterns (numpy uint8) -> exact float64 values."""
    lib = lib or _lib()
    x = np.ascontiguousarray(x)
    if x.dtype != np.uint8:
        raise TypeError("e4m3 inputs are bit patterns (numpy.uint8), got %s" % x.dtype)
    out = np.empty(x.shape, dtype=np.float64)
    lib.oracle_e4m3_to_f64(_ptr(x), x.size, _ptr(out))
    return out


def attention_fp8(q8, k8, v8, descale_q, descale_k, descale_v, causal=False, window=0, scale=None, rows=None,
                  nthreads=0, lib=None):
    """Exact attention on FP8 e4m3 inputs: q = q8 * descale_q, k = k8 * descale_k, v = v8 * descale_v
    (per-tensor scales), in fp64. Every e4m3 value is exactly a bf16 value, so the bf16-input
    attention runs on the converted bits with the score scale times descale_q * descale_k, and the
    output is multiplied by descale_v. Shapes and returns as ``attention``."""
    lib = lib or _lib()
    conv = []
    for x in (q8, k8, v8):
        val = e4m3_to_f64(x, lib=lib)
        b = round_bf16(val, lib=lib)
        if not np.array_equal(bf16_bits_to_f64(b), val):
            raise OracleError("e4m3 value not exact in bf16 (NaN input?)")
        conv.append(b)
    D = q8.shape[-1]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    o, lse = attention(conv[0], conv[1], conv[2], causal=causal, window=window, rope_base=0.0,
                       scale=float(scale) * float(descale_q) * float(descale_k), rows=rows, nthreads=nthreads, lib=lib)
    return o * float(descale_v), lse


def attention_bwd_dq_rows(q, k, v, dout, rows, causal=False, window=0, rope_base=0.0, scale=None, nthreads=0,
                          lib=None):
    """dq of the given query rows (flat ids (b*Hq + h)*N + i) for bf16 inputs, in fp64, with the steps
    of ``attention_bwd`` for one row. Returns [len(rows), D]."""
    lib = lib or _lib()
    q, k, v, dout = _bits(q), _bits(k), _bits(v), _bits(dout)
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    if D > 512:
        raise ValueError("D above 512")
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    rws = np.ascontiguousarray(rows, dtype=np.int64)
    dq = np.empty((rws.shape[0], D), dtype=np.float64)
    st = lib.oracle_attention_bwd_dq_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), B, Hq, Hkv, N, D, int(causal),
                                          int(window), float(rope_base), float(scale), _ptr(rws), rws.shape[0],
                                          _ptr(dq), int(nthreads))
    if st != 0:
        raise OracleError("oracle_attention_bwd_dq_rows failed with status %d" % st)
    return dq


def rope_bf16(x, pos, base, lib=None):
    """Rotate rows of x (uint16 [n, D]) at positions pos (int64 [n]); returns uint16 [n, D]."""
    lib = lib or _lib()
    x = _bits(x)
    n, D = x.shape
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    out = np.empty_like(x)
    st = lib.oracle_rope_bf16(_ptr(x), _ptr(pos), n, D, float(base), _ptr(out))
    if st != 0:
        raise OracleError("oracle_rope_bf16 failed with status %d" % st)
    return out


def round_bf16(x, lib=None):
    """Round float64 values to bf16 (ties to even); returns the uint16 bit patterns."""
    lib = lib or _lib()
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    lib.oracle_round_bf16_array(_ptr(x), x.size, _ptr(out))
    return out


def bf16_bits_to_f64(bits):
    """Exact value of bf16 bit patterns (plain reinterpretation, no arithmetic)."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
