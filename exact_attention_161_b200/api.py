"""Python binding of the C ABI in ``include/attn.h`` (argument marshalling only).

Every computation runs in ``libattn_b200.so``; this module checks tensor dtypes, shapes and
devices, allocates outputs when the caller passes none, and forwards raw device pointers and the
current CUDA stream. Importing it loads the library and raises if it is missing: there is no
CPU fallback.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattn_b200.so")

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_CUDA = 3
ATTN_ERR_DEVICE_CHECK = 4
ATTN_ERR_TIMEOUT = 5
STATUS_NAMES = {0: "ATTN_OK", 1: "ATTN_ERR_INVALID_ARG", 2: "ATTN_ERR_UNSUPPORTED", 3: "ATTN_ERR_CUDA",
                4: "ATTN_ERR_DEVICE_CHECK", 5: "ATTN_ERR_TIMEOUT"}
DEVICE_TIMEOUT, DEVICE_BAD_PAGE, DEVICE_BAD_SEQLEN = 1, 2, 4

# Every function include/attn.h declares, with its ctypes signature.
_p, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "attn_fwd": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _f, _f, _p]),
    "attn_fwd_pos": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _f, _i, _f, _f, _p, _f, _p]),
    "attn_fwd_fp8": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _f, _f, _f, _f, _p]),
    "attn_bwd_workspace_size": (_sz, [_i, _i, _i, _i, _i, _f]),
    "attn_bwd": (_i, [_p, _p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _f, _f, _p, _sz, _p]),
    "attn_decode_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "attn_decode_paged": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _f, _p, _p, _p, _sz, _p]),
    "attn_decode_paged_noalloc": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _f, _p, _p, _p]),
    "attn_decode_step_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "attn_decode_step": (_i, [_p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _f, _f, _p, _p, _p, _sz,
                              _p]),
    "attn_debug_drop_copy": (None, [_i]),
    "attn_get_device_status": (_i, [_p, ctypes.POINTER(ctypes.c_int)]),
    "attn_last_error": (ctypes.c_char_p, []),
    "attn_version": (ctypes.c_char_p, []),
    "attn_shutdown": (None, []),
}


class AttnError(RuntimeError):
    def __init__(self, status, message):
        super().__init__("%s: %s" % (STATUS_NAMES.get(status, status), message))
        self.status = status


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError("CUDA library %s is missing; build it with `python -m exact_attention_161_b200.build` "
                          "(there is no CPU fallback)" % path)
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = load()


def _check(status):
    if status != ATTN_OK:
        raise AttnError(status, lib.attn_last_error().decode())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dev_tensor(t, name, dtype):
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise TypeError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return ctypes.c_void_p(t.data_ptr())


def version() -> str:
    return lib.attn_version().decode()


def last_error() -> str:
    return lib.attn_last_error().decode()


def shutdown() -> None:
    lib.attn_shutdown()


def attn_fwd(q, k, v, causal=False, window=0, rope_base=0.0, scale=0.0, o=None, lse=None, want_lse=True,
             stream=None):
    """Exact attention forward. q [B,Hq,N,D], k/v [B,Hkv,N,D] bf16 CUDA tensors.
    Returns (o [B,Hq,N,D] bf16, lse [B,Hq,N] fp32 or None)."""
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, D) or v.shape != k.shape:
        raise ValueError("k and v must be [B, Hkv, N, D] matching q")
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    args = [_dev_tensor(q, "q", torch.bfloat16), _dev_tensor(k, "k", torch.bfloat16),
            _dev_tensor(v, "v", torch.bfloat16), _dev_tensor(o, "o", torch.bfloat16),
            _dev_tensor(lse, "lse", torch.float32) if lse is not None else None]
    _check(lib.attn_fwd(*args, B, Hq, Hkv, N, D, int(bool(causal)), int(window), float(rope_base), float(scale),
                        _stream(stream)))
    return o, lse


def attn_fwd_pos(q, k, v, causal=False, window=0, rope_base=0.0, rope_half_split=False, rope_pos_scale=1.0,
                 rope_ntk_factor=1.0, alibi_slopes=None, scale=0.0, o=None, lse=None, want_lse=True, stream=None):
    """attn_fwd with position variants: half-split RoPE pairing, Position Interpolation
    (rope_pos_scale), NTK-aware base scaling (rope_ntk_factor) and ALiBi (alibi_slopes: fp32 [Hq]
    CUDA tensor of per-head slopes, causal only). Returns (o, lse) as attn_fwd."""
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, D) or v.shape != k.shape:
        raise ValueError("k and v must be [B, Hkv, N, D] with q [B, Hq, N, D]")
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    if alibi_slopes is not None and tuple(alibi_slopes.shape) != (Hq,):
        raise ValueError("alibi_slopes must be [Hq]")
    _check(lib.attn_fwd_pos(_dev_tensor(q, "q", torch.bfloat16), _dev_tensor(k, "k", torch.bfloat16),
                            _dev_tensor(v, "v", torch.bfloat16), _dev_tensor(o, "o", torch.bfloat16),
                            _dev_tensor(lse, "lse", torch.float32) if lse is not None else None, B, Hq, Hkv, N, D,
                            int(causal), int(window), float(rope_base), int(bool(rope_half_split)),
                            float(rope_pos_scale), float(rope_ntk_factor),
                            _dev_tensor(alibi_slopes, "alibi_slopes", torch.float32) if alibi_slopes is not None
                            else None, float(scale), _stream(stream)))
    return o, lse


def attn_fwd_fp8(q8, k8, v8, descale_q, descale_k, descale_v, causal=False, window=0, scale=0.0, o=None, lse=None,
                 want_lse=True, stream=None):
    """FP8 attention forward. q8 [B,Hq,N,128], k8/v8 [B,Hkv,N,128]: e4m3 bit patterns as uint8 CUDA
    tensors, with per-tensor descales. Returns (o [B,Hq,N,128] bf16, lse [B,Hq,N] fp32 or None)."""
    B, Hq, N, D = q8.shape
    Hkv = k8.shape[1]
    if k8.shape != (B, Hkv, N, D) or v8.shape != k8.shape:
        raise ValueError("k8 and v8 must be [B, Hkv, N, D] with q8 [B, Hq, N, D]")
    if o is None:
        o = torch.empty((B, Hq, N, D), dtype=torch.bfloat16, device=q8.device)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q8.device)
    _check(lib.attn_fwd_fp8(_dev_tensor(q8, "q8", torch.uint8), _dev_tensor(k8, "k8", torch.uint8),
                            _dev_tensor(v8, "v8", torch.uint8), _dev_tensor(o, "o", torch.bfloat16),
                            _dev_tensor(lse, "lse", torch.float32) if lse is not None else None, B, Hq, Hkv, N, D,
                            int(causal), int(window), float(descale_q), float(descale_k), float(descale_v),
                            float(scale), _stream(stream)))
    return o, lse


def bwd_workspace_size(B, Hq, Hkv, N, D, rope_base=0.0) -> int:
    return int(lib.attn_bwd_workspace_size(B, Hq, Hkv, N, D, float(rope_base)))


def attn_bwd(q, k, v, o, lse, dout, causal=False, window=0, rope_base=0.0, scale=0.0, dq=None, dk=None, dv=None,
             workspace=None, stream=None):
    """Attention backward. q/o/dout [B,Hq,N,D], k/v [B,Hkv,N,D] bf16, lse [B,Hq,N] fp32 (from
    attn_fwd with the same arguments). Returns (dq, dk, dv), bf16."""
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, D) or v.shape != k.shape or o.shape != q.shape or dout.shape != q.shape:
        raise ValueError("shape mismatch")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace = torch.empty(bwd_workspace_size(B, Hq, Hkv, N, D, rope_base), dtype=torch.uint8, device=q.device)
    args = [_dev_tensor(t, n, torch.bfloat16) for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"))]
    args += [_dev_tensor(lse, "lse", torch.float32), _dev_tensor(dout, "dout", torch.bfloat16)]
    args += [_dev_tensor(t, n, torch.bfloat16) for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv"))]
    _check(lib.attn_bwd(*args, B, Hq, Hkv, N, D, int(bool(causal)), int(window), float(rope_base), float(scale),
                        _dev_tensor(workspace, "workspace", torch.uint8), workspace.numel(), _stream(stream)))
    return dq, dk, dv


def decode_workspace_size(num_seqs, max_blocks_per_seq, page_size, Hq, D) -> int:
    return int(lib.attn_decode_workspace_size(num_seqs, max_blocks_per_seq, page_size, Hq, D))


def attn_decode_paged(q, k_pages, v_pages, block_table, seq_lens, scale=0.0, o=None, lse=None, want_lse=True,
                      workspace=None, stream=None):
    """One decode step per sequence over a paged KV cache.
    q [S,Hq,D] bf16; k_pages/v_pages [num_pages,Hkv,page_size,D] bf16; block_table [S,max_blocks]
    int32; seq_lens [S] int32 (all CUDA). Returns (o [S,Hq,D] bf16, lse [S,Hq] fp32 or None)."""
    S, Hq, D = q.shape
    num_pages, Hkv, page_size, D2 = k_pages.shape
    if D2 != D or v_pages.shape != k_pages.shape:
        raise ValueError("k_pages/v_pages must be [num_pages, Hkv, page_size, D]")
    max_blocks = block_table.shape[1]
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((S, Hq), dtype=torch.float32, device=q.device)
    need = decode_workspace_size(S, max_blocks, page_size, Hq, D)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    args = [_dev_tensor(q, "q", torch.bfloat16), _dev_tensor(k_pages, "k_pages", torch.bfloat16),
            _dev_tensor(v_pages, "v_pages", torch.bfloat16), _dev_tensor(block_table, "block_table", torch.int32),
            _dev_tensor(seq_lens, "seq_lens", torch.int32)]
    _check(lib.attn_decode_paged(*args, S, max_blocks, num_pages, page_size, Hq, Hkv, D, float(scale),
                                 _dev_tensor(o, "o", torch.bfloat16),
                                 _dev_tensor(lse, "lse", torch.float32) if lse is not None else None,
                                 _dev_tensor(workspace, "workspace", torch.uint8),
                                 workspace.numel() * workspace.element_size(), _stream(stream)))
    return o, lse


def decode_step_workspace_size(num_seqs, q_len, max_blocks_per_seq, page_size, Hq, D) -> int:
    return int(lib.attn_decode_step_workspace_size(num_seqs, q_len, max_blocks_per_seq, page_size, Hq, D))


def attn_decode_step(q, k_pages, v_pages, block_table, seq_lens, k_new=None, v_new=None, rope_base=0.0, scale=0.0,
                     o=None, lse=None, want_lse=True, workspace=None, stream=None):
    """Decode step with q_len new tokens per sequence: append k_new/v_new (keys rotated) into their
    page slots, then attend with the new queries (rotated) causally over the cache.
    q [S,q_len,Hq,D] bf16; k_new/v_new [S,q_len,Hkv,D] bf16 or None; k_pages/v_pages
    [num_pages,Hkv,page_size,D] bf16 (updated in place); block_table [S,max_blocks] int32; seq_lens
    [S] int32 counting the new tokens (all CUDA). Returns (o [S,q_len,Hq,D] bf16, lse [S,q_len,Hq] fp32
    or None)."""
    S, T, Hq, D = q.shape
    num_pages, Hkv, page_size, D2 = k_pages.shape
    if D2 != D or v_pages.shape != k_pages.shape:
        raise ValueError("k_pages/v_pages must be [num_pages, Hkv, page_size, D]")
    if (k_new is None) != (v_new is None):
        raise ValueError("k_new and v_new go together")
    if k_new is not None and (k_new.shape != (S, T, Hkv, D) or v_new.shape != k_new.shape):
        raise ValueError("k_new/v_new must be [S, q_len, Hkv, D]")
    max_blocks = block_table.shape[1]
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((S, T, Hq), dtype=torch.float32, device=q.device)
    need = decode_step_workspace_size(S, T, max_blocks, page_size, Hq, D)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    kn = _dev_tensor(k_new, "k_new", torch.bfloat16) if k_new is not None else None
    vn = _dev_tensor(v_new, "v_new", torch.bfloat16) if v_new is not None else None
    _check(lib.attn_decode_step(_dev_tensor(q, "q", torch.bfloat16), kn, vn,
                                _dev_tensor(k_pages, "k_pages", torch.bfloat16),
                                _dev_tensor(v_pages, "v_pages", torch.bfloat16),
                                _dev_tensor(block_table, "block_table", torch.int32),
                                _dev_tensor(seq_lens, "seq_lens", torch.int32), S, T, max_blocks, num_pages, page_size,
                                Hq, Hkv, D, float(rope_base), float(scale), _dev_tensor(o, "o", torch.bfloat16),
                                _dev_tensor(lse, "lse", torch.float32) if lse is not None else None,
                                _dev_tensor(workspace, "workspace", torch.uint8),
                                workspace.numel() * workspace.element_size(), _stream(stream)))
    return o, lse


DECODE_NOALLOC_MAX_BYTES = 40 << 20


def attn_decode_paged_noalloc(q, k_pages, v_pages, block_table, seq_lens, scale=0.0, o=None, lse=None,
                              want_lse=True, stream=None):
    """attn_decode_paged without a workspace, for callers that cannot allocate device memory at
    call time; its scratch is a fixed 40 MiB array inside the library, shared by every call
    (calls that overlap on the GPU race). Outputs must be passed in to allocate nothing here."""
    S, Hq, D = q.shape
    num_pages, Hkv, page_size, _ = k_pages.shape
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((S, Hq), dtype=torch.float32, device=q.device)
    args = [_dev_tensor(q, "q", torch.bfloat16), _dev_tensor(k_pages, "k_pages", torch.bfloat16),
            _dev_tensor(v_pages, "v_pages", torch.bfloat16), _dev_tensor(block_table, "block_table", torch.int32),
            _dev_tensor(seq_lens, "seq_lens", torch.int32)]
    _check(lib.attn_decode_paged_noalloc(*args, S, block_table.shape[1], num_pages, page_size, Hq, Hkv, D,
                                         float(scale), _dev_tensor(o, "o", torch.bfloat16),
                                         _dev_tensor(lse, "lse", torch.float32) if lse is not None else None,
                                         _stream(stream)))
    return o, lse


def debug_drop_copy(enable: bool) -> None:
    """Test hook: make the next decode calls' first split CTA skip one page copy, so its bounded
    wait runs out and the device status reports a timeout (see attn.h)."""
    lib.attn_debug_drop_copy(1 if enable else 0)


def device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word's bits."""
    flags = ctypes.c_int(0)
    st = lib.attn_get_device_status(_stream(stream), ctypes.byref(flags))
    if st not in (ATTN_OK, ATTN_ERR_DEVICE_CHECK, ATTN_ERR_TIMEOUT):
        _check(st)
    return flags.value
