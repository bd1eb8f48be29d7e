"""Seeded synthetic inputs for the attention workloads.

This module holds no attention arithmetic. It only draws random numbers, rounds them to bf16
and lays out a paged KV cache. The CUDA path and the fp64 oracle both take their inputs from
here, so they see the same bits.

Every tensor is drawn on the CPU from ``torch.Generator('cpu').manual_seed(seed)``: fp32
``randn``, then rounded to bf16 (round to nearest even, which is what ``Tensor.to(bfloat16)``
does). The pages draw Q/K/V i.i.d. N(0, 1), which gives q.k/sqrt(d) unit variance
("attention-transformers", Q "Why is attention scaled by 1/sqrt(dk)?").
"""
import math
from dataclasses import dataclass
from typing import Optional

import torch

BF16_NAN_BITS = 0x7FC0


@dataclass(frozen=True)
class PrefillConfig:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    D: int
    causal: bool
    window: int
    rope_base: float
    seed: int

    @property
    def scale(self) -> float:
        return 1.0 / (self.D ** 0.5)


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    num_seqs: int
    Hq: int
    Hkv: int
    D: int
    page_size: int
    len_lo: int
    len_hi: int
    spare_frac: float
    seed: int

    @property
    def scale(self) -> float:
        return 1.0 / (self.D ** 0.5)


# The five workloads: one single-head case small enough for the oracle, three prefill cases
# (causal MHA + RoPE; causal GQA + RoPE; causal sliding-window GQA + RoPE) and one paged decode.
SINGLE_HEAD_N128 = PrefillConfig("single_head_n128_d64", 1, 1, 1, 128, 64, False, 0, 0.0, 1001)
MHA_CAUSAL_N2048 = PrefillConfig("mha_causal_rope_b4_h16_n2048_d128", 4, 16, 16, 2048, 128, True, 0,
                                 10000.0, 1002)
GQA_CAUSAL_N8192 = PrefillConfig("gqa_causal_rope_b2_hq32_hkv8_n8192_d128", 2, 32, 8, 8192, 128, True,
                                 0, 500000.0, 1003)
GQA_WINDOW_N32768 = PrefillConfig("gqa_window4096_rope_b1_hq32_hkv8_n32768_d128", 1, 32, 8, 32768, 128,
                                  True, 4096, 10000.0, 1004)
PAGED_DECODE_64 = DecodeConfig("paged_decode_s64_hq32_hkv8_d128_p16_len512_16384", 64, 32, 8, 128,
                               16, 512, 16384, 0.10, 1005)

PREFILL_CONFIGS = (SINGLE_HEAD_N128, MHA_CAUSAL_N2048, GQA_CAUSAL_N8192, GQA_WINDOW_N32768)


def _gen(seed: int) -> torch.Generator:
    return torch.Generator(device="cpu").manual_seed(int(seed))


def randn_bf16(shape, gen: torch.Generator) -> torch.Tensor:
    """i.i.d. N(0,1) drawn in fp32 and rounded to bf16."""
    return torch.randn(*shape, generator=gen, dtype=torch.float32).to(torch.bfloat16)


def prefill_inputs(B, Hq, Hkv, N, D, seed):
    """q [B,Hq,N,D], k and v [B,Hkv,N,D], contiguous bf16 CPU tensors."""
    g = _gen(seed)
    q = randn_bf16((B, Hq, N, D), g)
    k = randn_bf16((B, Hkv, N, D), g)
    v = randn_bf16((B, Hkv, N, D), g)
    return q, k, v


def prefill_inputs_for(cfg: PrefillConfig):
    return prefill_inputs(cfg.B, cfg.Hq, cfg.Hkv, cfg.N, cfg.D, cfg.seed)


def bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (a view change, no arithmetic)."""
    import numpy as np
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


@dataclass
class PagedCache:
    q: torch.Tensor            # [S, Hq, D] bf16
    k_pages: torch.Tensor      # [num_pages, Hkv, page_size, D] bf16
    v_pages: torch.Tensor      # same
    block_table: torch.Tensor  # [S, max_blocks] int32, unused tail = -1
    seq_lens: torch.Tensor     # [S] int32
    page_size: int
    Hq: int
    Hkv: int
    D: int

    @property
    def num_seqs(self) -> int:
        return self.q.shape[0]

    @property
    def num_pages(self) -> int:
        return self.k_pages.shape[0]

    @property
    def max_blocks(self) -> int:
        return self.block_table.shape[1]

    @property
    def total_tokens(self) -> int:
        return int(self.seq_lens.sum())


def paged_decode_inputs(num_seqs, Hq, Hkv, D, page_size, seq_lens=None, len_lo=None, len_hi=None,
                        spare_frac=0.10, seed=0, max_blocks: Optional[int] = None,
                        permute: bool = True, poison: bool = True, chunk_pages: int = 4096):
    """A paged KV cache in the layout [num_pages, Hkv, page_size, D].

    Sequence lengths are given, or drawn uniformly from [len_lo, len_hi]. Sequence s needs
    ceil(len_s / page_size) pages. The pool holds the sum of those plus ``spare_frac`` spare
    pages, and a seeded random permutation of the pool assigns physical pages to the block
    tables in table order (``permute=False`` gives the identity order, a contiguous cache).
    Spare pages and the slots past seq_len in each last page hold bf16 NaN (``poison``), so a
    stray read shows up in the output. Unused block-table entries are -1.
    """
    g = _gen(seed)
    if seq_lens is None:
        seq_lens = torch.randint(len_lo, len_hi + 1, (num_seqs,), generator=g, dtype=torch.int64)
    seq_lens = torch.as_tensor(seq_lens, dtype=torch.int64)
    assert seq_lens.shape == (num_seqs,) and int(seq_lens.min()) >= 1
    pages_per_seq = (seq_lens + page_size - 1) // page_size
    used = int(pages_per_seq.sum())
    spare = int(round(used * spare_frac))
    pool = used + spare
    if max_blocks is None:
        max_blocks = int(pages_per_seq.max())
    assert max_blocks >= int(pages_per_seq.max())
    # The permutation is always drawn, so both orders consume the same random stream and
    # hold the same token values.
    perm = torch.randperm(pool, generator=g)
    order = perm if permute else torch.arange(pool)
    block_table = torch.full((num_seqs, max_blocks), -1, dtype=torch.int32)
    cursor = 0
    for s in range(num_seqs):
        n = int(pages_per_seq[s])
        block_table[s, :n] = order[cursor:cursor + n].to(torch.int32)
        cursor += n
    q = randn_bf16((num_seqs, Hq, D), g)
    k_pages = torch.empty((pool, Hkv, page_size, D), dtype=torch.bfloat16)
    v_pages = torch.empty((pool, Hkv, page_size, D), dtype=torch.bfloat16)
    # Page contents are drawn in logical (table) order, so a permuted and an identity-ordered
    # cache built from the same seed hold the same tokens.
    logical = order[:used]
    for c0 in range(0, used, chunk_pages):
        c1 = min(used, c0 + chunk_pages)
        idx = logical[c0:c1]
        k_pages[idx] = randn_bf16((c1 - c0, Hkv, page_size, D), g)
        v_pages[idx] = randn_bf16((c1 - c0, Hkv, page_size, D), g)
    if spare:
        fill = torch.tensor(BF16_NAN_BITS, dtype=torch.int16).view(torch.bfloat16)
        if poison:
            k_pages[order[used:]] = fill
            v_pages[order[used:]] = fill
        else:
            k_pages[order[used:]] = 0
            v_pages[order[used:]] = 0
    if poison:
        fill = torch.tensor(BF16_NAN_BITS, dtype=torch.int16).view(torch.bfloat16)
        for s in range(num_seqs):
            n = int(pages_per_seq[s])
            tail = int(seq_lens[s]) - (n - 1) * page_size
            if tail < page_size:
                last = int(block_table[s, n - 1])
                k_pages[last, :, tail:, :] = fill
                v_pages[last, :, tail:, :] = fill
    return PagedCache(q, k_pages, v_pages, block_table, seq_lens.to(torch.int32), page_size, Hq,
                      Hkv, D)


def paged_decode_inputs_for(cfg: DecodeConfig, permute: bool = True, poison: bool = True):
    return paged_decode_inputs(cfg.num_seqs, cfg.Hq, cfg.Hkv, cfg.D, cfg.page_size,
                               len_lo=cfg.len_lo, len_hi=cfg.len_hi, spare_frac=cfg.spare_frac,
                               seed=cfg.seed, permute=permute, poison=poison)


def contiguous_copy(cache: PagedCache) -> PagedCache:
    """The same cache re-laid so that sequence s occupies consecutive pages in logical order
    (block_table[s][p] = base_s + p). Only data movement; the token values are unchanged."""
    S = cache.num_seqs
    pages_per_seq = (cache.seq_lens.to(torch.int64) + cache.page_size - 1) // cache.page_size
    used = int(pages_per_seq.sum())
    k = torch.empty((used,) + tuple(cache.k_pages.shape[1:]), dtype=cache.k_pages.dtype)
    v = torch.empty_like(k)
    bt = torch.full_like(cache.block_table, -1)
    cursor = 0
    for s in range(S):
        n = int(pages_per_seq[s])
        src = cache.block_table[s, :n].to(torch.int64)
        k[cursor:cursor + n] = cache.k_pages[src]
        v[cursor:cursor + n] = cache.v_pages[src]
        bt[s, :n] = torch.arange(cursor, cursor + n, dtype=torch.int32)
        cursor += n
    return PagedCache(cache.q, k, v, bt, cache.seq_lens, cache.page_size, cache.Hq, cache.Hkv,
                      cache.D)


@dataclass
class DecodeStepInputs:
    """A paged cache whose seq_lens already count T new tokens per sequence, with the slots of those
    tokens poisoned (NaN) until an append fills them, plus the new tokens' q, k, v (not rotated)."""
    cache: PagedCache
    q: torch.Tensor      # [S, T, Hq, D] bf16
    k_new: torch.Tensor  # [S, T, Hkv, D] bf16
    v_new: torch.Tensor  # [S, T, Hkv, D] bf16

    @property
    def T(self) -> int:
        return self.q.shape[1]


def decode_step_inputs(num_seqs, T, Hq, Hkv, D, page_size, seq_lens=None, len_lo=None, len_hi=None,
                       spare_frac=0.10, seed=0, permute: bool = True, poison: bool = True):
    """Inputs for a decode step that appends T tokens per sequence and attends with their queries.
    The cache is ``paged_decode_inputs`` with the same arguments; the new tokens are drawn from a
    second seeded stream, so the cache is the same whatever T is."""
    cache = paged_decode_inputs(num_seqs, Hq, Hkv, D, page_size, seq_lens=seq_lens, len_lo=len_lo, len_hi=len_hi,
                                spare_frac=spare_frac, seed=seed, permute=permute, poison=poison)
    assert int(cache.seq_lens.min()) >= T
    g = _gen(seed + 7919)
    q = randn_bf16((num_seqs, T, Hq, D), g)
    k_new = randn_bf16((num_seqs, T, Hkv, D), g)
    v_new = randn_bf16((num_seqs, T, Hkv, D), g)
    if poison:
        fill = torch.tensor(BF16_NAN_BITS, dtype=torch.int16).view(torch.bfloat16)
        for s in range(num_seqs):
            for pos in range(int(cache.seq_lens[s]) - T, int(cache.seq_lens[s])):
                page = int(cache.block_table[s, pos // page_size])
                cache.k_pages[page, :, pos % page_size, :] = fill
                cache.v_pages[page, :, pos % page_size, :] = fill
    return DecodeStepInputs(cache, q, k_new, v_new)


def decode_step_inputs_for(cfg: DecodeConfig, T: int, permute: bool = True, poison: bool = True):
    return decode_step_inputs(cfg.num_seqs, T, cfg.Hq, cfg.Hkv, cfg.D, cfg.page_size, len_lo=cfg.len_lo,
                              len_hi=cfg.len_hi, spare_frac=cfg.spare_frac, seed=cfg.seed, permute=permute,
                              poison=poison)


def alibi_slopes(H: int) -> torch.Tensor:
    """Per-head ALiBi slopes, the geometric sequence m_h = 2^(-8h/H), h = 1..H, of the ALiBi paper
    (Press et al., 2021; the pages name the method and say only that each head has a fixed slope).
    fp32 [H]; every value is a power of two, so both implementations see it exactly."""
    return torch.tensor([2.0 ** (-8.0 * h / H) for h in range(1, H + 1)], dtype=torch.float32)


@dataclass
class Fp8Inputs:
    """FP8 e4m3 Q/K/V (bit patterns, uint8) with per-tensor scales: the value of an element is its
    e4m3 value times the tensor's descale."""
    q8: torch.Tensor
    k8: torch.Tensor
    v8: torch.Tensor
    descale_q: float
    descale_k: float
    descale_v: float


E4M3_MAX = 448.0


def fp8_inputs(B, Hq, Hkv, N, D, seed) -> Fp8Inputs:
    """N(0,1) fp32 draws quantised to e4m3 per tensor: descale = max|x| / 448 rounded up to a power of
    two (so the scaling is exact), then x / descale rounded to e4m3 by torch (nearest even; no value
    exceeds 448)."""
    g = _gen(seed)
    out = []
    for shape in ((B, Hq, N, D), (B, Hkv, N, D), (B, Hkv, N, D)):
        x = torch.randn(shape, generator=g, dtype=torch.float32)
        amax = float(x.abs().max())
        descale = 2.0 ** math.ceil(math.log2(amax / E4M3_MAX))
        x8 = (x / descale).to(torch.float8_e4m3fn).view(torch.uint8)
        out.append((x8, descale))
    return Fp8Inputs(out[0][0], out[1][0], out[2][0], out[0][1], out[1][1], out[2][1])


def fp8_inputs_for(cfg: PrefillConfig) -> Fp8Inputs:
    return fp8_inputs(cfg.B, cfg.Hq, cfg.Hkv, cfg.N, cfg.D, cfg.seed + 2000)
