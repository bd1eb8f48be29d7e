/*
 * attn.h -- C ABI of libattn_b200.so: exact scaled dot-product attention on NVIDIA B200 (sm_100a).
 *
 * Operations computing softmax(Q K^T * scale) V exactly (up to floating-point rounding), never
 * materialising the n x n score matrix in device memory:
 *   attn_fwd           prefill over whole sequences (causal / sliding-window / full, GQA, RoPE);
 *   attn_bwd           its gradients, recomputing the scores from the saved logsumexp;
 *   attn_decode_paged  one new query token per sequence over a paged KV cache.
 *
 * Conventions shared by every entry point:
 *   - Tensor arguments are plain device pointers to caller-owned memory, contiguous, in the
 *     layouts stated below, each 16-byte aligned. bf16 means IEEE bfloat16 (uint16 storage).
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream). Calls are
 *     asynchronous on that stream; the return value covers argument validation and launch only.
 *   - Nothing throws, aborts or traps. Every failure returns a status and sets a thread-local
 *     message readable with attn_last_error(). Faults detected on the device (a bounded wait
 *     that gave up, an out-of-range block-table entry) set bits of a device status word read
 *     with attn_get_device_status().
 *   - The library owns only its caches (RoPE cos/sin tables per (device, base, head dim); a
 *     scratch per (device, stream) for the rotated queries and keys of attn_fwd and
 *     attn_fwd_pos, kept for at most 8 streams per device; the device status word);
 *     attn_shutdown releases them. A cache grows geometrically when a call needs more; the
 *     outgrown buffer is freed at once after a device synchronisation, so memory stays bounded.
 *   - There is no CPU fallback: without a B200 every compute call returns ATTN_ERR_CUDA.
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_INVALID_ARG = 1,  /* a pointer, size or flag violates the contract below */
    ATTN_ERR_UNSUPPORTED = 2,  /* valid request outside what the kernels implement (e.g. D) */
    ATTN_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed (no device, launch error) */
    ATTN_ERR_DEVICE_CHECK = 4, /* reported by attn_get_device_status: a device-side check fired */
    ATTN_ERR_TIMEOUT = 5       /* reported by attn_get_device_status: a bounded wait gave up */
} attn_status;

/* Bits of the device status word returned by attn_get_device_status(). */
#define ATTN_DEVICE_TIMEOUT 1u      /* a pipeline wait exceeded its limit; that CTA bailed out */
#define ATTN_DEVICE_BAD_PAGE 2u     /* a block-table entry outside [0, num_pages) was skipped */
#define ATTN_DEVICE_BAD_SEQLEN 4u   /* a seq_len outside [1, max_blocks*page_size]; row set to NaN */

/*
 * attn_fwd -- attention forward (prefill), FlashAttention-style.
 *
 * Computes, for every batch b, query head h and query position i,
 *   O[b,h,i,:] = sum_j softmax_j(scale * q_i . k_j) v_j,   LSE[b,h,i] = ln sum_j exp(scale * q_i . k_j)
 * over the visible keys j, where q_i = Q[b,h,i,:] and k_j, v_j come from K/V head h / (Hq/Hkv)
 * ("attention-transformers", Q "How does self-attention work in a transformer?";
 * "Transformer Complexity, Inference Optimization, GQA and FlashAttention", Part 3 for
 * grouped-query attention). The computation tiles Q, K and V through on-chip memory with the
 * online softmax of "Why is attention O(n^2), how does FlashAttention help, ...",
 * "Deep dive: FlashAttention"; LSE is the saved row statistic m + ln(l) of that section.
 *
 *   q      bf16 [B, Hq,  N, D] device, read only
 *   k, v   bf16 [B, Hkv, N, D] device, read only
 *   o      bf16 [B, Hq,  N, D] device, written
 *   lse    fp32 [B, Hq,  N]    device, written (natural log), or NULL to skip
 *   causal 1: key j visible to query i iff j <= i (mask on the logits, "Transformer Attention
 *          Mechanism Interview Deep Dive", "Causal masking"); 0: every key visible.
 *   window >0: additionally j >= i - window + 1 (sliding window of width `window`,
 *          "attention-transformers", Q "What is sparse / sliding-window attention?");
 *          requires causal = 1. <=0: no window.
 *   rope_base  >0: rotate q and k pairwise, pairs (2t, 2t+1) by pos * rope_base^(-2t/D), pos =
 *          the token index 0..N-1, counter-clockwise, then round to bf16 ("attention-transformers",
 *          Q "How does Rotary Position Embedding (RoPE) work?"); the rotation is computed in
 *          fp64 and rounded once, into the library's scratch, before the attention kernel.
 *          <=0: no rotation.
 *   scale  >0: softmax scale; <=0: 1/sqrt(D) ("Why is attention scaled by 1/sqrt(dk)?").
 * Constraints: B, Hq, Hkv, N >= 1; Hq % Hkv == 0; D in {64, 128} (else ATTN_ERR_UNSUPPORTED);
 * B * Hq * ceil(N/256) < 2^31. Fully masked key tiles are skipped, not computed.
 * Errors: ATTN_ERR_INVALID_ARG for NULL/misaligned pointers or inconsistent sizes/flags;
 * ATTN_ERR_CUDA when a runtime call or the launch fails. With RoPE, the first call for a new
 * (device, rope_base, D), a longer N than cached, or a new stream allocates cached device memory
 * (cudaMalloc) and synchronises the device; later calls of the same or smaller size do neither.
 */
attn_status attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                     int N, int D, int causal, int window, float rope_base, float scale, void* stream);

/*
 * attn_fwd_pos -- attn_fwd with the position-encoding variants ("attention-transformers": Q "How
 * does Rotary Position Embedding (RoPE) work?", Q "What are NTK-aware RoPE scaling and YaRN?",
 * Q "How does ALiBi encode position?"):
 *   rope_half_split  0: RoPE pairs (2i, 2i+1) as attn_fwd; 1: pairs (i, i + D/2) (the rotate-half
 *                    layout). The output is the same attention either way; only which
 *                    dimensions form a pair changes.
 *   rope_pos_scale   Position Interpolation: pair i of position pos is rotated by
 *                    (pos / rope_pos_scale) * b^(-2i/D); 1 = off. Finite, > 0.
 *   rope_ntk_factor  NTK-aware scaling: b = rope_base * rope_ntk_factor^(D/(D-2)), which leaves the
 *                    highest frequency as is and divides the lowest by the factor; 1 = off.
 *                    Finite, > 0. Both scalings change only the cos/sin table.
 *   alibi_slopes     device fp32 [Hq], 4-byte aligned, or NULL: ALiBi subtracts
 *                    alibi_slopes[h] * (i - j) from the scaled logit of query i and key j of head
 *                    h (then the softmax as usual; LSE includes the bias). Requires causal = 1.
 * Other arguments, constraints and errors as attn_fwd; attn_fwd is attn_fwd_pos with (0, 1, 1,
 * NULL). The scalings and pairing apply only when rope_base > 0.
 */
attn_status attn_fwd_pos(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                         int N, int D, int causal, int window, float rope_base, int rope_half_split,
                         float rope_pos_scale, float rope_ntk_factor, const float* alibi_slopes, float scale,
                         void* stream);

/*
 * attn_fwd_fp8 -- attn_fwd on FP8 e4m3 inputs ("Why is attention O(n^2), how does FlashAttention help,
 * ...": newer hardware's FP8). The value of an element of q is its e4m3 value times descale_q (per
 * tensor), likewise k and v. Both products run on the tensor cores in e4m3 with fp32 accumulation;
 * the probabilities P are rounded to e4m3 (nearest even) for the P V product, so O carries their
 * ~2.6% relative rounding (the LSE does not: the row sums stay fp32).
 *   q            e4m3 bytes [B, Hq, N, 128]; k, v e4m3 bytes [B, Hkv, N, 128]; device, 16-byte aligned
 *   descale_q, descale_k, descale_v   finite, > 0
 *   o, lse, B, Hq, Hkv, N, causal, window, scale, stream   as attn_fwd (scale applies to q.k of
 *                the dequantised values)
 * D must be 128 (else ATTN_ERR_UNSUPPORTED). No RoPE on this path: rotate before quantising.
 */
attn_status attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                         int N, int D, int causal, int window, float descale_q, float descale_k, float descale_v,
                         float scale, void* stream);

/*
 * attn_bwd_workspace_size -- bytes of device workspace attn_bwd needs: fp32 (-LSE*log2 e, -D_i)
 * and the fp32 dq sums (D values) per query row padded to 128-row tiles, plus, with RoPE, the
 * rotated Q and K (bf16). 0 for invalid sizes.
 */
size_t attn_bwd_workspace_size(int B, int Hq, int Hkv, int N, int D, float rope_base);

/*
 * attn_bwd -- attention backward: gradients of L = sum(O * dout) with respect to q, k and v for the
 * attention attn_fwd computes (same masks, GQA map, RoPE and scale). The scores are recomputed from
 * q, k and the forward's row logsumexp instead of being stored ("Self-Attention Complexity,
 * FlashAttention, PagedAttention, and RoPE in Code", Part 2: recomputation in the backward pass;
 * "Why is attention O(n^2), how does FlashAttention help, ...", "Deep dive: FlashAttention": the
 * backward recomputes scores from the saved m and l):
 *   dv_j = sum_i P_ij dO_i,  dS_ij = P_ij (dO_i . v_j - dO_i . O_i),
 *   dq_i = scale sum_j dS_ij k_j,  dk_j = scale sum_i dS_ij q_i,
 * with q, k rotated; the gradients of the unrotated inputs are rotated back. For GQA, dk and dv of a
 * K/V head sum over its query heads. dk and dv are accumulated in a fixed order and repeat bit for
 * bit; dq is a sum of fp32 partials (one per 128-key tile) added in device memory in the order the
 * tiles finish, so two calls may differ by one bf16 unit in the last place.
 *
 *   q, k, v, causal, window, rope_base, scale, B, Hq, Hkv, N, D   as given to attn_fwd
 *   o      bf16 [B, Hq, N, D] and lse fp32 [B, Hq, N]: attn_fwd's outputs for these inputs
 *   dout   bf16 [B, Hq, N, D] gradient of the loss with respect to o
 *   dq     bf16 [B, Hq, N, D]; dk, dv bf16 [B, Hkv, N, D]: written
 *   workspace  device scratch of at least attn_bwd_workspace_size(...) bytes, 16-byte aligned,
 *          owned by the caller, any initial contents; overlapping calls need their own.
 * Constraints and errors as attn_fwd (D in {64, 128}), with B * Hq * ceil(N/128) * 128 < 2^31.
 */
attn_status attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                     void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int D, int causal, int window,
                     float rope_base, float scale, void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_decode_workspace_size -- bytes of device workspace attn_decode_paged needs: fp32 partial
 * (max, sum, output) states for every (sequence, query head, 512-token split) -- the shortest split
 * the call may use, so the size covers every choice. Returns 0 for
 * invalid sizes.
 */
size_t attn_decode_workspace_size(int num_seqs, int max_blocks_per_seq, int page_size, int Hq, int D);

/*
 * attn_decode_paged -- one decode step per sequence over a PagedAttention KV cache.
 *
 * The cache is a pool of fixed-size pages; token t of sequence s lives in page
 * block_table[s][t / page_size], slot t % page_size ("Self-Attention Complexity,
 * FlashAttention, PagedAttention, and RoPE in Code", Part 3: fixed-size blocks, block tables).
 * The single query of sequence s (its newest token, position seq_lens[s]-1, already rotated)
 * attends to all seq_lens[s] cached tokens, which include that token itself. The key range is
 * split into chunks of 512, 1024 or 2048 tokens (the longest that still gives every SM several
 * CTAs for the call's num_seqs, heads and max_blocks_per_seq) whose partial softmax states are
 * merged in ascending order,
 * so the result depends only on logical token positions: a paged cache and a contiguous copy
 * of it give bit-identical outputs.
 *
 *   q            bf16 [num_seqs, Hq, D] device
 *   k_pages,
 *   v_pages      bf16 [num_pages, Hkv, page_size, D] device (RoPE already applied to keys)
 *   block_table  int32 [num_seqs, max_blocks_per_seq] device; entries past a sequence's last
 *                page are never read (any value, e.g. -1)
 *   seq_lens     int32 [num_seqs] device, each in [1, max_blocks_per_seq * page_size]
 *   o            bf16 [num_seqs, Hq, D] device, written
 *   lse          fp32 [num_seqs, Hq] device, written (natural log), or NULL
 *   workspace    device scratch of at least attn_decode_workspace_size(...) bytes, 16-byte
 *                aligned, owned by the caller; overwritten; calls that overlap on the GPU must
 *                use different workspaces.
 *   scale        >0 softmax scale, <=0: 1/sqrt(D)
 * Constraints: page_size == 16 and D in {64, 128} (else ATTN_ERR_UNSUPPORTED); Hq % Hkv == 0
 * and Hq / Hkv <= 16; num_seqs, Hkv <= 65535. Slots past seq_len in a sequence's last page may
 * hold anything (NaN included): they are masked and never reach the output.
 * Block-table entries and seq_lens are device data and are checked on the device: an invalid
 * entry sets a bit of the device status word (the page is skipped; the output is then wrong).
 */
attn_status attn_decode_paged(const void* q, const void* k_pages, const void* v_pages, const int32_t* block_table,
                              const int32_t* seq_lens, int num_seqs, int max_blocks_per_seq, int num_pages,
                              int page_size, int Hq, int Hkv, int D, float scale, void* o, float* lse,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_decode_step_workspace_size -- bytes of device workspace attn_decode_step needs: fp32 partial
 * outputs and (max, sum) per (sequence, new token, query head, 512-token chunk, the shortest a call
 * may use), rounded up to
 * 256 bytes. 0 for invalid sizes.
 */
size_t attn_decode_step_workspace_size(int num_seqs, int q_len, int max_blocks_per_seq, int page_size, int Hq, int D);

/*
 * attn_decode_step -- a decode step that brings q_len new tokens per sequence: it appends their
 * keys and values to the paged cache, then attends with their queries.
 *
 * The new tokens of sequence s sit at positions seq_lens[s]-q_len .. seq_lens[s]-1 (seq_lens
 * count them). With rope_base > 0, every new query and key is rotated at its position, on
 * interleaved pairs (2i, 2i+1) by pos * rope_base^(-2i/D) ("attention-transformers", Q "How does
 * Rotary Position Embedding (RoPE) work?"), in fp64 (an fp64 cos/sin table, unfused products) and
 * rounded once to bf16; values are never rotated.
 * 1. Append (when k_new is given): new token t's rotated key and its value go to page
 *    block_table[s][pos / page_size], slot pos % page_size ("Self-Attention Complexity,
 *    FlashAttention, PagedAttention, and RoPE in Code", Part 3: the cache grows one block-table
 *    slot at a time). k_new == NULL: the cache already holds the new tokens.
 * 2. Attend: new token t's queries attend causally to cached tokens 0..pos -- the last q_len rows of
 *    causal attention over the sequence (multi-token decode; q_len = 1 is one-token decode), with
 *    the split-and-merge of attn_decode_paged.
 *
 *   q            bf16 [num_seqs, q_len, Hq, D] device, not rotated (rotated here if rope_base > 0)
 *   k_new, v_new bf16 [num_seqs, q_len, Hkv, D] device, or both NULL; k_new not rotated
 *   k_pages,
 *   v_pages      bf16 [num_pages, Hkv, page_size, D] device; the new tokens' slots are written.
 *                Slots written by two sequences in one call are the caller's error.
 *   block_table, seq_lens   as attn_decode_paged, with seq_lens[s] in [q_len, max_blocks_per_seq * page_size]
 *   rope_base    > 0: RoPE base; <= 0: no rotation (q and k_new are used as given)
 *   o            bf16 [num_seqs, q_len, Hq, D] device, written
 *   lse          fp32 [num_seqs, q_len, Hq] device, written (natural log), or NULL
 *   workspace    device scratch of at least attn_decode_step_workspace_size(...) bytes, 16-byte
 *                aligned, owned by the caller; overwritten; overlapping calls need their own.
 *   scale        >0 softmax scale, <=0: 1/sqrt(D)
 * Constraints as attn_decode_paged, plus 1 <= q_len <= 64 (else ATTN_ERR_UNSUPPORTED above 64) and
 * Hkv * ceil(q_len * Hq / Hkv / 16) <= 65535. Bad block-table entries or lengths set device status
 * bits (see attn_get_device_status); the tokens concerned are not written.
 * The RoPE table covers positions up to max_blocks_per_seq * page_size and is cached per (device,
 * base, D); its first build synchronises the device.
 */
attn_status attn_decode_step(const void* q, const void* k_new, const void* v_new, void* k_pages, void* v_pages,
                             const int32_t* block_table, const int32_t* seq_lens, int num_seqs, int q_len,
                             int max_blocks_per_seq, int num_pages, int page_size, int Hq, int Hkv, int D,
                             float rope_base, float scale, void* o, float* lse, void* workspace,
                             size_t workspace_bytes, void* stream);

/*
 * attn_decode_paged_noalloc -- attn_decode_paged for callers that cannot allocate device memory.
 * The pages have no counterpart to this entry point; it exists for callers that cannot call
 * cudaMalloc when they call in -- for example a plugin inside a framework that owns the device's
 * memory pool and hands out no scratch buffers, or a serving loop that cannot afford cudaMalloc's
 * implicit device-wide synchronisation.
 *
 * Same arguments, computation, results and checks as attn_decode_paged, without the workspace:
 * the partial softmax states live in one fixed device array of ATTN_DECODE_NOALLOC_MAX_BYTES
 * compiled into the library (every GPU that loads the library holds it until the process exits).
 * The call itself allocates nothing. The array is reserved when the library's device code is
 * loaded on a device, which with CUDA's lazy module loading happens at the first call into the
 * library on that device, whichever entry point it is, and may synchronise the device: make one
 * warm-up call per device before the latency-sensitive path. Limits and sharing:
 *   - requests whose attn_decode_workspace_size(...) exceeds ATTN_DECODE_NOALLOC_MAX_BYTES are
 *     rejected with ATTN_ERR_INVALID_ARG and a message naming the limit;
 *   - every call, on every stream, uses the same array and leaves its contents behind; nothing in
 *     it needs to start at zero (each call writes every partial state it reads), but calls that
 *     overlap on the GPU race on it and must be serialised by the caller;
 *   - the first call on each device looks up the array's device address (cudaGetSymbolAddress,
 *     with that device current) and caches it; make that first call before any stream capture;
 *   - after a device reset (cudaDeviceReset) the cached address is stale: call attn_shutdown,
 *     which forgets it, before calling in again.
 */
#define ATTN_DECODE_NOALLOC_MAX_BYTES ((size_t)40 << 20)
attn_status attn_decode_paged_noalloc(const void* q, const void* k_pages, const void* v_pages,
                                      const int32_t* block_table, const int32_t* seq_lens, int num_seqs,
                                      int max_blocks_per_seq, int num_pages, int page_size, int Hq, int Hkv, int D,
                                      float scale, void* o, float* lse, void* stream);

/*
 * attn_get_device_status -- synchronises `stream` on the current device, returns the device
 * status word (ATTN_DEVICE_* bits) in *flags_out and clears it. Returns ATTN_ERR_TIMEOUT or
 * ATTN_ERR_DEVICE_CHECK when a bit was set, ATTN_OK otherwise.
 */
attn_status attn_get_device_status(void* stream, int* flags_out);

/*
 * attn_debug_drop_copy -- test hook for the timeout path (not for production use). While enabled,
 * the first CTA of a kernel sets up one copy but never issues it: its first page copy in the
 * paged-decode split kernel (attn_decode_paged, attn_decode_paged_noalloc, attn_decode_step), its
 * first key-tile copy in the prefill kernel (attn_fwd, attn_fwd_pos, attn_fwd_fp8), its first
 * query/dO copy in the backward's main kernel (attn_bwd). The bounded wait on that copy (about
 * 2 s of SM clocks) runs out: the CTA raises ATTN_DEVICE_TIMEOUT in the device status word, drains
 * its own copies and products, and returns; the outputs that CTA owns are then undefined. No
 * memory outside the call's buffers is touched and the CUDA context stays usable. Applies to
 * calls launched while enabled.
 */
void attn_debug_drop_copy(int enable);

/* Message of the last failure on the calling thread ("" if none). Owned by the library. */
const char* attn_last_error(void);

/* Library version string. */
const char* attn_version(void);

/* Frees every cache the library allocated (RoPE tables, query/key scratch), on every device, and
 * forgets the cached device address of the no-alloc decode's array. The caller must ensure no call
 * is still running on the GPU. */
void attn_shutdown(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
