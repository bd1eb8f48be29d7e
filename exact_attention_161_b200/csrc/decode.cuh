// decode.cuh -- one-token decode over a paged KV cache, split along the KV length.
//
// The cache is a pool of fixed-size pages [num_pages, Hkv, page_size, D]; sequence s reaches
// its t-th token through its block table: page block_table[s][t / page_size], slot
// t % page_size ("Self-Attention Complexity, FlashAttention, PagedAttention, and RoPE in Code",
// Part 3: fixed-size blocks, block tables). Each decode step reads the whole cache of the
// sequence and does little arithmetic per byte, so this path is bound by HBM bandwidth ("Why is
// attention O(n^2), how does FlashAttention help, ...", follow-up "Why is decode memory-bound").
//
// Split: the logical token range of every sequence is cut into chunks of 32 to 128 pages.
// One CTA handles one (chunk, KV head, sequence) and produces, for each of the G query heads
// of that KV head, a partial online-softmax state (m, l, o) over its chunk -- the recurrence of
// "Deep dive: FlashAttention" applied to a slice of the keys. A second kernel merges the
// partials of each (sequence, head) in ascending chunk order with the same rescaling identity,
// so the result depends only on logical positions: a paged cache and its contiguous copy give
// identical bits.
//
// Inside a CTA, each of the 4 warps takes every fourth page of the chunk and streams it
// through its own ring of shared-memory stages filled by TMA (the page's K and V slabs are
// contiguous 16 x D blocks; a 128-byte swizzle makes the ldmatrix reads conflict-free). The G
// query heads form the M rows of 16x8x16 bf16 tensor-core products (this path is HBM-bound,
// so the small MMA is not the limit): S = q K^T per page, then O += P V.
//
// A decode step may bring T >= 1 new tokens per sequence (multi-token decode: the last T rows of
// causal attention over the sequence). Their G*T query rows (G heads x T tokens) are cut into
// 16-row tiles, one tile per CTA, and row (t, head) sees the cached tokens up to its position
// len - T + t. A prep kernel runs first: it rotates each new query row once at its position (into
// the workspace) and writes the new tokens' keys (rotated) and values into their page slots, so
// the split kernel reads a cache that already holds them and queries that are already rotated.
#pragma once
#include "common.cuh"
#include "ptx.cuh"
#include "rope.cuh"

namespace attn {

constexpr int kPageSize = 16;
// Chunk lengths in pages: the host takes the longest of 128, 64 and 32 pages (2048, 1024, 512
// tokens) that still gives every SM several CTAs. Longer chunks spread a CTA's fixed cost (its
// set-up, the combine of its four warps' states and the partial states it writes) over more
// pages; the workspace is sized for the shortest.
constexpr int kChunkPages = 32;
constexpr int kMaxChunkPages = 128;
constexpr int kDecodeWarps = 4;
constexpr int kDecodeThreads = kDecodeWarps * 32;

struct DecodeParams {
    const __nv_bfloat16* q;      // [S, T, Hq, D], rotated
    const int32_t* block_table;  // [S, max_blocks]
    const int32_t* seq_lens;     // [S], counting the T new tokens
    __nv_bfloat16* o;            // [S, T, Hq, D]
    float* lse;                  // [S, T, Hq] or nullptr
    float* ws_o;                 // [S, T*Hq, max_chunks, D] unnormalised partial outputs
    float* ws_ml;                // [S, T*Hq, max_chunks, 2] partial (max in log2 units, sum)
    int S, Hq, Hkv, G, max_blocks, num_pages, max_chunks;
    int T, mtiles;               // new tokens per sequence; 16-row tiles per KV head = ceil(G*T / 16)
    int chunk_pages;             // pages per split chunk
    int debug_drop_copy;         // test hook: CTA (0,0,0) skips its first page copy (see attn.h)
    float scale_log2;
};

// Prep of a decode step: token t of sequence s sits at position pos = len - T + t. Its query rows
// are rotated at pos into q_rot (when a table is given), and its key (rotated at pos, rounded to
// bf16) and value are written to page block_table[s][pos / page_size], slot pos % page_size (when
// k_new is given).
struct StepPrepParams {
    const __nv_bfloat16* q;      // [S, T, Hq, D]
    __nv_bfloat16* q_rot;        // [S, T, Hq, D] or nullptr (no rotation)
    const __nv_bfloat16* k_new;  // [S, T, Hkv, D] or nullptr (no append)
    const __nv_bfloat16* v_new;  // [S, T, Hkv, D]
    __nv_bfloat16* k_pages;      // [num_pages, Hkv, page_size, D]
    __nv_bfloat16* v_pages;
    const int32_t* block_table;
    const int32_t* seq_lens;
    const double2* rope;
    int S, T, Hq, Hkv, max_blocks, num_pages;
};

template <int D>
struct DecCfg {
    static constexpr int NREG = D / 64;
    static constexpr int SLAB_BYTES = kPageSize * D * 2;   // one page of one KV head
    static constexpr int STAGES = 3;
    static constexpr int STAGE_BYTES = 2 * SLAB_BYTES;      // K then V
    static constexpr int WARP_BYTES = STAGES * STAGE_BYTES;
    static constexpr int NT = D / 8;                        // 8-wide output column tiles
    static constexpr int COMBINE_BYTES = (kDecodeWarps * 16 * (D + 3) + 32) * 4;
    static constexpr int SMEM_BYTES = kDecodeWarps * WARP_BYTES + 1024 /*align*/ + 256 /*barriers*/;
    static_assert(COMBINE_BYTES <= kDecodeWarps * WARP_BYTES, "combine buffer reuses the stages");
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
// D = A(16x16, row) * B(16x8, col) + D, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Byte offset of (row, 16-byte chunk) inside a 128-byte-swizzled slab of 16 rows per region.
__device__ __forceinline__ uint32_t slab_off(int row, int chunk) {
    return (chunk >> 3) * (kPageSize * 128) + row * 128 + (((chunk & 7) ^ (row & 7)) << 4);
}

// kStep = false: one token per sequence, q as given (the plain decode); true: the decode step's
// general form (T tokens, per-row causal limits, optional rotation of q).
template <int D, bool kStep>
__global__ void __launch_bounds__(kDecodeThreads)
    decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const DecodeParams p) {
    using C = DecCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kDecodeWarps * C::WARP_BYTES);  // [warps][STAGES]
    int* abort_ptr = reinterpret_cast<int*>(full + kDecodeWarps * C::STAGES);
    volatile int* abort_flag = abort_ptr;

    const int chunk = blockIdx.x, s = blockIdx.z;
    const int g = kStep ? blockIdx.y / p.mtiles : blockIdx.y, mt = kStep ? blockIdx.y % p.mtiles : 0;
    const int T = kStep ? p.T : 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int len = p.seq_lens[s];
    if (len < T || len > p.max_blocks * kPageSize) {
        if (chunk == 0 && blockIdx.y == 0 && threadIdx.x == 0) raise_status(kStatusBadSeqLen);
        return;
    }
    const int n_pages = (len + kPageSize - 1) / kPageSize;
    const int pg_begin = chunk * p.chunk_pages;
    if (pg_begin >= n_pages) return;
    const int pg_end = min(n_pages, pg_begin + p.chunk_pages);
    const int my_count = (pg_end - pg_begin - warp + kDecodeWarps - 1) / kDecodeWarps;  // may be <= 0

    if (threadIdx.x == 0) {
        for (int i = 0; i < kDecodeWarps * C::STAGES; ++i) ptx::mbar_init(&full[i], 1);
        *abort_ptr = 0;
        ptx::fence_mbar_init();
    }
    if (threadIdx.x == 32) {
        ptx::prefetch_tensormap(&tm_k);
        ptx::prefetch_tensormap(&tm_v);
    }
    __syncthreads();

    uint8_t* ring = smem + warp * C::WARP_BYTES;
    uint64_t* wfull = full + warp * C::STAGES;
    const int32_t* bt = p.block_table + static_cast<size_t>(s) * p.max_blocks;

    // Lane 0 issues the TMA copies of the warp's i-th page; returns false for an invalid page
    // index (then the stage barrier is completed without data and the page is skipped).
    auto issue = [&](int i) -> bool {
        const int pg = pg_begin + warp + kDecodeWarps * i;
        const int phys = bt[pg];
        const bool valid = phys >= 0 && phys < p.num_pages;
        if (lane == 0) {
            uint64_t* bar = &wfull[i % C::STAGES];
            if (valid) {
                uint8_t* st = ring + (i % C::STAGES) * C::STAGE_BYTES;
                const int z = phys * p.Hkv + g;
                ptx::fence_proxy_async_smem();
                ptx::mbar_arrive_expect_tx(bar, C::STAGE_BYTES);
                // test hook: expect the bytes but never copy them, so this stage's wait runs out
                if (p.debug_drop_copy && i == 0 && warp == 0 && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
                    return valid;
#pragma unroll
                for (int r = 0; r < C::NREG; ++r) {
                    ptx::tma_load_3d(st + r * kPageSize * 128, &tm_k, bar, r * 64, 0, z);
                    ptx::tma_load_3d(st + C::SLAB_BYTES + r * kPageSize * 128, &tm_v, bar, r * 64, 0, z);
                }
            } else {
                raise_status(kStatusBadPage);
                ptx::mbar_arrive(bar);
            }
        }
        return valid;
    };

    // Q fragments (A operand). Row r of this CTA's tile is query row mt*16 + r = t*G + head of the
    // KV head's G*T rows; rows past G*T are zero. lim: the last position the row sees (padding rows
    // see the whole sequence, so their scores stay finite).
    const int rowA = lane >> 2, colA = 2 * (lane & 3);
    uint32_t qa[D / 16][4];
    int lim[2];
    {
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            const int R = mt * 16 + rowA + 8 * hr;
            const bool live = R < p.G * T;
            const int t = kStep ? (live ? R / p.G : T - 1) : 0;
            const int pos = len - T + t;
            lim[hr] = pos;
            const __nv_bfloat16* qrow =
                p.q + ((static_cast<size_t>(s) * T + t) * p.Hq + g * p.G + (kStep ? R % p.G : R)) * D;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int d0 = kk * 16 + colA + 8 * half;
                    qa[kk][hr + 2 * half] = live ? *reinterpret_cast<const uint32_t*>(qrow + d0) : 0u;
                }
            }
        }
    }

    float m[2] = {-INFINITY, -INFINITY};  // rows rowA, rowA + 8 (log2 units)
    float l[2] = {0.f, 0.f};              // this lane's share of the row sums
    float o[C::NT][4];
#pragma unroll
    for (int nt = 0; nt < C::NT; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;

    const int prefetch = min(C::STAGES, max(my_count, 0));
    uint32_t valid_mask = 0;  // bit (i % STAGES): page i had a valid block-table entry
    int n_issued = 0, n_consumed = 0;
    for (int i = 0; i < prefetch; ++i, ++n_issued)
        if (issue(i)) valid_mask |= 1u << i;

    bool ok = true;
    for (int i = 0; i < my_count; ++i) {
        const int st = i % C::STAGES;
        if (!ptx::mbar_wait(&wfull[st], (i / C::STAGES) & 1, abort_flag)) {
            ok = false;
            break;
        }
        n_consumed = i + 1;
        const bool page_ok = (valid_mask >> st) & 1u;
        const int pg = pg_begin + warp + kDecodeWarps * i;
        const int valid = min(kPageSize, len - pg * kPageSize);  // tokens of this page in use
        if (page_ok) {
            const uint32_t sk = ptx::smem_u32(ring + st * C::STAGE_BYTES);
            const uint32_t sv = sk + C::SLAB_BYTES;
            // ---- S = q K^T for the 16 tokens of the page (two 8-token column tiles)
            float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            const int mat = lane >> 3, mrow = lane & 7;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const int tok = 8 * (mat >> 1) + mrow;
                const int chunkd = 2 * kk + (mat & 1);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(sk + slab_off(tok, chunkd), b0, b1, b2, b3);
                mma_16816(sc[0], qa[kk], b0, b1);
                mma_16816(sc[1], qa[kk], b2, b3);
            }
            // ---- online softmax over the page (row rowA: sc[.][0..1], row rowA+8: sc[.][2..3])
            float mx[2];
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                // last slot of this page the row sees (one token: the page's last valid slot)
                const int last = kStep ? lim[hr] - pg * kPageSize : valid - 1;
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int tok = nt * 8 + colA + e;
                        float v = sc[nt][2 * hr + e];
                        v = tok <= last ? v : -INFINITY;  // select: NaN-poisoned slots never leak
                        sc[nt][2 * hr + e] = v;
                    }
                float t = fmaxf(fmaxf(sc[0][2 * hr], sc[0][2 * hr + 1]), fmaxf(sc[1][2 * hr], sc[1][2 * hr + 1]));
                t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, 1));
                t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, 2));
                mx[hr] = t * p.scale_log2;
            }
            float alpha[2];
            uint32_t pa[4];
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                // -inf while the row has seen none of this warp's tokens (a later token of a
                // multi-token step): exponents then use 0, giving p = 0 and alpha = 0
                const float m_new = fmaxf(m[hr], mx[hr]);
                const float m_use = (kStep && m_new == -INFINITY) ? 0.f : m_new;
                alpha[hr] = ptx::ex2(m[hr] - m_use);
                m[hr] = m_new;
                float ps[4];
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e) ps[nt * 2 + e] = ptx::ex2(fmaf(sc[nt][2 * hr + e], p.scale_log2, -m_use));
                l[hr] = l[hr] * alpha[hr] + ((ps[0] + ps[1]) + (ps[2] + ps[3]));
                pa[hr] = ptx::pack_bf16x2(ps[0], ps[1]);       // tokens colA, colA+1
                pa[2 + hr] = ptx::pack_bf16x2(ps[2], ps[3]);   // tokens 8+colA, 8+colA+1
            }
            // ---- O = alpha * O + P V
            const uint32_t a_frag[4] = {pa[0], pa[1], pa[2], pa[3]};
            const uint32_t keep0 = (colA < valid ? 0x0000FFFFu : 0u) | (colA + 1 < valid ? 0xFFFF0000u : 0u);
            const uint32_t keep1 = (8 + colA < valid ? 0x0000FFFFu : 0u) | (9 + colA < valid ? 0xFFFF0000u : 0u);
#pragma unroll
            for (int np = 0; np < C::NT / 2; ++np) {
                const int tok = 8 * (mat & 1) + mrow;
                const int chunkd = 2 * np + (mat >> 1);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(sv + slab_off(tok, chunkd), b0, b1, b2, b3);
                // zero the value rows of unused slots: 0 * NaN would poison the sum
                b0 &= keep0;
                b1 &= keep1;
                b2 &= keep0;
                b3 &= keep1;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    o[2 * np][e] *= alpha[e >> 1];
                    o[2 * np + 1][e] *= alpha[e >> 1];
                }
                mma_16816(o[2 * np], a_frag, b0, b1);
                mma_16816(o[2 * np + 1], a_frag, b2, b3);
            }
        }
        __syncwarp();
        if (i + C::STAGES < my_count) {
            const bool v = issue(i + C::STAGES);
            ++n_issued;
            valid_mask = v ? (valid_mask | (1u << st)) : (valid_mask & ~(1u << st));
        }
    }
    if (!ok) {
        *abort_flag = 1;
        raise_status(kStatusTimeout);
    }
    // Drain: every copy this warp issued must land before the stages are reused or the CTA ends
    // (only copies issued but not yet waited for can still be in flight; each wait is bounded).
    {
        volatile int never = 0;
        for (int i = n_consumed; i < n_issued; ++i)
            if (lane == 0) ptx::mbar_wait(&wfull[i % C::STAGES], (i / C::STAGES) & 1, &never);
        __syncwarp();
    }
    __syncthreads();

    // ---- combine the 4 warps' states for this chunk (shared memory reuses the stage ring)
    float* cm = reinterpret_cast<float*>(smem);                 // [warps][16] max
    float* cl = cm + kDecodeWarps * 16;                          // [warps][16] sum
    float* cwt = cl + kDecodeWarps * 16;                         // [warps][16] merge weight
    float* crow = cwt + kDecodeWarps * 16;                       // [16][2] merged (max, sum)
    float* co = crow + 32;                                       // [warps][16][D]
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
        float lsum = l[hr];
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
        const int row = rowA + 8 * hr;
        if ((lane & 3) == 0) {
            cm[warp * 16 + row] = m[hr];
            cl[warp * 16 + row] = lsum;
        }
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt) {
            co[(warp * 16 + row) * D + nt * 8 + colA] = o[nt][2 * hr];
            co[(warp * 16 + row) * D + nt * 8 + colA + 1] = o[nt][2 * hr + 1];
        }
    }
    __syncthreads();
    // every warp that gave up set the shared abort flag before the barrier above, so this exit is
    // the same for the whole CTA (the combine below has another barrier)
    if (*abort_flag) return;
    const int rows_here = kStep ? min(16, p.G * T - mt * 16) : p.G;
    // per row, once: M = max of the warps' maxima, the warps' weights 2^(m_w - M) and the merged sum
    if (threadIdx.x < rows_here) {
        const int row = threadIdx.x;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; ++w) M = fmaxf(M, cm[w * 16 + row]);
        float lacc = 0.f;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; ++w) {
            const float mw = cm[w * 16 + row];
            const float sw = mw == -INFINITY ? 0.f : ptx::ex2(mw - M);
            cwt[w * 16 + row] = sw;
            lacc += sw * cl[w * 16 + row];
        }
        crow[2 * row] = M;
        crow[2 * row + 1] = lacc;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < rows_here * D; idx += kDecodeThreads) {
        const int row = idx / D, d = idx % D;
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; ++w) acc += cwt[w * 16 + row] * co[(w * 16 + row) * D + d];
        const int R = mt * 16 + row, t = kStep ? R / p.G : 0;
        const size_t out_row = (static_cast<size_t>(s) * T + t) * p.Hq + g * p.G + (kStep ? R % p.G : R);
        const size_t prow = out_row * p.max_chunks + chunk;
        p.ws_o[prow * D + d] = acc;
        if (d == 0) {
            p.ws_ml[prow * 2] = crow[2 * row];
            p.ws_ml[prow * 2 + 1] = crow[2 * row + 1];
        }
    }
}

// Merge the chunk partials of every (sequence, token, head) row in ascending chunk order:
// M = max m_c, L = sum 2^(m_c - M) l_c, O = sum 2^(m_c - M) o_c / L, LSE = (M + log2 L) ln 2.
// Chunks a row sees none of carry m_c = -inf and weigh 0.
template <int D>
__global__ void __launch_bounds__(128) decode_merge_kernel(const DecodeParams p) {
    const long long warp_global = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const long long rows_per_seq = static_cast<long long>(p.T) * p.Hq;
    if (warp_global >= p.S * rows_per_seq) return;
    const int s = static_cast<int>(warp_global / rows_per_seq);
    const size_t out_row = static_cast<size_t>(warp_global);
    const int len = p.seq_lens[s];
    constexpr int PER = D / 32;
    __nv_bfloat16* orow = p.o + out_row * D;
    if (len < p.T || len > p.max_blocks * kPageSize) {  // flagged by the split kernel
        for (int e = 0; e < PER; ++e) orow[lane * PER + e] = __float2bfloat16(__int_as_float(0x7fc00000));
        if (p.lse != nullptr && lane == 0) p.lse[out_row] = __int_as_float(0x7fc00000);
        return;
    }
    const int n_chunks = (len + p.chunk_pages * kPageSize - 1) / (p.chunk_pages * kPageSize);
    const size_t base = out_row * p.max_chunks;
    float M = -INFINITY;
    for (int c = 0; c < n_chunks; ++c) M = fmaxf(M, p.ws_ml[(base + c) * 2]);
    float acc[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = 0.f;
    float L = 0.f;
    for (int c = 0; c < n_chunks; ++c) {
        const float mc = p.ws_ml[(base + c) * 2];
        const float w = mc == -INFINITY ? 0.f : ptx::ex2(mc - M);
        L += w * p.ws_ml[(base + c) * 2 + 1];
        const float* oc = p.ws_o + (base + c) * D + lane * PER;
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] += w * oc[e];
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) orow[lane * PER + e] = __float2bfloat16_rn(acc[e] * inv);
    if (p.lse != nullptr && lane == 0) p.lse[out_row] = L > 0.f ? (M + ptx::lg2(L)) * kLn2 : -INFINITY;
}

// One warp per row: the first S*T*Hq warps rotate a new query row (when q_rot is given), the next
// S*T*Hkv warps append a new token's key and value for one KV head (when k_new is given). Each
// lane handles D/64 bf16 pairs. An invalid length or block-table entry raises a status bit and
// the row is left alone.
template <int D>
__global__ void __launch_bounds__(128) decode_step_prep_kernel(const StepPrepParams a) {
    const long long w = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const long long q_rows = a.q_rot != nullptr ? static_cast<long long>(a.S) * a.T * a.Hq : 0;
    const long long kv_rows = a.k_new != nullptr ? static_cast<long long>(a.S) * a.T * a.Hkv : 0;
    if (w >= q_rows + kv_rows) return;
    const bool is_q = w < q_rows;
    const long long r = is_q ? w : w - q_rows;
    const int H = is_q ? a.Hq : a.Hkv;
    const long long st = r / H;
    const int t = static_cast<int>(st % a.T), s = static_cast<int>(st / a.T);
    const int len = a.seq_lens[s];
    if (len < a.T || len > a.max_blocks * kPageSize) {
        if (lane == 0) raise_status(kStatusBadSeqLen);
        return;
    }
    const int pos = len - a.T + t;
    const double2* cs = a.rope != nullptr ? a.rope + static_cast<size_t>(pos) * (D / 2) : nullptr;
    if (is_q) {
        const uint32_t* src = reinterpret_cast<const uint32_t*>(a.q + static_cast<size_t>(r) * D);
        uint32_t* dst = reinterpret_cast<uint32_t*>(a.q_rot + static_cast<size_t>(r) * D);
#pragma unroll
        for (int i = lane; i < D / 2; i += 32) {
            const double2 c = __ldg(cs + i);
            dst[i] = rope_rotate_pair(src[i], c.x, c.y);
        }
        return;
    }
    const int g = static_cast<int>(r % a.Hkv);
    const int page = a.block_table[static_cast<size_t>(s) * a.max_blocks + pos / kPageSize];
    if (page < 0 || page >= a.num_pages) {
        if (lane == 0) raise_status(kStatusBadPage);
        return;
    }
    const size_t src = static_cast<size_t>(r) * D;
    const size_t dst = ((static_cast<size_t>(page) * a.Hkv + g) * kPageSize + pos % kPageSize) * D;
    const uint32_t* ks = reinterpret_cast<const uint32_t*>(a.k_new + src);
    const uint32_t* vs = reinterpret_cast<const uint32_t*>(a.v_new + src);
    uint32_t* kd = reinterpret_cast<uint32_t*>(a.k_pages + dst);
    uint32_t* vd = reinterpret_cast<uint32_t*>(a.v_pages + dst);
#pragma unroll
    for (int i = lane; i < D / 2; i += 32) {
        uint32_t kw = ks[i];
        if (cs != nullptr) {
            const double2 c = __ldg(cs + i);
            kw = rope_rotate_pair(kw, c.x, c.y);
        }
        kd[i] = kw;
        vd[i] = vs[i];
    }
}

}  // namespace attn
