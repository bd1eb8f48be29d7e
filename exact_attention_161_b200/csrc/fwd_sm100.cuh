// fwd_sm100.cuh -- FlashAttention-style exact attention forward for sm_100a.
//
// The kernel is persistent: one CTA per SM walks a list of work items, each being two 128-row
// query tiles (256 consecutive queries) of one (batch, query head), longest items first. Both
// tiles stream the same visible 128-key tiles of the matching K/V head through shared memory, so
// each K/V tile loaded serves 256 query rows; the K/V rings run on across items, and the next
// item's queries are loaded while the current item finishes. Per row the online softmax keeps the
// running max m, the normaliser l and the output accumulator o, rescaled as the max grows, then
// O = o / l and the row logsumexp ("Why is attention O(n^2), how does FlashAttention help, ...",
// "Deep dive: FlashAttention"). The n x n score matrix never leaves the SM: each 128x128 score
// tile lives in Tensor Memory only.
//
// Roles (320 threads):
//   warps 0-3, 4-7  softmax warpgroup i (i = 0, 1) owns query tile i; thread r owns row r (TMEM
//              lane r). Per key tile it reads its 128 scores from TMEM with one load, masks them,
//              updates m and l, writes P (bf16) back into TMEM over the first half of its score
//              buffer, rescales its row of O when the max moved by more than 2^8, and finally
//              reads O out of TMEM (releasing it for the next item's products) and writes O and
//              LSE. Q and K arrive already rotated (RoPE) by a streaming pass before the kernel.
//   warp 8     TMA producer: the Q tiles once, then K tiles into an NK-stage ring and V tiles into
//              an NV-stage ring.
//   warp 9     MMA issuer and TMEM owner: the warp walks the schedule, one elected lane issues.
//
// Tensor Memory (512 columns): S0 at 0, S1 at 128, O0 at 256, O1 at 256 + D. The MMA thread
// issues, per key tile j:  O0 += P0(j) V(j);  S0(j+1) = Q0 K(j+1)^T;  O1 += P1(j) V(j);
// S1(j+1) = Q1 K(j+1)^T. So while warpgroup 0 computes the softmax of S0(j+1), the tensor core
// works on tile 1's products, and the other way round. tcgen05.mma executes in issue order, so
// when a warpgroup sees S_i(j+1) complete, the product O_i += P_i(j) V(j) issued before it has
// completed too: the warpgroup may then overwrite P_i and rescale O_i without a further wait.
//
// Masks enter as -inf on the logits before the softmax ("Transformer Attention Mechanism
// Interview Deep Dive", "Causal masking"); key tiles fully masked for a query tile are never
// visited by it (causal: tiles past the diagonal; sliding window: tiles before the window), the
// block skipping of "Deep dive: FlashAttention".
#pragma once
#include "common.cuh"
#include "ptx.cuh"

namespace attn {

struct FwdParams {
    __nv_bfloat16* o;       // [B, Hq, N, D]
    float* lse;             // [B, Hq, N] natural-log row logsumexp, or nullptr
    const float* alibi;     // [Hq] ALiBi slopes m_h (logit minus m_h (i - j)), read when kAlibi
    float o_scale;          // output multiplier (the FP8 path's V descale; 1 otherwise)
    int B, Hq, Hkv, N;
    int causal, window;     // window > 0 only together with causal
    float scale_log2;       // softmax scale * log2(e)
    int nblk;               // 256-query blocks per (batch, head)
    int n_items;            // B * Hq * nblk work items
    int debug_drop_copy;    // test hook: CTA 0 skips its first key-tile copy (see attn.h)
};

template <int D, bool kFp8 = false>
struct FwdCfg {
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    static_assert(!kFp8 || D == 128, "the FP8 path takes D = 128");
    static constexpr int ELEM = kFp8 ? 1 : 2;         // bytes per Q/K/V element (e4m3 or bf16)
    static constexpr int BM = 128;                    // query rows per tile
    static constexpr int BN = 128;                    // keys per tile
    static constexpr int QT = 2;                      // query tiles per CTA
    static constexpr int ROW_BYTES = D * ELEM;
    static constexpr int NREG = ROW_BYTES / 128;      // 128-byte swizzle regions per row
    static constexpr int TMA_X = 128 / ELEM;          // elements per region row (TMA box width)
    static constexpr int REGION_BYTES = 128 * 128;    // 128 rows x 128 bytes
    static constexpr int TILE_BYTES = 128 * ROW_BYTES;  // one Q, K or V tile
    static constexpr int S_KSTEPS = ROW_BYTES / 32;   // MMAs per score tile (32 bytes of K each)
    static constexpr int O_KSTEPS = BN * ELEM / 32;   // MMAs per P V (32 bytes of P per row each)
    static constexpr int O_ROWS = 32 / ELEM;          // keys (V rows) per P V MMA
    static constexpr int P_COLS = BN * ELEM / 4;      // TMEM columns that hold P
    // K and V pipeline stages. K(u) is read one step before V(u) and both stages of a step are
    // released together, so at D = 128 (five 32 KB tiles fit beside Q) V gets the deeper ring.
    static constexpr int NK = kFp8 ? 4 : (D == 128) ? 2 : 4;
    static constexpr int NV = kFp8 ? 4 : (D == 128) ? 3 : 4;
    static constexpr int SMEM_TILES = QT + NK + NV;
    static constexpr int SMEM_BYTES = SMEM_TILES * TILE_BYTES + 1024 /*barriers*/ + 1024 /*align*/;
    static constexpr uint32_t TMEM_COLS = 512;
    // TMEM columns of the score buffer and the output accumulator of query tile i
    static __device__ __forceinline__ uint32_t tmem_s(int i) { return 128u * i; }
    static __device__ __forceinline__ uint32_t tmem_o(int i) { return 256u + uint32_t(D) * i; }
    static constexpr int THREADS = 320;
    static constexpr int PRODUCER_WARP = 8, MMA_WARP = 9;
    // Rescale the output only when the running max grew by more than this (log2 units): with a
    // stale max the probabilities stay below 2^8, exact after the final division by l.
    static constexpr float RESCALE_THRESHOLD = 8.0f;
};

template <int NK, int NV>
struct FwdBarriers {
    uint64_t q_loaded[2], q_empty[2];
    uint64_t k_full[NK], k_empty[NK], v_full[NV], v_empty[NV];
    uint64_t s_full[2], p_full[2], o_final[2], o_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

// Key-tile range of one query tile: [jb, jb + n) of 128-key tiles with at least one visible key.
struct TileRange {
    int q0, jb, n;
};

__device__ __forceinline__ TileRange tile_range(int q0, int N, int causal, int window) {
    TileRange t{q0, 0, 0};
    if (q0 >= N) return t;
    const int hi = causal ? min(N, q0 + 128) : N;             // exclusive
    const int lo = window > 0 ? max(0, q0 - window + 1) : 0;  // inclusive
    t.jb = lo / 128;
    t.n = (hi + 127) / 128 - t.jb;
    return t;
}

// One work item: (batch b, query head h, block of 256 queries); the longest causal blocks come
// first, and the query heads of one block are adjacent so heads sharing a K/V head run together.
struct Item {
    int b, h, blk;
    TileRange rng[2];
    int J0, T;  // union of the two key-tile ranges
    __device__ __forceinline__ bool active(int i, int u) const {
        const int j = J0 + u;
        return rng[i].n > 0 && j >= rng[i].jb && j < rng[i].jb + rng[i].n;
    }
};

// Item of round r for CTA c: rounds alternate direction over the CTAs (c, then G-1-c), which with
// the longest-first item order balances the causal work to within a fraction of a percent.
__device__ __forceinline__ int item_of_round(int r, int c, int G) { return r * G + ((r & 1) ? G - 1 - c : c); }

__device__ __forceinline__ Item make_item(const FwdParams& p, int it) {
    Item x;
    const int bh = it % (p.B * p.Hq);
    x.blk = p.nblk - 1 - it / (p.B * p.Hq);
    x.b = bh / p.Hq;
    x.h = bh % p.Hq;
    x.rng[0] = tile_range(x.blk * 256, p.N, p.causal, p.window);
    x.rng[1] = tile_range(x.blk * 256 + 128, p.N, p.causal, p.window);
    // Tile 1 starts no earlier and ends no earlier than tile 0, so the union is contiguous.
    x.J0 = x.rng[0].jb;
    const int end0 = x.rng[0].jb + x.rng[0].n;
    x.T = (x.rng[1].n > 0 ? max(end0, x.rng[1].jb + x.rng[1].n) : end0) - x.J0;
    return x;
}

#ifndef ATTN_FP8_POLY_EVERY
#define ATTN_FP8_POLY_EVERY 1
#endif
#ifndef ATTN_BF16_POLY_EVERY
#define ATTN_BF16_POLY_EVERY 2
#endif

// kFp8: Q, K, V in e4m3; both products run as kind::f8f6f4 (K = 32 per MMA) and P is packed to
// e4m3 for the second one; the scores' scale carries the Q and K descales (scale_log2) and the
// output the V descale (o_scale). No RoPE on this path.
template <int D, bool kAlibi, bool kFp8 = false>
__global__ void __launch_bounds__(FwdCfg<D, kFp8>::THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    using C = FwdCfg<D, kFp8>;
    constexpr int NK = C::NK, NV = C::NV;
    // the exponential pair of columns 6-7 of every kPolyEvery-th group of 8 is evaluated on the FMA
    // pipe (0: none); FP8 also moves the pair of columns 4-5 of every second group there
    constexpr int kPolyEvery = kFp8 ? ATTN_FP8_POLY_EVERY : ATTN_BF16_POLY_EVERY;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;                                  // QT tiles
    uint8_t* sK = sQ + C::QT * C::TILE_BYTES;            // NK tiles
    uint8_t* sV = sK + NK * C::TILE_BYTES;               // NV tiles
    auto* bar = reinterpret_cast<FwdBarriers<NK, NV>*>(sV + NV * C::TILE_BYTES);
    volatile int* abort_flag = &bar->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&bar->q_loaded[i], 1);
            ptx::mbar_init(&bar->q_empty[i], 1);
            ptx::mbar_init(&bar->s_full[i], 1);
            ptx::mbar_init(&bar->p_full[i], 128);
            ptx::mbar_init(&bar->o_final[i], 1);
            ptx::mbar_init(&bar->o_empty[i], 128);
        }
        for (int s = 0; s < NK; ++s) {
            ptx::mbar_init(&bar->k_full[s], 1);
            ptx::mbar_init(&bar->k_empty[s], 1);
        }
        for (int s = 0; s < NV; ++s) {
            ptx::mbar_init(&bar->v_full[s], 1);
            ptx::mbar_init(&bar->v_empty[s], 1);
        }
        ptx::mbar_init(&bar->drain, 1);
        bar->abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == C::PRODUCER_WARP && lane == 0) {
        ptx::prefetch_tensormap(&tm_q);
        ptx::prefetch_tensormap(&tm_k);
        ptx::prefetch_tensormap(&tm_v);
    }
    if (warp == C::MMA_WARP) {
        ptx::tmem_alloc(&bar->tmem_base, C::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    // Launched right behind the query/key rotation pass, the kernel may start before that pass
    // has finished: the set-up above overlaps its tail, and every thread waits here for it (and its
    // writes) to complete before any global memory is read or written.
    ptx::grid_dependency_wait();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = bar->tmem_base;

    if (warp == C::PRODUCER_WARP) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int kq[2] = {0, 0};  // items in which query tile i was loaded so far
            int g = 0;           // key tiles streamed so far (ring position)
            int k_issued = 0, v_issued = 0;
            bool ok = true;
            for (int rnd = 0, it = blockIdx.x; ok && it < p.n_items; it = item_of_round(++rnd, blockIdx.x, gridDim.x)) {
                const Item x = make_item(p, it);
                const int zq = x.b * p.Hq + x.h, zk = x.b * p.Hkv + x.h / (p.Hq / p.Hkv);
                for (int i = 0; i < 2 && ok; ++i) {
                    if (x.rng[i].n == 0) continue;
                    // the buffer is free once the previous item's last S_i has been computed
                    if (kq[i] > 0 && !ptx::mbar_wait(&bar->q_empty[i], (kq[i] - 1) & 1, abort_flag)) { ok = false; break; }
                    ptx::mbar_arrive_expect_tx(&bar->q_loaded[i], C::TILE_BYTES);
#pragma unroll
                    for (int r = 0; r < C::NREG; ++r)
                        ptx::tma_load_3d(sQ + i * C::TILE_BYTES + r * C::REGION_BYTES, &tm_q, &bar->q_loaded[i],
                                         r * C::TMA_X, x.rng[i].q0, zq);
                    ++kq[i];
                }
                for (int u = 0; u < x.T && ok; ++u, ++g) {
                    const int k0 = (x.J0 + u) * C::BN;
                    const int sk = g % NK, sv = g % NV;
                    if (g >= NK && !ptx::mbar_wait(&bar->k_empty[sk], ((g / NK) - 1) & 1, abort_flag)) { ok = false; break; }
                    ptx::mbar_arrive_expect_tx(&bar->k_full[sk], C::TILE_BYTES);
                    if (!(p.debug_drop_copy && g == 0 && blockIdx.x == 0)) {
#pragma unroll
                        for (int r = 0; r < C::NREG; ++r)
                            ptx::tma_load_3d(sK + sk * C::TILE_BYTES + r * C::REGION_BYTES, &tm_k, &bar->k_full[sk],
                                             r * C::TMA_X, k0, zk);
                    }
                    k_issued = g + 1;
                    if (g >= NV && !ptx::mbar_wait(&bar->v_empty[sv], ((g / NV) - 1) & 1, abort_flag)) { ok = false; break; }
                    ptx::mbar_arrive_expect_tx(&bar->v_full[sv], C::TILE_BYTES);
#pragma unroll
                    for (int r = 0; r < C::NREG; ++r)
                        ptx::tma_load_3d(sV + sv * C::TILE_BYTES + r * C::REGION_BYTES, &tm_v, &bar->v_full[sv],
                                         r * C::TMA_X, k0, zk);
                    v_issued = g + 1;
                }
            }
            if (!ok) {
                *abort_flag = 1;
                raise_status(kStatusTimeout);
                // Let the copies already in flight land before the CTA's shared memory is released
                // (each wait is still bounded).
                volatile int never = 0;
                for (int i = 0; i < 2; ++i)
                    if (kq[i] > 0) ptx::mbar_wait(&bar->q_loaded[i], (kq[i] - 1) & 1, &never);
                for (int u = max(0, k_issued - NK); u < k_issued; ++u)
                    ptx::mbar_wait(&bar->k_full[u % NK], (u / NK) & 1, &never);
                for (int u = max(0, v_issued - NV); u < v_issued; ++u)
                    ptx::mbar_wait(&bar->v_full[u % NV], (u / NV) & 1, &never);
            }
        }
    } else if (warp == C::MMA_WARP) {
        // ------------------------------------------------------------------ MMA issuer
        // The whole warp walks the schedule and takes the waits, so every index, TMEM address and
        // descriptor is warp-uniform; the tcgen05 instructions carry a lane predicate, so that one
        // elected lane issues them without the warp leaving the converged path. Descriptors are
        // 64-bit words built once; stepping through a tile adds a constant to their address field.
        const uint32_t issue = ptx::elect_one() ? 1u : 0u;
        const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
        // Q, K both K-major; P K-major, V MN-major
        constexpr uint32_t IDESC_S = kFp8 ? ptx::idesc_e4m3_f32(128, C::BN, 0, 0) : ptx::idesc_bf16_f32(128, C::BN, 0, 0);
        constexpr uint32_t IDESC_O = kFp8 ? ptx::idesc_e4m3_f32(128, D, 0, 1) : ptx::idesc_bf16_f32(128, D, 0, 1);
        constexpr uint32_t HI = ptx::sw128_desc_hi(1024);                    // 8-row groups 1024 B apart
        constexpr uint64_t TILE16 = C::TILE_BYTES >> 4;
        // descriptors of Q tile 0, K stage 0 and V stage 0 (K-major LBO unused = 16; V is MN-major
        // with its 64-column halves one region apart)
        const uint64_t q_d = ptx::desc64(__shfl_sync(0xffffffffu, ptx::sw128_desc_lo(ptx::smem_u32(sQ), 16), 0), HI);
        const uint64_t k_d = ptx::desc64(__shfl_sync(0xffffffffu, ptx::sw128_desc_lo(ptx::smem_u32(sK), 16), 0), HI);
        const uint64_t v_d =
            ptx::desc64(__shfl_sync(0xffffffffu, ptx::sw128_desc_lo(ptx::smem_u32(sV), C::REGION_BYTES), 0), HI);
        bool ok = true, issued_any = false;
        int kq0 = 0, kq1 = 0;  // items of query tile 0 / 1 started so far
        int cw0 = 0, cw1 = 0;  // score tiles of query tile 0 / 1 computed so far (all items)
        int g = 0;             // key tiles consumed so far (ring position)
        for (int rnd = 0, it = blockIdx.x; ok && it < p.n_items; it = item_of_round(++rnd, blockIdx.x, gridDim.x)) {
            const Item x = make_item(p, it);
            // per tile: first and one-past-last u of its key tiles (empty when the tile is past N)
            const int a0 = x.rng[0].jb - x.J0, e0 = x.rng[0].n > 0 ? a0 + x.rng[0].n : a0;
            const int a1 = x.rng[1].jb - x.J0, e1 = x.rng[1].n > 0 ? a1 + x.rng[1].n : a1;
            for (int u = -1; ok && u < x.T; ++u) {
                // u = -1: the prologue (scores of the first key tile only)
                if (u >= 0) {
                    if (!ptx::mbar_wait_warp(&bar->v_full[(g + u) % NV], ((g + u) / NV) & 1, abort_flag)) { ok = false; break; }
                }
                bool k_ready = false;
                for (int i = 0; i < 2; ++i) {
                    const int kq = i ? kq1 : kq0, cw = i ? cw1 : cw0;
                    const int a = i ? a1 : a0, e = i ? e1 : e0;
                    const uint32_t d_s = tm + C::tmem_s(i), d_o = tm + C::tmem_o(i);
                    if (u >= a && u < e) {
                        // O_i += P_i(u) V(u); P_i in TMEM over the first 64 columns of score buffer i
                        const int c = u - a;
                        if (c == 0 && kq > 0 && !ptx::mbar_wait_warp(&bar->o_empty[i], (kq - 1) & 1, abort_flag)) { ok = false; break; }
                        if (!ptx::mbar_wait_warp(&bar->p_full[i], (cw + c) & 1, abort_flag)) { ok = false; break; }
                        ptx::tc_fence_after();  // P was written to TMEM by the softmax warps
                        const uint64_t vb = v_d + ((g + u) % NV) * TILE16;
#pragma unroll
                        for (int kk = 0; kk < C::O_KSTEPS; ++kk) {
                            const uint64_t bd = vb + kk * ((C::O_ROWS * 128) >> 4);
                            if constexpr (kFp8)
                                ptx::mma_ts_f8_if(issue, d_o, d_s + kk * 8, bd, IDESC_O, (c > 0 || kk > 0) ? 1u : 0u);
                            else
                                ptx::mma_ts_if(issue, d_o, d_s + kk * 8, bd, IDESC_O, (c > 0 || kk > 0) ? 1u : 0u);
                        }
                        if (c == e - a - 1) ptx::mma_commit_if(issue, &bar->o_final[i]);
                    }
                    if (u + 1 >= a && u + 1 < e) {
                        // S_i(u+1) = Q_i K(u+1)^T into score buffer i
                        const int c = u + 1 - a;
                        // Q and K arrive by TMA: the barriers alone order them before the MMA's reads
                        if (c == 0 && !ptx::mbar_wait_warp(&bar->q_loaded[i], kq & 1, abort_flag)) { ok = false; break; }
                        if (!k_ready && !ptx::mbar_wait_warp(&bar->k_full[(g + u + 1) % NK], ((g + u + 1) / NK) & 1, abort_flag)) { ok = false; break; }
                        k_ready = true;
                        const uint64_t qa = q_d + i * TILE16, kb = k_d + ((g + u + 1) % NK) * TILE16;
#pragma unroll
                        for (int kk = 0; kk < C::S_KSTEPS; ++kk) {
                            const uint64_t off = ((kk >> 2) * C::REGION_BYTES + (kk & 3) * 32) >> 4;
                            if constexpr (kFp8)
                                ptx::mma_ss_f8_if(issue, d_s, qa + off, kb + off, IDESC_S, kk > 0);
                            else
                                ptx::mma_ss_if(issue, d_s, qa + off, kb + off, IDESC_S, kk > 0);
                        }
                        ptx::mma_commit_if(issue, &bar->s_full[i]);
                        if (c == e - a - 1) ptx::mma_commit_if(issue, &bar->q_empty[i]);  // Q_i no longer read
                        issued_any = true;
                    }
                }
                if (!ok) break;
                if (u >= 0) ptx::mma_commit_if(issue, &bar->v_empty[(g + u) % NV]);
                if (u + 1 < x.T) ptx::mma_commit_if(issue, &bar->k_empty[(g + u + 1) % NK]);
            }
            if (x.rng[0].n > 0) { ++kq0; cw0 += x.rng[0].n; }
            if (x.rng[1].n > 0) { ++kq1; cw1 += x.rng[1].n; }
            g += x.T;
        }
        if (!ok) {
            if (issue) {
                *abort_flag = 1;
                raise_status(kStatusTimeout);
                if (issued_any) {  // wait for the MMAs in flight before TMEM is released
                    ptx::mma_commit(&bar->drain);
                    volatile int never = 0;
                    ptx::mbar_wait(&bar->drain, 0, &never);
                }
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ softmax warpgroups
        const int wg = warp >> 2;            // query tile of this warpgroup
        const int r = threadIdx.x & 127;     // row within the tile == TMEM lane
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t t_s = tmem + lane_base + C::tmem_s(wg);
        const uint32_t t_o = tmem + lane_base + C::tmem_o(wg);
        const float sl = p.scale_log2;
        // The warpgroup never touches Q: the MMA warp computes an item's first scores as soon as
        // its query tile has landed (the tile's buffer was freed by the previous item's last score
        // MMA), which overlaps them with this warpgroup's epilogue of the previous item. Score
        // buffer reuse is ordered by the MMA warp issuing P(n, last) V before S(n+1, 0), and item
        // n+1's first P V waits for o_empty, which the epilogue arrives on. Waits are made uniform
        // per warp, because the tile loop holds warp-wide votes.
        bool ok = true;
        int kq = 0, cw = 0;
        for (int rnd = 0, it = blockIdx.x; ok && it < p.n_items; it = item_of_round(++rnd, blockIdx.x, gridDim.x)) {
            const Item x = make_item(p, it);
            const TileRange R = x.rng[wg];
            if (R.n == 0) continue;
            const int i_pos = R.q0 + r;  // query position
            // ALiBi: this head's slope in log2 units
            const float slope2 = kAlibi ? p.alibi[x.h] * kLog2e : 0.f;

            float m_used = -INFINITY, l = 0.f;
            for (int c = 0; ok && c < R.n; ++c) {
                const int j0 = (R.jb + c) * C::BN;
                if (!__all_sync(0xffffffffu, ptx::mbar_wait(&bar->s_full[wg], (cw + c) & 1, abort_flag))) { ok = false; break; }
                ptx::tc_fence_after();
                uint32_t sv[C::BN];
                ptx::tmem_ld128(t_s, sv);
                float s[C::BN];
#pragma unroll
                for (int k = 0; k < C::BN; ++k) s[k] = __uint_as_float(sv[k]);
                const bool need_mask = (j0 + C::BN > p.N) || (p.causal && j0 + C::BN - 1 > R.q0) ||
                                       (p.window > 0 && j0 < R.q0 + C::BM - p.window);
                if (need_mask) {
                    const int lo = p.window > 0 ? i_pos - p.window + 1 : -0x7fffffff;
                    const int hi = p.causal ? min(i_pos, p.N - 1) : p.N - 1;
#pragma unroll
                    for (int k = 0; k < C::BN; ++k) {
                        const int kj = j0 + k;
                        if (kj < lo || kj > hi) s[k] = -INFINITY;
                    }
                }
                // Row max. Plain: the max of the scores, scaled. ALiBi: an upper bound of the biased
                // logits s*scale_log2 + slope2*(j - i), from the max score of each 16-column group plus
                // the group's largest bias; it exceeds the true max by at most 15 slope steps, which
                // keeps P far from underflow, and the online softmax and the LSE are exact for any
                // upper bound. The bias then enters only the exponent argument below.
                float m_new;
                const float b0 = kAlibi ? slope2 * static_cast<float>(j0 - i_pos) : 0.f;
                if constexpr (kAlibi) {
                    const int kend = slope2 >= 0.f ? 15 : 0;
                    float bound = -INFINITY;
#pragma unroll
                    for (int g = 0; g < C::BN / 16; ++g) {
                        float a = fmaxf(s[16 * g], s[16 * g + 1]), b = fmaxf(s[16 * g + 2], s[16 * g + 3]);
#pragma unroll
                        for (int k = 16 * g + 4; k < 16 * g + 16; k += 4) {
                            a = ptx::fmax3(a, s[k], s[k + 1]);
                            b = ptx::fmax3(b, s[k + 2], s[k + 3]);
                        }
                        bound = fmaxf(bound, fmaf(fmaxf(a, b), sl, fmaf(slope2, static_cast<float>(16 * g + kend), b0)));
                    }
                    m_new = bound;
                } else {
                    // four independent chains over s[0..7], s[8..15], ...: every element exactly once
                    float mx0 = fmaxf(s[0], s[1]), mx1 = fmaxf(s[2], s[3]), mx2 = fmaxf(s[4], s[5]),
                          mx3 = fmaxf(s[6], s[7]);
#pragma unroll
                    for (int k = 8; k < C::BN; k += 8) {
                        mx0 = ptx::fmax3(mx0, s[k], s[k + 1]);
                        mx1 = ptx::fmax3(mx1, s[k + 2], s[k + 3]);
                        mx2 = ptx::fmax3(mx2, s[k + 4], s[k + 5]);
                        mx3 = ptx::fmax3(mx3, s[k + 6], s[k + 7]);
                    }
                    m_new = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl;
                }
                float alpha = 1.f;
                bool rescale = false;
                if (m_new > m_used + C::RESCALE_THRESHOLD) {  // also the first visible key (m_used = -inf)
                    alpha = ptx::ex2(m_used - m_new);          // 2^-inf = 0
                    m_used = m_new;
                    rescale = true;
                }
                const float m_eff = (m_used == -INFINITY) ? 0.f : m_used;
                const float2 sl2 = make_float2(sl, sl), nm2 = make_float2(-m_eff, -m_eff);
                // ALiBi: the addend of column k is slope2*k + b0 - m instead of -m; per group of 8
                // columns one FMA gives the group's base, the other columns follow from it
                const float bm = b0 - m_eff;
                float2 acc0 = make_float2(0.f, 0.f), acc1 = acc0, acc2 = acc0, acc3 = acc0;
                uint32_t pk[C::P_COLS];
#pragma unroll
                for (int k = 0; k < C::BN; k += 8) {
                    float2 a0, a1, a2, a3;
                    if constexpr (!kAlibi) {
                        a0 = a1 = a2 = a3 = nm2;
                    } else {
                        const float bg = fmaf(slope2, static_cast<float>(k), bm);
                        a0 = make_float2(bg, bg + slope2);
                        a1 = make_float2(fmaf(slope2, 2.f, bg), fmaf(slope2, 3.f, bg));
                        a2 = make_float2(fmaf(slope2, 4.f, bg), fmaf(slope2, 5.f, bg));
                        a3 = make_float2(fmaf(slope2, 6.f, bg), fmaf(slope2, 7.f, bg));
                    }
                    float2 x0 = ptx::ffma2(make_float2(s[k], s[k + 1]), sl2, a0);
                    float2 x1 = ptx::ffma2(make_float2(s[k + 2], s[k + 3]), sl2, a1);
                    float2 x2 = ptx::ffma2(make_float2(s[k + 4], s[k + 5]), sl2, a2);
                    float2 x3 = ptx::ffma2(make_float2(s[k + 6], s[k + 7]), sl2, a3);
                    x0 = make_float2(ptx::ex2(x0.x), ptx::ex2(x0.y));
                    x1 = make_float2(ptx::ex2(x1.x), ptx::ex2(x1.y));
                    // Some exponential pairs go to the FMA pipe, which the softmax leaves mostly idle
                    // while the SFU is busy. bf16: columns 6-7 of every second group of 8 (1/8 of
                    // the exponentials), one lane at a time (the packed form's extra registers
                    // spill there). FP8, whose SFU also packs P to e4m3 and whose P takes fewer
                    // registers: columns 6-7 of every group and 4-5 of every second one (3/8), on
                    // packed f32x2 instructions. Shares of 1/4, 5/16, 7/16 and 1/2 measured slower
                    // for FP8. The polynomial's 1e-4 relative error is far below the rounding of P
                    // to bf16 or e4m3; it gives exactly 1 at 0 and exactly 0 for masked scores.
                    if (kFp8 && (k / 8) % 2 == 0) x2 = ptx::ex2_poly2(x2);
                    else x2 = make_float2(ptx::ex2(x2.x), ptx::ex2(x2.y));
                    if constexpr (kPolyEvery > 0) {
                        if ((k / 8) % kPolyEvery == 0)
                            x3 = kFp8 ? ptx::ex2_poly2(x3) : make_float2(ptx::ex2_poly(x3.x), ptx::ex2_poly(x3.y));
                        else
                            x3 = make_float2(ptx::ex2(x3.x), ptx::ex2(x3.y));
                    } else {
                        x3 = make_float2(ptx::ex2(x3.x), ptx::ex2(x3.y));
                    }
                    acc0 = ptx::fadd2(acc0, x0);
                    acc1 = ptx::fadd2(acc1, x1);
                    acc2 = ptx::fadd2(acc2, x2);
                    acc3 = ptx::fadd2(acc3, x3);
                    if constexpr (kFp8) {
                        pk[k / 4] = ptx::pack_e4m3x4(x0.x, x0.y, x1.x, x1.y);
                        pk[k / 4 + 1] = ptx::pack_e4m3x4(x2.x, x2.y, x3.x, x3.y);
                    } else {
                        pk[k / 2] = ptx::pack_bf16x2(x0.x, x0.y);
                        pk[k / 2 + 1] = ptx::pack_bf16x2(x1.x, x1.y);
                        pk[k / 2 + 2] = ptx::pack_bf16x2(x2.x, x2.y);
                        pk[k / 2 + 3] = ptx::pack_bf16x2(x3.x, x3.y);
                    }
                }
                const float2 a01 = ptx::fadd2(acc0, acc1), a23 = ptx::fadd2(acc2, acc3);
                const float2 a = ptx::fadd2(a01, a23);
                l = l * alpha + (a.x + a.y);
                // P (bf16 pairs, or e4m3 quadruples) over the first columns of this tile's score buffer.
                if constexpr (kFp8)
                    ptx::tmem_st32(t_s, pk);
                else
                    ptx::tmem_st64(t_s, pk);
                if (c > 0 && __any_sync(0xffffffffu, rescale)) {
                    // The product with the previous P has completed (it was issued before this
                    // tile's scores), so O_i is stable here.
                    const float2 al2 = make_float2(alpha, alpha);
#pragma unroll
                    for (int cc = 0; cc < D / 32; ++cc) {
                        uint32_t v[32];
                        ptx::tmem_ld32(t_o + cc * 32, v);
#pragma unroll
                        for (int k = 0; k < 32; k += 2) {
                            const float2 y =
                                ptx::fmul2(make_float2(__uint_as_float(v[k]), __uint_as_float(v[k + 1])), al2);
                            v[k] = __float_as_uint(y.x);
                            v[k + 1] = __float_as_uint(y.y);
                        }
                        ptx::tmem_st32(t_o + cc * 32, v);
                    }
                }
                ptx::tc_fence_before();
                ptx::mbar_arrive(&bar->p_full[wg]);
            }
            if (!ok) break;
            cw += R.n;
            // ---- epilogue: O_i out of TMEM (then the next item may overwrite it), O = o / l, LSE
            if (!__all_sync(0xffffffffu, ptx::mbar_wait(&bar->o_final[wg], kq & 1, abort_flag))) { ok = false; break; }
            ptx::tc_fence_after();
            uint32_t w[D / 2];
            const float inv_l = l > 0.f ? p.o_scale / l : 0.f;
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t v[32];
                ptx::tmem_ld32(t_o + cc * 32, v);
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    w[cc * 16 + k] =
                        ptx::pack_bf16x2(__uint_as_float(v[2 * k]) * inv_l, __uint_as_float(v[2 * k + 1]) * inv_l);
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&bar->o_empty[wg]);
            if (i_pos < p.N) {
                uint4* dst = reinterpret_cast<uint4*>(p.o + ((static_cast<size_t>(x.b) * p.Hq + x.h) * p.N + i_pos) * D);
#pragma unroll
                for (int k = 0; k < D / 8; ++k) dst[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
                if (p.lse != nullptr)
                    p.lse[(static_cast<size_t>(x.b) * p.Hq + x.h) * p.N + i_pos] =
                        l > 0.f ? (m_used + ptx::lg2(l)) * kLn2 : -INFINITY;
            }
            ++kq;
        }
        if (!ok) {
            *abort_flag = 1;
            raise_status(kStatusTimeout);
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == C::MMA_WARP) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace attn
