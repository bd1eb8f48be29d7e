// bwd_sm100.cuh -- backward of exact attention for sm_100a, recomputing the scores.
//
// For L = sum(O * dO), with P the softmax rows of the forward and LSE its saved logsumexp, the
// gradients are (chain rule through the softmax; "Self-Attention Complexity, FlashAttention,
// PagedAttention, and RoPE in Code", Part 2, and "Why is attention O(n^2), how does FlashAttention
// help, ...", "Deep dive: FlashAttention": the backward recomputes the scores from the saved
// statistics instead of storing P):
//   P_ij  = 2^(s_ij * scale * log2(e) - LSE_i * log2(e))    (recomputed, never stored in HBM)
//   dV_j  = sum_i P_ij dO_i             dP_ij = dO_i . v_j
//   dS_ij = P_ij (dP_ij - D_i)          D_i   = dO_i . O_i  (= sum_j P_ij dP_ij)
//   dq_i  = scale sum_j dS_ij k_j       dk_j  = scale sum_i dS_ij q_i
// with q, k the rotated vectors; RoPE's gradient rotates dq, dk back by -angle.
//
// Three kernels: a prep pass (D_i and the log2-scaled LSE, padded per 128-row tile), the main
// kernel with one CTA per (128-key tile, K/V head) that walks every query head of the group and
// every query tile that sees the keys, and a pass that turns the fp32 dq sums into bf16. The five
// products of a tile pair (S^T, dP^T, dV, dK, dQ) run on tcgen05 with fp32 accumulators in Tensor
// Memory: dK and dV accumulate there over the whole walk; the dQ of each tile pair is added into an
// fp32 array in device memory by TMA reductions, since every key tile contributes to it.
// Sixteen elementwise warps (four groups, each owning 32 of the 128 query columns of a tile) turn
// scores into P and dS and move the dQ partials out; the products are issued in an order that
// lets the tensor core work while they do (see the issue loop). CTAs are numbered so that the
// ones with the most work start first.
#pragma once
#include "common.cuh"
#include "fwd_sm100.cuh"
#include "ptx.cuh"

namespace attn {

struct BwdParams {
    const __nv_bfloat16* o;     // [B, Hq, N, D] forward output
    const __nv_bfloat16* dout;  // [B, Hq, N, D]
    const float* lse;           // [B, Hq, N] forward logsumexp (natural log)
    float* vec;                 // [B*Hq, ntiles, 2, 128]: per 128-row tile -LSE*log2 e, then -D_i;
                                // rows >= N hold (-inf, 0)
    __nv_bfloat16* dq;          // [B, Hq, N, D]
    float* dqacc;               // [B*Hq, ntiles*128, D] fp32 sums of dS K, zeroed by the prep kernel
    __nv_bfloat16* dk;          // [B, Hkv, N, D]
    __nv_bfloat16* dv;          // [B, Hkv, N, D]
    const float2* rope;         // (cos, sin) table or nullptr
    int B, Hq, Hkv, N, ntiles;
    int causal, window;
    float scale, scale_log2;
    int debug_drop_copy;        // test hook: CTA 0 skips its first Q / dO copy (see attn.h)
};

// Per query row: -D_i = -(dO_i . O_i) and -LSE_i * log2(e), stored negated so that the kernels add
// them, and the row's fp32 dq sums set to zero. D/8 lanes share a row (16-byte loads), grid-stride
// over all padded rows; rows past N get (-inf, 0) so that their recomputed probabilities are
// exactly 0.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const BwdParams p) {
    constexpr int LPR = D / 8;     // lanes per row
    constexpr int RPW = 32 / LPR;  // rows per warp and pass
    const int lane = threadIdx.x & 31, sub = lane / LPR, l = lane % LPR;
    const long long npad = static_cast<long long>(p.ntiles) * 128;
    const long long rows = static_cast<long long>(p.B) * p.Hq * npad;
    const long long nwarps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
    for (long long base = (static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5)) * RPW;
         base < rows; base += nwarps * RPW) {
        const long long row = base + sub;
        const long long bh = row / npad;
        const int i = static_cast<int>(row - bh * npad);
        const bool valid = row < rows && i < p.N;
        float acc = 0.f;
        if (valid) {
            const size_t off = (static_cast<size_t>(bh) * p.N + i) * D + l * 8;
            const uint4 a = __ldg(reinterpret_cast<const uint4*>(p.o + off));
            const uint4 b = __ldg(reinterpret_cast<const uint4*>(p.dout + off));
            const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                acc = fmaf(ptx::bf16lo_to_f32(aw[e]), ptx::bf16lo_to_f32(bw[e]), acc);
                acc = fmaf(ptx::bf16hi_to_f32(aw[e]), ptx::bf16hi_to_f32(bw[e]), acc);
            }
        }
        if (row < rows) {
            float4* z = reinterpret_cast<float4*>(p.dqacc + static_cast<size_t>(row) * D + l * 8);
            z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
            z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int m = LPR / 2; m >= 1; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
        if (row < rows && l == 0) {
            float* v = p.vec + (static_cast<size_t>(bh) * p.ntiles + i / 128) * 256 + (i & 127);
            v[0] = valid ? -p.lse[static_cast<size_t>(bh) * p.N + i] * kLog2e : -INFINITY;
            v[128] = valid ? -acc : 0.f;
        }
    }
}

template <int D>
struct BwdCfg {
    static constexpr int NREG = D / 64;
    static constexpr int REGION_BYTES = 128 * 128;
    static constexpr int TILE_BYTES = 128 * D * 2;
    static constexpr int DS_BYTES = 2 * REGION_BYTES;  // dS^T of one tile pair: 128 keys x 128 queries, bf16
    static constexpr int VEC_BYTES = 256 * 4;  // -LSE*log2 e and -D of the 128 rows of a query tile
    // K, V fixed + two stages of Q, dO + dS + two stages of the vectors, from a 1024-byte boundary
    // (128-byte swizzled tiles), + 1024 bytes for the gap in front of that boundary and the barriers:
    // the barriers (128 bytes) sit in the gap when it is at least that large, else after the vectors
    static constexpr int SMEM_BYTES = 6 * TILE_BYTES + DS_BYTES + 2 * VEC_BYTES + 1024;
    static_assert(SMEM_BYTES <= 232448, "backward shared memory above 227 KiB per CTA");
    // warps 0-15 elementwise (four groups of 32 query columns), 16 TMA producer, 17 MMA issuer,
    // 18 dQ reduce
    static constexpr int THREADS = 608;
    static constexpr int PRODUCER_WARP = 16, MMA_WARP = 17, REDUCE_WARP = 18;
    static constexpr int EW_THREADS = 512;
    static constexpr uint32_t TMEM_COLS = 512;
};

struct BwdBarriers {
    uint64_t fixed_loaded;
    uint64_t full[2], empty[2];
    uint64_t staged[2];  // the dQ partial of the step held in stage s is in shared memory
    uint64_t s_full, dp_full, p_full, ds_full, dq_full, dq_free, acc_done, drain;
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(BwdBarriers) <= 128, "barrier block larger than its reserved bytes");

// 32 consecutive columns [c0, c0 + 32) of a gradient row held in registers (fp32, pairs (2t, 2t+1)):
// rotate each pair by -angle at position pos (the gradient of the unrotated vector is the
// rotated-back gradient), scale, and store as bf16. rope == nullptr: no rotation.
__device__ __forceinline__ void store_chunk_unrotated(const uint32_t (&v)[32], float scale, const float2* rope,
                                                      int D, int pos, int c0, __nv_bfloat16* dst_row) {
    float g[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) g[e] = __uint_as_float(v[e]) * scale;
    if (rope != nullptr) {
        const float2* cs = rope + static_cast<size_t>(pos) * (D / 2) + c0 / 2;
#pragma unroll
        for (int t = 0; t < 16; ++t) {
            const float2 c = __ldg(cs + t);
            const float x0 = g[2 * t], x1 = g[2 * t + 1];
            g[2 * t] = fmaf(x0, c.x, x1 * c.y);
            g[2 * t + 1] = fmaf(-x0, c.y, x1 * c.x);
        }
    }
    uint4* d4 = reinterpret_cast<uint4*>(dst_row + c0);
#pragma unroll
    for (int k = 0; k < 4; ++k)
        d4[k] = make_uint4(ptx::pack_bf16x2(g[8 * k], g[8 * k + 1]), ptx::pack_bf16x2(g[8 * k + 2], g[8 * k + 3]),
                           ptx::pack_bf16x2(g[8 * k + 4], g[8 * k + 5]), ptx::pack_bf16x2(g[8 * k + 6], g[8 * k + 7]));
}

// Visible query tiles for the key tile starting at j0: [ib, ie).
__device__ __forceinline__ void query_tiles_for_keys(int j0, int N, int causal, int window, int& ib, int& ie) {
    const int nq = (N + 127) / 128;
    ib = causal ? j0 / 128 : 0;
    ie = nq;
    if (window > 0) ie = min(nq, (j0 + 127 + window - 1) / 128 + 1);
}

// TMEM column of the k-th 16-element slice of a packed bf16 operand: each group of elementwise
// warps packs its 32 columns of a 128-column fp32 buffer into the first 16 of them.
__device__ __forceinline__ constexpr uint32_t packed_col(int kk) { return (kk >> 1) * 32 + (kk & 1) * 8; }

// P = 2^(s * scale_log2 + nlse) for 32 consecutive fp32 scores, the (-LSE*log2 e) values given per
// query column (from shared memory).
__device__ __forceinline__ void probs32_cols(const uint32_t (&sv)[32], float scale_log2, const float* nlse,
                                             float (&pr)[32]) {
    const float2 sc = make_float2(scale_log2, scale_log2);
#pragma unroll
    for (int c = 0; c < 32; c += 4) {
        const float4 l4 = *reinterpret_cast<const float4*>(nlse + c);
        const float2 a = ptx::ffma2(make_float2(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), sc,
                                    make_float2(l4.x, l4.y));
        const float2 b = ptx::ffma2(make_float2(__uint_as_float(sv[c + 2]), __uint_as_float(sv[c + 3])), sc,
                                    make_float2(l4.z, l4.w));
        pr[c] = ptx::ex2(a.x);
        pr[c + 1] = ptx::ex2(a.y);
        pr[c + 2] = ptx::ex2(b.x);
        pr[c + 3] = ptx::ex2(b.y);
    }
}
// Zero the probabilities of columns outside [lo, hi] (column indices relative to the 32-column block).
__device__ __forceinline__ void mask32(float (&pr)[32], int lo, int hi) {
#pragma unroll
    for (int c = 0; c < 32; ++c) pr[c] = (c < lo || c > hi) ? 0.f : pr[c];
}
// dS = P (dP - D) for 32 columns, packed to 16 bf16 pairs; nd holds -D per column.
__device__ __forceinline__ void dscores32_cols(const float* pr, const uint32_t (&dp)[32], const float* nd,
                                               uint32_t* out) {
#pragma unroll
    for (int c = 0; c < 32; c += 4) {
        const float4 d4 = *reinterpret_cast<const float4*>(nd + c);
        const float2 a = ptx::fmul2(make_float2(pr[c], pr[c + 1]),
                                    ptx::fadd2(make_float2(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1])),
                                               make_float2(d4.x, d4.y)));
        const float2 b = ptx::fmul2(make_float2(pr[c + 2], pr[c + 3]),
                                    ptx::fadd2(make_float2(__uint_as_float(dp[c + 2]), __uint_as_float(dp[c + 3])),
                                               make_float2(d4.z, d4.w)));
        out[c / 2] = ptx::pack_bf16x2(a.x, a.y);
        out[c / 2 + 1] = ptx::pack_bf16x2(b.x, b.y);
    }
}

// A warp's 32 x 32 fp32 block (lane = row, 32 columns in registers) into 4 KB of shared memory:
// 128-byte rows, 16-byte chunk e of row r at position e ^ (r & 7), so the eight lanes of each
// store phase hit distinct banks.
// blk is the 32-bit shared address of a 1024-byte aligned block, so chunk e of row r sits at
// (blk + 128 r + 16 (r & 7)) ^ 16 e.
__device__ __forceinline__ void stage_rows32(uint32_t blk, const uint32_t (&v)[32], int lane) {
    const uint32_t row = blk + lane * 128 + ((lane & 7) << 4);
#pragma unroll
    for (int e = 0; e < 8; ++e) ptx::st_shared_v4(row ^ (e << 4), v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
}
// Shared address of the 32 x 32 fp32 box that stages dQ columns [32 cg, 32 cg + 32), rows
// [32 qw, 32 qw + 32) of a query tile: the first D / 64 column groups in the Q buffer of ring stage
// s, the rest in its dO buffer, 4 KB per box.
template <int D>
__device__ __forceinline__ uint32_t dq_box(int cg, int qw, const uint8_t* sQ, const uint8_t* sDO, int s) {
    constexpr int TILE = 128 * D * 2;
    return ptx::smem_u32(cg < D / 64 ? sQ : sDO) + s * TILE + ((cg % (D / 64)) * 4 + qw) * 4096;
}

// =============================================================================== dQ, dK, dV
// CTA (key tile jt, K/V head g, batch b); block numbers run over key tiles slowest, so the causal
// key tiles with the most visible queries start first. Steps t walk the visible query tiles from
// the last one down, and the query heads of the group for each: under a causal mask every key
// tile's walk starts at the same query tile, so the CTAs of one K/V head that run side by side read
// each Q and dO tile at about the same time, and the repeats come from L2.
//
// TMEM: S^T at 0 (P^T packed into the first 16 of every 32 columns), dP^T at 128, which takes the dQ
// partial of the step once dS^T has been formed, dV at 256, dK at 256 + D. Shared memory holds dS^T
// once per step (keys as 128-byte swizzled rows, queries along them); dK reads it K-major as
// dS^T and dQ reads the same bytes MN-major as dS. The dQ partial (128 x D fp32) leaves through the
// step's Q and dO buffers, which the tensor core is done with by then: each elementwise warp
// stages its 32 rows there as 32 x 32 fp32 boxes; a reduce warp has the TMA add them into the fp32
// sums and hands the stage back to the producer once the TMA has read it. That read takes about a
// step's worth of time under load, so no warp on the per-step chain waits for it.
//
// Issue order per step t: dV(t) once P^T(t) is written; dK(t) and dQ(t) once dS^T(t) is written;
// S^T(t+1); dP^T(t+1) once the dQ(t) partial has been read out of TMEM. MMAs of one thread run in
// issue order, so S^T(t+1) may overwrite the scores that P^T(t) was packed over once dV(t) is
// issued. The tensor core runs S^T(t+1) while the elementwise warps move dQ(t) out, and dV(t+1)
// while they form dS^T(t+1). The ring stage that S^T(t+1) reads is held by the dQ reduce of two
// steps back until the TMA has read it (about 64 KB at ~20 bytes per clock per SM under load), so
// issuing it earlier in the step gains nothing.
template <int D>
__global__ void __launch_bounds__(BwdCfg<D>::THREADS, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
    using C = BwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sK = smem;
    uint8_t* sV = sK + C::TILE_BYTES;
    uint8_t* sQ = sV + C::TILE_BYTES;          // [2] stages
    uint8_t* sDO = sQ + 2 * C::TILE_BYTES;     // [2] stages
    uint8_t* sDS = sDO + 2 * C::TILE_BYTES;    // dS^T, two 64-query regions
    float* sVec = reinterpret_cast<float*>(sDS + C::DS_BYTES);  // [2][256]
    auto* bar = reinterpret_cast<BwdBarriers*>(smem - smem_raw >= 128 ? smem_raw
                                                                      : reinterpret_cast<uint8_t*>(sVec) + 2 * C::VEC_BYTES);
    volatile int* abort_flag = &bar->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int groups = p.B * p.Hkv;
    const int jt = static_cast<int>(blockIdx.x / groups);
    const int gb = static_cast<int>(blockIdx.x - static_cast<unsigned>(jt) * groups);
    const int g = gb % p.Hkv, b = gb / p.Hkv;
    const int j0 = jt * 128;
    const int G = p.Hq / p.Hkv;
    int ib, ie;
    query_tiles_for_keys(j0, p.N, p.causal, p.window, ib, ie);
    const int per_head = max(0, ie - ib);
    const int T = G * per_head;  // steps

    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar->fixed_loaded, 1);
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(&bar->full[s], 1);
            ptx::mbar_init(&bar->empty[s], 1);  // the reduce warp, after the TMA has read the dQ staged there
            ptx::mbar_init(&bar->staged[s], C::EW_THREADS);
        }
        ptx::mbar_init(&bar->s_full, 1);
        ptx::mbar_init(&bar->dp_full, 1);
        ptx::mbar_init(&bar->p_full, C::EW_THREADS);
        ptx::mbar_init(&bar->ds_full, C::EW_THREADS);
        ptx::mbar_init(&bar->dq_full, 1);
        ptx::mbar_init(&bar->dq_free, C::EW_THREADS);
        ptx::mbar_init(&bar->acc_done, 1);
        ptx::mbar_init(&bar->drain, 1);
        bar->abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == C::MMA_WARP) {
        ptx::tmem_alloc(&bar->tmem_base, C::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = bar->tmem_base;
    constexpr uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_DK = 256 + D;

    if (warp == C::PRODUCER_WARP) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0 && T > 0) {
            const int zk = b * p.Hkv + g;
            ptx::mbar_arrive_expect_tx(&bar->fixed_loaded, 2 * C::TILE_BYTES);
            for (int r = 0; r < C::NREG; ++r) {
                ptx::tma_load_3d(sK + r * C::REGION_BYTES, &tm_k, &bar->fixed_loaded, r * 64, j0, zk);
                ptx::tma_load_3d(sV + r * C::REGION_BYTES, &tm_v, &bar->fixed_loaded, r * 64, j0, zk);
            }
            int issued = 0;
            bool ok = true;
            for (int t = 0; t < T && ok; ++t) {
                const int s = t & 1;
                if (t >= 2 && !ptx::mbar_wait(&bar->empty[s], ((t >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
                const int qt = ie - 1 - t / G, h = g * G + t % G;
                const int zq = b * p.Hq + h;
                ptx::mbar_arrive_expect_tx(&bar->full[s], 2 * C::TILE_BYTES + C::VEC_BYTES);
                if (!(p.debug_drop_copy && t == 0 && blockIdx.x == 0)) {
                    for (int r = 0; r < C::NREG; ++r) {
                        ptx::tma_load_3d(sQ + s * C::TILE_BYTES + r * C::REGION_BYTES, &tm_q, &bar->full[s], r * 64,
                                         qt * 128, zq);
                        ptx::tma_load_3d(sDO + s * C::TILE_BYTES + r * C::REGION_BYTES, &tm_do, &bar->full[s], r * 64,
                                         qt * 128, zq);
                    }
                    ptx::bulk_load(sVec + s * 256, p.vec + (static_cast<size_t>(zq) * p.ntiles + qt) * 256,
                                   C::VEC_BYTES, &bar->full[s]);
                }
                issued = t + 1;
            }
            if (!ok) {
                *abort_flag = 1;
                raise_status(kStatusTimeout);
                volatile int never = 0;
                ptx::mbar_wait(&bar->fixed_loaded, 0, &never);
                for (int t = max(0, issued - 2); t < issued; ++t) ptx::mbar_wait(&bar->full[t & 1], (t >> 1) & 1, &never);
            }
        }
    } else if (warp == C::MMA_WARP) {
        // ------------------------------------------------------------------ MMA issuer
        // The whole warp walks the steps and takes the waits, so operands stay warp-uniform; one
        // elected lane issues the tcgen05 instructions.
        if (T > 0) {
            const bool leader = ptx::elect_one();
            const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
            constexpr uint32_t ID_S = ptx::idesc_bf16_f32(128, 128, 0, 0);  // K Q^T, V dO^T: both K-major
            constexpr uint32_t ID_G = ptx::idesc_bf16_f32(128, D, 0, 1);    // P^T (TMEM) / dS^T x dO / Q (MN-major)
            constexpr uint32_t ID_Q = ptx::idesc_bf16_f32(128, D, 1, 1);    // dS x K, both MN-major
            constexpr uint32_t HI = ptx::sw128_desc_hi(1024);
            constexpr uint32_t TILE16 = C::TILE_BYTES >> 4;
            const uint32_t k_lo = ptx::sw128_desc_lo(ptx::smem_u32(sK), 16);
            const uint32_t v_lo = ptx::sw128_desc_lo(ptx::smem_u32(sV), 16);
            const uint32_t q_lo = ptx::sw128_desc_lo(ptx::smem_u32(sQ), 16);
            const uint32_t do_lo = ptx::sw128_desc_lo(ptx::smem_u32(sDO), 16);
            const uint32_t ds_lo = ptx::sw128_desc_lo(ptx::smem_u32(sDS), 16);
            const uint32_t qmn_lo = ptx::sw128_desc_lo(ptx::smem_u32(sQ), C::REGION_BYTES);
            const uint32_t domn_lo = ptx::sw128_desc_lo(ptx::smem_u32(sDO), C::REGION_BYTES);
            const uint32_t dsmn_lo = ptx::sw128_desc_lo(ptx::smem_u32(sDS), C::REGION_BYTES);
            const uint32_t kmn_lo = ptx::sw128_desc_lo(ptx::smem_u32(sK), C::REGION_BYTES);
            // K-major 16-element slice kk of a tile stored as 64-column regions of 128-byte rows
            auto kslice = [](int kk) -> uint32_t {
                return static_cast<uint32_t>(((kk >> 2) * C::REGION_BYTES + (kk & 3) * 32) >> 4);
            };
            // S^T = K Q^T (M = 128 keys, N = 128 queries, K = D)
            auto issue_s = [&](int t) {
                const uint32_t st = (t & 1) * TILE16;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    ptx::mma_ss(tm + T_S, ptx::desc64(k_lo + kslice(kk), HI), ptx::desc64(q_lo + st + kslice(kk), HI),
                                ID_S, kk > 0);
            };
            // dP^T = V dO^T
            auto issue_dp = [&](int t) {
                const uint32_t st = (t & 1) * TILE16;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    ptx::mma_ss(tm + T_DP, ptx::desc64(v_lo + kslice(kk), HI), ptx::desc64(do_lo + st + kslice(kk), HI),
                                ID_S, kk > 0);
            };
            // dV += P^T dO (M = 128 keys, N = D, K = 128 queries; P^T packed in TMEM)
            auto issue_dv = [&](int t) {
                const uint32_t st = (t & 1) * TILE16;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    ptx::mma_ts(tm + T_DV, tm + T_S + packed_col(kk), ptx::desc64(domn_lo + st + kk * 128, HI), ID_G,
                                (t > 0 || kk > 0) ? 1u : 0u);
            };
            // dK += dS^T Q (M = 128 keys, N = D, K = 128 queries)
            auto issue_dk = [&](int t) {
                const uint32_t st = (t & 1) * TILE16;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    ptx::mma_ss(tm + T_DK, ptx::desc64(ds_lo + kslice(kk), HI), ptx::desc64(qmn_lo + st + kk * 128, HI),
                                ID_G, (t > 0 || kk > 0) ? 1u : 0u);
            };
            // dQ partial = dS K (M = 128 queries, N = D, K = 128 keys), into the dP^T columns
            auto issue_dq = [&]() {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    ptx::mma_ss(tm + T_DP, ptx::desc64(dsmn_lo + kk * 128, HI), ptx::desc64(kmn_lo + kk * 128, HI), ID_Q,
                                kk > 0);
            };
            bool ok = ptx::mbar_wait_warp(&bar->fixed_loaded, 0, abort_flag) &&
                      ptx::mbar_wait_warp(&bar->full[0], 0, abort_flag);
            bool issued_any = false;
            if (ok) {
                if (leader) {
                    issue_s(0);
                    ptx::mma_commit(&bar->s_full);
                    issue_dp(0);
                    ptx::mma_commit(&bar->dp_full);
                }
                __syncwarp();
                issued_any = true;
            }
            for (int t = 0; ok && t < T; ++t) {
                if (!ptx::mbar_wait_warp(&bar->p_full, t & 1, abort_flag)) { ok = false; break; }
                ptx::tc_fence_after();
                if (leader) issue_dv(t);
                __syncwarp();
                if (!ptx::mbar_wait_warp(&bar->ds_full, t & 1, abort_flag)) { ok = false; break; }
                ptx::tc_fence_after();
                if (leader) {
                    issue_dk(t);
                    issue_dq();
                    ptx::mma_commit(&bar->dq_full);
                    if (t + 1 == T) ptx::mma_commit(&bar->acc_done);
                }
                __syncwarp();
                if (t + 1 < T) {
                    if (!ptx::mbar_wait_warp(&bar->full[(t + 1) & 1], ((t + 1) >> 1) & 1, abort_flag)) { ok = false; break; }
                    if (leader) {
                        issue_s(t + 1);
                        ptx::mma_commit(&bar->s_full);
                    }
                    __syncwarp();
                    if (!ptx::mbar_wait_warp(&bar->dq_free, t & 1, abort_flag)) { ok = false; break; }
                    ptx::tc_fence_after();
                    if (leader) {
                        issue_dp(t + 1);
                        ptx::mma_commit(&bar->dp_full);
                    }
                    __syncwarp();
                }
            }
            if (!ok && leader) {
                *abort_flag = 1;
                raise_status(kStatusTimeout);
                if (issued_any) {
                    ptx::mma_commit(&bar->drain);
                    volatile int never = 0;
                    ptx::mbar_wait(&bar->drain, 0, &never);
                }
            }
        }
        __syncwarp();
    } else if (warp == C::REDUCE_WARP) {
        // ------------------------------------------------------------------ dQ reduce
        // Per step: the TMA adds the staged boxes into the fp32 sums; once it has read them the
        // stage goes back to the producer. The additions complete before the CTA exits.
        if (lane == 0 && T > 0) {
            bool ok = true;
            for (int t = 0; t < T; ++t) {
                const int s = t & 1;
                const int qt = ie - 1 - t / G, h = g * G + t % G;
                if (!ptx::mbar_wait(&bar->staged[s], (t >> 1) & 1, abort_flag)) { ok = false; break; }
                const int row0 = ((b * p.Hq + h) * p.ntiles + qt) * 128;
#pragma unroll 1
                for (int cg = 0; cg < D / 32; ++cg)
#pragma unroll
                    for (int qw = 0; qw < 4; ++qw)
                        ptx::tma_reduce_add_2d(&tm_dq, dq_box<D>(cg, qw, sQ, sDO, s), 32 * cg, row0 + 32 * qw);
                ptx::bulk_commit_group();
                ptx::bulk_wait_read<0>();
                ptx::mbar_arrive(&bar->empty[s]);
            }
            ptx::bulk_wait_all();
            if (!ok) {
                *abort_flag = 1;
                raise_status(kStatusTimeout);
            }
        }
    } else {
        // ------------------------------------------------------------------ elementwise warps
        const int cg = warp >> 2;                  // query columns [32 cg, 32 cg + 32) of each tile
        const int r = (warp & 3) * 32 + lane;      // TMEM lane: key row of S^T, dP^T; query row of dQ
        const int key = j0 + r;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t t_s = tmem + lane_base + T_S + 32 * cg, t_dp = tmem + lane_base + T_DP + 32 * cg;
        // this thread's dS^T row, queries [32 cg, 32 cg + 32): 128-byte row r of region cg / 2,
        // 16-byte chunks 4 (cg & 1) + c stored at (4 (cg & 1) + c) ^ (r & 7)
        const uint32_t ds_row = ptx::smem_u32(sDS) + (cg >> 1) * C::REGION_BYTES + r * 128;
        bool ok = true;
        for (int t = 0; ok && t < T; ++t) {
            const int s = t & 1;
            const int qt = ie - 1 - t / G;
            const int c0 = qt * 128 + 32 * cg;  // first query of this group's columns
            if (!ptx::mbar_wait(&bar->full[s], (t >> 1) & 1, abort_flag)) { ok = false; break; }
            if (!ptx::mbar_wait(&bar->s_full, t & 1, abort_flag)) { ok = false; break; }
            ptx::tc_fence_after();
            const float* vec = sVec + s * 256 + 32 * cg;
            float pr[32];
            {
                uint32_t sv[32];
                ptx::tmem_ld32(t_s, sv);
                probs32_cols(sv, p.scale_log2, vec, pr);
            }
            // query qpos sees this key iff qpos >= key (causal) and qpos - key < window
            const int lo = p.causal ? key - c0 : -1;
            const int hi = p.window > 0 ? key + p.window - 1 - c0 : 32;
            if (lo > 0 || hi < 31) mask32(pr, lo, hi);
            {
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 16; ++c) pk[c] = ptx::pack_bf16x2(pr[2 * c], pr[2 * c + 1]);
                ptx::tmem_st16(t_s, pk);
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&bar->p_full);
            if (!ptx::mbar_wait(&bar->dp_full, t & 1, abort_flag)) { ok = false; break; }
            ptx::tc_fence_after();
            {
                uint32_t dp[32], dsk[16];
                ptx::tmem_ld32(t_dp, dp);
                dscores32_cols(pr, dp, vec + 128, dsk);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    ptx::st_shared_v4(ds_row + ((((cg & 1) * 4 + c) ^ (r & 7)) << 4), dsk[4 * c], dsk[4 * c + 1],
                                      dsk[4 * c + 2], dsk[4 * c + 3]);
            }
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            ptx::mbar_arrive(&bar->ds_full);
            // dQ partial of this step: query row qt * 128 + r, columns [32 cg, 32 cg + 32) for the
            // first D / 32 groups, staged as one 32 x 32 box in the step's Q or dO buffer; the TMEM
            // columns are released as soon as it is in registers
            if (!ptx::mbar_wait(&bar->dq_full, t & 1, abort_flag)) { ok = false; break; }
            ptx::tc_fence_after();
            if (cg < D / 32) {
                uint32_t v[32];
                ptx::tmem_ld32(tmem + lane_base + T_DP + 32 * cg, v);
                ptx::tc_fence_before();
                ptx::mbar_arrive(&bar->dq_free);
                stage_rows32(dq_box<D>(cg, warp & 3, sQ, sDO, s), v, lane);
            } else {
                ptx::mbar_arrive(&bar->dq_free);
            }
            ptx::fence_proxy_async_smem();
            ptx::mbar_arrive(&bar->staged[s]);
        }
        // groups 0 and 1 write dV columns [0, D/2) and [D/2, D), groups 2 and 3 dK likewise
        const bool is_k = cg >= 2;
        const int col0 = (cg & 1) * (D / 2);
        if (ok && T > 0) ok = ptx::mbar_wait(&bar->acc_done, 0, abort_flag);
        if (ok && T > 0) {
            // every lane takes part in the warp-collective TMEM loads; rows past N store nothing
            ptx::tc_fence_after();
            const size_t row = (static_cast<size_t>(b) * p.Hkv + g) * p.N + min(key, p.N - 1);
#pragma unroll 1
            for (int c = 0; c < D / 64; ++c) {
                uint32_t v[32];
                ptx::tmem_ld32(tmem + lane_base + (is_k ? T_DK : T_DV) + col0 + c * 32, v);
                if (key < p.N) {
                    if (is_k)
                        store_chunk_unrotated(v, p.scale, p.rope, D, key, col0 + c * 32, p.dk + row * D);
                    else
                        store_chunk_unrotated(v, 1.f, nullptr, D, key, col0 + c * 32, p.dv + row * D);
                }
            }
        } else if (T == 0 && key < p.N) {
            // no query sees these keys: zero gradients
            const size_t row = (static_cast<size_t>(b) * p.Hkv + g) * p.N + key;
            uint4* d1 = reinterpret_cast<uint4*>((is_k ? p.dk : p.dv) + row * D + col0);
            for (int k = 0; k < D / 16; ++k) d1[k] = make_uint4(0, 0, 0, 0);
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

// dq = scale * (the fp32 sums) rotated back by -angle (RoPE), stored bf16. Eight columns per
// thread (one 16-byte store), grid-stride over the B * Hq * N rows.
template <int D>
__global__ void __launch_bounds__(256) bwd_dq_store_kernel(const BwdParams p) {
    constexpr int CPR = D / 8;  // threads per row
    const long long total = static_cast<long long>(p.B) * p.Hq * p.N * CPR;
    const size_t npad = static_cast<size_t>(p.ntiles) * 128;
    for (long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
         idx += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long row = idx / CPR;
        const int c0 = static_cast<int>(idx - row * CPR) * 8;
        const long long bh = row / p.N;
        const int i = static_cast<int>(row - bh * p.N);
        const float4* src = reinterpret_cast<const float4*>(p.dqacc + (static_cast<size_t>(bh) * npad + i) * D + c0);
        const float4 a = src[0], c = src[1];
        float g[8] = {a.x * p.scale, a.y * p.scale, a.z * p.scale, a.w * p.scale,
                      c.x * p.scale, c.y * p.scale, c.z * p.scale, c.w * p.scale};
        if (p.rope != nullptr) {
            const float2* cs = p.rope + static_cast<size_t>(i) * (D / 2) + c0 / 2;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const float2 r = __ldg(cs + t);
                const float x0 = g[2 * t], x1 = g[2 * t + 1];
                g[2 * t] = fmaf(x0, r.x, x1 * r.y);
                g[2 * t + 1] = fmaf(-x0, r.y, x1 * r.x);
            }
        }
        *reinterpret_cast<uint4*>(p.dq + static_cast<size_t>(row) * D + c0) =
            make_uint4(ptx::pack_bf16x2(g[0], g[1]), ptx::pack_bf16x2(g[2], g[3]), ptx::pack_bf16x2(g[4], g[5]),
                       ptx::pack_bf16x2(g[6], g[7]));
    }
}

}  // namespace attn
