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
// Three kernels: a prep pass (D_i and the log2-scaled LSE, padded per 128-row tile), a dK/dV
// kernel with one CTA per (128-key tile, K/V head) that walks every query head of the group and
// every query tile that sees the keys, and a dQ kernel with one CTA per (128-query tile, query
// head) that walks the visible key tiles. All five products per tile pair run on tcgen05 with
// fp32 accumulators in Tensor Memory. Eight elementwise warps (two warpgroups, each owning 64 of
// the 128 columns of a tile) turn scores into P and dS; the products are issued in an order that
// lets the tensor core work on the next tile while they do (see each kernel's issue loop).
// CTAs are numbered so that the ones with the most work start first.
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
    __nv_bfloat16* dk;          // [B, Hkv, N, D]
    __nv_bfloat16* dv;          // [B, Hkv, N, D]
    const float2* rope;         // (cos, sin) table or nullptr
    int B, Hq, Hkv, N, ntiles;
    int causal, window;
    float scale, scale_log2;
};

// Per query row: -D_i = -(dO_i . O_i) and -LSE_i * log2(e), stored negated so that the kernels add
// them. D/8 lanes share a row (16-byte loads), grid-stride over all padded rows; rows past N get
// (-inf, 0) so that their recomputed probabilities are exactly 0.
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
    static constexpr int VEC_BYTES = 256 * 4;  // -LSE*log2 e and -D of the 128 rows of a query tile
    // fixed pair (K,V or Q,dO) + two stages of the streamed pair, with their vectors
    static constexpr int SMEM_BYTES = 6 * TILE_BYTES + 2 * VEC_BYTES + 1024 /*barriers*/ + 1024 /*align*/;
    static constexpr int THREADS = 320;  // warps 0-7 elementwise, 8 TMA producer, 9 MMA issuer
    static constexpr int PRODUCER_WARP = 8, MMA_WARP = 9;
    static constexpr int EW_THREADS = 256;
    static constexpr uint32_t TMEM_COLS = 512;
};

struct BwdBarriers {
    uint64_t fixed_loaded;
    uint64_t full[2], empty[2];
    uint64_t s_full[2], dp_full, p_full, ds_full, acc_done, drain;
    uint32_t tmem_base;
    int abort;
};

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

// TMEM column of the k-th 16-element slice of a packed bf16 operand: each warpgroup packs its 64
// columns of a 128-column fp32 buffer into the first 32 columns of its own half.
__device__ __forceinline__ constexpr uint32_t packed_col(int kk) { return (kk >> 2) * 64 + (kk & 3) * 8; }

// P = 2^(s * scale_log2 + nlse) for 64 consecutive fp32 scores, the (-LSE*log2 e) values given per
// element (dK/dV: per query column, from shared memory) or as one value (dQ: per row).
__device__ __forceinline__ void probs64_cols(const uint32_t (&sv)[64], float scale_log2, const float* nlse,
                                             float (&pr)[64]) {
    const float2 sc = make_float2(scale_log2, scale_log2);
#pragma unroll
    for (int c = 0; c < 64; c += 4) {
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
__device__ __forceinline__ void probs64_row(const uint32_t (&sv)[64], float scale_log2, float nlse,
                                            float (&pr)[64]) {
    const float2 sc = make_float2(scale_log2, scale_log2), nl = make_float2(nlse, nlse);
#pragma unroll
    for (int c = 0; c < 64; c += 2) {
        const float2 a = ptx::ffma2(make_float2(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), sc, nl);
        pr[c] = ptx::ex2(a.x);
        pr[c + 1] = ptx::ex2(a.y);
    }
}
// Zero the probabilities of columns outside [lo, hi] (column indices relative to the 64-column block).
__device__ __forceinline__ void mask64(float (&pr)[64], int lo, int hi) {
#pragma unroll
    for (int c = 0; c < 64; ++c) pr[c] = (c < lo || c > hi) ? 0.f : pr[c];
}
// dS = P (dP - D) for 32 columns, packed to 16 bf16 pairs. nd: -D per element (pointer) or per row.
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
__device__ __forceinline__ void dscores32_row(const float* pr, const uint32_t (&dp)[32], float nd, uint32_t* out) {
    const float2 n2 = make_float2(nd, nd);
#pragma unroll
    for (int c = 0; c < 32; c += 2) {
        const float2 a = ptx::fmul2(make_float2(pr[c], pr[c + 1]),
                                    ptx::fadd2(make_float2(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1])), n2));
        out[c / 2] = ptx::pack_bf16x2(a.x, a.y);
    }
}

// =============================================================================== dK, dV
// CTA (key tile jt, K/V head g, batch b); block numbers run over key tiles slowest, so the causal
// key tiles with the most visible queries start first. Steps t walk the visible query tiles from
// the last one down, and the query heads of the group for each: under a causal mask every key
// tile's walk starts at the same query tile, so the CTAs of one K/V head that run side by side read
// each Q and dO tile at about the same time, and the repeats come from L2. TMEM: S^T at 0 (P^T packed into columns 0-31 and 64-95), dP^T at 128 (dS^T
// packed likewise), dV at 256, dK at 256 + D.
//
// Issue order per step t: dV(t) once P^T(t) is written, S^T(t+1), dK(t) once dS^T(t) is written,
// dP^T(t+1). MMAs of one thread run in issue order, so S^T(t+1) may overwrite the scores that P^T(t)
// was packed over once dV(t) is issued, and dP^T(t+1) the dS^T(t) buffer once dK(t) is issued; the
// elementwise warps compute P^T(t+1) while the tensor core runs dK(t) and dP^T(t+1), and dS^T(t)
// while it runs dV(t) and S^T(t+1).
template <int D>
__global__ void __launch_bounds__(BwdCfg<D>::THREADS, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                         const BwdParams p) {
    using C = BwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sK = smem;
    uint8_t* sV = sK + C::TILE_BYTES;
    uint8_t* sQ = sV + C::TILE_BYTES;          // [2] stages
    uint8_t* sDO = sQ + 2 * C::TILE_BYTES;     // [2] stages
    float* sVec = reinterpret_cast<float*>(sDO + 2 * C::TILE_BYTES);  // [2][256]
    auto* bar = reinterpret_cast<BwdBarriers*>(reinterpret_cast<uint8_t*>(sVec) + 2 * C::VEC_BYTES);
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
            ptx::mbar_init(&bar->empty[s], 1);
            ptx::mbar_init(&bar->s_full[s], 1);
        }
        ptx::mbar_init(&bar->dp_full, 1);
        ptx::mbar_init(&bar->p_full, C::EW_THREADS);
        ptx::mbar_init(&bar->ds_full, C::EW_THREADS);
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
                for (int r = 0; r < C::NREG; ++r) {
                    ptx::tma_load_3d(sQ + s * C::TILE_BYTES + r * C::REGION_BYTES, &tm_q, &bar->full[s], r * 64,
                                     qt * 128, zq);
                    ptx::tma_load_3d(sDO + s * C::TILE_BYTES + r * C::REGION_BYTES, &tm_do, &bar->full[s], r * 64,
                                     qt * 128, zq);
                }
                ptx::bulk_load(sVec + s * 256, p.vec + (static_cast<size_t>(zq) * p.ntiles + qt) * 256, C::VEC_BYTES,
                               &bar->full[s]);
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
            constexpr uint32_t ID_S = ptx::idesc_bf16_f32(128, 128, 0, 0);  // K (keys) x Q^T, both K-major
            constexpr uint32_t ID_G = ptx::idesc_bf16_f32(128, D, 0, 1);    // P^T/dS^T (TMEM) x dO/Q (MN-major)
            constexpr uint32_t HI = ptx::sw128_desc_hi(1024);
            constexpr uint32_t TILE16 = C::TILE_BYTES >> 4;
            const uint32_t k_lo = ptx::sw128_desc_lo(ptx::smem_u32(sK), 16);
            const uint32_t v_lo = ptx::sw128_desc_lo(ptx::smem_u32(sV), 16);
            const uint32_t q_lo = ptx::sw128_desc_lo(ptx::smem_u32(sQ), 16);
            const uint32_t do_lo = ptx::sw128_desc_lo(ptx::smem_u32(sDO), 16);
            const uint32_t qmn_lo = ptx::sw128_desc_lo(ptx::smem_u32(sQ), C::REGION_BYTES);
            const uint32_t domn_lo = ptx::sw128_desc_lo(ptx::smem_u32(sDO), C::REGION_BYTES);
            // S^T = K Q^T (M = 128 keys, N = 128 queries, K = D)
            auto issue_s = [&](int t) {
                const uint32_t st = (t & 1) * TILE16;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * C::REGION_BYTES + (kk & 3) * 32) >> 4;
                    ptx::mma_ss(tm + T_S, ptx::desc64(k_lo + off, HI), ptx::desc64(q_lo + st + off, HI), ID_S, kk > 0);
                }
            };
            // dP^T = V dO^T
            auto issue_dp = [&](int t) {
                const uint32_t st = (t & 1) * TILE16;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * C::REGION_BYTES + (kk & 3) * 32) >> 4;
                    ptx::mma_ss(tm + T_DP, ptx::desc64(v_lo + off, HI), ptx::desc64(do_lo + st + off, HI), ID_S, kk > 0);
                }
            };
            // dV += P^T dO, dK += dS^T Q (M = 128 keys, N = D, K = 128 queries)
            auto issue_grad = [&](int t, uint32_t acc_col, uint32_t a_col, uint32_t b_lo) {
                const uint32_t st = (t & 1) * TILE16;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    ptx::mma_ts(tm + acc_col, tm + a_col + packed_col(kk), ptx::desc64(b_lo + st + ((kk * 2048) >> 4), HI),
                                ID_G, (t > 0 || kk > 0) ? 1u : 0u);
            };
            bool ok = ptx::mbar_wait_warp(&bar->fixed_loaded, 0, abort_flag) &&
                      ptx::mbar_wait_warp(&bar->full[0], 0, abort_flag);
            bool issued_any = false;
            if (ok) {
                if (leader) {
                    issue_s(0);
                    ptx::mma_commit(&bar->s_full[0]);
                    issue_dp(0);
                    ptx::mma_commit(&bar->dp_full);
                }
                __syncwarp();
                issued_any = true;
            }
            for (int t = 0; ok && t < T; ++t) {
                if (!ptx::mbar_wait_warp(&bar->p_full, t & 1, abort_flag)) { ok = false; break; }
                ptx::tc_fence_after();
                if (leader) issue_grad(t, T_DV, T_S, domn_lo);
                __syncwarp();
                if (t + 1 < T) {
                    if (!ptx::mbar_wait_warp(&bar->full[(t + 1) & 1], ((t + 1) >> 1) & 1, abort_flag)) { ok = false; break; }
                    if (leader) {
                        issue_s(t + 1);
                        ptx::mma_commit(&bar->s_full[0]);
                    }
                    __syncwarp();
                }
                if (!ptx::mbar_wait_warp(&bar->ds_full, t & 1, abort_flag)) { ok = false; break; }
                ptx::tc_fence_after();
                if (leader) {
                    issue_grad(t, T_DK, T_DP, qmn_lo);
                    ptx::mma_commit(&bar->empty[t & 1]);
                    if (t + 1 < T) {
                        issue_dp(t + 1);
                        ptx::mma_commit(&bar->dp_full);
                    } else {
                        ptx::mma_commit(&bar->acc_done);
                    }
                }
                __syncwarp();
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
    } else {
        // ------------------------------------------------------------------ elementwise warps
        const int wg = warp >> 2;                  // query columns [64 wg, 64 wg + 64) of each tile
        const int r = (warp & 3) * 32 + lane;      // key row == TMEM lane
        const int key = j0 + r;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t t_s = tmem + lane_base + T_S + 64 * wg, t_dp = tmem + lane_base + T_DP + 64 * wg;
        bool ok = true;
        for (int t = 0; ok && t < T; ++t) {
            const int s = t & 1;
            const int c0 = (ie - 1 - t / G) * 128 + 64 * wg;  // first query of this warpgroup's columns
            if (!ptx::mbar_wait(&bar->full[s], (t >> 1) & 1, abort_flag)) { ok = false; break; }
            if (!ptx::mbar_wait(&bar->s_full[0], t & 1, abort_flag)) { ok = false; break; }
            ptx::tc_fence_after();
            const float* vec = sVec + s * 256 + 64 * wg;
            float pr[64];
            {
                uint32_t sv[64];
                ptx::tmem_ld64(t_s, sv);
                probs64_cols(sv, p.scale_log2, vec, pr);
            }
            // query qpos sees this key iff qpos >= key (causal) and qpos - key < window
            const int lo = p.causal ? key - c0 : -1;
            const int hi = p.window > 0 ? key + p.window - 1 - c0 : 64;
            if (lo > 0 || hi < 63) mask64(pr, lo, hi);
            {
                uint32_t pk[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) pk[c] = ptx::pack_bf16x2(pr[2 * c], pr[2 * c + 1]);
                ptx::tmem_st32(t_s, pk);
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&bar->p_full);
            if (!ptx::mbar_wait(&bar->dp_full, t & 1, abort_flag)) { ok = false; break; }
            ptx::tc_fence_after();
            uint32_t dsk[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t dp[32];
                ptx::tmem_ld32(t_dp + 32 * half, dp);
                dscores32_cols(pr + 32 * half, dp, vec + 128 + 32 * half, dsk + 16 * half);
            }
            ptx::tmem_st32(t_dp, dsk);
            ptx::tc_fence_before();
            ptx::mbar_arrive(&bar->ds_full);
        }
        if (ok && T > 0) ok = ptx::mbar_wait(&bar->acc_done, 0, abort_flag);
        if (ok && T > 0) {
            // warpgroup 0 writes dV, warpgroup 1 dK; every lane takes part in the warp-collective
            // TMEM loads, rows past N store nothing
            ptx::tc_fence_after();
            const size_t row = (static_cast<size_t>(b) * p.Hkv + g) * p.N + min(key, p.N - 1);
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t v[32];
                ptx::tmem_ld32(tmem + lane_base + (wg == 0 ? T_DV : T_DK) + c * 32, v);
                if (key < p.N) {
                    if (wg == 0)
                        store_chunk_unrotated(v, 1.f, nullptr, D, key, c * 32, p.dv + row * D);
                    else
                        store_chunk_unrotated(v, p.scale, p.rope, D, key, c * 32, p.dk + row * D);
                }
            }
        } else if (T == 0 && key < p.N) {
            // no query sees these keys: zero gradients
            const size_t row = (static_cast<size_t>(b) * p.Hkv + g) * p.N + key;
            uint4* d1 = reinterpret_cast<uint4*>((wg == 0 ? p.dv : p.dk) + row * D);
            for (int k = 0; k < D / 8; ++k) d1[k] = make_uint4(0, 0, 0, 0);
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

// =============================================================================== dQ
// CTA (query tile it, query head h, batch b); block numbers run over query tiles slowest, the last
// (causal: longest) tiles first. Steps walk the visible key tiles. TMEM: S in two buffers at 0 and
// 128, dP at 256 (dS packed into columns 256-287 and 320-351), dQ at 384.
//
// Issue order per step t: S(t+1) into the other buffer, dQ(t) once dS(t) is written, dP(t+1). P
// stays in registers, so the elementwise warps compute P(t+1) while the tensor core runs dQ(t) and
// dP(t+1).
template <int D>
__global__ void __launch_bounds__(BwdCfg<D>::THREADS, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                       const BwdParams p) {
    using C = BwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;
    uint8_t* sDO = sQ + C::TILE_BYTES;
    uint8_t* sK = sDO + C::TILE_BYTES;        // [2] stages
    uint8_t* sV = sK + 2 * C::TILE_BYTES;     // [2] stages
    auto* bar = reinterpret_cast<BwdBarriers*>(sV + 2 * C::TILE_BYTES + 2 * C::VEC_BYTES);
    volatile int* abort_flag = &bar->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int groups = p.B * p.Hq;
    const int rank = static_cast<int>(blockIdx.x / groups);
    const int hb = static_cast<int>(blockIdx.x - static_cast<unsigned>(rank) * groups);
    const int h = hb % p.Hq, b = hb / p.Hq;
    const int qt = p.ntiles - 1 - rank;
    const int q0 = qt * 128;
    const int g = h / (p.Hq / p.Hkv);
    const TileRange R = tile_range(q0, p.N, p.causal, p.window);
    const int T = R.n;

    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar->fixed_loaded, 1);
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(&bar->full[s], 1);
            ptx::mbar_init(&bar->empty[s], 1);
            ptx::mbar_init(&bar->s_full[s], 1);
        }
        ptx::mbar_init(&bar->dp_full, 1);
        ptx::mbar_init(&bar->p_full, 1);
        ptx::mbar_init(&bar->ds_full, C::EW_THREADS);
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
    constexpr uint32_t T_S = 0, T_DP = 256, T_DQ = 384;

    if (warp == C::PRODUCER_WARP) {
        if (lane == 0 && T > 0) {
            const int zq = b * p.Hq + h, zk = b * p.Hkv + g;
            ptx::mbar_arrive_expect_tx(&bar->fixed_loaded, 2 * C::TILE_BYTES);
            for (int r = 0; r < C::NREG; ++r) {
                ptx::tma_load_3d(sQ + r * C::REGION_BYTES, &tm_q, &bar->fixed_loaded, r * 64, q0, zq);
                ptx::tma_load_3d(sDO + r * C::REGION_BYTES, &tm_do, &bar->fixed_loaded, r * 64, q0, zq);
            }
            int issued = 0;
            bool ok = true;
            for (int t = 0; t < T && ok; ++t) {
                const int s = t & 1;
                if (t >= 2 && !ptx::mbar_wait(&bar->empty[s], ((t >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
                const int k0 = (R.jb + t) * 128;
                ptx::mbar_arrive_expect_tx(&bar->full[s], 2 * C::TILE_BYTES);
                for (int r = 0; r < C::NREG; ++r) {
                    ptx::tma_load_3d(sK + s * C::TILE_BYTES + r * C::REGION_BYTES, &tm_k, &bar->full[s], r * 64, k0, zk);
                    ptx::tma_load_3d(sV + s * C::TILE_BYTES + r * C::REGION_BYTES, &tm_v, &bar->full[s], r * 64, k0, zk);
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
        // The whole warp walks the steps and takes the waits; one elected lane issues.
        if (T > 0) {
            const bool leader = ptx::elect_one();
            const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
            constexpr uint32_t ID_S = ptx::idesc_bf16_f32(128, 128, 0, 0);  // Q K^T, dO V^T: K-major
            constexpr uint32_t ID_G = ptx::idesc_bf16_f32(128, D, 0, 1);    // dS (TMEM) x K (MN-major)
            constexpr uint32_t HI = ptx::sw128_desc_hi(1024);
            constexpr uint32_t TILE16 = C::TILE_BYTES >> 4;
            const uint32_t q_lo = ptx::sw128_desc_lo(ptx::smem_u32(sQ), 16);
            const uint32_t do_lo = ptx::sw128_desc_lo(ptx::smem_u32(sDO), 16);
            const uint32_t k_lo = ptx::sw128_desc_lo(ptx::smem_u32(sK), 16);
            const uint32_t v_lo = ptx::sw128_desc_lo(ptx::smem_u32(sV), 16);
            const uint32_t kmn_lo = ptx::sw128_desc_lo(ptx::smem_u32(sK), C::REGION_BYTES);
            // S = Q K^T into buffer t & 1 (M = 128 queries, N = 128 keys, K = D)
            auto issue_s = [&](int t) {
                const uint32_t st = (t & 1) * TILE16;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * C::REGION_BYTES + (kk & 3) * 32) >> 4;
                    ptx::mma_ss(tm + T_S + 128 * (t & 1), ptx::desc64(q_lo + off, HI), ptx::desc64(k_lo + st + off, HI),
                                ID_S, kk > 0);
                }
            };
            // dP = dO V^T
            auto issue_dp = [&](int t) {
                const uint32_t st = (t & 1) * TILE16;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * C::REGION_BYTES + (kk & 3) * 32) >> 4;
                    ptx::mma_ss(tm + T_DP, ptx::desc64(do_lo + off, HI), ptx::desc64(v_lo + st + off, HI), ID_S, kk > 0);
                }
            };
            bool ok = ptx::mbar_wait_warp(&bar->fixed_loaded, 0, abort_flag) &&
                      ptx::mbar_wait_warp(&bar->full[0], 0, abort_flag);
            bool issued_any = false;
            if (ok) {
                if (leader) {
                    issue_s(0);
                    ptx::mma_commit(&bar->s_full[0]);
                    issue_dp(0);
                    ptx::mma_commit(&bar->dp_full);
                }
                __syncwarp();
                issued_any = true;
            }
            for (int t = 0; ok && t < T; ++t) {
                if (t + 1 < T) {
                    if (!ptx::mbar_wait_warp(&bar->full[(t + 1) & 1], ((t + 1) >> 1) & 1, abort_flag)) { ok = false; break; }
                    if (leader) {
                        issue_s(t + 1);
                        ptx::mma_commit(&bar->s_full[(t + 1) & 1]);
                    }
                    __syncwarp();
                }
                if (!ptx::mbar_wait_warp(&bar->ds_full, t & 1, abort_flag)) { ok = false; break; }
                ptx::tc_fence_after();
                if (leader) {
                    // dQ += dS K (M = 128 queries, N = D, K = 128 keys)
                    const uint32_t st = (t & 1) * TILE16;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        ptx::mma_ts(tm + T_DQ, tm + T_DP + packed_col(kk),
                                    ptx::desc64(kmn_lo + st + ((kk * 2048) >> 4), HI), ID_G, (t > 0 || kk > 0) ? 1u : 0u);
                    ptx::mma_commit(&bar->empty[t & 1]);
                    if (t + 1 < T) {
                        issue_dp(t + 1);
                        ptx::mma_commit(&bar->dp_full);
                    } else {
                        ptx::mma_commit(&bar->acc_done);
                    }
                }
                __syncwarp();
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
    } else {
        const int wg = warp >> 2;              // key columns [64 wg, 64 wg + 64) of each tile
        const int r = (warp & 3) * 32 + lane;  // query row == TMEM lane
        const int qpos = q0 + r;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t t_dp = tmem + lane_base + T_DP + 64 * wg;
        const float* vrow = p.vec + (static_cast<size_t>(b * p.Hq + h) * p.ntiles + qt) * 256 + r;
        const float nlse = vrow[0], nd = vrow[128];
        bool ok = true;
        for (int t = 0; ok && t < T; ++t) {
            const int c0 = (R.jb + t) * 128 + 64 * wg;  // first key of this warpgroup's columns
            if (!ptx::mbar_wait(&bar->s_full[t & 1], (t >> 1) & 1, abort_flag)) { ok = false; break; }
            ptx::tc_fence_after();
            float pr[64];
            {
                uint32_t sv[64];
                ptx::tmem_ld64(tmem + lane_base + T_S + 128 * (t & 1) + 64 * wg, sv);
                probs64_row(sv, p.scale_log2, nlse, pr);
            }
            // key kpos is visible iff kpos <= qpos (causal) and qpos - kpos < window; keys past N
            // have zero K and V rows (zero-filled loads), so their dS meets a zero K row
            const int hi = p.causal ? qpos - c0 : 64;
            const int lo = p.window > 0 ? qpos - p.window + 1 - c0 : -1;
            if (lo > 0 || hi < 63) mask64(pr, lo, hi);
            if (!ptx::mbar_wait(&bar->dp_full, t & 1, abort_flag)) { ok = false; break; }
            ptx::tc_fence_after();
            uint32_t dsk[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t dp[32];
                ptx::tmem_ld32(t_dp + 32 * half, dp);
                dscores32_row(pr + 32 * half, dp, nd, dsk + 16 * half);
            }
            ptx::tmem_st32(t_dp, dsk);
            ptx::tc_fence_before();
            ptx::mbar_arrive(&bar->ds_full);
        }
        if (ok && T > 0) ok = ptx::mbar_wait(&bar->acc_done, 0, abort_flag);
        if (ok && T > 0) {
            // each warpgroup writes half of the D columns
            ptx::tc_fence_after();
            __nv_bfloat16* dst = p.dq + ((static_cast<size_t>(b) * p.Hq + h) * p.N + min(qpos, p.N - 1)) * D;
#pragma unroll 1
            for (int c = wg * (D / 64); c < (wg + 1) * (D / 64); ++c) {
                uint32_t v[32];
                ptx::tmem_ld32(tmem + lane_base + T_DQ + c * 32, v);
                if (qpos < p.N) store_chunk_unrotated(v, p.scale, p.rope, D, qpos, c * 32, dst);
            }
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
