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
// fp32 accumulators in Tensor Memory; the elementwise step runs one row per thread.
#pragma once
#include "common.cuh"
#include "fwd_sm100.cuh"
#include "ptx.cuh"

namespace attn {

struct BwdParams {
    const __nv_bfloat16* o;     // [B, Hq, N, D] forward output
    const __nv_bfloat16* dout;  // [B, Hq, N, D]
    const float* lse;           // [B, Hq, N] forward logsumexp (natural log)
    float* vec;                 // [B*Hq, Npad, 2]: (LSE * log2 e, D_i); rows >= N hold (+inf, 0)
    __nv_bfloat16* dq;          // [B, Hq, N, D]
    __nv_bfloat16* dk;          // [B, Hkv, N, D]
    __nv_bfloat16* dv;          // [B, Hkv, N, D]
    const float2* rope;         // (cos, sin) table or nullptr
    int B, Hq, Hkv, N, Npad;
    int causal, window;
    float scale, scale_log2;
};

// D_i = dO_i . O_i and LSE_i * log2(e), one warp per row; rows past N get (+inf, 0) so that their
// recomputed probabilities are exactly 0.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const BwdParams p) {
    const long long warp = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const long long rows = static_cast<long long>(p.B) * p.Hq * p.Npad;
    if (warp >= rows) return;
    const long long bh = warp / p.Npad;
    const int i = static_cast<int>(warp % p.Npad);
    float2 out = make_float2(INFINITY, 0.f);
    if (i < p.N) {
        const size_t off = (static_cast<size_t>(bh) * p.N + i) * D;
        float acc = 0.f;
        constexpr int PER = D / 32;  // consecutive elements per lane
        const __nv_bfloat16* po = p.o + off + lane * PER;
        const __nv_bfloat16* pd = p.dout + off + lane * PER;
#pragma unroll
        for (int e = 0; e < PER; ++e) acc = fmaf(__bfloat162float(po[e]), __bfloat162float(pd[e]), acc);
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
        out = make_float2(p.lse[static_cast<size_t>(bh) * p.N + i] * kLog2e, acc);
    }
    if (lane == 0) reinterpret_cast<float2*>(p.vec)[warp] = out;
}

template <int D>
struct BwdCfg {
    static constexpr int NREG = D / 64;
    static constexpr int REGION_BYTES = 128 * 128;
    static constexpr int TILE_BYTES = 128 * D * 2;
    static constexpr int VEC_BYTES = 128 * 8;  // (lse2, D) per row of a query tile
    // fixed pair (K,V or Q,dO) + two stages of the streamed pair, with their vectors
    static constexpr int SMEM_BYTES = 6 * TILE_BYTES + 2 * VEC_BYTES + 1024 /*barriers*/ + 1024 /*align*/;
    static constexpr int THREADS = 192;
    static constexpr uint32_t TMEM_COLS = 512;
};

struct BwdBarriers {
    uint64_t fixed_loaded;
    uint64_t full[2], empty[2];
    uint64_t s_full, p_full, acc_done, drain;
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

// =============================================================================== dK, dV
// CTA (key tile jt, K/V head g, batch b). Steps t walk (query head of the group, query tile).
// TMEM: S^T at 0 (P^T over its first 64 columns), dP^T at 128 (dS^T over its first 64),
// dV at 256, dK at 256 + D.
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
    float2* sVec = reinterpret_cast<float2*>(sDO + 2 * C::TILE_BYTES);  // [2][128]
    auto* bar = reinterpret_cast<BwdBarriers*>(reinterpret_cast<uint8_t*>(sVec) + 2 * C::VEC_BYTES);
    volatile int* abort_flag = &bar->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int jt = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
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
        }
        ptx::mbar_init(&bar->s_full, 1);
        ptx::mbar_init(&bar->p_full, 128);
        ptx::mbar_init(&bar->acc_done, 1);
        ptx::mbar_init(&bar->drain, 1);
        bar->abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 5) {
        ptx::tmem_alloc(&bar->tmem_base, C::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = bar->tmem_base;
    constexpr uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_DK = 256 + D;

    if (warp == 4) {
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
                const int h = g * G + t / per_head, i0 = (ib + t % per_head) * 128;
                const int zq = b * p.Hq + h;
                ptx::mbar_arrive_expect_tx(&bar->full[s], 2 * C::TILE_BYTES + C::VEC_BYTES);
                for (int r = 0; r < C::NREG; ++r) {
                    ptx::tma_load_3d(sQ + s * C::TILE_BYTES + r * C::REGION_BYTES, &tm_q, &bar->full[s], r * 64, i0, zq);
                    ptx::tma_load_3d(sDO + s * C::TILE_BYTES + r * C::REGION_BYTES, &tm_do, &bar->full[s], r * 64, i0, zq);
                }
                ptx::bulk_load(sVec + s * 128, p.vec + (static_cast<size_t>(zq) * p.Npad + i0) * 2, C::VEC_BYTES,
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
    } else if (warp == 5) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0 && T > 0) {
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
            bool ok = ptx::mbar_wait(&bar->fixed_loaded, 0, abort_flag);
            bool issued_any = false;
            for (int t = 0; ok && t < T; ++t) {
                const int s = t & 1;
                if (!ptx::mbar_wait(&bar->full[s], (t >> 1) & 1, abort_flag)) { ok = false; break; }
                // S^T = K Q^T and dP^T = V dO^T (M = 128 keys, N = 128 queries, K = D)
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * C::REGION_BYTES + (kk & 3) * 32) >> 4;
                    ptx::mma_ss(tmem + T_S, ptx::desc64(k_lo + off, HI), ptx::desc64(q_lo + s * TILE16 + off, HI), ID_S, kk > 0);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * C::REGION_BYTES + (kk & 3) * 32) >> 4;
                    ptx::mma_ss(tmem + T_DP, ptx::desc64(v_lo + off, HI), ptx::desc64(do_lo + s * TILE16 + off, HI), ID_S, kk > 0);
                }
                ptx::mma_commit(&bar->s_full);
                issued_any = true;
                if (!ptx::mbar_wait(&bar->p_full, t & 1, abort_flag)) { ok = false; break; }
                ptx::tc_fence_after();
                // dV += P^T dO and dK += dS^T Q (M = 128 keys, N = D, K = 128 queries)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk * 2048) >> 4;
                    ptx::mma_ts(tmem + T_DV, tmem + T_S + kk * 8, ptx::desc64(domn_lo + s * TILE16 + off, HI), ID_G,
                                (t > 0 || kk > 0) ? 1u : 0u);
                    ptx::mma_ts(tmem + T_DK, tmem + T_DP + kk * 8, ptx::desc64(qmn_lo + s * TILE16 + off, HI), ID_G,
                                (t > 0 || kk > 0) ? 1u : 0u);
                }
                ptx::mma_commit(&bar->empty[s]);
                if (t == T - 1) ptx::mma_commit(&bar->acc_done);
            }
            if (!ok) {
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
        const int r = threadIdx.x;           // key row == TMEM lane
        const int key = j0 + r;
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        bool ok = true;
        for (int t = 0; ok && t < T; ++t) {
            const int s = t & 1;
            const int i0 = (ib + t % per_head) * 128;
            if (!ptx::mbar_wait(&bar->full[s], (t >> 1) & 1, abort_flag)) { ok = false; break; }
            if (!ptx::mbar_wait(&bar->s_full, t & 1, abort_flag)) { ok = false; break; }
            ptx::tc_fence_after();
            const float2* vec = sVec + s * 128;
            const bool need_mask = (p.causal && i0 < j0 + 127) || (p.window > 0 && i0 + 127 - j0 > p.window - 1);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t sv[32], dv[32], sv2[32], dv2[32];
                ptx::tmem_ld32(tmem + lane_base + T_S + half * 64, sv);
                ptx::tmem_ld32(tmem + lane_base + T_S + half * 64 + 32, sv2);
                ptx::tmem_ld32(tmem + lane_base + T_DP + half * 64, dv);
                ptx::tmem_ld32(tmem + lane_base + T_DP + half * 64 + 32, dv2);
                uint32_t pk[32], dk[32];
#pragma unroll
                for (int c = 0; c < 64; c += 2) {
                    float pr[2], ds[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int col = half * 64 + c + e;  // query column within the tile
                        const float sraw = __uint_as_float(c + e < 32 ? sv[c + e] : sv2[c + e - 32]);
                        const float dp = __uint_as_float(c + e < 32 ? dv[c + e] : dv2[c + e - 32]);
                        const float2 ld = vec[col];  // (LSE * log2 e, D) of the query; +inf past N
                        float pe = ptx::ex2(fmaf(sraw, p.scale_log2, -ld.x));
                        if (need_mask) {
                            const int qpos = i0 + col;
                            const bool vis = (!p.causal || qpos >= key) && (p.window <= 0 || qpos - key < p.window);
                            pe = vis ? pe : 0.f;
                        }
                        pr[e] = pe;
                        ds[e] = pe * (dp - ld.y);
                    }
                    pk[c / 2] = ptx::pack_bf16x2(pr[0], pr[1]);
                    dk[c / 2] = ptx::pack_bf16x2(ds[0], ds[1]);
                }
                // P^T and dS^T (bf16 pairs) over the first 64 columns of their buffers; this half's
                // source columns were read above, the second half's lie beyond what is written now.
                ptx::tmem_st32(tmem + lane_base + T_S + half * 32, pk);
                ptx::tmem_st32(tmem + lane_base + T_DP + half * 32, dk);
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&bar->p_full);
        }
        if (ok && T > 0) ok = ptx::mbar_wait(&bar->acc_done, 0, abort_flag);
        if (ok && T > 0) {
            // every lane takes part in the warp-collective TMEM loads; rows past N store nothing
            ptx::tc_fence_after();
            const size_t row = (static_cast<size_t>(b) * p.Hkv + g) * p.N + min(key, p.N - 1);
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t v[32];
                ptx::tmem_ld32(tmem + lane_base + T_DV + c * 32, v);
                if (key < p.N) store_chunk_unrotated(v, 1.f, nullptr, D, key, c * 32, p.dv + row * D);
                ptx::tmem_ld32(tmem + lane_base + T_DK + c * 32, v);
                if (key < p.N) store_chunk_unrotated(v, p.scale, p.rope, D, key, c * 32, p.dk + row * D);
            }
        } else if (T == 0 && key < p.N) {
            // no query sees these keys: zero gradients
            const size_t row = (static_cast<size_t>(b) * p.Hkv + g) * p.N + key;
            uint4* d1 = reinterpret_cast<uint4*>(p.dv + row * D);
            uint4* d2 = reinterpret_cast<uint4*>(p.dk + row * D);
            for (int k = 0; k < D / 8; ++k) d1[k] = d2[k] = make_uint4(0, 0, 0, 0);
        }
        if (!ok) {
            *abort_flag = 1;
            raise_status(kStatusTimeout);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// =============================================================================== dQ
// CTA (query tile it, query head h, batch b). Steps walk the visible key tiles.
// TMEM: S at 0 (dS over its first 64 columns), dP at 128, dQ at 256.
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
    const int h = blockIdx.y, b = blockIdx.z;
    const int qt = gridDim.x - 1 - blockIdx.x;  // longest (causal) tiles first
    const int q0 = qt * 128;
    const int g = h / (p.Hq / p.Hkv);
    const TileRange R = tile_range(q0, p.N, p.causal, p.window);
    const int T = R.n;

    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar->fixed_loaded, 1);
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(&bar->full[s], 1);
            ptx::mbar_init(&bar->empty[s], 1);
        }
        ptx::mbar_init(&bar->s_full, 1);
        ptx::mbar_init(&bar->p_full, 128);
        ptx::mbar_init(&bar->acc_done, 1);
        ptx::mbar_init(&bar->drain, 1);
        bar->abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 5) {
        ptx::tmem_alloc(&bar->tmem_base, C::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = bar->tmem_base;
    constexpr uint32_t T_S = 0, T_DP = 128, T_DQ = 256;

    if (warp == 4) {
        if (lane == 0) {
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
    } else if (warp == 5) {
        if (lane == 0) {
            constexpr uint32_t ID_S = ptx::idesc_bf16_f32(128, 128, 0, 0);  // Q K^T, dO V^T: K-major
            constexpr uint32_t ID_G = ptx::idesc_bf16_f32(128, D, 0, 1);    // dS (TMEM) x K (MN-major)
            constexpr uint32_t HI = ptx::sw128_desc_hi(1024);
            constexpr uint32_t TILE16 = C::TILE_BYTES >> 4;
            const uint32_t q_lo = ptx::sw128_desc_lo(ptx::smem_u32(sQ), 16);
            const uint32_t do_lo = ptx::sw128_desc_lo(ptx::smem_u32(sDO), 16);
            const uint32_t k_lo = ptx::sw128_desc_lo(ptx::smem_u32(sK), 16);
            const uint32_t v_lo = ptx::sw128_desc_lo(ptx::smem_u32(sV), 16);
            const uint32_t kmn_lo = ptx::sw128_desc_lo(ptx::smem_u32(sK), C::REGION_BYTES);
            bool ok = ptx::mbar_wait(&bar->fixed_loaded, 0, abort_flag);
            bool issued_any = false;
            for (int t = 0; ok && t < T; ++t) {
                const int s = t & 1;
                if (!ptx::mbar_wait(&bar->full[s], (t >> 1) & 1, abort_flag)) { ok = false; break; }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * C::REGION_BYTES + (kk & 3) * 32) >> 4;
                    ptx::mma_ss(tmem + T_S, ptx::desc64(q_lo + off, HI), ptx::desc64(k_lo + s * TILE16 + off, HI), ID_S, kk > 0);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * C::REGION_BYTES + (kk & 3) * 32) >> 4;
                    ptx::mma_ss(tmem + T_DP, ptx::desc64(do_lo + off, HI), ptx::desc64(v_lo + s * TILE16 + off, HI), ID_S, kk > 0);
                }
                ptx::mma_commit(&bar->s_full);
                issued_any = true;
                if (!ptx::mbar_wait(&bar->p_full, t & 1, abort_flag)) { ok = false; break; }
                ptx::tc_fence_after();
                // dQ += dS K (M = 128 queries, N = D, K = 128 keys)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    ptx::mma_ts(tmem + T_DQ, tmem + T_S + kk * 8, ptx::desc64(kmn_lo + s * TILE16 + ((kk * 2048) >> 4), HI),
                                ID_G, (t > 0 || kk > 0) ? 1u : 0u);
                ptx::mma_commit(&bar->empty[s]);
                if (t == T - 1) ptx::mma_commit(&bar->acc_done);
            }
            if (!ok) {
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
        const int r = threadIdx.x;  // query row == TMEM lane
        const int qpos = q0 + r;
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        float2 ld = make_float2(INFINITY, 0.f);
        if (qpos < p.N) ld = reinterpret_cast<const float2*>(p.vec)[(static_cast<size_t>(b) * p.Hq + h) * p.Npad + qpos];
        bool ok = true;
        for (int t = 0; ok && t < T; ++t) {
            const int k0 = (R.jb + t) * 128;
            if (!ptx::mbar_wait(&bar->s_full, t & 1, abort_flag)) { ok = false; break; }
            ptx::tc_fence_after();
            const bool need_mask = (k0 + 128 > p.N) || (p.causal && k0 + 127 > q0) ||
                                   (p.window > 0 && k0 < q0 + 128 - p.window);
            const int lo = p.window > 0 ? qpos - p.window + 1 : -0x7fffffff;
            const int hi = p.causal ? min(qpos, p.N - 1) : p.N - 1;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t sv[32], dv[32], sv2[32], dv2[32];
                ptx::tmem_ld32(tmem + lane_base + T_S + half * 64, sv);
                ptx::tmem_ld32(tmem + lane_base + T_S + half * 64 + 32, sv2);
                ptx::tmem_ld32(tmem + lane_base + T_DP + half * 64, dv);
                ptx::tmem_ld32(tmem + lane_base + T_DP + half * 64 + 32, dv2);
                uint32_t dsk[32];
#pragma unroll
                for (int c = 0; c < 64; c += 2) {
                    float ds[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int col = half * 64 + c + e;
                        const float sraw = __uint_as_float(c + e < 32 ? sv[c + e] : sv2[c + e - 32]);
                        const float dp = __uint_as_float(c + e < 32 ? dv[c + e] : dv2[c + e - 32]);
                        float pe = ptx::ex2(fmaf(sraw, p.scale_log2, -ld.x));
                        if (need_mask) {
                            const int kj = k0 + col;
                            pe = (kj < lo || kj > hi) ? 0.f : pe;
                        }
                        ds[e] = pe * (dp - ld.y);
                    }
                    dsk[c / 2] = ptx::pack_bf16x2(ds[0], ds[1]);
                }
                ptx::tmem_st32(tmem + lane_base + T_S + half * 32, dsk);
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&bar->p_full);
        }
        if (ok && T > 0) ok = ptx::mbar_wait(&bar->acc_done, 0, abort_flag);
        if (ok && T > 0) {
            ptx::tc_fence_after();
            __nv_bfloat16* dst = p.dq + ((static_cast<size_t>(b) * p.Hq + h) * p.N + min(qpos, p.N - 1)) * D;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
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
    if (warp == 5) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace attn
