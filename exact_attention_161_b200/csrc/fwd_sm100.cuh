// fwd_sm100.cuh -- FlashAttention-style exact attention forward for sm_100a.
//
// One CTA computes one 128-row tile of queries of one (batch, query head). It streams the
// visible 128-key tiles of the matching K/V head through shared memory and keeps the online
// softmax state per row: running max m, normaliser l and output accumulator o, rescaled as the
// max grows, then O = o / l and the row logsumexp ("Why is attention O(n^2), how does
// FlashAttention help, ...", "Deep dive: FlashAttention"). The n x n score matrix never leaves
// the SM: each 128x128 score tile lives in Tensor Memory only.
//
// Roles (192 threads):
//   warps 0-3  softmax: thread r owns query row r of the tile; it rotates its Q row (RoPE) once,
//              then per key tile reads its 128 scores from TMEM, masks them, updates m and l,
//              writes P (bf16) back into TMEM over the first half of the scores, rescales its
//              row of O when the max moved by more than 2^8, and finally writes O and LSE.
//   warp 4     TMA producer: Q once, then K and V tiles into a NS-stage ring.
//   warp 5     MMA issuer (one thread) and TMEM owner: S = Q K^T into one of two TMEM score
//              buffers, O += P V with P read from TMEM, completion signalled by tcgen05.commit.
//
// Tensor Memory (512 columns x 128 lanes x 32 bit): S0 at column 0, S1 at 128, O at 256
// (D columns). The score buffers alternate per key tile, so the tensor core computes the next
// tile's scores while the softmax works on the current one.
//
// Masks enter as -inf on the logits before the softmax ("Transformer Attention Mechanism
// Interview Deep Dive", "Causal masking"); key tiles that are fully masked are never visited
// (causal: tiles past the diagonal; sliding window: tiles before the window), which is the
// block skipping of "Deep dive: FlashAttention".
#pragma once
#include "common.cuh"
#include "ptx.cuh"

namespace attn {

struct FwdParams {
    __nv_bfloat16* o;       // [B, Hq, N, D]
    float* lse;             // [B, Hq, N] natural-log row logsumexp, or nullptr
    const float2* rope;     // [>= N, D/2] (cos, sin) of pos * base^(-2i/D), or nullptr (no RoPE)
    int B, Hq, Hkv, N;
    int causal, window;     // window > 0 only together with causal
    float scale_log2;       // softmax scale * log2(e)
};

template <int D>
struct FwdCfg {
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    static constexpr int BM = 128;                    // query rows per tile
    static constexpr int BN = 128;                    // keys per tile
    static constexpr int NREG = D / 64;               // 128-byte swizzle regions per row
    static constexpr int REGION_BYTES = 128 * 128;    // 128 rows x 128 bytes
    static constexpr int TILE_BYTES = 128 * D * 2;    // one Q, K or V tile in bf16
    static constexpr int NS = (D == 128) ? 2 : 4;     // K/V pipeline stages
    static constexpr int SMEM_TILES = 1 + 2 * NS;
    static constexpr int SMEM_BYTES = SMEM_TILES * TILE_BYTES + 1024 /*barriers*/ + 1024 /*align*/;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t TMEM_S0 = 0, TMEM_S1 = 128, TMEM_O = 256;
    static constexpr int THREADS = 192;
    // Rescale the output only when the running max grew by more than this (log2 units): with a
    // stale max the probabilities stay below 2^8, exact after the final division by l.
    static constexpr float RESCALE_THRESHOLD = 8.0f;
};

template <int NS>
struct FwdBarriers {
    uint64_t q_loaded, q_ready;
    uint64_t k_full[NS], v_full[NS], kv_empty[NS];
    uint64_t s_full[2], p_full[2];
    uint64_t o_done, o_final, drain;
    uint32_t tmem_base;
    int abort;
};

// Rotate one 128-byte-swizzled row of a Q tile in place: pairs (2i, 2i+1) by pos * theta_i, in
// fp32 with the (cos, sin) table, rounded back to bf16 ("attention-transformers", Q "How does
// Rotary Position Embedding (RoPE) work?").
template <int D>
__device__ __forceinline__ void rope_rotate_smem_row(uint8_t* tile, int r, const float2* __restrict__ cs_row) {
    using C = FwdCfg<D>;
#pragma unroll
    for (int reg = 0; reg < C::NREG; ++reg) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint4* p = reinterpret_cast<uint4*>(tile + reg * C::REGION_BYTES + r * 128 + ((c ^ (r & 7)) << 4));
            uint4 w = *p;
            const int i0 = reg * 32 + c * 4;  // first pair index of this 16-byte chunk
            const float4 a = __ldg(reinterpret_cast<const float4*>(cs_row + i0));
            const float4 b = __ldg(reinterpret_cast<const float4*>(cs_row + i0 + 2));
            uint32_t* wv = reinterpret_cast<uint32_t*>(&w);
            const float cs[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float x0 = ptx::bf16lo_to_f32(wv[k]), x1 = ptx::bf16hi_to_f32(wv[k]);
                const float cth = cs[2 * k], sth = cs[2 * k + 1];
                wv[k] = ptx::pack_bf16x2(fmaf(x0, cth, -x1 * sth), fmaf(x0, sth, x1 * cth));
            }
            *p = w;
        }
    }
}

template <int D>
__global__ void __launch_bounds__(FwdCfg<D>::THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    using C = FwdCfg<D>;
    constexpr int NS = C::NS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;
    uint8_t* sK = sQ + C::TILE_BYTES;
    uint8_t* sV = sK + NS * C::TILE_BYTES;
    auto* bar = reinterpret_cast<FwdBarriers<NS>*>(sV + NS * C::TILE_BYTES);
    volatile int* abort_flag = &bar->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.x, b = blockIdx.y;
    const int qt = gridDim.z - 1 - blockIdx.z;  // longest (causal) tiles first
    const int q0 = qt * C::BM;
    const int g = h / (p.Hq / p.Hkv);           // query head h reads K/V head h / (Hq/Hkv)
    const int kv_hi = p.causal ? min(p.N, q0 + C::BM) : p.N;
    const int kv_lo = p.window > 0 ? max(0, q0 - p.window + 1) : 0;
    const int j_begin = kv_lo / C::BN;
    const int T = (kv_hi + C::BN - 1) / C::BN - j_begin;  // >= 1

    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar->q_loaded, 1);
        ptx::mbar_init(&bar->q_ready, 1);
        for (int s = 0; s < NS; ++s) {
            ptx::mbar_init(&bar->k_full[s], 1);
            ptx::mbar_init(&bar->v_full[s], 1);
            ptx::mbar_init(&bar->kv_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(&bar->s_full[s], 1);
            ptx::mbar_init(&bar->p_full[s], 128);
        }
        ptx::mbar_init(&bar->o_done, 1);
        ptx::mbar_init(&bar->o_final, 1);
        ptx::mbar_init(&bar->drain, 1);
        bar->abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 4 && lane == 0) {
        ptx::prefetch_tensormap(&tm_q);
        ptx::prefetch_tensormap(&tm_k);
        ptx::prefetch_tensormap(&tm_v);
    }
    if (warp == 5) {
        ptx::tmem_alloc(&bar->tmem_base, C::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = bar->tmem_base;

    if (warp == 4) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const int zq = b * p.Hq + h, zk = b * p.Hkv + g;
            ptx::mbar_arrive_expect_tx(&bar->q_loaded, C::TILE_BYTES);
#pragma unroll
            for (int r = 0; r < C::NREG; ++r)
                ptx::tma_load_3d(sQ + r * C::REGION_BYTES, &tm_q, &bar->q_loaded, r * 64, q0, zq);
            int issued = 0;
            bool ok = true;
            for (int t = 0; t < T && ok; ++t) {
                const int s = t % NS;
                if (t >= NS && !ptx::mbar_wait(&bar->kv_empty[s], ((t / NS) - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                const int k0 = (j_begin + t) * C::BN;
                ptx::mbar_arrive_expect_tx(&bar->k_full[s], C::TILE_BYTES);
#pragma unroll
                for (int r = 0; r < C::NREG; ++r)
                    ptx::tma_load_3d(sK + s * C::TILE_BYTES + r * C::REGION_BYTES, &tm_k, &bar->k_full[s], r * 64,
                                     k0, zk);
                ptx::mbar_arrive_expect_tx(&bar->v_full[s], C::TILE_BYTES);
#pragma unroll
                for (int r = 0; r < C::NREG; ++r)
                    ptx::tma_load_3d(sV + s * C::TILE_BYTES + r * C::REGION_BYTES, &tm_v, &bar->v_full[s], r * 64,
                                     k0, zk);
                issued = t + 1;
            }
            if (!ok) {
                *abort_flag = 1;
                raise_status(kStatusTimeout);
                // Let the copies already in flight land before the CTA's shared memory is released
                // (each wait is still bounded).
                volatile int never = 0;
                ptx::mbar_wait(&bar->q_loaded, 0, &never);
                for (int t = max(0, issued - NS); t < issued; ++t) {
                    const int s = t % NS;
                    ptx::mbar_wait(&bar->k_full[s], (t / NS) & 1, &never);
                    ptx::mbar_wait(&bar->v_full[s], (t / NS) & 1, &never);
                }
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC_S = ptx::idesc_bf16_f32(128, C::BN, 0, 0);  // Q, K both K-major
            constexpr uint32_t IDESC_O = ptx::idesc_bf16_f32(128, D, 0, 1);      // P K-major, V MN-major
            const uint32_t sq = ptx::smem_u32(sQ);
            bool ok = ptx::mbar_wait(&bar->q_ready, 0, abort_flag);
            bool issued_any = false;
            ptx::tc_fence_after();
            for (int t = 0; ok && t <= T; ++t) {
                if (t < T) {
                    const int s = t % NS;
                    if (!ptx::mbar_wait(&bar->k_full[s], (t / NS) & 1, abort_flag)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t sk = ptx::smem_u32(sK + s * C::TILE_BYTES);
                    const uint32_t d_s = tmem + ((t & 1) ? C::TMEM_S1 : C::TMEM_S0);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * C::REGION_BYTES + (kk & 3) * 32;
                        ptx::mma_ss(d_s, ptx::sw128_desc(sq + off, 16, 1024), ptx::sw128_desc(sk + off, 16, 1024),
                                    IDESC_S, kk > 0);
                    }
                    ptx::mma_commit(&bar->s_full[t & 1]);
                    issued_any = true;
                }
                if (t >= 1) {
                    const int u = t - 1, su = u % NS;
                    if (!ptx::mbar_wait(&bar->p_full[u & 1], (u >> 1) & 1, abort_flag)) { ok = false; break; }
                    if (!ptx::mbar_wait(&bar->v_full[su], (u / NS) & 1, abort_flag)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t sv = ptx::smem_u32(sV + su * C::TILE_BYTES);
                    const uint32_t a_p = tmem + ((u & 1) ? C::TMEM_S1 : C::TMEM_S0);
#pragma unroll
                    for (int kk = 0; kk < C::BN / 16; ++kk)
                        ptx::mma_ts(tmem + C::TMEM_O, a_p + kk * 8, ptx::sw128_desc(sv + kk * 2048, C::REGION_BYTES, 1024),
                                    IDESC_O, (u > 0 || kk > 0) ? 1u : 0u);
                    ptx::mma_commit(&bar->kv_empty[su]);
                    ptx::mma_commit(u == T - 1 ? &bar->o_final : &bar->o_done);
                }
            }
            if (!ok) {
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
        // ------------------------------------------------------------------ softmax warpgroup
        const int r = threadIdx.x;  // row within the tile == TMEM lane
        const int i = q0 + r;       // query position
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        bool ok = ptx::mbar_wait(&bar->q_loaded, 0, abort_flag);
        if (ok && p.rope != nullptr && i < p.N)
            rope_rotate_smem_row<D>(sQ, r, p.rope + static_cast<size_t>(i) * (D / 2));
        ptx::fence_proxy_async_smem();
        ptx::named_barrier_sync(1, 128);
        if (threadIdx.x == 0) ptx::mbar_arrive(&bar->q_ready);

        float m_used = -INFINITY, l = 0.f;
        for (int t = 0; ok && t < T; ++t) {
            const int j0 = (j_begin + t) * C::BN;
            if (!ptx::mbar_wait(&bar->s_full[t & 1], (t >> 1) & 1, abort_flag)) { ok = false; break; }
            ptx::tc_fence_after();
            const uint32_t t_s = tmem + lane_base + ((t & 1) ? C::TMEM_S1 : C::TMEM_S0);
            float s[C::BN];
#pragma unroll
            for (int c = 0; c < C::BN / 32; ++c) {
                uint32_t v[32];
                ptx::tmem_ld32(t_s + c * 32, v);
#pragma unroll
                for (int k = 0; k < 32; ++k) s[c * 32 + k] = __uint_as_float(v[k]);
            }
            const bool need_mask = (j0 + C::BN > p.N) || (p.causal && j0 + C::BN - 1 > q0) ||
                                   (p.window > 0 && j0 < q0 + C::BM - p.window);
            if (need_mask) {
                const int lo = p.window > 0 ? i - p.window + 1 : -0x7fffffff;
                const int hi = p.causal ? min(i, p.N - 1) : p.N - 1;
#pragma unroll
                for (int c = 0; c < C::BN; ++c) {
                    const int kj = j0 + c;
                    if (kj < lo || kj > hi) s[c] = -INFINITY;
                }
            }
            float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
            for (int c = 4; c < C::BN; c += 4) {
                mx0 = fmaxf(mx0, s[c]);
                mx1 = fmaxf(mx1, s[c + 1]);
                mx2 = fmaxf(mx2, s[c + 2]);
                mx3 = fmaxf(mx3, s[c + 3]);
            }
            const float m_new = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * p.scale_log2;
            float alpha = 1.f;
            bool rescale = false;
            if (m_new > m_used + C::RESCALE_THRESHOLD) {  // also the first visible key (m_used = -inf)
                alpha = ptx::ex2(m_used - m_new);          // 2^-inf = 0
                m_used = m_new;
                rescale = true;
            }
            const float m_eff = (m_used == -INFINITY) ? 0.f : m_used;
            float sum0 = 0.f, sum1 = 0.f, sum2 = 0.f, sum3 = 0.f;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t pk[32];
#pragma unroll
                for (int k = 0; k < 32; k += 2) {
                    const int c = half * 64 + 2 * k;
                    const float p0 = ptx::ex2(fmaf(s[c], p.scale_log2, -m_eff));
                    const float p1 = ptx::ex2(fmaf(s[c + 1], p.scale_log2, -m_eff));
                    const float p2 = ptx::ex2(fmaf(s[c + 2], p.scale_log2, -m_eff));
                    const float p3 = ptx::ex2(fmaf(s[c + 3], p.scale_log2, -m_eff));
                    sum0 += p0;
                    sum1 += p1;
                    sum2 += p2;
                    sum3 += p3;
                    pk[k] = ptx::pack_bf16x2(p0, p1);
                    pk[k + 1] = ptx::pack_bf16x2(p2, p3);
                }
                // P (bf16 pairs) over the first 64 columns of this score buffer.
                ptx::tmem_st32(t_s + half * 32, pk);
            }
            l = l * alpha + ((sum0 + sum1) + (sum2 + sum3));
            if (t > 0 && __any_sync(0xffffffffu, rescale)) {
                // O must hold the previous tile's product before it is rescaled.
                if (!ptx::mbar_wait(&bar->o_done, (t - 1) & 1, abort_flag)) { ok = false; break; }
                ptx::tc_fence_after();
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t v[32];
                    const uint32_t t_o = tmem + lane_base + C::TMEM_O + c * 32;
                    ptx::tmem_ld32(t_o, v);
#pragma unroll
                    for (int k = 0; k < 32; ++k) v[k] = __float_as_uint(__uint_as_float(v[k]) * alpha);
                    ptx::tmem_st32(t_o, v);
                }
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&bar->p_full[t & 1]);
        }
        if (ok) ok = ptx::mbar_wait(&bar->o_final, 0, abort_flag);
        if (ok) {
            ptx::tc_fence_after();
            const float inv_l = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16* orow = p.o + ((static_cast<size_t>(b) * p.Hq + h) * p.N + i) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t v[32];
                ptx::tmem_ld32(tmem + lane_base + C::TMEM_O + c * 32, v);
                uint32_t w[16];
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    w[k] = ptx::pack_bf16x2(__uint_as_float(v[2 * k]) * inv_l, __uint_as_float(v[2 * k + 1]) * inv_l);
                if (i < p.N) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                    for (int k = 0; k < 4; ++k) dst[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
                }
            }
            if (p.lse != nullptr && i < p.N)
                p.lse[(static_cast<size_t>(b) * p.Hq + h) * p.N + i] =
                    l > 0.f ? (m_used + ptx::lg2(l)) * kLn2 : -INFINITY;
        } else {
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
