// rope.cuh -- rotary position embedding of the key rows, once per call.
//
// RoPE rotates each pair (2i, 2i+1) of a query or key vector by the angle pos * base^(-2i/D)
// ("attention-transformers", Q "How does Rotary Position Embedding (RoPE) work?"; pairs are the
// interleaved 2-D subspaces). Queries are rotated inside the attention kernel right after their
// tile lands in shared memory (once per query tile). Keys are rotated here, by one streaming
// pass over K: every key tile is read by many query tiles (all of its query heads, and every
// later query tile under a causal mask), so rotating it inside the attention kernel would
// repeat the same rotation tens of times per tile and compete with the softmax for the FP32
// pipes. This pass moves 2 bytes in and 2 bytes out per element, about 1% of the attention
// kernel's time at N = 8192.
#pragma once
#include "ptx.cuh"

namespace attn {

// One interleaved pair (x0 in the low half, x1 in the high half of a bf16x2 word) rotated by the
// angle whose (cos, sin) is given: x0 cos - x1 sin and x0 sin + x1 cos, each product and the sum
// rounded once in fp64 (no fused multiply-add), then rounded to bf16 (nearest even). With the
// fp64 cos/sin of the host-built table this is the rotation rounded exactly as an fp64 reference
// computes it, so rotated operands carry no fp32 rotation error.
__device__ __forceinline__ uint32_t rope_rotate_pair(uint32_t w, double cth, double sth) {
    const double x0 = static_cast<double>(ptx::bf16lo_to_f32(w)), x1 = static_cast<double>(ptx::bf16hi_to_f32(w));
    const double y0 = __dsub_rn(__dmul_rn(x0, cth), __dmul_rn(x1, sth));
    const double y1 = __dadd_rn(__dmul_rn(x0, sth), __dmul_rn(x1, cth));
    const uint32_t lo = __bfloat16_as_ushort(__double2bfloat16(y0));
    const uint32_t hi = __bfloat16_as_ushort(__double2bfloat16(y1));
    return lo | (hi << 16);
}

// k, k_rot: [rows, D] bf16 with row r at position r % N (rows = BH * N); cs: [>= N, D/2] (cos, sin)
// in fp64. A thread takes one 16-byte output chunk (4 pairs) of one position, loads that chunk's 4
// table entries once and applies them to the chunk in every one of the BH rows at the position;
// consecutive threads take consecutive chunks, so each row's loads and stores are coalesced.
// kHalf: the pairs are (i, i + D/2) and the rotated pair i is written interleaved at (2i, 2i+1) --
// the dimensions are permuted so that the attention kernel, which rotates its queries the same
// way, can treat both pairings alike.
template <int D, bool kHalf = false>
__global__ void __launch_bounds__(256) rope_rotate_rows_kernel(const uint4* __restrict__ k, uint4* __restrict__ k_rot,
                                                               const double2* __restrict__ cs, long long rows, int N) {
    constexpr int CHUNKS = D / 8;
    const long long bh_count = rows / N;
    const long long total = static_cast<long long>(N) * CHUNKS;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int pos = static_cast<int>(idx / CHUNKS);
        const int c = static_cast<int>(idx % CHUNKS);
        double2 t[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) t[e] = __ldg(cs + static_cast<size_t>(pos) * (D / 2) + c * 4 + e);
#pragma unroll 4
        for (long long bh = 0; bh < bh_count; ++bh) {
            const long long row = bh * N + pos;
            uint4 w;
            if constexpr (kHalf) {
                // pairs 4c .. 4c+3: first members at elements 4c.., second members at D/2 + 4c..
                const uint2* src = reinterpret_cast<const uint2*>(k + row * CHUNKS);
                const uint2 a = __ldg(src + c), b = __ldg(src + c + D / 8);
                const uint32_t av[2] = {a.x, a.y}, bv[2] = {b.x, b.y};
                uint32_t* wv = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const uint32_t lo = (e & 1) ? (av[e / 2] >> 16) : (av[e / 2] & 0xFFFFu);
                    const uint32_t hi = (e & 1) ? (bv[e / 2] >> 16) : (bv[e / 2] & 0xFFFFu);
                    wv[e] = lo | (hi << 16);
                }
            } else {
                w = __ldg(k + row * CHUNKS + c);
            }
            uint32_t* wv = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
            for (int e = 0; e < 4; ++e) wv[e] = rope_rotate_pair(wv[e], t[e].x, t[e].y);
            k_rot[row * CHUNKS + c] = w;
        }
    }
}

}  // namespace attn
