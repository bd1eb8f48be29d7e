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

// k, k_rot: [rows, D] bf16 with row r at position r % N; cs: [>= N, D/2] (cos, sin) float2.
// Each thread handles 16-byte chunks (4 pairs); consecutive threads take consecutive chunks, so
// loads and stores are fully coalesced.
template <int D>
__global__ void __launch_bounds__(256) rope_rotate_rows_kernel(const uint4* __restrict__ k, uint4* __restrict__ k_rot,
                                                               const float2* __restrict__ cs, long long rows, int N) {
    constexpr int CHUNKS = D / 8;
    const long long total = rows * CHUNKS;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const long long row = idx / CHUNKS;
        const int c = static_cast<int>(idx % CHUNKS);
        const int pos = static_cast<int>(row % N);
        uint4 w = __ldg(k + idx);
        const float4* t = reinterpret_cast<const float4*>(cs + static_cast<size_t>(pos) * (D / 2) + c * 4);
        const float4 a = __ldg(t), b = __ldg(t + 1);
        const float csv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        uint32_t* wv = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float x0 = ptx::bf16lo_to_f32(wv[e]), x1 = ptx::bf16hi_to_f32(wv[e]);
            const float cth = csv[2 * e], sth = csv[2 * e + 1];
            wv[e] = ptx::pack_bf16x2(fmaf(x0, cth, -x1 * sth), fmaf(x0, sth, x1 * cth));
        }
        k_rot[idx] = w;
    }
}

}  // namespace attn
