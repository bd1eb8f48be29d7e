// rope.cuh -- rotary position embedding of the query and key rows, once per call.
//
// RoPE rotates each pair (2i, 2i+1) of a query or key vector by the angle pos * base^(-2i/D)
// ("attention-transformers", Q "How does Rotary Position Embedding (RoPE) work?"; pairs are the
// interleaved 2-D subspaces). Queries and keys are rotated here, by one streaming pass over Q and
// K in one launch, before the attention kernel reads them. Every key tile is read by many query
// tiles, so rotating keys inside the attention kernel would repeat the same rotation tens of
// times per tile; a query tile is used once, but rotating it inside the kernel puts 64 KB of
// cos/sin table per query tile through the SM and the rotation on the tensor core's critical
// path at every work item, which measured slower than this pass's extra read and write of Q.
// The rotation itself is exact (fp64, below), so rotated operands equal an fp64 reference's.
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

// Up to two tensors per launch, blockIdx.z selecting one: src[z], dst[z]: [bh[z] * N, D] bf16
// with row r at position r % N; cs: [>= N, D/2] (cos, sin) in fp64.
struct RopeRowsArgs {
    const uint4* src[2];
    uint4* dst[2];
    long long bh[2];
    const double2* cs;
    int N;
};

// A thread takes one 16-byte output chunk (4 pairs) of one position, loads that chunk's 4 table
// entries once and applies them to the chunk in rows blockIdx.y, blockIdx.y + gridDim.y, ... of
// the bh rows at that position, loading 4 such rows before it stores any, so that several loads
// are in flight per thread. Consecutive threads take consecutive chunks, so each row's loads and
// stores are coalesced; the y split keeps a short sequence (few positions, many rows) from
// running on fewer blocks than there are SMs.
// kHalf: the pairs are (i, i + D/2) and the rotated pair i is written interleaved at (2i, 2i+1) --
// the dimensions are permuted, the same for queries and keys, which leaves every score q.k
// unchanged, so the attention kernel treats both pairings alike.
template <int D, bool kHalf = false>
__global__ void __launch_bounds__(256) rope_rotate_rows_kernel(RopeRowsArgs a) {
    constexpr int CHUNKS = D / 8;
    constexpr int U = 4;  // rows in flight per thread
    // The attention kernel that reads the rotated rows is launched as this kernel's programmatic
    // dependent: it may be scheduled now and run its set-up, and it waits for this grid to
    // complete before it touches global memory.
    ptx::grid_launch_dependents();
    const int z = blockIdx.z;
    const uint4* __restrict__ src = z ? a.src[1] : a.src[0];
    uint4* __restrict__ dst = z ? a.dst[1] : a.dst[0];
    const long long bh_count = z ? a.bh[1] : a.bh[0];
    const int N = a.N;
    const long long total = static_cast<long long>(N) * CHUNKS;
    const long long ys = gridDim.y;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int pos = static_cast<int>(idx / CHUNKS);
        const int c = static_cast<int>(idx % CHUNKS);
        double2 t[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) t[e] = __ldg(a.cs + static_cast<size_t>(pos) * (D / 2) + c * 4 + e);
        for (long long bh0 = blockIdx.y; bh0 < bh_count; bh0 += U * ys) {
            uint4 w[U];
#pragma unroll
            for (int j = 0; j < U; ++j) {
                const long long bh = bh0 + j * ys;
                if (bh >= bh_count) continue;
                const long long row = bh * N + pos;
                if constexpr (kHalf) {
                    // pairs 4c .. 4c+3: first members at elements 4c.., second members at D/2 + 4c..
                    const uint2* s2 = reinterpret_cast<const uint2*>(src + row * CHUNKS);
                    const uint2 lo = __ldg(s2 + c), hi = __ldg(s2 + c + D / 8);
                    w[j].x = (lo.x & 0xFFFFu) | (hi.x << 16);
                    w[j].y = (lo.x >> 16) | (hi.x & 0xFFFF0000u);
                    w[j].z = (lo.y & 0xFFFFu) | (hi.y << 16);
                    w[j].w = (lo.y >> 16) | (hi.y & 0xFFFF0000u);
                } else {
                    w[j] = __ldg(src + row * CHUNKS + c);
                }
            }
#pragma unroll
            for (int j = 0; j < U; ++j) {
                const long long bh = bh0 + j * ys;
                if (bh >= bh_count) continue;
                uint32_t* wv = reinterpret_cast<uint32_t*>(&w[j]);
#pragma unroll
                for (int e = 0; e < 4; ++e) wv[e] = rope_rotate_pair(wv[e], t[e].x, t[e].y);
                dst[(bh * N + pos) * CHUNKS + c] = w[j];
            }
        }
    }
}

}  // namespace attn
