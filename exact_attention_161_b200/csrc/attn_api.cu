// attn_api.cu -- the C ABI declared in include/attn.h: argument checks, TMA descriptors, the
// cached RoPE tables and key scratch, and the kernel launches. The whole library is this one
// translation unit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <tuple>
#include <vector>

#include "attn.h"
#include "common.cuh"
#include "bwd_sm100.cuh"
#include "decode.cuh"
#include "fwd_sm100.cuh"
#include "rope.cuh"

#define ATTN_VERSION_STRING "exact_attention_161_b200 0.2.0 (sm_100a)"

namespace {

thread_local std::string g_last_error;

attn_status fail(attn_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

#define CUDA_TRY(expr)                                                                          \
    do {                                                                                        \
        cudaError_t e_ = (expr);                                                                \
        if (e_ != cudaSuccess) return fail(ATTN_ERR_CUDA, "%s: %s", #expr, cudaGetErrorString(e_)); \
    } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------------ cuTensorMapEncodeTiled
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// A rank-3 tensor map of bf16 (elem = 2) or 8-bit (elem = 1) elements: dims {d0 (contiguous), d1,
// d2}, box {128 bytes of d0, box1, 1}, 128-byte swizzle, out-of-bounds elements read as zero.
attn_status make_map_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box1,
                        int elem = 2) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable (no CUDA driver?)");
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {d0 * elem, d0 * d1 * elem};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / elem), box1, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, elem == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                    const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return ATTN_OK;
}

// 2-D fp32 map [d1 rows][d0 columns] with 32 x 32 boxes, 128-byte swizzled (reduce targets).
attn_status make_map_2d_f32(CUtensorMap* map, void* base, uint64_t d0, uint64_t d1) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable (no CUDA driver?)");
    const cuuint64_t dims[2] = {d0, d1};
    const cuuint64_t strides[1] = {d0 * 4};
    const cuuint32_t box[2] = {32, 32};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return ATTN_OK;
}

// ------------------------------------------------------------------ caches
struct DevBuf {
    void* ptr = nullptr;
    size_t bytes = 0;
    int dev = 0;
};

std::atomic<bool> g_debug_drop_copy{false};  // test hook of attn_debug_drop_copy

// Caches. A table or scratch buffer that is outgrown is replaced by a larger one; the old one is
// freed at once, after a device synchronisation (a launch still queued on any stream may read
// it). Growth is geometric, so this happens a few times in a process's life, not per call.
std::mutex g_cache_mu;
// Layouts of a cos/sin table covering positions [0, cap): (cos, sin) pairs, [cap][D/2], one
// position's pairs contiguous, in fp32 (kTab32) or fp64 (kTab64)
enum TabLayout { kTab32 = 0, kTab64 = 1 };
// (device, base, D, position scale, NTK factor, layout) -> table and its capacity
std::map<std::tuple<int, double, int, double, double, int>, std::pair<DevBuf, int>> g_rope_tables;
// (device, stream) -> scratch for the rotated queries and keys of attn_fwd; at most
// kMaxScratchStreams streams per device keep one (a new stream beyond that frees the device's
// others first, after a device synchronisation)
std::map<std::pair<int, void*>, DevBuf> g_key_scratch;
constexpr int kMaxScratchStreams = 8;

// Frees an outgrown buffer of device `dev` once every launch queued on that device has finished.
cudaError_t free_after_device_sync(const DevBuf& b) {
    if (!b.ptr) return cudaSuccess;
    int cur = 0;
    cudaError_t e = cudaGetDevice(&cur);
    if (e != cudaSuccess) return e;
    if (cur != b.dev && (e = cudaSetDevice(b.dev)) != cudaSuccess) return e;
    e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaFree(b.ptr);
    if (cur != b.dev) cudaSetDevice(cur);
    return e;
}

size_t grow_geometric(size_t need, size_t have) {
    size_t cap = have > 0 ? have : 1;
    while (cap < need) cap *= 2;
    return cap;
}

// (cos, sin) of (pos / pos_scale) * b^(-2i/D), b = base * ntk^(D/(D-2)), for pos < n, i < D/2:
// angles and trigonometry in fp64 (Position Interpolation divides the positions; NTK-aware scaling
// raises the base), stored in fp64 or rounded to fp32.
attn_status rope_table_any(int dev, double base, int D, int n, double pos_scale, double ntk, int layout,
                           const void** out) {
    std::lock_guard<std::mutex> lock(g_cache_mu);
    auto key = std::make_tuple(dev, base, D, pos_scale, ntk, layout);
    auto it = g_rope_tables.find(key);
    if (it != g_rope_tables.end() && it->second.second >= n) {
        *out = it->second.first.ptr;
        return ATTN_OK;
    }
    const bool wide = layout == kTab64;
    // capacity: a power of two of at least 1024 positions (so regrowth is rare), never beyond the
    // int range of positions
    int cap = 1024;
    while (cap < n && cap < (1 << 30)) cap *= 2;
    if (cap < n) cap = n;
    const size_t pairs = static_cast<size_t>(cap) * (D / 2);
    std::vector<double2> host64(wide ? pairs : 0);
    std::vector<float2> host32(wide ? 0 : pairs);
    std::vector<double> theta(D / 2);
    const double b = base * std::pow(ntk, static_cast<double>(D) / static_cast<double>(D - 2));
    for (int i = 0; i < D / 2; ++i) theta[i] = std::pow(b, -2.0 * static_cast<double>(i) / static_cast<double>(D));
    for (int pos = 0; pos < cap; ++pos)
        for (int i = 0; i < D / 2; ++i) {
            const double a = (static_cast<double>(pos) / pos_scale) * theta[i];
            const size_t at = static_cast<size_t>(pos) * (D / 2) + i;
            if (wide)
                host64[at] = make_double2(std::cos(a), std::sin(a));
            else
                host32[at] = make_float2(static_cast<float>(std::cos(a)), static_cast<float>(std::sin(a)));
        }
    DevBuf buf;
    buf.dev = dev;
    buf.bytes = pairs * (wide ? sizeof(double2) : sizeof(float2));
    CUDA_TRY(cudaMalloc(&buf.ptr, buf.bytes));
    cudaError_t e = cudaMemcpy(buf.ptr, wide ? static_cast<const void*>(host64.data()) : host32.data(), buf.bytes,
                               cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
        cudaFree(buf.ptr);
        return fail(ATTN_ERR_CUDA, "rope table upload: %s", cudaGetErrorString(e));
    }
    if (it != g_rope_tables.end()) {
        e = free_after_device_sync(it->second.first);
        if (e != cudaSuccess) {
            cudaFree(buf.ptr);
            return fail(ATTN_ERR_CUDA, "freeing an outgrown rope table: %s", cudaGetErrorString(e));
        }
    }
    g_rope_tables[key] = std::make_pair(buf, cap);
    *out = buf.ptr;
    return ATTN_OK;
}
attn_status rope_table(int dev, double base, int D, int n, const float2** out, double pos_scale = 1.0,
                       double ntk = 1.0) {
    const void* p = nullptr;
    attn_status st = rope_table_any(dev, base, D, n, pos_scale, ntk, kTab32, &p);
    *out = static_cast<const float2*>(p);
    return st;
}
attn_status rope_table64(int dev, double base, int D, int n, const double2** out, double pos_scale = 1.0,
                         double ntk = 1.0) {
    const void* p = nullptr;
    attn_status st = rope_table_any(dev, base, D, n, pos_scale, ntk, kTab64, &p);
    *out = static_cast<const double2*>(p);
    return st;
}
attn_status key_scratch(int dev, void* stream, size_t bytes, void** out) {
    std::lock_guard<std::mutex> lock(g_cache_mu);
    const auto key = std::make_pair(dev, stream);
    if (g_key_scratch.find(key) == g_key_scratch.end()) {
        int on_dev = 0;
        for (const auto& kv : g_key_scratch) on_dev += kv.first.first == dev;
        if (on_dev >= kMaxScratchStreams) {
            for (auto it = g_key_scratch.begin(); it != g_key_scratch.end();) {
                if (it->first.first != dev) { ++it; continue; }
                const cudaError_t e = free_after_device_sync(it->second);
                if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "freeing stream scratch: %s", cudaGetErrorString(e));
                it = g_key_scratch.erase(it);
            }
        }
    }
    DevBuf& b = g_key_scratch[key];
    if (b.bytes < bytes) {
        const size_t cap = grow_geometric(bytes, b.bytes);
        const cudaError_t e = free_after_device_sync(b);
        if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "freeing outgrown scratch: %s", cudaGetErrorString(e));
        b = DevBuf();
        CUDA_TRY(cudaMalloc(&b.ptr, cap));
        b.bytes = cap;
        b.dev = dev;
    }
    *out = b.ptr;
    return ATTN_OK;
}

// Opt a kernel into more than 48 KB of dynamic shared memory, once per (kernel, device).
std::mutex g_attr_mu;
std::map<std::pair<const void*, int>, bool> g_smem_set;

template <typename K>
attn_status ensure_smem(K kernel, int bytes, int dev) {
    std::lock_guard<std::mutex> lock(g_attr_mu);
    const auto key = std::make_pair(reinterpret_cast<const void*>(kernel), dev);
    if (!g_smem_set[key]) {
        CUDA_TRY(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
        g_smem_set[key] = true;
    }
    return ATTN_OK;
}

// Rotate Q (bhq rows of N positions) and K (bhk rows) into qr and kr with one launch of
// rope_rotate_rows_kernel: x covers the N * D/8 (position, chunk) pairs with 256 threads a block,
// at most 8 blocks per SM (the x loop strides over the rest); z picks the tensor; y splits the
// rows so that about 8 blocks per SM are resident however few positions there are.
template <int D>
attn_status launch_rope_rows(bool half, const void* q, void* qr, long long bhq, const void* k, void* kr, long long bhk,
                             const double2* cs, int N, int sms, cudaStream_t stream) {
    attn::RopeRowsArgs a{};
    a.src[0] = static_cast<const uint4*>(q);
    a.dst[0] = static_cast<uint4*>(qr);
    a.bh[0] = bhq;
    a.src[1] = static_cast<const uint4*>(k);
    a.dst[1] = static_cast<uint4*>(kr);
    a.bh[1] = bhk;
    a.cs = cs;
    a.N = N;
    const long long want = (static_cast<long long>(N) * (D / 8) + 255) / 256;
    const long long gx = want < 8LL * sms ? want : 8LL * sms;
    const long long bh_max = bhq > bhk ? bhq : bhk;
    long long gy = (8LL * sms + 2 * gx - 1) / (2 * gx);
    if (gy > bh_max) gy = bh_max;
    if (gy > 65535) gy = 65535;
    if (gy < 1) gy = 1;
    const dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy), 2);
    if (half)
        attn::rope_rotate_rows_kernel<D, true><<<grid, 256, 0, stream>>>(a);
    else
        attn::rope_rotate_rows_kernel<D, false><<<grid, 256, 0, stream>>>(a);
    CUDA_TRY(cudaGetLastError());
    return ATTN_OK;
}

struct PosVariant {
    int half_split = 0;
    double pos_scale = 1.0, ntk = 1.0;
    const float* alibi = nullptr;
};

template <int D>
attn_status launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                       int N, int causal, int window, float rope_base, float scale, cudaStream_t stream, int dev,
                       const PosVariant& pv = PosVariant()) {
    using C = attn::FwdCfg<D>;
    const void* q_use = q;
    const void* k_use = k;
    attn::FwdParams p{};
    if (rope_base > 0.f) {
        const double2* table64 = nullptr;
        attn_status st = rope_table64(dev, static_cast<double>(rope_base), D, N, &table64, pv.pos_scale, pv.ntk);
        if (st != ATTN_OK) return st;
        // rotated Q, then rotated K (256-byte aligned), in the stream's scratch
        const size_t qbytes = static_cast<size_t>(B) * Hq * N * D * 2;
        const size_t kbytes = static_cast<size_t>(B) * Hkv * N * D * 2;
        const size_t koff = (qbytes + 255) / 256 * 256;
        void* scratch = nullptr;
        st = key_scratch(dev, stream, koff + kbytes, &scratch);
        if (st != ATTN_OK) return st;
        void* q_rot = scratch;
        void* k_rot = static_cast<char*>(scratch) + koff;
        int sms = 148;
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        st = launch_rope_rows<D>(pv.half_split != 0, q, q_rot, static_cast<long long>(B) * Hq, k, k_rot,
                                 static_cast<long long>(B) * Hkv, table64, N, sms, stream);
        if (st != ATTN_OK) return st;
        q_use = q_rot;
        k_use = k_rot;
    }
    p.alibi = pv.alibi;
    p.o_scale = 1.f;
    CUtensorMap tq, tk, tv;
    attn_status st;
    if ((st = make_map_3d(&tq, q_use, D, N, static_cast<uint64_t>(B) * Hq, 128)) != ATTN_OK) return st;
    if ((st = make_map_3d(&tk, k_use, D, N, static_cast<uint64_t>(B) * Hkv, 128)) != ATTN_OK) return st;
    if ((st = make_map_3d(&tv, v, D, N, static_cast<uint64_t>(B) * Hkv, 128)) != ATTN_OK) return st;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.N = N;
    p.causal = causal;
    p.window = window > 0 ? window : 0;
    p.scale_log2 = scale * attn::kLog2e;
    p.nblk = (N + C::QT * C::BM - 1) / (C::QT * C::BM);
    p.n_items = B * Hq * p.nblk;
    p.debug_drop_copy = g_debug_drop_copy.load() ? 1 : 0;
    int sms = 148;
    CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    const int grid = p.n_items < sms ? p.n_items : sms;  // persistent: one CTA per SM
    // With RoPE the kernel is the rotation pass's programmatic dependent (see the kernel's set-up):
    // it is scheduled while the pass finishes and waits for it on the device.
    cudaLaunchConfig_t lc{};
    lc.gridDim = dim3(static_cast<unsigned>(grid));
    lc.blockDim = dim3(C::THREADS);
    lc.dynamicSmemBytes = C::SMEM_BYTES;
    lc.stream = stream;
    cudaLaunchAttribute la[1];
    la[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    la[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = la;
    lc.numAttrs = rope_base > 0.f ? 1 : 0;
    if (pv.alibi != nullptr) {
        if ((st = ensure_smem(attn::attn_fwd_kernel<D, true>, C::SMEM_BYTES, dev)) != ATTN_OK) return st;
        CUDA_TRY(cudaLaunchKernelEx(&lc, attn::attn_fwd_kernel<D, true, false>, tq, tk, tv, p));
    } else {
        if ((st = ensure_smem(attn::attn_fwd_kernel<D, false>, C::SMEM_BYTES, dev)) != ATTN_OK) return st;
        CUDA_TRY(cudaLaunchKernelEx(&lc, attn::attn_fwd_kernel<D, false, false>, tq, tk, tv, p));
    }
    CUDA_TRY(cudaGetLastError());
    return ATTN_OK;
}

size_t decode_chunks(int max_blocks) { return (static_cast<size_t>(max_blocks) + attn::kChunkPages - 1) / attn::kChunkPages; }

// FP8 prefill: e4m3 Q, K, V with per-tensor descales; the persistent kernel's kFp8 instance.
attn_status launch_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                           int N, int causal, int window, float scale, float descale_v, cudaStream_t stream, int dev) {
    constexpr int D = 128;
    using C = attn::FwdCfg<D, true>;
    attn::FwdParams p{};
    CUtensorMap tq, tk, tv;
    attn_status st;
    if ((st = make_map_3d(&tq, q, D, N, static_cast<uint64_t>(B) * Hq, 128, 1)) != ATTN_OK) return st;
    if ((st = make_map_3d(&tk, k, D, N, static_cast<uint64_t>(B) * Hkv, 128, 1)) != ATTN_OK) return st;
    if ((st = make_map_3d(&tv, v, D, N, static_cast<uint64_t>(B) * Hkv, 128, 1)) != ATTN_OK) return st;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.o_scale = descale_v;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.N = N;
    p.causal = causal;
    p.window = window > 0 ? window : 0;
    p.scale_log2 = scale * attn::kLog2e;
    p.nblk = (N + C::QT * C::BM - 1) / (C::QT * C::BM);
    p.n_items = B * Hq * p.nblk;
    p.debug_drop_copy = g_debug_drop_copy.load() ? 1 : 0;
    int sms = 148;
    CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    const int grid = p.n_items < sms ? p.n_items : sms;
    if ((st = ensure_smem(attn::attn_fwd_kernel<D, false, true>, C::SMEM_BYTES, dev)) != ATTN_OK) return st;
    attn::attn_fwd_kernel<D, false, true><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
    CUDA_TRY(cudaGetLastError());
    return ATTN_OK;
}

template <int D>
attn_status launch_step_prep(const void* q, void* q_rot, const void* k_new, const void* v_new, void* k_pages,
                             void* v_pages, const int32_t* block_table, const int32_t* seq_lens, int S, int T,
                             int max_blocks, int num_pages, int Hq, int Hkv, const double2* rope,
                             cudaStream_t stream) {
    attn::StepPrepParams a{};
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.q_rot = static_cast<__nv_bfloat16*>(q_rot);
    a.k_new = static_cast<const __nv_bfloat16*>(k_new);
    a.v_new = static_cast<const __nv_bfloat16*>(v_new);
    a.k_pages = static_cast<__nv_bfloat16*>(k_pages);
    a.v_pages = static_cast<__nv_bfloat16*>(v_pages);
    a.block_table = block_table;
    a.seq_lens = seq_lens;
    a.rope = rope;
    a.S = S;
    a.T = T;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.max_blocks = max_blocks;
    a.num_pages = num_pages;
    const long long warps = static_cast<long long>(S) * T * ((q_rot ? Hq : 0) + (k_new ? Hkv : 0));
    if (warps == 0) return ATTN_OK;
    attn::decode_step_prep_kernel<D><<<static_cast<unsigned>((warps * 32 + 127) / 128), 128, 0, stream>>>(a);
    CUDA_TRY(cudaGetLastError());
    return ATTN_OK;
}

template <int D>
attn_status launch_decode(const void* q, const void* k_pages, const void* v_pages, const int32_t* block_table,
                          const int32_t* seq_lens, int S, int T, int max_blocks, int num_pages, int Hq, int Hkv,
                          float scale, void* o, float* lse, void* ws, cudaStream_t stream, int dev) {
    using C = attn::DecCfg<D>;
    CUtensorMap tk, tv;
    attn_status st;
    const uint64_t slabs = static_cast<uint64_t>(num_pages) * Hkv;
    if ((st = make_map_3d(&tk, k_pages, D, attn::kPageSize, slabs, attn::kPageSize)) != ATTN_OK) return st;
    if ((st = make_map_3d(&tv, v_pages, D, attn::kPageSize, slabs, attn::kPageSize)) != ATTN_OK) return st;
    // chunk length: the longest that still gives at least 8 CTAs per SM (the grid's upper bound,
    // from max_blocks; the workspace is sized for the shortest chunk, so any choice fits)
    int sms = 148;
    CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    const long long rows = static_cast<long long>(S) * Hkv * ((Hq / Hkv * T + 15) / 16);
    int chunk_pages = attn::kMaxChunkPages;
    while (chunk_pages > attn::kChunkPages && rows * ((max_blocks + chunk_pages - 1) / chunk_pages) < 8LL * sms)
        chunk_pages /= 2;
    const int max_chunks = (max_blocks + chunk_pages - 1) / chunk_pages;  // never more than decode_chunks()
    attn::DecodeParams p{};
    p.chunk_pages = chunk_pages;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.block_table = block_table;
    p.seq_lens = seq_lens;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.ws_o = static_cast<float*>(ws);
    p.ws_ml = p.ws_o + static_cast<size_t>(S) * T * Hq * max_chunks * D;
    p.T = T;
    p.mtiles = (Hq / Hkv * T + 15) / 16;
    p.debug_drop_copy = g_debug_drop_copy.load() ? 1 : 0;
    p.S = S;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.G = Hq / Hkv;
    p.max_blocks = max_blocks;
    p.num_pages = num_pages;
    p.max_chunks = max_chunks;
    p.scale_log2 = scale * attn::kLog2e;
    const bool step = T > 1;
    if (step) {
        if ((st = ensure_smem(attn::decode_split_kernel<D, true>, C::SMEM_BYTES, dev)) != ATTN_OK) return st;
        attn::decode_split_kernel<D, true><<<dim3(max_chunks, Hkv * p.mtiles, S), attn::kDecodeThreads, C::SMEM_BYTES,
                                             stream>>>(tk, tv, p);
    } else {
        if ((st = ensure_smem(attn::decode_split_kernel<D, false>, C::SMEM_BYTES, dev)) != ATTN_OK) return st;
        attn::decode_split_kernel<D, false><<<dim3(max_chunks, Hkv, S), attn::kDecodeThreads, C::SMEM_BYTES, stream>>>(
            tk, tv, p);
    }
    CUDA_TRY(cudaGetLastError());
    const long long warps = static_cast<long long>(S) * T * Hq;
    attn::decode_merge_kernel<D><<<static_cast<unsigned>((warps * 32 + 127) / 128), 128, 0, stream>>>(p);
    CUDA_TRY(cudaGetLastError());
    return ATTN_OK;
}

struct BwdLayout {
    size_t vec, dqacc, qrot, krot, total;  // byte offsets within the workspace
};

BwdLayout bwd_layout(int B, int Hq, int Hkv, int N, int D, bool rope) {
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    const size_t npad = static_cast<size_t>((N + 127) / 128) * 128;
    BwdLayout L{};
    L.vec = 0;
    L.dqacc = up(static_cast<size_t>(B) * Hq * npad * 2 * sizeof(float));
    L.qrot = L.dqacc + up(static_cast<size_t>(B) * Hq * npad * D * sizeof(float));
    L.krot = L.qrot + (rope ? up(static_cast<size_t>(B) * Hq * N * D * 2) : 0);
    L.total = L.krot + (rope ? up(static_cast<size_t>(B) * Hkv * N * D * 2) : 0);
    return L;
}

template <int D>
attn_status launch_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                       void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int causal, int window,
                       float rope_base, float scale, void* ws, cudaStream_t stream, int dev) {
    using C = attn::BwdCfg<D>;
    const bool rope = rope_base > 0.f;
    const BwdLayout L = bwd_layout(B, Hq, Hkv, N, D, rope);
    uint8_t* w = static_cast<uint8_t*>(ws);
    attn::BwdParams p{};
    p.o = static_cast<const __nv_bfloat16*>(o);
    p.dout = static_cast<const __nv_bfloat16*>(dout);
    p.lse = lse;
    p.vec = reinterpret_cast<float*>(w + L.vec);
    p.dq = static_cast<__nv_bfloat16*>(dq);
    p.dqacc = reinterpret_cast<float*>(w + L.dqacc);
    p.dk = static_cast<__nv_bfloat16*>(dk);
    p.dv = static_cast<__nv_bfloat16*>(dv);
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.N = N;
    p.ntiles = (N + 127) / 128;
    p.causal = causal;
    p.window = window > 0 ? window : 0;
    p.scale = scale;
    p.scale_log2 = scale * attn::kLog2e;
    p.debug_drop_copy = g_debug_drop_copy.load() ? 1 : 0;
    int sms = 148;
    CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    const void* q_use = q;
    const void* k_use = k;
    if (rope) {
        const float2* table = nullptr;
        attn_status st = rope_table(dev, static_cast<double>(rope_base), D, N, &table);
        if (st != ATTN_OK) return st;
        const double2* table64 = nullptr;
        st = rope_table64(dev, static_cast<double>(rope_base), D, N, &table64);
        if (st != ATTN_OK) return st;
        p.rope = table;
        void* qr = w + L.qrot;
        void* kr = w + L.krot;
        st = launch_rope_rows<D>(false, q, qr, static_cast<long long>(B) * Hq, k, kr, static_cast<long long>(B) * Hkv,
                                 table64, N, sms, stream);
        if (st != ATTN_OK) return st;
        q_use = qr;
        k_use = kr;
    }
    const long long vec_rows = static_cast<long long>(B) * Hq * p.ntiles * 128;
    const long long prep_blocks = (vec_rows / (256 / 32 * (32 / (D / 8)))) + 1;
    attn::bwd_prep_kernel<D><<<static_cast<unsigned>(prep_blocks < 16LL * sms ? prep_blocks : 16LL * sms), 256, 0,
                               stream>>>(p);
    CUDA_TRY(cudaGetLastError());
    CUtensorMap tq, tk, tv, tdo, tdq;
    attn_status st;
    if ((st = make_map_3d(&tq, q_use, D, N, static_cast<uint64_t>(B) * Hq, 128)) != ATTN_OK) return st;
    if ((st = make_map_3d(&tk, k_use, D, N, static_cast<uint64_t>(B) * Hkv, 128)) != ATTN_OK) return st;
    if ((st = make_map_3d(&tv, v, D, N, static_cast<uint64_t>(B) * Hkv, 128)) != ATTN_OK) return st;
    if ((st = make_map_3d(&tdo, dout, D, N, static_cast<uint64_t>(B) * Hq, 128)) != ATTN_OK) return st;
    if ((st = make_map_2d_f32(&tdq, p.dqacc, D, static_cast<uint64_t>(B) * Hq * p.ntiles * 128)) != ATTN_OK) return st;
    if ((st = ensure_smem(attn::attn_bwd_kernel<D>, C::SMEM_BYTES, dev)) != ATTN_OK) return st;
    // one-dimensional grid, key tile index slowest (the longest causal walks start first)
    const unsigned nt = static_cast<unsigned>(p.ntiles);
    attn::attn_bwd_kernel<D><<<nt * static_cast<unsigned>(B * Hkv), C::THREADS, C::SMEM_BYTES, stream>>>(
        tq, tk, tv, tdo, tdq, p);
    CUDA_TRY(cudaGetLastError());
    const long long dq_threads = static_cast<long long>(B) * Hq * N * (D / 8);
    const long long dq_blocks = (dq_threads + 255) / 256;
    attn::bwd_dq_store_kernel<D><<<static_cast<unsigned>(dq_blocks < 16LL * sms ? dq_blocks : 16LL * sms), 256, 0,
                                   stream>>>(p);
    CUDA_TRY(cudaGetLastError());
    return ATTN_OK;
}

// Forgets the cached device addresses of the no-alloc decode's array (defined with it below).
void noalloc_forget();

}  // namespace

extern "C" {

attn_status attn_fwd_pos(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                         int N, int D, int causal, int window, float rope_base, int rope_half_split,
                         float rope_pos_scale, float rope_ntk_factor, const float* alibi_slopes, float scale,
                         void* stream) {
    g_last_error.clear();
    if (!q || !k || !v || !o) return fail(ATTN_ERR_INVALID_ARG, "q, k, v and o must be non-NULL");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (lse && !aligned16(lse)))
        return fail(ATTN_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (alibi_slopes && (reinterpret_cast<uintptr_t>(alibi_slopes) & 3u))
        return fail(ATTN_ERR_INVALID_ARG, "alibi_slopes must be 4-byte aligned");
    if (B < 1 || Hq < 1 || Hkv < 1 || N < 1) return fail(ATTN_ERR_INVALID_ARG, "B, Hq, Hkv, N must be >= 1");
    if (Hq % Hkv != 0) return fail(ATTN_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
    if (causal != 0 && causal != 1) return fail(ATTN_ERR_INVALID_ARG, "causal must be 0 or 1");
    if (window > 0 && !causal) return fail(ATTN_ERR_INVALID_ARG, "a sliding window requires causal = 1");
    if (alibi_slopes && !causal) return fail(ATTN_ERR_INVALID_ARG, "ALiBi requires causal = 1");
    if (rope_half_split != 0 && rope_half_split != 1) return fail(ATTN_ERR_INVALID_ARG, "rope_half_split must be 0 or 1");
    if (!std::isfinite(scale) || !std::isfinite(rope_base)) return fail(ATTN_ERR_INVALID_ARG, "scale and rope_base must be finite");
    if (!(std::isfinite(rope_pos_scale) && rope_pos_scale > 0.f) || !(std::isfinite(rope_ntk_factor) && rope_ntk_factor > 0.f))
        return fail(ATTN_ERR_INVALID_ARG, "rope_pos_scale and rope_ntk_factor must be finite and > 0");
    if (D != 64 && D != 128) return fail(ATTN_ERR_UNSUPPORTED, "head dim %d not supported (64 or 128)", D);
    if (static_cast<long long>(B) * Hq * ((N + 255) / 256) > 0x7fffffffLL)
        return fail(ATTN_ERR_UNSUPPORTED, "too many 256-query work items");
    if (static_cast<double>(B) * Hq * N * D * 2 >= 1099511627776.0)
        return fail(ATTN_ERR_UNSUPPORTED, "tensor larger than 1 TiB");
    if (scale <= 0.f) scale = 1.0f / std::sqrt(static_cast<float>(D));
    int dev = 0;
    CUDA_TRY(cudaGetDevice(&dev));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    PosVariant pv;
    pv.half_split = rope_half_split;
    pv.pos_scale = rope_pos_scale;
    pv.ntk = rope_ntk_factor;
    pv.alibi = alibi_slopes;
    if (D == 64) return launch_fwd<64>(q, k, v, o, lse, B, Hq, Hkv, N, causal, window, rope_base, scale, s, dev, pv);
    return launch_fwd<128>(q, k, v, o, lse, B, Hq, Hkv, N, causal, window, rope_base, scale, s, dev, pv);
}

attn_status attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                         int N, int D, int causal, int window, float descale_q, float descale_k, float descale_v,
                         float scale, void* stream) {
    g_last_error.clear();
    if (!q || !k || !v || !o) return fail(ATTN_ERR_INVALID_ARG, "q, k, v and o must be non-NULL");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (lse && !aligned16(lse)))
        return fail(ATTN_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (B < 1 || Hq < 1 || Hkv < 1 || N < 1) return fail(ATTN_ERR_INVALID_ARG, "B, Hq, Hkv, N must be >= 1");
    if (Hq % Hkv != 0) return fail(ATTN_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
    if (causal != 0 && causal != 1) return fail(ATTN_ERR_INVALID_ARG, "causal must be 0 or 1");
    if (window > 0 && !causal) return fail(ATTN_ERR_INVALID_ARG, "a sliding window requires causal = 1");
    if (!std::isfinite(scale)) return fail(ATTN_ERR_INVALID_ARG, "scale must be finite");
    if (!(std::isfinite(descale_q) && descale_q > 0.f) || !(std::isfinite(descale_k) && descale_k > 0.f) ||
        !(std::isfinite(descale_v) && descale_v > 0.f))
        return fail(ATTN_ERR_INVALID_ARG, "descale factors must be finite and > 0");
    if (D != 128) return fail(ATTN_ERR_UNSUPPORTED, "the FP8 path supports head dim 128, got %d", D);
    if (static_cast<long long>(B) * Hq * ((N + 255) / 256) > 0x7fffffffLL)
        return fail(ATTN_ERR_UNSUPPORTED, "too many 256-query work items");
    if (static_cast<double>(B) * Hq * N * D * 2 >= 1099511627776.0)
        return fail(ATTN_ERR_UNSUPPORTED, "tensor larger than 1 TiB");
    if (scale <= 0.f) scale = 1.0f / std::sqrt(static_cast<float>(D));
    int dev = 0;
    CUDA_TRY(cudaGetDevice(&dev));
    return launch_fwd_fp8(q, k, v, o, lse, B, Hq, Hkv, N, causal, window, scale * descale_q * descale_k, descale_v,
                          static_cast<cudaStream_t>(stream), dev);
}

attn_status attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                     int N, int D, int causal, int window, float rope_base, float scale, void* stream) {
    return attn_fwd_pos(q, k, v, o, lse, B, Hq, Hkv, N, D, causal, window, rope_base, 0, 1.f, 1.f, nullptr, scale,
                        stream);
}

size_t attn_bwd_workspace_size(int B, int Hq, int Hkv, int N, int D, float rope_base) {
    if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || D < 1) return 0;
    return bwd_layout(B, Hq, Hkv, N, D, rope_base > 0.f).total;
}

attn_status attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                     void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int D, int causal, int window,
                     float rope_base, float scale, void* workspace, size_t workspace_bytes, void* stream) {
    g_last_error.clear();
    if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !workspace)
        return fail(ATTN_ERR_INVALID_ARG, "q, k, v, o, lse, dout, dq, dk, dv and workspace must be non-NULL");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv) || !aligned16(workspace) || (reinterpret_cast<uintptr_t>(lse) & 3u))
        return fail(ATTN_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned (lse 4-byte)");
    if (B < 1 || Hq < 1 || Hkv < 1 || N < 1) return fail(ATTN_ERR_INVALID_ARG, "B, Hq, Hkv, N must be >= 1");
    if (Hq % Hkv != 0) return fail(ATTN_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
    if (causal != 0 && causal != 1) return fail(ATTN_ERR_INVALID_ARG, "causal must be 0 or 1");
    if (window > 0 && !causal) return fail(ATTN_ERR_INVALID_ARG, "a sliding window requires causal = 1");
    if (!std::isfinite(scale) || !std::isfinite(rope_base)) return fail(ATTN_ERR_INVALID_ARG, "scale and rope_base must be finite");
    if (D != 64 && D != 128) return fail(ATTN_ERR_UNSUPPORTED, "head dim %d not supported (64 or 128)", D);
    if (static_cast<double>(B) * Hq * ((N + 127) / 128) * 128 >= 2147483648.0)
        return fail(ATTN_ERR_UNSUPPORTED, "too many query rows: B * Hq * ceil(N/128) * 128 must be < 2^31");
    if (static_cast<double>(B) * Hq * N * D * 2 >= 1099511627776.0) return fail(ATTN_ERR_UNSUPPORTED, "tensor larger than 1 TiB");
    const size_t need = attn_bwd_workspace_size(B, Hq, Hkv, N, D, rope_base);
    if (workspace_bytes < need)
        return fail(ATTN_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", workspace_bytes, need);
    if (scale <= 0.f) scale = 1.0f / std::sqrt(static_cast<float>(D));
    int dev = 0;
    CUDA_TRY(cudaGetDevice(&dev));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (D == 64)
        return launch_bwd<64>(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, N, causal, window, rope_base, scale,
                              workspace, s, dev);
    return launch_bwd<128>(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, N, causal, window, rope_base, scale,
                           workspace, s, dev);
}

size_t attn_decode_workspace_size(int num_seqs, int max_blocks_per_seq, int page_size, int Hq, int D) {
    if (num_seqs < 1 || max_blocks_per_seq < 1 || page_size < 1 || Hq < 1 || D < 1) return 0;
    const size_t rows = static_cast<size_t>(num_seqs) * Hq * decode_chunks(max_blocks_per_seq);
    const size_t bytes = rows * (static_cast<size_t>(D) + 2) * sizeof(float);
    return (bytes + 255) / 256 * 256;
}

attn_status attn_decode_paged(const void* q, const void* k_pages, const void* v_pages, const int32_t* block_table,
                              const int32_t* seq_lens, int num_seqs, int max_blocks_per_seq, int num_pages,
                              int page_size, int Hq, int Hkv, int D, float scale, void* o, float* lse,
                              void* workspace, size_t workspace_bytes, void* stream) {
    g_last_error.clear();
    if (!q || !k_pages || !v_pages || !block_table || !seq_lens || !o || !workspace)
        return fail(ATTN_ERR_INVALID_ARG, "q, k_pages, v_pages, block_table, seq_lens, o and workspace must be non-NULL");
    if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(o) || !aligned16(workspace) ||
        (reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u) ||
        (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
        return fail(ATTN_ERR_INVALID_ARG, "misaligned pointer (tensors 16-byte, int32/fp32 arrays 4-byte)");
    if (num_seqs < 1 || max_blocks_per_seq < 1 || num_pages < 1 || page_size < 1 || Hq < 1 || Hkv < 1)
        return fail(ATTN_ERR_INVALID_ARG, "sizes must be >= 1");
    if (Hq % Hkv != 0) return fail(ATTN_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
    if (!std::isfinite(scale)) return fail(ATTN_ERR_INVALID_ARG, "scale must be finite");
    if (page_size != attn::kPageSize) return fail(ATTN_ERR_UNSUPPORTED, "page_size %d not supported (16)", page_size);
    if (D != 64 && D != 128) return fail(ATTN_ERR_UNSUPPORTED, "head dim %d not supported (64 or 128)", D);
    if (Hq / Hkv > 16) return fail(ATTN_ERR_UNSUPPORTED, "more than 16 query heads per KV head");
    if (num_seqs > 65535 || Hkv > 65535) return fail(ATTN_ERR_UNSUPPORTED, "num_seqs or Hkv too large for the grid");
    if (static_cast<double>(num_pages) * Hkv * page_size * D * 2 >= 1099511627776.0)
        return fail(ATTN_ERR_UNSUPPORTED, "KV pool larger than 1 TiB");
    const size_t need = attn_decode_workspace_size(num_seqs, max_blocks_per_seq, page_size, Hq, D);
    if (workspace_bytes < need)
        return fail(ATTN_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", workspace_bytes, need);
    if (scale <= 0.f) scale = 1.0f / std::sqrt(static_cast<float>(D));
    int dev = 0;
    CUDA_TRY(cudaGetDevice(&dev));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (D == 64)
        return launch_decode<64>(q, k_pages, v_pages, block_table, seq_lens, num_seqs, 1, max_blocks_per_seq,
                                 num_pages, Hq, Hkv, scale, o, lse, workspace, s, dev);
    return launch_decode<128>(q, k_pages, v_pages, block_table, seq_lens, num_seqs, 1, max_blocks_per_seq,
                              num_pages, Hq, Hkv, scale, o, lse, workspace, s, dev);
}

// Partial states of the split (as attn_decode_workspace_size, per new token), then the rotated
// queries (bf16).
size_t step_partials_bytes(int num_seqs, int q_len, int max_blocks_per_seq, int Hq, int D) {
    const size_t rows = static_cast<size_t>(num_seqs) * q_len * Hq * decode_chunks(max_blocks_per_seq);
    return (rows * (static_cast<size_t>(D) + 2) * sizeof(float) + 255) / 256 * 256;
}

size_t attn_decode_step_workspace_size(int num_seqs, int q_len, int max_blocks_per_seq, int page_size, int Hq, int D) {
    if (num_seqs < 1 || q_len < 1 || max_blocks_per_seq < 1 || page_size < 1 || Hq < 1 || D < 1) return 0;
    const size_t qrot = (static_cast<size_t>(num_seqs) * q_len * Hq * D * 2 + 255) / 256 * 256;
    return step_partials_bytes(num_seqs, q_len, max_blocks_per_seq, Hq, D) + qrot;
}

attn_status attn_decode_step(const void* q, const void* k_new, const void* v_new, void* k_pages, void* v_pages,
                             const int32_t* block_table, const int32_t* seq_lens, int num_seqs, int q_len,
                             int max_blocks_per_seq, int num_pages, int page_size, int Hq, int Hkv, int D,
                             float rope_base, float scale, void* o, float* lse, void* workspace,
                             size_t workspace_bytes, void* stream) {
    g_last_error.clear();
    if (!q || !k_pages || !v_pages || !block_table || !seq_lens || !o || !workspace)
        return fail(ATTN_ERR_INVALID_ARG, "q, k_pages, v_pages, block_table, seq_lens, o and workspace must be non-NULL");
    if ((k_new == nullptr) != (v_new == nullptr))
        return fail(ATTN_ERR_INVALID_ARG, "k_new and v_new must both be given or both be NULL");
    if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(o) || !aligned16(workspace) ||
        (k_new && (!aligned16(k_new) || !aligned16(v_new))) ||
        (reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u) ||
        (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
        return fail(ATTN_ERR_INVALID_ARG, "misaligned pointer (tensors 16-byte, int32/fp32 arrays 4-byte)");
    if (num_seqs < 1 || q_len < 1 || max_blocks_per_seq < 1 || num_pages < 1 || page_size < 1 || Hq < 1 || Hkv < 1)
        return fail(ATTN_ERR_INVALID_ARG, "sizes must be >= 1");
    if (Hq % Hkv != 0) return fail(ATTN_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
    if (!std::isfinite(scale) || !std::isfinite(rope_base)) return fail(ATTN_ERR_INVALID_ARG, "scale and rope_base must be finite");
    if (page_size != attn::kPageSize) return fail(ATTN_ERR_UNSUPPORTED, "page_size %d not supported (16)", page_size);
    if (D != 64 && D != 128) return fail(ATTN_ERR_UNSUPPORTED, "head dim %d not supported (64 or 128)", D);
    if (Hq / Hkv > 16) return fail(ATTN_ERR_UNSUPPORTED, "more than 16 query heads per KV head");
    if (q_len > 64) return fail(ATTN_ERR_UNSUPPORTED, "q_len %d above 64 new tokens per sequence", q_len);
    if (num_seqs > 65535 || static_cast<long long>(Hkv) * ((Hq / Hkv * q_len + 15) / 16) > 65535)
        return fail(ATTN_ERR_UNSUPPORTED, "num_seqs or Hkv * row tiles too large for the grid");
    if (static_cast<double>(num_pages) * Hkv * page_size * D * 2 >= 1099511627776.0)
        return fail(ATTN_ERR_UNSUPPORTED, "KV pool larger than 1 TiB");
    const size_t need = attn_decode_step_workspace_size(num_seqs, q_len, max_blocks_per_seq, page_size, Hq, D);
    if (workspace_bytes < need)
        return fail(ATTN_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", workspace_bytes, need);
    if (scale <= 0.f) scale = 1.0f / std::sqrt(static_cast<float>(D));
    int dev = 0;
    CUDA_TRY(cudaGetDevice(&dev));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const double2* table = nullptr;
    if (rope_base > 0.f) {
        attn_status st = rope_table64(dev, static_cast<double>(rope_base), D, max_blocks_per_seq * page_size, &table);
        if (st != ATTN_OK) return st;
    }
    // rotated queries live after the partial states
    void* q_rot = table != nullptr ? static_cast<uint8_t*>(workspace) +
                                         step_partials_bytes(num_seqs, q_len, max_blocks_per_seq, Hq, D)
                                   : nullptr;
    attn_status st = D == 64 ? launch_step_prep<64>(q, q_rot, k_new, v_new, k_pages, v_pages, block_table, seq_lens,
                                                     num_seqs, q_len, max_blocks_per_seq, num_pages, Hq, Hkv, table, s)
                             : launch_step_prep<128>(q, q_rot, k_new, v_new, k_pages, v_pages, block_table, seq_lens,
                                                      num_seqs, q_len, max_blocks_per_seq, num_pages, Hq, Hkv, table, s);
    if (st != ATTN_OK) return st;
    const void* q_use = q_rot != nullptr ? q_rot : q;
    if (D == 64)
        return launch_decode<64>(q_use, k_pages, v_pages, block_table, seq_lens, num_seqs, q_len, max_blocks_per_seq,
                                 num_pages, Hq, Hkv, scale, o, lse, workspace, s, dev);
    return launch_decode<128>(q_use, k_pages, v_pages, block_table, seq_lens, num_seqs, q_len, max_blocks_per_seq,
                              num_pages, Hq, Hkv, scale, o, lse, workspace, s, dev);
}

attn_status attn_get_device_status(void* stream, int* flags_out) {
    g_last_error.clear();
    if (!flags_out) return fail(ATTN_ERR_INVALID_ARG, "flags_out must be non-NULL");
    *flags_out = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned int word = 0;
    CUDA_TRY(cudaMemcpyFromSymbolAsync(&word, attn::g_attn_status, sizeof word, 0, cudaMemcpyDeviceToHost, s));
    CUDA_TRY(cudaStreamSynchronize(s));
    if (word) {
        const unsigned int zero = 0;
        CUDA_TRY(cudaMemcpyToSymbolAsync(attn::g_attn_status, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, s));
        CUDA_TRY(cudaStreamSynchronize(s));
    }
    *flags_out = static_cast<int>(word);
    if (word & attn::kStatusTimeout) return fail(ATTN_ERR_TIMEOUT, "a device-side wait timed out (flags 0x%x)", word);
    if (word) return fail(ATTN_ERR_DEVICE_CHECK, "a device-side check fired (flags 0x%x)", word);
    return ATTN_OK;
}

void attn_debug_drop_copy(int enable) { g_debug_drop_copy.store(enable != 0); }

const char* attn_last_error(void) { return g_last_error.c_str(); }

const char* attn_version(void) { return ATTN_VERSION_STRING; }

void attn_shutdown(void) {
    std::lock_guard<std::mutex> lock(g_cache_mu);
    int cur = 0;
    const bool have_dev = cudaGetDevice(&cur) == cudaSuccess;
    auto release = [](const DevBuf& b) {
        if (b.ptr && cudaSetDevice(b.dev) == cudaSuccess) cudaFree(b.ptr);
    };
    for (auto& kv : g_rope_tables) release(kv.second.first);
    for (auto& kv : g_key_scratch) release(kv.second);
    if (have_dev) cudaSetDevice(cur);
    g_rope_tables.clear();
    g_key_scratch.clear();
    noalloc_forget();
}

}  // extern "C"

// ------------------------------------------------------------------ decode without allocation
// Some callers cannot allocate device memory when they call in: a plugin hosted by a framework
// that owns the device's memory pool and hands out no scratch buffers, or a serving loop that
// cannot afford cudaMalloc's implicit device-wide synchronisation. For them the split-KV decode
// runs with its partial states in this fixed array instead of a caller workspace. Every GPU that
// loads the library holds the array until the process exits.
namespace {

constexpr size_t kNoAllocScratchBytes = ATTN_DECODE_NOALLOC_MAX_BYTES;  // 40 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {};  // device address of g_noalloc_scratch, per device

// Host code must not use g_noalloc_scratch's name as an address (on the host it is only a
// stand-in); the device address is looked up once per device with that device current.
attn_status noalloc_scratch(int dev, void** out) {
    if (dev < 0 || dev >= 64) return fail(ATTN_ERR_CUDA, "device index %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr)
            return fail(ATTN_ERR_CUDA, "cudaGetSymbolAddress(no-alloc scratch): %s", cudaGetErrorString(e));
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return ATTN_OK;
}

void noalloc_forget() {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    for (auto& ptr : g_noalloc_ptr) ptr = nullptr;
}

}  // namespace

extern "C" attn_status attn_decode_paged_noalloc(const void* q, const void* k_pages, const void* v_pages,
                                                 const int32_t* block_table, const int32_t* seq_lens, int num_seqs,
                                                 int max_blocks_per_seq, int num_pages, int page_size, int Hq,
                                                 int Hkv, int D, float scale, void* o, float* lse, void* stream) {
    g_last_error.clear();
    if (num_seqs < 1 || max_blocks_per_seq < 1 || page_size < 1 || Hq < 1 || D < 1)
        return fail(ATTN_ERR_INVALID_ARG, "sizes must be >= 1");
    const size_t need = attn_decode_workspace_size(num_seqs, max_blocks_per_seq, page_size, Hq, D);
    if (need > kNoAllocScratchBytes)
        return fail(ATTN_ERR_INVALID_ARG,
                    "decode needs %zu bytes of scratch, above the no-alloc limit of %zu bytes (40 MiB); "
                    "use attn_decode_paged with a caller workspace",
                    need, kNoAllocScratchBytes);
    int dev = 0;
    CUDA_TRY(cudaGetDevice(&dev));
    void* scratch = nullptr;
    const attn_status st = noalloc_scratch(dev, &scratch);
    if (st != ATTN_OK) return st;
    // Same checks and kernels as attn_decode_paged; the split kernel writes every partial state
    // the merge reads within the call, so nothing in the scratch has to start at zero.
    return attn_decode_paged(q, k_pages, v_pages, block_table, seq_lens, num_seqs, max_blocks_per_seq, num_pages,
                             page_size, Hq, Hkv, D, scale, o, lse, scratch, kNoAllocScratchBytes, stream);
}
