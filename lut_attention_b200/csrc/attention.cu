// Decode attention after the LUT scores: for query head h*G + g,
//     out[h*G + g, :] = sum_t softmax(s[h*G + g, :])_t * V[h, t, :]
// The pages define the scores (AXELRAM, arXiv 2604.02638, abstract: scores read
// straight from the stored indices); the softmax over a query's scores and the
// weighted sum of the value rows is the attention those scores feed.  Values
// are read as stored (fp32, fp16 or bf16), not quantized.
//
// Split over keys, two kernels:
//   partial : grid (splits, KV heads); a CTA takes a chunk of 4096/G keys of one
//             KV head and its G (padded to 1, 2, 4 or 8) query heads: the chunk's
//             scores are staged in shared memory with their maxima m_g and turned
//             into weights exp(s - m_g) and sums l_g once; then every warp walks
//             keys (one value row per warp step, d/32 elements per lane)
//             accumulating weight * V; the warps' sums are added in shared
//             memory in warp order and (m, l, o) written to the workspace.
//   combine : one CTA per query head merges the splits,
//             out = sum_c e^(m_c - M) o_c / sum_c e^(m_c - M) l_c,  M = max_c m_c.
// The value rows are the traffic (2d bytes per key in bf16); both kernels are
// plain CUDA-core code.
#include <mutex>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "axr_internal.cuh"

namespace axr {

// Fixed scratch for the partial sums of axr_attention_static, for callers that
// cannot supply device memory of their own.  Part of the module image: it exists
// once per device from the time the library's kernels are loaded there, and
// every call of that entry point on the device uses the same bytes.
constexpr int64_t kStaticScratchBytes = static_cast<int64_t>(16) << 20;
static __device__ __align__(256) float g_static_scratch[kStaticScratchBytes / sizeof(float)];
namespace {

constexpr int kChunkScores = 4096;    // scores staged per CTA (16 KB): chunk = 4096 / G keys
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

// query heads padded to the kernel's G (1, 2, 4 or 8)
__host__ __device__ constexpr int padded_group(int group)
{
    return group <= 1 ? 1 : group <= 2 ? 2 : group <= 4 ? 4 : 8;
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// E consecutive elements of a value row (16-byte pieces where the row allows)
template <typename T, int E>
__device__ __forceinline__ void load_values(const T *src, float (&v)[E])
{
    constexpr int kBytes = E * static_cast<int>(sizeof(T));
    if constexpr (kBytes % 16 == 0) {
        T buf[E];
#pragma unroll
        for (int i = 0; i < kBytes / 16; ++i)
            reinterpret_cast<uint4 *>(buf)[i] = __ldcs(reinterpret_cast<const uint4 *>(src) + i);
#pragma unroll
        for (int e = 0; e < E; ++e) v[e] = to_f32<T>(buf[e]);
    } else if constexpr (kBytes == 8) {
        T buf[E];
        *reinterpret_cast<uint2 *>(buf) = __ldcs(reinterpret_cast<const uint2 *>(src));
#pragma unroll
        for (int e = 0; e < E; ++e) v[e] = to_f32<T>(buf[e]);
    } else {
#pragma unroll
        for (int e = 0; e < E; ++e) v[e] = to_f32<T>(src[e]);
    }
}

struct AttnParams {
    const float *scores;       // (heads*group, n)
    const void *V;             // (heads, n, D)
    float *part;               // (heads, splits, G, D + 2): o[D], m, l
    float *out;                // (heads*group, D)
    int n;
    int group;
    int splits;
    AXR_DEBUG_ONLY(dbg::Span sp_scores, sp_V, sp_part, sp_out;)
};

// partial sums of one chunk of keys for the query heads of one KV head
template <int D, int G, typename T>
__global__ void __launch_bounds__(kThreads) attention_partial_kernel(const AttnParams p)
{
    constexpr int E = D / 32;                  // value elements per lane
    constexpr int C = kChunkScores / G;        // keys per CTA
    __shared__ float s_w[G][C];                // scores, then weights exp(s - m)
    __shared__ float s_red[kWarps][G];
    __shared__ float s_m[G], s_l[G];
    __shared__ float s_o[G][D];
    const int h = blockIdx.y, c = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = c * C;
    const int len = min(C, p.n - t0);

    // 1. stage the chunk's scores and take each query's maximum
    float red[G];
#pragma unroll
    for (int g = 0; g < G; ++g) red[g] = -INFINITY;
    for (int i = threadIdx.x; i < len; i += kThreads) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float *src = p.scores + (static_cast<int64_t>(h) * p.group + g) * p.n + t0 + i;
            const float v = (g < p.group && AXR_IN(p.sp_scores, src, 4)) ? *src : 0.0f;
            s_w[g][i] = v;
            red[g] = fmaxf(red[g], v);
        }
    }
    for (int i = threadIdx.x; i < G * D; i += kThreads) (&s_o[0][0])[i] = 0.0f;
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) red[g] = fmaxf(red[g], __shfl_xor_sync(0xffffffffu, red[g], o));
        if (lane == 0) s_red[warp][g] = red[g];
    }
    __syncthreads();
    if (threadIdx.x < G) {
        float m = -INFINITY;
        for (int w = 0; w < kWarps; ++w) m = fmaxf(m, s_red[w][threadIdx.x]);
        s_m[threadIdx.x] = m;
    }
    __syncthreads();

    // 2. weights once per (query, key), and their sums
    float m[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m[g] = s_m[g];
        red[g] = 0.0f;
    }
    for (int i = threadIdx.x; i < len; i += kThreads) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float w = (g < p.group) ? expf(s_w[g][i] - m[g]) : 0.0f;
            s_w[g][i] = w;
            red[g] += w;
        }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) red[g] += __shfl_xor_sync(0xffffffffu, red[g], o);
    }
    __syncthreads();                          // s_red reuse, weights complete
#pragma unroll
    for (int g = 0; g < G; ++g)
        if (lane == 0) s_red[warp][g] = red[g];
    __syncthreads();
    if (threadIdx.x < G) {
        float l = 0.0f;
        for (int w = 0; w < kWarps; ++w) l += s_red[w][threadIdx.x];
        s_l[threadIdx.x] = l;
    }

    // 3. weighted value rows: warp w takes keys w, w + 8, ...; lane owns elements
    //    lane*E .. lane*E + E - 1 of every row
    float acc[G][E];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < E; ++e) acc[g][e] = 0.0f;
    const T *Vh = static_cast<const T *>(p.V) + (static_cast<int64_t>(h) * p.n + t0) * D + lane * E;
    for (int i = warp; i < len; i += kWarps) {
        float v[E];
        const T *src = Vh + static_cast<int64_t>(i) * D;
        if (AXR_IN(p.sp_V, src, E * sizeof(T))) {
            load_values<T, E>(src, v);
        } else {
#pragma unroll
            for (int e = 0; e < E; ++e) v[e] = 0.0f;
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float w = s_w[g][i];
#pragma unroll
            for (int e = 0; e < E; ++e) acc[g][e] = fmaf(w, v[e], acc[g][e]);
        }
    }
    // the warps' sums, added in warp order (deterministic)
    for (int w = 0; w < kWarps; ++w) {
        if (warp == w) {
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int e = 0; e < E; ++e) s_o[g][lane * E + e] += acc[g][e];
        }
        __syncthreads();
    }
    float *part = p.part + (static_cast<int64_t>(h) * p.splits + c) * G * (D + 2);
    for (int i = threadIdx.x; i < G * D; i += kThreads) {
        float *dst = part + (i / D) * (D + 2) + i % D;
        if (AXR_IN(p.sp_part, dst, 4)) *dst = s_o[i / D][i % D];
    }
    if (threadIdx.x < G) {
        float *dst = part + threadIdx.x * (D + 2) + D;
        if (AXR_IN(p.sp_part, dst, 8)) {
            dst[0] = s_m[threadIdx.x];
            dst[1] = s_l[threadIdx.x];
        }
    }
}

// merge the splits of one query head (blockIdx.x = h*group + g)
template <int D, int G>
__global__ void attention_combine_kernel(const AttnParams p)
{
    const int hq = blockIdx.x;
    const int h = hq / p.group, g = hq % p.group;
    const float *part = p.part + static_cast<int64_t>(h) * p.splits * G * (D + 2) + g * (D + 2);
    float M = -INFINITY;
    for (int c = 0; c < p.splits; ++c) {
        const float *pm = part + static_cast<int64_t>(c) * G * (D + 2) + D;
        if (AXR_IN(p.sp_part, pm, 4)) M = fmaxf(M, *pm);
    }
    for (int j = threadIdx.x; j < D; j += blockDim.x) {
        float o = 0.0f, l = 0.0f;
        for (int c = 0; c < p.splits; ++c) {
            const float *pc = part + static_cast<int64_t>(c) * G * (D + 2);
            if (!AXR_IN(p.sp_part, pc + j, 4) || !AXR_IN(p.sp_part, pc + D, 8)) continue;
            const float sc = expf(pc[D] - M);
            o = fmaf(sc, pc[j], o);
            l = fmaf(sc, pc[D + 1], l);
        }
        float *dst = p.out + static_cast<int64_t>(hq) * D + j;
        if (AXR_IN(p.sp_out, dst, 4)) *dst = o / l;
    }
}

template <int D, int G, typename T>
cudaError_t launch_dgt(const AttentionArgs &a, cudaStream_t stream)
{
    static_assert(padded_group(G) == G, "G is a padded group size");
    AttnParams p;
    p.scores = a.scores;
    p.V = a.V;
    p.part = static_cast<float *>(a.workspace);
    p.out = a.out;
    p.n = static_cast<int>(a.n);
    p.group = a.group;
    p.splits = attention_splits(a.n, a.group);
    AXR_DEBUG_ONLY(const uint64_t rows_q = static_cast<uint64_t>(a.heads) * a.group;
                   p.sp_scores = dbg::span(a.scores, rows_q * a.n * sizeof(float));
                   p.sp_V = dbg::span(a.V, static_cast<uint64_t>(a.heads) * a.n * D * sizeof(T));
                   p.sp_part = dbg::span(a.workspace, attention_workspace_bytes(a.n, a.heads, a.group, D));
                   p.sp_out = dbg::span(a.out, rows_q * D * sizeof(float));)
    attention_partial_kernel<D, G, T><<<dim3(p.splits, a.heads), kThreads, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    attention_combine_kernel<D, G><<<a.heads * a.group, D < 256 ? D : 256, 0, stream>>>(p);
    return cudaGetLastError();
}

template <int D, int G>
cudaError_t launch_dg(const AttentionArgs &a, cudaStream_t stream)
{
    switch (a.vdtype) {
    case AXR_F32: return launch_dgt<D, G, float>(a, stream);
    case AXR_F16: return launch_dgt<D, G, __half>(a, stream);
    default: return launch_dgt<D, G, __nv_bfloat16>(a, stream);
    }
}

template <int D>
cudaError_t launch_d(const AttentionArgs &a, cudaStream_t stream)
{
    if (a.group <= 1) return launch_dg<D, 1>(a, stream);
    if (a.group <= 2) return launch_dg<D, 2>(a, stream);
    if (a.group <= 4) return launch_dg<D, 4>(a, stream);
    return launch_dg<D, 8>(a, stream);
}

}  // namespace

int attention_splits(int64_t n, int group)
{
    const int chunk = kChunkScores / padded_group(group);
    return static_cast<int>((n + chunk - 1) / chunk);
}

int64_t attention_workspace_bytes(int64_t n, int heads, int group, int d)
{
    return static_cast<int64_t>(heads) * attention_splits(n, group) * padded_group(group) * (d + 2) *
           static_cast<int64_t>(sizeof(float));
}

int64_t static_attention_scratch_bytes() { return kStaticScratchBytes; }

cudaError_t static_attention_scratch(void **ptr)
{
    constexpr int kMaxDevices = 64;
    static std::mutex mu;
    static void *addr[kMaxDevices] = {};      // per device, filled on its first call
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);      // with device `dev` current
        if (e != cudaSuccess) return e;
        addr[dev] = p;
    }
    *ptr = addr[dev];
    return cudaSuccess;
}

cudaError_t launch_attention(const AttentionArgs &a, cudaStream_t stream)
{
    switch (a.d) {
    case 32: return launch_d<32>(a, stream);
    case 64: return launch_d<64>(a, stream);
    case 128: return launch_d<128>(a, stream);
    case 256: return launch_d<256>(a, stream);
    default: return launch_d<512>(a, stream);
    }
}

}  // namespace axr
