// Quantize-on-write kernel (AXELRAM, arXiv 2604.02638, abstract: keys are
// transformed once on write and stored as indices into a design-time codebook).
//
// Per key row k of length D:
//   x = diag(signs) k                         sign flip
//   y = H x                                   Walsh-Hadamard (Sylvester order)
//   norm = sqrt(sum k_j^2)                    fp32, stored
//   u = y / (sqrt(D) norm)                    unit key in the rotated basis
//   idx_j = #{i : u_j > t_i}                  binary search on the boundaries
//   bit-pack idx into D*B/8 bytes, LSB-first
//
// Thread layout.  A row is split over TPR = D/E threads of one warp, E = min(D,32)
// elements each, in 8-element chunks: thread t of a row holds chunk k at elements
// j = 8t + 8*TPR*k + e (e < 8).  So one warp-wide 16-byte load instruction reads
// TPR*16 contiguous bytes of each of its rows (coalesced), the Hadamard stages on
// bits 0-2 and on the chunk bits run inside a thread, and the stages on the
// thread bits run as xor-shuffles inside the row's TPR lanes.  Each chunk's 8
// indices fill exactly B bytes of the packed row, so packing needs no exchange:
// the chunks are assembled in shared memory and leave with 16-byte stores.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "axr_internal.cuh"
#include "row_load.cuh"

namespace axr {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr unsigned kFull = 0xffffffffu;

struct QParams {
    const void *K;
    int64_t n;
    const int8_t *signs;
    uint8_t *idx;
    float *norms;
    int64_t out_stride;        // key r goes to row r * out_stride + out_offset
    int64_t out_offset;
    float bnd[kMaxLevels - 1];
    AXR_DEBUG_ONLY(dbg::Span sp_K, sp_signs, sp_idx, sp_norms;)
};

template <int D, int B, typename T>
__global__ void __launch_bounds__(kThreads) quantize_keys_kernel(QParams p)
{
    constexpr int E = D >= 32 ? 32 : D;   // elements per thread
    constexpr int TPR = D / E;            // threads per row
    constexpr int RW = 32 / TPR;          // rows per warp step
    constexpr int NCH = E / 8;            // 8-element chunks per thread
    constexpr int L = 1 << B;
    constexpr int P = D * B / 8;          // packed bytes per row
    constexpr int WBYTES = RW * P;        // packed bytes per warp step
    static_assert(WBYTES % 16 == 0 && WBYTES <= 512, "warp step must be whole 16-byte words");

    __shared__ float s_bnd[kMaxLevels];
    __shared__ __align__(16) uint8_t s_pack[kWarps][WBYTES];

    if (threadIdx.x == 0) {
#pragma unroll
        for (int i = 0; i < L - 1; ++i) s_bnd[i] = p.bnd[i];   // constant indices: p stays in param space
    }
    __syncthreads();

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int t = lane % TPR;
    const int slot = lane / TPR;

    float sg[E];
#pragma unroll
    for (int k = 0; k < NCH; ++k)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int8_t *sp = p.signs + 8 * t + 8 * TPR * k + e;
            sg[8 * k + e] = (AXR_IN(p.sp_signs, sp, 1) && *sp < 0) ? -1.0f : 1.0f;
        }

    const float sqrt_d = sqrtf(static_cast<float>(D));
    const int64_t nsteps = (p.n + RW - 1) / RW;
    uint8_t *stage = s_pack[warp];

    for (int64_t s = static_cast<int64_t>(blockIdx.x) * kWarps + warp; s < nsteps;
         s += static_cast<int64_t>(gridDim.x) * kWarps) {
        const int64_t row = s * RW + slot;
        const bool valid = row < p.n;

        float v[E];
#pragma unroll
        for (int k = 0; k < NCH; ++k) {
            const int64_t at = row * D + 8 * t + 8 * TPR * k;
            if (valid && AXR_IN(p.sp_K, static_cast<const T *>(p.K) + at, 8 * sizeof(T))) {
                Load8<T>::run(p.K, at, v + 8 * k);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) v[8 * k + e] = 0.0f;
            }
        }

        // sign flip and the squared norm
        float ss = 0.0f;
#pragma unroll
        for (int i = 0; i < E; ++i) {
            v[i] *= sg[i];
            ss = fmaf(v[i], v[i], ss);
        }
#pragma unroll
        for (int m = 1; m < TPR; m <<= 1) ss += __shfl_xor_sync(kFull, ss, m);

        // Hadamard stages held inside the thread (element bits 0-2 and the chunk bits)
#pragma unroll
        for (int h = 1; h < E; h <<= 1)
#pragma unroll
            for (int i = 0; i < E; ++i)
                if (!(i & h)) {
                    const float a = v[i], b = v[i + h];
                    v[i] = a + b;
                    v[i + h] = a - b;
                }
        // Hadamard stages across the row's threads (element bits 3 .. 3+log2(TPR)-1)
#pragma unroll
        for (int m = 1; m < TPR; m <<= 1) {
            const bool upper = (t & m) != 0;
#pragma unroll
            for (int i = 0; i < E; ++i) {
                const float o = __shfl_xor_sync(kFull, v[i], m);
                v[i] = upper ? (o - v[i]) : (v[i] + o);
            }
        }

        const float norm = sqrtf(ss);
        // a zero key has u = 0, which the search maps to 2^(B-1) - 1
        const float inv = (norm > 0.0f) ? 1.0f / (sqrt_d * norm) : 0.0f;

        // quantize (binary search on the boundaries) and pack each 8-element chunk
        uint8_t *rowstage = stage + slot * P;
#pragma unroll
        for (int k = 0; k < NCH; ++k) {
            uint32_t word = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float u = v[8 * k + e] * inv;
                int c = 0;
#pragma unroll
                for (int step = L / 2; step >= 1; step >>= 1)
                    if (u > s_bnd[c + step - 1]) c += step;
                word |= static_cast<uint32_t>(c) << (B * e);
            }
            const int off = B * (t + TPR * k);
            if constexpr (B == 4) {
                *reinterpret_cast<uint32_t *>(rowstage + off) = word;
            } else if constexpr (B == 2) {
                *reinterpret_cast<uint16_t *>(rowstage + off) = static_cast<uint16_t>(word);
            } else {
#pragma unroll
                for (int i = 0; i < B; ++i) rowstage[off + i] = static_cast<uint8_t>(word >> (8 * i));
            }
        }
        __syncwarp();

        const int64_t first = s * RW;
        const int64_t rows_here = (p.n - first < RW) ? (p.n - first) : RW;
        if (p.out_stride == 1 && p.out_offset == 0) {
            // the warp step's rows are contiguous in idx: write them out
            uint8_t *dst = p.idx + first * P;
            if (rows_here == RW) {
                if (lane < WBYTES / 16 && AXR_IN(p.sp_idx, reinterpret_cast<uint4 *>(dst) + lane, 16))
                    __stcs(reinterpret_cast<uint4 *>(dst) + lane, reinterpret_cast<const uint4 *>(stage)[lane]);
            } else {
                const int nbytes = static_cast<int>(rows_here) * P;
                for (int i = lane; i < nbytes; i += 32)
                    if (AXR_IN(p.sp_idx, dst + i, 1)) dst[i] = stage[i];
            }
        } else {
            // rows land out_stride rows apart (one key appended per cache head)
            for (int i = lane; i < static_cast<int>(rows_here) * P; i += 32) {
                const int64_t rr = first + i / P;
                uint8_t *o = p.idx + (rr * p.out_stride + p.out_offset) * P + i % P;
                if (AXR_IN(p.sp_idx, o, 1)) *o = stage[i];
            }
        }
        float *nd = p.norms + row * p.out_stride + p.out_offset;
        if (valid && t == 0 && AXR_IN(p.sp_norms, nd, 4)) __stcs(nd, norm);
        __syncwarp();
    }
}

template <int D, int B, typename T>
cudaError_t launch_typed(const QuantizeArgs &a, cudaStream_t stream)
{
    auto kernel = quantize_keys_kernel<D, B, T>;
    // resident blocks per SM (the same on every device of one model; it sizes the
    // grid, and the kernel strides over the rows, so any value is correct)
    static std::atomic<int> blocks_cached{0};
    int blocks_per_sm = blocks_cached.load(std::memory_order_relaxed);
    if (blocks_per_sm == 0) {
        int v = 0;
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, kernel, kThreads, 0);
        if (e != cudaSuccess) return e;
        blocks_per_sm = v > 0 ? v : 1;
        blocks_cached.store(blocks_per_sm, std::memory_order_relaxed);
    }
    constexpr int E = D >= 32 ? 32 : D;
    constexpr int RW = 32 / (D / E);
    const int64_t nsteps = (a.n + RW - 1) / RW;
    const int64_t want = (nsteps + kWarps - 1) / kWarps;
    const int64_t cap = static_cast<int64_t>(device_sm_count()) * blocks_per_sm;
    const int grid = static_cast<int>(want < cap ? want : cap);

    QParams p;
    p.K = a.K;
    p.n = a.n;
    p.signs = a.signs;
    p.idx = a.idx;
    p.norms = a.norms;
    p.out_stride = a.out_stride;
    p.out_offset = a.out_offset;
    for (int i = 0; i < kMaxLevels - 1; ++i) p.bnd[i] = a.cb.boundaries[i];
    AXR_DEBUG_ONLY(const int64_t rows = a.out_rows ? a.out_rows : a.n;
                   p.sp_K = dbg::span(a.K, static_cast<uint64_t>(a.n) * D * sizeof(T));
                   p.sp_signs = dbg::span(a.signs, D);
                   p.sp_idx = dbg::span(a.idx, static_cast<uint64_t>(rows) * (D * B / 8));
                   p.sp_norms = dbg::span(a.norms, static_cast<uint64_t>(rows) * sizeof(float));)
    kernel<<<grid, kThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

template <int D, int B>
cudaError_t launch_db(const QuantizeArgs &a, cudaStream_t stream)
{
    switch (a.kdtype) {
    case AXR_F32: return launch_typed<D, B, float>(a, stream);
    case AXR_F16: return launch_typed<D, B, __half>(a, stream);
    default: return launch_typed<D, B, __nv_bfloat16>(a, stream);
    }
}

template <int D>
cudaError_t launch_d(const QuantizeArgs &a, cudaStream_t stream)
{
    switch (a.b) {
    case 1: return launch_db<D, 1>(a, stream);
    case 2: return launch_db<D, 2>(a, stream);
    case 3: return launch_db<D, 3>(a, stream);
    default: return launch_db<D, 4>(a, stream);
    }
}

}  // namespace

cudaError_t launch_quantize_keys(const QuantizeArgs &a, cudaStream_t stream)
{
    switch (a.d) {
    case 8: return launch_d<8>(a, stream);
    case 16: return launch_d<16>(a, stream);
    case 32: return launch_d<32>(a, stream);
    case 64: return launch_d<64>(a, stream);
    case 128: return launch_d<128>(a, stream);
    case 256: return launch_d<256>(a, stream);
    default: return launch_d<512>(a, stream);
    }
}

}  // namespace axr
