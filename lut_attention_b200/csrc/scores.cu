// Score-on-read kernel (AXELRAM, arXiv 2604.02638, abstract: scores come from
// table lookups on the stored indices, with no inverse transform of the keys).
//
// One CTA serves one KV head h (batch folded in) and a tile of its keys.
//   prologue: q''_g = H diag(signs) q_g / D for the G query heads of h
//             (the orthonormal 1/sqrt(D) of the rotation times the attention
//             temperature 1/sqrt(D); D is a power of two, so 1/D is exact),
//             or q''_g = T q_g / sqrt(D) with the IsoQuant block rotation T
//             (arXiv 2603.28430, abstract) when the keys were written with it;
//   per key t: s_g[t] = norms[t] * sum_j q''_g[j] * c[idx_t[j]]
// The index stream of a key is read once and serves all G queries (GQA).
//
// Lane layout.  Each lane owns CL consecutive coordinates of a key (CL*B/8
// bytes of its packed row) and keeps q'' for those coordinates and all G
// queries in registers; LR = D/CL lanes cover one row, so a warp scores 32/LR
// rows per step.  A lane decodes each code once (centroid from a shared-memory
// table of 2^B entries: every entry sits in its own bank) and feeds it to G
// FMAs; the LR partial sums of a row meet in an xor-shuffle reduction.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "axr_internal.cuh"
#include "quat.cuh"

namespace axr {
namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kTile = 1024;   // keys per CTA
constexpr unsigned kFull = 0xffffffffu;

struct SParams {
    const void *q;
    int qdtype;
    const uint8_t *idx;
    const float *norms;
    int n;
    int64_t head_stride;       // rows between KV heads in idx and norms
    int group;
    const int8_t *signs;
    const float *quats;        // block rotation of the queries instead of H diag(signs), or null
    float *scores;
    float cent[kMaxLevels];
    AXR_DEBUG_ONLY(dbg::Span sp_q, sp_idx, sp_norms, sp_signs, sp_quats, sp_scores;)
};

__device__ __forceinline__ float load_q(const void *q, int dtype, int64_t i)
{
    switch (dtype) {
    case AXR_F32: return static_cast<const float *>(q)[i];
    case AXR_F16: return __half2float(static_cast<const __half *>(q)[i]);
    default: return __bfloat162float(static_cast<const __nv_bfloat16 *>(q)[i]);
    }
}

// WB bytes at p (aligned to the largest power of two dividing WB, up to 16),
// as little-endian 32-bit words; zero when !valid.
template <int WB>
__device__ __forceinline__ void load_bytes(const uint8_t *p, bool valid, uint32_t *w)
{
    constexpr int NW = (WB + 3) / 4;
#pragma unroll
    for (int i = 0; i < NW; ++i) w[i] = 0;
    if (!valid) return;
    if constexpr (WB % 16 == 0) {
#pragma unroll
        for (int i = 0; i < WB / 16; ++i) {
            const uint4 x = __ldcs(reinterpret_cast<const uint4 *>(p) + i);
            w[4 * i] = x.x; w[4 * i + 1] = x.y; w[4 * i + 2] = x.z; w[4 * i + 3] = x.w;
        }
    } else if constexpr (WB % 8 == 0) {
#pragma unroll
        for (int i = 0; i < WB / 8; ++i) {
            const uint2 x = __ldcs(reinterpret_cast<const uint2 *>(p) + i);
            w[2 * i] = x.x; w[2 * i + 1] = x.y;
        }
    } else if constexpr (WB % 4 == 0) {
#pragma unroll
        for (int i = 0; i < WB / 4; ++i) w[i] = __ldcs(reinterpret_cast<const unsigned int *>(p) + i);
    } else if constexpr (WB % 2 == 0) {
#pragma unroll
        for (int i = 0; i < WB / 2; ++i)
            w[i / 2] |= static_cast<uint32_t>(__ldcs(reinterpret_cast<const unsigned short *>(p) + i))
                        << (16 * (i % 2));
    } else {
#pragma unroll
        for (int i = 0; i < WB; ++i) w[i / 4] |= static_cast<uint32_t>(__ldcs(p + i)) << (8 * (i % 4));
    }
}

// code c (bits [c*B, c*B+B) of the little-endian word stream)
template <int B, int NW>
__device__ __forceinline__ uint32_t extract(const uint32_t *w, int c)
{
    const int o = c * B;
    const int wi = o >> 5, sh = o & 31;
    uint32_t x = w[wi] >> sh;
    if (sh + B > 32 && wi + 1 < NW) x |= w[wi + 1] << (32 - sh);
    return x & ((1u << B) - 1u);
}

template <int D, int G>
struct ScoresShape {
    static constexpr int kRawCL = (G <= 2) ? 32 : (G == 4 ? 16 : 8);
    static constexpr int kMinCL = D / 32 > 0 ? D / 32 : 1;       // at most 32 lanes per row
    static constexpr int kCL0 = kRawCL > kMinCL ? kRawCL : kMinCL;
    static constexpr int CL = kCL0 < D ? kCL0 : D;                // codes per lane
    static constexpr int LR = D / CL;                             // lanes per row
    static constexpr int RS = 32 / LR;                            // rows per warp step
};

template <int D, int B, int G>
__global__ void __launch_bounds__(kThreads) scores_kernel(SParams p)
{
    using S = ScoresShape<D, G>;
    constexpr int CL = S::CL, LR = S::LR, RS = S::RS;
    constexpr int WB = CL * B / 8;   // bytes per lane per row
    constexpr int NW = (WB + 3) / 4;
    constexpr int P = D * B / 8;
    constexpr int L = 1 << B;

    __shared__ float s_q[G][D];
    __shared__ float s_cb[kMaxLevels];

    const int h = blockIdx.y;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;

    if (threadIdx.x == 0) {
#pragma unroll
        for (int i = 0; i < L; ++i) s_cb[i] = p.cent[i];   // constant indices: p stays in param space
    }

    // prologue: rotate this KV head's queries once (fp32, in shared memory)
    for (int g = warp; g < G; g += kWarps) {
        float *sq = s_q[g];
        if (g < p.group) {
            const int64_t qrow = static_cast<int64_t>(h) * p.group + g;
            const int qb = dtype_bytes(p.qdtype);
            for (int j = lane; j < D; j += 32) {
                const int64_t qi = qrow * D + j;
                const bool flip = !p.quats && AXR_IN(p.sp_signs, p.signs + j, 1) && p.signs[j] < 0;
                const float qv =
                    AXR_IN(p.sp_q, static_cast<const char *>(p.q) + qi * qb, qb) ? load_q(p.q, p.qdtype, qi) : 0.0f;
                sq[j] = flip ? -qv : qv;
            }
        } else {
            for (int j = lane; j < D; j += 32) sq[j] = 0.0f;
        }
        __syncwarp();
        if (p.quats) {
            // q'' = T q / sqrt(D): the block rotation is orthonormal, 1/sqrt(D) is the temperature
            const float inv_sqrt_d = 1.0f / sqrtf(static_cast<float>(D));
            for (int m = lane; m < D / 4; m += 32) {
                Quat qL, qRc;
                if (AXR_IN(p.sp_quats, p.quats + 8 * m, 32)) {
                    block_quats(p.quats, m, qL, qRc);
                } else {
                    unit_quats(qL, qRc);
                }
                const Quat y = block_rotate(qL, qRc, {sq[4 * m], sq[4 * m + 1], sq[4 * m + 2], sq[4 * m + 3]});
                sq[4 * m] = y.w * inv_sqrt_d;
                sq[4 * m + 1] = y.x * inv_sqrt_d;
                sq[4 * m + 2] = y.y * inv_sqrt_d;
                sq[4 * m + 3] = y.z * inv_sqrt_d;
            }
            __syncwarp();
        } else {
            for (int hh = 1; hh < D; hh <<= 1) {
                for (int pi = lane; pi < D / 2; pi += 32) {
                    const int i = (pi / hh) * 2 * hh + (pi % hh);
                    const float a = sq[i], b = sq[i + hh];
                    sq[i] = a + b;
                    sq[i + hh] = a - b;
                }
                __syncwarp();
            }
            for (int j = lane; j < D; j += 32) sq[j] *= 1.0f / static_cast<float>(D);
            __syncwarp();
        }
    }
    __syncthreads();

    const int part = lane % LR;
    const int slot = lane / LR;
    float qr[G][CL];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int c = 0; c < CL; ++c) qr[g][c] = s_q[g][part * CL + c];

    const int n = p.n;
    const int tile0 = blockIdx.x * kTile;
    const int tile1 = (n - tile0 < kTile) ? n : tile0 + kTile;
    const uint8_t *idx_h = p.idx + static_cast<int64_t>(h) * p.head_stride * P;
    const float *norms_h = p.norms + static_cast<int64_t>(h) * p.head_stride;

    for (int r0 = tile0 + warp * RS; r0 < tile1; r0 += kWarps * RS) {
        const int r = r0 + slot;
        const bool valid = r < tile1;
        uint32_t w[NW];
        const uint8_t *src = idx_h + static_cast<int64_t>(r) * P + part * WB;
        load_bytes<WB>(src, valid && AXR_IN(p.sp_idx, src, WB), w);
        float acc[G];
#pragma unroll
        for (int g = 0; g < G; ++g) acc[g] = 0.0f;
#pragma unroll
        for (int c = 0; c < CL; ++c) {
            const float cv = s_cb[extract<B, NW>(w, c)];
#pragma unroll
            for (int g = 0; g < G; ++g) acc[g] = fmaf(qr[g][c], cv, acc[g]);
        }
#pragma unroll
        for (int m = 1; m < LR; m <<= 1)
#pragma unroll
            for (int g = 0; g < G; ++g) acc[g] += __shfl_xor_sync(kFull, acc[g], m);
        if (valid) {
            const float nk = AXR_IN(p.sp_norms, norms_h + r, 4) ? __ldg(norms_h + r) : 0.0f;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float *dst = p.scores + (static_cast<int64_t>(h) * p.group + g) * n + r;
                if (g % LR == part && g < p.group && AXR_IN(p.sp_scores, dst, 4)) __stcs(dst, nk * acc[g]);
            }
        }
    }
}

template <int D, int B, int G>
cudaError_t launch_dbg(const ScoresArgs &a, cudaStream_t stream)
{
    SParams p;
    p.q = a.q;
    p.qdtype = a.qdtype;
    p.idx = a.idx;
    p.norms = a.norms;
    p.n = static_cast<int>(a.n);
    p.head_stride = a.head_stride;
    p.group = a.group;
    p.signs = a.signs;
    p.quats = a.quats;
    p.scores = a.scores;
    for (int i = 0; i < kMaxLevels; ++i) p.cent[i] = a.cb.centroids[i];
    AXR_DEBUG_ONLY(const uint64_t rows_q = static_cast<uint64_t>(a.heads) * a.group;
                   const uint64_t rows_k = static_cast<uint64_t>(a.heads) * a.head_stride;
                   p.sp_q = dbg::span(a.q, rows_q * D * dtype_bytes(a.qdtype));
                   p.sp_idx = dbg::span(a.idx, rows_k * (D * B / 8));
                   p.sp_norms = dbg::span(a.norms, rows_k * sizeof(float));
                   p.sp_signs = dbg::span(a.signs, a.signs ? D : 0);
                   p.sp_quats = dbg::span(a.quats, a.quats ? (D / 4) * 8 * sizeof(float) : 0);
                   p.sp_scores = dbg::span(a.scores, rows_q * a.n * sizeof(float));)
    const dim3 grid(static_cast<unsigned>((a.n + kTile - 1) / kTile), static_cast<unsigned>(a.heads));
    scores_kernel<D, B, G><<<grid, kThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

template <int D, int B>
cudaError_t launch_db(const ScoresArgs &a, cudaStream_t stream)
{
    if (a.group <= 1) return launch_dbg<D, B, 1>(a, stream);
    if (a.group <= 2) return launch_dbg<D, B, 2>(a, stream);
    if (a.group <= 4) return launch_dbg<D, B, 4>(a, stream);
    return launch_dbg<D, B, 8>(a, stream);
}

template <int D>
cudaError_t launch_d(const ScoresArgs &a, cudaStream_t stream)
{
    switch (a.b) {
    case 1: return launch_db<D, 1>(a, stream);
    case 2: return launch_db<D, 2>(a, stream);
    case 3: return launch_db<D, 3>(a, stream);
    default: return launch_db<D, 4>(a, stream);
    }
}

}  // namespace

cudaError_t launch_scores(const ScoresArgs &a, cudaStream_t stream)
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
