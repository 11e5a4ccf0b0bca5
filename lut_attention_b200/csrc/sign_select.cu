// Sign-pattern choice (AXELRAM, arXiv 2604.02638, abstract: the sign pattern is
// chosen once, without gradients, among candidates on a few calibration
// samples, which removes the spikes that some patterns cause when key norms
// differ between heads).
//
// The criterion is the error of the attention logits the quantized cache gives.
// For candidate D_c and KV head h:
//     E[c][h] = mean over samples s, query heads g < G and keys t of e^2,
//     e = score_c(q, k) - q.k / sqrt(D)
//       = |k| / sqrt(D) * sum_j q'_j (c[idx_j] - u_j),      q' = H D_c q / sqrt(D),
// where u = H D_c k / (sqrt(D) |k|) is the rotated unit key and idx its codes.
// The second form holds because R = H D_c / sqrt(D) is orthonormal: q.k =
// (R q).(R k) = |k| q'.u.  It needs no exact logit and no cancellation: only the
// quantization residual c[idx] - u enters.  The chosen pattern is the candidate
// whose worst head has the smallest E, the lowest index among equal values.
//
// One CTA per (candidate, KV head) walks every calibration key of that head, so
// each E[c][h] is a fixed-order sum and the result does not depend on
// scheduling.  Per sample the CTA rotates its G queries once in shared memory
// (q' for this candidate); the keys go through the write kernel's thread layout
// (a row over D/E threads, E = min(D, 32) elements each, Walsh-Hadamard stages
// in registers and across the row's lanes), then the residuals are projected on
// the G rotated queries.  The calibration keys are read once per candidate and
// stay in L2 between candidates (cached loads).
#include <climits>
#include <cmath>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "axr_internal.cuh"
#include "row_load.cuh"

namespace axr {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr unsigned kFull = 0xffffffffu;

struct SelParams {
    const void *K;            // [samples][heads][n][D]
    const void *q;            // [samples][heads * group][D]
    int qdtype;
    const int8_t *cand;       // [C][D]
    float *errors;            // [C][heads]
    int64_t n;
    int samples;
    int heads;
    int group;
    double inv_count;         // 1 / (samples * group * n)
    float bnd[kMaxLevels - 1];
    float cent[kMaxLevels];
};

__device__ __forceinline__ float load_query(const void *q, int dtype, int64_t i)
{
    switch (dtype) {
    case AXR_F32: return static_cast<const float *>(q)[i];
    case AXR_F16: return __half2float(static_cast<const __half *>(q)[i]);
    default: return __bfloat162float(static_cast<const __nv_bfloat16 *>(q)[i]);
    }
}

template <int D, int B, typename T>
__global__ void __launch_bounds__(kThreads) sign_errors_kernel(const __grid_constant__ SelParams p)
{
    constexpr int E = D >= 32 ? 32 : D;   // elements per thread
    constexpr int TPR = D / E;            // threads per key row
    constexpr int RW = 32 / TPR;          // rows per warp step
    constexpr int NCH = E / 8;            // 8-element chunks per thread
    constexpr int L = 1 << B;

    extern __shared__ float s_q[];        // [group][D]: H D_c q of this sample's query heads
    __shared__ float s_bnd[kMaxLevels];
    __shared__ float s_cent[kMaxLevels];
    __shared__ double s_red[kWarps];

    const int c = blockIdx.x / p.heads;
    const int h = blockIdx.x % p.heads;
    const int G = p.group;
    const int8_t *dc = p.cand + static_cast<int64_t>(c) * D;

    if (threadIdx.x == 0) {
#pragma unroll
        for (int i = 0; i < L - 1; ++i) s_bnd[i] = p.bnd[i];   // constant indices: p stays in param space
#pragma unroll
        for (int i = 0; i < L; ++i) s_cent[i] = p.cent[i];
    }

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int t = lane % TPR;
    const int slot = lane / TPR;

    float sg[E];
#pragma unroll
    for (int k = 0; k < NCH; ++k)
#pragma unroll
        for (int e = 0; e < 8; ++e) sg[8 * k + e] = (dc[8 * t + 8 * TPR * k + e] < 0) ? -1.0f : 1.0f;

    const float sqrt_d = sqrtf(static_cast<float>(D));
    const int64_t nsteps = (p.n + RW - 1) / RW;
    double acc = 0.0;                     // this thread's sum of e^2 (the row's lane t = 0)

    for (int s = 0; s < p.samples; ++s) {
        __syncthreads();                  // the previous sample's reads of s_q are done
        const int64_t q0 = (static_cast<int64_t>(s) * p.heads + h) * G * D;
        for (int i = threadIdx.x; i < G * D; i += kThreads)
            s_q[i] = (dc[i % D] < 0) ? -load_query(p.q, p.qdtype, q0 + i) : load_query(p.q, p.qdtype, q0 + i);
        __syncthreads();
        // Walsh-Hadamard butterflies (Sylvester order) over each of the G rows;
        // the 1/sqrt(D) of q' is folded into the key's factor below
        for (int len = 1; len < D; len <<= 1) {
            for (int i = threadIdx.x; i < G * (D / 2); i += kThreads) {
                const int g = i / (D / 2), r = i % (D / 2);
                float *v = s_q + g * D + (r / len) * 2 * len + (r % len);
                const float a = v[0], b = v[len];
                v[0] = a + b;
                v[len] = a - b;
            }
            __syncthreads();
        }

        const void *Ks = static_cast<const T *>(p.K) + (static_cast<int64_t>(s) * p.heads + h) * p.n * D;
        for (int64_t st = warp; st < nsteps; st += kWarps) {
            const int64_t row = st * RW + slot;
            const bool valid = row < p.n;

            float v[E];
#pragma unroll
            for (int k = 0; k < NCH; ++k) {
                if (valid) {
                    Load8<T, false>::run(Ks, row * D + 8 * t + 8 * TPR * k, v + 8 * k);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[8 * k + e] = 0.0f;
                }
            }

            // sign flip with D_c and the squared norm
            float ss = 0.0f;
#pragma unroll
            for (int i = 0; i < E; ++i) {
                v[i] *= sg[i];
                ss = fmaf(v[i], v[i], ss);
            }
#pragma unroll
            for (int m = 1; m < TPR; m <<= 1) ss += __shfl_xor_sync(kFull, ss, m);

            // Hadamard stages inside the thread, then across the row's threads
#pragma unroll
            for (int hb = 1; hb < E; hb <<= 1)
#pragma unroll
                for (int i = 0; i < E; ++i)
                    if (!(i & hb)) {
                        const float a = v[i], b = v[i + hb];
                        v[i] = a + b;
                        v[i + hb] = a - b;
                    }
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
            // a zero key has u = 0 and |k| = 0: its logit and its error are 0
            const float inv = (norm > 0.0f) ? 1.0f / (sqrt_d * norm) : 0.0f;
            const float alpha = norm / static_cast<float>(D);   // |k| / sqrt(D), times the 1/sqrt(D) of q'

            // residuals c[idx] - u, idx by binary search on the boundaries
#pragma unroll
            for (int i = 0; i < E; ++i) {
                const float u = v[i] * inv;
                int code = 0;
#pragma unroll
                for (int step = L / 2; step >= 1; step >>= 1)
                    if (u > s_bnd[code + step - 1]) code += step;
                v[i] = s_cent[code] - u;
            }

            for (int g = 0; g < G; ++g) {
                const float *w = s_q + g * D;
                float part = 0.0f;
#pragma unroll
                for (int k = 0; k < NCH; ++k) {
                    const float4 a = *reinterpret_cast<const float4 *>(w + 8 * t + 8 * TPR * k);
                    const float4 b = *reinterpret_cast<const float4 *>(w + 8 * t + 8 * TPR * k + 4);
                    part = fmaf(a.x, v[8 * k + 0], part);
                    part = fmaf(a.y, v[8 * k + 1], part);
                    part = fmaf(a.z, v[8 * k + 2], part);
                    part = fmaf(a.w, v[8 * k + 3], part);
                    part = fmaf(b.x, v[8 * k + 4], part);
                    part = fmaf(b.y, v[8 * k + 5], part);
                    part = fmaf(b.z, v[8 * k + 6], part);
                    part = fmaf(b.w, v[8 * k + 7], part);
                }
#pragma unroll
                for (int m = 1; m < TPR; m <<= 1) part += __shfl_xor_sync(kFull, part, m);
                const float e = alpha * part;
                if (valid && t == 0) acc = fma(static_cast<double>(e), static_cast<double>(e), acc);
            }
        }
    }

    // fixed-order reduction over the CTA
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) acc += __shfl_xor_sync(kFull, acc, m);
    if (lane == 0) s_red[warp] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double tot = 0.0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) tot += s_red[w];
        p.errors[static_cast<int64_t>(c) * p.heads + h] = static_cast<float>(tot * p.inv_count);
    }
}

// best = argmin over c of max over h of errors[c][h], the lowest c among equal
// values; -1 if no candidate compares (every error NaN).
__global__ void __launch_bounds__(kThreads) select_best_kernel(const float *errors, int C, int heads, int *best)
{
    __shared__ float s_v[kThreads];
    __shared__ int s_i[kThreads];
    float bv = INFINITY;
    int bi = INT_MAX;
    for (int c = threadIdx.x; c < C; c += kThreads) {   // increasing c: strict < keeps the lowest
        float worst = -INFINITY;
        for (int h = 0; h < heads; ++h) {
            const float e = errors[static_cast<int64_t>(c) * heads + h];
            if (e > worst || e != e) worst = e;             // a NaN head makes the candidate's worst NaN
        }
        if (worst < bv || (worst == bv && bi == INT_MAX)) {
            bv = worst;
            bi = c;
        }
    }
    s_v[threadIdx.x] = bv;
    s_i[threadIdx.x] = bi;
    __syncthreads();
    for (int m = kThreads / 2; m >= 1; m >>= 1) {
        if (threadIdx.x < m) {
            const float v2 = s_v[threadIdx.x + m];
            const int i2 = s_i[threadIdx.x + m];
            if (v2 < s_v[threadIdx.x] || (v2 == s_v[threadIdx.x] && i2 < s_i[threadIdx.x])) {
                s_v[threadIdx.x] = v2;
                s_i[threadIdx.x] = i2;
            }
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) *best = (s_i[0] == INT_MAX) ? -1 : s_i[0];
}

template <int D, int B, typename T>
cudaError_t launch_typed(const SignSelectArgs &a, cudaStream_t stream)
{
    SelParams p;
    p.K = a.K;
    p.q = a.q;
    p.qdtype = a.qdtype;
    p.cand = a.candidates;
    p.errors = a.errors;
    p.n = a.n;
    p.samples = a.samples;
    p.heads = a.heads;
    p.group = a.group;
    p.inv_count = 1.0 / (static_cast<double>(a.samples) * a.group * static_cast<double>(a.n));
    for (int i = 0; i < kMaxLevels - 1; ++i) p.bnd[i] = a.cb.boundaries[i];
    for (int i = 0; i < kMaxLevels; ++i) p.cent[i] = a.cb.centroids[i];
    const size_t smem = static_cast<size_t>(a.group) * D * sizeof(float);
    sign_errors_kernel<D, B, T><<<a.candidates_count * a.heads, kThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

template <int D, int B>
cudaError_t launch_db(const SignSelectArgs &a, cudaStream_t stream)
{
    switch (a.kdtype) {
    case AXR_F32: return launch_typed<D, B, float>(a, stream);
    case AXR_F16: return launch_typed<D, B, __half>(a, stream);
    default: return launch_typed<D, B, __nv_bfloat16>(a, stream);
    }
}

template <int D>
cudaError_t launch_d(const SignSelectArgs &a, cudaStream_t stream)
{
    switch (a.b) {
    case 1: return launch_db<D, 1>(a, stream);
    case 2: return launch_db<D, 2>(a, stream);
    case 3: return launch_db<D, 3>(a, stream);
    default: return launch_db<D, 4>(a, stream);
    }
}

}  // namespace

cudaError_t launch_sign_select(const SignSelectArgs &a, cudaStream_t stream)
{
    cudaError_t e;
    switch (a.d) {
    case 8: e = launch_d<8>(a, stream); break;
    case 16: e = launch_d<16>(a, stream); break;
    case 32: e = launch_d<32>(a, stream); break;
    case 64: e = launch_d<64>(a, stream); break;
    case 128: e = launch_d<128>(a, stream); break;
    case 256: e = launch_d<256>(a, stream); break;
    default: e = launch_d<512>(a, stream); break;
    }
    if (e != cudaSuccess || !a.best) return e;
    select_best_kernel<<<1, kThreads, 0, stream>>>(a.errors, a.candidates_count, a.heads, a.best);
    return cudaGetLastError();
}

}  // namespace axr
