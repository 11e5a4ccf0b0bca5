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

constexpr uint32_t kMagicBits = 0x4B400000u;    // bits of 1.5 * 2^23
constexpr float kMagic = 12582912.0f;

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
    float g_scale;            // bucket table of the codebook (see BucketTable)
    float g_off;
    int nt;
    float cent[kMaxLevels];
    float bnd[kMaxLevels];    // decision boundaries (L - 1 used)
    float tau[kMaxBuckets];
    int base[kMaxBuckets];
    AXR_DEBUG_ONLY(dbg::Span sp_K, sp_q, sp_cand, sp_errors;)
};

__device__ __forceinline__ float load_query(const void *q, int dtype, int64_t i)
{
    switch (dtype) {
    case AXR_F32: return static_cast<const float *>(q)[i];
    case AXR_F16: return __half2float(static_cast<const __half *>(q)[i]);
    default: return __bfloat162float(static_cast<const __nv_bfloat16 *>(q)[i]);
    }
}

__device__ __forceinline__ float2 sub2(float2 a, float2 b) { return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a); }

// The centroid nearest to a rotated unit coordinate u, given the bits of
// f = round(u * g_scale + g_off) + 1.5 * 2^23: bucket j = round(g) holds at most
// one decision boundary t[j] (+inf where it holds none).  Below it the centroid
// is clo[j] = c[base[j]]; above it c[base[j] + 1], which is clo[j + 1] (the next
// bucket starts one code higher exactly when this one holds a boundary).  The
// bucket only names the boundary; the decision compares u itself with it, as
// the definition does.  Two conflict-free 4-byte lookups: the buckets a warp
// touches at once lie in a window narrower than the 32 banks.  The index is
// clamped to the table, which only non-finite keys can leave.
__device__ __forceinline__ float nearest_centroid(float u, float f, const float *t, const float *clo,
                                                  uint32_t last)
{
    const uint32_t j = min(__float_as_uint(f) - kMagicBits, last);
    return clo[j + (u > t[j] ? 1u : 0u)];
}

// Element i < E of a thread's row segment sits at 8 t + 8 TPR (i / 8) + i % 8;
// the thread holds it in pair i % (E/2), half i / (E/2).
template <int E, int TPR>
__device__ __forceinline__ int element_of(int t, int i)
{
    return 8 * t + 8 * TPR * (i / 8) + i % 8;
}

template <int D, int B, typename T>
__global__ void __launch_bounds__(kThreads) sign_errors_kernel(const __grid_constant__ SelParams p)
{
    constexpr int E = D >= 32 ? 32 : D;   // elements per thread
    constexpr int EH = E / 2;             // element pairs per thread: (i, i + E/2)
    constexpr int TPR = D / E;            // threads per key row
    constexpr int RW = 32 / TPR;          // rows per warp step
    constexpr int NCH = E / 8;            // 8-element chunks per thread
    constexpr int QS = EH + 2;            // float2 stride of a thread's query pairs (padded: no bank conflicts)

    // dynamic: s_q [group][D] (H D_c q, natural order), then s_q2 [group][TPR][QS]
    // float2 (the pairs each thread multiplies, in its register order)
    extern __shared__ __align__(16) float s_dyn[];
    __shared__ float s_t[kMaxBuckets];            // the boundary in each bucket, u units
    __shared__ float s_clo[kMaxBuckets + 1];      // the centroid below it
    __shared__ double s_red[kWarps];

    const int c = blockIdx.x / p.heads;
    const int h = blockIdx.x % p.heads;
    const int G = p.group;
    const int8_t *dc = p.cand + static_cast<int64_t>(c) * D;
    float *s_q = s_dyn;
    float2 *s_q2 = reinterpret_cast<float2 *>(s_dyn + G * D);

    for (int j = threadIdx.x; j <= p.nt; j += kThreads) {
        const int lo = j < p.nt ? p.base[j] : (1 << B) - 1;
        if (j < p.nt) s_t[j] = p.tau[j] < INFINITY ? p.bnd[lo] : INFINITY;
        s_clo[j] = p.cent[lo];
    }

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int t = lane % TPR;
    const int slot = lane / TPR;

    float2 sg[EH];
#pragma unroll
    for (int i = 0; i < EH; ++i) {
        const int8_t *c0 = dc + element_of<E, TPR>(t, i), *c1 = dc + element_of<E, TPR>(t, i + EH);
        sg[i] = make_float2(AXR_IN(p.sp_cand, c0, 1) && *c0 < 0 ? -1.0f : 1.0f,
                            AXR_IN(p.sp_cand, c1, 1) && *c1 < 0 ? -1.0f : 1.0f);
    }
    const int qb = dtype_bytes(p.qdtype);

    const float sqrt_d = sqrtf(static_cast<float>(D));
    const uint32_t last = static_cast<uint32_t>(p.nt - 1);
    const int64_t nsteps = (p.n + RW - 1) / RW;
    double acc = 0.0;                     // this thread's sum of e^2 (the row's lane t = 0)

    for (int s = 0; s < p.samples; ++s) {
        __syncthreads();                  // the previous sample's reads of the queries are done
        const int64_t q0 = (static_cast<int64_t>(s) * p.heads + h) * G * D;
        for (int i = threadIdx.x; i < G * D; i += kThreads) {
            const bool flip = AXR_IN(p.sp_cand, dc + i % D, 1) && dc[i % D] < 0;
            const float qv = AXR_IN(p.sp_q, static_cast<const char *>(p.q) + (q0 + i) * qb, qb)
                                 ? load_query(p.q, p.qdtype, q0 + i) : 0.0f;
            s_q[i] = flip ? -qv : qv;
        }
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
        for (int i = threadIdx.x; i < G * TPR * EH; i += kThreads) {
            const int g = i / (TPR * EH), tt = (i / EH) % TPR, k = i % EH;
            s_q2[(g * TPR + tt) * QS + k] = make_float2(s_q[g * D + element_of<E, TPR>(tt, k)],
                                                        s_q[g * D + element_of<E, TPR>(tt, k + EH)]);
        }
        __syncthreads();

        const void *Ks = static_cast<const T *>(p.K) + (static_cast<int64_t>(s) * p.heads + h) * p.n * D;
        for (int64_t st = warp; st < nsteps; st += kWarps) {
            const int64_t row = st * RW + slot;
            const bool valid = row < p.n;

            float v[E];
#pragma unroll
            for (int k = 0; k < NCH; ++k) {
                const int64_t at = row * D + 8 * t + 8 * TPR * k;
                if (valid && AXR_IN(p.sp_K, static_cast<const T *>(Ks) + at, 8 * sizeof(T))) {
                    Load8<T, false>::run(Ks, at, v + 8 * k);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[8 * k + e] = 0.0f;
                }
            }

            // sign flip with D_c and the squared norm, two elements at a time
            float2 w[EH];
            float2 ss2 = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int i = 0; i < EH; ++i) {
                w[i] = __fmul2_rn(make_float2(v[i], v[i + EH]), sg[i]);
                ss2 = __ffma2_rn(w[i], w[i], ss2);
            }
            float ss = ss2.x + ss2.y;
#pragma unroll
            for (int m = 1; m < TPR; m <<= 1) ss += __shfl_xor_sync(kFull, ss, m);

            // Hadamard stages inside the thread: bits below E/2 on both halves
            // at once, then the top bit between the halves
#pragma unroll
            for (int hb = 1; hb < EH; hb <<= 1)
#pragma unroll
                for (int i = 0; i < EH; ++i)
                    if (!(i & hb)) {
                        const float2 a = w[i], b = w[i + hb];
                        w[i] = __fadd2_rn(a, b);
                        w[i + hb] = sub2(a, b);
                    }
#pragma unroll
            for (int i = 0; i < EH; ++i) w[i] = make_float2(w[i].x + w[i].y, w[i].x - w[i].y);
            // stages across the row's threads: the upper lane keeps (other - own)
#pragma unroll
            for (int m = 1; m < TPR; m <<= 1) {
                const float sgn = (t & m) ? -1.0f : 1.0f;
                const float2 sgn2 = make_float2(sgn, sgn);
#pragma unroll
                for (int i = 0; i < EH; ++i) {
                    const float2 o = make_float2(__shfl_xor_sync(kFull, w[i].x, m), __shfl_xor_sync(kFull, w[i].y, m));
                    w[i] = __ffma2_rn(w[i], sgn2, o);
                }
            }

            const float norm = sqrtf(ss);
            // a zero key has u = 0 and |k| = 0: its logit and its error are 0
            const float inv = (norm > 0.0f) ? 1.0f / (sqrt_d * norm) : 0.0f;
            const float alpha = norm / static_cast<float>(D);   // |k| / sqrt(D), times the 1/sqrt(D) of q'
            const float a = p.g_scale * inv;
            const float2 a2 = make_float2(a, a);
            const float2 inv2 = make_float2(inv, inv);
            const float2 offm2 = make_float2(p.g_off + kMagic, p.g_off + kMagic);

            // residuals c[idx] - u, the bucket of u naming the boundary to compare with
#pragma unroll
            for (int i = 0; i < EH; ++i) {
                const float2 u = __fmul2_rn(w[i], inv2);
                const float2 f = __ffma2_rn(w[i], a2, offm2);
                const float2 cc = make_float2(nearest_centroid(u.x, f.x, s_t, s_clo, last),
                                              nearest_centroid(u.y, f.y, s_t, s_clo, last));
                w[i] = sub2(cc, u);
            }

            for (int g = 0; g < G; ++g) {
                const float4 *qv = reinterpret_cast<const float4 *>(s_q2 + (g * TPR + t) * QS);
                float2 part2 = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int i = 0; i < EH / 2; ++i) {
                    const float4 qq = qv[i];
                    part2 = __ffma2_rn(make_float2(qq.x, qq.y), w[2 * i], part2);
                    part2 = __ffma2_rn(make_float2(qq.z, qq.w), w[2 * i + 1], part2);
                }
                float part = part2.x + part2.y;
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
        float *dst = p.errors + static_cast<int64_t>(c) * p.heads + h;
        if (AXR_IN(p.sp_errors, dst, 4)) *dst = static_cast<float>(tot * p.inv_count);
    }
}

// best = argmin over c of max over h of errors[c][h], the lowest c among equal
// values; -1 if no candidate compares (every error NaN).
__global__ void __launch_bounds__(kThreads)
    select_best_kernel(const float *errors, int C, int heads, int *best AXR_DEBUG_ONLY(, dbg::Span sp_errors,
                                                                                        dbg::Span sp_best))
{
    __shared__ float s_v[kThreads];
    __shared__ int s_i[kThreads];
    float bv = INFINITY;
    int bi = INT_MAX;
    for (int c = threadIdx.x; c < C; c += kThreads) {   // increasing c: strict < keeps the lowest
        float worst = -INFINITY;
        for (int h = 0; h < heads; ++h) {
            const float *src = errors + static_cast<int64_t>(c) * heads + h;
            const float e = AXR_IN(sp_errors, src, 4) ? *src : NAN;
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
    if (threadIdx.x == 0 && AXR_IN(sp_best, best, 4)) *best = (s_i[0] == INT_MAX) ? -1 : s_i[0];
}

template <int D, int B, typename T>
cudaError_t launch_typed(const SignSelectArgs &a, const BucketTable &tab, cudaStream_t stream)
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
    p.g_scale = tab.g_scale;
    p.g_off = tab.g_off;
    p.nt = tab.nt;
    for (int i = 0; i < kMaxLevels; ++i) p.cent[i] = a.cb.centroids[i];
    for (int i = 0; i < kMaxLevels; ++i) p.bnd[i] = i < kMaxLevels - 1 ? a.cb.boundaries[i] : INFINITY;
    for (int j = 0; j < kMaxBuckets; ++j) {
        p.tau[j] = tab.tau[j];
        p.base[j] = tab.base[j];
    }
    constexpr int E = D >= 32 ? 32 : D;
    constexpr int TPR = D / E;
    const size_t smem = static_cast<size_t>(a.group) * (D + TPR * (E / 2 + 2) * 2) * sizeof(float);
    AXR_DEBUG_ONLY(const uint64_t rows = static_cast<uint64_t>(a.samples) * a.heads;
                   p.sp_K = dbg::span(a.K, rows * a.n * D * sizeof(T));
                   p.sp_q = dbg::span(a.q, rows * a.group * D * dtype_bytes(a.qdtype));
                   p.sp_cand = dbg::span(a.candidates, static_cast<uint64_t>(a.candidates_count) * D);
                   p.sp_errors = dbg::span(a.errors, static_cast<uint64_t>(a.candidates_count) * a.heads * 4);)
    sign_errors_kernel<D, B, T><<<a.candidates_count * a.heads, kThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

template <int D, int B>
cudaError_t launch_db(const SignSelectArgs &a, const BucketTable &tab, cudaStream_t stream)
{
    switch (a.kdtype) {
    case AXR_F32: return launch_typed<D, B, float>(a, tab, stream);
    case AXR_F16: return launch_typed<D, B, __half>(a, tab, stream);
    default: return launch_typed<D, B, __nv_bfloat16>(a, tab, stream);
    }
}

template <int D>
cudaError_t launch_d(const SignSelectArgs &a, const BucketTable &tab, cudaStream_t stream)
{
    switch (a.b) {
    case 1: return launch_db<D, 1>(a, tab, stream);
    case 2: return launch_db<D, 2>(a, tab, stream);
    case 3: return launch_db<D, 3>(a, tab, stream);
    default: return launch_db<D, 4>(a, tab, stream);
    }
}

}  // namespace

cudaError_t launch_sign_select(const SignSelectArgs &a, cudaStream_t stream)
{
    BucketTable tab;
    if (!get_bucket_table(a.d, a.b, &tab)) return cudaErrorInvalidValue;
    cudaError_t e;
    switch (a.d) {
    case 8: e = launch_d<8>(a, tab, stream); break;
    case 16: e = launch_d<16>(a, tab, stream); break;
    case 32: e = launch_d<32>(a, tab, stream); break;
    case 64: e = launch_d<64>(a, tab, stream); break;
    case 128: e = launch_d<128>(a, tab, stream); break;
    case 256: e = launch_d<256>(a, tab, stream); break;
    default: e = launch_d<512>(a, tab, stream); break;
    }
    if (e != cudaSuccess || !a.best) return e;
    select_best_kernel<<<1, kThreads, 0, stream>>>(
        a.errors, a.candidates_count, a.heads,
        a.best AXR_DEBUG_ONLY(, dbg::span(a.errors, static_cast<uint64_t>(a.candidates_count) * a.heads * 4),
                              dbg::span(a.best, 4)));
    return cudaGetLastError();
}

}  // namespace axr
