// Quantize-on-write with the IsoQuant block rotation in place of the sign flip
// and Walsh-Hadamard transform (IsoQuant, arXiv 2603.28430, abstract: each
// 4-element block v of a key turns into qL v conj(qR); AXELRAM, arXiv
// 2604.02638, abstract: the rotated unit key is quantized with the design-time
// codebook of N(0, 1/d)).
//
// Per key row k of length D:
//   norm = sqrt(sum k_j^2)                    fp32, stored
//   y = T k                                   block by block, T orthonormal
//   u = y / norm                              unit key in the rotated basis
//   idx_j = #{i : u_j > t_i}                  the codebook's boundaries
//   bit-pack idx into D*B/8 bytes, LSB-first
//
// The rotation has no exchange between blocks, so a thread owns EPT consecutive
// coordinates of a row (EPT = 8, 16 at D = 512), i.e. EPT/4 whole blocks, and
// keeps their 4 x 4 matrices in registers for the whole kernel: each matrix is
// composed once from the two quaternion products (columns T e_c), and a block
// then costs 16 FMAs (8 paired) for either variant.  TPR = D/EPT threads share a
// row; they meet only in the xor-reduction of the squared norm.  Codes: the
// bucket of u (the bucket table of the codebook) names the one boundary that can
// decide it, and u itself is compared with that boundary.  Each thread's codes
// fill EPT*B/8 whole bytes of the packed row, stored straight from registers.
#include <cstring>
#include <type_traits>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "axr_internal.cuh"
#include "quat.cuh"

namespace axr {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr unsigned kFull = 0xffffffffu;
constexpr uint32_t kMagicBits = 0x4B400000u;    // bits of 1.5 * 2^23
constexpr float kMagic = 12582912.0f;
constexpr int kBytesInFlight = 2048;            // key bytes per warp and group of rows (two groups in flight)

// Warp steps per loop iteration: about kBytesInFlight of keys per warp, at most
// 64 staged values per thread.
template <int D, int RW, int EPT, typename T>
__host__ __device__ constexpr int steps_per_iteration()
{
    constexpr int by_bytes = kBytesInFlight / (RW * D * static_cast<int>(sizeof(T)));
    constexpr int by_regs = 64 / EPT;
    return by_bytes < 1 ? 1 : (by_bytes < by_regs ? by_bytes : by_regs);
}

struct BParams {
    const void *K;
    int64_t n;
    const float *quats;       // (D/4) x 8: qL, qR per block
    uint8_t *idx;
    float *norms;
    float g_scale;
    float g_off;
    int nt;
    float bnd[kMaxLevels];
    float tau[kMaxBuckets];
    int base[kMaxBuckets];
    AXR_DEBUG_ONLY(dbg::Span sp_K, sp_quats, sp_idx, sp_norms;)
};

// Code of one rotated unit coordinate u, given the bits of f = round(g) + 1.5 * 2^23
// for its bucket value g: entry {boundary, code below it} of bucket round(g) sits
// at bits * 8 + (table - 1.5 * 2^23 * 8), one multiply-add (the bias wraps mod
// 2^32 by design).  kClamp bounds the bucket to the table instead, for rows whose
// squared norm is zero, tiny or not finite, where |u| <= 1 can fail.
// One thread's EPT coordinates of a row as loaded (16-byte words), converted to
// fp32 only when the row is processed, so the next rows' loads stay in flight.
template <typename T, int EPT>
struct RawRow {
    static constexpr int N = EPT * static_cast<int>(sizeof(T)) / 16;
    uint4 w[N];
};

template <typename T, int EPT>
__device__ __forceinline__ void load_row(const void *K, int64_t elem, bool ok, RawRow<T, EPT> &r)
{
    const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const T *>(K) + elem);
#pragma unroll
    for (int i = 0; i < RawRow<T, EPT>::N; ++i) r.w[i] = ok ? __ldcs(src + i) : make_uint4(0u, 0u, 0u, 0u);
}

template <typename T, int EPT>
__device__ __forceinline__ void to_f32(const RawRow<T, EPT> &r, float (&v)[EPT])
{
#pragma unroll
    for (int i = 0; i < RawRow<T, EPT>::N; ++i) {
        const uint32_t ws[4] = {r.w[i].x, r.w[i].y, r.w[i].z, r.w[i].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if constexpr (std::is_same<T, float>::value) {
                v[4 * i + k] = __uint_as_float(ws[k]);
            } else if constexpr (std::is_same<T, __nv_bfloat16>::value) {
                v[8 * i + 2 * k] = __uint_as_float(ws[k] << 16);
                v[8 * i + 2 * k + 1] = __uint_as_float(ws[k] & 0xffff0000u);
            } else {
                __half2 h2;
                memcpy(&h2, &ws[k], 4);
                const float2 f = __half22float2(h2);
                v[8 * i + 2 * k] = f.x;
                v[8 * i + 2 * k + 1] = f.y;
            }
        }
    }
}

template <bool kClamp>
__device__ __forceinline__ uint32_t code_of(float u, float f, uint32_t tab, uint32_t bias, uint32_t last)
{
    uint32_t addr;
    if constexpr (kClamp) {
        addr = tab + min(__float_as_uint(f) - kMagicBits, last) * 8u;
    } else {
        addr = __float_as_uint(f) * 8u + bias;
    }
    float t;
    uint32_t base;
    asm("ld.shared.v2.b32 {%0, %1}, [%2];" : "=f"(t), "=r"(base) : "r"(addr));
    return base + (u > t ? 1u : 0u);
}

template <int B, int EPT, bool kClamp, typename Word>
__device__ __forceinline__ Word pack_codes(const float (&y)[EPT], float inv, float a, float2 offm2, uint32_t tab,
                                           uint32_t bias, uint32_t last)
{
    const float2 inv2 = make_float2(inv, inv), a2 = make_float2(a, a);
    Word word = 0;
#pragma unroll
    for (int e = 0; e < EPT; e += 2) {
        const float2 ye = make_float2(y[e], y[e + 1]);
        const float2 u = __fmul2_rn(ye, inv2);
        const float2 f = __ffma2_rn(ye, a2, offm2);
        word |= static_cast<Word>(code_of<kClamp>(u.x, f.x, tab, bias, last)) << (B * e);
        word |= static_cast<Word>(code_of<kClamp>(u.y, f.y, tab, bias, last)) << (B * (e + 1));
    }
    return word;
}

template <int D, int B, typename T>
__global__ void __launch_bounds__(kThreads, 2) quantize_keys_block_kernel(const __grid_constant__ BParams p)
{
    constexpr int EPT = D >= 512 ? 16 : 8;   // coordinates per thread
    constexpr int TPR = D / EPT;              // threads per row
    constexpr int RW = 32 / TPR;              // rows per warp step
    constexpr int NB = EPT / 4;               // quaternion blocks per thread
    constexpr int P = D * B / 8;              // packed bytes per row
    constexpr int TB = EPT * B / 8;           // packed bytes per thread
    constexpr int U = steps_per_iteration<D, RW, EPT, T>();   // warp steps per iteration
    using Word = typename std::conditional<(EPT * B > 32), unsigned long long, uint32_t>::type;

    __shared__ float2 s_tab[kMaxBuckets];     // {boundary in u units (+inf: none), code below it}
    for (int j = threadIdx.x; j < p.nt; j += kThreads)
        s_tab[j] = make_float2(p.tau[j] < INFINITY ? p.bnd[p.base[j]] : INFINITY, __int_as_float(p.base[j]));
    __syncthreads();

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int t = lane % TPR;
    const int slot = lane / TPR;

    // this thread's blocks as 4 x 4 matrices, rows paired: m01[i][c] = (T_0c, T_1c)
    float2 m01[NB][4], m23[NB][4];
#pragma unroll
    for (int i = 0; i < NB; ++i) {
        Quat qL, qRc;
        if (AXR_IN(p.sp_quats, p.quats + 8 * (t * NB + i), 32)) {
            block_quats(p.quats, t * NB + i, qL, qRc);
        } else {
            unit_quats(qL, qRc);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const Quat e = {c == 0 ? 1.0f : 0.0f, c == 1 ? 1.0f : 0.0f, c == 2 ? 1.0f : 0.0f, c == 3 ? 1.0f : 0.0f};
            const Quat y = block_rotate(qL, qRc, e);
            m01[i][c] = make_float2(y.w, y.x);
            m23[i][c] = make_float2(y.y, y.z);
        }
    }
    const float2 offm2 = make_float2(p.g_off + kMagic, p.g_off + kMagic);
    const uint32_t last = static_cast<uint32_t>(p.nt - 1);
    const uint32_t tab = static_cast<uint32_t>(__cvta_generic_to_shared(s_tab));
    const uint32_t bias = tab - kMagicBits * 8u;     // wraps mod 2^32 by design
    // U warp steps per group: a group's loads are issued together, one group ahead
    // of the one being processed (one step at a time leaves HBM latency-bound)
    const int64_t nsteps = (p.n + RW - 1) / RW;
    const int64_t ngroups = (nsteps + U - 1) / U;

    const int64_t stride = static_cast<int64_t>(gridDim.x) * kWarps;
    RawRow<T, EPT> cur[U], nxt[U];
    int64_t grp = static_cast<int64_t>(blockIdx.x) * kWarps + warp;
    if (grp < ngroups) {
#pragma unroll
        for (int uu = 0; uu < U; ++uu) {
            const int64_t row = (grp * U + uu) * RW + slot;
            const bool ok = row < p.n && AXR_IN(p.sp_K, static_cast<const T *>(p.K) + row * D + t * EPT, EPT * sizeof(T));
            load_row<T, EPT>(p.K, row * D + t * EPT, ok, cur[uu]);
        }
    }
    for (; grp < ngroups; grp += stride) {
        // the next group's loads go out before this group is processed
        const int64_t gn = grp + stride;
        if (gn < ngroups) {
#pragma unroll
            for (int uu = 0; uu < U; ++uu) {
                const int64_t row = (gn * U + uu) * RW + slot;
                const bool ok =
                    row < p.n && AXR_IN(p.sp_K, static_cast<const T *>(p.K) + row * D + t * EPT, EPT * sizeof(T));
                load_row<T, EPT>(p.K, row * D + t * EPT, ok, nxt[uu]);
            }
        }
#pragma unroll
        for (int uu = 0; uu < U; ++uu) {
            const int64_t row = (grp * U + uu) * RW + slot;
            const bool valid = row < p.n;
            float v[EPT];
            to_f32<T, EPT>(cur[uu], v);
            float2 ss2 = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int e = 0; e < EPT; e += 2) {
                const float2 x = make_float2(v[e], v[e + 1]);
                ss2 = __ffma2_rn(x, x, ss2);
            }
            float ss = ss2.x + ss2.y;
#pragma unroll
            for (int m = 1; m < TPR; m <<= 1) ss += __shfl_xor_sync(kFull, ss, m);

            float y[EPT];
#pragma unroll
            for (int i = 0; i < NB; ++i) {
                float2 a01 = make_float2(0.0f, 0.0f), a23 = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float2 vc = make_float2(v[4 * i + c], v[4 * i + c]);
                    a01 = __ffma2_rn(m01[i][c], vc, a01);
                    a23 = __ffma2_rn(m23[i][c], vc, a23);
                }
                y[4 * i + 0] = a01.x;
                y[4 * i + 1] = a01.y;
                y[4 * i + 2] = a23.x;
                y[4 * i + 3] = a23.y;
            }

            const float norm = sqrtf(ss);
            // a zero key has u = 0, which the codes map to 2^(B-1) - 1
            const float inv = (norm > 0.0f) ? 1.0f / norm : 0.0f;
            const float a = p.g_scale * inv;
            const Word word = (ss >= 1e-36f && ss <= 3.402823466e38f)
                                  ? pack_codes<B, EPT, false, Word>(y, inv, a, offm2, tab, bias, last)
                                  : pack_codes<B, EPT, true, Word>(y, inv, a, offm2, tab, bias, last);
            uint8_t *dst = p.idx + row * P + t * TB;
            if (valid && AXR_IN(p.sp_idx, dst, TB)) {
                if constexpr (TB == 8) {
                    *reinterpret_cast<uint2 *>(dst) = make_uint2(static_cast<uint32_t>(word),
                                                                 static_cast<uint32_t>(word >> 32));
                } else if constexpr (TB == 4) {
                    *reinterpret_cast<uint32_t *>(dst) = static_cast<uint32_t>(word);
                } else if constexpr (TB == 2) {
                    *reinterpret_cast<uint16_t *>(dst) = static_cast<uint16_t>(word);
                } else {
#pragma unroll
                    for (int i = 0; i < TB; ++i) dst[i] = static_cast<uint8_t>(word >> (8 * i));
                }
            }
            if (valid && t == 0 && AXR_IN(p.sp_norms, p.norms + row, 4)) p.norms[row] = norm;
        }
#pragma unroll
        for (int uu = 0; uu < U; ++uu) cur[uu] = nxt[uu];
    }
}

template <int D, int B, typename T>
cudaError_t launch_typed(const QuantizeArgs &a, const BucketTable &tab, cudaStream_t stream)
{
    auto kernel = quantize_keys_block_kernel<D, B, T>;
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
    constexpr int EPT = D >= 512 ? 16 : 8;
    constexpr int RW = 32 / (D / EPT);
    constexpr int U = steps_per_iteration<D, RW, EPT, T>();
    const int64_t nsteps = (a.n + RW - 1) / RW;
    const int64_t ngroups = (nsteps + U - 1) / U;
    const int64_t want = (ngroups + kWarps - 1) / kWarps;
    const int64_t cap = static_cast<int64_t>(device_sm_count()) * blocks_per_sm;
    const int grid = static_cast<int>(want < cap ? want : cap);

    BParams p;
    p.K = a.K;
    p.n = a.n;
    p.quats = a.quats;
    p.idx = a.idx;
    p.norms = a.norms;
    p.g_scale = tab.g_scale;
    p.g_off = tab.g_off;
    p.nt = tab.nt;
    for (int i = 0; i < kMaxLevels; ++i) p.bnd[i] = i < kMaxLevels - 1 ? a.cb.boundaries[i] : INFINITY;
    for (int j = 0; j < kMaxBuckets; ++j) {
        p.tau[j] = tab.tau[j];
        p.base[j] = tab.base[j];
    }
    AXR_DEBUG_ONLY(p.sp_K = dbg::span(a.K, static_cast<uint64_t>(a.n) * D * sizeof(T));
                   p.sp_quats = dbg::span(a.quats, (D / 4) * 8 * sizeof(float));
                   p.sp_idx = dbg::span(a.idx, static_cast<uint64_t>(a.n) * (D * B / 8));
                   p.sp_norms = dbg::span(a.norms, static_cast<uint64_t>(a.n) * sizeof(float));)
    kernel<<<grid, kThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

template <int D, int B>
cudaError_t launch_db(const QuantizeArgs &a, const BucketTable &tab, cudaStream_t stream)
{
    switch (a.kdtype) {
    case AXR_F32: return launch_typed<D, B, float>(a, tab, stream);
    case AXR_F16: return launch_typed<D, B, __half>(a, tab, stream);
    default: return launch_typed<D, B, __nv_bfloat16>(a, tab, stream);
    }
}

template <int D>
cudaError_t launch_d(const QuantizeArgs &a, const BucketTable &tab, cudaStream_t stream)
{
    switch (a.b) {
    case 1: return launch_db<D, 1>(a, tab, stream);
    case 2: return launch_db<D, 2>(a, tab, stream);
    case 3: return launch_db<D, 3>(a, tab, stream);
    default: return launch_db<D, 4>(a, tab, stream);
    }
}

}  // namespace

cudaError_t launch_quantize_keys_block(const QuantizeArgs &a, cudaStream_t stream)
{
    BucketTable tab;
    if (!get_bucket_table(a.d, a.b, &tab)) return cudaErrorInvalidValue;
    switch (a.d) {
    case 8: return launch_d<8>(a, tab, stream);
    case 16: return launch_d<16>(a, tab, stream);
    case 32: return launch_d<32>(a, tab, stream);
    case 64: return launch_d<64>(a, tab, stream);
    case 128: return launch_d<128>(a, tab, stream);
    case 256: return launch_d<256>(a, tab, stream);
    default: return launch_d<512>(a, tab, stream);
    }
}

}  // namespace axr
