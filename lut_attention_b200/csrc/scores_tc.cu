// Score-on-read on the 5th-generation tensor cores, head dimension 128 (AXELRAM,
// arXiv 2604.02638, abstract: scores come from table lookups on the stored
// indices, never from dequantized keys).
//
// For the G query heads of a KV head the scores of a tile of 128 keys form one
// small contraction, s[t][g] = norm_t * sum_j c[idx_t[j]] * q''_g[j], so the
// lookups feed the tensor cores instead of G FMAs per coordinate:
//   * every centroid becomes two signed 8-bit digits of a fixed-point number,
//     c * 128 * S_c = 128 * hi + lo  (|hi| <= 127, |lo| <= 64);
//   * every rotated query coordinate becomes three signed 8-bit digits,
//     q'' * S_q = D0 + D1/128 + D2/128^2  (|D| <= 64);
//   * A (tensor memory) holds the hi and lo digits of the looked-up centroids,
//     K = 2 * 128; B (shared memory) holds the query digits, N = 4 columns per
//     query with weights (128, 1, 1/128, 1/128^2):
//         hi rows (D0, D1, D2, 0),   lo rows (0, D0, D1, D2)
//     so one kind::i8 product per 32-wide K step yields, for every query,
//     sum_j q'' c * 128 * S_q * S_c as four exact int32 partial sums.
// The digit error is at most 0.5 / (128 * 127) of the largest centroid per
// coordinate, so |score error| <= 8.5e-5 * ||q|| * ||k|| / sqrt(d) in the worst
// case, inside the 1e-4 the method's tests use; query digits add < 1e-6.
//
// Decoding a packed index row into A is a table walk: each lookup takes one
// field of the row (one byte = 2 codes at b = 4 or 4 codes at b = 2, a 6-bit
// pair at b = 3, a nibble of 4 codes at b = 1) and reads the digits of all its
// codes from a table replicated per lane (address = field * 256 + lane * entry
// size), which is conflict-free in shared memory.
//
// One CTA per SM, persistent over a contiguous range of 128-key tiles:
//   warp 4 (TMA) : packed index tiles HBM -> shared memory (6 stages);
//   warp 5 (MMA) : 8 tcgen05.mma (M=128, N=16|32, K=32) per tile;
//   warps 0-3    : one thread per key: read its packed row, look up its digits,
//                  store them to tensor memory (A); for the previous tile read
//                  the int32 sums (D), scale by the key norm, store the scores.
// Whenever the range enters a new KV head the worker warps rotate that head's
// queries (sign flip, Walsh-Hadamard butterflies, 1/d) and write its digits
// into the other of two B buffers.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "axr_internal.cuh"
#include "sm100.cuh"

namespace axr {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kTileRows = 128;
constexpr int kStages = 6;
constexpr int kWorkWarps = 4;
constexpr int kWorkers = kWorkWarps * 32;
constexpr int kThreads = (kWorkWarps + 2) * 32;
constexpr int kWarpTma = kWorkWarps, kWarpMma = kWorkWarps + 1;
constexpr int kK = 2 * kD;            // two digits per coordinate
constexpr int kACols = kK / 4;        // tensor-memory columns of one A buffer
constexpr int kTmemCols = 256;
constexpr int kAOff = 0;              // A buffers: columns [0, 128)
constexpr int kDOff = 128;            // D buffers: columns [128, 128 + 2*N)
constexpr int kNMax = 32;             // at most 8 queries x 4 digit columns
constexpr int kBBytesMax = kNMax * kK; // one B buffer: N rows x K bytes
constexpr int kStageBytes = kTileRows * 64;   // packed rows of one tile (P <= 64)
constexpr int kLutBytes = 256 * 256;          // up to 256 fields x 256 bytes

__device__ unsigned int g_status;

// geometry of one lookup for b bits: C codes per lookup, FB field bits
template <int B>
struct Lookup {
    static constexpr int C = (B >= 3) ? 2 : 4;
    static constexpr int FB = C * B;              // 8, 6, 8, 4
    static constexpr int EB = 2 * C;              // entry bytes: C hi digits, C lo digits
    static constexpr int NL = kD / C;             // lookups per row
    static constexpr int NF = 1 << FB;            // table fields
};

struct TcParams {
    CUtensorMap tmap;          // packed rows as a [heads*n, P] byte tensor, box P x 128
    const void *q;
    int qdtype;
    const float *norms;
    const int8_t *signs;
    float *scores;
    int n;                     // keys per head
    int group;
    int tiles_per_head;
    int total_tiles;
    int tiles_per_cta;
    float inv_sc;              // 1 / (128 * S_c)
    int8_t hi[kMaxLevels];     // centroid digits
    int8_t lo[kMaxLevels];
};

struct Smem {
    uint64_t full[kStages], empty[kStages], a_full[2], a_empty[2], d_full[2], d_empty[2], drain;
    uint64_t wsync;            // all worker threads (query rotation steps)
    uint32_t tmem_base;
    float inv[2][8];           // per B buffer and query: 1 / (128 * S_q * S_c)
    float q[8][kD];            // rotation scratch
    float qmax[kWorkWarps][8];
};

__device__ __forceinline__ float load_q(const void *q, int dtype, int64_t i)
{
    switch (dtype) {
    case AXR_F32: return static_cast<const float *>(q)[i];
    case AXR_F16: return __half2float(static_cast<const __half *>(q)[i]);
    default: return __bfloat162float(static_cast<const __nv_bfloat16 *>(q)[i]);
    }
}

// bounded barrier of the worker threads; `phase` counts the syncs so far
__device__ __forceinline__ bool workers_sync(Smem &S, int &phase)
{
    mbar_arrive(smem_u32(&S.wsync));
    const bool ok = mbar_wait_warp(smem_u32(&S.wsync), phase & 1);
    ++phase;
    return ok;
}

// B offset of element (n, k) in the no-swizzle K-major layout: 8-row x 16-byte
// core matrices, K-adjacent ones 128 bytes apart, N-adjacent ones kK*8 bytes apart
__device__ __forceinline__ int b_offset(int n, int k)
{
    return ((n >> 3) * (kK / 16) + (k >> 4)) * 128 + (n & 7) * 16 + (k & 15);
}

// Rotate the G queries of KV head h and write their digits into B buffer `bbuf`
// (all worker threads; thread j owns coordinate j).
template <int B, int NQ>
__device__ bool build_b(const TcParams &p, Smem &S, uint8_t *sB, int bbuf, int h, int &phase)
{
    using LK = Lookup<B>;
    const int tid = threadIdx.x;
    const float sg = p.signs[tid] < 0 ? -1.0f : 1.0f;
#pragma unroll
    for (int g = 0; g < NQ; ++g)
        S.q[g][tid] = (g < p.group) ? sg * load_q(p.q, p.qdtype, (static_cast<int64_t>(h) * p.group + g) * kD + tid)
                                    : 0.0f;
    if (!workers_sync(S, phase)) return false;
    for (int hh = 1; hh < kD; hh <<= 1) {
        for (int t = tid; t < NQ * (kD / 2); t += kWorkers) {
            const int g = t / (kD / 2), pi = t % (kD / 2);
            const int i = (pi / hh) * 2 * hh + (pi % hh);
            const float a = S.q[g][i], b = S.q[g][i + hh];
            S.q[g][i] = a + b;
            S.q[g][i + hh] = a - b;
        }
        if (!workers_sync(S, phase)) return false;
    }
    // q'' = H diag(s) q / d  (rotation 1/sqrt(d) times temperature 1/sqrt(d))
    float qq[NQ];
#pragma unroll
    for (int g = 0; g < NQ; ++g) {
        qq[g] = S.q[g][tid] * (1.0f / kD);
        float m = fabsf(qq[g]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if ((tid & 31) == 0) S.qmax[tid >> 5][g] = m;
    }
    if (!workers_sync(S, phase)) return false;
    // this coordinate's hi and lo K rows: lookup l = j / C covers K indices EB*l ..
    const int l = tid / LK::C, t = tid % LK::C;
    const int k_hi = LK::EB * l + t, k_lo = LK::EB * l + LK::C + t;
    uint8_t *b = sB + bbuf * kBBytesMax;
#pragma unroll
    for (int g = 0; g < NQ; ++g) {
        float m = 0.0f;
#pragma unroll
        for (int w = 0; w < kWorkWarps; ++w) m = fmaxf(m, S.qmax[w][g]);
        const float sq = (m > 0.0f) ? 64.0f / m : 1.0f;
        if (tid == 0) S.inv[bbuf][g] = p.inv_sc / sq;
        const float Q = qq[g] * sq;                       // |Q| <= 64
        const float d0 = rintf(Q);
        const float r1 = (Q - d0) * 128.0f;
        const float d1 = rintf(r1);
        const float d2 = rintf((r1 - d1) * 128.0f);
        const uint8_t D0 = static_cast<uint8_t>(static_cast<int8_t>(d0));
        const uint8_t D1 = static_cast<uint8_t>(static_cast<int8_t>(d1));
        const uint8_t D2 = static_cast<uint8_t>(static_cast<int8_t>(d2));
        // column weights (128, 1, 1/128, 1/128^2): hi rows (D0, D1, D2, 0), lo rows (0, D0, D1, D2)
        b[b_offset(4 * g + 0, k_hi)] = D0;
        b[b_offset(4 * g + 1, k_hi)] = D1;
        b[b_offset(4 * g + 2, k_hi)] = D2;
        b[b_offset(4 * g + 3, k_hi)] = 0;
        b[b_offset(4 * g + 0, k_lo)] = 0;
        b[b_offset(4 * g + 1, k_lo)] = D0;
        b[b_offset(4 * g + 2, k_lo)] = D1;
        b[b_offset(4 * g + 3, k_lo)] = D2;
    }
    fence_proxy_async_smem();
    return workers_sync(S, phase);
}

// table entry of one field value: C hi digits then C lo digits
template <int B>
__device__ void build_lut(const TcParams &p, uint8_t *lut)
{
    using LK = Lookup<B>;
    constexpr uint32_t mask = (1u << B) - 1u;
    for (int e = threadIdx.x; e < LK::NF * 32; e += kWorkers) {
        const int field = e / 32, ln = e % 32;
        uint8_t bytes[LK::EB];
#pragma unroll
        for (int i = 0; i < LK::C; ++i) {
            const int code = (field >> (B * i)) & mask;
            bytes[i] = static_cast<uint8_t>(p.hi[code]);
            bytes[LK::C + i] = static_cast<uint8_t>(p.lo[code]);
        }
        uint8_t *dst = lut + field * 256 + ln * LK::EB;
#pragma unroll
        for (int i = 0; i < LK::EB; ++i) dst[i] = bytes[i];
    }
}

// byte offset of 16-byte chunk c of tile row r in a stage, with the swizzle
// the tensor map applies for this row size (P = 64: 64-byte, P = 32: 32-byte)
template <int P>
__device__ __forceinline__ int chunk_offset(int r, int c)
{
    if constexpr (P == 64) return r * 64 + ((c ^ ((r >> 1) & 3)) << 4);
    else if constexpr (P == 32) return r * 32 + ((c ^ ((r >> 2) & 1)) << 4);
    else return r * P + (c << 4);
}

// shared-memory address of the table entry for lookup l of a row held in w[]
template <int B>
__device__ __forceinline__ uint32_t lut_addr(const uint32_t *w, int l, uint32_t lane_off)
{
    using LK = Lookup<B>;
    constexpr int o = LK::FB * 0;   // (placeholder to keep the form uniform)
    (void)o;
    const int bit = l * LK::FB;
    const int wi = bit >> 5, sh = bit & 31;
    if constexpr (LK::FB == 8) {
        // one PRMT: byte (sh/8) of w[wi] into bits 8..15, lane offset into bits 0..7
        const uint32_t sel = 0x5504u | (static_cast<uint32_t>(sh >> 3) << 4);
        return __byte_perm(w[wi], lane_off, sel);
    } else {
        constexpr uint32_t fmask = ((1u << LK::FB) - 1u) << 8;
        uint32_t x;
        if (sh >= 8) {
            x = (sh + LK::FB <= 32) ? (w[wi] >> (sh - 8))
                                    : __funnelshift_r(w[wi], w[wi + 1], sh - 8);
        } else {
            x = w[wi] << (8 - sh);
        }
        return (x & fmask) | lane_off;
    }
}

template <int B, int NQ>
__global__ void __launch_bounds__(kThreads, 1) scores_tc_kernel(const __grid_constant__ TcParams p)
{
    using LK = Lookup<B>;
    constexpr int P = kD * B / 8;
    constexpr int N = 4 * NQ;
    static_assert(N <= kNMax && N * kK <= kBBytesMax, "B buffer too small for N");
    static_assert(kTileRows * P <= kStageBytes, "stage too small for a tile of packed rows");
    static_assert(LK::NF * 256 <= kLutBytes, "lookup table too large");
    constexpr int NW = P / 4;                      // words of a packed row
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *base = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    uint8_t *sStage = base;                         // kStages x 8 KB
    uint8_t *sLut = sStage + kStages * kStageBytes; // 64 KB
    uint8_t *sB = sLut + kLutBytes;                 // 2 x 8 KB
    Smem &S = *reinterpret_cast<Smem *>(sB + 2 * kBBytesMax);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int t0 = blockIdx.x * p.tiles_per_cta;
    const int t1 = min(p.total_tiles, t0 + p.tiles_per_cta);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&S.full[s]), 1);
            mbar_init(smem_u32(&S.empty[s]), kWorkers);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&S.a_full[a]), kWorkers);
            mbar_init(smem_u32(&S.a_empty[a]), 1);
            mbar_init(smem_u32(&S.d_full[a]), 1);
            mbar_init(smem_u32(&S.d_empty[a]), kWorkers);
        }
        mbar_init(smem_u32(&S.drain), 1);
        mbar_init(smem_u32(&S.wsync), kWorkers);
        fence_mbar_init();
    }
    if (warp == kWarpTma && lane == 0) prefetch_tensormap(&p.tmap);
    if (warp < kWorkWarps) build_lut<B>(p, sLut);
    if (warp == 0) {
        tmem_alloc(smem_u32(&S.tmem_base), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = S.tmem_base;

    if (warp == kWarpTma) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            int it = 0;
            for (int tile = t0; tile < t1; ++tile, ++it) {
                const int s = it % kStages;
                const uint32_t ph = (it / kStages) & 1;
                if (!mbar_wait(smem_u32(&S.empty[s]), ph ^ 1)) {
                    atomicOr(&g_status, kErrTimeoutDrain);
                    break;
                }
                const int h = tile / p.tiles_per_head, i = tile % p.tiles_per_head;
                const uint32_t full = smem_u32(&S.full[s]);
                mbar_arrive_expect_tx(full, kTileRows * P);
                tma_load_2d(smem_u32(sStage + s * kStageBytes), &p.tmap, 0, h * p.n + i * kTileRows, full);
            }
            for (int k = 0; k < kStages && k < it; ++k) {
                const int j = it - 1 - k;
                mbar_wait(smem_u32(&S.full[j % kStages]), (j / kStages) & 1);
            }
        }
    } else if (warp == kWarpMma) {
        // --------------------------------------------------------------- MMA
        if (lane == 0) {
            const uint32_t id = idesc(kAccS32, kFmtS8, kFmtS8, 128, N);
            const uint32_t b0 = smem_u32(sB);
            int it = 0, bsel = -1, prev_h = -1;
            for (int tile = t0; tile < t1; ++tile, ++it) {
                const int h = tile / p.tiles_per_head;
                if (h != prev_h) {
                    bsel ^= 1;
                    prev_h = h;
                    if (bsel < 0) bsel = 0;
                }
                const int ab = it & 1;
                const uint32_t aph = (it >> 1) & 1;
                if (!mbar_wait(smem_u32(&S.a_full[ab]), aph)) {
                    atomicOr(&g_status, kErrTimeoutLoad);
                    break;
                }
                if (!mbar_wait(smem_u32(&S.d_empty[ab]), aph ^ 1)) {
                    atomicOr(&g_status, kErrTimeoutDrain);
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d = tmem + kDOff + ab * N;
                const uint32_t a = tmem + kAOff + ab * kACols;
#pragma unroll
                for (int k = 0; k < kK / 32; ++k) {
                    const uint64_t bd = desc_k_interleave(b0 + bsel * kBBytesMax + k * 256, 128, (kK / 16) * 128);
                    mma_i8_ts(d, a + 8 * k, bd, id, k > 0);
                }
                mma_commit(smem_u32(&S.a_empty[ab]));
                mma_commit(smem_u32(&S.d_full[ab]));
            }
            mma_commit(smem_u32(&S.drain));
            mbar_wait(smem_u32(&S.drain), 0);
        }
    } else {
        // ------------------------------------------------------------ workers
        const int r = threadIdx.x;                  // key within the tile = tensor-memory lane
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        const uint32_t lane_off = static_cast<uint32_t>(lane * LK::EB);
        const uint32_t lut0 = smem_u32(sLut);
        int it = 0, bsel = -1, prev_h = -1;
        int prev_tile = -1;
        float prev_norm = 0.0f;
        bool ok = true;
        int sync_phase = 0;

        auto output = [&](int tile, int itp, float nk) {
            const int ab = itp & 1;
            if (!mbar_wait_warp(smem_u32(&S.d_full[ab]), (itp >> 1) & 1)) {
                if (lane == 0) atomicOr(&g_status, kErrTimeoutMma);
                return false;
            }
            tc_fence_after_sync();
            uint32_t acc[16];
            float sc[NQ];
#pragma unroll
            for (int c = 0; c < N / 16; ++c) {
                tmem_ld16(tmem + lane_base + kDOff + ab * N + 16 * c, acc);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int g = 4 * c + e;
                    const float v = fmaf(128.0f, __int2float_rn(static_cast<int>(acc[4 * e])),
                                         fmaf(1.0f / 16384.0f, __int2float_rn(static_cast<int>(acc[4 * e + 3])),
                                              fmaf(1.0f / 128.0f, __int2float_rn(static_cast<int>(acc[4 * e + 2])),
                                                   __int2float_rn(static_cast<int>(acc[4 * e + 1])))));
                    sc[g] = v;
                }
            }
            tc_fence_before_sync();
            mbar_arrive(smem_u32(&S.d_empty[ab]));
            const int h = tile / p.tiles_per_head;
            const int t = (tile % p.tiles_per_head) * kTileRows + r;
            const int hb = ((tile / p.tiles_per_head) == prev_h) ? bsel : (bsel ^ 1);
            if (t < p.n) {
#pragma unroll
                for (int g = 0; g < NQ; ++g)
                    if (g < p.group)
                        __stcs(p.scores + (static_cast<int64_t>(h) * p.group + g) * p.n + t, nk * S.inv[hb][g] * sc[g]);
            }
            return true;
        };

        for (int tile = t0; tile < t1; ++tile, ++it) {
            const int h = tile / p.tiles_per_head;
            const int t = (tile % p.tiles_per_head) * kTileRows + r;
            // the packed row of this thread's key
            const int s = it % kStages;
            if (!mbar_wait_warp(smem_u32(&S.full[s]), (it / kStages) & 1)) {
                if (lane == 0) atomicOr(&g_status, kErrTimeoutLoad);
                ok = false;
                break;
            }
            uint32_t w[NW + 1];
            {
                const uint8_t *st = sStage + s * kStageBytes;
#pragma unroll
                for (int c = 0; c < P / 16; ++c) {
                    const uint4 x = *reinterpret_cast<const uint4 *>(st + chunk_offset<P>(r, c));
                    w[4 * c] = x.x; w[4 * c + 1] = x.y; w[4 * c + 2] = x.z; w[4 * c + 3] = x.w;
                }
                w[NW] = 0;
            }
            mbar_arrive(smem_u32(&S.empty[s]));
            const float nk = (t < p.n) ? __ldg(p.norms + static_cast<int64_t>(h) * p.n + t) : 0.0f;

            if (h != prev_h) {
                bsel = (bsel < 0) ? 0 : (bsel ^ 1);
                prev_h = h;
                if (!build_b<B, NQ>(p, S, sB, bsel, h, sync_phase)) {
                    if (lane == 0) atomicOr(&g_status, kErrTimeoutDrain);
                    ok = false;
                    break;
                }
            }

            // A = the digits of this key's centroids, into tensor memory
            const int ab = it & 1;
            if (!mbar_wait_warp(smem_u32(&S.a_empty[ab]), ((it >> 1) & 1) ^ 1)) {
                if (lane == 0) atomicOr(&g_status, kErrTimeoutMma);
                ok = false;
                break;
            }
            tc_fence_after_sync();
#pragma unroll
            for (int q4 = 0; q4 < kACols / 16; ++q4) {
                uint32_t a[16];
                if constexpr (LK::EB == 4) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const uint32_t ad = lut0 + lut_addr<B>(w, 16 * q4 + i, lane_off);
                        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a[i]) : "r"(ad));
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const uint32_t ad = lut0 + lut_addr<B>(w, 8 * q4 + i, lane_off);
                        asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(a[2 * i]), "=r"(a[2 * i + 1]) : "r"(ad));
                    }
                }
                tmem_st16(tmem + lane_base + kAOff + ab * kACols + 16 * q4, a);
            }
            tmem_wait_st();
            tc_fence_before_sync();
            mbar_arrive(smem_u32(&S.a_full[ab]));

            if (prev_tile >= 0 && !output(prev_tile, it - 1, prev_norm)) {
                ok = false;
                break;
            }
            prev_tile = tile;
            prev_norm = nk;
        }
        if (ok && prev_tile >= 0) output(prev_tile, it - 1, prev_norm);
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ host side

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

template <int B, int NQ>
cudaError_t launch_bn(const ScoresArgs &a, cudaStream_t stream)
{
    constexpr int P = kD * B / 8;
    auto kernel = scores_tc_kernel<B, NQ>;
    const size_t smem = 1024 + kStages * kStageBytes + kLutBytes + 2 * kBBytesMax + sizeof(Smem);
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        configured = true;
    }
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return cudaErrorNotSupported;
    TcParams p{};
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(P),
                                static_cast<cuuint64_t>(a.heads) * static_cast<cuuint64_t>(a.n)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(P)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(P), kTileRows};
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapSwizzle swz = (P == 64) ? CU_TENSOR_MAP_SWIZZLE_64B
                                  : (P == 32) ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_NONE;
    CUresult r = enc(&p.tmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(a.idx), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    p.q = a.q;
    p.qdtype = a.qdtype;
    p.norms = a.norms;
    p.signs = a.signs;
    p.scores = a.scores;
    p.n = static_cast<int>(a.n);
    p.group = a.group;
    p.tiles_per_head = static_cast<int>((a.n + kTileRows - 1) / kTileRows);
    p.total_tiles = p.tiles_per_head * a.heads;
    const int sms = device_sm_count();
    const int grid = p.total_tiles < sms ? p.total_tiles : sms;
    p.tiles_per_cta = (p.total_tiles + grid - 1) / grid;
    // centroid digits: c * 128 * S_c = 128 * hi + lo, S_c = 127 / max |c|
    const int L = 1 << a.b;
    const float cmax = fabsf(a.cb.centroids[L - 1]);
    const double sc = 127.0 / cmax;
    p.inv_sc = static_cast<float>(1.0 / (128.0 * sc));
    for (int i = 0; i < kMaxLevels; ++i) {
        const double v = (i < L) ? a.cb.centroids[i] * 128.0 * sc : 0.0;
        const long vi = lrint(v);
        const long hi = lrint(static_cast<double>(vi) / 128.0);
        p.hi[i] = static_cast<int8_t>(hi);
        p.lo[i] = static_cast<int8_t>(vi - 128 * hi);
    }
    const int used = (p.total_tiles + p.tiles_per_cta - 1) / p.tiles_per_cta;
    kernel<<<used, kThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

template <int B>
cudaError_t launch_b(const ScoresArgs &a, cudaStream_t stream)
{
    return a.group <= 4 ? launch_bn<B, 4>(a, stream) : launch_bn<B, 8>(a, stream);
}

}  // namespace

bool scores_tc_supported(const ScoresArgs &a)
{
    return a.d == kD && a.b >= 1 && a.b <= 4 && a.group <= 8 && a.n > 0 &&
           static_cast<int64_t>(a.heads) * a.n < (static_cast<int64_t>(1) << 31) - kTileRows &&
           encode_tiled() != nullptr;
}

cudaError_t launch_scores_tc(const ScoresArgs &a, cudaStream_t stream)
{
    switch (a.b) {
    case 1: return launch_b<1>(a, stream);
    case 2: return launch_b<2>(a, stream);
    case 3: return launch_b<3>(a, stream);
    default: return launch_b<4>(a, stream);
    }
}

unsigned int scores_tc_status(bool clear)
{
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return ~0u;
    if (clear) {
        const unsigned int z = 0;
        cudaMemcpyToSymbol(g_status, &z, sizeof(z));
    }
    return v;
}

}  // namespace axr
