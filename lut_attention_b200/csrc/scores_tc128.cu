// Score-on-read for 128-wide heads on the 5th-generation tensor cores (AXELRAM,
// arXiv 2604.02638, abstract: scores come from table lookups on the stored
// indices, never from dequantized keys; queries are rotated once).
//
// The lookups feed an exact int32 contraction over a tile of 128 keys and the G
// query heads of a KV head (fixed-point digits, lut_read.cuh):
//   * one CTA per SM, persistent over a contiguous range of 128-key tiles (split
//     so that each CTA's tiles plus its KV-head changes cost the same,
//     lut::balanced_ranges), dealt round-robin to S tile streams (S = 3 for up to 4 queries per KV head, 2
//     for up to 8), each of 4 worker warps (one thread per key = tensor-memory
//     lane) and one MMA warp;
//   * one TMA warp streams every tile's packed rows and key norms into a ring of
//     6 shared-memory stages (54 KB in flight per SM at b = 4: measured, 12
//     stages were 1 us slower); a worker reads its row with 16-byte loads, which
//     the tensor map's swizzle keeps free of bank conflicts;
//   * for tile k a worker reads the int32 sums of tile k - 2 out of D once its
//     products are done, turns them into scores, and looks up tile k's digits
//     into the A buffer tile k - 2 used (two A and two D buffers per stream), so
//     it never waits for the tensor cores of the tile just published;
//   * the MMA warp runs 8 products (M = 128, N = 4G, K = 32) per tile and one
//     commit, which frees A and publishes D at once.
// Tensor memory per stream: two A buffers of 64 columns and two D buffers of 4G
// columns: 3 x (128 + 32) = 480 columns for G <= 4, 2 x (128 + 64) = 384 for
// G <= 8.  Each stream has one B buffer: on entering a new KV head it waits
// for its last products before writing the head's query digits.
//
// In a decode step the stream that scores a head's last tile first quantizes
// the head's new key (sign flip, Walsh-Hadamard butterflies, norm, nearest
// centroid, packing), stores it in the cache and scores it from registers.
#include <cuda.h>
#include <cuda_runtime.h>

#include "axr_internal.cuh"
#include "lut_read.cuh"
#include "quat.cuh"
#include "sm100.cuh"

namespace axr {
namespace {

using namespace sm100;
using lut::kD;
using lut::kK;

constexpr int kMaxStreams = 3;
constexpr int kTileRows = 128;
constexpr int kStreamThreads = 128;
constexpr int kACols = kK / 4;          // 64 tensor-memory columns hold one tile's digits
constexpr int kTmemCols = 512;
constexpr float kInvSqrtD = 0.08838834764831845f;   // 1 / sqrt(128), the attention temperature

struct Params {
    CUtensorMap tmap;          // packed rows as a [heads * head_stride, P] byte tensor, box P x 128
    CUtensorMap nmap;          // key norms as a 1-D fp32 tensor from a 16-byte boundary, box kNormBox
    int nshift;                // norms[0] is element nshift of nmap
    const void *q;
    int qdtype;
    const int8_t *signs;
    const float *quats;        // block rotation of the queries instead of H diag(signs), or null
    float *scores;             // [heads * group, n]
    int n;                     // keys scored per head
    int head_stride;           // rows between KV heads (>= n)
    int group;
    int tiles_per_head;
    int total_tiles;
    int tile_start[lut::kMaxCtas + 1];   // CTA c scores tiles [tile_start[c], tile_start[c + 1])
    float inv_sc;              // 1 / (128 * S_c)
    int8_t hi[kMaxLevels];     // centroid digits
    int8_t lo[kMaxLevels];
    // decode step: the key of KV head h in k_new (heads x 128, kdtype) is
    // quantized into row append_pos of that head (the last key scored)
    int append_pos;            // -1: no key to append
    int kdtype;
    const void *k_new;
    uint8_t *idx_out;
    float *norms_out;
    float bnd[kMaxLevels - 1];
    AXR_DEBUG_ONLY(dbg::Span sp_q, sp_signs, sp_quats, sp_scores, sp_k_new, sp_idx_out, sp_norms_out;)
};

// stages planned below the 64 KB-aligned table: at most 62 KB, which the window
// holds when it starts within 2 KB past a 64 KB boundary (a window whose gap is
// neither that large nor nearly empty is refused with kErrLayout)
constexpr int kGap = 65536 - 2048;

// The norms of a tile come as a TMA box that starts on the 16-byte boundary at
// or below the tile's first norm, so it holds 128 + 3 floats; the tile's norms
// start (first norm index + nshift) mod 4 floats into it.
constexpr int kNormBox = kTileRows + 4;

// Stages: one tile's packed rows (128 x P bytes), then its norms box; 6 of them
// (a multiple of 2 and 3, so that every stream owns every S-th stage).  Those
// that fit go below the table, the rest after it.
template <int B>
struct Stages {
    static constexpr int P = kD * B / 8;
    static constexpr int kBytes = (kTileRows * P + kNormBox * 4 + 1023) / 1024 * 1024;
    static constexpr int kCount = 6;
    static_assert(kCount % 6 == 0, "every stream owns whole stages");
    static constexpr int kLow = (kGap / kBytes < kCount) ? kGap / kBytes : kCount;
};

// Addresses of the stages: the first kLow from `lo`, the rest from `hi`.
template <int B>
struct StageMap {
    uint8_t *lo, *hi;
    __device__ __forceinline__ uint8_t *at(int s) const
    {
        using St = Stages<B>;
        return s < St::kLow ? lo + s * St::kBytes : hi + (s - St::kLow) * St::kBytes;
    }
};

template <int NQ>
struct Cfg {
    static constexpr int N = 4 * NQ;                       // B rows = D columns
    static constexpr int S = (NQ <= 4) ? 3 : 2;            // tile streams
    static constexpr int kBBytes = N * kK;                 // one stream's B buffer (one head's query digits)
    static constexpr int kWorkerThreads = S * kStreamThreads;
    static constexpr int kWarpTma = kWorkerThreads / 32;
    static constexpr int kWarpMma0 = kWarpTma + 1;         // one MMA warp per stream
    static constexpr int kThreads = kWorkerThreads + 32 * (1 + S);
    static constexpr int kDOff = S * 2 * kACols;           // A buffers first, then D buffers
    static_assert(S <= kMaxStreams, "streams");
    static_assert(kDOff + S * 2 * N <= kTmemCols, "tensor memory budget");
    static_assert(kBBytes >= NQ * kD * 4, "the B buffer holds the query rotation's scratch");
};

constexpr int kMaxStages = 32;
struct Book {
    uint64_t full[kMaxStages], empty[kMaxStages];
    // per stream and buffer: A written (workers); products done (one commit: A
    // may be overwritten, D may be read)
    uint64_t a_full[kMaxStreams][2], mma_done[kMaxStreams][2];
    uint64_t wsync[kMaxStreams];       // the threads of one stream
    uint64_t drain[kMaxStreams];
    uint32_t tmem_base;
    float inv[kMaxStreams][4][8];      // per stream, head number mod 4 and query: 1 / (128 S_q S_c)
    float qmax[kMaxStreams][4][8];     // per stream, warp and query: max |q''|
    float ksum[kMaxStreams][4];        // per stream and warp: sum of squares of an appended key
    uint32_t arow[kMaxStreams][17];    // per stream: packed row of an appended key
    float y[kMaxStreams][kD];          // per stream: rotation scratch of an appended key
};

__device__ unsigned int g_status;

// shared memory: the low stages in the 64 KB below the table, the table on a
// 64 KB boundary, then the high stages, the B buffers and the bookkeeping
template <int B, int NQ>
__host__ __device__ constexpr size_t smem_request()
{
    using St = Stages<B>;
    return 65536 + lut::kLutBytes + (St::kCount - St::kLow) * St::kBytes + Cfg<NQ>::S * Cfg<NQ>::kBBytes +
           sizeof(Book);
}
static_assert(smem_request<4, 8>() <= 232448 && smem_request<3, 8>() <= 232448 && smem_request<2, 8>() <= 232448 &&
                  smem_request<1, 8>() <= 232448,
              "shared memory per block");

// bounded barrier of the 128 threads of stream g; `phase` counts the syncs so
// far.  Its waits are short (the stream's own threads), so it polls.
__device__ __forceinline__ bool stream_sync(Book &S, int g, int &phase)
{
    const uint32_t bar = smem_u32(&S.wsync[g]);
    mbar_arrive(bar);
    const bool ok = mbar_wait_spin(bar, phase & 1);
    ++phase;
    return __all_sync(0xffffffffu, ok) != 0;
}

// This thread's coordinate (its index in the stream) of the G queries of KV
// head h, times the sign pattern D unless the keys were written with the block
// rotation; 0 for the padding queries past the group.
template <int NQ>
__device__ __forceinline__ void load_queries(const Params &p, int h, float (&qq)[NQ])
{
    const int tid = threadIdx.x & (kStreamThreads - 1);
    const float sg = (p.quats || !AXR_IN(p.sp_signs, p.signs + tid, 1) || p.signs[tid] >= 0) ? 1.0f : -1.0f;
    [[maybe_unused]] const int qb = dtype_bytes(p.qdtype);
#pragma unroll
    for (int qi = 0; qi < NQ; ++qi) {
        const int64_t at = (static_cast<int64_t>(h) * p.group + qi) * kD + tid;
        qq[qi] = (qi < p.group && AXR_IN(p.sp_q, static_cast<const char *>(p.q) + at * qb, qb))
                     ? sg * lut::load_q(p.q, p.qdtype, at) : 0.0f;
    }
}

// Rotate the G queries qq (as load_queries gives them) and write their digits
// into the stream's B buffer b (thread j of the stream owns coordinate j of
// every query), and each query's score scale 1 / (128 S_q S_c) into inv[]
// (every thread writes the same values, so each reads back its own).  The
// Walsh-Hadamard transform runs its strides 1-16 with shuffles and its strides
// 32 and 64 as one 4-point transform across the stream's warps, through the B
// buffer (free: its last products are done; every read of it precedes the
// barrier before the digits are written).
template <int B, int NQ>
__device__ bool build_b(const Params &p, Book &S, int g, uint8_t *b, float (&qq)[NQ], float *inv, int &phase)
{
    const int tid = threadIdx.x & (kStreamThreads - 1);
    const int lane = tid & 31, wq = tid >> 5;
    if (p.quats) {
        // q'' = T q / sqrt(d): the IsoQuant block rotation times the temperature;
        // the 4 coordinates of a block sit in 4 consecutive lanes
        Quat qL, qRc;
        if (AXR_IN(p.sp_quats, p.quats + 8 * (tid >> 2), 32)) {
            block_quats(p.quats, tid >> 2, qL, qRc);
        } else {
            unit_quats(qL, qRc);
        }
        const int b0 = lane & ~3;
#pragma unroll
        for (int qi = 0; qi < NQ; ++qi) {
            const Quat v{__shfl_sync(0xffffffffu, qq[qi], b0), __shfl_sync(0xffffffffu, qq[qi], b0 + 1),
                         __shfl_sync(0xffffffffu, qq[qi], b0 + 2), __shfl_sync(0xffffffffu, qq[qi], b0 + 3)};
            const Quat y = block_rotate(qL, qRc, v);
            const float c = (tid & 3) == 0 ? y.w : (tid & 3) == 1 ? y.x : (tid & 3) == 2 ? y.y : y.z;
            qq[qi] = c * kInvSqrtD;
        }
    } else {
#pragma unroll
        for (int st = 1; st < 32; st <<= 1)
#pragma unroll
            for (int qi = 0; qi < NQ; ++qi) {
                const float o = __shfl_xor_sync(0xffffffffu, qq[qi], st);
                qq[qi] = (lane & st) ? o - qq[qi] : qq[qi] + o;
            }
        float(*x)[kD] = reinterpret_cast<float(*)[kD]>(b);
#pragma unroll
        for (int qi = 0; qi < NQ; ++qi) x[qi][tid] = qq[qi];
        if (!stream_sync(S, g, phase)) return false;
        // q'' = H diag(s) q / d  (rotation 1/sqrt(d) times temperature 1/sqrt(d)):
        // coordinate (w, lane) = sum over warps v of (-1)^popcount(w & v) x(v, lane)
#pragma unroll
        for (int qi = 0; qi < NQ; ++qi) {
            const float v0 = x[qi][lane], v1 = x[qi][lane + 32], v2 = x[qi][lane + 64], v3 = x[qi][lane + 96];
            const float a = (wq & 1) ? v0 - v1 : v0 + v1;
            const float c = (wq & 1) ? v2 - v3 : v2 + v3;
            qq[qi] = ((wq & 2) ? a - c : a + c) * (1.0f / kD);
        }
    }
#pragma unroll
    for (int qi = 0; qi < NQ; ++qi) {
        float m = fabsf(qq[qi]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) S.qmax[g][wq][qi] = m;
    }
    if (!stream_sync(S, g, phase)) return false;
    int k_hi, k_lo;
    lut::digit_rows<B>(tid, k_hi, k_lo);
#pragma unroll
    for (int qi = 0; qi < NQ; ++qi) {
        const float m = fmaxf(fmaxf(S.qmax[g][0][qi], S.qmax[g][1][qi]), fmaxf(S.qmax[g][2][qi], S.qmax[g][3][qi]));
        const float sq = (m > 0.0f) ? 64.0f / m : 1.0f;
        inv[qi] = p.inv_sc / sq;
        lut::write_query_digits(b, qi, k_hi, k_lo, qq[qi] * sq);
    }
    fence_proxy_async_smem();
    return true;
}

// Decode step: quantize the appended key of KV head h exactly as the write path
// defines it (sign flip, Walsh-Hadamard, norm, nearest centroid, packing) with
// the stream's 128 threads (thread j owns coordinate j).  Stores its codes and
// norm in the cache and leaves the packed row in S.arow[g] and the norm in *norm.
template <int B>
__device__ bool append_key(const Params &p, Book &S, int g, int h, float *y, float *norm, int &phase)
{
    constexpr int P = kD * B / 8;
    constexpr int L = 1 << B;
    const int tid = threadIdx.x & (kStreamThreads - 1);
    [[maybe_unused]] const int kb = dtype_bytes(p.kdtype);
    const int64_t at = static_cast<int64_t>(h) * kD + tid;
    const bool flip = AXR_IN(p.sp_signs, p.signs + tid, 1) && p.signs[tid] < 0;
    const float kv =
        AXR_IN(p.sp_k_new, static_cast<const char *>(p.k_new) + at * kb, kb) ? lut::load_q(p.k_new, p.kdtype, at) : 0.0f;
    const float x = flip ? -kv : kv;
    y[tid] = x;
    float ss = x * x;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((tid & 31) == 0) S.ksum[g][tid >> 5] = ss;
    if (tid <= P / 4) S.arow[g][tid] = 0u;
    if (!stream_sync(S, g, phase)) return false;
    for (int hh = 1; hh < kD; hh <<= 1) {
        if (tid < kD / 2) {
            const int i = (tid / hh) * 2 * hh + (tid % hh);
            const float a = y[i], c = y[i + hh];
            y[i] = a + c;
            y[i + hh] = a - c;
        }
        if (!stream_sync(S, g, phase)) return false;
    }
    const float nk = sqrtf((S.ksum[g][0] + S.ksum[g][1]) + (S.ksum[g][2] + S.ksum[g][3]));
    // u = y / (sqrt(d) ||k||); idx = number of boundaries below u (a zero key has
    // u = 0 and takes the central index)
    const float u = (nk > 0.0f) ? y[tid] / (sqrtf(static_cast<float>(kD)) * nk) : 0.0f;
    uint32_t code = 0;
#pragma unroll
    for (int i = 0; i < L - 1; ++i) code += (u > p.bnd[i]) ? 1u : 0u;
    const int bit = tid * B;
    atomicOr(&S.arow[g][bit >> 5], code << (bit & 31));
    if ((bit & 31) + B > 32) atomicOr(&S.arow[g][(bit >> 5) + 1], code >> (32 - (bit & 31)));
    if (!stream_sync(S, g, phase)) return false;
    const int64_t row = static_cast<int64_t>(h) * p.head_stride + p.append_pos;
    uint32_t *dst = reinterpret_cast<uint32_t *>(p.idx_out + row * P) + tid;
    if (tid < P / 4 && AXR_IN(p.sp_idx_out, dst, 4)) *dst = S.arow[g][tid];
    if (tid == 0 && AXR_IN(p.sp_norms_out, p.norms_out + row, 4)) p.norms_out[row] = nk;
    *norm = nk;
    return true;
}

// byte offset of 16-byte chunk c of tile row r in a stage, with the swizzle
// the tensor map applies for this row size (P = 64: 64-byte, P = 32: 32-byte;
// rows of 48 and 16 bytes already spread a warp's chunks over all banks)
template <int P>
__device__ __forceinline__ int chunk_offset(int r, int c)
{
    if constexpr (P == 64) return r * 64 + ((c ^ ((r >> 1) & 3)) << 4);
    else if constexpr (P == 32) return r * 32 + ((c ^ ((r >> 2) & 1)) << 4);
    else return r * P + (c << 4);
}

// Worker threads of tile stream g (local tiles k = 0, 1, ... are the CTA's
// tiles t0 + g + S k): one thread per key of a tile.  kAppend: the
// instantiation that serves the decode step (axr_append_scores); plain scoring
// runs the one without the append code.
template <int B, int NQ, bool kAppend>
struct Worker {
    using LK = lut::Lookup<B>;
    using C = Cfg<NQ>;
    using St = Stages<B>;
    static constexpr int P = kD * B / 8;     // bytes of a packed row
    static constexpr int NV = P / 16;        // 16-byte loads per row
    static constexpr int NW = P / 4;

    // digits of 16 tensor-memory columns starting at column 16 q
    static __device__ __forceinline__ void decode16(const uint32_t *w, int q, uint32_t base_lane, uint32_t (&a)[16])
    {
        if constexpr (LK::EB == 4) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint32_t ad = lut::lut_addr<B>(w, 16 * q + i, base_lane);
                asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a[i]) : "r"(ad));
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t ad = lut::lut_addr<B>(w, 8 * q + i, base_lane);
                asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(a[2 * i]), "=r"(a[2 * i + 1]) : "r"(ad));
            }
        }
    }

    // scores of this thread's key of tile (h, ti) from the int32 sums in D.  The
    // query scales of the tile's head (head number hc) are reloaded from shared
    // memory only when the head changes (inv_hc: the head number `inv` holds).
    static __device__ __forceinline__ void emit(const Params &p, const Book &S, int g, uint32_t d_addr, int h,
                                                int ti, int r, float nk, int hc, int &inv_hc, float (&inv)[NQ])
    {
        if (hc != inv_hc) {
            inv_hc = hc;
#pragma unroll
            for (int qi = 0; qi < NQ; ++qi) inv[qi] = S.inv[g][hc & 3][qi];
        }
        uint32_t acc[C::N];
        if constexpr (C::N == 16) {
            tmem_ld16(d_addr, acc);
        } else {
            tmem_ld32(d_addr, acc);
        }
        const int t = ti * kTileRows + r;
        if (t < p.n) {
            float *dst = p.scores + static_cast<int64_t>(h) * p.group * p.n + t;
#pragma unroll
            for (int qi = 0; qi < NQ; ++qi) {
                if (qi < p.group) {
                    if (AXR_IN(p.sp_scores, dst, 4)) __stcs(dst, nk * inv[qi] * lut::join_sums(acc + 4 * qi));
                    dst += p.n;
                }
            }
        }
    }

    // On entering a KV head (the first one too) the stream writes the head's
    // query digits before it waits for the tile's stage.  The first head's
    // queries were loaded before the CTA's set-up (so that their latency
    // overlaps it) and wait in the B buffer, this thread's coordinate of query i
    // at float i * 128 + (thread in stream).
    static __device__ void run(const Params &p, Book &S, int g, const StageMap<B> &stage, uint8_t *sB,
                               uint32_t lut_base, uint32_t tmem, int t0, int t1)
    {
        const int r = threadIdx.x & (kStreamThreads - 1);    // key within the tile = tensor-memory lane
        const int lane = threadIdx.x & 31;
        const uint32_t tl = tmem + (static_cast<uint32_t>(r & ~31) << 16);
        const uint32_t base_lane = lut_base | static_cast<uint32_t>(lane * LK::EB);
        uint8_t *const b = sB + g * C::kBBytes;
        int tile = t0 + g;
        if (tile >= t1) return;
        int h = tile / p.tiles_per_head, ti = tile - h * p.tiles_per_head;
        int prev_h = -1, hc = 0, sync_phase = 0;
        // (head, tile in head, head number, key norm) of tiles k - 1 and k - 2,
        // whose scores are still due
        int h1 = 0, ti1 = 0, hc1 = 0, h2 = 0, ti2 = 0, hc2 = 0;
        float nk1 = 0.0f, nk2 = 0.0f;
        int inv_hc = -1;                    // head number whose query scales `inv` holds
        float inv[NQ];
        // this stream's tiles are the CTA's tiles g, g + S, ...: stages g, g + S, ...
        int s = g;
        uint32_t sph = 0;
        int k = 0;
        for (; tile < t1; tile += C::S, ++k) {
            const int ab = k & 1;
            if (h != prev_h) {
                // one B buffer: the products of tile k - 1 (the last to read it) must be done
                if (k >= 1 && !mbar_wait_warp(smem_u32(&S.mma_done[g][ab ^ 1]), ((k - 1) >> 1) & 1)) {
                    if (lane == 0) atomicOr(&g_status, kErrTimeoutMma);
                    return;
                }
                tc_fence_after_sync();
                prev_h = h;
                ++hc;
                float qq[NQ];
                if (k == 0) {
#pragma unroll
                    for (int qi = 0; qi < NQ; ++qi) qq[qi] = reinterpret_cast<const float *>(b)[qi * kD + r];
                } else {
                    load_queries<NQ>(p, h, qq);
                }
                if (!build_b<B, NQ>(p, S, g, b, qq, S.inv[g][hc & 3], sync_phase)) {
                    if (lane == 0) atomicOr(&g_status, kErrTimeoutDrain);
                    return;
                }
            }
            if (!mbar_wait_warp(smem_u32(&S.full[s]), sph)) {
                if (lane == 0) atomicOr(&g_status, kErrTimeoutLoad);
                return;
            }
            uint32_t w[NW + 1];
            {
                const uint8_t *st = stage.at(s);
#pragma unroll
                for (int c = 0; c < NV; ++c) {
                    const uint4 x = *reinterpret_cast<const uint4 *>(st + chunk_offset<P>(r, c));
                    w[4 * c] = x.x;
                    w[4 * c + 1] = x.y;
                    w[4 * c + 2] = x.z;
                    w[4 * c + 3] = x.w;
                }
                w[NW] = 0u;
            }
            float nk = reinterpret_cast<const float *>(stage.at(s) + kTileRows * P)
                [((h * p.head_stride + ti * kTileRows + p.nshift) & 3) + r];
            mbar_arrive(smem_u32(&S.empty[s]));
            s += C::S;
            if (s >= St::kCount) {
                s -= St::kCount;
                sph ^= 1u;
            }
            // the products of tile k - 2 are done: its A buffer is free, and its D
            // buffer holds its sums
            if (!mbar_wait_warp(smem_u32(&S.mma_done[g][ab]), ((k >> 1) & 1) ^ 1)) {
                if (lane == 0) atomicOr(&g_status, kErrTimeoutMma);
                return;
            }
            tc_fence_after_sync();
            if (k >= 2) emit(p, S, g, tl + C::kDOff + (2 * g + ab) * C::N, h2, ti2, r, nk2, hc2, inv_hc, inv);
            // decode step: this head's last tile holds the appended key, whose row
            // the stage has only as it was before this launch
            if (kAppend && p.append_pos >= 0 && ti == (p.append_pos >> 7)) {
                float nka;
                if (!append_key<B>(p, S, g, h, S.y[g], &nka, sync_phase)) {
                    if (lane == 0) atomicOr(&g_status, kErrTimeoutDrain);
                    return;
                }
                if (r == (p.append_pos & (kTileRows - 1))) {
#pragma unroll
                    for (int v = 0; v < NW; ++v) w[v] = S.arow[g][v];
                    nk = nka;
                }
            }
            // tile k's digits into A buffer ab
            const uint32_t a_addr = tl + (2 * g + ab) * kACols;
#pragma unroll
            for (int qt = 0; qt < 4; ++qt) {
                uint32_t a[16];
                decode16(w, qt, base_lane, a);
                tmem_st16(a_addr + 16 * qt, a);
            }
            tmem_wait_st();
            tc_fence_before_sync();
            mbar_arrive(smem_u32(&S.a_full[g][ab]));
            h2 = h1; ti2 = ti1; hc2 = hc1; nk2 = nk1;
            h1 = h; ti1 = ti; hc1 = hc; nk1 = nk;
            ti += C::S;
            while (ti >= p.tiles_per_head) {
                ti -= p.tiles_per_head;
                ++h;
            }
        }
        // the last two tiles' scores
        for (int j = (k >= 2 ? k - 2 : 0); j < k; ++j) {
            const bool last = (j == k - 1);
            if (!mbar_wait_warp(smem_u32(&S.mma_done[g][j & 1]), (j >> 1) & 1)) {
                if (lane == 0) atomicOr(&g_status, kErrTimeoutMma);
                return;
            }
            tc_fence_after_sync();
            emit(p, S, g, tl + C::kDOff + (2 * g + (j & 1)) * C::N, last ? h1 : h2, last ? ti1 : ti2, r,
                 last ? nk1 : nk2, last ? hc1 : hc2, inv_hc, inv);
        }
    }
};

template <int B, int NQ, bool kAppend>
__global__ void __launch_bounds__(Cfg<NQ>::kThreads, 1) scores_tc128_kernel(const __grid_constant__ Params p)
{
    using C = Cfg<NQ>;
    using St = Stages<B>;
    constexpr int P = kD * B / 8;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base1k = (raw + 1023u) & ~1023u;
    const uint32_t lut_pos = (base1k + 65535u) & ~65535u;
    // low stages in the gap below the table when it holds them, else after it
    const bool low = lut_pos - base1k >= static_cast<uint32_t>(St::kLow * St::kBytes);
    const uint32_t hi_pos = lut_pos + lut::kLutBytes;
    const uint32_t st_lo = low ? base1k : hi_pos;
    const uint32_t st_hi = low ? hi_pos : hi_pos + St::kLow * St::kBytes;
    const uint32_t b_pos = st_hi + (St::kCount - St::kLow) * St::kBytes;
    const uint32_t book_pos = b_pos + C::S * C::kBBytes;
    if (book_pos + sizeof(Book) > raw + static_cast<uint32_t>(smem_request<B, NQ>())) {
        if (threadIdx.x == 0) atomicOr(&g_status, kErrLayout);
        return;
    }
    uint8_t *sLut = smem_raw + (lut_pos - raw);
    uint8_t *sB = smem_raw + (b_pos - raw);
    Book &S = *reinterpret_cast<Book *>(smem_raw + (book_pos - raw));
    const StageMap<B> stage{smem_raw + (st_lo - raw), smem_raw + (st_hi - raw)};

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int t0 = p.tile_start[blockIdx.x];
    const int t1 = p.tile_start[blockIdx.x + 1];
    // the worker threads' coordinates of their first KV head's queries, loaded
    // now and left in their stream's B buffer after the set-up
    float q0[NQ];
    const int first_tile = t0 + static_cast<int>(threadIdx.x / kStreamThreads);
    const bool has_first = threadIdx.x < C::kWorkerThreads && first_tile < t1;
    if (has_first) load_queries<NQ>(p, first_tile / p.tiles_per_head, q0);

    if (threadIdx.x == 0) {
        for (int s = 0; s < St::kCount; ++s) {
            mbar_init(smem_u32(&S.full[s]), 1);
            mbar_init(smem_u32(&S.empty[s]), kStreamThreads);     // consumed by one stream
        }
        for (int g = 0; g < C::S; ++g) {
            for (int a = 0; a < 2; ++a) {
                mbar_init(smem_u32(&S.a_full[g][a]), kStreamThreads);
                mbar_init(smem_u32(&S.mma_done[g][a]), 1);
            }
            mbar_init(smem_u32(&S.wsync[g]), kStreamThreads);
            mbar_init(smem_u32(&S.drain[g]), 1);
        }
        fence_mbar_init();
    }
    if (warp == C::kWarpTma && lane == 0) {
        prefetch_tensormap(&p.tmap);
        prefetch_tensormap(&p.nmap);
    }
    lut::build_lut<B>(p.hi, p.lo, sLut, threadIdx.x, C::kThreads);
    if (has_first) {
        float *x = reinterpret_cast<float *>(sB + (threadIdx.x / kStreamThreads) * C::kBBytes);
#pragma unroll
        for (int qi = 0; qi < NQ; ++qi) x[qi * kD + (threadIdx.x & (kStreamThreads - 1))] = q0[qi];
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&S.tmem_base), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = S.tmem_base;

    if (threadIdx.x < C::kWorkerThreads) {
        const int g = threadIdx.x / kStreamThreads;
        Worker<B, NQ, kAppend>::run(p, S, g, stage, sB, lut_pos, tmem, t0, t1);
    } else if (warp == C::kWarpTma) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            int h = t0 / p.tiles_per_head, ti = t0 - h * p.tiles_per_head;
            int s = 0;
            uint32_t ph = 0;
            for (int tile = t0; tile < t1; ++tile) {
                if (!mbar_wait(smem_u32(&S.empty[s]), ph ^ 1u)) {
                    atomicOr(&g_status, kErrTimeoutDrain);
                    break;
                }
                const int row = h * p.head_stride + ti * kTileRows;
                const uint32_t full = smem_u32(&S.full[s]);
                mbar_arrive_expect_tx(full, kTileRows * P + kNormBox * 4);
                const uint32_t dst = smem_u32(stage.at(s));
                tma_load_2d(dst, &p.tmap, 0, row, full);
                tma_load_1d(dst + kTileRows * P, &p.nmap, (row + p.nshift) & ~3, full);
                if (++s == St::kCount) {
                    s = 0;
                    ph ^= 1u;
                }
                if (++ti == p.tiles_per_head) {
                    ti = 0;
                    ++h;
                }
            }
            // every load issued has landed before the CTA may exit
            const int n_loaded = t1 - t0;
            for (int j = n_loaded - 1; j >= 0 && j >= n_loaded - St::kCount; --j)
                mbar_wait(smem_u32(&S.full[j % St::kCount]), static_cast<uint32_t>(j / St::kCount) & 1u);
        }
    } else if (lane == 0) {
        // ------------------------------------------- MMA issue, one warp per stream
        const int g = warp - C::kWarpMma0;
        const uint32_t id = idesc(kAccS32, kFmtS8, kFmtS8, 128, C::N);
        const uint64_t bd = desc_k_interleave(smem_u32(sB) + g * C::kBBytes, 128, (kK / 16) * 128);
        for (int tile = t0 + g, k = 0; tile < t1; tile += C::S, ++k) {
            const int ab = k & 1;
            if (!mbar_wait(smem_u32(&S.a_full[g][ab]), (k >> 1) & 1)) {
                atomicOr(&g_status, kErrTimeoutLoad);
                break;
            }
            tc_fence_after_sync();
            const uint32_t a = tmem + (2 * g + ab) * kACols;
            const uint32_t d = tmem + C::kDOff + (2 * g + ab) * C::N;
            // K step kk covers A columns 8 kk .. 8 kk + 7 and B 256 bytes further on
#pragma unroll
            for (int kk = 0; kk < kK / 32; ++kk) mma_i8_ts(d, a + 8 * kk, bd + 16 * kk, id, kk > 0);
            mma_commit(smem_u32(&S.mma_done[g][ab]));
        }
        mma_commit(smem_u32(&S.drain[g]));
        mbar_wait(smem_u32(&S.drain[g]), 0);
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int B, int NQ>
cudaError_t launch_bn(const ScoresArgs &a, cudaStream_t stream)
{
    constexpr int P = kD * B / 8;
    const bool append = a.k_new != nullptr;
    auto kernel = append ? scores_tc128_kernel<B, NQ, true> : scores_tc128_kernel<B, NQ, false>;
    constexpr size_t smem = smem_request<B, NQ>();
    static std::atomic<unsigned long long> smem_allowed[2] = {0, 0};     // one bit per device
    if (cudaError_t e = allow_dynamic_smem(reinterpret_cast<const void *>(kernel), smem, smem_allowed[append]);
        e != cudaSuccess)
        return e;
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return cudaErrorNotSupported;
    Params p{};
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(P),
                                static_cast<cuuint64_t>(a.heads) * static_cast<cuuint64_t>(a.head_stride)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(P)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(P), kTileRows};
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapSwizzle swz = (P == 64) ? CU_TENSOR_MAP_SWIZZLE_64B
                                  : (P == 32) ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_NONE;
    CUresult r = enc(&p.tmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(a.idx), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    // norms as a 1-D fp32 tensor whose base is the 16-byte boundary at or below
    // a.norms (TMA wants an aligned base and element offsets that are multiples
    // of 4 floats); boxes running past the end read zeros
    const uintptr_t nbase = reinterpret_cast<uintptr_t>(a.norms) & ~static_cast<uintptr_t>(15);
    p.nshift = static_cast<int>((reinterpret_cast<uintptr_t>(a.norms) - nbase) / sizeof(float));
    const cuuint64_t ndims[1] = {static_cast<cuuint64_t>(a.heads) * static_cast<cuuint64_t>(a.head_stride) +
                                 static_cast<cuuint64_t>(p.nshift)};
    const cuuint64_t nstrides[1] = {0};      // unused for one dimension
    const cuuint32_t nbox[1] = {kNormBox};
    const cuuint32_t nestr[1] = {1};
    r = enc(&p.nmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 1, reinterpret_cast<void *>(nbase), ndims, nstrides, nbox,
            nestr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    p.q = a.q;
    p.qdtype = a.qdtype;
    p.signs = a.signs;
    p.quats = a.quats;
    p.scores = a.scores;
    p.n = static_cast<int>(a.n);
    p.head_stride = static_cast<int>(a.head_stride);
    p.group = a.group;
    p.tiles_per_head = static_cast<int>((a.n + kTileRows - 1) / kTileRows);
    p.total_tiles = p.tiles_per_head * a.heads;
    p.append_pos = a.k_new ? static_cast<int>(a.append_pos) : -1;
    p.kdtype = a.kdtype;
    p.k_new = a.k_new;
    p.idx_out = a.idx_out;
    p.norms_out = a.norms_out;
    for (int i = 0; i < kMaxLevels - 1; ++i) p.bnd[i] = a.cb.boundaries[i];
    lut::centroid_digits(a.cb, p.hi, p.lo, &p.inv_sc);
    AXR_DEBUG_ONLY(const uint64_t rows_q = static_cast<uint64_t>(a.heads) * a.group;
                   const uint64_t rows_k = static_cast<uint64_t>(a.heads) * a.head_stride;
                   p.sp_q = dbg::span(a.q, rows_q * kD * dtype_bytes(a.qdtype));
                   p.sp_signs = dbg::span(a.signs, a.signs ? kD : 0);
                   p.sp_quats = dbg::span(a.quats, a.quats ? (kD / 4) * 8 * sizeof(float) : 0);
                   p.sp_scores = dbg::span(a.scores, rows_q * a.n * sizeof(float));
                   p.sp_k_new = dbg::span(a.k_new, a.k_new ? static_cast<uint64_t>(a.heads) * kD * dtype_bytes(a.kdtype) : 0);
                   p.sp_idx_out = dbg::span(a.idx_out, a.idx_out ? rows_k * P : 0);
                   p.sp_norms_out = dbg::span(a.norms_out, a.norms_out ? rows_k * sizeof(float) : 0);)
    const int sms = device_sm_count() < lut::kMaxCtas ? device_sm_count() : lut::kMaxCtas;
    const int grid = p.total_tiles < sms ? p.total_tiles : sms;
    // a head change costs a stream about 4 us, some 12 tiles of a CTA's time
    lut::balanced_ranges(p.total_tiles, p.tiles_per_head, grid, 12, p.tile_start);
    kernel<<<grid, Cfg<NQ>::kThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

template <int B>
cudaError_t launch_b(const ScoresArgs &a, cudaStream_t stream)
{
    return a.group <= 4 ? launch_bn<B, 4>(a, stream) : launch_bn<B, 8>(a, stream);
}

}  // namespace

bool scores_tc128_supported(const ScoresArgs &a)
{
    return a.d == kD && a.b >= 1 && a.b <= 4 && a.group >= 1 && a.group <= 8 && a.n > 0 &&
           static_cast<int64_t>(a.heads) * a.head_stride < (static_cast<int64_t>(1) << 31) - kTileRows &&
           encode_tiled() != nullptr;
}

cudaError_t launch_scores_tc128(const ScoresArgs &a, cudaStream_t stream)
{
    switch (a.b) {
    case 1: return launch_b<1>(a, stream);
    case 2: return launch_b<2>(a, stream);
    case 3: return launch_b<3>(a, stream);
    default: return launch_b<4>(a, stream);
    }
}

unsigned int scores_tc128_status(bool clear)
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
