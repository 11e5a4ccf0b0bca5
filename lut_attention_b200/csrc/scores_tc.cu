// Score-on-read on the 5th-generation tensor cores, head dimension 256 or 512
// (AXELRAM, arXiv 2604.02638, abstract: scores come from table lookups on the
// stored indices, never from dequantized keys).  Each 128-key tile runs as 2 or
// 4 subtiles of 128 coordinates into one accumulator (see Cfg); the queries are
// rotated by the Walsh-Hadamard transform or, for keys written with it, by the
// IsoQuant block rotation.  128-wide heads have their own kernel
// (scores_tc128.cu); the digits and lookup tables are shared (lut_read.cuh).
// A decode step (one new key per KV head, axr_append_scores) runs in the same
// launch: the stream that meets a head's last tile quantizes the new key itself
// (append_key), stores its codes and norm in the cache and scores it with the
// rest of the tile.
//
// The lookups become fixed-point digits that feed an exact int32 tcgen05.mma
// kind::i8 contraction over a tile of 128 keys and the G queries of a KV head
// (lut_read.cuh states the digits and their error bound).
//
// One CTA per SM, persistent over a contiguous range of 128-key tiles (split so
// that each CTA's tiles plus its KV-head changes cost the same), which it
// deals round-robin to S tile streams (S = 3 for up to 4 queries per KV head,
// else 2).  Per stream:
//   4 worker warps : one thread per key (= tensor-memory lane).  For tile k:
//                    read the packed row and the key norm; once the products
//                    of tile k - 2 are done, read its int32 sums (D), scale
//                    them by the key norm and the query scale and store the
//                    scores; then look up tile k's digits and store them to
//                    A in the same buffer.  On entering a new KV head they
//                    wait for the stream's last products, rotate the head's
//                    queries (sign flip, Walsh-Hadamard butterflies, 1/d) and
//                    write their digits into the stream's B buffer.
//   1 MMA warp     : 8 tcgen05.mma (M = 128, N = 4G, K = 32) per tile and one
//                    commit, which frees A and publishes D at once.
// plus one TMA warp loading each tile's packed rows and key norms HBM -> shared
// memory (6 stages).
// A tcgen05.mma issue blocks while the tensor pipe works, and a tile's 8
// products take longer than its decode, so every stream has its own issuer:
// together they keep the pipe fed while each waits for its own workers.
#include <cstdlib>
#include <cstring>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
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
using lut::kLutBytes;
using lut::Lookup;

constexpr int kTileRows = 128;
// Stages of packed rows in flight per CTA: 12, each one slice of a tile (a tile
// takes NH of them).  Stages 0-5 sit in the gap below the lookup table when it
// holds them (otherwise after it), stages 6-11 after it.
constexpr int kStagesMax = 12;
constexpr int kLowStages = 6;
constexpr int kGroupThreads = 128;    // worker threads of one stream (one per key of a tile)
constexpr int kACols = kK / 4;        // tensor-memory columns of one A buffer
constexpr int kTmemCols = 512;
// One stage: the packed rows of a tile (P <= 64 bytes each), then its key norms.
// The norms come as a TMA box that starts on a 16-byte boundary at or below the
// tile's first norm, so it holds 128 + 3 floats; its offset in the box is
// (first norm index + nshift) mod 4.
constexpr int kStageCodeBytes = kTileRows * 64;
constexpr int kNormBox = kTileRows + 4;
constexpr int kStageBytes = kStageCodeBytes + 1024;   // keeps every stage 512-byte aligned
constexpr int kInvSlots = 8;          // per-stream ring of query scales, one slot per head
constexpr int kBBytesMax = 32 * kK;   // one B buffer at most: 8 queries x 4 digit rows x K bytes

// launch shape for NQ query columns per KV head (G <= NQ) and head dimension
// 128 * NH (NH = 2 or 4).  A tile of 128 keys is processed as NH subtiles of 128
// coordinates (one stage, one A buffer and one K = 256 block of B each)
// accumulating into one D.  Each stream keeps one B buffer (shared memory), and
// waits for its products before writing a new head's digits.
template <int NQ, int NH>
struct Cfg {
    static_assert(NH == 2 || NH == 4, "128-wide heads run in scores_tc128.cu");
    static constexpr int N = 4 * NQ;                  // B rows = D columns
    // tile streams: 3 wherever tensor memory and the B buffers allow it
    static constexpr int S = (NH == 2) ? ((NQ <= 4) ? 3 : 2) : ((NQ <= 4) ? 3 : 1);
    static constexpr int kBBufs = 1;                  // B buffers per stream
    static constexpr int kWorkerWarps = 4 * S;
    static constexpr int kWarpTma = kWorkerWarps;
    static constexpr int kWarpMma0 = kWorkerWarps + 1;
    static constexpr int kThreads = (kWorkerWarps + 1 + S) * 32;
    static constexpr int kDOff = S * 2 * kACols;      // A buffers first, then D buffers
    static constexpr int kSliceB = N * kK;            // B bytes of one subtile's K block
    static constexpr int kBBytes = kSliceB * NH;      // one B buffer
    // stages in flight: 12, or 9 at d = 512 with three streams, whose B buffers
    // (3 x 16 KB) take the shared memory of three stages
    static constexpr int kStages = (NH == 4 && NQ <= 4) ? 9 : kStagesMax;
    static constexpr int kBRegion = S * kBBufs * kBBytes;   // the streams' B buffers
    static_assert(kStages % S == 0, "streams must own whole stages");
    static_assert(kStages > kLowStages, "stages below and after the table");
    static_assert(kDOff + S * 2 * N <= kTmemCols, "tensor memory budget");
    static_assert(kSliceB <= kBBytesMax, "B buffer");
    static_assert(kBBytes >= NQ * kD * NH * 4, "a wide head's B buffer holds its rotation scratch");
};

__device__ unsigned int g_status;

struct TcParams {
    CUtensorMap tmap;          // packed rows as a [heads*n, P] byte tensor, box P x 128
    CUtensorMap nmap;          // key norms as a 1-D fp32 tensor from a 16-byte boundary, box kNormBox
    const void *q;
    int qdtype;
    int nshift;                // norms[0] is element nshift of nmap
    const int8_t *signs;
    const float *quats;              // block rotation of the queries instead of H diag(signs), or null
    float *scores;
    int n;                     // keys per head
    int head_stride;           // rows between KV heads in the packed rows and norms (>= n)
    int group;
    int tiles_per_head;
    int total_tiles;
    int tile_start[lut::kMaxCtas + 1];   // CTA c scores tiles [tile_start[c], tile_start[c + 1])
    float inv_sc;              // 1 / (128 * S_c)
    int8_t hi[kMaxLevels];     // centroid digits
    int8_t lo[kMaxLevels];
    // decode step: the key of KV head h in k_new (heads x d, kdtype) is quantized
    // into row append_pos of that head (the last key scored)
    int append_pos;            // -1: no key to append
    int kdtype;
    const void *k_new;
    uint8_t *idx_out;
    float *norms_out;
    float bnd[kMaxLevels - 1];
    AXR_DEBUG_ONLY(dbg::Span sp_q, sp_signs, sp_quats, sp_scores, sp_k_new, sp_idx_out, sp_norms_out;)
};

constexpr int kMaxStreams = 3;
constexpr int kMaxD = 4 * kD;
struct Smem {
    uint64_t full[kStagesMax], empty[kStagesMax];
    // per stream and buffer: A written (workers); products done (one commit: A
    // may be overwritten, D may be read)
    uint64_t a_full[kMaxStreams][2], mma_done[kMaxStreams][2];
    uint64_t drain[kMaxStreams];
    uint64_t wsync[kMaxStreams];       // the threads of one stream (query rotation steps)
    uint32_t tmem_base;
    float inv[kMaxStreams][kInvSlots][8];   // per stream, head slot and query: 1 / (128 * S_q * S_c)
    float qmax[kMaxStreams][4][8];           // per stream, warp and query: max |q''|
    // decode step, per stream: the appended key after the in-warp transform
    // stages, its per-warp sums of squares, and its packed row (+1 spare word)
    float ky[kMaxStreams][kMaxD];
    float ksum[kMaxStreams][4];
    uint32_t arow[kMaxStreams][kMaxD * kMaxBits / 32 + 1];
};
constexpr int kSmemBook = 10240;
static_assert(sizeof(Smem) <= kSmemBook, "bookkeeping area too small");

// bounded barrier of the threads of stream g; `phase` counts the syncs so far
__device__ __forceinline__ bool stream_sync(Smem &S, int g, int &phase)
{
    mbar_arrive(smem_u32(&S.wsync[g]));
    const bool ok = mbar_wait_warp(smem_u32(&S.wsync[g]), phase & 1);
    ++phase;
    return ok;
}

// Rotate the G queries of KV head h and write their digits into B buffer `b`
// of stream g (the stream's 128 threads; thread j owns coordinates j + 128 l of
// the NH slices l).  Slice l's digits form their own K = 256 block of B, at
// l * N * kK bytes.  The B buffer itself is the rotation scratch (it is free,
// and every byte of it is written with digits only after the last read of the
// rotated values).
template <int B, int NQ, int NH>
__device__ bool build_b(const TcParams &p, Smem &S, int g, uint8_t *b, float *inv, int h, int &phase)
{
    constexpr int D = kD * NH;
    constexpr int kSliceB = 4 * NQ * kK;        // bytes of one slice's digits (N rows x K)
    const int tid = threadIdx.x & (kGroupThreads - 1);
    float(*q)[D] = reinterpret_cast<float(*)[D]>(b);
#pragma unroll
    for (int sl = 0; sl < NH; ++sl) {
        const int j = tid + kD * sl;
        const float sg = (p.quats || !AXR_IN(p.sp_signs, p.signs + j, 1) || p.signs[j] >= 0) ? 1.0f : -1.0f;
        [[maybe_unused]] const int qb = dtype_bytes(p.qdtype);
#pragma unroll
        for (int qi = 0; qi < NQ; ++qi) {
            const int64_t at = (static_cast<int64_t>(h) * p.group + qi) * D + j;
            q[qi][j] = (qi < p.group && AXR_IN(p.sp_q, static_cast<const char *>(p.q) + at * qb, qb))
                           ? sg * lut::load_q(p.q, p.qdtype, at) : 0.0f;
        }
    }
    if (!stream_sync(S, g, phase)) return false;
    float qq[NQ][NH];
    if (p.quats) {
        // q'' = T q / sqrt(d): the IsoQuant block rotation T (orthonormal) times the
        // temperature; each coordinate from its 4-element block
        const float inv_sqrt_d = 1.0f / sqrtf(static_cast<float>(D));
#pragma unroll
        for (int sl = 0; sl < NH; ++sl) {
            const int j = tid + kD * sl;
            Quat qL, qRc;
            if (AXR_IN(p.sp_quats, p.quats + 8 * (j >> 2), 32)) {
                block_quats(p.quats, j >> 2, qL, qRc);
            } else {
                unit_quats(qL, qRc);
            }
            const int b0 = j & ~3;
#pragma unroll
            for (int qi = 0; qi < NQ; ++qi) {
                const Quat y = block_rotate(qL, qRc, {q[qi][b0], q[qi][b0 + 1], q[qi][b0 + 2], q[qi][b0 + 3]});
                const float c = (j & 3) == 0 ? y.w : (j & 3) == 1 ? y.x : (j & 3) == 2 ? y.y : y.z;
                qq[qi][sl] = c * inv_sqrt_d;
            }
        }
    } else {
        for (int hh = 1; hh < D; hh <<= 1) {
            for (int t = tid; t < NQ * (D / 2); t += kGroupThreads) {
                const int qi = t / (D / 2), pi = t % (D / 2);
                const int i = (pi / hh) * 2 * hh + (pi % hh);
                const float x = q[qi][i], y = q[qi][i + hh];
                q[qi][i] = x + y;
                q[qi][i + hh] = x - y;
            }
            if (!stream_sync(S, g, phase)) return false;
        }
        // q'' = H diag(s) q / d  (rotation 1/sqrt(d) times temperature 1/sqrt(d))
#pragma unroll
        for (int qi = 0; qi < NQ; ++qi)
#pragma unroll
            for (int sl = 0; sl < NH; ++sl) qq[qi][sl] = q[qi][tid + kD * sl] * (1.0f / D);
    }
#pragma unroll
    for (int qi = 0; qi < NQ; ++qi) {
        float m = 0.0f;
#pragma unroll
        for (int sl = 0; sl < NH; ++sl) m = fmaxf(m, fabsf(qq[qi][sl]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if ((tid & 31) == 0) S.qmax[g][tid >> 5][qi] = m;
    }
    if (!stream_sync(S, g, phase)) return false;
    // this coordinate's hi and lo K rows (the same in every slice)
    int k_hi, k_lo;
    lut::digit_rows<B>(tid, k_hi, k_lo);
#pragma unroll
    for (int qi = 0; qi < NQ; ++qi) {
        float m = 0.0f;
#pragma unroll
        for (int w = 0; w < 4; ++w) m = fmaxf(m, S.qmax[g][w][qi]);
        const float sq = (m > 0.0f) ? 64.0f / m : 1.0f;
        if (tid == 0) inv[qi] = p.inv_sc / sq;
#pragma unroll
        for (int sl = 0; sl < NH; ++sl) {
            lut::write_query_digits(b + sl * kSliceB, qi, k_hi, k_lo, qq[qi][sl] * sq);   // |Q| <= 64
        }
    }
    fence_proxy_async_smem();
    return stream_sync(S, g, phase);
}

// Decode step: quantize the appended key of KV head h exactly as the write path
// defines it (sign flip, Walsh-Hadamard, norm, nearest centroid, packing) with
// the stream's 128 threads; thread j holds coordinates j + 128 l of the NH
// slices l.  The transform's strides 128 and 256 run inside the thread, strides
// 1-16 as shuffles, strides 32 and 64 as one 4-point transform across the
// stream's warps through shared memory.  Stores the codes and the norm in the
// cache.
template <int B, int NH>
__device__ bool append_key(const TcParams &p, Smem &S, int g, int h, int &phase)
{
    constexpr int D = kD * NH;
    constexpr int PT = D * B / 8;             // bytes of the whole packed row
    constexpr int L = 1 << B;
    static_assert(D <= kMaxD && PT / 4 < kGroupThreads, "append scratch");
    const int tid = threadIdx.x & (kGroupThreads - 1);
    const int lane = tid & 31, wq = tid >> 5;
    [[maybe_unused]] const int kb = dtype_bytes(p.kdtype);
    float x[NH];
    float ss = 0.0f;
#pragma unroll
    for (int sl = 0; sl < NH; ++sl) {
        const int j = tid + kD * sl;
        const int64_t at = static_cast<int64_t>(h) * D + j;
        const bool flip = AXR_IN(p.sp_signs, p.signs + j, 1) && p.signs[j] < 0;
        const float kv = AXR_IN(p.sp_k_new, static_cast<const char *>(p.k_new) + at * kb, kb)
                             ? lut::load_q(p.k_new, p.kdtype, at) : 0.0f;
        x[sl] = flip ? -kv : kv;
        ss = fmaf(x[sl], x[sl], ss);
    }
#pragma unroll
    for (int st = 1; st < NH; st <<= 1)
#pragma unroll
        for (int sl = 0; sl < NH; ++sl)
            if (!(sl & st)) {
                const float a = x[sl], c = x[sl + st];
                x[sl] = a + c;
                x[sl + st] = a - c;
            }
#pragma unroll
    for (int st = 1; st < 32; st <<= 1)
#pragma unroll
        for (int sl = 0; sl < NH; ++sl) {
            const float o = __shfl_xor_sync(0xffffffffu, x[sl], st);
            x[sl] = (lane & st) ? o - x[sl] : x[sl] + o;
        }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) S.ksum[g][wq] = ss;
    float *y = S.ky[g];
#pragma unroll
    for (int sl = 0; sl < NH; ++sl) y[kD * sl + tid] = x[sl];
    if (tid <= PT / 4) S.arow[g][tid] = 0u;
    if (!stream_sync(S, g, phase)) return false;
    const float nk = sqrtf((S.ksum[g][0] + S.ksum[g][1]) + (S.ksum[g][2] + S.ksum[g][3]));
    // u = y / (sqrt(d) ||k||); idx = number of boundaries below u (a zero key has
    // u = 0 and takes the central index)
    const float den = sqrtf(static_cast<float>(D)) * nk;
#pragma unroll
    for (int sl = 0; sl < NH; ++sl) {
        // coordinate (wq, lane) of slice sl = sum over warps v of (-1)^popcount(wq & v) y(v, lane)
        const float *ys = y + kD * sl;
        const float v0 = ys[lane], v1 = ys[lane + 32], v2 = ys[lane + 64], v3 = ys[lane + 96];
        const float a = (wq & 1) ? v0 - v1 : v0 + v1;
        const float c = (wq & 1) ? v2 - v3 : v2 + v3;
        const float yv = (wq & 2) ? a - c : a + c;
        const float u = (nk > 0.0f) ? yv / den : 0.0f;
        uint32_t code = 0;
#pragma unroll
        for (int i = 0; i < L - 1; ++i) code += (u > p.bnd[i]) ? 1u : 0u;
        const int bit = (kD * sl + tid) * B;
        atomicOr(&S.arow[g][bit >> 5], code << (bit & 31));
        if ((bit & 31) + B > 32) atomicOr(&S.arow[g][(bit >> 5) + 1], code >> (32 - (bit & 31)));
    }
    if (!stream_sync(S, g, phase)) return false;
    const int64_t row = static_cast<int64_t>(h) * p.head_stride + p.append_pos;
    uint32_t *dst = reinterpret_cast<uint32_t *>(p.idx_out + row * PT) + tid;
    if (tid < PT / 4 && AXR_IN(p.sp_idx_out, dst, 4)) *dst = S.arow[g][tid];
    if (tid == 0 && AXR_IN(p.sp_norms_out, p.norms_out + row, 4)) p.norms_out[row] = nk;
    return true;
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

// Dynamic shared memory: the table on a 64 KB boundary of the shared window
// (so one PRMT forms a full address).  The request covers the table's
// alignment gap (at most 64 KB, which holds stages 0-5 when it is large
// enough), the table, and after it kRestBytes: stages 6-11 (6-8 with nine
// stages), the B buffers and the bookkeeping.
constexpr int kBRegionMax = 32768;    // B buffers with 12 stages
constexpr int kRestBytes = (kStagesMax - kLowStages) * kStageBytes + kBRegionMax + kSmemBook;
static_assert(kLowStages * kStageBytes == (kStagesMax - kLowStages) * kStageBytes, "either half of the stages");
constexpr size_t kSmemRequest = 1024 + 65536 + kLutBytes + kRestBytes;
static_assert(kSmemRequest <= 232448, "shared memory per block");

// Addresses of the NS stages: the first kLowStages from `lo`, the rest from `hi`.
template <int NS>
struct StageMap {
    uint8_t *lo, *hi;
    __device__ __forceinline__ uint8_t *at(int s) const
    {
        if constexpr (NS <= kLowStages) return lo + s * kStageBytes;
        return s < kLowStages ? lo + s * kStageBytes : hi + (s - kLowStages) * kStageBytes;
    }
};
// the stages after the table, the B buffers and the bookkeeping fit in kRestBytes
template <int NQ, int NH>
constexpr bool b_fits()
{
    using C = Cfg<NQ, NH>;
    return (C::kStages - kLowStages) * kStageBytes + C::kBRegion + kSmemBook <= kRestBytes && C::kBRegion % 1024 == 0;
}
static_assert(b_fits<4, 2>() && b_fits<8, 2>() && b_fits<4, 4>() && b_fits<8, 4>(),
              "B buffers of every stream fit");

// Worker threads of tile stream g (local tiles k = 0, 1, ... are the CTA's
// tiles t0 + g + S*k): one thread per key of a tile.
// kAppend: the instantiation that serves the decode step (axr_append_scores);
// plain scoring runs the one without the append code
template <int B, int NQ, int NH, bool kAppend>
struct Worker {
    using LK = Lookup<B>;
    using C = Cfg<NQ, NH>;
    static constexpr int P = kD * B / 8;      // bytes of one 128-coordinate slice of a packed row
    static constexpr int NW = P / 4;

    static constexpr int NL = C::N / 16;      // 16-column loads of one D buffer

    // scores of this thread's key from its int32 digit sums.  D columns 4q .. 4q+3
    // of query q carry weights 128, 1, 1/128, 1/128^2; the pairs are joined in
    // int32 first (|128 c0 + c1| < 1.4e8, |128 c2 + c3| < 2.1e8), so two
    // conversions serve a query.  nk is the key norm; the query scales of the
    // stream's head number `hc` (slot hc mod kInvSlots) are kept in `inv` while
    // that head lasts.
    static __device__ __forceinline__ void store_sums(const TcParams &p, const Smem &S, int g,
                                                      const uint32_t (&acc)[NL][16], float nk, int hc, int h,
                                                      int t, int &inv_hc, float (&inv)[NQ])
    {
        if (hc != inv_hc) {
            inv_hc = hc;
#pragma unroll
            for (int qi = 0; qi < NQ; ++qi) inv[qi] = S.inv[g][hc & (kInvSlots - 1)][qi];
        }
        if (t < p.n) {
            float *dst = p.scores + static_cast<int64_t>(h) * p.group * p.n + t;
#pragma unroll
            for (int qi = 0; qi < NQ; ++qi) {
                const int *x = reinterpret_cast<const int *>(&acc[qi / 4][4 * (qi % 4)]);
                const float hi = __int2float_rn(x[0] * 128 + x[1]);
                const float lo = __int2float_rn(x[2] * 128 + x[3]);
                if (qi < p.group) {
                    if (AXR_IN(p.sp_scores, dst, 4)) __stcs(dst, nk * inv[qi] * fmaf(lo, 1.0f / 16384.0f, hi));
                    dst += p.n;
                }
            }
        }
    }

    // int32 digit sums of this thread's key out of D (load and wait)
    static __device__ __forceinline__ void load_sums(uint32_t taddr, uint32_t (&acc)[NL][16])
    {
#pragma unroll
        for (int c = 0; c < NL; ++c) tmem_ld16(taddr + 16 * c, acc[c]);
    }

    static __device__ void run(const TcParams &p, Smem &S, int g, const StageMap<C::kStages> &sm, uint8_t *sB,
                               uint32_t lut_base,
                               uint32_t tmem, int t0, int t1)
    {
        const int lane = threadIdx.x & 31;
        const int r = threadIdx.x & (kGroupThreads - 1);   // key within the tile = tensor-memory lane
        const uint32_t tmem_lane = tmem + (static_cast<uint32_t>(r & ~31) << 16);
        const uint32_t base_lane = lut_base | static_cast<uint32_t>(lane * LK::EB);
        int bsel = -1, prev_h = -1, hc = -1, sync_phase = 0;
        int h = (t0 + g) / p.tiles_per_head, ti = (t0 + g) - h * p.tiles_per_head;
        // (head, key offset, stream head number, key norm) of tiles k - 1 and k - 2,
        // whose scores are still due
        int h1 = 0, t1k = 0, hs1 = 0, h2 = 0, t2k = 0, hs2 = 0;
        float nk1 = 0.0f, nk2 = 0.0f;
        int s = g, k = 0;
        uint32_t sph = 0;
        bool ok = true;
        int inv_hc = -1;                    // head number whose query scales `inv` holds
        float inv[NQ];

        if constexpr (kAppend) {
            // decode step: before any tile, quantize the appended key of every head
            // whose last tile (the one holding append_pos) this stream scores, and
            // store it in the cache; then one barrier, so that every thread's
            // stores are visible to the key's owner in the loop below
            if (p.append_pos >= 0) {
                const int at = p.append_pos >> 7;
                for (int hh = (t0 + g) / p.tiles_per_head; ok && hh * p.tiles_per_head + at < t1; ++hh) {
                    const int tile = hh * p.tiles_per_head + at;
                    if (tile < t0 + g || (tile - t0 - g) % C::S != 0) continue;
                    ok = append_key<B, NH>(p, S, g, hh, sync_phase);
                }
                ok = ok && stream_sync(S, g, sync_phase);
                if (!ok) {
                    if (lane == 0) atomicOr(&g_status, kErrTimeoutDrain);
                    t1 = t0;                   // no tiles
                }
            }
        }

        for (int tile = t0 + g; tile < t1; tile += C::S, ++k) {
            float nk = 0.0f;
            // decode step: the appended key's row and norm, which the stages may hold
            // as they were before this launch, come from the cache for its thread
            const bool mine = kAppend && p.append_pos >= 0 && ti == (p.append_pos >> 7) &&
                              r == (p.append_pos & (kTileRows - 1));
#pragma unroll 1
            for (int sl = 0; sl < NH; ++sl) {
                const int m = k * NH + sl;      // this stream's subtile count
                if constexpr (NH > 1) {
                    // the CTA's load of (tile, slice) went to stage i mod kStages
                    const int i = (tile - t0) * NH + sl;
                    s = i % C::kStages;
                    sph = static_cast<uint32_t>(i / C::kStages) & 1u;
                }
                if (!mbar_wait_warp(smem_u32(&S.full[s]), sph)) {
                    if (lane == 0) atomicOr(&g_status, kErrTimeoutLoad);
                    ok = false;
                    break;
                }
                uint32_t w[NW + 1];
                {
                    const uint8_t *st = sm.at(s);
#pragma unroll
                    for (int c = 0; c < P / 16; ++c) {
                        const uint4 x = *reinterpret_cast<const uint4 *>(st + chunk_offset<P>(r, c));
                        w[4 * c] = x.x; w[4 * c + 1] = x.y; w[4 * c + 2] = x.z; w[4 * c + 3] = x.w;
                    }
                    w[NW] = 0;
                }
                // this tile's key norm, with its first slice (its scores are due two tiles from now)
                if (sl == 0)
                    nk = reinterpret_cast<const float *>(sm.at(s) + kStageCodeBytes)
                        [((h * p.head_stride + ti * kTileRows + p.nshift) & 3) + r];
                mbar_arrive(smem_u32(&S.empty[s]));

                // products of subtile m - 2 done: its A buffer is free, and with it
                // every product of tile k - 2 (its D is readable) and of the B
                // buffer of two heads back
                const int ab = m & 1;
                if (!mbar_wait_warp(smem_u32(&S.mma_done[g][ab]), ((m >> 1) & 1) ^ 1)) {
                    if (lane == 0) atomicOr(&g_status, kErrTimeoutMma);
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                if (sl == 0) {
                    // scores of tile k - 2, read out of D before tile k's products may overwrite it
                    if (k >= 2) {
                        uint32_t acc[NL][16];
                        load_sums(tmem_lane + C::kDOff + (2 * g + (k & 1)) * C::N, acc);
                        store_sums(p, S, g, acc, nk2, hs2, h2, t2k + r, inv_hc, inv);
                    }
                    if (h != prev_h) {
                        // one B buffer: the last head's products must be done with it
                        if (m >= 1 && !mbar_wait_warp(smem_u32(&S.mma_done[g][(m - 1) & 1]), ((m - 1) >> 1) & 1)) {
                            if (lane == 0) atomicOr(&g_status, kErrTimeoutMma);
                            ok = false;
                            break;
                        }
                        tc_fence_after_sync();
                        bsel = 0;
                        prev_h = h;
                        ++hc;
                        if (!build_b<B, NQ, NH>(p, S, g, sB + (C::kBBufs * g + bsel) * C::kBBytes,
                                                S.inv[g][hc & (kInvSlots - 1)], h, sync_phase)) {
                            if (lane == 0) atomicOr(&g_status, kErrTimeoutDrain);
                            ok = false;
                            break;
                        }
                    }
                }
                if (mine) {
                    const int64_t row = static_cast<int64_t>(h) * p.head_stride + p.append_pos;
                    const uint32_t *src = reinterpret_cast<const uint32_t *>(p.idx_out + row * (P * NH)) + sl * NW;
#pragma unroll
                    for (int v = 0; v < NW; ++v) w[v] = AXR_IN(p.sp_idx_out, src + v, 4) ? __ldcg(src + v) : 0u;
                    if (sl == 0) nk = AXR_IN(p.sp_norms_out, p.norms_out + row, 4) ? __ldcg(p.norms_out + row) : 0.0f;
                }

                // lookup l fills A columns l (4-byte entries) or 2l, 2l+1 (8-byte entries)
                const uint32_t a_addr = tmem_lane + (2 * g + ab) * kACols;
#pragma unroll
                for (int qt = 0; qt < 4; ++qt) {
                    uint32_t a[16];
                    if constexpr (LK::EB == 4) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const uint32_t ad = lut::lut_addr<B>(w, 16 * qt + i, base_lane);
                            asm("ld.shared.u32 %0, [%1];" : "=r"(a[i]) : "r"(ad));
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const uint32_t ad = lut::lut_addr<B>(w, 8 * qt + i, base_lane);
                            asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(a[2 * i]), "=r"(a[2 * i + 1]) : "r"(ad));
                        }
                    }
                    tmem_st16(a_addr + 16 * qt, a);
                }
                tmem_wait_st();
                tc_fence_before_sync();
                mbar_arrive(smem_u32(&S.a_full[g][ab]));
            }
            if (!ok) break;

            h2 = h1; t2k = t1k; hs2 = hs1; nk2 = nk1;
            h1 = h; t1k = ti * kTileRows; hs1 = hc; nk1 = nk;
            ti += C::S;
            while (ti >= p.tiles_per_head) {
                ti -= p.tiles_per_head;
                ++h;
            }
        }

        // the last two tiles' scores (each complete with the products of its last subtile)
        if (ok) {
            for (int j = (k >= 2 ? k - 2 : 0); j < k; ++j) {
                const bool last = (j == k - 1);
                const int mj = j * NH + NH - 1;
                if (!mbar_wait_warp(smem_u32(&S.mma_done[g][mj & 1]), (mj >> 1) & 1)) {
                    if (lane == 0) atomicOr(&g_status, kErrTimeoutMma);
                    break;
                }
                tc_fence_after_sync();
                uint32_t acc[NL][16];
                load_sums(tmem_lane + C::kDOff + (2 * g + (j & 1)) * C::N, acc);
                store_sums(p, S, g, acc, last ? nk1 : nk2, last ? hs1 : hs2, last ? h1 : h2,
                           (last ? t1k : t2k) + r, inv_hc, inv);
            }
        }
    }
};

template <int B, int NQ, int NH, bool kAppend>
__global__ void __launch_bounds__(Cfg<NQ, NH>::kThreads, 1) scores_tc_kernel(const __grid_constant__ TcParams p)
{
    using LK = Lookup<B>;
    using C = Cfg<NQ, NH>;
    constexpr int P = kD * B / 8;             // bytes of one 128-coordinate slice of a packed row
    static_assert(kTileRows * P <= kStageCodeBytes && kStageCodeBytes + kNormBox * 4 <= kStageBytes,
                  "stage too small for a tile of packed rows and its norms");
    static_assert(LK::kRows * 256 <= kLutBytes, "lookup table too large");
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base1k = (raw + 1023u) & ~1023u;
    const uint32_t lut_pos = (base1k + 65535u) & ~65535u;
    // stages 0-5 in the gap below the table when it holds them, else after it;
    // then stages 6-11 (wide heads), B and the bookkeeping.  A shared window whose
    // gap is neither large nor small enough is refused before any barrier exists.
    const bool low = lut_pos - base1k >= static_cast<uint32_t>(kLowStages * kStageBytes);
    const uint32_t hi_pos = lut_pos + kLutBytes;
    const uint32_t st_lo = low ? base1k : hi_pos;
    const uint32_t st_hi = low ? hi_pos : hi_pos + kLowStages * kStageBytes;
    const uint32_t b_pos = st_hi + (C::kStages - kLowStages) * kStageBytes;
    if (b_pos + C::kBRegion + kSmemBook > raw + static_cast<uint32_t>(kSmemRequest)) {
        if (threadIdx.x == 0) atomicOr(&g_status, kErrLayout);
        return;
    }
    uint8_t *sLut = smem_raw + (lut_pos - raw);
    const StageMap<C::kStages> sm{smem_raw + (st_lo - raw), smem_raw + (st_hi - raw)};
    uint8_t *sB = smem_raw + (b_pos - raw);                          // S streams x 2 B buffers
    Smem &S = *reinterpret_cast<Smem *>(sB + C::kBRegion);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int t0 = p.tile_start[blockIdx.x];
    const int t1 = p.tile_start[blockIdx.x + 1];

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(smem_u32(&S.full[s]), 1);
            mbar_init(smem_u32(&S.empty[s]), kGroupThreads);     // consumed by one stream
        }
        for (int g = 0; g < C::S; ++g) {
            for (int a = 0; a < 2; ++a) {
                mbar_init(smem_u32(&S.a_full[g][a]), kGroupThreads);
                mbar_init(smem_u32(&S.mma_done[g][a]), 1);
            }
            mbar_init(smem_u32(&S.wsync[g]), kGroupThreads);
            mbar_init(smem_u32(&S.drain[g]), 1);
        }
        fence_mbar_init();
    }
    if (warp == C::kWarpTma && lane == 0) {
        prefetch_tensormap(&p.tmap);
        prefetch_tensormap(&p.nmap);
    }
    if (warp < C::kWorkerWarps) lut::build_lut<B>(p.hi, p.lo, sLut, threadIdx.x, C::kWorkerWarps * 32);
    if (warp == 0) {
        tmem_alloc(smem_u32(&S.tmem_base), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = S.tmem_base;

    if (warp == C::kWarpTma) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            int it = 0, s = 0;
            uint32_t ph = 0;
            int h = t0 / p.tiles_per_head, ti = t0 - h * p.tiles_per_head;
            bool stop = false;
            for (int tile = t0; tile < t1 && !stop; ++tile) {
                const int row = h * p.head_stride + ti * kTileRows;
                // one stage per 128-coordinate slice of the tile; the norms come with the first
                for (int sl = 0; sl < NH; ++sl, ++it) {
                    if (!mbar_wait(smem_u32(&S.empty[s]), ph ^ 1)) {
                        atomicOr(&g_status, kErrTimeoutDrain);
                        stop = true;
                        break;
                    }
                    const uint32_t full = smem_u32(&S.full[s]);
                    mbar_arrive_expect_tx(full, kTileRows * P + (sl == 0 ? kNormBox * 4 : 0));
                    const uint32_t stg = smem_u32(sm.at(s));
                    tma_load_2d(stg, &p.tmap, sl * P, row, full);
                    if (sl == 0)
                        tma_load_1d(stg + kStageCodeBytes, &p.nmap,
                                    (row + p.nshift) & ~3, full);
                    if (++s == C::kStages) {
                        s = 0;
                        ph ^= 1;
                    }
                }
                if (++ti == p.tiles_per_head) {
                    ti = 0;
                    ++h;
                }
            }
            // every load issued has landed before the CTA may exit
            for (int k = 0; k < C::kStages && k < it; ++k) {
                const int j = it - 1 - k;
                mbar_wait(smem_u32(&S.full[j % C::kStages]), (j / C::kStages) & 1);
            }
        }
    } else if (warp >= C::kWarpMma0) {
        // ------------------------------------------------- MMA, one per stream
        if (lane == 0) {
            const int g = warp - C::kWarpMma0;
            const uint32_t id = idesc(kAccS32, kFmtS8, kFmtS8, 128, C::N);
            const uint32_t b0 = smem_u32(sB) + C::kBBufs * g * C::kBBytes;
            const uint32_t a0 = tmem + 2 * g * kACols;
            const uint32_t d0 = tmem + C::kDOff + 2 * g * C::N;
            // the stream's B buffer flips whenever its tiles enter a new head,
            // exactly as the workers flip it
            int bsel = 1, prev_h = -1;
            int h = (t0 + g) / p.tiles_per_head, ti = (t0 + g) - h * p.tiles_per_head;
            int k = 0;
            bool stop = false;
            for (int tile = t0 + g; tile < t1 && !stop; tile += C::S, ++k) {
                if (h != prev_h) {
                    bsel = (C::kBBufs == 1) ? 0 : (bsel ^ 1);
                    prev_h = h;
                }
                const uint32_t d = d0 + (k & 1) * C::N;
                for (int sl = 0; sl < NH; ++sl) {
                    const int m = k * NH + sl;
                    const int ab = m & 1;
                    // A of this subtile written (which also means the workers have read
                    // the D of tile k - 2 out of this tile's D buffer)
                    if (!mbar_wait(smem_u32(&S.a_full[g][ab]), (m >> 1) & 1)) {
                        atomicOr(&g_status, kErrTimeoutLoad);
                        stop = true;
                        break;
                    }
                    tc_fence_after_sync();
                    // K step kk reads B 256 bytes further on: +16 in the address field;
                    // slice sl's digits are the sl-th K block of the buffer
                    const uint64_t bd =
                        desc_k_interleave(b0 + bsel * C::kBBytes + sl * C::kSliceB, 128, (kK / 16) * 128);
                    const uint32_t a = a0 + ab * kACols;
#pragma unroll
                    for (int kk = 0; kk < kK / 32; ++kk)
                        mma_i8_ts(d, a + 8 * kk, bd + 16 * kk, id, sl > 0 || kk > 0);
                    mma_commit(smem_u32(&S.mma_done[g][ab]));
                }
                ti += C::S;
                while (ti >= p.tiles_per_head) {
                    ti -= p.tiles_per_head;
                    ++h;
                }
            }
            mma_commit(smem_u32(&S.drain[g]));
            mbar_wait(smem_u32(&S.drain[g]), 0);
        }
    } else {
        // ----------------------------------------------------------- workers
        Worker<B, NQ, NH, kAppend>::run(p, S, warp / 4, sm, sB, lut_pos, tmem, t0, t1);
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ host side

template <int B, int NQ, int NH>
cudaError_t launch_bn(const ScoresArgs &a, cudaStream_t stream)
{
    constexpr int P = kD * B / 8;             // one slice of a row: the TMA box width
    constexpr int PT = P * NH;                // the whole packed row
    const bool append = a.k_new != nullptr;
    auto kernel = append ? scores_tc_kernel<B, NQ, NH, true> : scores_tc_kernel<B, NQ, NH, false>;
    const size_t smem = kSmemRequest;
    static std::atomic<unsigned long long> smem_allowed[2] = {0, 0};     // one bit per device
    if (cudaError_t e = allow_dynamic_smem(reinterpret_cast<const void *>(kernel), smem, smem_allowed[append]);
        e != cudaSuccess)
        return e;
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return cudaErrorNotSupported;
    TcParams p{};
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(PT),
                                static_cast<cuuint64_t>(a.heads) * static_cast<cuuint64_t>(a.head_stride)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(PT)};
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
    const int sms = device_sm_count() < lut::kMaxCtas ? device_sm_count() : lut::kMaxCtas;
    const int grid = p.total_tiles < sms ? p.total_tiles : sms;
    // a head change (the query rotation over d coordinates) costs a stream a few
    // microseconds: about 12 tiles of 128 coordinates
    lut::balanced_ranges(p.total_tiles, p.tiles_per_head, grid, 12 / NH, p.tile_start);
    lut::centroid_digits(a.cb, p.hi, p.lo, &p.inv_sc);
    AXR_DEBUG_ONLY(constexpr int D = kD * NH;
                   const uint64_t rows_q = static_cast<uint64_t>(a.heads) * a.group;
                   const uint64_t rows_k = static_cast<uint64_t>(a.heads) * a.head_stride;
                   p.sp_q = dbg::span(a.q, rows_q * D * dtype_bytes(a.qdtype));
                   p.sp_signs = dbg::span(a.signs, a.signs ? D : 0);
                   p.sp_quats = dbg::span(a.quats, a.quats ? (D / 4) * 8 * sizeof(float) : 0);
                   p.sp_scores = dbg::span(a.scores, rows_q * a.n * sizeof(float));
                   p.sp_k_new = dbg::span(a.k_new, a.k_new ? static_cast<uint64_t>(a.heads) * D * dtype_bytes(a.kdtype) : 0);
                   p.sp_idx_out = dbg::span(a.idx_out, a.idx_out ? rows_k * PT : 0);
                   p.sp_norms_out = dbg::span(a.norms_out, a.norms_out ? rows_k * sizeof(float) : 0);)
    kernel<<<grid, Cfg<NQ, NH>::kThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

template <int B, int NH>
cudaError_t launch_b(const ScoresArgs &a, cudaStream_t stream)
{
    return a.group <= 4 ? launch_bn<B, 4, NH>(a, stream) : launch_bn<B, 8, NH>(a, stream);
}

template <int NH>
cudaError_t launch_h(const ScoresArgs &a, cudaStream_t stream)
{
    switch (a.b) {
    case 1: return launch_b<1, NH>(a, stream);
    case 2: return launch_b<2, NH>(a, stream);
    case 3: return launch_b<3, NH>(a, stream);
    default: return launch_b<4, NH>(a, stream);
    }
}

}  // namespace

// AXR_READ_KERNEL=cuda_core in the environment routes every read to the
// CUDA-core kernel (scores.cu), to compare the two on the same calls; read once
// per process.
static bool read_forced_to_cuda_cores()
{
    static const bool forced = [] {
        const char *v = std::getenv("AXR_READ_KERNEL");
        return v != nullptr && std::strcmp(v, "cuda_core") == 0;
    }();
    return forced;
}

bool scores_tc_supported(const ScoresArgs &a)
{
    if (read_forced_to_cuda_cores()) return false;
    if (a.d == kD) return scores_tc128_supported(a);
    // d = 256 and 512 run as 2 and 4 slices of 128 coordinates
    const bool width = a.d == 2 * kD || a.d == 4 * kD;
    return width && a.b >= 1 && a.b <= 4 && a.group <= 8 && a.n > 0 &&
           static_cast<int64_t>(a.heads) * a.head_stride < (static_cast<int64_t>(1) << 31) - kTileRows &&
           encode_tiled() != nullptr;
}

cudaError_t launch_scores_tc(const ScoresArgs &a, cudaStream_t stream)
{
    switch (a.d) {
    case 2 * kD: return launch_h<2>(a, stream);
    case 4 * kD: return launch_h<4>(a, stream);
    default: return launch_scores_tc128(a, stream);
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
    return v | scores_tc128_status(clear);
}

}  // namespace axr

