// Quantize-on-write on the 5th-generation tensor cores, head dimension 128, 256
// or 512, bf16 or fp16 keys (AXELRAM, arXiv 2604.02638, abstract: keys are
// transformed once on write and stored as indices into a design-time codebook).
//
// The sign-flipped Walsh-Hadamard transform is a matrix product:
//     y = H diag(s) k   for every key   <=>   Y = K (H diag(s))^T
// H diag(s) has entries +-1, exact in bf16/fp16, and the keys are bf16/fp16, so
// every product is exact and tcgen05 accumulates in fp32: the same arithmetic as
// a butterfly transform, without spending CUDA-core instructions on it.  Wider
// heads follow Sylvester's recursion: with H_256 = [[H, H], [H, -H]] and
// H_512 = H_4 (x) H, y is a signed sum of z_l = H diag(s_l) k_l over the
// 128-coordinate slices l of the key, which the tensor cores compute slice by
// slice and the epilogue combines.  The IsoQuant block rotation (quats) takes
// the same path with another B (see the block-rotation helpers below).
//
// One CTA per SM, persistent over 128-key tiles:
//   warp 16 (TMA) : streams key slices HBM -> shared memory (a ring of 32 KB
//                   stages, 128-byte swizzle, one 128-coordinate slice of a
//                   tile per stage);
//   warp 17 (MMA) : 8 tcgen05.mma (M=128, N=128, K=16) per slice into the
//                   tile's 128-column fp32 accumulator for that slice;
//   warps 0-15    : at d = 128 and 256, two epilogue groups of 8 warps, group e
//                   draining the accumulators of the CTA's even or odd tiles, so
//                   two tiles are in the epilogue at once.  In a group, two warps
//                   per 32 keys (a tensor-memory lane quadrant), one per half of
//                   the 128 columns: read y, exchange the partial sums of y^2
//                   (= d ||k||^2 in total), quantize, pack, store.  At d = 512
//                   the four accumulators fill tensor memory: one tile at a time,
//                   drained by all 16 warps (a 32-column quarter each).
// Quantization: u = y / sqrt(sum y^2); with g = u * G_SCALE + G_OFF every
// bucket [j - 0.5, j + 0.5) of g holds at most one decision boundary, so
//     idx = base[j] + (u > tau[j]),   j = round(g)
// is the count of boundaries below u (one table lookup and one compare instead
// of a b-level binary search).  tau[j] is the boundary inside bucket j (+inf if
// none); no boundary lies near a bucket edge, so the rounding of j never
// changes the result.  Each bucket is one 32-bit word in shared memory (tau with
// base in its low 4 bits, see place_code): one wavefront per warp-wide lookup,
// which buckets 32 apart would have to share a bank to conflict.  Zero keys and
// exact zeros land on the central boundary (0) and take the lower index, as
// ties do.  A key with a non-finite entry (outside the contract) stores its
// non-finite norm and the central index instead of reading the table out of
// range.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "axr_internal.cuh"
#include "quat.cuh"
#include "sm100.cuh"

namespace axr {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kTileRows = 128;
constexpr int kStages = 4;
constexpr int kABytes = kTileRows * kD * 2;     // one tile of keys, 32 KB
constexpr int kBBytes = kD * kD * 2;            // H diag(s), 32 KB
constexpr int kHalfBytes = kTileRows * 128;     // one 64-element K block of a tile
constexpr int kGroupWarps = 8;                  // one epilogue group: two warps per lane quadrant
constexpr int kEpiWarps = 2 * kGroupWarps;      // two groups, one per accumulator
constexpr int kThreads = (kEpiWarps + 2) * 32;
// d = 128 * NH: a tile's keys arrive as NH stages of 128 coordinates, and each
// 128-key tile has NH accumulators of 128 columns (two tiles in flight)
template <int NH>
__host__ __device__ constexpr int tmem_cols() { return NH == 4 ? 512 : 256 * NH; }
// Stages of the key ring: d = 512 fills tensor memory with one tile's four
// accumulators (single buffered, drained by all epilogue warps together) and
// shared memory with its four B matrices, which leaves room for two stages;
// d = 256 keeps four; d = 128 three, which measured 2.6 % faster than four and
// 10 % faster than two on gqa_decode_128k (and the same on mha_decode_32k)
template <int NH>
__host__ __device__ constexpr int stages() { return NH == 4 ? 2 : (NH == 2 ? kStages : 3); }
template <int NH>
__host__ __device__ constexpr int acc_bufs() { return NH == 4 ? 1 : 2; }
constexpr int kWarpTma = kEpiWarps, kWarpMma = kEpiWarps + 1;
constexpr uint32_t kMagicBits = 0x4B400000u;    // bits of 1.5 * 2^23
constexpr float kMagic = 12582912.0f;

__device__ unsigned int g_status;

struct TcParams {
    CUtensorMap tmap;              // keys as a [n, 128] tensor, box 64 x 128, 128-byte swizzle
    uint8_t *idx;
    float *norms;
    const int8_t *signs;
    const float *quats;            // block rotation (d/4 x 8 floats) in place of the signs, or null
    int64_t n;
    int ntiles;
    float g_scale;
    float g_off;
    float inv_sqrt_d;
    int nt;
    float tau[kMaxBuckets];
    int base[kMaxBuckets];
    AXR_DEBUG_ONLY(dbg::Span sp_idx, sp_norms, sp_signs, sp_quats;)
};

struct Smem {
    uint64_t full[kStages], empty[kStages], acc_full[2], acc_empty[2], drain;
    uint64_t pair[2][4];           // [accumulator][lane quadrant]: both halves posted their sums
    uint32_t tmem_base;
    float ss[2][2][kTileRows];     // [accumulator][column half][key]: partial sums of y^2
};

// Insert the code of one coordinate (unit value u) into the packed words at bit
// offset O.  Its bucket is round(g) for g = u g_scale + g_off, read from the
// bits of f = g + 1.5 * 2^23 (entry address bits(f) * 4 + bias, or the clamped
// bucket).  An entry is the codebook boundary the bucket holds (u units; 2 if
// none, which no |u| <= 1 exceeds) with its low 4 mantissa bits replaced by the
// bucket's base code (the number of boundaries below the bucket).  Read as a
// float it is the boundary moved by at most 15 ulp (at most 2.3e-7 for
// d >= 128, inside the 1e-6 boundary window).  u > entry is the sign bit of
// entry - u (exact in sign, and +0 when the two are equal), so the code is the
// low bits of entry + that bit.  At b = 1, 2, 4 the codes of a 32-bit word
// arrive in coordinate order and each enters at the top of the word with one
// funnel shift, moving the earlier ones down; at b = 3 they are masked and
// added at their offsets.
template <int B, int O, bool kClamp>
__device__ __forceinline__ void place_code(float u, float f, uint32_t tab, uint32_t bias, uint32_t *w)
{
    uint32_t addr;
    if constexpr (kClamp) {
        const uint32_t bucket = min(__float_as_uint(f) - kMagicBits, static_cast<uint32_t>(kMaxBuckets - 1));
        addr = tab + bucket * 4u;
    } else {
        addr = __float_as_uint(f) * 4u + bias;
    }
    uint32_t e;
    asm("ld.shared.b32 %0, [%1];" : "=r"(e) : "r"(addr));
    e += __float_as_uint(__fsub_rn(__uint_as_float(e), u)) >> 31;
    constexpr int k = O >> 5, sh = O & 31;
    if constexpr (32 % B == 0) {
        w[k] = __funnelshift_r(w[k], e, B);
    } else {
        const uint32_t code = e & ((1u << B) - 1u);
        w[k] += code << sh;
        if constexpr (sh + B > 32) w[k + 1] += code >> (32 - sh);
    }
}

// Table entry of bucket j: boundary tau (u units; 2 for none, tau = +inf) with
// its low 4 bits replaced by the base code
__device__ __forceinline__ uint32_t table_entry(float tau, int base)
{
    const float t = tau < 2.0f ? tau : 2.0f;
    return (__float_as_uint(t) & ~15u) | static_cast<uint32_t>(base);
}

// Quantize coordinates C0 + E, C0 + E + 1 (two at a time: one paired multiply
// gives both unit values u = y / |y|, one paired FMA both f = y a + g_off +
// 1.5 * 2^23, rounded exactly as two scalar operations would be).
template <int B, int C0, int E, bool kClamp>
__device__ __forceinline__ void quantize_chunk(const uint32_t (&v)[32], float2 ug2, float2 a2, float2 offm2,
                                               uint32_t tab, uint32_t bias, uint32_t *w)
{
    if constexpr (E < 32) {
        const float2 y = make_float2(__uint_as_float(v[E]), __uint_as_float(v[E + 1]));
        const float2 u = __fmul2_rn(y, ug2);
        const float2 f = __ffma2_rn(y, a2, offm2);
        place_code<B, (C0 + E) * B, kClamp>(u.x, f.x, tab, bias, w);
        place_code<B, (C0 + E + 1) * B, kClamp>(u.y, f.y, tab, bias, w);
        quantize_chunk<B, C0, E + 2, kClamp>(v, ug2, a2, offm2, tab, bias, w);
    }
}

// y_q = sum_l (-1)^popcount(q & l) z_l (Sylvester H_4) for columns e, e + 1 of
// the four accumulators' pieces z[l][0 .. 7]
// (kIdentity: the block rotation, whose slices do not mix: y_q = z_q)
template <bool kIdentity>
__device__ __forceinline__ void h4(const uint32_t (&z)[4][8], int e, float2 (&y)[4])
{
    const float2 m1 = make_float2(-1.0f, -1.0f);
    const float2 z0 = make_float2(__uint_as_float(z[0][e]), __uint_as_float(z[0][e + 1]));
    const float2 z1 = make_float2(__uint_as_float(z[1][e]), __uint_as_float(z[1][e + 1]));
    const float2 z2 = make_float2(__uint_as_float(z[2][e]), __uint_as_float(z[2][e + 1]));
    const float2 z3 = make_float2(__uint_as_float(z[3][e]), __uint_as_float(z[3][e + 1]));
    if constexpr (kIdentity) {
        y[0] = z0;
        y[1] = z1;
        y[2] = z2;
        y[3] = z3;
        return;
    }
    const float2 s01 = __fadd2_rn(z0, z1), d01 = __ffma2_rn(z1, m1, z0);
    const float2 s23 = __fadd2_rn(z2, z3), d23 = __ffma2_rn(z3, m1, z2);
    y[0] = __fadd2_rn(s01, s23);
    y[1] = __fadd2_rn(d01, d23);
    y[2] = __ffma2_rn(s23, m1, s01);
    y[3] = __ffma2_rn(d23, m1, d01);
}

// codes of 8 coordinates held in v[24 .. 31] at positions 8 pc .. 8 pc + 7 of a
// 32-coordinate run (quantize_chunk on the top quarter of v, offset back by 24)
template <int B, bool kClamp>
__device__ __forceinline__ void quantize_piece(int pc, const uint32_t (&v)[32], float2 ug2, float2 a2, float2 offm2,
                                               uint32_t tab, uint32_t bias, uint32_t *w)
{
    switch (pc) {
    case 0: quantize_chunk<B, -24, 24, kClamp>(v, ug2, a2, offm2, tab, bias, w); break;
    case 1: quantize_chunk<B, -16, 24, kClamp>(v, ug2, a2, offm2, tab, bias, w); break;
    case 2: quantize_chunk<B, -8, 24, kClamp>(v, ug2, a2, offm2, tab, bias, w); break;
    default: quantize_chunk<B, 0, 24, kClamp>(v, ug2, a2, offm2, tab, bias, w); break;
    }
}

// NWQ packed words (32 coordinates) to global memory, streaming
template <int NWQ>
__device__ __forceinline__ void store_words(uint8_t *dst, const uint32_t *w)
{
    if constexpr (NWQ == 4) {
        __stcs(reinterpret_cast<uint4 *>(dst), make_uint4(w[0], w[1], w[2], w[3]));
    } else if constexpr (NWQ == 2) {
        __stcs(reinterpret_cast<uint2 *>(dst), make_uint2(w[0], w[1]));
    } else {
#pragma unroll
        for (int i = 0; i < NWQ; ++i) __stcs(reinterpret_cast<unsigned int *>(dst) + i, w[i]);
    }
}

// Block rotation (IsoQuant, arXiv 2603.28430, abstract: 4-element blocks v turn
// into qL v conj(qR)).  T is block diagonal, so each 16-coordinate group of a
// 128-coordinate slice only mixes within itself: output columns 16 j .. 16 j + 15
// of z_l are one M = 128, N = 16, K = 16 product of the keys' columns 16 j ..
// with the group's 16 x 16 piece of T.  Those pieces are fp32; they enter the
// tensor cores as kParts terms in the key type (bf16: 3 terms, 24 bits; fp16:
// 2 terms, 22 bits), each product of a bf16/fp16 key with a term is exact, and
// fp32 accumulation adds them, so y = T k comes out at fp32 accuracy.
template <bool kBF16>
__host__ __device__ constexpr int block_parts() { return kBF16 ? 3 : 2; }
constexpr int kBlkBytes = 16 * 16 * 2;           // one 16 x 16 piece, no swizzle (core matrices)

// byte offset of element (n = output, k = input) in a 16 x 16 K-major piece:
// 8 x 8-element core matrices, K-adjacent ones 128 bytes apart, N-adjacent 256
__device__ __forceinline__ int blk_offset(int n, int k)
{
    return ((n >> 3) * 2 + (k >> 3)) * 128 + (n & 7) * 16 + (k & 7) * 2;
}

template <bool kBF16>
__device__ __forceinline__ uint16_t to_half_bits(float v, float &back)
{
    if constexpr (kBF16) {
        const __nv_bfloat16 h = __float2bfloat16_rn(v);
        back = __bfloat162float(h);
        return __bfloat16_as_ushort(h);
    } else {
        const __half h = __float2half_rn(v);
        back = __half2float(h);
        return __half_as_ushort(h);
    }
}

// one run of NWH packed words (64 coordinates), 16- or 8-byte streaming stores
template <int NWH>
__device__ __forceinline__ void store_run(uint8_t *dst, const uint32_t *w)
{
    if constexpr (NWH % 4 == 0) {
#pragma unroll
        for (int i = 0; i < NWH / 4; ++i)
            __stcs(reinterpret_cast<uint4 *>(dst) + i, make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]));
    } else {
#pragma unroll
        for (int i = 0; i < NWH / 2; ++i) __stcs(reinterpret_cast<uint2 *>(dst) + i, make_uint2(w[2 * i], w[2 * i + 1]));
    }
}

template <int B, bool kBF16, int NH, bool kBlock>
__global__ void __launch_bounds__(kThreads, 1) quantize_keys_tc_kernel(const __grid_constant__ TcParams p)
{
    constexpr int kParts = block_parts<kBF16>();
    constexpr int kBRegion = kBlock ? kParts * NH * 8 * kBlkBytes : NH * kBBytes;
    constexpr int D = kD * NH;
    constexpr int kTmemCols = tmem_cols<NH>();
    constexpr int kSt = stages<NH>();
    constexpr int P = D * B / 8;             // packed bytes per key
    constexpr int NW = kD * B / 8 / 4;       // packed 32-bit words per 128 coordinates
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *base = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    uint8_t *sA = base;                                      // kStages x 32 KB
    uint8_t *sB = sA + kSt * kABytes;                        // NH x 32 KB
    uint32_t *sTab = reinterpret_cast<uint32_t *>(sB + kBRegion);     // kMaxBuckets entries (table_entry)
    Smem &S = *reinterpret_cast<Smem *>(sTab + kMaxBuckets);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&S.full[s]), 1);
            mbar_init(smem_u32(&S.empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&S.acc_full[a]), 1);
            // the group that drains it (d <= 256), or all epilogue warps (d = 512)
            mbar_init(smem_u32(&S.acc_empty[a]), (NH == 4 ? kEpiWarps : kGroupWarps) * 32);
        }
        mbar_init(smem_u32(&S.drain), 1);
        for (int a = 0; a < 2; ++a)
            for (int q = 0; q < 4; ++q) mbar_init(smem_u32(&S.pair[a][q]), NH == 4 ? 128 : 64);   // warps of a quadrant
        fence_mbar_init();
    }
    if (warp == kWarpTma && lane == 0) prefetch_tensormap(&p.tmap);

    // B_l = H diag(s_l), s_l the signs of coordinates 128 l .. 128 l + 127, as
    // [n = output coordinate][k = input coordinate], K-major, two 64-column blocks
    // of 128-byte swizzled rows (the layout TMA gives A).  For d = 256 the
    // Sylvester recursion H_256 = [[H, H], [H, -H]] gives y = (z_0 + z_1, z_0 - z_1)
    // with z_l = B_l k_l, which the epilogue forms.
    if constexpr (kBlock) {
        // piece (part, slice l, group j) at ((part * NH + l) * 8 + j) * kBlkBytes
        for (int e = threadIdx.x; e < NH * 8 * 256; e += kThreads) {
            const int l = e / (8 * 256), j = (e / 256) % 8, n = (e / 16) % 16, k = e % 16;
            float v = 0.0f;
            if ((n >> 2) == (k >> 2)) {
                Quat qL, qRc;
                const int m = 32 * l + 4 * j + (n >> 2);
                if (AXR_IN(p.sp_quats, p.quats + 8 * m, 32)) {
                    block_quats(p.quats, m, qL, qRc);
                } else {
                    unit_quats(qL, qRc);
                }
                const int c = k & 3;
                const Quat y = block_rotate(qL, qRc, {c == 0 ? 1.0f : 0.0f, c == 1 ? 1.0f : 0.0f,
                                                      c == 2 ? 1.0f : 0.0f, c == 3 ? 1.0f : 0.0f});
                const int r = n & 3;
                v = r == 0 ? y.w : r == 1 ? y.x : r == 2 ? y.y : y.z;
            }
            float rest = v;
#pragma unroll
            for (int part = 0; part < kParts; ++part) {
                float back;
                const uint16_t bits = to_half_bits<kBF16>(rest, back);
                rest -= back;
                *reinterpret_cast<uint16_t *>(sB + ((part * NH + l) * 8 + j) * kBlkBytes + blk_offset(n, k)) = bits;
            }
        }
    } else
    for (int chunk = threadIdx.x; chunk < NH * kD * (kD / 8); chunk += kThreads) {
        const int l = chunk / (kD * (kD / 8));
        const int n = (chunk / (kD / 8)) % kD;
        const int c = chunk % (kD / 8);          // 8-element chunk along k
        uint32_t w[4];
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
            uint32_t pair = 0;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int k = 8 * c + 2 * e2 + h;
                const int8_t *sg = p.signs + kD * l + k;
                const bool neg = ((__popc(n & k) & 1) != 0) != (AXR_IN(p.sp_signs, sg, 1) && *sg < 0);
                const uint16_t one = kBF16 ? (neg ? 0xBF80 : 0x3F80) : (neg ? 0xBC00 : 0x3C00);
                pair |= static_cast<uint32_t>(one) << (16 * h);
            }
            w[e2] = pair;
        }
        const int kb = c / 8, cc = c % 8;
        uint4 *dst = reinterpret_cast<uint4 *>(sB + l * kBBytes + kb * kHalfBytes + n * 128 + ((cc ^ (n & 7)) * 16));
        *dst = make_uint4(w[0], w[1], w[2], w[3]);
    }
    for (int j = threadIdx.x; j < kMaxBuckets; j += kThreads)
        sTab[j] = table_entry(j < p.nt ? p.tau[j] : __int_as_float(0x7f800000), p.base[j]);
    fence_proxy_async_smem();
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
            bool stop = false;
            for (int t = blockIdx.x; t < p.ntiles && !stop; t += gridDim.x) {
                for (int l = 0; l < NH; ++l, ++it) {         // one stage per 128 coordinates
                    const int s = it % kSt;
                    const uint32_t ph = (it / kSt) & 1;
                    if (!mbar_wait(smem_u32(&S.empty[s]), ph ^ 1)) {
                        atomicOr(&g_status, kErrTimeoutMma);
                        stop = true;
                        break;
                    }
                    const uint32_t full = smem_u32(&S.full[s]);
                    mbar_arrive_expect_tx(full, kABytes);
                    tma_load_2d(smem_u32(sA + s * kABytes), &p.tmap, kD * l, t * kTileRows, full);
                    tma_load_2d(smem_u32(sA + s * kABytes + kHalfBytes), &p.tmap, kD * l + 64, t * kTileRows, full);
                }
            }
            // let every load this thread issued land before the CTA exits
            for (int k = 0; k < kSt && k < it; ++k) {
                const int j = it - 1 - k;
                mbar_wait(smem_u32(&S.full[j % kSt]), (j / kSt) & 1);
            }
        }
    } else if (warp == kWarpMma) {
        // --------------------------------------------------------------- MMA
        if (lane == 0) {
            const uint32_t id = idesc(kAccF32, kBF16 ? kFmtBF16 : kFmtF16, kBF16 ? kFmtBF16 : kFmtF16, 128, kD);
            const uint32_t id16 = idesc(kAccF32, kBF16 ? kFmtBF16 : kFmtF16, kBF16 ? kFmtBF16 : kFmtF16, 128, 16);
            const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
            int it = 0, st = 0;                               // tiles, stages
            bool stop = false;
            for (int t = blockIdx.x; t < p.ntiles && !stop; t += gridDim.x, ++it) {
                const int acc = (acc_bufs<NH>() == 1) ? 0 : (it & 1);
                const uint32_t aph = (acc_bufs<NH>() == 1) ? (it & 1) : ((it >> 1) & 1);
                if (!mbar_wait(smem_u32(&S.acc_empty[acc]), aph ^ 1)) {
                    atomicOr(&g_status, kErrTimeoutDrain);
                    break;
                }
                for (int l = 0; l < NH; ++l, ++st) {
                    const int s = st % kSt;
                    const uint32_t ph = (st / kSt) & 1;
                    if (!mbar_wait(smem_u32(&S.full[s]), ph)) {
                        atomicOr(&g_status, kErrTimeoutLoad);
                        stop = true;
                        break;
                    }
                    tc_fence_after_sync();
                    // accumulator acc holds z_0 .. z_{NH-1}, 128 columns each
                    const uint32_t d = tmem + (acc * NH + l) * kD;
                    if constexpr (kBlock) {
                        // 16 output columns per group, from the group's 16 key columns
                        // and the kParts terms of its piece of T
#pragma unroll
                        for (int k = 0; k < kD / 16; ++k) {
                            const uint32_t off = (k >> 2) * kHalfBytes + (k & 3) * 32;
                            const uint64_t ad = desc_k_sw128(a0 + s * kABytes + off);
#pragma unroll
                            for (int part = 0; part < kParts; ++part)
                                mma_f16_ss(d + 16 * k, ad,
                                           desc_k_interleave(b0 + ((part * NH + l) * 8 + k) * kBlkBytes, 128, 256),
                                           id16, part > 0);
                        }
                    } else {
#pragma unroll
                        for (int k = 0; k < kD / 16; ++k) {
                            const uint32_t off = (k >> 2) * kHalfBytes + (k & 3) * 32;
                            mma_f16_ss(d, desc_k_sw128(a0 + s * kABytes + off), desc_k_sw128(b0 + l * kBBytes + off),
                                       id, k > 0);
                        }
                    }
                    mma_commit(smem_u32(&S.empty[s]));
                }
                if (stop) break;
                mma_commit(smem_u32(&S.acc_full[acc]));
            }
            // all MMAs of this thread complete before the tensor memory is freed
            mma_commit(smem_u32(&S.drain));
            mbar_wait(smem_u32(&S.drain), 0);
        }
    } else {
        // ---------------------------------------------------------- epilogue
      if constexpr (NH == 4) {
        // d = 512: y = (H_4 (x) H) diag(s) k, so y_q = sum_l (-1)^popcount(q & l) z_l over
        // the four accumulators z_l = B_l k_l.  All 16 warps drain each tile: lane
        // quadrant `quad`, 32-column quarter `cq` of every z_l, 8 columns at a time.
        constexpr int NWQ = B;                       // packed words of 32 coordinates
        const int quad = warp & 3, cq = warp >> 2;
        const uint32_t col0 = tmem + (static_cast<uint32_t>(quad * 32) << 16) + cq * 32;
        const int key = quad * 32 + lane;
        float *ss4 = &S.ss[0][0][0];                 // [quarter][key]
        constexpr uint32_t kCentral = (1u << (B - 1)) - 1u;
        const uint32_t tab_u32 = smem_u32(sTab);
        const uint32_t tab_bias = tab_u32 - kMagicBits * 4u;     // wraps mod 2^32 by design
        int it = 0;
        for (int t = blockIdx.x; t < p.ntiles; t += gridDim.x, ++it) {
            const uint32_t aph = it & 1;
            if (!mbar_wait_warp(smem_u32(&S.acc_full[0]), aph)) {
                if (lane == 0) atomicOr(&g_status, kErrTimeoutMma);
                break;
            }
            tc_fence_after_sync();
            // pass 1: this quarter's sum of y^2 over the four outputs
            float2 p01 = make_float2(0.0f, 0.0f), p23 = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int pc = 0; pc < 4; ++pc) {
                uint32_t z[4][8];
#pragma unroll
                for (int l = 0; l < 4; ++l) tmem_ld8(col0 + l * kD + 8 * pc, z[l]);
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    float2 y[4];
                    h4<kBlock>(z, e, y);
                    p01 = __ffma2_rn(y[0], y[0], p01);
                    p01 = __ffma2_rn(y[1], y[1], p01);
                    p23 = __ffma2_rn(y[2], y[2], p23);
                    p23 = __ffma2_rn(y[3], y[3], p23);
                }
            }
            ss4[cq * kTileRows + key] = (p01.x + p01.y) + (p23.x + p23.y);
            mbar_arrive(smem_u32(&S.pair[0][quad]));
            if (!mbar_wait_warp(smem_u32(&S.pair[0][quad]), aph)) {
                if (lane == 0) atomicOr(&g_status, kErrTimeoutDrain);
                break;
            }
            const float ss = (ss4[key] + ss4[kTileRows + key]) + (ss4[2 * kTileRows + key] + ss4[3 * kTileRows + key]);
            const float norm = sqrtf(ss) * p.inv_sqrt_d;
            const bool finite = ss <= 3.402823466e38f;
            const bool clamp = !(ss >= 1e-36f);
            const float a = (finite && ss > 0.0f) ? p.g_scale / sqrtf(ss) : 0.0f;
            const float2 a2 = make_float2(a, a);
            const float2 offm2 = make_float2(p.g_off + kMagic, p.g_off + kMagic);
            const float ug = (finite && ss > 0.0f) ? 1.0f / sqrtf(ss) : 0.0f;
            const float2 ug2 = make_float2(ug, ug);
            uint32_t w[4][NWQ + 1];
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int i = 0; i <= NWQ; ++i) w[q][i] = 0;
            // pass 2: codes of y_q at coordinates 128 q + 32 cq + (8 pc .. 8 pc + 7)
#pragma unroll
            for (int pc = 0; pc < 4; ++pc) {
                uint32_t z[4][8];
#pragma unroll
                for (int l = 0; l < 4; ++l) tmem_ld8(col0 + l * kD + 8 * pc, z[l]);
                uint32_t v[4][32];                   // y_q in v[q][24 .. 31]
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    float2 y[4];
                    h4<kBlock>(z, e, y);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        v[q][24 + e] = __float_as_uint(y[q].x);
                        v[q][25 + e] = __float_as_uint(y[q].y);
                    }
                }
                if (pc == 3) {                       // every read of this tile's accumulators done
                    tc_fence_before_sync();
                    mbar_arrive(smem_u32(&S.acc_empty[0]));
                }
                if (finite) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        if (!clamp) quantize_piece<B, false>(pc, v[q], ug2, a2, offm2, tab_u32, tab_bias, w[q]);
                        else quantize_piece<B, true>(pc, v[q], ug2, a2, offm2, tab_u32, tab_bias, w[q]);
                    }
                }
            }
            if (!finite) {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int o = j * B;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        w[q][o >> 5] |= kCentral << (o & 31);
                        if ((o & 31) + B > 32) w[q][(o >> 5) + 1] |= kCentral >> (32 - (o & 31));
                    }
                }
            }
            const int64_t row = static_cast<int64_t>(t) * kTileRows + key;
            if (row < p.n) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint8_t *dst = p.idx + row * P + (4 * q + cq) * NWQ * 4;
                    if (AXR_IN(p.sp_idx, dst, NWQ * 4)) store_words<NWQ>(dst, w[q]);
                }
                if (cq == 0 && AXR_IN(p.sp_norms, p.norms + row, 4)) __stcs(p.norms + row, norm);
            }
        }
      } else {
        constexpr int kHalfCols = kD / 2;
        constexpr int NWH = NW / 2;                  // packed words per half row
        // group e drains accumulator e: the CTA's tiles 2m + e, so two tiles are
        // in the epilogue at once
        const int grp = warp / kGroupWarps;
        const int quad = warp & 3, half = (warp >> 2) & 1;
        const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
        const int key = quad * 32 + lane;            // key within the tile
        constexpr uint32_t kCentral = (1u << (B - 1)) - 1u;
        const uint32_t tab_u32 = smem_u32(sTab);
        const uint32_t tab_bias = tab_u32 - kMagicBits * 4u;     // wraps mod 2^32 by design
        int it = 0;
        const int acc = grp;
        for (int t = blockIdx.x + grp * gridDim.x; t < p.ntiles; t += 2 * gridDim.x, ++it) {
            const uint32_t aph = it & 1;
            if (!mbar_wait_warp(smem_u32(&S.acc_full[acc]), aph)) {
                if (lane == 0) atomicOr(&g_status, kErrTimeoutMma);
                break;
            }
            tc_fence_after_sync();
            // this warp's 64 columns of z_0 (and of z_1 at d = 256)
            const uint32_t col_addr = tmem + lane_base + acc * NH * kD + half * kHalfCols;
            // pass 1: this half's sum of y^2 (four interleaved partial sums); the
            // pair adds both halves in a fixed order
            // (partial sums 0,1 and 2,3 in paired FMAs: coordinates e = 0, 1 mod 4 and 2, 3 mod 4;
            // at d = 256, 0,1 for y = z_0 + z_1 and 2,3 for y = z_0 - z_1)
            float2 p01 = make_float2(0.0f, 0.0f), p23 = make_float2(0.0f, 0.0f);
            // d = 128: the half's 64 columns are read once, with one wait, and held
            // for pass 2; the accumulator is released once both halves' sums are read
            uint32_t vh[NH == 1 ? 2 * 32 : 1];
            if constexpr (NH == 1) {
                tmem_ld64(col_addr, vh);
#pragma unroll
                for (int e = 0; e < 2 * 32; e += 4) {
                    const float2 x01 = make_float2(__uint_as_float(vh[e]), __uint_as_float(vh[e + 1]));
                    const float2 x23 = make_float2(__uint_as_float(vh[e + 2]), __uint_as_float(vh[e + 3]));
                    p01 = __ffma2_rn(x01, x01, p01);
                    p23 = __ffma2_rn(x23, x23, p23);
                }
            } else {
#pragma unroll
                for (int c = 0; c < kHalfCols / 32; ++c) {
                    uint32_t v[32];
                    tmem_ld32(col_addr + 32 * c, v);
                    uint32_t v1[32];
                    tmem_ld32(col_addr + kD + 32 * c, v1);
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const float2 z0 = make_float2(__uint_as_float(v[e]), __uint_as_float(v[e + 1]));
                        const float2 z1 = make_float2(__uint_as_float(v1[e]), __uint_as_float(v1[e + 1]));
                        const float2 ya = kBlock ? z0 : __fadd2_rn(z0, z1);
                        const float2 yb = kBlock ? z1 : __ffma2_rn(z1, make_float2(-1.0f, -1.0f), z0);
                        p01 = __ffma2_rn(ya, ya, p01);
                        p23 = __ffma2_rn(yb, yb, p23);
                    }
                }
            }
            S.ss[acc][half][key] = (p01.x + p01.y) + (p23.x + p23.y);
            mbar_arrive(smem_u32(&S.pair[acc][quad]));
            if (!mbar_wait_warp(smem_u32(&S.pair[acc][quad]), aph)) {
                if (lane == 0) atomicOr(&g_status, kErrTimeoutDrain);
                break;
            }
            const float ss = S.ss[acc][0][key] + S.ss[acc][1][key];
            if constexpr (NH == 1) {
                // the accumulator is in registers.  Releasing it only now, after the
                // read of the other half's sum, keeps the group's next tile on this
                // accumulator (which needs every thread's release) from overwriting
                // S.ss[acc] before that read
                tc_fence_before_sync();
                mbar_arrive(smem_u32(&S.acc_empty[acc]));
            }
            const float norm = sqrtf(ss) * p.inv_sqrt_d;

            uint32_t w[NWH + 1], w1[NWH + 1];      // codes of y (z_0 + z_1 at d = 256) and of z_0 - z_1
#pragma unroll
            for (int i = 0; i <= NWH; ++i) w[i] = w1[i] = 0;
            // pass 2: quantize and pack this half, 32 coordinates at a time.  The
            // tensor-memory loads stay outside the per-key branches (warp-collective).
            // |y| <= sqrt(ss) keeps round(g) inside the table; a zero or denormal
            // sum, where that bound can fail, takes the clamped copy of the body; a
            // non-finite key stores the central index.
            const bool finite = ss <= 3.402823466e38f;
            const bool clamp = !(ss >= 1e-36f);
            const float a = (finite && ss > 0.0f) ? p.g_scale / sqrtf(ss) : 0.0f;
            const float2 a2 = make_float2(a, a);
            const float2 offm2 = make_float2(p.g_off + kMagic, p.g_off + kMagic);
            const float ug = (finite && ss > 0.0f) ? 1.0f / sqrtf(ss) : 0.0f;
            const float2 ug2 = make_float2(ug, ug);
            if constexpr (NH == 1) {
                const uint32_t(&va)[32] = *reinterpret_cast<const uint32_t(*)[32]>(&vh[0]);
                const uint32_t(&vb)[32] = *reinterpret_cast<const uint32_t(*)[32]>(&vh[32]);
                if (finite && !clamp) quantize_chunk<B, 0, 0, false>(va, ug2, a2, offm2, tab_u32, tab_bias, w);
                else if (finite) quantize_chunk<B, 0, 0, true>(va, ug2, a2, offm2, tab_u32, tab_bias, w);
                if (finite && !clamp) quantize_chunk<B, 32, 0, false>(vb, ug2, a2, offm2, tab_u32, tab_bias, w);
                else if (finite) quantize_chunk<B, 32, 0, true>(vb, ug2, a2, offm2, tab_u32, tab_bias, w);
            } else {
#pragma unroll
                for (int c = 0; c < kHalfCols / 32; ++c) {
                    uint32_t v[32], v1[32];
                    tmem_ld32(col_addr + 32 * c, v);
                    tmem_ld32(col_addr + kD + 32 * c, v1);
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const float2 z0 = make_float2(__uint_as_float(v[e]), __uint_as_float(v[e + 1]));
                        const float2 z1 = make_float2(__uint_as_float(v1[e]), __uint_as_float(v1[e + 1]));
                        const float2 ya = kBlock ? z0 : __fadd2_rn(z0, z1);
                        const float2 yb = kBlock ? z1 : __ffma2_rn(z1, make_float2(-1.0f, -1.0f), z0);
                        v[e] = __float_as_uint(ya.x);
                        v[e + 1] = __float_as_uint(ya.y);
                        v1[e] = __float_as_uint(yb.x);
                        v1[e + 1] = __float_as_uint(yb.y);
                    }
                    if (c == 0) {
                        if (finite && !clamp) {
                            quantize_chunk<B, 0, 0, false>(v, ug2, a2, offm2, tab_u32, tab_bias, w);
                            quantize_chunk<B, 0, 0, false>(v1, ug2, a2, offm2, tab_u32, tab_bias, w1);
                        } else if (finite) {
                            quantize_chunk<B, 0, 0, true>(v, ug2, a2, offm2, tab_u32, tab_bias, w);
                            quantize_chunk<B, 0, 0, true>(v1, ug2, a2, offm2, tab_u32, tab_bias, w1);
                        }
                    } else {
                        if (finite && !clamp) {
                            quantize_chunk<B, 32, 0, false>(v, ug2, a2, offm2, tab_u32, tab_bias, w);
                            quantize_chunk<B, 32, 0, false>(v1, ug2, a2, offm2, tab_u32, tab_bias, w1);
                        } else if (finite) {
                            quantize_chunk<B, 32, 0, true>(v, ug2, a2, offm2, tab_u32, tab_bias, w);
                            quantize_chunk<B, 32, 0, true>(v1, ug2, a2, offm2, tab_u32, tab_bias, w1);
                        }
                    }
                }
            }
            if (!finite) {
#pragma unroll
                for (int j = 0; j < kHalfCols; ++j) {
                    const int o = j * B;
                    w[o >> 5] |= kCentral << (o & 31);
                    w1[o >> 5] |= kCentral << (o & 31);
                    if ((o & 31) + B > 32) {
                        w[(o >> 5) + 1] |= kCentral >> (32 - (o & 31));
                        w1[(o >> 5) + 1] |= kCentral >> (32 - (o & 31));
                    }
                }
            }
            if constexpr (NH != 1) {
                tc_fence_before_sync();
                mbar_arrive(smem_u32(&S.acc_empty[acc]));
            }

            const int64_t row = static_cast<int64_t>(t) * kTileRows + key;
            if (row < p.n) {
                // this warp's 64 coordinates of each 128: runs of NWH words at
                // coordinates 64 half and (d = 256) 128 + 64 half
                uint8_t *dst = p.idx + row * P + half * (NWH * 4);
                if (AXR_IN(p.sp_idx, dst, NWH * 4)) store_run<NWH>(dst, w);
                if constexpr (NH == 2) {
                    if (AXR_IN(p.sp_idx, dst + 2 * NWH * 4, NWH * 4)) store_run<NWH>(dst + 2 * NWH * 4, w1);
                }
                if (half == 0 && AXR_IN(p.sp_norms, p.norms + row, 4)) __stcs(p.norms + row, norm);
            }
        }
      }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ host side

template <int B, bool kBF16, int NH, bool kBlock>
cudaError_t launch_tc(const QuantizeArgs &a, const BucketTable &tab, cudaStream_t stream)
{
    constexpr int D = kD * NH;
    auto kernel = quantize_keys_tc_kernel<B, kBF16, NH, kBlock>;
    constexpr size_t kBReg = kBlock ? block_parts<kBF16>() * NH * 8 * kBlkBytes : NH * kBBytes;
    const size_t smem = 1024 + stages<NH>() * kABytes + kBReg + kMaxBuckets * sizeof(uint32_t) + sizeof(Smem);
    static_assert(1024 + stages<NH>() * kABytes + kBReg + kMaxBuckets * sizeof(uint32_t) + sizeof(Smem) <= 232448,
                  "shared memory per block");
    static std::atomic<unsigned long long> smem_allowed{0};     // one bit per device
    if (cudaError_t e = allow_dynamic_smem(reinterpret_cast<const void *>(kernel), smem, smem_allowed);
        e != cudaSuccess)
        return e;
    TcParams p{};
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(a.n)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
    const cuuint32_t box[2] = {64, kTileRows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(&p.tmap, kBF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                     const_cast<void *>(a.K), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    p.idx = a.idx;
    p.norms = a.norms;
    p.signs = a.signs;
    p.n = a.n;
    p.ntiles = static_cast<int>((a.n + kTileRows - 1) / kTileRows);
    p.g_scale = tab.g_scale;
    p.g_off = tab.g_off;
    // |y|^2 = d |k|^2 for the unnormalised Walsh-Hadamard product, |k|^2 for the
    // (orthonormal) block rotation
    p.inv_sqrt_d = kBlock ? 1.0f : 1.0f / sqrtf(static_cast<float>(D));
    p.quats = a.quats;
    p.nt = tab.nt;
    // the codebook boundary each bucket holds, in u units (the kernel compares u itself)
    for (int j = 0; j < kMaxBuckets; ++j) {
        const bool has = j < tab.nt && tab.tau[j] < INFINITY;
        p.tau[j] = has ? a.cb.boundaries[tab.base[j]] : INFINITY;
        p.base[j] = tab.base[j];
    }
    AXR_DEBUG_ONLY(const int64_t rows = a.out_rows ? a.out_rows : a.n;
                   p.sp_idx = dbg::span(a.idx, static_cast<uint64_t>(rows) * (D * B / 8));
                   p.sp_norms = dbg::span(a.norms, static_cast<uint64_t>(rows) * sizeof(float));
                   p.sp_signs = dbg::span(a.signs, a.signs ? D : 0);
                   p.sp_quats = dbg::span(a.quats, a.quats ? (D / 4) * 8 * sizeof(float) : 0);)
    const int grid = p.ntiles < device_sm_count() ? p.ntiles : device_sm_count();
    kernel<<<grid, kThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

template <bool kBF16, int NH, bool kBlock>
cudaError_t launch_typed(const QuantizeArgs &a, const BucketTable &tab, cudaStream_t stream)
{
    switch (a.b) {
    case 1: return launch_tc<1, kBF16, NH, kBlock>(a, tab, stream);
    case 2: return launch_tc<2, kBF16, NH, kBlock>(a, tab, stream);
    case 3: return launch_tc<3, kBF16, NH, kBlock>(a, tab, stream);
    default: return launch_tc<4, kBF16, NH, kBlock>(a, tab, stream);
    }
}

template <int NH, bool kBlock>
cudaError_t launch_width(const QuantizeArgs &a, const BucketTable &tab, cudaStream_t stream)
{
    return a.kdtype == AXR_BF16 ? launch_typed<true, NH, kBlock>(a, tab, stream)
                                : launch_typed<false, NH, kBlock>(a, tab, stream);
}

template <bool kBlock>
cudaError_t launch_transform(const QuantizeArgs &a, const BucketTable &tab, cudaStream_t stream)
{
    switch (a.d) {
    case 2 * kD: return launch_width<2, kBlock>(a, tab, stream);
    case 4 * kD: return launch_width<4, kBlock>(a, tab, stream);
    default: return launch_width<1, kBlock>(a, tab, stream);
    }
}

}  // namespace

bool quantize_tc_supported(const QuantizeArgs &a)
{
    return (a.d == kD || a.d == 2 * kD || a.d == 4 * kD) && (a.kdtype == AXR_BF16 || a.kdtype == AXR_F16) &&
           a.n > 0 &&
           a.out_stride == 1 &&
           a.out_offset == 0 &&
           a.n <= static_cast<int64_t>(0x7fffffff) - kTileRows && encode_tiled() != nullptr;
}

cudaError_t launch_quantize_keys_tc(const QuantizeArgs &a, cudaStream_t stream)
{
    BucketTable tab;
    if (!get_bucket_table(a.d, a.b, &tab)) return cudaErrorInvalidValue;
    return a.quats ? launch_transform<true>(a, tab, stream) : launch_transform<false>(a, tab, stream);
}

unsigned int quantize_tc_status(bool clear)
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
