// Pieces shared by the tensor-core read kernels (scores_tc.cu for 256- and
// 512-wide heads, scores_tc128.cu for 128-wide heads): the fixed-point digits
// that turn the per-coordinate lookup tables of the read path into an exact
// int32 contraction, and the per-lane table the digits are looked up in.
//
// AXELRAM (arXiv 2604.02638), abstract: scores come from table lookups on the
// stored indices, never from dequantized keys.  For the G query heads of a KV
// head the scores of a tile of 128 keys form one small contraction,
// s[t][g] = norm_t * sum_j c[idx_t[j]] * q''_g[j]:
//   * every centroid becomes two signed 8-bit digits of a fixed-point number,
//     c * 128 * S_c = 128 * hi + lo  (|hi| <= 127, |lo| <= 64, S_c = 127/max|c|);
//   * every rotated query coordinate becomes three signed 8-bit digits,
//     q'' * S_q = D0 + D1/128 + D2/128^2  (|D| <= 64, S_q = 64/max|q''|);
//   * A (tensor memory) holds the hi and lo digits of the looked-up centroids,
//     K = 2 * 128 per 128 coordinates; B (shared memory) holds the query
//     digits, N = 4 columns per query with weights (128, 1, 1/128, 1/128^2):
//         hi rows (D0, D1, D2, 0),   lo rows (0, D0, D1, D2)
//     so one kind::i8 product yields, for every query, sum_j q'' c 128 S_q S_c
//     as four exact int32 partial sums.
// The digit error is at most 0.5 / (128 * 127) of the largest centroid per
// coordinate; with the query digits the score error stays below 1e-4 of
// ||q|| ||k|| / sqrt(d) for every head width and bit count served (the worst
// case is about 8.6e-5, at b = 4).
//
// Decoding a packed index row into A is a table walk: each lookup takes one
// field of the row (one byte = 2 codes at b = 4 or 4 codes at b = 2, a 6-bit
// pair at b = 3, a nibble of 4 codes at b = 1) and reads the digits of all its
// codes from a table replicated per lane (entry (field, lane) at
// field * 256 + lane * entry size), which is conflict-free in shared memory.
// The table sits on a 64 KB boundary of the shared window, so one PRMT forms a
// whole address from a byte field.
#pragma once

#include <cmath>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "axr_internal.cuh"

namespace axr {
namespace lut {

constexpr int kD = 128;               // coordinates of one slice (one K block of 2 * 128 digits)
constexpr int kK = 2 * kD;            // two digits per coordinate
constexpr int kLutBytes = 256 * 256;  // up to 256 fields x 256 bytes

// geometry of one lookup for b bits: C codes per lookup, FB field bits
template <int B>
struct Lookup {
    static constexpr int C = (B >= 3) ? 2 : 4;
    static constexpr int FB = C * B;              // 8, 6, 8, 4
    static constexpr int EB = 2 * C;              // entry bytes: C hi digits, C lo digits
    static constexpr int NF = 1 << FB;            // table fields
    // b = 3: the table is indexed by a whole byte, and a second one sits in the
    // unused upper half of every 256-byte row (lane offsets 128 + 4 lane):
    // the first reads the 6-bit field in bits 0..5 of the byte, the second in
    // bits 2..7, so a field that starts 0 or 2 bits into a byte costs one PRMT
    static constexpr bool kByteTables = (B == 3);
    static constexpr int kRows = kByteTables ? 256 : NF;
    static constexpr int kLookups = kD / C;       // per 128 coordinates
    static constexpr int kColsPerLookup = EB / 4; // 32-bit tensor-memory columns each lookup fills
};

// Centroid digits of a codebook (host): hi[i], lo[i] and 1 / (128 S_c).
inline void centroid_digits(const Codebook &cb, int8_t hi[kMaxLevels], int8_t lo[kMaxLevels], float *inv_sc)
{
    const int L = 1 << cb.b;
    const float cmax = std::fabs(cb.centroids[L - 1]);
    const double sc = 127.0 / cmax;
    *inv_sc = static_cast<float>(1.0 / (128.0 * sc));
    for (int i = 0; i < kMaxLevels; ++i) {
        const double v = (i < L) ? cb.centroids[i] * 128.0 * sc : 0.0;
        const long vi = std::lrint(v);
        const long h = std::lrint(static_cast<double>(vi) / 128.0);
        hi[i] = static_cast<int8_t>(h);
        lo[i] = static_cast<int8_t>(vi - 128 * h);
    }
}

// Contiguous tile ranges for the persistent CTAs of a read kernel (host): CTA c
// scores tiles [starts[c], starts[c + 1]).  A CTA whose range crosses into a new
// KV head rebuilds its query digits there, which the split charges as
// change_cost tiles: the cost of the tiles before t is
//     t + change_cost * floor(t / tiles_per_head),
// and each CTA gets an equal share of the total cost, so CTAs with a head change
// get fewer tiles and all end together.
constexpr int kMaxCtas = 160;
inline void balanced_ranges(int total_tiles, int tiles_per_head, int ctas, int change_cost, int *starts)
{
    const int64_t tph = tiles_per_head, cc = change_cost;
    const int64_t total = total_tiles + cc * (total_tiles / tiles_per_head - 1);
    starts[0] = 0;
    for (int c = 1; c < ctas; ++c) {
        const int64_t target = total * c / ctas;
        // first t whose cost reaches target: inside head h (cost h (tph + cc) + r)
        // at t = h tph + r, or at the next head's first tile if target falls
        // into the jump at the boundary
        const int64_t h = target / (tph + cc);
        const int64_t r = target - h * (tph + cc);
        const int64_t t = r < tph ? h * tph + r : (h + 1) * tph;
        starts[c] = static_cast<int>(t < total_tiles ? t : total_tiles);
    }
    starts[ctas] = total_tiles;
}

__device__ __forceinline__ float load_q(const void *q, int dtype, int64_t i)
{
    switch (dtype) {
    case AXR_F32: return static_cast<const float *>(q)[i];
    case AXR_F16: return __half2float(static_cast<const __half *>(q)[i]);
    default: return __bfloat162float(static_cast<const __nv_bfloat16 *>(q)[i]);
    }
}

// B offset of element (n, k) in the no-swizzle K-major layout: 8-row x 16-byte
// core matrices, K-adjacent ones 128 bytes apart, N-adjacent ones kK*8 bytes apart
__device__ __forceinline__ int b_offset(int n, int k)
{
    return ((n >> 3) * (kK / 16) + (k >> 4)) * 128 + (n & 7) * 16 + (k & 15);
}

// K rows of coordinate j's hi and lo digits: lookup l = j / C fills K indices
// EB*l .. EB*l + EB - 1 (C hi digits, then C lo digits)
template <int B>
__device__ __forceinline__ void digit_rows(int j, int &k_hi, int &k_lo)
{
    using LK = Lookup<B>;
    const int l = j / LK::C, t = j % LK::C;
    k_hi = LK::EB * l + t;
    k_lo = LK::EB * l + LK::C + t;
}

// The three digits of one rotated query coordinate Q = q'' S_q (|Q| <= 64) in
// the B rows of query qi: hi row (D0, D1, D2, 0), lo row (0, D0, D1, D2)
__device__ __forceinline__ void write_query_digits(uint8_t *b, int qi, int k_hi, int k_lo, float Q)
{
    const float d0 = rintf(Q);
    const float r1 = (Q - d0) * 128.0f;
    const float d1 = rintf(r1);
    const float d2 = rintf((r1 - d1) * 128.0f);
    const uint8_t D0 = static_cast<uint8_t>(static_cast<int8_t>(d0));
    const uint8_t D1 = static_cast<uint8_t>(static_cast<int8_t>(d1));
    const uint8_t D2 = static_cast<uint8_t>(static_cast<int8_t>(d2));
    b[b_offset(4 * qi + 0, k_hi)] = D0;
    b[b_offset(4 * qi + 1, k_hi)] = D1;
    b[b_offset(4 * qi + 2, k_hi)] = D2;
    b[b_offset(4 * qi + 3, k_hi)] = 0;
    b[b_offset(4 * qi + 0, k_lo)] = 0;
    b[b_offset(4 * qi + 1, k_lo)] = D0;
    b[b_offset(4 * qi + 2, k_lo)] = D1;
    b[b_offset(4 * qi + 3, k_lo)] = D2;
}

// The four int32 sums of one query (columns weighted 128, 1, 1/128, 1/128^2)
// joined into one float: pairs in int32 first (|128 c0 + c1| < 1.4e8,
// |128 c2 + c3| < 2.1e8), then one fused multiply-add
__device__ __forceinline__ float join_sums(const uint32_t *x)
{
    const int *v = reinterpret_cast<const int *>(x);
    const float hi = __int2float_rn(v[0] * 128 + v[1]);
    const float lo = __int2float_rn(v[2] * 128 + v[3]);
    return fmaf(lo, 1.0f / 16384.0f, hi);
}

// Table entry of one field value: C hi digits then C lo digits, replicated for
// the 32 lanes (entry (field, lane) at field * 256 + lane * EB).  One thread
// per (row, table) forms the entry once and writes its 32 copies as 16-byte
// chunks (4 or 2 copies each), starting at a chunk that rotates with the row so
// that the threads of a warp spread their stores over all banks.  Also built as
// host code, so that a CPU test can check the table against its definition.
template <int B>
__host__ __device__ void build_lut(const int8_t *hi, const int8_t *lo, uint8_t *lut, int tid, int nthreads)
{
    using LK = Lookup<B>;
    constexpr uint32_t mask = (1u << B) - 1u;
    constexpr int kTables = LK::kByteTables ? 2 : 1;
    constexpr int kChunks = 32 * LK::EB / 16;       // 16-byte chunks of one row of one table
    static_assert(LK::EB == 4 || LK::EB == 8, "entries of one or two words");
    static_assert(kTables * 32 * LK::EB <= 256, "a row holds every table's 32 entries");
    for (int e = tid; e < LK::kRows * kTables; e += nthreads) {
        const int row = e / kTables, tab = e % kTables;
        const int field = LK::kByteTables ? ((tab == 0) ? (row & (LK::NF - 1)) : (row >> 2)) : row;
        uint32_t words[2] = {0u, 0u};
#pragma unroll
        for (int i = 0; i < LK::C; ++i) {
            const int code = (field >> (B * i)) & mask;
            const int bh = i, bl = LK::C + i;       // byte positions of the hi and lo digit
            words[bh / 4] |= static_cast<uint32_t>(static_cast<uint8_t>(hi[code])) << (8 * (bh % 4));
            words[bl / 4] |= static_cast<uint32_t>(static_cast<uint8_t>(lo[code])) << (8 * (bl % 4));
        }
        const uint4 v = (LK::EB == 4) ? make_uint4(words[0], words[0], words[0], words[0])
                                      : make_uint4(words[0], words[1], words[0], words[1]);
        uint8_t *dst = lut + row * 256 + tab * 128;
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
            const int j = (c + e) & (kChunks - 1);
            *reinterpret_cast<uint4 *>(dst + 16 * j) = v;
        }
    }
}

// Shared-memory address of the table entry for lookup l of a row held in w[]
// (w[P/4] must be 0).  base_lane = table base (64 KB aligned) | lane * entry
// size, so the field only has to be placed in bits 8.. of it: one PRMT for
// byte fields (and, at b = 3, for fields starting 0 or 2 bits into a byte), a
// shift and one LOP3 otherwise.
template <int B>
__device__ __forceinline__ uint32_t lut_addr(const uint32_t *w, int l, uint32_t base_lane)
{
    using LK = Lookup<B>;
    const int bit = l * LK::FB;
    const int wi = bit >> 5, sh = bit & 31;
    if constexpr (LK::FB == 8) {
        // bytes: [lane offset, field, table base bits 16..23, 24..31]
        const uint32_t sel = 0x7604u | (static_cast<uint32_t>(sh >> 3) << 4);
        return __byte_perm(w[wi], base_lane, sel);
    } else if (LK::kByteTables && ((sh & 7) == 0 || (sh & 7) == 2)) {
        // the byte holding the field indexes the first table (field in bits
        // 0..5) or the second (bits 2..7, lane offsets + 128)
        const uint32_t sel = 0x7604u | (static_cast<uint32_t>(sh >> 3) << 4);
        return __byte_perm(w[wi], (sh & 7) == 0 ? base_lane : (base_lane | 128u), sel);
    } else {
        constexpr uint32_t fmask = ((1u << LK::FB) - 1u) << 8;
        uint32_t x;
        if (sh >= 8) {
            x = (sh + LK::FB <= 32) ? (w[wi] >> (sh - 8)) : __funnelshift_r(w[wi], w[wi + 1], sh - 8);
        } else {
            x = w[wi] << (8 - sh);
        }
        return (x & fmask) | base_lane;
    }
}

}  // namespace lut
}  // namespace axr
