// Internal declarations shared by the libaxr translation units (not installed).
#pragma once

#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "axr.h"
#include "bounds.cuh"

namespace axr {

constexpr int kMaxBits = 4;
constexpr int kMaxLevels = 1 << kMaxBits;
constexpr int kMaxGroup = 8;

// bytes of one element of an axr_dtype, 0 for anything else
__host__ __device__ inline int dtype_bytes(int dtype)
{
    return dtype == AXR_F32 ? 4 : (dtype == AXR_F16 || dtype == AXR_BF16) ? 2 : 0;
}

// fp32 codebook for one (d, b): what the kernels receive by value.
struct Codebook {
    int d = 0;
    int b = 0;
    float centroids[kMaxLevels] = {};
    float boundaries[kMaxLevels - 1] = {};
};

// Host solver and cache (codebook.cpp).  Returns false for unsupported (d, b).
bool get_codebook(int d, int b, Codebook *out);

// Bucket table for quantizing without a search (codebook.cpp).  A rotated unit
// coordinate u maps to g = u * g_scale + g_off; bucket j covers g in
// [j - 0.5, j + 0.5) and holds at most one decision boundary, tau[j] (in g
// units, +inf if none); base[j] is the number of boundaries below the bucket.
// Then idx(u) = base[round(g)] + (g > tau[round(g)]).  g_off is an integer and
// no boundary lies within `margin` (in g units) of a bucket edge.
constexpr int kMaxBuckets = 256;
struct BucketTable {
    int d = 0, b = 0, nt = 0;
    float g_scale = 0.0f, g_off = 0.0f, margin = 0.0f;
    float tau[kMaxBuckets] = {};
    int base[kMaxBuckets] = {};
};
bool get_bucket_table(int d, int b, BucketTable *out);

struct QuantizeArgs {
    const void *K;
    int kdtype;
    int64_t n;
    int d;
    int b;
    const int8_t *signs;
    uint8_t *idx;
    float *norms;
    Codebook cb;
    // key r is stored at row r * out_stride + out_offset of idx and norms
    // (1 and 0 for a dense batch; a cache's capacity and the write slot when one
    // key per head is appended)
    int64_t out_stride = 1;
    int64_t out_offset = 0;
    int64_t out_rows = 0;      // rows of idx and norms (0: n); what the bounds checks of the debug build allow
    // IsoQuant block rotation in place of diag(signs) and H: (d/4) x 8 floats,
    // qL then qR of every 4-element block (quantize_keys_block.cu)
    const float *quats = nullptr;
};

struct ScoresArgs {
    const void *q;
    int qdtype;
    const uint8_t *idx;
    const float *norms;
    int64_t n;
    int heads;
    int group;
    int d;
    int b;
    const int8_t *signs;
    float *scores;
    Codebook cb;
    int64_t head_stride = 0;   // rows between KV heads in idx and norms (n for a dense cache)
    // decode step fused into the read (tensor-core path): quantize k_new[h] into
    // row append_pos (= n - 1) of head h of idx_out / norms_out (the same cache)
    // before scoring it
    const void *k_new = nullptr;
    int kdtype = 0;
    int64_t append_pos = -1;
    uint8_t *idx_out = nullptr;
    float *norms_out = nullptr;
    // queries rotated by the IsoQuant block rotation instead of H diag(signs)
    const float *quats = nullptr;
};

// Kernel launchers (quantize_keys.cu, scores.cu).  They return cudaSuccess or
// the launch error; arguments are already validated.
cudaError_t launch_quantize_keys(const QuantizeArgs &a, cudaStream_t stream);
// Write path with the block rotation (quantize_keys_block.cu): every d, dense output.
cudaError_t launch_quantize_keys_block(const QuantizeArgs &a, cudaStream_t stream);

// Tensor-core write path (quantize_keys_tc.cu): d = 128, 256, 512, bf16/fp16 keys,
// with the Walsh-Hadamard transform or (quats set) the block rotation.
bool quantize_tc_supported(const QuantizeArgs &a);
cudaError_t launch_quantize_keys_tc(const QuantizeArgs &a, cudaStream_t stream);
unsigned int quantize_tc_status(bool clear);
cudaError_t launch_scores(const ScoresArgs &a, cudaStream_t stream);

// Tensor-core read path: d = 128 (scores_tc128.cu), d = 256 and 512
// (scores_tc.cu).  scores_tc_* dispatch on d and cover both.
bool scores_tc_supported(const ScoresArgs &a);
cudaError_t launch_scores_tc(const ScoresArgs &a, cudaStream_t stream);
unsigned int scores_tc_status(bool clear);
bool scores_tc128_supported(const ScoresArgs &a);
cudaError_t launch_scores_tc128(const ScoresArgs &a, cudaStream_t stream);
unsigned int scores_tc128_status(bool clear);

// Decode attention after the scores (attention.cu): softmax over each query
// head's n scores, weighted sum of its KV head's value rows.
struct AttentionArgs {
    const float *scores;       // (heads*group, n), already computed
    const void *V;             // (heads, n, d), vdtype
    int vdtype;
    int64_t n;
    int heads;
    int group;
    int d;
    void *workspace;           // attention_workspace_bytes(n, heads, group, d)
    float *out;                // (heads*group, d)
};
int attention_splits(int64_t n, int group);
int64_t attention_workspace_bytes(int64_t n, int heads, int group, int d);
cudaError_t launch_attention(const AttentionArgs &a, cudaStream_t stream);
// The fixed device scratch of axr_attention_static: its size, and its address on
// the current device (looked up on the device's first call, cached after).
int64_t static_attention_scratch_bytes();
cudaError_t static_attention_scratch(void **ptr);

// Sign-pattern choice (sign_select.cu): the calibration logit error of every
// candidate pattern per KV head, and the candidate with the smallest worst head.
struct SignSelectArgs {
    const void *K;             // (samples, heads, n, d), kdtype
    int kdtype;
    const void *q;             // (samples, heads*group, d), qdtype
    int qdtype;
    int64_t n;
    int samples;
    int heads;
    int group;
    int d;
    int b;
    const int8_t *candidates;  // (candidates_count, d)
    int candidates_count;
    float *errors;             // (candidates_count, heads)
    int *best;                 // one int, or nullptr
    Codebook cb;
};
cudaError_t launch_sign_select(const SignSelectArgs &a, cudaStream_t stream);

// Number of SMs of the current device (cached per device).
int device_sm_count();

// cuTensorMapEncodeTiled from the driver, looked up once; nullptr when the
// driver does not provide it (the tensor-core kernels are then not used).
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled();

// Raise a kernel's dynamic shared-memory limit to `bytes` on the current
// device.  The limit belongs to the kernel's instance in each device's context,
// so it is set once per device; `done` holds one bit per device (devices 64 and
// up are set on every call).  Safe to call from several host threads.
cudaError_t allow_dynamic_smem(const void *kernel, size_t bytes, std::atomic<unsigned long long> &done);

}  // namespace axr
