// Internal declarations shared by the libaxr translation units (not installed).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "axr.h"

namespace axr {

constexpr int kMaxBits = 4;
constexpr int kMaxLevels = 1 << kMaxBits;
constexpr int kMaxGroup = 8;

// fp32 codebook for one (d, b): what the kernels receive by value.
struct Codebook {
    int d = 0;
    int b = 0;
    float centroids[kMaxLevels] = {};
    float boundaries[kMaxLevels - 1] = {};
};

// Host solver and cache (codebook.cpp).  Returns false for unsupported (d, b).
bool get_codebook(int d, int b, Codebook *out);

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
};

// Kernel launchers (quantize_keys.cu, scores.cu).  They return cudaSuccess or
// the launch error; arguments are already validated.
cudaError_t launch_quantize_keys(const QuantizeArgs &a, cudaStream_t stream);
cudaError_t launch_scores(const ScoresArgs &a, cudaStream_t stream);

// Number of SMs of the current device (cached per device).
int device_sm_count();

}  // namespace axr
