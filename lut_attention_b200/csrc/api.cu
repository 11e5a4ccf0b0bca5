// extern "C" entry points of libaxr: argument validation, codebook lookup and
// kernel launch.  Every check runs on the host before anything is enqueued.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "axr_internal.cuh"

namespace axr {
namespace {

thread_local char g_last_error[512] = "";

int fail(int status, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    std::vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return status;
}

int ok()
{
    g_last_error[0] = '\0';
    return AXR_OK;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool pow2_in_range(int d) { return d >= 8 && d <= 512 && (d & (d - 1)) == 0; }

int elem_size(int dtype) { return dtype_bytes(dtype); }

// Where a pointer lives, for the current device's kernels: device memory of the
// current device, managed memory, or host memory mapped into the device address
// space are usable; memory of another device is reported as such (a kernel here
// would fault on it without peer access).
enum class Access { kUsable, kOtherDevice, kNone };

Access device_access(const void *p, int *owner)
{
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
        cudaGetLastError();
        return Access::kNone;
    }
    switch (attr.type) {
    case cudaMemoryTypeDevice: {
        int cur = 0;
        if (cudaGetDevice(&cur) != cudaSuccess) return Access::kNone;
        *owner = attr.device;
        return attr.device == cur ? Access::kUsable : Access::kOtherDevice;
    }
    case cudaMemoryTypeManaged: return Access::kUsable;
    case cudaMemoryTypeHost: return attr.devicePointer != nullptr ? Access::kUsable : Access::kNone;
    default: return Access::kNone;
    }
}

int check_device_ptr(const void *p, uintptr_t align, const char *name)
{
    if (!p) return fail(AXR_EINVAL, "%s is NULL", name);
    if (!aligned(p, align)) return fail(AXR_EINVAL, "%s is not %u-byte aligned", name, (unsigned)align);
    int owner = -1;
    switch (device_access(p, &owner)) {
    case Access::kUsable: return AXR_OK;
    case Access::kOtherDevice:
        return fail(AXR_EINVAL, "%s is memory of device %d, not of the current device", name, owner);
    default: return fail(AXR_EINVAL, "%s is not device-accessible memory", name);
    }
}

int check_shape(int d, int b)
{
    if (!pow2_in_range(d)) return fail(AXR_EUNSUPPORTED, "d=%d: must be a power of two in [8, 512]", d);
    if (b < 1 || b > kMaxBits) return fail(AXR_EUNSUPPORTED, "b=%d: must be in [1, %d]", b, kMaxBits);
    return AXR_OK;
}

}  // namespace

int device_sm_count()
{
    static std::mutex mu;
    static std::vector<int> counts;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    std::lock_guard<std::mutex> lock(mu);
    if ((int)counts.size() <= dev) counts.resize(dev + 1, 0);
    if (counts[dev] == 0) {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
            sms = 148;
        counts[dev] = sms;
    }
    return counts[dev];
}

EncodeTiledFn encode_tiled()
{
    static const EncodeTiledFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiledFn>(p);
        return static_cast<EncodeTiledFn>(nullptr);
    }();
    return fn;
}

cudaError_t allow_dynamic_smem(const void *kernel, size_t bytes, std::atomic<unsigned long long> &done)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = dev < 64 ? (1ull << dev) : 0ull;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

namespace dbg {
namespace {
std::mutex g_reader_mu;
std::vector<Reader> &readers()
{
    static std::vector<Reader> v;
    return v;
}
#ifdef AXR_DEBUG
std::atomic<int64_t> g_slack{0};
#endif
}  // namespace

bool register_reader(Reader r)
{
    std::lock_guard<std::mutex> lock(g_reader_mu);
    readers().push_back(r);
    return true;
}

unsigned read_all(bool clear)
{
    std::lock_guard<std::mutex> lock(g_reader_mu);
    unsigned v = 0;
    for (Reader r : readers()) {
        const unsigned x = r(clear);
        if (x == ~0u) return ~0u;
        v |= x;
    }
    return v;
}

#ifdef AXR_DEBUG
void set_slack(int64_t bytes) { g_slack.store(bytes, std::memory_order_relaxed); }

Span span(const void *base, uint64_t bytes)
{
    const uint64_t slack = static_cast<uint64_t>(g_slack.load(std::memory_order_relaxed));
    return Span{reinterpret_cast<uintptr_t>(base), bytes > slack ? bytes - slack : 0};
}
#endif
}  // namespace dbg

}  // namespace axr

using namespace axr;

extern "C" int axr_make_codebook(int d, int b, float *centroids, float *boundaries)
{
    int rc = check_shape(d, b);
    if (rc != AXR_OK) return rc;
    if (!centroids) return fail(AXR_EINVAL, "centroids is NULL");
    Codebook cb;
    if (!get_codebook(d, b, &cb)) return fail(AXR_EUNSUPPORTED, "no codebook for d=%d b=%d", d, b);
    const int L = 1 << b;
    std::memcpy(centroids, cb.centroids, sizeof(float) * L);
    if (boundaries) std::memcpy(boundaries, cb.boundaries, sizeof(float) * (L - 1));
    return ok();
}

extern "C" int axr_quantize_keys(const void *K, int kdtype, int64_t n, int d, int b,
                                 const int8_t *signs, uint8_t *idx, float *norms,
                                 axr_stream stream)
{
    int rc = check_shape(d, b);
    if (rc != AXR_OK) return rc;
    if (elem_size(kdtype) == 0) return fail(AXR_EINVAL, "kdtype=%d is not an axr_dtype", kdtype);
    if (n < 0) return fail(AXR_EINVAL, "n=%lld is negative", (long long)n);
    if (n == 0) return ok();
    if ((rc = check_device_ptr(K, 16, "K")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(signs, 1, "signs")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(idx, 16, "idx")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(norms, 4, "norms")) != AXR_OK) return rc;

    QuantizeArgs a{K, kdtype, n, d, b, signs, idx, norms, Codebook{}};
    if (!get_codebook(d, b, &a.cb)) return fail(AXR_EUNSUPPORTED, "no codebook for d=%d b=%d", d, b);
    cudaError_t e = quantize_tc_supported(a) ? launch_quantize_keys_tc(a, reinterpret_cast<cudaStream_t>(stream))
                                             : launch_quantize_keys(a, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(AXR_ECUDA, "quantize_keys launch: %s", cudaGetErrorString(e));
    return ok();
}

extern "C" int axr_scores(const void *q, int qdtype, const uint8_t *idx, const float *norms,
                          int64_t n, int heads, int group, int d, int b, const int8_t *signs,
                          float *scores, axr_stream stream)
{
    int rc = check_shape(d, b);
    if (rc != AXR_OK) return rc;
    if (elem_size(qdtype) == 0) return fail(AXR_EINVAL, "qdtype=%d is not an axr_dtype", qdtype);
    if (n < 0) return fail(AXR_EINVAL, "n=%lld is negative", (long long)n);
    if (heads < 1) return fail(AXR_EINVAL, "heads=%d must be >= 1", heads);
    if (group < 1) return fail(AXR_EINVAL, "group=%d must be >= 1", group);
    if (group > kMaxGroup) return fail(AXR_EUNSUPPORTED, "group=%d: at most %d", group, kMaxGroup);
    if (n == 0) return ok();
    if (n > (int64_t)INT32_MAX) return fail(AXR_EUNSUPPORTED, "n=%lld: at most 2^31-1 keys per head", (long long)n);
    if ((rc = check_device_ptr(q, 16, "q")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(idx, 16, "idx")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(norms, 4, "norms")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(signs, 1, "signs")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(scores, 4, "scores")) != AXR_OK) return rc;

    ScoresArgs a{q, qdtype, idx, norms, n, heads, group, d, b, signs, scores, Codebook{}};
    a.head_stride = n;
    if (!get_codebook(d, b, &a.cb)) return fail(AXR_EUNSUPPORTED, "no codebook for d=%d b=%d", d, b);
    cudaError_t e = scores_tc_supported(a) ? launch_scores_tc(a, reinterpret_cast<cudaStream_t>(stream))
                                           : launch_scores(a, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(AXR_ECUDA, "scores launch: %s", cudaGetErrorString(e));
    return ok();
}

extern "C" int axr_append_scores(const void *k_new, int kdtype, const void *q, int qdtype, uint8_t *idx,
                                 float *norms, int64_t capacity, int64_t pos, int heads, int group, int d, int b,
                                 const int8_t *signs, float *scores, axr_stream stream)
{
    int rc = check_shape(d, b);
    if (rc != AXR_OK) return rc;
    if (elem_size(kdtype) == 0) return fail(AXR_EINVAL, "kdtype=%d is not an axr_dtype", kdtype);
    if (elem_size(qdtype) == 0) return fail(AXR_EINVAL, "qdtype=%d is not an axr_dtype", qdtype);
    if (heads < 1) return fail(AXR_EINVAL, "heads=%d must be >= 1", heads);
    if (group < 1) return fail(AXR_EINVAL, "group=%d must be >= 1", group);
    if (group > kMaxGroup) return fail(AXR_EUNSUPPORTED, "group=%d: at most %d", group, kMaxGroup);
    if (capacity < 1) return fail(AXR_EINVAL, "capacity=%lld must be >= 1", (long long)capacity);
    if (capacity > (int64_t)INT32_MAX)
        return fail(AXR_EUNSUPPORTED, "capacity=%lld: at most 2^31-1 keys per head", (long long)capacity);
    if (pos < 0 || pos >= capacity)
        return fail(AXR_EINVAL, "pos=%lld is outside the cache [0, %lld)", (long long)pos, (long long)capacity);
    if ((rc = check_device_ptr(k_new, 16, "k_new")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(q, 16, "q")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(idx, 16, "idx")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(norms, 4, "norms")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(signs, 1, "signs")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(scores, 4, "scores")) != AXR_OK) return rc;

    Codebook cb;
    if (!get_codebook(d, b, &cb)) return fail(AXR_EUNSUPPORTED, "no codebook for d=%d b=%d", d, b);
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // every query head against keys 0 .. pos of its KV head
    ScoresArgs sa{q, qdtype, idx, norms, pos + 1, heads, group, d, b, signs, scores, cb};
    sa.head_stride = capacity;
    ScoresArgs fused = sa;
    fused.k_new = k_new;
    fused.kdtype = kdtype;
    fused.append_pos = pos;
    fused.idx_out = idx;
    fused.norms_out = norms;
    cudaError_t e;
    if (scores_tc_supported(fused)) {
        // one launch: the tensor-core read kernel quantizes the new key of each
        // head into row h * capacity + pos itself, in the CTA that scores it
        e = launch_scores_tc(fused, st);
    } else {
        // two launches: the new key of KV head h goes to cache row h * capacity + pos
        QuantizeArgs qa{k_new, kdtype, heads, d, b, signs, idx, norms, cb};
        qa.out_stride = capacity;
        qa.out_offset = pos;
        qa.out_rows = static_cast<int64_t>(heads) * capacity;
        e = launch_quantize_keys(qa, st);
        if (e == cudaSuccess) e = scores_tc_supported(sa) ? launch_scores_tc(sa, st) : launch_scores(sa, st);
    }
    if (e != cudaSuccess) return fail(AXR_ECUDA, "decode step launch: %s", cudaGetErrorString(e));
    return ok();
}

extern "C" int axr_attention_workspace_bytes(int64_t n, int heads, int group, int d, int64_t *bytes)
{
    if (!bytes) return fail(AXR_EINVAL, "bytes is NULL");
    if (!pow2_in_range(d) || d < 32) return fail(AXR_EUNSUPPORTED, "d=%d: attention needs a power of two in [32, 512]", d);
    if (n < 0 || heads < 1 || group < 1) return fail(AXR_EINVAL, "n, heads or group out of range");
    if (group > kMaxGroup) return fail(AXR_EUNSUPPORTED, "group=%d: at most %d", group, kMaxGroup);
    *bytes = n == 0 ? 0 : attention_workspace_bytes(n, heads, group, d);
    return ok();
}

extern "C" int axr_attention(const void *q, int qdtype, const uint8_t *idx, const float *norms, const void *V,
                             int vdtype, int64_t n, int heads, int group, int d, int b, const int8_t *signs,
                             float *scores, void *workspace, int64_t workspace_bytes, float *out,
                             axr_stream stream)
{
    int rc = check_shape(d, b);
    if (rc != AXR_OK) return rc;
    if (d < 32) return fail(AXR_EUNSUPPORTED, "d=%d: attention needs d >= 32", d);
    if (elem_size(qdtype) == 0) return fail(AXR_EINVAL, "qdtype=%d is not an axr_dtype", qdtype);
    if (elem_size(vdtype) == 0) return fail(AXR_EINVAL, "vdtype=%d is not an axr_dtype", vdtype);
    if (n < 1) return fail(AXR_EINVAL, "n=%lld: attention needs at least one key", (long long)n);
    if (heads < 1) return fail(AXR_EINVAL, "heads=%d must be >= 1", heads);
    if (group < 1) return fail(AXR_EINVAL, "group=%d must be >= 1", group);
    if (group > kMaxGroup) return fail(AXR_EUNSUPPORTED, "group=%d: at most %d", group, kMaxGroup);
    if (n > (int64_t)INT32_MAX) return fail(AXR_EUNSUPPORTED, "n=%lld: at most 2^31-1 keys per head", (long long)n);
    const int64_t need = attention_workspace_bytes(n, heads, group, d);
    if (workspace_bytes < need)
        return fail(AXR_EINVAL, "workspace_bytes=%lld: needs %lld", (long long)workspace_bytes, (long long)need);
    if ((rc = check_device_ptr(q, 16, "q")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(idx, 16, "idx")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(norms, 4, "norms")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(V, 16, "V")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(signs, 1, "signs")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(scores, 16, "scores")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(workspace, 16, "workspace")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(out, 4, "out")) != AXR_OK) return rc;

    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    ScoresArgs sa{q, qdtype, idx, norms, n, heads, group, d, b, signs, scores, Codebook{}};
    sa.head_stride = n;
    if (!get_codebook(d, b, &sa.cb)) return fail(AXR_EUNSUPPORTED, "no codebook for d=%d b=%d", d, b);
    cudaError_t e = scores_tc_supported(sa) ? launch_scores_tc(sa, st) : launch_scores(sa, st);
    if (e != cudaSuccess) return fail(AXR_ECUDA, "scores launch: %s", cudaGetErrorString(e));
    AttentionArgs aa{scores, V, vdtype, n, heads, group, d, workspace, out};
    e = launch_attention(aa, st);
    if (e != cudaSuccess) return fail(AXR_ECUDA, "attention launch: %s", cudaGetErrorString(e));
    return ok();
}

extern "C" int axr_attention_static(const void *q, int qdtype, const uint8_t *idx, const float *norms,
                                    const void *V, int vdtype, int64_t n, int heads, int group, int d, int b,
                                    const int8_t *signs, float *scores, float *out, axr_stream stream)
{
    int rc = check_shape(d, b);
    if (rc != AXR_OK) return rc;
    if (d < 32) return fail(AXR_EUNSUPPORTED, "d=%d: attention needs d >= 32", d);
    if (elem_size(qdtype) == 0) return fail(AXR_EINVAL, "qdtype=%d is not an axr_dtype", qdtype);
    if (elem_size(vdtype) == 0) return fail(AXR_EINVAL, "vdtype=%d is not an axr_dtype", vdtype);
    if (n < 1) return fail(AXR_EINVAL, "n=%lld: attention needs at least one key", (long long)n);
    if (heads < 1) return fail(AXR_EINVAL, "heads=%d must be >= 1", heads);
    if (group < 1) return fail(AXR_EINVAL, "group=%d must be >= 1", group);
    if (group > kMaxGroup) return fail(AXR_EUNSUPPORTED, "group=%d: at most %d", group, kMaxGroup);
    if (n > (int64_t)INT32_MAX) return fail(AXR_EUNSUPPORTED, "n=%lld: at most 2^31-1 keys per head", (long long)n);
    const int64_t need = attention_workspace_bytes(n, heads, group, d);
    if (need > static_attention_scratch_bytes())
        return fail(AXR_EUNSUPPORTED,
                    "this shape needs %lld bytes of scratch; the fixed scratch holds %lld (use axr_attention "
                    "with a workspace)",
                    (long long)need, (long long)static_attention_scratch_bytes());
    if ((rc = check_device_ptr(q, 16, "q")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(idx, 16, "idx")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(norms, 4, "norms")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(V, 16, "V")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(signs, 1, "signs")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(scores, 16, "scores")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(out, 4, "out")) != AXR_OK) return rc;

    void *scratch = nullptr;
    cudaError_t e = static_attention_scratch(&scratch);
    if (e != cudaSuccess) return fail(AXR_ECUDA, "fixed scratch address: %s", cudaGetErrorString(e));
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    ScoresArgs sa{q, qdtype, idx, norms, n, heads, group, d, b, signs, scores, Codebook{}};
    sa.head_stride = n;
    if (!get_codebook(d, b, &sa.cb)) return fail(AXR_EUNSUPPORTED, "no codebook for d=%d b=%d", d, b);
    e = scores_tc_supported(sa) ? launch_scores_tc(sa, st) : launch_scores(sa, st);
    if (e != cudaSuccess) return fail(AXR_ECUDA, "scores launch: %s", cudaGetErrorString(e));
    AttentionArgs aa{scores, V, vdtype, n, heads, group, d, scratch, out};
    e = launch_attention(aa, st);
    if (e != cudaSuccess) return fail(AXR_ECUDA, "attention launch: %s", cudaGetErrorString(e));
    return ok();
}

extern "C" int axr_quantize_keys_block(const void *K, int kdtype, int64_t n, int d, int b, const float *quats,
                                       uint8_t *idx, float *norms, axr_stream stream)
{
    int rc = check_shape(d, b);
    if (rc != AXR_OK) return rc;
    if (elem_size(kdtype) == 0) return fail(AXR_EINVAL, "kdtype=%d is not an axr_dtype", kdtype);
    if (n < 0) return fail(AXR_EINVAL, "n=%lld is negative", (long long)n);
    if (n == 0) return ok();
    if ((rc = check_device_ptr(K, 16, "K")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(quats, 16, "quats")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(idx, 16, "idx")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(norms, 4, "norms")) != AXR_OK) return rc;
    QuantizeArgs a{K, kdtype, n, d, b, nullptr, idx, norms, Codebook{}};
    a.quats = quats;
    if (!get_codebook(d, b, &a.cb)) return fail(AXR_EUNSUPPORTED, "no codebook for d=%d b=%d", d, b);
    // bf16/fp16 keys of d = 128, 256, 512 on the tensor cores, the rest on CUDA cores
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const cudaError_t e = quantize_tc_supported(a) ? launch_quantize_keys_tc(a, st) : launch_quantize_keys_block(a, st);
    if (e != cudaSuccess) return fail(AXR_ECUDA, "block-rotation quantize launch: %s", cudaGetErrorString(e));
    return ok();
}

extern "C" int axr_scores_block(const void *q, int qdtype, const uint8_t *idx, const float *norms, int64_t n,
                                int heads, int group, int d, int b, const float *quats, float *scores,
                                axr_stream stream)
{
    int rc = check_shape(d, b);
    if (rc != AXR_OK) return rc;
    if (elem_size(qdtype) == 0) return fail(AXR_EINVAL, "qdtype=%d is not an axr_dtype", qdtype);
    if (n < 0) return fail(AXR_EINVAL, "n=%lld is negative", (long long)n);
    if (heads < 1) return fail(AXR_EINVAL, "heads=%d must be >= 1", heads);
    if (group < 1) return fail(AXR_EINVAL, "group=%d must be >= 1", group);
    if (group > kMaxGroup) return fail(AXR_EUNSUPPORTED, "group=%d: at most %d", group, kMaxGroup);
    if (n > (int64_t)INT32_MAX) return fail(AXR_EUNSUPPORTED, "n=%lld: at most 2^31-1 keys per head", (long long)n);
    if (n == 0) return ok();
    if ((rc = check_device_ptr(q, 16, "q")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(idx, 16, "idx")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(norms, 4, "norms")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(quats, 16, "quats")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(scores, 4, "scores")) != AXR_OK) return rc;
    ScoresArgs a{q, qdtype, idx, norms, n, heads, group, d, b, nullptr, scores, Codebook{}};
    a.head_stride = n;
    a.quats = quats;
    if (!get_codebook(d, b, &a.cb)) return fail(AXR_EUNSUPPORTED, "no codebook for d=%d b=%d", d, b);
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const cudaError_t e = scores_tc_supported(a) ? launch_scores_tc(a, st) : launch_scores(a, st);
    if (e != cudaSuccess) return fail(AXR_ECUDA, "block-rotation scores launch: %s", cudaGetErrorString(e));
    return ok();
}

extern "C" int axr_select_signs(const void *K, int kdtype, const void *q, int qdtype, int64_t n, int samples,
                                int heads, int group, int d, int b, const int8_t *candidates, int n_candidates,
                                float *errors, int32_t *best, axr_stream stream)
{
    int rc = check_shape(d, b);
    if (rc != AXR_OK) return rc;
    if (elem_size(kdtype) == 0) return fail(AXR_EINVAL, "kdtype=%d is not an axr_dtype", kdtype);
    if (elem_size(qdtype) == 0) return fail(AXR_EINVAL, "qdtype=%d is not an axr_dtype", qdtype);
    if (n < 1) return fail(AXR_EINVAL, "n=%lld: the choice needs at least one calibration key", (long long)n);
    if (samples < 1) return fail(AXR_EINVAL, "samples=%d must be >= 1", samples);
    if (heads < 1) return fail(AXR_EINVAL, "heads=%d must be >= 1", heads);
    if (group < 1) return fail(AXR_EINVAL, "group=%d must be >= 1", group);
    if (n_candidates < 1) return fail(AXR_EINVAL, "n_candidates=%d must be >= 1", n_candidates);
    if (group > kMaxGroup) return fail(AXR_EUNSUPPORTED, "group=%d: at most %d", group, kMaxGroup);
    if ((int64_t)n_candidates * heads > (int64_t)INT32_MAX)
        return fail(AXR_EINVAL, "%d candidates x %d heads: at most 2^31-1 pairs", n_candidates, heads);
    if ((rc = check_device_ptr(K, 16, "K")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(q, (uintptr_t)elem_size(qdtype), "q")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(candidates, 1, "candidates")) != AXR_OK) return rc;
    if ((rc = check_device_ptr(errors, 4, "errors")) != AXR_OK) return rc;
    if (best && (rc = check_device_ptr(best, 4, "best")) != AXR_OK) return rc;

    SignSelectArgs a{K, kdtype, q, qdtype, n, samples, heads, group, d, b, candidates, n_candidates, errors, best,
                     Codebook{}};
    if (!get_codebook(d, b, &a.cb)) return fail(AXR_EUNSUPPORTED, "no codebook for d=%d b=%d", d, b);
    const cudaError_t e = launch_sign_select(a, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(AXR_ECUDA, "sign selection launch: %s", cudaGetErrorString(e));
    return ok();
}

extern "C" const char *axr_status_string(int status)
{
    switch (status) {
    case AXR_OK: return "AXR_OK";
    case AXR_EINVAL: return "AXR_EINVAL: invalid argument";
    case AXR_EUNSUPPORTED: return "AXR_EUNSUPPORTED: unsupported d, b or group";
    case AXR_ECUDA: return "AXR_ECUDA: CUDA error";
    default: return "unknown axr status";
    }
}

extern "C" int axr_device_status(int clear, unsigned int *status)
{
    if (!status) return fail(AXR_EINVAL, "status is NULL");
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return fail(AXR_ECUDA, "device synchronize: %s", cudaGetErrorString(e));
    const unsigned int q = quantize_tc_status(clear != 0);
    const unsigned int r = scores_tc_status(clear != 0);
    const unsigned int bnd = dbg::read_all(clear != 0);
    if (q == ~0u || r == ~0u || bnd == ~0u) return fail(AXR_ECUDA, "reading the device status words failed");
    *status = q | r | bnd;
    return ok();
}

extern "C" int axr_debug_build(void)
{
#ifdef AXR_DEBUG
    return 1;
#else
    return 0;
#endif
}

extern "C" int axr_debug_set_span_slack(int64_t bytes)
{
    if (bytes < 0) return fail(AXR_EINVAL, "bytes=%lld must be >= 0", (long long)bytes);
#ifdef AXR_DEBUG
    dbg::set_slack(bytes);
    return ok();
#else
    return fail(AXR_EUNSUPPORTED, "span slack exists only in the debug build (libaxr_debug.so)");
#endif
}

extern "C" const char *axr_last_error(void) { return g_last_error; }

extern "C" int axr_version(void) { return 100; }
