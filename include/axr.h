/*
 * axr.h -- C ABI of libaxr: AXELRAM-style quantize-on-write and LUT score-on-read
 * for the key cache of attention, on NVIDIA B200 (sm_100a).
 *
 * Method: "AXELRAM: Quantize Once, Never Dequantize" (arXiv 2604.02638), abstract.
 * Keys are rotated by a sign-flipped orthonormal Walsh-Hadamard transform, which
 * makes every coordinate of a unit key close to N(0, 1/d); each coordinate is then
 * scalar-quantized to a codebook fixed at design time by d and b alone.  Scores
 * are read straight from the stored indices through lookup tables built from the
 * once-rotated query; the keys are never dequantized or rotated back.
 *
 * Conventions shared by every entry point
 *   - All buffers are owned by the caller.  The library never allocates device
 *     memory; it keeps only a host-side, thread-safe cache of codebooks.
 *   - Device-pointer arguments must be device (or managed) memory of the current
 *     device; memory of another device is refused with AXR_EINVAL.  Calls
 *     enqueue work on `stream` and return without synchronising;
 *     results are valid once the stream has reached that point.
 *   - Argument errors are detected on the host before any launch and return
 *     AXR_EINVAL / AXR_EUNSUPPORTED with nothing enqueued.  A failed launch
 *     returns AXR_ECUDA.  axr_last_error() gives a message for the calling thread.
 *   - n == 0 is a no-op that returns AXR_OK.
 *   - Inputs must be finite, with squared key norms inside the fp32 range.
 *   - The sign pattern `signs` is an int8 device vector of length d with entries
 *     +1 or -1 (any negative entry counts as -1, anything else as +1).  One
 *     pattern serves a whole layer: keys and queries of that layer must use the
 *     same one (AXELRAM abstract: the transform's sign pattern, chosen once).
 *   - Supported shapes: d a power of two in [8, 512]; b in {1, 2, 3, 4};
 *     group in [1, 8].
 *   - The read calls run the tensor-core kernels at d = 128, 256 and 512 and the
 *     CUDA-core kernel otherwise.  AXR_READ_KERNEL=cuda_core in the environment
 *     (read once per process) routes every read to the CUDA-core kernel, to
 *     compare the two; the results agree within the score tolerance.
 *
 * Packed index layout (one row per key, P = d*b/8 bytes, rows back to back):
 *   bit i of idx_j is bit (j*b + i) of the row's bit stream, and byte k of the
 *   row holds stream bits 8k .. 8k+7, least significant first.  idx 0 is the most
 *   negative centroid.  (The pages only say the indices are stored; this dense
 *   little-endian layout is this library's choice.)
 */
#ifndef AXR_H
#define AXR_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum axr_status {
    AXR_OK = 0,
    AXR_EINVAL = -1,        /* null/misaligned pointer, negative size, bad dtype   */
    AXR_EUNSUPPORTED = -2,  /* d, b or group outside the supported set            */
    AXR_ECUDA = -3          /* a CUDA call failed; see axr_last_error()           */
} axr_status;

typedef enum axr_dtype {
    AXR_F32 = 0,
    AXR_F16 = 1,
    AXR_BF16 = 2
} axr_dtype;

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *axr_stream;

/*
 * Design-time codebook (AXELRAM abstract: the optimal scalar quantizer of a
 * rotated coordinate depends on d and b only, never on the data; the paper's
 * repository lists a Lloyd-Max solver for it).
 *
 * Host only.  Fills caller-owned HOST arrays:
 *   centroids[2^b]   Lloyd-Max centroids of N(0, 1/d), ascending, fp32,
 *                    exactly symmetric (c[L-1-i] == -c[i]);
 *   boundaries[2^b-1] fp32 of the midpoint of neighbouring centroids
 *                    (may be NULL if not wanted).
 * Returns AXR_OK, AXR_EINVAL (centroids NULL) or AXR_EUNSUPPORTED (d, b).
 */
int axr_make_codebook(int d, int b, float *centroids, float *boundaries);

/*
 * Quantize-on-write (AXELRAM abstract: keys are transformed once, on write).
 * For every key row k (length d):
 *   norm = ||k||_2 (fp32 accumulation), stored;
 *   y = H * diag(signs) * k, H the Sylvester-ordered Walsh-Hadamard matrix;
 *   u = y / (sqrt(d) * norm)          (the unit key in the rotated basis);
 *   idx_j = number of codebook boundaries t_i with u_j > t_i
 *           (= nearest centroid, ties to the lower index);
 *   the d indices are bit-packed into P = d*b/8 bytes (layout above).
 * A key of norm 0 stores norm 0 and idx_j = 2^(b-1) - 1 for every j.
 *
 * K      device, n x d row-major, element type kdtype; 16-byte aligned.
 * signs  device int8[d].
 * idx    device uint8[n * P] output; 16-byte aligned.
 * norms  device float[n] output; 4-byte aligned.
 */
int axr_quantize_keys(const void *K, int kdtype, int64_t n, int d, int b,
                      const int8_t *signs, uint8_t *idx, float *norms,
                      axr_stream stream);

/*
 * Score-on-read (AXELRAM abstract: table lookup on read, no inverse transform).
 * Each query is rotated once, q' = H * diag(signs) * q / sqrt(d); then for every
 * stored key t of its KV head
 *   scores[t] = norms[t] * sum_j q'_j * c[idx_t[j]] / sqrt(d)
 * where the last 1/sqrt(d) is the attention temperature.  The keys are never
 * dequantized.  Grouped-query attention: query head h*group + g reads KV head h,
 * so one index stream serves all `group` queries of a KV head.  A batch is
 * folded into `heads` (heads = batch * KV heads).
 *
 * q       device, (heads*group) x d row-major, element type qdtype; 16-byte aligned.
 * idx     device, heads x n x P bytes (as written by axr_quantize_keys); 16-byte aligned.
 * norms   device float[heads * n].
 * signs   device int8[d], the pattern the keys were written with.
 * scores  device float[(heads*group) * n] output, row h*group+g holds the n
 *         scores of that query head.
 */
int axr_scores(const void *q, int qdtype, const uint8_t *idx, const float *norms,
               int64_t n, int heads, int group, int d, int b, const int8_t *signs,
               float *scores, axr_stream stream);

/*
 * One decode step on a key cache (AXELRAM abstract: keys are quantized once, when
 * written; every read is a table lookup on the stored indices).  For every KV
 * head h the new key k_new[h] is quantized exactly as axr_quantize_keys would
 * and stored in slot `pos` of that head's cache; then every query head scores
 * keys 0 .. pos of its KV head exactly as axr_scores would.
 *
 * k_new   device, heads x d row-major, element type kdtype; 16-byte aligned.
 * q       device, (heads*group) x d row-major, element type qdtype; 16-byte aligned.
 * idx     device, heads x capacity x P bytes (P = d*b/8): the packed cache, head h
 *         at rows [h*capacity, (h+1)*capacity); 16-byte aligned.  Rows < pos hold
 *         earlier keys; row pos is overwritten; rows > pos are neither read for
 *         scores nor written.
 * norms   device float[heads * capacity], laid out like idx; row pos is overwritten.
 * capacity  keys each head's cache holds, >= 1; 0 <= pos < capacity (else AXR_EINVAL).
 * scores  device float[(heads*group) * (pos+1)] output; row h*group+g holds the
 *         pos+1 scores of that query head (row stride pos+1).
 * At d = 128, 256 and 512 both parts run in one kernel launch (the tensor-core
 * read quantizes the new keys itself); at smaller d they are two launches,
 * enqueued on `stream` in order.  The call is asynchronous like the others.
 */
int axr_append_scores(const void *k_new, int kdtype, const void *q, int qdtype, uint8_t *idx,
                      float *norms, int64_t capacity, int64_t pos, int heads, int group, int d, int b,
                      const int8_t *signs, float *scores, axr_stream stream);

/*
 * Decode attention on the quantized keys.  The pages define the scores only; this
 * is the standard attention that consumes them: for query head h*group + g,
 *   p = softmax over t of scores[h*group + g, t]     (t = 0 .. n-1)
 *   out[h*group + g, :] = sum_t p_t * V[h, t, :]
 * with the scores exactly as axr_scores computes them (they are also returned).
 * The values are read as stored (not quantized).
 *
 * q, idx, norms, signs as for axr_scores (16/16/4/1-byte aligned).
 * V          device, heads x n x d row-major, element type vdtype; 16-byte aligned.
 * scores     device float[(heads*group) * n] output (the scores); 16-byte aligned.
 * workspace  device scratch of at least axr_attention_workspace_bytes(...) bytes,
 *            16-byte aligned, owned by the caller; its contents on entry do not
 *            matter and on exit are unspecified.  Calls that share a workspace
 *            must not overlap in time.
 * out        device float[(heads*group) * d] output.
 * d must be a power of two in [32, 512]; n >= 1.  Three kernels are enqueued on
 * `stream` in order (scores, per-chunk partial softmax sums, their merge).
 */
int axr_attention_workspace_bytes(int64_t n, int heads, int group, int d, int64_t *bytes);
int axr_attention(const void *q, int qdtype, const uint8_t *idx, const float *norms, const void *V, int vdtype,
                  int64_t n, int heads, int group, int d, int b, const int8_t *signs, float *scores,
                  void *workspace, int64_t workspace_bytes, float *out, axr_stream stream);

/*
 * axr_attention without a workspace argument: the same computation, with the
 * partial sums kept in a fixed 16 MiB scratch area that the library carries in
 * device memory (one per device).  The method has no counterpart to this call;
 * it exists for callers that cannot hand the library device memory of their own:
 * a plain C program with no device allocator at hand, code that runs with a fixed
 * device-memory budget that must not grow, or a latency-bound decode loop that
 * cannot afford the synchronisation an allocation may cause.
 *
 * Arguments as for axr_attention, less workspace and workspace_bytes.
 * Limit: shapes whose axr_attention_workspace_bytes exceed 16 MiB (16777216
 *   bytes) return AXR_EUNSUPPORTED with nothing enqueued; 131072 keys x 32 KV heads
 *   x 4 queries per head at d = 128 need 8.5 MB.
 * Set-up: the first call on a device looks up the scratch address there (with
 *   that device current), and the first call for a (d, b) pair solves its
 *   codebook on the host; later calls allocate nothing, on the host or the
 *   device.  Make the first call on each device before any stream capture.
 * Nothing in the scratch needs clearing: every call writes each partial sum it
 *   later reads.
 * Overlapping calls race: all calls on one device share the scratch, so two of
 *   them in flight at once (on different streams or from different threads)
 *   corrupt each other's results.  Order them (one stream, or events).
 */
int axr_attention_static(const void *q, int qdtype, const uint8_t *idx, const float *norms, const void *V,
                         int vdtype, int64_t n, int heads, int group, int d, int b, const int8_t *signs,
                         float *scores, float *out, axr_stream stream);

/*
 * Quantize-on-write with a block rotation in place of the sign flip and the
 * Walsh-Hadamard transform (IsoQuant, arXiv 2603.28430, abstract: the d
 * coordinates form d/4 blocks of 4, each read as a quaternion v = v0 + v1 i +
 * v2 j + v3 k and turned into qL v conj(qR); IsoQuant-Full, or IsoQuant-Fast
 * when every qR is 1).  Then as axr_quantize_keys: the fp32 norm of the key is
 * stored, the rotated unit key u = T k / |k| is quantized to the same Lloyd-Max
 * codebook of N(0, 1/d) and bit-packed in the same layout.
 *
 *   K      device, (n, d) row-major keys of kdtype, 16-byte aligned;
 *   quats  device float (d/4, 8), 16-byte aligned: block m's qL then qR, each
 *          (w, x, y, z), unit quaternions (used as given; the transform is
 *          orthonormal only if they are unit);
 *   idx    device uint8 (n, d*b/8), 16-byte aligned, written;
 *   norms  device float (n), written.
 *
 * The caller owns every buffer; one kernel on `stream`, no allocation.  Both
 * variants cost the same here (each block's two products are composed into one
 * 4 x 4 matrix).  Errors as axr_quantize_keys; n = 0 is a no-op.  Keys written
 * this way are read with axr_scores_block and the same quats.
 */
int axr_quantize_keys_block(const void *K, int kdtype, int64_t n, int d, int b, const float *quats,
                            uint8_t *idx, float *norms, axr_stream stream);

/*
 * Score-on-read for keys written by axr_quantize_keys_block: each query is
 * rotated once by the same block rotation, q' = T q, and
 * score[t] = |k_t| * sum_j q'_j c[idx_t[j]] / sqrt(d), with no inverse transform
 * of the keys.  Arguments, layouts and errors as axr_scores, with quats (as in
 * axr_quantize_keys_block) in place of signs.
 */
int axr_scores_block(const void *q, int qdtype, const uint8_t *idx, const float *norms, int64_t n, int heads,
                     int group, int d, int b, const float *quats, float *scores, axr_stream stream);

/*
 * Sign-pattern choice (AXELRAM, arXiv 2604.02638, abstract: the sign pattern is
 * chosen once, without gradients, among candidates (200) on a few calibration
 * samples (8); some patterns cause large errors on heads whose key norms stand
 * out).  The pages rank candidates by perplexity, which needs a model; this call
 * ranks them by the error of the attention logits that the quantized cache
 * gives.  For candidate c and KV head h,
 *   errors[c*heads + h] = mean over samples s, query heads g < group and keys t
 *                         of (score_c - q.k / sqrt(d))^2,
 * with score_c the score that axr_quantize_keys + axr_scores would give with
 * signs = candidate c, q = q[s, h*group + g] and k = K[s, h, t] (fp32 arithmetic,
 * accumulated in fp64 in a fixed order: the result is deterministic).  *best
 * (if best is not NULL) receives the index of the candidate whose worst head
 * has the smallest error, the lowest index among equal values (-1 only if every
 * candidate has a NaN error, which only non-finite inputs give).
 *
 *   K           device, (samples, heads, n, d) row-major keys of kdtype, 16-byte
 *               aligned: the calibration keys of one layer, sample by sample;
 *   q           device, (samples, heads*group, d) queries of qdtype (element
 *               aligned); query head h*group + g of sample s reads KV head h;
 *   candidates  device int8 (n_candidates, d): candidate sign patterns, a
 *               negative entry is -1, any other +1;
 *   errors      device float (n_candidates, heads), written;
 *   best        device int32, one element, written; or NULL.
 *
 * The caller owns every buffer; the call allocates nothing and enqueues two
 * kernels on `stream` (one if best is NULL).  AXR_EINVAL for NULL or misaligned
 * pointers, n < 1, samples, heads, group or n_candidates < 1, or more than
 * 2^31 - 1 (candidate, head) pairs; AXR_EUNSUPPORTED for d or b outside the
 * write path's range or group above 8.
 */
int axr_select_signs(const void *K, int kdtype, const void *q, int qdtype, int64_t n, int samples, int heads,
                     int group, int d, int b, const int8_t *candidates, int n_candidates, float *errors,
                     int32_t *best, axr_stream stream);

/*
 * Device-side status of the kernels (no counterpart in the method; a
 * diagnostic).  Every wait inside the tensor-core kernels is bounded; a wait that
 * runs out records a bit here instead of hanging: 1 = a tile load never arrived,
 * 2 = a matrix product never completed, 4 = an accumulator was never released;
 * 8 = the read kernel found its shared-memory window laid out so that its stages
 * do not fit, and scored nothing.  In the debug build (libaxr_debug.so) every
 * kernel also checks each plain global load and store against the buffer the
 * call's arguments describe, skips one that falls outside (a load reads zeros)
 * and records 16.
 * Synchronizes the current device, writes the OR of the recorded bits to
 * *status (0 = none) and clears them if `clear` is non-zero.
 */
int axr_device_status(int clear, unsigned int *status);

/* 1 in the debug build (libaxr_debug.so, compiled with AXR_DEBUG: device-side
 * bounds checks, status bit 16), 0 in the release build (libaxr.so). */
int axr_debug_build(void);

/*
 * Debug build only: shorten, for every later launch, each buffer span the bounds
 * checks allow by `bytes` (>= 0; 0 restores the exact spans), so that the last
 * accesses of every buffer count as outside and are skipped with status bit 16
 * although they lie in the real allocation.  For testing that the checks fire
 * without any access leaving its buffer.  Process-wide, not thread-safe against
 * concurrent launches.  AXR_EINVAL for bytes < 0; AXR_EUNSUPPORTED in the
 * release build.
 */
int axr_debug_set_span_slack(int64_t bytes);

/* Static string naming a status code. */
const char *axr_status_string(int status);

/* Message describing the last failure on the calling thread ("" if none). */
const char *axr_last_error(void);

/* Library version, major*10000 + minor*100 + patch. */
int axr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* AXR_H */
