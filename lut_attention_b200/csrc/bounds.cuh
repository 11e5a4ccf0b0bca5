// Bounds checks of the debug build (libaxr_debug.so, compiled with -DAXR_DEBUG).
//
// In that build every kernel carries, for each global buffer it reads or
// writes with plain loads and stores, the span [base, base + bytes) that the
// call's own arguments describe (shapes times element sizes, computed on the
// host independently of the kernel's index arithmetic).  Each such access is
// checked against its span first; one that falls outside is not made (a load
// yields zeros) and sets kErrBounds in the bounds word of its translation
// unit, which axr_device_status reports.  Nothing traps or aborts: the kernel
// runs to its end, every barrier and wait stays matched, and the host reads
// the bit.  Tile loads through tensor maps (TMA) are bounded by the map's
// extents in hardware and need no check here.
//
// A test can shorten every span by a few bytes (axr_debug_set_span_slack):
// the last accesses of each buffer then count as outside although they stay in
// the real allocation, which shows that the checks fire without any access
// leaving its buffer.
//
// In the release build the spans do not exist, AXR_IN(...) is the constant
// true and AXR_DEBUG_ONLY(...) expands to nothing.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace axr {

constexpr unsigned kErrBounds = 16u;   // a plain load or store fell outside its buffer (debug build)

namespace dbg {

// Reader of one translation unit's bounds word; register_reader() is called
// once per unit at load time, read_all() ORs the words of all units.
using Reader = unsigned (*)(bool clear);
bool register_reader(Reader r);
unsigned read_all(bool clear);

#ifdef AXR_DEBUG
struct Span {
    uintptr_t base = 0;
    uint64_t bytes = 0;
};

// host: the span of `bytes` bytes at `base`, less the slack a test has set
Span span(const void *base, uint64_t bytes);
void set_slack(int64_t bytes);
#endif

// the bounds word and its checks exist in CUDA translation units only
#if defined(AXR_DEBUG) && defined(__CUDACC__)
namespace {
__device__ unsigned g_bounds;

[[maybe_unused]] unsigned read_bounds(bool clear)
{
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_bounds, sizeof(v)) != cudaSuccess) return ~0u;
    if (clear && v) {
        const unsigned z = 0;
        if (cudaMemcpyToSymbol(g_bounds, &z, sizeof(z)) != cudaSuccess) return ~0u;
    }
    return v;
}

[[maybe_unused]] const bool g_registered = register_reader(&read_bounds);
}  // namespace

// true when the n bytes at p lie inside s; otherwise records kErrBounds
__device__ __forceinline__ bool admit(const Span &s, const void *p, uint64_t n)
{
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    if (a >= s.base && a - s.base <= s.bytes && n <= s.bytes - (a - s.base)) return true;
    atomicOr(&g_bounds, kErrBounds);
    return false;
}
#endif

}  // namespace dbg
}  // namespace axr

#ifdef AXR_DEBUG
#define AXR_IN(span, ptr, nbytes) (::axr::dbg::admit((span), (ptr), (nbytes)))
#define AXR_DEBUG_ONLY(...) __VA_ARGS__
#else
#define AXR_IN(span, ptr, nbytes) true
#define AXR_DEBUG_ONLY(...)
#endif
