// kvq_debug.cuh -- device bounds checks of the debug build.
//
// Built with -DKVQ_DEBUG (libkvq_debug.so), every kernel checks the global
// addresses it computes against the extents of the buffers they fall in: the
// rows of a view's head, the ring of its window, the caller's q / out /
// workspace arrays, the card image.  A failed check sets its kernel family's
// bit in one device word (kvq_debug_flags reads it back) and the access is
// skipped, so a bad index never becomes an out-of-bounds access and nothing
// traps.  In the normal build dcheck() is the constant true and the checks
// compile away.
#pragma once

#include <cstdint>

namespace kvq {

enum DebugBit : uint32_t {
    kDbgAttnPacked = 1u << 0,     // a packed-row copy outside its head's rows
    kDbgAttnWindow = 1u << 1,     // a window copy outside its head's ring
    kDbgAttnStage = 1u << 2,      // a shared-memory stage outside the warp's ring
    kDbgAttnIo = 1u << 3,         // q, out or scores outside their arrays
    kDbgAttnWorkspace = 1u << 4,  // partials or arrival counters outside the workspace
    kDbgCodec = 1u << 5,          // quantize / dequantize rows outside the tensors
    kDbgAppend = 1u << 6,         // append rows or ring slots outside the view
    kDbgCard = 1u << 7,           // card pieces outside the card or the views
    kDbgScore = 1u << 8,          // score kernel rows or scores outside their arrays
    kDbgSelect = 1u << 9,         // selections or scores outside their arrays
    kDbgSens = 1u << 10,          // sensitivity window rows outside the ring
};

#ifdef KVQ_DEBUG
__device__ uint32_t g_debug_flags;

__device__ __forceinline__ bool dcheck(bool ok, uint32_t bit) {
    if (!ok) atomicOr(&g_debug_flags, bit);
    return ok;
}
#else
__device__ __forceinline__ bool dcheck(bool, uint32_t) { return true; }
#endif

// [p, p + n) within [base, base + extent) (bytes)
__device__ __forceinline__ bool within(const void *p, int64_t n, const void *base, int64_t extent) {
    const char *a = static_cast<const char *>(p), *b = static_cast<const char *>(base);
    return n >= 0 && a >= b && a + n <= b + extent;
}

}  // namespace kvq
