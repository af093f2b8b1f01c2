// device_error.cuh -- the per-device error word the kernels report into.
//
// Kernels never trap.  A pipeline wait that runs out of time, or an input the
// host could not check (a seqlens value in device memory), sets a bit here;
// the host reads and clears it with attn_device_error().
#pragma once

namespace attn {

constexpr unsigned int kDevErrTimeout = 0x1u;   // ATTN_DEVERR_TIMEOUT
constexpr unsigned int kDevErrSeqlen = 0x2u;    // ATTN_DEVERR_SEQLEN
constexpr unsigned int kDevErrPage = 0x4u;      // ATTN_DEVERR_PAGE
constexpr unsigned int kDevErrSched = 0x8u;     // ATTN_DEVERR_SCHED
constexpr unsigned int kDevErrBounds = 0x10u;   // ATTN_DEVERR_BOUNDS (builds with ATTN_DEBUG_BOUNDS)

__device__ unsigned int g_attn_err;

// Debug builds (-DATTN_DEBUG_BOUNDS=1) check, at the points where the kernels
// turn work-unit numbers, ring positions and tile indices into addresses, that
// the result lies inside the tensor it addresses, and record a violation in the
// error word (they never trap).  Ordinary builds compile the checks away.
#ifndef ATTN_DEBUG_BOUNDS
#define ATTN_DEBUG_BOUNDS 0
#endif
#if ATTN_DEBUG_BOUNDS
#define ATTN_CHECK(cond)                                         \
    do {                                                         \
        if (!(cond)) atomicOr(&::attn::g_attn_err, ::attn::kDevErrBounds); \
    } while (0)
#else
#define ATTN_CHECK(cond) \
    do {                 \
    } while (0)
#endif

}  // namespace attn
