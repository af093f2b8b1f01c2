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

__device__ unsigned int g_attn_err;

}  // namespace attn
