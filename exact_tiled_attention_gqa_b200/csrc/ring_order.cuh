// ring_order.cuh -- the order in which K and V tiles pass through a shared-
// memory ring, for kernels that issue their MMAs in one of two orders:
//
//   NQ = 2 (two Q tiles, one S buffer each):  K_0 V_0 K_1 V_1 ...
//   NQ = 1 (one Q tile, two S buffers):       K_0 K_1 V_0 K_2 V_1 K_3 V_2 ... V_{n-1}
//
// With two S buffers the MMA issuer runs S(0), S(1), then per tile j
// O += P(j) V_j and S(j+2), so K_{j+2} is needed right after V_j.  A producer
// that loads in this order never waits for an entry the consumer releases later.
#pragma once

namespace attn {

// position (in tiles) of K_j and V_j in the ring order, n_kt tiles in all
template <int NQ>
__device__ __forceinline__ int ring_pos_k(int j) { return NQ == 2 ? 2 * j : (j == 0 ? 0 : 2 * j - 1); }
template <int NQ>
__device__ __forceinline__ int ring_pos_v(int j, int n_kt) {
    return NQ == 2 ? 2 * j + 1 : (j + 1 < n_kt ? 2 * j + 2 : 2 * n_kt - 1);
}
// the inverse: which tile (K or V, index j) sits at position pos
template <int NQ>
__device__ __forceinline__ void ring_tile(int pos, int n_kt, bool& is_v, int& j) {
    if (NQ == 2) {
        is_v = pos & 1;
        j = pos >> 1;
    } else if (pos == 0) {
        is_v = false;
        j = 0;
    } else if (pos == 2 * n_kt - 1) {
        is_v = true;
        j = n_kt - 1;
    } else if (pos & 1) {
        is_v = false;
        j = (pos + 1) >> 1;
    } else {
        is_v = true;
        j = (pos - 2) >> 1;
    }
}

}  // namespace attn
