// decode_kv8_sm100.cuh -- split-KV decode against an 8-bit KV cache.
//
// Same computation, grid, splits and partial format as attn_decode_split_kernel
// (decode_sm100.cuh), and the same combine kernel; only the cache element
// changes.  Decode is bound by reading the cache (NVIDIA attention page,
// "Prefill and decode are two different tasks"), so a cache of one byte per
// element halves the bytes each token costs.  Two element formats:
//
//   E4M3  OCP FP8 E4M3 codes (sign, 4 exponent bits with bias 7, 3 mantissa
//         bits; subnormals; no infinities; S.1111.111 is NaN), one fp32 scale
//         per KV head for K and one for V: element = scale[g] * code value.
//   Q8_0  int8 codes and one fp16 scale per 32 consecutive values of a cache
//         row (the q8_0 cache type of the llama.cpp page), stored as a plane
//         of codes [B, Hkv, Lmax, D] and a plane of scales [B, Hkv, Lmax, D/32]
//         so TMA can stage both: element = scale[row][d / 32] * code.
//
// The MMAs run in f16 (m16n8k16, fp32 accumulation).  Every E4M3 value and
// every int8 value is an f16 value, so the codes enter the tensor cores
// exactly; Q is rescaled per row by a power of two into f16 range (exact) and
// the factor is folded into that row's score scale.  The scales are applied
// where they factor out of the sums:
//   E4M3  S = s_k[g] (Q . codes_K): folded into the score scale; O gets s_v[g]
//         once, at the end.
//   Q8_0  S = sum over 32-column blocks c of s_k[key][c] (Q_c . codes_K,c):
//         one MMA accumulator per block, scaled in fp32 and summed; P V =
//         sum over keys of (P s_v[key][c]) codes_V: P is scaled per block c of
//         output columns before it is rounded to f16.
// P is rounded to f16 (11 significant bits), a finer grid than the bf16 P of
// the other kernels.
//
// Two kernels: attn_decode_kv8t_kernel (below) for up to 16 query rows per KV
// head, with the cache rows as the MMA's M dimension, and
// attn_decode_kv8_kernel for 17 to 64 rows, with the query rows as M.
//
// Shared-memory reads without bank conflicts (row-major kernel; the
// transposed one is described with it).  A cache tile is 64 rows x D bytes,
// TMA-swizzled (128-byte swizzle for D = 128, 64-byte for D = 64).
//  - K (the B operand of S = Q K^T): the MMA sums over d, so any d order used
//    by both Q and K is valid.  Lane (grp, tq) takes the 4 contiguous bytes
//    d = 16 kk + 4 tq .. + 3 of key grp as its k slots {2tq, 2tq+1, 2tq+8,
//    2tq+9}; Q's A fragments are built in the same order.  One 32-bit load.
//  - V (the B operand of O += P V): the k slots are keys, so a lane needs one
//    byte from each of 4 rows.  It loads the 4 contiguous bytes d = 32 c +
//    4 grp .. + 3 of each of its 4 keys and byte-permutes them into the key
//    pairs of 4 n-tiles: n-tile 4 c + i, column n holds d = 32 c + 4 n + i.
//    The output columns are put back in d order when O is written.
#pragma once

#include "decode_sm100.cuh"
#include "device_error.cuh"
#include "ptx_sm100.cuh"

namespace attn {

constexpr int kKvFmtE4M3 = 1;
constexpr int kKvFmtQ8_0 = 2;

template <int D, int FMT>
struct DecodeKv8Smem {
    static constexpr int kBlk = D / 32;
    static constexpr int kTileBytes = kDecKT * D;                       // 64 rows of codes
    static constexpr int kScaleBytes = (FMT == kKvFmtQ8_0) ? kDecKT * (D / 32) * 2 : 0;
    static constexpr int kVOff = kTileBytes;
    static constexpr int kKsOff = 2 * kTileBytes;
    static constexpr int kVsOff = kKsOff + kScaleBytes;
    static constexpr int kStageBytes = ((2 * kTileBytes + 2 * kScaleBytes) + 1023) & ~1023;
    static constexpr int kStageTx = 2 * kTileBytes + 2 * kScaleBytes;
    static constexpr int kStages = (D == 128) ? 6 : 10;
    static constexpr int kRingBytes = kStages * kStageBytes;
    // end-of-CTA merge area (reuses the ring): m[4][16], l[4][16], O[4][16][D]
    static constexpr int kMergeBytes = 4 * 16 * 4 * 2 + 4 * 16 * D * 4;
    static_assert(kMergeBytes <= kRingBytes, "merge area must fit in the ring");
    static constexpr int kBarOff = kRingBytes;
    static constexpr int kBytes = kBarOff + 2 * kStages * 8 + 16;
    static constexpr int kAlloc = kBytes + 1024;
};

// byte offset of (row, byte col) in a TMA-swizzled tile of rows of D bytes
template <int D>
__device__ __forceinline__ uint32_t kv8_swz(int row, int col) {
    if constexpr (D == 128)
        return static_cast<uint32_t>(row * 128 + ((((col >> 4) ^ row) & 7) << 4) + (col & 15));
    else
        return static_cast<uint32_t>(row * 64 + ((((col >> 4) ^ (row >> 1)) & 3) << 4) + (col & 15));
}

// A 32-bit word of codes as the converters below take it: E4M3 codes as they
// are, int8 codes in offset form (sign bits flipped once per word, not per pair).
template <int FMT>
__device__ __forceinline__ uint32_t kv8_word(uint32_t raw) {
    return FMT == kKvFmtE4M3 ? raw : raw ^ 0x80808080u;
}

// two codes (bytes 0 and 1 of a kv8_word) -> f16x2
template <int FMT>
__device__ __forceinline__ uint32_t kv8_pair(uint32_t x) {
    if constexpr (FMT == kKvFmtE4M3)
        return e4m3x2_to_f16x2(x);
    else
        return offset_u8x2_to_f16x2(x);
}

// TMA producer of both kernels (one thread): the 64-row tiles of cache rows
// k_begin .. of (b, g) into the ring, codes and (q8_0) scales.  Contiguous
// cache: tile of rows r .. r+63 is box (0, r, b * Hkv + g).  Paged cache: row r
// lives in page block_table[b][r / page_size] at row r % page_size (page_size
// a multiple of 64, so a tile never straddles pages): box (0, r % page_size,
// page * Hkv + g).  A page outside the pool is flagged and replaced by page 0.
template <typename L, int FMT>
__device__ __forceinline__ void kv8_produce(const CUtensorMap* tm_k, const CUtensorMap* tm_v, const CUtensorMap* tm_ks,
                                            const CUtensorMap* tm_vs, const DecodeParams& p, int b, int g,
                                            int k_begin, int n_tiles, uint32_t ring, uint32_t bar0,
                                            volatile int* abort_flag) {
    constexpr int kBlk = L::kBlk;
    auto bar_full = [&](int s) { return bar0 + 8u * s; };
    auto bar_empty = [&](int s) { return bar0 + 8u * (L::kStages + s); };
    tma_prefetch_desc(tm_k);
    tma_prefetch_desc(tm_v);
    if constexpr (FMT == kKvFmtQ8_0) {
        tma_prefetch_desc(tm_ks);
        tma_prefetch_desc(tm_vs);
    }
    int issued = 0;
    for (int t = 0; t < n_tiles; ++t) {
        const int s = t % L::kStages;
        const uint32_t round = static_cast<uint32_t>(t / L::kStages);
        const int key0 = k_begin + t * kDecKT;
        int row = key0, outer = b * p.Hkv + g;
        if (p.block_table != nullptr) {
            int page = __ldg(p.block_table + static_cast<size_t>(b) * p.max_pages + key0 / p.page_size);
            if (page < 0 || page >= p.n_pages) {   // the tile would read another tenant's rows
                atomicOr(&g_attn_err, kDevErrPage);
                page = 0;
            }
            row = key0 % p.page_size;
            outer = page * p.Hkv + g;
        }
        decode_check_tile(p, row, outer);
        if (!mbar_wait(bar_empty(s), (round & 1u) ^ 1u, abort_flag, &g_attn_err, kDevErrTimeout)) break;
        mbar_arrive_expect_tx(bar_full(s), L::kStageTx);
        const uint32_t dst = ring + s * L::kStageBytes;
        tma_load_3d(dst, tm_k, bar_full(s), 0, row, outer);
        tma_load_3d(dst + L::kVOff, tm_v, bar_full(s), 0, row, outer);
        if constexpr (FMT == kKvFmtQ8_0) {
            tma_load_2d(dst + L::kKsOff, tm_ks, bar_full(s), row * kBlk, outer);
            tma_load_2d(dst + L::kVsOff, tm_vs, bar_full(s), row * kBlk, outer);
        }
        issued = t + 1;
    }
    if (issued < n_tiles) {
        // unwinding after a timeout: let issued copies land first
        for (int t = max(0, issued - L::kStages); t < issued; ++t) {
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(bar_full(t % L::kStages), static_cast<uint32_t>(t / L::kStages) & 1u) &&
                   global_timer_ns() - t0 < 100000000ull) {
            }
        }
    }
}

// KPW = cache rows of each 64-row tile handled by one compute warp (16, 32 or 64).
template <int D, int KPW, int FMT>
__global__ void __maxnreg__(200)
    attn_decode_kv8_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                           const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_vs,
                           const DecodeParams p) {
    grid_dep_release();   // the combine launch may be scheduled now
    using L = DecodeKv8Smem<D, FMT>;
    constexpr int kNT = KPW / 8;          // 8-key n-tiles of S per warp
    constexpr int kWPM = kDecKT / KPW;    // warps per 16-row block
    constexpr int kBlk = D / 32;          // 32-column blocks (q8_0 scale blocks)
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_base);

    const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int seqlen = decode_seqlen(p, b);
    const int k_begin = split * p.chunk;
    if (k_begin >= seqlen) return;   // uniform: this split has no rows
    const int k_end = min(k_begin + p.chunk, seqlen);
    const int n_tiles = (k_end - k_begin + kDecKT - 1) / kDecKT;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t ring = base;
    const uint32_t bar0 = base + L::kBarOff;
    auto bar_full = [&](int s) { return bar0 + 8u * s; };
    auto bar_empty = [&](int s) { return bar0 + 8u * (L::kStages + s); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kBarOff + 2 * L::kStages * 8);

    if (threadIdx.x == 0) {
        for (int s = 0; s < L::kStages; ++s) {
            mbar_init(bar_full(s), 1);
            mbar_init(bar_empty(s), 4);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == 4) {
        // ================= TMA producer =================
        if (lane == 0) kv8_produce<L, FMT>(&tm_k, &tm_v, &tm_ks, &tm_vs, p, b, g, k_begin, n_tiles, ring, bar0, abort_flag);
        __syncwarp();
        return;   // the producer takes no part in the merge below
    }

    // ================= compute warps =================
    const int mt = warp / kWPM;           // 16-row block of query heads
    const int ws = warp % kWPM;           // which slice of each tile's keys
    const int key_off = ws * KPW;
    const int grp = lane >> 2, tq = lane & 3;
    const int R = p.G * p.Lq;             // query rows of the group
    const int row_a = mt * 16 + grp, row_b = row_a + 8;
    const size_t group_row0 = (static_cast<size_t>(b) * p.Hq + static_cast<size_t>(g) * p.G) * p.Lq;
    const int lim_a = min(k_end, seqlen - p.Lq + row_a % p.Lq + 1);
    const int lim_b = min(k_end, seqlen - p.Lq + row_b % p.Lq + 1);
    const int lim_lo = min(k_end, seqlen - p.Lq + 1);

    // ---- Q as f16 A fragments, d order 16 kk + 4 tq + {0,1 | 2,3}, each row
    // scaled by 2^-e so its largest |q| lies in [2^14, 2^15) ----
    uint32_t qa[D / 16][4];
    float sl2_a, sl2_b;
    {
        const uint2* qrow_a = reinterpret_cast<const uint2*>(p.q + (group_row0 + row_a) * D);
        const uint2* qrow_b = reinterpret_cast<const uint2*>(p.q + (group_row0 + row_b) * D);
        const bool va = row_a < R, vb = row_b < R;
        uint2 wa[D / 16], wb[D / 16];
        float mxa = 0.0f, mxb = 0.0f;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            wa[kk] = va ? __ldg(qrow_a + (kk * 16 + 4 * tq) / 4) : make_uint2(0u, 0u);
            wb[kk] = vb ? __ldg(qrow_b + (kk * 16 + 4 * tq) / 4) : make_uint2(0u, 0u);
            const uint32_t ua[4] = {wa[kk].x << 16, wa[kk].x & 0xffff0000u, wa[kk].y << 16, wa[kk].y & 0xffff0000u};
            const uint32_t ub[4] = {wb[kk].x << 16, wb[kk].x & 0xffff0000u, wb[kk].y << 16, wb[kk].y & 0xffff0000u};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                mxa = fmaxf(mxa, fabsf(__uint_as_float(ua[i])));
                mxb = fmaxf(mxb, fabsf(__uint_as_float(ub[i])));
            }
        }
        mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 1));
        mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 2));
        mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 1));
        mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 2));
        // e = exponent of the row max - 14, kept in [-100, 100]; 2^-e and 2^e are exact
        auto row_exp = [](float mx) {
            if (!(mx > 0.0f) || !(mx < INFINITY)) return 0;
            const int ex = static_cast<int>((__float_as_uint(mx) >> 23) & 0xff) - 127;
            return max(-100, min(100, ex - 14));
        };
        const int ea = row_exp(mxa), eb = row_exp(mxb);
        const float fa = __uint_as_float(static_cast<uint32_t>(127 - ea) << 23);
        const float fb = __uint_as_float(static_cast<uint32_t>(127 - eb) << 23);
        const float ks = (FMT == kKvFmtE4M3) ? p.k_scale[g] : 1.0f;
        sl2_a = p.scale_log2 * ks * __uint_as_float(static_cast<uint32_t>(127 + ea) << 23);
        sl2_b = p.scale_log2 * ks * __uint_as_float(static_cast<uint32_t>(127 + eb) << 23);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            qa[kk][0] = pack_f16x2(__uint_as_float(wa[kk].x << 16) * fa, __uint_as_float(wa[kk].x & 0xffff0000u) * fa);
            qa[kk][1] = pack_f16x2(__uint_as_float(wb[kk].x << 16) * fb, __uint_as_float(wb[kk].x & 0xffff0000u) * fb);
            qa[kk][2] = pack_f16x2(__uint_as_float(wa[kk].y << 16) * fa, __uint_as_float(wa[kk].y & 0xffff0000u) * fa);
            qa[kk][3] = pack_f16x2(__uint_as_float(wb[kk].y << 16) * fb, __uint_as_float(wb[kk].y & 0xffff0000u) * fb);
        }
    }

    float oacc[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.0f;
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.0f, l_b = 0.0f;
    bool ok = true;

    for (int t = 0; t < n_tiles; ++t) {
        const int s = t % L::kStages;
        ok = mbar_wait(bar_full(s), static_cast<uint32_t>(t / L::kStages) & 1u, abort_flag, &g_attn_err, kDevErrTimeout);
        if (!ok) break;
        const uint32_t kbase = ring + s * L::kStageBytes;
        const uint32_t vbase = kbase + L::kVOff;
        const __half* ks_tile = reinterpret_cast<const __half*>(smem + s * L::kStageBytes + L::kKsOff);
        const __half* vs_tile = reinterpret_cast<const __half*>(smem + s * L::kStageBytes + L::kVsOff);
        const int tile_key0 = k_begin + t * kDecKT + key_off;   // absolute row of this warp's first key
        const bool tail = (k_begin + (t + 1) * kDecKT > k_end);
        const bool masked = (k_begin + (t + 1) * kDecKT > lim_lo);

        // ---- S = Q K^T over this warp's KPW keys ----
        float sacc[kNT][4];
#pragma unroll
        for (int i = 0; i < kNT; ++i) sacc[i][0] = sacc[i][1] = sacc[i][2] = sacc[i][3] = 0.0f;
#pragma unroll
        for (int c = 0; c < kBlk; ++c) {
            float bacc[kNT][4];   // this 32-column block's part (Q8_0 scales it per key)
#pragma unroll
            for (int i = 0; i < kNT; ++i) bacc[i][0] = bacc[i][1] = bacc[i][2] = bacc[i][3] = 0.0f;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int kk = 2 * c + h;
#pragma unroll
                for (int nt = 0; nt < kNT; ++nt) {
                    const int key_local = key_off + nt * 8 + grp;
                    const uint32_t w = kv8_word<FMT>(ld_shared_u32(kbase + kv8_swz<D>(key_local, kk * 16 + 4 * tq)));
                    mma_f16_16816(FMT == kKvFmtQ8_0 ? bacc[nt] : sacc[nt], qa[kk], kv8_pair<FMT>(w),
                                  kv8_pair<FMT>(w >> 16));
                }
            }
            if constexpr (FMT == kKvFmtQ8_0) {
#pragma unroll
                for (int nt = 0; nt < kNT; ++nt) {
                    const int k0 = key_off + nt * 8 + 2 * tq;   // keys of columns 2 tq, 2 tq + 1
                    const float s0 = __half2float(ks_tile[k0 * kBlk + c]);
                    const float s1 = __half2float(ks_tile[(k0 + 1) * kBlk + c]);
                    sacc[nt][0] = fmaf(bacc[nt][0], s0, sacc[nt][0]);
                    sacc[nt][1] = fmaf(bacc[nt][1], s1, sacc[nt][1]);
                    sacc[nt][2] = fmaf(bacc[nt][2], s0, sacc[nt][2]);
                    sacc[nt][3] = fmaf(bacc[nt][3], s1, sacc[nt][3]);
                }
            }
        }
        // ---- mask keys a row may not see (also every row past the valid length) ----
        if (masked) {
#pragma unroll
            for (int nt = 0; nt < kNT; ++nt) {
                const int key = tile_key0 + nt * 8 + 2 * tq;
                if (key >= lim_a) sacc[nt][0] = -INFINITY;
                if (key + 1 >= lim_a) sacc[nt][1] = -INFINITY;
                if (key >= lim_b) sacc[nt][2] = -INFINITY;
                if (key + 1 >= lim_b) sacc[nt][3] = -INFINITY;
            }
        }
        // ---- online softmax (log2 domain), rows a and b ----
        float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) {
            mx_a = fmaxf(mx_a, fmaxf(sacc[nt][0], sacc[nt][1]));
            mx_b = fmaxf(mx_b, fmaxf(sacc[nt][2], sacc[nt][3]));
        }
        mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
        mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
        mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
        mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
        const float mn_a = fmaxf(m_a, mx_a * sl2_a), mn_b = fmaxf(m_b, mx_b * sl2_b);
        const float f_a = (m_a == -INFINITY) ? 0.0f : ex2_approx(m_a - mn_a);
        const float f_b = (m_b == -INFINITY) ? 0.0f : ex2_approx(m_b - mn_b);
        const float ms_a = (mn_a == -INFINITY) ? 0.0f : mn_a;
        const float ms_b = (mn_b == -INFINITY) ? 0.0f : mn_b;
        m_a = mn_a;
        m_b = mn_b;
        float ps_a = 0.0f, ps_b = 0.0f;
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) {
            sacc[nt][0] = ex2_approx(fmaf(sacc[nt][0], sl2_a, -ms_a));
            sacc[nt][1] = ex2_approx(fmaf(sacc[nt][1], sl2_a, -ms_a));
            sacc[nt][2] = ex2_approx(fmaf(sacc[nt][2], sl2_b, -ms_b));
            sacc[nt][3] = ex2_approx(fmaf(sacc[nt][3], sl2_b, -ms_b));
            ps_a += sacc[nt][0] + sacc[nt][1];
            ps_b += sacc[nt][2] + sacc[nt][3];
        }
        l_a = l_a * f_a + ps_a;
        l_b = l_b * f_b + ps_b;
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
            oacc[i][0] *= f_a;
            oacc[i][1] *= f_a;
            oacc[i][2] *= f_b;
            oacc[i][3] *= f_b;
        }
        // ---- O += P V ----
#pragma unroll
        for (int k2 = 0; k2 < KPW / 16; ++k2) {
            // this lane's keys (tile rows): klo, klo + 1 (k slots 2 tq, 2 tq + 1), klo + 8, klo + 9
            const int klo = key_off + k2 * 16 + 2 * tq;
            const int kabs = tile_key0 - key_off + klo;   // absolute row of klo
            // rows past the valid length may hold anything (NaN codes included): use code 0
            const bool v0 = !tail || kabs < k_end, v1 = !tail || kabs + 1 < k_end;
            const bool v8 = !tail || kabs + 8 < k_end, v9 = !tail || kabs + 9 < k_end;
            float pa0 = sacc[2 * k2][0], pa1 = sacc[2 * k2][1], pb0 = sacc[2 * k2][2], pb1 = sacc[2 * k2][3];
            float pa8 = sacc[2 * k2 + 1][0], pa9 = sacc[2 * k2 + 1][1], pb8 = sacc[2 * k2 + 1][2],
                  pb9 = sacc[2 * k2 + 1][3];
            uint32_t a[4];
            if constexpr (FMT == kKvFmtE4M3) {
                a[0] = pack_f16x2(pa0, pa1);
                a[1] = pack_f16x2(pb0, pb1);
                a[2] = pack_f16x2(pa8, pa9);
                a[3] = pack_f16x2(pb8, pb9);
            }
#pragma unroll
            for (int c = 0; c < kBlk; ++c) {
                if constexpr (FMT == kKvFmtQ8_0) {
                    // P scaled by each key's V scale for this 32-column block (0 past the valid length)
                    const float s0 = v0 ? __half2float(vs_tile[klo * kBlk + c]) : 0.0f;
                    const float s1 = v1 ? __half2float(vs_tile[(klo + 1) * kBlk + c]) : 0.0f;
                    const float s8 = v8 ? __half2float(vs_tile[(klo + 8) * kBlk + c]) : 0.0f;
                    const float s9 = v9 ? __half2float(vs_tile[(klo + 9) * kBlk + c]) : 0.0f;
                    a[0] = pack_f16x2(pa0 * s0, pa1 * s1);
                    a[1] = pack_f16x2(pb0 * s0, pb1 * s1);
                    a[2] = pack_f16x2(pa8 * s8, pa9 * s9);
                    a[3] = pack_f16x2(pb8 * s8, pb9 * s9);
                }
                const int col = c * 32 + 4 * grp;
                const uint32_t w0 = kv8_word<FMT>(v0 ? ld_shared_u32(vbase + kv8_swz<D>(klo, col)) : 0u);
                const uint32_t w1 = kv8_word<FMT>(v1 ? ld_shared_u32(vbase + kv8_swz<D>(klo + 1, col)) : 0u);
                const uint32_t w8 = kv8_word<FMT>(v8 ? ld_shared_u32(vbase + kv8_swz<D>(klo + 8, col)) : 0u);
                const uint32_t w9 = kv8_word<FMT>(v9 ? ld_shared_u32(vbase + kv8_swz<D>(klo + 9, col)) : 0u);
                // key pairs of byte i: {w0.i, w1.i} and {w8.i, w9.i}; two bytes per permute
                const uint32_t lo01 = prmt(w0, w1, 0x5140u), hi01 = prmt(w0, w1, 0x7362u);
                const uint32_t lo89 = prmt(w8, w9, 0x5140u), hi89 = prmt(w8, w9, 0x7362u);
                mma_f16_16816(oacc[4 * c + 0], a, kv8_pair<FMT>(lo01), kv8_pair<FMT>(lo89));
                mma_f16_16816(oacc[4 * c + 1], a, kv8_pair<FMT>(lo01 >> 16), kv8_pair<FMT>(lo89 >> 16));
                mma_f16_16816(oacc[4 * c + 2], a, kv8_pair<FMT>(hi01), kv8_pair<FMT>(hi89));
                mma_f16_16816(oacc[4 * c + 3], a, kv8_pair<FMT>(hi01 >> 16), kv8_pair<FMT>(hi89 >> 16));
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_empty(s));
    }

    // ---- merge the warps of each 16-row block through shared memory ----
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
    asm volatile("bar.sync 1, 128;" ::: "memory");   // every compute warp is done with the ring
    float* sm_m = reinterpret_cast<float*>(smem);
    float* sm_l = sm_m + 4 * 16;
    float* sm_o = sm_l + 4 * 16;
    if (tq == 0) {
        sm_m[warp * 16 + grp] = m_a;
        sm_m[warp * 16 + grp + 8] = m_b;
        sm_l[warp * 16 + grp] = l_a;
        sm_l[warp * 16 + grp + 8] = l_b;
    }
    // n-tile 4 c + i, columns 2 tq and 2 tq + 1, hold d = 32 c + 8 tq + i and 32 c + 8 tq + 4 + i
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
        const int d = (nt >> 2) * 32 + 8 * tq + (nt & 3);
        float* oa = sm_o + (warp * 16 + grp) * D;
        float* ob = sm_o + (warp * 16 + grp + 8) * D;
        oa[d] = oacc[nt][0];
        oa[d + 4] = oacc[nt][1];
        ob[d] = oacc[nt][2];
        ob[d + 4] = oacc[nt][3];
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (!ok) return;
    const float vscale = (FMT == kKvFmtE4M3) ? p.v_scale[g] : 1.0f;
    for (int idx = threadIdx.x; idx < R * D; idx += 128) {
        const int row = idx / D, d = idx % D;
        const int blk = row >> 4, rr = row & 15;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWPM; ++w) M = fmaxf(M, sm_m[(blk * kWPM + w) * 16 + rr]);
        float Lsum = 0.0f, acc = 0.0f;
#pragma unroll
        for (int w = 0; w < kWPM; ++w) {
            const int ww = blk * kWPM + w;
            const float mw = sm_m[ww * 16 + rr];
            const float sc = (mw == -INFINITY) ? 0.0f : ex2_approx(mw - M);
            Lsum += sm_l[ww * 16 + rr] * sc;
            acc += sm_o[(ww * 16 + rr) * D + d] * sc;
        }
        const size_t prow = (group_row0 + row) * p.n_splits + split;
        decode_check_prow(p, prow);
        p.o_part[prow * D + d] = (Lsum > 0.0f) ? acc * vscale / Lsum : 0.0f;
        if (d == 0) p.lse_part[prow] = (Lsum > 0.0f) ? M + __log2f(Lsum) : -INFINITY;
    }
}

// ---------------------------------------------------------------------------
// Up to 16 query rows per KV head (NR = 1 or 2 groups of 8): the transposed
// form.  With R <= 16 rows, an m16 MMA over query rows is mostly padding, so
// the cache rows take the M dimension instead:
//   S^T = K Q^T     M = 16 cache rows, N = 8 query rows, K = 16 columns of d
//   O^T = V^T P^T   M = 16 columns of d, N = 8 query rows, K = 16 cache rows
// Half the MMAs and half the accumulator registers of the row-major form, so
// more CTAs fit on an SM.  The S^T accumulator holds a cache row per lane
// group and query rows across the quad; P^T reaches the B-operand layout of
// the second MMA by one 8x8 transpose (movmatrix) per 8 cache rows.
//  - K (A operand of S^T): lane (grp, tq) loads the 4 bytes d = 16 kk + 4 tq
//    .. + 3 of cache rows grp and grp + 8 (Q's B fragments use the same d order).
//  - V^T (A operand of O^T): lane loads 4 bytes d = 32 c + 4 grp .. + 3 of cache
//    rows 2 tq, 2 tq + 1, 2 tq + 8, 2 tq + 9 and byte-permutes them into the key
//    pairs of two M tiles: M tile (c, h) row grp holds d = 32 c + 4 grp + 2 h,
//    row grp + 8 holds d + 1.
template <int D, int FMT>
struct DecodeKv8tSmem {
    static constexpr int kBlk = D / 32;
    static constexpr int kTileBytes = kDecKT * D;
    static constexpr int kScaleBytes = (FMT == kKvFmtQ8_0) ? kDecKT * (D / 32) * 2 : 0;
    static constexpr int kVOff = kTileBytes;
    static constexpr int kKsOff = 2 * kTileBytes;
    static constexpr int kVsOff = kKsOff + kScaleBytes;
    static constexpr int kStageBytes = ((2 * kTileBytes + 2 * kScaleBytes) + 1023) & ~1023;
    static constexpr int kStageTx = 2 * kTileBytes + 2 * kScaleBytes;
    // 3 (D = 128) or 5 (D = 64) stages: four CTAs fit in an SM's shared memory,
    // with 192 KB of cache rows in flight per SM
    static constexpr int kStages = (D == 128) ? 3 : 5;
    static constexpr int kRingBytes = kStages * kStageBytes;
    // merge area (reuses the ring): m[4][16], l[4][16], O[4][16][D]
    static constexpr int kMergeBytes = 4 * 16 * 4 * 2 + 4 * 16 * D * 4;
    static_assert(kMergeBytes <= kRingBytes, "merge area must fit in the ring");
    static constexpr int kBarOff = kRingBytes;
    static constexpr int kBytes = kBarOff + 2 * kStages * 8 + 16;
    static constexpr int kAlloc = kBytes + 1024;
};

// CTAs per SM the register budget is sized for (one query-row group: 4; two: 2)
template <int NR>
constexpr int kv8t_min_blocks() { return NR == 1 ? 4 : 2; }

template <int D, int NR, int FMT>
__global__ void __launch_bounds__(kDecThreads, kv8t_min_blocks<NR>())
    attn_decode_kv8t_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                            const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_vs,
                            const DecodeParams p) {
    grid_dep_release();   // the combine launch may be scheduled now
    using L = DecodeKv8tSmem<D, FMT>;
    constexpr int kBlk = D / 32;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_base);

    const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int seqlen = decode_seqlen(p, b);
    const int k_begin = split * p.chunk;
    if (k_begin >= seqlen) return;   // uniform: this split has no rows
    const int k_end = min(k_begin + p.chunk, seqlen);
    const int n_tiles = (k_end - k_begin + kDecKT - 1) / kDecKT;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t ring = base;
    const uint32_t bar0 = base + L::kBarOff;
    auto bar_full = [&](int s) { return bar0 + 8u * s; };
    auto bar_empty = [&](int s) { return bar0 + 8u * (L::kStages + s); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kBarOff + 2 * L::kStages * 8);

    if (threadIdx.x == 0) {
        for (int s = 0; s < L::kStages; ++s) {
            mbar_init(bar_full(s), 1);
            mbar_init(bar_empty(s), 4);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == 4) {
        // ================= TMA producer =================
        if (lane == 0) kv8_produce<L, FMT>(&tm_k, &tm_v, &tm_ks, &tm_vs, p, b, g, k_begin, n_tiles, ring, bar0, abort_flag);
        __syncwarp();
        return;
    }

    // ================= compute warps: warp w owns cache rows 16 w .. 16 w + 15 of each tile =================
    const int grp = lane >> 2, tq = lane & 3;
    const int key_off = warp * 16;
    const int R = p.G * p.Lq;
    const size_t group_row0 = (static_cast<size_t>(b) * p.Hq + static_cast<size_t>(g) * p.G) * p.Lq;
    const int lim_lo = min(k_end, seqlen - p.Lq + 1);

    // ---- Q^T as B fragments: n-tile j, column grp = query row 8 j + grp; rows
    // scaled by 2^-e into f16 range (e per row, folded into that row's score scale) ----
    uint32_t qb[D / 16][NR][2];
    float sl2[NR][2];   // score scale of the rows this lane's accumulators hold: 8 j + 2 tq (+1)
    int lim[NR][2];
    {
        const float ks = (FMT == kKvFmtE4M3) ? p.k_scale[g] : 1.0f;
#pragma unroll
        for (int j = 0; j < NR; ++j) {
            const int r = 8 * j + grp;
            const bool valid = r < R;
            const uint2* qrow = reinterpret_cast<const uint2*>(p.q + (group_row0 + (valid ? r : 0)) * D);
            uint2 w[D / 16];
            float mx = 0.0f;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                w[kk] = valid ? __ldg(qrow + 4 * kk + tq) : make_uint2(0u, 0u);
                mx = fmaxf(mx, fmaxf(fmaxf(fabsf(__uint_as_float(w[kk].x << 16)),
                                           fabsf(__uint_as_float(w[kk].x & 0xffff0000u))),
                                     fmaxf(fabsf(__uint_as_float(w[kk].y << 16)),
                                           fabsf(__uint_as_float(w[kk].y & 0xffff0000u)))));
            }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            int e = 0;
            if (mx > 0.0f && mx < INFINITY) e = max(-100, min(100, static_cast<int>((__float_as_uint(mx) >> 23) & 0xff) - 141));
            const float f = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                qb[kk][j][0] = pack_f16x2(__uint_as_float(w[kk].x << 16) * f, __uint_as_float(w[kk].x & 0xffff0000u) * f);
                qb[kk][j][1] = pack_f16x2(__uint_as_float(w[kk].y << 16) * f, __uint_as_float(w[kk].y & 0xffff0000u) * f);
            }
            // the exponents of rows 8 j + 2 tq and 8 j + 2 tq + 1 live in lanes 8 tq and 8 tq + 4
            const int e0 = __shfl_sync(0xffffffffu, e, 8 * tq);
            const int e1 = __shfl_sync(0xffffffffu, e, 8 * tq + 4);
            sl2[j][0] = p.scale_log2 * ks * __uint_as_float(static_cast<uint32_t>(127 + e0) << 23);
            sl2[j][1] = p.scale_log2 * ks * __uint_as_float(static_cast<uint32_t>(127 + e1) << 23);
            const int r0 = 8 * j + 2 * tq;
            lim[j][0] = min(k_end, seqlen - p.Lq + r0 % p.Lq + 1);
            lim[j][1] = min(k_end, seqlen - p.Lq + (r0 + 1) % p.Lq + 1);
        }
    }

    float oacc[D / 16][NR][4];
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
        for (int j = 0; j < NR; ++j) oacc[mt][j][0] = oacc[mt][j][1] = oacc[mt][j][2] = oacc[mt][j][3] = 0.0f;
    float m_run[NR][2], l_run[NR][2];
#pragma unroll
    for (int j = 0; j < NR; ++j) {
        m_run[j][0] = m_run[j][1] = -INFINITY;
        l_run[j][0] = l_run[j][1] = 0.0f;
    }
    bool ok = true;

    for (int t = 0; t < n_tiles; ++t) {
        const int s = t % L::kStages;
        ok = mbar_wait(bar_full(s), static_cast<uint32_t>(t / L::kStages) & 1u, abort_flag, &g_attn_err, kDevErrTimeout);
        if (!ok) break;
        const uint32_t kbase = ring + s * L::kStageBytes;
        const uint32_t vbase = kbase + L::kVOff;
        const __half* ks_tile = reinterpret_cast<const __half*>(smem + s * L::kStageBytes + L::kKsOff);
        const __half* vs_tile = reinterpret_cast<const __half*>(smem + s * L::kStageBytes + L::kVsOff);
        const int tile_key0 = k_begin + t * kDecKT + key_off;   // absolute row of this warp's cache row 0
        const bool tail = (k_begin + (t + 1) * kDecKT > k_end);
        const bool masked = (k_begin + (t + 1) * kDecKT > lim_lo);

        // ---- S^T = K Q^T: rows key_off + grp (c0, c1) and + 8 (c2, c3), columns 8 j + 2 tq (+1) ----
        float sacc[NR][4];
#pragma unroll
        for (int j = 0; j < NR; ++j) sacc[j][0] = sacc[j][1] = sacc[j][2] = sacc[j][3] = 0.0f;
#pragma unroll
        for (int c = 0; c < kBlk; ++c) {
            float bacc[NR][4];
#pragma unroll
            for (int j = 0; j < NR; ++j) bacc[j][0] = bacc[j][1] = bacc[j][2] = bacc[j][3] = 0.0f;
            // For h = 0, 1 the words of cache rows grp (w[2h]) and grp + 8 (w[2h + 1]) at
            // d = 16 (2 c + h) + 4 tq .. + 3.  E4M3: the block's codes in one ldmatrix
            // (lane l addresses row l % 8, + 8 for odd l / 8, of columns 32 c + 16 (l / 16)
            // .. + 15, and receives from each of the four 8 x 16-byte matrices the 4
            // bytes 4 tq .. + 3 of row grp); q8_0 with four 32-bit loads, which measured
            // about 5 % faster for it on B200 (the ldmatrix form about 2 % faster for E4M3).
            uint32_t w[4];
            if constexpr (FMT == kKvFmtE4M3) {
                ldmatrix_x4(kbase + kv8_swz<D>(key_off + (lane & 7) + ((lane >> 3) & 1) * 8, c * 32 + (lane >> 4) * 16),
                            w[0], w[1], w[2], w[3]);
            } else {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    w[2 * h] = ld_shared_u32(kbase + kv8_swz<D>(key_off + grp, (2 * c + h) * 16 + 4 * tq));
                    w[2 * h + 1] = ld_shared_u32(kbase + kv8_swz<D>(key_off + grp + 8, (2 * c + h) * 16 + 4 * tq));
                }
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int kk = 2 * c + h;
                const uint32_t wl = kv8_word<FMT>(w[2 * h]);
                const uint32_t wh = kv8_word<FMT>(w[2 * h + 1]);
                const uint32_t a[4] = {kv8_pair<FMT>(wl), kv8_pair<FMT>(wh), kv8_pair<FMT>(wl >> 16),
                                       kv8_pair<FMT>(wh >> 16)};
#pragma unroll
                for (int j = 0; j < NR; ++j)
                    mma_f16_16816(FMT == kKvFmtQ8_0 ? bacc[j] : sacc[j], a, qb[kk][j][0], qb[kk][j][1]);
            }
            if constexpr (FMT == kKvFmtQ8_0) {
                const float s_lo = __half2float(ks_tile[(key_off + grp) * kBlk + c]);
                const float s_hi = __half2float(ks_tile[(key_off + grp + 8) * kBlk + c]);
#pragma unroll
                for (int j = 0; j < NR; ++j) {
                    sacc[j][0] = fmaf(bacc[j][0], s_lo, sacc[j][0]);
                    sacc[j][1] = fmaf(bacc[j][1], s_lo, sacc[j][1]);
                    sacc[j][2] = fmaf(bacc[j][2], s_hi, sacc[j][2]);
                    sacc[j][3] = fmaf(bacc[j][3], s_hi, sacc[j][3]);
                }
            }
        }
        // ---- masking, online softmax per query row (a column of S^T) ----
        const int key_lo = tile_key0 + grp, key_hi = key_lo + 8;
#pragma unroll
        for (int j = 0; j < NR; ++j) {
            if (masked) {
                if (key_lo >= lim[j][0]) sacc[j][0] = -INFINITY;
                if (key_lo >= lim[j][1]) sacc[j][1] = -INFINITY;
                if (key_hi >= lim[j][0]) sacc[j][2] = -INFINITY;
                if (key_hi >= lim[j][1]) sacc[j][3] = -INFINITY;
            }
            float mx0 = fmaxf(sacc[j][0], sacc[j][2]), mx1 = fmaxf(sacc[j][1], sacc[j][3]);
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
            }
            const float mn0 = fmaxf(m_run[j][0], mx0 * sl2[j][0]), mn1 = fmaxf(m_run[j][1], mx1 * sl2[j][1]);
            const float f0 = (m_run[j][0] == -INFINITY) ? 0.0f : ex2_approx(m_run[j][0] - mn0);
            const float f1 = (m_run[j][1] == -INFINITY) ? 0.0f : ex2_approx(m_run[j][1] - mn1);
            const float ms0 = (mn0 == -INFINITY) ? 0.0f : mn0;
            const float ms1 = (mn1 == -INFINITY) ? 0.0f : mn1;
            m_run[j][0] = mn0;
            m_run[j][1] = mn1;
            sacc[j][0] = ex2_approx(fmaf(sacc[j][0], sl2[j][0], -ms0));
            sacc[j][1] = ex2_approx(fmaf(sacc[j][1], sl2[j][1], -ms1));
            sacc[j][2] = ex2_approx(fmaf(sacc[j][2], sl2[j][0], -ms0));
            sacc[j][3] = ex2_approx(fmaf(sacc[j][3], sl2[j][1], -ms1));
            l_run[j][0] = l_run[j][0] * f0 + (sacc[j][0] + sacc[j][2]);
            l_run[j][1] = l_run[j][1] * f1 + (sacc[j][1] + sacc[j][3]);
            if (__any_sync(0xffffffffu, f0 != 1.0f || f1 != 1.0f)) {
#pragma unroll
                for (int mt = 0; mt < D / 16; ++mt) {
                    oacc[mt][j][0] *= f0;
                    oacc[mt][j][1] *= f1;
                    oacc[mt][j][2] *= f0;
                    oacc[mt][j][3] *= f1;
                }
            }
        }
        // ---- O^T += V^T P^T ----
        // cache rows past the valid length may hold anything (NaN codes or scales included)
        const int vk = key_off + 2 * tq;           // this lane's V rows: vk, vk+1, vk+8, vk+9
        const int vabs = tile_key0 + 2 * tq;
        const bool v0 = !tail || vabs < k_end, v1 = !tail || vabs + 1 < k_end;
        const bool v8 = !tail || vabs + 8 < k_end, v9 = !tail || vabs + 9 < k_end;
        // P^T B fragments, transposed once per tile: after the transpose this lane
        // holds cache rows vk, vk + 1 (fragment 0) and vk + 8, vk + 9 (fragment 1),
        // the rows whose V codes it loads.  q8_0 scales P per row and column
        // block, so each block multiplies the fragments by those rows' V scales.
        uint32_t pt[NR][2];
#pragma unroll
        for (int j = 0; j < NR; ++j) {
            pt[j][0] = movmatrix_trans(pack_f16x2(sacc[j][0], sacc[j][1]));
            pt[j][1] = movmatrix_trans(pack_f16x2(sacc[j][2], sacc[j][3]));
        }
        // q8_0: the V scales of those rows, one word (two blocks) at a time; zero for
        // rows past the valid length (their scales may be NaN)
        const uint32_t* vsw = reinterpret_cast<const uint32_t*>(vs_tile);
        uint32_t w0s = 0u, w1s = 0u, w8s = 0u, w9s = 0u;
        uint32_t pb[NR][2];
#pragma unroll
        for (int c = 0; c < kBlk; ++c) {
            if constexpr (FMT == kKvFmtQ8_0) {
                if ((c & 1) == 0) {
                    constexpr int kW = kBlk / 2;   // scale words per row
                    w0s = v0 ? vsw[vk * kW + (c >> 1)] : 0u;
                    w1s = v1 ? vsw[(vk + 1) * kW + (c >> 1)] : 0u;
                    w8s = v8 ? vsw[(vk + 8) * kW + (c >> 1)] : 0u;
                    w9s = v9 ? vsw[(vk + 9) * kW + (c >> 1)] : 0u;
                }
                const uint32_t sel = (c & 1) ? 0x7632u : 0x5410u;
                const uint32_t s01 = prmt(w0s, w1s, sel), s89 = prmt(w8s, w9s, sel);
#pragma unroll
                for (int j = 0; j < NR; ++j) {
                    pb[j][0] = hmul2(pt[j][0], s01);
                    pb[j][1] = hmul2(pt[j][1], s89);
                }
            } else {
#pragma unroll
                for (int j = 0; j < NR; ++j) {
                    pb[j][0] = pt[j][0];
                    pb[j][1] = pt[j][1];
                }
            }
            const int col = c * 32 + 4 * grp;
            const uint32_t w0 = kv8_word<FMT>(v0 ? ld_shared_u32(vbase + kv8_swz<D>(vk, col)) : 0u);
            const uint32_t w1 = kv8_word<FMT>(v1 ? ld_shared_u32(vbase + kv8_swz<D>(vk + 1, col)) : 0u);
            const uint32_t w8 = kv8_word<FMT>(v8 ? ld_shared_u32(vbase + kv8_swz<D>(vk + 8, col)) : 0u);
            const uint32_t w9 = kv8_word<FMT>(v9 ? ld_shared_u32(vbase + kv8_swz<D>(vk + 9, col)) : 0u);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t sel = h ? 0x7362u : 0x5140u;
                const uint32_t p01 = prmt(w0, w1, sel), p89 = prmt(w8, w9, sel);
                const uint32_t a[4] = {kv8_pair<FMT>(p01), kv8_pair<FMT>(p01 >> 16), kv8_pair<FMT>(p89),
                                       kv8_pair<FMT>(p89 >> 16)};
#pragma unroll
                for (int j = 0; j < NR; ++j) mma_f16_16816(oacc[2 * c + h][j], a, pb[j][0], pb[j][1]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_empty(s));
    }

    // ---- merge the four warps' key slices through shared memory ----
#pragma unroll
    for (int j = 0; j < NR; ++j)
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) l_run[j][i] += __shfl_xor_sync(0xffffffffu, l_run[j][i], o);
    asm volatile("bar.sync 1, 128;" ::: "memory");   // every compute warp is done with the ring
    float* sm_m = reinterpret_cast<float*>(smem);
    float* sm_l = sm_m + 4 * 16;
    float* sm_o = sm_l + 4 * 16;
#pragma unroll
    for (int j = 0; j < NR; ++j) {
        const int r0 = 8 * j + 2 * tq;
        if (grp == 0) {
            sm_m[warp * 16 + r0] = m_run[j][0];
            sm_m[warp * 16 + r0 + 1] = m_run[j][1];
            sm_l[warp * 16 + r0] = l_run[j][0];
            sm_l[warp * 16 + r0 + 1] = l_run[j][1];
        }
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
            const int d = (mt >> 1) * 32 + 4 * grp + 2 * (mt & 1);   // row grp; row grp + 8 is d + 1
            float* o0 = sm_o + (warp * 16 + r0) * D;
            float* o1 = o0 + D;
            o0[d] = oacc[mt][j][0];
            o1[d] = oacc[mt][j][1];
            o0[d + 1] = oacc[mt][j][2];
            o1[d + 1] = oacc[mt][j][3];
        }
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (!ok) return;
    const float vscale = (FMT == kKvFmtE4M3) ? p.v_scale[g] : 1.0f;
    for (int idx = threadIdx.x; idx < R * D; idx += 128) {
        const int row = idx / D, d = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, sm_m[w * 16 + row]);
        float Lsum = 0.0f, acc = 0.0f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const float mw = sm_m[w * 16 + row];
            const float sc = (mw == -INFINITY) ? 0.0f : ex2_approx(mw - M);
            Lsum += sm_l[w * 16 + row] * sc;
            acc += sm_o[(w * 16 + row) * D + d] * sc;
        }
        const size_t prow = (group_row0 + row) * p.n_splits + split;
        decode_check_prow(p, prow);
        p.o_part[prow * D + d] = (Lsum > 0.0f) ? acc * vscale / Lsum : 0.0f;
        if (d == 0) p.lse_part[prow] = (Lsum > 0.0f) ? M + __log2f(Lsum) : -INFINITY;
    }
}

}  // namespace attn
