// decode_sm100.cuh -- split-KV GQA decode and its log-sum-exp combine.
//
// What it computes: for each sequence b and query head h, Lq new query rows
// (Lq = 1: plain decode; Lq > 1: the speculative-decoding verify step or a
// small chunk) against cache rows of KV head h / G.  The Lq new tokens are the
// last Lq of the sequence's seqlens[b] cached rows, so new token i sees rows
// 0 .. seqlens[b] - Lq + i (the bottom-right alignment of the is_causal
// section of the SDPA / FlashAttention selection guide; for Lq = 1 every
// cached row, as its "use_cache" section has it).  Decode is bound by reading the
// cache (NVIDIA attention page, "Prefill and decode are two different
// tasks"), so the kernel is built around streaming K and V once at full HBM
// bandwidth:
//
//   split kernel  grid (split, KV head, batch).  A CTA owns `chunk` cache rows
//                 of one (b, KV head): a producer warp streams 64-row K and V
//                 tiles into a ring of shared-memory stages with TMA (128-byte
//                 swizzle, so the ldmatrix reads below are conflict-free); four
//                 compute warps multiply the G x Lq query rows of the group (as
//                 the M rows of m16n8k16 tensor-core MMAs, padded to 16) with
//                 each tile once, run an online softmax, and accumulate P V.
//                 Warps sharing a 16-row block split the tile's keys and merge
//                 through shared memory at the end; the CTA writes one
//                 normalised partial output and its log2-sum-exp per row.
//   combine       one warp per query row: LSE-weighted sum of its partials.
//
// Splitting the cache length and merging by log-sum-exp is the single-GPU
// form of the KV parallelism on the NVIDIA page ("Parameter four").
//
// Two cache layouts share these kernels:
//   contiguous  K/V [B, Hkv, Lmax, D]; a tile of rows r .. r+63 of (b, g) is
//               TMA box (0/64, r, b * Hkv + g) of the [B*Hkv, Lmax, D] view.
//   paged       K/V pools [n_pages, Hkv, page_size, D] and a block table
//               [B, max_pages]: logical row r of sequence b lives in page
//               block_table[b][r / page_size] at row r % page_size.  page_size
//               is a multiple of 64, so a tile never straddles two pages; the
//               box is (0/64, r % page_size, page * Hkv + g) of the
//               [n_pages*Hkv, page_size, D] view.
#pragma once

#include "ptx_sm100.cuh"
#include "device_error.cuh"

namespace attn {

constexpr int kDecThreads = 160;   // warps 0-3 compute, warp 4 TMA producer
constexpr int kDecKT = 64;         // cache rows per tile

template <int D>
struct DecodeSmem {
    static constexpr int kKB = D / 64;
    static constexpr int kBlockBytes = kDecKT * 128;        // 64 rows x 128 bytes
    static constexpr int kTileBytes = kDecKT * D * 2;       // one K or V tile
    static constexpr int kStageBytes = 2 * kTileBytes;      // K then V
    static constexpr int kStages = (D == 128) ? 3 : 6;
    static constexpr int kRingBytes = kStages * kStageBytes;
    // end-of-CTA merge area (reuses the ring): m[4][16], l[4][16], l_exact[4][16], O[4][16][D]
    static constexpr int kMergeBytes = 4 * 16 * 4 * 3 + 4 * 16 * D * 4;
    static_assert(kMergeBytes <= kRingBytes, "merge area must fit in the ring");
    static constexpr int kBarOff = kRingBytes;
    static constexpr int kBytes = kBarOff + 2 * kStages * 8 + 16;
    static constexpr int kAlloc = kBytes + 1024;
};

struct DecodeParams {
    const __nv_bfloat16* q;   // [B,Hq,Lq,D]
    const int* seqlens;       // [B]
    float* o_part;            // [B,Hq,Lq,n_splits,D]
    float* lse_part;          // [B,Hq,Lq,n_splits] (log2 domain)
    int B, Hq, Hkv, Lmax, G;
    int Lq;                   // new query rows per sequence (1 = plain decode)
    const int* block_table;   // [B, max_pages] for the paged layout, nullptr for the contiguous one
    int page_size, max_pages, n_pages;
    int chunk;                // cache rows per split (multiple of 64)
    int n_splits;
    float scale_log2;
    const float* k_scale = nullptr;   // 8-bit E4M3 cache: per-KV-head scales [Hkv] (decode_kv8_sm100.cuh)
    const float* v_scale = nullptr;
};

__device__ __forceinline__ int decode_seqlen(const DecodeParams& p, int b) {
    int n = p.seqlens[b];
    if (n < 0 || n > p.Lmax) {
        atomicOr(&g_attn_err, kDevErrSeqlen);
        n = n < 0 ? 0 : p.Lmax;
    }
    return n;
}

// (debug builds) a tile starting at cache row `row` of slab `outer` lies in the
// view TMA reads: [B * Hkv, Lmax] rows, or [n_pages * Hkv, page_size] when paged
__device__ __forceinline__ void decode_check_tile(const DecodeParams& p, int row, int outer) {
    const int rows = p.block_table ? p.page_size : p.Lmax;
    const long long outers = p.block_table ? static_cast<long long>(p.n_pages) * p.Hkv
                                           : static_cast<long long>(p.B) * p.Hkv;
    ATTN_CHECK(row >= 0 && row < rows && outer >= 0 && outer < outers);
}

// (debug builds) a partial row index lies in [B * Hq * Lq * n_splits)
__device__ __forceinline__ void decode_check_prow(const DecodeParams& p, size_t prow) {
    ATTN_CHECK(prow < static_cast<size_t>(p.B) * p.Hq * p.Lq * p.n_splits);
}

// KPW = cache rows of each 64-row tile handled by one compute warp (16, 32 or 64).
// A group's query rows are the G heads x Lq new tokens, head-major (row r = head
// r / Lq, token r % Lq), which is also their order in q, out and lse.
template <int D, int KPW>
__global__ void __maxnreg__(200)
    attn_decode_split_kernel(const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
    grid_dep_release();   // the combine launch may be scheduled now
    using L = DecodeSmem<D>;
    constexpr int kNT = KPW / 8;          // 8-key n-tiles of S per warp
    constexpr int kWPM = kDecKT / KPW;    // warps per 16-row block
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
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            int issued = 0;
            for (int t = 0; t < n_tiles; ++t) {
                const int s = t % L::kStages;
                const uint32_t round = static_cast<uint32_t>(t / L::kStages);
                // where rows k_begin + 64 t .. + 63 of (b, g) live
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
                mbar_arrive_expect_tx(bar_full(s), L::kStageBytes);
                const uint32_t dst = ring + s * L::kStageBytes;
                for (int kb = 0; kb < L::kKB; ++kb) {
                    tma_load_3d(dst + kb * L::kBlockBytes, &tm_k, bar_full(s), kb * 64, row, outer);
                    tma_load_3d(dst + L::kTileBytes + kb * L::kBlockBytes, &tm_v, bar_full(s), kb * 64, row, outer);
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
        __syncwarp();
        return;   // the producer takes no part in the merge below
    }

    // ================= compute warps =================
    const int mt = warp / kWPM;           // 16-row block of query heads
    const int ws = warp % kWPM;           // which slice of each tile's keys
    const int key_off = ws * KPW;
    const int grp = lane >> 2, tq = lane & 3;
    const int R = p.G * p.Lq;             // query rows of the group
    const int row_a = mt * 16 + grp, row_b = row_a + 8;   // rows (within the group) this thread holds
    const size_t group_row0 = (static_cast<size_t>(b) * p.Hq + static_cast<size_t>(g) * p.G) * p.Lq;
    // keys this thread's rows may see: below min(k_end, seqlen - Lq + token + 1)
    const int lim_a = min(k_end, seqlen - p.Lq + row_a % p.Lq + 1);
    const int lim_b = min(k_end, seqlen - p.Lq + row_b % p.Lq + 1);
    const int lim_lo = min(k_end, seqlen - p.Lq + 1);   // the smallest limit of any row

    // Q as m16n8k16 A fragments (rows beyond R are zero)
    uint32_t qa[D / 16][4];
    {
        const uint32_t* qrow_a = reinterpret_cast<const uint32_t*>(p.q + (group_row0 + row_a) * D);
        const uint32_t* qrow_b = reinterpret_cast<const uint32_t*>(p.q + (group_row0 + row_b) * D);
        const bool va = row_a < R, vb = row_b < R;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const int c = (kk * 16 + 2 * tq) >> 1;   // bf16x2 index
            qa[kk][0] = va ? __ldg(qrow_a + c) : 0u;
            qa[kk][1] = vb ? __ldg(qrow_b + c) : 0u;
            qa[kk][2] = va ? __ldg(qrow_a + c + 4) : 0u;
            qa[kk][3] = vb ? __ldg(qrow_b + c + 4) : 0u;
        }
    }

    float oacc[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.0f;
    // l: row sum of P as rounded to bf16 (the weights P.V applies; normalises O);
    // le: row sum of the unrounded exponentials (for the log-sum-exp)
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.0f, l_b = 0.0f, le_a = 0.0f, le_b = 0.0f;
    const float sl2 = p.scale_log2;
    bool ok = true;

    for (int t = 0; t < n_tiles; ++t) {
        const int s = t % L::kStages;
        ok = mbar_wait(bar_full(s), static_cast<uint32_t>(t / L::kStages) & 1u, abort_flag, &g_attn_err, kDevErrTimeout);
        if (!ok) break;
        const uint32_t kbase = ring + s * L::kStageBytes;
        const uint32_t vbase = kbase + L::kTileBytes;
        const int tile_key0 = k_begin + t * kDecKT + key_off;   // absolute row of this warp's first key
        const bool tail = (k_begin + (t + 1) * kDecKT > k_end);            // rows past the valid length
        const bool masked = (k_begin + (t + 1) * kDecKT > lim_lo);        // keys some row may not see

        // ---- S = Q K^T over this warp's KPW keys ----
        float sacc[kNT][4];
#pragma unroll
        for (int i = 0; i < kNT; ++i) sacc[i][0] = sacc[i][1] = sacc[i][2] = sacc[i][3] = 0.0f;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t region = kbase + (kk >> 2) * L::kBlockBytes;
            const int cbase = (kk & 3) * 2;
#pragma unroll
            for (int np = 0; np < kNT / 2; ++np) {
                const int mi = lane >> 3, rr = lane & 7;
                const int key_local = key_off + np * 16 + ((mi >> 1) << 3) + rr;
                const int c = cbase + (mi & 1);
                const uint32_t addr = region + key_local * 128 + ((c ^ (key_local & 7)) << 4);
                uint32_t r0, r1, r2, r3;
                ldmatrix_x4(addr, r0, r1, r2, r3);
                mma_bf16_16816(sacc[2 * np], qa[kk], r0, r1);
                mma_bf16_16816(sacc[2 * np + 1], qa[kk], r2, r3);
            }
        }
        // ---- mask keys a row may not see (only in the last tiles of a sequence) ----
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
        const float mn_a = fmaxf(m_a, mx_a * sl2), mn_b = fmaxf(m_b, mx_b * sl2);
        const float f_a = (m_a == -INFINITY) ? 0.0f : ex2_approx(m_a - mn_a);
        const float f_b = (m_b == -INFINITY) ? 0.0f : ex2_approx(m_b - mn_b);
        const float ms_a = (mn_a == -INFINITY) ? 0.0f : mn_a;
        const float ms_b = (mn_b == -INFINITY) ? 0.0f : mn_b;
        m_a = mn_a;
        m_b = mn_b;
        float ps_a = 0.0f, ps_b = 0.0f, pe_a = 0.0f, pe_b = 0.0f;
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) {
            sacc[nt][0] = ex2_approx(fmaf(sacc[nt][0], sl2, -ms_a));
            sacc[nt][1] = ex2_approx(fmaf(sacc[nt][1], sl2, -ms_a));
            sacc[nt][2] = ex2_approx(fmaf(sacc[nt][2], sl2, -ms_b));
            sacc[nt][3] = ex2_approx(fmaf(sacc[nt][3], sl2, -ms_b));
            pe_a += sacc[nt][0] + sacc[nt][1];
            pe_b += sacc[nt][2] + sacc[nt][3];
            // round P to bf16 here, as the MMA will see it, so the row sum
            // matches the weights actually applied to V
            f2_unpack(bf16x2_to_f2(pack_bf16x2(sacc[nt][0], sacc[nt][1])), sacc[nt][0], sacc[nt][1]);
            f2_unpack(bf16x2_to_f2(pack_bf16x2(sacc[nt][2], sacc[nt][3])), sacc[nt][2], sacc[nt][3]);
            ps_a += sacc[nt][0] + sacc[nt][1];
            ps_b += sacc[nt][2] + sacc[nt][3];
        }
        l_a = l_a * f_a + ps_a;
        l_b = l_b * f_b + ps_b;
        le_a = le_a * f_a + pe_a;
        le_b = le_b * f_b + pe_b;
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
            uint32_t a[4];
            a[0] = pack_bf16x2(sacc[2 * k2][0], sacc[2 * k2][1]);
            a[1] = pack_bf16x2(sacc[2 * k2][2], sacc[2 * k2][3]);
            a[2] = pack_bf16x2(sacc[2 * k2 + 1][0], sacc[2 * k2 + 1][1]);
            a[3] = pack_bf16x2(sacc[2 * k2 + 1][2], sacc[2 * k2 + 1][3]);
            // keys held by this thread's V fragments: rows klo, klo+1 (r0, r2) and klo+8, klo+9 (r1, r3)
            const int klo = tile_key0 + k2 * 16 + 2 * tq;
            uint32_t keep_lo = 0xffffffffu, keep_hi = 0xffffffffu;
            if (tail) {
                keep_lo = (klo < k_end ? 0x0000ffffu : 0u) | (klo + 1 < k_end ? 0xffff0000u : 0u);
                keep_hi = (klo + 8 < k_end ? 0x0000ffffu : 0u) | (klo + 9 < k_end ? 0xffff0000u : 0u);
            }
#pragma unroll
            for (int nd = 0; nd < D / 16; ++nd) {
                const int mi = lane >> 3, rr = lane & 7;
                const int key_local = key_off + k2 * 16 + ((mi & 1) << 3) + rr;
                const int dchunk = nd * 2 + (mi >> 1);
                const uint32_t addr = vbase + (dchunk >> 3) * L::kBlockBytes + key_local * 128 +
                                      (((dchunk & 7) ^ (key_local & 7)) << 4);
                uint32_t r0, r1, r2, r3;
                ldmatrix_x4_trans(addr, r0, r1, r2, r3);
                // rows past the valid length may hold anything (NaN): zero them so 0 * NaN cannot appear
                r0 &= keep_lo;
                r2 &= keep_lo;
                r1 &= keep_hi;
                r3 &= keep_hi;
                mma_bf16_16816(oacc[2 * nd], a, r0, r1);
                mma_bf16_16816(oacc[2 * nd + 1], a, r2, r3);
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
    le_a += __shfl_xor_sync(0xffffffffu, le_a, 1);
    le_a += __shfl_xor_sync(0xffffffffu, le_a, 2);
    le_b += __shfl_xor_sync(0xffffffffu, le_b, 1);
    le_b += __shfl_xor_sync(0xffffffffu, le_b, 2);
    asm volatile("bar.sync 1, 128;" ::: "memory");   // every compute warp is done with the ring
    float* sm_m = reinterpret_cast<float*>(smem);
    float* sm_l = sm_m + 4 * 16;
    float* sm_le = sm_l + 4 * 16;
    float* sm_o = sm_le + 4 * 16;
    if (tq == 0) {
        sm_m[warp * 16 + grp] = m_a;
        sm_m[warp * 16 + grp + 8] = m_b;
        sm_l[warp * 16 + grp] = l_a;
        sm_l[warp * 16 + grp + 8] = l_b;
        sm_le[warp * 16 + grp] = le_a;
        sm_le[warp * 16 + grp + 8] = le_b;
    }
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
        const int d = nt * 8 + 2 * tq;
        float* oa = sm_o + (warp * 16 + grp) * D + d;
        float* ob = sm_o + (warp * 16 + grp + 8) * D + d;
        oa[0] = oacc[nt][0];
        oa[1] = oacc[nt][1];
        ob[0] = oacc[nt][2];
        ob[1] = oacc[nt][3];
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (!ok) return;
    for (int idx = threadIdx.x; idx < R * D; idx += 128) {
        const int row = idx / D, d = idx % D;
        const int blk = row >> 4, rr = row & 15;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWPM; ++w) M = fmaxf(M, sm_m[(blk * kWPM + w) * 16 + rr]);
        float Lsum = 0.0f, Lexact = 0.0f, acc = 0.0f;
#pragma unroll
        for (int w = 0; w < kWPM; ++w) {
            const int ww = blk * kWPM + w;
            const float mw = sm_m[ww * 16 + rr];
            const float sc = (mw == -INFINITY) ? 0.0f : ex2_approx(mw - M);
            Lsum += sm_l[ww * 16 + rr] * sc;
            Lexact += sm_le[ww * 16 + rr] * sc;
            acc += sm_o[(ww * 16 + rr) * D + d] * sc;
        }
        const size_t prow = (group_row0 + row) * p.n_splits + split;
        decode_check_prow(p, prow);
        p.o_part[prow * D + d] = (Lsum > 0.0f) ? acc / Lsum : 0.0f;
        if (d == 0) p.lse_part[prow] = (Lexact > 0.0f) ? M + __log2f(Lexact) : -INFINITY;
    }
}

// out = sum_s 2^(lse_s - lse) O_s,  lse = log2 sum_s 2^lse_s, per query row.
// WPR warps per row (1: four rows per CTA; 4: one row per CTA, for rows with many
// splits).  Warp w of a row takes splits w, w + WPR, w + 2 WPR, ... in chunks of
// kChunk; lane i holds the LSE of the chunk's split i and every lane D / 32
// columns of each of its O rows.  All loads of the first chunk -- the row's LSEs
// for the max, the chunk's LSEs and O rows -- are issued before any of them is
// used, so a row with up to WPR * kChunk splits costs one round trip to memory.
// The warps' sums meet in shared memory.
// F32: out is fp32 [rows, D] instead of bf16 (a partial result that is merged later).
template <int D, bool F32 = false, int WPR = 1>
__global__ void __launch_bounds__(128)
    attn_decode_combine_kernel(const DecodeParams p, void* out_ptr, float* lse) {
    grid_dep_wait();   // launched as a programmatic dependent of the split kernel
    static_assert(WPR == 1 || WPR == 4, "one or four warps per row");
    constexpr int kPer = D / 32;                  // columns per lane
    constexpr int kChunk = (D >= 256) ? 8 : 16;   // splits per warp whose O rows are in registers
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * (4 / WPR) + warp / WPR;
    const int sub = warp % WPR;
    if (row >= p.B * p.Hq * p.Lq) return;   // (uniform over a CTA when WPR = 4)
    const int b = row / (p.Hq * p.Lq);
    const int seqlen = decode_seqlen(p, b);
    const int n_valid = (seqlen + p.chunk - 1) / p.chunk;
    ATTN_CHECK(n_valid >= 0 && n_valid <= p.n_splits);
    const float* lp = p.lse_part + static_cast<size_t>(row) * p.n_splits;
    const float* op = p.o_part + static_cast<size_t>(row) * p.n_splits * D + lane * kPer;
    float ov[kChunk][kPer];
    float my_ls;
    // this warp's chunk from split `base`: lane i's LSE, every lane's columns of the O rows
    auto load_chunk = [&](int base) {
        const int sl = base + sub + WPR * lane;
        my_ls = (lane < kChunk && sl < n_valid) ? lp[sl] : -INFINITY;
#pragma unroll
        for (int i = 0; i < kChunk; ++i) {
            const int s = base + sub + WPR * i;
            if (s < n_valid) {
                const float* src = op + static_cast<size_t>(s) * D;
#pragma unroll
                for (int c = 0; c < kPer; c += 2) {
                    const float2 v = *reinterpret_cast<const float2*>(src + c);
                    ov[i][c] = v.x;
                    ov[i][c + 1] = v.y;
                }
            } else {
#pragma unroll
                for (int c = 0; c < kPer; ++c) ov[i][c] = 0.0f;
            }
        }
    };
    load_chunk(0);
    float M = -INFINITY;
    for (int s = lane; s < n_valid; s += 32) M = fmaxf(M, lp[s]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float acc[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) acc[i] = 0.0f;
    float Lsum = 0.0f;   // lane i: the weights of its splits
    for (int base = 0; base < n_valid; base += WPR * kChunk) {
        if (base > 0) load_chunk(base);
        const float wl = (my_ls == -INFINITY) ? 0.0f : ex2_approx(my_ls - M);   // split weight (lane < kChunk)
        Lsum += wl;
#pragma unroll
        for (int i = 0; i < kChunk; ++i) {
            const float w = __shfl_sync(0xffffffffu, wl, i);
#pragma unroll
            for (int c = 0; c < kPer; ++c) acc[c] = fmaf(w, ov[i][c], acc[c]);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Lsum += __shfl_xor_sync(0xffffffffu, Lsum, o);
    if constexpr (WPR > 1) {
        __shared__ float red_acc[WPR][D];
        __shared__ float red_l[WPR];
#pragma unroll
        for (int i = 0; i < kPer; ++i) red_acc[sub][lane * kPer + i] = acc[i];
        if (lane == 0) red_l[sub] = Lsum;
        __syncthreads();
        if (sub != 0) return;
#pragma unroll
        for (int w = 1; w < WPR; ++w) {
#pragma unroll
            for (int i = 0; i < kPer; ++i) acc[i] += red_acc[w][lane * kPer + i];
            Lsum += red_l[w];
        }
    }
    const float inv = (Lsum > 0.0f) ? 1.0f / Lsum : 0.0f;
    if constexpr (F32) {
        float* o = static_cast<float*>(out_ptr) + static_cast<size_t>(row) * D + lane * kPer;
#pragma unroll
        for (int i = 0; i < kPer; i += 2) *reinterpret_cast<float2*>(o + i) = make_float2(acc[i] * inv, acc[i + 1] * inv);
    } else {
        __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out_ptr) + static_cast<size_t>(row) * D + lane * kPer;
#pragma unroll
        for (int i = 0; i < kPer; i += 2) {
            const uint32_t v2 = pack_bf16x2(acc[i] * inv, acc[i + 1] * inv);
            *reinterpret_cast<uint32_t*>(o + i) = v2;
        }
    }
    if (lse != nullptr && lane == 0) lse[row] = (Lsum > 0.0f) ? (M + __log2f(Lsum)) * kLn2 : -INFINITY;
}

// Merge of decode results over disjoint sets of cache rows (KV parallelism: each
// set held by one GPU, the NVIDIA attention page, "Parameter four: parallelism"):
// out[r] = sum_p exp(lse_p[r] - lse[r]) O_p[r],  lse[r] = ln sum_p exp(lse_p[r]).
// o_parts [n_parts][rows][D] fp32 (each normalised over its own rows), lse_parts
// [n_parts][rows] natural log (-inf: no rows).  One warp per row, as the combine.
template <int D>
__global__ void __launch_bounds__(128)
    attn_decode_merge_kernel(const float* o_parts, const float* lse_parts, int n_parts, int rows,
                             __nv_bfloat16* out, float* lse) {
    const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    constexpr int kPer = D / 32;
    float M = -INFINITY;
    for (int q = lane; q < n_parts; q += 32) M = fmaxf(M, lse_parts[static_cast<size_t>(q) * rows + row]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float acc[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) acc[i] = 0.0f;
    float Lsum = 0.0f;
    for (int q0 = 0; q0 < n_parts; q0 += 32) {
        const int q = q0 + lane;
        const float ls = (q < n_parts) ? lse_parts[static_cast<size_t>(q) * rows + row] : -INFINITY;
        const float wl = (ls == -INFINITY) ? 0.0f : ex2_approx((ls - M) * kLog2e);
        Lsum += wl;
        const int cnt = min(32, n_parts - q0);
#pragma unroll 4
        for (int i = 0; i < cnt; ++i) {
            const float w = __shfl_sync(0xffffffffu, wl, i);
            const float* src = o_parts + (static_cast<size_t>(q0 + i) * rows + row) * D + lane * kPer;
#pragma unroll
            for (int c = 0; c < kPer; c += 2) {
                const float2 v = *reinterpret_cast<const float2*>(src + c);
                acc[c] = fmaf(w, v.x, acc[c]);
                acc[c + 1] = fmaf(w, v.y, acc[c + 1]);
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Lsum += __shfl_xor_sync(0xffffffffu, Lsum, o);
    const float inv = (Lsum > 0.0f) ? 1.0f / Lsum : 0.0f;
    __nv_bfloat16* o = out + static_cast<size_t>(row) * D + lane * kPer;
#pragma unroll
    for (int i = 0; i < kPer; i += 2) *reinterpret_cast<uint32_t*>(o + i) = pack_bf16x2(acc[i] * inv, acc[i + 1] * inv);
    if (lse != nullptr && lane == 0) lse[row] = (Lsum > 0.0f) ? M + __logf(Lsum) : -INFINITY;
}

// ---------------------------------------------------------------------------
// KV parallelism with the exchange fused into the merge.  Each GPU writes its
// partial results into its own memory; the merge on every GPU then reads all
// parts where they lie (plain loads: this GPU's memory, or a peer's over
// NVLink), instead of first copying them with an all-gather.  Flags order the
// steps, each a 32-bit epoch counter compared wraparound-safely:
//   ready[p]    part p is complete (set by part p's GPU after its partial)
//   consumed[p] GPU p has finished reading every part of that epoch (set after
//               its merge), so a part's buffer may be overwritten next epoch.
// Every wait is bounded: after kWaitLimitNs it sets ATTN_DEVERR_TIMEOUT and the
// kernel skips its work instead of hanging.
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t ld_acquire_sys(const unsigned int* p) {
    uint32_t v;
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_sys(unsigned int* p, uint32_t v) {
    asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// flag has reached `value` (epochs only grow; compared modulo 2^32)
__device__ __forceinline__ bool epoch_reached(uint32_t flag, uint32_t value) {
    return static_cast<int32_t>(flag - value) >= 0;
}

// One thread waits until flags[0 .. n) have all reached `value`; false after the time limit.
__device__ __forceinline__ bool wait_flags(const unsigned int* flags, int n, uint32_t value) {
    const uint64_t t0 = global_timer_ns();
    for (int i = 0; i < n; ++i) {
        while (!epoch_reached(ld_acquire_sys(flags + i), value)) {
            if (global_timer_ns() - t0 > kWaitLimitNs) {
                atomicOr(&g_attn_err, kDevErrTimeout);
                return false;
            }
            __nanosleep(64);
        }
    }
    return true;
}

// flag_ptrs[i] <- value for i < n, after everything this GPU wrote before this
// kernel (in stream order) is visible system-wide.
__global__ void attn_kvp_signal_kernel(unsigned int* const* flag_ptrs, int n, uint32_t value) {
    __threadfence_system();
    for (int i = threadIdx.x; i < n; i += blockDim.x) st_release_sys(flag_ptrs[i], value);
}

__global__ void attn_kvp_wait_kernel(const unsigned int* flags, int n, uint32_t value) {
    if (threadIdx.x == 0) wait_flags(flags, n, value);
}

// attn_decode_merge_kernel over parts reached through pointers: part p's O at
// o_ptrs[p] ([rows][D] fp32) and LSE at lse_ptrs[p] ([rows]), read only after
// ready[p] has reached `value`.
template <int D>
__global__ void __launch_bounds__(128)
    attn_decode_merge_peers_kernel(const float* const* o_ptrs, const float* const* lse_ptrs,
                                   const unsigned int* ready, uint32_t value, int n_parts, int rows,
                                   __nv_bfloat16* out, float* lse) {
    __shared__ int go;
    if (threadIdx.x == 0) go = wait_flags(ready, n_parts, value) ? 1 : 0;
    __syncthreads();
    if (!go) return;
    const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    constexpr int kPer = D / 32;
    float M = -INFINITY;
    // parts are read at L2 (.cg): the same addresses held last epoch's values
    for (int q = lane; q < n_parts; q += 32) M = fmaxf(M, __ldcg(lse_ptrs[q] + row));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float acc[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) acc[i] = 0.0f;
    float Lsum = 0.0f;
    for (int q0 = 0; q0 < n_parts; q0 += 32) {
        const int q = q0 + lane;
        const float ls = (q < n_parts) ? __ldcg(lse_ptrs[q] + row) : -INFINITY;
        const float wl = (ls == -INFINITY) ? 0.0f : ex2_approx((ls - M) * kLog2e);
        Lsum += wl;
        const int cnt = min(32, n_parts - q0);
        for (int i = 0; i < cnt; ++i) {
            const float w = __shfl_sync(0xffffffffu, wl, i);
            const float* src = o_ptrs[q0 + i] + static_cast<size_t>(row) * D + lane * kPer;
#pragma unroll
            for (int c = 0; c < kPer; c += 2) {
                const float2 v = __ldcg(reinterpret_cast<const float2*>(src + c));
                acc[c] = fmaf(w, v.x, acc[c]);
                acc[c + 1] = fmaf(w, v.y, acc[c + 1]);
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Lsum += __shfl_xor_sync(0xffffffffu, Lsum, o);
    const float inv = (Lsum > 0.0f) ? 1.0f / Lsum : 0.0f;
    __nv_bfloat16* o = out + static_cast<size_t>(row) * D + lane * kPer;
#pragma unroll
    for (int i = 0; i < kPer; i += 2) *reinterpret_cast<uint32_t*>(o + i) = pack_bf16x2(acc[i] * inv, acc[i + 1] * inv);
    if (lse != nullptr && lane == 0) lse[row] = (Lsum > 0.0f) ? M + __logf(Lsum) : -INFINITY;
}

}  // namespace attn
