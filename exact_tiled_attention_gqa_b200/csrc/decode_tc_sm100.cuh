// decode_tc_sm100.cuh -- split-KV decode on the tcgen05 tensor cores, for KV
// heads with many query rows (G x Lq > 16) and for every group size at D = 256.
//
// Same computation, split and partial format as attn_decode_split_kernel
// (decode_sm100.cuh): a CTA owns `chunk` cache rows of one (b, KV head) and
// writes one normalised partial output and log2-sum-exp per query row; the
// same combine kernel merges the splits.  The difference is where the
// arithmetic runs.  Decode reads G x Lq query rows per cache row, i.e. G x Lq
// FLOPs per byte (NVIDIA attention page, "Parameter one: group size": more
// query heads per KV head raise the arithmetic intensity), so at G = 32..64
// the warp-level mma.sync path runs out of math before the cache runs out of
// bandwidth.  Here the group's rows are the M = 128 rows of tcgen05 MMAs, over
// tiles of 64 cache rows:
//
//   S  = Q K_j^T   (M = 128 rows, N = 64 cache rows, K = D)
//   P  = 2^(S * scale * log2 e - m)  (softmax warpgroup, thread = row = TMEM lane)
//   O += P V_j     (P from TMEM, V MN-major from shared memory)
//
// 6 warps: warps 0-3 softmax, warp 4 TMA producer, warp 5 TMEM allocator and
// MMA issuer.  Latency, not math, bounds decode, so the design keeps the tensor
// cores and the softmax overlapped and loads in flight:
//  - two S buffers in TMEM: the issuer runs S(0), S(1), then per tile
//    O += P(j) V_j and S(j+2), so S(j+1) is computed while the softmax works on
//    S(j).  Each P V gets its own commit; the softmax waits on it only when it
//    rescales O (lazy max: the running max moves only when a tile's max beats
//    it by more than 2^8);
//  - 64-row tiles keep TMEM at 256 columns (S0 [0,64), S1 [64,128) with P over
//    the first 32 columns of its S, O [128, 128 + D)), so two CTAs share an SM
//    for D <= 128 and one's softmax overlaps the other's (D = 256: 512 columns,
//    one CTA per SM);
//  - a ring of 64-row K and V tiles (each one TMA box per 64 columns, so paged
//    caches with 64-row pages work), filled in the order the MMAs use them
//    (K_0 K_1 V_0 K_2 V_1 ..., ring_order.cuh).
//
// The softmax reads a tile's S from TMEM once into registers (row max, then the
// exponentials).  Warps whose 32 rows are all padding only keep the pipeline moving.  Cache rows past
// the split's valid length may hold anything (NaN included); P is 0 there but
// 0 * NaN is NaN, so the MMA warp zeroes those V rows in shared memory first.
#pragma once

#include "decode_sm100.cuh"
#include "device_error.cuh"
#include "ptx_sm100.cuh"
#include "ring_order.cuh"

namespace attn {

constexpr int kDtcThreads = 192;
constexpr int kDtcBN = 64;           // cache rows per tile
constexpr int kDtcProducerWarp = 4;
constexpr int kDtcMmaWarp = 5;
constexpr float kDtcRescaleLog2 = 8.0f;

template <int D>
struct DecodeTcSmem {
    static constexpr int kKB = D / 64;
    static constexpr int kCtasPerSm = (D <= 128) ? 2 : 1;
    static constexpr int kQBlockBytes = 128 * 128;         // Q: 128 rows x 128 bytes per 64 columns
    static constexpr int kQBytes = 128 * D * 2;
    static constexpr int kHalfBlockBytes = 64 * 128;        // a tile: 64 rows x 128 bytes per 64 columns
    static constexpr int kHalfBytes = 64 * D * 2;           // one K or V tile
    // as many tiles as fit beside Q when kCtasPerSm CTAs share the SM's 228 KB
    // (1 KB reserved per CTA, 1 KB alignment slack, 2 KB for barriers), at most 16
    static constexpr int kStagesFit = (233472 / kCtasPerSm - 1024 - 1024 - 2048 - kQBytes) / kHalfBytes;
    static constexpr int kStages = kStagesFit > 16 ? 16 : kStagesFit;
    static constexpr uint32_t kTmemCols = (128 + D <= 256) ? 256u : 512u;   // S0 + S1 + O, rounded up
    static constexpr int kQOff = 0;
    static constexpr int kKVOff = kQBytes;
    static constexpr int kBarOff = kKVOff + kStages * kHalfBytes;
    // q_full, full[S], empty[S], s_full[2], p_full[2], o_ready, o_done, drain
    static constexpr int kNumBars = 1 + 2 * kStages + 2 + 2 + 3;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;  // tmem base, abort flag
    static constexpr int kTagOff = kMiscOff + 16;             // debug builds: ring entry -> item index
    static constexpr int kBytes = kTagOff + 4 * kStages;
    static constexpr int kAlloc = kBytes + 1024;
    static_assert(kAlloc <= 232448, "dynamic shared memory per CTA");
    static_assert(kStages >= 4, "ring too shallow");
};

template <int D>
__global__ void __launch_bounds__(kDtcThreads, DecodeTcSmem<D>::kCtasPerSm)
    attn_decode_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
    grid_dep_release();   // the combine launch may be scheduled now
    using L = DecodeTcSmem<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_base);

    const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int seqlen = decode_seqlen(p, b);
    const int k_begin = split * p.chunk;
    if (k_begin >= seqlen) return;   // uniform: this split has no rows
    const int k_end = min(k_begin + p.chunk, seqlen);
    const int n_tiles = (k_end - k_begin + kDtcBN - 1) / kDtcBN;
    const int R = p.G * p.Lq;          // query rows of the group (<= 128)
    const size_t group_row0 = (static_cast<size_t>(b) * p.Hq + static_cast<size_t>(g) * p.G) * p.Lq;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t sQ = base + L::kQOff;
    const uint32_t sKV = base + L::kKVOff;
    const uint32_t bar0 = base + L::kBarOff;
    const uint32_t bar_q_full = bar0;
    auto bar_full = [&](int s) { return bar0 + 8u * (1 + s); };
    auto bar_empty = [&](int s) { return bar0 + 8u * (1 + L::kStages + s); };
    auto bar_s_full = [&](int i) { return bar0 + 8u * (1 + 2 * L::kStages + i); };
    auto bar_p_full = [&](int i) { return bar0 + 8u * (3 + 2 * L::kStages + i); };
    const uint32_t bar_o_ready = bar0 + 8u * (5 + 2 * L::kStages);
    const uint32_t bar_o_done = bar_o_ready + 8u;
    const uint32_t bar_drain = bar_o_ready + 16u;
    uint32_t* tmem_base_ptr = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
    // (debug builds) the ring position the producer put in each entry, checked by the MMA warp
    volatile int* ring_tag = reinterpret_cast<volatile int*>(smem + L::kTagOff);

    if (threadIdx.x == 0) {
        mbar_init(bar_q_full, 1);
        for (int s = 0; s < L::kStages; ++s) {
            mbar_init(bar_full(s), 1);
            mbar_init(bar_empty(s), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar_s_full(i), 1);
            mbar_init(bar_p_full(i), 128);
        }
        mbar_init(bar_o_ready, 1);
        mbar_init(bar_o_done, 1);
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // query rows R .. 127 are not loaded: make them zero (finite) for the MMA
    if (R < 128) {
        const int pad = (128 - R) * 128;
        for (int kb = 0; kb < L::kKB; ++kb) {
            uint8_t* blk = smem + L::kQOff + kb * L::kQBlockBytes + R * 128;
            for (int i = threadIdx.x * 16; i < pad; i += kDtcThreads * 16)
                *reinterpret_cast<uint4*>(blk + i) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
    }
    if (warp == kDtcMmaWarp) {
        tmem_alloc(smem_u32(tmem_base_ptr), L::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_base_ptr;
    const uint32_t tS[2] = {tmem, tmem + 64u};    // S buffers (P over the first 32 columns)
    const uint32_t tO = tmem + 128u;               // O

    // ring entry t holds the tile at ring position t (K_0 K_1 V_0 K_2 V_1 ...)
    const int n_items = 2 * n_tiles;
    auto slot_of = [&](int t) { return t % L::kStages; };
    auto par_of = [&](int t) { return static_cast<uint32_t>(t / L::kStages) & 1u; };

    if (warp == kDtcProducerWarp) {
        // ================= TMA producer =================
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            mbar_arrive_expect_tx(bar_q_full, static_cast<uint32_t>(L::kKB * R * 128));
            for (int kb = 0; kb < L::kKB; ++kb)
                tma_load_3d(sQ + kb * L::kQBlockBytes, &tm_q, bar_q_full, kb * 64, static_cast<int>(group_row0), 0);
            int issued = 0;
            for (int t = 0; t < n_items; ++t) {
                const int s = slot_of(t);
                if (!mbar_wait(bar_empty(s), par_of(t) ^ 1u, abort_flag, &g_attn_err, kDevErrTimeout)) break;
                bool is_v;
                int j;
                ring_tile<1>(t, n_tiles, is_v, j);
                const int key0 = k_begin + j * kDtcBN;   // split starts are multiples of 64
                int row = key0, outer = b * p.Hkv + g;
                if (p.block_table != nullptr) {
                    int page = __ldg(p.block_table + static_cast<size_t>(b) * p.max_pages + key0 / p.page_size);
                    if (page < 0 || page >= p.n_pages) {
                        atomicOr(&g_attn_err, kDevErrPage);
                        page = 0;
                    }
                    row = key0 % p.page_size;
                    outer = page * p.Hkv + g;
                }
                decode_check_tile(p, row, outer);
                ATTN_CHECK(j >= 0 && j < n_tiles);
                if (ATTN_DEBUG_BOUNDS) ring_tag[s] = t;
                mbar_arrive_expect_tx(bar_full(s), L::kHalfBytes);
                const CUtensorMap* map = is_v ? &tm_v : &tm_k;
                const uint32_t dst = sKV + s * L::kHalfBytes;
                for (int kb = 0; kb < L::kKB; ++kb)
                    tma_load_3d(dst + kb * L::kHalfBlockBytes, map, bar_full(s), kb * 64, row, outer);
                issued = t + 1;
            }
            if (issued < n_items) {
                // unwinding after a timeout: let issued copies land first
                for (int t = max(0, issued - L::kStages); t < issued; ++t) {
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(bar_full(slot_of(t)), par_of(t)) && global_timer_ns() - t0 < 100000000ull) {
                    }
                }
                const uint64_t t0 = global_timer_ns();
                while (!mbar_try_wait(bar_q_full, 0) && global_timer_ns() - t0 < 100000000ull) {
                }
            }
        }
        __syncwarp();
    } else if (warp == kDtcMmaWarp) {
        // ================= MMA issuer (lane 0 issues; the warp clears stale V rows) =================
        constexpr uint32_t kIdescQK = umma_idesc_bf16_f32(128, kDtcBN, false);
        constexpr uint32_t kIdescPV = umma_idesc_bf16_f32(128, D, true);
        const uint64_t dQ = umma_sdesc_sw128(sQ, 16, 1024);
        const uint64_t dK0 = umma_sdesc_sw128(sKV, 16, 1024);
        const uint64_t dV0 = umma_sdesc_sw128(sKV, L::kHalfBlockBytes, 1024);
        constexpr uint64_t kSlotStep = L::kHalfBytes >> 4;
        auto wait_item = [&](int it) {
            const bool got = mbar_wait(bar_full(slot_of(it)), par_of(it), abort_flag, &g_attn_err, kDevErrTimeout);
            if (got) ATTN_CHECK(ring_tag[slot_of(it)] == it);   // (debug builds) the entry holds that item
            return got;
        };
        // S(j) = Q K_j^T into buffer j % 2 (N = 64 cache rows)
        auto qk = [&](int j) {
            const int it = ring_pos_k<1>(j);
            if (!wait_item(it)) return false;
            tc_fence_after_sync();
            if (lane == 0) {
                const uint64_t b0 = dK0 + static_cast<uint64_t>(slot_of(it)) * kSlotStep;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t qoff = static_cast<uint64_t>(((kk >> 2) * L::kQBlockBytes + (kk & 3) * 32) >> 4);
                    const uint64_t koff = static_cast<uint64_t>(((kk >> 2) * L::kHalfBlockBytes + (kk & 3) * 32) >> 4);
                    umma_ss(tS[j & 1], dQ + qoff, b0 + koff, kIdescQK, kk > 0 ? 1u : 0u);
                }
                umma_commit(bar_empty(slot_of(it)));
                umma_commit(bar_s_full(j & 1));
            }
            __syncwarp();
            return true;
        };
        bool ok = mbar_wait(bar_q_full, 0, abort_flag, &g_attn_err, kDevErrTimeout);
        if (ok) ok = qk(0);
        if (ok && n_tiles > 1) ok = qk(1);
        for (int j = 0; j < n_tiles && ok; ++j) {
            const int buf = j & 1;
            const uint32_t ph = static_cast<uint32_t>(j >> 1) & 1u;
            const int itv = ring_pos_v<1>(j, n_tiles);
            ok = wait_item(itv) && mbar_wait(bar_p_full(buf), ph, abort_flag, &g_attn_err, kDevErrTimeout);
            if (!ok) break;
            // V rows past this split's last row: zero them (P is 0 there, but 0 * NaN is NaN)
            const int valid = k_end - (k_begin + j * kDtcBN);
            if (valid < kDtcBN) {
                uint8_t* ent = smem + L::kKVOff + slot_of(itv) * L::kHalfBytes;
                for (int kb = 0; kb < L::kKB; ++kb) {
                    uint8_t* blk = ent + kb * L::kHalfBlockBytes + valid * 128;
                    for (int i = lane * 16; i < (kDtcBN - valid) * 128; i += 32 * 16)
                        *reinterpret_cast<uint4*>(blk + i) = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();
            }
            __syncwarp();
            tc_fence_after_sync();
            if (lane == 0) {
                // O += P(j) V_j: 4 steps of 16 cache rows
                const uint64_t b0 = dV0 + static_cast<uint64_t>(slot_of(itv)) * kSlotStep;
#pragma unroll
                for (int kk = 0; kk < kDtcBN / 16; ++kk)
                    umma_ts(tO, tS[buf] + kk * 8, b0 + static_cast<uint64_t>((kk * 2048) >> 4), kIdescPV,
                            (j > 0 || kk > 0) ? 1u : 0u);
                umma_commit(bar_o_ready);
                if (j + 1 == n_tiles) umma_commit(bar_o_done);
                umma_commit(bar_empty(slot_of(itv)));
            }
            __syncwarp();
            if (j + 2 < n_tiles) ok = qk(j + 2);
        }
        if (lane == 0) {
            // Drain: no MMA may still be running when TMEM is released.
            umma_commit(bar_drain);
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(bar_drain, 0) && global_timer_ns() - t0 < 100000000ull) {
            }
        }
        __syncwarp();
    } else {
        // ================= softmax warpgroup (thread = row = TMEM lane) =================
        const int r = threadIdx.x;               // 0..127
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        const uint32_t tOr = tO + lane_off;
        // keys this row may see: below min(k_end, seqlen - Lq + token + 1)
        const int lim = min(k_end, seqlen - p.Lq + r % p.Lq + 1);
        const int lim_lo = min(k_end, seqlen - p.Lq + 1);
        const float sl2 = p.scale_log2;
        const uint64_t sl2x2 = f2_pack(sl2, sl2);
        // l_run: row sum of P as rounded to bf16 (normalises O); l_exact: of the
        // unrounded exponentials (for the log-sum-exp)
        float m_run = -INFINITY, l_run = 0.0f, l_exact = 0.0f;
        // A warp whose 32 rows are all padding (row >= R) only keeps the pipeline
        // moving: its P rows are never read into a real output row (the MMA keeps
        // rows apart), so it skips the softmax and just signals.
        const bool idle_warp = warp * 32 >= R;
        bool ok = true;
        for (int j = 0; j < n_tiles; ++j) {
            const int buf = j & 1;
            ok = mbar_wait(bar_s_full(buf), static_cast<uint32_t>(j >> 1) & 1u, abort_flag, &g_attn_err,
                           kDevErrTimeout);
            if (!ok) break;
            tc_fence_after_sync();
            if (idle_warp) {
                tc_fence_before_sync();
                mbar_arrive(bar_p_full(buf));
                continue;
            }
            const uint32_t tSr = tS[buf] + lane_off;
            const int key0 = k_begin + j * kDtcBN;
            const bool masked = key0 + kDtcBN > lim_lo;
            // the tile's 64 scores of this row, read from TMEM once
            uint32_t v[kDtcBN];
            tmem_ld_32x32b_x32(tSr, v);
            tmem_ld_32x32b_x32(tSr + 32, v + 32);
            tmem_wait_ld();
            reg_fence<kDtcBN>(v);
            if (masked) {
#pragma unroll
                for (int i = 0; i < kDtcBN; ++i)
                    if (key0 + i >= lim) v[i] = __float_as_uint(-INFINITY);
            }
            float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
            for (int i = 0; i < kDtcBN; i += 8) {
                mx0 = fmax3(mx0, __uint_as_float(v[i]), __uint_as_float(v[i + 1]));
                mx1 = fmax3(mx1, __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
                mx2 = fmax3(mx2, __uint_as_float(v[i + 4]), __uint_as_float(v[i + 5]));
                mx3 = fmax3(mx3, __uint_as_float(v[i + 6]), __uint_as_float(v[i + 7]));
            }
            const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
            float factor = 1.0f;
            if (m_tile > m_run + kDtcRescaleLog2) {
                factor = (m_run == -INFINITY) ? 0.0f : ex2_approx(m_run - m_tile);
                m_run = m_tile;
                l_run *= factor;
                l_exact *= factor;
            }
            if (j > 0 && __any_sync(0xffffffffu, factor != 1.0f)) {
                // O must hold tiles 0..j-1: O += P(j-1) V_{j-1} is the only one that can be in flight
                if (!mbar_wait(bar_o_ready, static_cast<uint32_t>(j - 1) & 1u, abort_flag, &g_attn_err,
                               kDevErrTimeout)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint64_t f2 = f2_pack(factor, factor);
#pragma unroll 1
                for (int c = 0; c < D; c += 32) {
                    uint32_t o[32];
                    tmem_ld_32x32b_x32(tOr + c, o);
                    tmem_wait_ld();
                    reg_fence<32>(o);
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        float a0, a1;
                        f2_unpack(f2_mul(f2_pack(__uint_as_float(o[i]), __uint_as_float(o[i + 1])), f2), a0, a1);
                        o[i] = __float_as_uint(a0);
                        o[i + 1] = __float_as_uint(a1);
                    }
                    tmem_st_32x32b_x32(tOr + c, o);
                }
                tmem_wait_st();
            }
            // exponentials, row sums, P (bf16) over the S columns already read
            const float m_sub = (m_run == -INFINITY) ? 0.0f : m_run;
            const uint64_t negm2 = f2_pack(-m_sub, -m_sub);
            uint64_t acc_r = 0ull, acc_e = 0ull;
#pragma unroll
            for (int c = 0; c < kDtcBN; c += 32) {
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const uint64_t t = f2_fma(f2_pack(__uint_as_float(v[c + 2 * i]), __uint_as_float(v[c + 2 * i + 1])),
                                              sl2x2, negm2);
                    float t0, t1;
                    f2_unpack(t, t0, t1);
                    const float e0 = ex2_approx(t0), e1 = ex2_approx(t1);
                    pk[i] = pack_bf16x2(e0, e1);
                    acc_e = f2_add(acc_e, f2_pack(e0, e1));
                    acc_r = f2_add(acc_r, bf16x2_to_f2(pk[i]));   // P as the MMA sees it
                }
                tmem_st_32x32b_x16(tSr + c / 2, pk);
            }
            tmem_wait_st();
            tc_fence_before_sync();
            mbar_arrive(bar_p_full(buf));
            float a0, a1, e0, e1;
            f2_unpack(acc_r, a0, a1);
            f2_unpack(acc_e, e0, e1);
            l_run += a0 + a1;
            l_exact += e0 + e1;
        }
        // ---- this split's partial: O / l (fp32) and m + log2 l per row ----
        bool have_o = ok && n_tiles > 0;
        if (have_o) {
            have_o = mbar_wait(bar_o_done, 0, abort_flag, &g_attn_err, kDevErrTimeout);
            tc_fence_after_sync();
        }
        const bool row_valid = r < R;
        const float inv_l = (l_run > 0.0f) ? 1.0f / l_run : 0.0f;
        const size_t prow = (group_row0 + static_cast<size_t>(row_valid ? r : 0)) * p.n_splits + split;
        decode_check_prow(p, prow);
        float* dst = p.o_part + prow * D;
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
            uint32_t o[32];
            if (have_o) {
                tmem_ld_32x32b_x32(tOr + c, o);
                tmem_wait_ld();
                reg_fence<32>(o);
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = 0u;
            }
            if (row_valid) {
#pragma unroll
                for (int i = 0; i < 32; i += 4)
                    *reinterpret_cast<float4*>(dst + c + i) =
                        make_float4(__uint_as_float(o[i]) * inv_l, __uint_as_float(o[i + 1]) * inv_l,
                                    __uint_as_float(o[i + 2]) * inv_l, __uint_as_float(o[i + 3]) * inv_l);
            }
        }
        if (row_valid) p.lse_part[prow] = (l_exact > 0.0f) ? m_run + __log2f(l_exact) : -INFINITY;
    }

    // ---- teardown ----
    tc_fence_before_sync();
    __syncthreads();
    if (warp == kDtcMmaWarp) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, L::kTmemCols);
    }
}

}  // namespace attn
