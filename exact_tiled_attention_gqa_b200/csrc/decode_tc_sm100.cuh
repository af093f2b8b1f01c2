// decode_tc_sm100.cuh -- split-KV decode on the tcgen05 tensor cores, for KV
// heads with many query rows (G x Lq > 16), and for every group size at
// D = 256 (a 256-wide O does not fit the mma.sync kernel's registers; there
// Q, the two slots and 384 TMEM columns make it one CTA per SM).
//
// Same computation, split and partial format as attn_decode_split_kernel
// (decode_sm100.cuh): a CTA owns `chunk` cache rows of one (b, KV head) and
// writes one normalised partial output and log2-sum-exp per query row; the
// same combine kernel merges the splits.  The difference is where the
// arithmetic runs.  Decode reads G x Lq query rows per cache row, i.e. G x Lq
// FLOPs per byte (NVIDIA attention page, "Parameter one: group size": more
// query heads per KV head raise the arithmetic intensity), so at G = 32..64
// the warp-level mma.sync path runs out of math before the cache runs out of
// bandwidth.  Here the group's rows are the M = 128 rows of one tcgen05 MMA:
//
//   S  = Q K_j^T   (M = 128 rows, N = 128 keys, K = D), into TMEM
//   P  = 2^(S * scale * log2 e - m)  (softmax warpgroup, thread = row = TMEM lane)
//   O += P V_j     (P from TMEM, V MN-major from shared memory)
//
// One CTA is 6 warps: warps 0-3 softmax, warp 4 TMA producer (K_j and V_j
// into a two-slot ring, each 128-row tile as two 64-row boxes so paged caches
// with 64-row pages work too), warp 5 TMEM allocator and MMA issuer.  TMEM:
// S [0,128) with P over its first 64 columns, O [128, 128 + D); 256 columns,
// so two CTAs share an SM and one's softmax overlaps the other's MMAs.  The
// pipeline per tile is serial (S(j+1) waits for O += P(j) V_j, which frees
// the TMEM P lives in); the cache stream is what bounds this kernel.
//
// The softmax reads S twice from TMEM (row max, then the exponentials) to
// keep registers low enough for two CTAs per SM, and uses the same lazy
// rescale as the prefill kernel: the running max only moves when a tile's
// max beats it by more than 2^8.
#pragma once

#include "decode_sm100.cuh"
#include "device_error.cuh"
#include "ptx_sm100.cuh"

namespace attn {

constexpr int kDtcThreads = 192;
constexpr int kDtcBN = 128;          // cache rows per tile
constexpr int kDtcProducerWarp = 4;
constexpr int kDtcMmaWarp = 5;
constexpr float kDtcRescaleLog2 = 8.0f;

template <int D>
struct DecodeTcSmem {
    static constexpr int kKB = D / 64;
    static constexpr int kBlockBytes = 128 * 128;           // 128 rows x 128 bytes
    static constexpr int kQBytes = 128 * D * 2;
    static constexpr int kTileBytes = kDtcBN * D * 2;       // one K or V tile
    static constexpr int kStages = 2;                       // K_j in slot 0, V_j in slot 1
    static constexpr int kQOff = 0;
    static constexpr int kKVOff = kQBytes;
    static constexpr int kBarOff = kKVOff + kStages * kTileBytes;
    // q_full, kv_full[2], kv_empty[2], s_full, p_full, o_done, drain
    static constexpr int kNumBars = 1 + 2 * kStages + 4;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;  // tmem base, abort flag
    static constexpr int kBytes = kMiscOff + 16;
    static constexpr int kAlloc = kBytes + 1024;
    static constexpr uint32_t kTmemCols = (128 + D <= 256) ? 256u : 512u;   // S + O, rounded up
};

template <int D>
__global__ void __launch_bounds__(kDtcThreads, 2)
    attn_decode_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
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
    auto bar_kv_full = [&](int s) { return bar0 + 8u * (1 + s); };
    auto bar_kv_empty = [&](int s) { return bar0 + 8u * (1 + L::kStages + s); };
    const uint32_t bar_s_full = bar0 + 8u * (1 + 2 * L::kStages);
    const uint32_t bar_p_full = bar_s_full + 8u;
    const uint32_t bar_o_done = bar_s_full + 16u;
    const uint32_t bar_drain = bar_s_full + 24u;
    uint32_t* tmem_base_ptr = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

    if (threadIdx.x == 0) {
        mbar_init(bar_q_full, 1);
        for (int s = 0; s < L::kStages; ++s) {
            mbar_init(bar_kv_full(s), 1);
            mbar_init(bar_kv_empty(s), 1);
        }
        mbar_init(bar_s_full, 1);
        mbar_init(bar_p_full, 128);
        mbar_init(bar_o_done, 1);
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // query rows R .. 127 are not loaded: make them zero (finite) for the MMA
    if (R < 128) {
        const int pad = (128 - R) * 128;
        for (int kb = 0; kb < L::kKB; ++kb) {
            uint8_t* blk = smem + L::kQOff + kb * L::kBlockBytes + R * 128;
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
    const uint32_t tS_base = tmem;           // S, and P over its first 64 columns
    const uint32_t tO_base = tmem + 128u;    // O

    if (warp == kDtcProducerWarp) {
        // ================= TMA producer =================
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            mbar_arrive_expect_tx(bar_q_full, static_cast<uint32_t>(L::kKB * R * 128));
            for (int kb = 0; kb < L::kKB; ++kb)
                tma_load_3d(sQ + kb * L::kBlockBytes, &tm_q, bar_q_full, kb * 64, static_cast<int>(group_row0), 0);
            int issued = 0;
            for (int t = 0; t < 2 * n_tiles; ++t) {
                const int s = t & 1;                         // K in slot 0, V in slot 1
                const uint32_t round = static_cast<uint32_t>(t >> 1);
                if (!mbar_wait(bar_kv_empty(s), (round & 1u) ^ 1u, abort_flag, &g_attn_err, kDevErrTimeout)) break;
                mbar_arrive_expect_tx(bar_kv_full(s), L::kTileBytes);
                const CUtensorMap* map = s ? &tm_v : &tm_k;
                const uint32_t dst = sKV + s * L::kTileBytes;
                for (int hh = 0; hh < 2; ++hh) {           // two 64-row boxes per 128-row tile
                    // a box wholly past this split's rows re-reads the last valid one (masked / zeroed)
                    const int key0 = min(k_begin + static_cast<int>(round) * kDtcBN + hh * 64, (k_end - 1) & ~63);
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
                    for (int kb = 0; kb < L::kKB; ++kb)
                        tma_load_3d(dst + kb * L::kBlockBytes + hh * 64 * 128, map, bar_kv_full(s), kb * 64, row, outer);
                }
                issued = t + 1;
            }
            if (issued < 2 * n_tiles) {
                for (int t = max(0, issued - 2); t < issued; ++t) {
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(bar_kv_full(t & 1), static_cast<uint32_t>(t >> 1) & 1u) &&
                           global_timer_ns() - t0 < 100000000ull) {
                    }
                }
                const uint64_t t0 = global_timer_ns();
                while (!mbar_try_wait(bar_q_full, 0) && global_timer_ns() - t0 < 100000000ull) {
                }
            }
        }
        __syncwarp();
    } else if (warp == kDtcMmaWarp) {
        // ================= MMA issuer (one lane issues; the warp clears stale V rows) =================
        constexpr uint32_t kIdescQK = umma_idesc_bf16_f32(128, kDtcBN, false);
        constexpr uint32_t kIdescPV = umma_idesc_bf16_f32(128, D, true);
        const uint64_t dQ = umma_sdesc_sw128(sQ, 16, 1024);
        const uint64_t dK = umma_sdesc_sw128(sKV, 16, 1024);
        const uint64_t dV = umma_sdesc_sw128(sKV + L::kTileBytes, L::kBlockBytes, 1024);
        bool ok = mbar_wait(bar_q_full, 0, abort_flag, &g_attn_err, kDevErrTimeout);
        for (int j = 0; j < n_tiles && ok; ++j) {
            const uint32_t par = static_cast<uint32_t>(j) & 1u;
            // S(j) = Q K_j^T (the TMEM it writes held P(j-1), consumed by the O += P V issued before)
            ok = mbar_wait(bar_kv_full(0), par, abort_flag, &g_attn_err, kDevErrTimeout);
            if (!ok) break;
            tc_fence_after_sync();
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = static_cast<uint64_t>(((kk >> 2) * L::kBlockBytes + (kk & 3) * 32) >> 4);
                    umma_ss(tS_base, dQ + off, dK + off, kIdescQK, kk > 0 ? 1u : 0u);
                }
                umma_commit(bar_s_full);
                umma_commit(bar_kv_empty(0));
            }
            __syncwarp();
            // O += P(j) V_j
            ok = mbar_wait(bar_kv_full(1), par, abort_flag, &g_attn_err, kDevErrTimeout) &&
                 mbar_wait(bar_p_full, par, abort_flag, &g_attn_err, kDevErrTimeout);
            if (!ok) break;
            // V rows past this split's last row may hold anything (NaN included) and P is 0
            // there, but 0 * NaN is NaN: clear them before the tensor cores read the tile
            const int valid = k_end - (k_begin + j * kDtcBN);
            if (valid < kDtcBN) {
                for (int kb = 0; kb < L::kKB; ++kb) {
                    uint8_t* blk = smem + L::kKVOff + L::kTileBytes + kb * L::kBlockBytes + valid * 128;
                    for (int i = lane * 16; i < (kDtcBN - valid) * 128; i += 32 * 16)
                        *reinterpret_cast<uint4*>(blk + i) = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();
            }
            __syncwarp();
            tc_fence_after_sync();
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < kDtcBN / 16; ++kk)
                    umma_ts(tO_base, tS_base + kk * 8, dV + static_cast<uint64_t>((kk * 2048) >> 4), kIdescPV,
                            (j > 0 || kk > 0) ? 1u : 0u);
                umma_commit(bar_kv_empty(1));
            }
            __syncwarp();
        }
        if (lane == 0) {
            umma_commit(bar_o_done);
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
        const uint32_t tS = tS_base + lane_off;
        const uint32_t tO = tO_base + lane_off;
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
            ok = mbar_wait(bar_s_full, static_cast<uint32_t>(j) & 1u, abort_flag, &g_attn_err, kDevErrTimeout);
            if (!ok) break;
            tc_fence_after_sync();
            if (idle_warp) {
                tc_fence_before_sync();
                mbar_arrive(bar_p_full);
                continue;
            }
            const int key0 = k_begin + j * kDtcBN;
            const bool masked = key0 + kDtcBN > lim_lo;
            // pass 1: the row max of this tile
            float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll 1
            for (int c = 0; c < kDtcBN; c += 32) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tS + c, v);
                tmem_wait_ld();
                reg_fence<32>(v);
                if (masked) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (key0 + c + i >= lim) v[i] = __float_as_uint(-INFINITY);
                }
#pragma unroll
                for (int i = 0; i < 32; i += 8) {
                    mx0 = fmax3(mx0, __uint_as_float(v[i]), __uint_as_float(v[i + 1]));
                    mx1 = fmax3(mx1, __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
                    mx2 = fmax3(mx2, __uint_as_float(v[i + 4]), __uint_as_float(v[i + 5]));
                    mx3 = fmax3(mx3, __uint_as_float(v[i + 6]), __uint_as_float(v[i + 7]));
                }
            }
            const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
            float factor = 1.0f;
            if (m_tile > m_run + kDtcRescaleLog2) {
                factor = (m_run == -INFINITY) ? 0.0f : ex2_approx(m_run - m_tile);
                m_run = m_tile;
                l_run *= factor;
                l_exact *= factor;
            }
            // O holds the sum over tiles < j (S(j) was issued after O += P(j-1) V_{j-1})
            if (j > 0 && __any_sync(0xffffffffu, factor != 1.0f)) {
                const uint64_t f2 = f2_pack(factor, factor);
#pragma unroll 1
                for (int c = 0; c < D; c += 32) {
                    uint32_t o[32];
                    tmem_ld_32x32b_x32(tO + c, o);
                    tmem_wait_ld();
                    reg_fence<32>(o);
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        float a0, a1;
                        f2_unpack(f2_mul(f2_pack(__uint_as_float(o[i]), __uint_as_float(o[i + 1])), f2), a0, a1);
                        o[i] = __float_as_uint(a0);
                        o[i + 1] = __float_as_uint(a1);
                    }
                    tmem_st_32x32b_x32(tO + c, o);
                }
                tmem_wait_st();
            }
            // pass 2: exponentials, row sum, P (bf16) over the S columns already read
            const float m_sub = (m_run == -INFINITY) ? 0.0f : m_run;
            const uint64_t negm2 = f2_pack(-m_sub, -m_sub);
            uint64_t acc_r = 0ull, acc_e = 0ull;
#pragma unroll 1
            for (int c = 0; c < kDtcBN; c += 32) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tS + c, v);
                tmem_wait_ld();
                reg_fence<32>(v);
                if (masked) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (key0 + c + i >= lim) v[i] = __float_as_uint(-INFINITY);
                }
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const uint64_t t =
                        f2_fma(f2_pack(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])), sl2x2, negm2);
                    float t0, t1;
                    f2_unpack(t, t0, t1);
                    const float e0 = ex2_approx(t0), e1 = ex2_approx(t1);
                    pk[i] = pack_bf16x2(e0, e1);
                    acc_e = f2_add(acc_e, f2_pack(e0, e1));
                    acc_r = f2_add(acc_r, bf16x2_to_f2(pk[i]));   // P as the MMA sees it
                }
                tmem_st_32x32b_x16(tS + c / 2, pk);
            }
            tmem_wait_st();
            tc_fence_before_sync();
            mbar_arrive(bar_p_full);
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
        float* dst = p.o_part + prow * D;
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
            uint32_t o[32];
            if (have_o) {
                tmem_ld_32x32b_x32(tO + c, o);
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
