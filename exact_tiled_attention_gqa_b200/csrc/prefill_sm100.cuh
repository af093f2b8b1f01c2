// prefill_sm100.cuh -- exact tiled GQA prefill on the sm_100a tensor cores.
//
// What it computes: O = softmax(scale * Q K^T + bottom-right causal mask) V
// and LSE per row, for Q [B,Hq,Lq,D], K/V [B,Hkv,Lk,D] (bf16), exactly, with
// an online softmax so the score table only ever exists one 128x128 tile at a
// time in tensor memory.  Sources: the SDPA / FlashAttention selection guide
// ("eager attention memory": tile the table, keep a max and a sum per row;
// "is_causal mask alignment": bottom-right alignment, query i sees key j iff
// j <= i + Lk - Lq; "long inputs": a block kernel skips fully masked blocks)
// and the NVIDIA attention page ("Parameter one: group size": G query heads
// share one KV head).
//
// Work unit: one batch b, one KV head g, and NQ*P consecutive query
// positions, as NQ "Q tiles" of M = 128 rows (NQ = 2 for D <= 128; NQ = 1 for
// D = 256, whose O accumulator alone takes 256 TMEM columns).  A Q tile packs the G query
// heads of the group with P = 128 / G positions each (row r = head r / P,
// position p0 + r % P), so every K/V tile staged in shared memory feeds all
// G heads of the group and both Q tiles.
//
// Persistent CTAs (NQ = 2): one CTA per SM takes unit after unit from an
// atomic counter, in the unit order of prefill_unit (heaviest first within a
// group), so the SMs stay balanced whatever the causal mix.  The producer
// loads the next unit's Q as soon as the last Q K^T of the current unit has
// read the Q tiles, and its first K/V tiles as ring entries free up, so a
// unit's start (Q and K_0 in flight, the first Q K^T) overlaps the previous
// unit's last P.V and epilogue.  An NQ = 1 CTA takes a single unit.
//
// Roles for NQ = 2 (384 threads = 3 warpgroups; for NQ = 1 the second softmax
// warpgroup is absent, warps 4 and 5 are producer and MMA issuer, 256 threads,
// and no registers are exchanged):
//   warps 0-3  softmax warpgroup for Q tile 0 (thread = TMEM lane = row)
//   warps 4-7  softmax warpgroup for Q tile 1
//   warp  8    TMA producer: per unit the Q tiles, then K_j, V_j into a ring of stages
//   warp  9    TMEM allocator and single-thread tcgen05.mma issuer
//   warps 10-11 idle
// The block launches at 168 registers per thread (3 warps per SM sub-partition
// x 168 x 32 = 16128 of its 16384).  The third warpgroup then gives registers
// back (setmaxnreg.dec to 104) and the softmax warpgroups take them
// (setmaxnreg.inc to 200): 2 x 200 + 104 = 3 x 168, so the exchange balances
// exactly and neither side waits.
//
// TMEM (512 columns): two S buffers at [0,128) and [128,256), then O.  For
// NQ = 2 buffer q holds S_q and O_q sits at [256 + D q, 256 + D q + D).  For
// NQ = 1 (D = 256) the two buffers alternate between key tiles (S(j) in buffer
// j mod 2) and O takes [256, 512).  P (bf16, two per column) overwrites the
// first 64 columns of its S buffer once the softmax has read S, and feeds
// O += P V_j as the TMEM A operand -- except at D = 64, where O0 and O1 end at
// column 384 and P_q gets columns of its own (P0 at 384, P1 at 448): there the
// softmax signals s_free_q once S_q(j) is in registers, S_q(j+1) = Q_q K_{j+1}^T
// is issued before O_q += P_q(j) V_j, and pv_done_q (committed after each P.V)
// tells the softmax when it may overwrite P_q or rescale O_q.
//
// Per key tile j the MMA thread issues, in order:
//   O0 += P0(j) V_j ; S0(j+1) = Q0 K_{j+1}^T ; O1 += P1(j) V_j ; S1(j+1) = Q1 K_{j+1}^T
// so the tensor cores work on one Q tile while the other's softmax runs.  The
// softmax hands P over in two halves (keys 0-63, then 64-127), and each half of
// O_q += P_q V_j is issued as soon as its half is in TMEM.
// A commit after S_q(j+1) also covers O_q += P_q(j) V_j, so when the softmax
// sees S_q(j+1) its O_q is settled and may be rescaled in place (with P in its
// own columns, D = 64, the softmax waits on pv_done_q instead).
//
// NQ = 1 (D = 256): one Q tile, so the overlap comes from the second S buffer:
//   S(0) ; S(1) ; then per j:  O += P(j) V_j ; S(j+2) = Q K_{j+2}^T
// The tensor cores compute S(j+1) while the softmax works on S(j).  Here the
// commit after S(j+1) does not cover O += P(j-1) V_{j-1}, so each P.V gets its
// own commit (o_ready) and the softmax waits on it only when it rescales O.
// The K/V ring holds half tiles (128 keys x 128 columns, 32 KB): K and V each
// arrive in two halves, in the order the MMAs use them (K0 K1 V0 K2 V1 ...),
// and the P.V product is issued as two N = 128 halves of O.
//
// The exponentials run on the MUFU unit (ex2.approx).  Scale-and-subtract,
// sums and O rescales use packed f32x2 instructions, maxima a 3-input max.
//
// Online softmax, in the log2 domain (x2 = x * scale * log2 e): per row a
// running max m and sum l.  The max used for the exponentials is only raised
// when a tile's max exceeds it by more than kRescaleLog2 (= 8, a factor 256);
// otherwise exponentials up to 2^8 are accumulated as they are.  The result
// is the same exact quantity -- O = sum_j 2^(s2_j - m) v_j / sum_j 2^(s2_j - m)
// holds for any m -- and the O rescale in TMEM is skipped on most tiles.
#pragma once

#include "ptx_sm100.cuh"
#include "device_error.cuh"
#include "ring_order.cuh"

namespace attn {

template <int NQ>
__host__ __device__ constexpr int prefill_threads() { return 32 * (4 * NQ + 4); }
__host__ __device__ constexpr int prefill_nq(int D) { return D == 256 ? 1 : 2; }
constexpr int kPrefillLaunchRegs = 168;    // must equal the compiled register count (checked by the build)
constexpr int kSoftmaxRegs = 200;
constexpr int kControlRegs = 104;
static_assert(2 * kSoftmaxRegs + kControlRegs == 3 * kPrefillLaunchRegs, "register exchange must balance");
constexpr int kBM = 128;               // rows per Q tile (MMA M)
constexpr int kBN = 128;               // keys per K/V tile
constexpr float kRescaleLog2 = 8.0f;
constexpr int kPrefillSplitParts = 4;  // runs of key tiles a key-split unit is cut into

template <int D>
struct PrefillSmem {
    static constexpr int kKB = D / 64;                    // 128-byte column blocks per row
    static constexpr int kQTileBytes = kBM * D * 2;      // one Q tile
    static constexpr int kKVTileBytes = kBN * D * 2;     // one K or V tile
    static constexpr int kBlockBytes = 128 * 128;        // one 128-row x 128-byte block
    static constexpr int kNQ = prefill_nq(D);
    // NQ = 2 CTAs are persistent and take work units from a counter; an NQ = 1
    // CTA takes one unit (its shared memory has no room for the O staging block)
    static constexpr bool kPersistent = (kNQ == 2);
    // D = 64: S0 | S1 | O0 | O1 take 384 TMEM columns, so P gets columns of its
    // own (P0 at 384, P1 at 448) instead of overwriting S; see the file comment
    static constexpr bool kSplitP = (D == 64);
    // ring entries: whole K or V tiles, or half tiles (32 KB each) for D = 256
    static constexpr int kItemsPerTile = (D == 256) ? 2 : 1;
    static constexpr int kItemBytes = kKVTileBytes / kItemsPerTile;
    static constexpr int kItemKB = kKB / kItemsPerTile;   // 128-byte column blocks per entry
    static constexpr int kStages = (D == 256) ? 5 : (D == 128) ? 4 : 8;
    static constexpr int kQOff = 0;
    static constexpr int kKVOff = kNQ * kQTileBytes;
    // O staging for the epilogue, one 64-column block per softmax warpgroup
    // (persistent CTAs: the Q tiles may already hold the next unit's queries)
    static constexpr int kStgOff = kKVOff + kStages * kItemBytes;
    static constexpr int kBarOff = kStgOff + (kPersistent ? kNQ * kBlockBytes : 0);
    // barriers: q_full, kv_full[S], kv_empty[S], s_full[2], p_half[2], p_full[2], o_done[2], drain,
    //           q_empty, unit_full[2], unit_empty[2], s_free[2], pv_done[2]
    static constexpr int kNumBars = 1 + 2 * kStages + 2 + 2 + 2 + 2 + 1 + 1 + 2 + 2 + 2 + 2;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;   // tmem base, abort flag, two unit slots (int each)
    static constexpr int kTagOff = kMiscOff + 16;             // debug builds: ring entry -> item index
    static constexpr int kBytes = kTagOff + 4 * kStages;
    static constexpr int kAlloc = kBytes + 1024;              // slack to align the base to 1 KiB
    static_assert(kAlloc <= 232448, "dynamic shared memory per CTA");
    static_assert(kStgOff % 1024 == 0, "swizzled TMA blocks start on 1 KiB");
};

// Scheduling counters of persistent launches: slot i is {next unit, CTAs
// done}.  Each launch takes a slot from the host; the last of its CTAs to
// finish puts both counters back to zero, so a slot is ready for its next
// launch without a memset.  Ordinary launches take the first
// kPrefillEagerSlots slots in turn; launches recorded into a CUDA graph take
// the next kPrefillCaptureSlots in turn (a graph keeps its slot for every
// replay, so the two kinds never share one).
constexpr int kPrefillEagerSlots = 256;
constexpr int kPrefillCaptureSlots = 1024;
constexpr int kPrefillSchedSlots = kPrefillEagerSlots + kPrefillCaptureSlots;
__device__ int g_prefill_sched[2 * kPrefillSchedSlots];

struct PrefillParams {
    void* out;          // [B,Hq,Lq,D] bf16
    float* lse;         // [B,Hq,Lq] or nullptr
    int B, Hq, Hkv, Lq, Lk;
    int G, P;           // group size, positions per Q tile (P = 128 / G)
    int n_mblk;         // ceil(Lq / (NQ P))
    int n_units;        // B * Hkv * n_mblk
    int band;           // (b, KV head) groups per band of the unit order (see prefill_unit)
    int is_causal;
    float scale_log2;   // scale * log2(e)
    int* sched;         // persistent launches: this launch's two counters (zero at launch)
    // Key-split tail (persistent launches with a workspace): units n_full .. of the
    // order are each cut into n_parts runs of key tiles; work items n_full + t
    // (t = split unit * n_parts + part) write fp32 partials to part_o
    // [t][NQ * 128 rows][D] and log2-sum-exps to part_l [t][NQ * 128], merged by
    // attn_prefill_merge_kernel.  n_units counts items; n_full == n_units: no split.
    int n_full, n_parts;
    float* part_o;
    float* part_l;
};

// One work item: batch b, KV head g, the NQ * P query positions from p_begin,
// and the key tiles kt0 .. kt0 + n_kt - 1 it covers (all the latest position
// sees, unless part >= 0: a run of them, partial results to item slot `part`).
struct PrefillUnit {
    int b, g, p_begin, n_kt, kt0, part;
};

// Unit `idx` of a launch.  Units run band by band: a band is `band`
// consecutive (b, KV head) groups (the last band may hold fewer), as many as
// keep their K/V in about half the L2, so the units that run at the same time
// find their K/V there.  Within a band the heaviest (latest) position blocks
// of all its groups come first: the longest-first order that keeps the tail of
// a causal launch short, since the last units handed out are the lightest.
// Items past n_full are the parts of the units n_full .. of this order (the
// lightest, handed out last), each a contiguous run of about n_kt / n_parts key tiles.
// kSplit = false: a launch without a key split (every item a whole unit).
template <int NQ, bool kSplit = true>
__host__ __device__ __forceinline__ PrefillUnit prefill_unit(const PrefillParams& p, int idx) {
    int part = -1, kpart = 0;
    if (kSplit && idx >= p.n_full) {
        part = idx - p.n_full;
        kpart = part % p.n_parts;
        idx = p.n_full + part / p.n_parts;
    }
    const int n_bh = p.B * p.Hkv;
    const int per_band = p.band * p.n_mblk;
    const int k = idx / per_band;
    const int g0 = k * p.band;
    const int bs = (p.band < n_bh - g0) ? p.band : n_bh - g0;   // groups in this band
    const int local = idx - k * per_band;
    const int mblk = p.n_mblk - 1 - local / bs;
    const int bh = g0 + local % bs;
    PrefillUnit u;
    u.b = bh / p.Hkv;
    u.g = bh % p.Hkv;
    u.p_begin = mblk * NQ * p.P;
    const long off = static_cast<long>(p.Lk) - static_cast<long>(p.Lq);
    const int p_end = (u.p_begin + NQ * p.P < p.Lq) ? u.p_begin + NQ * p.P : p.Lq;
    const long lk1 = static_cast<long>(p.Lk) - 1;
    const long last_key = p.is_causal ? ((p_end - 1 + off < lk1) ? p_end - 1 + off : lk1) : lk1;
    u.n_kt = last_key < 0 ? 0 : static_cast<int>(last_key / kBN) + 1;
    u.kt0 = 0;
    u.part = part;
    if (kSplit && part >= 0) {
        const int total = u.n_kt;
        u.kt0 = kpart * total / p.n_parts;
        u.n_kt = (kpart + 1) * total / p.n_parts - u.kt0;
    }
    return u;
}

// kSplit: the launch has a key-split tail (items past p.n_full write partials);
// launches without one use the kSplit = false build of the kernel.
template <int D, int NQ, bool kSplit>
__global__ void __launch_bounds__(prefill_threads<NQ>(), 1)
    attn_prefill_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                              const __grid_constant__ CUtensorMap tm_k,
                              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                              const PrefillParams p) {
    if constexpr (kSplit) grid_dep_release();   // the merge launch may be scheduled now
    using L = PrefillSmem<D>;
    static_assert(L::kNQ == NQ, "Q tiles per CTA follow from D");
    constexpr bool kPersistent = L::kPersistent;
    constexpr bool kSplitP = L::kSplitP;
    constexpr int kThreads = prefill_threads<NQ>();
    constexpr int kProducerWarp = 4 * NQ;
    constexpr int kMmaWarp = 4 * NQ + 1;
    constexpr int kUnitReaders = 1 + 4 * NQ;   // the MMA thread and every softmax warp
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_base);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int P = p.P;
    const int rows_used = p.G * P;

    // ---- shared memory map ----
    const uint32_t sQ = base + L::kQOff;
    const uint32_t sKV = base + L::kKVOff;
    const uint32_t bar0 = base + L::kBarOff;
    const uint32_t bar_q_full = bar0;
    auto bar_kv_full = [&](int s) { return bar0 + 8u * (1 + s); };
    auto bar_kv_empty = [&](int s) { return bar0 + 8u * (1 + L::kStages + s); };
    auto bar_s_full = [&](int q) { return bar0 + 8u * (1 + 2 * L::kStages + q); };
    auto bar_p_half = [&](int q) { return bar0 + 8u * (3 + 2 * L::kStages + q); };
    auto bar_p_full = [&](int q) { return bar0 + 8u * (5 + 2 * L::kStages + q); };
    auto bar_o_done = [&](int q) { return bar0 + 8u * (7 + 2 * L::kStages + q); };
    const uint32_t bar_drain = bar0 + 8u * (9 + 2 * L::kStages);
    const uint32_t bar_q_empty = bar0 + 8u * (10 + 2 * L::kStages);
    auto bar_unit_full = [&](int s) { return bar0 + 8u * (11 + 2 * L::kStages + s); };
    auto bar_unit_empty = [&](int s) { return bar0 + 8u * (13 + 2 * L::kStages + s); };
    // (split P only) the softmax has read S_q into registers / O_q += P_q V has completed
    auto bar_s_free = [&](int q) { return bar0 + 8u * (15 + 2 * L::kStages + q); };
    auto bar_pv_done = [&](int q) { return bar0 + 8u * (17 + 2 * L::kStages + q); };
    // P_q (or, for NQ = 1, S buffer q's P) is handed over in two halves: keys 0-63 on p_half, 64-127 on p_full
    auto bar_p_part = [&](int q, int half) { return half == 0 ? bar_p_half(q) : bar_p_full(q); };
    uint32_t* tmem_base_ptr = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
    volatile int* unit_slot = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 8);
    // (debug builds) the ring position the producer put in each entry, checked by the MMA thread
    volatile int* ring_tag = reinterpret_cast<volatile int*>(smem + L::kTagOff);

    if (threadIdx.x == 0) {
        mbar_init(bar_q_full, 1);
        mbar_init(bar_q_empty, 1);
        for (int s = 0; s < L::kStages; ++s) {
            mbar_init(bar_kv_full(s), 1);
            mbar_init(bar_kv_empty(s), 1);
        }
        for (int q = 0; q < 2; ++q) {   // per Q tile (NQ = 2) or per S buffer (NQ = 1)
            mbar_init(bar_s_full(q), 1);
            mbar_init(bar_p_half(q), 4);   // one arrival per softmax warp
            mbar_init(bar_p_full(q), 4);
            mbar_init(bar_o_done(q), 1);
            mbar_init(bar_unit_full(q), 1);
            mbar_init(bar_unit_empty(q), kUnitReaders);
            mbar_init(bar_s_free(q), 4);   // one arrival per softmax warp
            mbar_init(bar_pv_done(q), 1);
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // Q rows the TMA box does not cover (G does not divide 128) must hold
    // finite values: zero them through the generic proxy, then hand them over.
    // No TMA load writes them, so this holds for every unit.
    if (rows_used < kBM) {
        const int pad_bytes_per_block = (kBM - rows_used) * 128;
        for (int q = 0; q < NQ; ++q)
            for (int kb = 0; kb < L::kKB; ++kb) {
                uint8_t* blk = smem + L::kQOff + q * L::kQTileBytes + kb * L::kBlockBytes + rows_used * 128;
                for (int i = threadIdx.x * 16; i < pad_bytes_per_block; i += kThreads * 16)
                    *reinterpret_cast<uint4*>(blk + i) = make_uint4(0, 0, 0, 0);
            }
        fence_proxy_async_smem();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(tmem_base_ptr), 512);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_base_ptr;

    // Work units reach the CTA through two shared-memory slots: the producer
    // writes unit k (or -1: no more) into slot k % 2 and arrives on unit_full;
    // the MMA thread and the softmax warps read it and arrive on unit_empty.
    // The first unit is blockIdx.x; a persistent CTA then takes gridDim.x + c,
    // c from the launch's counter, until the units run out.  Barrier phases
    // and ring positions run on across units.

    if (warp >= kProducerWarp) {
      if constexpr (NQ == 2) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kControlRegs));
      if (warp == kProducerWarp) {
        // ================= TMA producer =================
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_o);
            const uint32_t q_bytes = static_cast<uint32_t>(NQ * L::kKB * rows_used * 128);
            int idx = blockIdx.x;
            int t = 0;    // ring entries issued, over all units
            int nu = 0;   // units with at least one key tile (Q loads)
            bool ok = true;
            for (int k = 0;; ++k) {
                const int s = k & 1;
                ok = mbar_wait(bar_unit_empty(s), static_cast<uint32_t>((k >> 1) & 1) ^ 1u, abort_flag, &g_attn_err,
                               kDevErrTimeout);
                if (!ok) break;
                const bool have = idx < p.n_units;
                unit_slot[s] = have ? idx : -1;
                mbar_arrive(bar_unit_full(s));
                if (!have) break;
                const PrefillUnit u = prefill_unit<NQ, kSplit>(p, idx);
                ATTN_CHECK(idx >= 0 && u.b >= 0 && u.b < p.B && u.g >= 0 && u.g < p.Hkv && u.p_begin >= 0 &&
                           u.p_begin < p.Lq && u.p_begin % (NQ * P) == 0 && u.n_kt >= 0 && u.kt0 >= 0 &&
                           u.kt0 + u.n_kt <= (p.Lk + kBN - 1) / kBN);
                // The next unit is taken once this one's loads are all issued (about
                // two key tiles before its MMAs end), not earlier: a CTA that claimed
                // its next unit at the start of a long one would hold it back from SMs
                // that run dry at the end of the launch.
                auto next_unit = [&]() {
                    return kPersistent ? static_cast<int>(gridDim.x) + atomicAdd(p.sched, 1) : p.n_units;
                };
                if (u.n_kt == 0) {
                    idx = next_unit();
                    continue;
                }
                if (nu > 0) {   // the previous unit's last Q K^T has read the Q tiles
                    ok = mbar_wait(bar_q_empty, static_cast<uint32_t>(nu - 1) & 1u, abort_flag, &g_attn_err,
                                   kDevErrTimeout);
                    if (!ok) break;
                }
                const int q_head0 = u.b * p.Hq + u.g * p.G;
                ATTN_CHECK(q_head0 >= 0 && q_head0 + p.G <= p.B * p.Hq);
                mbar_arrive_expect_tx(bar_q_full, q_bytes);
                for (int q = 0; q < NQ; ++q)
                    for (int kb = 0; kb < L::kKB; ++kb)
                        tma_load_3d(sQ + q * L::kQTileBytes + kb * L::kBlockBytes, &tm_q, bar_q_full, kb * 64,
                                    u.p_begin + q * P, q_head0);
                ++nu;
                const int kv_row = u.b * p.Hkv + u.g;
                const int n_items = 2 * u.n_kt * L::kItemsPerTile;
                for (int i = 0; i < n_items; ++i) {
                    const int st = t % L::kStages;
                    const uint32_t round = static_cast<uint32_t>(t / L::kStages);
                    ok = mbar_wait(bar_kv_empty(st), (round & 1u) ^ 1u, abort_flag, &g_attn_err, kDevErrTimeout);
                    if (!ok) break;
                    bool is_v;
                    int j;
                    ring_tile<NQ>(i / L::kItemsPerTile, u.n_kt, is_v, j);
                    const int kb0 = (i % L::kItemsPerTile) * L::kItemKB;
                    ATTN_CHECK(j >= 0 && j < u.n_kt && kv_row >= 0 && kv_row < p.B * p.Hkv &&
                               (kb0 + L::kItemKB) * 64 <= D);
                    if (ATTN_DEBUG_BOUNDS) ring_tag[st] = t;
                    mbar_arrive_expect_tx(bar_kv_full(st), L::kItemBytes);
                    const CUtensorMap* map = is_v ? &tm_v : &tm_k;
                    for (int kb = 0; kb < L::kItemKB; ++kb)
                        tma_load_3d(sKV + st * L::kItemBytes + kb * L::kBlockBytes, map, bar_kv_full(st),
                                    (kb0 + kb) * 64, (u.kt0 + j) * kBN, kv_row);
                    ++t;
                }
                if (!ok) break;
                idx = next_unit();
            }
            if (!ok) {
                // Unwinding: let the copies already issued land before the CTA exits.
                for (int t2 = max(0, t - L::kStages); t2 < t; ++t2) {
                    const int st = t2 % L::kStages;
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(bar_kv_full(st), static_cast<uint32_t>(t2 / L::kStages) & 1u) &&
                           global_timer_ns() - t0 < 100000000ull) {
                    }
                }
                if (nu > 0) {
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(bar_q_full, static_cast<uint32_t>(nu - 1) & 1u) &&
                           global_timer_ns() - t0 < 100000000ull) {
                    }
                }
            }
            if constexpr (kPersistent) {
                // This CTA takes no more units.  The last CTA to get here leaves
                // both counters at zero for the slot's next launch.  Every CTA
                // that ran to the end made one claim per unit it ran after its
                // first, plus one that came back empty, so a launch that had its
                // counters to itself ends with exactly n_units claims; any other
                // count means another launch used the same slot at the same time
                // (units may have been skipped), which is flagged.
                __threadfence();
                if (atomicAdd(p.sched + 1, 1) == static_cast<int>(gridDim.x) - 1) {
                    const int claims = atomicExch(p.sched, 0);
                    atomicExch(p.sched + 1, 0);
                    if (ok && claims != p.n_units && !(atomicOr(&g_attn_err, 0u) & kDevErrTimeout))
                        atomicOr(&g_attn_err, kDevErrSched);   // (a timed-out CTA stops claiming early)
                }
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ================= MMA issuer =================
        if (lane == 0) {
            constexpr uint32_t kIdescQK = umma_idesc_bf16_f32(kBM, kBN, false);
            constexpr uint32_t kIdescPV = umma_idesc_bf16_f32(kBM, D, true);
            const uint32_t tS[2] = {tmem + 0u, tmem + 128u};
            const uint32_t tO[2] = {tmem + 256u, tmem + 256u + D};
            const uint32_t tP[2] = {kSplitP ? tmem + 384u : tS[0], kSplitP ? tmem + 448u : tS[1]};
            int tb = 0;      // ring entries of earlier units
            int tiles = 0;   // key tiles of earlier units (phases of the per-tile barriers)
            int nu = 0;      // earlier units with key tiles
            // Ring positions in unsigned arithmetic: this thread's instruction latency
            // sits on the S -> P -> MMA chain, and signed % and / with a runtime base
            // cost about 60 cycles per key tile (measured).
            auto slot_of = [&](int t) { return static_cast<int>(static_cast<unsigned>(tb + t) % L::kStages); };
            auto par_of = [&](int t) { return (static_cast<unsigned>(tb + t) / L::kStages) & 1u; };
            // (debug builds) the entry holds the item this thread expects there
            auto check_item = [&](int t) { ATTN_CHECK(ring_tag[slot_of(t)] == tb + t); };
            // Shared-memory descriptors are built once; a k-step only moves the
            // start-address field (bits 0-13, address >> 4), so each MMA issue
            // costs one 64-bit add.
            const uint64_t dQ[2] = {umma_sdesc_sw128(sQ, 16, 1024), umma_sdesc_sw128(sQ + L::kQTileBytes, 16, 1024)};
            const uint64_t dK0 = umma_sdesc_sw128(sKV, 16, 1024);
            const uint64_t dV0 = umma_sdesc_sw128(sKV, L::kBlockBytes, 1024);
            constexpr uint64_t kSlotStep = L::kItemBytes >> 4;
            // S_q = Q_q K^T : M=128, N=128, K=D in steps of 16 (32 bytes)
            auto issue_qk = [&](int q, int t) {
                const uint64_t b0 = dK0 + static_cast<uint64_t>(slot_of(t)) * kSlotStep;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t koff = static_cast<uint64_t>(((kk >> 2) * L::kBlockBytes + (kk & 3) * 32) >> 4);
                    umma_ss(tS[q], dQ[q] + koff, b0 + koff, kIdescQK, kk > 0 ? 1u : 0u);
                }
            };
            // O_q += P_q V : M=128, N=D, K=128 keys in steps of 16 (8 TMEM columns of P);
            // `half` 0 covers keys 0-63 (P columns 0-31), half 1 keys 64-127
            auto issue_pv = [&](int q, int t, bool acc, int half) {
                const uint64_t b0 = dV0 + static_cast<uint64_t>(slot_of(t)) * kSlotStep;
#pragma unroll
                for (int k4 = 0; k4 < kBN / 32; ++k4) {
                    const int kk = half * (kBN / 32) + k4;
                    umma_ts(tO[q], tP[q] + kk * 8, b0 + static_cast<uint64_t>((kk * 2048) >> 4), kIdescPV,
                            (acc || kk > 0) ? 1u : 0u);
                }
            };
            // both halves of O_q += P_q(j) V_j, each as soon as the softmax has released it
            auto pv_tile = [&](int q, int t, int j) {
                const uint32_t ph = static_cast<uint32_t>(tiles + j) & 1u;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    if (!mbar_wait(bar_p_part(q, half), ph, abort_flag, &g_attn_err, kDevErrTimeout)) return false;
                    tc_fence_after_sync();
                    issue_pv(q, t, half > 0 || j > 0, half);
                }
                return true;
            };
            bool ok = true;
            for (int k = 0; ok; ++k) {
                const int s = k & 1;
                ok = mbar_wait(bar_unit_full(s), static_cast<uint32_t>(k >> 1) & 1u, abort_flag, &g_attn_err,
                               kDevErrTimeout);
                if (!ok) break;
                const int idx = unit_slot[s];
                mbar_arrive(bar_unit_empty(s));
                if (idx < 0) break;
                const int n_kt = prefill_unit<NQ, kSplit>(p, idx).n_kt;
                if (n_kt == 0) continue;
                ok = mbar_wait(bar_q_full, static_cast<uint32_t>(nu) & 1u, abort_flag, &g_attn_err, kDevErrTimeout);
              if constexpr (kSplitP) {
                // P has TMEM columns of its own: S_q(j+1) = Q_q K_{j+1}^T is issued as soon
                // as the softmax has read S_q(j) into registers, and O_q += P_q(j) V_j once
                // P_q(j) is in TMEM, so the next tile's scores are ready when the softmax
                // finishes this one.  pv_done_q tells the softmax when P_q and O_q are free.
                if (ok) ok = mbar_wait(bar_kv_full(slot_of(0)), par_of(0), abort_flag, &g_attn_err, kDevErrTimeout);
                if (ok) check_item(0);
                if (ok) {
                    tc_fence_after_sync();
                    issue_qk(0, 0);
                    umma_commit(bar_s_full(0));
                    issue_qk(1, 0);
                    umma_commit(bar_s_full(1));
                    if (n_kt == 1) umma_commit(bar_q_empty);
                    umma_commit(bar_kv_empty(slot_of(0)));
                }
                for (int j = 0; j < n_kt && ok; ++j) {
                    const int tv = 2 * j + 1, tk = 2 * j + 2;
                    const bool last = (j + 1 == n_kt);
                    const uint32_t ph = static_cast<uint32_t>(tiles + j) & 1u;
                    ok = mbar_wait(bar_kv_full(slot_of(tv)), par_of(tv), abort_flag, &g_attn_err, kDevErrTimeout);
                    if (ok) check_item(tv);
                    if (ok && !last)
                        ok = mbar_wait(bar_kv_full(slot_of(tk)), par_of(tk), abort_flag, &g_attn_err, kDevErrTimeout);
                    if (ok && !last) check_item(tk);
                    if (ok && !last) {
                        ok = mbar_wait(bar_s_free(0), ph, abort_flag, &g_attn_err, kDevErrTimeout);
                        if (ok) {
                            tc_fence_after_sync();
                            issue_qk(0, tk);
                            umma_commit(bar_s_full(0));
                        }
                    }
                    ok = ok && pv_tile(0, tv, j);
                    if (!ok) break;
                    umma_commit(bar_pv_done(0));
                    if (!last) {
                        ok = mbar_wait(bar_s_free(1), ph, abort_flag, &g_attn_err, kDevErrTimeout);
                        if (!ok) break;
                        tc_fence_after_sync();
                        issue_qk(1, tk);
                        umma_commit(bar_s_full(1));
                        if (j + 2 == n_kt) umma_commit(bar_q_empty);   // the unit's last reads of Q
                        umma_commit(bar_kv_empty(slot_of(tk)));
                    }
                    ok = pv_tile(1, tv, j);
                    if (!ok) break;
                    umma_commit(bar_pv_done(1));
                    umma_commit(bar_kv_empty(slot_of(tv)));
                }
              } else if constexpr (NQ == 2) {
                if (ok) ok = mbar_wait(bar_kv_full(slot_of(0)), par_of(0), abort_flag, &g_attn_err, kDevErrTimeout);
                if (ok) check_item(0);
                if (ok) {
                    tc_fence_after_sync();
                    issue_qk(0, 0);
                    umma_commit(bar_s_full(0));
                    issue_qk(1, 0);
                    umma_commit(bar_s_full(1));
                    if (n_kt == 1) umma_commit(bar_q_empty);
                    umma_commit(bar_kv_empty(slot_of(0)));
                }
                for (int j = 0; j < n_kt && ok; ++j) {
                    const int tv = 2 * j + 1, tk = 2 * j + 2;
                    const bool last = (j + 1 == n_kt);
                    // operands first (normally long landed), so only the P waits sit on the chain
                    ok = mbar_wait(bar_kv_full(slot_of(tv)), par_of(tv), abort_flag, &g_attn_err, kDevErrTimeout);
                    if (ok) check_item(tv);
                    if (ok && !last)
                        ok = mbar_wait(bar_kv_full(slot_of(tk)), par_of(tk), abort_flag, &g_attn_err, kDevErrTimeout);
                    if (ok && !last) check_item(tk);
                    ok = ok && pv_tile(0, tv, j);
                    if (!ok) break;
                    if (last) umma_commit(bar_o_done(0));
                    if (!last) {
                        issue_qk(0, tk);
                        umma_commit(bar_s_full(0));
                    }
                    ok = pv_tile(1, tv, j);
                    if (!ok) break;
                    if (last) umma_commit(bar_o_done(1));
                    umma_commit(bar_kv_empty(slot_of(tv)));
                    if (!last) {
                        issue_qk(1, tk);
                        umma_commit(bar_s_full(1));
                        if (j + 2 == n_kt) umma_commit(bar_q_empty);   // the unit's last reads of Q
                        umma_commit(bar_kv_empty(slot_of(tk)));
                    }
                }
              } else if (ok) {
                // ---- one Q tile, S double-buffered (D = 256; one unit per CTA, so
                // ring positions and phases start at zero) ----
                constexpr uint32_t kIdescPVh = umma_idesc_bf16_f32(kBM, 128, true);
                const uint32_t tOq = tmem + 256u;
                auto wait_item = [&](int it) {
                    const bool got =
                        mbar_wait(bar_kv_full(slot_of(it)), par_of(it), abort_flag, &g_attn_err, kDevErrTimeout);
                    if (got) check_item(it);
                    return got;
                };
                // S(j) into buffer j % 2, K_j in two half entries (columns 0-127, 128-255)
                auto qk = [&](int j) {
                    const int it0 = L::kItemsPerTile * ring_pos_k<NQ>(j);
                    const uint32_t tSb = tS[j & 1];
                    for (int hh = 0; hh < 2; ++hh) {
                        if (!wait_item(it0 + hh)) return false;
                        tc_fence_after_sync();
                        const uint64_t b0 = dK0 + static_cast<uint64_t>(slot_of(it0 + hh)) * kSlotStep;
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const int kq = hh * 8 + kk;
                            const uint64_t koff =
                                static_cast<uint64_t>(((kk >> 2) * L::kBlockBytes + (kk & 3) * 32) >> 4);
                            const uint64_t qoff =
                                static_cast<uint64_t>(((kq >> 2) * L::kBlockBytes + (kq & 3) * 32) >> 4);
                            umma_ss(tSb, dQ[0] + qoff, b0 + koff, kIdescQK, kq > 0 ? 1u : 0u);
                        }
                        umma_commit(bar_kv_empty(slot_of(it0 + hh)));
                    }
                    umma_commit(bar_s_full(j & 1));
                    return true;
                };
                // O[:, 128 hv .. +128) += P(j)[:, keys of `half`] V_j^(hv)
                auto pv_part = [&](int j, int itv, int half) {
                    const uint32_t tSb = tS[j & 1];
#pragma unroll
                    for (int hv = 0; hv < 2; ++hv) {
                        const uint64_t b0 = dV0 + static_cast<uint64_t>(slot_of(itv + hv)) * kSlotStep;
#pragma unroll
                        for (int k4 = 0; k4 < kBN / 32; ++k4) {
                            const int kk = half * (kBN / 32) + k4;
                            umma_ts(tOq + 128u * hv, tSb + kk * 8, b0 + static_cast<uint64_t>((kk * 2048) >> 4),
                                    kIdescPVh, (j > 0 || kk > 0) ? 1u : 0u);
                        }
                    }
                };
                ok = qk(0);
                if (ok && n_kt > 1) ok = qk(1);
                for (int j = 0; j < n_kt && ok; ++j) {
                    const int buf = j & 1;
                    const uint32_t ph = static_cast<uint32_t>(j >> 1) & 1u;
                    const int itv = L::kItemsPerTile * ring_pos_v<NQ>(j, n_kt);
                    ok = wait_item(itv) && wait_item(itv + 1);
                    ok = ok && mbar_wait(bar_p_half(buf), ph, abort_flag, &g_attn_err, kDevErrTimeout);
                    if (!ok) break;
                    tc_fence_after_sync();
                    pv_part(j, itv, 0);
                    ok = mbar_wait(bar_p_full(buf), ph, abort_flag, &g_attn_err, kDevErrTimeout);
                    if (!ok) break;
                    tc_fence_after_sync();
                    pv_part(j, itv, 1);
                    umma_commit(bar_o_done(1));              // o_ready: O holds tiles 0..j
                    if (j + 1 == n_kt) umma_commit(bar_o_done(0));
                    umma_commit(bar_kv_empty(slot_of(itv)));
                    umma_commit(bar_kv_empty(slot_of(itv + 1)));
                    if (j + 2 < n_kt) ok = qk(j + 2);
                }
              }
                tb += 2 * n_kt * L::kItemsPerTile;
                tiles += n_kt;
                ++nu;
            }
            // Drain: no MMA may still be running when TMEM is released.
            umma_commit(bar_drain);
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(bar_drain, 0) && global_timer_ns() - t0 < 100000000ull) {
            }
        }
        __syncwarp();
      }
    } else {
        if constexpr (NQ == 2) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
        // ================= softmax warpgroups =================
        const int q = warp >> 2;                 // Q tile of this warpgroup
        const int r = threadIdx.x & 127;         // row = TMEM lane
        const int wg_bar = 1 + q;                // this warpgroup's named barrier
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS_q = tmem + (q ? 128u : 0u) + lane_off;
        const uint32_t tO = tmem + 256u + (q ? static_cast<uint32_t>(D) : 0u) + lane_off;
        const uint32_t tP_q = kSplitP ? tmem + (q ? 448u : 384u) + lane_off : tS_q;
        const int head_local = r / P;
        const long off = static_cast<long>(p.Lk) - static_cast<long>(p.Lq);
        const long lk1 = static_cast<long>(p.Lk) - 1;
        const float sl2 = p.scale_log2;
        int tiles = 0;   // key tiles of earlier units (barrier phases)
        int nu = 0;      // earlier units with key tiles (o_done phase)
        bool ok = true;
        for (int k = 0;; ++k) {
            const int s = k & 1;
            int idx = -1;
            if (ok) {
                ok = mbar_wait(bar_unit_full(s), static_cast<uint32_t>(k >> 1) & 1u, abort_flag, &g_attn_err,
                               kDevErrTimeout);
                if (ok) idx = unit_slot[s];
            }
            // The warpgroup decides together (its threads meet at named barriers
            // in the epilogue); the barrier also orders every lane's read of the
            // slot before the warp's release of it.
            if (named_bar_or(wg_bar, 128, !ok || idx < 0)) break;
            if (lane == 0) mbar_arrive(bar_unit_empty(s));
            const PrefillUnit u = prefill_unit<NQ, kSplit>(p, idx);
            const int n_kt = u.n_kt;
            const int pos = u.p_begin + q * P + (r % P);
            const bool row_valid = (r < rows_used) && (pos < p.Lq);
            const int h = u.g * p.G + head_local;
            // last visible key of this row, and the smallest such bound over the tile's rows
            const long bound = p.is_causal ? min(static_cast<long>(pos) + off, lk1) : lk1;
            const int tile_p0 = u.p_begin + q * P;
            const long tile_min_bound = p.is_causal ? min(static_cast<long>(tile_p0) + off, lk1) : lk1;

            float m_run = -INFINITY;   // running max used for the exponentials (log2 domain)
            float l_run = 0.0f;        // running sum normalising O (see the exponentials below)
            float l_exact = 0.0f;      // running sum of the unrounded exponentials (for the LSE)
            for (int j = 0; j < n_kt; ++j) {
                // S buffer of this tile, and the phase of its barriers
                const int buf = (NQ == 2) ? q : (j & 1);
                const uint32_t ph = static_cast<uint32_t>(NQ == 2 ? tiles + j : (j >> 1)) & 1u;
                const uint32_t tS = (NQ == 2) ? tS_q : tS_q + (static_cast<uint32_t>(j & 1) << 7);
                ok = mbar_wait(bar_s_full(buf), ph, abort_flag, &g_attn_err, kDevErrTimeout);
                if (!ok) break;
                tc_fence_after_sync();
                uint32_t sr[128];
                tmem_ld_32x32b_x32(tS + 0, sr + 0);
                tmem_ld_32x32b_x32(tS + 32, sr + 32);
                tmem_ld_32x32b_x32(tS + 64, sr + 64);
                tmem_ld_32x32b_x32(tS + 96, sr + 96);
                tmem_wait_ld();
                reg_fence<128>(sr);
                if constexpr (kSplitP) {   // S_q is in registers: the next Q K^T may overwrite it
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar_s_free(q));
                }
                // (split P) O_q += P_q(j-1) V_{j-1} must have completed before O_q is
                // rescaled or P_q(j) overwrites P_q(j-1)
                bool pv_prev_done = !kSplitP || j == 0;
                auto wait_pv_prev = [&]() {
                    if (pv_prev_done) return true;
                    pv_prev_done = true;
                    if (!mbar_wait(bar_pv_done(q), static_cast<uint32_t>(tiles + j - 1) & 1u, abort_flag,
                                   &g_attn_err, kDevErrTimeout))
                        return false;
                    tc_fence_after_sync();
                    return true;
                };
                float sv[kBN];
#pragma unroll
                for (int c = 0; c < kBN; ++c) sv[c] = __uint_as_float(sr[c]);
                const long key0 = static_cast<long>(u.kt0 + j) * kBN;
                ATTN_CHECK(key0 < p.Lk);
                const bool masked = key0 + kBN - 1 > tile_min_bound;
                if (masked) {
                    // diagonal or ragged tile: mask keys beyond this row's bound
#pragma unroll
                    for (int c = 0; c < kBN; ++c)
                        if (key0 + c > bound) sv[c] = -INFINITY;
                }
                float mx[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) mx[i] = fmax3(sv[i], sv[8 + i], sv[16 + i]);
#pragma unroll
                for (int c = 24; c < kBN - 8; c += 16)
#pragma unroll
                    for (int i = 0; i < 8; ++i) mx[i] = fmax3(mx[i], sv[c + i], sv[c + 8 + i]);
#pragma unroll
                for (int i = 0; i < 8; ++i) mx[i] = fmaxf(mx[i], sv[kBN - 8 + i]);
                const float tmax =
                    fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(fmax3(mx[3], mx[4], mx[5]), mx[6], mx[7]));
                const float m_tile = tmax * sl2;   // -inf stays -inf
                float factor = 1.0f;
                if (m_tile > m_run + kRescaleLog2) {
                    factor = (m_run == -INFINITY) ? 0.0f : ex2_approx(m_run - m_tile);
                    m_run = m_tile;
                    l_run *= factor;
                    l_exact *= factor;
                }
                // rescale O_q in TMEM if any row of this warp raised its max (O holds
                // the sum over tiles < j, settled: see the file comment)
                if (j > 0 && __any_sync(0xffffffffu, factor != 1.0f)) {
                    if (!wait_pv_prev()) {
                        ok = false;
                        break;
                    }
                    if constexpr (NQ == 1) {
                        // O += P(j-1) V_{j-1} must have landed (at most one P.V is outstanding)
                        if (!mbar_wait(bar_o_done(1), static_cast<uint32_t>(j - 1) & 1u, abort_flag, &g_attn_err,
                                       kDevErrTimeout)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after_sync();
                    }
                    const uint64_t f2 = f2_pack(factor, factor);
#pragma unroll 1
                    for (int c = 0; c < D; c += 32) {
                        uint32_t orr[32];
                        tmem_ld_32x32b_x32(tO + c, orr);
                        tmem_wait_ld();
                        reg_fence<32>(orr);
#pragma unroll
                        for (int i = 0; i < 32; i += 2) {
                            float a0, a1;
                            f2_unpack(f2_mul(f2_pack(__uint_as_float(orr[i]), __uint_as_float(orr[i + 1])), f2), a0,
                                      a1);
                            orr[i] = __float_as_uint(a0);
                            orr[i + 1] = __float_as_uint(a1);
                        }
                        tmem_st_32x32b_x32(tO + c, orr);
                    }
                    tmem_wait_st();
                }
                // exponentials 2^(s * scale * log2 e - m), the row sum, and P (bf16)
                // into TMEM in two halves, each handed to the MMA thread at once
                const float m_sub = (m_run == -INFINITY) ? 0.0f : m_run;
                const uint64_t sl2x2 = f2_pack(sl2, sl2);
                const uint64_t negm2 = f2_pack(-m_sub, -m_sub);
                // the row sum in independent f32x2 chains: four at D=128 (shorter
                // dependency chain, measured faster there), two at D=64 (fewer registers)
                constexpr int kSumChains = (D == 128) ? 4 : 2;
                uint64_t acc_e[4] = {0ull, 0ull, 0ull, 0ull};
                auto exp_half = [&](int hf) {
                    uint32_t pk[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int c = hf * 64 + 2 * i;
                        const uint64_t t = f2_fma(f2_pack(sv[c], sv[c + 1]), sl2x2, negm2);
                        float t0, t1;
                        f2_unpack(t, t0, t1);
                        const float e0 = ex2_approx(t0), e1 = ex2_approx(t1);
                        pk[i] = pack_bf16x2(e0, e1);
                        acc_e[i % kSumChains] = f2_add(acc_e[i % kSumChains], f2_pack(e0, e1));
                    }
                    tmem_st_32x32b_x32((kSplitP ? tP_q : tS) + hf * 32, pk);
                    tmem_wait_st();
                    tc_fence_before_sync();
                    __syncwarp();   // every lane's P is in TMEM: one arrival for the warp
                    if (lane == 0) mbar_arrive(bar_p_part(buf, hf));
                };
                if (!wait_pv_prev()) {
                    ok = false;
                    break;
                }
                exp_half(0);
                exp_half(1);
                // P reaches the MMA rounded to bf16.  O is normalised by the sum with the
                // tile's largest P taken as rounded (its exponential is recomputed
                // exactly as in the loop above): a key that dominates a row then has
                // its rounding cancel in O / l, which is where rounding P costs most.
                // The LSE takes the unrounded sum.
                float d_round = 0.0f;
                if (tmax != -INFINITY) {
                    const float pm = ex2_approx(fmaf(tmax, sl2, -m_sub));
                    d_round = __uint_as_float(pack_bf16x2(pm, 0.0f) << 16) - pm;
                }
                float b0, b1;
                f2_unpack(kSumChains == 4 ? f2_add(f2_add(acc_e[0], acc_e[1]), f2_add(acc_e[2], acc_e[3]))
                                          : f2_add(acc_e[0], acc_e[1]),
                          b0, b1);
                l_run += (b0 + b1) + d_round;
                l_exact += b0 + b1;
            }

            // ---- epilogue: O / l -> bf16, staged in shared memory in the TMA box
            // layout (128-byte swizzle) and written with TMA stores, 64 columns
            // per store (positions past Lq are clipped by TMA); LSE per row ----
            bool have_o = ok && n_kt > 0;
            if (have_o) {
                // the unit's last P.V has completed: o_done, or (split P) its pv_done
                have_o = kSplitP ? mbar_wait(bar_pv_done(q), static_cast<uint32_t>(tiles + n_kt - 1) & 1u,
                                             abort_flag, &g_attn_err, kDevErrTimeout)
                                 : mbar_wait(bar_o_done(q), static_cast<uint32_t>(nu) & 1u, abort_flag, &g_attn_err,
                                             kDevErrTimeout);
                ok = have_o;
                tc_fence_after_sync();
            }
            const float inv_l = (l_run > 0.0f) ? 1.0f / l_run : 0.0f;
            if (kSplit && u.part >= 0) {
                // a run of the unit's key tiles: O / l in fp32 and the log2-sum-exp to
                // this item's slot, every row of the tile (attn_prefill_merge_kernel
                // combines the unit's parts and skips padding rows)
                ATTN_CHECK(p.part_o != nullptr && u.part < (p.n_units - p.n_full));
                const size_t prow = (static_cast<size_t>(u.part) * NQ + q) * kBM + r;
                float* dst = p.part_o + prow * D;
#pragma unroll 1
                for (int c = 0; c < D; c += 32) {
                    uint32_t orr[32];
                    if (have_o) {
                        tmem_ld_32x32b_x32(tO + c, orr);
                        tmem_wait_ld();
                        reg_fence<32>(orr);
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) orr[i] = 0u;
                    }
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4*>(dst + c + i) =
                            make_float4(__uint_as_float(orr[i]) * inv_l, __uint_as_float(orr[i + 1]) * inv_l,
                                        __uint_as_float(orr[i + 2]) * inv_l, __uint_as_float(orr[i + 3]) * inv_l);
                }
                p.part_l[prow] = (l_exact > 0.0f) ? m_run + __log2f(l_exact) : -INFINITY;
                tiles += n_kt;
                if (n_kt > 0) ++nu;
                continue;
            }
            const int q_head0 = u.b * p.Hq + u.g * p.G;
            ATTN_CHECK(tile_p0 >= 0 && q_head0 >= 0 && q_head0 + p.G <= p.B * p.Hq);
            auto o_cols = [&](int c, uint32_t* ob) {   // 32 columns from c, packed into 16 words
                uint32_t orr[32];
                if (have_o) {
                    tmem_ld_32x32b_x32(tO + c, orr);
                    tmem_wait_ld();
                    reg_fence<32>(orr);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) orr[i] = 0u;
                }
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    ob[i] = pack_bf16x2(__uint_as_float(orr[2 * i]) * inv_l, __uint_as_float(orr[2 * i + 1]) * inv_l);
            };
            if constexpr (kPersistent) {
                // One 64-column staging block per warpgroup: the next unit's Q may
                // already be landing in the Q tiles.
                uint8_t* stg = smem + L::kStgOff + q * L::kBlockBytes;
#pragma unroll 1
                for (int kb = 0; kb < L::kKB; ++kb) {
                    uint32_t ob[32];
                    o_cols(kb * 64, ob);
                    o_cols(kb * 64 + 32, ob + 16);
                    if (r == 0) tma_store_wait_read();   // the previous store from the block has read it
                    named_bar_sync(wg_bar, 128);
                    uint8_t* rowp = stg + r * 128;
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        *reinterpret_cast<uint4*>(rowp + ((i ^ (r & 7)) << 4)) =
                            make_uint4(ob[4 * i], ob[4 * i + 1], ob[4 * i + 2], ob[4 * i + 3]);
                    fence_proxy_async_smem();
                    named_bar_sync(wg_bar, 128);   // the warpgroup's rows are all staged
                    if (r == 0) {
                        tma_store_3d(&tm_o, smem_u32(stg), kb * 64, tile_p0, q_head0);
                        tma_store_commit();
                    }
                }
            } else {
                // One unit per CTA: the Q tile is free (its last reader, the last
                // Q K^T, precedes the last P.V, which o_done follows).
                uint8_t* stile = smem + L::kQOff + q * L::kQTileBytes;
#pragma unroll 1
                for (int c = 0; c < D; c += 32) {
                    uint32_t ob[16];
                    o_cols(c, ob);
                    uint8_t* rowp = stile + (c >> 6) * L::kBlockBytes + r * 128;
                    const int chunk0 = (c & 63) >> 3;   // 16-byte chunk of the 128-byte row: 0 or 4
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        *reinterpret_cast<uint4*>(rowp + (((chunk0 + i) ^ (r & 7)) << 4)) =
                            make_uint4(ob[4 * i], ob[4 * i + 1], ob[4 * i + 2], ob[4 * i + 3]);
                }
                fence_proxy_async_smem();
                named_bar_sync(wg_bar, 128);   // the warpgroup's rows are all staged
                if (r == 0) {
                    for (int kb = 0; kb < L::kKB; ++kb)
                        tma_store_3d(&tm_o, smem_u32(stile) + kb * L::kBlockBytes, kb * 64, tile_p0, q_head0);
                    tma_store_commit();
                }
            }
            ATTN_CHECK(!row_valid || (h >= 0 && h < p.Hq && pos >= 0 && pos < p.Lq));
            if (row_valid && p.lse != nullptr) {
                const float lse = (l_exact > 0.0f) ? (m_run + __log2f(l_exact)) * kLn2 : -INFINITY;
                p.lse[(static_cast<size_t>(u.b) * p.Hq + h) * p.Lq + pos] = lse;
            }
            tiles += n_kt;
            if (n_kt > 0) ++nu;
        }
        if (r == 0) tma_store_wait_all();   // shared memory stays until the stores are done with it
    }

    // ---- teardown ----
    tc_fence_before_sync();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

// Merge of the key-split units' parts (PrefillParams: n_full, n_parts, part_o,
// part_l): out = sum_k 2^(lse_k - lse) O_k and lse = log2 sum_k 2^lse_k (stored
// as natural log), per query row; one warp per row of a unit's NQ Q tiles, each
// lane D / 32 columns, all of a row's loads issued before any is used.  Rows
// past G * P or past Lq are padding: skipped.
template <int D, int NQ>
__global__ void __launch_bounds__(128) attn_prefill_merge_kernel(const PrefillParams p) {
    grid_dep_wait();   // launched as a programmatic dependent of the prefill kernel
    constexpr int kPer = D / 32;
    constexpr int kParts = kPrefillSplitParts;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * 4 + warp;                  // over split units x NQ x 128
    const int n_split = (p.n_units - p.n_full) / kParts;
    if (row >= n_split * NQ * kBM) return;
    const int su = row / (NQ * kBM);
    const int q = (row / kBM) % NQ;
    const int r = row % kBM;
    const PrefillUnit u = prefill_unit<NQ>(p, p.n_full + su * kParts);   // b, g, p_begin of the unit
    const int pos = u.p_begin + q * p.P + r % p.P;
    if (r >= p.G * p.P || pos >= p.Lq) return;
    const int h = u.g * p.G + r / p.P;
    float lk[kParts], ov[kParts][kPer];
#pragma unroll
    for (int k = 0; k < kParts; ++k) {
        const size_t prow = (static_cast<size_t>(su * kParts + k) * NQ + q) * kBM + r;
        lk[k] = p.part_l[prow];
        const float* src = p.part_o + prow * D + lane * kPer;
#pragma unroll
        for (int i = 0; i < kPer; i += 2) {
            const float2 v = *reinterpret_cast<const float2*>(src + i);
            ov[k][i] = v.x;
            ov[k][i + 1] = v.y;
        }
    }
    float M = -INFINITY;
#pragma unroll
    for (int k = 0; k < kParts; ++k) M = fmaxf(M, lk[k]);
    float acc[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) acc[i] = 0.0f;
    float L = 0.0f;
#pragma unroll
    for (int k = 0; k < kParts; ++k) {
        const float w = (lk[k] == -INFINITY) ? 0.0f : ex2_approx(lk[k] - M);
        L += w;
#pragma unroll
        for (int i = 0; i < kPer; ++i) acc[i] = fmaf(w, ov[k][i], acc[i]);
    }
    const float inv = (L > 0.0f) ? 1.0f / L : 0.0f;
    const size_t orow = (static_cast<size_t>(u.b) * p.Hq + h) * p.Lq + pos;
    ATTN_CHECK(u.b < p.B && h < p.Hq && pos < p.Lq);
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) + orow * D + lane * kPer;
#pragma unroll
    for (int i = 0; i < kPer; i += 2) *reinterpret_cast<uint32_t*>(o + i) = pack_bf16x2(acc[i] * inv, acc[i + 1] * inv);
    if (p.lse != nullptr && lane == 0) p.lse[orow] = (L > 0.0f) ? (M + __log2f(L)) * kLn2 : -INFINITY;
}

}  // namespace attn
