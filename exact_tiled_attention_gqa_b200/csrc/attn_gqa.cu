// attn_gqa.cu -- the C ABI of include/attn_gqa.h: argument checks, TMA
// descriptors and kernel launches.  All arithmetic happens in the kernels of
// prefill_sm100.cuh and decode_sm100.cuh; this file only validates, describes
// the caller's tensors to the TMA unit and enqueues work on the caller's
// stream.  There is no other code path: no fallback, no host compute.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include "../../include/attn_gqa.h"
#include "decode_kv8_sm100.cuh"
#include "decode_sm100.cuh"
#include "decode_tc_sm100.cuh"
#include "prefill_sm100.cuh"

namespace attn {
namespace {

thread_local char g_last_error[320] = "";

int fail(int status, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return status;
}

int ok() {
    g_last_error[0] = '\0';
    return ATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---- cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda) ----
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* sym = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &sym, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(sym);
    });
    return fn;
}

// A dense bf16 tensor [d2][d1][d0] (d0 contiguous) read in boxes of
// (box0, box1, box2) elements with 128-byte swizzle; out-of-range rows read as 0.
int encode_bf16_3d(CUtensorMap* map, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box0,
                   uint32_t box1, uint32_t box2, const char* what) {
    auto enc = tensor_map_encoder();
    if (!enc) return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the CUDA driver");
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
    cuuint32_t box[3] = {box0, box1, box2};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for %s", (int)r, what);
    return ATTN_OK;
}

// An 8-bit [d2][d1][d0] tensor (d0 bytes innermost) read in boxes of
// (box0, box1, 1), swizzled to match the box's row length (128 or 64 bytes).
int encode_u8_3d(CUtensorMap* map, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box0,
                 uint32_t box1, const char* what) {
    auto enc = tensor_map_encoder();
    if (!enc) return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the CUDA driver");
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {d0, d0 * d1};
    cuuint32_t box[3] = {box0, box1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapSwizzle swz = (box0 == 128) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for %s", (int)r, what);
    return ATTN_OK;
}

// A 16-bit [d1][d0] tensor read in boxes of (box0, 1), unswizzled.
int encode_u16_2d(CUtensorMap* map, const void* ptr, uint64_t d0, uint64_t d1, uint32_t box0, const char* what) {
    auto enc = tensor_map_encoder();
    if (!enc) return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the CUDA driver");
    cuuint64_t dims[2] = {d0, d1};
    cuuint64_t strides[1] = {d0 * 2};
    cuuint32_t box[2] = {box0, 1};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for %s", (int)r, what);
    return ATTN_OK;
}

// Allow a kernel its dynamic shared memory (once per device and kernel).
template <typename Kernel>
int ensure_smem(Kernel kernel, int bytes, int* done_mask_per_device) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= 64) return fail(ATTN_ERR_CUDA, "device ordinal %d out of range", dev);
    if (__atomic_load_n(&done_mask_per_device[dev], __ATOMIC_ACQUIRE)) return ATTN_OK;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    __atomic_store_n(&done_mask_per_device[dev], 1, __ATOMIC_RELEASE);
    return ATTN_OK;
}

// SMs of the current device, and this launch's scheduling counters for a
// persistent prefill.  Ordinary launches take the eager slots in turn; a launch
// being recorded into a CUDA graph (a stream capture) takes the next capture
// slot instead, which the graph then uses on every replay (see g_prefill_sched).
int device_sms_and_sched(cudaStream_t stream, int* n_sm, int** sched) {
    static int sms[64];
    static int* sched_base[64];
    static std::atomic<unsigned> eager_ticket{0};
    static std::atomic<unsigned> capture_ticket{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= 64) return fail(ATTN_ERR_CUDA, "device ordinal %d out of range", dev);
    int n = __atomic_load_n(&sms[dev], __ATOMIC_ACQUIRE);
    int* b = __atomic_load_n(&sched_base[dev], __ATOMIC_ACQUIRE);
    if (n == 0 || b == nullptr) {
        e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
        void* addr = nullptr;
        e = cudaGetSymbolAddress(&addr, g_prefill_sched);
        if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
        b = static_cast<int*>(addr);
        __atomic_store_n(&sched_base[dev], b, __ATOMIC_RELEASE);
        __atomic_store_n(&sms[dev], n, __ATOMIC_RELEASE);
    }
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(stream, &cap);
    if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "cudaStreamIsCapturing: %s", cudaGetErrorString(e));
    unsigned slot;
    if (cap == cudaStreamCaptureStatusActive)
        slot = kPrefillEagerSlots + capture_ticket.fetch_add(1, std::memory_order_relaxed) % kPrefillCaptureSlots;
    else
        slot = eager_ticket.fetch_add(1, std::memory_order_relaxed) % kPrefillEagerSlots;
    *n_sm = n;
    *sched = b + 2 * slot;
    return ATTN_OK;
}

int check_launch(const char* what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "%s launch failed: %s", what, cudaGetErrorString(e));
    return ATTN_OK;
}

// Launches a kernel that starts with grid_dep_wait() as a programmatic dependent
// of the kernel before it on the stream: it may be scheduled while that kernel's
// last CTAs still run (they release it when they start), and reads nothing before
// that kernel has completed.  Saves the launch gap between a split kernel and its
// combine.  Static shared memory only.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), unsigned grid, unsigned block, cudaStream_t stream,
                             Args... args) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// The split combine: one warp per row (four rows per CTA) when rows have few
// splits, four warps per row when they have more than 16 (their reads then take
// four times fewer dependent rounds).
template <int D, bool F32>
int launch_combine(const DecodeParams& prm, void* out, float* lse, int rows, cudaStream_t stream) {
    const cudaError_t e =
        (prm.n_splits > 16)
            ? launch_dependent(attn_decode_combine_kernel<D, F32, 4>, static_cast<unsigned>(rows), 128u, stream, prm,
                               out, lse)
            : launch_dependent(attn_decode_combine_kernel<D, F32, 1>, static_cast<unsigned>((rows + 3) / 4), 128u,
                               stream, prm, out, lse);
    if (e != cudaSuccess)
        return fail(ATTN_ERR_CUDA, "attn_decode_combine_kernel launch failed: %s", cudaGetErrorString(e));
    return check_launch("attn_decode_combine_kernel");
}

// Rows that see no key at all (Lk == 0): O = 0, LSE = -inf.
__global__ void fill_no_key_rows_kernel(__nv_bfloat16* out, float* lse, size_t rows, int D) {
    const size_t n = rows * static_cast<size_t>(D);
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        out[i] = __float2bfloat16(0.0f);
        if (lse != nullptr && i % D == 0) lse[i / D] = -INFINITY;
    }
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// The launch's parameters that depend only on the sizes (pointers and the
// scheduling counters are set by the caller).
template <int D>
PrefillParams prefill_params(int B, int Hq, int Hkv, int Lq, int Lk, float scale, int is_causal) {
    using L = PrefillSmem<D>;
    constexpr int NQ = L::kNQ;
    PrefillParams prm{};
    prm.B = B;
    prm.Hq = Hq;
    prm.Hkv = Hkv;
    prm.Lq = Lq;
    prm.Lk = Lk;
    prm.G = Hq / Hkv;
    prm.P = kBM / prm.G;
    prm.n_mblk = (Lq + NQ * prm.P - 1) / (NQ * prm.P);
    // Unit order: one band of every group when all of K and V fit in half the
    // L2 (126 MB); otherwise bands of as many groups as fit in 16 MB.  (Bands of
    // 60 MB raised DRAM reads of the Qwen3-8B B4 L8192 prefill from 403 to about
    // 710 MB on B200: a tile read from both dies is held in both halves of L2.)
    {
        const double group_kv_bytes = static_cast<double>(Lk) * D * 2 * 2;
        const double n_bh = static_cast<double>(B) * Hkv;
        const double fit = (group_kv_bytes * n_bh <= 63e6) ? n_bh : std::floor(16e6 / std::max(group_kv_bytes, 1.0));
        prm.band = static_cast<int>(std::min(std::max(fit, 1.0), n_bh));
    }
    prm.is_causal = is_causal ? 1 : 0;
    prm.scale_log2 = scale * kLog2e;
    const long long units = static_cast<long long>(B) * Hkv * prm.n_mblk;
    prm.n_units = units > 0x7fffffffLL ? -1 : static_cast<int>(units);
    prm.n_full = prm.n_units;
    prm.n_parts = 1;
    return prm;
}

// Key-split tail.  Units are near-equal when every query of a launch sees most
// keys (chunked prefill: Lq << Lk), and a persistent launch whose unit count is
// not a multiple of the SM count then ends in a part-filled wave: 256 units on
// 148 SMs keep 40 SMs idle for half of the launch.  The last (units mod SMs)
// units of the order are cut into 4 runs of key tiles instead, handed out after
// the full units, and merged by attn_prefill_merge_kernel.  Only for 1 to 3 full
// waves (beyond that the tail is a small part of the launch) and only when every
// unit cut has at least 8 key tiles (2 per part; lighter units cost less than a
// part's start-up).
struct PrefillSplit {
    int n_full = 0, n_items = 0;
    size_t o_bytes = 0, total = 0;   // partial outputs, then log2-sum-exps
};

template <int D>
PrefillSplit prefill_split_plan(const PrefillParams& prm, int n_sm) {
    using L = PrefillSmem<D>;
    constexpr int NQ = L::kNQ;
    PrefillSplit sp;
    sp.n_full = sp.n_items = prm.n_units;
    if (!L::kPersistent || prm.n_units <= n_sm || prm.n_units >= 4 * n_sm) return sp;
    const int R = prm.n_units % n_sm;
    if (R == 0) return sp;
    for (int i = prm.n_units - R; i < prm.n_units; ++i)
        if (prefill_unit<NQ>(prm, i).n_kt < 2 * kPrefillSplitParts) return sp;
    sp.n_full = prm.n_units - R;
    sp.n_items = sp.n_full + R * kPrefillSplitParts;
    const size_t rows = static_cast<size_t>(R) * kPrefillSplitParts * NQ * kBM;
    sp.o_bytes = align256(rows * D * sizeof(float));
    sp.total = sp.o_bytes + align256(rows * sizeof(float));
    return sp;
}

int device_sm_count(int* n_sm) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(n_sm, cudaDevAttrMultiProcessorCount, dev);
    return e == cudaSuccess ? ATTN_OK : fail(ATTN_ERR_CUDA, "SM count: %s", cudaGetErrorString(e));
}

template <int D>
int launch_prefill(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv,
                   int Lq, int Lk, float scale, int is_causal, cudaStream_t stream, bool ws_call = false,
                   void* workspace = nullptr, size_t workspace_bytes = 0) {
    static int smem_done[64], smem_done_split[64];
    using L = PrefillSmem<D>;
    constexpr int NQ = L::kNQ;
    const int G = Hq / Hkv;
    const int P = kBM / G;
    CUtensorMap tq, tk, tv;
    int st;
    if ((st = encode_bf16_3d(&tq, q, D, Lq, static_cast<uint64_t>(B) * Hq, 64, P, G, "q")) != ATTN_OK) return st;
    if ((st = encode_bf16_3d(&tk, k, D, Lk, static_cast<uint64_t>(B) * Hkv, 64, kBN, 1, "k")) != ATTN_OK) return st;
    if ((st = encode_bf16_3d(&tv, v, D, Lk, static_cast<uint64_t>(B) * Hkv, 64, kBN, 1, "v")) != ATTN_OK) return st;
    CUtensorMap to;   // O is written in the same boxes Q is read in
    if ((st = encode_bf16_3d(&to, out, D, Lq, static_cast<uint64_t>(B) * Hq, 64, P, G, "out")) != ATTN_OK) return st;
    PrefillParams prm = prefill_params<D>(B, Hq, Hkv, Lq, Lk, scale, is_causal);
    if (prm.n_units < 0) return fail(ATTN_ERR_UNSUPPORTED, "prefill has too many work units");
    prm.out = out;
    prm.lse = lse;
    prm.sched = nullptr;
    long long grid = prm.n_units;
    bool split = false;
    if (L::kPersistent) {   // one CTA per SM, each taking units until they run out
        int n_sm = 0;
        if ((st = device_sms_and_sched(stream, &n_sm, &prm.sched)) != ATTN_OK) return st;
        if (ws_call) {
            const PrefillSplit sp = prefill_split_plan<D>(prm, n_sm);
            if (sp.n_items != prm.n_units) {
                if (workspace == nullptr || workspace_bytes < sp.total)
                        return fail(ATTN_ERR_WORKSPACE, "prefill workspace needs %zu bytes, got %zu", sp.total,
                                workspace ? workspace_bytes : static_cast<size_t>(0));
                prm.n_full = sp.n_full;
                prm.n_parts = kPrefillSplitParts;
                prm.n_units = sp.n_items;
                prm.part_o = static_cast<float*>(workspace);
                prm.part_l = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + sp.o_bytes);
                split = true;
            }
        }
        grid = std::min<long long>(prm.n_units, n_sm);
    }
    if (!split) {
        if ((st = ensure_smem(attn_prefill_sm100_kernel<D, NQ, false>, L::kAlloc, smem_done)) != ATTN_OK) return st;
        attn_prefill_sm100_kernel<D, NQ, false>
            <<<static_cast<unsigned>(grid), prefill_threads<NQ>(), L::kAlloc, stream>>>(tq, tk, tv, to, prm);
        return check_launch("attn_prefill_sm100_kernel");
    }
    if constexpr (L::kPersistent) {
        if ((st = ensure_smem(attn_prefill_sm100_kernel<D, NQ, true>, L::kAlloc, smem_done_split)) != ATTN_OK)
            return st;
        attn_prefill_sm100_kernel<D, NQ, true>
            <<<static_cast<unsigned>(grid), prefill_threads<NQ>(), L::kAlloc, stream>>>(tq, tk, tv, to, prm);
        if ((st = check_launch("attn_prefill_sm100_kernel")) != ATTN_OK) return st;
        const long long rows = static_cast<long long>(prm.n_units - prm.n_full) / prm.n_parts * NQ * kBM;
        const cudaError_t e =
            launch_dependent(attn_prefill_merge_kernel<D, NQ>, static_cast<unsigned>((rows + 3) / 4), 128u, stream, prm);
        if (e != cudaSuccess)
            return fail(ATTN_ERR_CUDA, "attn_prefill_merge_kernel launch failed: %s", cudaGetErrorString(e));
        return check_launch("attn_prefill_merge_kernel");
    }
    return st;
}

// Cache rows per decode split (always a multiple of 64, the tile height).
//  - mma.sync split kernel: the largest power of two in [256, 4096] that still
//    gives about four waves of CTAs on a 148-SM part (1184 CTAs).
//  - tcgen05 kernel, D <= 128 (more than 16 query rows per KV head): its CTAs
//    carry more setup than the split kernel's (TMEM, the Q tile, a partial per
//    row for the combine), so splits are long, and the split length balances
//    the waves: of the multiples of 64 in [512, 8192], the one that minimises
//    waves x (rows per split + 512), with waves = splits / 256 rounded up and
//    the split count taken at Lmax.  256 CTAs per wave is measured, not the
//    148 SMs x 2 CTAs that fit: at 131072 cached rows and batch 8, splits of
//    4096 rows (G = 64, 256 CTAs) took 0.0938 ms against 0.0960 for 3584 (296
//    CTAs), 0.098 for 4608 and 0.106 for 1792; splits of 8192 rows (G = 32,
//    256 CTAs) took 0.163-0.164 ms against 0.165-0.166 for 7296 (288 CTAs) and
//    0.178 for 10240.
//  - tcgen05 kernel, D = 256 (one CTA per SM): the largest power of two in
//    [512, 4096] that still gives 148 CTAs (the balanced rule above, at one CTA
//    per SM, made the head-dim-256 decode batch 8 % slower: with lengths spread
//    over [1024, 32768] the split count at Lmax says little about real waves).
// The result depends only on the arguments (workspace sizes do too).
bool decode_uses_tc(int D, int rows_per_group) { return D == 256 || rows_per_group > 16; }

int decode_chunk(int B, int Hkv, int Lmax, bool tc_path, int D) {
    const long long groups = static_cast<long long>(B) * Hkv;
    if (!tc_path || D == 256) {
        const long long target = tc_path ? 148LL : 148LL * 2 * 4;
        const int min_chunk = tc_path ? 512 : 256;
        int chunk = 4096;
        while (chunk > min_chunk && groups * ((Lmax + chunk - 1) / chunk) < target) chunk >>= 1;
        return chunk;
    }
    const long long slots = 256;
    int best = 512;
    long long best_cost = -1;
    for (int c = 512; c <= 8192; c += 64) {
        const long long splits = (Lmax + c - 1) / c;
        const long long waves = (groups * splits + slots - 1) / slots;
        const long long cost = waves * (c + 512);
        if (best_cost < 0 || cost < best_cost) {   // ties keep the shorter split (more parallel partials)
            best_cost = cost;
            best = c;
        }
        if (splits == 1) break;   // longer splits change nothing
    }
    return best;
}


struct DecodeLayout {
    int chunk, n_splits;
    size_t o_bytes, lse_off, total;
};

DecodeLayout decode_layout(int B, int Hq, int Hkv, int Lmax, int D, int Lq = 1, bool kv8 = false) {
    DecodeLayout d;
    d.chunk = decode_chunk(B, Hkv, Lmax, !kv8 && decode_uses_tc(D, (Hq / Hkv) * Lq), D);
    d.n_splits = (Lmax + d.chunk - 1) / d.chunk;
    const size_t rows = static_cast<size_t>(B) * Hq * Lq * d.n_splits;
    d.o_bytes = align256(rows * D * sizeof(float));
    d.lse_off = d.o_bytes;
    d.total = d.o_bytes + align256(rows * sizeof(float));
    return d;
}

template <int D, int KPW>
int launch_decode_split(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& prm, cudaStream_t stream) {
    static int smem_done[64];
    using L = DecodeSmem<D>;
    int st;
    if ((st = ensure_smem(attn_decode_split_kernel<D, KPW>, L::kAlloc, smem_done)) != ATTN_OK) return st;
    dim3 grid(prm.n_splits, prm.Hkv, prm.B);
    attn_decode_split_kernel<D, KPW><<<grid, kDecThreads, L::kAlloc, stream>>>(tk, tv, prm);
    return check_launch("attn_decode_split_kernel");
}

// Paged cache description (block_table == nullptr: the contiguous layout).
struct PagedKV {
    const int32_t* block_table = nullptr;
    int page_size = 0, max_pages = 0, n_pages = 0;
};

template <int D, int KPW, int FMT>
int launch_decode_kv8_split(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tks,
                            const CUtensorMap& tvs, const DecodeParams& prm, cudaStream_t stream) {
    static int smem_done[64];
    using L = DecodeKv8Smem<D, FMT>;
    int st;
    if ((st = ensure_smem(attn_decode_kv8_kernel<D, KPW, FMT>, L::kAlloc, smem_done)) != ATTN_OK) return st;
    dim3 grid(prm.n_splits, prm.Hkv, prm.B);
    attn_decode_kv8_kernel<D, KPW, FMT><<<grid, kDecThreads, L::kAlloc, stream>>>(tk, tv, tks, tvs, prm);
    return check_launch("attn_decode_kv8_kernel");
}

template <int D, int NR, int FMT>
int launch_decode_kv8t(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tks, const CUtensorMap& tvs,
                       const DecodeParams& prm, cudaStream_t stream) {
    static int smem_done[64];
    using L = DecodeKv8tSmem<D, FMT>;
    int st;
    if ((st = ensure_smem(attn_decode_kv8t_kernel<D, NR, FMT>, L::kAlloc, smem_done)) != ATTN_OK) return st;
    dim3 grid(prm.n_splits, prm.Hkv, prm.B);
    attn_decode_kv8t_kernel<D, NR, FMT><<<grid, kDecThreads, L::kAlloc, stream>>>(tk, tv, tks, tvs, prm);
    return check_launch("attn_decode_kv8t_kernel");
}

template <int D, int FMT>
int launch_decode_kv8(const void* q, const void* kc, const void* vc, const void* k_scale, const void* v_scale,
                      const int32_t* seqlens, void* out, float* lse, int B, int Hq, int Hkv, int Lq, int Lmax,
                      float scale, void* workspace, cudaStream_t stream, PagedKV paged = PagedKV()) {
    const DecodeLayout lay = decode_layout(B, Hq, Hkv, Lmax, D, Lq, true);
    CUtensorMap tk, tv, tks, tvs;
    int st;
    // the [outer, rows, D] view TMA reads 64-row boxes from (pages: [n_pages * Hkv, page_size, D])
    const uint64_t view_rows = paged.block_table ? static_cast<uint64_t>(paged.page_size) : static_cast<uint64_t>(Lmax);
    const uint64_t outer = paged.block_table ? static_cast<uint64_t>(paged.n_pages) * Hkv
                                             : static_cast<uint64_t>(B) * Hkv;
    if ((st = encode_u8_3d(&tk, kc, D, view_rows, outer, D, kDecKT, "k_cache")) != ATTN_OK) return st;
    if ((st = encode_u8_3d(&tv, vc, D, view_rows, outer, D, kDecKT, "v_cache")) != ATTN_OK) return st;
    if (FMT == kKvFmtQ8_0) {
        const uint64_t per_row = D / 32;
        if ((st = encode_u16_2d(&tks, k_scale, per_row * view_rows, outer, kDecKT * (D / 32), "k_scale")) != ATTN_OK)
            return st;
        if ((st = encode_u16_2d(&tvs, v_scale, per_row * view_rows, outer, kDecKT * (D / 32), "v_scale")) != ATTN_OK)
            return st;
    } else {
        tks = tk;   // unused
        tvs = tv;
    }
    DecodeParams prm;
    prm.q = static_cast<const __nv_bfloat16*>(q);
    prm.seqlens = seqlens;
    prm.o_part = static_cast<float*>(workspace);
    prm.lse_part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + lay.lse_off);
    prm.B = B;
    prm.Hq = Hq;
    prm.Hkv = Hkv;
    prm.Lmax = Lmax;
    prm.G = Hq / Hkv;
    prm.Lq = Lq;
    prm.block_table = paged.block_table;
    prm.page_size = paged.page_size;
    prm.max_pages = paged.max_pages;
    prm.n_pages = paged.n_pages;
    prm.chunk = lay.chunk;
    prm.n_splits = lay.n_splits;
    prm.scale_log2 = scale * kLog2e;
    prm.k_scale = (FMT == kKvFmtE4M3) ? static_cast<const float*>(k_scale) : nullptr;
    prm.v_scale = (FMT == kKvFmtE4M3) ? static_cast<const float*>(v_scale) : nullptr;
    if (prm.n_splits > 65535 || Hkv > 65535 || B > 65535)
        return fail(ATTN_ERR_UNSUPPORTED, "decode grid (%d, %d, %d) exceeds launch limits", prm.n_splits, Hkv, B);
    const int rows = prm.G * Lq;
    if (rows <= 8)
        st = launch_decode_kv8t<D, 1, FMT>(tk, tv, tks, tvs, prm, stream);
    else if (rows <= 16)
        st = launch_decode_kv8t<D, 2, FMT>(tk, tv, tks, tvs, prm, stream);
    else if (rows <= 32)
        st = launch_decode_kv8_split<D, 32, FMT>(tk, tv, tks, tvs, prm, stream);
    else
        st = launch_decode_kv8_split<D, 64, FMT>(tk, tv, tks, tvs, prm, stream);
    if (st != ATTN_OK) return st;
    const int n_rows = B * Hq * Lq;
    return launch_combine<D, false>(prm, out, lse, n_rows, stream);
}


template <int D>
int launch_decode(const void* q, const void* kc, const void* vc, const int32_t* seqlens, void* out, float* lse, int B,
                  int Hq, int Hkv, int Lmax, float scale, void* workspace, cudaStream_t stream, int Lq = 1,
                  PagedKV paged = PagedKV(), bool f32_out = false) {
    const DecodeLayout lay = decode_layout(B, Hq, Hkv, Lmax, D, Lq);
    CUtensorMap tk, tv;
    int st;
    // the [outer, rows, D] view TMA reads boxes of 64 rows from
    const uint64_t view_rows = paged.block_table ? static_cast<uint64_t>(paged.page_size) : static_cast<uint64_t>(Lmax);
    const uint64_t view_outer = paged.block_table ? static_cast<uint64_t>(paged.n_pages) * Hkv
                                                  : static_cast<uint64_t>(B) * Hkv;
    if ((st = encode_bf16_3d(&tk, kc, D, view_rows, view_outer, 64, kDecKT, 1, "k_cache")) != ATTN_OK) return st;
    if ((st = encode_bf16_3d(&tv, vc, D, view_rows, view_outer, 64, kDecKT, 1, "v_cache")) != ATTN_OK) return st;
    DecodeParams prm;
    prm.q = static_cast<const __nv_bfloat16*>(q);
    prm.seqlens = seqlens;
    prm.o_part = static_cast<float*>(workspace);
    prm.lse_part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + lay.lse_off);
    prm.B = B;
    prm.Hq = Hq;
    prm.Hkv = Hkv;
    prm.Lmax = Lmax;
    prm.G = Hq / Hkv;
    prm.Lq = Lq;
    prm.block_table = paged.block_table;
    prm.page_size = paged.page_size;
    prm.max_pages = paged.max_pages;
    prm.n_pages = paged.n_pages;
    prm.chunk = lay.chunk;
    prm.n_splits = lay.n_splits;
    prm.scale_log2 = scale * kLog2e;
    if (prm.n_splits > 65535 || Hkv > 65535 || B > 65535)
        return fail(ATTN_ERR_UNSUPPORTED, "decode grid (%d, %d, %d) exceeds launch limits", prm.n_splits, Hkv, B);
    const int rows_per_group = prm.G * Lq;
    if (decode_uses_tc(D, rows_per_group)) {
        // many query rows per cache row: the tcgen05 split kernel (decode_tc_sm100.cuh)
        static int smem_done_tc[64];
        using LT = DecodeTcSmem<D>;
        CUtensorMap tq;
        if ((st = encode_bf16_3d(&tq, q, D, static_cast<uint64_t>(B) * Hq * Lq, 1, 64, rows_per_group, 1, "q")) !=
            ATTN_OK)
            return st;
        if ((st = ensure_smem(attn_decode_tc_kernel<D>, LT::kAlloc, smem_done_tc)) != ATTN_OK) return st;
        dim3 grid(prm.n_splits, prm.Hkv, prm.B);
        attn_decode_tc_kernel<D><<<grid, kDtcThreads, LT::kAlloc, stream>>>(tq, tk, tv, prm);
        st = check_launch("attn_decode_tc_kernel");
    } else if constexpr (D == 256) {
        st = fail(ATTN_ERR_UNSUPPORTED, "unreachable");   // D = 256 always takes the branch above
    } else if (rows_per_group <= 16)
        st = launch_decode_split<D, 16>(tk, tv, prm, stream);
    else if (rows_per_group <= 32)
        st = launch_decode_split<D, 32>(tk, tv, prm, stream);
    else
        st = launch_decode_split<D, 64>(tk, tv, prm, stream);
    if (st != ATTN_OK) return st;
    const int rows = B * Hq * Lq;
    return f32_out ? launch_combine<D, true>(prm, out, lse, rows, stream)
                   : launch_combine<D, false>(prm, out, lse, rows, stream);
}

// q/out may be null only when they are empty (B == 0 or L1 == 0); k/v only when
// they are empty (B == 0 or L2 == 0) -- an empty tensor has no storage.
int check_common(const void* q, const void* k, const void* v, const void* out, const float* lse, int B, int Hq,
                 int Hkv, int L1, int L2, int D, float scale, const char* l1name, const char* l2name) {
    const bool q_empty = (B == 0 || L1 == 0), kv_empty = (B == 0 || L2 == 0);
    if ((!q && !q_empty) || (!out && !q_empty)) return fail(ATTN_ERR_INVALID_ARG, "null q or out pointer");
    if ((!k || !v) && !kv_empty) return fail(ATTN_ERR_INVALID_ARG, "null k or v pointer");
    if (B < 0 || L1 < 0 || L2 < 0)
        return fail(ATTN_ERR_INVALID_ARG, "negative size (B=%d %s=%d %s=%d)", B, l1name, L1, l2name, L2);
    if (Hq < 1 || Hkv < 1) return fail(ATTN_ERR_INVALID_ARG, "head counts must be >= 1 (Hq=%d Hkv=%d)", Hq, Hkv);
    if (Hq % Hkv != 0) return fail(ATTN_ERR_INVALID_ARG, "Hq=%d is not a multiple of Hkv=%d", Hq, Hkv);
    if (!(std::isfinite(scale) && scale > 0.0f)) return fail(ATTN_ERR_INVALID_ARG, "scale must be finite and > 0");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return fail(ATTN_ERR_INVALID_ARG, "tensor base addresses must be 16-byte aligned");
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u))
        return fail(ATTN_ERR_INVALID_ARG, "lse must be 4-byte aligned");
    if (D != 64 && D != 128 && D != 256) return fail(ATTN_ERR_UNSUPPORTED, "head dim D=%d (built: 64, 128, 256)", D);
    return ATTN_OK;
}

}  // namespace
}  // namespace attn

using namespace attn;

namespace {
// attn_prefill and attn_prefill_ws: checks, empty cases, then the launch (with
// the key-split tail when a workspace is given and the plan uses one).
int prefill_checked(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv,
                    int Lq, int Lk, int D, float scale, int is_causal, bool ws_call, void* workspace,
                    size_t workspace_bytes, void* stream) {
    int st = check_common(q, k, v, out, lse, B, Hq, Hkv, Lq, Lk, D, scale, "Lq", "Lk");
    if (st != ATTN_OK) return st;
    if (Hq / Hkv > kBM) return fail(ATTN_ERR_UNSUPPORTED, "group size G=%d > %d", Hq / Hkv, kBM);
    if (static_cast<long long>(B) * Hq > 0x7fffffffLL || static_cast<long long>(B) * Hkv > 0x7fffffffLL)
        return fail(ATTN_ERR_UNSUPPORTED, "B*H too large");
    if (workspace != nullptr && (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return fail(ATTN_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    if (B == 0 || Lq == 0) return ok();
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (Lk == 0) {
        const size_t rows = static_cast<size_t>(B) * Hq * Lq;
        fill_no_key_rows_kernel<<<1184, 256, 0, s>>>(static_cast<__nv_bfloat16*>(out), lse, rows, D);
        st = check_launch("fill_no_key_rows_kernel");
        return st == ATTN_OK ? ok() : st;
    }
    st = (D == 256) ? launch_prefill<256>(q, k, v, out, lse, B, Hq, Hkv, Lq, Lk, scale, is_causal, s, ws_call,
                                          workspace, workspace_bytes)
         : (D == 128)
             ? launch_prefill<128>(q, k, v, out, lse, B, Hq, Hkv, Lq, Lk, scale, is_causal, s, ws_call, workspace,
                                   workspace_bytes)
             : launch_prefill<64>(q, k, v, out, lse, B, Hq, Hkv, Lq, Lk, scale, is_causal, s, ws_call, workspace,
                                  workspace_bytes);
    return st == ATTN_OK ? ok() : st;
}
}  // namespace

extern "C" int attn_prefill(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
                            int Hkv, int Lq, int Lk, int D, float scale, int is_causal, void* stream) {
    return prefill_checked(q, k, v, out, lse, B, Hq, Hkv, Lq, Lk, D, scale, is_causal, false, nullptr, 0, stream);
}

extern "C" size_t attn_prefill_split_plan(int B, int Hq, int Hkv, int Lq, int Lk, int D, int is_causal, int n_sm,
                                          int* n_full, int* n_items) {
    PrefillSplit sp;
    if (B >= 1 && Hq >= 1 && Hkv >= 1 && Hq % Hkv == 0 && Hq / Hkv <= kBM && Lq >= 1 && Lk >= 1 && n_sm >= 1) {
        if (D == 128) {
            const PrefillParams prm = prefill_params<128>(B, Hq, Hkv, Lq, Lk, 1.0f, is_causal);
            if (prm.n_units > 0) sp = prefill_split_plan<128>(prm, n_sm);
        } else if (D == 64) {
            const PrefillParams prm = prefill_params<64>(B, Hq, Hkv, Lq, Lk, 1.0f, is_causal);
            if (prm.n_units > 0) sp = prefill_split_plan<64>(prm, n_sm);
        }
    }
    if (n_full) *n_full = sp.n_full;
    if (n_items) *n_items = sp.n_items;
    return sp.total;
}

extern "C" size_t attn_prefill_workspace_size(int B, int Hq, int Hkv, int Lq, int Lk, int D, int is_causal) {
    if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || Hq / Hkv > kBM || Lq < 1 || Lk < 1 ||
        (D != 64 && D != 128 && D != 256))
        return 0;
    int n_sm = 0;
    if (device_sm_count(&n_sm) != ATTN_OK) return 0;
    return attn_prefill_split_plan(B, Hq, Hkv, Lq, Lk, D, is_causal, n_sm, nullptr, nullptr);
}

extern "C" int attn_prefill_ws(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
                               int Hkv, int Lq, int Lk, int D, float scale, int is_causal, void* workspace,
                               size_t workspace_bytes, void* stream) {
    return prefill_checked(q, k, v, out, lse, B, Hq, Hkv, Lq, Lk, D, scale, is_causal, true, workspace,
                           workspace_bytes, stream);
}

namespace attn {
namespace {
// ---- attn_prefill_host: host buffers in, host buffers out, copies overlapped ----
//
// Work is cut into units of (sequence b, hc consecutive KV heads); the slabs of
// q, k, v, out and lse that a unit touches are contiguous in [B, H, L, D], so a
// unit is three host-to-device copies, one prefill launch (B = 1, Hq = hc G,
// Hkv = hc) and two device-to-host copies.  Units alternate between two device
// slots; copies in run on one library stream, copies out on another, the
// kernels on the caller's stream, ordered by events per slot, so unit u's
// copy in, unit u-1's kernel and unit u-2's copy out can run at once.
struct HostPipe {
    bool ready = false;
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t start = nullptr, in_done[2] = {}, comp_done[2] = {}, out_done[2] = {};
};
HostPipe g_pipes[64];
std::mutex g_pipe_mu;

int host_pipe(HostPipe** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= 64) return fail(ATTN_ERR_CUDA, "device ordinal %d out of range", dev);
    HostPipe& p = g_pipes[dev];
    if (!p.ready) {
        const unsigned ef = cudaEventDisableTiming;
        e = cudaStreamCreateWithFlags(&p.h2d, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&p.d2h, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p.start, ef);
        for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
            e = cudaEventCreateWithFlags(&p.in_done[i], ef);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p.comp_done[i], ef);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p.out_done[i], ef);
        }
        if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "creating the copy streams: %s", cudaGetErrorString(e));
        p.ready = true;
    }
    *out = &p;
    return ATTN_OK;
}

struct HostUnits {
    int hc = 1, n_units = 0;
    size_t q_bytes = 0, kv_bytes = 0, lse_bytes = 0;   // one unit's slabs
    size_t q_off = 0, k_off = 0, v_off = 0, o_off = 0, l_off = 0, slot_bytes = 0;
};

HostUnits host_units(int B, int Hq, int Hkv, int Lq, int Lk, int D) {
    HostUnits u;
    const int G = Hq / Hkv;
    const int NQ = (D == 256) ? 1 : 2;
    const long long n_mblk = (Lq + static_cast<long long>(NQ) * (kBM / G) - 1) / (static_cast<long long>(NQ) * (kBM / G));
    // the smallest run of KV heads (a divisor of Hkv) whose kernel still fills a wave of CTAs:
    // small units keep the pipeline's fill and drain short
    u.hc = Hkv;
    for (int hc = 1; hc <= Hkv; ++hc)
        if (Hkv % hc == 0 && hc * n_mblk >= 148) {
            u.hc = hc;
            break;
        }
    u.n_units = B * (Hkv / u.hc);
    u.q_bytes = static_cast<size_t>(u.hc) * G * Lq * D * 2;
    u.kv_bytes = static_cast<size_t>(u.hc) * Lk * D * 2;
    u.lse_bytes = static_cast<size_t>(u.hc) * G * Lq * 4;
    u.q_off = 0;
    u.k_off = align256(u.q_off + u.q_bytes);
    u.v_off = align256(u.k_off + u.kv_bytes);
    u.o_off = align256(u.v_off + u.kv_bytes);
    u.l_off = align256(u.o_off + u.q_bytes);
    u.slot_bytes = align256(u.l_off + u.lse_bytes);
    return u;
}
}  // namespace
}  // namespace attn

extern "C" size_t attn_prefill_host_scratch_size(int B, int Hq, int Hkv, int Lq, int Lk, int D) {
    if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || Lq < 1 || Lk < 0 || (D != 64 && D != 128 && D != 256) ||
        Hq / Hkv > kBM)
        return 0;
    return 2 * host_units(B, Hq, Hkv, Lq, Lk, D).slot_bytes;
}

extern "C" int attn_prefill_host(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
                                 int Hkv, int Lq, int Lk, int D, float scale, int is_causal, void* scratch,
                                 size_t scratch_bytes, void* stream) {
    int st = check_common(q, k, v, out, lse, B, Hq, Hkv, Lq, Lk, D, scale, "Lq", "Lk");
    if (st != ATTN_OK) return st;
    if (Hq / Hkv > kBM) return fail(ATTN_ERR_UNSUPPORTED, "group size G=%d > %d", Hq / Hkv, kBM);
    if (static_cast<long long>(B) * Hq > 0x7fffffffLL || static_cast<long long>(B) * Hkv > 0x7fffffffLL)
        return fail(ATTN_ERR_UNSUPPORTED, "B*H too large");
    if (B == 0 || Lq == 0) return ok();
    const HostUnits u = host_units(B, Hq, Hkv, Lq, Lk, D);
    if (!scratch || scratch_bytes < 2 * u.slot_bytes)
        return fail(ATTN_ERR_WORKSPACE, "prefill host scratch needs %zu bytes, got %zu", 2 * u.slot_bytes,
                    scratch ? scratch_bytes : static_cast<size_t>(0));
    if (reinterpret_cast<uintptr_t>(scratch) & 255u)
        return fail(ATTN_ERR_INVALID_ARG, "scratch must be 256-byte aligned");
    std::lock_guard<std::mutex> lock(g_pipe_mu);
    HostPipe* hp = nullptr;
    if ((st = host_pipe(&hp)) != ATTN_OK) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const int G = Hq / Hkv, chunks = Hkv / u.hc;
    auto cuda_ok = [](cudaError_t e, const char* what) {
        return e == cudaSuccess ? ATTN_OK : fail(ATTN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    };
    // the copies must not overtake work the caller queued before (it may still use the scratch)
    if ((st = cuda_ok(cudaEventRecord(hp->start, cs), "cudaEventRecord")) != ATTN_OK) return st;
    if ((st = cuda_ok(cudaStreamWaitEvent(hp->h2d, hp->start, 0), "cudaStreamWaitEvent")) != ATTN_OK) return st;
    for (int n = 0; n < u.n_units; ++n) {
        const int slot = n & 1, b = n / chunks, c = n % chunks;
        uint8_t* base = static_cast<uint8_t*>(scratch) + slot * u.slot_bytes;
        const size_t qrow = (static_cast<size_t>(b) * Hq + static_cast<size_t>(c) * u.hc * G) * Lq;   // first q row
        const size_t krow = (static_cast<size_t>(b) * Hkv + static_cast<size_t>(c) * u.hc) * Lk;     // first k row
        const uint8_t* qh = static_cast<const uint8_t*>(q) + qrow * D * 2;
        const uint8_t* kh = static_cast<const uint8_t*>(k) + krow * D * 2;
        const uint8_t* vh = static_cast<const uint8_t*>(v) + krow * D * 2;
        uint8_t* oh = static_cast<uint8_t*>(out) + qrow * D * 2;
        float* lh = lse ? lse + qrow : nullptr;
        // in: after the kernel that last read this slot's inputs
        st = cuda_ok(cudaStreamWaitEvent(hp->h2d, hp->comp_done[slot], 0), "cudaStreamWaitEvent");
        if (st == ATTN_OK) st = cuda_ok(cudaMemcpyAsync(base + u.q_off, qh, u.q_bytes, cudaMemcpyHostToDevice, hp->h2d), "copy q in");
        if (st == ATTN_OK && u.kv_bytes) {
            st = cuda_ok(cudaMemcpyAsync(base + u.k_off, kh, u.kv_bytes, cudaMemcpyHostToDevice, hp->h2d), "copy k in");
            if (st == ATTN_OK)
                st = cuda_ok(cudaMemcpyAsync(base + u.v_off, vh, u.kv_bytes, cudaMemcpyHostToDevice, hp->h2d), "copy v in");
        }
        if (st == ATTN_OK) st = cuda_ok(cudaEventRecord(hp->in_done[slot], hp->h2d), "cudaEventRecord");
        // kernel: after its inputs are in and the slot's previous outputs are out
        if (st == ATTN_OK) st = cuda_ok(cudaStreamWaitEvent(cs, hp->in_done[slot], 0), "cudaStreamWaitEvent");
        if (st == ATTN_OK) st = cuda_ok(cudaStreamWaitEvent(cs, hp->out_done[slot], 0), "cudaStreamWaitEvent");
        if (st != ATTN_OK) return st;
        void* od = base + u.o_off;
        float* ld = lh ? reinterpret_cast<float*>(base + u.l_off) : nullptr;
        if (Lk == 0) {
            fill_no_key_rows_kernel<<<1184, 256, 0, cs>>>(static_cast<__nv_bfloat16*>(od), ld,
                                                          static_cast<size_t>(u.hc) * G * Lq, D);
            st = check_launch("fill_no_key_rows_kernel");
        } else {
            const void *qd = base + u.q_off, *kd = base + u.k_off, *vd = base + u.v_off;
            st = (D == 256)   ? launch_prefill<256>(qd, kd, vd, od, ld, 1, u.hc * G, u.hc, Lq, Lk, scale, is_causal, cs)
                 : (D == 128) ? launch_prefill<128>(qd, kd, vd, od, ld, 1, u.hc * G, u.hc, Lq, Lk, scale, is_causal, cs)
                              : launch_prefill<64>(qd, kd, vd, od, ld, 1, u.hc * G, u.hc, Lq, Lk, scale, is_causal, cs);
        }
        if (st != ATTN_OK) return st;
        if ((st = cuda_ok(cudaEventRecord(hp->comp_done[slot], cs), "cudaEventRecord")) != ATTN_OK) return st;
        // out: after the kernel
        st = cuda_ok(cudaStreamWaitEvent(hp->d2h, hp->comp_done[slot], 0), "cudaStreamWaitEvent");
        if (st == ATTN_OK) st = cuda_ok(cudaMemcpyAsync(oh, od, u.q_bytes, cudaMemcpyDeviceToHost, hp->d2h), "copy out");
        if (st == ATTN_OK && lh) st = cuda_ok(cudaMemcpyAsync(lh, ld, u.lse_bytes, cudaMemcpyDeviceToHost, hp->d2h), "copy lse out");
        if (st == ATTN_OK) st = cuda_ok(cudaEventRecord(hp->out_done[slot], hp->d2h), "cudaEventRecord");
        if (st != ATTN_OK) return st;
    }
    // the caller's stream passes this call only once every result is in host memory
    for (int slot = 0; slot < 2; ++slot)
        if ((st = cuda_ok(cudaStreamWaitEvent(cs, hp->out_done[slot], 0), "cudaStreamWaitEvent")) != ATTN_OK) return st;
    return ok();
}

extern "C" size_t attn_decode_workspace_size(int B, int Hq, int Hkv, int Lmax, int D) {
    if (B < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || Lmax < 1 || (D != 64 && D != 128 && D != 256) || Hq / Hkv > 128)
        return 0;
    if (B == 0) return 0;
    return decode_layout(B, Hq, Hkv, Lmax, D).total;
}

namespace attn {
namespace {
void* decode_scratch_address(int* status);
}  // namespace
}  // namespace attn

namespace {
// Argument checks and launch shared by attn_decode, attn_decode_partial and
// attn_decode_noalloc.  With noalloc the workspace arguments are ignored and the
// split partials go to the library's static scratch array, if they fit.
int decode_checked(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens, void* out,
                   float* lse, int B, int Hq, int Hkv, int Lmax, int D, float scale, void* workspace,
                   size_t workspace_bytes, void* stream, bool f32_out, bool noalloc = false) {
    int st = check_common(q, k_cache, v_cache, out, lse, B, Hq, Hkv, Lmax, Lmax, D, scale, "Lmax", "Lmax");
    if (st != ATTN_OK) return st;
    if (!seqlens && B > 0) return fail(ATTN_ERR_INVALID_ARG, "null seqlens");
    if (reinterpret_cast<uintptr_t>(seqlens) & 3u) return fail(ATTN_ERR_INVALID_ARG, "seqlens must be 4-byte aligned");
    if (Lmax < 1) return fail(ATTN_ERR_INVALID_ARG, "Lmax must be >= 1");
    if (Hq / Hkv > 128) return fail(ATTN_ERR_UNSUPPORTED, "decode group size G=%d > 128", Hq / Hkv);
    if (static_cast<long long>(B) * Hq > 0x7fffffffLL) return fail(ATTN_ERR_UNSUPPORTED, "B*Hq too large");
    if (B == 0) return ok();
    const size_t need = decode_layout(B, Hq, Hkv, Lmax, D).total;
    if (noalloc) {
        if (need > ATTN_DECODE_NOALLOC_SCRATCH_BYTES)
            return fail(ATTN_ERR_WORKSPACE,
                        "attn_decode_noalloc: these sizes need %zu bytes of split partials; the static scratch "
                        "holds %u (use attn_decode with a caller workspace)",
                        need, ATTN_DECODE_NOALLOC_SCRATCH_BYTES);
        workspace = decode_scratch_address(&st);
        if (st != ATTN_OK) return st;
    } else {
        if (!workspace || workspace_bytes < need)
            return fail(ATTN_ERR_WORKSPACE, "decode workspace needs %zu bytes, got %zu", need,
                        workspace ? workspace_bytes : static_cast<size_t>(0));
        if (reinterpret_cast<uintptr_t>(workspace) & 255u)
            return fail(ATTN_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const PagedKV none;
    st = (D == 256)   ? launch_decode<256>(q, k_cache, v_cache, seqlens, out, lse, B, Hq, Hkv, Lmax, scale, workspace, s,
                                           1, none, f32_out)
         : (D == 128) ? launch_decode<128>(q, k_cache, v_cache, seqlens, out, lse, B, Hq, Hkv, Lmax, scale, workspace, s,
                                           1, none, f32_out)
                      : launch_decode<64>(q, k_cache, v_cache, seqlens, out, lse, B, Hq, Hkv, Lmax, scale, workspace, s,
                                          1, none, f32_out);
    return st == ATTN_OK ? ok() : st;
}
}  // namespace

extern "C" int attn_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens, void* out,
                           float* lse, int B, int Hq, int Hkv, int Lmax, int D, float scale, void* workspace,
                           size_t workspace_bytes, void* stream) {
    return decode_checked(q, k_cache, v_cache, seqlens, out, lse, B, Hq, Hkv, Lmax, D, scale, workspace,
                          workspace_bytes, stream, false);
}

namespace {
// attn_decode_host's workspace: attn_decode's partials, then device copies of
// q, out, lse and seqlens, each 256-byte aligned.
struct HostDecodeLayout {
    size_t q_off, o_off, l_off, s_off, total;
};
HostDecodeLayout host_decode_layout(int B, int Hq, int D, size_t partial_bytes) {
    auto al = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    const size_t rows = static_cast<size_t>(B) * Hq;
    HostDecodeLayout L;
    L.q_off = al(partial_bytes);
    L.o_off = L.q_off + al(rows * D * 2);
    L.l_off = L.o_off + al(rows * D * 2);
    L.s_off = L.l_off + al(rows * 4);
    L.total = L.s_off + al(static_cast<size_t>(B) * 4);
    return L;
}
}  // namespace

extern "C" size_t attn_decode_host_workspace_size(int B, int Hq, int Hkv, int Lmax, int D) {
    const size_t partial = attn_decode_workspace_size(B, Hq, Hkv, Lmax, D);
    return partial == 0 ? 0 : host_decode_layout(B, Hq, D, partial).total;
}

extern "C" int attn_decode_host(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens,
                                void* out, float* lse, int B, int Hq, int Hkv, int Lmax, int D, float scale,
                                void* workspace, size_t workspace_bytes, void* stream) {
    int st = check_common(q, k_cache, v_cache, out, lse, B, Hq, Hkv, Lmax, Lmax, D, scale, "Lmax", "Lmax");
    if (st != ATTN_OK) return st;
    if (!seqlens && B > 0) return fail(ATTN_ERR_INVALID_ARG, "null seqlens");
    if (reinterpret_cast<uintptr_t>(seqlens) & 3u) return fail(ATTN_ERR_INVALID_ARG, "seqlens must be 4-byte aligned");
    if (Lmax < 1) return fail(ATTN_ERR_INVALID_ARG, "Lmax must be >= 1");
    if (Hq / Hkv > 128) return fail(ATTN_ERR_UNSUPPORTED, "decode group size G=%d > 128", Hq / Hkv);
    if (static_cast<long long>(B) * Hq > 0x7fffffffLL) return fail(ATTN_ERR_UNSUPPORTED, "B*Hq too large");
    if (B == 0) return ok();
    const size_t partial = attn_decode_workspace_size(B, Hq, Hkv, Lmax, D);
    const HostDecodeLayout L = host_decode_layout(B, Hq, D, partial);
    if (!workspace || workspace_bytes < L.total)
        return fail(ATTN_ERR_WORKSPACE, "decode host workspace needs %zu bytes, got %zu", L.total,
                    workspace ? workspace_bytes : static_cast<size_t>(0));
    if (reinterpret_cast<uintptr_t>(workspace) & 255u)
        return fail(ATTN_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const size_t rows = static_cast<size_t>(B) * Hq;
    auto copy = [&](void* dst, const void* src, size_t bytes, cudaMemcpyKind kind, const char* what) {
        const cudaError_t e = cudaMemcpyAsync(dst, src, bytes, kind, s);
        return e == cudaSuccess ? ATTN_OK : fail(ATTN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    };
    if ((st = copy(ws + L.q_off, q, rows * D * 2, cudaMemcpyHostToDevice, "copy q in")) != ATTN_OK) return st;
    if ((st = copy(ws + L.s_off, seqlens, static_cast<size_t>(B) * 4, cudaMemcpyHostToDevice, "copy seqlens in")) !=
        ATTN_OK)
        return st;
    float* lse_dev = lse ? reinterpret_cast<float*>(ws + L.l_off) : nullptr;
    st = decode_checked(ws + L.q_off, k_cache, v_cache, reinterpret_cast<const int32_t*>(ws + L.s_off), ws + L.o_off,
                        lse_dev, B, Hq, Hkv, Lmax, D, scale, workspace, partial, stream, false);
    if (st != ATTN_OK) return st;
    if ((st = copy(out, ws + L.o_off, rows * D * 2, cudaMemcpyDeviceToHost, "copy out")) != ATTN_OK) return st;
    if (lse && (st = copy(lse, lse_dev, rows * 4, cudaMemcpyDeviceToHost, "copy lse out")) != ATTN_OK) return st;
    return ok();
}

extern "C" int attn_decode_partial(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens,
                                   float* o_part, float* lse_part, int B, int Hq, int Hkv, int Lmax, int D, float scale,
                                   void* workspace, size_t workspace_bytes, void* stream) {
    if (B > 0 && !lse_part) return fail(ATTN_ERR_INVALID_ARG, "null lse_part");
    return decode_checked(q, k_cache, v_cache, seqlens, o_part, lse_part, B, Hq, Hkv, Lmax, D, scale, workspace,
                          workspace_bytes, stream, true);
}

extern "C" int attn_decode_merge(const float* o_parts, const float* lse_parts, int n_parts, int rows, int D,
                                 void* out, float* lse, void* stream) {
    if (n_parts < 1 || rows < 0) return fail(ATTN_ERR_INVALID_ARG, "n_parts must be >= 1 and rows >= 0");
    if (D != 64 && D != 128 && D != 256) return fail(ATTN_ERR_UNSUPPORTED, "head dim D=%d (built: 64, 128, 256)", D);
    if (rows == 0) return ok();
    if (!o_parts || !lse_parts || !out) return fail(ATTN_ERR_INVALID_ARG, "null o_parts, lse_parts or out");
    if (!aligned16(o_parts) || !aligned16(out) || (reinterpret_cast<uintptr_t>(lse_parts) & 3u) ||
        (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
        return fail(ATTN_ERR_INVALID_ARG, "o_parts and out must be 16-byte aligned, lse arrays 4-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const unsigned grid = static_cast<unsigned>((rows + 3) / 4);
    auto* o = static_cast<__nv_bfloat16*>(out);
    if (D == 256)
        attn_decode_merge_kernel<256><<<grid, 128, 0, s>>>(o_parts, lse_parts, n_parts, rows, o, lse);
    else if (D == 128)
        attn_decode_merge_kernel<128><<<grid, 128, 0, s>>>(o_parts, lse_parts, n_parts, rows, o, lse);
    else
        attn_decode_merge_kernel<64><<<grid, 128, 0, s>>>(o_parts, lse_parts, n_parts, rows, o, lse);
    const int st = check_launch("attn_decode_merge_kernel");
    return st == ATTN_OK ? ok() : st;
}

extern "C" int attn_kvp_signal(unsigned int* const* flag_ptrs, int n, unsigned int value, void* stream) {
    if (n < 0 || (n > 0 && !flag_ptrs)) return fail(ATTN_ERR_INVALID_ARG, "bad flag pointer array");
    if (n == 0) return ok();
    attn_kvp_signal_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(flag_ptrs, n, value);
    const int st = check_launch("attn_kvp_signal_kernel");
    return st == ATTN_OK ? ok() : st;
}

extern "C" int attn_kvp_wait(const unsigned int* flags, int n, unsigned int value, void* stream) {
    if (n < 0 || (n > 0 && !flags) || (reinterpret_cast<uintptr_t>(flags) & 3u))
        return fail(ATTN_ERR_INVALID_ARG, "bad flags array");
    if (n == 0) return ok();
    attn_kvp_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(flags, n, value);
    const int st = check_launch("attn_kvp_wait_kernel");
    return st == ATTN_OK ? ok() : st;
}

extern "C" int attn_decode_merge_peers(const float* const* o_ptrs, const float* const* lse_ptrs,
                                       const unsigned int* ready, unsigned int value, int n_parts, int rows, int D,
                                       void* out, float* lse, void* stream) {
    if (n_parts < 1 || rows < 0) return fail(ATTN_ERR_INVALID_ARG, "n_parts must be >= 1 and rows >= 0");
    if (D != 64 && D != 128 && D != 256) return fail(ATTN_ERR_UNSUPPORTED, "head dim D=%d (built: 64, 128, 256)", D);
    if (rows == 0) return ok();
    if (!o_ptrs || !lse_ptrs || !ready || !out) return fail(ATTN_ERR_INVALID_ARG, "null pointer array, flags or out");
    if (!aligned16(out) || (reinterpret_cast<uintptr_t>(ready) & 3u) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
        return fail(ATTN_ERR_INVALID_ARG, "out must be 16-byte aligned, ready and lse 4-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const unsigned grid = static_cast<unsigned>((rows + 3) / 4);
    auto* o = static_cast<__nv_bfloat16*>(out);
    if (D == 256)
        attn_decode_merge_peers_kernel<256><<<grid, 128, 0, s>>>(o_ptrs, lse_ptrs, ready, value, n_parts, rows, o, lse);
    else if (D == 128)
        attn_decode_merge_peers_kernel<128><<<grid, 128, 0, s>>>(o_ptrs, lse_ptrs, ready, value, n_parts, rows, o, lse);
    else
        attn_decode_merge_peers_kernel<64><<<grid, 128, 0, s>>>(o_ptrs, lse_ptrs, ready, value, n_parts, rows, o, lse);
    const int st = check_launch("attn_decode_merge_peers_kernel");
    return st == ATTN_OK ? ok() : st;
}


namespace attn {
namespace {
// The pipelines' bounded wait, made to run out: warp 0 plays a producer that
// announces 16 bytes on `full` that never arrive (no copy is issued), then waits
// for the consumer to free the entry (`empty`) with the kernels' 2 s limit;
// warp 1 plays the consumer and waits on `full` with `limit_ns`.  The consumer's
// wait gives up, records the timeout and raises the abort flag; the producer's
// wait then ends through the flag, long before its own limit.  No asynchronous
// copy is in flight at any point.
__global__ void wait_selftest_kernel(unsigned long long limit_ns, int* result) {
    __shared__ __align__(8) uint64_t bars[2];
    __shared__ int abort_word;
    volatile int* abort_flag = &abort_word;
    const uint32_t full = smem_u32(&bars[0]), empty = smem_u32(&bars[1]);
    if (threadIdx.x == 0) {
        mbar_init(full, 1);
        mbar_init(empty, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if ((threadIdx.x & 31) != 0) return;
    const uint64_t t0 = global_timer_ns();
    bool ok;
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(full, 16);
        ok = mbar_wait(empty, 0, abort_flag, &g_attn_err, kDevErrTimeout);
    } else {
        ok = mbar_wait(full, 0, abort_flag, &g_attn_err, kDevErrTimeout, limit_ns);
    }
    const int role = threadIdx.x >> 5;
    result[2 * role] = ok ? 1 : 0;
    const uint64_t us = (global_timer_ns() - t0) / 1000u;
    result[2 * role + 1] = us > 0x7fffffffull ? 0x7fffffff : static_cast<int>(us);
}
}  // namespace
}  // namespace attn

extern "C" int attn_selftest_wait(unsigned long long limit_ns, int* result, void* stream) {
    if (!result || (reinterpret_cast<uintptr_t>(result) & 3u))
        return fail(ATTN_ERR_INVALID_ARG, "result must be a 4-byte aligned device array of 4 ints");
    if (limit_ns == 0 || limit_ns > kWaitLimitNs)
        return fail(ATTN_ERR_INVALID_ARG, "limit_ns must be in (0, %llu]", static_cast<unsigned long long>(kWaitLimitNs));
    wait_selftest_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, result);
    const int st = check_launch("wait_selftest_kernel");
    return st == ATTN_OK ? ok() : st;
}

extern "C" int attn_prefill_sched_busy(int* busy) {
    if (!busy) return fail(ATTN_ERR_INVALID_ARG, "null busy");
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "cudaDeviceSynchronize: %s", cudaGetErrorString(e));
    static int host[2 * kPrefillSchedSlots];
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    e = cudaMemcpyFromSymbol(host, g_prefill_sched, sizeof host);
    if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "reading the scheduling counters: %s", cudaGetErrorString(e));
    int n = 0;
    for (int i = 0; i < 2 * kPrefillSchedSlots; ++i) n += host[i] != 0;
    *busy = n;
    return ok();
}

extern "C" size_t attn_decode_mq_workspace_size(int B, int Hq, int Hkv, int Lq, int Lmax, int D) {
    if (B < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || Lmax < 1 || Lq < 1 || (D != 64 && D != 128 && D != 256) ||
        static_cast<long long>(Hq / Hkv) * Lq > 128)
        return 0;
    if (B == 0) return 0;
    return decode_layout(B, Hq, Hkv, Lmax, D, Lq).total;
}

extern "C" int attn_decode_mq(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens,
                              void* out, float* lse, int B, int Hq, int Hkv, int Lq, int Lmax, int D, float scale,
                              void* workspace, size_t workspace_bytes, void* stream) {
    int st = check_common(q, k_cache, v_cache, out, lse, B, Hq, Hkv, Lq, Lmax, D, scale, "Lq", "Lmax");
    if (st != ATTN_OK) return st;
    if (Lq < 1) return fail(ATTN_ERR_INVALID_ARG, "Lq must be >= 1");
    if (!seqlens && B > 0) return fail(ATTN_ERR_INVALID_ARG, "null seqlens");
    if (reinterpret_cast<uintptr_t>(seqlens) & 3u) return fail(ATTN_ERR_INVALID_ARG, "seqlens must be 4-byte aligned");
    if (Lmax < 1) return fail(ATTN_ERR_INVALID_ARG, "Lmax must be >= 1");
    if (static_cast<long long>(Hq / Hkv) * Lq > 128)
        return fail(ATTN_ERR_UNSUPPORTED, "G * Lq = %lld query rows per KV head (built: up to 128)",
                    static_cast<long long>(Hq / Hkv) * Lq);
    if (static_cast<long long>(B) * Hq * Lq > 0x7fffffffLL) return fail(ATTN_ERR_UNSUPPORTED, "B*Hq*Lq too large");
    if (B == 0) return ok();
    const size_t need = decode_layout(B, Hq, Hkv, Lmax, D, Lq).total;
    if (!workspace || workspace_bytes < need)
        return fail(ATTN_ERR_WORKSPACE, "decode workspace needs %zu bytes, got %zu", need,
                    workspace ? workspace_bytes : static_cast<size_t>(0));
    if (reinterpret_cast<uintptr_t>(workspace) & 255u)
        return fail(ATTN_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    st = (D == 256)
             ? launch_decode<256>(q, k_cache, v_cache, seqlens, out, lse, B, Hq, Hkv, Lmax, scale, workspace, s, Lq)
         : (D == 128)
             ? launch_decode<128>(q, k_cache, v_cache, seqlens, out, lse, B, Hq, Hkv, Lmax, scale, workspace, s, Lq)
             : launch_decode<64>(q, k_cache, v_cache, seqlens, out, lse, B, Hq, Hkv, Lmax, scale, workspace, s, Lq);
    return st == ATTN_OK ? ok() : st;
}

extern "C" size_t attn_decode_paged_workspace_size(int B, int Hq, int Hkv, int Lq, int page_size, int max_pages,
                                                    int D) {
    if (page_size < 64 || page_size % 64 != 0 || max_pages < 1 ||
        static_cast<long long>(page_size) * max_pages > 0x7fffffffLL)
        return 0;
    return attn_decode_mq_workspace_size(B, Hq, Hkv, Lq, page_size * max_pages, D);
}

extern "C" int attn_decode_paged(const void* q, const void* k_pages, const void* v_pages, const int32_t* block_table,
                                 const int32_t* seqlens, void* out, float* lse, int B, int Hq, int Hkv, int Lq,
                                 int n_pages, int page_size, int max_pages, int D, float scale, void* workspace,
                                 size_t workspace_bytes, void* stream) {
    if (page_size < 64 || page_size % 64 != 0)
        return fail(ATTN_ERR_INVALID_ARG, "page_size=%d must be a positive multiple of 64", page_size);
    if (n_pages < 1 || max_pages < 1) return fail(ATTN_ERR_INVALID_ARG, "n_pages and max_pages must be >= 1");
    if (static_cast<long long>(page_size) * max_pages > 0x7fffffffLL ||
        static_cast<long long>(n_pages) * Hkv > 0x7fffffffLL)
        return fail(ATTN_ERR_UNSUPPORTED, "page pool too large");
    const int Lmax = page_size * max_pages;   // the longest sequence the block table can describe
    int st = check_common(q, k_pages, v_pages, out, lse, B, Hq, Hkv, Lq, Lmax, D, scale, "Lq", "Lmax");
    if (st != ATTN_OK) return st;
    if (Lq < 1) return fail(ATTN_ERR_INVALID_ARG, "Lq must be >= 1");
    if (B > 0 && (!seqlens || !block_table)) return fail(ATTN_ERR_INVALID_ARG, "null seqlens or block_table");
    if ((reinterpret_cast<uintptr_t>(seqlens) | reinterpret_cast<uintptr_t>(block_table)) & 3u)
        return fail(ATTN_ERR_INVALID_ARG, "seqlens and block_table must be 4-byte aligned");
    if (static_cast<long long>(Hq / Hkv) * Lq > 128)
        return fail(ATTN_ERR_UNSUPPORTED, "G * Lq = %lld query rows per KV head (built: up to 128)",
                    static_cast<long long>(Hq / Hkv) * Lq);
    if (static_cast<long long>(B) * Hq * Lq > 0x7fffffffLL) return fail(ATTN_ERR_UNSUPPORTED, "B*Hq*Lq too large");
    if (B == 0) return ok();
    const size_t need = decode_layout(B, Hq, Hkv, Lmax, D, Lq).total;
    if (!workspace || workspace_bytes < need)
        return fail(ATTN_ERR_WORKSPACE, "decode workspace needs %zu bytes, got %zu", need,
                    workspace ? workspace_bytes : static_cast<size_t>(0));
    if (reinterpret_cast<uintptr_t>(workspace) & 255u)
        return fail(ATTN_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    PagedKV pg;
    pg.block_table = block_table;
    pg.page_size = page_size;
    pg.max_pages = max_pages;
    pg.n_pages = n_pages;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    st = (D == 256)
             ? launch_decode<256>(q, k_pages, v_pages, seqlens, out, lse, B, Hq, Hkv, Lmax, scale, workspace, s, Lq, pg)
         : (D == 128)
             ? launch_decode<128>(q, k_pages, v_pages, seqlens, out, lse, B, Hq, Hkv, Lmax, scale, workspace, s, Lq, pg)
             : launch_decode<64>(q, k_pages, v_pages, seqlens, out, lse, B, Hq, Hkv, Lmax, scale, workspace, s, Lq, pg);
    return st == ATTN_OK ? ok() : st;
}

extern "C" const char* attn_status_string(int status) {
    switch (status) {
        case ATTN_OK: return "ATTN_OK";
        case ATTN_ERR_INVALID_ARG: return "ATTN_ERR_INVALID_ARG";
        case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED";
        case ATTN_ERR_WORKSPACE: return "ATTN_ERR_WORKSPACE";
        case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA";
        default: return "ATTN_ERR_UNKNOWN";
    }
}

extern "C" const char* attn_last_error(void) { return g_last_error; }

extern "C" int attn_device_error(unsigned int* flags, int reset) {
    if (!flags) return fail(ATTN_ERR_INVALID_ARG, "null flags");
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "cudaDeviceSynchronize: %s", cudaGetErrorString(e));
    e = cudaMemcpyFromSymbol(flags, g_attn_err, sizeof(unsigned int));
    if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "reading the device error word: %s", cudaGetErrorString(e));
    if (reset) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_attn_err, &zero, sizeof zero);
        if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "clearing the device error word: %s", cudaGetErrorString(e));
    }
    return ok();
}

// ---------------------------------------------------------------------------
// attn_decode_noalloc: attn_decode whose split partials live in a scratch
// array declared here, for callers that cannot allocate device memory.
// ---------------------------------------------------------------------------
namespace attn {
namespace {

static __device__ __align__(256) uint8_t g_decode_scratch[ATTN_DECODE_NOALLOC_SCRATCH_BYTES];

// In host code `g_decode_scratch` only names a host-side stand-in; the device
// address is looked up once per device, with that device current.
void* decode_scratch_address(int* status) {
    static std::mutex mu;
    static void* addr[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        *status = fail(ATTN_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
        return nullptr;
    }
    if (dev < 0 || dev >= 64) {
        *status = fail(ATTN_ERR_CUDA, "device ordinal %d out of range", dev);
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (addr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess || p == nullptr) {
            *status = fail(ATTN_ERR_CUDA, "cudaGetSymbolAddress(decode scratch): %s", cudaGetErrorString(e));
            return nullptr;
        }
        addr[dev] = p;
    }
    *status = ATTN_OK;
    return addr[dev];
}

}  // namespace
}  // namespace attn

extern "C" int attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens,
                                   void* out, float* lse, int B, int Hq, int Hkv, int Lmax, int D, float scale,
                                   void* stream) {
    return decode_checked(q, k_cache, v_cache, seqlens, out, lse, B, Hq, Hkv, Lmax, D, scale, nullptr, 0, stream,
                          false, /*noalloc=*/true);
}

extern "C" size_t attn_decode_kv8_workspace_size(int B, int Hq, int Hkv, int Lq, int Lmax, int D) {
    if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || Lmax < 1 || Lq < 1 || (D != 64 && D != 128) ||
        static_cast<long long>(Hq / Hkv) * Lq > 64)
        return 0;
    return decode_layout(B, Hq, Hkv, Lmax, D, Lq, true).total;
}

extern "C" size_t attn_decode_kv8_paged_workspace_size(int B, int Hq, int Hkv, int Lq, int page_size, int max_pages,
                                                       int D) {
    if (page_size < 64 || page_size % 64 != 0 || max_pages < 1 ||
        static_cast<long long>(page_size) * max_pages > 0x7fffffffLL)
        return 0;
    return attn_decode_kv8_workspace_size(B, Hq, Hkv, Lq, page_size * max_pages, D);
}

namespace {
// Checks and launch shared by the contiguous and the paged 8-bit entry points.
// Lmax: the cache rows one sequence can have (paged: page_size * max_pages);
// scale_rows: rows of one (b or page, KV head) slab of the q8_0 scale plane.
int decode_kv8_checked(const void* q, const void* k_cache, const void* v_cache, const void* k_scale,
                       const void* v_scale, int kv_format, const int32_t* seqlens, void* out, float* lse, int B,
                       int Hq, int Hkv, int Lq, int Lmax, int scale_rows, int D, float scale, void* workspace,
                       size_t workspace_bytes, void* stream, PagedKV paged) {
    int st = check_common(q, k_cache, v_cache, out, lse, B, Hq, Hkv, Lq, Lmax, D, scale, "Lq", "Lmax");
    if (st != ATTN_OK) return st;
    if (kv_format != ATTN_KV_E4M3 && kv_format != ATTN_KV_Q8_0)
        return fail(ATTN_ERR_INVALID_ARG, "kv_format %d (E4M3 = %d, Q8_0 = %d)", kv_format, ATTN_KV_E4M3,
                    ATTN_KV_Q8_0);
    if (Lq < 1) return fail(ATTN_ERR_INVALID_ARG, "Lq must be >= 1");
    if (Lmax < 1) return fail(ATTN_ERR_INVALID_ARG, "Lmax must be >= 1");
    if (!seqlens && B > 0) return fail(ATTN_ERR_INVALID_ARG, "null seqlens");
    if (reinterpret_cast<uintptr_t>(seqlens) & 3u) return fail(ATTN_ERR_INVALID_ARG, "seqlens must be 4-byte aligned");
    if (B > 0 && (!k_scale || !v_scale)) return fail(ATTN_ERR_INVALID_ARG, "null k_scale or v_scale");
    if (kv_format == ATTN_KV_E4M3 && ((reinterpret_cast<uintptr_t>(k_scale) | reinterpret_cast<uintptr_t>(v_scale)) & 3u))
        return fail(ATTN_ERR_INVALID_ARG, "E4M3 scales must be 4-byte aligned");
    if (kv_format == ATTN_KV_Q8_0) {
        if (!aligned16(k_scale) || !aligned16(v_scale))
            return fail(ATTN_ERR_INVALID_ARG, "Q8_0 scale planes must be 16-byte aligned");
        if (scale_rows % 4 != 0)
            return fail(ATTN_ERR_INVALID_ARG, "Q8_0 caches need Lmax %% 4 == 0 (got %d)", scale_rows);
    }
    if (D != 64 && D != 128) return fail(ATTN_ERR_UNSUPPORTED, "8-bit cache head dim D=%d (built: 64, 128)", D);
    if (static_cast<long long>(Hq / Hkv) * Lq > 64)
        return fail(ATTN_ERR_UNSUPPORTED, "G * Lq = %lld query rows per KV head (8-bit cache: up to 64)",
                    static_cast<long long>(Hq / Hkv) * Lq);
    if (static_cast<long long>(B) * Hq * Lq > 0x7fffffffLL) return fail(ATTN_ERR_UNSUPPORTED, "B*Hq*Lq too large");
    if (B == 0) return ok();
    const size_t need = decode_layout(B, Hq, Hkv, Lmax, D, Lq, true).total;
    if (!workspace || workspace_bytes < need)
        return fail(ATTN_ERR_WORKSPACE, "decode workspace needs %zu bytes, got %zu", need,
                    workspace ? workspace_bytes : static_cast<size_t>(0));
    if (reinterpret_cast<uintptr_t>(workspace) & 255u)
        return fail(ATTN_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (kv_format == ATTN_KV_E4M3)
        st = (D == 128) ? launch_decode_kv8<128, kKvFmtE4M3>(q, k_cache, v_cache, k_scale, v_scale, seqlens, out, lse,
                                                              B, Hq, Hkv, Lq, Lmax, scale, workspace, s, paged)
                        : launch_decode_kv8<64, kKvFmtE4M3>(q, k_cache, v_cache, k_scale, v_scale, seqlens, out, lse,
                                                             B, Hq, Hkv, Lq, Lmax, scale, workspace, s, paged);
    else
        st = (D == 128) ? launch_decode_kv8<128, kKvFmtQ8_0>(q, k_cache, v_cache, k_scale, v_scale, seqlens, out, lse,
                                                              B, Hq, Hkv, Lq, Lmax, scale, workspace, s, paged)
                        : launch_decode_kv8<64, kKvFmtQ8_0>(q, k_cache, v_cache, k_scale, v_scale, seqlens, out, lse,
                                                             B, Hq, Hkv, Lq, Lmax, scale, workspace, s, paged);
    return st == ATTN_OK ? ok() : st;
}
}  // namespace

extern "C" int attn_decode_kv8(const void* q, const void* k_cache, const void* v_cache, const void* k_scale,
                               const void* v_scale, int kv_format, const int32_t* seqlens, void* out, float* lse,
                               int B, int Hq, int Hkv, int Lq, int Lmax, int D, float scale, void* workspace,
                               size_t workspace_bytes, void* stream) {
    return decode_kv8_checked(q, k_cache, v_cache, k_scale, v_scale, kv_format, seqlens, out, lse, B, Hq, Hkv, Lq,
                              Lmax, Lmax, D, scale, workspace, workspace_bytes, stream, PagedKV());
}

extern "C" int attn_decode_kv8_paged(const void* q, const void* k_pages, const void* v_pages, const void* k_scale,
                                     const void* v_scale, int kv_format, const int32_t* block_table,
                                     const int32_t* seqlens, void* out, float* lse, int B, int Hq, int Hkv, int Lq,
                                     int n_pages, int page_size, int max_pages, int D, float scale, void* workspace,
                                     size_t workspace_bytes, void* stream) {
    if (page_size < 64 || page_size % 64 != 0)
        return fail(ATTN_ERR_INVALID_ARG, "page_size=%d must be a positive multiple of 64", page_size);
    if (n_pages < 1 || max_pages < 1) return fail(ATTN_ERR_INVALID_ARG, "n_pages and max_pages must be >= 1");
    if (static_cast<long long>(page_size) * max_pages > 0x7fffffffLL ||
        static_cast<long long>(n_pages) * Hkv > 0x7fffffffLL)
        return fail(ATTN_ERR_UNSUPPORTED, "page pool too large");
    if (B > 0 && !block_table) return fail(ATTN_ERR_INVALID_ARG, "null block_table");
    if (reinterpret_cast<uintptr_t>(block_table) & 3u)
        return fail(ATTN_ERR_INVALID_ARG, "block_table must be 4-byte aligned");
    PagedKV pg;
    pg.block_table = block_table;
    pg.page_size = page_size;
    pg.max_pages = max_pages;
    pg.n_pages = n_pages;
    return decode_kv8_checked(q, k_pages, v_pages, k_scale, v_scale, kv_format, seqlens, out, lse, B, Hq, Hkv, Lq,
                              page_size * max_pages, page_size, D, scale, workspace, workspace_bytes, stream, pg);
}

namespace attn {
namespace {
__global__ void kv8_convert_selftest_kernel(const uint16_t* codes, uint32_t* out, int n, int fmt) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const uint32_t x = codes[i];
    out[i] = (fmt == kKvFmtE4M3) ? e4m3x2_to_f16x2(x) : int8x2_to_f16x2(x);
}
}  // namespace
}  // namespace attn

extern "C" int attn_selftest_kv8_convert(const uint16_t* codes, uint32_t* out, int n, int kv_format, void* stream) {
    if (n < 0 || (n > 0 && (!codes || !out)) || (kv_format != ATTN_KV_E4M3 && kv_format != ATTN_KV_Q8_0))
        return fail(ATTN_ERR_INVALID_ARG, "bad selftest arguments");
    if (n == 0) return ok();
    kv8_convert_selftest_kernel<<<(n + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(codes, out, n,
                                                                                                 kv_format);
    const int st = check_launch("kv8_convert_selftest_kernel");
    return st == ATTN_OK ? ok() : st;
}
