// libpa host side: argument checks, launch planning and the C entry points of
// include/pa.h.  One translation unit, so the device error word has one definition.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "pa_cache.cuh"
#include "pa_common.cuh"
#include "pa_decode.cuh"
#include "pa_merge.cuh"
#include "pa_decode_streamk.cuh"
#include "pa_decode_dynamic.cuh"
#include "pa_prefill.cuh"

using namespace pa;

namespace {

constexpr int kMaxDevices = 64;
// Default fixed split (measured on B200 over the decode workloads): one pass for
// contexts up to kAutoSingleMax tokens, else 1024-token partitions when there are at
// least as many (sequence, kv head) pairs as SMs, 2048-token partitions when fewer.
constexpr int kAutoSplitTokens = 1024;
constexpr int kAutoSplitTokensFew = 2048;
constexpr int kAutoSingleMax = 1280;
// Pages of at least this many tokens: warps start their tiles at rotated offsets (measured
// on the long-context workload at 512-token pages: 59.8 -> 58.5 us per step; no gain at 16).
constexpr int kRotateMinBlock = 64;

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }
int ilog2_host(int x) {
    int r = 0;
    while ((1 << r) < x) ++r;
    return r;
}
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 2-D map over a cache seen as [rows][D] 16-bit elements; box 64 columns x boxr rows,
// 128-byte swizzle (the layout the decode kernel's shared-memory reads assume).
bool make_cache_map(CUtensorMap *m, const void *base, unsigned long long rows, int D,
                    pa_dtype dt, int boxr) {
    auto enc = encode_fn();
    if (!enc) return false;
    const CUtensorMapDataType t =
        dt == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    cuuint32_t box[2] = {64u, (cuuint32_t)boxr};
    cuuint32_t estr[2] = {1u, 1u};
    return enc(m, t, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over q [num_tokens][Hq][D]: box 64 columns x G heads x 128/G tokens (the
// 128 query rows of one kv head's group), 128-byte swizzle.
bool make_q_map(CUtensorMap *m, const void *base, int num_tokens, int Hq, int D, int G,
                pa_dtype dt) {
    auto enc = encode_fn();
    if (!enc) return false;
    const CUtensorMapDataType t =
        dt == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)num_tokens};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hq * D * 2};
    cuuint32_t box[3] = {64u, (cuuint32_t)G, (cuuint32_t)(kPfRows / G)};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    return enc(m, t, 3, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Plan {
    bool streamk = false;   // balanced split over persistent warps
    bool dynamic = false;   // dynamic split over persistent CTAs
    int grid = 0;           // stream-K / dynamic CTAs
    int partition_tokens = 0;
    int num_parts = 1;
    size_t ws_bytes = 0;
    // every split leaves the first kDynCounterBytes (the dynamic split's counters) alone,
    // so that one workspace can serve calls with different splits
    size_t off_o = kDynCounterBytes, off_m = 0, off_l = 0, off_pre = 0;
    size_t off_co = 0, off_cm = 0, off_cl = 0;  // balanced split: CTA-level records
    size_t off_us = 0, off_ro = 0, off_rm = 0, off_rl = 0;  // dynamic split
};


constexpr int kSmPerSmBytes = 233472;  // shared memory per SM usable by CTAs (228 KiB)

template <int D>
int streamk_ctas_per_sm() {
    const int per_cta = SkGeom<D>::kSmem + 16 + 1024;  // + static smem + per-CTA reserve
    const int n = kSmPerSmBytes / per_cta;
    return n < 1 ? 1 : (n > 16 ? 16 : n);
}

int device_sms(int dev) {
    static std::atomic<int> cache[kMaxDevices];
    if (dev < 0 || dev >= kMaxDevices) return 148;
    int v = cache[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        return 148;  // no device visible: size for a B200
    }
    cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

int current_device_or_zero() {
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return d;
}

Plan make_plan(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
               int max_blocks_per_seq, int max_context_len, int sliding_window,
               int partition_size, int sms) {
    Plan pl;
    const long long cap = (long long)max_blocks_per_seq * block_size;
    long long bound = cap;
    if (max_context_len > 0 && max_context_len < cap) bound = max_context_len;
    // under a window the tiles of a context span at most W + 15 tokens (span_begin
    // rounds the window start down to a tile)
    if (sliding_window > 0 && (long long)sliding_window + kTile - 1 < bound)
        bound = (long long)sliding_window + kTile - 1;
    if (bound < 1) bound = 1;
    const int G = num_kv_heads > 0 ? num_q_heads / num_kv_heads : 1;
    const int max_seqs = head_dim == 64 ? SkGeom<64>::kMaxSeqs : SkGeom<128>::kMaxSeqs;
    const bool fits32 = (long long)num_seqs * ((cap + kTile - 1) / kTile) < (1LL << 31);
    const bool balanced_ok = num_seqs <= max_seqs && fits32;
    const bool want_balanced = partition_size == PA_PARTITION_BALANCED;
    const long long units = (long long)num_seqs * num_kv_heads;
    const int dyn_grid = sms * kDynCtasPerSm;
    if (partition_size == PA_PARTITION_DYNAMIC && units >= 1 && units <= dyn_grid &&
        units <= kDynMaxUnits && fits32) {
        pl.dynamic = true;
        pl.grid = dyn_grid;
        const size_t recs = (size_t)dyn_grid * G;
        pl.off_us = kDynCounterBytes;
        pl.off_ro = pl.off_us + round_up(((size_t)units + 1) * sizeof(int32_t), 256);
        pl.off_rm = pl.off_ro + round_up(recs * head_dim * sizeof(float), 256);
        pl.off_rl = pl.off_rm + round_up(recs * sizeof(float), 256);
        pl.ws_bytes = pl.off_rl + round_up(recs * sizeof(float), 256);
        pl.partition_tokens = 0;
        pl.num_parts = 0;
        return pl;
    }
    if (want_balanced && balanced_ok) {
        pl.streamk = true;
        const int per_sm = head_dim == 64 ? streamk_ctas_per_sm<64>() : streamk_ctas_per_sm<128>();
        pl.grid = sms * per_sm;
        const size_t recs = (size_t)pl.grid * kSkWarps * 2 * G;  // warp pieces
        const size_t crecs = (size_t)pl.grid * 2 * G;            // CTA records
        const size_t o_bytes = round_up(recs * head_dim * sizeof(float), 256);
        const size_t v_bytes = round_up(recs * sizeof(float), 256);
        const size_t co_bytes = round_up(crecs * head_dim * sizeof(float), 256);
        const size_t cv_bytes = round_up(crecs * sizeof(float), 256);
        pl.off_m = pl.off_o + o_bytes;
        pl.off_l = pl.off_m + v_bytes;
        pl.off_co = pl.off_l + v_bytes;
        pl.off_cm = pl.off_co + co_bytes;
        pl.off_cl = pl.off_cm + cv_bytes;
        pl.off_pre = pl.off_cl + cv_bytes;
        pl.ws_bytes = pl.off_pre + round_up(((size_t)num_seqs + 1) * sizeof(int32_t), 256);
        pl.partition_tokens = 0;
        pl.num_parts = 0;
        return pl;
    }
    long long P;
    if (partition_size > 0)
        P = partition_size;
    else if (bound <= kAutoSingleMax)
        P = round_up((size_t)bound, 64);
    else
        P = (long long)num_seqs * num_kv_heads >= sms ? kAutoSplitTokens : kAutoSplitTokensFew;
    if (P > (1LL << 30)) P = 1LL << 30;
    pl.partition_tokens = (int)P;
    pl.num_parts = (int)((bound + P - 1) / P);
    if (pl.num_parts > 1) {
        const size_t n = (size_t)num_seqs * num_q_heads * pl.num_parts;
        const size_t o_bytes = round_up(n * head_dim * sizeof(float), 256);
        const size_t v_bytes = round_up(n * sizeof(float), 256);
        pl.off_m = pl.off_o + o_bytes;
        pl.off_l = pl.off_m + v_bytes;
        pl.ws_bytes = pl.off_l + v_bytes;
    }
    return pl;
}

// A stride coprime with n (a prime that does not divide it), so that b -> b * stride % n
// permutes [0, n) and scatters consecutive values.
int coprime_stride(int n) {
    for (int pr : {97, 101, 103, 107, 109, 113, 127, 131, 137, 139})
        if (n % pr != 0 && pr < n) return pr;
    return 1;
}

// Launch with programmatic stream serialisation (see pdl_wait_and_release).
template <typename Kern, typename P>
cudaError_t launch_pdl(Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       const P &p) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, p);
    return e != cudaSuccess ? e : cudaGetLastError();
}

int current_device() {
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess) return -1;
    return d;
}

template <typename K>
cudaError_t ensure_smem(K kernel, int bytes, std::atomic<bool> *flags, int dev) {
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (flags[dev].load(std::memory_order_acquire)) return cudaSuccess;
    cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) flags[dev].store(true, std::memory_order_release);
    return e;
}

template <typename T, int D, int G, int BOXR, bool WIN, bool COW = false>
cudaError_t launch_partition(const DecodeParams &p, dim3 grid, cudaStream_t st, int dev) {
    static std::atomic<bool> flags[kMaxDevices];
    auto kernel = pa_decode_partition_kernel<T, D, G, BOXR, WIN, COW>;
    cudaError_t e = ensure_smem(kernel, Geom<D>::kSmem, flags, dev);
    if (e != cudaSuccess) return e;
    return launch_pdl(kernel, grid, dim3(kWarps * 32), Geom<D>::kSmem, st, p);
}

// A host-planned launch: grid (kv heads, units), the unit list in the parameters.
template <typename T, int D, int G, int BOXR>
cudaError_t launch_planned(const PlannedParams &pp, int units, cudaStream_t st, int dev) {
    static std::atomic<bool> flags[kMaxDevices];
    auto kernel = pa_decode_partition_kernel<T, D, G, BOXR, false, false, true>;
    cudaError_t e = ensure_smem(kernel, Geom<D>::kSmem, flags, dev);
    if (e != cudaSuccess) return e;
    return launch_pdl(kernel, dim3((unsigned)pp.base.num_kv_heads, (unsigned)units),
                      dim3(kWarps * 32), Geom<D>::kSmem, st, pp);
}

template <typename T, int D>
cudaError_t planned_group(const PlannedParams &pp, int units, cudaStream_t st, int dev, int G,
                          int boxr) {
    switch (G) {
        case 1: return boxr == 8 ? launch_planned<T, D, 1, 8>(pp, units, st, dev)
                                 : launch_planned<T, D, 1, 16>(pp, units, st, dev);
        case 2: return boxr == 8 ? launch_planned<T, D, 2, 8>(pp, units, st, dev)
                                 : launch_planned<T, D, 2, 16>(pp, units, st, dev);
        case 4: return boxr == 8 ? launch_planned<T, D, 4, 8>(pp, units, st, dev)
                                 : launch_planned<T, D, 4, 16>(pp, units, st, dev);
        case 8: return boxr == 8 ? launch_planned<T, D, 8, 8>(pp, units, st, dev)
                                 : launch_planned<T, D, 8, 16>(pp, units, st, dev);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t planned_dispatch(const PlannedParams &pp, int units, cudaStream_t st, int dev, int D,
                             int G, int boxr) {
    return D == 64 ? planned_group<T, 64>(pp, units, st, dev, G, boxr)
                   : planned_group<T, 128>(pp, units, st, dev, G, boxr);
}

// The (sequence, partition) units of a fixed-split launch from host copies of the context
// lengths, longest first: every full partition (partition-major, so CTAs scheduled together
// read neighbouring heads of the same blocks), then the shorter last partitions by
// decreasing length.  Returns the unit count, or -1 when the plan does not fit (the caller
// then launches the full grid).
int plan_units(const int32_t *lens, int num_seqs, long long cap, int P, int num_parts,
               uint32_t *units) {
    if (num_parts > kPlanMaxParts || num_seqs > 65535) return -1;
    long long total = 0;
    for (int s = 0; s < num_seqs; ++s) {
        long long L = lens[s] < 0 ? 0 : (lens[s] > cap ? cap : lens[s]);
        long long n = L == 0 ? 1 : (L + P - 1) / P;
        total += n < num_parts ? n : num_parts;
    }
    if (total > kPlanMaxUnits) return -1;
    int k = 0;
    for (int part = 0; part < num_parts; ++part)
        for (int s = 0; s < num_seqs; ++s) {
            const long long L = lens[s] < 0 ? 0 : (lens[s] > cap ? cap : lens[s]);
            const long long n = L == 0 ? 1 : (L + P - 1) / P;
            const int np = (int)(n < num_parts ? n : num_parts);
            if (part < np && (long long)(part + 1) * P <= L)
                units[k++] = ((uint32_t)s << 16) | ((uint32_t)part << 8) | (uint32_t)np;
        }
    const int full = k;
    for (int s = 0; s < num_seqs; ++s) {  // the last, shorter partition of each context
        const long long L = lens[s] < 0 ? 0 : (lens[s] > cap ? cap : lens[s]);
        const long long n = L == 0 ? 1 : (L + P - 1) / P;
        const int np = (int)(n < num_parts ? n : num_parts);
        const int last = np - 1;
        if ((long long)(last + 1) * P > L)
            units[k++] = ((uint32_t)s << 16) | ((uint32_t)last << 8) | (uint32_t)np;
    }
    auto rem = [&](uint32_t u) {
        const int s = (int)(u >> 16);
        const long long L = lens[s] < 0 ? 0 : (lens[s] > cap ? cap : lens[s]);
        return L - (long long)((u >> 8) & 0xffu) * P;
    };
    std::stable_sort(units + full, units + k,
                     [&](uint32_t a, uint32_t b) { return rem(a) > rem(b); });
    return k;
}

// The units pa_decode_planned launches for a fixed split, or 0 for the full grid (a
// window, or no empty row to leave out).  Where the plan leaves out at least 30% of the
// grid's rows the units go longest first; otherwise in the full grid's own order without
// its empty rows: partition 0 of every sequence in order, then each later partition index
// longest first.  A/B on B200 against the full grid: GQA (20% of the rows real) -5% and
// long 8/1 (61%) -1 to -2% longest first, where the full grid's order gained nothing;
// Llama-2 (75%) +2% longest first but -2% in the grid's order.
int planned_units(const int32_t *lens, int num_seqs, int max_blocks_per_seq, int block_size,
                  int sliding_window, const Plan &pl, uint32_t *units) {
    if (sliding_window > 0 || pl.streamk || pl.dynamic || pl.partition_tokens <= 0) return 0;
    const int n = plan_units(lens, num_seqs, (long long)max_blocks_per_seq * block_size,
                             pl.partition_tokens, pl.num_parts, units);
    if (n <= 0) return 0;
    if ((long long)n * 10 <= 7LL * num_seqs * pl.num_parts) return n;  // longest first
    if ((long long)n >= (long long)num_seqs * pl.num_parts) return 0;  // no empty row
    const long long cap = (long long)max_blocks_per_seq * block_size;
    const int P = pl.partition_tokens;
    auto size = [&](uint32_t u) {
        const int s = (int)(u >> 16);
        const long long L = lens[s] < 0 ? 0 : (lens[s] > cap ? cap : lens[s]);
        const long long r = L - (long long)((u >> 8) & 0xffu) * P;
        return r < P ? r : (long long)P;
    };
    std::stable_sort(units, units + n, [&](uint32_t a, uint32_t b) {
        const uint32_t pa_ = (a >> 8) & 0xffu, pb = (b >> 8) & 0xffu;
        if (pa_ != pb) return pa_ < pb;
        if (pa_ == 0) return (a >> 16) < (b >> 16);
        return size(a) > size(b);
    });
    return n;
}

template <typename T, int D>
cudaError_t launch_merge(const MergeParams &p, dim3 grid, cudaStream_t st) {
    if (p.num_parts <= kMergeFew)
        return launch_pdl(pa_merge_kernel<T, D, false>, grid, dim3(kMergeThreads), 0, st, p);
    return launch_pdl(pa_merge_kernel<T, D, true>, grid, dim3(kMergeThreads), 0, st, p);
}

template <typename T, int D, int G>
cudaError_t dispatch_boxr(const DecodeParams &p, dim3 grid, cudaStream_t st, int dev, int boxr) {
    if (p.cow != nullptr && p.sliding_window > 0)  // the instances with copy-on-write
        return boxr == 8 ? launch_partition<T, D, G, 8, true, true>(p, grid, st, dev)
                         : launch_partition<T, D, G, 16, true, true>(p, grid, st, dev);
    if (p.cow != nullptr)
        return boxr == 8 ? launch_partition<T, D, G, 8, false, true>(p, grid, st, dev)
                         : launch_partition<T, D, G, 16, false, true>(p, grid, st, dev);
    if (p.sliding_window > 0)
        return boxr == 8 ? launch_partition<T, D, G, 8, true>(p, grid, st, dev)
                         : launch_partition<T, D, G, 16, true>(p, grid, st, dev);
    return boxr == 8 ? launch_partition<T, D, G, 8, false>(p, grid, st, dev)
                     : launch_partition<T, D, G, 16, false>(p, grid, st, dev);
}

template <typename T, int D>
cudaError_t dispatch_group(const DecodeParams &p, dim3 grid, cudaStream_t st, int dev, int G,
                           int boxr) {
    switch (G) {
        case 1: return dispatch_boxr<T, D, 1>(p, grid, st, dev, boxr);
        case 2: return dispatch_boxr<T, D, 2>(p, grid, st, dev, boxr);
        case 4: return dispatch_boxr<T, D, 4>(p, grid, st, dev, boxr);
        case 8: return dispatch_boxr<T, D, 8>(p, grid, st, dev, boxr);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t dispatch_dim(const DecodeParams &p, dim3 grid, cudaStream_t st, int dev, int D,
                         int G, int boxr) {
    return D == 64 ? dispatch_group<T, 64>(p, grid, st, dev, G, boxr)
                   : dispatch_group<T, 128>(p, grid, st, dev, G, boxr);
}

template <typename T, int D, int G, int BOXR>
cudaError_t launch_streamk(const StreamKParams &p, int grid_max, cudaStream_t st, int dev,
                           int *grid_used) {
    static std::atomic<bool> flags[kMaxDevices];
    static std::atomic<int> occ[kMaxDevices];
    auto kernel = pa_decode_streamk_kernel<T, D, G, BOXR>;
    cudaError_t e = ensure_smem(kernel, SkGeom<D>::kSmem, flags, dev);
    if (e != cudaSuccess) return e;
    int n = occ[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kSkWarps * 32,
                                                          SkGeom<D>::kSmem);
        if (e != cudaSuccess || n < 1) return e != cudaSuccess ? e : cudaErrorInvalidConfiguration;
        occ[dev].store(n, std::memory_order_relaxed);
    }
    const int sms = device_sms(dev);
    int grid = sms * n;
    if (grid > grid_max) grid = grid_max;
    *grid_used = grid;
    return launch_pdl(kernel, dim3(grid), dim3(kSkWarps * 32), SkGeom<D>::kSmem, st, p);
}

template <typename T, int D, int G>
cudaError_t sk_dispatch_boxr(const StreamKParams &p, int gmax, cudaStream_t st, int dev, int boxr,
                             int *gu) {
    return boxr == 8 ? launch_streamk<T, D, G, 8>(p, gmax, st, dev, gu)
                     : launch_streamk<T, D, G, 16>(p, gmax, st, dev, gu);
}

template <typename T, int D>
cudaError_t sk_dispatch_group(const StreamKParams &p, int gmax, cudaStream_t st, int dev, int G,
                              int boxr, int *gu) {
    switch (G) {
        case 1: return sk_dispatch_boxr<T, D, 1>(p, gmax, st, dev, boxr, gu);
        case 2: return sk_dispatch_boxr<T, D, 2>(p, gmax, st, dev, boxr, gu);
        case 4: return sk_dispatch_boxr<T, D, 4>(p, gmax, st, dev, boxr, gu);
        case 8: return sk_dispatch_boxr<T, D, 8>(p, gmax, st, dev, boxr, gu);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t sk_dispatch(const StreamKParams &p, int gmax, cudaStream_t st, int dev, int D, int G,
                        int boxr, int *gu) {
    return D == 64 ? sk_dispatch_group<T, 64>(p, gmax, st, dev, G, boxr, gu)
                   : sk_dispatch_group<T, 128>(p, gmax, st, dev, G, boxr, gu);
}

template <typename T>
cudaError_t sk_merge(const SkMergeParams &p, dim3 grid, int D, cudaStream_t st) {
    return D == 64 ? launch_pdl(pa_merge_streamk_kernel<T, 64>, grid, dim3(kMergeThreads), 0, st, p)
                   : launch_pdl(pa_merge_streamk_kernel<T, 128>, grid, dim3(kMergeThreads), 0, st,
                                p);
}

template <typename T, int D, int G, int BOXR>
cudaError_t launch_dynamic(const DynParams &p, int grid, cudaStream_t st, int dev) {
    static std::atomic<bool> flags[kMaxDevices];
    static std::atomic<int> occ[kMaxDevices];
    auto kernel = pa_decode_dynamic_kernel<T, D, G, BOXR>;
    cudaError_t e = ensure_smem(kernel, Geom<D>::kSmem, flags, dev);
    if (e != cudaSuccess) return e;
    int n = occ[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kWarps * 32,
                                                          Geom<D>::kSmem);
        if (e != cudaSuccess) return e;
        occ[dev].store(n, std::memory_order_relaxed);
    }
    // the plan gives every warp two chunks of its own: all CTAs must be resident at once
    if (n < kDynCtasPerSm) return cudaErrorInvalidConfiguration;
    return launch_pdl(kernel, dim3(grid), dim3(kWarps * 32), Geom<D>::kSmem, st, p);
}

template <typename T, int D, int G>
cudaError_t dyn_dispatch_boxr(const DynParams &p, int grid, cudaStream_t st, int dev, int boxr) {
    return boxr == 8 ? launch_dynamic<T, D, G, 8>(p, grid, st, dev)
                     : launch_dynamic<T, D, G, 16>(p, grid, st, dev);
}

template <typename T, int D>
cudaError_t dyn_dispatch_group(const DynParams &p, int grid, cudaStream_t st, int dev, int G,
                               int boxr) {
    switch (G) {
        case 1: return dyn_dispatch_boxr<T, D, 1>(p, grid, st, dev, boxr);
        case 2: return dyn_dispatch_boxr<T, D, 2>(p, grid, st, dev, boxr);
        case 4: return dyn_dispatch_boxr<T, D, 4>(p, grid, st, dev, boxr);
        case 8: return dyn_dispatch_boxr<T, D, 8>(p, grid, st, dev, boxr);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t dyn_dispatch(const DynParams &p, int grid, cudaStream_t st, int dev, int D, int G,
                         int boxr) {
    return D == 64 ? dyn_dispatch_group<T, 64>(p, grid, st, dev, G, boxr)
                   : dyn_dispatch_group<T, 128>(p, grid, st, dev, G, boxr);
}

template <typename T>
cudaError_t dyn_merge(const DynMergeParams &p, dim3 grid, int D, cudaStream_t st) {
    return D == 64 ? launch_pdl(pa_merge_dynamic_kernel<T, 64>, grid, dim3(kMergeThreads), 0, st, p)
                   : launch_pdl(pa_merge_dynamic_kernel<T, 128>, grid, dim3(kMergeThreads), 0, st,
                                p);
}

template <typename T, int D, int G>
cudaError_t launch_prefill(const PrefillParams &p, dim3 grid, cudaStream_t st, int dev) {
    static std::atomic<bool> flags[kMaxDevices];
    auto kernel = pa_prefill_kernel<T, D, G>;
    cudaError_t e = ensure_smem(kernel, PfGeom<D>::kSmem, flags, dev);
    if (e != cudaSuccess) return e;
    return launch_pdl(kernel, grid, dim3(kPfThreads), PfGeom<D>::kSmem, st, p);
}

template <typename T, int D>
cudaError_t prefill_dispatch_group(const PrefillParams &p, dim3 grid, cudaStream_t st, int dev,
                                   int G) {
    switch (G) {
        case 1: return launch_prefill<T, D, 1>(p, grid, st, dev);
        case 2: return launch_prefill<T, D, 2>(p, grid, st, dev);
        case 4: return launch_prefill<T, D, 4>(p, grid, st, dev);
        case 8: return launch_prefill<T, D, 8>(p, grid, st, dev);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t prefill_dispatch(const PrefillParams &p, dim3 grid, cudaStream_t st, int dev, int D,
                             int G) {
    return D == 64 ? prefill_dispatch_group<T, 64>(p, grid, st, dev, G)
                   : prefill_dispatch_group<T, 128>(p, grid, st, dev, G);
}

pa_status check_decode_shape(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                             int block_size, int num_blocks, int max_blocks_per_seq,
                             int max_context_len, int sliding_window, int partition_size) {
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 ||
        max_blocks_per_seq <= 0 || max_context_len < 0 || sliding_window < 0 ||
        partition_size < PA_PARTITION_DYNAMIC)
        return PA_ERR_INVALID_ARG;
    if (num_q_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
    const int G = num_q_heads / num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return PA_ERR_UNSUPPORTED;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (!pow2(block_size) || block_size < 8 || block_size > 512) return PA_ERR_UNSUPPORTED;
    if (partition_size > 0 && partition_size % 64 != 0) return PA_ERR_INVALID_ARG;
    if ((unsigned long long)num_blocks * num_kv_heads * block_size >= (1ull << 31))
        return PA_ERR_UNSUPPORTED;
    if ((long long)max_blocks_per_seq * block_size >= (1ll << 31)) return PA_ERR_INVALID_ARG;
    if (num_seqs > 65535 || num_kv_heads > 65535) return PA_ERR_UNSUPPORTED;
    return PA_OK;
}

}  // namespace

extern "C" {

int pa_version(void) { return 201; }

const char *pa_status_str(pa_status s) {
    switch (s) {
        case PA_OK: return "ok";
        case PA_ERR_INVALID_ARG: return "invalid argument";
        case PA_ERR_UNSUPPORTED: return "unsupported configuration";
        case PA_ERR_CUDA: return "CUDA runtime error";
        case PA_ERR_OUT_OF_RANGE: return "index out of range (device error word)";
        case PA_ERR_TIMEOUT: return "bounded wait expired (device error word)";
        case PA_ERR_NO_FREE_BLOCK: return "no free block in the pool";
        case PA_ERR_HOST_ALLOC: return "host memory allocation failed";
    }
    return "unknown status";
}

pa_status pa_get_device_error(int device, uint32_t *bits_out, int clear) {
    if (!bits_out) return PA_ERR_INVALID_ARG;
    int prev = 0;
    if (cudaGetDevice(&prev) != cudaSuccess) return PA_ERR_CUDA;
    if (cudaSetDevice(device) != cudaSuccess) return PA_ERR_INVALID_ARG;
    pa_status st = PA_OK;
    unsigned int v = 0;
    if (cudaDeviceSynchronize() != cudaSuccess ||
        cudaMemcpyFromSymbol(&v, g_error_word, sizeof v) != cudaSuccess) {
        st = PA_ERR_CUDA;
    } else if (clear) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof zero) != cudaSuccess) st = PA_ERR_CUDA;
    }
    *bits_out = v;
    cudaSetDevice(prev);
    return st;
}

pa_status pa_kv_write(const void *key, const void *value, const int64_t *slot_mapping,
                      int num_tokens, int num_kv_heads, int head_dim, int64_t key_token_stride,
                      int64_t value_token_stride, void *k_cache, void *v_cache, int num_blocks,
                      int block_size, pa_dtype dtype, void *stream) {
    if (dtype != PA_FP16 && dtype != PA_BF16) return PA_ERR_INVALID_ARG;
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || head_dim % 8 != 0 ||
        num_blocks <= 0 || block_size <= 0)
        return PA_ERR_INVALID_ARG;
    if (num_tokens == 0) return PA_OK;
    if (!key || !value || !slot_mapping || !k_cache || !v_cache) return PA_ERR_INVALID_ARG;
    if (!aligned(key, 16) || !aligned(value, 16) || !aligned(k_cache, 16) ||
        !aligned(v_cache, 16) || !aligned(slot_mapping, 8))
        return PA_ERR_INVALID_ARG;
    if (key_token_stride % 8 != 0 || value_token_stride % 8 != 0 ||
        key_token_stride < (int64_t)num_kv_heads * head_dim ||
        value_token_stride < (int64_t)num_kv_heads * head_dim)
        return PA_ERR_INVALID_ARG;
    KvWriteParams p;
    p.key = static_cast<const uint8_t *>(key);
    p.value = static_cast<const uint8_t *>(value);
    p.slot_mapping = slot_mapping;
    p.k_cache = static_cast<uint8_t *>(k_cache);
    p.v_cache = static_cast<uint8_t *>(v_cache);
    p.key_stride_b = (long long)key_token_stride * 2;
    p.value_stride_b = (long long)value_token_stride * 2;
    p.num_slots = (long long)num_blocks * block_size;
    p.num_tokens = num_tokens;
    p.num_kv_heads = num_kv_heads;
    p.row_chunks = head_dim / 8;
    p.block_size = block_size;
    const long long total = (long long)num_tokens * num_kv_heads * p.row_chunks;
    if (total >= (1ll << 31)) return PA_ERR_UNSUPPORTED;  // split the call
    const long long per_cta = (long long)kKvwThreads * kKvwUnroll;
    const unsigned grid = (unsigned)((total + per_cta - 1) / per_cta);
    return launch_pdl(pa_kv_write_kernel, dim3(grid), dim3(kKvwThreads), 0,
                      static_cast<cudaStream_t>(stream), p) == cudaSuccess
               ? PA_OK
               : PA_ERR_CUDA;
}

pa_status pa_copy_blocks(void *k_cache, void *v_cache, const int64_t *src_dst_pairs,
                         int num_pairs, int num_kv_heads, int block_size, int head_dim,
                         int num_blocks, pa_dtype dtype, void *stream) {
    if (dtype != PA_FP16 && dtype != PA_BF16) return PA_ERR_INVALID_ARG;
    if (num_pairs < 0 || num_kv_heads <= 0 || block_size <= 0 || head_dim <= 0 || num_blocks <= 0)
        return PA_ERR_INVALID_ARG;
    if (num_pairs == 0) return PA_OK;
    if (!k_cache || !v_cache || !src_dst_pairs) return PA_ERR_INVALID_ARG;
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(src_dst_pairs, 8))
        return PA_ERR_INVALID_ARG;
    const long long elems = (long long)num_kv_heads * block_size * head_dim;
    if (elems % 8 != 0) return PA_ERR_INVALID_ARG;
    CopyBlocksParams p;
    p.k_cache = static_cast<uint8_t *>(k_cache);
    p.v_cache = static_cast<uint8_t *>(v_cache);
    p.pairs = src_dst_pairs;
    p.block_chunks = elems / 8;
    p.num_blocks = num_blocks;
    p.num_pairs = num_pairs;
    const long long per_cta = (long long)kCopyThreads * kCopyUnroll;
    const long long chunks = (p.block_chunks + per_cta - 1) / per_cta;
    if (chunks > 65535 || num_pairs > 65535) return PA_ERR_UNSUPPORTED;
    dim3 grid((unsigned)chunks, (unsigned)num_pairs, 2);
    return launch_pdl(pa_copy_blocks_kernel, grid, dim3(kCopyThreads), 0,
                      static_cast<cudaStream_t>(stream), p) == cudaSuccess
               ? PA_OK
               : PA_ERR_CUDA;
}

pa_status pa_swap_blocks(void *dst_k_cache, void *dst_v_cache, const void *src_k_cache,
                         const void *src_v_cache, const int64_t *src_dst_pairs, int num_pairs,
                         int num_kv_heads, int block_size, int head_dim, int src_num_blocks,
                         int dst_num_blocks, pa_dtype dtype, void *stream) {
    if (dtype != PA_FP16 && dtype != PA_BF16) return PA_ERR_INVALID_ARG;
    if (num_pairs < 0 || num_kv_heads <= 0 || block_size <= 0 || head_dim <= 0 ||
        src_num_blocks <= 0 || dst_num_blocks <= 0)
        return PA_ERR_INVALID_ARG;
    if (num_pairs == 0) return PA_OK;
    if (!dst_k_cache || !dst_v_cache || !src_k_cache || !src_v_cache || !src_dst_pairs)
        return PA_ERR_INVALID_ARG;
    if (!aligned(dst_k_cache, 16) || !aligned(dst_v_cache, 16) || !aligned(src_k_cache, 16) ||
        !aligned(src_v_cache, 16) || !aligned(src_dst_pairs, 8))
        return PA_ERR_INVALID_ARG;
    const long long elems = (long long)num_kv_heads * block_size * head_dim;
    if (elems % 8 != 0) return PA_ERR_INVALID_ARG;
    // Every pointer must be reachable by the kernel at that address: device memory,
    // managed memory, or pinned host memory mapped into the unified address space.
    // Anything else (pageable host memory) is refused here, before any launch.
    for (const void *ptr : {static_cast<const void *>(dst_k_cache),
                            static_cast<const void *>(dst_v_cache), src_k_cache, src_v_cache,
                            static_cast<const void *>(src_dst_pairs)}) {
        cudaPointerAttributes a;
        if (cudaPointerGetAttributes(&a, ptr) != cudaSuccess) {
            cudaGetLastError();
            return PA_ERR_INVALID_ARG;
        }
        const bool ok = a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged ||
                        (a.type == cudaMemoryTypeHost && a.devicePointer == ptr);
        if (!ok) return PA_ERR_INVALID_ARG;
    }
    SwapBlocksParams p;
    p.dst_k = static_cast<uint8_t *>(dst_k_cache);
    p.dst_v = static_cast<uint8_t *>(dst_v_cache);
    p.src_k = static_cast<const uint8_t *>(src_k_cache);
    p.src_v = static_cast<const uint8_t *>(src_v_cache);
    p.pairs = src_dst_pairs;
    p.block_chunks = elems / 8;
    p.src_blocks = src_num_blocks;
    p.dst_blocks = dst_num_blocks;
    const long long per_cta = (long long)kCopyThreads * kCopyUnroll;
    const long long chunks = (p.block_chunks + per_cta - 1) / per_cta;
    if (chunks > 65535) return PA_ERR_UNSUPPORTED;
    dim3 grid((unsigned)num_pairs, (unsigned)chunks, 2);
    return launch_pdl(pa_swap_blocks_kernel, grid, dim3(kCopyThreads), 0,
                      static_cast<cudaStream_t>(stream), p) == cudaSuccess
               ? PA_OK
               : PA_ERR_CUDA;
}

size_t pa_decode_workspace_bytes(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                 int block_size, int max_blocks_per_seq, int max_context_len,
                                 int sliding_window, int partition_size) {
    if (num_seqs <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        block_size <= 0 || max_blocks_per_seq <= 0 || partition_size < PA_PARTITION_DYNAMIC ||
        max_context_len < 0 || sliding_window < 0)
        return 0;
    return make_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                     max_blocks_per_seq, max_context_len, sliding_window, partition_size,
                     device_sms(current_device_or_zero()))
        .ws_bytes;
}

int pa_decode_partition_tokens(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                               int block_size, int max_blocks_per_seq, int max_context_len,
                               int sliding_window, int partition_size) {
    if (num_kv_heads <= 0 || block_size <= 0 || max_blocks_per_seq <= 0 ||
        partition_size < PA_PARTITION_DYNAMIC || max_context_len < 0 || sliding_window < 0)
        return 0;
    return make_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                     max_blocks_per_seq, max_context_len, sliding_window, partition_size,
                     device_sms(current_device_or_zero()))
        .partition_tokens;
}

}  // extern "C"

namespace {

// pa_decode, optionally with the step's cache write fused in (new_k != nullptr).
pa_status decode_impl(void *out, const void *q, const void *k_cache, const void *v_cache,
                      const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                      int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                      int num_blocks, int max_blocks_per_seq, float scale, int max_context_len,
                      int sliding_window, int partition_size, void *workspace,
                      size_t workspace_bytes, pa_dtype dtype, void *stream, const void *new_k,
                      const void *new_v, long long new_k_stride, long long new_v_stride,
                      const int32_t *cow = nullptr, const int32_t *host_lens = nullptr) {
    if (dtype != PA_FP16 && dtype != PA_BF16) return PA_ERR_INVALID_ARG;
    pa_status st = check_decode_shape(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                      num_blocks, max_blocks_per_seq, max_context_len,
                                      sliding_window, partition_size);
    if (st != PA_OK) return st;
    if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
    if (num_seqs == 0) return PA_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
        return PA_ERR_INVALID_ARG;
    if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(block_tables, 4) || !aligned(context_lens, 4))
        return PA_ERR_INVALID_ARG;
    const int dev = current_device();
    const Plan pl = make_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                              max_blocks_per_seq, max_context_len, sliding_window,
                              partition_size, device_sms(dev));
    if (pl.ws_bytes > 0 &&
        (!workspace || !aligned(workspace, 256) || workspace_bytes < pl.ws_bytes))
        return PA_ERR_INVALID_ARG;

    const int G = num_q_heads / num_kv_heads;
    const int boxr = block_size < 16 ? block_size : 16;
    cudaStream_t st_ = static_cast<cudaStream_t>(stream);
    const unsigned long long rows = (unsigned long long)num_blocks * num_kv_heads * block_size;
    if (pl.streamk && new_k != nullptr) return PA_ERR_UNSUPPORTED;  // fixed split only
    if ((pl.streamk || pl.dynamic) && cow != nullptr) return PA_ERR_UNSUPPORTED;
    if (pl.streamk) {
        StreamKParams sp;
        std::memset(&sp, 0, sizeof sp);
        if (!make_cache_map(&sp.kmap, k_cache, rows, head_dim, dtype, boxr) ||
            !make_cache_map(&sp.vmap, v_cache, rows, head_dim, dtype, boxr))
            return PA_ERR_CUDA;
        uint8_t *ws = static_cast<uint8_t *>(workspace);
        sp.out = out;
        sp.q = q;
        sp.block_tables = block_tables;
        sp.context_lens = context_lens;
        sp.rec_o = reinterpret_cast<float *>(ws + pl.off_o);
        sp.rec_m = reinterpret_cast<float *>(ws + pl.off_m);
        sp.rec_l = reinterpret_cast<float *>(ws + pl.off_l);
        sp.crec_o = reinterpret_cast<float *>(ws + pl.off_co);
        sp.crec_m = reinterpret_cast<float *>(ws + pl.off_cm);
        sp.crec_l = reinterpret_cast<float *>(ws + pl.off_cl);
        sp.ws_pre = reinterpret_cast<int32_t *>(ws + pl.off_pre);
        sp.num_seqs = num_seqs;
        sp.num_q_heads = num_q_heads;
        sp.num_kv_heads = num_kv_heads;
        sp.block_size = block_size;
        sp.bs_shift = ilog2_host(block_size);
        sp.num_blocks = num_blocks;
        sp.max_blocks_per_seq = max_blocks_per_seq;
        sp.sliding_window = sliding_window;
        sp.scale_log2 = scale * 1.4426950408889634f;
        int grid_used = 0;
        cudaError_t e = dtype == PA_BF16
                            ? sk_dispatch<__nv_bfloat16>(sp, pl.grid, st_, dev, head_dim, G, boxr,
                                                         &grid_used)
                            : sk_dispatch<__half>(sp, pl.grid, st_, dev, head_dim, G, boxr,
                                                  &grid_used);
        if (e != cudaSuccess) return PA_ERR_CUDA;
        SkMergeParams mp;
        mp.out = out;
        mp.ws_pre = sp.ws_pre;
        mp.rec_o = sp.crec_o;
        mp.rec_m = sp.crec_m;
        mp.rec_l = sp.crec_l;
        mp.num_seqs = num_seqs;
        mp.num_q_heads = num_q_heads;
        mp.num_kv_heads = num_kv_heads;
        mp.num_workers = grid_used;  // records are per CTA
        dim3 mgrid((unsigned)num_q_heads, (unsigned)num_seqs);
        e = dtype == PA_BF16 ? sk_merge<__nv_bfloat16>(mp, mgrid, head_dim, st_)
                             : sk_merge<__half>(mp, mgrid, head_dim, st_);
        return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
    }

    if (pl.dynamic) {
        DynParams dp;
        std::memset(&dp, 0, sizeof dp);
        if (!make_cache_map(&dp.kmap, k_cache, rows, head_dim, dtype, boxr) ||
            !make_cache_map(&dp.vmap, v_cache, rows, head_dim, dtype, boxr))
            return PA_ERR_CUDA;
        uint8_t *ws = static_cast<uint8_t *>(workspace);
        dp.out = out;
        dp.q = q;
        dp.block_tables = block_tables;
        dp.context_lens = context_lens;
        dp.claim = reinterpret_cast<int32_t *>(ws);
        dp.done = dp.claim + kDynMaxUnits;
        dp.ustart = reinterpret_cast<int32_t *>(ws + pl.off_us);
        dp.rec_o = reinterpret_cast<float *>(ws + pl.off_ro);
        dp.rec_m = reinterpret_cast<float *>(ws + pl.off_rm);
        dp.rec_l = reinterpret_cast<float *>(ws + pl.off_rl);
        dp.num_seqs = num_seqs;
        dp.num_q_heads = num_q_heads;
        dp.num_kv_heads = num_kv_heads;
        dp.block_size = block_size;
        dp.bs_shift = ilog2_host(block_size);
        dp.num_blocks = num_blocks;
        dp.max_blocks_per_seq = max_blocks_per_seq;
        dp.sliding_window = sliding_window;
        dp.cta_stride = coprime_stride(pl.grid);
        dp.scale_log2 = scale * 1.4426950408889634f;
        dp.new_k = new_k;
        dp.new_v = new_v;
        dp.new_k_stride = new_k_stride;
        dp.new_v_stride = new_v_stride;
        dp.k_cache = const_cast<void *>(k_cache);
        dp.v_cache = const_cast<void *>(v_cache);
        cudaError_t e = dtype == PA_BF16
                            ? dyn_dispatch<__nv_bfloat16>(dp, pl.grid, st_, dev, head_dim, G, boxr)
                            : dyn_dispatch<__half>(dp, pl.grid, st_, dev, head_dim, G, boxr);
        if (e != cudaSuccess) return PA_ERR_CUDA;
        DynMergeParams mp;
        mp.out = out;
        mp.context_lens = context_lens;
        mp.claim = dp.claim;
        mp.done = dp.done;
        mp.ustart = dp.ustart;
        mp.rec_o = dp.rec_o;
        mp.rec_m = dp.rec_m;
        mp.rec_l = dp.rec_l;
        mp.num_q_heads = num_q_heads;
        mp.num_kv_heads = num_kv_heads;
        mp.cap = max_blocks_per_seq * block_size;
        mp.sliding_window = sliding_window;
        dim3 mgrid((unsigned)num_q_heads, (unsigned)num_seqs);
        e = dtype == PA_BF16 ? dyn_merge<__nv_bfloat16>(mp, mgrid, head_dim, st_)
                             : dyn_merge<__half>(mp, mgrid, head_dim, st_);
        return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
    }

    DecodeParams p;
    std::memset(&p, 0, sizeof p);
    if (!make_cache_map(&p.kmap, k_cache, rows, head_dim, dtype, boxr) ||
        !make_cache_map(&p.vmap, v_cache, rows, head_dim, dtype, boxr))
        return PA_ERR_CUDA;
    p.out = out;
    p.q = q;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    if (pl.ws_bytes > 0) {
        uint8_t *ws = static_cast<uint8_t *>(workspace);
        p.ws_o = reinterpret_cast<float *>(ws + pl.off_o);
        p.ws_m = reinterpret_cast<float *>(ws + pl.off_m);
        p.ws_l = reinterpret_cast<float *>(ws + pl.off_l);
    }
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.block_size = block_size;
    p.bs_shift = ilog2_host(block_size);
    p.num_blocks = num_blocks;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.partition_tokens = pl.partition_tokens;
    p.num_parts = pl.num_parts;
    p.sliding_window = sliding_window;
    p.rotate = block_size >= kRotateMinBlock ? 1 : 0;
    p.sort_second = (pl.num_parts == 2 && num_seqs <= kSortMaxSeqs) ? 1 : 0;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.new_k = new_k;
    p.new_v = new_v;
    p.new_k_stride = new_k_stride;
    p.new_v_stride = new_v_stride;
    p.k_cache = const_cast<void *>(k_cache);
    p.v_cache = const_cast<void *>(v_cache);
    p.cow = cow;

    if (pl.num_parts > 65535) return PA_ERR_UNSUPPORTED;  // use a larger partition_size
    cudaError_t e = cudaSuccess;
    bool launched = false;
    if (host_lens != nullptr && cow == nullptr) {
        // the units that exist, longest first, from the host's copy of the lengths
        PlannedParams pp;
        const int units = planned_units(host_lens, num_seqs, max_blocks_per_seq, block_size,
                                        sliding_window, pl, pp.units);
        if (units > 0) {
            pp.base = p;
            pp.base.sort_second = 0;
            e = dtype == PA_BF16
                    ? planned_dispatch<__nv_bfloat16>(pp, units, st_, dev, head_dim, G, boxr)
                    : planned_dispatch<__half>(pp, units, st_, dev, head_dim, G, boxr);
            launched = true;
        }
    }
    if (!launched) {
        dim3 grid((unsigned)num_kv_heads, (unsigned)num_seqs, (unsigned)pl.num_parts);
        e = dtype == PA_BF16 ? dispatch_dim<__nv_bfloat16>(p, grid, st_, dev, head_dim, G, boxr)
                             : dispatch_dim<__half>(p, grid, st_, dev, head_dim, G, boxr);
    }
    if (e != cudaSuccess) return PA_ERR_CUDA;
    if (pl.num_parts > 1) {
        MergeParams mp;
        mp.out = out;
        mp.context_lens = context_lens;
        mp.ws_o = p.ws_o;
        mp.ws_m = p.ws_m;
        mp.ws_l = p.ws_l;
        mp.num_q_heads = num_q_heads;
        mp.cap = max_blocks_per_seq * block_size;
        mp.partition_tokens = pl.partition_tokens;
        mp.num_parts = pl.num_parts;
        mp.sliding_window = sliding_window;
        dim3 mgrid((unsigned)num_q_heads, (unsigned)num_seqs);
        if (dtype == PA_BF16)
            e = head_dim == 64 ? launch_merge<__nv_bfloat16, 64>(mp, mgrid, st_)
                               : launch_merge<__nv_bfloat16, 128>(mp, mgrid, st_);
        else
            e = head_dim == 64 ? launch_merge<__half, 64>(mp, mgrid, st_)
                               : launch_merge<__half, 128>(mp, mgrid, st_);
        if (e != cudaSuccess) return PA_ERR_CUDA;
    }
    return PA_OK;
}

}  // namespace

extern "C" {

pa_status pa_decode(void *out, const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                    int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                    int num_blocks, int max_blocks_per_seq, float scale, int max_context_len,
                    int sliding_window, int partition_size, void *workspace,
                    size_t workspace_bytes, pa_dtype dtype, void *stream) {
    return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs,
                       num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                       max_blocks_per_seq, scale, max_context_len, sliding_window,
                       partition_size, workspace, workspace_bytes, dtype, stream, nullptr,
                       nullptr, 0, 0);
}

pa_status pa_decode_append(void *out, const void *q, const void *key, const void *value,
                           int64_t key_token_stride, int64_t value_token_stride, void *k_cache,
                           void *v_cache, const int32_t *block_tables,
                           const int32_t *context_lens, int num_seqs, int num_q_heads,
                           int num_kv_heads, int head_dim, int block_size, int num_blocks,
                           int max_blocks_per_seq, float scale, int max_context_len,
                           int sliding_window, int partition_size, void *workspace,
                           size_t workspace_bytes, pa_dtype dtype, void *stream) {
    if (num_seqs > 0) {
        if (!key || !value || !aligned(key, 16) || !aligned(value, 16)) return PA_ERR_INVALID_ARG;
        if (key_token_stride % 8 != 0 || value_token_stride % 8 != 0 ||
            key_token_stride < (int64_t)num_kv_heads * head_dim ||
            value_token_stride < (int64_t)num_kv_heads * head_dim)
            return PA_ERR_INVALID_ARG;
    }
    return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs,
                       num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                       max_blocks_per_seq, scale, max_context_len, sliding_window,
                       partition_size, workspace, workspace_bytes, dtype, stream, key, value,
                       key_token_stride, value_token_stride);
}

pa_status pa_decode_planned(void *out, const void *q, const void *key, const void *value,
                            int64_t key_token_stride, int64_t value_token_stride,
                            void *k_cache, void *v_cache, const int32_t *block_tables,
                            const int32_t *context_lens, const int32_t *host_context_lens,
                            int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                            int block_size, int num_blocks, int max_blocks_per_seq, float scale,
                            int max_context_len, int sliding_window, int partition_size,
                            void *workspace, size_t workspace_bytes, pa_dtype dtype,
                            void *stream) {
    if (num_seqs > 0) {
        if (!host_context_lens) return PA_ERR_INVALID_ARG;
        if ((key == nullptr) != (value == nullptr)) return PA_ERR_INVALID_ARG;
        if (key != nullptr) {
            if (!aligned(key, 16) || !aligned(value, 16)) return PA_ERR_INVALID_ARG;
            if (key_token_stride % 8 != 0 || value_token_stride % 8 != 0 ||
                key_token_stride < (int64_t)num_kv_heads * head_dim ||
                value_token_stride < (int64_t)num_kv_heads * head_dim)
                return PA_ERR_INVALID_ARG;
        }
    }
    return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs,
                       num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                       max_blocks_per_seq, scale, max_context_len, sliding_window,
                       partition_size, workspace, workspace_bytes, dtype, stream, key, value,
                       key != nullptr ? key_token_stride : 0,
                       value != nullptr ? value_token_stride : 0, nullptr, host_context_lens);
}

int pa_decode_planned_units(const int32_t *host_context_lens, int num_seqs, int num_q_heads,
                            int num_kv_heads, int head_dim, int block_size,
                            int max_blocks_per_seq, int max_context_len, int sliding_window,
                            int partition_size, uint32_t *units, int max_units) {
    if (check_decode_shape(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, 1,
                           max_blocks_per_seq, max_context_len, sliding_window,
                           partition_size) != PA_OK ||
        (num_seqs > 0 && !host_context_lens) || max_units < 0 || (max_units > 0 && !units))
        return -1;
    if (num_seqs == 0) return 0;
    const Plan pl = make_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                              max_blocks_per_seq, max_context_len, sliding_window,
                              partition_size, device_sms(current_device_or_zero()));
    static thread_local uint32_t buf[kPlanMaxUnits];
    const int n = planned_units(host_context_lens, num_seqs, max_blocks_per_seq, block_size,
                                sliding_window, pl, buf);
    for (int i = 0; i < n && i < max_units; ++i) units[i] = buf[i];
    return n;
}

pa_status pa_decode_cow(void *out, const void *q, const void *key, const void *value,
                        int64_t key_token_stride, int64_t value_token_stride, void *k_cache,
                        void *v_cache, const int32_t *block_tables, const int32_t *context_lens,
                        const int32_t *cow, int num_seqs, int num_q_heads, int num_kv_heads,
                        int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
                        float scale, int max_context_len, int sliding_window,
                        int partition_size, void *workspace, size_t workspace_bytes,
                        pa_dtype dtype, void *stream) {
    if (num_seqs > 0) {
        if (!cow || !aligned(cow, 4)) return PA_ERR_INVALID_ARG;
        if ((key == nullptr) != (value == nullptr)) return PA_ERR_INVALID_ARG;
        if (key != nullptr) {
            if (!aligned(key, 16) || !aligned(value, 16)) return PA_ERR_INVALID_ARG;
            if (key_token_stride % 8 != 0 || value_token_stride % 8 != 0 ||
                key_token_stride < (int64_t)num_kv_heads * head_dim ||
                value_token_stride < (int64_t)num_kv_heads * head_dim)
                return PA_ERR_INVALID_ARG;
        }
    }
    return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs,
                       num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                       max_blocks_per_seq, scale, max_context_len, sliding_window,
                       partition_size, workspace, workspace_bytes, dtype, stream, key, value,
                       key != nullptr ? key_token_stride : 0,
                       value != nullptr ? value_token_stride : 0, cow);
}

}  // extern "C"

// ------------------------------------------------------------------------------
// Decode without any allocation: the split-K partials live in a scratch array the
// library holds in device memory (one copy per GPU that loads the library, kept
// until the process exits).  Host code cannot use the array's name as a device
// address, so the address is looked up once per device with cudaGetSymbolAddress
// while that device is current, and passed to the kernels as their workspace.

static __device__ __align__(256) unsigned char pa_static_scratch[PA_STATIC_SCRATCH_BYTES];

namespace {

std::mutex g_static_scratch_mu;
void *g_static_scratch_addr[kMaxDevices];

pa_status static_scratch_address(int dev, void **addr) {
    if (dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_static_scratch_mu);
    if (g_static_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, pa_static_scratch) != cudaSuccess || p == nullptr)
            return PA_ERR_CUDA;
        g_static_scratch_addr[dev] = p;
    }
    *addr = g_static_scratch_addr[dev];
    return PA_OK;
}

}  // namespace

extern "C" pa_status pa_decode_static_scratch(
    void *out, const void *q, const void *k_cache, const void *v_cache,
    const int32_t *block_tables, const int32_t *context_lens, int num_seqs, int num_q_heads,
    int num_kv_heads, int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
    float scale, int max_context_len, int sliding_window, int partition_size, pa_dtype dtype,
    void *stream) {
    if (dtype != PA_FP16 && dtype != PA_BF16) return PA_ERR_INVALID_ARG;
    pa_status st = check_decode_shape(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                      num_blocks, max_blocks_per_seq, max_context_len,
                                      sliding_window, partition_size);
    if (st != PA_OK) return st;
    if (num_seqs == 0) return PA_OK;
    const Plan pl = make_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                              max_blocks_per_seq, max_context_len, sliding_window,
                              partition_size, device_sms(current_device_or_zero()));
    if (pl.ws_bytes > PA_STATIC_SCRATCH_BYTES) return PA_ERR_INVALID_ARG;  // over the limit
    void *scratch = nullptr;
    if (pl.ws_bytes > 0) {
        const int dev = current_device();
        st = static_scratch_address(dev, &scratch);
        if (st != PA_OK) return st;
    }
    return pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs, num_q_heads,
                     num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq, scale,
                     max_context_len, sliding_window, partition_size, scratch,
                     pl.ws_bytes > 0 ? (size_t)PA_STATIC_SCRATCH_BYTES : 0, dtype, stream);
}

// ------------------------------------------------------------------------------
// Multi-query (prefill / chunked prefill) attention on the tcgen05 tensor cores.

extern "C" pa_status pa_prefill(void *out, const void *q, const void *k_cache,
                                const void *v_cache, const int32_t *block_tables,
                                const int32_t *context_lens, const int32_t *query_start_loc,
                                int num_seqs, int num_tokens, int num_q_heads, int num_kv_heads,
                                int head_dim, int block_size, int num_blocks,
                                int max_blocks_per_seq, float scale, int sliding_window,
                                pa_dtype dtype, void *stream) {
    if (dtype != PA_FP16 && dtype != PA_BF16) return PA_ERR_INVALID_ARG;
    if (num_seqs < 0 || num_tokens < 0 || num_q_heads <= 0 || num_kv_heads <= 0 ||
        num_blocks <= 0 || max_blocks_per_seq <= 0 || sliding_window < 0 ||
        !std::isfinite(scale) || !(scale > 0.f))
        return PA_ERR_INVALID_ARG;
    if (num_q_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
    const int G = num_q_heads / num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return PA_ERR_UNSUPPORTED;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (!pow2(block_size) || block_size < 8 || block_size > 512) return PA_ERR_UNSUPPORTED;
    if ((unsigned long long)num_blocks * num_kv_heads * block_size >= (1ull << 31))
        return PA_ERR_UNSUPPORTED;
    if ((long long)max_blocks_per_seq * block_size >= (1ll << 31)) return PA_ERR_INVALID_ARG;
    if (num_kv_heads > 65535) return PA_ERR_UNSUPPORTED;
    if (num_seqs == 0 || num_tokens == 0) return PA_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start_loc)
        return PA_ERR_INVALID_ARG;
    if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(block_tables, 4) || !aligned(context_lens, 4) || !aligned(query_start_loc, 4))
        return PA_ERR_INVALID_ARG;
    const int dev = current_device();
    PrefillParams p;
    std::memset(&p, 0, sizeof p);
    const int boxr = block_size < kPfKeys ? block_size : kPfKeys;
    const unsigned long long rows = (unsigned long long)num_blocks * num_kv_heads * block_size;
    if (!make_q_map(&p.qmap, q, num_tokens, num_q_heads, head_dim, G, dtype) ||
        !make_cache_map(&p.kmap, k_cache, rows, head_dim, dtype, boxr) ||
        !make_cache_map(&p.vmap, v_cache, rows, head_dim, dtype, boxr))
        return PA_ERR_CUDA;
    p.out = out;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.query_start_loc = query_start_loc;
    p.num_seqs = num_seqs;
    p.num_tokens = num_tokens;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.block_size = block_size;
    p.bs_shift = ilog2_host(block_size);
    p.box_rows = boxr;
    p.num_blocks = num_blocks;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.sliding_window = sliding_window;
    p.scale_log2 = scale * 1.4426950408889634f;
    // a CTA takes two query tiles of tpt tokens: sum over sequences of
    // ceil(ceil(n_s / tpt) / 2) <= num_tokens / (2 tpt) + num_seqs
    const long long tpt = kPfRows / G;
    const long long pairs = (long long)num_tokens / (2 * tpt) + num_seqs;
    if (pairs >= (1ll << 31)) return PA_ERR_UNSUPPORTED;
    p.heads_inner = pairs <= 65535 ? 1 : 0;
    const dim3 grid = p.heads_inner ? dim3((unsigned)num_kv_heads, (unsigned)pairs)
                                    : dim3((unsigned)pairs, (unsigned)num_kv_heads);
    cudaStream_t st_ = static_cast<cudaStream_t>(stream);
    const cudaError_t e = dtype == PA_BF16
                              ? prefill_dispatch<__nv_bfloat16>(p, grid, st_, dev, head_dim, G)
                              : prefill_dispatch<__half>(p, grid, st_, dev, head_dim, G);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
