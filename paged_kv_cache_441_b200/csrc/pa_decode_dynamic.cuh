// Dynamic split of paged decode attention, for a few long contexts.
//
// What is computed is the decode of pa_decode.cuh ("IO-5 vLLM Paged Attention" note,
// sections 3-4): out[s][h] = softmax_t(scale * q[s][h] . K_s[t]) V_s[t] over the
// sequence's pages in block-table order.  Only the division of the work differs.
//
// When there are fewer (sequence s, kv head g) units than the GPU holds CTAs, a fixed
// split leaves each CTA a long, equal share of one context, and the call ends when the
// slowest SM has streamed its share: B200 SMs differ in streaming rate by about +-10%,
// so a ~50 us call loses several microseconds to that tail.  Here the grid is
// persistent (as many CTAs as are resident at once) and the work is handed out while
// it runs:
//
//  * Every CTA computes the same plan from the context lengths: unit u gets
//    n_u >= 1 CTAs, in proportion to its 16-token tiles (start(u) = u +
//    floor((C - U) * tiles before u / all tiles), C CTAs, U units).
//  * A unit's tiles form chunks of kDynChunk tiles.  Warp r of the unit's
//    NW = 4 n_u warps first takes chunks r and r + NW, then claims chunk
//    2 NW + atomicAdd(claim[u], 1) until the claims run past the end.  A claim is
//    issued one chunk ahead, and each chunk's table entries are loaded a chunk ahead,
//    so neither latency stalls the warp's TMA ring (the ring of pa_decode.cuh: per-warp
//    stages of K and V tiles, one mbarrier each).  Warps on faster SMs simply claim
//    more chunks, and every warp of a unit ends within about one chunk of the others.
//  * A warp keeps one online-softmax state for all of its chunks (they all belong to
//    the unit), the CTA merges its warps in shared memory, and writes one fp32 record
//    (m, l, O/l) -- or the output itself when the unit has a single CTA.
//  * pa_merge_dynamic_kernel combines a unit's records by log-sum-exp, then checks
//    the unit's counters -- the claims the plan implies, and every chunk processed
//    exactly once -- and resets them to zero for the next call.
//
// The counters live in the first kDynCounterBytes of the caller's workspace, which
// must be zero before its first use; every call leaves them zero.  A claim result
// outside the unit's chunks (a workspace that was not zeroed) ends the warp's claims
// and is reported by the merge; it never forms an address.  The sum over
// a context is split differently from run to run, so results may differ in the last
// bits between runs (always within the fp32 rounding of the online softmax).
#pragma once

#include "pa_decode.cuh"
#include "pa_merge.cuh"

namespace pa {

constexpr int kDynChunk = 2;             // 16-token tiles per chunk
constexpr int kDynMaxUnits = 1024;       // (sequence, kv head) units of one call
constexpr int kDynCounterBytes = 8192;   // counters at the start of the workspace
constexpr int kDynCtasPerSm = 3;         // resident CTAs per SM the grid is sized for
static_assert(2 * kDynMaxUnits * 4 <= kDynCounterBytes, "two int32 counters per unit");
static_assert(2 * kDynChunk + 1 <= 32, "a chunk's pages are held one per lane");

struct DynParams {
    CUtensorMap kmap;  // as DecodeParams
    CUtensorMap vmap;
    void *out;
    const void *q;
    const int32_t *block_tables;
    const int32_t *context_lens;
    int32_t *claim;    // [kDynMaxUnits] claim counters (zero between calls)
    int32_t *done;     // [kDynMaxUnits] chunks processed (zero between calls)
    int32_t *ustart;   // [U + 1] first CTA of each unit (written by CTA 0)
    float *rec_o;      // [grid][G][D]  per-CTA records
    float *rec_m;      // [grid][G]
    float *rec_l;      // [grid][G]
    int num_seqs;
    int num_q_heads;
    int num_kv_heads;
    int block_size;
    int bs_shift;
    int num_blocks;
    int max_blocks_per_seq;
    int sliding_window;
    int cta_stride;    // coprime with the grid: CTA b takes plan slot (b * cta_stride) % grid
    float scale_log2;
    // fused cache write (pa_decode_append): the warp that produces the tile holding
    // position L-1 stores the new token's K and V row there before that tile's copy
    const void *new_k;
    const void *new_v;
    long long new_k_stride;
    long long new_v_stride;
    void *k_cache;
    void *v_cache;
};

// First CTA of unit u (u in [0, U]): u + floor((C - U) * before / total), where
// `before` counts the tiles of the units ahead of u; with no tiles at all the spare
// CTAs are spread evenly.
__device__ __forceinline__ int dyn_unit_start(int u, int U, int C, long long before,
                                              long long total) {
    const long long spare = (long long)(C - U);
    if (total <= 0) return u + (int)(spare * u / U);
    return u + (int)(spare * before / total);
}

// Claims a unit's warps make in one call when all goes well: one claim per chunk past
// the two static rounds, plus the one failed claim of every warp that claimed at all.
__host__ __device__ __forceinline__ int dyn_expected_claims(int nch, int nw) {
    const int ok = nch > 2 * nw ? nch - 2 * nw : 0;
    const int failed = nch > nw ? (nch - nw < nw ? nch - nw : nw) : 0;
    return ok + failed;
}

template <typename T, int D, int G, int BOXR>
__global__ void __launch_bounds__(kWarps * 32, kDynCtasPerSm)
    pa_decode_dynamic_kernel(const __grid_constant__ DynParams p) {
    pdl_wait_and_release();
    using Gm = Geom<D>;
    extern __shared__ uint8_t smem_raw[];
    __shared__ int unit_s;
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *base_ptr = smem_raw + (base - raw);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int B = p.num_seqs, Hkv = p.num_kv_heads, Hq = p.num_q_heads;
    // plan slot of this CTA: consecutive slots (the CTAs of one unit) are spread over
    // the grid, so no unit sits on one corner of the GPU's SMs
    const int U = B * Hkv, C = gridDim.x;
    const int c = (int)(((long long)blockIdx.x * p.cta_stride) % C);
    const int W = p.sliding_window;
    const int cap = p.max_blocks_per_seq << p.bs_shift;

    // ---- 1. plan: tiles per sequence, exclusive prefix (block scan, aliasing the ring);
    // the lengths are kept beside it
    int *pre = reinterpret_cast<int *>(base_ptr);
    int *lens_sm = pre + (B + 1);
    {
        constexpr int nthr = kWarps * 32;
        const int per = (B + nthr - 1) / nthr;
        const int s_lo = min(B, tid * per), s_hi = min(B, s_lo + per);
        int local = 0;
        for (int s = s_lo; s < s_hi; ++s) {
            const int L0 = __ldg(p.context_lens + s);
            lens_sm[s] = L0;
            const int L = L0 < 0 ? 0 : (L0 > cap ? cap : L0);
            local += (L - span_begin(L, W) + kTile - 1) / kTile;
        }
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += v;
        }
        __shared__ int wsum[kWarps];
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        int off = 0;
        for (int w = 0; w < warp; ++w) off += wsum[w];
        int run = off + incl - local;
        for (int s = s_lo; s < s_hi; ++s) {
            int L = lens_sm[s];
            L = L < 0 ? 0 : (L > cap ? cap : L);
            pre[s] = run;
            run += (L - span_begin(L, W) + kTile - 1) / kTile;
        }
        if (tid == nthr - 1) pre[B] = off + incl;
        __syncthreads();
    }
    const long long total = (long long)pre[B] * Hkv;
    auto before = [&](int u) -> long long {  // tiles of the units ahead of u
        const int s = u / Hkv, g = u - s * Hkv;
        return (long long)pre[s] * Hkv + (long long)g * (pre[s + 1] - pre[s]);
    };
    auto ustart = [&](int u) -> int {
        return u >= U ? C : dyn_unit_start(u, U, C, before(u), total);
    };
    if (c == 0)
        for (int u = tid; u <= U; u += kWarps * 32) p.ustart[u] = ustart(u);
    if (tid == 0) {  // the unit of this CTA: the largest u with ustart(u) <= c
        int lo = 0, hi = U - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (ustart(mid) <= c) lo = mid;
            else hi = mid - 1;
        }
        unit_s = lo;
    }
    __syncthreads();
    const int u = unit_s;
    const int s = u / Hkv, g = u - s * Hkv;
    const int c0 = ustart(u), nctas = ustart(u + 1) - c0;
    int L = lens_sm[s];
    __syncthreads();  // pre[] and the lengths (in the ring) are no longer read

    if (L < 0 || L > cap) {
        if (tid == 0 && c == c0) raise_error(PA_DEVERR_CONTEXT);
        L = L < 0 ? 0 : cap;
    }
    const int wlo = window_lo(L, W), span0 = span_begin(L, W);
    const int ntile = (L - span0 + kTile - 1) / kTile;
    const int nch = (ntile + kDynChunk - 1) / kDynChunk;
    const int NW = nctas * kWarps;
    const int r = (c - c0) * kWarps + warp;
    const int32_t *table = p.block_tables + (size_t)s * p.max_blocks_per_seq;
    int *claim = p.claim + u;

    // ---- 2. chunk pipeline of this warp (all values warp-uniform except the per-lane
    // table entries and lane 0's claim result).  The table entries of the first two
    // chunks and the first claim are in flight while q is read.
    auto chunk_pages = [&](int ch, int &pg_lo) -> int {
        const int t_lo = span0 + ch * (kDynChunk * kTile);
        const int t_hi = min(t_lo + kDynChunk * kTile, L);
        pg_lo = t_lo >> p.bs_shift;
        return ((t_hi - 1) >> p.bs_shift) - pg_lo + 1;
    };
    auto load_tab = [&](int ch, int &pg_lo) -> int {
        if (ch >= nch) return -1;
        const int npg = chunk_pages(ch, pg_lo);
        return lane < npg ? __ldg(table + pg_lo + lane) : -1;
    };
    int q0 = r, q1 = r + NW;       // chunk being produced, next chunk
    int pg0 = 0, pg1 = 0;          // first page of each
    int tab0 = load_tab(q0, pg0), tab1 = load_tab(q1, pg1);
    int off0 = 0;                  // next tile of q0
    int claim_res = 0;             // lane 0: result of the claim in flight
    bool pending = false;          // a claim is in flight
    if (q1 < nch) {
        if (lane == 0) claim_res = atomicAdd(claim, 1);
        pending = true;
    }
    int nchunks = q0 < nch ? 1 : 0;  // chunks this warp has started

    const T *q_item = reinterpret_cast<const T *>(p.q) + ((size_t)s * Hq + (size_t)g * G) * D;
    T *out = reinterpret_cast<T *>(p.out) + ((size_t)s * Hq + (size_t)g * G) * D;
    WarpCompute<T, D, G> wc;
    wc.init(q_item, lane);

    const uint32_t bars_all = base + Gm::kRing;
    const uint32_t ring = base + warp * kStages * Gm::kStage;
    const uint32_t bars = bars_all + warp * kStages * 8;
    if (tid == 0) {
        tma_prefetch_desc(&p.kmap);
        tma_prefetch_desc(&p.vmap);
        for (int i = 0; i < kWarps * kStages; ++i) mbar_init(bars_all + 8 * i, 1);
        fence_barrier_init();
    }

    auto advance = [&]() {         // q0 exhausted: move to q1, resolve the claim
        q0 = q1;
        if (q0 < nch) ++nchunks;
        tab0 = tab1;
        pg0 = pg1;
        off0 = 0;
        if (pending) {
            const int res = __shfl_sync(kFull, claim_res, 0);
            q1 = (res >= 0 && res < nch - 2 * NW) ? 2 * NW + res : nch;
            pending = false;
        } else {
            q1 = nch;
        }
        tab1 = load_tab(q1, pg1);
        if (q1 < nch) {
            if (lane == 0) claim_res = atomicAdd(claim, 1);
            pending = true;
        }
    };

    const uint64_t pol = l2_policy_evict_first();
    int st_tok[kStages], st_rows[kStages];
#pragma unroll
    for (int k = 0; k < kStages; ++k) st_tok[k] = st_rows[k] = 0;

    __syncthreads();  // barriers initialised

    auto produce = [&](int jt) {
        const int stage = jt % kStages;
        const int tok = span0 + (q0 * kDynChunk + off0) * kTile;
        const int nrows = min(kTile, L - tok);
        const int row_lo = max(0, wlo - tok);
        if (p.new_k != nullptr && tok + nrows == L) {
            // fused cache write of position L-1, before the copy of its tile
            const int pos = L - 1;
            const int blk = __shfl_sync(kFull, tab0, (pos >> p.bs_shift) - pg0);
            if ((unsigned)blk < (unsigned)p.num_blocks) {
                const size_t row = ((size_t)blk * Hkv + g) * p.block_size +
                                   (pos & (p.block_size - 1));
                constexpr int kChunks = D / 8;
                for (int cc = lane; cc < 2 * kChunks; cc += 32) {
                    const bool isv = cc >= kChunks;
                    const int c8 = isv ? cc - kChunks : cc;
                    const T *src = reinterpret_cast<const T *>(isv ? p.new_v : p.new_k) +
                                   (size_t)s * (isv ? p.new_v_stride : p.new_k_stride) +
                                   (size_t)g * D + 8 * c8;
                    T *dst = reinterpret_cast<T *>(isv ? p.v_cache : p.k_cache) + row * D + 8 * c8;
                    *reinterpret_cast<uint4 *>(dst) = ld_global_nc_v4(src);
                }
                fence_proxy_async_global();  // this tile's TMA reads the new row
                __syncwarp();
            } else if (lane == 0) {
                raise_error(PA_DEVERR_BLOCK_ID);
            }
        }
        constexpr int kBoxes = kTile / BOXR;
        int ys[kBoxes];
        unsigned boxes = 0;
        bool ok = true;
#pragma unroll
        for (int b = 0; b < kBoxes; ++b) {
            ys[b] = 0;
            if (b * BOXR < nrows && (b + 1) * BOXR > row_lo) {
                const int tb = tok + b * BOXR;
                const int blk = __shfl_sync(kFull, tab0, (tb >> p.bs_shift) - pg0);
                if ((unsigned)blk < (unsigned)p.num_blocks)
                    ys[b] = (blk * Hkv + g) * p.block_size + (tb & (p.block_size - 1));
                else
                    ok = false;
                boxes |= 1u << b;
            }
        }
        const uint32_t bar = bars + 8 * stage;
        const uint32_t kd = ring + stage * Gm::kStage, vd = kd + Gm::kMat;
        if (lane == 0) {
            if (ok) {
                mbar_arrive_expect_tx(bar,
                                      (uint32_t)(__popc(boxes) * Gm::kHalves * BOXR * 128 * 2));
#pragma unroll
                for (int b = 0; b < kBoxes; ++b) {
                    if ((boxes >> b) & 1u) {
#pragma unroll
                        for (int hf = 0; hf < Gm::kHalves; ++hf) {
                            const uint32_t off = hf * Gm::kRegion + b * BOXR * 128;
                            tma_load_2d(kd + off, &p.kmap, bar, 64 * hf, ys[b], pol);
                            tma_load_2d(vd + off, &p.vmap, bar, 64 * hf, ys[b], pol);
                        }
                    }
                }
            } else {
                raise_error(PA_DEVERR_BLOCK_ID);
                mbar_arrive(bar);
            }
        }
#pragma unroll
        for (int k = 0; k < kStages; ++k) {
            if (k == stage) {
                st_tok[k] = tok;
                st_rows[k] = ok ? nrows : 0;
            }
        }
        if (++off0 == min(kDynChunk, ntile - q0 * kDynChunk)) advance();
    };

    int nprod = 0;
    for (; nprod < kStages && q0 < nch; ++nprod) produce(nprod);
    bool failed = false;
    for (int jt = 0; jt < nprod; ++jt) {
        const int stage = jt % kStages;
        const uint32_t parity = (uint32_t)((jt / kStages) & 1);
        const bool got = mbar_wait_bounded(bars + 8 * stage, parity);
        if (!__all_sync(kFull, got)) {
            if (lane == 0) raise_error(PA_DEVERR_TIMEOUT);
            for (int k = jt + 1; k < nprod; ++k)
                (void)mbar_wait_bounded(bars + 8 * (k % kStages), (uint32_t)((k / kStages) & 1));
            failed = true;
            break;
        }
        int tok = 0, nrows = 0;
#pragma unroll
        for (int k = 0; k < kStages; ++k) {
            if (k == stage) {
                tok = st_tok[k];
                nrows = st_rows[k];
            }
        }
        const uint32_t kd = ring + stage * Gm::kStage, vd = kd + Gm::kMat;
        wc.tile(kd, vd, max(0, wlo - tok), nrows, p.scale_log2, lane);
        __syncwarp();
        if (q0 < nch) produce(nprod++);
    }
    if (failed) wc.init(q_item, lane);  // contributes nothing (m = -inf, l = 0)
    else if (lane == 0 && nchunks > 0) atomicAdd(p.done + u, nchunks);

    // ---- 3. merge the warps; one record per CTA, or the output for a one-CTA unit
    float *mine = reinterpret_cast<float *>(base_ptr + warp * kStages * Gm::kStage);
    wc.finish(mine, lane);
    __syncthreads();
    const bool single = nctas == 1;
    for (int e = tid; e < G * D; e += kWarps * 32) {
        const int h = e / D, d = e % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float *src = reinterpret_cast<const float *>(base_ptr + w * kStages * Gm::kStage);
            M = fmaxf(M, src[G * D + h]);
        }
        float num = 0.f, den = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float *src = reinterpret_cast<const float *>(base_ptr + w * kStages * Gm::kStage);
            const float mw = src[G * D + h];
            if (mw != -INFINITY) {
                const float wt = fast_exp2(mw - M);
                num = fmaf(src[h * D + d], wt, num);
                den = fmaf(src[G * D + G + h], wt, den);
            }
        }
        const float val = den > 0.f ? num / den : 0.f;
        if (single) {
            out[e] = Fmt<T>::from_float(val);
        } else {
            const size_t idx = (size_t)c * G + h;
            p.rec_o[idx * D + d] = val;
            if (d == 0) {
                p.rec_m[idx] = M;
                p.rec_l[idx] = den;
            }
        }
    }
}

struct DynMergeParams {
    void *out;
    const int32_t *context_lens;
    int32_t *claim;
    int32_t *done;
    const int32_t *ustart;
    const float *rec_o;
    const float *rec_m;
    const float *rec_l;
    int num_q_heads;
    int num_kv_heads;
    int cap;
    int sliding_window;
};

// One CTA of kMergeThreads per (q head, sequence): the unit's CTA records merged in one
// round of loads (lse_merge_warps), or by lse_merge_block when there are more of them.
template <typename T, int D>
__global__ void __launch_bounds__(kMergeThreads)
    pa_merge_dynamic_kernel(const __grid_constant__ DynMergeParams p) {
    pdl_wait_and_release();
    constexpr int kW = kMergeThreads / 32;
    const int h = blockIdx.x, s = blockIdx.y, tid = threadIdx.x;
    const int Hkv = p.num_kv_heads, G = p.num_q_heads / Hkv;
    const int g = h / G, hh = h - g * G, u = s * Hkv + g;
    const int c0 = p.ustart[u], n = p.ustart[u + 1] - c0;
    if (hh == 0 && tid == 0) {
        // the claims and chunks this call counted for the unit, then zero for the next call
        int L = p.context_lens[s];
        L = L < 0 ? 0 : (L > p.cap ? p.cap : L);
        const int ntile = (L - span_begin(L, p.sliding_window) + kTile - 1) / kTile;
        const int nch = (ntile + kDynChunk - 1) / kDynChunk;
        if (p.claim[u] != dyn_expected_claims(nch, n * kWarps) || p.done[u] != nch)
            raise_error(PA_DEVERR_WORKSPACE);
        p.claim[u] = 0;
        p.done[u] = 0;
    }
    if (n <= 1) return;  // the unit's only CTA wrote the output
    T *out = reinterpret_cast<T *>(p.out) + ((size_t)s * p.num_q_heads + h) * D;
    const auto rec = [&](int i) -> long long { return (long long)(c0 + i) * G + hh; };
    const float v = n <= kW * kMergeWarpRecs
                        ? lse_merge_warps<D>(n, rec, p.rec_m, p.rec_l, p.rec_o)
                        : lse_merge_block<D>(n, rec, p.rec_m, p.rec_l, p.rec_o);
    if (tid < D) out[tid] = Fmt<T>::from_float(v);
}

}  // namespace pa
