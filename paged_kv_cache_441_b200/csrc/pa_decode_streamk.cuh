// Balanced ("stream-K") split of paged decode attention over persistent warps.
//
// The work of one decode call is the list of 16-token tiles of every
// (sequence s, kv head g) segment, laid out s-major:
//     tile index = pre[s] * Hkv + g * n_s + j,   n_s = ceil(L_s / 16),  j < n_s,
// with pre[] the exclusive prefix sum of n_s.  The grid holds as many CTAs as fit
// on the GPU at once, and warp k of NW = grid * kSkWarps warps takes the contiguous
// tile range [T k / NW, T (k+1) / NW) of the T tiles, so every warp streams the
// same number of K/V bytes (to within one tile) however ragged the context lengths
// are.  The warp's TMA ring runs straight across segment boundaries: tile metadata
// travels with each stage, so the copy of the next segment's first tiles overlaps
// the end of the current one and no warp waits on another.
//
// A segment that lies inside one warp's range is finished by that warp (output
// written directly).  A segment cut by range boundaries is a context partition in
// the split-K sense: each warp that holds part of it writes an fp32 record
// (m, l, O/l) -- slot 0 for the first segment of its range, slot 1 for the last --
// and pa_merge_streamk_kernel combines the records of the segment by log-sum-exp,
// exactly as the fixed-partition path does.
//
// Start-up: every CTA computes pre[] with a block-wide scan into its (not yet used)
// TMA ring, each warp finds its first tile by binary search, and CTA 0 publishes
// pre[] for the merge kernel (which also writes the zero outputs of empty sequences).
#pragma once

#include "pa_decode.cuh"
#include "pa_merge.cuh"

namespace pa {

constexpr int kSkWarps = 4;
constexpr int kSkStages = 2;

struct StreamKParams {
    CUtensorMap kmap;
    CUtensorMap vmap;
    void *out;
    const void *q;
    const int32_t *block_tables;
    const int32_t *context_lens;
    int32_t *ws_pre;  // [B + 1] tiles per kv head, exclusive prefix (written by CTA 0)
    float *rec_o;     // warp pieces  [NW * 2][G][D]   (NW = grid * kSkWarps)
    float *rec_m;     //              [NW * 2][G]
    float *rec_l;     //              [NW * 2][G]
    float *crec_o;    // CTA records  [grid * 2][G][D]
    float *crec_m;    //              [grid * 2][G]
    float *crec_l;    //              [grid * 2][G]
    int num_seqs;
    int num_q_heads;
    int num_kv_heads;
    int block_size;
    int bs_shift;
    int num_blocks;
    int max_blocks_per_seq;
    int sliding_window;  // > 0: each query attends to its last sliding_window tokens
    float scale_log2;
};

template <int D>
struct SkGeom {
    static constexpr int kHalves = D / 64;
    static constexpr int kRegion = kTile * 128;
    static constexpr int kMat = kHalves * kRegion;
    static constexpr int kStage = 2 * kMat;
    static constexpr int kRing = kSkWarps * kSkStages * kStage;
    static constexpr int kBars = kSkWarps * kSkStages * 8;
    static constexpr int kMeta = kSkWarps * kSkStages * 16;
    static constexpr int kSmem = kRing + kBars + kMeta + 1024;
    static constexpr int kMaxSeqs = kRing / 4 - 1;  // pre[] aliases the ring at start-up
};

// tile-metadata flags carried by each ring stage
constexpr int kSkFirst = 1;     // first tile of a segment in this warp: reset the state
constexpr int kSkLast = 2;      // last tile of a segment in this warp: store it
constexpr int kSkWhole = 4;     // the segment is entirely in this warp: final output
constexpr int kSkFirstSeg = 8;  // the segment is the first of this warp's range: slot 0
constexpr int kSkOk = 16;       // block ids valid, data loaded
constexpr int kSkStarts = 32;   // the segment starts (j = 0) inside this warp
constexpr int kSkEnds = 64;     // the segment ends (last tile) inside this warp
constexpr int kSkRowLoShift = 8;  // bits 8+: first context row of the tile (window start)

__host__ __device__ __forceinline__ long long sk_range_begin(long long T, int k, int NW) {
    return T * k / NW;
}

// The warp whose range holds tile x: the largest k with T k / NW <= x.
__host__ __device__ __forceinline__ int sk_worker_of(long long x, long long T, int NW) {
    return (int)(((x + 1) * (long long)NW - 1) / T);
}

__device__ __forceinline__ int clamp_len(int L, int cap) { return L < 0 ? 0 : (L > cap ? cap : L); }

// 16-token tiles of a (sequence, kv head) segment: from span_begin(L, W) to L.
__device__ __forceinline__ int seg_tiles(int L, int W) {
    return (L - span_begin(L, W) + kTile - 1) / kTile;
}

// T k / NW without a 64-bit division per call: T = q NW + r, so T k / NW = q k + r k / NW
// with r k < NW k < 2^32.
struct RangeSplit {
    long long q;
    unsigned r, nw;
    __device__ __forceinline__ RangeSplit(long long T, int NW)
        : q(T / NW), r((unsigned)(T % NW)), nw((unsigned)NW) {}
    __device__ __forceinline__ long long begin(int k) const {
        return q * k + (long long)((r * (unsigned)k) / nw);
    }
};

template <typename T, int D, int G, int BOXR>
__global__ void __launch_bounds__(kSkWarps * 32)
    pa_decode_streamk_kernel(const __grid_constant__ StreamKParams p) {
    pdl_wait_and_release();
    using Gm = SkGeom<D>;
    extern __shared__ uint8_t smem_raw[];
    __shared__ int warp_tot[kSkWarps];
    __shared__ int4 piece[kSkWarps][2];  // partial segments of each warp: {s, g, flags}
    __shared__ float jw_[2 * kSkWarps][G];  // CTA join: piece weights per head
    __shared__ float jm_[2][G];             // CTA join: max and weight sum per head
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *base_ptr = smem_raw + (base - raw);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int B = p.num_seqs, Hq = p.num_q_heads, Hkv = p.num_kv_heads;
    const int cap = p.max_blocks_per_seq << p.bs_shift;

    // ---- 1. pre[] = exclusive prefix of per-sequence tile counts (block-wide scan)
    int *pre = reinterpret_cast<int *>(base_ptr);
    const int nthr = kSkWarps * 32;
    const int per = (B + nthr - 1) / nthr;
    const int s_lo = min(B, tid * per), s_hi = min(B, s_lo + per);
    int local = 0;
    for (int s = s_lo; s < s_hi; ++s) {
        const int L = p.context_lens[s];
        if ((L < 0 || L > cap) && blockIdx.x == 0) raise_error(PA_DEVERR_CONTEXT);
        local += seg_tiles(clamp_len(L, cap), p.sliding_window);
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int woff = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kSkWarps; ++w) {
        woff += (w < warp) ? warp_tot[w] : 0;
        total += warp_tot[w];
    }
    int run = woff + incl - local;
    for (int s = s_lo; s < s_hi; ++s) {
        pre[s] = run;
        run += seg_tiles(clamp_len(p.context_lens[s], cap), p.sliding_window);
    }
    if (tid == 0) pre[B] = total;
    __syncthreads();

    const long long Ttot = (long long)total * Hkv;
    const int NW = gridDim.x * kSkWarps;
    const int k = blockIdx.x * kSkWarps + warp;
    const long long a = Ttot > 0 ? sk_range_begin(Ttot, k, NW) : 0;
    const long long b = Ttot > 0 ? sk_range_begin(Ttot, k + 1, NW) : 0;

    if (blockIdx.x == 0)
        for (int i = tid; i <= B; i += nthr) p.ws_pre[i] = pre[i];

    // ---- 2. this warp's first tile: sequence s0 (largest s with pre[s]*Hkv <= a)
    int s0 = 0, n0 = 1, r0 = 0;
    if (a < b) {
        if (lane == 0) {
            int lo = 0, hi = B - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if ((long long)pre[mid] * Hkv <= a) lo = mid; else hi = mid - 1;
            }
            s0 = lo;
        }
        s0 = __shfl_sync(kFull, s0, 0);
        n0 = pre[s0 + 1] - pre[s0];
        r0 = (int)(a - (long long)pre[s0] * Hkv);
    }
    if (lane < 2) piece[warp][lane] = make_int4(0, 0, 0, 0);
    fence_proxy_async_smem();  // the ring was written through the generic proxy
    const uint32_t bars = base + Gm::kRing + warp * kSkStages * 8;
    int4 *meta = reinterpret_cast<int4 *>(base_ptr + Gm::kRing + Gm::kBars) + warp * kSkStages;
    if (tid == 0) {
        tma_prefetch_desc(&p.kmap);
        tma_prefetch_desc(&p.vmap);
        for (int i = 0; i < kSkWarps * kSkStages; ++i) mbar_init(base + Gm::kRing + 8 * i, 1);
        fence_barrier_init();
    }
    __syncthreads();
    T *out_all = reinterpret_cast<T *>(p.out);
    if (a < b) {
        const uint32_t ring = base + warp * kSkStages * Gm::kStage;
        const int nt = (int)(b - a);
        const uint64_t pol = l2_policy_evict_first();

        // producer cursor
        int ps = s0, pg = r0 / n0, pj = r0 % n0, pn = n0;
        int pL = clamp_len(p.context_lens[s0], cap);
        int p_left = nt, p_seg_j0 = pj, p_segidx = 0;
        bool p_segfirst = true;
        // caches: context lengths of 32 sequences, 32 block-table entries of one sequence
        int lc_base = -(1 << 30), lc_reg = 0;
        int tab_s = -1, tab_base = 0, tab_reg = -1;

        auto get_len = [&](int s) -> int {
            if (s < lc_base || s >= lc_base + 32) {  // warp-uniform
                lc_base = s;
                const int e = s + lane;
                lc_reg = e < B ? clamp_len(__ldg(p.context_lens + e), cap) : 0;
            }
            return __shfl_sync(kFull, lc_reg, s - lc_base);
        };
        auto lookup = [&](int s, int pg_idx, int npages) -> int {
            if (s != tab_s || pg_idx < tab_base || pg_idx >= tab_base + 32) {  // warp-uniform
                tab_s = s;
                tab_base = pg_idx;
                const int e = pg_idx + lane;
                tab_reg = e < npages ? __ldg(p.block_tables + (size_t)s * p.max_blocks_per_seq + e) : -1;
            }
            return __shfl_sync(kFull, tab_reg, pg_idx - tab_base);
        };

        auto produce = [&](int t) {
            const int stage = t % kSkStages;
            const int tok = span_begin(pL, p.sliding_window) + pj * kTile;
            const int nrows = min(kTile, pL - tok);
            const int row_lo = max(0, window_lo(pL, p.sliding_window) - tok);
            const int npages = (pL + p.block_size - 1) >> p.bs_shift;
            constexpr int kBoxes = kTile / BOXR;
            int ys[kBoxes];
            unsigned boxes = 0;  // boxes holding context rows (below the window: skipped)
            bool ok = true;
    #pragma unroll
            for (int bx = 0; bx < kBoxes; ++bx) {
                ys[bx] = 0;
                if (bx * BOXR < nrows && (bx + 1) * BOXR > row_lo) {
                    const int tb = tok + bx * BOXR;
                    const int blk = lookup(ps, tb >> p.bs_shift, npages);
                    if ((unsigned)blk < (unsigned)p.num_blocks)
                        ys[bx] = (blk * Hkv + pg) * p.block_size + (tb & (p.block_size - 1));
                    else
                        ok = false;
                    boxes |= 1u << bx;
                }
            }
            int flags = 0;
            if (p_segfirst) flags |= kSkFirst;
            if (pj == pn - 1 || p_left == 1) flags |= kSkLast;
            if (p_seg_j0 == 0 && pj == pn - 1) flags |= kSkWhole;
            if (p_seg_j0 == 0) flags |= kSkStarts;
            if (pj == pn - 1) flags |= kSkEnds;
            if (p_segidx == 0) flags |= kSkFirstSeg;
            if (ok) flags |= kSkOk;
            flags |= row_lo << kSkRowLoShift;
            const uint32_t bar = bars + 8 * stage;
            const uint32_t kd = ring + stage * Gm::kStage, vd = kd + Gm::kMat;
            if (lane == 0) {
                meta[stage] = make_int4(ps, pg, nrows, flags);
                if (ok) {
                    mbar_arrive_expect_tx(
                        bar, (uint32_t)(__popc(boxes) * Gm::kHalves * BOXR * 128 * 2));
    #pragma unroll
                    for (int bx = 0; bx < kBoxes; ++bx) {
                        if ((boxes >> bx) & 1u) {
    #pragma unroll
                            for (int hf = 0; hf < Gm::kHalves; ++hf) {
                                const uint32_t off = hf * Gm::kRegion + bx * BOXR * 128;
                                tma_load_2d(kd + off, &p.kmap, bar, 64 * hf, ys[bx], pol);
                                tma_load_2d(vd + off, &p.vmap, bar, 64 * hf, ys[bx], pol);
                            }
                        }
                    }
                } else {
                    raise_error(PA_DEVERR_BLOCK_ID);
                    mbar_arrive(bar);
                }
            }
            // advance the cursor (warp-uniform)
            --p_left;
            p_segfirst = false;
            ++pj;
            if (pj == pn && p_left > 0) {
                pj = 0;
                if (++pg == Hkv) {
                    pg = 0;
                    do {
                        ++ps;
                        pL = get_len(ps);
                    } while (pL == 0 && ps + 1 < B);
                    pn = seg_tiles(pL, p.sliding_window);
                }
                p_segfirst = true;
                p_seg_j0 = 0;
                ++p_segidx;
            }
        };

        const int npre = min(kSkStages, nt);
        for (int t = 0; t < npre; ++t) produce(t);

        WarpCompute<T, D, G> wc;
        for (int t = 0; t < nt; ++t) {
            const int stage = t % kSkStages;
            const uint32_t parity = (uint32_t)((t / kSkStages) & 1);
            const bool got = mbar_wait_bounded(bars + 8 * stage, parity);
            if (!__all_sync(kFull, got)) {
                if (lane == 0) raise_error(PA_DEVERR_TIMEOUT);
                for (int u = t + 1; u < min(t + kSkStages, nt); ++u)
                    (void)mbar_wait_bounded(bars + 8 * (u % kSkStages),
                                            (uint32_t)((u / kSkStages) & 1));
                break;
            }
            const int4 md = meta[stage];
            const int cs = md.x, cg = md.y, flags = md.w;
            const size_t head0 = (size_t)cs * Hq + (size_t)cg * G;
            if (flags & kSkFirst)
                wc.init(reinterpret_cast<const T *>(p.q) + head0 * D, lane);
            const uint32_t kd = ring + stage * Gm::kStage, vd = kd + Gm::kMat;
            wc.tile(kd, vd, flags >> kSkRowLoShift, (flags & kSkOk) ? md.z : 0, p.scale_log2,
                    lane);
            if (flags & kSkLast) {
                const int slot = (flags & kSkFirstSeg) ? 0 : 1;
                const size_t rec = (size_t)k * 2 + slot;
                wc.store((flags & kSkWhole) != 0, out_all + head0 * D, p.rec_o + rec * G * D,
                         p.rec_m + rec * G, p.rec_l + rec * G, lane);
                if (!(flags & kSkWhole) && lane == 0)
                    piece[warp][slot] = make_int4(cs, cg, 1 | (flags & (kSkStarts | kSkEnds)), 0);
            }
            __syncwarp();
            if (t + kSkStages < nt) produce(t + kSkStages);
        }
    }  // a < b

    // ---- 3. CTA level: join the pieces of segments that several warps of this CTA cut.
    // The CTA's range [T c / grid, T (c+1) / grid) is the union of its warps' ranges.
    // A joined segment that starts and ends inside the CTA is final; otherwise it is
    // the CTA's first segment (slot 0) or last segment (slot 1) for the merge kernel.
    __syncthreads();
    {
        int pw[2 * kSkWarps], ps_[2 * kSkWarps];
        int np = 0, w_first = -1;
        const RangeSplit rsw(Ttot > 0 ? Ttot : 1, NW);
#pragma unroll
        for (int w = 0; w < kSkWarps; ++w) {
            const int kw = blockIdx.x * kSkWarps + w;
            if (w_first < 0 && Ttot > 0 && rsw.begin(kw) < rsw.begin(kw + 1)) w_first = w;
#pragma unroll
            for (int sl = 0; sl < 2; ++sl)
                if (piece[w][sl].z & 1) {
                    pw[np] = w;
                    ps_[np] = sl;
                    ++np;
                }
        }
        int i = 0;
        while (i < np) {
            const int4 pi = piece[pw[i]][ps_[i]];
            int j = i;
            while (j + 1 < np && piece[pw[j + 1]][ps_[j + 1]].x == pi.x &&
                   piece[pw[j + 1]][ps_[j + 1]].y == pi.y)
                ++j;
            const bool starts = (pi.z & kSkStarts) != 0;
            const bool ends = (piece[pw[j]][ps_[j]].z & kSkEnds) != 0;
            bool has_first = false;
            for (int u = i; u <= j; ++u) has_first |= (pw[u] == w_first && ps_[u] == 0);
            const int slot = has_first ? 0 : 1;
            const size_t crec = (size_t)blockIdx.x * 2 + slot;
            const size_t head0 = (size_t)pi.x * Hq + (size_t)pi.y * G;
            const int npc = j - i + 1;
            // weights of the pieces, per head, staged once: wgt[u][h] = l 2^(m - M_h)
            __syncthreads();  // jw_/jm_ of the previous group fully read
            if (tid < G) {
                float M = -INFINITY;
                for (int u = 0; u < npc; ++u) {
                    const size_t r = ((size_t)(blockIdx.x * kSkWarps + pw[i + u]) * 2 + ps_[i + u]) * G + tid;
                    M = fmaxf(M, __ldcg(p.rec_m + r));
                }
                float den = 0.f;
                for (int u = 0; u < npc; ++u) {
                    const size_t r = ((size_t)(blockIdx.x * kSkWarps + pw[i + u]) * 2 + ps_[i + u]) * G + tid;
                    const float mu = __ldcg(p.rec_m + r);
                    const float w = mu == -INFINITY ? 0.f : __ldcg(p.rec_l + r) * fast_exp2(mu - M);
                    jw_[u][tid] = w;
                    den += w;
                }
                jm_[0][tid] = M;
                jm_[1][tid] = den;
            }
            __syncthreads();
            for (int e = tid; e < G * D; e += nthr) {
                const int h = e / D, d = e % D;
                float v[2 * kSkWarps];
#pragma unroll
                for (int u = 0; u < 2 * kSkWarps; ++u) {  // all loads in flight together
                    v[u] = 0.f;
                    if (u < npc && jw_[u][h] != 0.f) {
                        const size_t r = ((size_t)(blockIdx.x * kSkWarps + pw[i + u]) * 2 + ps_[i + u]) * G + h;
                        v[u] = __ldcg(p.rec_o + r * D + d);
                    }
                }
                float num = 0.f;
#pragma unroll
                for (int u = 0; u < 2 * kSkWarps; ++u)
                    if (u < npc) num = fmaf(jw_[u][h], v[u], num);
                const float den = jm_[1][h];
                const float val = den > 0.f ? num / den : 0.f;
                if (starts && ends) {
                    out_all[head0 * D + e] = Fmt<T>::from_float(val);
                } else {
                    p.crec_o[(crec * G + h) * D + d] = val;
                    if (d == 0) {
                        p.crec_m[crec * G + h] = jm_[0][h];
                        p.crec_l[crec * G + h] = den;
                    }
                }
            }
            i = j + 1;
        }
    }
}

struct SkMergeParams {
    void *out;
    const int32_t *ws_pre;
    const float *rec_o;  // CTA records [num_workers * 2][G][D]
    const float *rec_m;
    const float *rec_l;
    int num_seqs;
    int num_q_heads;
    int num_kv_heads;
    int num_workers;  // CTAs of the decode grid: CTA c held tiles [T c / n, T (c+1) / n)
};

// One CTA per (q head, sequence): log-sum-exp merge of the records of a segment that
// several CTAs shared (slot 1 for the CTA whose range began before the segment, slot 0
// for the others); nothing to do otherwise, zeros for an empty context.
template <typename T, int D>
__global__ void __launch_bounds__(kMergeThreads)
    pa_merge_streamk_kernel(const __grid_constant__ SkMergeParams p) {
    pdl_wait_and_release();
    const int h = blockIdx.x, s = blockIdx.y, d = threadIdx.x;
    const int G = p.num_q_heads / p.num_kv_heads;
    const int g = h / G, jh = h % G;
    const int pre_s = p.ws_pre[s];
    const int n = p.ws_pre[s + 1] - pre_s;
    T *out = reinterpret_cast<T *>(p.out) + ((size_t)s * p.num_q_heads + h) * D;
    if (n == 0) {  // empty context: no warp touched this sequence
        if (d < D) out[d] = Fmt<T>::from_float(0.f);
        return;
    }
    const long long Ttot = (long long)p.ws_pre[p.num_seqs] * p.num_kv_heads;
    const int NW = p.num_workers;
    const long long A = (long long)pre_s * p.num_kv_heads + (long long)g * n;
    const long long E = A + n - 1;
    const int k0 = sk_worker_of(A, Ttot, NW), k1 = sk_worker_of(E, Ttot, NW);
    if (k0 == k1) return;
    const RangeSplit rs(Ttot, NW);
    const long long a0 = rs.begin(k0);
    // record of warp k for this segment: slot 1 when the segment is the last of k0's
    // range (k0 started before it), slot 0 otherwise; warps with empty ranges have none
    auto rec = [&](int i) -> long long {
        const int k = k0 + i;
        if (rs.begin(k) == rs.begin(k + 1)) return -1;
        return ((long long)k * 2 + ((k == k0 && a0 < A) ? 1 : 0)) * G + jh;
    };
    const float v = lse_merge_block<D>(k1 - k0 + 1, rec, p.rec_m, p.rec_l, p.rec_o);
    if (d < D) out[d] = Fmt<T>::from_float(v);
}

}  // namespace pa
