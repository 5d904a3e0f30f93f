// Paged decode attention kernels (sm_100a).
//
// What is computed ("IO-5 vLLM Paged Attention" note, sections 3-4): for sequence s
// and query head h (kv head g = h / G),
//     out[s][h] = softmax_t(scale * q[s][h] . K_s[t]) V_s[t],  t < L_s,
// where K_s is the sequence's pages concatenated in block-table order.  The
// arithmetic is the textbook one evaluated as an online softmax in fp32 (running
// max m, running sum l, rescaled accumulator), so the pages' statement that paging
// leaves the attention unchanged holds up to fp32 rounding.
//
// Work decomposition.  One CTA owns one item (sequence s, kv head g, context
// partition p of `partition_tokens` tokens); grid = (kv heads, sequences, partitions).  Its kWarps warps split the item's
// 16-token tiles into contiguous runs.  Each warp streams its tiles through its own
// kStages-deep ring in shared memory: lane 0 issues 2-D TMA loads (128-byte
// swizzled boxes of 64 columns x min(bs, 16) rows) for the K and V rows of a tile
// into a stage, completion is tracked by one mbarrier per stage, and the whole warp
// consumes the stage once the barrier flips.  The block-table row is read 32
// entries at a time with one coalesced load and broadcast by shuffles, so the table
// lookup for tile j+kStages is done while tile j is being consumed.
//
// Compute per tile:
//  * G <= 2 (SIMT): 16 (or 8) lanes cover one 128-wide (64-wide) row with 16-byte
//    shared loads; q.k partial sums are reduced with a transposing butterfly
//    (one shuffle per row and head), p.V with one broadcast shuffle per row and head.
//  * G >= 4 (tensor cores): S^T[16 tokens x 8 heads] = K_tile . Q^T with
//    mma.m16n8k16 (K from ldmatrix, Q^T kept in registers), then
//    O^T[d x 8 heads] += V_tile^T . P^T with the probabilities P split into a
//    high and a low 16-bit part (two mma per tile), so P keeps ~16 significant bits
//    (fp32-grade accuracy for the weights) while the one page read serves all G heads.
//
// The warps' (m, l, O) are merged in shared memory.  A sequence that fits one
// partition is written to `out` directly; otherwise the partition writes its fp32
// (m, l, O/l) to the workspace and pa_merge_kernel combines the partitions by
// log-sum-exp:  M = max m_p,  w_p = l_p 2^(m_p - M),  out = sum w_p o_p / sum w_p
// (m is kept in the log2 domain: scores are pre-multiplied by scale * log2(e)).
#pragma once

#include <type_traits>

#include "pa_common.cuh"

namespace pa {

#ifndef PA_DECODE_WARPS
#define PA_DECODE_WARPS 4
#endif
#ifndef PA_DECODE_STAGES
#define PA_DECODE_STAGES 2
#endif

constexpr int kTile = 16;                  // tokens per tile (one mma M/K extent)
constexpr int kTabSmem = 256;              // block-table entries of a partition kept in smem
constexpr int kWarps = PA_DECODE_WARPS;    // warps per CTA
constexpr int kStages = PA_DECODE_STAGES;  // ring depth per warp
constexpr unsigned kFull = 0xffffffffu;

struct DecodeParams {
    CUtensorMap kmap;  // [rows = num_blocks*Hkv*bs][D] 16-bit, box 64 x min(bs,16), swizzle 128B
    CUtensorMap vmap;
    void *out;
    const void *q;
    const int32_t *block_tables;
    const int32_t *context_lens;
    float *ws_o;  // [B][Hq][num_parts][D]
    float *ws_m;  // [B][Hq][num_parts]
    float *ws_l;  // [B][Hq][num_parts]
    int num_q_heads;
    int num_kv_heads;
    int block_size;
    int bs_shift;
    int num_blocks;
    int max_blocks_per_seq;
    int partition_tokens;
    int num_parts;
    int sliding_window;  // > 0: attend to the last sliding_window tokens only; 0: all
    int rotate;          // != 0: each warp starts its tiles at a pseudo-random offset
    int sort_second;     // != 0 (two partitions, few sequences): second partitions longest first
    float scale_log2;
    // Cache write fused into the decode (pa_decode_append): the new token of sequence s
    // (key/value rows new_k + s * new_k_stride, heads contiguous) is stored at position
    // L-1 by the CTA of the last partition before its first copy.  nullptr = no write.
    const void *new_k;
    const void *new_v;
    long long new_k_stride;  // elements between tokens
    long long new_v_stride;
    void *k_cache;
    void *v_cache;
    // Copy-on-write folded into the decode (pa_decode_cow): int32 [B][3] = (source block,
    // logical block index, rows); rows [0, rows) of every kv head of the source block are
    // copied into the sequence's own block at that index before any of them is read.
    // Source < 0: no copy for that sequence.  nullptr = no copies at all.
    const int32_t *cow;
};

// A launch planned on the host (pa_decode_planned): the (sequence, partition) units that
// exist, in the order the CTAs should take them, carried in the kernel's parameter space.
// Unit = sequence << 16 | partition << 8 | the sequence's partition count.
constexpr int kPlanMaxUnits = 4096;
constexpr int kPlanMaxParts = 255;
struct PlannedParams {
    DecodeParams base;
    uint32_t units[kPlanMaxUnits];
};
__device__ __forceinline__ const DecodeParams &param_base(const DecodeParams &p) { return p; }
__device__ __forceinline__ const DecodeParams &param_base(const PlannedParams &p) {
    return p.base;
}

template <int D>
struct Geom {
    static constexpr int kHalves = D / 64;             // 128-byte column blocks per row
    static constexpr int kRegion = kTile * 128;        // one column block of a tile
    static constexpr int kMat = kHalves * kRegion;     // a 16 x D tile
    static constexpr int kStage = 2 * kMat;            // K tile + V tile
    static constexpr int kRing = kWarps * kStages * kStage;
    static constexpr int kSmem = kRing + kWarps * kStages * 8 + 1024;  // + barriers + align
};

// Byte offset of 16-byte chunk `chunk` of row `row` in a tile as the TMA stores it:
// column block chunk/8, then the 128-byte swizzle (chunk%8) ^ (row%8).
__device__ __forceinline__ uint32_t tile_off(int row, int chunk) {
    return (chunk >> 3) * (kTile * 128) + row * 128 + (((chunk & 7) ^ (row & 7)) << 4);
}

// Sliding window: the attended tokens of a context of L are [window_lo, L); the
// tiles that cover them start at the 16-aligned position span_begin, so every tile
// stays inside one page (block sizes are powers of two) and its rows below
// window_lo are masked.  Without a window both are 0.
__host__ __device__ __forceinline__ int window_lo(int L, int W) {
    return (W > 0 && L > W) ? L - W : 0;
}
__host__ __device__ __forceinline__ int span_begin(int L, int W) {
    return window_lo(L, W) & ~(kTile - 1);
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "r"(addr));
    return r;
}

__device__ __forceinline__ void sts128_zero(uint32_t addr) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0) : "memory");
}

// Transposing butterfly sum over the lanes that differ in bits MASK, MASK/2, ..., 1:
// N values per lane in, the full sum of value index (lane bits from MASK down) out
// in v[0].  N/2 + N/4 + ... shuffles instead of N * log2(lanes).
template <int N, int MASK>
struct Butterfly {
    __device__ __forceinline__ static void run(float *v, int lane) {
        if constexpr (MASK == 0) {
            return;
        } else if constexpr (N > 1) {
            const bool upper = (lane & MASK) != 0;
#pragma unroll
            for (int k = 0; k < N / 2; ++k) {
                const float send = upper ? v[k] : v[k + N / 2];
                const float keep = upper ? v[k + N / 2] : v[k];
                v[k] = keep + __shfl_xor_sync(kFull, send, MASK);
            }
            Butterfly<N / 2, MASK / 2>::run(v, lane);
        } else {
            v[0] += __shfl_xor_sync(kFull, v[0], MASK);
            Butterfly<1, MASK / 2>::run(v, lane);
        }
    }
};

constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }

// --------------------------------------------------------------------------- SIMT path

template <typename T, int D, int G>
struct SimtWarp {
    static constexpr int kCpr = D / 8;               // 16-byte chunks per row
    static constexpr int kRps = 32 / kCpr;           // rows per warp step
    static constexpr int kSteps = kTile / kRps;      // steps per tile
    static constexpr int kN = kSteps * G;            // partial sums per lane per tile
    static constexpr int kShift = ilog2(kCpr) - ilog2(kN);  // replicated low lane bits
    static_assert(kN <= kCpr, "SIMT path needs steps*G <= chunks per row");

    float qf[G][8];
    float acc[G][8];
    float m;  // running max (log2 domain) of this lane's head
    float l;  // this lane's share of the running sum of its head
    int lig, rr, c, my_v, my_i, my_h, my_row;
    bool owner;

    __device__ __forceinline__ void init(const T *q_item, int lane) {
        lig = lane & (kCpr - 1);
        rr = lane / kCpr;
        c = lig;
        my_v = lig >> kShift;
        my_i = my_v / G;
        my_h = my_v % G;
        my_row = my_i * kRps + rr;
        owner = (lig & ((1 << kShift) - 1)) == 0;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const uint4 w = *reinterpret_cast<const uint4 *>(q_item + h * D + 8 * c);
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = Fmt<T>::unpack(ws[e]);
                qf[h][2 * e] = f.x;
                qf[h][2 * e + 1] = f.y;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[h][e] = 0.f;
        }
        m = -INFINITY;
        l = 0.f;
    }

    // Rows [row_lo, nrows) of the tile are context tokens; the others are masked.
    __device__ __forceinline__ void tile(uint32_t kd, uint32_t vd, int row_lo, int nrows,
                                         float sl2, int lane) {
        float v[kN];
#pragma unroll
        for (int i = 0; i < kSteps; ++i) {
            const int r = i * kRps + rr;
            const uint4 w = lds128(kd + tile_off(r, c));
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
            float kf[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = Fmt<T>::unpack(ws[e]);
                kf[2 * e] = f.x;
                kf[2 * e + 1] = f.y;
            }
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float a = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) a = fmaf(qf[h][e], kf[e], a);
                v[i * G + h] = a;
            }
        }
        Butterfly<kN, kCpr / 2>::run(v, lane);
        const bool valid = my_row >= row_lo && my_row < nrows;
        const float sc = valid ? v[0] * sl2 : -INFINITY;
        // tile max of this lane's head: all lane bits except the head bits
        float mx = sc;
#pragma unroll
        for (int mask = 1; mask < 32; mask <<= 1) {
            if (G > 1 && mask >= (1 << kShift) && mask < ((1 << kShift) * G)) continue;
            mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, mask));
        }
        const float mn = fmaxf(m, mx);
        const float alpha = (mn == -INFINITY) ? 1.f : fast_exp2(m - mn);
        const float pr = valid ? fast_exp2(sc - mn) : 0.f;
        m = mn;
        l = l * alpha + (owner ? pr : 0.f);
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float ah = (G == 1) ? alpha : __shfl_sync(kFull, alpha, h << kShift);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[h][e] *= ah;
        }
        const int grp = lane & ~(kCpr - 1);
#pragma unroll
        for (int i = 0; i < kSteps; ++i) {
            float ph[G];
#pragma unroll
            for (int h = 0; h < G; ++h) ph[h] = __shfl_sync(kFull, pr, grp | ((i * G + h) << kShift));
            const int r = i * kRps + rr;
            if (r >= row_lo && r < nrows) {
                const uint4 w = lds128(vd + tile_off(r, c));
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = Fmt<T>::unpack(ws[e]);
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        acc[h][2 * e] = fmaf(ph[h], f.x, acc[h][2 * e]);
                        acc[h][2 * e + 1] = fmaf(ph[h], f.y, acc[h][2 * e + 1]);
                    }
                }
            }
        }
    }

    // Writes this warp's O[G][D], m[G], l[G] (fp32) at `dst`.
    __device__ __forceinline__ void finish(float *dst, int lane) {
#pragma unroll
        for (int mask = kCpr; mask < 32; mask <<= 1)
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[h][e] += __shfl_xor_sync(kFull, acc[h][e], mask);
        float lt = l;
#pragma unroll
        for (int mask = 1; mask < 32; mask <<= 1) {
            if (G > 1 && mask >= (1 << kShift) && mask < ((1 << kShift) * G)) continue;
            lt += __shfl_xor_sync(kFull, lt, mask);
        }
        if (lane < kCpr) {
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int e = 0; e < 8; ++e) dst[h * D + 8 * c + e] = acc[h][e];
        }
        if (lane < (G << kShift) && (lane & ((1 << kShift) - 1)) == 0) {
            dst[G * D + my_h] = m;
            dst[G * D + G + my_h] = lt;
        }
    }

    // Ends a segment straight from registers: `whole` -> out[h][:] = O/l rounded to T;
    // otherwise the fp32 partial record ro[h][:] = O/l, rm[h] = m, rl[h] = l.
    __device__ __forceinline__ void store(bool whole, T *out, float *ro, float *rm, float *rl,
                                          int lane) {
#pragma unroll
        for (int mask = kCpr; mask < 32; mask <<= 1)
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[h][e] += __shfl_xor_sync(kFull, acc[h][e], mask);
        float lt = l;
#pragma unroll
        for (int mask = 1; mask < 32; mask <<= 1) {
            if (G > 1 && mask >= (1 << kShift) && mask < ((1 << kShift) * G)) continue;
            lt += __shfl_xor_sync(kFull, lt, mask);
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float lh = __shfl_sync(kFull, lt, h << kShift);
            const float mh = __shfl_sync(kFull, m, h << kShift);
            if (lane < kCpr) {
                float v[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] = lh > 0.f ? acc[h][e] / lh : 0.f;
                if (whole) {
                    uint4 w;
                    w.x = Fmt<T>::pack_rn(v[0], v[1]);
                    w.y = Fmt<T>::pack_rn(v[2], v[3]);
                    w.z = Fmt<T>::pack_rn(v[4], v[5]);
                    w.w = Fmt<T>::pack_rn(v[6], v[7]);
                    *reinterpret_cast<uint4 *>(out + h * D + 8 * c) = w;
                } else {
                    float4 *dst = reinterpret_cast<float4 *>(ro + h * D + 8 * c);
                    dst[0] = make_float4(v[0], v[1], v[2], v[3]);
                    dst[1] = make_float4(v[4], v[5], v[6], v[7]);
                }
            }
            if (!whole && lane == 0) {
                rm[h] = mh;
                rl[h] = lh;
            }
        }
    }
};

// ---------------------------------------------------------------- tensor-core path

template <typename T, int D, int G>
struct MmaWarp {
    static constexpr int kK = D / 16;  // k-steps of QK^T, m-tiles of PV
    static_assert(G <= 8, "one mma N extent holds at most 8 heads");

    uint32_t qb[kK][2];  // Q^T B-fragments (heads >= G are zero)
    float o[kK][4];      // O^T accumulators: (d = 16mt + gq (+8), heads 2tq, 2tq+1)
    float m0, m1, l0, l1;
    int gq, tq;

    __device__ __forceinline__ void init(const T *q_item, int lane) {
        gq = lane >> 2;
        tq = lane & 3;
#pragma unroll
        for (int kk = 0; kk < kK; ++kk) {
            if (gq < G) {
                const T *qh = q_item + gq * D + 16 * kk + 2 * tq;
                qb[kk][0] = *reinterpret_cast<const uint32_t *>(qh);
                qb[kk][1] = *reinterpret_cast<const uint32_t *>(qh + 8);
            } else {
                qb[kk][0] = 0u;
                qb[kk][1] = 0u;
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) o[kk][e] = 0.f;
        }
        m0 = m1 = -INFINITY;
        l0 = l1 = 0.f;
    }

    // Rows [row_lo, nrows) of the tile are context tokens; the others are masked.
    __device__ __forceinline__ void tile(uint32_t kd, uint32_t vd, int row_lo, int nrows,
                                         float sl2, int lane) {
        const int j = lane >> 3, r8 = lane & 7;
        // S^T = K . Q^T  (A = K rows from ldmatrix: matrix j -> rows +8*(j&1), k +8*(j>>1))
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
        {
            const int row = r8 + ((j & 1) << 3);
#pragma unroll
            for (int kk = 0; kk < kK; ++kk) {
                uint32_t a[4];
                ldsm_x4(kd + tile_off(row, 2 * kk + (j >> 1)), a[0], a[1], a[2], a[3]);
                Mma<T>::run(sc, a, qb[kk][0], qb[kk][1]);
            }
        }
        const bool v0 = gq >= row_lo && gq < nrows, v1 = gq + 8 >= row_lo && gq + 8 < nrows;
        const float s0 = v0 ? sc[0] * sl2 : -INFINITY;
        const float s1 = v0 ? sc[1] * sl2 : -INFINITY;
        const float s2 = v1 ? sc[2] * sl2 : -INFINITY;
        const float s3 = v1 ? sc[3] * sl2 : -INFINITY;
        float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
        for (int mask = 4; mask < 32; mask <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, mask));
            mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, mask));
        }
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float al0 = (mn0 == -INFINITY) ? 1.f : fast_exp2(m0 - mn0);
        const float al1 = (mn1 == -INFINITY) ? 1.f : fast_exp2(m1 - mn1);
        m0 = mn0;
        m1 = mn1;
        const float p0 = v0 ? fast_exp2(s0 - mn0) : 0.f;
        const float p1 = v0 ? fast_exp2(s1 - mn1) : 0.f;
        const float p2 = v1 ? fast_exp2(s2 - mn0) : 0.f;
        const float p3 = v1 ? fast_exp2(s3 - mn1) : 0.f;
        l0 = l0 * al0 + (p0 + p2);
        l1 = l1 * al1 + (p1 + p3);
#pragma unroll
        for (int mt = 0; mt < kK; ++mt) {
            o[mt][0] *= al0;
            o[mt][1] *= al1;
            o[mt][2] *= al0;
            o[mt][3] *= al1;
        }
        // P^T as B fragments: hi = RN(p), lo = RN(p - hi); the 8x8 transposes turn the
        // (token row, head pair) layout of S^T into the (token pair, head) layout of B.
        const uint32_t x0 = Fmt<T>::pack_rn(p0, p1), x1 = Fmt<T>::pack_rn(p2, p3);
        const float2 h0 = Fmt<T>::unpack(x0), h1 = Fmt<T>::unpack(x1);
        const uint32_t y0 = Fmt<T>::pack_rn(p0 - h0.x, p1 - h0.y);
        const uint32_t y1 = Fmt<T>::pack_rn(p2 - h1.x, p3 - h1.y);
        const uint32_t bh0 = movmatrix_trans(x0), bh1 = movmatrix_trans(x1);
        const uint32_t bl0 = movmatrix_trans(y0), bl1 = movmatrix_trans(y1);
        // rows outside the context may hold anything (NaN, or rows that were never
        // loaded): zero them so 0 * V stays 0
        if (nrows < kTile) {
            constexpr int kChunks = Geom<D>::kHalves * 8;
            for (int idx = lane; idx < (kTile - nrows) * kChunks; idx += 32) {
                const int r = nrows + idx / kChunks;
                const int ch = idx % kChunks;
                sts128_zero(vd + (ch >> 3) * (kTile * 128) + r * 128 + ((ch & 7) << 4));
            }
        }
        if (row_lo > 0) {
            constexpr int kChunks = Geom<D>::kHalves * 8;
            const int nlo = min(row_lo, kTile);
            for (int idx = lane; idx < nlo * kChunks; idx += 32) {
                const int r = idx / kChunks;
                const int ch = idx % kChunks;
                sts128_zero(vd + (ch >> 3) * (kTile * 128) + r * 128 + ((ch & 7) << 4));
            }
        }
        if (nrows < kTile || row_lo > 0) {
            fence_proxy_async_smem();
            __syncwarp();
        }
        // O^T += V^T . P^T  (A = V^T via ldmatrix.trans: matrix j -> tokens +8*(j>>1),
        // dims +8*(j&1))
        {
            const int row = r8 + ((j >> 1) << 3);
#pragma unroll
            for (int mt = 0; mt < kK; ++mt) {
                uint32_t a[4];
                ldsm_x4_trans(vd + tile_off(row, 2 * mt + (j & 1)), a[0], a[1], a[2], a[3]);
                Mma<T>::run(o[mt], a, bh0, bh1);
                Mma<T>::run(o[mt], a, bl0, bl1);
            }
        }
    }

    __device__ __forceinline__ void finish(float *dst, int lane) {
        float lt0 = l0, lt1 = l1;
#pragma unroll
        for (int mask = 4; mask < 32; mask <<= 1) {
            lt0 += __shfl_xor_sync(kFull, lt0, mask);
            lt1 += __shfl_xor_sync(kFull, lt1, mask);
        }
        const int h0 = 2 * tq, h1 = 2 * tq + 1;
#pragma unroll
        for (int mt = 0; mt < kK; ++mt) {
            const int d = 16 * mt + gq;
            if (h0 < G) {
                dst[h0 * D + d] = o[mt][0];
                dst[h0 * D + d + 8] = o[mt][2];
            }
            if (h1 < G) {
                dst[h1 * D + d] = o[mt][1];
                dst[h1 * D + d + 8] = o[mt][3];
            }
        }
        if (gq == 0) {
            if (h0 < G) {
                dst[G * D + h0] = m0;
                dst[G * D + G + h0] = lt0;
            }
            if (h1 < G) {
                dst[G * D + h1] = m1;
                dst[G * D + G + h1] = lt1;
            }
        }
    }

    // Ends a segment straight from registers (see SimtWarp::store).
    __device__ __forceinline__ void store(bool whole, T *out, float *ro, float *rm, float *rl,
                                          int lane) {
        float lt0 = l0, lt1 = l1;
#pragma unroll
        for (int mask = 4; mask < 32; mask <<= 1) {
            lt0 += __shfl_xor_sync(kFull, lt0, mask);
            lt1 += __shfl_xor_sync(kFull, lt1, mask);
        }
        const int h0 = 2 * tq, h1 = 2 * tq + 1;
#pragma unroll
        for (int mt = 0; mt < kK; ++mt) {
            const int d = 16 * mt + gq;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int h = half ? h1 : h0;
                const float lh = half ? lt1 : lt0;
                if (h < G) {
                    const float a = lh > 0.f ? o[mt][half] / lh : 0.f;
                    const float b = lh > 0.f ? o[mt][2 + half] / lh : 0.f;
                    if (whole) {
                        out[h * D + d] = Fmt<T>::from_float(a);
                        out[h * D + d + 8] = Fmt<T>::from_float(b);
                    } else {
                        ro[h * D + d] = a;
                        ro[h * D + d + 8] = b;
                    }
                }
            }
        }
        if (!whole && gq == 0) {
            if (h0 < G) {
                rm[h0] = m0;
                rl[h0] = lt0;
            }
            if (h1 < G) {
                rm[h1] = m1;
                rl[h1] = lt1;
            }
        }
    }
};

template <typename T, int D, int G>
using WarpCompute = typename std::conditional<(G >= 4), MmaWarp<T, D, G>, SimtWarp<T, D, G>>::type;

// ------------------------------------------------------------------ partition kernel

constexpr int kSortMaxSeqs = kWarps * 32;  // one sequence per thread

// Launches of at most two partitions per context: the second partitions -- the grid's
// last CTAs, and so the tail -- are taken longest first.  Returns the sequence whose second
// partition has rank k in that order (by decreasing length, ties by sequence), or -1
// past the last one.  Every thread of the CTA calls it; at most kSortMaxSeqs sequences.
template <bool WIN>
__device__ __forceinline__ int second_partition_seq(const DecodeParams &p, int k, int S) {
    __shared__ __align__(16) int sh_len2[kSortMaxSeqs];  // second partition's length, or -1
    __shared__ int sh_sel;
    const int tid = threadIdx.x;
    const int P = p.partition_tokens;
    const int cap = p.max_blocks_per_seq << p.bs_shift;
    int r = -1;
    if (tid < S) {
        int L = __ldg(p.context_lens + tid);
        L = L < 0 ? 0 : (L > cap ? cap : L);
        const int len = WIN ? L - span_begin(L, p.sliding_window) : L;
        r = len > P ? len - P : -1;
    }
    sh_len2[tid] = r;
    if (tid == 0) sh_sel = -1;
    __syncthreads();
    if (r >= 0) {
        int rank = 0;
#pragma unroll 4
        for (int t = 0; t < kSortMaxSeqs; t += 4) {
            const int4 v = *reinterpret_cast<const int4 *>(sh_len2 + t);
            rank += (v.x > r || (v.x == r && t < tid)) ? 1 : 0;
            rank += (v.y > r || (v.y == r && t + 1 < tid)) ? 1 : 0;
            rank += (v.z > r || (v.z == r && t + 2 < tid)) ? 1 : 0;
            rank += (v.w > r || (v.w == r && t + 3 < tid)) ? 1 : 0;
        }
        if (rank == k) sh_sel = tid;
    }
    __syncthreads();
    return sh_sel;
}

// Copy-on-write (p.cow): rows [a, b) of kv head g of block src into block dst, in both
// caches, by `n` threads numbered `t` (a warp's lanes or the whole CTA).
template <int D>
__device__ __forceinline__ void cow_rows(const DecodeParams &p, int src, int dst, int g, int a,
                                         int b, int t, int n) {
    constexpr int kChunks = D / 8;  // 16-byte chunks of a head row
    if (a >= b) return;
    const size_t head_rows = (size_t)p.num_kv_heads * p.block_size;
    const size_t from = ((size_t)src * head_rows + (size_t)g * p.block_size + a) * kChunks;
    const size_t to = ((size_t)dst * head_rows + (size_t)g * p.block_size + a) * kChunks;
    uint4 *kc = reinterpret_cast<uint4 *>(p.k_cache);
    uint4 *vc = reinterpret_cast<uint4 *>(p.v_cache);
    for (int c = t; c < (b - a) * kChunks; c += n) {
        const uint4 k = ld_global_nc_v4(kc + from + c), v = ld_global_nc_v4(vc + from + c);
        kc[to + c] = k;
        vc[to + c] = v;
    }
}

// WIN: compiled with sliding-window support (p.sliding_window > 0); the instances
// without it keep the whole-context path free of the window's bookkeeping.  COW: compiled
// with the copy-on-write of p.cow, so that calls without copies run code without it.
// PLAN: the grid is (kv head, unit) over a host-planned unit list (PlannedParams).
template <typename T, int D, int G, int BOXR, bool WIN, bool COW = false, bool PLAN = false>
__global__ void __launch_bounds__(kWarps * 32)
    pa_decode_partition_kernel(
        const __grid_constant__ typename std::conditional<PLAN, PlannedParams, DecodeParams>::type
            pp) {
    const DecodeParams &p = param_base(pp);
    pdl_wait_and_release();
    using Gm = Geom<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *base_ptr = smem_raw + (base - raw);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    // grid (kv head, sequence, partition): every first partition is scheduled before any
    // second one, so the smaller remainder partitions run last and shorten the tail, and
    // CTAs scheduled together read neighbouring heads of the same physical blocks.  With
    // p.sort_second the second partitions are moreover taken longest first.
    const int g = blockIdx.x;
    int s, part, planned_parts = 0;
    if constexpr (PLAN) {
        const uint32_t u = pp.units[blockIdx.y];
        s = (int)(u >> 16);
        part = (int)((u >> 8) & 0xffu);
        planned_parts = (int)(u & 0xffu);
    } else {
        s = blockIdx.y;
        part = blockIdx.z;
        if (p.sort_second && part == 1) {
            s = second_partition_seq<WIN>(p, (int)blockIdx.y, (int)gridDim.y);
            if (s < 0) return;
        }
    }
    const int Hq = p.num_q_heads;

    // Start the three independent loads of this item at once: its context length, the
    // block-table entries of its partition (without a sliding window the page range
    // does not depend on L) and q.  Under a window the table is read through the
    // per-warp lookup below once L is known.
    const int P = p.partition_tokens;
    const int W = WIN ? p.sliding_window : 0;
    const int32_t *table = p.block_tables + (size_t)s * p.max_blocks_per_seq;
    int cw_src = -1, cw_lb = 0, cw_rows = 0;  // this sequence's copy-on-write, loaded early
    if constexpr (COW) {
        cw_src = __ldg(p.cow + 3 * (size_t)s);
        cw_lb = __ldg(p.cow + 3 * (size_t)s + 1);
        cw_rows = __ldg(p.cow + 3 * (size_t)s + 2);
    }
    const int pg_first = (int)(((long long)part * P) >> p.bs_shift);
    const int pg_count = min((int)((((long long)part * P + P - 1) >> p.bs_shift) - pg_first + 1),
                             p.max_blocks_per_seq - pg_first);
    const bool tab_in_smem = W == 0 && pg_count <= kTabSmem;
    __shared__ int tab_smem[kTabSmem];
    if (tab_in_smem)
        for (int i = tid; i < pg_count; i += kWarps * 32) tab_smem[i] = __ldg(table + pg_first + i);
    const T *q_item = reinterpret_cast<const T *>(p.q) + ((size_t)s * Hq + (size_t)g * G) * D;
    WarpCompute<T, D, G> wc;
    wc.init(q_item, lane);
    int L = __ldg(p.context_lens + s);
    const int cap = p.max_blocks_per_seq << p.bs_shift;
    if (L < 0 || L > cap) {
        if (tid == 0 && part == 0) raise_error(PA_DEVERR_CONTEXT);
        L = L < 0 ? 0 : cap;
    }
    const int wlo = WIN ? window_lo(L, W) : 0, span0 = WIN ? span_begin(L, W) : 0;
    const int nparts = (L - span0 + P - 1) / P;
    if (nparts > p.num_parts && tid == 0 && part == 0) raise_error(PA_DEVERR_CONTEXT);
    // a plan made from host lengths that disagree with the device's: flagged (a partition
    // the plan left out is not computed)
    if (PLAN && part == 0 && tid == 0 && max(nparts, 1) != planned_parts)
        raise_error(PA_DEVERR_CONTEXT);
    // Copy-on-write: every row of the copied block goes to the CTA whose partition holds
    // its position (rows before the first partition to the first, rows past the last to
    // the last), so the CTA that reads a row copies it.  This CTA's share: rows [cr0, cr1).
    int cr0 = 0, cr1 = 0;
    long long cw_pos0 = 0;  // position of the block's first row
    if constexpr (COW) {
        const int owners = max(min(nparts, p.num_parts), 1);
        if (cw_src >= 0 && part < owners) {
            if (cw_src >= p.num_blocks || (unsigned)cw_lb >= (unsigned)p.max_blocks_per_seq ||
                (unsigned)cw_rows > (unsigned)p.block_size) {
                if (tid == 0 && part == 0 && g == 0) raise_error(PA_DEVERR_PAIR);
            } else {
                cw_pos0 = (long long)cw_lb << p.bs_shift;
                const long long Pl = P;
                const long long lo = part == 0 ? cw_pos0 : span0 + part * Pl;
                const long long hi = part == owners - 1 ? cw_pos0 + cw_rows
                                                        : span0 + (part + 1) * Pl;
                cr0 = (int)max(0LL, min((long long)cw_rows, lo - cw_pos0));
                cr1 = (int)max(0LL, min((long long)cw_rows, hi - cw_pos0));
            }
        }
    }
    T *out = reinterpret_cast<T *>(p.out) + ((size_t)s * Hq + (size_t)g * G) * D;
    if (L == 0) {
        if constexpr (COW) {
            if (cr0 < cr1) {  // no tiles: the whole CTA copies the rows
                const int dst = __ldg(table + cw_lb);
                if ((unsigned)dst < (unsigned)p.num_blocks)
                    cow_rows<D>(p, cw_src, dst, g, cr0, cr1, tid, kWarps * 32);
                else if (tid == 0)
                    raise_error(PA_DEVERR_BLOCK_ID);
            }
        }
        if (part == 0)
            for (int e = tid; e < G * D; e += kWarps * 32) out[e] = Fmt<T>::from_float(0.f);
        return;
    }
    if (part >= nparts) return;

    // Fused cache write of this step's token (position L-1, always in the last partition).
    if (p.new_k != nullptr && part == nparts - 1) {
        const int pos = L - 1;
        const int blk = __ldg(table + (pos >> p.bs_shift));
        if ((unsigned)blk < (unsigned)p.num_blocks) {
            const size_t row =
                ((size_t)blk * p.num_kv_heads + g) * p.block_size + (pos & (p.block_size - 1));
            constexpr int kChunks = D / 8;  // 16-byte chunks of a head row
            for (int c = tid; c < 2 * kChunks; c += kWarps * 32) {
                const bool isv = c >= kChunks;
                const int cc = isv ? c - kChunks : c;
                const T *src = reinterpret_cast<const T *>(isv ? p.new_v : p.new_k) +
                               (size_t)s * (isv ? p.new_v_stride : p.new_k_stride) +
                               (size_t)g * D + 8 * cc;
                T *dst = reinterpret_cast<T *>(isv ? p.v_cache : p.k_cache) + row * D + 8 * cc;
                *reinterpret_cast<uint4 *>(dst) = ld_global_nc_v4(src);
            }
            fence_proxy_async_global();  // the TMA of the last tile reads this row
        } else if (tid == 0) {
            raise_error(PA_DEVERR_BLOCK_ID);
        }
    }

    const int t0 = span0 + part * P, t1 = min(t0 + P, L);
    const int ntiles = (t1 - t0 + kTile - 1) / kTile;
    const int qd = ntiles / kWarps, rm = ntiles % kWarps;
    const int wt0 = warp * qd + min(warp, rm);
    const int nt = qd + (warp < rm ? 1 : 0);
    const int tok_begin = t0 + wt0 * kTile;
    const int tok_end = min(tok_begin + nt * kTile, t1);
    // With large pages every warp's range starts at the same offset of a page, and all
    // warps would walk their pages in step; `rotate` starts each warp at its own offset
    // and wraps around (the softmax is order-independent; the order is fixed per call
    // shape, so results stay the same from call to call).
    int rot = 0;
    if (p.rotate && nt > 1) {
        const unsigned hsh = ((unsigned)s * 2654435761u) ^ ((unsigned)g * 2246822519u) ^
                             ((unsigned)part * 3266489917u) ^ ((unsigned)warp * 668265263u);
        rot = (int)((hsh >> 8) % (unsigned)nt);
    }
    auto tile_tok = [&](int jt) {
        const int j = jt + rot < nt ? jt + rot : jt + rot - nt;
        return tok_begin + j * kTile;
    };

    const uint32_t bars_all = base + Gm::kRing;
    const uint32_t ring = base + warp * kStages * Gm::kStage;
    const uint32_t bars = bars_all + warp * kStages * 8;
    if (tid == 0) {
        tma_prefetch_desc(&p.kmap);
        tma_prefetch_desc(&p.vmap);
        for (int i = 0; i < kWarps * kStages; ++i) mbar_init(bars_all + 8 * i, 1);
        fence_barrier_init();
    }

    const int npages = (L + p.block_size - 1) >> p.bs_shift;
    int tab_base = -(1 << 30), tab_reg = -1;
    const uint64_t pol = l2_policy_evict_first();
    unsigned okmask = 0;

    __syncthreads();

    auto lookup = [&](int pg) -> int {
        if (tab_in_smem) return tab_smem[pg - pg_first];  // CTA-uniform
        if (pg < tab_base || pg >= tab_base + 32) {  // warp-uniform
            tab_base = pg;
            const int e = pg + lane;
            tab_reg = e < npages ? __ldg(table + e) : -1;
        }
        return __shfl_sync(kFull, tab_reg, pg - tab_base);
    };

    auto produce = [&](int jt) {
        const int stage = jt % kStages;
        const int tok = tile_tok(jt);
        const int nrows = min(kTile, tok_end - tok);
        const int row_lo = WIN ? max(0, wlo - tok) : 0;
        constexpr int kBoxes = kTile / BOXR;
        int ys[kBoxes];
        unsigned boxes = 0;  // boxes that hold context rows (a box below the window is skipped)
        bool ok = true;
#pragma unroll
        for (int b = 0; b < kBoxes; ++b) {
            ys[b] = 0;
            if (b * BOXR < nrows && (b + 1) * BOXR > row_lo) {
                const int tb = tok + b * BOXR;
                const int blk = lookup(tb >> p.bs_shift);
                if ((unsigned)blk < (unsigned)p.num_blocks)
                    ys[b] = (blk * p.num_kv_heads + g) * p.block_size + (tb & (p.block_size - 1));
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
        okmask = ok ? (okmask | (1u << stage)) : (okmask & ~(1u << stage));
    };

    // Copy-on-write rows of this CTA's share, after the barrier and before the first TMA:
    // the warp whose tiles hold rows copies those (only that warp waits for the copy; the
    // others start streaming), and the rows no tile of the call reads -- before the first
    // tile or past the context -- are copied by the whole CTA.  The row the fused cache
    // write stored is left out (the write wins either way).  Deferring the warp's copy
    // until after its first TMA issues measured slower.
    if constexpr (COW) {
        if (cr0 < cr1) {  // CTA-uniform
            const int o1 = (int)max((long long)cr0, min((long long)cr1, (long long)t0 - cw_pos0));
            const int o2 = (int)min((long long)cr1, max((long long)cr0, (long long)t1 - cw_pos0));
            long long wb = min((long long)cr1, (long long)tok_end - cw_pos0);
            if (p.new_k != nullptr) wb = min(wb, (long long)(L - 1) - cw_pos0);
            const int wa = (int)max((long long)cr0, (long long)tok_begin - cw_pos0);
            const bool outside = cr0 < o1 || o2 < cr1;
            const bool reads_rows = nt > 0 && wa < wb;  // warp-uniform
            if (outside || reads_rows) {
                const int dst = __ldg(table + cw_lb);
                if ((unsigned)dst < (unsigned)p.num_blocks) {
                    if (reads_rows) {
                        cow_rows<D>(p, cw_src, dst, g, wa, (int)wb, lane, 32);
                        fence_proxy_async_global();  // this warp's TMA reads the rows
                    }
                    if (outside) {
                        cow_rows<D>(p, cw_src, dst, g, cr0, o1, tid, kWarps * 32);
                        cow_rows<D>(p, cw_src, dst, g, o2, cr1, tid, kWarps * 32);
                    }
                } else if (lane == 0) {
                    raise_error(PA_DEVERR_BLOCK_ID);
                }
                __syncwarp();
            }
        }
    }
    const int npre = min(kStages, nt);
    for (int jt = 0; jt < npre; ++jt) produce(jt);

    bool failed = false;
    for (int jt = 0; jt < nt; ++jt) {
        const int stage = jt % kStages;
        const uint32_t parity = (uint32_t)((jt / kStages) & 1);
        const bool got = mbar_wait_bounded(bars + 8 * stage, parity);
        if (!__all_sync(kFull, got)) {
            // give up on this item: record it, wait (bounded) for the copies in flight
            if (lane == 0) raise_error(PA_DEVERR_TIMEOUT);
            for (int k = jt + 1; k < min(jt + kStages, nt); ++k)
                (void)mbar_wait_bounded(bars + 8 * (k % kStages), (uint32_t)((k / kStages) & 1));
            failed = true;
            break;
        }
        const int tok = tile_tok(jt);
        const int nrows = ((okmask >> stage) & 1u) ? min(kTile, tok_end - tok) : 0;
        const uint32_t kd = ring + stage * Gm::kStage, vd = kd + Gm::kMat;
        wc.tile(kd, vd, WIN ? max(0, wlo - tok) : 0, nrows, p.scale_log2, lane);
        __syncwarp();
        if (jt + kStages < nt) produce(jt + kStages);
    }
    if (failed) wc.init(q_item, lane);  // contributes nothing (m = -inf, l = 0)
    // ---- merge the warps' partial softmax states (each warp uses its own ring)
    float *mine = reinterpret_cast<float *>(base_ptr + warp * kStages * Gm::kStage);
    wc.finish(mine, lane);
    __syncthreads();

    const bool single = (nparts == 1);
    const size_t item = ((size_t)s * Hq + (size_t)g * G) * p.num_parts + part;
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
            const size_t idx = item + (size_t)h * p.num_parts;
            p.ws_o[idx * D + d] = val;
            if (d == 0) {
                p.ws_m[idx] = M;
                p.ws_l[idx] = den;
            }
        }
    }
}

}  // namespace pa
