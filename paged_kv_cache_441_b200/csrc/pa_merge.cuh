// Log-sum-exp merge of split-K partial results (fixed-partition path).
//
// A context cut into pieces yields, per piece i and query head, the running max m_i
// (log2 domain), the running sum l_i and the normalised partial output o_i = O_i/l_i.
// The exact softmax result is  out = sum_i l_i 2^(m_i - M) o_i / sum_i l_i 2^(m_i - M)
// with M = max_i m_i -- the standard identity that lets a softmax be evaluated over a
// split sum.
#pragma once

#include "pa_decode.cuh"

namespace pa {

// Log-sum-exp merge of n partial results of one (sequence, q head):
//     M = max_i m_i,  w_i = l_i 2^(m_i - M),  out[:] = sum_i w_i o_i[:] / sum_i w_i.
// rec(i) gives the record index of partial i, or -1 for "no record"; m at rm[rec],
// l at rl[rec], o at ro[rec * D].  Block of kMergeThreads threads:
//   1. all threads reduce M over the records;
//   2. per chunk of kMergeChunk records, all threads compute w_i and the record index
//      into shared memory at once;
//   3. each warp takes every 8th record of the chunk, four records per step, each an
//      independent vector load of o (D/32 floats per lane), so the loads overlap;
//   4. the warps' sums are added in shared memory.
// Thread e (e < D) returns element e of the merged output.
constexpr int kMergeThreads = 256;
constexpr int kMergeChunk = 512;
constexpr int kMergeFew = 8;  // up to this many partials: one load round per thread

template <int D, typename RecFn>
__device__ __forceinline__ float lse_merge_block(int n, RecFn rec, const float *rm,
                                                 const float *rl, const float *ro) {
    constexpr int kW = kMergeThreads / 32;
    constexpr int kV = D / 32;  // floats per lane
    __shared__ float red[kW];
    __shared__ float w_s[kMergeChunk];
    __shared__ int r_s[kMergeChunk];
    __shared__ float part[kW][D];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    float M = -INFINITY;
    for (int i = tid; i < n; i += kMergeThreads) {
        const long long r = rec(i);
        if (r >= 0) M = fmaxf(M, rm[r]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, o));
    if (lane == 0) red[wid] = M;
    __syncthreads();
    M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kW; ++w) M = fmaxf(M, red[w]);
    float acc[kV];
#pragma unroll
    for (int e = 0; e < kV; ++e) acc[e] = 0.f;
    float den = 0.f;
    for (int c0 = 0; c0 < n; c0 += kMergeChunk) {
        const int cnt = min(kMergeChunk, n - c0);
        __syncthreads();  // previous chunk fully consumed (and red[] read)
        for (int i = tid; i < cnt; i += kMergeThreads) {
            const long long r = rec(c0 + i);
            float w = 0.f;
            if (r >= 0) {
                const float mi = rm[r];
                if (mi != -INFINITY) w = rl[r] * fast_exp2(mi - M);
            }
            w_s[i] = w;
            r_s[i] = r >= 0 ? (int)r : 0;
            den += w;
        }
        __syncthreads();
        int j = wid;
        for (; j + 3 * kW < cnt; j += 4 * kW) {
            float wv[4];
            const float *src[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                wv[u] = w_s[j + u * kW];
                src[u] = ro + (long long)r_s[j + u * kW] * D + lane * kV;
            }
            // a zero weight marks a partial without a record: its slot may hold
            // anything (even NaN), so it is not read at all
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (wv[u] == 0.f) continue;
                if constexpr (kV == 4) {
                    const float4 v = *reinterpret_cast<const float4 *>(src[u]);
                    acc[0] = fmaf(wv[u], v.x, acc[0]);
                    acc[1] = fmaf(wv[u], v.y, acc[1]);
                    acc[2] = fmaf(wv[u], v.z, acc[2]);
                    acc[3] = fmaf(wv[u], v.w, acc[3]);
                } else {
                    const float2 v = *reinterpret_cast<const float2 *>(src[u]);
                    acc[0] = fmaf(wv[u], v.x, acc[0]);
                    acc[1] = fmaf(wv[u], v.y, acc[1]);
                }
            }
        }
        for (; j < cnt; j += kW) {
            const float wv = w_s[j];
            if (wv == 0.f) continue;
            const float *src = ro + (long long)r_s[j] * D + lane * kV;
#pragma unroll
            for (int e = 0; e < kV; ++e) acc[e] = fmaf(wv, src[e], acc[e]);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(kFull, den, o);
    __syncthreads();
#pragma unroll
    for (int e = 0; e < kV; ++e) part[wid][lane * kV + e] = acc[e];
    if (lane == 0) red[wid] = den;
    __syncthreads();
    if (tid >= D) return 0.f;
    float num = 0.f, dsum = 0.f;
#pragma unroll
    for (int w = 0; w < kW; ++w) {
        num += part[w][tid];
        dsum += red[w];
    }
    return dsum > 0.f ? num / dsum : 0.f;
}

// Log-sum-exp merge of n <= (kMergeThreads / 32) * kMergeWarpRecs partials in one round of
// loads: warp w takes partials w, w + 8, w + 16, ... -- o as D/32 floats per lane in one
// vector load, m and l as broadcast loads -- all issued before any is used; the maximum is
// combined through shared memory, then each warp's weighted sum, and the warps' sums.
// rec(i) as in lse_merge_block; a partial whose m is -inf (nothing attended) gets no
// weight, and whatever its o slot holds is not used.  Thread e (e < D) returns element e.
constexpr int kMergeWarpRecs = 16;

template <int D, typename RecFn>
__device__ __forceinline__ float lse_merge_warps(int n, RecFn rec, const float *rm,
                                                 const float *rl, const float *ro) {
    constexpr int kW = kMergeThreads / 32, kV = D / 32;
    __shared__ float red[kW];
    __shared__ float den_s[kW];
    __shared__ float part[kW][D];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    float m[kMergeWarpRecs], l[kMergeWarpRecs];
    float o[kMergeWarpRecs][kV];
#pragma unroll
    for (int i = 0; i < kMergeWarpRecs; ++i) {
        const int j = wid + i * kW;
        m[i] = -INFINITY;
        l[i] = 0.f;
#pragma unroll
        for (int e = 0; e < kV; ++e) o[i][e] = 0.f;
        if (j < n) {
            const long long r = rec(j);
            m[i] = rm[r];
            l[i] = rl[r];
            const float *src = ro + r * D + lane * kV;
            if constexpr (kV == 4) {
                const float4 v = *reinterpret_cast<const float4 *>(src);
                o[i][0] = v.x;
                o[i][1] = v.y;
                o[i][2] = v.z;
                o[i][3] = v.w;
            } else {
                const float2 v = *reinterpret_cast<const float2 *>(src);
                o[i][0] = v.x;
                o[i][1] = v.y;
            }
        }
    }
    float Mw = -INFINITY;
#pragma unroll
    for (int i = 0; i < kMergeWarpRecs; ++i) Mw = fmaxf(Mw, m[i]);
    if (lane == 0) red[wid] = Mw;
    __syncthreads();
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kW; ++w) M = fmaxf(M, red[w]);
    float acc[kV], den = 0.f;
#pragma unroll
    for (int e = 0; e < kV; ++e) acc[e] = 0.f;
#pragma unroll
    for (int i = 0; i < kMergeWarpRecs; ++i) {
        if (m[i] == -INFINITY) continue;
        const float w = l[i] * fast_exp2(m[i] - M);
        den += w;
#pragma unroll
        for (int e = 0; e < kV; ++e) acc[e] = fmaf(w, o[i][e], acc[e]);
    }
#pragma unroll
    for (int e = 0; e < kV; ++e) part[wid][lane * kV + e] = acc[e];
    if (lane == 0) den_s[wid] = den;
    __syncthreads();
    if (tid >= D) return 0.f;
    float num = 0.f, dsum = 0.f;
#pragma unroll
    for (int w = 0; w < kW; ++w) {
        num += part[w][tid];
        dsum += den_s[w];
    }
    return dsum > 0.f ? num / dsum : 0.f;
}

struct MergeParams {
    void *out;
    const int32_t *context_lens;
    const float *ws_o;
    const float *ws_m;
    const float *ws_l;
    int num_q_heads;
    int cap;  // max_blocks_per_seq * block_size
    int partition_tokens;
    int num_parts;
    int sliding_window;  // as in DecodeParams: partitions start at span_begin(L, W)
};

// One CTA per (q head, sequence) with more than one partition.  WIDE: compiled with the
// warp and block paths (more than kMergeFew partitions possible); the instance for at
// most kMergeFew keeps its register count, and so its occupancy, low.
template <typename T, int D, bool WIDE>
__global__ void __launch_bounds__(kMergeThreads) pa_merge_kernel(const __grid_constant__ MergeParams p) {
    pdl_wait_and_release();
    const int h = blockIdx.x, s = blockIdx.y;
    int L = p.context_lens[s];
    L = L < 0 ? 0 : (L > p.cap ? p.cap : L);
    int n = (L - span_begin(L, p.sliding_window) + p.partition_tokens - 1) / p.partition_tokens;
    if (n <= 1) return;
    n = min(n, p.num_parts);
    const long long base = ((long long)s * p.num_q_heads + h) * p.num_parts;
    if (!WIDE || n <= kMergeFew) {
        // few partitions: every load of this thread's element is issued at once
        const int d = threadIdx.x;
        if (d >= D) return;
        float m[kMergeFew], l[kMergeFew], o[kMergeFew];
#pragma unroll
        for (int i = 0; i < kMergeFew; ++i) {
            m[i] = i < n ? p.ws_m[base + i] : -INFINITY;
            l[i] = i < n ? p.ws_l[base + i] : 0.f;
            o[i] = i < n ? p.ws_o[(base + i) * D + d] : 0.f;
        }
        float M = -INFINITY;
#pragma unroll
        for (int i = 0; i < kMergeFew; ++i) M = fmaxf(M, m[i]);
        float num = 0.f, den = 0.f;
#pragma unroll
        for (int i = 0; i < kMergeFew; ++i) {
            if (m[i] == -INFINITY) continue;
            const float w = l[i] * fast_exp2(m[i] - M);
            num = fmaf(w, o[i], num);
            den += w;
        }
        T *out = reinterpret_cast<T *>(p.out) + ((size_t)s * p.num_q_heads + h) * D;
        out[d] = Fmt<T>::from_float(den > 0.f ? num / den : 0.f);
        return;
    }
    if constexpr (!WIDE) return;
    T *out = reinterpret_cast<T *>(p.out) + ((size_t)s * p.num_q_heads + h) * D;
    if (n <= (kMergeThreads / 32) * kMergeWarpRecs) {
        const float v = lse_merge_warps<D>(
            n, [&](int i) -> long long { return base + i; }, p.ws_m, p.ws_l, p.ws_o);
        if (threadIdx.x < D) out[threadIdx.x] = Fmt<T>::from_float(v);
        return;
    }
    const float v = lse_merge_block<D>(
        n, [&](int i) -> long long { return base + i; }, p.ws_m, p.ws_l, p.ws_o);
    if (threadIdx.x < D) out[threadIdx.x] = Fmt<T>::from_float(v);
}

}  // namespace pa
