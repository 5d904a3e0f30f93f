// Multi-query (prefill / chunked-prefill) attention over the paged cache, on the
// fifth-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// What is computed ("IO-5 vLLM Paged Attention" note, section 4, with a matrix Q: one
// row per new token of a request, as continuous batching -- section 6 -- brings new
// prompts into the running batch).  Sequence s holds L_s tokens in the cache; its n_s
// new tokens (rows query_start_loc[s] .. +n_s of q) sit at positions L_s - n_s .. L_s - 1,
// and the token at position p attends causally to positions 0 .. p (the last W of them
// under a sliding window):
//     out[t][h] = sum_{u <= p} softmax_u(scale * q[t][h] . K_s[u][g]) V_s[u][g],  g = h / G.
//
// Work decomposition.  One CTA owns 128 query rows of one (sequence, kv head): 128/G
// consecutive tokens times the G query heads that share the kv head (row r = token
// r / G, head r % G), so one K/V tile read serves all G heads.  It walks the keys the
// rows need in tiles of 128:
//   S     = Q K^T      tcgen05.mma (M 128, N 128, K head_dim), Q and K K-major in
//                      128-byte swizzled shared memory, fp32 S in tensor memory;
//   softmax            row r is thread r is tensor-memory lane r: the row is read back
//                      with tcgen05.ld, masked (causal, window, context end), and its
//                      online-softmax state (m, l) updated in fp32; the 16-bit
//                      probabilities P go to shared memory in the K-major layout;
//   O += P V           tcgen05.mma (M 128, N head_dim, K 128) with V as an MN-major
//                      operand (the cache rows as TMA lays them down), accumulated in
//                      tensor memory; before it, each warp rescales its rows of O in
//                      tensor memory by 2^(m_old - m_new) (skipped when no row of the
//                      warp changed its maximum).  P is split into a high and a low
//                      16-bit part (two products) so the weights keep ~16 bits, as in
//                      the decode kernels' tensor-core path.
// K/V tiles stream through a two-stage TMA ring (one mbarrier per stage and operand);
// the tile two ahead is loaded while the current one is used.  Scores are kept in the
// log2 domain (scale * log2 e folded in), as in the decode kernels.
//
// Every wait is bounded: on a timeout the CTA records PA_DEVERR_TIMEOUT, waits (again
// bounded) for its copies and matrix operations in flight, frees its tensor memory and
// returns.
#pragma once

#include "pa_common.cuh"

namespace pa {

constexpr int kPfRows = 128;     // query rows per CTA = UMMA M = tensor-memory lanes
constexpr int kPfKeys = 128;     // keys per tile = UMMA N of S and K of P.V
constexpr int kPfThreads = 128;  // row r <-> thread r
constexpr int kPfStages = 2;     // K/V ring depth
constexpr int kPfTmemCols = 256; // S: columns [0, 128), O tile: [128, 128 + D)

struct PrefillParams {
    CUtensorMap qmap;  // 3-D [num_tokens][Hq][D] 16-bit, box {64, G, 128/G}, swizzle 128B
    CUtensorMap kmap;  // 2-D [num_blocks * Hkv * bs][D], box {64, min(bs, 128)}, swizzle 128B
    CUtensorMap vmap;
    void *out;
    const int32_t *block_tables;
    const int32_t *context_lens;
    const int32_t *query_start_loc;
    int num_seqs;
    int num_tokens;
    int num_q_heads;
    int num_kv_heads;
    int block_size;
    int bs_shift;
    int box_rows;  // min(block_size, 128)
    int num_blocks;
    int max_blocks_per_seq;
    int sliding_window;
    float scale_log2;
};

template <int D>
struct PfGeom {
    static constexpr int kHalves = D / 64;                // 128-byte column blocks of a row
    static constexpr int kRegion = 128 * 128;             // 128 rows of one column block
    static constexpr int kQ = kHalves * kRegion;          // Q tile
    static constexpr int kKV = kHalves * kRegion;         // one K (or V) stage
    static constexpr int kP = 2 * kRegion;                // P: 128 rows x 128 keys
    static constexpr int kOffK = kQ;
    static constexpr int kOffV = kOffK + kPfStages * kKV;
    static constexpr int kOffP = kOffV + kPfStages * kKV;  // high part of P
    static constexpr int kOffPlo = kOffP + kP;             // low part of P
    static constexpr int kOffBar = kOffPlo + kP;
    static constexpr int kBars = 1 + 2 * kPfStages + 2;  // q, k[2], v[2], s, o
    static constexpr int kSmem = kOffBar + 8 * kBars + 1024;  // + alignment slack
};

// ---------------------------------------------------------------- tcgen05 helpers

// Shared-memory matrix descriptor (sm_100 format): start address, leading and stride
// byte offsets (16-byte units), descriptor version 1, 128-byte swizzle.  K-major
// operands: rows of 128 bytes, 8-row groups 1024 bytes apart (stride offset); the
// leading offset is unused.  MN-major operand: 64-element column blocks `lbo` bytes
// apart, 8-row groups along K 1024 bytes apart.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr, uint32_t lbo) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1 << 46;  // version
    d |= (uint64_t)2 << 61;  // SWIZZLE_128B
    return d;
}

// Instruction descriptor of kind::f16: fp32 accumulate, A and B of type T, A K-major,
// B K-major or MN-major, shape M x N.
template <typename T>
__device__ __forceinline__ uint32_t umma_idesc(int M, int N, bool b_mn_major) {
    const uint32_t fmt = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
    return (1u << 4) | (fmt << 7) | (fmt << 10) | ((b_mn_major ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}

// Arrives on `bar` once every tcgen05.mma this thread issued before has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 consecutive fp32 columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}

// Stores 32 consecutive fp32 columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 3-D tiled TMA load (the q rows of one kv head's query-head group).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int x, int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void sts_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                       uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

// ---------------------------------------------------------------- the kernel

// grid = (an upper bound of the number of 128-row tiles, kv heads); CTAs past the last
// tile return at once.
template <typename T, int D, int G>
__global__ void __launch_bounds__(kPfThreads, 1)
    pa_prefill_kernel(const __grid_constant__ PrefillParams p) {
    pdl_wait_and_release();
    using Gm = PfGeom<D>;
    constexpr int kTpt = kPfRows / G;  // tokens per tile
    extern __shared__ uint8_t smem_raw[];
    __shared__ int sh_item[2];  // sequence, tile index within it
    __shared__ int warp_tot[kPfThreads / 32];
    __shared__ uint32_t sh_tmem;
    __shared__ int stage_ok[kPfStages];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = blockIdx.y;
    const int cta = blockIdx.x;

    // ---- 1. this CTA's (sequence, q tile): block-wide prefix sum of tiles per sequence.
    // Within a sequence the last (longest-context) tile comes first.
    if (tid == 0) sh_item[0] = -1;
    __syncthreads();
    int run = 0;
    for (int s0 = 0; s0 < p.num_seqs; s0 += kPfThreads) {
        const int s = s0 + tid;
        int nt = 0;
        if (s < p.num_seqs) {
            const int n = __ldg(p.query_start_loc + s + 1) - __ldg(p.query_start_loc + s);
            nt = n > 0 ? (n + kTpt - 1) / kTpt : 0;
        }
        int incl = nt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) warp_tot[warp] = incl;
        __syncthreads();
        int woff = 0, total = 0;
#pragma unroll
        for (int w = 0; w < kPfThreads / 32; ++w) {
            woff += (w < warp) ? warp_tot[w] : 0;
            total += warp_tot[w];
        }
        const int excl = run + woff + incl - nt;
        if (nt > 0 && cta >= excl && cta < excl + nt) {
            sh_item[0] = s;
            sh_item[1] = nt - 1 - (cta - excl);
        }
        run += total;
        __syncthreads();
        if (sh_item[0] >= 0 || cta < run) break;
    }
    const int s = sh_item[0];
    if (s < 0) return;
    const int qt = sh_item[1];
    const int q0 = __ldg(p.query_start_loc + s);
    const int n = __ldg(p.query_start_loc + s + 1) - q0;
    const int L = __ldg(p.context_lens + s);
    if (q0 < 0 || q0 + n > p.num_tokens || n > L || L > (p.max_blocks_per_seq << p.bs_shift)) {
        if (tid == 0 && qt == 0) raise_error(PA_DEVERR_CONTEXT);
        return;
    }
    const int W = p.sliding_window;
    const int tok0 = qt * kTpt;               // first token of the tile within the chunk
    const int ntok = min(kTpt, n - tok0);     // its valid tokens
    const int pos0 = L - n + tok0;            // position of its first token
    const int posN = pos0 + ntok - 1;         // position of its last valid token
    const int kv_begin = W > 0 ? max(0, pos0 - W + 1) : 0;  // first key any row attends
    const int j0 = kv_begin / kPfKeys, j1 = posN / kPfKeys + 1;

    // this thread's row
    const int rtok = tid / G, rh = tid % G;
    const bool rvalid = rtok < ntok;
    const int rpos = rvalid ? pos0 + rtok : -1;              // invalid rows attend nothing
    const int rlo = (W > 0 && rvalid) ? rpos - W + 1 : 0;

    // ---- 2. barriers, tensor memory
    const uint32_t sq = base, sk = base + Gm::kOffK, sv = base + Gm::kOffV, sp = base + Gm::kOffP;
    const uint32_t splo = base + Gm::kOffPlo;
    const uint32_t bar_q = base + Gm::kOffBar;
    const uint32_t bar_k0 = bar_q + 8, bar_v0 = bar_k0 + 8 * kPfStages;
    const uint32_t bar_s = bar_v0 + 8 * kPfStages, bar_o = bar_s + 8;
    if (tid == 0) {
        tma_prefetch_desc(&p.qmap);
        tma_prefetch_desc(&p.kmap);
        tma_prefetch_desc(&p.vmap);
        for (int i = 0; i < Gm::kBars; ++i) mbar_init(bar_q + 8 * i, 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&sh_tmem)),
                     "r"(kPfTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh_tmem;
    const uint32_t tmem_s = tmem, tmem_o = tmem + 128;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

    const int32_t *table = p.block_tables + (size_t)s * p.max_blocks_per_seq;
    const int BR = p.box_rows;
    // K/V tile jt -> stage: boxes of BR rows that overlap [kv_begin, L) are loaded
    auto load_kv = [&](int jt) {  // thread 0 only
        const int st = (jt - j0) % kPfStages;
        const int kv0 = jt * kPfKeys;
        int nload = 0;
        bool ok = true;
        for (int b = 0; b < kPfKeys / BR; ++b) {
            const int r0 = kv0 + b * BR;
            if (r0 < L && r0 + BR > kv_begin) {
                ++nload;
                const int blk = __ldg(table + (r0 >> p.bs_shift));
                ok = ok && (unsigned)blk < (unsigned)p.num_blocks;
            }
        }
        stage_ok[st] = ok ? 1 : 0;
        const uint32_t bk = bar_k0 + 8 * st, bv = bar_v0 + 8 * st;
        if (!ok) {
            raise_error(PA_DEVERR_BLOCK_ID);
            mbar_arrive(bk);
            mbar_arrive(bv);
            return;
        }
        const uint32_t bytes = (uint32_t)(nload * BR * 128 * Gm::kHalves);
        mbar_arrive_expect_tx(bk, bytes);
        mbar_arrive_expect_tx(bv, bytes);
        const uint64_t pol = l2_policy_evict_first();
        for (int b = 0; b < kPfKeys / BR; ++b) {
            const int r0 = kv0 + b * BR;
            if (r0 < L && r0 + BR > kv_begin) {
                const int blk = __ldg(table + (r0 >> p.bs_shift));
                const int y = (blk * p.num_kv_heads + g) * p.block_size + (r0 & (p.block_size - 1));
#pragma unroll
                for (int hf = 0; hf < Gm::kHalves; ++hf) {
                    const uint32_t off = hf * Gm::kRegion + b * BR * 128;
                    tma_load_2d(sk + st * Gm::kKV + off, &p.kmap, bk, 64 * hf, y, pol);
                    tma_load_2d(sv + st * Gm::kKV + off, &p.vmap, bv, 64 * hf, y, pol);
                }
            }
        }
    };

    int issued = j0;  // tiles whose K/V loads were issued: [j0, issued)
    if (tid == 0) {
        mbar_arrive_expect_tx(bar_q, (uint32_t)Gm::kQ);
#pragma unroll
        for (int hf = 0; hf < Gm::kHalves; ++hf)
            tma_load_3d(sq + hf * Gm::kRegion, &p.qmap, bar_q, 64 * hf, g * G, q0 + tok0);
        for (; issued < min(j1, j0 + kPfStages); ++issued) load_kv(issued);
    }
    __syncthreads();  // stage_ok of the first tiles

    const uint32_t idesc_s = umma_idesc<T>(kPfRows, kPfKeys, false);
    const uint32_t idesc_o = umma_idesc<T>(kPfRows, D, true);
    float m_run = -INFINITY, l_run = 0.f;
    bool failed = false;
    // thread 0: parity of a commit not yet waited for, or -1 (for the cleanup)
    int s_pending = -1, o_pending = -1;

    for (int jt = j0; jt < j1; ++jt) {
        const int it = jt - j0, st = it % kPfStages;
        const uint32_t ph = (uint32_t)((it / kPfStages) & 1);
        const int kv0 = jt * kPfKeys;
        bool bad = false;
        // (a) S = Q K^T
        if (tid == 0) {
            bool ok = (it > 0 || mbar_wait_bounded(bar_q, 0));
            ok = ok && mbar_wait_bounded(bar_k0 + 8 * st, ph);
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * Gm::kRegion + (kk & 3) * 32;
                    umma_f16(tmem_s, umma_desc_sw128(sq + koff, 16),
                             umma_desc_sw128(sk + st * Gm::kKV + koff, 16), idesc_s, kk > 0);
                }
                umma_commit(bar_s);
                s_pending = it & 1;
            } else {
                bad = true;
            }
        }
        // (b) the previous tile's P V has finished (P and its stage are free again; the
        // tensor core runs the S product above after it, so this rarely waits)
        if (it > 0) {
            const bool got = mbar_wait_bounded(bar_o, (uint32_t)((it - 1) & 1));
            if (tid == 0 && got) o_pending = -1;
            bad = bad || !got;
            if (tid == 0 && got && issued < j1) load_kv(issued++);  // into the freed stage
        }
        // (c) softmax of row `tid` over the tile's keys
        const bool got_s = mbar_wait_bounded(bar_s, (uint32_t)(it & 1));
        if (tid == 0 && got_s) s_pending = -1;
        bad = bad || !got_s;
        tc_fence_after();
        const bool tile_ok = stage_ok[st] != 0;
        float mx = -INFINITY;
#pragma unroll
        for (int cc = 0; cc < kPfKeys / 32; ++cc) {
            uint32_t v[32];
            tmem_ld32(tmem_s + lane_off + cc * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int key = kv0 + cc * 32 + e;
                const bool ok = tile_ok && key <= rpos && key >= rlo;
                mx = fmaxf(mx, ok ? __uint_as_float(v[e]) * p.scale_log2 : -INFINITY);
            }
        }
        const float m_new = fmaxf(m_run, mx);
        const float alpha = (m_new == -INFINITY) ? 1.f : fast_exp2(m_run - m_new);
        float sum = 0.f;
#pragma unroll
        for (int cc = 0; cc < kPfKeys / 32; ++cc) {
            uint32_t v[32];
            tmem_ld32(tmem_s + lane_off + cc * 32, v);
            tmem_wait_ld();
            // P = hi + lo: hi = RN(p), lo = RN(p - hi) in the input type, so that the two
            // P V products keep ~16 significant bits of every weight
            uint32_t ph_[16], pl_[16];
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
                const int key = kv0 + cc * 32 + e;
                const bool ok0 = tile_ok && key <= rpos && key >= rlo;
                const bool ok1 = tile_ok && key + 1 <= rpos && key + 1 >= rlo;
                const float p0 =
                    ok0 ? fast_exp2(__uint_as_float(v[e]) * p.scale_log2 - m_new) : 0.f;
                const float p1 =
                    ok1 ? fast_exp2(__uint_as_float(v[e + 1]) * p.scale_log2 - m_new) : 0.f;
                sum += p0 + p1;
                ph_[e >> 1] = Fmt<T>::pack_rn(p0, p1);
                const float2 h = Fmt<T>::unpack(ph_[e >> 1]);
                pl_[e >> 1] = Fmt<T>::pack_rn(p0 - h.x, p1 - h.y);
            }
            // keys cc*32 .. +31 of row tid: column block cc/2, 16-byte chunks 4(cc%2) .. +3
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                const int ch = (cc & 1) * 4 + c4;
                const uint32_t off = (cc >> 1) * Gm::kRegion + tid * 128 + ((ch ^ (tid & 7)) << 4);
                sts_v4(sp + off, ph_[4 * c4], ph_[4 * c4 + 1], ph_[4 * c4 + 2], ph_[4 * c4 + 3]);
                sts_v4(splo + off, pl_[4 * c4], pl_[4 * c4 + 1], pl_[4 * c4 + 2], pl_[4 * c4 + 3]);
            }
        }
        l_run = l_run * alpha + sum;
        m_run = m_new;
        // (d) rescale the running output in tensor memory by alpha (rows of this warp)
        if (it > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t v[32];
                tmem_ld32(tmem_o + lane_off + cc * 32, v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
                tmem_st32(tmem_o + lane_off + cc * 32, v);
            }
            tmem_wait_st();
        }
        // V rows outside [kv_begin, L) (not loaded, or past the context) -> 0, so that
        // their zero probabilities cannot meet a NaN
        const bool edge = !tile_ok || kv0 < kv_begin || kv0 + kPfKeys > L;
        if (edge) {
            bad = bad || !mbar_wait_bounded(bar_v0 + 8 * st, ph);
            const int key = kv0 + tid;
            if (!tile_ok || key < kv_begin || key >= L) {
#pragma unroll
                for (int hf = 0; hf < Gm::kHalves; ++hf)
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        sts_v4(sv + st * Gm::kKV + hf * Gm::kRegion + tid * 128 + c * 16, 0, 0,
                               0, 0);
            }
        }
        fence_proxy_async_smem();  // P (and zeroed V rows) -> the tensor-core reads
        tc_fence_before();
        if (__syncthreads_or(bad)) {
            failed = true;
            break;
        }
        // (e) O += P V
        if (tid == 0) {
            tc_fence_after();
            if (mbar_wait_bounded(bar_v0 + 8 * st, ph)) {
#pragma unroll
                for (int kk = 0; kk < 2 * (kPfKeys / 16); ++kk) {  // P_hi V, then P_lo V
                    const int k = kk % (kPfKeys / 16);
                    const uint32_t aoff = (kk < kPfKeys / 16 ? sp : splo) + (k >> 2) * Gm::kRegion +
                                          (k & 3) * 32;
                    umma_f16(tmem_o, umma_desc_sw128(aoff, 16),
                             umma_desc_sw128(sv + st * Gm::kKV + k * 16 * 128, Gm::kRegion),
                             idesc_o, (it > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(bar_o);
                o_pending = it & 1;
            } else {
                // nothing was issued: the next wait on bar_o times out and ends the tile
                // loop through the barrier above
            }
        }
    }
    // the last P V
    if (!failed && j1 > j0) {
        const bool got = mbar_wait_bounded(bar_o, (uint32_t)((j1 - j0 - 1) & 1));
        if (tid == 0 && got) o_pending = -1;
        failed = __syncthreads_or(!got);
    }

    if (failed) {
        if (tid == 0) {
            raise_error(PA_DEVERR_TIMEOUT);
            // let the copies and matrix operations in flight finish (bounded)
            (void)mbar_wait_bounded(bar_q, 0);
            for (int jt = j0; jt < issued; ++jt) {
                const int it = jt - j0, st = it % kPfStages;
                const uint32_t ph = (uint32_t)((it / kPfStages) & 1);
                (void)mbar_wait_bounded(bar_k0 + 8 * st, ph);
                (void)mbar_wait_bounded(bar_v0 + 8 * st, ph);
            }
            if (s_pending >= 0) (void)mbar_wait_bounded(bar_s, (uint32_t)s_pending);
            if (o_pending >= 0) (void)mbar_wait_bounded(bar_o, (uint32_t)o_pending);
        }
    } else {
        tc_fence_after();
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        T *dst = reinterpret_cast<T *>(p.out) +
                 ((size_t)(q0 + tok0 + rtok) * p.num_q_heads + (size_t)g * G + rh) * D;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t v[32];
            tmem_ld32(tmem_o + lane_off + cc * 32, v);
            tmem_wait_ld();
            if (rvalid) {
#pragma unroll
                for (int e = 0; e < 32; e += 8) {
                    uint4 w;
                    w.x = Fmt<T>::pack_rn(__uint_as_float(v[e]) * inv, __uint_as_float(v[e + 1]) * inv);
                    w.y = Fmt<T>::pack_rn(__uint_as_float(v[e + 2]) * inv, __uint_as_float(v[e + 3]) * inv);
                    w.z = Fmt<T>::pack_rn(__uint_as_float(v[e + 4]) * inv, __uint_as_float(v[e + 5]) * inv);
                    w.w = Fmt<T>::pack_rn(__uint_as_float(v[e + 6]) * inv, __uint_as_float(v[e + 7]) * inv);
                    *reinterpret_cast<uint4 *>(dst + cc * 32 + e) = w;
                }
            }
        }
    }

    // ---- teardown: free the tensor memory (the warp that allocated it)
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kPfTmemCols)
                     : "memory");
    }
}

}  // namespace pa
