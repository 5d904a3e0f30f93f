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
// Work decomposition.  A query tile is 128 rows of one (sequence, kv head): 128/G
// consecutive tokens times the G query heads that share the kv head (row r = token r / G,
// head r % G), so one K/V tile read serves all G heads.  A CTA owns two consecutive
// query tiles, A and B, and walks the keys they need in tiles of 64:
//   S_X   = Q_X K^T     tcgen05.mma (M 128, N 64, K head_dim): Q_X and K K-major in
//                       128-byte swizzled shared memory, fp32 S_X in tensor memory, two
//                       buffers per query tile so that the product for key tile j+2 can
//                       run while the softmax of tile j+1 and P V of tile j are pending;
//   softmax             a warpgroup per query tile; row r is thread r is tensor-memory
//                       lane r.  The row is read from tensor memory in two 32-column
//                       chunks (double-buffered), masked (causal, window, context end;
//                       tiles wholly inside every row's range skip the masks), and the
//                       online-softmax state (m, l) updated in fp32; the probabilities go
//                       back over S_X in tensor memory as a high and a low 16-bit part
//                       (tcgen05.st);
//   O_X  += P_X V       tcgen05.mma with P_X read from tensor memory and V as an MN-major
//                       shared-memory operand (the cache rows as TMA lays them down), two
//                       products (high and low part) so the weights keep ~16 bits.  The
//                       reference maximum of a row moves only when the row maximum
//                       exceeds it by more than 2^8; only then does the warp rescale its
//                       rows of O_X (in tensor memory) by 2^(m_old - m_new).
// Roles (warp specialisation): warps 0-3 softmax A, warps 4-7 softmax B, warps 8 and 9
// issue the matrix products of A and of B, warp 10 issues the TMA loads of Q and of a
// four-stage K/V ring (and zeroes the V rows of edge tiles outside the attended keys).
// The products of one query tile overlap the softmax of the other, and a query tile's next
// scores are computed while its current softmax runs.  Scores are kept in the log2 domain
// (scale * log2 e folded into one FFMA), as in the decode kernels.
//
// Every wait is bounded: on a timeout a role records PA_DEVERR_TIMEOUT and stops, the
// others see the shared failure flag (or time out themselves), the copies and products
// in flight are waited for (bounded), and the tensor memory is freed.
#pragma once

#include "pa_common.cuh"

namespace pa {

constexpr int kPfRows = 128;        // query rows per tile = UMMA M = tensor-memory lanes
constexpr int kPfKeys = 64;         // keys per tile = UMMA N of S and K of P.V
constexpr int kPfSoftWarps = 8;     // two softmax warpgroups
constexpr int kPfMmaWarp = 8;       // warps 8 and 9: the P V products of query tiles A and B
constexpr int kPfLoadWarp = 10;     // TMA loads of Q and K (and the tensor-memory allocation)
constexpr int kPfLoadWarpV = 11;    // TMA loads of V (and the zeroing of edge-tile V rows)
constexpr int kPfSWarp = 12;        // warps 12 and 13: the S products of query tiles A and B
constexpr int kPfThreads = 448;
constexpr int kPfStages = 4;        // K/V ring depth
// tensor memory of query tile X: two S/P buffers at [256X, 256X + 64) and [256X + 64,
// 256X + 128) (key tile i of X uses buffer i % 2), O at [256X + 128, 256X + 128 + D)
constexpr int kPfTmemCols = 512;
constexpr float kPfRescaleLog2 = 8.f;  // move the softmax reference max only past 2^8
#ifndef PA_PREFILL_SPLIT_P
#define PA_PREFILL_SPLIT_P 1
#endif
// P as high + low 16-bit parts (two P V products): weights keep ~16 significant bits
constexpr bool kPfSplitP = PA_PREFILL_SPLIT_P != 0;

struct PrefillParams {
    CUtensorMap qmap;  // 3-D [num_tokens][Hq][D] 16-bit, box {64, G, 128/G}, swizzle 128B
    CUtensorMap kmap;  // 2-D [num_blocks * Hkv * bs][D], box {64, min(bs, 64)}, swizzle 128B
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
    int box_rows;  // min(block_size, 64)
    int num_blocks;
    int max_blocks_per_seq;
    int sliding_window;
    float scale_log2;
    int heads_inner;  // 1: blockIdx.x is the kv head and blockIdx.y the tile pair; 0: swapped
};

template <int D>
struct PfGeom {
    static constexpr int kHalves = D / 64;                // 128-byte column blocks of a row
    static constexpr int kRegion = kPfRows * 128;         // 128 query rows of one column block
    static constexpr int kKVRegion = kPfKeys * 128;       // 64 key rows of one column block
    static constexpr int kQ = kHalves * kRegion;          // one Q tile
    static constexpr int kKV = kHalves * kKVRegion;       // one K (or V) stage
    static constexpr int kOffK = 2 * kQ;
    static constexpr int kOffV = kOffK + kPfStages * kKV;
    static constexpr int kOffBar = kOffV + kPfStages * kKV;
    // q, k[stages], v[stages], v_edge[stages], k_empty[stages], v_empty[stages], s[2][2],
    // p[2][2], o[2], fin[2], pv_done[2][2], s_fin[2]
    static constexpr int kBars = 1 + 5 * kPfStages + 18;
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

// Stores 16 consecutive 32-bit columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t *r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// tcgen05.wait::ld that also names the 32 registers of the load it completes, so the
// compiler cannot move their uses above it.
__device__ __forceinline__ void tmem_wait_ld_regs(uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.wait::ld.sync.aligned;"
        : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
          "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]),
          "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]),
          "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]),
          "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]),
          "+r"(r[31])
        :
        : "memory");
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

// A from tensor memory (lane = row, a 32-bit column holds two consecutive 16-bit K
// elements, the first in the low half), B from shared memory.
__device__ __forceinline__ void umma_f16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t b,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(b), "r"(idesc), "r"(accumulate));
}

// ---------------------------------------------------------------- the kernel

// One query tile's place in its sequence.
struct PfTile {
    bool live;
    int tok0, ntok;   // first token (within the chunk) and valid tokens
    int pos0;         // position of its first token
    int kv_begin;     // first key any row attends
    int j0, j1;       // key tiles [j0, j1)
};

__device__ __forceinline__ PfTile pf_tile(int qt, int tpt, int n, int L, int W) {
    PfTile t;
    t.tok0 = qt * tpt;
    t.live = t.tok0 < n;
    t.ntok = t.live ? min(tpt, n - t.tok0) : 0;
    t.pos0 = L - n + t.tok0;
    t.kv_begin = W > 0 ? max(0, t.pos0 - W + 1) : 0;
    t.j0 = t.kv_begin / kPfKeys;
    t.j1 = t.live ? (t.pos0 + t.ntok - 1) / kPfKeys + 1 : t.j0;
    return t;
}

// grid = (kv heads, an upper bound of the number of tile pairs), or the two swapped when
// the bound exceeds the grid's y limit; CTAs past the last pair return at once.
template <typename T, int D, int G>
__global__ void __launch_bounds__(kPfThreads, 1)
    pa_prefill_kernel(const __grid_constant__ PrefillParams p) {
    pdl_wait_and_release();
    using Gm = PfGeom<D>;
    constexpr int kTpt = kPfRows / G;  // tokens per query tile
    extern __shared__ uint8_t smem_raw[];
    __shared__ int sh_item[2];  // sequence, pair index within it
    __shared__ int warp_tot[kPfThreads / 32];
    __shared__ uint32_t sh_tmem;
    __shared__ volatile int sh_fail;
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // kv head and tile-pair slot.  With the kv head as blockIdx.x, the hardware hands out
    // every head of one pair before the next pair, so the last CTAs are the shortest pairs
    // of the last sequence instead of all pairs of the last kv head.
    const int g = p.heads_inner ? blockIdx.x : blockIdx.y;
    const int cta = p.heads_inner ? blockIdx.y : blockIdx.x;

    // ---- 1. this CTA's (sequence, tile pair): block-wide prefix sum of pairs per
    // sequence; within a sequence the last (longest-context) pair comes first.
    if (tid == 0) {
        sh_item[0] = -1;
        sh_fail = 0;
    }
    __syncthreads();
    int run = 0;
    for (int s0 = 0; s0 < p.num_seqs; s0 += kPfThreads) {
        const int s = s0 + tid;
        int np = 0;
        if (s < p.num_seqs) {
            const int n = __ldg(p.query_start_loc + s + 1) - __ldg(p.query_start_loc + s);
            const int nt = n > 0 ? (n + kTpt - 1) / kTpt : 0;
            np = (nt + 1) / 2;
        }
        int incl = np;
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
        const int excl = run + woff + incl - np;
        if (np > 0 && cta >= excl && cta < excl + np) {
            sh_item[0] = s;
            sh_item[1] = np - 1 - (cta - excl);
        }
        run += total;
        __syncthreads();
        if (sh_item[0] >= 0 || cta < run) break;
    }
    const int s = sh_item[0];
    if (s < 0) return;
    const int q0 = __ldg(p.query_start_loc + s);
    const int n = __ldg(p.query_start_loc + s + 1) - q0;
    const int L = __ldg(p.context_lens + s);
    if (q0 < 0 || q0 + n > p.num_tokens || n > L || L > (p.max_blocks_per_seq << p.bs_shift)) {
        if (tid == 0 && sh_item[1] == 0) raise_error(PA_DEVERR_CONTEXT);
        return;
    }
    const int W = p.sliding_window;
    const PfTile ta = pf_tile(2 * sh_item[1], kTpt, n, L, W);
    const PfTile tb = pf_tile(2 * sh_item[1] + 1, kTpt, n, L, W);
    const int j0 = ta.j0, j1 = max(ta.j1, tb.live ? tb.j1 : ta.j1);  // tb.j0 >= ta.j0
    const int kv_begin = ta.kv_begin;  // first key either tile attends

    // ---- 2. barriers, tensor memory
    const uint32_t sq = base, sk = base + Gm::kOffK, sv = base + Gm::kOffV;
    const uint32_t bar_q = base + Gm::kOffBar;
    const uint32_t bar_k0 = bar_q + 8, bar_v0 = bar_k0 + 8 * kPfStages;
    const uint32_t bar_vt0 = bar_v0 + 8 * kPfStages;     // V of an edge tile landed (producer)
    // a stage's K and its V are released separately (both MMA warps commit each): K once
    // the S product that reads it has finished, V once the P V product has
    const uint32_t bar_ek0 = bar_vt0 + 8 * kPfStages;
    const uint32_t bar_ev0 = bar_ek0 + 8 * kPfStages;
    // per query tile X = 0 (A), 1 (B) and S/P buffer b: S ready, P written (one barrier
    // per buffer, so that neither side can get two phases ahead of the other)
    const uint32_t bar_s0 = bar_ev0 + 8 * kPfStages;     // + 8 (2X + b)
    const uint32_t bar_p0 = bar_s0 + 32;                 // + 8 (2X + b)
    const uint32_t bar_o0 = bar_p0 + 32;                 // + 8X: P_X V done
    const uint32_t bar_f0 = bar_o0 + 16;                 // + 8X: every P V of X done
    // per query tile X and buffer b: the P V that read the buffer's P has finished (the S
    // warp may then overwrite it); one barrier per buffer, as for S and P
    const uint32_t bar_pv0 = bar_f0 + 16;                // + 8 (2X + b)
    const uint32_t bar_sf0 = bar_pv0 + 32;               // + 8X: every S product of X done
    if (tid == 0) {
        tma_prefetch_desc(&p.qmap);
        tma_prefetch_desc(&p.kmap);
        tma_prefetch_desc(&p.vmap);
        mbar_init(bar_q, 1);
        for (int i = 0; i < kPfStages; ++i) {
            mbar_init(bar_k0 + 8 * i, 1);
            mbar_init(bar_v0 + 8 * i, 1);
            mbar_init(bar_vt0 + 8 * i, 1);
            mbar_init(bar_ek0 + 8 * i, 2);  // one commit per MMA warp
            mbar_init(bar_ev0 + 8 * i, 2);
        }
        for (int i = 0; i < 4; ++i) {
            mbar_init(bar_s0 + 8 * i, 1);
            mbar_init(bar_p0 + 8 * i, 4);  // one arrival per softmax warp
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(bar_o0 + 8 * x, 1);
            mbar_init(bar_f0 + 8 * x, 1);
            mbar_init(bar_sf0 + 8 * x, 1);
        }
        for (int i = 0; i < 4; ++i) mbar_init(bar_pv0 + 8 * i, 1);
        fence_barrier_init();
    }
    if (warp == kPfLoadWarp) {
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

    if (warp == kPfLoadWarp || warp == kPfLoadWarpV) {
        // ============================ TMA producers (lane 0 issues): warp 10 loads Q and
        // the K ring, warp 11 the V ring and zeroes edge V rows.  Each ring stage is reused
        // once both MMA warps have released it: K after its S product, V after its P V, so
        // the K loads run ahead of the V loads by the two key tiles S is computed ahead.
        const bool is_k = warp == kPfLoadWarp;
        const int32_t *table = p.block_tables + (size_t)s * p.max_blocks_per_seq;
        const int BR = p.box_rows;
        const uint64_t pol = l2_policy_evict_first();
        if (is_k && lane == 0) {
            mbar_arrive_expect_tx(bar_q, (uint32_t)((tb.live ? 2 : 1) * Gm::kQ));
#pragma unroll
            for (int hf = 0; hf < Gm::kHalves; ++hf) {
                tma_load_3d(sq + hf * Gm::kRegion, &p.qmap, bar_q, 64 * hf, g * G, q0 + ta.tok0);
                if (tb.live)
                    tma_load_3d(sq + Gm::kQ + hf * Gm::kRegion, &p.qmap, bar_q, 64 * hf, g * G,
                                q0 + tb.tok0);
            }
        }
        const uint32_t bar_empty0 = is_k ? bar_ek0 : bar_ev0;
        const uint32_t sbase = is_k ? sk : sv;
        const CUtensorMap *map = is_k ? &p.kmap : &p.vmap;
        int issued = j0;
        int vt_uses[kPfStages];
#pragma unroll
        for (int i = 0; i < kPfStages; ++i) vt_uses[i] = 0;
        // the table entries of a tile's boxes, one per lane (lane b: box b; the boxes of
        // keys outside [kv_begin, L) read nothing), loaded one tile ahead of their use
        const int nbox = kPfKeys / BR;
        auto tab_load = [&](int jt) -> int {
            const int r0 = jt * kPfKeys + lane * BR;
            if (jt >= j1 || lane >= nbox || r0 >= L || r0 + BR <= kv_begin) return -1;
            return __ldg(table + (r0 >> p.bs_shift));
        };
        int tab_next = tab_load(j0);
        bool ok = true;
        for (int jt = j0; jt < j1 && ok; ++jt) {
            const int it = jt - j0, st = it % kPfStages;
            if (it >= kPfStages) {
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(
                                                 bar_empty0 + 8 * st,
                                                 (uint32_t)(((it / kPfStages) - 1) & 1)));
                if (!ok) break;
            }
            if (__any_sync(0xffffffffu, sh_fail != 0)) {
                ok = false;
                break;
            }
            const int kv0 = jt * kPfKeys;
            const int tab_cur = tab_next;
            tab_next = tab_load(jt + 1);
            const int r0l = kv0 + lane * BR;
            const bool live = lane < nbox && r0l < L && r0l + BR > kv_begin;
            const unsigned live_mask = __ballot_sync(0xffffffffu, live);
            const bool tab_ok =
                !__any_sync(0xffffffffu, live && (unsigned)tab_cur >= (unsigned)p.num_blocks);
            // nothing loaded after a bad entry: the tile reads as all-masked
            const int nload = tab_ok ? __popc(live_mask) : 0;
            const int y_l = live && tab_ok ? (tab_cur * p.num_kv_heads + g) * p.block_size +
                                                 (r0l & (p.block_size - 1))
                                           : 0;
            int ys[kPfKeys / 8];  // box rows are at least 8
#pragma unroll
            for (int b = 0; b < kPfKeys / 8; ++b) ys[b] = __shfl_sync(0xffffffffu, y_l, b);
            // an edge tile (keys outside [kv_begin, L), or a bad table entry): its V lands
            // on a private barrier, the rows outside the attended keys are zeroed, then V
            // is released
            const bool edge = !is_k && (!tab_ok || kv0 < kv_begin || kv0 + kPfKeys > L);
            const uint32_t bk = bar_k0 + 8 * st, bv = bar_v0 + 8 * st, bvt = bar_vt0 + 8 * st;
            const uint32_t bar = is_k ? bk : (edge ? bvt : bv);
            const uint32_t bytes = (uint32_t)(nload * BR * 128 * Gm::kHalves);
            if (lane == 0) {
                if (!tab_ok && is_k) raise_error(PA_DEVERR_BLOCK_ID);
                mbar_arrive_expect_tx(bar, bytes);
                if (tab_ok) {
#pragma unroll
                    for (int b = 0; b < kPfKeys / 8; ++b) {
                        if ((live_mask >> b) & 1u) {
#pragma unroll
                            for (int hf = 0; hf < Gm::kHalves; ++hf) {
                                const uint32_t off = hf * Gm::kKVRegion + b * BR * 128;
                                tma_load_2d(sbase + st * Gm::kKV + off, map, bar, 64 * hf, ys[b],
                                            pol);
                            }
                        }
                    }
                }
            }
            __syncwarp();
            issued = jt + 1;
            if (edge) {
                ok = __all_sync(0xffffffffu,
                                mbar_wait_bounded(bvt, (uint32_t)(vt_uses[st] & 1)));
                ++vt_uses[st];
                if (!ok) break;
                const int lo = tab_ok ? max(0, kv_begin - kv0) : kPfKeys;
                const int hi = tab_ok ? min(kPfKeys, L - kv0) : 0;
                for (int idx = lane; idx < kPfKeys * Gm::kHalves * 8; idx += 32) {
                    const int r = idx / (Gm::kHalves * 8), c = idx % (Gm::kHalves * 8);
                    if (r < lo || r >= hi)
                        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(
                                         sv + st * Gm::kKV + (c >> 3) * Gm::kKVRegion + r * 128 +
                                         (c & 7) * 16),
                                     "r"(0)
                                     : "memory");
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bv);
            }
        }
        if (!ok) {
            if (lane == 0) raise_error(PA_DEVERR_TIMEOUT);
            sh_fail = 1;
        }
        // cleanup: the loads this warp issued have landed (bounded)
        if (lane == 0) {
            if (is_k) (void)mbar_wait_bounded(bar_q, 0);
            for (int jt = max(j0, issued - kPfStages); jt < issued; ++jt) {
                const int it = jt - j0, st = it % kPfStages;
                const uint32_t ph = (uint32_t)((it / kPfStages) & 1);
                (void)mbar_wait_bounded((is_k ? bar_k0 : bar_v0) + 8 * st, ph);
            }
        }
        __syncwarp();
    } else if (warp >= kPfMmaWarp) {
        // ============================ products of query tile X (lane 0 issues): warps 8
        // and 9 the P V products, warps 12 and 13 the S products, so that the P V of a tile
        // is issued as soon as its P is written, even while the S products queue
        const bool s_role = warp >= kPfSWarp;
        const int x = warp - (s_role ? kPfSWarp : kPfMmaWarp);
        const PfTile &t = x == 0 ? ta : tb;
        const uint32_t idesc_s = umma_idesc<T>(kPfRows, kPfKeys, false);
        const uint32_t idesc_o = umma_idesc<T>(kPfRows, D, true);
        auto wait_all = [&](uint32_t bar, uint32_t par) {
            return __all_sync(0xffffffffu, mbar_wait_bounded(bar, par));
        };
        auto need = [&](int jt) { return t.live && jt >= t.j0 && jt < t.j1; };
        auto stage_of = [&](int jt) { return (jt - j0) % kPfStages; };
        auto phase_of = [&](int jt) { return (uint32_t)(((jt - j0) / kPfStages) & 1); };
        // descriptors built once; each product adds a constant start-address offset
        const uint64_t dq = umma_desc_sw128(sq + x * Gm::kQ, 16);
        const uint64_t dk = umma_desc_sw128(sk, 16);
        const uint64_t dv = umma_desc_sw128(sv, Gm::kKVRegion);
        // S_X = Q_X K_jt into X's buffer (jt - j0_X) % 2
        auto issue_s = [&](int jt) {
            const int st = stage_of(jt);
            const int b = (jt - t.j0) & 1;
            if (lane == 0) {
                tc_fence_after();
                const uint64_t dks = dk + (uint64_t)((st * Gm::kKV) >> 4);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t qoff = ((kk >> 2) * Gm::kRegion + (kk & 3) * 32) >> 4;
                    const uint32_t koff = ((kk >> 2) * Gm::kKVRegion + (kk & 3) * 32) >> 4;
                    umma_f16(tmem + 256 * x + 64 * b, dq + qoff, dks + koff, idesc_s, kk > 0);
                }
                umma_commit(bar_s0 + 8 * (2 * x + b));
            }
            __syncwarp();
        };
        // O_X += P_X V_jt (high, then low part of P from X's buffer)
        auto issue_pv = [&](int jt) {
            const int st = stage_of(jt);
            const uint32_t pcol = 256 * x + 64 * ((jt - t.j0) & 1);
            const bool first = jt == t.j0;
            if (lane == 0) {
                tc_fence_after();
                const uint64_t dvs = dv + (uint64_t)((st * Gm::kKV) >> 4);
#pragma unroll
                for (int kk = 0; kk < (kPfSplitP ? 2 : 1) * (kPfKeys / 16); ++kk) {
                    const int k = kk % (kPfKeys / 16);
                    const uint32_t acol = pcol + (kk >= kPfKeys / 16 ? 32 : 0) + k * 8;
                    umma_f16_ts(tmem + 256 * x + 128, tmem + acol, dvs + (uint64_t)((k * 16 * 128) >> 4),
                                idesc_o, (!first || kk > 0) ? 1u : 0u);
                }
                umma_commit(bar_o0 + 8 * x);
                umma_commit(bar_pv0 + 8 * (2 * x + ((jt - t.j0) & 1)));
            }
            __syncwarp();
        };
        if (s_role) {
            // S of every key tile this query tile needs, two tiles ahead of its softmax:
            // into buffer i % 2 once the P V that read that buffer (tile i - 2) is done.
            // Each tile's K is released by both S warps (whether or not this one needs
            // it) once the products issued so far are done; every S warp waits each K
            // before releasing it, so that neither releases a stage a ring's length ahead
            // of the loads.
            bool ok = wait_all(bar_q, 0);
            for (int jn = j0; ok && jn < j1; ++jn) {
                if (__any_sync(0xffffffffu, sh_fail != 0)) {
                    ok = false;
                    break;
                }
                ok = wait_all(bar_k0 + 8 * stage_of(jn), phase_of(jn));
                if (!ok) break;
                if (need(jn)) {
                    const int i = jn - t.j0;
                    if (i >= 2) {
                        ok = wait_all(bar_pv0 + 8 * (2 * x + (i & 1)),
                                      (uint32_t)(((i - 2) >> 1) & 1));
                        if (!ok) break;
                    }
                    issue_s(jn);
                }
                if (lane == 0) umma_commit(bar_ek0 + 8 * stage_of(jn));
                __syncwarp();
            }
            if (!ok) {
                if (lane == 0) raise_error(PA_DEVERR_TIMEOUT);
                sh_fail = 1;
            }
            // the S products this warp issued have finished (bounded) before the tensor
            // memory is freed
            if (lane == 0) {
                umma_commit(bar_sf0 + 8 * x);
                (void)mbar_wait_bounded(bar_sf0 + 8 * x, 0);
            }
            __syncwarp();
        } else {
            bool ok = true;
            for (int jt = j0; ok && jt < j1; ++jt) {
                if (__any_sync(0xffffffffu, sh_fail != 0)) {
                    ok = false;
                    break;
                }
                const int st = stage_of(jt);
                // every P V warp waits each tile's V, so that neither commits a stage's
                // release a ring's length ahead of the loads
                ok = wait_all(bar_v0 + 8 * st, phase_of(jt));
                if (!ok) break;
                if (need(jt)) {
                    const int i = jt - t.j0;
                    ok = wait_all(bar_p0 + 8 * (2 * x + (i & 1)), (uint32_t)((i >> 1) & 1));
                    if (!ok) break;
                    issue_pv(jt);
                }
                if (lane == 0) umma_commit(bar_ev0 + 8 * st);  // V of stage st, after this P V
                __syncwarp();
            }
            if (ok) {
                // completes when every P V of this query tile (its last included) is done
                if (lane == 0 && t.live) umma_commit(bar_f0 + 8 * x);
                __syncwarp();
            } else {
                if (lane == 0) raise_error(PA_DEVERR_TIMEOUT);
                sh_fail = 1;
                // cleanup: the products issued so far have finished (bounded)
                if (lane == 0) {
                    umma_commit(bar_f0 + 8 * x);
                    (void)mbar_wait_bounded(bar_f0 + 8 * x, 0);
                }
                __syncwarp();
            }
        }
    } else {
        // ============================ softmax warpgroup X (rows = threads 128X .. 128X+127)
        const int x = warp / 4;
        const PfTile &t = x == 0 ? ta : tb;
        const int row = tid & 127;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tO = tmem + 256 * x + 128 + lane_off;
        const int rtok = row / G, rh = row % G;
        const bool rvalid = t.live && rtok < t.ntok;
        const int rpos = rvalid ? t.pos0 + rtok : -1;
        const int rlo = (W > 0 && rvalid) ? rpos - W + 1 : 0;
        // this row attends keys [key_base, key_base + key_span]: a key is in iff
        // key - key_base <= key_span as unsigned (one compare per element); a row that
        // attends nothing gets a base every key is below, modulo 2^32
        const int key_lo = max(rlo, kv_begin);
        const bool row_any = rpos >= key_lo;
        const unsigned key_base = row_any ? (unsigned)key_lo : 0x80000000u;
        const unsigned key_span = row_any ? (unsigned)(rpos - key_lo) : 0u;
        // every row of the tile attends keys [key_all_lo, key_all_hi] (valid tokens only)
        const bool all_rows = t.live && t.ntok == kTpt;
        const int key_all_hi = t.pos0;                          // min over rows of rpos
        const int key_all_lo = W > 0 ? t.pos0 + t.ntok - W : 0;  // max over rows of rlo
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        int i = 0;
        for (int jt = t.j0; t.live && jt < t.j1; ++jt, ++i) {
            if (__any_sync(0xffffffffu, sh_fail != 0)) {
                ok = false;
                break;
            }
            const int kv0 = jt * kPfKeys;
            const uint32_t tS = tmem + 256 * x + 64 * (i & 1) + lane_off;  // S/P buffer
            ok = mbar_wait_bounded(bar_s0 + 8 * (2 * x + (i & 1)), (uint32_t)((i >> 1) & 1));
            if (!__all_sync(0xffffffffu, ok)) {
                ok = false;
                break;
            }
            tc_fence_after();
            // keys inside every row's range, and nothing past the context or before the
            // loaded keys: no per-element mask
            const bool full = all_rows && kv0 + kPfKeys - 1 <= key_all_hi && kv0 >= key_all_lo &&
                              kv0 >= kv_begin;
            const float c2 = p.scale_log2;  // > 0 (checked on the host)
            // pass 1: the tile's row maximum of the raw scores (8 independent partial
            // maxima; scale > 0 keeps the order); the load of chunk c+1 overlaps chunk c
            float mxp[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) mxp[k] = -INFINITY;
            {
                uint32_t va[32], vb[32];
                tmem_ld32(tS, va);
                tmem_wait_ld_regs(va);
#pragma unroll
                for (int c = 0; c < kPfKeys / 32; ++c) {
                    uint32_t(&cur)[32] = (c & 1) ? vb : va;
                    uint32_t(&nxt)[32] = (c & 1) ? va : vb;
                    if (c + 1 < kPfKeys / 32) tmem_ld32(tS + 32 * (c + 1), nxt);
                    if (full) {
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            mxp[e & 7] = fmaxf(mxp[e & 7], __uint_as_float(cur[e]));
                    } else {
                        const unsigned dlo = (unsigned)(kv0 + 32 * c) - key_base;
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const bool in = dlo + (unsigned)e <= key_span;
                            mxp[e & 7] = fmaxf(mxp[e & 7], in ? __uint_as_float(cur[e]) : -INFINITY);
                        }
                    }
                    if (c + 1 < kPfKeys / 32) tmem_wait_ld_regs(nxt);
                }
            }
            const float mraw = fmaxf(fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3])),
                                     fmaxf(fmaxf(mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7])));
            const float mx = mraw * c2;  // -inf stays -inf
            // The reference maximum moves only when the row maximum exceeds it by more
            // than 2^8 (weights stay <= 256; O and l share the reference, so the result is
            // exact either way) -- most tiles then need no rescale of O.
            const bool upd = mx > m_run + kPfRescaleLog2 || (m_run == -INFINITY && mx > -INFINITY);
            const float m_new = upd ? mx : m_run;
            const float alpha = (upd && m_run != -INFINITY) ? fast_exp2(m_run - m_new) : 1.f;
            // a row of this warp moved its reference: once the previous P_X V has
            // finished, rescale the warp's rows of O_X (otherwise the next P V simply
            // accumulates onto O_X after the previous one, same accumulator, in order)
            if (i > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                ok = mbar_wait_bounded(bar_o0 + 8 * x, (uint32_t)((i - 1) & 1));
                if (!__all_sync(0xffffffffu, ok)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t o[32];
                    tmem_ld32(tO + cc * 32, o);
                    tmem_wait_ld_regs(o);
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_st32(tO + cc * 32, o);
                }
            }
            // pass 2: P = hi + lo, written over S in its buffer: the 64 keys' high part in
            // columns 0 .. 31, the low part in 32 .. 63 (two keys per column).  A row with
            // nothing attended yet (m = -inf) gets zeros.  Chunk 1 is loaded before chunk 0
            // is stored (chunk 0's low part lands in chunk 1's columns).
            const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
            float sump[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) sump[k] = 0.f;
            {
                uint32_t va[32], vb[32];
                tmem_ld32(tS, va);
                tmem_wait_ld_regs(va);
#pragma unroll
                for (int c = 0; c < kPfKeys / 32; ++c) {
                    uint32_t(&cur)[32] = (c & 1) ? vb : va;
                    uint32_t(&nxt)[32] = (c & 1) ? va : vb;
                    if (c + 1 < kPfKeys / 32) tmem_ld32(tS + 32 * (c + 1), nxt);
                    // exponent = score * scale log2 e - reference, one FFMA; masked -> 0
                    float xe[32];
                    if (full) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) xe[e] = fmaf(__uint_as_float(cur[e]), c2, -m_use);
                    } else {
                        const unsigned dlo = (unsigned)(kv0 + 32 * c) - key_base;
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const bool in = dlo + (unsigned)e <= key_span;
                            xe[e] = in ? fmaf(__uint_as_float(cur[e]), c2, -m_use) : -INFINITY;
                        }
                    }
                    uint32_t ph_[16], pl_[16];
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const float p0 = fast_exp2(xe[e]);
                        const float p1 = fast_exp2(xe[e + 1]);
                        sump[(e >> 1) & 7] += p0 + p1;
                        ph_[e >> 1] = Fmt<T>::pack_rn(p0, p1);
                        if (kPfSplitP) {
                            const float2 hv = Fmt<T>::unpack(ph_[e >> 1]);
                            pl_[e >> 1] = Fmt<T>::pack_rn(p0 - hv.x, p1 - hv.y);
                        }
                    }
                    if (c + 1 < kPfKeys / 32) tmem_wait_ld_regs(nxt);
                    tmem_st16(tS + 16 * c, ph_);
                    if (kPfSplitP) tmem_st16(tS + 32 + 16 * c, pl_);
                }
            }
            tmem_wait_st();
            const float sum = ((sump[0] + sump[1]) + (sump[2] + sump[3])) +
                              ((sump[4] + sump[5]) + (sump[6] + sump[7]));
            l_run = l_run * alpha + sum;
            m_run = m_new;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_p0 + 8 * (2 * x + (i & 1)));
        }
        if (t.live && ok && i > 0) {
            ok = mbar_wait_bounded(bar_f0 + 8 * x, 0);
            ok = __all_sync(0xffffffffu, ok);
        }
        if (!ok) {
            if (lane == 0) raise_error(PA_DEVERR_TIMEOUT);
            sh_fail = 1;
        } else if (t.live) {
            tc_fence_after();
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            T *dst = reinterpret_cast<T *>(p.out) +
                     ((size_t)(q0 + t.tok0 + rtok) * p.num_q_heads + (size_t)g * G + rh) * D;
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t v[32];
                tmem_ld32(tO + cc * 32, v);
                tmem_wait_ld_regs(v);
                if (rvalid) {
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        uint4 w;
                        w.x = Fmt<T>::pack_rn(__uint_as_float(v[e]) * inv,
                                              __uint_as_float(v[e + 1]) * inv);
                        w.y = Fmt<T>::pack_rn(__uint_as_float(v[e + 2]) * inv,
                                              __uint_as_float(v[e + 3]) * inv);
                        w.z = Fmt<T>::pack_rn(__uint_as_float(v[e + 4]) * inv,
                                              __uint_as_float(v[e + 5]) * inv);
                        w.w = Fmt<T>::pack_rn(__uint_as_float(v[e + 6]) * inv,
                                              __uint_as_float(v[e + 7]) * inv);
                        *reinterpret_cast<uint4 *>(dst + cc * 32 + e) = w;
                    }
                }
            }
        }
    }

    // ---- teardown: free the tensor memory (the warp that allocated it)
    tc_fence_before();
    __syncthreads();
    if (warp == kPfLoadWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kPfTmemCols)
                     : "memory");
    }
}

}  // namespace pa
