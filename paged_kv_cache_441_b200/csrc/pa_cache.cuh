// Cache write (slot-mapped scatter of new tokens) and block copy (copy-on-write).
//
// Both are pure data movement at HBM bandwidth: 16-byte vector loads and stores,
// several independent 16-byte transfers in flight per thread, bit-exact.
#pragma once

#include "pa_common.cuh"

namespace pa {

struct KvWriteParams {
    const uint8_t *key;
    const uint8_t *value;
    const int64_t *slot_mapping;
    uint8_t *k_cache;
    uint8_t *v_cache;
    long long key_stride_b;    // bytes between tokens of key
    long long value_stride_b;  // bytes between tokens of value
    long long num_slots;       // num_blocks * block_size
    int num_tokens;
    int num_kv_heads;
    int row_chunks;            // head_dim / 8 (16-byte chunks per head row)
    int block_size;
};

constexpr int kKvwThreads = 256;
constexpr int kKvwUnroll = 4;

// One CTA per kKvwThreads * kKvwUnroll consecutive 16-byte chunks of the (token, kv head,
// chunk) rows, K and V together; each thread issues its kKvwUnroll K and V loads before any
// store (32-bit index math: the host keeps the chunk count below 2^31).
// PagedAttention and dynamic memory management blog, first section: the cache keeps the
// K and V of each token the model produces; here that store goes to
// k_cache[slot / bs][h][slot % bs][:] (and the same for V).
__global__ void __launch_bounds__(kKvwThreads) pa_kv_write_kernel(const __grid_constant__ KvWriteParams p) {
    pdl_wait_and_release();
    const unsigned per_tok = (unsigned)(p.num_kv_heads * p.row_chunks);
    const unsigned total = per_tok * (unsigned)p.num_tokens;
    const unsigned i0 = blockIdx.x * (unsigned)(kKvwThreads * kKvwUnroll) + threadIdx.x;
    uint4 kv[kKvwUnroll], vv[kKvwUnroll];
    long long dst[kKvwUnroll];
#pragma unroll
    for (int u = 0; u < kKvwUnroll; ++u) {
        const unsigned i = i0 + (unsigned)(u * kKvwThreads);
        dst[u] = -1;
        if (i >= total) continue;
        const unsigned t = i / per_tok, rem = i - t * per_tok;
        const unsigned h = rem / (unsigned)p.row_chunks, c = rem - h * (unsigned)p.row_chunks;
        const long long slot = p.slot_mapping[t];
        if (slot < 0) continue;
        if (slot >= p.num_slots) {
            if (rem == 0) raise_error(PA_DEVERR_SLOT);
            continue;
        }
        const long long blk = slot / p.block_size, off = slot - blk * p.block_size;
        dst[u] = ((blk * p.num_kv_heads + h) * p.block_size + off) * p.row_chunks + c;
        const long long src_off = (long long)rem * 16;
        kv[u] = ld_global_nc_v4(p.key + (long long)t * p.key_stride_b + src_off);
        vv[u] = ld_global_nc_v4(p.value + (long long)t * p.value_stride_b + src_off);
    }
#pragma unroll
    for (int u = 0; u < kKvwUnroll; ++u) {
        if (dst[u] < 0) continue;
        reinterpret_cast<uint4 *>(p.k_cache)[dst[u]] = kv[u];
        reinterpret_cast<uint4 *>(p.v_cache)[dst[u]] = vv[u];
    }
}

struct CopyBlocksParams {
    uint8_t *k_cache;
    uint8_t *v_cache;
    const int64_t *pairs;
    long long block_chunks;  // 16-byte chunks per block per cache
    int num_blocks;
    int num_pairs;
};

constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 4;

// grid = (chunks_of_a_block / (256 * 4) rounded up, num_pairs, 2 caches).
// Each thread keeps kCopyUnroll 16-byte loads in flight before storing.
__global__ void __launch_bounds__(kCopyThreads)
    pa_copy_blocks_kernel(const __grid_constant__ CopyBlocksParams p) {
    pdl_wait_and_release();
    const int pair = blockIdx.y;
    const long long src = p.pairs[2 * pair], dst = p.pairs[2 * pair + 1];
    if (src < 0 || src >= p.num_blocks || dst < 0 || dst >= p.num_blocks) {
        if (blockIdx.x == 0 && blockIdx.z == 0 && threadIdx.x == 0) raise_error(PA_DEVERR_PAIR);
        return;
    }
    uint4 *cache = reinterpret_cast<uint4 *>(blockIdx.z == 0 ? p.k_cache : p.v_cache);
    const uint4 *from = cache + src * p.block_chunks;
    uint4 *to = cache + dst * p.block_chunks;
    const long long c0 = (long long)blockIdx.x * kCopyThreads * kCopyUnroll + threadIdx.x;
    uint4 buf[kCopyUnroll];
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
        const long long c = c0 + (long long)u * kCopyThreads;
        if (c < p.block_chunks) buf[u] = ld_global_nc_v4(from + c);
    }
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
        const long long c = c0 + (long long)u * kCopyThreads;
        if (c < p.block_chunks) to[c] = buf[u];
    }
}

struct SwapBlocksParams {
    uint8_t *dst_k;
    uint8_t *dst_v;
    const uint8_t *src_k;
    const uint8_t *src_v;
    const int64_t *pairs;     // [n][2]: block in the source pool, block in the destination pool
    long long block_chunks;   // 16-byte chunks per block per cache
    int src_blocks;
    int dst_blocks;
};

// Block copy between two pools, one of which may be pinned host memory reached
// through unified addressing (swap out: device -> host, swap in: host -> device).
// grid = (pairs, chunks of a block, 2 caches); kCopyUnroll 16-byte loads in flight
// per thread, which is what keeps the host link busy.
__global__ void __launch_bounds__(kCopyThreads)
    pa_swap_blocks_kernel(const __grid_constant__ SwapBlocksParams p) {
    pdl_wait_and_release();
    const int pair = blockIdx.x;
    const long long src = p.pairs[2 * pair], dst = p.pairs[2 * pair + 1];
    if (src < 0 || src >= p.src_blocks || dst < 0 || dst >= p.dst_blocks) {
        if (blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0) raise_error(PA_DEVERR_PAIR);
        return;
    }
    const uint4 *from = reinterpret_cast<const uint4 *>(blockIdx.z == 0 ? p.src_k : p.src_v) +
                        src * p.block_chunks;
    uint4 *to = reinterpret_cast<uint4 *>(blockIdx.z == 0 ? p.dst_k : p.dst_v) +
                dst * p.block_chunks;
    const long long c0 = (long long)blockIdx.y * kCopyThreads * kCopyUnroll + threadIdx.x;
    uint4 buf[kCopyUnroll];
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
        const long long c = c0 + (long long)u * kCopyThreads;
        if (c < p.block_chunks) buf[u] = from[c];
    }
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
        const long long c = c0 + (long long)u * kCopyThreads;
        if (c < p.block_chunks) to[c] = buf[u];
    }
}

}  // namespace pa
