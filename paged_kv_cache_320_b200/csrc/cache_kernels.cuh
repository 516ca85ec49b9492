// Cache maintenance kernels: the cache write through a slot mapping and the
// copy-on-write block copy ("vLLM / PagedAttention — 分页 KV Cache 分析" §3.2: a new
// token goes into its page; a shared page is copied before it is changed).
//
// Both are pure data movement: 16-byte vector loads/stores, every 32-byte sector
// fully used (a (token, KV head) row is head_dim*2 = 128 or 256 contiguous bytes).
#pragma once

#include <stdint.h>

#include "pkv_ptx.cuh"

namespace pkv {

// One thread per 16-byte vector of one (token, KV head) row; K and V together.
//   k_cache[slot / BS][h][slot % BS][:] = k_new[t][h][:]   (V alike), slot >= 0
template <int D>
__global__ void __launch_bounds__(256)
reshape_and_cache_kernel(const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new,
                         uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache,
                         const int64_t *__restrict__ slot_mapping, int num_tokens, int Hkv,
                         int BS, int num_blocks, unsigned *status) {
    pdl_wait_and_release();
    constexpr int VPR = D * 2 / 16;   // vectors per row
    const int64_t total = (int64_t)num_tokens * Hkv * VPR;
    const int64_t limit = (int64_t)num_blocks * BS;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = i / VPR;          // t * Hkv + h
        const int v = (int)(i - row * VPR);
        const int64_t t = row / Hkv;
        const int h = (int)(row - t * Hkv);
        const int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        if (slot >= limit) {
            if (h == 0 && v == 0) atomicOr(status, 1u /* bad slot */);
            continue;
        }
        const int64_t blk = slot / BS;
        const int64_t r = slot - blk * BS;
        const int64_t dst = ((blk * Hkv + h) * BS + r) * VPR + v;
        k_cache[dst] = k_new[i];
        v_cache[dst] = v_new[i];
    }
}

// One CTA per (pair, layer, K|V): copies the whole block (all KV heads).
__global__ void __launch_bounds__(256)
copy_blocks_kernel(void *const *__restrict__ k_caches, void *const *__restrict__ v_caches,
                   const int32_t *__restrict__ block_pairs, int num_blocks, int block_vecs,
                   unsigned *status) {
    pdl_wait_and_release();
    const int pair = blockIdx.x;
    const int layer = blockIdx.y;
    const int src = block_pairs[2 * pair];
    const int dst = block_pairs[2 * pair + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
        if (threadIdx.x == 0 && blockIdx.z == 0) atomicOr(status, 2u /* bad pair */);
        return;
    }
    uint4 *base = reinterpret_cast<uint4 *>(blockIdx.z ? v_caches[layer] : k_caches[layer]);
    const uint4 *s = base + (int64_t)src * block_vecs;
    uint4 *d = base + (int64_t)dst * block_vecs;
    int i = threadIdx.x;
    for (; i + 3 * 256 < block_vecs; i += 4 * 256) {
        const uint4 a = s[i], b = s[i + 256], c = s[i + 512], e = s[i + 768];
        d[i] = a; d[i + 256] = b; d[i + 512] = c; d[i + 768] = e;
    }
    for (; i < block_vecs; i += 256) d[i] = s[i];
}

// Swap of whole blocks between the device caches and a pinned host buffer, for
// preemption ("vLLM/PagedAttention — L3 Cross-Paper Synthesis" §3: all-or-nothing
// eviction swaps every block of a request; "vLLM" entity page, observation 2: copies
// of small fragments one cudaMemcpyAsync at a time leave the host link mostly idle).
// One kernel moves every listed block of every layer through mapped host memory.
// Host buffer layout: [layer][K, V][i][Hkv * BS * D elements] for block_ids[i].
//   to_host = 1: host[l][kv][i] = cache_l,kv[block_ids[i]]
//   to_host = 0: cache_l,kv[block_ids[i]] = host[l][kv][i]
// One CTA per (block, layer, K|V); 16-byte vectors, four in flight per thread.
__global__ void __launch_bounds__(256)
swap_blocks_kernel(void *const *__restrict__ k_caches, void *const *__restrict__ v_caches,
                   const int32_t *__restrict__ block_ids, int n_blocks, uint4 *host,
                   int num_blocks, int block_vecs, int to_host, unsigned *status) {
    pdl_wait_and_release();
    const int i = blockIdx.x;
    const int layer = blockIdx.y;
    const int kv = blockIdx.z;
    const int b = block_ids[i];
    if (b < 0 || b >= num_blocks) {
        if (threadIdx.x == 0 && kv == 0 && layer == 0) atomicOr(status, 2u /* bad pair */);
        return;
    }
    uint4 *cache = reinterpret_cast<uint4 *>(kv ? v_caches[layer] : k_caches[layer]) +
                   (int64_t)b * block_vecs;
    uint4 *h = host + (((int64_t)layer * 2 + kv) * n_blocks + i) * block_vecs;
    const uint4 *src = to_host ? cache : h;
    uint4 *dst = to_host ? h : cache;
    int t = threadIdx.x;
    for (; t + 3 * 256 < block_vecs; t += 4 * 256) {
        const uint4 a = src[t], c = src[t + 256], d = src[t + 512], e = src[t + 768];
        dst[t] = a; dst[t + 256] = c; dst[t + 512] = d; dst[t + 768] = e;
    }
    for (; t < block_vecs; t += 256) dst[t] = src[t];
}

// Staged swap: tiles t0 .. t0 + count - 1 of the swap's flat order (tile t = the block
// block_ids[t % n_blocks] of layer (t / n_blocks) / 2, K for even t / n_blocks, V for odd,
// the host buffer's order) between the caches and a device staging buffer, one CTA per
// tile, so that each chunk crosses the host link as one large copy.
//   to_staging = 1: staging[j] = tile t0 + j   (a tile with a bad id is zero-filled)
//   to_staging = 0: tile t0 + j = staging[j]    (a tile with a bad id is not written)
__global__ void __launch_bounds__(256)
swap_stage_kernel(void *const *__restrict__ k_caches, void *const *__restrict__ v_caches,
                  const int32_t *__restrict__ block_ids, int n_blocks, uint4 *staging,
                  long long t0, int num_blocks, int block_vecs, int to_staging,
                  unsigned *status) {
    pdl_wait_and_release();
    const long long t = t0 + blockIdx.x;
    const long long lk = t / n_blocks;
    const int i = (int)(t - lk * n_blocks);
    const int layer = (int)(lk >> 1);
    const int kv = (int)(lk & 1);
    const int b = block_ids[i];
    uint4 *st = staging + (long long)blockIdx.x * block_vecs;
    if (b < 0 || b >= num_blocks) {
        if (threadIdx.x == 0 && kv == 0 && layer == 0) atomicOr(status, 2u /* bad pair */);
        if (to_staging)
            for (int v = threadIdx.x; v < block_vecs; v += 256) st[v] = make_uint4(0, 0, 0, 0);
        return;
    }
    uint4 *cache = reinterpret_cast<uint4 *>(kv ? v_caches[layer] : k_caches[layer]) +
                   (long long)b * block_vecs;
    const uint4 *src = to_staging ? cache : st;
    uint4 *dst = to_staging ? st : cache;
    int v = threadIdx.x;
    for (; v + 3 * 256 < block_vecs; v += 4 * 256) {
        const uint4 a = src[v], c = src[v + 256], d = src[v + 512], e = src[v + 768];
        dst[v] = a; dst[v + 256] = c; dst[v + 512] = d; dst[v + 768] = e;
    }
    for (; v < block_vecs; v += 256) dst[v] = src[v];
}

}  // namespace pkv
