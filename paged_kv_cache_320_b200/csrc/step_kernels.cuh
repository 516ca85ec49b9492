// Decode step with the block-table update on the device and the cache write, the
// decode and the partition merge in one launch per layer.
//
// "vLLM / PagedAttention — 分页 KV Cache 分析" §3.1 (each step the new token's K/V is
// written into its page, then attention runs over the pages) and §2.3 (the block
// manager maps a sequence's logical blocks to physical pages and hands out a new page
// when the last one is full). "vLLM" entity page, 关键观察: every extra kernel launch
// costs a few microseconds, which at decode sizes is a visible share of the step.
//
//  * device_append_kernel (once per step, one CTA): appends one token to every
//    sequence. A sequence whose length is a multiple of the block size takes the next
//    block of a caller-given free list; sequences are served in index order, so the
//    result is the host block manager's in-order append when the list holds the host's
//    free blocks in pop order. All or nothing: if the list runs short, a table would
//    overflow or a length would pass the stated maximum, nothing changes and a status
//    bit is set.
//  * paged_decode_step_kernel (once per layer, cooperative persistent grid): the
//    decode work-item loop of paged_decode_partition_kernel in which the producer
//    writes each sequence's newest token (position len_s - 1) before loading its page;
//    then, when some context spans several partitions, a grid barrier and the
//    log-sum-exp merge by every warp of the grid.
#pragma once

#include "decode_kernels.cuh"
#include "shared_prefix_kernels.cuh"

namespace pkv {

constexpr unsigned kStatusNoBlocks = 1u << 5;
constexpr unsigned kStatusWorkspace = 1u << 6;
constexpr unsigned kStatusSharedBlock = 1u << 7;

// Workspace header of the step kernel: SchedHeader, whose `arrive`, `gen` and `exit`
// hold the grid barrier and the exit count. Valid at launch: zero-filled (armed, gen
// and exit 0), left by a previous step launch (armed == kStepArmed: the last CTA out
// cleared the counters) or re-armed by paged_decode_reduce_kernel (armed ==
// kSchedArmed: it cleared them too), always with exit == 0. Anything else is refused
// before any write. `arrive` cannot be checked at the start (a CTA may reach the
// barrier before another has started); a stale value is caught at the barrier instead.
constexpr unsigned kStepArmed = 0x57E9A11Du;
using StepHeader = SchedHeader;

constexpr uint32_t kBarrierPolls = 1u << 22;

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Grid-wide barrier for a co-resident grid; bounded (returns false when it gave up).
// gen0 is the header's generation read at kernel start (it cannot change before every
// CTA has arrived, so every CTA read the same value). An arrival count at or past the
// grid size means the header came in with a stale count: flagged as a workspace error
// (the release may then have come early, so the launch's output is not to be used).
__device__ __forceinline__ bool grid_barrier(StepHeader *h, unsigned gen0, int *flag,
                                             unsigned *status) {
    __syncthreads();
    if (threadIdx.x == 0) {
        int ok = 1;
        __threadfence();
        const unsigned t = atomicAdd(&h->arrive, 1u);
        if (t >= gridDim.x) atomicOr(status, kStatusWorkspace);
        if (t == gridDim.x - 1) {
            h->arrive = 0;
            __threadfence();
            atomicExch(&h->gen, gen0 + 1);
        } else {
            uint32_t i = 0;
            while (ld_acquire_gpu(&h->gen) == gen0) {
                if (++i > kBarrierPolls) {
                    ok = 0;
                    break;
                }
                __nanosleep(64);
            }
        }
        __threadfence();
        *flag = ok;
    }
    __syncthreads();
    return *flag != 0;
}

template <typename T, int D, int BS>
__global__ void __launch_bounds__(kDecodeThreads, 2)
paged_decode_step_kernel(const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v,
                         const __grid_constant__ CUtensorMap tmap_q, DecodeParams prm,
                         int merge) {
    __shared__ int s_flag;
    __shared__ unsigned s_gen;
    DecodeSmem<D> sm(aligned_dynamic_smem(), prm.group);
    sm.init_barriers();
    StepHeader *hdr = reinterpret_cast<StepHeader *>(prm.sched);
    if (threadIdx.x == 0) {
        int ok = 1;
        if (hdr) {
            // Read before this launch can change them: `armed` is written only by the last
            // CTA out, `gen` only at the barrier's release and, with the merge (the only
            // way this kernel is launched with a header), `exit` only after the barrier,
            // which every CTA reaches after this check. So every CTA decides alike.
            const unsigned a = *(volatile unsigned *)&hdr->armed;
            const unsigned g = *(volatile unsigned *)&hdr->gen;
            const unsigned ex = merge ? *(volatile unsigned *)&hdr->exit : 0u;
            ok = (a == kStepArmed || a == kSchedArmed || (a == 0u && g == 0u)) && ex == 0u;
            s_gen = g;
            if (!ok && blockIdx.x == 0) atomicOr(prm.status, kStatusWorkspace);
        }
        s_flag = ok;
    }
    __syncthreads();
    if (!s_flag) return;   // same decision in every CTA: nothing has written the header

    decode_items<T, D, BS, true>(&tmap_k, &tmap_v, &tmap_q, prm, sm, hdr != nullptr);
    if (!hdr) return;

    if (merge) {
        if (grid_barrier(hdr, s_gen, &s_flag, prm.status)) {
            const int lane = threadIdx.x & 31;
            const int nwarps = gridDim.x * (kDecodeThreads / 32);
            const int G = prm.group, P = prm.partition;
            for (int pair = blockIdx.x * (kDecodeThreads / 32) + (threadIdx.x >> 5);
                 pair < prm.num_seqs * prm.num_heads; pair += nwarps) {
                const int s = pair / prm.num_heads;
                const int h = pair - s * prm.num_heads;
                int len = prm.context_lens[s];
                len = len < 0 ? 0 : (len > prm.max_context_len ? prm.max_context_len : len);
                const int np = max(1, (len + P - 1) / P);
                if (np == 1) continue;
                const int hk = h / G, g = h - hk * G;
                const size_t row0 = (size_t)(prm.ws_seq_base[s] + hk * np) * G + g;
                warp_merge<T, D>(reinterpret_cast<const float2 *>(prm.ws_ml) + row0, G,
                                 prm.ws_o + row0 * D, (size_t)G * D, np,
                                 reinterpret_cast<T *>(prm.out) + ((size_t)s * prm.num_heads + h) * D,
                                 lane);
            }
        } else if (threadIdx.x == 0) {
            atomicOr(prm.status, kStatusTimeout);
        }
    }
    // the last CTA out leaves the header ready for the next launch
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned t = atomicAdd(&hdr->exit, 1u);
        if (t == gridDim.x - 1) {
            hdr->next = 0;
            hdr->arrive = 0;
            hdr->exit = 0;
            __threadfence();
            hdr->armed = kStepArmed;
        }
    }
}

// One token appended to each of B sequences on the device (one CTA of kPlanThreads).
//   n = context_lens[s];  if n % BS == 0: block_tables[s][n / BS] = free_blocks[used + r_s]
//   (r_s = number of sequences before s that take a block);  slot_s =
//   block_tables[s][n / BS] * BS + n % BS;  context_lens[s] = n + 1;  *free_used += taken.
// With refcounts (the host manager's per-block counts), a sequence that would write into
// a partly filled block held by more than one sequence refuses the step: that write
// needs the copy-on-write of the host manager first.
__global__ void __launch_bounds__(kPlanThreads)
device_append_kernel(int32_t *block_tables, int32_t *context_lens, const int32_t *free_blocks,
                     int free_count, int *free_used, const int32_t *refcounts, int64_t *slots_out,
                     int B, int MB, int BS, int num_blocks, int max_len, unsigned *status) {
    pdl_wait_and_release();
    __shared__ int sm[kPlanThreads / 32];
    __shared__ int s_used, s_bad, s_shared;
    const int tid = threadIdx.x;
    if (tid == 0) {
        s_used = *free_used;
        s_bad = 0;
        s_shared = 0;
    }
    __syncthreads();
    const int used = s_used;
    // pass 1: blocks needed, and every reason to refuse the whole step
    int need = 0, bad = 0, shared = 0;
    for (int s = tid; s < B; s += kPlanThreads) {
        const int n = context_lens[s];
        if (n < 0 || n + 1 > max_len || n / BS >= MB) {
            bad = 1;
        } else if (n % BS == 0) {
            need += 1;
        } else if (refcounts) {
            const int b = block_tables[(size_t)s * MB + n / BS];
            if (b >= 0 && b < num_blocks && refcounts[b] > 1) shared = 1;
        }
    }
    int total;
    block_exclusive_scan(need, sm, &total);
    if (bad || shared) atomicOr(&s_bad, 1);
    if (shared) atomicOr(&s_shared, 1);
    __syncthreads();
    if (!s_bad && (used < 0 || used > free_count || total > free_count - used)) bad = 1;
    if (!s_bad && !bad)
        for (int i = tid; i < total; i += kPlanThreads) {
            const int b = free_blocks[used + i];
            if (b < 0 || b >= num_blocks) bad = 1;
        }
    if (bad) atomicOr(&s_bad, 1);
    __syncthreads();
    if (s_bad) {
        if (tid == 0) atomicOr(status, kStatusNoBlocks | (s_shared ? kStatusSharedBlock : 0u));
        return;
    }
    // pass 2: ranks in sequence order, table / length / slot updates
    int base = 0;
    for (int c0 = 0; c0 < B; c0 += kPlanThreads) {
        const int s = c0 + tid;
        const int n = s < B ? context_lens[s] : 0;
        const int takes = s < B && n % BS == 0;
        int chunk;
        const int r = block_exclusive_scan(takes, sm, &chunk);
        if (s < B) {
            int32_t *row = block_tables + (size_t)s * MB;
            int b;
            if (takes) {
                b = free_blocks[used + base + r];
                row[n / BS] = b;
            } else {
                b = row[n / BS];
            }
            int64_t slot = -1;
            if (b >= 0 && b < num_blocks) slot = (int64_t)b * BS + n % BS;
            else atomicOr(status, kStatusBadBlock);
            context_lens[s] = n + 1;
            if (slots_out) slots_out[s] = slot;
        }
        base += chunk;
    }
    if (tid == 0) *free_used = used + total;
}

}  // namespace pkv
