// Shared-prefix-aware paged decode attention for sm_100a.
//
// Parallel sampling and common prompts make several sequences point at the same
// physical prefix pages ("vLLM" entity page, 是什么; "vLLM / PagedAttention — 分页 KV
// Cache 分析" §3.2). Plain decode streams such a page once per sequence. Here the
// sequences of a group share the prefix: every prefix page of a KV head is streamed
// once for up to 16 query rows (the G heads of several member sequences on the MMA's
// M dimension), each sequence's private suffix is streamed for its own G rows, and
// the partial softmax states of the pieces are merged exactly (log-sum-exp). The
// result is the same attention as plain decode:
//   out[s][h] = sum_t softmax_t(scale * q[s][h] . K_s[t]) V_s[t],  t < len_s.
//
// Three launches: a one-CTA plan builds the item list in the workspace (and checks
// the declared prefix against the block tables: the shared length of a group is cut
// at the first logical block where a member's table differs from the group's first
// member, so a wrong declaration costs sharing, never correctness); the decode kernel
// runs the items with the same TMA / mbarrier / tensor-core pipeline as plain decode;
// the reduce merges the partials of the (sequence, head) pairs whose work was split.
//
// Work items. The members of a group are taken R = 16 / G at a time ("chunks", 16 query
// rows). A chunk's tokens are its prefix, cut into partitions of P tokens, and its
// members' suffixes, cut into partitions of P tokens per member (suffix partition k of a
// chunk holds every member's tokens [pre + kP, pre + (k+1)P)). An item is one of them
// for one KV head, or the last prefix partition and the first suffix partition
// together when their 64-token stages fit in one partition's budget. The item's stages
// come in segments (the prefix pages, then each member's own pages); during a member's
// segment only that member's G rows attend. A chunk that is one item writes its output
// directly; otherwise each item leaves one partial per row (empty for rows it did not
// touch) for the reduce.
#pragma once

#include "decode_kernels.cuh"

namespace pkv {

struct SharedItem {
    int table_seq;   // the group's first member: its block-table row holds the prefix pages
    int pre;         // the group's shared tokens (a multiple of the block size)
    int first_seq;   // query rows: sequences first_seq .. first_seq + nseq - 1, G heads each
    int nseq;
    int hk;          // KV head
    int part;        // index of this item among its chunk's items (its partials' index)
    int npp;         // prefix partitions of the chunk
    int nps2;        // 2 x suffix partitions of the chunk, + 1 if the last prefix partition
                     // and the first suffix partition are one item
};

// Items of a chunk: prefix partitions, then suffix partitions, one fewer if fused.
__host__ __device__ __forceinline__ int chunk_parts(int npp, int nps2) {
    return npp + (nps2 >> 1) - (nps2 & 1);
}

struct SharedCounters {
    unsigned next;    // next work item (0 after the plan and after every reduce)
    int count;        // items in the list
    int sig[4];       // sizes the plan was built for (kPlanMagic, B, Hq | Hkv << 16, P)
    int pad[58];
};

// The plan stays valid for every layer of a step (it depends on the tables, lengths and
// groups only): decode and reduce launches check that the workspace holds a plan for
// their sizes and otherwise write nothing and set the workspace status bit.
constexpr int kPlanMagic = 0x51A9ED01;
constexpr unsigned kStatusPlanMismatch = 1u << 6;   // the status word's workspace bit

__device__ __forceinline__ bool plan_matches(const SharedCounters *c, int B, int Hq, int Hkv,
                                             int P) {
    return c->sig[0] == kPlanMagic && c->sig[1] == B && c->sig[2] == (Hq | (Hkv << 16)) &&
           c->sig[3] == P;
}

struct SharedParams {
    SharedCounters *counters;
    SharedItem *items;
    int *np;           // [B] partials per (sequence, head)
    int *row_base;     // [B] scratch row of (s, h, j) = row_base[s] + h * np[s] + j
    int *seq_group;    // [B] group of each sequence (plan scratch)
    int *gpre;         // [B] shared tokens per group (plan scratch)
    int *gmin;         // [B] shortest member, then first chunk, per group (plan scratch)
    int *gmis;         // [B] first block where a member's table differs per group, then
                       //     first item per chunk (plan scratch)
    int *ioff;         // [B] 2 x suffix partitions + fused, per chunk (plan scratch)
    float *ws_o;       // [rows][D]
    float *ws_ml;      // [rows][2]
    void *out;
    const void *q;
    const int32_t *block_tables;
    const int32_t *context_lens;
    const int32_t *group_start;   // [num_groups + 1]
    const int32_t *prefix_lens;   // [num_groups] declared shared tokens
    unsigned *status;
    int num_groups, num_seqs, num_heads, num_kv_heads, group;
    int max_blocks_per_seq, num_blocks, max_context_len, partition, block_size, max_items;
    int sms, slots;      // the decode launch's SMs and CTAs per SM (item placement)
    float scale_log2;
};

constexpr int kPlanThreads = 1024;
constexpr int kPlanBins = 1024;   // stage-count bins of the item placement (longer ones share the top)

__device__ __forceinline__ int clamp_len(int len, int max_len) {
    return len < 0 ? 0 : (len > max_len ? max_len : len);
}

// Exclusive block-wide prefix sum of one value per thread (kPlanThreads threads);
// returns the exclusive sum and writes the block total to *total.
__device__ __forceinline__ int block_exclusive_scan(int v, int *sm, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sm[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < kPlanThreads / 32 ? sm[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        sm[lane] = w;   // inclusive sums of warps
    }
    __syncthreads();
    const int before = warp ? sm[warp - 1] : 0;
    *total = sm[kPlanThreads / 32 - 1];
    __syncthreads();
    return before + x - v;
}

// Per-sequence scratch arrays of the plan kept in shared memory up to this batch size
// (7 ints per sequence); larger batches use the workspace copies.
constexpr int kPlanSmemSeqs = 6144;

// Largest i in [0, n) with off[i] <= x (off ascending, off[0] = 0).
__device__ __forceinline__ int owner_of(const int *off, int n, int x) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= x) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// One CTA builds the item list. Groups are contiguous runs of sequences; a malformed
// group_start makes every sequence its own group (no sharing) and sets the length
// status bit. A group's shared length is its declared prefix cut to a multiple of the
// block size, to its shortest member and at the first logical block where a member's
// table differs from the first member's; a group of one shares nothing.
__global__ void __launch_bounds__(kPlanThreads)
shared_prefix_plan_kernel(SharedParams p) {
    pdl_wait_and_release();
    extern __shared__ int plan_smem[];
    __shared__ int sm[kPlanThreads / 32];
    __shared__ int plan_bins[kPlanBins];
    __shared__ int bad, max_pre_blocks;
    const int B = p.num_seqs, Hkv = p.num_kv_heads, G = p.group, P = p.partition;
    const int BS = p.block_size;
    const int R = kMaxGroup / G;   // member sequences per 16-row prefix item
    const int tid = threadIdx.x;
    // scratch: in shared memory when it fits (generic pointers address either space)
    const bool in_smem = B <= kPlanSmemSeqs;
    int *seq_group = in_smem ? plan_smem : p.seq_group;
    int *gpre = in_smem ? plan_smem + B : p.gpre;
    int *gmin = in_smem ? plan_smem + 2 * B : p.gmin;
    int *gmis = in_smem ? plan_smem + 3 * B : p.gmis;
    int *slen = in_smem ? plan_smem + 4 * B : p.np;          // clamped lengths
    int *gfirst = in_smem ? plan_smem + 5 * B : p.row_base;  // first member of each group
    int *ioff = in_smem ? plan_smem + 6 * B : p.ioff;        // per-chunk partition counts
    if (tid == 0) {
        bad = 0;
        max_pre_blocks = 0;
        p.counters->next = 0u;
        const int ng = p.num_groups;
        if (ng < 1 || ng > B || p.group_start[0] != 0 || p.group_start[ng] != B) bad = 1;
    }
    __syncthreads();
    if (!bad)
        for (int g = tid; g < p.num_groups; g += kPlanThreads)
            if (p.group_start[g + 1] <= p.group_start[g]) atomicOr(&bad, 1);
    __syncthreads();
    if (tid == 0 && bad) atomicOr(p.status, kStatusBadLen);
    const int ng = bad ? B : p.num_groups;
    // pass 0 (per group): membership, declared prefix, identities for the minima;
    // (per sequence): clamped length
    for (int g = tid; g < ng; g += kPlanThreads) {
        const int first = bad ? g : p.group_start[g];
        const int last = bad ? g + 1 : p.group_start[g + 1];
        int pre = (bad || last - first < 2) ? 0 : p.prefix_lens[g];
        pre = pre < 0 ? 0 : pre - pre % BS;
        gpre[g] = pre;
        gmin[g] = 0x7fffffff;
        gmis[g] = 0x7fffffff;
        gfirst[g] = first;
        for (int s = first; s < last; ++s) seq_group[s] = g;
        atomicMax(&max_pre_blocks, pre / BS);
    }
    for (int s = tid; s < B; s += kPlanThreads)
        slen[s] = clamp_len(p.context_lens[s], p.max_context_len);
    __syncthreads();
    // pass 1 (per sequence): shortest member
    for (int s = tid; s < B; s += kPlanThreads) atomicMin(&gmin[seq_group[s]], slen[s]);
    // pass 2 (per (sequence, 8 prefix blocks)): first block where a member's table
    // differs from the group's first member (independent loads, one atomic per chunk)
    const int nch = (max_pre_blocks + 7) / 8;
    for (long long i = tid; i < (long long)B * nch; i += kPlanThreads) {
        const int s = (int)(i / nch), c = (int)(i - (long long)s * nch);
        const int g = seq_group[s];
        const int first = gfirst[g];
        const int nb = gpre[g] / BS;
        if (s == first || c * 8 >= nb) continue;
        const int32_t *mine = p.block_tables + (size_t)s * p.max_blocks_per_seq;
        const int32_t *ref = p.block_tables + (size_t)first * p.max_blocks_per_seq;
        int a[8], r[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int b = c * 8 + k;
            a[k] = b < nb ? mine[b] : 0;
            r[k] = b < nb ? ref[b] : 0;
        }
        int mis = 0x7fffffff;
#pragma unroll
        for (int k = 7; k >= 0; --k)
            if (a[k] != r[k]) mis = c * 8 + k;
        if (mis != 0x7fffffff) atomicMin(&gmis[g], mis);
    }
    __syncthreads();
    // pass 3 (per group): shared length; chunks of R members; first chunk of each group
    const int S = P / kStageTokens;   // 64-token stages per partition
    int n_chunks = 0;
    for (int g0 = 0; g0 < ng; g0 += kPlanThreads) {
        const int g = g0 + tid;
        int cnt = 0;
        if (g < ng) {
            const int first = gfirst[g];
            const int last = bad ? g + 1 : p.group_start[g + 1];
            const int shortest = gmin[g];
            int pre = min(gpre[g], shortest - shortest % BS);
            pre = min(pre, min(gmis[g], pre / BS) * BS);
            gpre[g] = pre;
            cnt = (last - first + R - 1) / R;
        }
        int total;
        const int at = n_chunks + block_exclusive_scan(cnt, sm, &total);
        if (g < ng) gmin[g] = at;   // first chunk of group g (only thread g reads gmin[g] here)
        n_chunks += total;
    }
    int *chunk_base = gmin;
    int *item_base = gmis;    // per chunk (n_chunks <= B)
    int *chunk_nps2 = ioff;   // per chunk
    __syncthreads();
    // pass 4 (per chunk): prefix and suffix partitions, fusion, first item
    int n_items = 0;
    for (int c0 = 0; c0 < n_chunks; c0 += kPlanThreads) {
        const int ch = c0 + tid;
        int cnt = 0;
        if (ch < n_chunks) {
            const int g = owner_of(chunk_base, ng, ch);
            const int first = gfirst[g] + (ch - chunk_base[g]) * R;
            const int last = bad ? g + 1 : p.group_start[g + 1];
            const int nseq = min(R, last - first);
            const int pre = gpre[g];
            const int npp = (pre + P - 1) / P;
            int nps = 0, st0 = 0;
            for (int m = 0; m < nseq; ++m) {
                const int suf = slen[first + m] - pre;   // >= 0: pre <= the shortest member
                nps = max(nps, (suf + P - 1) / P);
                st0 += (min(P, suf) + kStageTokens - 1) / kStageTokens;
            }
            if (npp == 0 && nps == 0) nps = 1;   // empty contexts: one item writes zeros
            const int pre_last = npp ? (pre - (npp - 1) * P + kStageTokens - 1) / kStageTokens : 0;
            const int fuse = npp > 0 && nps > 0 && pre_last + st0 <= S;
            chunk_nps2[ch] = 2 * nps + fuse;
            cnt = Hkv * chunk_parts(npp, 2 * nps + fuse);
        }
        int total;
        const int at = n_items + block_exclusive_scan(cnt, sm, &total);
        if (ch < n_chunks) item_base[ch] = at;
        n_items += total;
    }
    __syncthreads();
    // pass 5 (per item): chunk, KV head and part; the item's 64-token stages
    auto make_item = [&](int i, int *stages) {
        const int ch = owner_of(item_base, n_chunks, i);
        const int g = owner_of(chunk_base, ng, ch);
        const int first = gfirst[g] + (ch - chunk_base[g]) * R;
        const int last = bad ? g + 1 : p.group_start[g + 1];
        const int pre = gpre[g];
        const int npp = (pre + P - 1) / P;
        const int nps2 = chunk_nps2[ch];
        const int np = chunk_parts(npp, nps2);
        const int local = i - item_base[ch];
        SharedItem it;
        it.table_seq = gfirst[g];
        it.pre = pre;
        it.first_seq = first;
        it.nseq = min(R, last - first);
        it.hk = local / np;
        it.part = local - it.hk * np;
        it.npp = npp;
        it.nps2 = nps2;
        const int j = it.part, k = j - npp + (nps2 & 1);
        int st = j < npp ? (min(P, pre - j * P) + kStageTokens - 1) / kStageTokens : 0;
        if (k >= 0 && k < (nps2 >> 1))
            for (int m = 0; m < it.nseq; ++m)
                st += (max(0, min(P, slen[first + m] - pre - k * P)) + kStageTokens - 1) /
                      kStageTokens;
        *stages = max(st, 1);
        return it;
    };
    // Placement: every CTA starts on the item at its own index. Items are ranked longest
    // first (counting sort on stage counts); the sms longest are items 0 .. sms-1 and, with
    // two CTAs per SM, the others follow shortest first, so that item sms + c goes to CTA
    // sms + c, which shares CTA c's SM when the launch fills the SMs in index order (on
    // B200 it does so for part of the SMs only: the first wave is spread GPC by GPC). That
    // pairs long items with short ones on an SM and evens out the SMs' loads. With more
    // items than CTAs, or another number of slots, the order is longest first. The
    // placement moves items only: results do not depend on it.
    for (int c = tid; c < kPlanBins; c += kPlanThreads) plan_bins[c] = 0;
    __syncthreads();
    const int n_put = min(n_items, p.max_items);
    for (int i = tid; i < n_put; i += kPlanThreads) {
        int st;
        make_item(i, &st);
        atomicAdd(&plan_bins[kPlanBins - 1 - min(st, kPlanBins - 1)], 1);   // longest first
    }
    __syncthreads();
    {
        int total;
        const int v = tid < kPlanBins ? plan_bins[tid] : 0;
        const int at = block_exclusive_scan(v, sm, &total);
        if (tid < kPlanBins) plan_bins[tid] = at;
    }
    __syncthreads();
    const bool paired = p.slots == 2 && n_put <= p.sms * 2 && n_put > p.sms;
    for (int i = tid; i < n_put; i += kPlanThreads) {
        int st;
        const SharedItem it = make_item(i, &st);
        const int r = atomicAdd(&plan_bins[kPlanBins - 1 - min(st, kPlanBins - 1)], 1);
        const int pos = paired && r >= p.sms ? p.sms + (n_put - 1 - r) : r;
        p.items[pos] = it;
    }
    __syncthreads();
    // pass 6 (per sequence): partials per (sequence, head) = its chunk's items, then the
    // scratch rows. slen becomes the partial count (in the workspace it is p.np itself),
    // and row_base may overwrite gfirst only once every count is known.
    for (int s = tid; s < B; s += kPlanThreads) {
        const int g = seq_group[s];
        const int ch = chunk_base[g] + (s - gfirst[g]) / R;
        slen[s] = chunk_parts((gpre[g] + P - 1) / P, chunk_nps2[ch]);
    }
    __syncthreads();
    int base_rows = 0;
    for (int s0 = 0; s0 < B; s0 += kPlanThreads) {
        const int s = s0 + tid;
        const int np = s < B ? slen[s] : 0;
        int total_rows;
        const int row = base_rows + block_exclusive_scan(np, sm, &total_rows);
        if (s < B) {
            p.row_base[s] = row * p.num_heads;
            p.np[s] = np;
        }
        base_rows += total_rows;
    }
    if (tid == 0) {
        if (n_items > p.max_items) atomicOr(p.status, kStatusBadLen);
        p.counters->count = min(n_items, p.max_items);
        p.counters->sig[0] = kPlanMagic;
        p.counters->sig[1] = B;
        p.counters->sig[2] = p.num_heads | (Hkv << 16);
        p.counters->sig[3] = P;
    }
}

// The producer's view of an item: its descriptor (lane k < 8 holds field k), each
// member's token count in this item's suffix partition (lane m), and which segments
// have tokens (bit 0: the prefix partition, bit 1 + m: member m's suffix part).
struct SharedItemCtx {
    int idx;
    int f;
    int mtok;
    unsigned mask;
    bool valid;
};

// One segment: tokens [tok0, tok0 + ntok) of sequence `seq`'s pages, attended by query
// rows [r0, r1) of the item.
struct SharedSeg {
    int seq, tok0, ntok, r0, r1;
    int sidx;        // 0: prefix partition, 1 + m: member m's suffix partition
    bool first, last, valid;
};

template <typename T, int D, int BS>
__global__ void __launch_bounds__(kDecodeThreads, 2)
paged_decode_shared_kernel(const __grid_constant__ CUtensorMap tmap_k,
                           const __grid_constant__ CUtensorMap tmap_v, SharedParams prm) {
    using L = DecodeLayout<D>;
    constexpr int kBPS = kStageTokens / BS;
    constexpr int H = L::kHalves;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ring = smem;
    float *obuf = reinterpret_cast<float *>(smem + L::kRingBytes);
    StageInfo *info = reinterpret_cast<StageInfo *>(reinterpret_cast<uint8_t *>(obuf) +
                                                    L::obuf_bytes(kMaxGroup));
    uint64_t *full = reinterpret_cast<uint64_t *>(info + L::kStages);
    uint64_t *empty = full + L::kStages;
    float2 *ml = reinterpret_cast<float2 *>(empty + L::kStages);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = prm.group;
    const int Hkv = prm.num_kv_heads;
    const int P = prm.partition;

    if (threadIdx.x == 0) {
        for (int i = 0; i < L::kStages; ++i) {
            mbar_init(smem_u32(&full[i]), 1);
            mbar_init(smem_u32(&empty[i]), kConsumerWarps);
        }
        fence_mbar_init();
    }
    pdl_wait_and_release();
    __syncthreads();
    // every CTA reads the same signature (nothing writes it during this launch)
    if (!plan_matches(prm.counters, prm.num_seqs, prm.num_heads, Hkv, prm.partition)) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(prm.status, kStatusPlanMismatch);
        return;
    }

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&tmap_k);
            prefetch_tensormap(&tmap_v);
        }
        const uint64_t kv_policy = l2_evict_first_policy();
        const int count = prm.counters->count;
        int it = 0;
        bool ok = true;
        // CTA c starts on item c (the plan's placement); the counter hands out the rest
        auto take = [&]() {
            unsigned v = 0;
            if (lane == 0) v = atomicAdd(&prm.counters->next, 1u) + gridDim.x;
            return v > 0x7fffffffu ? 0x7fffffff : (int)v;   // lives in lane 0
        };
        auto field = [&](const SharedItemCtx &c, int k) { return __shfl_sync(0xffffffffu, c.f, k); };
        // descriptor, members' suffix-part token counts, non-empty segments
        auto load_item = [&](int idx) {
            SharedItemCtx c;
            c.idx = idx;
            c.valid = idx < count;
            c.f = c.valid && lane < 8 ? reinterpret_cast<const int *>(prm.items + idx)[lane] : 0;
            c.mtok = 0;
            c.mask = 0u;
            if (!c.valid) return c;
            const int pre = field(c, 1), first = field(c, 2), nseq = field(c, 3);
            const int j = field(c, 5), npp = field(c, 6), nps2 = field(c, 7);
            const int k = j - npp + (nps2 & 1);   // suffix partition of this item, if any
            if (k >= 0 && k < (nps2 >> 1) && lane < nseq) {
                const int len = clamp_len(prm.context_lens[first + lane], prm.max_context_len);
                c.mtok = max(0, min(P, len - pre - k * P));
            }
            c.mask = (__ballot_sync(0xffffffffu, c.mtok > 0) << 1) | (j < npp ? 1u : 0u);
            return c;
        };
        // segment sidx of item c (sidx < 0: the empty item's single stage of no tokens)
        auto make_seg = [&](const SharedItemCtx &c, int sidx) {
            SharedSeg g;
            g.valid = c.valid;
            g.sidx = sidx;
            const int nseq = field(c, 3);
            const int m = sidx - 1;
            const int mt = __shfl_sync(0xffffffffu, c.mtok, max(m, 0));
            if (sidx <= 0) {
                const int j = field(c, 5), pre = field(c, 1);
                g.seq = sidx == 0 ? field(c, 0) : field(c, 2);
                g.tok0 = sidx == 0 ? j * P : 0;
                g.ntok = sidx == 0 ? min(P, pre - j * P) : 0;
                g.r0 = 0;
                g.r1 = nseq * G;
            } else {
                const int j = field(c, 5), npp = field(c, 6), nps2 = field(c, 7);
                g.seq = field(c, 2) + m;
                g.tok0 = field(c, 1) + (j - npp + (nps2 & 1)) * P;
                g.ntok = mt;
                g.r0 = m * G;
                g.r1 = (m + 1) * G;
            }
            const unsigned below = sidx <= 0 ? 0u : (c.mask & ((1u << sidx) - 1u));
            const unsigned above = sidx < 0 ? 0u : (c.mask & ~((2u << sidx) - 1u));
            g.first = below == 0u;
            g.last = above == 0u;
            return g;
        };
        auto first_seg = [&](const SharedItemCtx &c) {
            return make_seg(c, c.mask ? __ffs(c.mask) - 1 : -1);
        };
        // a segment's slice of its block-table row: entry e in lane e % 32, register e / 32
        auto load_entries = [&](const SharedSeg &g, int (&ent)[kMaxItemBlocks / 32]) {
            const int nblk = g.valid ? (g.ntok + BS - 1) / BS : 0;
            const int32_t *bt =
                prm.block_tables + (size_t)(g.valid ? g.seq : 0) * prm.max_blocks_per_seq +
                (g.valid ? g.tok0 / BS : 0);
#pragma unroll
            for (int k = 0; k < kMaxItemBlocks / 32; ++k) {
                const int e = k * 32 + lane;
                ent[k] = e < nblk ? bt[e] : 0;
            }
        };
        SharedItemCtx cur_item = load_item(blockIdx.x);
        int pending = take();
        SharedSeg cur = first_seg(cur_item);
        int ent[kMaxItemBlocks / 32];
        load_entries(cur, ent);
        // The next item is looked up while the current item's first segment streams (its
        // descriptor and lengths are a chain of dependent loads), and each segment's table
        // slice while the segment before it streams.
        SharedItemCtx nxt_item = cur_item;
        nxt_item.valid = false;
        while (cur.valid && ok) {
            const int hk = field(cur_item, 4);
            const int first_seq = field(cur_item, 2);
            const int nseq = field(cur_item, 3);
            const int part = field(cur_item, 5);
            const int nparts = chunk_parts(field(cur_item, 6), field(cur_item, 7));
            const int nst = max(1, (cur.ntok + kStageTokens - 1) / kStageTokens);
            SharedSeg nxt;
            nxt.valid = false;
            int nxt_ent[kMaxItemBlocks / 32];
            for (int st = 0; st < nst; ++st, ++it) {
                const int slot = it % L::kStages;
                const uint32_t ph = ((it / L::kStages) & 1) ^ 1;
                if (!warp_wait(smem_u32(&empty[slot]), ph)) {
                    if (lane == 0) atomicOr(prm.status, kStatusTimeout);
                    ok = false;
                    break;
                }
                const int sntok = max(0, min(kStageTokens, cur.ntok - st * kStageTokens));
                const int nb_st = (sntok + BS - 1) / BS;
                const int e0 = st * kBPS;
                const int reg = e0 >> 5;
                int v = ent[0];
#pragma unroll
                for (int k = 1; k < kMaxItemBlocks / 32; ++k)
                    if (reg == k) v = ent[k];
                const int bid = __shfl_sync(0xffffffffu, v, (e0 + lane) & 31);
                const uint32_t bar = smem_u32(&full[slot]);
                if (lane == 0) {
                    StageInfo in;
                    in.s = first_seq; in.hk = hk; in.p = part; in.npart = nparts;
                    in.item = nseq;
                    in.ntok = sntok;
                    in.flags = (cur.first && st == 0 ? kFirst : 0) |
                               (cur.last && st == nst - 1 ? kLast : 0);
                    in.pad = cur.r0 | (cur.r1 << 16);
                    info[slot] = in;
                    mbar_arrive_expect_tx(bar, (uint32_t)(nb_st * BS * L::kRowBytes * 2));
                }
                __syncwarp();
                if (lane < nb_st) {
                    int y;
                    if (bid >= 0 && bid < prm.num_blocks) {
                        y = (bid * Hkv + hk) * BS;
                    } else {
                        atomicOr(prm.status, kStatusBadBlock);
                        y = prm.num_blocks * Hkv * BS;
                    }
                    uint8_t *stage = ring + slot * L::kStageBytes;
                    const uint32_t off = lane * BS * L::kRowBytes;
                    if (H == 2) {
                        tma_load_3d(smem_u32(stage + off), &tmap_k, 0, y, 0, bar, kv_policy);
                        tma_load_3d(smem_u32(stage + L::kKBytes + off), &tmap_v, 0, y, 0, bar,
                                    kv_policy);
                    } else {
                        tma_load_2d(smem_u32(stage + off), &tmap_k, 0, y, bar, kv_policy);
                        tma_load_2d(smem_u32(stage + L::kKBytes + off), &tmap_v, 0, y, bar,
                                    kv_policy);
                    }
                }
                if (st == 0) {
                    if (cur.first) {
                        nxt_item = load_item(__shfl_sync(0xffffffffu, pending, 0));
                        if (nxt_item.valid) pending = take();
                    }
                    if (!cur.last) {
                        const unsigned above = cur_item.mask & ~((2u << cur.sidx) - 1u);
                        nxt = make_seg(cur_item, __ffs(above) - 1);
                    } else {
                        nxt = first_seg(nxt_item);
                    }
                    load_entries(nxt, nxt_ent);
                }
            }
            if (cur.last) cur_item = nxt_item;
            cur = nxt;
#pragma unroll
            for (int k = 0; k < kMaxItemBlocks / 32; ++k) ent[k] = nxt_ent[k];
        }
        if (ok) {
            const int slot = it % L::kStages;
            const uint32_t ph = ((it / L::kStages) & 1) ^ 1;
            if (warp_wait(smem_u32(&empty[slot]), ph)) {
                if (lane == 0) {
                    StageInfo in = {};
                    in.s = -1;
                    in.flags = kEnd;
                    info[slot] = in;
                    mbar_arrive(smem_u32(&full[slot]));
                }
            } else {
                if (lane == 0) atomicOr(prm.status, kStatusTimeout);
                ok = false;
            }
        }
        if (!ok) {
            for (int j = max(0, it - L::kStages); j < it; ++j)
                warp_wait(smem_u32(&full[j % L::kStages]), (j / L::kStages) & 1);
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int w = warp;
    const int gid = lane >> 2;
    const int tig = lane & 3;
    constexpr int KS = D / 16;
    WarpState<D> st;
    reset_state(st);
    const T *qg = reinterpret_cast<const T *>(prm.q);

    for (int it = 0;; ++it) {
        const int slot = it % L::kStages;
        if (!warp_wait(smem_u32(&full[slot]), (it / L::kStages) & 1)) {
            if (lane == 0) atomicOr(prm.status, kStatusTimeout);
            break;
        }
        const StageInfo in = info[slot];
        if (in.flags & kEnd) break;
        const int nrows = in.item * G;

        if (in.flags & kFirst) {
            // A fragments of the item's rows r = member * G + head (rows >= nrows are zero)
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int r = gid + 8 * half;
                const uint32_t *qr = nullptr;
                if (r < nrows) {
                    const int s = in.s + r / G, h = in.hk * G + r % G;
                    qr = reinterpret_cast<const uint32_t *>(
                        qg + ((size_t)s * prm.num_heads + h) * D);
                }
#pragma unroll
                for (int ks = 0; ks < KS; ++ks) {
                    st.qa[ks][half] = qr ? __ldg(qr + ks * 8 + tig) : 0u;
                    st.qa[ks][2 + half] = qr ? __ldg(qr + ks * 8 + tig + 4) : 0u;
                }
            }
            reset_state(st);
        }

        const int valid = in.ntok - 16 * w;
        if (valid > 0) {
            const uint8_t *stage = ring + slot * L::kStageBytes;
            consume_stage<T, D, BS, true>(st, smem_u32(stage), smem_u32(stage + L::kKBytes),
                                          16 * w, lane, valid, prm.scale_log2, in.pad & 0xffff,
                                          in.pad >> 16);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[slot]));

        if (in.flags & kLast) {
            merge_warps<D>(st, nrows, obuf, L::kObufStride, ml, w, lane);
            const int tid = threadIdx.x;
            if (in.npart == 1) {
                // the chunk is this one item: final output
                for (int idx = tid; idx < nrows * D; idx += kConsumerWarps * 32) {
                    const int r = idx / D, dim = idx - r * D;
                    const int s = in.s + r / G, h = in.hk * G + r % G;
                    reinterpret_cast<T *>(prm.out)[((size_t)s * prm.num_heads + h) * D + dim] =
                        from_float<T>(obuf[r * L::kObufStride + dim]);
                }
            } else {
                for (int idx = tid; idx < nrows * D; idx += kConsumerWarps * 32) {
                    const int r = idx / D, dim = idx - r * D;
                    const int s = in.s + r / G, h = in.hk * G + r % G;
                    const size_t row = (size_t)prm.row_base[s] + (size_t)h * prm.np[s] + in.p;
                    prm.ws_o[row * D + dim] = obuf[r * L::kObufStride + dim];
                }
                if (tid < nrows) {
                    const int s = in.s + tid / G, h = in.hk * G + tid % G;
                    const size_t row = (size_t)prm.row_base[s] + (size_t)h * prm.np[s] + in.p;
                    reinterpret_cast<float2 *>(prm.ws_ml)[row] = row_stats(ml, tid);
                }
            }
        }
    }
}

// Merge of the partials of every (sequence, head) whose chunk was split into several
// items: rows row_base[s] + h*np[s] + j, j < np[s]; one warp per pair.
template <typename T, int D>
__global__ void __launch_bounds__(kReduceWarps * 32)
paged_decode_shared_reduce_kernel(SharedParams prm) {
    pdl_wait_and_release();
    if (!plan_matches(prm.counters, prm.num_seqs, prm.num_heads, prm.num_kv_heads, prm.partition))
        return;
    // the decode launch has finished (stream order): re-arm the work counter for the next
    // decode over the same plan
    if (blockIdx.x == 0 && threadIdx.x == 0) prm.counters->next = 0u;
    const int lane = threadIdx.x & 31;
    const int pair = blockIdx.x * kReduceWarps + (threadIdx.x >> 5);
    if (pair >= prm.num_seqs * prm.num_heads) return;
    const int s = pair / prm.num_heads;
    const int h = pair - s * prm.num_heads;
    const int np = prm.np[s];
    if (np == 1) return;   // written by the decode kernel
    const size_t row0 = (size_t)prm.row_base[s] + (size_t)h * np;
    warp_merge<T, D>(reinterpret_cast<const float2 *>(prm.ws_ml) + row0, 1,
                     prm.ws_o + row0 * D, D, np,
                     reinterpret_cast<T *>(prm.out) + ((size_t)s * prm.num_heads + h) * D, lane);
}

}  // namespace pkv
