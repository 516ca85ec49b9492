// Paged single-query decode attention for sm_100a.
//
// What it computes ("vLLM / PagedAttention — 分页 KV Cache 分析" §3.1, the per-page
// loop read as the streaming form of ONE softmax per (sequence, query head)):
//   out[s][h] = sum_t softmax_t(scale * q[s][h] . K_s[t]) V_s[t],  t < len_s,
// with K_s[t] in page block_tables[s][t / bs], row t % bs, KV head h / G.
//
// Work decomposition. A work item is (sequence s, KV head hk, partition p): the
// tokens [p*P, min((p+1)*P, len_s)) of one KV head, for all G query heads that read
// it, so every K/V byte is read from HBM once. Items are numbered sequence-major
// (then KV head, then partition); persistent CTAs (two per SM where shared memory
// allows) take the next free item from a counter in the workspace (or, without
// one, items blockIdx.x, blockIdx.x + gridDim.x, ...). A sequence with one
// partition writes `out` directly; otherwise each item leaves (max, sum,
// normalised partial output) in fp32 scratch and paged_decode_reduce merges them
// exactly (log-sum-exp).
//
// Inside a CTA (160 threads): warp 4 is the producer. It walks the item list one
// item ahead, prefetching the next item's block-table slice into registers (one
// coalesced load per lane) while the current one streams, and for every 64-token
// stage issues one TMA box per page for K and one for V (the whole
// block_size x head_dim tile, 128-byte swizzle) plus, with an item's first stage,
// one box for the item's G query rows; all complete on the stage's mbarrier.
// Warps 0-3 are consumers: each takes 16 of the stage's 64 tokens, computes the
// scores of the whole GQA group with m16n8k16 tensor-core MMAs (query heads on M,
// padded to 16; tokens on N; head_dim on K), keeps an online max / sum in fp32,
// and accumulates P.V with a second MMA (P stays in registers as the A operand).
// At the end of an item the four warps merge their softmax states through
// shared memory. Masking is by selection: scores of tokens at or past len_s are
// -inf and their V rows are zeroed in registers, so stale bits (NaN) never reach
// the result.
#pragma once

#include "pkv_ptx.cuh"

namespace pkv {

// L2 policy of the K/V tile loads: evict-first (each byte is read once per call)
// unless built with PKV_KV_EVICT_FIRST=0.
#ifndef PKV_KV_EVICT_FIRST
#define PKV_KV_EVICT_FIRST 1
#endif

constexpr int kStageTokens = 64;
constexpr int kConsumerWarps = 4;
constexpr int kDecodeThreads = (kConsumerWarps + 1) * 32;
constexpr int kMaxGroup = 16;               // query heads per KV head (MMA M)
constexpr int kMaxItemBlocks = 256;         // block-table entries held per item (8 per lane)
constexpr uint32_t kWaitLimit = 1u << 22;   // polls before a pipeline wait gives up

constexpr unsigned kStatusBadSlot = 1u << 0;
constexpr unsigned kStatusBadPair = 1u << 1;
constexpr unsigned kStatusBadBlock = 1u << 2;
constexpr unsigned kStatusBadLen = 1u << 3;
constexpr unsigned kStatusTimeout = 1u << 4;

struct StageInfo {
    int s, hk, p, npart;
    int item;   // compact item index (scratch row)
    int ntok;   // tokens of this stage that belong to the sequence (0..64)
    int flags;  // bit 0: first stage of the item, bit 1: last stage, bit 2: end of work
    int pad;
};
constexpr int kFirst = 1, kLast = 2, kEnd = 4;

// Dynamic work distribution: producers take item indices from `next`. A launch that
// found the header armed leaves it armed: its last CTA out (counted in `exit`) resets
// the counters. The reduce kernel, which follows every decode that has a workspace,
// re-arms it too (next = 0, arrive = exit = 0, armed = kSchedArmed); a header that is
// not armed (a workspace never used before) makes that call fall back to the static
// schedule. The same header serves paged_decode_step_kernel, whose grid barrier lives
// in `arrive` and `gen`.
constexpr unsigned kSchedArmed = 0x9A6EDC0Du;
struct SchedHeader {
    unsigned armed;
    int next;         // dynamic work counter
    unsigned arrive;  // step kernel: CTAs arrived at the grid barrier
    unsigned gen;     // step kernel: barrier generation
    unsigned exit;    // step kernel: CTAs finished
    int pad[59];
};
static_assert(sizeof(SchedHeader) == 256, "workspace header size");

struct DecodeParams {
    SchedHeader *sched;  // null: static schedule (items blockIdx.x + k * gridDim.x)
    void *out;
    const int32_t *block_tables;
    const int32_t *context_lens;
    float *ws_o;         // [items * G][D]
    float *ws_ml;        // [items * G][2]  (max in log2 units, sum)
    int32_t *ws_seq_base;// [B] first item of each sequence
    unsigned *status;
    int num_seqs, num_heads, num_kv_heads, group;
    int max_blocks_per_seq, num_blocks, max_context_len, partition;
    float scale_log2;    // scale * log2(e)
    // fused decode step only: this step's K/V rows [B][Hkv][D] and the caches they go to
    const void *k_new, *v_new;
    void *k_cache, *v_cache;
};

// Shared-memory plan. A stage holds 64 tokens of K then V as [token][head_dim]
// rows (head_dim*2 bytes each); TMA's 128-byte swizzle permutes the 16-byte
// chunks of every 128-byte line by (line index mod 8), so line L = token*halves +
// half has chunk c at L*128 + ((c ^ (L & 7)) * 16).
template <int D>
struct DecodeLayout {
    static constexpr int kHalves = D / 64;
    static constexpr int kRowBytes = D * 2;
    static constexpr int kKBytes = kStageTokens * kRowBytes;
    static constexpr int kStageBytes = 2 * kKBytes;            // K + V
    static constexpr int kStages = D == 128 ? 3 : 6;
    static constexpr int kRingBytes = kStages * kStageBytes;
    static constexpr int kObufStride = D + 8;                  // floats per merge row
    static constexpr int kMetaBytes = 2048;    // infos + barriers + ml + item-order table
    __host__ __device__ static constexpr int q_slot_bytes(int group) {
        return (group * kRowBytes + 1023) / 1024 * 1024;
    }
    __host__ __device__ static constexpr int obuf_bytes(int group) {
        return (group * kObufStride * 4 + 127) / 128 * 128;
    }
    static constexpr size_t smem_bytes(int group) {
        return 1024 /*alignment slack*/ + kRingBytes + (size_t)kStages * q_slot_bytes(group) +
               obuf_bytes(group) + kMetaBytes;
    }
};

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void named_bar_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity) {
    const bool mine = mbar_wait_bounded(bar, parity, kWaitLimit);
    return __all_sync(0xffffffffu, mine);
}

// Byte offset of 16-byte chunk c of 128-byte line L in a 128B-swizzled region.
__device__ __forceinline__ uint32_t swz(int line, int c) {
    return (uint32_t)(line * 128 + ((c ^ (line & 7)) << 4));
}

// Line of (stage token t, column half h) in a stage: each page tile lands as
// [half][row][64 elements], so eight consecutive tokens of one half occupy eight
// consecutive lines (eight different swizzle phases: conflict-free ldmatrix).
template <int H, int BS>
__device__ __forceinline__ int kv_line(int t, int h) {
    if (H == 1) return t;
    return (t / BS) * (2 * BS) + h * BS + (t % BS);
}

// Position of one work item in the list (lane-uniform).
struct ItemPos {
    int item, s, hk, p, np, ntok, nst, nblk;
    int ticket;   // position in the hand-out order (== item in sequence-major order)
    bool valid;
};

// Walks the item list in increasing order, 32 sequences at a time (one context
// length per lane, warp prefix sum of items per sequence).
struct ItemWalker {
    int cs = 0, chunk_base = 0, chunk_total = 0, incl = 0, my_items = 0, my_np = 0, my_len = 0;
    bool loaded = false;

    __device__ ItemPos find(int item, const DecodeParams &prm, int lane) {
        ItemPos r;
        r.item = item;
        r.ticket = item;
        r.valid = false;
        const int B = prm.num_seqs, P = prm.partition, Hkv = prm.num_kv_heads;
        for (;;) {
            if (cs >= B) return r;
            if (!loaded) {
                const int s = cs + lane;
                int len = 0;
                if (s < B) {
                    len = prm.context_lens[s];
                    if (len < 0 || len > prm.max_context_len) {
                        if (blockIdx.x == 0) atomicOr(prm.status, kStatusBadLen);
                        len = len < 0 ? 0 : prm.max_context_len;
                    }
                }
                my_len = len;
                my_np = s < B ? max(1, (len + P - 1) / P) : 0;
                my_items = my_np * Hkv;
                incl = my_items;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int v = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += v;
                }
                chunk_total = __shfl_sync(0xffffffffu, incl, 31);
                loaded = true;
            }
            if (item < chunk_base + chunk_total) break;
            chunk_base += chunk_total;
            cs += 32;
            loaded = false;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, item < chunk_base + incl);
        const int ln = __ffs(hit) - 1;
        const int excl = __shfl_sync(0xffffffffu, incl - my_items, ln);
        const int len = __shfl_sync(0xffffffffu, my_len, ln);
        r.s = cs + ln;
        r.np = __shfl_sync(0xffffffffu, my_np, ln);
        const int rem = item - chunk_base - excl;
        r.hk = rem / r.np;
        r.p = rem - r.hk * r.np;
        r.ntok = max(0, min(P, len - r.p * P));
        r.nst = max(1, (r.ntok + kStageTokens - 1) / kStageTokens);
        r.valid = true;
        return r;
    }
};

// Longest-first order, for small batches of long contexts. Items are handed out by
// their number of 64-token stages, largest first (within a count: sequence, then KV
// head, then partition), so the last items any CTA takes are the shortest and the
// launch drains evenly (long context: 99.3 % instead of 97.9 % of the copy peak). With
// many sequences the sequence-major order is kept: it measured faster there (GQA, 256
// sequences: 2.3 % ahead), as concurrently running CTAs then read neighbouring pages of
// the same sequences and the walker never rescans the batch. An item's stage
// count is P/64 for every partition but a sequence's last, which holds the remainder.
// Tickets of stage count c are [first[c], first[c - 1]); first[S] = 0 and first[0] is
// the item total (S = P/64). The table is built in shared memory by order_table() at
// the start of the kernel; the walker keeps, per count, a cursor over the sequences
// (32 at a time), so tickets must reach it in increasing order. Results carry the
// canonical item number (sequence-major, as ItemWalker numbers them), which indexes
// the partials.
constexpr int kMaxStageCount = kMaxItemBlocks * 32 / kStageTokens;   // P <= 256 blocks of 32
#ifndef PKV_ORDER_MAX_SEQS
#define PKV_ORDER_MAX_SEQS 64
#endif
constexpr int kOrderMaxSeqs = PKV_ORDER_MAX_SEQS;   // longest-first order up to this batch size

__device__ __forceinline__ int clamp_ctx(int len, const DecodeParams &prm, bool flag) {
    if (len < 0 || len > prm.max_context_len) {
        if (flag) atomicOr(prm.status, kStatusBadLen);
        len = len < 0 ? 0 : prm.max_context_len;
    }
    return len;
}

// Last partition's stage count of a context of len tokens (1 for an empty context).
__device__ __forceinline__ int last_stages(int len, int np, int P) {
    const int ntok = len - (np - 1) * P;
    return ntok <= 0 ? 1 : (ntok + kStageTokens - 1) / kStageTokens;
}

// All threads of the CTA: first[0..S] (int[kMaxStageCount + 1]) from the context lengths;
// cnt is scratch of the same size. Ends with a barrier.
__device__ __forceinline__ void order_table(const DecodeParams &prm, int *first, int *cnt) {
    const int P = prm.partition, S = P / kStageTokens, Hkv = prm.num_kv_heads;
    for (int c = threadIdx.x; c <= S; c += blockDim.x) cnt[c] = 0;
    __syncthreads();
    for (int s = threadIdx.x; s < prm.num_seqs; s += blockDim.x) {
        const int len = clamp_ctx(prm.context_lens[s], prm, blockIdx.x == 0);
        const int np = max(1, (len + P - 1) / P);
        if (np > 1) atomicAdd(&cnt[S], (np - 1) * Hkv);
        atomicAdd(&cnt[last_stages(len, np, P)], Hkv);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int c = S; c >= 1; --c) {
            first[c] = acc;
            acc += cnt[c];
        }
        first[0] = acc;
    }
    __syncthreads();
}

struct OrderWalker {
    const int *first;
    int c = 0;   // stage count whose sequences are being walked (0: none yet)
    int cs = 0, base = 0, cbase = 0, total = 0, ctotal = 0;
    int my_len = 0, my_np = 0, my_k = 0, incl = 0, cincl = 0;
    bool loaded = false;

    __device__ ItemPos find(int ticket, const DecodeParams &prm, int lane) {
        ItemPos r;
        r.item = ticket;
        r.ticket = ticket;
        r.valid = false;
        const int B = prm.num_seqs, P = prm.partition, Hkv = prm.num_kv_heads;
        const int S = P / kStageTokens;
        if (ticket < 0 || ticket >= first[0]) return r;
        int cc = c ? c : S;
        while (cc > 1 && ticket >= first[cc - 1]) --cc;
        if (cc != c) {   // a new stage count: walk the sequences from the start
            c = cc;
            cs = 0;
            base = 0;
            cbase = 0;
            loaded = false;
        }
        const int rank = ticket - first[c];
        for (;;) {
            if (cs >= B) return r;   // cannot happen while first[] matches the lengths
            if (!loaded) {
                const int s = cs + lane;
                int len = 0, np = 0, k = 0;
                if (s < B) {
                    len = clamp_ctx(prm.context_lens[s], prm, false);
                    np = max(1, (len + P - 1) / P);
                    const int cl = last_stages(len, np, P);
                    k = (c == S ? np - 1 : 0) + (cl == c ? 1 : 0);
                }
                my_len = len;
                my_np = np;
                my_k = k;
                incl = k * Hkv;
                cincl = np * Hkv;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int v = __shfl_up_sync(0xffffffffu, incl, o);
                    const int w = __shfl_up_sync(0xffffffffu, cincl, o);
                    if (lane >= o) {
                        incl += v;
                        cincl += w;
                    }
                }
                total = __shfl_sync(0xffffffffu, incl, 31);
                ctotal = __shfl_sync(0xffffffffu, cincl, 31);
                loaded = true;
            }
            if (rank < base + total) break;
            base += total;
            cbase += ctotal;
            cs += 32;
            loaded = false;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, rank < base + incl);
        const int ln = __ffs(hit) - 1;
        const int k = __shfl_sync(0xffffffffu, my_k, ln);
        const int excl = __shfl_sync(0xffffffffu, incl - my_k * Hkv, ln);
        const int cexcl = __shfl_sync(0xffffffffu, cincl - my_np * Hkv, ln);
        const int len = __shfl_sync(0xffffffffu, my_len, ln);
        r.s = cs + ln;
        r.np = __shfl_sync(0xffffffffu, my_np, ln);
        const int rem = rank - base - excl;
        r.hk = rem / k;
        const int j = rem - r.hk * k;
        r.p = (c == S) ? j : r.np - 1;
        r.item = cbase + cexcl + r.hk * r.np + r.p;
        r.ntok = max(0, min(P, len - r.p * P));
        r.nst = max(1, (r.ntok + kStageTokens - 1) / kStageTokens);
        r.valid = true;
        return r;
    }
};

// Online-softmax state of one consumer warp for a 16-row query tile: lane (gid, tig)
// holds rows gid and gid + 8 (max m, partial sum l, output accumulators o).
template <int D>
struct WarpState {
    uint32_t qa[D / 16][4];   // A fragments of Q (rows >= the tile's row count are zero)
    float o[D / 8][4];
    float m0, m1, l0, l1;
};

template <int D>
__device__ __forceinline__ void reset_state(WarpState<D> &st) {
#pragma unroll
    for (int n = 0; n < D / 8; ++n) st.o[n][0] = st.o[n][1] = st.o[n][2] = st.o[n][3] = 0.f;
    st.m0 = st.m1 = -INFINITY;
    st.l0 = st.l1 = 0.f;
}

// One warp's share of a stage: tokens tok0 .. tok0+15 of the stage's K and V tiles
// (tok0 a multiple of 16), of which the first `valid` belong to the sequence.
//   S = Q K^T (two n-tiles of 8 tokens), scale, mask, online softmax, O += P V.
// kRows: only query rows r0 <= row < r1 attend to these tokens (the others' scores are
// -inf); a row that has attended to nothing yet keeps m = -inf, l = 0, o = 0.
template <typename T, int D, int BS, bool kRows = false>
__device__ __forceinline__ void consume_stage(WarpState<D> &st, uint32_t kbase, uint32_t vbase,
                                              int tok0, int lane, int valid, float scale_log2,
                                              int r0 = 0, int r1 = kMaxGroup) {
    constexpr int H = D / 64;
    constexpr int NT = D / 8;
    const int tig = lane & 3;
    float sc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
        const int t = tok0 + 8 * nt + (lane & 7);
        const int mi = lane >> 3;
#pragma unroll
        for (int hf = 0; hf < H; ++hf) {
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(kbase + swz(kv_line<H, BS>(t, hf), c2 * 4 + mi), b0, b1, b2, b3);
                const int ks = hf * 4 + c2 * 2;
                Mma<T>::run(sc[nt], st.qa[ks], b0, b1);
                Mma<T>::run(sc[nt], st.qa[ks + 1], b2, b3);
            }
        }
    }
    // scale, mask, online softmax (rows gid and gid+8)
    const int gid = lane >> 2;
    const bool row0_in = !kRows || (gid >= r0 && gid < r1);
    const bool row1_in = !kRows || (gid + 8 >= r0 && gid + 8 < r1);
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const bool in_seq = 8 * nt + 2 * tig + e < valid;
            sc[nt][e] = in_seq && row0_in ? sc[nt][e] * scale_log2 : -INFINITY;
            sc[nt][2 + e] = in_seq && row1_in ? sc[nt][2 + e] * scale_log2 : -INFINITY;
            mx0 = fmaxf(mx0, sc[nt][e]);
            mx1 = fmaxf(mx1, sc[nt][2 + e]);
        }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(st.m0, mx0), mn1 = fmaxf(st.m1, mx1);
    // with row masks a row may still have seen nothing (max -inf): subtract 0 instead,
    // so that its weights are 0 rather than NaN
    const float ms0 = kRows && mn0 == -INFINITY ? 0.f : mn0;
    const float ms1 = kRows && mn1 == -INFINITY ? 0.f : mn1;
    const float a0 = ex2(st.m0 - ms0), a1 = ex2(st.m1 - ms1);
    st.m0 = mn0;
    st.m1 = mn1;
    float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            sc[nt][e] = ex2(sc[nt][e] - ms0);
            sc[nt][2 + e] = ex2(sc[nt][2 + e] - ms1);
            ps0 += sc[nt][e];
            ps1 += sc[nt][2 + e];
        }
    }
    st.l0 = st.l0 * a0 + ps0;
    st.l1 = st.l1 * a1 + ps1;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        st.o[n][0] *= a0; st.o[n][1] *= a0;
        st.o[n][2] *= a1; st.o[n][3] *= a1;
    }
    uint32_t pa[4];
    pa[0] = Mma<T>::pack(sc[0][0], sc[0][1]);
    pa[1] = Mma<T>::pack(sc[0][2], sc[0][3]);
    pa[2] = Mma<T>::pack(sc[1][0], sc[1][1]);
    pa[3] = Mma<T>::pack(sc[1][2], sc[1][3]);
    // O += P V  (V rows of tokens past the sequence are zeroed)
    uint32_t keep_lo = 0xffffffffu, keep_hi = 0xffffffffu;
    if (valid < 16) {
        const int t0 = 2 * tig, t1 = 2 * tig + 8;
        keep_lo = (t0 < valid ? 0x0000ffffu : 0u) | (t0 + 1 < valid ? 0xffff0000u : 0u);
        keep_hi = (t1 < valid ? 0x0000ffffu : 0u) | (t1 + 1 < valid ? 0xffff0000u : 0u);
    }
    const int mi = lane >> 3;
    const int tv = tok0 + (mi & 1) * 8 + (lane & 7);
#pragma unroll
    for (int dp = 0; dp < D / 16; ++dp) {
        const int hf = dp >> 2;
        const int c = 2 * (dp & 3) + (mi >> 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_trans(vbase + swz(kv_line<H, BS>(tv, hf), c), b0, b1, b2, b3);
        b0 &= keep_lo; b1 &= keep_hi; b2 &= keep_lo; b3 &= keep_hi;
        Mma<T>::run(st.o[2 * dp], pa, b0, b1);
        Mma<T>::run(st.o[2 * dp + 1], pa, b2, b3);
    }
}

// End of an item: combine the four consumer warps' states. Leaves the normalised
// output of rows < nrows in obuf (row stride obuf_stride floats) and every warp's
// (m, l) per row in ml[warp * 16 + row]. All 128 consumer threads call it; the first
// barrier also protects obuf and ml from the previous item's readers.
template <int D>
__device__ __forceinline__ void merge_warps(WarpState<D> &st, int nrows, float *obuf,
                                            int obuf_stride, float2 *ml, int w, int lane) {
    constexpr int NT = D / 8;
    const int gid = lane >> 2;
    const int tig = lane & 3;
    float lt0 = st.l0 + __shfl_xor_sync(0xffffffffu, st.l0, 1);
    lt0 += __shfl_xor_sync(0xffffffffu, lt0, 2);
    float lt1 = st.l1 + __shfl_xor_sync(0xffffffffu, st.l1, 1);
    lt1 += __shfl_xor_sync(0xffffffffu, lt1, 2);
    named_bar_sync(1, kConsumerWarps * 32);
    if (tig == 0) {
        ml[w * kMaxGroup + gid] = make_float2(st.m0, lt0);
        ml[w * kMaxGroup + gid + 8] = make_float2(st.m1, lt1);
    }
    named_bar_sync(1, kConsumerWarps * 32);
    // my rows' scale factors f = 2^(m_self - M) / L  (0 when the item is empty)
    float fr[2];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        const int row = min(gid + 8 * rr, nrows - 1);
        float M = -INFINITY;
#pragma unroll
        for (int ww = 0; ww < kConsumerWarps; ++ww) M = fmaxf(M, ml[ww * kMaxGroup + row].x);
        float Lsum = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int ww = 0; ww < kConsumerWarps; ++ww) {
                const float2 v = ml[ww * kMaxGroup + row];
                Lsum += v.y * ex2(v.x - M);
            }
        }
        const float mself = rr ? st.m1 : st.m0;
        fr[rr] = (Lsum > 0.f) ? ex2(mself - M) / Lsum : 0.f;
    }
    // accumulate the four warps' scaled outputs in a fixed order (deterministic)
#pragma unroll
    for (int ww = 0; ww < kConsumerWarps; ++ww) {
        if (w == ww) {
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const int row = gid + 8 * rr;
                if (row < nrows) {
                    float2 *dst = reinterpret_cast<float2 *>(obuf + row * obuf_stride + 2 * tig);
#pragma unroll
                    for (int n = 0; n < NT; ++n) {
                        float2 v = make_float2(st.o[n][2 * rr] * fr[rr], st.o[n][2 * rr + 1] * fr[rr]);
                        if (ww > 0) {
                            const float2 prev = dst[n * 4];
                            v.x += prev.x;
                            v.y += prev.y;
                        }
                        dst[n * 4] = v;
                    }
                }
            }
        }
        named_bar_sync(1, kConsumerWarps * 32);
    }
}

// (M, L) of one row over the four warps' (m, l) pairs.
__device__ __forceinline__ float2 row_stats(const float2 *ml, int row) {
    float M = -INFINITY;
    for (int ww = 0; ww < kConsumerWarps; ++ww) M = fmaxf(M, ml[ww * kMaxGroup + row].x);
    float Lsum = 0.f;
    if (M != -INFINITY)
        for (int ww = 0; ww < kConsumerWarps; ++ww) {
            const float2 v = ml[ww * kMaxGroup + row];
            Lsum += v.y * ex2(v.x - M);
        }
    return make_float2(M, Lsum);
}

// Carve-up of the decode kernels' dynamic shared memory (base aligned to 1024 B).
template <int D>
struct DecodeSmem {
    uint8_t *ring, *qring;
    float *obuf;
    StageInfo *info;
    uint64_t *full, *empty;
    float2 *ml;   // [4][16]
    int *order_first, *order_cnt;   // [kMaxStageCount + 1] each
    int qslot_bytes;
    __device__ DecodeSmem(uint8_t *smem, int G) {
        using L = DecodeLayout<D>;
        qslot_bytes = L::q_slot_bytes(G);
        ring = smem;
        qring = smem + L::kRingBytes;
        obuf = reinterpret_cast<float *>(qring + L::kStages * qslot_bytes);
        info = reinterpret_cast<StageInfo *>(reinterpret_cast<uint8_t *>(obuf) + L::obuf_bytes(G));
        full = reinterpret_cast<uint64_t *>(info + L::kStages);
        empty = full + L::kStages;
        ml = reinterpret_cast<float2 *>(empty + L::kStages);
        order_first = reinterpret_cast<int *>(ml + kConsumerWarps * kMaxGroup);
        order_cnt = order_first + kMaxStageCount + 1;
    }
    __device__ void init_barriers() {
        if (threadIdx.x == 0) {
            for (int i = 0; i < DecodeLayout<D>::kStages; ++i) {
                mbar_init(smem_u32(&full[i]), 1);
                mbar_init(smem_u32(&empty[i]), kConsumerWarps);
            }
            fence_mbar_init();
        }
    }
};

__device__ __forceinline__ uint8_t *aligned_dynamic_smem() {
    extern __shared__ uint8_t smem_raw[];
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                       ~uintptr_t(1023));
}

__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// The work-item loop shared by the decode kernels: warp 4 produces, warps 0-3
// consume, until the item list is exhausted (barriers already initialised).
// dynamic: take items from prm.sched->next (the caller checked the header), else the
// static schedule.
// kStep: before loading the page that holds a sequence's last token (position
// len_s - 1), the producer writes that token's K and V rows (prm.k_new / prm.v_new,
// [B][Hkv][D]) for its KV head into the cache, so the cache write of the decode step
// needs no launch of its own.
template <typename T, int D, int BS, bool kStep>
__device__ __forceinline__ void decode_items(const CUtensorMap *tmap_k, const CUtensorMap *tmap_v,
                                             const CUtensorMap *tmap_q, const DecodeParams &prm,
                                             DecodeSmem<D> &sm, bool dynamic) {
    using L = DecodeLayout<D>;
    constexpr int kBPS = kStageTokens / BS;   // blocks per stage
    constexpr int H = L::kHalves;
    const int G = prm.group;
    const int qslot_bytes = sm.qslot_bytes;
    uint8_t *ring = sm.ring;
    uint8_t *qring = sm.qring;
    float *obuf = sm.obuf;
    StageInfo *info = sm.info;
    uint64_t *full = sm.full;
    uint64_t *empty = sm.empty;
    float2 *ml = sm.ml;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int Hkv = prm.num_kv_heads;
    const int P = prm.partition;

    if (prm.num_seqs <= kOrderMaxSeqs) order_table(prm, sm.order_first, sm.order_cnt);

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(tmap_k);
            prefetch_tensormap(tmap_v);
            prefetch_tensormap(tmap_q);
        }
#if PKV_KV_EVICT_FIRST
        const uint64_t kv_policy = l2_evict_first_policy();
#else
        const uint64_t kv_policy = l2_evict_normal_policy();
#endif
        ItemWalker walker;
        OrderWalker owalk;
        owalk.first = sm.order_first;
        const bool ordered = prm.num_seqs <= kOrderMaxSeqs;
        int it = 0;
        bool ok = true;

        // this item's slice of the block table: entry e lives in lane e % 32, register e / 32
#define PKV_LOAD_ENTRIES(ip, ent)                                                         \
    {                                                                                   \
        const int nblk_ = (ip).valid ? ((ip).ntok + BS - 1) / BS : 0;                   \
        const int32_t *bt_ = prm.block_tables +                                         \
                             ((ip).valid ? (size_t)(ip).s * prm.max_blocks_per_seq +    \
                                               (size_t)(ip).p * (P / BS)                \
                                         : 0);                                          \
        _Pragma("unroll") for (int k_ = 0; k_ < kMaxItemBlocks / 32; ++k_) {            \
            const int e_ = k_ * 32 + lane;                                              \
            ent[k_] = e_ < nblk_ ? bt_[e_] : 0;                                         \
        }                                                                               \
    }

        // Every CTA's first item is its index (the grid never exceeds the item count);
        // later tickets come from the counter, offset by the grid. A ticket is requested
        // one item before it is resolved, so the atomic's latency overlaps a whole item;
        // the value lives in lane 0 until used.
        auto request = [&](int static_item) {
            int v = static_item;
            if (dynamic && lane == 0) v = (int)gridDim.x + atomicAdd(&prm.sched->next, 1);
            return v;
        };
        auto redeem = [&](int ticket) { return __shfl_sync(0xffffffffu, ticket, 0); };
        ItemPos cur = ordered ? owalk.find((int)blockIdx.x, prm, lane)
                              : walker.find((int)blockIdx.x, prm, lane);
        int pending = request(cur.ticket + gridDim.x);
        int cur_ent[kMaxItemBlocks / 32];
        PKV_LOAD_ENTRIES(cur, cur_ent);
        while (cur.valid) {
            if (cur.hk == 0 && cur.p == 0 && lane == 0 && prm.ws_seq_base)
                prm.ws_seq_base[cur.s] = cur.item;
            ItemPos nxt;
            nxt.valid = false;
            int nxt_ent[kMaxItemBlocks / 32];
            for (int st = 0; st < cur.nst; ++st, ++it) {
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
                int v = cur_ent[0];
#pragma unroll
                for (int k = 1; k < kMaxItemBlocks / 32; ++k)
                    if (reg == k) v = cur_ent[k];
                const int bid = __shfl_sync(0xffffffffu, v, (e0 + lane) & 31);
                const uint32_t bar = smem_u32(&full[slot]);
                if (lane == 0) {
                    StageInfo in;
                    in.s = cur.s; in.hk = cur.hk; in.p = cur.p; in.npart = cur.np;
                    in.item = cur.item;
                    in.ntok = sntok;
                    in.flags = (st == 0 ? kFirst : 0) | (st == cur.nst - 1 ? kLast : 0);
                    in.pad = 0;
                    info[slot] = in;
                    const uint32_t qbytes = st == 0 ? (uint32_t)(G * L::kRowBytes) : 0u;
                    mbar_arrive_expect_tx(bar, (uint32_t)(nb_st * BS * L::kRowBytes * 2) + qbytes);
                }
                if constexpr (kStep) {
                    if (cur.p == cur.np - 1 && st == cur.nst - 1 && cur.ntok > 0) {
                        // this stage holds the sequence's last token: write its K/V row first
                        const int tl = cur.ntok - 1 - st * kStageTokens;
                        const int wb = __shfl_sync(0xffffffffu, bid, tl / BS);
                        constexpr int VPR = D * 2 / 16;   // 16-byte vectors per row
                        if (wb >= 0 && wb < prm.num_blocks && lane < 2 * VPR) {
                            const bool isv = lane >= VPR;
                            const int vi = lane - (isv ? VPR : 0);
                            const uint4 *src = reinterpret_cast<const uint4 *>(isv ? prm.v_new : prm.k_new) +
                                               ((size_t)cur.s * Hkv + cur.hk) * VPR + vi;
                            uint4 *dst = reinterpret_cast<uint4 *>(isv ? prm.v_cache : prm.k_cache) +
                                         (((size_t)wb * Hkv + cur.hk) * BS + tl % BS) * VPR + vi;
                            *dst = *src;
                            fence_proxy_async_global();   // before the tensor-map read of it
                        }
                        __syncwarp();
                        fence_proxy_async_global();
                    }
                }
                __syncwarp();
                uint8_t *stage = ring + slot * L::kStageBytes;
                if (lane < nb_st) {
                    int y;
                    if (bid >= 0 && bid < prm.num_blocks) {
                        y = (bid * Hkv + cur.hk) * BS;
                    } else {
                        atomicOr(prm.status, kStatusBadBlock);
                        y = prm.num_blocks * Hkv * BS;   // fully out of range: reads zeros
                    }
                    const uint32_t off = lane * BS * L::kRowBytes;
                    if (H == 2) {
                        tma_load_3d(smem_u32(stage + off), tmap_k, 0, y, 0, bar, kv_policy);
                        tma_load_3d(smem_u32(stage + L::kKBytes + off), tmap_v, 0, y, 0, bar,
                                    kv_policy);
                    } else {
                        tma_load_2d(smem_u32(stage + off), tmap_k, 0, y, bar, kv_policy);
                        tma_load_2d(smem_u32(stage + L::kKBytes + off), tmap_v, 0, y, bar,
                                    kv_policy);
                    }
                }
                if (st == 0 && lane == 31) {
                    const int qrow = cur.s * prm.num_heads + cur.hk * G;
                    const uint32_t qdst = smem_u32(qring + slot * qslot_bytes);
                    if (H == 2)
                        tma_load_3d(qdst, tmap_q, 0, qrow, 0, bar, kv_policy);
                    else
                        tma_load_2d(qdst, tmap_q, 0, qrow, bar, kv_policy);
                }
                if (st == 0) {
                    // look one item ahead: position and block-table slice
                    nxt = ordered ? owalk.find(redeem(pending), prm, lane)
                                  : walker.find(redeem(pending), prm, lane);
                    PKV_LOAD_ENTRIES(nxt, nxt_ent);
                    if (nxt.valid) pending = request(nxt.ticket + gridDim.x);
                }
            }
            if (!ok) break;
            cur = nxt;
#pragma unroll
            for (int k = 0; k < kMaxItemBlocks / 32; ++k) cur_ent[k] = nxt_ent[k];
        }
#undef PKV_LOAD_ENTRIES
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
            // leave only after every tile load this warp issued has landed
            for (int j = max(0, it - L::kStages); j < it; ++j)
                warp_wait(smem_u32(&full[j % L::kStages]), (j / L::kStages) & 1);
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int w = warp;
    const int gid = lane >> 2;
    constexpr int KS = D / 16;   // k-steps of QK
    WarpState<D> st;
    reset_state(st);

    for (int it = 0;; ++it) {
        const int slot = it % L::kStages;
        if (!warp_wait(smem_u32(&full[slot]), (it / L::kStages) & 1)) {
            if (lane == 0) atomicOr(prm.status, kStatusTimeout);
            break;
        }
        const StageInfo in = info[slot];
        if (in.flags & kEnd) break;

        if (in.flags & kFirst) {
            // A fragments of the G query rows (rows >= G are zero)
            const uint32_t qbase = smem_u32(qring + slot * qslot_bytes);
            const int mi = lane >> 3;
            const int row = min((mi & 1) * 8 + (lane & 7), G - 1);
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                const int hf = ks >> 2;
                const int c = 2 * (ks & 3) + (mi >> 1);
                ldsm_x4(qbase + swz(hf * G + row, c), st.qa[ks][0], st.qa[ks][1], st.qa[ks][2],
                        st.qa[ks][3]);
                if (gid >= G) st.qa[ks][0] = st.qa[ks][2] = 0u;
                if (gid + 8 >= G) st.qa[ks][1] = st.qa[ks][3] = 0u;
            }
            reset_state(st);
        }

        const int valid = in.ntok - 16 * w;   // tokens of my 16-token slice in the sequence
        if (valid > 0) {
            const uint8_t *stage = ring + slot * L::kStageBytes;
            consume_stage<T, D, BS>(st, smem_u32(stage), smem_u32(stage + L::kKBytes), 16 * w,
                                    lane, valid, prm.scale_log2);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[slot]));

        if (in.flags & kLast) {
            merge_warps<D>(st, G, obuf, L::kObufStride, ml, w, lane);
            const int tid = threadIdx.x;   // 0..127
            if (in.npart == 1) {
                T *out = reinterpret_cast<T *>(prm.out) +
                         ((size_t)in.s * prm.num_heads + (size_t)in.hk * G) * D;
                for (int idx = tid; idx < G * D; idx += kConsumerWarps * 32) {
                    const int row = idx / D, dim = idx - row * D;
                    out[idx] = from_float<T>(obuf[row * L::kObufStride + dim]);
                }
            } else {
                float *dst = prm.ws_o + (size_t)in.item * G * D;
                for (int idx = tid; idx < G * D; idx += kConsumerWarps * 32) {
                    const int row = idx / D, dim = idx - row * D;
                    dst[idx] = obuf[row * L::kObufStride + dim];
                }
                if (tid < G)
                    reinterpret_cast<float2 *>(prm.ws_ml)[(size_t)in.item * G + tid] =
                        row_stats(ml, tid);
            }
        }
    }
}

// How a launch uses the workspace header: kSchedDynamic when it is armed (items from the
// counter, the last CTA out re-arms it); kSchedArmZero when it is zero and the caller
// guarantees a zero-filled workspace (static schedule, and the last CTA out arms it);
// kSchedStatic otherwise. Read by every CTA before it changes anything; `armed` is
// written again only by the last CTA out (sched_exit), so every CTA decides alike.
constexpr int kSchedStatic = 0, kSchedDynamic = 1, kSchedArmZero = 2;
__device__ __forceinline__ int sched_mode(const DecodeParams &prm, bool zero_filled, int *flag) {
    if (threadIdx.x == 0) {
        int m = kSchedStatic;
        if (prm.sched != nullptr) {
            const unsigned a = *(volatile unsigned *)&prm.sched->armed;
            m = a == kSchedArmed ? kSchedDynamic : (zero_filled && a == 0u ? kSchedArmZero
                                                                           : kSchedStatic);
        }
        *flag = m;
    }
    __syncthreads();
    return *flag;
}

// End of a launch that found the header armed or zero: the last CTA out (re-)arms it
// (counter and step counters 0), so the next launch on the workspace may run without a
// merge kernel in between. Every CTA of the launch calls it (all threads).
__device__ __forceinline__ void sched_exit(SchedHeader *h) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned t = atomicAdd(&h->exit, 1u);
        if (t == gridDim.x - 1) {
            h->next = 0;
            h->arrive = 0;
            h->exit = 0;
            __threadfence();
            h->armed = kSchedArmed;
        }
    }
}

template <typename T, int D, int BS>
__global__ void __launch_bounds__(kDecodeThreads, 2)
paged_decode_partition_kernel(const __grid_constant__ CUtensorMap tmap_k,
                              const __grid_constant__ CUtensorMap tmap_v,
                              const __grid_constant__ CUtensorMap tmap_q, DecodeParams prm) {
    __shared__ int s_mode;
    DecodeSmem<D> sm(aligned_dynamic_smem(), prm.group);
    sm.init_barriers();
    pdl_wait_and_release();
    const int mode = sched_mode(prm, false, &s_mode);   // a decode workspace may hold anything
    decode_items<T, D, BS, false>(&tmap_k, &tmap_v, &tmap_q, prm, sm, mode == kSchedDynamic);
    // reread: nothing held across the loop
    if (*(volatile int *)&s_mode != kSchedStatic) sched_exit(prm.sched);
}

// The same with the decode step's cache write (each sequence's newest token written by
// the producer before its page is loaded); partitions are merged by
// paged_decode_reduce_kernel.
template <typename T, int D, int BS>
__global__ void __launch_bounds__(kDecodeThreads, 2)
paged_decode_partition_write_kernel(const __grid_constant__ CUtensorMap tmap_k,
                                    const __grid_constant__ CUtensorMap tmap_v,
                                    const __grid_constant__ CUtensorMap tmap_q, DecodeParams prm) {
    __shared__ int s_mode;
    DecodeSmem<D> sm(aligned_dynamic_smem(), prm.group);
    sm.init_barriers();
    pdl_wait_and_release();
    const int mode = sched_mode(prm, true, &s_mode);    // a step workspace starts zero-filled
    decode_items<T, D, BS, true>(&tmap_k, &tmap_v, &tmap_q, prm, sm, mode == kSchedDynamic);
    // reread: nothing held across the loop
    if (*(volatile int *)&s_mode != kSchedStatic) sched_exit(prm.sched);
}

// Log-sum-exp merge of n partials (m_j in log2 units, l_j, normalised o_j) of one
// (sequence, query head), by one warp: lane k owns output dims k*D/32 .. (k+1)*D/32-1.
//   M = max m_j;  w_j = l_j 2^(m_j - M);  out = sum_j w_j o_j / sum_j w_j
// Partial j's (m, l) is at ml[j * ml_stride], its output row at o + j * o_stride.
template <typename T, int D>
__device__ __forceinline__ void warp_merge(const float2 *ml, size_t ml_stride, const float *o,
                                           size_t o_stride, int n, T *out, int lane) {
    constexpr int V = D / 32;   // dims per lane (4 or 2)
    float M = -INFINITY;
    for (int j = lane; j < n; j += 32) M = fmaxf(M, ml[(size_t)j * ml_stride].x);
#pragma unroll
    for (int x = 16; x > 0; x >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, x));
    float L = 0.f;
    if (M != -INFINITY)
        for (int j = lane; j < n; j += 32) {
            const float2 v = ml[(size_t)j * ml_stride];
            L += v.y * ex2(v.x - M);
        }
#pragma unroll
    for (int x = 16; x > 0; x >>= 1) L += __shfl_xor_sync(0xffffffffu, L, x);
    float acc[V];
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = 0.f;
    if (L > 0.f) {
        const float inv = 1.f / L;
        for (int j0 = 0; j0 < n; j0 += 32) {
            float wmine = 0.f;
            if (j0 + lane < n) {
                const float2 v = ml[(size_t)(j0 + lane) * ml_stride];
                wmine = v.y * ex2(v.x - M) * inv;
            }
            const int cnt = min(32, n - j0);
#pragma unroll 4
            for (int k = 0; k < cnt; ++k) {
                const float wj = __shfl_sync(0xffffffffu, wmine, k);
                const float *row = o + (size_t)(j0 + k) * o_stride + lane * V;
                if (V == 4) {
                    const float4 x = *reinterpret_cast<const float4 *>(row);
                    acc[0] += wj * x.x; acc[1] += wj * x.y; acc[2] += wj * x.z; acc[3] += wj * x.w;
                } else {
                    const float2 x = *reinterpret_cast<const float2 *>(row);
                    acc[0] += wj * x.x; acc[1] += wj * x.y;
                }
            }
        }
    }
#pragma unroll
    for (int i = 0; i < V; ++i) out[lane * V + i] = from_float<T>(acc[i]);
}

constexpr int kReduceWarps = 8;

// Merge of a sequence's partitions for one query head; one warp per (sequence,
// query head) pair, pairs of single-partition sequences skipped. Block 0 re-arms the
// work counter of the workspace for the next decode.
template <typename T, int D>
__global__ void __launch_bounds__(kReduceWarps * 32)
paged_decode_reduce_kernel(DecodeParams prm) {
    pdl_wait_and_release();
    if (blockIdx.x == 0 && threadIdx.x == 0 && prm.sched) {
        // every decode CTA has finished (stream order): re-arm the scheduler, and clear
        // the step kernel's counters so that a workspace a plain decode used is also a
        // valid step workspace
        prm.sched->next = 0;
        prm.sched->arrive = 0;
        prm.sched->exit = 0;
        __threadfence();
        prm.sched->armed = kSchedArmed;
    }
    const int lane = threadIdx.x & 31;
    const int pair = blockIdx.x * kReduceWarps + (threadIdx.x >> 5);
    if (pair >= prm.num_seqs * prm.num_heads) return;
    const int s = pair / prm.num_heads;
    const int h = pair - s * prm.num_heads;
    int len = prm.context_lens[s];
    len = len < 0 ? 0 : (len > prm.max_context_len ? prm.max_context_len : len);
    const int P = prm.partition;
    const int np = max(1, (len + P - 1) / P);
    if (np == 1) return;
    const int G = prm.group;
    const int hk = h / G, g = h - hk * G;
    const size_t row0 = (size_t)(prm.ws_seq_base[s] + hk * np) * G + g;   // partition 0
    warp_merge<T, D>(reinterpret_cast<const float2 *>(prm.ws_ml) + row0, G,
                     prm.ws_o + row0 * D, (size_t)G * D, np,
                     reinterpret_cast<T *>(prm.out) + ((size_t)s * prm.num_heads + h) * D, lane);
}

}  // namespace pkv
