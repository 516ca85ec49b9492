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
// (then KV head, then partition); persistent CTAs take items blockIdx.x,
// blockIdx.x + gridDim.x, ... A sequence with one partition writes `out` directly;
// otherwise each item leaves (max, sum, normalised partial output) in fp32 scratch
// and paged_decode_reduce merges them exactly (log-sum-exp).
//
// Inside a CTA (160 threads): warp 4 is the producer. It walks the item list, reads
// each item's block-table slice into registers (one coalesced load per lane), and
// for every 64-token stage issues TMA tile loads of the K and V pages into a ring of
// shared-memory stages (128-byte swizzle), completing on a per-stage mbarrier.
// Warps 0-3 are consumers: each takes 16 of the stage's 64 tokens, computes the
// scores for the whole GQA group with m16n8k16 tensor-core MMAs (query heads on M,
// padded to 16; tokens on N; head_dim on K), keeps an online max / sum in fp32,
// and accumulates P.V with a second MMA (P kept in registers as the A operand).
// At the end of an item the four warps merge their partial softmax states through
// shared memory. Masking is by selection: scores of tokens at or past len_s become
// -inf and their V rows are zeroed in registers, so stale bits (NaN) never reach
// the result.
#pragma once

#include "pkv_ptx.cuh"

namespace pkv {

constexpr int kStageTokens = 64;
constexpr int kConsumerWarps = 4;
constexpr int kDecodeThreads = (kConsumerWarps + 1) * 32;
constexpr int kMaxGroup = 16;               // query heads per KV head (MMA M)
constexpr int kMaxItemBlocks = 128;         // block-table entries held per item (4 per lane)
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

struct DecodeParams {
    void *out;
    const void *q;
    const int32_t *block_tables;
    const int32_t *context_lens;
    float *ws_o;         // [items * G][D]
    float *ws_ml;        // [items * G][2]  (max in log2 units, sum)
    int32_t *ws_seq_base;// [B] first item of each sequence
    unsigned *status;
    int num_seqs, num_heads, num_kv_heads, group;
    int max_blocks_per_seq, num_blocks, max_context_len, partition;
    float scale_log2;    // scale * log2(e)
};

template <int D>
struct DecodeLayout {
    static constexpr int kHalves = D / 64;                     // 128-byte column slabs
    static constexpr int kSlabBytes = kStageTokens * 128;      // one slab of 64 tokens
    static constexpr int kKBytes = kHalves * kSlabBytes;
    static constexpr int kStageBytes = 2 * kKBytes;            // K + V
    static constexpr int kStages = D == 128 ? 4 : 8;
    static constexpr int kRingBytes = kStages * kStageBytes;
    static constexpr int kObufStride = D + 8;                  // floats per merge row
    static constexpr int kMetaBytes = 1024;                    // infos + barriers + ml
    static constexpr size_t smem_bytes(int group) {
        return 1024 /*alignment slack*/ + kRingBytes + kMetaBytes +
               (size_t)kConsumerWarps * group * kObufStride * sizeof(float);
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

template <typename T, int D, int BS>
__global__ void __launch_bounds__(kDecodeThreads, 1)
paged_decode_partition_kernel(const __grid_constant__ CUtensorMap tmap_k,
                              const __grid_constant__ CUtensorMap tmap_v, DecodeParams prm) {
    using L = DecodeLayout<D>;
    constexpr int kBPS = kStageTokens / BS;   // blocks per stage
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ring = smem;
    StageInfo *info = reinterpret_cast<StageInfo *>(smem + L::kRingBytes);
    uint64_t *full = reinterpret_cast<uint64_t *>(info + L::kStages);
    uint64_t *empty = full + L::kStages;
    float2 *ml = reinterpret_cast<float2 *>(empty + L::kStages);            // [4][16]
    float *obuf = reinterpret_cast<float *>(smem + L::kRingBytes + L::kMetaBytes);

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
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&tmap_k);
            prefetch_tensormap(&tmap_v);
        }
        const uint64_t policy = l2_evict_first_policy();
        const int B = prm.num_seqs;
        int it = 0;
        bool ok = true;
        // cursor over chunks of 32 sequences
        int cs = 0, chunk_base = 0, chunk_total = 0, incl = 0, my_items = 0, my_np = 0,
            my_len = 0;
        bool loaded = false;
        for (int item = blockIdx.x; ok; item += gridDim.x) {
            bool done = false;
            for (;;) {
                if (cs >= B) { done = true; break; }
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
            if (done) break;
            const unsigned hit = __ballot_sync(0xffffffffu, item < chunk_base + incl);
            const int ln = __ffs(hit) - 1;
            const int s = cs + ln;
            const int excl = __shfl_sync(0xffffffffu, incl - my_items, ln);
            const int np = __shfl_sync(0xffffffffu, my_np, ln);
            const int len = __shfl_sync(0xffffffffu, my_len, ln);
            const int r = item - chunk_base - excl;
            const int hk = r / np;
            const int p = r - hk * np;
            const int tok0 = p * P;
            const int ntok = max(0, min(P, len - tok0));
            const int nst = max(1, (ntok + kStageTokens - 1) / kStageTokens);
            const int nblk = (ntok + BS - 1) / BS;
            if (hk == 0 && p == 0 && lane == 0 && prm.ws_seq_base) prm.ws_seq_base[s] = item;
            // this item's slice of the block table: entry e lives in lane e%32, reg e/32
            int ent[kMaxItemBlocks / 32];
            const int32_t *bt = prm.block_tables + (size_t)s * prm.max_blocks_per_seq + tok0 / BS;
#pragma unroll
            for (int k = 0; k < kMaxItemBlocks / 32; ++k) {
                const int e = k * 32 + lane;
                ent[k] = e < nblk ? bt[e] : 0;
            }
            for (int st = 0; st < nst; ++st, ++it) {
                const int slot = it % L::kStages;
                const uint32_t ph = ((it / L::kStages) & 1) ^ 1;
                if (!warp_wait(smem_u32(&empty[slot]), ph)) {
                    if (lane == 0) atomicOr(prm.status, kStatusTimeout);
                    ok = false;
                    break;
                }
                const int sntok = max(0, min(kStageTokens, ntok - st * kStageTokens));
                const int nb_st = (sntok + BS - 1) / BS;
                const int e0 = st * kBPS;
                const int reg = e0 >> 5;
                int v = ent[0];
#pragma unroll
                for (int k = 1; k < kMaxItemBlocks / 32; ++k)
                    if (reg == k) v = ent[k];
                const int bid = __shfl_sync(0xffffffffu, v, (e0 + lane) & 31);
                if (lane == 0) {
                    StageInfo in;
                    in.s = s; in.hk = hk; in.p = p; in.npart = np; in.item = item;
                    in.ntok = sntok;
                    in.flags = (st == 0 ? kFirst : 0) | (st == nst - 1 ? kLast : 0);
                    in.pad = 0;
                    info[slot] = in;
                    mbar_arrive_expect_tx(smem_u32(&full[slot]),
                                          (uint32_t)(nb_st * BS * D * 2 * 2));
                }
                __syncwarp();
                if (lane < nb_st) {
                    int y;
                    if (bid >= 0 && bid < prm.num_blocks) {
                        y = (bid * Hkv + hk) * BS;
                    } else {
                        atomicOr(prm.status, kStatusBadBlock);
                        y = prm.num_blocks * Hkv * BS;   // fully out of range: reads zeros
                    }
                    uint8_t *stage = ring + slot * L::kStageBytes;
                    const uint32_t bar = smem_u32(&full[slot]);
#pragma unroll
                    for (int hf = 0; hf < L::kHalves; ++hf) {
                        const uint32_t off = hf * L::kSlabBytes + lane * BS * 128;
                        tma_load_2d(smem_u32(stage + off), &tmap_k, hf * 64, y, bar, policy);
                        tma_load_2d(smem_u32(stage + L::kKBytes + off), &tmap_v, hf * 64, y, bar,
                                    policy);
                    }
                }
            }
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
            // leave only after every tile load this warp issued has landed
            for (int j = max(0, it - L::kStages); j < it; ++j)
                warp_wait(smem_u32(&full[j % L::kStages]), (j / L::kStages) & 1);
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int w = warp;
    const int gid = lane >> 2;
    const int tig = lane & 3;
    constexpr int KS = D / 16;   // k-steps of QK
    constexpr int NT = D / 8;    // n-tiles of PV
    uint32_t qa[KS][4];
    float o[NT][4];
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    const T *qbase = reinterpret_cast<const T *>(prm.q);

    for (int it = 0;; ++it) {
        const int slot = it % L::kStages;
        if (!warp_wait(smem_u32(&full[slot]), (it / L::kStages) & 1)) {
            if (lane == 0) atomicOr(prm.status, kStatusTimeout);
            break;
        }
        const StageInfo in = info[slot];
        if (in.flags & kEnd) break;

        if (in.flags & kFirst) {
            const T *qs = qbase + ((size_t)in.s * prm.num_heads + (size_t)in.hk * G) * D;
            const bool r0 = gid < G, r1 = gid + 8 < G;
            const uint32_t *q0 = reinterpret_cast<const uint32_t *>(qs + gid * D);
            const uint32_t *q1 = reinterpret_cast<const uint32_t *>(qs + (gid + 8) * D);
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                const int c = ks * 8 + tig;   // 32-bit word index of dims 16ks + 2tig
                qa[ks][0] = r0 ? __ldg(q0 + c) : 0u;
                qa[ks][1] = r1 ? __ldg(q1 + c) : 0u;
                qa[ks][2] = r0 ? __ldg(q0 + c + 4) : 0u;
                qa[ks][3] = r1 ? __ldg(q1 + c + 4) : 0u;
            }
#pragma unroll
            for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
            m0 = m1 = -INFINITY;
            l0 = l1 = 0.f;
        }

        const int valid = in.ntok - 16 * w;   // tokens of my 16-token slice in the sequence
        if (valid > 0) {
            const uint8_t *stage = ring + slot * L::kStageBytes;
            const uint32_t kbase = smem_u32(stage);
            const uint32_t vbase = smem_u32(stage + L::kKBytes);
            // ---- S = Q K^T for tokens 16w .. 16w+15 (two n-tiles of 8)
            float sc[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
                const int t = 16 * w + 8 * nt + (lane & 7);
                const int mi = lane >> 3;
#pragma unroll
                for (int hf = 0; hf < L::kHalves; ++hf) {
#pragma unroll
                    for (int c2 = 0; c2 < 2; ++c2) {
                        const int c = c2 * 4 + mi;
                        const uint32_t addr =
                            kbase + hf * L::kSlabBytes + t * 128 + ((c ^ (t & 7)) << 4);
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4(addr, b0, b1, b2, b3);
                        const int ks = hf * 4 + c2 * 2;
                        Mma<T>::run(sc[nt], qa[ks], b0, b1);
                        Mma<T>::run(sc[nt], qa[ks + 1], b2, b3);
                    }
                }
            }
            // ---- scale, mask, online softmax (rows gid and gid+8)
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const bool in_seq = 8 * nt + 2 * tig + e < valid;
                    sc[nt][e] = in_seq ? sc[nt][e] * prm.scale_log2 : -INFINITY;
                    sc[nt][2 + e] = in_seq ? sc[nt][2 + e] * prm.scale_log2 : -INFINITY;
                    mx0 = fmaxf(mx0, sc[nt][e]);
                    mx1 = fmaxf(mx1, sc[nt][2 + e]);
                }
            }
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
            const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
            const float a0 = ex2(m0 - mn0), a1 = ex2(m1 - mn1);
            m0 = mn0;
            m1 = mn1;
            float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    sc[nt][e] = ex2(sc[nt][e] - mn0);
                    sc[nt][2 + e] = ex2(sc[nt][2 + e] - mn1);
                    ps0 += sc[nt][e];
                    ps1 += sc[nt][2 + e];
                }
            }
            l0 = l0 * a0 + ps0;
            l1 = l1 * a1 + ps1;
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                o[n][0] *= a0; o[n][1] *= a0;
                o[n][2] *= a1; o[n][3] *= a1;
            }
            uint32_t pa[4];
            pa[0] = Mma<T>::pack(sc[0][0], sc[0][1]);
            pa[1] = Mma<T>::pack(sc[0][2], sc[0][3]);
            pa[2] = Mma<T>::pack(sc[1][0], sc[1][1]);
            pa[3] = Mma<T>::pack(sc[1][2], sc[1][3]);
            // ---- O += P V  (V rows of tokens past the sequence are zeroed)
            uint32_t keep_lo = 0xffffffffu, keep_hi = 0xffffffffu;
            if (valid < 16) {
                const int t0 = 2 * tig, t1 = 2 * tig + 8;
                keep_lo = (t0 < valid ? 0x0000ffffu : 0u) | (t0 + 1 < valid ? 0xffff0000u : 0u);
                keep_hi = (t1 < valid ? 0x0000ffffu : 0u) | (t1 + 1 < valid ? 0xffff0000u : 0u);
            }
            const int mi = lane >> 3;
            const int tv = 16 * w + (mi & 1) * 8 + (lane & 7);
#pragma unroll
            for (int dp = 0; dp < D / 16; ++dp) {
                const int hf = dp >> 2;
                const int c = 2 * (dp & 3) + (mi >> 1);
                const uint32_t addr =
                    vbase + hf * L::kSlabBytes + tv * 128 + ((c ^ (tv & 7)) << 4);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_trans(addr, b0, b1, b2, b3);
                b0 &= keep_lo; b1 &= keep_hi; b2 &= keep_lo; b3 &= keep_hi;
                Mma<T>::run(o[2 * dp], pa, b0, b1);
                Mma<T>::run(o[2 * dp + 1], pa, b2, b3);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[slot]));

        if (in.flags & kLast) {
            // ---- merge the four warps' softmax states, then write
            float lt0 = l0 + __shfl_xor_sync(0xffffffffu, l0, 1);
            lt0 += __shfl_xor_sync(0xffffffffu, lt0, 2);
            float lt1 = l1 + __shfl_xor_sync(0xffffffffu, l1, 1);
            lt1 += __shfl_xor_sync(0xffffffffu, lt1, 2);
            named_bar_sync(1, kConsumerWarps * 32);
            if (tig == 0) {
                ml[w * kMaxGroup + gid] = make_float2(m0, lt0);
                ml[w * kMaxGroup + gid + 8] = make_float2(m1, lt1);
            }
            named_bar_sync(1, kConsumerWarps * 32);
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const int row = gid + 8 * rr;
                if (row < G) {
                    float M = -INFINITY;
#pragma unroll
                    for (int ww = 0; ww < kConsumerWarps; ++ww)
                        M = fmaxf(M, ml[ww * kMaxGroup + row].x);
                    float Lsum = 0.f;
                    if (M != -INFINITY) {
#pragma unroll
                        for (int ww = 0; ww < kConsumerWarps; ++ww) {
                            const float2 v = ml[ww * kMaxGroup + row];
                            Lsum += v.y * ex2(v.x - M);
                        }
                    }
                    const float mself = rr ? m1 : m0;
                    const float f = (Lsum > 0.f) ? ex2(mself - M) / Lsum : 0.f;
                    float *dst = obuf + ((size_t)w * G + row) * L::kObufStride + 2 * tig;
#pragma unroll
                    for (int n = 0; n < NT; ++n)
                        *reinterpret_cast<float2 *>(dst + n * 8) =
                            make_float2(o[n][2 * rr] * f, o[n][2 * rr + 1] * f);
                }
            }
            named_bar_sync(1, kConsumerWarps * 32);
            const int tid = threadIdx.x;   // 0..127
            if (in.npart == 1) {
                T *out = reinterpret_cast<T *>(prm.out) +
                         ((size_t)in.s * prm.num_heads + (size_t)in.hk * G) * D;
                for (int idx = tid; idx < G * D; idx += kConsumerWarps * 32) {
                    const int row = idx / D, dim = idx - row * D;
                    float acc = 0.f;
#pragma unroll
                    for (int ww = 0; ww < kConsumerWarps; ++ww)
                        acc += obuf[((size_t)ww * G + row) * L::kObufStride + dim];
                    out[idx] = from_float<T>(acc);
                }
            } else {
                float *dst = prm.ws_o + (size_t)in.item * G * D;
                for (int idx = tid; idx < G * D; idx += kConsumerWarps * 32) {
                    const int row = idx / D, dim = idx - row * D;
                    float acc = 0.f;
#pragma unroll
                    for (int ww = 0; ww < kConsumerWarps; ++ww)
                        acc += obuf[((size_t)ww * G + row) * L::kObufStride + dim];
                    dst[idx] = acc;
                }
                if (tid < G) {
                    float M = -INFINITY;
                    for (int ww = 0; ww < kConsumerWarps; ++ww)
                        M = fmaxf(M, ml[ww * kMaxGroup + tid].x);
                    float Lsum = 0.f;
                    if (M != -INFINITY)
                        for (int ww = 0; ww < kConsumerWarps; ++ww) {
                            const float2 v = ml[ww * kMaxGroup + tid];
                            Lsum += v.y * ex2(v.x - M);
                        }
                    reinterpret_cast<float2 *>(prm.ws_ml)[(size_t)in.item * G + tid] =
                        make_float2(M, Lsum);
                }
            }
        }
    }
}

// Merge of a sequence's partitions for one query head (log-sum-exp):
//   M = max_p m_p;  w_p = l_p 2^(m_p - M);  out = sum_p w_p o_p / sum_p w_p
// (m_p in log2 units, o_p normalised). One CTA per (query head, sequence), D threads.
template <typename T, int D>
__global__ void __launch_bounds__(D)
paged_decode_reduce_kernel(DecodeParams prm) {
    const int h = blockIdx.x;
    const int s = blockIdx.y;
    int len = prm.context_lens[s];
    len = len < 0 ? 0 : (len > prm.max_context_len ? prm.max_context_len : len);
    const int P = prm.partition;
    const int np = max(1, (len + P - 1) / P);
    if (np == 1) return;
    const int G = prm.group;
    const int hk = h / G, g = h - hk * G;
    const int base = prm.ws_seq_base[s] + hk * np;
    extern __shared__ float wsm[];   // [np] weights
    __shared__ float red[D / 32];
    __shared__ float bcast;
    const float2 *mlp = reinterpret_cast<const float2 *>(prm.ws_ml);
    const int tid = threadIdx.x;

    float M = -INFINITY;
    for (int p = tid; p < np; p += D) M = fmaxf(M, mlp[(size_t)(base + p) * G + g].x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    if ((tid & 31) == 0) red[tid >> 5] = M;
    __syncthreads();
    if (tid == 0) {
        float v = red[0];
        for (int i = 1; i < D / 32; ++i) v = fmaxf(v, red[i]);
        bcast = v;
    }
    __syncthreads();
    M = bcast;
    float Ls = 0.f;
    for (int p = tid; p < np; p += D) {
        const float2 v = mlp[(size_t)(base + p) * G + g];
        const float wv = (M == -INFINITY) ? 0.f : v.y * ex2(v.x - M);
        wsm[p] = wv;
        Ls += wv;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, o);
    __syncthreads();
    if ((tid & 31) == 0) red[tid >> 5] = Ls;
    __syncthreads();
    if (tid == 0) {
        float v = 0.f;
        for (int i = 0; i < D / 32; ++i) v += red[i];
        bcast = v;
    }
    __syncthreads();
    Ls = bcast;
    const float *op = prm.ws_o + ((size_t)base * G + g) * D + tid;
    const size_t stride = (size_t)G * D;
    float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
    int p = 0;
    for (; p + 4 <= np; p += 4) {
        acc0 += wsm[p] * op[(size_t)p * stride];
        acc1 += wsm[p + 1] * op[(size_t)(p + 1) * stride];
        acc2 += wsm[p + 2] * op[(size_t)(p + 2) * stride];
        acc3 += wsm[p + 3] * op[(size_t)(p + 3) * stride];
    }
    for (; p < np; ++p) acc0 += wsm[p] * op[(size_t)p * stride];
    const float acc = (acc0 + acc1) + (acc2 + acc3);
    T *out = reinterpret_cast<T *>(prm.out) + ((size_t)s * prm.num_heads + h) * D;
    out[tid] = from_float<T>(Ls > 0.f ? acc / Ls : 0.f);
}

}  // namespace pkv
