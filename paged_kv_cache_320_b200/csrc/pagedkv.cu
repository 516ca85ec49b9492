// C-ABI entry points of libpagedkv.so (declared and documented in pagedkv.h):
// host-side argument checks, TMA descriptor encoding, launch configuration and the
// per-device status word. All device work is in decode_kernels.cuh and
// cache_kernels.cuh.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstring>
#include <atomic>
#include <mutex>
#include <utility>

#include "cache_kernels.cuh"
#include "decode_kernels.cuh"
#include "shared_prefix_kernels.cuh"
#include "step_kernels.cuh"
#include "pagedkv.h"

namespace {

// One status word per device (each device that loads the library gets its own copy).
__device__ unsigned int g_pkv_status;

constexpr int kMaxDevices = 64;

std::mutex g_mu;
unsigned int *g_status_ptr[kMaxDevices];
int g_sm_count[kMaxDevices];

int current_device(int *dev) {
    if (cudaGetDevice(dev) != cudaSuccess || *dev < 0 || *dev >= kMaxDevices) return PKV_ERR_CUDA;
    return PKV_OK;
}

int device_status_ptr(unsigned int **out) {
    int dev;
    if (current_device(&dev) != PKV_OK) return PKV_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_status_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_pkv_status) != cudaSuccess) return PKV_ERR_CUDA;
        g_status_ptr[dev] = static_cast<unsigned int *>(p);
    }
    *out = g_status_ptr[dev];
    return PKV_OK;
}

// Scratch of pkv_paged_attention_decode_noalloc: a fixed device array (one copy per
// device that loads the library). Host code must not pass the symbol itself to a
// kernel (on the host it only names the array); its device address is looked up
// once per device with cudaGetSymbolAddress.
constexpr size_t kNoAllocScratchBytes = PKV_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
// Per device: the library's copy stream and events of the staged swap (created on first
// use, kept until exit), and the lock that keeps one call's sequence of them whole.
struct SwapSide {
    bool ready = false;
    cudaStream_t cs = nullptr;
    cudaEvent_t start = nullptr, fill[2] = {nullptr, nullptr}, drain[2] = {nullptr, nullptr};
};
SwapSide g_swap_side[kMaxDevices];
std::mutex g_swap_mu;

void *g_noalloc_ptr[kMaxDevices];

int noalloc_scratch_ptr(void **out) {
    int dev;
    if (current_device(&dev) != PKV_OK) return PKV_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return PKV_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return PKV_OK;
}

int sm_count(int *out) {
    int dev;
    if (current_device(&dev) != PKV_OK) return PKV_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_sm_count[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            return PKV_ERR_CUDA;
        g_sm_count[dev] = n;
    }
    *out = g_sm_count[dev];
    return PKV_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link-time
// dependency on libcuda, so the library also loads on a machine without a GPU).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// View of one layer's cache for TMA: rows = num_blocks*Hkv*BS of head_dim elements.
// head_dim 128: 3-D (64 elements, rows, 2 halves of a row) with a box of one page tile
// (64 x BS x 2), landing half-major in shared memory; head_dim 64: 2-D (64, rows) with a
// box of 64 x BS. 128-byte swizzle.
int encode_rows_map(CUtensorMap *map, const void *base, int dtype, int D, long long rows,
                    int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return PKV_ERR_CUDA;
    const CUtensorMapDataType dt =
        dtype == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUresult r;
    if (D == 128) {
        const cuuint64_t dims[3] = {64, (cuuint64_t)rows, 2};
        const cuuint64_t strides[2] = {256, 128};
        const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 2};
        const cuuint32_t estr[3] = {1, 1, 1};
        r = fn(map, dt, 3, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    } else {
        const cuuint64_t dims[2] = {64, (cuuint64_t)rows};
        const cuuint64_t strides[1] = {128};
        const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
        const cuuint32_t estr[2] = {1, 1};
        r = fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    }
    return r == CUDA_SUCCESS ? PKV_OK : PKV_ERR_CUDA;
}

// Launch with programmatic stream serialization: the kernel may begin while the
// previous kernel of the stream finishes; every kernel of this library waits
// (griddepcontrol.wait) before touching global memory, so stream order is kept.
// Built with PKV_USE_PDL=0 the launches are ordinary.
#ifndef PKV_USE_PDL
#define PKV_USE_PDL 1
#endif
template <typename... KArgs, typename... Args>
int launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
           Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = PKV_USE_PDL;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) != cudaSuccess)
        return PKV_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int cdiv(int a, int b) { return (a + b - 1) / b; }

// Automatic partition size. One partition per context (no partials, no merge) when
// every context fits one work item (256 blocks), the batch is small enough for the
// longest-first item order (so the long items start first and the launch drains on
// short ones) and offers at least 1024 items. Otherwise 512 tokens for GQA groups up to 4
// and 2048 above (the fp32 partials grow with the group; measured best at the GQA-4 and
// GQA-8 workloads), at most 256 blocks, halved while the batch offers fewer than 1024
// work items (about 7 per CTA on 148 SMs).
int auto_partition(int B, int Hq, int Hkv, int BS, int max_len) {
    const int G = Hq / Hkv;
    if (max_len <= pkv::kMaxItemBlocks * BS && B <= pkv::kOrderMaxSeqs &&
        (long long)B * Hkv >= 1024)
        return std::max(pkv::kStageTokens, cdiv(max_len, pkv::kStageTokens) * pkv::kStageTokens);
    int p = G <= 4 ? 512 : 2048;
    if (p > pkv::kMaxItemBlocks * BS) p = pkv::kMaxItemBlocks * BS;
    while (p > 64 && (long long)B * Hkv * cdiv(max_len, p) < 1024) p /= 2;
    return p;
}

// Automatic partition size of the shared-prefix decode: 2048 tokens (same block and
// batch limits as the plain decode's). An item carries up to 16 query rows and, where
// they fit in one partition's stages, a chunk's last prefix partition and its members'
// first suffix partition together, which then need no merge.
int auto_shared_partition(int B, int Hq, int Hkv, int BS, int max_len) {
    (void)Hq;
    int p = 2048;
    if (p > pkv::kMaxItemBlocks * BS) p = pkv::kMaxItemBlocks * BS;
    while (p > 64 && (long long)B * Hkv * cdiv(max_len, p) < 1024) p /= 2;
    return p;
}

int check_decode_sizes(int B, int Hq, int Hkv, int D, int BS, int max_len, int partition,
                       int *P_out, bool shared = false) {
    if (B < 0 || Hkv < 1 || Hq < 1 || Hq % Hkv != 0 || Hq / Hkv > pkv::kMaxGroup)
        return PKV_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return PKV_ERR_INVALID_ARG;
    if (BS != 8 && BS != 16 && BS != 32) return PKV_ERR_INVALID_ARG;
    if (max_len < 0) return PKV_ERR_INVALID_ARG;
    int P = partition;
    if (P == 0)
        P = shared ? auto_shared_partition(B, Hq, Hkv, BS, max_len)
                   : auto_partition(B, Hq, Hkv, BS, max_len);
    if (P <= 0 || P % pkv::kStageTokens != 0 || P > pkv::kMaxItemBlocks * BS)
        return PKV_ERR_INVALID_ARG;
    const long long pmax = max_len <= P ? 1 : cdiv(max_len, P);
    if ((long long)B * Hkv * pmax >= INT_MAX) return PKV_ERR_INVALID_ARG;
    if ((long long)B * Hq >= INT_MAX) return PKV_ERR_INVALID_ARG;   // (sequence, head) pairs
    *P_out = P;
    return PKV_OK;
}

// Workspace: [scheduler header 256 B][first item of each sequence][partials (max,
// sum)][partial outputs]. Only needed when some context spans several partitions.
struct WsLayout {
    size_t seq_base, ml, o, total;
};

WsLayout ws_layout(int B, int Hq, int D, int max_len, int P) {
    WsLayout w{0, 0, 0, 0};
    const long long pmax = max_len <= P ? 1 : cdiv(max_len, P);
    if (pmax <= 1 || B == 0) return w;
    const size_t rows = (size_t)B * Hq * pmax;
    w.seq_base = sizeof(pkv::SchedHeader);
    w.ml = w.seq_base + align_up((size_t)B * sizeof(int32_t), 256);
    w.o = w.ml + align_up(rows * 2 * sizeof(float), 256);
    w.total = w.o + rows * D * sizeof(float);
    return w;
}

template <typename T, int D, int BS, bool kWrite = false>
int launch_decode(const CUtensorMap &mk, const CUtensorMap &mv, const CUtensorMap &mq,
                  const pkv::DecodeParams &prm, long long items_upper, cudaStream_t st) {
    using L = pkv::DecodeLayout<D>;
    auto kern = kWrite ? pkv::paged_decode_partition_write_kernel<T, D, BS>
                       : pkv::paged_decode_partition_kernel<T, D, BS>;
    const size_t smem = L::smem_bytes(prm.group);
    int dev;
    if (current_device(&dev) != PKV_OK) return PKV_ERR_CUDA;
    // blocks per SM, cached per device and group size (read without the lock)
    static std::atomic<int> occ[kMaxDevices][pkv::kMaxGroup + 1];
    static bool attr_set[kMaxDevices];
    int nsm;
    if (sm_count(&nsm) != PKV_OK) return PKV_ERR_CUDA;
    std::atomic<int> &o = occ[dev][prm.group];
    int per_sm = o.load(std::memory_order_acquire);
    if (per_sm == 0) {
        std::lock_guard<std::mutex> lk(g_mu);
        // the largest layout any group size needs, so every later launch fits
        if (!attr_set[dev]) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)L::smem_bytes(pkv::kMaxGroup)) != cudaSuccess)
                return PKV_ERR_CUDA;
            attr_set[dev] = true;
        }
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, pkv::kDecodeThreads, smem) !=
                cudaSuccess ||
            n <= 0)
            return PKV_ERR_CUDA;
        o.store(n, std::memory_order_release);
        per_sm = n;
    }
    long long grid = (long long)nsm * per_sm;
    if (grid > items_upper) grid = items_upper;
    if (grid < 1) grid = 1;
    return launch(kern, dim3((unsigned)grid), dim3(pkv::kDecodeThreads), smem, st, mk, mv, mq, prm);
}

template <typename T, int D>
int launch_reduce(const pkv::DecodeParams &prm, cudaStream_t st) {
    const long long pairs = (long long)prm.num_seqs * prm.num_heads;
    const long long grid = (pairs + pkv::kReduceWarps - 1) / pkv::kReduceWarps;
    return launch(pkv::paged_decode_reduce_kernel<T, D>, dim3((unsigned)grid),
                  dim3(pkv::kReduceWarps * 32), 0, st, prm);
}

template <typename T, int D>
int dispatch_bs(int BS, const CUtensorMap &mk, const CUtensorMap &mv, const CUtensorMap &mq,
                const pkv::DecodeParams &prm, long long items, cudaStream_t st) {
    switch (BS) {
        case 8: return launch_decode<T, D, 8>(mk, mv, mq, prm, items, st);
        case 16: return launch_decode<T, D, 16>(mk, mv, mq, prm, items, st);
        case 32: return launch_decode<T, D, 32>(mk, mv, mq, prm, items, st);
    }
    return PKV_ERR_INVALID_ARG;
}

// ---- shared-prefix decode ------------------------------------------------
// Workspace: [counters 256 B][np, row_base, seq_group, gpre, gmin, gmis, ioff: B ints each]
// [items][partials (max, sum)][partial outputs].
struct SharedWs {
    size_t ints, items, ml, o, total;
    int max_items;
    long long rows;
};

SharedWs shared_ws_layout(int B, int Hq, int Hkv, int D, int max_len, int P) {
    SharedWs w{};
    const long long pmax = max_len <= P ? 1 : cdiv(max_len, P);
    w.max_items = (int)std::min<long long>(2LL * Hkv * B * pmax, INT_MAX / 2);
    w.rows = (long long)B * Hq * (pmax + 1);
    w.ints = sizeof(pkv::SharedCounters);
    w.items = w.ints + 7 * align_up((size_t)B * sizeof(int), 256);
    w.ml = w.items + align_up((size_t)w.max_items * sizeof(pkv::SharedItem), 256);
    w.o = w.ml + align_up((size_t)w.rows * 2 * sizeof(float), 256);
    w.total = w.o + (size_t)w.rows * D * sizeof(float);
    return w;
}

template <typename T, int D, int BS>
int launch_shared_decode(const CUtensorMap &mk, const CUtensorMap &mv,
                         const pkv::SharedParams &prm, cudaStream_t st) {
    using L = pkv::DecodeLayout<D>;
    auto kern = pkv::paged_decode_shared_kernel<T, D, BS>;
    const size_t smem = 1024 + L::kRingBytes + L::obuf_bytes(pkv::kMaxGroup) + L::kMetaBytes;
    int dev;
    if (current_device(&dev) != PKV_OK) return PKV_ERR_CUDA;
    static std::atomic<int> occ[kMaxDevices];   // blocks per SM (read without the lock)
    int nsm;
    if (sm_count(&nsm) != PKV_OK) return PKV_ERR_CUDA;
    int per_sm = occ[dev].load(std::memory_order_acquire);
    if (per_sm == 0) {
        std::lock_guard<std::mutex> lk(g_mu);
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return PKV_ERR_CUDA;
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, pkv::kDecodeThreads, smem) !=
                cudaSuccess ||
            n <= 0)
            return PKV_ERR_CUDA;
        occ[dev].store(n, std::memory_order_release);
        per_sm = n;
    }
    long long grid = (long long)nsm * per_sm;
    if (grid > prm.max_items) grid = prm.max_items;
    if (grid < 1) grid = 1;
    return launch(kern, dim3((unsigned)grid), dim3(pkv::kDecodeThreads), smem, st, mk, mv, prm);
}

// CTAs per SM of the shared-prefix decode launch (its shared memory against the SM's;
// launch bounds allow two), for the plan's item placement.
int shared_decode_slots(int D, int *slots) {
    int dev;
    if (current_device(&dev) != PKV_OK) return PKV_ERR_CUDA;
    int cap = 0;
    if (cudaDeviceGetAttribute(&cap, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) !=
        cudaSuccess)
        return PKV_ERR_CUDA;
    const size_t smem =
        D == 128 ? 1024 + pkv::DecodeLayout<128>::kRingBytes +
                       pkv::DecodeLayout<128>::obuf_bytes(pkv::kMaxGroup) +
                       pkv::DecodeLayout<128>::kMetaBytes
                 : 1024 + pkv::DecodeLayout<64>::kRingBytes +
                       pkv::DecodeLayout<64>::obuf_bytes(pkv::kMaxGroup) +
                       pkv::DecodeLayout<64>::kMetaBytes;
    *slots = (int)std::min<size_t>(2, (size_t)cap / (smem + 1024));
    return PKV_OK;
}

int launch_shared_plan(const pkv::SharedParams &prm, cudaStream_t st) {
    const size_t plan_smem =
        prm.num_seqs <= pkv::kPlanSmemSeqs ? (size_t)7 * prm.num_seqs * sizeof(int) : 0;
    {
        int dev;
        if (current_device(&dev) != PKV_OK) return PKV_ERR_CUDA;
        static bool attr[kMaxDevices];
        std::lock_guard<std::mutex> lk(g_mu);
        if (!attr[dev]) {
            if (cudaFuncSetAttribute(pkv::shared_prefix_plan_kernel,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     7 * pkv::kPlanSmemSeqs * (int)sizeof(int)) != cudaSuccess)
                return PKV_ERR_CUDA;
            attr[dev] = true;
        }
    }
    return launch(pkv::shared_prefix_plan_kernel, dim3(1), dim3(pkv::kPlanThreads), plan_smem,
                  st, prm);
}

template <typename T, int D>
int launch_shared_decode_reduce(int BS, const CUtensorMap &mk, const CUtensorMap &mv,
                                const pkv::SharedParams &prm, cudaStream_t st) {
    int rc;
    switch (BS) {
        case 8: rc = launch_shared_decode<T, D, 8>(mk, mv, prm, st); break;
        case 16: rc = launch_shared_decode<T, D, 16>(mk, mv, prm, st); break;
        case 32: rc = launch_shared_decode<T, D, 32>(mk, mv, prm, st); break;
        default: return PKV_ERR_INVALID_ARG;
    }
    if (rc != PKV_OK) return rc;
    const long long pairs = (long long)prm.num_seqs * prm.num_heads;
    const long long grid = (pairs + pkv::kReduceWarps - 1) / pkv::kReduceWarps;
    return launch(pkv::paged_decode_shared_reduce_kernel<T, D>, dim3((unsigned)grid),
                  dim3(pkv::kReduceWarps * 32), 0, st, prm);
}

// Workspace pointers and sizes of the shared-prefix path (no output, query or scale).
pkv::SharedParams shared_params(const SharedWs &ws, void *workspace, int num_seqs, int num_heads,
                                int num_kv_heads, int block_size, int max_blocks_per_seq,
                                int num_blocks, int max_context_len, int P,
                                const int32_t *block_tables, const int32_t *context_lens,
                                unsigned *status) {
    uint8_t *wsb = static_cast<uint8_t *>(workspace);
    const size_t ib = align_up((size_t)num_seqs * sizeof(int), 256);
    pkv::SharedParams prm{};
    prm.counters = reinterpret_cast<pkv::SharedCounters *>(wsb);
    prm.np = reinterpret_cast<int *>(wsb + ws.ints);
    prm.row_base = reinterpret_cast<int *>(wsb + ws.ints + ib);
    prm.seq_group = reinterpret_cast<int *>(wsb + ws.ints + 2 * ib);
    prm.gpre = reinterpret_cast<int *>(wsb + ws.ints + 3 * ib);
    prm.gmin = reinterpret_cast<int *>(wsb + ws.ints + 4 * ib);
    prm.gmis = reinterpret_cast<int *>(wsb + ws.ints + 5 * ib);
    prm.ioff = reinterpret_cast<int *>(wsb + ws.ints + 6 * ib);
    prm.items = reinterpret_cast<pkv::SharedItem *>(wsb + ws.items);
    prm.ws_ml = reinterpret_cast<float *>(wsb + ws.ml);
    prm.ws_o = reinterpret_cast<float *>(wsb + ws.o);
    prm.block_tables = block_tables;
    prm.context_lens = context_lens;
    prm.status = status;
    prm.num_seqs = num_seqs;
    prm.num_heads = num_heads;
    prm.num_kv_heads = num_kv_heads;
    prm.group = num_heads / num_kv_heads;
    prm.max_blocks_per_seq = max_blocks_per_seq;
    prm.num_blocks = num_blocks;
    prm.max_context_len = max_context_len;
    prm.partition = P;
    prm.block_size = block_size;
    prm.max_items = ws.max_items;
    return prm;
}

// ---- fused decode step -----------------------------------------------------
// Workspace: the decode workspace when some context spans several partitions,
// else the 256-byte header alone (dynamic schedule).
size_t step_ws_bytes(int B, int Hq, int D, int max_len, int P) {
    const size_t t = ws_layout(B, Hq, D, max_len, P).total;
    return t ? t : sizeof(pkv::StepHeader);
}

template <typename T, int D, int BS>
int launch_step(const CUtensorMap &mk, const CUtensorMap &mv, const CUtensorMap &mq,
                const pkv::DecodeParams &prm, long long items, int merge, cudaStream_t st) {
    using L = pkv::DecodeLayout<D>;
    auto kern = pkv::paged_decode_step_kernel<T, D, BS>;
    const size_t smem = L::smem_bytes(prm.group);
    int dev;
    if (current_device(&dev) != PKV_OK) return PKV_ERR_CUDA;
    // blocks per SM, cached per device and group size (read without the lock)
    static std::atomic<int> occ[kMaxDevices][pkv::kMaxGroup + 1];
    static bool attr_set[kMaxDevices];
    int nsm;
    if (sm_count(&nsm) != PKV_OK) return PKV_ERR_CUDA;
    std::atomic<int> &o = occ[dev][prm.group];
    int per_sm = o.load(std::memory_order_acquire);
    if (per_sm == 0) {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!attr_set[dev]) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)L::smem_bytes(pkv::kMaxGroup)) != cudaSuccess)
                return PKV_ERR_CUDA;
            attr_set[dev] = true;
        }
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, pkv::kDecodeThreads, smem) !=
                cudaSuccess ||
            n <= 0)
            return PKV_ERR_CUDA;
        o.store(n, std::memory_order_release);
        per_sm = n;
    }
    long long grid = (long long)nsm * per_sm;
    if (grid > items) grid = items;
    if (grid < 1) grid = 1;
    // the merge phase waits at a grid barrier: all CTAs must be resident at once
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(pkv::kDecodeThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = merge ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, mk, mv, mq, prm, merge) != cudaSuccess) return PKV_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

// Where a decode step with several partitions merges them: in the step launch (one
// cooperative launch; after a grid barrier every warp of the persistent grid merges
// pairs) when every (sequence, query head) pair gets a warp of its own, so the merge is
// one pass; otherwise in paged_decode_reduce_kernel after the write-and-decode kernel
// (two launches, both with programmatic dependent launch), which runs all pairs at once
// across the GPU. The grid is two CTAs of kDecodeThreads per SM (the launch bounds and
// shared-memory plan of the decode kernels), at most one per work item.
// Built with PKV_STEP_INKERNEL_MERGE=0 the reduce kernel is always used.
#ifndef PKV_STEP_INKERNEL_MERGE
#define PKV_STEP_INKERNEL_MERGE 1
#endif

int step_merges_in_kernel(int B, int Hq, long long items, int pmax, int nsm) {
    if (!PKV_STEP_INKERNEL_MERGE || pmax <= 1) return 0;
    const long long grid = std::min<long long>(2LL * nsm, items);
    return (long long)B * Hq <= grid * (pkv::kDecodeThreads / 32);
}

template <typename T, int D>
int dispatch_step(int BS, const CUtensorMap &mk, const CUtensorMap &mv, const CUtensorMap &mq,
                  const pkv::DecodeParams &prm, long long items, int merge, int in_kernel,
                  bool launch_merge, cudaStream_t st) {
    if (in_kernel) {
        switch (BS) {
            case 8: return launch_step<T, D, 8>(mk, mv, mq, prm, items, merge, st);
            case 16: return launch_step<T, D, 16>(mk, mv, mq, prm, items, merge, st);
            case 32: return launch_step<T, D, 32>(mk, mv, mq, prm, items, merge, st);
        }
        return PKV_ERR_INVALID_ARG;
    }
    // the header (zero-filled at first, then armed by the last CTA out of each launch)
    // holds the work counter whether or not the contexts span several partitions
    const pkv::DecodeParams &p = prm;
    int rc = PKV_ERR_INVALID_ARG;
    switch (BS) {
        case 8: rc = launch_decode<T, D, 8, true>(mk, mv, mq, p, items, st); break;
        case 16: rc = launch_decode<T, D, 16, true>(mk, mv, mq, p, items, st); break;
        case 32: rc = launch_decode<T, D, 32, true>(mk, mv, mq, p, items, st); break;
    }
    if (rc == PKV_OK && merge && launch_merge) rc = launch_reduce<T, D>(p, st);
    return rc;
}

}  // namespace

extern "C" {

const char *pkv_status_string(int code) {
    switch (code) {
        case PKV_OK: return "ok";
        case PKV_ERR_INVALID_ARG: return "invalid argument";
        case PKV_ERR_OUT_OF_BLOCKS: return "out of blocks";
        case PKV_ERR_UNKNOWN_SEQ: return "unknown sequence";
        case PKV_ERR_SEQ_EXISTS: return "sequence id already in use";
        case PKV_ERR_TABLE_FULL: return "block table full";
        case PKV_ERR_BAD_INDEX: return "out-of-pool index met on the device";
        case PKV_ERR_TIMEOUT: return "bounded device wait gave up";
        case PKV_ERR_CUDA: return "CUDA runtime error";
        case PKV_ERR_WORKSPACE: return "workspace missing or too small";
        case PKV_ERR_HOST_MEMORY: return "host allocation failed in the block manager";
    }
    return "unknown status";
}

int pkv_decode_partition_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                              int block_size, int max_context_len, int partition_size,
                              int *partition_out) {
    if (!partition_out) return PKV_ERR_INVALID_ARG;
    return check_decode_sizes(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                              max_context_len, partition_size, partition_out);
}

int pkv_decode_shared_prefix_partition_size(int num_seqs, int num_heads, int num_kv_heads,
                                            int head_dim, int block_size, int max_context_len,
                                            int partition_size, int *partition_out) {
    if (!partition_out) return PKV_ERR_INVALID_ARG;
    return check_decode_sizes(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                              max_context_len, partition_size, partition_out, true);
}

int pkv_decode_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                              int block_size, int max_context_len, int partition_size,
                              size_t *bytes_out) {
    if (!bytes_out) return PKV_ERR_INVALID_ARG;
    int P;
    const int rc = check_decode_sizes(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                      max_context_len, partition_size, &P);
    if (rc != PKV_OK) return rc;
    *bytes_out = ws_layout(num_seqs, num_heads, head_dim, max_context_len, P).total;
    return PKV_OK;
}

}  // extern "C"

namespace {

// pkv_paged_attention_decode (with_merge) or its partition launch alone.
int decode_impl(void *out, const void *q, const void *k_cache, const void *v_cache,
                const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                int num_heads, int num_kv_heads, int head_dim, int block_size,
                int max_blocks_per_seq, int num_blocks, int max_context_len, float scale,
                int dtype, int partition_size, void *workspace, size_t workspace_bytes,
                pkv_stream_t stream, bool with_merge) {
    int P;
    int rc = check_decode_sizes(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                max_context_len, partition_size, &P);
    if (rc != PKV_OK) return rc;
    if (dtype != PKV_F16 && dtype != PKV_BF16) return PKV_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return PKV_ERR_INVALID_ARG;
    if (max_blocks_per_seq < 1 || num_blocks < 1) return PKV_ERR_INVALID_ARG;
    if ((long long)max_context_len > (long long)max_blocks_per_seq * block_size)
        return PKV_ERR_INVALID_ARG;
    if ((long long)num_blocks * num_kv_heads * block_size >= INT_MAX) return PKV_ERR_INVALID_ARG;
    if (num_seqs == 0) return PKV_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
        return PKV_ERR_INVALID_ARG;
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(q, 16) || !aligned(out, 2) ||
        !aligned(block_tables, 4) || !aligned(context_lens, 4))
        return PKV_ERR_INVALID_ARG;
    const WsLayout ws = ws_layout(num_seqs, num_heads, head_dim, max_context_len, P);
    if (ws.total > 0 && (!workspace || workspace_bytes < ws.total || !aligned(workspace, 16)))
        return PKV_ERR_WORKSPACE;

    unsigned int *status;
    if ((rc = device_status_ptr(&status)) != PKV_OK) return rc;
    CUtensorMap mk, mv, mq;
    const long long cache_rows = (long long)num_blocks * num_kv_heads * block_size;
    const int group = num_heads / num_kv_heads;
    if ((rc = encode_rows_map(&mk, k_cache, dtype, head_dim, cache_rows, block_size)) != PKV_OK)
        return rc;
    if ((rc = encode_rows_map(&mv, v_cache, dtype, head_dim, cache_rows, block_size)) != PKV_OK)
        return rc;
    if ((rc = encode_rows_map(&mq, q, dtype, head_dim, (long long)num_seqs * num_heads, group)) !=
        PKV_OK)
        return rc;

    pkv::DecodeParams prm{};
    prm.out = out;
    prm.block_tables = block_tables;
    prm.context_lens = context_lens;
    uint8_t *wsb = static_cast<uint8_t *>(workspace);
    prm.sched = ws.total ? reinterpret_cast<pkv::SchedHeader *>(wsb) : nullptr;
    prm.ws_seq_base = ws.total ? reinterpret_cast<int32_t *>(wsb + ws.seq_base) : nullptr;
    prm.ws_ml = ws.total ? reinterpret_cast<float *>(wsb + ws.ml) : nullptr;
    prm.ws_o = ws.total ? reinterpret_cast<float *>(wsb + ws.o) : nullptr;
    prm.status = status;
    prm.num_seqs = num_seqs;
    prm.num_heads = num_heads;
    prm.num_kv_heads = num_kv_heads;
    prm.group = num_heads / num_kv_heads;
    prm.max_blocks_per_seq = max_blocks_per_seq;
    prm.num_blocks = num_blocks;
    prm.max_context_len = max_context_len;
    prm.partition = P;
    prm.scale_log2 = (float)((double)scale * 1.4426950408889634);

    const int pmax = max_context_len <= P ? 1 : cdiv(max_context_len, P);
    const long long items = (long long)num_seqs * num_kv_heads * pmax;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dtype == PKV_BF16) {
        rc = head_dim == 128 ? dispatch_bs<__nv_bfloat16, 128>(block_size, mk, mv, mq, prm, items, st)
                             : dispatch_bs<__nv_bfloat16, 64>(block_size, mk, mv, mq, prm, items, st);
        if (rc == PKV_OK && pmax > 1 && with_merge)
            rc = head_dim == 128 ? launch_reduce<__nv_bfloat16, 128>(prm, st)
                                 : launch_reduce<__nv_bfloat16, 64>(prm, st);
    } else {
        rc = head_dim == 128 ? dispatch_bs<__half, 128>(block_size, mk, mv, mq, prm, items, st)
                             : dispatch_bs<__half, 64>(block_size, mk, mv, mq, prm, items, st);
        if (rc == PKV_OK && pmax > 1 && with_merge)
            rc = head_dim == 128 ? launch_reduce<__half, 128>(prm, st)
                                 : launch_reduce<__half, 64>(prm, st);
    }
    return rc;
}

}  // namespace

extern "C" {

int pkv_paged_attention_decode(void *out, const void *q, const void *k_cache,
                               const void *v_cache, const int32_t *block_tables,
                               const int32_t *context_lens, int num_seqs, int num_heads,
                               int num_kv_heads, int head_dim, int block_size,
                               int max_blocks_per_seq, int num_blocks, int max_context_len,
                               float scale, int dtype, int partition_size, void *workspace,
                               size_t workspace_bytes, pkv_stream_t stream) {
    return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs, num_heads,
                       num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                       max_context_len, scale, dtype, partition_size, workspace, workspace_bytes,
                       stream, true);
}

int pkv_paged_attention_decode_partitions(void *out, const void *q, const void *k_cache,
                                          const void *v_cache, const int32_t *block_tables,
                                          const int32_t *context_lens, int num_seqs,
                                          int num_heads, int num_kv_heads, int head_dim,
                                          int block_size, int max_blocks_per_seq, int num_blocks,
                                          int max_context_len, float scale, int dtype,
                                          int partition_size, void *workspace,
                                          size_t workspace_bytes, pkv_stream_t stream) {
    return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs, num_heads,
                       num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                       max_context_len, scale, dtype, partition_size, workspace, workspace_bytes,
                       stream, false);
}

int pkv_paged_attention_merge(void *out, const int32_t *context_lens, int num_seqs, int num_heads,
                              int num_kv_heads, int head_dim, int block_size, int max_context_len,
                              int partition_size, int dtype, void *workspace,
                              size_t workspace_bytes, pkv_stream_t stream) {
    int P;
    int rc = check_decode_sizes(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                max_context_len, partition_size, &P);
    if (rc != PKV_OK) return rc;
    if (dtype != PKV_F16 && dtype != PKV_BF16) return PKV_ERR_INVALID_ARG;
    const WsLayout ws = ws_layout(num_seqs, num_heads, head_dim, max_context_len, P);
    if (num_seqs == 0 || ws.total == 0) return PKV_OK;   // every context is one partition
    if (!out || !context_lens || !aligned(out, 2) || !aligned(context_lens, 4))
        return PKV_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < ws.total || !aligned(workspace, 16))
        return PKV_ERR_WORKSPACE;
    unsigned int *status;
    if ((rc = device_status_ptr(&status)) != PKV_OK) return rc;
    uint8_t *wsb = static_cast<uint8_t *>(workspace);
    pkv::DecodeParams prm{};
    prm.out = out;
    prm.context_lens = context_lens;
    prm.sched = reinterpret_cast<pkv::SchedHeader *>(wsb);
    prm.ws_seq_base = reinterpret_cast<int32_t *>(wsb + ws.seq_base);
    prm.ws_ml = reinterpret_cast<float *>(wsb + ws.ml);
    prm.ws_o = reinterpret_cast<float *>(wsb + ws.o);
    prm.status = status;
    prm.num_seqs = num_seqs;
    prm.num_heads = num_heads;
    prm.num_kv_heads = num_kv_heads;
    prm.group = num_heads / num_kv_heads;
    prm.max_context_len = max_context_len;
    prm.partition = P;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dtype == PKV_BF16)
        return head_dim == 128 ? launch_reduce<__nv_bfloat16, 128>(prm, st)
                               : launch_reduce<__nv_bfloat16, 64>(prm, st);
    return head_dim == 128 ? launch_reduce<__half, 128>(prm, st)
                           : launch_reduce<__half, 64>(prm, st);
}

int pkv_paged_attention_decode_noalloc(void *out, const void *q, const void *k_cache,
                                       const void *v_cache, const int32_t *block_tables,
                                       const int32_t *context_lens, int num_seqs, int num_heads,
                                       int num_kv_heads, int head_dim, int block_size,
                                       int max_blocks_per_seq, int num_blocks,
                                       int max_context_len, float scale, int dtype,
                                       int partition_size, pkv_stream_t stream) {
    int P;
    const int rc = check_decode_sizes(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                      max_context_len, partition_size, &P);
    if (rc != PKV_OK) return rc;
    const size_t need = ws_layout(num_seqs, num_heads, head_dim, max_context_len, P).total;
    if (need > kNoAllocScratchBytes) return PKV_ERR_WORKSPACE;
    void *scratch = nullptr;
    if (need > 0) {
        const int r = noalloc_scratch_ptr(&scratch);
        if (r != PKV_OK) return r;
    }
    return pkv_paged_attention_decode(out, q, k_cache, v_cache, block_tables, context_lens,
                                      num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                      max_blocks_per_seq, num_blocks, max_context_len, scale,
                                      dtype, P, scratch, need > 0 ? kNoAllocScratchBytes : 0,
                                      stream);
}

int pkv_decode_step_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                   int block_size, int max_context_len, int partition_size,
                                   size_t *bytes_out) {
    if (!bytes_out) return PKV_ERR_INVALID_ARG;
    int P;
    const int rc = check_decode_sizes(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                      max_context_len, partition_size, &P);
    if (rc != PKV_OK) return rc;
    *bytes_out = step_ws_bytes(num_seqs, num_heads, head_dim, max_context_len, P);
    return PKV_OK;
}

}  // extern "C"

namespace {

// pkv_paged_decode_step (split = false) or the write-and-decode launch alone (split).
int step_impl(void *out, const void *q, const void *k_new, const void *v_new, void *k_cache,
              void *v_cache, const int32_t *block_tables, const int32_t *context_lens,
              int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
              int max_blocks_per_seq, int num_blocks, int max_context_len, float scale, int dtype,
              int partition_size, void *workspace, size_t workspace_bytes, pkv_stream_t stream,
              bool split) {
    int P;
    int rc = check_decode_sizes(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                max_context_len, partition_size, &P);
    if (rc != PKV_OK) return rc;
    if (dtype != PKV_F16 && dtype != PKV_BF16) return PKV_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return PKV_ERR_INVALID_ARG;
    if (max_blocks_per_seq < 1 || num_blocks < 1) return PKV_ERR_INVALID_ARG;
    if ((long long)max_context_len > (long long)max_blocks_per_seq * block_size)
        return PKV_ERR_INVALID_ARG;
    if ((long long)num_blocks * num_kv_heads * block_size >= INT_MAX) return PKV_ERR_INVALID_ARG;
    if (num_seqs == 0) return PKV_OK;
    if (!out || !q || !k_new || !v_new || !k_cache || !v_cache || !block_tables || !context_lens)
        return PKV_ERR_INVALID_ARG;
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(q, 16) || !aligned(k_new, 16) ||
        !aligned(v_new, 16) || !aligned(out, 2) || !aligned(block_tables, 4) ||
        !aligned(context_lens, 4))
        return PKV_ERR_INVALID_ARG;
    const size_t need = step_ws_bytes(num_seqs, num_heads, head_dim, max_context_len, P);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return PKV_ERR_WORKSPACE;
    const WsLayout ws = ws_layout(num_seqs, num_heads, head_dim, max_context_len, P);

    unsigned int *status;
    if ((rc = device_status_ptr(&status)) != PKV_OK) return rc;
    CUtensorMap mk, mv, mq;
    const long long cache_rows = (long long)num_blocks * num_kv_heads * block_size;
    const int group = num_heads / num_kv_heads;
    if ((rc = encode_rows_map(&mk, k_cache, dtype, head_dim, cache_rows, block_size)) != PKV_OK)
        return rc;
    if ((rc = encode_rows_map(&mv, v_cache, dtype, head_dim, cache_rows, block_size)) != PKV_OK)
        return rc;
    if ((rc = encode_rows_map(&mq, q, dtype, head_dim, (long long)num_seqs * num_heads, group)) !=
        PKV_OK)
        return rc;

    pkv::DecodeParams prm{};
    prm.out = out;
    prm.block_tables = block_tables;
    prm.context_lens = context_lens;
    uint8_t *wsb = static_cast<uint8_t *>(workspace);
    prm.sched = reinterpret_cast<pkv::SchedHeader *>(wsb);
    prm.ws_seq_base = ws.total ? reinterpret_cast<int32_t *>(wsb + ws.seq_base) : nullptr;
    prm.ws_ml = ws.total ? reinterpret_cast<float *>(wsb + ws.ml) : nullptr;
    prm.ws_o = ws.total ? reinterpret_cast<float *>(wsb + ws.o) : nullptr;
    prm.status = status;
    prm.num_seqs = num_seqs;
    prm.num_heads = num_heads;
    prm.num_kv_heads = num_kv_heads;
    prm.group = group;
    prm.max_blocks_per_seq = max_blocks_per_seq;
    prm.num_blocks = num_blocks;
    prm.max_context_len = max_context_len;
    prm.partition = P;
    prm.scale_log2 = (float)((double)scale * 1.4426950408889634);
    prm.k_new = k_new;
    prm.v_new = v_new;
    prm.k_cache = k_cache;
    prm.v_cache = v_cache;

    const int pmax = max_context_len <= P ? 1 : cdiv(max_context_len, P);
    const long long items = (long long)num_seqs * num_kv_heads * pmax;
    const int merge = pmax > 1;
    int nsm;
    if ((rc = sm_count(&nsm)) != PKV_OK) return rc;
    const int ink = split ? 0 : step_merges_in_kernel(num_seqs, num_heads, items, pmax, nsm);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dtype == PKV_BF16)
        return head_dim == 128 ? dispatch_step<__nv_bfloat16, 128>(block_size, mk, mv, mq, prm,
                                                                   items, merge, ink, !split, st)
                               : dispatch_step<__nv_bfloat16, 64>(block_size, mk, mv, mq, prm,
                                                                  items, merge, ink, !split, st);
    return head_dim == 128
               ? dispatch_step<__half, 128>(block_size, mk, mv, mq, prm, items, merge, ink,
                                            !split, st)
               : dispatch_step<__half, 64>(block_size, mk, mv, mq, prm, items, merge, ink,
                                           !split, st);
}

}  // namespace

extern "C" {

int pkv_paged_decode_step(void *out, const void *q, const void *k_new, const void *v_new,
                          void *k_cache, void *v_cache, const int32_t *block_tables,
                          const int32_t *context_lens, int num_seqs, int num_heads,
                          int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                          int num_blocks, int max_context_len, float scale, int dtype,
                          int partition_size, void *workspace, size_t workspace_bytes,
                          pkv_stream_t stream) {
    return step_impl(out, q, k_new, v_new, k_cache, v_cache, block_tables, context_lens, num_seqs,
                     num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                     num_blocks, max_context_len, scale, dtype, partition_size, workspace,
                     workspace_bytes, stream, false);
}

int pkv_paged_decode_step_partitions(void *out, const void *q, const void *k_new,
                                     const void *v_new, void *k_cache, void *v_cache,
                                     const int32_t *block_tables, const int32_t *context_lens,
                                     int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                     int block_size, int max_blocks_per_seq, int num_blocks,
                                     int max_context_len, float scale, int dtype,
                                     int partition_size, void *workspace, size_t workspace_bytes,
                                     pkv_stream_t stream) {
    return step_impl(out, q, k_new, v_new, k_cache, v_cache, block_tables, context_lens, num_seqs,
                     num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                     num_blocks, max_context_len, scale, dtype, partition_size, workspace,
                     workspace_bytes, stream, true);
}

int pkv_decode_step_launches(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                             int block_size, int max_context_len, int partition_size,
                             int *launches_out) {
    if (!launches_out) return PKV_ERR_INVALID_ARG;
    int P;
    int rc = check_decode_sizes(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                max_context_len, partition_size, &P);
    if (rc != PKV_OK) return rc;
    if (num_seqs == 0) {
        *launches_out = 0;
        return PKV_OK;
    }
    const int pmax = max_context_len <= P ? 1 : cdiv(max_context_len, P);
    const long long items = (long long)num_seqs * num_kv_heads * pmax;
    int nsm;
    if ((rc = sm_count(&nsm)) != PKV_OK) return rc;
    *launches_out =
        pmax > 1 && !step_merges_in_kernel(num_seqs, num_heads, items, pmax, nsm) ? 2 : 1;
    return PKV_OK;
}

int pkv_device_append(int32_t *block_tables, int32_t *context_lens, const int32_t *free_blocks,
                      int free_count, int32_t *free_used, const int32_t *block_refcounts,
                      int64_t *slots_out, int num_seqs, int max_blocks_per_seq, int block_size,
                      int num_blocks, int max_context_len, pkv_stream_t stream) {
    if (num_seqs < 0 || free_count < 0 || max_blocks_per_seq < 1 || block_size < 1 ||
        num_blocks < 1 || max_context_len < 0)
        return PKV_ERR_INVALID_ARG;
    if ((long long)num_blocks * block_size >= (1LL << 62)) return PKV_ERR_INVALID_ARG;
    if (!free_used) return PKV_ERR_INVALID_ARG;
    if (num_seqs > 0 && (!block_tables || !context_lens)) return PKV_ERR_INVALID_ARG;
    if (free_count > 0 && !free_blocks) return PKV_ERR_INVALID_ARG;
    if (!aligned(block_tables, 4) || !aligned(context_lens, 4) || !aligned(free_blocks, 4) ||
        !aligned(free_used, 4) || !aligned(block_refcounts, 4) || !aligned(slots_out, 8))
        return PKV_ERR_INVALID_ARG;
    unsigned int *status;
    int rc;
    if ((rc = device_status_ptr(&status)) != PKV_OK) return rc;
    return launch(pkv::device_append_kernel, dim3(1), dim3(pkv::kPlanThreads), 0,
                  reinterpret_cast<cudaStream_t>(stream), block_tables, context_lens, free_blocks,
                  free_count, reinterpret_cast<int *>(free_used), block_refcounts, slots_out,
                  num_seqs,
                  max_blocks_per_seq, block_size, num_blocks, max_context_len, status);
}

int pkv_decode_shared_prefix_workspace_size(int num_seqs, int num_heads, int num_kv_heads,
                                            int head_dim, int block_size, int max_context_len,
                                            int partition_size, size_t *bytes_out) {
    if (!bytes_out) return PKV_ERR_INVALID_ARG;
    int P;
    const int rc = check_decode_sizes(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                      max_context_len, partition_size, &P, true);
    if (rc != PKV_OK) return rc;
    *bytes_out = num_seqs ? shared_ws_layout(num_seqs, num_heads, num_kv_heads, head_dim,
                                             max_context_len, P).total
                          : 0;
    return PKV_OK;
}

// Host checks shared by the shared-prefix entry points; resolves the partition size.
static int check_shared(int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                 int max_blocks_per_seq, int num_blocks, int max_context_len, int partition_size,
                 int *P) {
    int rc = check_decode_sizes(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                max_context_len, partition_size, P, true);
    if (rc != PKV_OK) return rc;
    if (max_blocks_per_seq < 1 || num_blocks < 1) return PKV_ERR_INVALID_ARG;
    if ((long long)max_context_len > (long long)max_blocks_per_seq * block_size)
        return PKV_ERR_INVALID_ARG;
    if ((long long)num_blocks * num_kv_heads * block_size >= INT_MAX) return PKV_ERR_INVALID_ARG;
    return PKV_OK;
}

int pkv_shared_prefix_plan(const int32_t *block_tables, const int32_t *context_lens,
                           const int32_t *group_start, const int32_t *prefix_lens, int num_groups,
                           int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                           int block_size, int max_blocks_per_seq, int max_context_len,
                           int partition_size, void *workspace, size_t workspace_bytes,
                           pkv_stream_t stream) {
    int P;
    int rc = check_shared(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                          max_blocks_per_seq, 1, max_context_len, partition_size, &P);
    if (rc != PKV_OK) return rc;
    if (num_seqs == 0) return PKV_OK;
    if (num_groups < 1 || num_groups > num_seqs) return PKV_ERR_INVALID_ARG;
    if (!block_tables || !context_lens || !group_start || !prefix_lens) return PKV_ERR_INVALID_ARG;
    if (!aligned(block_tables, 4) || !aligned(context_lens, 4) || !aligned(group_start, 4) ||
        !aligned(prefix_lens, 4))
        return PKV_ERR_INVALID_ARG;
    const SharedWs ws =
        shared_ws_layout(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len, P);
    if (!workspace || workspace_bytes < ws.total || !aligned(workspace, 16))
        return PKV_ERR_WORKSPACE;
    unsigned int *status;
    if ((rc = device_status_ptr(&status)) != PKV_OK) return rc;
    pkv::SharedParams prm = shared_params(ws, workspace, num_seqs, num_heads, num_kv_heads,
                                          block_size, max_blocks_per_seq, 1, max_context_len, P,
                                          block_tables, context_lens, status);
    prm.group_start = group_start;
    prm.prefix_lens = prefix_lens;
    prm.num_groups = num_groups;
    if ((rc = sm_count(&prm.sms)) != PKV_OK) return rc;
    if ((rc = shared_decode_slots(head_dim, &prm.slots)) != PKV_OK) return rc;
    return launch_shared_plan(prm, reinterpret_cast<cudaStream_t>(stream));
}

int pkv_paged_attention_decode_shared_prefix_planned(
    void *out, const void *q, const void *k_cache, const void *v_cache,
    const int32_t *block_tables, const int32_t *context_lens, int num_seqs, int num_heads,
    int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq, int num_blocks,
    int max_context_len, float scale, int dtype, int partition_size, void *workspace,
    size_t workspace_bytes, pkv_stream_t stream) {
    int P;
    int rc = check_shared(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                          max_blocks_per_seq, num_blocks, max_context_len, partition_size, &P);
    if (rc != PKV_OK) return rc;
    if (dtype != PKV_F16 && dtype != PKV_BF16) return PKV_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return PKV_ERR_INVALID_ARG;
    if (num_seqs == 0) return PKV_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
        return PKV_ERR_INVALID_ARG;
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(q, 4) || !aligned(out, 2) ||
        !aligned(block_tables, 4) || !aligned(context_lens, 4))
        return PKV_ERR_INVALID_ARG;
    const SharedWs ws =
        shared_ws_layout(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len, P);
    if (!workspace || workspace_bytes < ws.total || !aligned(workspace, 16))
        return PKV_ERR_WORKSPACE;
    unsigned int *status;
    if ((rc = device_status_ptr(&status)) != PKV_OK) return rc;
    CUtensorMap mk, mv;
    const long long cache_rows = (long long)num_blocks * num_kv_heads * block_size;
    if ((rc = encode_rows_map(&mk, k_cache, dtype, head_dim, cache_rows, block_size)) != PKV_OK)
        return rc;
    if ((rc = encode_rows_map(&mv, v_cache, dtype, head_dim, cache_rows, block_size)) != PKV_OK)
        return rc;
    pkv::SharedParams prm = shared_params(ws, workspace, num_seqs, num_heads, num_kv_heads,
                                          block_size, max_blocks_per_seq, num_blocks,
                                          max_context_len, P, block_tables, context_lens, status);
    prm.out = out;
    prm.q = q;
    prm.scale_log2 = (float)((double)scale * 1.4426950408889634);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dtype == PKV_BF16)
        return head_dim == 128
                   ? launch_shared_decode_reduce<__nv_bfloat16, 128>(block_size, mk, mv, prm, st)
                   : launch_shared_decode_reduce<__nv_bfloat16, 64>(block_size, mk, mv, prm, st);
    return head_dim == 128 ? launch_shared_decode_reduce<__half, 128>(block_size, mk, mv, prm, st)
                           : launch_shared_decode_reduce<__half, 64>(block_size, mk, mv, prm, st);
}

int pkv_paged_attention_decode_shared_prefix(
    void *out, const void *q, const void *k_cache, const void *v_cache,
    const int32_t *block_tables, const int32_t *context_lens, const int32_t *group_start,
    const int32_t *prefix_lens, int num_groups, int num_seqs, int num_heads, int num_kv_heads,
    int head_dim, int block_size, int max_blocks_per_seq, int num_blocks, int max_context_len,
    float scale, int dtype, int partition_size, void *workspace, size_t workspace_bytes,
    pkv_stream_t stream) {
    int P;
    int rc = check_shared(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                          max_blocks_per_seq, num_blocks, max_context_len, partition_size, &P);
    if (rc != PKV_OK) return rc;
    if (dtype != PKV_F16 && dtype != PKV_BF16) return PKV_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return PKV_ERR_INVALID_ARG;
    if (num_seqs == 0) return PKV_OK;
    if (num_groups < 1 || num_groups > num_seqs) return PKV_ERR_INVALID_ARG;
    if (!out || !q || !k_cache || !v_cache) return PKV_ERR_INVALID_ARG;
    rc = pkv_shared_prefix_plan(block_tables, context_lens, group_start, prefix_lens, num_groups,
                                num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                max_blocks_per_seq, max_context_len, P, workspace,
                                workspace_bytes, stream);
    if (rc != PKV_OK) return rc;
    return pkv_paged_attention_decode_shared_prefix_planned(
        out, q, k_cache, v_cache, block_tables, context_lens, num_seqs, num_heads, num_kv_heads,
        head_dim, block_size, max_blocks_per_seq, num_blocks, max_context_len, scale, dtype, P,
        workspace, workspace_bytes, stream);
}

int pkv_reshape_and_cache(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                          const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                          int head_dim, int block_size, int num_blocks, int dtype,
                          pkv_stream_t stream) {
    if (num_tokens < 0 || num_kv_heads < 1 || num_blocks < 1) return PKV_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return PKV_ERR_INVALID_ARG;
    if (block_size != 8 && block_size != 16 && block_size != 32) return PKV_ERR_INVALID_ARG;
    if (dtype != PKV_F16 && dtype != PKV_BF16) return PKV_ERR_INVALID_ARG;
    if (num_tokens == 0) return PKV_OK;
    if (!k_new || !v_new || !k_cache || !v_cache || !slot_mapping) return PKV_ERR_INVALID_ARG;
    if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_cache, 16) ||
        !aligned(v_cache, 16) || !aligned(slot_mapping, 8))
        return PKV_ERR_INVALID_ARG;
    unsigned int *status;
    int rc;
    if ((rc = device_status_ptr(&status)) != PKV_OK) return rc;
    int nsm;
    if ((rc = sm_count(&nsm)) != PKV_OK) return rc;
    const long long total = (long long)num_tokens * num_kv_heads * (head_dim * 2 / 16);
    long long blocks = (total + 255) / 256;
    if (blocks > (long long)nsm * 16) blocks = (long long)nsm * 16;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    auto *kn = static_cast<const uint4 *>(k_new);
    auto *vn = static_cast<const uint4 *>(v_new);
    auto *kc = static_cast<uint4 *>(k_cache);
    auto *vc = static_cast<uint4 *>(v_cache);
    if (head_dim == 128)
        return launch(pkv::reshape_and_cache_kernel<128>, dim3((unsigned)blocks), dim3(256), 0, st,
                      kn, vn, kc, vc, slot_mapping, num_tokens, num_kv_heads, block_size,
                      num_blocks, status);
    return launch(pkv::reshape_and_cache_kernel<64>, dim3((unsigned)blocks), dim3(256), 0, st, kn,
                  vn, kc, vc, slot_mapping, num_tokens, num_kv_heads, block_size, num_blocks,
                  status);
}

int pkv_copy_blocks(void *const *k_caches, void *const *v_caches, int num_layers,
                    const int32_t *block_pairs, int num_pairs, int num_kv_heads, int head_dim,
                    int block_size, int num_blocks, int dtype, pkv_stream_t stream) {
    if (num_pairs < 0 || num_layers < 1 || num_layers > 65535 || num_kv_heads < 1 ||
        num_blocks < 1)
        return PKV_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return PKV_ERR_INVALID_ARG;
    if (block_size != 8 && block_size != 16 && block_size != 32) return PKV_ERR_INVALID_ARG;
    if (dtype != PKV_F16 && dtype != PKV_BF16) return PKV_ERR_INVALID_ARG;
    if (num_pairs == 0) return PKV_OK;
    if (!k_caches || !v_caches || !block_pairs) return PKV_ERR_INVALID_ARG;
    const long long vecs = (long long)num_kv_heads * block_size * head_dim * 2 / 16;
    if (vecs >= INT_MAX) return PKV_ERR_INVALID_ARG;
    unsigned int *status;
    int rc;
    if ((rc = device_status_ptr(&status)) != PKV_OK) return rc;
    dim3 grid((unsigned)num_pairs, (unsigned)num_layers, 2);
    return launch(pkv::copy_blocks_kernel, grid, dim3(256), 0,
                  reinterpret_cast<cudaStream_t>(stream), k_caches, v_caches, block_pairs,
                  num_blocks, (int)vecs, status);
}

int pkv_swap_blocks(void *const *k_caches, void *const *v_caches, int num_layers,
                    const int32_t *block_ids, int num_ids, void *host_buffer,
                    size_t host_buffer_bytes, int to_host, int num_kv_heads, int head_dim,
                    int block_size, int num_blocks, int dtype, pkv_stream_t stream) {
    if (num_ids < 0 || num_layers < 1 || num_layers > 65535 || num_kv_heads < 1 ||
        num_blocks < 1 || (to_host != 0 && to_host != 1))
        return PKV_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return PKV_ERR_INVALID_ARG;
    if (block_size != 8 && block_size != 16 && block_size != 32) return PKV_ERR_INVALID_ARG;
    if (dtype != PKV_F16 && dtype != PKV_BF16) return PKV_ERR_INVALID_ARG;
    if (num_ids == 0) return PKV_OK;
    if (!k_caches || !v_caches || !block_ids || !host_buffer || !aligned(host_buffer, 16))
        return PKV_ERR_INVALID_ARG;
    const long long vecs = (long long)num_kv_heads * block_size * head_dim * 2 / 16;
    if (vecs >= INT_MAX) return PKV_ERR_INVALID_ARG;
    const unsigned long long need = (unsigned long long)num_layers * 2 * num_ids * vecs * 16;
    if (host_buffer_bytes < need) return PKV_ERR_INVALID_ARG;
    // the kernel reads / writes the buffer through unified addressing: it must be
    // pinned host memory that this device can reach
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, host_buffer) != cudaSuccess) {
        cudaGetLastError();
        return PKV_ERR_INVALID_ARG;
    }
    if (attr.type != cudaMemoryTypeHost || attr.devicePointer != host_buffer)
        return PKV_ERR_INVALID_ARG;
    unsigned int *status;
    int rc;
    if ((rc = device_status_ptr(&status)) != PKV_OK) return rc;
    dim3 grid((unsigned)num_ids, (unsigned)num_layers, 2);
    return launch(pkv::swap_blocks_kernel, grid, dim3(256), 0,
                  reinterpret_cast<cudaStream_t>(stream), k_caches, v_caches, block_ids,
                  num_ids, static_cast<uint4 *>(host_buffer), num_blocks, (int)vecs, to_host,
                  status);
}

int pkv_swap_blocks_staged(void *const *k_caches, void *const *v_caches, int num_layers,
                           const int32_t *block_ids, int num_ids, void *host_buffer,
                           size_t host_buffer_bytes, int to_host, int num_kv_heads,
                           int head_dim, int block_size, int num_blocks, int dtype,
                           void *staging, size_t staging_bytes, pkv_stream_t stream) {
    if (num_ids < 0 || num_layers < 1 || num_layers > 65535 || num_kv_heads < 1 ||
        num_blocks < 1 || (to_host != 0 && to_host != 1))
        return PKV_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return PKV_ERR_INVALID_ARG;
    if (block_size != 8 && block_size != 16 && block_size != 32) return PKV_ERR_INVALID_ARG;
    if (dtype != PKV_F16 && dtype != PKV_BF16) return PKV_ERR_INVALID_ARG;
    if (num_ids == 0) return PKV_OK;
    if (!k_caches || !v_caches || !block_ids || !host_buffer || !aligned(host_buffer, 16))
        return PKV_ERR_INVALID_ARG;
    const long long vecs = (long long)num_kv_heads * block_size * head_dim * 2 / 16;
    if (vecs >= INT_MAX) return PKV_ERR_INVALID_ARG;
    const unsigned long long tile = (unsigned long long)vecs * 16;
    const long long total = (long long)num_layers * 2 * num_ids;
    if (host_buffer_bytes < (unsigned long long)total * tile) return PKV_ERR_INVALID_ARG;
    if (!staging || !aligned(staging, 16) || staging_bytes < 2 * tile) return PKV_ERR_WORKSPACE;
    // the copies are asynchronous only from pinned memory: anything else is refused
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, host_buffer) != cudaSuccess) {
        cudaGetLastError();
        return PKV_ERR_INVALID_ARG;
    }
    if (attr.type != cudaMemoryTypeHost) return PKV_ERR_INVALID_ARG;
    if (cudaPointerGetAttributes(&attr, staging) != cudaSuccess) {
        cudaGetLastError();
        return PKV_ERR_INVALID_ARG;
    }
    if (attr.type != cudaMemoryTypeDevice) return PKV_ERR_INVALID_ARG;
    unsigned int *status;
    int rc;
    if ((rc = device_status_ptr(&status)) != PKV_OK) return rc;
    int dev;
    if ((rc = current_device(&dev)) != PKV_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // Two halves of the staging buffer: while the copy engine moves one half over the link
    // (on a stream of the library's, `cs`), the next gather fills the other half on `st`
    // (or, into the device, the next copy fills one half while the previous scatter drains
    // the other). Events order each half's fill after its last drain.
    const long long per = (long long)std::min<unsigned long long>(staging_bytes / 2 / tile,
                                                                  INT_MAX);
    if (per < 1) return PKV_ERR_WORKSPACE;
    std::lock_guard<std::mutex> lk(g_swap_mu);   // the side stream and events are shared
    SwapSide &side = g_swap_side[dev];
    if (!side.ready) {
        if (cudaStreamCreateWithFlags(&side.cs, cudaStreamNonBlocking) != cudaSuccess)
            return PKV_ERR_CUDA;
        for (cudaEvent_t *e : {&side.start, &side.fill[0], &side.fill[1], &side.drain[0],
                               &side.drain[1]})
            if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess)
                return PKV_ERR_CUDA;
        side.ready = true;
    }
    cudaStream_t cs = side.cs;
    char *host = static_cast<char *>(host_buffer);
    char *halves[2] = {static_cast<char *>(staging),
                       static_cast<char *>(staging) + (size_t)per * tile};
    if (cudaEventRecord(side.start, st) != cudaSuccess) return PKV_ERR_CUDA;
    if (cudaStreamWaitEvent(cs, side.start, 0) != cudaSuccess) return PKV_ERR_CUDA;
    long long k = 0;
    for (long long t0 = 0; t0 < total; t0 += per, ++k) {
        const int h = (int)(k & 1);
        const long long cnt = std::min(per, total - t0);
        char *hp = host + (unsigned long long)t0 * tile;
        const size_t bytes = (size_t)((unsigned long long)cnt * tile);
        uint4 *stg = reinterpret_cast<uint4 *>(halves[h]);
        if (to_host) {
            // gather k into half h once copy k-2 has read it, then copy it out
            if (k >= 2 && cudaStreamWaitEvent(st, side.drain[h], 0) != cudaSuccess)
                return PKV_ERR_CUDA;
            if ((rc = launch(pkv::swap_stage_kernel, dim3((unsigned)cnt), dim3(256), 0, st,
                             k_caches, v_caches, block_ids, num_ids, stg, t0, num_blocks,
                             (int)vecs, 1, status)) != PKV_OK)
                return rc;
            if (cudaEventRecord(side.fill[h], st) != cudaSuccess ||
                cudaStreamWaitEvent(cs, side.fill[h], 0) != cudaSuccess ||
                cudaMemcpyAsync(hp, stg, bytes, cudaMemcpyDeviceToHost, cs) != cudaSuccess ||
                cudaEventRecord(side.drain[h], cs) != cudaSuccess)
                return PKV_ERR_CUDA;
        } else {
            // copy k into half h once scatter k-2 has read it, then scatter it
            if (k >= 2 && cudaStreamWaitEvent(cs, side.drain[h], 0) != cudaSuccess)
                return PKV_ERR_CUDA;
            if (cudaMemcpyAsync(stg, hp, bytes, cudaMemcpyHostToDevice, cs) != cudaSuccess ||
                cudaEventRecord(side.fill[h], cs) != cudaSuccess ||
                cudaStreamWaitEvent(st, side.fill[h], 0) != cudaSuccess)
                return PKV_ERR_CUDA;
            if ((rc = launch(pkv::swap_stage_kernel, dim3((unsigned)cnt), dim3(256), 0, st,
                             k_caches, v_caches, block_ids, num_ids, stg, t0, num_blocks,
                             (int)vecs, 0, status)) != PKV_OK)
                return rc;
            if (cudaEventRecord(side.drain[h], st) != cudaSuccess) return PKV_ERR_CUDA;
        }
    }
    if (to_host) {
        // `st` reaches the end of the call once every copy has landed in host memory
        for (int h = 0; h < 2 && h < k; ++h)
            if (cudaStreamWaitEvent(st, side.drain[h], 0) != cudaSuccess) return PKV_ERR_CUDA;
    }
    return PKV_OK;
}

int pkv_get_device_status(uint32_t *status_out, int clear, pkv_stream_t stream) {
    if (!status_out) return PKV_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return PKV_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_pkv_status, sizeof(v)) != cudaSuccess) return PKV_ERR_CUDA;
    if (clear) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_pkv_status, &zero, sizeof(zero)) != cudaSuccess)
            return PKV_ERR_CUDA;
    }
    *status_out = v;
    return PKV_OK;
}

}  // extern "C"
