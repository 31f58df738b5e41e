// libdsa.so: the C ABI declared in include/dsa.h.  Host side: argument validation, workspace
// carving, TMA descriptor encoding, launch configuration and the fused prefill/decode drivers.
// Every computation of the path runs in the kernels of indexer.cuh, topk.cuh and attn.cuh.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "attn.cuh"
#include "attn_dedup.cuh"
#include "kl.cuh"
#include "dsa.h"
#include "indexer.cuh"
#include "ptx.cuh"
#include "topk.cuh"

using namespace dsa;

namespace {

constexpr int kVersion = 10000;
constexpr int kMaxTopk = 65536;
constexpr int kMaxDecodeSplits = 16;
static_assert(kMaxDecodeSplits <= 32, "attn_combine_kernel holds one split per lane");
constexpr int kDecodeIdxStages = 8;
constexpr int kPrefillIdxStages = 4;

// ------------------------------------------------------------------ launch accounting / profiling
std::atomic<long long> g_launches{0};
std::mutex g_prof_mu;
bool g_prof_on = false;
struct ProfRec {
    int kind;
    cudaEvent_t a, b;
};
std::vector<ProfRec> g_prof_recs;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t pooled_event() {
    if (!g_event_pool.empty()) {
        cudaEvent_t e = g_event_pool.back();
        g_event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

struct LaunchScope {
    int kind;
    cudaStream_t s;
    cudaEvent_t a = nullptr, b = nullptr;
    LaunchScope(int kind_, cudaStream_t s_) : kind(kind_), s(s_) {
        g_launches.fetch_add(1);
        std::lock_guard<std::mutex> lk(g_prof_mu);
        if (g_prof_on) {
            a = pooled_event();
            b = pooled_event();
            cudaEventRecord(a, s);
        }
    }
    ~LaunchScope() {
        if (a) {
            cudaEventRecord(b, s);
            std::lock_guard<std::mutex> lk(g_prof_mu);
            g_prof_recs.push_back({kind, a, b});
        }
    }
};

enum { K_INDEX = 0, K_TOPK = 1, K_ATTN = 2, K_COMBINE = 3, K_APPEND = 4, K_ADVANCE = 5, K_SELFTEST = 6, K_KL = 7 };

dsa_status launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// ------------------------------------------------------------------ device properties
// The SM count and the kernels' shared-memory limits belong to a device: both are cached per
// device id, so that a process which moves between devices (cudaSetDevice) between calls still
// configures each device before its first launch there.
constexpr int kMaxDevices = 256;

int current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
    return dev;
}

int num_sms() {
    static std::atomic<int> n[kMaxDevices];
    const int dev = current_device();
    if (dev < 0) return 0;
    int v = n[dev].load(std::memory_order_relaxed);
    if (v <= 0) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) return 0;
        n[dev].store(v, std::memory_order_relaxed);
    }
    return v;
}

// One flag per device: the kernel's dynamic shared-memory limit has been raised there.
using DeviceFlags = std::atomic<bool>[kMaxDevices];

// Raise `kern`'s dynamic shared-memory limit to `bytes` on the current device, once per device.
template <typename Kern>
bool set_smem_limit(Kern* kern, int bytes, DeviceFlags& done) {
    const int dev = current_device();
    if (dev < 0) return false;
    if (done[dev].load(std::memory_order_acquire)) return true;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
    done[dev].store(true, std::memory_order_release);
    return true;
}

// ------------------------------------------------------------------ TMA descriptors
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// bf16 tensor [d2][d1][64] (rows of 128 bytes), box {64, box_rows, 1}, 128-byte swizzle.
bool make_rows_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t batch, uint64_t batch_stride_bytes,
                   uint32_t box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {64, rows, batch};
    cuuint64_t strides[2] = {128, batch_stride_bytes};
    cuuint32_t box[3] = {64, box_rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool hi_supported_prefill(int HI) {
    return HI == 1 || HI == 2 || HI == 4 || HI == 8 || HI == 16 || HI == 32 || HI == 64;
}
bool hi_supported_decode(int HI) { return HI == 16 || HI == 32 || HI == 64; }

dsa_status check_attn_shape(int Hq, int Hkv, int D) {
    if (Hq <= 0 || Hkv <= 0 || D <= 0) return DSA_ERR_INVALID_ARG;
    if (D != kAttnD) return DSA_ERR_UNSUPPORTED;
    if (!(Hkv == 1 || Hkv == 2 || Hkv == 4)) return DSA_ERR_UNSUPPORTED;
    if (Hq % Hkv != 0 || Hq / Hkv > 16) return DSA_ERR_UNSUPPORTED;
    return DSA_OK;
}

// ------------------------------------------------------------------ indexer launch
template <int HI, int BN, int STAGES>
dsa_status launch_indexer_t(const CUtensorMap& mq, const CUtensorMap& mk, const IndexerParams& P, int grid,
                            cudaStream_t s) {
    using C = IndexerCfg<HI, BN, STAGES>;
    auto kern = indexer_kernel<HI, BN, STAGES>;
    static DeviceFlags attr_set;
    if (!set_smem_limit(kern, C::SMEM, attr_set)) return DSA_ERR_CUDA;
    LaunchScope ls(K_INDEX, s);
    kern<<<grid, C::THREADS, C::SMEM, s>>>(mq, mk, P);
    return launch_status();
}

// Query tokens per indexer work block: a 256-column tile of whole tokens (prefill), or the one new
// token of a sequence (decode).
int indexer_tb(int HI, bool decode) { return decode ? 1 : 256 / HI; }

// Shared by dsa_index (P = 1) and the decode step (P = B, one query each).
dsa_status run_indexer(const void* qI, const void* kI, const __nv_bfloat16* w, int P_, int Lq, int64_t q_pos0,
                       const int* ctx_len, int64_t Lk, int HI, float* scores, int64_t ld, cudaStream_t s,
                       int64_t window = 0, const IndexerParams* append = nullptr) {
    const bool decode = ctx_len != nullptr;
    const int TB = indexer_tb(HI, decode);
    IndexerParams P{};
    P.P = P_;
    P.Lq = Lq;
    P.q_pos0 = q_pos0;
    P.ctx_len = ctx_len;
    P.Lk = Lk;
    P.w = w;
    P.scores = scores;
    P.ld = ld;
    P.num_qb = (Lq + TB - 1) / TB;
    P.window = decode ? 0 : window;
    if (append) {
        P.new_k = append->new_k;
        P.new_v = append->new_v;
        P.new_kI = append->new_kI;
        P.cache_k = append->cache_k;
        P.cache_v = append->cache_v;
        P.cache_kI = append->cache_kI;
        P.kv16 = append->kv16;
        P.kI16 = append->kI16;
    }
    const int sms = num_sms();
    if (sms <= 0) return DSA_ERR_CUDA;
    const int64_t ktiles = (Lk + kIdxBM - 1) / kIdxBM;
    if (decode) {
        // about 4 units per SM, the same count on every SM when B divides 4*SMs
        int ns = std::max(1, (4 * sms + P_ - 1) / P_);
        ns = (int)std::min<int64_t>(ns, ktiles);
        P.kt_per_split = (int)((ktiles + ns - 1) / ns);
        P.nsplit = (int)((ktiles + P.kt_per_split - 1) / P.kt_per_split);
    } else {
        P.nsplit = 1;
        P.kt_per_split = (int)ktiles;
    }
    P.num_units = P_ * P.num_qb * P.nsplit;
    const uint64_t qrows = (uint64_t)Lq * HI;
    const uint32_t qbox = (uint32_t)std::min<uint64_t>((uint64_t)TB * HI, qrows);  // one block's qI rows
    const uint32_t kbox = (uint32_t)std::min<int64_t>(kIdxBM, Lk);
    P.q_box_bytes = qbox * 128u;
    P.k_box_bytes = kbox * 128u;
    CUtensorMap mq, mk;
    if (!make_rows_map(&mq, qI, qrows, (uint64_t)P_, qrows * 128ull, qbox)) return DSA_ERR_CUDA;
    if (!make_rows_map(&mk, kI, (uint64_t)Lk, (uint64_t)P_, (uint64_t)Lk * 128ull, kbox)) return DSA_ERR_CUDA;
    const int grid = std::min(P.num_units, sms);
    if (grid <= 0) return DSA_OK;
    if (!decode) {
        switch (HI) {
        case 1: return launch_indexer_t<1, 256, kPrefillIdxStages>(mq, mk, P, grid, s);
        case 2: return launch_indexer_t<2, 256, kPrefillIdxStages>(mq, mk, P, grid, s);
        case 4: return launch_indexer_t<4, 256, kPrefillIdxStages>(mq, mk, P, grid, s);
        case 8: return launch_indexer_t<8, 256, kPrefillIdxStages>(mq, mk, P, grid, s);
        case 16: return launch_indexer_t<16, 256, kPrefillIdxStages>(mq, mk, P, grid, s);
        case 32: return launch_indexer_t<32, 256, kPrefillIdxStages>(mq, mk, P, grid, s);
        case 64: return launch_indexer_t<64, 256, kPrefillIdxStages>(mq, mk, P, grid, s);
        }
    } else {
        switch (HI) {
        case 16: return launch_indexer_t<16, 16, kDecodeIdxStages>(mq, mk, P, grid, s);
        case 32: return launch_indexer_t<32, 32, kDecodeIdxStages>(mq, mk, P, grid, s);
        case 64: return launch_indexer_t<64, 64, kDecodeIdxStages>(mq, mk, P, grid, s);
        }
    }
    return DSA_ERR_UNSUPPORTED;
}

// ------------------------------------------------------------------ top-k launch
// Clusters of the top-k cluster kernel that fit on the device at once with `smem` bytes of
// dynamic shared memory per CTA (cached per device and size; 0 if the query fails).
int cluster_residency(int smem, cudaLaunchConfig_t cfg) {
    static std::mutex mu;
    static std::vector<std::pair<std::pair<int, int>, int>> cache;
    const int dev = current_device();
    std::lock_guard<std::mutex> lock(mu);
    for (const auto& e : cache)
        if (e.first.first == dev && e.first.second == smem) return e.second;
    cfg.dynamicSmemBytes = smem;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, topk_cluster_kernel, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        n = 0;
    }
    cache.push_back({{dev, smem}, n});
    return n;
}

dsa_status run_topk(const float* scores, int64_t ld, int rows, int64_t q_pos0, const int* ctx_len, int64_t n_max,
                    int k, int* idx, cudaStream_t s, int64_t window = 0) {
    TopkParams P{scores, ld, rows, q_pos0, ctx_len, n_max, k, idx, window};
    const int sms = num_sms();
    const int smem = (int)sizeof(TopkSmem);
    // Few long rows: a cluster of CTAs per row; otherwise one CTA per row.
    if ((long long)rows * kTkCluster <= 2LL * sms && n_max > 4LL * kTkCap) {
        static DeviceFlags cattr;
        if (!set_smem_limit(topk_cluster_kernel, kTkStageOffset + kTkStageMaxF4 * 16, cattr)) return DSA_ERR_CUDA;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(rows * kTkCluster);
        cfg.blockDim = dim3(kTkThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = kTkCluster;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        // Stage every CTA's segment in shared memory when the largest one fits and every cluster
        // of the launch is still co-resident with the larger footprint (one wave).
        const int64_t n4 = (n_max + 3) / 4;
        const int seg_f4 = (int)(((n4 + kTkCluster - 1) / kTkCluster + 31) & ~31LL);
        if (seg_f4 <= kTkStageMaxF4) {
            const int ssmem = kTkStageOffset + seg_f4 * 16;
            if (cluster_residency(ssmem, cfg) >= rows) {
                P.stage_f4 = seg_f4;
                cfg.dynamicSmemBytes = ssmem;
            }
        }
        LaunchScope ls(K_TOPK, s);
        if (cudaLaunchKernelEx(&cfg, topk_cluster_kernel, P) != cudaSuccess) return DSA_ERR_CUDA;
        return launch_status();
    }
    static DeviceFlags attr_set;
    if (!set_smem_limit(topk_kernel, smem, attr_set)) return DSA_ERR_CUDA;
    LaunchScope ls(K_TOPK, s);
    topk_kernel<<<rows, kTkThreads, smem, s>>>(P);
    return launch_status();
}

// ------------------------------------------------------------------ attention launch
template <int NT>
dsa_status launch_attn_t(const AttnParams& P, cudaStream_t s) {
    const int smem = attn_smem_bytes(P.Hkv, NT);
    auto kern = sparse_attn_kernel<NT>;
    static DeviceFlags attr_set;
    const int most = std::max(attn_smem_bytes(1, NT), std::max(attn_smem_bytes(2, NT), attn_smem_bytes(4, NT)));
    if (!set_smem_limit(kern, most, attr_set)) return DSA_ERR_CUDA;
    LaunchScope ls(K_ATTN, s);
    kern<<<P.T * P.nsplit, kAttnThreads, smem, s>>>(P);
    return launch_status();
}

// ------------------------------------------------------------------ dedup attention launch
// q bf16 [T][Hq][128] as a 3D map {128, Hq, T}; box {64, G, TBA}: the 128 (token, head) rows of one
// KV group and block, one 64-dim half per load, 128-byte swizzle.
bool make_dedup_q_map(CUtensorMap* m, const void* q, int T, int Hq, int G, int TBA) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)kAttnD, (cuuint64_t)Hq, (cuuint64_t)T};
    cuuint64_t strides[2] = {(cuuint64_t)kAttnD * 2, (cuuint64_t)Hq * kAttnD * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)G, (cuuint32_t)TBA};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int G>
dsa_status launch_dedup_t(const CUtensorMap& qm, const DedupParams& P, cudaStream_t s) {
    auto kern = attn_dedup_kernel<G>;
    static DeviceFlags attr_set;
    if (!set_smem_limit(kern, kDdSmemBytes, attr_set)) return DSA_ERR_CUDA;
    LaunchScope ls(K_ATTN, s);
    kern<<<P.nblk * P.Hkv, kDdThreads, kDdSmemBytes, s>>>(qm, P);
    return launch_status();
}

// Query heads per KV group the dedup kernel supports: 128 / G adjacent tokens fill one 128-row tile.
bool dedup_supported(int Hq, int Hkv) { return Hkv > 0 && Hq % Hkv == 0 && (Hq / Hkv == 8 || Hq / Hkv == 16); }

dsa_status run_attn_dedup(const void* q, DedupParams P, cudaStream_t s) {
    const int G = P.Hq / P.Hkv;
    const int TBA = kDdRows / G;
    P.nblk = (P.T + TBA - 1) / TBA;
    CUtensorMap qm;
    if (!make_dedup_q_map(&qm, q, P.T, P.Hq, G, TBA)) return DSA_ERR_CUDA;
    switch (G) {
    case 8: return launch_dedup_t<8>(qm, P, s);
    case 16: return launch_dedup_t<16>(qm, P, s);
    }
    return DSA_ERR_UNSUPPORTED;
}

// ------------------------------------------------------------------ warm-up KL launches
// k bf16 [Lk][Hkv][128] as a 3D map {128, Hkv, Lk}; box {64, 1, 128}: 128 keys of one KV group, one
// 64-dim half per load, 128-byte swizzle.
bool make_k_tile_map(CUtensorMap* m, const void* k, int64_t Lk, int Hkv) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)kAttnD, (cuuint64_t)Hkv, (cuuint64_t)Lk};
    cuuint64_t strides[2] = {(cuuint64_t)kAttnD * 2, (cuuint64_t)Hkv * kAttnD * 2};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)kKlKeys};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(k), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool kl_shape_supported(int Hq, int Hkv) {
    return (Hq == 8 || Hq == 16 || Hq == 32 || Hq == 64) && (Hkv == 1 || Hkv == 2 || Hkv == 4) && Hq % Hkv == 0 &&
           Hq / Hkv >= 2;
}

template <int G>
dsa_status launch_kl_lse_t(const CUtensorMap& qm, const CUtensorMap& km, const KlLseParams& P, cudaStream_t s) {
    auto kern = kl_lse_kernel<G>;
    static DeviceFlags attr_set;
    if (!set_smem_limit(kern, kKlLseSmem, attr_set)) return DSA_ERR_CUDA;
    LaunchScope ls(K_KL, s);
    kern<<<P.nblk * P.Hkv, kKlThreads, kKlLseSmem, s>>>(qm, km, P);
    return launch_status();
}

template <int HQ, int HKV>
dsa_status launch_kl_div_t(const CUtensorMap& qm, const CUtensorMap& km, const KlDivParams& P, cudaStream_t s) {
    auto kern = kl_div_kernel<HQ, HKV>;
    static DeviceFlags attr_set;
    if (!set_smem_limit(kern, kKlDivSmem, attr_set)) return DSA_ERR_CUDA;
    LaunchScope ls(K_KL, s);
    kern<<<P.nblk, kKlThreads, kKlDivSmem, s>>>(qm, km, P);
    return launch_status();
}

// Both passes for n query rows at positions t0 .. t0+n-1 whose indexer score rows are in `scores`.
dsa_status run_kl(const __nv_bfloat16* q, const void* k, const float* scores, int64_t ld, int n, int64_t t0, int Hq,
                  int Hkv, float scale, float* lse2, float* kl, cudaStream_t s) {
    const int G = Hq / Hkv;
    CUtensorMap km, qa, qb;
    if (!make_k_tile_map(&km, k, t0 + n, Hkv)) return DSA_ERR_CUDA;
    KlLseParams A{};
    A.T = n;
    A.q_pos0 = t0;
    A.Hq = Hq;
    A.Hkv = Hkv;
    A.scale_log2 = scale * 1.4426950408889634f;
    A.lse2 = lse2;
    A.nblk = (n + 128 / G - 1) / (128 / G);
    if (!make_dedup_q_map(&qa, q, n, Hq, G, 128 / G)) return DSA_ERR_CUDA;
    dsa_status st = DSA_ERR_UNSUPPORTED;
    switch (G) {
    case 2: st = launch_kl_lse_t<2>(qa, km, A, s); break;
    case 4: st = launch_kl_lse_t<4>(qa, km, A, s); break;
    case 8: st = launch_kl_lse_t<8>(qa, km, A, s); break;
    case 16: st = launch_kl_lse_t<16>(qa, km, A, s); break;
    case 32: st = launch_kl_lse_t<32>(qa, km, A, s); break;
    case 64: st = launch_kl_lse_t<64>(qa, km, A, s); break;
    }
    if (st != DSA_OK) return st;
    KlDivParams B{};
    B.scores = scores;
    B.ld = ld;
    B.T = n;
    B.q_pos0 = t0;
    B.scale_log2 = A.scale_log2;
    B.lse2 = lse2;
    B.kl = kl;
    const int TB = 256 / Hq;
    B.nblk = (n + TB - 1) / TB;
    if (!make_dedup_q_map(&qb, q, n, Hq, G, TB)) return DSA_ERR_CUDA;
#define DSA_KL_DIV(HQ_, HKV_) \
    if (Hq == HQ_ && Hkv == HKV_) return launch_kl_div_t<HQ_, HKV_>(qb, km, B, s);
    DSA_KL_DIV(8, 1) DSA_KL_DIV(8, 2) DSA_KL_DIV(8, 4)
    DSA_KL_DIV(16, 1) DSA_KL_DIV(16, 2) DSA_KL_DIV(16, 4)
    DSA_KL_DIV(32, 1) DSA_KL_DIV(32, 2) DSA_KL_DIV(32, 4)
    DSA_KL_DIV(64, 1) DSA_KL_DIV(64, 2) DSA_KL_DIV(64, 4)
#undef DSA_KL_DIV
    return DSA_ERR_UNSUPPORTED;
}

dsa_status run_attn(const AttnParams& P, cudaStream_t s) {
    const int G = P.Hq / P.Hkv;
    if (G <= 8) return launch_attn_t<1>(P, s);
    return launch_attn_t<2>(P, s);
}

// ------------------------------------------------------------------ decode helpers
// Sequences whose ctx_len is out of range must not be read past the caches by the other kernels;
// the indexer, top-k and attention kernels clamp their key counts to the cache capacity, and the
// indexer (which appends the new token) reports the bad input.

__global__ void selftest_timeout_kernel(unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // nothing ever arrives on `bar`: the wait must end by its time limit
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(&bar, 0)) {
            if (globaltimer_ns() - t0 > limit_ns) {
                record_error(DSA_DEV_ERR_TIMEOUT, 0x901);
                break;
            }
        }
    }
}

// Key splits per sequence for the decode attention: enough CTAs for two per SM (the kernel's
// residency), so every SM keeps two rings of K/V copies in flight.
int decode_attn_splits(int B) {
    const int sms = std::max(1, num_sms());
    return std::max(1, std::min(kMaxDecodeSplits, 2 * sms / std::max(1, B)));
}

struct DecodeWs {
    size_t scores, idx, part, total;
};
DecodeWs decode_ws_layout(int64_t Lmax, int B, int Hq, int topk, bool need_idx) {
    DecodeWs w{};
    const int64_t ld = (int64_t)align_up((size_t)Lmax, 4);
    w.scores = 0;
    size_t off = align_up((size_t)B * ld * 4, 256);
    w.idx = off;
    if (need_idx) off = align_up(off + (size_t)B * topk * 4, 256);
    w.part = off;
    off = align_up(off + (size_t)B * kMaxDecodeSplits * Hq * kAttnPartStride * 4, 256);
    w.total = off;
    return w;
}

int64_t prefill_ld(int64_t L) { return (int64_t)align_up((size_t)L, 4); }

// Bytes of a chunk of C query rows: C score rows of ld floats, then (idx_per_row > 0) C index
// rows starting at a 256-byte boundary.
size_t chunk_bytes(int64_t C, int64_t ld, int64_t idx_per_row) {
    return align_up((size_t)C * ld * 4, 256) + (size_t)C * idx_per_row * 4;
}

// Query rows per chunk for a workspace of ws_bytes laid out as chunk_bytes says: the most that
// fit, whole query blocks of TB rows unless the chunk covers every remaining row.  0 = too small.
int64_t chunk_rows(size_t ws_bytes, int64_t ld, int64_t idx_per_row, int64_t rows, int TB) {
    const size_t per_row = (size_t)(ld + idx_per_row) * 4;
    int64_t C = std::min<int64_t>(rows, (int64_t)(ws_bytes / per_row));
    while (C > 0 && chunk_bytes(C, ld, idx_per_row) > ws_bytes) --C;
    if (C < rows && C >= TB) C = C / TB * TB;
    return C;
}

}  // namespace

// ------------------------------------------------------------------ allocation-free decode
// Scratch of dsa_decode_noalloc: a fixed array in the library's own device memory.  Every GPU on
// which the library is loaded holds it until the process exits.  Host code must not pass the
// array's name to a kernel (on the host it is only a stand-in for the symbol); its device
// address is looked up once per device with cudaGetSymbolAddress.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up on first use).
dsa_status noalloc_scratch(void** out) {
    const int dev = current_device();
    if (dev < 0) return DSA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return DSA_ERR_CUDA;
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return DSA_OK;
}

// ====================================================================== C ABI
extern "C" {

const char* dsa_status_string(int status) {
    switch (status) {
    case DSA_OK: return "DSA_OK";
    case DSA_ERR_INVALID_ARG: return "DSA_ERR_INVALID_ARG: invalid argument (null/misaligned pointer or bad size)";
    case DSA_ERR_UNSUPPORTED: return "DSA_ERR_UNSUPPORTED: shape outside the supported set";
    case DSA_ERR_WORKSPACE: return "DSA_ERR_WORKSPACE: workspace missing or too small";
    case DSA_ERR_CUDA: return "DSA_ERR_CUDA: a CUDA call or kernel launch failed";
    case DSA_ERR_TIMEOUT: return "DSA_ERR_TIMEOUT: a kernel's bounded wait expired";
    case DSA_ERR_DEVICE_INPUT: return "DSA_ERR_DEVICE_INPUT: a device-side input check failed";
    default: return "DSA_ERR_UNKNOWN";
    }
}

int dsa_version(void) { return kVersion; }

dsa_status dsa_index(const void* qI, const void* kI, const void* w, int Lq, int64_t Lk, int HI, int dI,
                     int64_t q_pos0, float* scores, int64_t ld_scores, dsa_stream_t stream) {
    if (!qI || !kI || !w || !scores) return DSA_ERR_INVALID_ARG;
    if (!aligned16(qI) || !aligned16(kI) || !aligned16(w) || !aligned16(scores)) return DSA_ERR_INVALID_ARG;
    if (Lq <= 0 || Lk <= 0 || HI <= 0 || dI <= 0 || q_pos0 < 0) return DSA_ERR_INVALID_ARG;
    if (q_pos0 + Lq > Lk || ld_scores < q_pos0 + Lq || ld_scores % 4 != 0) return DSA_ERR_INVALID_ARG;
    if (dI != kIdxBK || !hi_supported_prefill(HI)) return DSA_ERR_UNSUPPORTED;
    if ((int64_t)Lq * HI > (int64_t)INT32_MAX || Lk > (int64_t)INT32_MAX) return DSA_ERR_UNSUPPORTED;
    return run_indexer(qI, kI, static_cast<const __nv_bfloat16*>(w), 1, Lq, q_pos0, nullptr, Lk, HI, scores,
                       ld_scores, reinterpret_cast<cudaStream_t>(stream));
}

dsa_status dsa_topk_window(const float* scores, int64_t ld_scores, int Lq, int64_t q_pos0, int k, int64_t window,
                           int32_t* idx, dsa_stream_t stream) {
    if (!scores || !idx) return DSA_ERR_INVALID_ARG;
    if (!aligned16(scores) || !aligned16(idx)) return DSA_ERR_INVALID_ARG;
    if (Lq <= 0 || q_pos0 < 0 || ld_scores % 4 != 0 || ld_scores < q_pos0 + Lq) return DSA_ERR_INVALID_ARG;
    if (k <= 0 || window < 0) return DSA_ERR_INVALID_ARG;
    if (k > kMaxTopk || q_pos0 + Lq > (int64_t)INT32_MAX) return DSA_ERR_UNSUPPORTED;
    return run_topk(scores, ld_scores, Lq, q_pos0, nullptr, q_pos0 + Lq, k, idx,
                    reinterpret_cast<cudaStream_t>(stream), window);
}

dsa_status dsa_topk(const float* scores, int64_t ld_scores, int Lq, int64_t q_pos0, int k, int32_t* idx, void* ws,
                    size_t ws_bytes, dsa_stream_t stream) {
    (void)ws;
    (void)ws_bytes;
    return dsa_topk_window(scores, ld_scores, Lq, q_pos0, k, 0, idx, stream);
}

dsa_status dsa_sparse_attn(const void* q, const void* k, const void* v, const int32_t* idx, int Lq, int64_t Lk,
                           int64_t q_pos0, int Hq, int Hkv, int D, int topk, float scale, void* out, float* lse,
                           dsa_stream_t stream) {
    if (!q || !k || !v || !idx || !out) return DSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(out))
        return DSA_ERR_INVALID_ARG;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return DSA_ERR_INVALID_ARG;
    if (Lq <= 0 || Lk <= 0 || q_pos0 < 0 || topk <= 0 || !(scale == scale)) return DSA_ERR_INVALID_ARG;
    dsa_status st = check_attn_shape(Hq, Hkv, D);
    if (st != DSA_OK) return st;
    if (topk > kMaxTopk || Lk > (int64_t)INT32_MAX) return DSA_ERR_UNSUPPORTED;
    AttnParams P{};
    P.q = static_cast<const __nv_bfloat16*>(q);
    P.k = static_cast<const __nv_bfloat16*>(k);
    P.v = static_cast<const __nv_bfloat16*>(v);
    P.kv_bstride = 0;
    P.idx = idx;
    P.topk = topk;
    P.T = Lq;
    P.q_pos0 = q_pos0;
    P.ctx_len = nullptr;
    P.n_keys = Lk;
    P.Hq = Hq;
    P.Hkv = Hkv;
    P.scale_log2 = scale * 1.4426950408889634f;
    P.out = static_cast<__nv_bfloat16*>(out);
    P.lse = lse;
    P.nsplit = 1;
    P.part = nullptr;
    return run_attn(P, reinterpret_cast<cudaStream_t>(stream));
}

dsa_status dsa_sparse_attn_dedup(const void* q, const void* k, const void* v, const int32_t* idx, int Lq, int64_t Lk,
                                 int64_t q_pos0, int Hq, int Hkv, int D, int topk, float scale, void* out, float* lse,
                                 dsa_stream_t stream) {
    if (!q || !k || !v || !idx || !out) return DSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(out))
        return DSA_ERR_INVALID_ARG;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return DSA_ERR_INVALID_ARG;
    if (Lq <= 0 || Lk <= 0 || q_pos0 < 0 || topk <= 0 || !(scale == scale)) return DSA_ERR_INVALID_ARG;
    dsa_status st = check_attn_shape(Hq, Hkv, D);
    if (st != DSA_OK) return st;
    if (!dedup_supported(Hq, Hkv) || topk > kMaxTopk || Lk > (int64_t)kDdMaxWin * kDdWin)
        return DSA_ERR_UNSUPPORTED;
    DedupParams P{};
    P.k = static_cast<const __nv_bfloat16*>(k);
    P.v = static_cast<const __nv_bfloat16*>(v);
    P.idx = idx;
    P.topk = topk;
    P.T = Lq;
    P.q_pos0 = q_pos0;
    P.n_keys = Lk;
    P.window = 0;
    P.Hq = Hq;
    P.Hkv = Hkv;
    P.scale_log2 = scale * 1.4426950408889634f;
    P.out = static_cast<__nv_bfloat16*>(out);
    P.lse = lse;
    return run_attn_dedup(q, P, reinterpret_cast<cudaStream_t>(stream));
}

size_t dsa_workspace_size(int op, int64_t L, int B, int Hq, int HI, int topk) {
    if (op == DSA_OP_INDEXER_KL) {  // score rows and per-head log-sum-exps of a chunk (topk unused)
        if (L <= 0 || HI <= 0 || Hq <= 0) return 0;
        const int64_t ld = prefill_ld(L);
        int64_t rows = (int64_t(4) << 30) / (ld * 4);
        rows = std::max<int64_t>(256, rows / 256 * 256);
        rows = std::min<int64_t>(rows, L);
        return align_up(chunk_bytes(rows, ld, Hq), 256);
    }
    if (L <= 0 || topk <= 0 || HI <= 0) return 0;
    switch (op) {
    case DSA_OP_INDEX:
    case DSA_OP_TOPK:
    case DSA_OP_SPARSE_ATTN: return 0;
    case DSA_OP_PREFILL: {
        // score rows of up to 16 GiB per chunk: fewer, longer chunks shorten every kernel's
        // per-launch tail (128K: 1.32 M tokens/s at 8192-row chunks, 1.38 M at 16384 or 32768;
        // 256K: 0.82 M at 4096, 0.86 M at 8192, 0.87 M at 16384)
        const int64_t ld = prefill_ld(L);
        int64_t rows = (int64_t(16) << 30) / (ld * 4);
        rows = std::max<int64_t>(256, rows / 256 * 256);
        rows = std::min<int64_t>(rows, L);
        return align_up(chunk_bytes(rows, ld, topk), 256);
    }
    case DSA_OP_DECODE:
        if (B <= 0 || Hq <= 0) return 0;
        return decode_ws_layout(L, B, Hq, topk, true).total;
    default: return 0;
    }
}

dsa_status dsa_indexer_kl(const void* q, const void* k, const void* qI, const void* kI, const void* w, int64_t L,
                          int Hq, int Hkv, int D, int HI, int dI, float scale, float* kl, void* ws, size_t ws_bytes,
                          dsa_stream_t stream) {
    if (!q || !k || !qI || !kI || !w || !kl) return DSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(qI) || !aligned16(kI) || !aligned16(w) ||
        (reinterpret_cast<uintptr_t>(kl) & 3u))
        return DSA_ERR_INVALID_ARG;
    if (L <= 0 || HI <= 0 || dI <= 0 || !(scale == scale)) return DSA_ERR_INVALID_ARG;
    dsa_status st = check_attn_shape(Hq, Hkv, D);
    if (st != DSA_OK) return st;
    if (!kl_shape_supported(Hq, Hkv) || dI != kIdxBK || !hi_supported_prefill(HI) || L * HI > (int64_t)INT32_MAX)
        return DSA_ERR_UNSUPPORTED;
    if (!ws || !aligned16(ws)) return DSA_ERR_WORKSPACE;
    const int64_t ld = prefill_ld(L);
    // chunks of whole blocks of every kernel (indexer 256/HI, pass 1 128/G, pass 2 256/Hq rows), so
    // that a row's arithmetic does not depend on the chunk size
    const int TB = std::max(indexer_tb(HI, false), 128);
    const int64_t C = chunk_rows(ws_bytes, ld, Hq, L, TB);
    if (C < std::min<int64_t>(L, TB)) return DSA_ERR_WORKSPACE;
    float* scores = static_cast<float*>(ws);
    float* lse2 = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + align_up((size_t)C * ld * 4, 256));
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    for (int64_t t0 = 0; t0 < L; t0 += C) {
        const int n = (int)std::min<int64_t>(C, L - t0);
        st = run_indexer(static_cast<const __nv_bfloat16*>(qI) + t0 * HI * dI, kI,
                         static_cast<const __nv_bfloat16*>(w) + t0 * HI, 1, n, t0, nullptr, t0 + n, HI, scores, ld, s);
        if (st != DSA_OK) return st;
        st = run_kl(static_cast<const __nv_bfloat16*>(q) + t0 * Hq * D, k, scores, ld, n, t0, Hq, Hkv, scale, lse2,
                    kl + t0, s);
        if (st != DSA_OK) return st;
    }
    return DSA_OK;
}

dsa_status dsa_prefill_rows(const void* q, const void* k, const void* v, const void* qI, const void* kI,
                            const void* w, int64_t row0, int64_t rows, int Hq, int Hkv, int D, int HI, int dI,
                            int topk, int64_t window, float scale, void* out, int32_t* idx_out, void* ws,
                            size_t ws_bytes, dsa_stream_t stream) {
    if (!q || !k || !v || !qI || !kI || !w || !out) return DSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(qI) || !aligned16(kI) || !aligned16(w) ||
        !aligned16(out) || (idx_out && !aligned16(idx_out)))
        return DSA_ERR_INVALID_ARG;
    if (row0 < 0 || rows <= 0 || topk <= 0 || HI <= 0 || dI <= 0 || window < 0 || !(scale == scale))
        return DSA_ERR_INVALID_ARG;
    dsa_status st = check_attn_shape(Hq, Hkv, D);
    if (st != DSA_OK) return st;
    const int64_t Lk = row0 + rows;  // keys the last row needs
    if (dI != kIdxBK || !hi_supported_prefill(HI) || topk > kMaxTopk || Lk * HI > (int64_t)INT32_MAX)
        return DSA_ERR_UNSUPPORTED;
    if (!ws || !aligned16(ws)) return DSA_ERR_WORKSPACE;
    const int64_t ld = prefill_ld(Lk);
    const int TB = indexer_tb(HI, false);
    const int64_t ipr = idx_out ? 0 : topk;
    const int64_t C = chunk_rows(ws_bytes, ld, ipr, rows, TB);
    if (C < std::min<int64_t>(rows, TB)) return DSA_ERR_WORKSPACE;
    float* scores = static_cast<float*>(ws);
    int32_t* idx_ws = idx_out ? nullptr
                              : reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) +
                                                           align_up((size_t)C * ld * 4, 256));
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const auto* qb = static_cast<const __nv_bfloat16*>(q);
    const auto* qIb = static_cast<const __nv_bfloat16*>(qI);
    const auto* wb = static_cast<const __nv_bfloat16*>(w);
    auto* ob = static_cast<__nv_bfloat16*>(out);
    for (int64_t c0 = 0; c0 < rows; c0 += C) {   // c0: offset inside the row range
        const int n = (int)std::min<int64_t>(C, rows - c0);
        const int64_t t0 = row0 + c0;            // absolute position of the chunk's first row
        int32_t* idx_c = idx_out ? idx_out + c0 * topk : idx_ws;
        st = run_indexer(qIb + c0 * HI * dI, kI, wb + c0 * HI, 1, n, t0, nullptr, t0 + n, HI, scores, ld, s, window);
        if (st != DSA_OK) return st;
        st = run_topk(scores, ld, n, t0, nullptr, t0 + n, topk, idx_c, s, window);
        if (st != DSA_OK) return st;
        AttnParams P{};
        P.q = qb + c0 * Hq * D;
        P.k = static_cast<const __nv_bfloat16*>(k);
        P.v = static_cast<const __nv_bfloat16*>(v);
        P.idx = idx_c;
        P.topk = topk;
        P.T = n;
        P.q_pos0 = t0;
        P.n_keys = Lk;
        P.Hq = Hq;
        P.Hkv = Hkv;
        P.scale_log2 = scale * 1.4426950408889634f;
        P.out = ob + c0 * Hq * D;
        P.nsplit = 1;
        P.window = window;
        st = run_attn(P, s);
        if (st != DSA_OK) return st;
    }
    return DSA_OK;
}

dsa_status dsa_prefill_window(const void* q, const void* k, const void* v, const void* qI, const void* kI,
                              const void* w, int64_t L, int Hq, int Hkv, int D, int HI, int dI, int topk,
                              int64_t window, float scale, void* out, int32_t* idx_out, void* ws, size_t ws_bytes,
                              dsa_stream_t stream) {
    if (L <= 0) return DSA_ERR_INVALID_ARG;
    return dsa_prefill_rows(q, k, v, qI, kI, w, 0, L, Hq, Hkv, D, HI, dI, topk, window, scale, out, idx_out, ws,
                            ws_bytes, stream);
}

dsa_status dsa_prefill(const void* q, const void* k, const void* v, const void* qI, const void* kI, const void* w,
                       int64_t L, int Hq, int Hkv, int D, int HI, int dI, int topk, float scale, void* out,
                       int32_t* idx_out, void* ws, size_t ws_bytes, dsa_stream_t stream) {
    return dsa_prefill_window(q, k, v, qI, kI, w, L, Hq, Hkv, D, HI, dI, topk, 0, scale, out, idx_out, ws, ws_bytes,
                              stream);
}

}  // extern "C"

namespace {
// Host-side checks of a decode step's arguments (everything except the workspace).
dsa_status check_decode_args(const void* q, const void* qI, const void* w, const void* k_new, const void* v_new,
                             const void* kI_new, const void* k_cache, const void* v_cache, const void* kI_cache,
                             const int32_t* ctx_len, int B, int64_t Lmax, int Hq, int Hkv, int D, int HI, int dI,
                             int topk, float scale, const void* out, const int32_t* idx_out) {
    const void* ptrs[] = {q, qI, w, k_new, v_new, kI_new, k_cache, v_cache, kI_cache, ctx_len, out};
    for (const void* p : ptrs)
        if (!p || !aligned16(p)) return DSA_ERR_INVALID_ARG;
    if (idx_out && !aligned16(idx_out)) return DSA_ERR_INVALID_ARG;
    if (B <= 0 || Lmax <= 0 || topk <= 0 || HI <= 0 || dI <= 0 || !(scale == scale)) return DSA_ERR_INVALID_ARG;
    dsa_status st = check_attn_shape(Hq, Hkv, D);
    if (st != DSA_OK) return st;
    if (dI != kIdxBK || !hi_supported_decode(HI) || topk > kMaxTopk || Lmax > (int64_t)INT32_MAX)
        return DSA_ERR_UNSUPPORTED;
    return DSA_OK;
}
}  // namespace

extern "C" {

dsa_status dsa_decode(const void* q, const void* qI, const void* w, const void* k_new, const void* v_new,
                      const void* kI_new, void* k_cache, void* v_cache, void* kI_cache, int32_t* ctx_len, int B,
                      int64_t Lmax, int Hq, int Hkv, int D, int HI, int dI, int topk, float scale, int update_ctx,
                      void* out, int32_t* idx_out, void* ws, size_t ws_bytes, dsa_stream_t stream) {
    dsa_status st = check_decode_args(q, qI, w, k_new, v_new, kI_new, k_cache, v_cache, kI_cache, ctx_len, B, Lmax,
                                      Hq, Hkv, D, HI, dI, topk, scale, out, idx_out);
    if (st != DSA_OK) return st;
    const DecodeWs L = decode_ws_layout(Lmax, B, Hq, topk, idx_out == nullptr);
    if (!ws || !aligned16(ws)) return DSA_ERR_WORKSPACE;
    if (ws_bytes < L.total) return DSA_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    float* scores = reinterpret_cast<float*>(wsb + L.scores);
    int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(wsb + L.idx);
    float* part = reinterpret_cast<float*>(wsb + L.part);
    const int64_t ld = (int64_t)align_up((size_t)Lmax, 4);
    // the indexer appends the new tokens' K, V and kI rows to the caches (ahead of its own loads)
    IndexerParams app{};
    app.new_k = static_cast<const uint4*>(k_new);
    app.new_v = static_cast<const uint4*>(v_new);
    app.new_kI = static_cast<const uint4*>(kI_new);
    app.cache_k = static_cast<uint4*>(k_cache);
    app.cache_v = static_cast<uint4*>(v_cache);
    app.cache_kI = static_cast<uint4*>(kI_cache);
    app.kv16 = Hkv * D / 8;
    app.kI16 = dI / 8;
    st = run_indexer(qI, kI_cache, static_cast<const __nv_bfloat16*>(w), B, 1, 0, ctx_len, Lmax, HI, scores, ld, s, 0,
                     &app);
    if (st != DSA_OK) return st;
    st = run_topk(scores, ld, B, 0, ctx_len, Lmax, topk, idx, s);
    if (st != DSA_OK) return st;
    AttnParams P{};
    P.q = static_cast<const __nv_bfloat16*>(q);
    P.k = static_cast<const __nv_bfloat16*>(k_cache);
    P.v = static_cast<const __nv_bfloat16*>(v_cache);
    P.kv_bstride = Lmax * Hkv * D;
    P.idx = idx;
    P.topk = topk;
    P.T = B;
    P.ctx_len = ctx_len;
    P.n_keys = Lmax;
    P.Hq = Hq;
    P.Hkv = Hkv;
    P.scale_log2 = scale * 1.4426950408889634f;
    P.out = static_cast<__nv_bfloat16*>(out);
    P.nsplit = decode_attn_splits(B);
    P.part = part;
    P.advance_ctx = (update_ctx && P.nsplit == 1) ? ctx_len : nullptr;
    st = run_attn(P, s);
    if (st != DSA_OK) return st;
    if (P.nsplit > 1) {
        LaunchScope ls(K_COMBINE, s);
        const int warps = B * Hq;
        attn_combine_kernel<<<(warps + 3) / 4, 128, 0, s>>>(part, B, P.nsplit, Hq, P.out, nullptr,
                                                            update_ctx ? ctx_len : nullptr, Lmax);
        if ((st = launch_status()) != DSA_OK) return st;
    }
    return DSA_OK;
}

dsa_status dsa_decode_noalloc(const void* q, const void* qI, const void* w, const void* k_new, const void* v_new,
                              const void* kI_new, void* k_cache, void* v_cache, void* kI_cache, int32_t* ctx_len, int B,
                              int64_t Lmax, int Hq, int Hkv, int D, int HI, int dI, int topk, float scale,
                              int update_ctx, void* out, int32_t* idx_out, dsa_stream_t stream) {
    // The same checks and work as dsa_decode, with its workspace in the library's fixed scratch
    // array: argument errors are reported exactly as dsa_decode reports them, and only a valid
    // step that needs more scratch than the array holds gets DSA_ERR_WORKSPACE.
    dsa_status st0 = check_decode_args(q, qI, w, k_new, v_new, kI_new, k_cache, v_cache, kI_cache, ctx_len, B, Lmax,
                                       Hq, Hkv, D, HI, dI, topk, scale, out, idx_out);
    if (st0 != DSA_OK) return st0;
    if (decode_ws_layout(Lmax, B, Hq, topk, idx_out == nullptr).total > kNoAllocScratchBytes)
        return DSA_ERR_WORKSPACE;
    void* scratch = nullptr;
    dsa_status st = noalloc_scratch(&scratch);
    if (st != DSA_OK) return st;
    return dsa_decode(q, qI, w, k_new, v_new, kI_new, k_cache, v_cache, kI_cache, ctx_len, B, Lmax, Hq, Hkv, D, HI,
                      dI, topk, scale, update_ctx, out, idx_out, scratch, kNoAllocScratchBytes, stream);
}

size_t dsa_decode_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

dsa_status dsa_sync_status(dsa_stream_t stream) {
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return DSA_ERR_CUDA;
    if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
    unsigned int err = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&err, g_dev_error, sizeof(err)) != cudaSuccess) return DSA_ERR_CUDA;
    if (err) {
        if (cudaMemcpyToSymbol(g_dev_error, &zero, sizeof(zero)) != cudaSuccess) return DSA_ERR_CUDA;
    }
    if (err & DSA_DEV_ERR_TIMEOUT) return DSA_ERR_TIMEOUT;
    if (err & DSA_DEV_ERR_BOUNDS) return DSA_ERR_DEVICE_INPUT;
    return DSA_OK;
}

unsigned int dsa_error_site(void) {
    unsigned int where = 0;
    if (cudaMemcpyFromSymbol(&where, g_dev_error_where, sizeof(where)) != cudaSuccess) return 0;
    return where;
}

void dsa_profile_begin(void) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    for (auto& r : g_prof_recs) {
        g_event_pool.push_back(r.a);
        g_event_pool.push_back(r.b);
    }
    g_prof_recs.clear();
    g_prof_on = true;
}

dsa_status dsa_profile_end(int64_t* launches, double* total_ms) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_on = false;
    dsa_status st = DSA_OK;
    for (int i = 0; i < DSA_PROFILE_KINDS; ++i) {
        if (launches) launches[i] = 0;
        if (total_ms) total_ms[i] = 0.0;
    }
    for (auto& r : g_prof_recs) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) {
            st = DSA_ERR_CUDA;
            continue;
        }
        if (launches) launches[r.kind] += 1;
        if (total_ms) total_ms[r.kind] += ms;
    }
    for (auto& r : g_prof_recs) {
        g_event_pool.push_back(r.a);
        g_event_pool.push_back(r.b);
    }
    g_prof_recs.clear();
    return st;
}

int64_t dsa_launch_count(void) { return g_launches.load(); }

dsa_status dsa_read_counters(int64_t* out, int n, int reset) {
    if (!out || n < 0 || n > DSA_NUM_COUNTERS) return DSA_ERR_INVALID_ARG;
    unsigned long long c[DSA_NUM_COUNTERS] = {};
    if (cudaDeviceSynchronize() != cudaSuccess) return DSA_ERR_CUDA;
    if (cudaMemcpyFromSymbol(c, g_counters, sizeof(c)) != cudaSuccess) return DSA_ERR_CUDA;
    for (int i = 0; i < n; ++i) out[i] = (int64_t)c[i];
    if (reset) {
        unsigned long long z[DSA_NUM_COUNTERS] = {};
        if (cudaMemcpyToSymbol(g_counters, z, sizeof(z)) != cudaSuccess) return DSA_ERR_CUDA;
    }
    return DSA_OK;
}

dsa_status dsa_selftest_timeout(int64_t wait_ns, dsa_stream_t stream) {
    if (wait_ns <= 0 || wait_ns > 2000000000ll) return DSA_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    LaunchScope ls(K_SELFTEST, s);
    selftest_timeout_kernel<<<1, 32, 0, s>>>((unsigned long long)wait_ns);
    return launch_status();
}

}  // extern "C"
