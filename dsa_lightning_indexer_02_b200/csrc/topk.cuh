// Per-row top-k of indexer scores: the min(k, n) keys with the largest score, ties to the lower
// key index, written as int32 key indices followed by -1 padding.
//
// The pages keep the 2048 best-scored positions per token (page "快手开源大模型Keye-VL-2.0：
// 一个能“看懂“两小时视频AI", gsyq.cn, section 一) and require a deterministic top-k so that
// training and inference select the same keys (same page, section 八).  This kernel is exact
// and deterministic: the output of a row depends only on the row's scores.
//
// One CTA per row, order-preserving 32-bit keys (larger score -> larger key).
// Fast path (one HBM read of the row):
//   sample   256 evenly spaced float4 of the row give an estimate T0 of the key at rank ~2k
//            (rows with n <= 8192 skip this: T0 = 0 keeps every key);
//   collect  stream the row once; keys >= T0 are compacted, in index order, into a shared
//            candidate list through block scans;
//   refine   if the list holds at least k and at most 8192 keys it contains the exact top-k:
//            radix rounds over the candidates' offsets from T0 (first round scaled to the key
//            range, so the bins spread evenly) find the exact k-th key tau and the number of
//            keys equal to tau to take; an ordered scan emits keys > tau and the first keys
//            == tau.  Output order: ascending key index.
// Fallback (the estimate missed): a two-pass radix select over the row -- histogram of the top
// 12 bits, then keys above the threshold bin are written in index order and the bin's keys are
// collected (or, past the buffer, re-read from memory) and refined the same way.
#pragma once

#include <cooperative_groups.h>

#include "ptx.cuh"

namespace dsa {

constexpr int kTopkThreads = 512;
constexpr int kTopkCap = 8192;   // candidate list capacity (shared memory)
constexpr int kTopkSampleVec = 256;  // float4 samples per row for the threshold estimate
constexpr int kTopkUnroll = 4;       // float4 loads in flight per thread
constexpr int kTopkBins = 4096;

struct TopkParams {
    const float* scores;     // row r at scores + r*ld (16-byte aligned rows)
    long long ld;
    int rows;
    long long q_pos0;        // prefill: row r has n = q_pos0 + r + 1 keys
    const int* ctx_len;      // decode: row r has n = ctx_len[r] + 1 keys (null for prefill)
    long long n_max;         // upper bound on n (keys addressable in a row)
    int k;
    int* idx;                // [rows, k]
};

// Order-preserving map float -> uint32 (larger float -> larger key); -0 is folded onto +0 so
// that the two zeros tie exactly as they do in real arithmetic.
__device__ __forceinline__ uint32_t score_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct TopkShared {
    uint32_t hist[kTopkBins];
    uint32_t cand_key[kTopkCap];
    int cand_idx[kTopkCap];
    uint32_t warp_sum[2][kTopkThreads / 32];
    uint32_t sel_bin, sel_gt;  // result of a threshold search
    uint32_t red[kTopkThreads / 32];
};

// Exclusive prefix sum over the block of a packed counter; returns the block total.  `buf`
// alternates between calls so that one __syncthreads per scan suffices.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t& total, uint32_t* warp_sum) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sum[warp] = x;
    __syncthreads();
    uint32_t before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kTopkThreads / 32; ++w) {
        const uint32_t s = warp_sum[w];
        before += (w < warp) ? s : 0u;
        tot += s;
    }
    total = tot;
    return before + x - v;
}

// Find bin b with (count of bins above b) < need <= (count above b) + hist[b].  Bins [0, nbins).
__device__ __forceinline__ void find_threshold_bin(TopkShared& S, int nbins, uint32_t need, int& scan_buf) {
    const int per = nbins >= kTopkThreads ? nbins / kTopkThreads : 1;
    const int lo = threadIdx.x * per;
    uint32_t mine = 0;
    if (lo < nbins)
        for (int b = 0; b < per; ++b) mine += S.hist[lo + b];
    // suffix sums: scan on reversed thread order
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_down_sync(0xffffffffu, x, o);
        if (lane + o < 32) x += y;
    }
    uint32_t* ws = S.warp_sum[scan_buf];
    scan_buf ^= 1;
    if (lane == 0) ws[warp] = x;
    __syncthreads();
    uint32_t above = x - mine;  // bins of later lanes in this warp
#pragma unroll
    for (int w = 0; w < kTopkThreads / 32; ++w) above += (w > warp) ? ws[w] : 0u;
    if (lo < nbins && above < need && need <= above + mine) {
        uint32_t cum = above;
        for (int b = lo + per - 1; b >= lo; --b) {
            const uint32_t h = S.hist[b];
            if (cum + h >= need) {
                S.sel_bin = (uint32_t)b;
                S.sel_gt = cum;
                break;
            }
            cum += h;
        }
    }
    __syncthreads();
}

__device__ __forceinline__ void clear_hist(TopkShared& S, int nbins) {
    for (int b = threadIdx.x; b < nbins; b += kTopkThreads) S.hist[b] = 0;
}

// Items of a refinement round: either the shared-memory candidate list or the global row
// filtered to the threshold bin of pass 1.
struct CandSource {
    const TopkShared* S;
    int m;
    __device__ __forceinline__ int count() const { return m; }
    __device__ __forceinline__ bool get(int e, uint32_t& key, int& idx) const {
        if (e >= m) return false;
        key = S->cand_key[e];
        idx = S->cand_idx[e];
        return true;
    }
};
struct RowSource {
    const float* row;
    int n;
    uint32_t b0;
    __device__ __forceinline__ int count() const { return n; }
    __device__ __forceinline__ bool get(int e, uint32_t& key, int& idx) const {
        if (e >= n) return false;
        key = score_key(row[e]);
        idx = e;
        return (key >> 20) == b0;
    }
};

template <class Src>
__device__ __forceinline__ void refine_round(TopkShared& S, const Src& src, int shift, int width, uint32_t pmask,
                                             uint32_t pval, uint32_t& need, uint32_t& out_bin, int& scan_buf) {
    const int nbins = 1 << width;
    clear_hist(S, nbins);
    __syncthreads();
    for (int e = threadIdx.x; e < src.count(); e += kTopkThreads) {
        uint32_t key;
        int idx;
        if (src.get(e, key, idx) && (key & pmask) == pval) atomicAdd(&S.hist[(key >> shift) & (nbins - 1)], 1u);
    }
    __syncthreads();
    find_threshold_bin(S, nbins, need, scan_buf);
    out_bin = S.sel_bin;
    need -= S.sel_gt;
}

// Emit, in source order, items with key > tau and the first `ties` items with key == tau.
template <class Src>
__device__ __forceinline__ void emit_final(TopkShared& S, const Src& src, uint32_t tau, uint32_t ties, int* out,
                                           uint32_t out_base, int& scan_buf) {
    uint32_t gt_seen = 0, eq_seen = 0;
    const int cnt = src.count();
    for (int e0 = 0; e0 < cnt; e0 += kTopkThreads) {
        const int e = e0 + threadIdx.x;
        uint32_t key = 0;
        int idx = 0;
        const bool in = src.get(e, key, idx);
        const uint32_t gt = (in && key > tau) ? 1u : 0u;
        const uint32_t eq = (in && key == tau) ? 1u : 0u;
        uint32_t total;
        const uint32_t ex = block_excl_scan(gt | (eq << 16), total, S.warp_sum[scan_buf]);
        scan_buf ^= 1;
        const uint32_t eq_before = eq_seen + (ex >> 16);
        if (gt || (eq && eq_before < ties)) {
            const uint32_t pos = out_base + gt_seen + (ex & 0xFFFFu) + min(eq_before, ties);
            out[pos] = idx;
        }
        gt_seen += total & 0xFFFFu;
        eq_seen += total >> 16;
    }
}

// Two-pass radix select over the global row (the fallback path).
__device__ __noinline__ void topk_two_pass(TopkShared& S, const float* row, int n, int k, int* out, int& scan_buf) {
    const int tid = threadIdx.x;
    const float4* row4 = reinterpret_cast<const float4*>(row);
    // ---- pass 1: histogram of the top 12 key bits
    clear_hist(S, kTopkBins);
    __syncthreads();
    const int n4 = (n + 3) >> 2;
    for (int g = tid; g < n4; g += kTopkThreads) {
        const float4 v = row4[g];
        const int e = g * 4;
        atomicAdd(&S.hist[score_key(v.x) >> 20], 1u);
        if (e + 1 < n) atomicAdd(&S.hist[score_key(v.y) >> 20], 1u);
        if (e + 2 < n) atomicAdd(&S.hist[score_key(v.z) >> 20], 1u);
        if (e + 3 < n) atomicAdd(&S.hist[score_key(v.w) >> 20], 1u);
    }
    __syncthreads();
    find_threshold_bin(S, kTopkBins, (uint32_t)k, scan_buf);
    const uint32_t b0 = S.sel_bin;
    const uint32_t gt0 = S.sel_gt;  // keys strictly above bin b0 (< k)

    // ---- pass 2: emit keys above b0, collect candidates inside b0 (both in index order)
    uint32_t sel_base = 0, cand_base = 0;
    for (int g0 = 0; g0 < n4; g0 += kTopkThreads) {
        const int g = g0 + tid;
        uint32_t key[4] = {0, 0, 0, 0};
        uint32_t nsel = 0, ncand = 0, selmask = 0, candmask = 0;
        if (g < n4) {
            const float4 v = __ldcs(row4 + g);
            const float f[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (g * 4 + j < n) {
                    key[j] = score_key(f[j]);
                    const uint32_t d = key[j] >> 20;
                    if (d > b0) { selmask |= 1u << j; ++nsel; }
                    else if (d == b0) { candmask |= 1u << j; ++ncand; }
                }
            }
        }
        uint32_t total;
        const uint32_t ex = block_excl_scan(nsel | (ncand << 16), total, S.warp_sum[scan_buf]);
        scan_buf ^= 1;
        uint32_t ps = sel_base + (ex & 0xFFFFu), pc = cand_base + (ex >> 16);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (selmask & (1u << j)) out[ps++] = g * 4 + j;
            if (candmask & (1u << j)) {
                if (pc < (uint32_t)kTopkCap) {
                    S.cand_key[pc] = key[j];
                    S.cand_idx[pc] = g * 4 + j;
                }
                ++pc;
            }
        }
        sel_base += total & 0xFFFFu;
        cand_base += total >> 16;
    }
    __syncthreads();

    // ---- refine inside bin b0: 12 more bits, then the last 8 bits
    uint32_t need = (uint32_t)k - gt0;
    uint32_t b1, b2;
    const uint32_t p0 = b0 << 20;
    if (cand_base <= (uint32_t)kTopkCap) {
        const CandSource src{&S, (int)cand_base};
        refine_round(S, src, 8, 12, 0xFFF00000u, p0, need, b1, scan_buf);
        refine_round(S, src, 0, 8, 0xFFFFFF00u, p0 | (b1 << 8), need, b2, scan_buf);
        emit_final(S, src, p0 | (b1 << 8) | b2, need, out, gt0, scan_buf);
    } else {
        const RowSource src{row, n, b0};
        refine_round(S, src, 8, 12, 0xFFF00000u, p0, need, b1, scan_buf);
        refine_round(S, src, 0, 8, 0xFFFFFF00u, p0 | (b1 << 8), need, b2, scan_buf);
        emit_final(S, src, p0 | (b1 << 8) | b2, need, out, gt0, scan_buf);
    }
}

// Block-wide max of a uint32.
__device__ __forceinline__ uint32_t block_max_u32(TopkShared& S, uint32_t v) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    __syncthreads();
    if (lane == 0) S.red[warp] = v;
    __syncthreads();
    uint32_t m = 0;
#pragma unroll
    for (int w = 0; w < kTopkThreads / 32; ++w) m = max(m, S.red[w]);
    return m;
}

// Exact top-k among the m <= kTopkCap candidates (all keys >= lo), emitted in candidate order.
__device__ __forceinline__ void refine_candidates(TopkShared& S, int m, uint32_t lo, int k, int* out, int& scan_buf) {
    uint32_t kmax = 0;
    for (int e = threadIdx.x; e < m; e += kTopkThreads) kmax = max(kmax, S.cand_key[e] - lo);
    const uint32_t R = block_max_u32(S, kmax);
    int fixed = R ? 32 - __clz(R) : 0;   // offsets are < 2^fixed; bits >= fixed are all zero
    uint32_t pv = 0, need = (uint32_t)k;
    while (fixed > 0) {
        const int sh = fixed > 12 ? fixed - 12 : 0;
        const int width = fixed - sh;
        const int nbins = 1 << width;
        clear_hist(S, nbins);
        __syncthreads();
        for (int e = threadIdx.x; e < m; e += kTopkThreads) {
            const uint32_t d = S.cand_key[e] - lo;
            const bool match = fixed >= 32 ? true : ((d >> fixed) == (pv >> fixed));
            if (match) atomicAdd(&S.hist[(d >> sh) & (nbins - 1)], 1u);
        }
        __syncthreads();
        find_threshold_bin(S, nbins, need, scan_buf);
        need -= S.sel_gt;
        pv |= S.sel_bin << sh;
        fixed = sh;
    }
    const CandSource src{&S, m};
    emit_final(S, src, lo + pv, need, out, 0u, scan_buf);
}

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const TopkParams P) {
    extern __shared__ __align__(1024) uint8_t topk_smem[];
    TopkShared& S = *reinterpret_cast<TopkShared*>(topk_smem);
    const int r = blockIdx.x;
    const int tid = threadIdx.x;
    long long n_ll = P.ctx_len ? (long long)P.ctx_len[r] + 1 : P.q_pos0 + r + 1;
    if (n_ll > P.n_max || n_ll < 1) {
        if (tid == 0) record_error(DSA_DEV_ERR_BOUNDS, 0x401);
        n_ll = n_ll < 1 ? 1 : P.n_max;
    }
    const int n = (int)n_ll;
    const int k = P.k;
    int* out = P.idx + (long long)r * k;
    if (n <= k) {
        for (int j = tid; j < k; j += kTopkThreads) out[j] = j < n ? j : -1;
        return;
    }
    const float* row = P.scores + (long long)r * P.ld;
    const float4* row4 = reinterpret_cast<const float4*>(row);
    const int n4 = (n + 3) >> 2;
    int scan_buf = 0;

    // ---- threshold estimate T0 from a sample (two 12-bit histogram rounds over ~1024 keys)
    uint32_t T0 = 0;
    if (n > kTopkCap) {
        uint32_t sk[4] = {0, 0, 0, 0};
        int sv = 0;
        if (tid < kTopkSampleVec) {
            const int g = (int)(((long long)tid * n4) / kTopkSampleVec);
            const float4 v = row4[g];
            const float f[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (g * 4 + j < n) sk[j] = score_key(f[j]), sv |= 1 << j;
        }
        clear_hist(S, kTopkBins);
        __syncthreads();
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (sv & (1 << j)) atomicAdd(&S.hist[sk[j] >> 20], 1u);
        __syncthreads();
        // aim at rank 2k of the row: r_s = 2k * m / n of the ~m = 4*256 samples
        const uint32_t rs = (uint32_t)min(4LL * kTopkSampleVec - 1,
                                          (2LL * k * 4 * kTopkSampleVec + n - 1) / n);
        find_threshold_bin(S, kTopkBins, rs, scan_buf);
        const uint32_t b = S.sel_bin, need2 = rs - S.sel_gt;
        clear_hist(S, kTopkBins);
        __syncthreads();
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if ((sv & (1 << j)) && (sk[j] >> 20) == b) atomicAdd(&S.hist[(sk[j] >> 8) & 0xFFF], 1u);
        __syncthreads();
        find_threshold_bin(S, kTopkBins, need2, scan_buf);
        T0 = (b << 20) | (S.sel_bin << 8);
    }

    // ---- single streaming pass: compact keys >= T0 in index order
    uint32_t cbase = 0;
    for (int g0 = 0; g0 < n4; g0 += kTopkUnroll * kTopkThreads) {
        float4 v[kTopkUnroll];
#pragma unroll
        for (int u = 0; u < kTopkUnroll; ++u) {
            const int g = g0 + u * kTopkThreads + tid;
            v[u] = g < n4 ? __ldcs(row4 + g) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < kTopkUnroll; ++u) {
            const int g = g0 + u * kTopkThreads + tid;
            const float f[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
            uint32_t key[4], mask = 0, cnt = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                key[j] = score_key(f[j]);
                if (g * 4 + j < n && key[j] >= T0) mask |= 1u << j, ++cnt;
            }
            uint32_t total;
            const uint32_t ex = block_excl_scan(cnt, total, S.warp_sum[scan_buf]);
            scan_buf ^= 1;
            uint32_t pos = cbase + ex;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (mask & (1u << j)) {
                    if (pos < (uint32_t)kTopkCap) {
                        S.cand_key[pos] = key[j];
                        S.cand_idx[pos] = g * 4 + j;
                    }
                    ++pos;
                }
            cbase += total;
            if (g0 + (u + 1) * kTopkThreads >= n4) break;  // uniform across the block
        }
    }
    __syncthreads();
    if (cbase >= (uint32_t)k && cbase <= (uint32_t)kTopkCap) {
        refine_candidates(S, (int)cbase, T0, k, out, scan_buf);
    } else {
        topk_two_pass(S, row, n, k, out, scan_buf);
    }
}

// ---------------------------------------------------------------------------------------------
// Few long rows (decode: B rows of ~131K keys): a cluster of kTopkCluster CTAs shares one row.
// Each CTA samples and streams 1/kTopkCluster of the row; the sample histograms are summed and
// the per-CTA candidate lists are gathered through distributed shared memory, so the row is
// still read once from HBM but by kTopkCluster SMs.  CTA 0 of the cluster refines and writes
// the row (or, if the estimate missed, runs the two-pass fallback over the whole row).
constexpr int kTopkCluster = 8;

namespace cg = cooperative_groups;

// Sum the histograms of every CTA of the cluster into `merged` (a local array).
__device__ __forceinline__ void cluster_merge_hist(TopkShared& S, uint32_t* merged) {
    cg::cluster_group cluster = cg::this_cluster();
    for (int b = threadIdx.x; b < kTopkBins; b += kTopkThreads) {
        uint32_t sum = 0;
#pragma unroll
        for (int c = 0; c < kTopkCluster; ++c) sum += cluster.map_shared_rank(S.hist, c)[b];
        merged[b] = sum;
    }
}

__global__ void __launch_bounds__(kTopkThreads) topk_cluster_kernel(const TopkParams P) {
    extern __shared__ __align__(1024) uint8_t topk_smem[];
    TopkShared& S = *reinterpret_cast<TopkShared*>(topk_smem);
    cg::cluster_group cluster = cg::this_cluster();
    const int crank = (int)cluster.block_rank();
    const int r = blockIdx.x / kTopkCluster;
    const int tid = threadIdx.x;
    long long n_ll = P.ctx_len ? (long long)P.ctx_len[r] + 1 : P.q_pos0 + r + 1;
    if (n_ll > P.n_max || n_ll < 1) {
        if (tid == 0 && crank == 0) record_error(DSA_DEV_ERR_BOUNDS, 0x402);
        n_ll = n_ll < 1 ? 1 : P.n_max;
    }
    const int n = (int)n_ll;
    const int k = P.k;
    int* out = P.idx + (long long)r * k;
    if (n <= k) {  // uniform over the cluster
        if (crank == 0)
            for (int j = tid; j < k; j += kTopkThreads) out[j] = j < n ? j : -1;
        return;
    }
    const float* row = P.scores + (long long)r * P.ld;
    const float4* row4 = reinterpret_cast<const float4*>(row);
    const int n4 = (n + 3) >> 2;
    const int seg = (n4 + kTopkCluster - 1) / kTopkCluster;
    const int g_lo = min(n4, crank * seg), g_hi = min(n4, g_lo + seg);
    int scan_buf = 0;
    uint32_t* merged = S.cand_key;  // scratch until candidates are collected

    // ---- threshold estimate over the whole row from kTopkSampleVec float4 samples
    constexpr int kPer = kTopkSampleVec / kTopkCluster;
    uint32_t sk[4] = {0, 0, 0, 0};
    int sv = 0;
    if (tid < kPer) {
        const int gi = crank * kPer + tid;
        const int g = (int)(((long long)gi * n4) / kTopkSampleVec);
        const float4 v = row4[g];
        const float f[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (g * 4 + j < n) sk[j] = score_key(f[j]), sv |= 1 << j;
    }
    clear_hist(S, kTopkBins);
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 4; ++j)
        if (sv & (1 << j)) atomicAdd(&S.hist[sk[j] >> 20], 1u);
    cluster.sync();
    cluster_merge_hist(S, merged);
    cluster.sync();  // every CTA has read every histogram
    for (int b = tid; b < kTopkBins; b += kTopkThreads) S.hist[b] = merged[b];
    __syncthreads();
    const uint32_t rs = (uint32_t)min(4LL * kTopkSampleVec - 1, (2LL * k * 4 * kTopkSampleVec + n - 1) / n);
    find_threshold_bin(S, kTopkBins, rs, scan_buf);
    const uint32_t b = S.sel_bin, need2 = rs - S.sel_gt;
    __syncthreads();
    clear_hist(S, kTopkBins);
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 4; ++j)
        if ((sv & (1 << j)) && (sk[j] >> 20) == b) atomicAdd(&S.hist[(sk[j] >> 8) & 0xFFF], 1u);
    cluster.sync();
    cluster_merge_hist(S, merged);
    cluster.sync();
    for (int bb = tid; bb < kTopkBins; bb += kTopkThreads) S.hist[bb] = merged[bb];
    __syncthreads();
    find_threshold_bin(S, kTopkBins, need2, scan_buf);
    const uint32_t T0 = (b << 20) | (S.sel_bin << 8);
    __syncthreads();

    // ---- stream this CTA's segment, compact keys >= T0 (index order) into the local list
    uint32_t cbase = 0;
    for (int g0 = g_lo; g0 < g_hi; g0 += kTopkUnroll * kTopkThreads) {
        float4 v[kTopkUnroll];
#pragma unroll
        for (int u = 0; u < kTopkUnroll; ++u) {
            const int g = g0 + u * kTopkThreads + tid;
            v[u] = g < g_hi ? __ldcs(row4 + g) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < kTopkUnroll; ++u) {
            const int g = g0 + u * kTopkThreads + tid;
            const float f[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
            uint32_t key[4], mask = 0, cnt = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                key[j] = score_key(f[j]);
                if (g < g_hi && g * 4 + j < n && key[j] >= T0) mask |= 1u << j, ++cnt;
            }
            uint32_t total;
            const uint32_t ex = block_excl_scan(cnt, total, S.warp_sum[scan_buf]);
            scan_buf ^= 1;
            uint32_t pos = cbase + ex;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (mask & (1u << j)) {
                    if (pos < (uint32_t)kTopkCap) {
                        S.cand_key[pos] = key[j];
                        S.cand_idx[pos] = g * 4 + j;
                    }
                    ++pos;
                }
            cbase += total;
            if (g0 + (u + 1) * kTopkThreads >= g_hi) break;
        }
    }
    if (tid == 0) S.sel_gt = cbase;  // publish this CTA's candidate count
    cluster.sync();

    if (crank == 0) {
        uint32_t counts[kTopkCluster], total = 0;
        bool fits = true;
#pragma unroll
        for (int c = 0; c < kTopkCluster; ++c) {
            counts[c] = cluster.map_shared_rank(&S.sel_gt, c)[0];
            fits = fits && counts[c] <= (uint32_t)kTopkCap;
            total += counts[c];
        }
        fits = fits && total >= (uint32_t)k && total <= (uint32_t)kTopkCap;
        if (fits) {
            uint32_t off = counts[0];
            for (int c = 1; c < kTopkCluster; ++c) {
                const uint32_t* pk = cluster.map_shared_rank(S.cand_key, c);
                const int* pi = cluster.map_shared_rank(S.cand_idx, c);
                for (uint32_t e = tid; e < counts[c]; e += kTopkThreads) {
                    S.cand_key[off + e] = pk[e];
                    S.cand_idx[off + e] = pi[e];
                }
                off += counts[c];
            }
        }
        __syncthreads();
        if (fits) refine_candidates(S, (int)total, T0, k, out, scan_buf);
        else topk_two_pass(S, row, n, k, out, scan_buf);
    }
    cluster.sync();  // peers keep their shared memory alive until CTA 0 has read it
}

}  // namespace dsa
