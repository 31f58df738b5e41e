// Per-row top-k of indexer scores: the min(k, n) keys with the largest score, ties to the lower
// key index, written as int32 key indices followed by -1 padding.
//
// The pages keep the 2048 best-scored positions per token (page "快手开源大模型Keye-VL-2.0：
// 一个能“看懂“两小时视频AI", gsyq.cn, section 一) and require a deterministic top-k so that
// training and inference select the same keys (same page, section 八).  This kernel is exact
// and deterministic: the output of a row depends only on the row's scores.
//
// Method (one CTA per row, radix select on order-preserving 32-bit keys):
//   pass 1  stream the row once from HBM, histogram of the top 12 key bits in shared memory,
//           find the bin b0 that holds the k-th largest key;
//   pass 2  stream the row again (mostly L2 hits): keys above b0 are selected and written out
//           in index order through a block scan; keys inside b0 are compacted, in index order,
//           into a shared-memory candidate list;
//   refine  two more histogram rounds (12 + 8 bits) over the candidates fix the exact k-th key
//           tau and how many keys equal to tau are taken; a last ordered scan over the
//           candidates emits keys > tau and the first keys == tau.
// If the threshold bin holds more candidates than shared memory can keep, the refinement reads
// the row from global memory instead (same rounds, same result).
// Output order: first the keys above the threshold bin (ascending index), then the selected
// candidates (ascending index).
#pragma once

#include "ptx.cuh"

namespace dsa {

constexpr int kTopkThreads = 512;
constexpr int kTopkCap = 6144;   // candidate list capacity (shared memory)
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
    int scan_buf = 0;

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

}  // namespace dsa
