// Per-row top-k of indexer scores: the min(k, n) keys with the largest score, ties to the lower
// key index, written as int32 key indices followed by -1 padding.
//
// The pages keep the 2048 best-scored positions per token (page "快手开源大模型Keye-VL-2.0：
// 一个能“看懂“两小时视频AI", gsyq.cn, section 一) and require a deterministic top-k so that
// training and inference select the same keys (same page, section 八).  This kernel is exact
// and deterministic: the output of a row depends only on the row's scores.
//
// Scores are compared through an order-preserving map float -> uint32 ("key"; -0 folded onto
// +0).  One CTA of 4 warps per row (a cluster of CTAs per row when rows are few and long):
//   sample   ~n/32 scores at evenly spaced float4s give T0, an estimate of the key at rank
//            1.5k (two histogram rounds over the sample keys, bins spanning the samples'
//            own key range);
//   stream   the row is read once, 8 float4 per lane per batch with the next batch's loads in
//            flight while the current one is filtered; each warp takes every 4th 128-byte piece
//            (so frames of correlated scores spread evenly over the warps) and compacts the
//            scores >= T0 into its own shared-memory region: one warp-wide scan of the lanes'
//            packed per-float4 counts places every candidate, then each lane walks only its own
//            candidate bits -- no block barrier per load;
//   refine   if every region fits and the total is >= k, the candidates contain the exact
//            top-k: radix rounds over the key offsets from T0 (first round scaled to the
//            candidates' key range) narrow the bin that holds the k-th key until it is small, and
//            that bin's members are ranked once by (key desc, index asc);
//   emit     the kept keys are written region by region, each region in ascending key order.
// If the candidates miss the window [k, capacity], the estimate is redone once, aimed using the
// observed count, and the row streamed again.  Rows that still miss (or where more than 512
// keys tie in the boundary bin) take an exact radix select over the row itself (10-bit rounds
// with eight 16-byte loads in flight per thread, then one ordered pass per warp region): slower,
// and rare.
// Output order, the same on every path: when every competing key is kept, ascending; otherwise
// grouped by region ((index / 32) mod 4, the pieces of one warp) and ascending within a region.
// Sliding window (SW-DSA, page "DSA注意力机制：多模态学习中的强化推理新范式", showapi.com,
// section 1.4: the selection is restricted to a local window): with window W > 0 only keys
// s > t - W compete; everything else is unchanged.
#pragma once

#include <cooperative_groups.h>

#include "ptx.cuh"

namespace dsa {

namespace cg = cooperative_groups;

constexpr int kTkThreads = 128;               // 4 warps per row (per cluster CTA)
constexpr int kTkWarps = kTkThreads / 32;
constexpr int kTkBins = 1024;                 // 10-bit radix digits
constexpr int kTkRegion = 1024;               // candidates per warp region
constexpr int kTkCap = kTkWarps * kTkRegion;  // 4096 candidates per CTA
constexpr int kTkMaxSample4 = kTkCap / 4;     // at most 1024 sampled float4 (4096 keys)
constexpr int kTkUnroll = 8;                  // float4 loads in flight per lane
constexpr int kTkCluster = 8;                 // CTAs per row in the cluster kernel
constexpr int kTkMaxRegions = kTkCluster * kTkWarps;

// The 128 threads (4 warps) of a CTA that select one row; tid is the thread's index in the CTA.
struct Grp {
    int tid;
    __device__ __forceinline__ int lane() const { return tid & 31; }
    __device__ __forceinline__ int warp() const { return tid >> 5; }
    __device__ __forceinline__ void sync() const { __syncthreads(); }
};

struct TopkParams {
    const float* scores;  // row r at scores + r*ld (16-byte aligned rows)
    long long ld;
    int rows;
    long long q_pos0;     // prefill: row r has n = q_pos0 + r + 1 keys
    const int* ctx_len;   // decode: row r has n = ctx_len[r] + 1 keys (null for prefill)
    long long n_max;      // upper bound on n (keys addressable in a row)
    int k;
    int* idx;             // [rows, k]
    long long window;     // > 0: only the last `window` keys of a row (s > t - window) compete
    int stage_f4;         // cluster kernel: > 0 copies each CTA's segment (up to this many float4)
                          // into shared memory first; 0 reads it from global memory
};

struct TopkSmem {
    uint32_t hist[kTkBins];
    uint32_t cand_key[kTkCap];  // also holds the sample keys before streaming
    int cand_idx[kTkCap];
    // candidate regions: keys/indices may live in this CTA's or (cluster) another CTA's shared memory
    const uint32_t* reg_kp[kTkMaxRegions];
    int* reg_ip[kTkMaxRegions];
    int reg_cnt[kTkMaxRegions], reg_gt[kTkMaxRegions], reg_eq[kTkMaxRegions];
    int nreg;
    uint32_t red[kTkWarps];
    uint32_t sel_bin, sel_gt;
    uint32_t T0;
};

__device__ __forceinline__ uint32_t score_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
// Smallest float whose key is >= T, so that (f >= key_floor_float(T)) == (score_key(f) >= T).
__device__ __forceinline__ float key_floor_float(uint32_t T) {
    if (T == 0u) return -INFINITY;
    return (T & 0x80000000u) ? __uint_as_float(T & 0x7FFFFFFFu) : __uint_as_float(~T);
}

__device__ __forceinline__ long long row_length(const TopkParams& P, int r, bool report) {
    long long n = P.ctx_len ? (long long)P.ctx_len[r] + 1 : P.q_pos0 + r + 1;
    if (n > P.n_max || n < 1) {
        if (report) record_error(DSA_DEV_ERR_BOUNDS, 0x401);
        n = n < 1 ? 1 : P.n_max;
    }
    return n;
}

// First key of row r's candidate range: 0, or n - window under a sliding window.
__device__ __forceinline__ int row_first_key(const TopkParams& P, int n) {
    return (P.window > 0 && (long long)n > P.window) ? (int)(n - P.window) : 0;
}

// Inclusive warp prefix sum.
__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t x) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    return x;
}

// Exclusive block prefix sum (4 warps); returns the block total.
__device__ __forceinline__ uint32_t block_excl_scan(TopkSmem& S, const Grp& G, uint32_t v, uint32_t& total) {
    const int lane = G.lane(), warp = G.warp();
    const uint32_t x = warp_incl_scan(v);
    G.sync();
    if (lane == 31) S.red[warp] = x;
    G.sync();
    uint32_t before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kTkWarps; ++w) {
        before += (w < warp) ? S.red[w] : 0u;
        tot += S.red[w];
    }
    total = tot;
    return before + x - v;
}

// Bin b of S.hist[0, nbins) with (count above b) < need <= (count above b) + hist[b]; result in
// S.sel_bin / S.sel_gt.  nbins <= kTkBins; needs the histogram total >= need.
__device__ __forceinline__ void find_threshold_bin(TopkSmem& S, const Grp& G, int nbins, uint32_t need) {
    constexpr int kMaxPer = kTkBins / kTkThreads;
    const int per = (nbins + kTkThreads - 1) / kTkThreads;
    const int lo = G.tid * per;
    uint32_t mine = 0;
#pragma unroll
    for (int b = 0; b < kMaxPer; ++b)
        if (b < per && lo + b < nbins) mine += S.hist[lo + b];
    // suffix sums over threads (a higher thread owns higher bins)
    const int lane = G.lane(), warp = G.warp();
    uint32_t x = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, x, o);
        if (lane + o < 32) x += y;
    }
    G.sync();
    if (lane == 0) S.red[warp] = x;
    G.sync();
    uint32_t above = x - mine;
#pragma unroll
    for (int w = 0; w < kTkWarps; ++w) above += (w > warp) ? S.red[w] : 0u;
    if (lo < nbins && above < need && need <= above + mine) {
        uint32_t cum = above;
        for (int b = min(lo + per, nbins) - 1; b >= lo; --b) {
            const uint32_t h = S.hist[b];
            if (cum + h >= need) {
                S.sel_bin = (uint32_t)b;
                S.sel_gt = cum;
                break;
            }
            cum += h;
        }
    }
    G.sync();
}

__device__ __forceinline__ void clear_hist(TopkSmem& S, const Grp& G, int nbins) {
    for (int b = G.tid; b < nbins; b += kTkThreads) S.hist[b] = 0;
}

// T0 from m sample keys in S.cand_key[0, m): a lower bound on the key at rank rs (counted from
// the top), found with two histogram rounds of 1024 bins over the samples' own key range
// [kmin, kmax] (key 0 marks a masked sample and counts with the lowest bin).  Round 1 bins
// have width 2^sh1, the smallest power of two that covers the range; round 2 splits the bin
// holding rank rs again into up to 1024 parts.  Every sample key >= T0 is counted, so at least
// rs samples are >= T0.  Bins that follow the data (rather than fixed top bits of the key) keep
// the shared-memory atomics spread out when the scores sit in a narrow range.
__device__ __forceinline__ uint32_t sample_threshold(TopkSmem& S, const Grp& G, int m, uint32_t rs,
                                                    uint32_t* kmax_out = nullptr) {
    const int lane = G.lane(), warp = G.warp();
    G.sync();  // the samples were written by other threads
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
    for (int e = G.tid; e < m; e += kTkThreads) {
        const uint32_t key = S.cand_key[e];
        if (key) {
            kmin = min(kmin, key);
            kmax = max(kmax, key);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    }
    if (lane == 0) {
        S.hist[warp] = kmin;
        S.hist[kTkWarps + warp] = kmax;
    }
    G.sync();
#pragma unroll
    for (int w = 0; w < kTkWarps; ++w) {
        kmin = min(kmin, S.hist[w]);
        kmax = max(kmax, S.hist[kTkWarps + w]);
    }
    G.sync();
    if (kmin > kmax) kmin = kmax = 0u;  // every sample masked
    if (kmax_out) *kmax_out = kmax;
    const uint32_t span = kmax - kmin;
    const int sh1 = (span >> 10) ? 32 - __clz(span >> 10) : 0;  // (span >> sh1) < 1024
    clear_hist(S, G, kTkBins);
    G.sync();
    for (int e = G.tid; e < m; e += kTkThreads) {
        const uint32_t key = S.cand_key[e];
        atomicAdd(&S.hist[min((key > kmin ? key - kmin : 0u) >> sh1, (uint32_t)kTkBins - 1u)], 1u);
    }
    G.sync();
    find_threshold_bin(S, G, kTkBins, rs);
    const uint32_t b1 = S.sel_bin, need = rs - S.sel_gt;
    if (sh1 == 0) return kmin + b1;  // bins of single key values: exact
    const int sh2 = sh1 > 10 ? sh1 - 10 : 0;
    const uint32_t base = b1 << sh1;
    clear_hist(S, G, kTkBins);
    G.sync();
    for (int e = G.tid; e < m; e += kTkThreads) {
        const uint32_t key = S.cand_key[e];
        const uint32_t d = key > kmin ? key - kmin : 0u;
        if (min(d >> sh1, (uint32_t)kTkBins - 1u) == b1) atomicAdd(&S.hist[min((d - base) >> sh2, (uint32_t)kTkBins - 1u)], 1u);
    }
    G.sync();
    find_threshold_bin(S, G, kTkBins, need);
    return kmin + base + (S.sel_bin << sh2);
}

// Stream float4 groups [g_lo, g_hi) of a row whose keys e_lo <= e < n compete and compact the
// scores >= F0 into this warp's region, in index order.  Warp w takes the 128-byte pieces p
// (keys 32p .. 32p+31 of the row) with p % 4 == w: region w.
// Each batch of kTkUnroll (8) float4 loads per lane is filtered as a whole; the next batch's loads
// are issued before the current batch is filtered (software pipelining).  The per-float4
// candidate counts of a lane (0..4 each) ride in the bytes of two registers through one warp-wide
// inclusive scan (5 shuffle steps), which gives every lane the position of each of its
// candidates.  Candidates are sparse (about one per lane per batch), so each lane then walks only
// the set bits of its 32-bit candidate mask -- the warp takes as many steps as its busiest lane
// has candidates -- and picks the score out of its registers with a select tree, instead of a
// predicated store slot for every score (8 % faster per 128K chunk) or a divergent branch per
// float4.  Positions: float4 u first, then lane, then component, i.e. index order.
// Returns how many scores of this warp qualified (may exceed the region; the excess is dropped).
__device__ __forceinline__ uint32_t stream_collect(TopkSmem& S, const Grp& G, const float4* row4, int g_lo, int g_hi,
                                                   int e_lo, int n, float F0, int region_base) {
    constexpr int UN = kTkUnroll;
    static_assert(UN == 8, "the candidate mask holds 8 float4 x 4 bits, the counts two words");
    const int g_first = g_lo;
    const int lane = G.lane(), warp = G.warp();
    // float4 offset inside a 128-float4 round: piece (lane/8)*4 + warp, float4 lane%8 of it
    const int lane_off = (lane >> 3) * 32 + warp * 8 + (lane & 7);
    // float4 groups whose four keys all lie in [e_lo, n): [g_in_lo, g_in_hi)
    const int g_in_lo = max(g_first, (e_lo + 3) >> 2), g_in_hi = min(g_hi, n >> 2);
    uint32_t cnt = 0;
    // pieces are numbered from the start of the row: start at a multiple of 4 pieces (32 float4)
    // so that warp w takes exactly the pieces p with p % 4 == w (keys below g_lo are masked)
    g_lo &= ~31;
    constexpr int kStep = UN * 128;  // float4 per iteration
    float4 vn[UN];
    auto load_batch = [&](int gb) {
        const bool in = gb >= g_in_lo && gb + kStep <= g_in_hi;
#pragma unroll
        for (int u = 0; u < UN; ++u) {
            const int g = gb + u * 128 + lane_off;
            vn[u] = (in || g < g_hi) ? __ldcs(row4 + g) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    if (g_lo < g_hi) load_batch(g_lo);
    for (int g0 = g_lo; g0 < g_hi; g0 += kStep) {
        // warp-uniform: every float4 of this iteration is in range, so only the score is tested
        const bool interior = g0 >= g_in_lo && g0 + kStep <= g_in_hi;
        float4 v[UN];
#pragma unroll
        for (int u = 0; u < UN; ++u) v[u] = vn[u];
        if (g0 + kStep < g_hi) load_batch(g0 + kStep);
        uint32_t mk = 0;              // 4-bit candidate mask of float4 u at bits 4u .. 4u+3
        uint32_t c[2];                // candidate count (0..4) of float4 u in byte u % 4 of word u / 4
#pragma unroll
        for (int u = 0; u < UN; ++u) {
            const int g = g0 + u * 128 + lane_off;
            const float f[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
            uint32_t mask = 0;
            if (interior) {
#pragma unroll
                for (int j = 0; j < 4; ++j) mask |= (f[j] >= F0 ? 1u : 0u) << j;
            } else if (g < g_hi) {
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (f[j] >= F0 && g * 4 + j < n && g * 4 + j >= e_lo && g >= g_first) mask |= 1u << j;
            }
            mk |= mask << (4 * u);
        }
        if (__ballot_sync(0xffffffffu, mk != 0u) == 0) continue;
        {
            // the counts from the packed mask: nibble popcounts (0..4 each), then nibbles 0..3 and
            // 4..7 spread into the bytes of c[0] and c[1] (fewer instructions than a popcount and
            // a shift-or per float4)
            uint32_t x = mk - ((mk >> 1) & 0x55555555u);
            x = (x & 0x33333333u) + ((x >> 2) & 0x33333333u);
            uint32_t y0 = x & 0xFFFFu, y1 = x >> 16;
            y0 = (y0 | (y0 << 8)) & 0x00FF00FFu;
            y1 = (y1 | (y1 << 8)) & 0x00FF00FFu;
            c[0] = (y0 | (y0 << 4)) & 0x0F0F0F0Fu;
            c[1] = (y1 | (y1 << 4)) & 0x0F0F0F0Fu;
        }
        // inclusive scan over lanes of the packed counts (each prefix <= 128 fits its byte)
        uint32_t sc[2] = {c[0], c[1]};
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y0 = __shfl_up_sync(0xffffffffu, sc[0], o), y1 = __shfl_up_sync(0xffffffffu, sc[1], o);
            if (lane >= o) {
                sc[0] += y0;
                sc[1] += y1;
            }
        }
        const uint32_t t0 = __shfl_sync(0xffffffffu, sc[0], 31), t1 = __shfl_sync(0xffffffffu, sc[1], 31);
        sc[0] -= c[0];  // exclusive prefixes, bytewise
        sc[1] -= c[1];
        // lane u < 8: the candidates of float4s before u over the whole warp (exclusive prefix)
        const uint32_t tot_l = lane < UN ? (((lane & 4) ? t1 : t0) >> (8 * (lane & 3))) & 0xFFu : 0u;
        uint32_t incl = tot_l;
#pragma unroll
        for (int o = 1; o < UN; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const uint32_t pre_l = incl - tot_l;
        const uint32_t batch_total = __shfl_sync(0xffffffffu, incl, UN - 1);
        uint32_t bits = mk;
        const int trips = (int)__reduce_max_sync(0xffffffffu, (unsigned)__popc(mk));
        for (int it = 0; it < trips; ++it) {
            const bool has = bits != 0u;
            const int b = has ? __ffs(bits) - 1 : 0;
            bits &= bits - 1u;
            const int u = b >> 2, j = b & 3;
            const uint32_t pre = __shfl_sync(0xffffffffu, pre_l, u);
            const uint32_t sw = u < 4 ? sc[0] : sc[1];
            const uint32_t pos = cnt + pre + ((sw >> (8 * (u & 3))) & 0xFFu) + __popc(mk & (((1u << j) - 1u) << (4 * u)));
            // v[u] component j through a select tree on the bits of b
            float4 a4[4], b4[2];
#pragma unroll
            for (int q = 0; q < 4; ++q) a4[q] = (u & 1) ? v[2 * q + 1] : v[2 * q];
#pragma unroll
            for (int q = 0; q < 2; ++q) b4[q] = (u & 2) ? a4[2 * q + 1] : a4[2 * q];
            const float4 c4 = (u & 4) ? b4[1] : b4[0];
            const float f = (j & 2) ? ((j & 1) ? c4.w : c4.z) : ((j & 1) ? c4.y : c4.x);
            if (has && pos < (uint32_t)kTkRegion) {
                const int g = g0 + u * 128 + lane_off;
                S.cand_key[region_base + pos] = score_key(f);
                S.cand_idx[region_base + pos] = g * 4 + j;
            }
        }
        cnt += batch_total;
    }
    return cnt;
}

// stream_collect for a segment staged in shared memory (src4[g - g_base]), 16 float4 per lane
// per batch.  Candidates are sparse (a few per lane per batch), so instead of a predicated store
// slot for every score, each lane walks the set bits of its 64-bit candidate mask and re-reads the
// score from shared memory: the warp runs as many steps as its busiest lane has candidates.
// Positions are the same as stream_collect's (float4 u first, then lane, then component), so the
// regions hold the same candidates in the same order.
__device__ __forceinline__ uint32_t stream_collect_staged(TopkSmem& S, const Grp& G, const float4* src4, int g_lo,
                                                          int g_hi, int e_lo, int n, float F0, int region_base,
                                                          int g_base) {
    constexpr int UN = 16, kW = UN / 4;
    const int g_first = g_lo;
    const int lane = G.lane(), warp = G.warp();
    const int lane_off = (lane >> 3) * 32 + warp * 8 + (lane & 7);
    const int g_in_lo = max(g_first, (e_lo + 3) >> 2), g_in_hi = min(g_hi, n >> 2);
    const float* src = reinterpret_cast<const float*>(src4);
    uint32_t cnt = 0;
    g_lo &= ~31;
    constexpr int kStep = UN * 128;
    for (int g0 = g_lo; g0 < g_hi; g0 += kStep) {
        const bool interior = g0 >= g_in_lo && g0 + kStep <= g_in_hi;
        unsigned long long mk = 0;  // 4-bit candidate mask of float4 u at bits 4u .. 4u+3
        uint32_t c[kW];             // candidate count (0..4) of float4 u in byte u % 4 of word u / 4
#pragma unroll
        for (int w = 0; w < kW; ++w) c[w] = 0;
#pragma unroll
        for (int u = 0; u < UN; ++u) {
            const int g = g0 + u * 128 + lane_off;
            uint32_t mask = 0;
            if (interior || g < g_hi) {
                const float4 v = src4[g - g_base];
                const float f[4] = {v.x, v.y, v.z, v.w};
                if (interior) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) mask |= (f[j] >= F0 ? 1u : 0u) << j;
                } else {
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        if (f[j] >= F0 && g * 4 + j < n && g * 4 + j >= e_lo && g >= g_first) mask |= 1u << j;
                }
            }
            mk |= (unsigned long long)mask << (4 * u);
            c[u >> 2] |= (uint32_t)__popc(mask) << (8 * (u & 3));
        }
        if (__ballot_sync(0xffffffffu, mk != 0ull) == 0) continue;
        // exclusive scan over lanes of the packed counts, and the per-float4 totals
        uint32_t sc[kW], t[kW];
#pragma unroll
        for (int w = 0; w < kW; ++w) sc[w] = c[w];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t y[kW];
#pragma unroll
            for (int w = 0; w < kW; ++w) y[w] = __shfl_up_sync(0xffffffffu, sc[w], o);
            if (lane >= o) {
#pragma unroll
                for (int w = 0; w < kW; ++w) sc[w] += y[w];
            }
        }
#pragma unroll
        for (int w = 0; w < kW; ++w) {
            t[w] = __shfl_sync(0xffffffffu, sc[w], 31);
            sc[w] -= c[w];
        }
        // lane u < UN: the candidates of float4s before u, over the whole warp (exclusive prefix)
        const int lw = (lane >> 2) & (kW - 1);
        const uint32_t tw = lw == 0 ? t[0] : lw == 1 ? t[1] : lw == 2 ? t[2] : t[3];
        const uint32_t tot_l = lane < UN ? (tw >> (8 * (lane & 3))) & 0xFFu : 0u;
        uint32_t incl = tot_l;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const uint32_t pre_l = incl - tot_l;
        const uint32_t batch_total = __shfl_sync(0xffffffffu, incl, UN - 1);
        unsigned long long bits = mk;
        const int trips = (int)__reduce_max_sync(0xffffffffu, (unsigned)__popcll(mk));
        for (int it = 0; it < trips; ++it) {
            const bool has = bits != 0ull;
            const int b = has ? __ffsll((long long)bits) - 1 : 0;
            bits &= bits - 1ull;
            const int u = b >> 2, j = b & 3;
            const uint32_t pre = __shfl_sync(0xffffffffu, pre_l, u);
            const uint32_t sw = u < 8 ? (u < 4 ? sc[0] : sc[1]) : (u < 12 ? sc[2] : sc[3]);
            const uint32_t mu = (uint32_t)(mk >> (4 * u)) & 0xFu;
            const uint32_t pos = cnt + pre + ((sw >> (8 * (u & 3))) & 0xFFu) + __popc(mu & ((1u << j) - 1u));
            if (has && pos < (uint32_t)kTkRegion) {
                const int g = g0 + u * 128 + lane_off;
                S.cand_key[region_base + pos] = score_key(src[(g - g_base) * 4 + j]);
                S.cand_idx[region_base + pos] = g * 4 + j;
            }
        }
        cnt += batch_total;
    }
    return cnt;
}

// Exact top-k among the candidates in S's regions (every candidate key >= lo; their total is
// >= k and includes every key of the row >= lo).  Radix rounds over the key offsets narrow down
// the bin holding the k-th key until it holds at most kTkSmallBin candidates (or one key value);
// keys above that bin are all kept, and the bin's members are ranked by (key desc, index asc).
// Returns false, writing nothing, when more than kTkBins / 2 candidates share the last bin.
constexpr int kTkSmallBin = 64;
constexpr int kTkBatch = 4;  // shared-memory loads batched per thread in the refinement passes

__device__ __forceinline__ bool refine_and_emit(TopkSmem& S, const Grp& G, uint32_t lo, int k, int* out) {
    const int tid = G.tid, lane = G.lane(), warp = G.warp();
    const int nreg = S.nreg;
    // The passes below hoist each region's pointers and count into registers and batch their
    // shared-memory loads (kTkBatch per thread ahead of the use), so that they overlap instead of
    // each waiting for the one before (stores and atomics in the loops would otherwise make the
    // compiler reload the bounds and serialise the loads).
    uint32_t mx = 0;
    for (int r = 0; r < nreg; ++r) {
        const uint32_t* kp = S.reg_kp[r];
        const int cnt = S.reg_cnt[r];
#pragma unroll 4
        for (int e = tid; e < cnt; e += kTkThreads) mx = max(mx, kp[e] - lo);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    G.sync();
    if (lane == 0) S.red[warp] = mx;
    G.sync();
    uint32_t R = 0;
#pragma unroll
    for (int w = 0; w < kTkWarps; ++w) R = max(R, S.red[w]);
    int fixed = R ? 32 - __clz(R) : 0;  // every offset is < 2^fixed
    uint32_t pv = 0, need = (uint32_t)k, cnt_b = 0;
    if (fixed == 0)
        for (int r = 0; r < nreg; ++r) cnt_b += (uint32_t)S.reg_cnt[r];  // one key value for all
    while (fixed > 0) {
        const int sh = fixed > 10 ? fixed - 10 : 0;
        const int nbins = 1 << (fixed - sh);
        G.sync();
        clear_hist(S, G, nbins);
        G.sync();
        for (int r = 0; r < nreg; ++r) {
            const uint32_t* kp = S.reg_kp[r];
            const int cnt = S.reg_cnt[r];
            for (int e0 = tid; e0 < cnt; e0 += kTkBatch * kTkThreads) {
                uint32_t d[kTkBatch];
#pragma unroll
                for (int j = 0; j < kTkBatch; ++j) {
                    const int e = e0 + j * kTkThreads;
                    d[j] = e < cnt ? kp[e] - lo : 0u;
                }
#pragma unroll
                for (int j = 0; j < kTkBatch; ++j) {
                    const bool match = fixed >= 32 ? true : ((d[j] >> fixed) == (pv >> fixed));
                    if (e0 + j * kTkThreads < cnt && match) atomicAdd(&S.hist[(d[j] >> sh) & (nbins - 1)], 1u);
                }
            }
        }
        G.sync();
        find_threshold_bin(S, G, nbins, need);
        need -= S.sel_gt;
        cnt_b = S.hist[S.sel_bin];
        pv |= S.sel_bin << sh;
        fixed = sh;
        if (cnt_b <= (uint32_t)kTkSmallBin) break;  // uniform: every thread read the same count
    }
    G.sync();
    // boundary bin: offsets d with d >> fixed == pv >> fixed; kept outright: d >> fixed > pv >> fixed
    if (cnt_b > (uint32_t)(kTkBins / 2)) return false;
    const uint32_t bin = fixed >= 32 ? 0u : (pv >> fixed);
    auto above = [&](uint32_t d) { return fixed < 32 && (d >> fixed) > bin; };
    auto in_bin = [&](uint32_t d) { return fixed >= 32 || (d >> fixed) == bin; };
    // the bin's members: (key, location) into a small list, order irrelevant; each is ranked once
    // by (key desc, index asc) and the ones not kept are marked (index -1) in place, so that the
    // passes below test a candidate in O(1)
    uint32_t* bkey = S.hist;                      // reused: up to kTkBins / 2 members
    uint32_t* bloc = S.hist + kTkBins / 2;        // region << 16 | position
    auto loc_idx = [&](uint32_t l) { return S.reg_ip[l >> 16][l & 0xFFFFu]; };
    if (tid == 0) S.sel_bin = 0;
    G.sync();
    for (int r = 0; r < nreg; ++r) {
        const uint32_t* kp = S.reg_kp[r];
        const int cnt = S.reg_cnt[r];
        for (int e0 = tid; e0 < cnt; e0 += kTkBatch * kTkThreads) {
            uint32_t key[kTkBatch];
#pragma unroll
            for (int j = 0; j < kTkBatch; ++j) {
                const int e = e0 + j * kTkThreads;
                key[j] = e < cnt ? kp[e] : 0u;
            }
#pragma unroll
            for (int j = 0; j < kTkBatch; ++j) {
                const int e = e0 + j * kTkThreads;
                if (e < cnt && in_bin(key[j] - lo)) {
                    const uint32_t p = atomicAdd(&S.sel_bin, 1u);
                    bkey[p] = key[j];
                    bloc[p] = ((uint32_t)r << 16) | (uint32_t)e;
                }
            }
        }
    }
    G.sync();
    bool drop[(kTkBins / 2 + kTkThreads - 1) / kTkThreads];
#pragma unroll
    for (int j = 0; j < (int)(sizeof(drop) / sizeof(drop[0])); ++j) {
        const uint32_t a = tid + j * kTkThreads;
        drop[j] = false;
        if (a < cnt_b) {
            const uint32_t ka = bkey[a];
            const int ia = loc_idx(bloc[a]);
            uint32_t rank = 0;
            for (uint32_t b2 = 0; b2 < cnt_b; ++b2) {
                const uint32_t kb = bkey[b2];
                rank += (kb > ka) || (kb == ka && loc_idx(bloc[b2]) < ia);
            }
            drop[j] = rank >= need;
        }
    }
    G.sync();  // every rank used the original indices
#pragma unroll
    for (int j = 0; j < (int)(sizeof(drop) / sizeof(drop[0])); ++j) {
        const uint32_t a = tid + j * kTkThreads;
        if (a < cnt_b && drop[j]) S.reg_ip[bloc[a] >> 16][bloc[a] & 0xFFFFu] = -1;
    }
    G.sync();
    auto kept = [&](uint32_t key, int ix) {
        const uint32_t d = key - lo;
        return above(d) || (in_bin(d) && ix >= 0);
    };
    // write the kept keys region by region, each region in its own (ascending) order
    for (int r = warp; r < nreg; r += kTkWarps) {
        uint32_t c = 0;
        const uint32_t* kp = S.reg_kp[r];
        const int* ip = S.reg_ip[r];
        const int cnt = S.reg_cnt[r];
#pragma unroll 4
        for (int e = lane; e < cnt; e += 32) c += kept(kp[e], ip[e]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        if (lane == 0) S.reg_gt[r] = (int)c;
    }
    G.sync();
    for (int r = warp; r < nreg; r += kTkWarps) {
        uint32_t base = 0;
        for (int q = 0; q < r; ++q) base += (uint32_t)S.reg_gt[q];
        const uint32_t* kp = S.reg_kp[r];
        const int* ip = S.reg_ip[r];
        const int cnt = S.reg_cnt[r];
        for (int e0 = 0; e0 < cnt; e0 += 32 * kTkBatch) {
            int ix[kTkBatch];
            bool keep[kTkBatch];
#pragma unroll
            for (int j = 0; j < kTkBatch; ++j) {
                const int e = e0 + 32 * j + lane;
                const bool in = e < cnt;
                ix[j] = in ? ip[e] : 0;
                keep[j] = in && kept(in ? kp[e] : 0u, ix[j]);
            }
#pragma unroll
            for (int j = 0; j < kTkBatch; ++j) {
                const uint32_t bk = __ballot_sync(0xffffffffu, keep[j]);
                if (keep[j]) out[base + __popc(bk & ((1u << lane) - 1u))] = ix[j];
                base += __popc(bk);
            }
        }
    }
    return true;
}

// Exact radix select over the row (the fallback): histogram passes of 10 + 10 + 10 + 2 bits over
// the row's keys fix tau and the number of ties to keep; when that is every key equal to tau (the
// usual case: one boundary key) no tie scan is needed, else a scan finds the last kept tie; then
// warp w writes region w's kept keys ((index / 32) mod 4 == w) in ascending order after the
// counts of the regions before it -- the fast path's order.  Every pass keeps eight 16-byte loads
// per thread (radix) or eight loads per lane (emission) in flight: a row that misses twice costs a
// few passes over it, not a latency-bound crawl.  `row` is 16-byte aligned.
__device__ __noinline__ void topk_global(TopkSmem& S, const Grp& G, const float* row, int lo, int n, int k, int* out) {
    const int tid = G.tid, lane = G.lane(), warp = G.warp();
    const float4* row4 = reinterpret_cast<const float4*>(row);
    const int g_lo = lo >> 2, g_hi = (n + 3) >> 2;
    uint32_t pval = 0, need = (uint32_t)k, eq_cnt = 0;
    int fixed = 32;
    while (fixed > 0) {
        const int width = fixed >= 10 ? 10 : fixed;
        const int sh = fixed - width;
        const int nbins = 1 << width;
        G.sync();
        clear_hist(S, G, nbins);
        G.sync();
        for (int g0 = g_lo + tid; g0 < g_hi; g0 += 8 * kTkThreads) {
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int g = g0 + u * kTkThreads;
                v[u] = g < g_hi ? __ldcs(row4 + g) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int g = g0 + u * kTkThreads;
                const float f[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int e = 4 * g + j;
                    if (g >= g_hi || e < lo || e >= n) continue;
                    const uint32_t key = score_key(f[j]);
                    if (fixed >= 32 || (key >> fixed) == (pval >> fixed))
                        atomicAdd(&S.hist[(key >> sh) & (nbins - 1)], 1u);
                }
            }
        }
        G.sync();
        find_threshold_bin(S, G, nbins, need);
        need -= S.sel_gt;
        pval |= S.sel_bin << sh;
        if (sh == 0) eq_cnt = S.hist[S.sel_bin];  // every bit fixed: the keys equal to tau
        fixed = sh;
    }
    const uint32_t tau = pval, ties = need;
    int tie_end = n;  // keys == tau with index < tie_end are kept
    if (ties < eq_cnt) {
        // keep only the `ties` lowest-index keys equal to tau: count them per 128 keys in order
        uint32_t eq_seen = 0;
        for (int e0 = lo; e0 < n; e0 += kTkThreads) {
            const int e = e0 + tid;
            const uint32_t eq = (e < n && score_key(row[e]) == tau) ? 1u : 0u;
            uint32_t total;
            const uint32_t ex = block_excl_scan(S, G, eq, total);
            if (eq && eq_seen + ex == ties - 1) S.sel_gt = (uint32_t)e + 1;  // the last kept tie
            G.sync();
            eq_seen += total;
            if (eq_seen >= ties) {
                tie_end = (int)S.sel_gt;
                break;
            }
        }
    }
    // emission: warp w owns region w, pieces p = 4 i + w (keys 32p .. 32p+31), lane = key
    const int p_first = ((lo >> 5) & ~3) + warp, p_end = (n + 31) >> 5;
    auto kept = [&](int e, float f) {
        if (e < lo || e >= n) return false;
        const uint32_t key = score_key(f);
        return key > tau || (key == tau && e < tie_end);
    };
    uint32_t cnt = 0;
    for (int p0 = p_first; p0 < p_end; p0 += 4 * 8) {
        float f[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = (p0 + 4 * u) * 32 + lane;
            f[u] = (p0 + 4 * u < p_end && e < n) ? __ldcs(row + e) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) cnt += __popc(__ballot_sync(0xffffffffu, kept((p0 + 4 * u) * 32 + lane, f[u])));
    }
    if (lane == 0) S.red[warp] = cnt;
    G.sync();
    uint32_t base = 0;
    for (int w = 0; w < warp; ++w) base += S.red[w];
    for (int p0 = p_first; p0 < p_end; p0 += 4 * 8) {
        float f[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = (p0 + 4 * u) * 32 + lane;
            f[u] = (p0 + 4 * u < p_end && e < n) ? __ldcs(row + e) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = (p0 + 4 * u) * 32 + lane;
            const bool keep = kept(e, f[u]);
            const uint32_t bal = __ballot_sync(0xffffffffu, keep);
            if (keep) out[base + __popc(bal & ((1u << lane) - 1u))] = e;
            base += __popc(bal);
        }
    }
    G.sync();  // S.red is reused by the caller's next phase
}

__device__ __forceinline__ uint32_t rank_target(long long m, long long n, int k) {
    // aim at rank 1.5k of the row, i.e. rank 1.5k * m / n of the m samples
    return (uint32_t)max(1LL, min(m - 1, (3LL * k * m + 2LL * n - 1) / (2LL * n)));
}

// Sample s4 evenly spaced float4 of float4 range [g_lo, g_hi) into keys[base .. base + 4*s4); all
// of a thread's loads are issued before any is used.  Float4 group g is read at src4[g - g_base]
// (the row itself with g_base = 0, or a shared-memory copy of a segment starting at g_base).
__device__ __forceinline__ void take_samples(const Grp& G, uint32_t* keys, int base, const float4* src4, int g_base,
                                             int g_lo, int g_hi, int e_lo, int n, int s4) {
    constexpr int kPer = kTkMaxSample4 / kTkThreads;
    float4 v[kPer];
    int gg[kPer];
    // position of sample i: g_lo + floor(i * span / s4), via a 32.32 fixed-point step
    const unsigned long long step = ((unsigned long long)(g_hi - g_lo) << 32) / (unsigned)max(s4, 1);
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int i = G.tid + u * kTkThreads;
        gg[u] = g_lo + (int)(((unsigned long long)i * step) >> 32);
        v[u] = (i < s4 && gg[u] < g_hi) ? src4[gg[u] - g_base] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int i = G.tid + u * kTkThreads;
        if (i >= s4) continue;
        const int g = gg[u];
        const float f[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
            keys[base + 4 * i + j] = (g < g_hi && g * 4 + j < n && g * 4 + j >= e_lo) ? score_key(f[j]) : 0u;
    }
}

// Sampled float4 groups per part for n4 groups of competing keys: about n/32 scores (at least 1024,
// at most 4096) in all.  (An earlier n4/8 rule sampled n/8 to n/16 of the shorter rows: 6 % slower
// over a 128K sequence's chunks, no fewer misses.)
__device__ __forceinline__ int sample_count4(int n4, int parts) {
    return min(kTkMaxSample4, max(256, n4 / 32)) / parts;
}

// Second aim after a miss: the observed count c at rank rs scales about linearly with the rank.
__device__ __forceinline__ uint32_t retarget(uint32_t rs, uint32_t c, long long m, int k) {
    const long long want = (3LL * k) / 2;
    const long long r2 = ((long long)rs * want + (c > 0 ? c : 1) - 1) / (c > 0 ? (long long)c : 1LL);
    return (uint32_t)max(1LL, min(m - 1, r2));
}

__global__ void __launch_bounds__(kTkThreads, 5) topk_kernel(const TopkParams P) {
    extern __shared__ __align__(1024) uint8_t topk_smem[];
    TopkSmem& S = *reinterpret_cast<TopkSmem*>(topk_smem);
    const int r = blockIdx.x, tid = threadIdx.x, warp = tid >> 5;
    const Grp G{tid};
    const int n = (int)row_length(P, r, tid == 0);
    const int lo = row_first_key(P, n), ne = n - lo;  // competing keys: [lo, n)
    const int k = P.k;
    int* out = P.idx + (long long)r * k;
    if (ne <= k) {
        for (int j = tid; j < k; j += kTkThreads) out[j] = j < ne ? lo + j : -1;
        return;
    }
    const float* row = P.scores + (long long)r * P.ld;
    const float4* row4 = reinterpret_cast<const float4*>(row);
    const int n4 = (n + 3) >> 2, g0 = lo >> 2;
    const int s4 = sample_count4(n4 - g0, 1);
    const long long m = 4LL * s4;
    uint32_t rs = (uint32_t)rank_target(m, ne, k);
    bool done = false;
    for (int attempt = 0; attempt < 2 && !done; ++attempt) {
        // ---- threshold estimate (rows of up to kTkCap scores keep them all)
        uint32_t T0 = 0;
        if (ne > kTkCap) {
            if (attempt > 0) __syncthreads();
            take_samples(G, S.cand_key, 0, row4, 0, g0, n4, lo, n, s4);
            T0 = sample_threshold(S, G, (int)m, rs);
        }
        // ---- one streaming pass: scores >= T0 into the 4 warp regions
        const uint32_t c = stream_collect(S, G, row4, g0, n4, lo, n, key_floor_float(T0), warp * kTkRegion);
        if ((tid & 31) == 0) {
            S.reg_kp[warp] = S.cand_key + warp * kTkRegion;
            S.reg_ip[warp] = S.cand_idx + warp * kTkRegion;
            S.reg_cnt[warp] = (int)min(c, (uint32_t)kTkRegion);
            S.reg_gt[warp] = (int)c;
        }
        if (tid == 0) S.nreg = kTkWarps;
        __syncthreads();
        uint32_t total = 0;
        bool fits = true;
#pragma unroll
        for (int w = 0; w < kTkWarps; ++w) {
            total += (uint32_t)S.reg_gt[w];
            fits = fits && S.reg_gt[w] <= kTkRegion;
        }
        fits = fits && total >= (uint32_t)k;
        done = fits && refine_and_emit(S, G, T0, k, out);
        if (!done) rs = retarget(rs, total, m, k);
        if (tid == 0) {
            atomicAdd(&g_counters[0], attempt == 0 ? 1ull : 0ull);
            if (!done) atomicAdd(&g_counters[1 + 3 * attempt], 1ull);  // [1] first miss, [4] second miss
        }
    }
    if (!done) topk_global(S, G, row, lo, n, k, out);
}

// Few long rows (decode): a cluster of kTkCluster CTAs per row, each sampling and streaming
// 1/kTkCluster of the row.  CTA 0 turns the samples (sent to it through distributed shared
// memory) into the threshold T0, aimed at rank 2k so that a miss is rare, and into the scale of a
// histogram of the candidates' key offsets from T0.  Every CTA streams its segment into its own
// warp regions and a local histogram of its candidates, which it then adds to CTA 0's
// (distributed shared-memory atomics, one per non-empty bin).
// The refinement is then spread over the cluster: CTA 0 finds the bin that holds the k-th key
// (narrowing it with further distributed histogram rounds while it holds more than kTkBndMax
// keys), the CTAs send that bin's members to CTA 0, which ranks them and broadcasts the exact
// cutoff (key, index); each CTA counts its kept keys per region, the counts are exchanged, and
// every CTA writes its own kept keys at its offsets.  The output order is the one-CTA kernel's:
// region w of the row is region w of CTA 0, then of CTA 1, ... (contiguous segments).  A miss
// (the candidates do not hold k keys, or a region overflows) re-aims and streams once more; a
// final bin of more than kTkBndMax equal keys, or a second miss, takes the exact radix select
// on CTA 0.  Dynamic shared memory: sizeof(TopkSmem).
constexpr int kTkBndMax = 256;
// Staged segments: after TopkSmem in the cluster kernel's dynamic shared memory, moved by bulk
// copies of at most kTkStageCopy bytes each; at most kTkStageMaxF4 float4 groups per CTA.
constexpr int kTkStageOffset = (int)((sizeof(TopkSmem) + 127) / 128 * 128);
constexpr uint32_t kTkStageCopy = 32768;
constexpr int kTkStageMaxF4 = 10240;  // 160 KiB

struct TopkClusterShared {
    int kept[kTkCluster][kTkWarps];  // kept keys per (CTA, region); every CTA writes its row into all
    uint32_t bkey[kTkBndMax];         // boundary-bin members (CTA 0)
    int bidx[kTkBndMax];
    int bn;                           // boundary-bin members received (CTA 0)
    uint32_t T0, sh;                  // threshold key and candidate-histogram shift (broadcast)
    uint32_t pv, need, cnt_b;         // refinement state (broadcast): prefix of the bin, keys still
    int fixed;                        // needed from it, its size, low offset bits not yet fixed
    uint32_t cut_key;                 // last kept key of the boundary bin (broadcast)
    int cut_idx;
    int above[kTkCluster][kTkWarps];  // keys above the boundary bin per (CTA, region) (CTA 0)
    int bkept[kTkCluster * kTkWarps]; // kept boundary-bin members per (CTA, region) (CTA 0)
    uint8_t borg[kTkBndMax];          // (CTA, region) of each boundary-bin member (CTA 0)
    int lab[kTkWarps];                // this CTA's above-bin counts per region
    uint32_t lhist[kTkBins];          // this CTA's candidate histogram, added to CTA 0's after the stream
};

__device__ __forceinline__ uint32_t rank_target_2k(long long m, long long n, int k) {
    // aim at rank 2k of the row, i.e. rank 2k * m / n of the m samples
    return (uint32_t)max(1LL, min(m - 1, (2LL * k * m + n - 1) / n));
}

// Float4 groups [g_lo, g_hi) of a row's competing keys [lo, n) that CTA `crank` of a cluster
// samples and streams: segments of whole groups of 4 pieces (32 float4), so that regions keep
// their meaning across CTAs.  Returns the segment length in float4 groups.
__device__ __forceinline__ int cluster_segment(int lo, int n, int crank, int& g_lo, int& g_hi) {
    const int n4 = (n + 3) >> 2, gw = lo >> 2;
    const int seg = ((n4 - (gw & ~31) + kTkCluster - 1) / kTkCluster + 31) & ~31;
    g_lo = min(n4, max(gw, (gw & ~31) + crank * seg));
    g_hi = min(n4, (gw & ~31) + (crank + 1) * seg);
    return seg;
}

// One row's selection by the cluster (every thread of every CTA calls it): ne = n - lo > k.
// This CTA reads its segment [g_lo, g_hi) of float4 groups at src4[g - g_base]: the row itself
// (staged false, g_base 0) or its shared-memory copy (staged true).  CTA 0's exact fallback reads
// the whole row.
__device__ __forceinline__ void cluster_select(TopkSmem& S, TopkClusterShared& C, int* src_cnt,
                                               cg::cluster_group& cluster, const float4* src4, int g_base,
                                               bool staged, int g_lo, int g_hi, int lo, int n, int k, int* out,
                                               const float* row) {
    const int crank = (int)cluster.block_rank();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const Grp G{tid};
    const int ne = n - lo;
    const int n4 = (n + 3) >> 2, gw = lo >> 2;
    TopkSmem* S0 = cluster.map_shared_rank(&S, 0);
    TopkClusterShared* C0 = cluster.map_shared_rank(&C, 0);

    // a quarter of the one-CTA kernel's samples (about n/128, 1024 for a 128K row): aimed at rank
    // 2k with no tight candidate capacity behind it, the estimate needs less precision (about 32
    // samples above the aim, so more than half of them falling below k is a rare miss), and CTA 0
    // turns every sample into the threshold alone (26.7 -> 24.7 us per call for 16 rows of 128K
    // keys against n/64 samples)
    const int s4 = sample_count4(n4 - gw, 4 * kTkCluster);  // per CTA
    const long long m = 4LL * s4 * kTkCluster;
    uint32_t rs = rank_target_2k(m, ne, k);
    bool done = false;
    for (int attempt = 0; attempt < 2 && !done; ++attempt) {
        // ---- samples of every segment into CTA 0, which sets T0 and the histogram scale
        take_samples(G, S0->cand_key, 4 * crank * s4, src4, g_base, g_lo, g_hi, lo, n, s4);
        cluster.sync();
        if (crank == 0) {
            uint32_t kmax = 0;
            const uint32_t t0 = sample_threshold(S, G, (int)m, rs, &kmax);
            // bins of width 2^sh over [T0, kmax] fill at most half the histogram: keys up to twice
            // the sampled range above T0 still get bins of their own
            const uint32_t span = kmax > t0 ? kmax - t0 : 0u;
            const uint32_t sh = (span >> 9) ? 32 - __clz(span >> 9) : 0;
            clear_hist(S, G, kTkBins);
            if (tid < kTkCluster) {
                TopkClusterShared* D = cluster.map_shared_rank(&C, tid);
                D->T0 = t0;
                D->sh = sh;
            }
        }
        cluster.sync();  // T0 everywhere, CTA 0's histogram cleared
        const uint32_t T0 = C.T0, sh = C.sh;

        // ---- stream this CTA's segment into its warp regions (a staged segment in batches of
        // 16 float4 per lane, each lane walking only its own candidates), then count the stored
        // candidates into a local histogram (a pass over shared memory whose atomics overlap,
        // instead of one inside the compaction loop) and add it to CTA 0's once (a remote atomic
        // per candidate made the stream 4x slower)
        for (int i = tid; i < kTkBins; i += kTkThreads) C.lhist[i] = 0u;
        const uint32_t c = staged ? stream_collect_staged(S, G, src4, g_lo, g_hi, lo, n, key_floor_float(T0),
                                                          warp * kTkRegion, g_base)
                                  : stream_collect(S, G, src4, g_lo, g_hi, lo, n, key_floor_float(T0),
                                                   warp * kTkRegion);
        if (lane == 0) S.reg_gt[warp] = (int)c;
        __syncthreads();
        for (int w = 0; w < kTkWarps; ++w) {
            const int cw = min(S.reg_gt[w], kTkRegion);
            for (int e = tid; e < cw; e += kTkThreads)
                atomicAdd(&C.lhist[min((S.cand_key[w * kTkRegion + e] - T0) >> sh, (uint32_t)kTkBins - 1u)], 1u);
        }
        __syncthreads();
        for (int i = tid; i < kTkBins; i += kTkThreads) {
            const uint32_t h = C.lhist[i];
            if (h) atomicAdd(&S0->hist[i], h);
        }
        cluster.sync();
        if (tid < kTkMaxRegions) src_cnt[tid] = cluster.map_shared_rank(&S, tid / kTkWarps)->reg_gt[tid % kTkWarps];
        __syncthreads();
        uint32_t total = 0;
        bool fits = true;
        for (int q = 0; q < kTkMaxRegions; ++q) {
            total += (uint32_t)src_cnt[q];
            fits = fits && src_cnt[q] <= kTkRegion;
        }
        fits = fits && total >= (uint32_t)k;  // uniform over the cluster
        if (crank == 0 && tid == 0) {
            atomicAdd(&g_counters[2], attempt == 0 ? 1ull : 0ull);
            if (!fits && attempt == 0) atomicAdd(&g_counters[3], 1ull);  // first miss
        }
        if (!fits) {
            rs = retarget(rs, total, m, k);
            cluster.sync();  // every CTA has read the counts before the next attempt rewrites them
            continue;
        }

        // ---- distributed refinement: the bin holding the k-th key, narrowed while it is large
        if (tid < kTkWarps) C.lab[tid] = 0;
        if (crank == 0) {
            // the member list and its per-region tallies start empty (filled after this barrier)
            if (tid == 0) C.bn = 0;
            if (tid < kTkCluster * kTkWarps) C.bkept[tid] = 0;
            find_threshold_bin(S, G, kTkBins, (uint32_t)k);
            if (tid < kTkCluster) {
                TopkClusterShared* D = cluster.map_shared_rank(&C, tid);
                D->pv = S.sel_bin << sh;
                D->fixed = (int)sh;
                D->need = (uint32_t)k - S.sel_gt;
                // a clamped top bin has no prefix: treat it as too large to resolve (exact fallback)
                D->cnt_b = S.sel_bin == (uint32_t)kTkBins - 1u ? 0xFFFFFFFFu : S.hist[S.sel_bin];
            }
        }
        cluster.sync();
        while (C.cnt_b != 0xFFFFFFFFu && C.cnt_b > (uint32_t)kTkBndMax && C.fixed > 0) {  // uniform
            const int fixed = C.fixed;
            const uint32_t pv = C.pv;
            const int sh2 = fixed > 10 ? fixed - 10 : 0;
            const int nb = 1 << (fixed - sh2);
            if (crank == 0) clear_hist(S, G, nb);
            cluster.sync();
            for (int w = 0; w < kTkWarps; ++w) {
                const int cw = min(S.reg_gt[w], kTkRegion);
                for (int e = tid; e < cw; e += kTkThreads) {
                    const uint32_t d = S.cand_key[w * kTkRegion + e] - T0;
                    if ((d >> fixed) == (pv >> fixed)) atomicAdd(&S0->hist[(d >> sh2) & (nb - 1)], 1u);
                }
            }
            cluster.sync();
            if (crank == 0) {
                find_threshold_bin(S, G, nb, C.need);
                if (tid < kTkCluster) {
                    TopkClusterShared* D = cluster.map_shared_rank(&C, tid);
                    D->need = C.need - S.sel_gt;
                    D->cnt_b = S.hist[S.sel_bin];
                    D->pv = pv | (S.sel_bin << sh2);
                    D->fixed = sh2;
                }
            }
            cluster.sync();
        }
        if (C.cnt_b > (uint32_t)kTkBndMax) break;  // more equal keys than the ranking handles: exact fallback
        const int fixed = C.fixed;
        const uint32_t pv = C.pv;
        auto in_bin = [&](uint32_t d) { return fixed >= 32 || (d >> fixed) == (pv >> fixed); };
        auto above = [&](uint32_t d) { return fixed < 32 && (d >> fixed) > (pv >> fixed); };
        // ---- the boundary bin's members (with their (CTA, region)) and every region's count of
        // keys above the bin go to CTA 0, which ranks the members, and broadcasts the cutoff and
        // each (CTA, region)'s kept count: the row offsets need no further exchange
        {
            uint32_t abv[kTkWarps];
#pragma unroll
            for (int w = 0; w < kTkWarps; ++w) {
                abv[w] = 0;
                const int cw = min(S.reg_gt[w], kTkRegion);
                for (int e = tid; e < cw; e += kTkThreads) {
                    const uint32_t key = S.cand_key[w * kTkRegion + e];
                    abv[w] += above(key - T0) ? 1u : 0u;
                    if (in_bin(key - T0)) {
                        const int p = atomicAdd(&C0->bn, 1);
                        if (p < kTkBndMax) {
                            C0->bkey[p] = key;
                            C0->bidx[p] = S.cand_idx[w * kTkRegion + e];
                            C0->borg[p] = (uint8_t)(crank * kTkWarps + w);
                        }
                    }
                }
            }
#pragma unroll
            for (int w = 0; w < kTkWarps; ++w) {
                uint32_t v = abv[w];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0 && v) atomicAdd(&C.lab[w], (int)v);
            }
            __syncthreads();
            if (tid < kTkWarps) C0->above[crank][tid] = C.lab[tid];
        }
        cluster.sync();
        if (crank == 0) {
            const int bn = min(C.bn, kTkBndMax);
            const uint32_t need = C.need;
            for (int a = tid; a < bn; a += kTkThreads) {
                const uint32_t ka = C.bkey[a];
                const int ia = C.bidx[a];
                uint32_t rank = 0;
                for (int b = 0; b < bn; ++b) {
                    const uint32_t kb = C.bkey[b];
                    rank += (kb > ka) || (kb == ka && C.bidx[b] < ia);
                }
                if (rank < need) atomicAdd(&C.bkept[C.borg[a]], 1);
                if (rank == need - 1u)  // exactly one member: the last kept one
                    for (int q = 0; q < kTkCluster; ++q) {
                        TopkClusterShared* D = cluster.map_shared_rank(&C, q);
                        D->cut_key = ka;
                        D->cut_idx = ia;
                    }
            }
            __syncthreads();  // CTA 0 only (uniform branch): every member tallied
            if (tid < kTkCluster * kTkWarps) {
                const int q = tid / kTkWarps, w = tid % kTkWarps;
                const int kq = C.above[q][w] + C.bkept[tid];
                for (int r2 = 0; r2 < kTkCluster; ++r2) cluster.map_shared_rank(&C, r2)->kept[q][w] = kq;
            }
        }
        cluster.sync();
        const uint32_t cut_key = C.cut_key;
        const int cut_idx = C.cut_idx;
        auto kept = [&](uint32_t key, int ix) {
            const uint32_t d = key - T0;
            return above(d) || (in_bin(d) && (key > cut_key || (key == cut_key && ix <= cut_idx)));
        };
        // ---- each CTA writes its own kept keys at the row's offsets
        {
            uint32_t base = 0;
            for (int w = 0; w < warp; ++w)
                for (int q = 0; q < kTkCluster; ++q) base += (uint32_t)C.kept[q][w];
            for (int q = 0; q < crank; ++q) base += (uint32_t)C.kept[q][warp];
            const int cw = min(S.reg_gt[warp], kTkRegion);
            for (int e0 = 0; e0 < cw; e0 += 32) {
                const int e = e0 + lane;
                const int ix = e < cw ? S.cand_idx[warp * kTkRegion + e] : 0;
                const bool keep = e < cw && kept(S.cand_key[warp * kTkRegion + e], ix);
                const uint32_t bk = __ballot_sync(0xffffffffu, keep);
                if (keep) out[base + __popc(bk & ((1u << lane) - 1u))] = ix;
                base += __popc(bk);
            }
        }
        done = true;
    }
    if (!done && crank == 0) {
        if (tid == 0) atomicAdd(&g_counters[5], 1ull);  // exact fallback
        topk_global(S, G, row, lo, n, k, out);
    }
    cluster.sync();  // peers keep their shared memory alive until every remote access is done
}

__global__ void __launch_bounds__(kTkThreads, 1) topk_cluster_kernel(const TopkParams P) {
    extern __shared__ __align__(1024) uint8_t topk_smem[];
    __shared__ TopkClusterShared C;
    __shared__ int src_cnt[kTkMaxRegions];
    __shared__ uint64_t stage_bar;
    TopkSmem& S = *reinterpret_cast<TopkSmem*>(topk_smem);
    cg::cluster_group cluster = cg::this_cluster();
    const int crank = (int)cluster.block_rank();
    const int r = blockIdx.x / kTkCluster, tid = threadIdx.x;
    const int n = (int)row_length(P, r, tid == 0 && crank == 0);
    const int lo = row_first_key(P, n), ne = n - lo;  // competing keys: [lo, n)
    const int k = P.k;
    int* out = P.idx + (long long)r * k;
    if (ne <= k) {  // uniform over the cluster
        if (crank == 0)
            for (int j = tid; j < k; j += kTkThreads) out[j] = j < ne ? lo + j : -1;
        return;
    }
    const float* row = P.scores + (long long)r * P.ld;
    int g_lo, g_hi;
    cluster_segment(lo, n, crank, g_lo, g_hi);
    // Staging: one bulk copy brings this CTA's segment (from its 32-group boundary, where the
    // stream starts) into shared memory while nothing else is waiting on it, so the samples and
    // the stream read shared memory instead of paying a DRAM round trip per batch.
    const int gs = g_lo & ~31;
    const bool stage = P.stage_f4 > 0 && g_hi > gs && g_hi - gs <= P.stage_f4;  // uniform in the CTA
    bool staged = false;
    const float4* src4 = reinterpret_cast<const float4*>(row);
    int g_base = 0;
    if (stage) {
        uint8_t* buf = topk_smem + kTkStageOffset;
        if (tid == 0) {
            mbar_init(&stage_bar, 1);
            fence_mbar_init();
            const uint32_t bytes = (uint32_t)(g_hi - gs) * 16u;
            const uint8_t* src = reinterpret_cast<const uint8_t*>(row) + (size_t)gs * 16;
            mbar_arrive_expect_tx(&stage_bar, bytes);
            for (uint32_t off = 0; off < bytes; off += kTkStageCopy)
                bulk_load(buf + off, src + off, min(kTkStageCopy, bytes - off), &stage_bar);
        }
        __syncthreads();
        staged = wait_parity(&stage_bar, 0, 0xA01u);
        if (staged) {
            src4 = reinterpret_cast<const float4*>(buf);
            g_base = gs;
        }
    }
    cluster_select(S, C, src_cnt, cluster, src4, g_base, staged, g_lo, g_hi, lo, n, k, out, row);
    // a copy that outlived a timed-out wait must land before this CTA's shared memory is released
    if (stage && !staged) wait_parity(&stage_bar, 0, 0xA02u);
}


}  // namespace dsa
