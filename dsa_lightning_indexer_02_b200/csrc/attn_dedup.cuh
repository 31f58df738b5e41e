// Sparse attention with adjacent-query deduplication (prefill).
//
// Page "快手开源大模型Keye-VL-2.0：一个能“看懂“两小时视频AI" (gsyq.cn), section 八: adjacent query
// tokens select largely the same keys, so a block of adjacent queries gathers the union of their
// index sets once and masks, per query, the union keys it did not select.  The result equals
// per-token sparse attention (the same softmax over each token's own selected keys, shared by its
// GQA KV group); only the order of the fp32 sums and the bf16 rounding of the probabilities differ.
//
// One CTA per (block of TBA = 128/G adjacent tokens, KV group g), G = Hq/Hkv query heads per group.
// The block's TBA x G (token, head) rows of group g are the M = 128 rows of every tcgen05 MMA:
//   S = Q K^T   (Q: 128 rows x 128 dims by TMA, K: 64 union keys x 128 dims, S in TMEM)
//   O += P V    (P: 128 rows x 64 keys in shared memory, V: 64 keys x 128 dims MN-major, O in TMEM)
// Roles (12 warps):
//   warps 0-3   union builder: counts the block's index entries per window of 2048 keys, groups
//               consecutive windows into super-windows of at most 8192 entries, scatters each
//               super-window's entries into a shared-memory bucket by window (one pass over the
//               rows per super-window, 16-byte loads), then per window ORs each token's bit into a
//               16-bit mask per key, compacts the keys with a non-zero mask into a ring of 64-key
//               tile descriptors and transposes the masks into one 64-bit mask per (tile, token).
//               Rows may list their keys in any order; empty windows cost nothing;
//   warps 4-7   softmax: warp w owns TMEM lanes 32(w%4)..+31, i.e. rows (token, head); reads S,
//               masks the keys its token did not select, online softmax in the exp2 domain with
//               the running maximum raised only when it grows by more than 2^8 (O then rescaled in
//               TMEM), writes P as bf16 into the 128-byte-swizzled K-major layout, and at the end
//               normalises O and stores it;
//   warp 8      TMEM allocation, the Q TMA loads and the single-thread MMA issue;
//   warps 9-11  K/V producers: warp i gathers tiles i, i+3, ... with 16-byte cp.async copies into
//               the swizzled layouts the MMA descriptors describe (K K-major, V MN-major).
// Every wait is bounded and sleeps while it waits (wait_parity_sleep); each waiter waits for every phase of the barriers it uses.
#pragma once

#include <climits>

#include "attn.cuh"
#include "ptx.cuh"

namespace dsa {

constexpr int kDdRows = 128;        // MMA M: (token, head) rows of one KV group
constexpr int kDdKeys = 64;         // union keys per tile
constexpr int kDdStages = 3;        // K/V stages = producer warps
constexpr int kDdRing = 39;         // tile descriptors (a multiple of kDdStages, > kDdWin/kDdKeys + 1)
constexpr int kDdWin = 2048;        // keys per union window (at most 32 tiles + 1 partial each)
constexpr int kDdBucket = 8192;     // entries of one super-window held in shared memory
constexpr int kDdMaxWin = 1024;     // windows per key range: n_keys <= kDdMaxWin * kDdWin
constexpr int kDdMaxTok = 16;       // tokens per block at most (masks are 16 bits per key)
constexpr int kDdBuildWarps = 4;
constexpr int kDdSoftWarps = 4;
constexpr int kDdMmaWarp = kDdBuildWarps + kDdSoftWarps;
constexpr int kDdProdWarp0 = kDdMmaWarp + 1;
constexpr int kDdThreads = (kDdProdWarp0 + kDdStages) * 32;
constexpr uint32_t kDdTmemCols = 256;  // S double buffer (2 x 64 columns) + O (128 columns)
constexpr int kDdTiltLog2 = 8;         // the running maximum is raised when exceeded by > 2^8

struct DedupParams {
    const __nv_bfloat16* k;  // [n_keys, Hkv, D]
    const __nv_bfloat16* v;
    const int* idx;           // [T, topk]
    int topk;
    int T;                    // tokens in this launch (rows of q, idx, out)
    long long q_pos0;         // token t sees the first min(topk, q_pos0 + t + 1 [, window]) entries
    long long n_keys;         // entries outside [0, n_keys) are skipped
    long long window;         // > 0: a row holds at most min(topk, window) entries
    int Hq, Hkv;
    float scale_log2;         // scale * log2(e)
    __nv_bfloat16* out;       // [T, Hq, D]
    float* lse;               // [T, Hq] natural-log LSE, may be null
    int nblk;                 // blocks of tokens per KV group
};

struct DdSlot {                 // one tile descriptor, 512 bytes
    int keys[kDdKeys];          // union keys (padding columns repeat a valid key)
    uint16_t emask[kDdKeys];    // per key: bit j = token j of the block selected it
    uint32_t tmask[kDdMaxTok][2];  // per token: bit c = it selected column c
};

struct DdMisc {
    uint64_t tfull[kDdRing], tempty[kDdRing];
    uint64_t kvfull[kDdStages], kvempty[kDdStages];
    uint64_t sfull[2], sempty[2], pfull[2], odone, qfull, mdone;
    int ring_cnt[kDdRing], ring_last[kDdRing];
    int scan[kDdBuildWarps];
    int bstop;                  // builder: stop (decided by its thread 0 before a barrier)
    uint32_t tmem_base;
    int abort;
};

constexpr int kDdQBytes = kDdRows * 128;          // one 64-dim half of Q (16 KB)
constexpr int kDdPBytes = kDdRows * 128;          // one P buffer (16 KB)
constexpr int kDdHalfBytes = kDdKeys * 128;       // 64 keys x 64 dims (8 KB)
constexpr int kDdStageBytes = 4 * kDdHalfBytes;   // K (2 halves) + V (2 halves)
constexpr int kDdOffQ = 0;
constexpr int kDdOffP = kDdOffQ + 2 * kDdQBytes;
constexpr int kDdOffKV = kDdOffP + 2 * kDdPBytes;
constexpr int kDdOffRing = kDdOffKV + kDdStages * kDdStageBytes;
constexpr int kDdOffWin = kDdOffRing + kDdRing * (int)sizeof(DdSlot);
constexpr int kDdOffBucket = kDdOffWin + kDdWin * 2;                 // uint32 [kDdBucket]
constexpr int kDdOffHist = kDdOffBucket + kDdBucket * 4;             // int [kDdMaxWin]: entries per window
constexpr int kDdOffWofs = kDdOffHist + kDdMaxWin * 4;               // int [kDdMaxWin]: bucket cursors
constexpr int kDdOffMisc = kDdOffWofs + kDdMaxWin * 4;
constexpr int kDdSmemBytes = kDdOffMisc + (int)sizeof(DdMisc);
static_assert(sizeof(DdSlot) == 512, "tile descriptor layout");
static_assert(kDdRing % kDdStages == 0, "a producer warp must see every phase of its ring slots");
static_assert(kDdSmemBytes <= 232448, "shared memory of one CTA");

// Entries a token's row holds (0 for tokens past the launch).
__device__ __forceinline__ int dd_row_count(const DedupParams& P, int t) {
    if (t >= P.T) return 0;
    long long n = P.q_pos0 + t + 1;
    if (P.window > 0 && n > P.window) n = P.window;
    return (int)min((long long)P.topk, n);
}

// Key of an index entry, INT_MAX for an entry naming no key.
__device__ __forceinline__ int dd_key(int e, long long n_keys) { return (e >= 0 && e < n_keys) ? e : INT_MAX; }

// Publish tile ti: transpose its per-key masks into per-token masks, then hand it to the roles.
template <int TBA>
__device__ __forceinline__ void dd_publish(DdSlot* ring, DdMisc& M, int ti, int cnt, int last, int lane) {
    const int slot = ti % kDdRing;
    DdSlot& S = ring[slot];
    const uint32_t m0 = S.emask[lane], m1 = S.emask[lane + 32];
    uint32_t my0 = 0, my1 = 0;
#pragma unroll
    for (int j = 0; j < TBA; ++j) {
        const uint32_t b0 = __ballot_sync(0xffffffffu, (m0 >> j) & 1u);
        const uint32_t b1 = __ballot_sync(0xffffffffu, (m1 >> j) & 1u);
        if (lane == j) {
            my0 = b0;
            my1 = b1;
        }
    }
    if (lane < TBA) {
        S.tmask[lane][0] = my0;
        S.tmask[lane][1] = my1;
    }
    if (lane == 0) {
        M.ring_cnt[slot] = cnt;
        M.ring_last[slot] = last;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&M.tfull[slot]);
}

// Calls fn(j, e) for every valid entry e of the block's token rows j = 0 .. TBA-1, spread over the
// builder's threads (bt = 0..127): 16-byte loads with eight in flight per thread when the rows are
// 16-byte aligned (topk % 4 == 0), else 4-byte loads.
template <int TBA, class Fn>
__device__ __forceinline__ void dd_for_entries(const DedupParams& P, int tb0, int bt, Fn fn) {
    constexpr int NT = 32 * kDdBuildWarps;
    if ((P.topk & 3) == 0) {
        const int q4 = P.topk >> 2;  // int4 per row
        const int total = TBA * q4;
        const int4* base = reinterpret_cast<const int4*>(P.idx + (long long)tb0 * P.topk);
        for (int g0 = bt; g0 < total; g0 += 8 * NT) {
            int4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int g = g0 + u * NT;
                const int j = g / q4;
                v[u] = (g < total && tb0 + j < P.T) ? __ldg(base + g) : make_int4(-1, -1, -1, -1);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int g = g0 + u * NT;
                const int j = g / q4, i = 4 * (g - j * q4);
                const int cnt = g < total ? dd_row_count(P, tb0 + j) : 0;
                const int ev[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int e = dd_key(ev[c], P.n_keys);
                    if (i + c < cnt && e != INT_MAX) fn(j, e);
                }
            }
        }
    } else {
        const int total = TBA * P.topk;
        const int* base = P.idx + (long long)tb0 * P.topk;
        for (int g0 = bt; g0 < total; g0 += 8 * NT) {
            int v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int g = g0 + u * NT;
                v[u] = (g < total && tb0 + g / P.topk < P.T) ? __ldg(base + g) : -1;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int g = g0 + u * NT;
                const int j = g / P.topk, i = g - j * P.topk;
                const int e = dd_key(v[u], P.n_keys);
                if (g < total && i < dd_row_count(P, tb0 + j) && e != INT_MAX) fn(j, e);
            }
        }
    }
}

template <int G>
__global__ void __launch_bounds__(kDdThreads, 1) attn_dedup_kernel(const __grid_constant__ CUtensorMap qmap,
                                                                    const DedupParams P) {
    constexpr int TBA = kDdRows / G;
    static_assert(TBA <= kDdMaxTok && TBA * G == kDdRows, "128 (token, head) rows per block");
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* sQ = smem + kDdOffQ;
    uint8_t* sP = smem + kDdOffP;
    uint8_t* sKV = smem + kDdOffKV;
    DdSlot* ring = reinterpret_cast<DdSlot*>(smem + kDdOffRing);
    uint32_t* wm = reinterpret_cast<uint32_t*>(smem + kDdOffWin);  // 16-bit token masks, two keys a word
    DdMisc& M = *reinterpret_cast<DdMisc*>(smem + kDdOffMisc);
    volatile int* abort_flag = &M.abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int blk = P.nblk - 1 - (int)(blockIdx.x / P.Hkv);  // the longest rows first
    const int g = (int)(blockIdx.x % P.Hkv);
    const int tb0 = blk * TBA;                                // first token of the block

    if (threadIdx.x == 0) {
        for (int i = 0; i < kDdRing; ++i) {
            mbar_init(&M.tfull[i], 1);
            mbar_init(&M.tempty[i], 2 + kDdSoftWarps);  // producer, MMA, softmax warps
        }
        for (int i = 0; i < kDdStages; ++i) {
            mbar_init(&M.kvfull[i], 32);
            mbar_init(&M.kvempty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&M.sfull[i], 1);
            mbar_init(&M.sempty[i], kDdSoftWarps);
            mbar_init(&M.pfull[i], kDdSoftWarps);
        }
        mbar_init(&M.odone, 1);
        mbar_init(&M.qfull, 1);
        mbar_init(&M.mdone, 1);
        M.abort = 0;
        fence_mbar_init();
        prefetch_tensormap(&qmap);
    }
    if (warp == kDdMmaWarp) {
        tmem_alloc(&M.tmem_base, kDdTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = M.tmem_base;

    if (warp < kDdBuildWarps) {
        // ================================================================ union builder
        const int bt = threadIdx.x;  // 0..127
        int* whist = reinterpret_cast<int*>(smem + kDdOffHist);
        int* wofs = reinterpret_cast<int*>(smem + kDdOffWofs);
        uint32_t* bucket = reinterpret_cast<uint32_t*>(smem + kDdOffBucket);
        const int nwin = (int)((P.n_keys + kDdWin - 1) / kDdWin);
        constexpr int NT = 32 * kDdBuildWarps;
        // ---- entries per window
        for (int i = bt; i < nwin; i += NT) whist[i] = 0;
        for (int i = bt; i < kDdWin / 2; i += NT) wm[i] = 0u;  // each window's compaction clears what it read
        named_bar_sync(1, NT);
        dd_for_entries<TBA>(P, tb0, bt, [&](int, int e) { atomicAdd(&whist[e / kDdWin], 1); });
        named_bar_sync(1, NT);

        int fill = 0;     // union keys emitted so far
        int claimed = 0;  // tiles whose slot is free for writing (thread 0's count)
        int pub = 0;      // tiles published
        bool ok = true;
        // Compaction of window [a, a + kDdWin) from wm into the tile ring; publishes completed tiles.
        auto emit_window = [&](int a) -> bool {
            constexpr int KPT = kDdWin / NT;  // keys per thread
            uint32_t wv[KPT / 2];
            int c = 0;
#pragma unroll
            for (int q = 0; q < KPT / 2; ++q) {
                wv[q] = wm[(KPT / 2) * bt + q];
                wm[(KPT / 2) * bt + q] = 0u;
                c += ((wv[q] & 0xFFFFu) != 0u) + ((wv[q] >> 16) != 0u);
            }
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            if (lane == 31) M.scan[warp] = incl;
            named_bar_sync(1, NT);
            int wbase = 0, total = 0;
#pragma unroll
            for (int w = 0; w < kDdBuildWarps; ++w) {
                const int sc = M.scan[w];
                wbase += w < warp ? sc : 0;
                total += sc;
            }
            if (bt == 0) {  // the slots of every position below fill + total must be free
                while (claimed * kDdKeys < fill + total) {
                    const int u = claimed / kDdRing;
                    if (u >= 1 && !wait_parity_sleep(&M.tempty[claimed % kDdRing], (u - 1) & 1,
                                               0xA01u | ((unsigned)claimed << 12), abort_flag))
                        break;
                    ++claimed;
                }
                M.bstop = *abort_flag;
            }
            // every builder thread takes the same branch: a named barrier has no time limit
            named_bar_sync(1, NT);
            if (M.bstop) return false;
            int pos = fill + wbase + incl - c;
#pragma unroll
            for (int q = 0; q < KPT / 2; ++q) {
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const uint32_t mk = (wv[q] >> (16 * hh)) & 0xFFFFu;
                    if (mk) {
                        DdSlot& S = ring[(pos / kDdKeys) % kDdRing];
                        S.keys[pos % kDdKeys] = a + KPT * bt + 2 * q + hh;
                        S.emask[pos % kDdKeys] = (uint16_t)mk;
                        ++pos;
                    }
                }
            }
            named_bar_sync(1, NT);
            // the tiles this window completed; later windows write only at positions >= fill
            fill += total;
            const int done = fill / kDdKeys;
            for (int ti = pub + warp; ti < done; ti += kDdBuildWarps) dd_publish<TBA>(ring, M, ti, kDdKeys, 0, lane);
            pub = done;
            return true;
        };
        auto set_bit = [&](int off, int j) { atomicOr(&wm[off >> 1], (1u << j) << ((off & 1) * 16)); };

        // ---- windows in key order; consecutive windows share one bucket fill (a super-window)
        for (int w = 0; ok;) {
            while (w < nwin && whist[w] == 0) ++w;
            if (w >= nwin) break;
            if (whist[w] > kDdBucket) {
                // more entries than the bucket holds (early rows select all their keys): read the
                // rows directly for this one window
                const int a = w * kDdWin;
                dd_for_entries<TBA>(P, tb0, bt, [&](int j, int e) {
                    if (e >= a && e < a + kDdWin) set_bit(e - a, j);
                });
                named_bar_sync(1, NT);
                ok = emit_window(a);
                ++w;
                continue;
            }
            int w2 = w, tot = 0;
            while (w2 < nwin && tot + whist[w2] <= kDdBucket) tot += whist[w2++];
            if (bt == 0) {
                int o = 0;
                for (int x = w; x < w2; ++x) {
                    wofs[x] = o;
                    o += whist[x];
                }
            }
            named_bar_sync(1, NT);
            const int lo = w * kDdWin, hi = w2 * kDdWin;
            dd_for_entries<TBA>(P, tb0, bt, [&](int j, int e) {
                if (e >= lo && e < hi) bucket[atomicAdd(&wofs[e / kDdWin], 1)] = ((uint32_t)(e - lo) << 4) | (uint32_t)j;
            });
            named_bar_sync(1, NT);
            for (int x = w; x < w2 && ok; ++x) {
                const int n = whist[x];
                if (n == 0) continue;
                const int start = wofs[x] - n, woff = (x - w) * kDdWin;
                for (int i = bt; i < n; i += NT) {
                    const uint32_t v = bucket[start + i];
                    set_bit((int)(v >> 4) - woff, (int)(v & 15u));
                }
                named_bar_sync(1, NT);
                ok = emit_window(x * kDdWin);
            }
            named_bar_sync(1, NT);  // the bucket and cursors are refilled next
            w = w2;
        }
        named_bar_sync(1, NT);
        if (ok) {
            // The last tile: the partial one (padded), or an empty end marker.  Every producer warp
            // waits on its own tiles only, so end markers follow for the next kDdStages - 1 indices.
            const int ti = fill / kDdKeys, rem = fill % kDdKeys;
            if (bt == 0) {
                while (claimed < ti + kDdStages) {
                    const int u = claimed / kDdRing;
                    if (u >= 1 && !wait_parity_sleep(&M.tempty[claimed % kDdRing], (u - 1) & 1, 0xA02u | ((unsigned)claimed << 12), abort_flag)) break;
                    ++claimed;
                }
                M.bstop = *abort_flag;
            }
            named_bar_sync(1, 32 * kDdBuildWarps);
            if (!M.bstop && warp == 0) {
                DdSlot& S = ring[ti % kDdRing];
                if (rem > 0) {
                    for (int col = rem + lane; col < kDdKeys; col += 32) {
                        S.keys[col] = S.keys[0];
                        S.emask[col] = 0;
                    }
                }
                __syncwarp();
                dd_publish<TBA>(ring, M, ti, rem, 1, lane);
                for (int m = 1; m < kDdStages; ++m) dd_publish<TBA>(ring, M, ti + m, 0, 1, lane);
            }
        }
    } else if (warp < kDdMmaWarp) {
        // ================================================================ softmax
        const int q4 = warp & 3;           // TMEM lane quarter
        const int r = q4 * 32 + lane;      // row = token * G + head
        const int jt = r / G, h = r % G;
        const uint32_t trow = tmem + ((uint32_t)(q4 * 32) << 16);
        float m_st = -INFINITY, l = 0.f;
        int j = 0, pv_seen = 0;  // PV completions waited for, in order
        bool ok = true;
        // wait, in order, for the completion of PV(0 .. upto-1)
        auto wait_pv = [&](int upto) {
            while (ok && pv_seen < upto) {
                ok = wait_parity_sleep(&M.odone, pv_seen & 1, 0xA32u | ((unsigned)pv_seen << 12), abort_flag);
                ++pv_seen;
            }
        };
        for (;; ++j) {
            const int slot = j % kDdRing;
            ok = wait_parity_sleep(&M.tfull[slot], (j / kDdRing) & 1, 0xA30u | ((unsigned)j << 12), abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            const int cnt = M.ring_cnt[slot], last = M.ring_last[slot];
            const uint32_t mk0 = ring[slot].tmask[jt][0], mk1 = ring[slot].tmask[jt][1];
            __syncwarp();
            if (lane == 0) mbar_arrive(&M.tempty[slot]);
            if (cnt == 0 && last) break;
            const int b = j & 1;
            ok = __all_sync(0xffffffffu, wait_parity_sleep(&M.sfull[b], (j >> 1) & 1, 0xA31u | ((unsigned)j << 12), abort_flag));
            if (!ok) break;
            tc_fence_after();
            float x[kDdKeys];
            tmem_ld_32x32b_x32(trow + b * kDdKeys, *reinterpret_cast<float(*)[32]>(x));
            tmem_ld_32x32b_x32(trow + b * kDdKeys + 32, *reinterpret_cast<float(*)[32]>(x + 32));
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&M.sempty[b]);
            // row maximum over the selected columns (eight independent partial maxima: a single
            // warp per SM sub-partition runs this, so dependent chains would set its pace)
            float mx[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) mx[i] = -INFINITY;
#pragma unroll
            for (int c = 0; c < kDdKeys; ++c) {
                const uint32_t sel = c < 32 ? (mk0 >> c) & 1u : (mk1 >> (c - 32)) & 1u;
                x[c] = sel ? x[c] * P.scale_log2 : -INFINITY;
                mx[c & 7] = fmaxf(mx[c & 7], x[c]);
            }
            const float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                   fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
            const bool raise = mt > m_st + (float)kDdTiltLog2;
            const bool rescale_o = raise && m_st != -INFINITY;  // O holds this row's earlier terms
            if (__any_sync(0xffffffffu, rescale_o)) {
                wait_pv(j);  // PV(j-1) must have landed in O
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after();
                const float alpha = rescale_o ? ex2_approx(m_st - mt) : 1.f;
#pragma unroll 1
                for (int cc = 0; cc < 4; ++cc) {
                    float o[32];
                    tmem_ld_32x32b_x32(trow + 128 + 32 * cc, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] *= alpha;
                    tmem_st_32x32b_x32(trow + 128 + 32 * cc, o);
                }
                tmem_st_wait();
                l *= alpha;
            }
            if (raise) m_st = mt;
            const float mref = m_st == -INFINITY ? 0.f : m_st;
            uint32_t pk[kDdKeys / 2];
            float sm[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) sm[i] = 0.f;
#pragma unroll
            for (int c = 0; c < kDdKeys / 2; ++c) {
                const float p0 = ex2_approx(x[2 * c] - mref), p1 = ex2_approx(x[2 * c + 1] - mref);
                sm[c & 7] += p0 + p1;
                pk[c] = pack_bf16x2(p0, p1);
            }
            l += ((sm[0] + sm[1]) + (sm[2] + sm[3])) + ((sm[4] + sm[5]) + (sm[6] + sm[7]));
            // P row r, K-major with 128-byte swizzle: 16-byte chunk c8 (keys 8c8..8c8+7) at c8 ^ (r & 7)
            uint8_t* prow = sP + b * kDdPBytes + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8)
                *reinterpret_cast<uint4*>(prow + ((c8 ^ (r & 7)) << 4)) =
                    make_uint4(pk[4 * c8], pk[4 * c8 + 1], pk[4 * c8 + 2], pk[4 * c8 + 3]);
            fence_proxy_async_smem();
            wait_pv(j);  // keeps the PV waits in order (PV(j-1) is normally long done)
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&M.pfull[b]);
            if (last) {
                ++j;
                break;
            }
        }
        // j = tiles processed; wait for the last PV, then normalise and store
        if (ok) {
            wait_pv(j);
            ok = __all_sync(0xffffffffu, ok);
        }
        if (ok) {
            tc_fence_after();
            const int t = tb0 + jt;
            const float inv = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16* orow = P.out + ((long long)t * P.Hq + g * G + h) * kAttnD;
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
                float o[32];
                if (j > 0) {
                    tmem_ld_32x32b_x32(trow + 128 + 32 * cc, o);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = 0.f;
                }
                if (t < P.T) {
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        reinterpret_cast<uint4*>(orow + 32 * cc)[i] =
                            make_uint4(pack_bf16x2(o[8 * i] * inv, o[8 * i + 1] * inv),
                                       pack_bf16x2(o[8 * i + 2] * inv, o[8 * i + 3] * inv),
                                       pack_bf16x2(o[8 * i + 4] * inv, o[8 * i + 5] * inv),
                                       pack_bf16x2(o[8 * i + 6] * inv, o[8 * i + 7] * inv));
                }
            }
            if (P.lse && t < P.T)
                P.lse[(long long)t * P.Hq + g * G + h] = l > 0.f ? (m_st + log2f(l)) * 0.6931471805599453f : -INFINITY;
        }
    } else if (warp == kDdMmaWarp) {
        // ================================================================ TMA for Q, MMA issue
        if (lane == 0) {
            mbar_arrive_expect_tx(&M.qfull, 2 * kDdQBytes);
            tma_load_3d(sQ, &qmap, &M.qfull, 0, g * G, tb0);
            tma_load_3d(sQ + kDdQBytes, &qmap, &M.qfull, 64, g * G, tb0);
            constexpr uint32_t idS = idesc_bf16_f32<kDdRows, kDdKeys>();
            constexpr uint32_t idO = idesc_bf16_f32_bmn<kDdRows, kAttnD>();
            bool ok = wait_parity_sleep(&M.qfull, 0, 0xA20, abort_flag);
            const uint64_t qd[2] = {smem_desc_k128_sw128(sQ), smem_desc_k128_sw128(sQ + kDdQBytes)};
            // O += P(jp) V(jp): K = 16 keys per MMA (32 bytes of a P row, two 8-key groups of V)
            auto issue_pv = [&](int jp) {
                const int b = jp & 1, s = jp % kDdStages;
                if (!wait_parity_sleep(&M.pfull[b], (jp >> 1) & 1, 0xA21u | ((unsigned)jp << 12), abort_flag)) return false;
                tc_fence_after();
                const uint64_t pd = smem_desc_k128_sw128(sP + b * kDdPBytes);
                const uint64_t vd = smem_desc_mn_sw128(sKV + s * kDdStageBytes + 2 * kDdHalfBytes, kDdHalfBytes);
#pragma unroll
                for (int kk = 0; kk < kDdKeys / 16; ++kk)
                    umma_bf16(tmem + 128, pd + 2 * kk, vd + (2048 >> 4) * kk, idO, (jp > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&M.kvempty[s]);
                umma_commit(&M.odone);
                return true;
            };
            int j = 0;
            for (; ok; ++j) {
                const int slot = j % kDdRing;
                if (!(ok = wait_parity_sleep(&M.tfull[slot], (j / kDdRing) & 1, 0xA22u | ((unsigned)j << 12), abort_flag))) break;
                const int cnt = M.ring_cnt[slot], last = M.ring_last[slot];
                mbar_arrive(&M.tempty[slot]);
                if (cnt == 0 && last) break;
                const int s = j % kDdStages, b = j & 1;
                ok = wait_parity_sleep(&M.kvfull[s], (j / kDdStages) & 1, 0xA23u | ((unsigned)j << 12), abort_flag) &&
                     (j < 2 || wait_parity_sleep(&M.sempty[b], ((j >> 1) - 1) & 1, 0xA24u | ((unsigned)j << 12), abort_flag));
                if (!ok) break;
                tc_fence_after();
                const uint8_t* kst = sKV + s * kDdStageBytes;
                const uint64_t kd[2] = {smem_desc_k128_sw128(kst), smem_desc_k128_sw128(kst + kDdHalfBytes)};
                // S = Q K^T: K = 16 dims per MMA, 32 bytes along the 128-byte rows of each half
#pragma unroll
                for (int kk = 0; kk < kAttnD / 16; ++kk)
                    umma_bf16(tmem + b * kDdKeys, qd[kk >> 2] + 2 * (kk & 3), kd[kk >> 2] + 2 * (kk & 3), idS,
                              kk > 0 ? 1u : 0u);
                umma_commit(&M.sfull[b]);
                if (j >= 1 && !(ok = issue_pv(j - 1))) break;
                if (last) {
                    ++j;
                    break;
                }
            }
            if (ok && j >= 1) issue_pv(j - 1);
            if (!ok) wait_parity_sleep(&M.qfull, 0, 0xA25, nullptr);  // the Q copy must land before exit
            // every MMA issued has completed before the CTA frees TMEM
            umma_commit(&M.mdone);
            wait_parity_sleep(&M.mdone, 0, 0xA26, nullptr);
        }
        __syncwarp();
    } else {
        // ================================================================ K/V producers
        const int pw = warp - kDdProdWarp0;
        uint8_t* sK = sKV + pw * kDdStageBytes;
        uint8_t* sV = sK + 2 * kDdHalfBytes;
        const long long rs = (long long)P.Hkv * kAttnD;  // elements per key row
        const __nv_bfloat16* kb = P.k + g * kAttnD;
        const __nv_bfloat16* vb = P.v + g * kAttnD;
        // lanes 0-15 copy the 16 chunks of one key's row, lanes 16-31 the next key's
        const int sub = lane >> 4, c = lane & 15, half = c >> 3, cc = c & 7;
        for (int j = pw;; j += kDdStages) {
            const int slot = j % kDdRing;
            if (!__all_sync(0xffffffffu, wait_parity_sleep(&M.tfull[slot], (j / kDdRing) & 1, 0xA10u | ((unsigned)j << 12), abort_flag))) break;
            const int cnt = M.ring_cnt[slot], last = M.ring_last[slot];
            if (cnt == 0 && last) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&M.tempty[slot]);
                break;
            }
            const int use = j / kDdStages;
            if (use >= 1 &&
                !__all_sync(0xffffffffu, wait_parity_sleep(&M.kvempty[pw], (use - 1) & 1, 0xA11u | ((unsigned)j << 12), abort_flag)))
                break;
#pragma unroll 4
            for (int i = 0; i < kDdKeys / 2; ++i) {
                const int kk = 2 * i + sub;
                const long long key = ring[slot].keys[kk];
                // 128-byte swizzle: 16-byte chunk cc of row kk (within its 8-row group) at cc ^ (kk & 7)
                const uint32_t off = half * kDdHalfBytes + (kk >> 3) * 1024 + (kk & 7) * 128 + ((cc ^ (kk & 7)) << 4);
                cp_async_16(sK + off, kb + key * rs + c * 8, true);
                cp_async_16(sV + off, vb + key * rs + c * 8, true);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&M.tempty[slot]);
            cp_async_commit();
            cp_async_wait<0>();
            fence_proxy_async_smem();
            mbar_arrive(&M.kvfull[pw]);
            if (last) break;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kDdMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kDdTmemCols);
    }
}

}  // namespace dsa
