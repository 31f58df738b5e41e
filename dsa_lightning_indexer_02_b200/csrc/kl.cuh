// Indexer warm-up target, forward only: for every query row t of a causal sequence
//   P_t(s) = (1/Hq) sum_h softmax_s(scale * q[t,h] . k[s,g(h)])     s = 0..t (dense attention)
//   Q_t(s) = softmax_s(score(t, s))                                  (the lightning indexer's scores)
//   KL_t   = sum_s P_t(s) * (log P_t(s) - log Q_t(s))
//          = sum_s P_t(s) * (ln P_t(s) - score(t, s)) + LSE_s score(t, s)      (sum_s P_t(s) = 1)
// (page "快手开源大模型Keye-VL-2.0：一个能“看懂“两小时视频AI", gsyq.cn, section 一: training stage 1
// fits the scout to the full attention distribution by minimising a KL divergence; the pages give
// no formula, this is the plainest reading of it).
//
// Dense and tensor-core bound: 2 x 2 x Hq x D flop per causal (t, s) pair over two passes, plus
// about 2 x Hq exponentials per pair.  Two tcgen05 kernels, each fed by TMA:
//   kl_lse_kernel (pass 1): one CTA per (block of 128/G tokens, KV group g).  S = Q_g K^T with the
//     block's 128 (token, head) rows as M and 128-key tiles as N, in TMEM (double buffered).  Four
//     epilogue warpgroups take 32 of the 128 columns each and keep an online (max, sum) of
//     2^(scale log2e z) per row; the four partial results merge once at the end into the row's
//     log2-domain log-sum-exp, lse2[t, h].
//   kl_div_kernel (pass 2): one CTA per block of 256/Hq tokens, all heads.  Per 128-key tile and
//     KV group, S^T = K_g Q_g^T with the keys as M (TMEM lanes) and the block's (token, head)
//     columns of group g as N, so that a thread holds every head of its key for its tokens: the
//     head sum P_t(s) = sum_h 2^(scale log2e z - lse2[t,h]) / Hq stays in registers (the block's
//     lse2 values are a shared-memory broadcast).  The thread accumulates P (ln P - score) and an
//     online log-sum-exp of the indexer scores over its keys; the 128 key lanes are reduced at
//     the end.
// Both: warp 0 issues the TMA loads, warp 1 allocates TMEM and issues the MMAs (one thread), warps
// 2-3 idle, warpgroups 1-4 run the epilogue.  Every wait is bounded (wait_parity_sleep).
#pragma once

#include "ptx.cuh"

namespace dsa {

constexpr int kKlD = 128;
constexpr int kKlKeys = 128;          // keys per tile
constexpr int kKlStages = 4;          // K tile ring (32 KB per stage)
constexpr int kKlThreads = 640;       // role warpgroup + 4 epilogue warpgroups
constexpr int kKlHalfBytes = kKlKeys * 128;   // 128 rows x 64 dims
constexpr int kKlStageBytes = 2 * kKlHalfBytes;

// ------------------------------------------------------------------ pass 1: per-head LSE
struct KlLseParams {
    int T;               // tokens in this launch
    long long q_pos0;    // row i is query position q_pos0 + i
    int Hq, Hkv;
    float scale_log2;    // scale * log2(e)
    float* lse2;         // [T, Hq] log2-domain log-sum-exp of scale_log2 * q.k over keys 0..t
    int nblk;            // blocks of 128/G tokens
};

// Q (2 x 16 KB) | K ring | barriers | partial (max, sum) per (column quarter, row) | misc
constexpr int kKlLseOffK = 2 * 128 * 128;
constexpr int kKlLseOffBar = kKlLseOffK + kKlStages * kKlStageBytes;
constexpr int kKlLseOffPart = kKlLseOffBar + 256;
constexpr int kKlLseOffMisc = kKlLseOffPart + 4 * 128 * 8;
constexpr int kKlLseSmem = kKlLseOffMisc + 16;

template <int G>
__global__ void __launch_bounds__(kKlThreads, 1) kl_lse_kernel(const __grid_constant__ CUtensorMap qmap,
                                                                const __grid_constant__ CUtensorMap kmap,
                                                                const KlLseParams P) {
    constexpr int TBA = 128 / G;  // tokens per block
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* sQ = smem;
    uint8_t* sK = smem + kKlLseOffK;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kKlLseOffBar);
    uint64_t *kfull = bars, *kempty = bars + kKlStages, *sfull = bars + 2 * kKlStages;
    uint64_t *sempty = sfull + 2, *qfull = sfull + 4;
    float2* part = reinterpret_cast<float2*>(smem + kKlLseOffPart);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kKlLseOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kKlLseOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int blk = P.nblk - 1 - (int)(blockIdx.x / P.Hkv);  // the most keys first
    const int g = (int)(blockIdx.x % P.Hkv);
    const int tb0 = blk * TBA;
    const long long t_last = P.q_pos0 + min(tb0 + TBA, P.T) - 1;
    const int ntiles = (int)(t_last / kKlKeys) + 1;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kKlStages; ++i) {
            mbar_init(&kfull[i], 1);
            mbar_init(&kempty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sfull[i], 1);
            mbar_init(&sempty[i], 16);  // one arrival per epilogue warp
        }
        mbar_init(qfull, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&qmap);
        prefetch_tensormap(&kmap);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            mbar_arrive_expect_tx(qfull, 2 * 128 * 128);
            tma_load_3d(sQ, &qmap, qfull, 0, g * G, tb0);
            tma_load_3d(sQ + 128 * 128, &qmap, qfull, 64, g * G, tb0);
            int kt = 0;
            for (; kt < ntiles; ++kt) {
                const int st = kt % kKlStages, use = kt / kKlStages;
                if (use >= 1 && !wait_parity_sleep(&kempty[st], (use - 1) & 1, 0xB01, abort_flag)) break;
                mbar_arrive_expect_tx(&kfull[st], kKlStageBytes);
                tma_load_3d(sK + st * kKlStageBytes, &kmap, &kfull[st], 0, g, kt * kKlKeys);
                tma_load_3d(sK + st * kKlStageBytes + kKlHalfBytes, &kmap, &kfull[st], 64, g, kt * kKlKeys);
            }
            if (kt < ntiles) {  // gave up: let the copies in flight land (bounded) before leaving
                wait_parity_sleep(qfull, 0, 0xB02, nullptr);
                for (int i = max(0, kt - kKlStages); i < kt; ++i)
                    wait_parity_sleep(&kfull[i % kKlStages], (i / kKlStages) & 1, 0xB03, nullptr);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32<128, kKlKeys>();
            bool ok = wait_parity_sleep(qfull, 0, 0xB10, abort_flag);
            const uint64_t qd[2] = {smem_desc_k128_sw128(sQ), smem_desc_k128_sw128(sQ + 128 * 128)};
            for (int kt = 0; ok && kt < ntiles; ++kt) {
                const int st = kt % kKlStages, b = kt & 1;
                ok = wait_parity_sleep(&kfull[st], (kt / kKlStages) & 1, 0xB11, abort_flag) &&
                     (kt < 2 || wait_parity_sleep(&sempty[b], ((kt >> 1) - 1) & 1, 0xB12, abort_flag));
                if (!ok) break;
                tc_fence_after();
                const uint8_t* kst = sK + st * kKlStageBytes;
                const uint64_t kd[2] = {smem_desc_k128_sw128(kst), smem_desc_k128_sw128(kst + kKlHalfBytes)};
#pragma unroll
                for (int kk = 0; kk < kKlD / 16; ++kk)
                    umma_bf16(tmem + b * kKlKeys, qd[kk >> 2] + 2 * (kk & 3), kd[kk >> 2] + 2 * (kk & 3), idesc,
                              kk > 0 ? 1u : 0u);
                umma_commit(&kempty[st]);
                umma_commit(&sfull[b]);
            }
        }
    } else if (warp >= 4) {
        // epilogue: warpgroup wg takes columns 32 wg .. 32 wg + 31 of every S tile
        const int et = threadIdx.x - 128, wg = et >> 7, q4 = warp & 3;
        const int r = q4 * 32 + lane;  // row = token * G + head
        const int jt = r / G;
        const long long t = P.q_pos0 + tb0 + jt;
        const uint32_t trow = tmem + ((uint32_t)(q4 * 32) << 16) + wg * 32;
        float m = -INFINITY, sum = 0.f;
        bool ok = true;
        for (int kt = 0; kt < ntiles; ++kt) {
            const int b = kt & 1;
            ok = __all_sync(0xffffffffu, wait_parity_sleep(&sfull[b], (kt >> 1) & 1, 0xB20, abort_flag));
            if (!ok) break;
            tc_fence_after();
            float x[32];
            tmem_ld_32x32b_x32(trow + b * kKlKeys, x);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sempty[b]);
            // keys of this thread's columns: kt*128 + 32 wg + c; only the row's last tiles hold keys
            // past t (masked: logit -inf)
            const int past = (int)((long long)kt * kKlKeys + wg * 32 - t);  // key - t at c = 0
            float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            if (past + 31 <= 0) {
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    x[c] *= P.scale_log2;
                    mx[c & 3] = fmaxf(mx[c & 3], x[c]);
                }
            } else {
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    x[c] = past + c <= 0 ? x[c] * P.scale_log2 : -INFINITY;
                    mx[c & 3] = fmaxf(mx[c & 3], x[c]);
                }
            }
            const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            if (mt > m) {
                sum *= ex2_approx(m - mt);  // m = -inf: 0 * 0
                m = mt;
            }
            float sm[4] = {0.f, 0.f, 0.f, 0.f};
            const float mref = m == -INFINITY ? 0.f : m;
#pragma unroll
            for (int c = 0; c < 32; ++c) sm[c & 3] += ex2_approx(x[c] - mref);
            sum += (sm[0] + sm[1]) + (sm[2] + sm[3]);
        }
        // merge the four column quarters of each row
        part[wg * 128 + r] = make_float2(m, sum);
        named_bar_sync(1, 512);
        if (ok && wg == 0 && tb0 + jt < P.T) {
            float M = -INFINITY;
#pragma unroll
            for (int i = 0; i < 4; ++i) M = fmaxf(M, part[i * 128 + r].x);
            float S = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 pi = part[i * 128 + r];
                if (pi.x != -INFINITY) S += pi.y * ex2_approx(pi.x - M);
            }
            P.lse2[(long long)(tb0 + jt) * P.Hq + g * G + (r % G)] = M + log2f(S);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ------------------------------------------------------------------ pass 2: KL per row
struct KlDivParams {
    const float* scores;   // indexer scores of this launch's rows: row i at scores + i * ld, keys 0..q_pos0+i
    long long ld;
    int T;
    long long q_pos0;
    float scale_log2;
    const float* lse2;     // [T, Hq] from pass 1
    float* kl;             // [T]
    int nblk;              // blocks of 256/Hq tokens
};

// Q (256 rows x 256 bytes) | K ring | barriers | reduction scratch | lse2 of the block | misc
constexpr int kKlDivOffK = 256 * 256;
constexpr int kKlDivOffBar = kKlDivOffK + kKlStages * kKlStageBytes;
constexpr int kKlDivOffRed = kKlDivOffBar + 256;
constexpr int kKlDivOffL2 = kKlDivOffRed + 16 * 16 * 12;
constexpr int kKlDivOffMisc = kKlDivOffL2 + 256 * 4;
constexpr int kKlDivSmem = kKlDivOffMisc + 16;

template <int HQ, int HKV>
__global__ void __launch_bounds__(kKlThreads, 1) kl_div_kernel(const __grid_constant__ CUtensorMap qmap,
                                                                const __grid_constant__ CUtensorMap kmap,
                                                                const KlDivParams P) {
    constexpr int G = HQ / HKV;
    constexpr int TB = 256 / HQ;        // tokens per block
    constexpr int NG = TB * G;          // MMA N per group (= 256 / HKV)
    constexpr int TPW = TB / 4;         // tokens per epilogue warpgroup
    constexpr int CPG = TPW * G;        // a warpgroup's columns per group (= 64 / HKV)
    static_assert(TB % 4 == 0 && TPW <= 16 && NG % 16 == 0 && NG <= 256 && CPG % 16 == 0, "block shape");
    constexpr float kLn2 = 0.69314718055994531f;
    constexpr float kLog2e = 1.4426950408889634f;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* sQ = smem;  // group g: rows g*NG .. as two 64-dim halves of NG rows
    uint8_t* sK = smem + kKlDivOffK;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kKlDivOffBar);
    uint64_t *kfull = bars, *kempty = bars + kKlStages, *afull = bars + 2 * kKlStages;
    uint64_t *aempty = afull + 2, *qfull = afull + 4;
    float* red = reinterpret_cast<float*>(smem + kKlDivOffRed);
    float* l2s = reinterpret_cast<float*>(smem + kKlDivOffL2);  // [TB][HQ]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kKlDivOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kKlDivOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int blk = P.nblk - 1 - (int)blockIdx.x;
    const int tb0 = blk * TB;
    const long long t_last = P.q_pos0 + min(tb0 + TB, P.T) - 1;
    const int ntiles = (int)(t_last / kKlKeys) + 1;
    const int nloads = ntiles * HKV;  // K tiles (key tile, group) in order

    if (threadIdx.x == 0) {
        for (int i = 0; i < kKlStages; ++i) {
            mbar_init(&kfull[i], 1);
            mbar_init(&kempty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&afull[i], 1);
            mbar_init(&aempty[i], 16);
        }
        mbar_init(qfull, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&qmap);
        prefetch_tensormap(&kmap);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            mbar_arrive_expect_tx(qfull, 256 * 256);
#pragma unroll
            for (int gg = 0; gg < HKV; ++gg) {
                tma_load_3d(sQ + gg * NG * 256, &qmap, qfull, 0, gg * G, tb0);
                tma_load_3d(sQ + gg * NG * 256 + NG * 128, &qmap, qfull, 64, gg * G, tb0);
            }
            int i = 0;
            for (; i < nloads; ++i) {
                const int st = i % kKlStages, use = i / kKlStages;
                if (use >= 1 && !wait_parity_sleep(&kempty[st], (use - 1) & 1, 0xB31, abort_flag)) break;
                const int kt = i / HKV, gg = i % HKV;
                mbar_arrive_expect_tx(&kfull[st], kKlStageBytes);
                tma_load_3d(sK + st * kKlStageBytes, &kmap, &kfull[st], 0, gg, kt * kKlKeys);
                tma_load_3d(sK + st * kKlStageBytes + kKlHalfBytes, &kmap, &kfull[st], 64, gg, kt * kKlKeys);
            }
            if (i < nloads) {
                wait_parity_sleep(qfull, 0, 0xB32, nullptr);
                for (int j = max(0, i - kKlStages); j < i; ++j)
                    wait_parity_sleep(&kfull[j % kKlStages], (j / kKlStages) & 1, 0xB33, nullptr);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32<kKlKeys, NG>();
            bool ok = wait_parity_sleep(qfull, 0, 0xB40, abort_flag);
            for (int kt = 0; ok && kt < ntiles; ++kt) {
                const int b = kt & 1;
                if (kt >= 2 && !(ok = wait_parity_sleep(&aempty[b], ((kt >> 1) - 1) & 1, 0xB41, abort_flag))) break;
#pragma unroll 1
                for (int gg = 0; gg < HKV; ++gg) {
                    const int i = kt * HKV + gg, st = i % kKlStages;
                    if (!(ok = wait_parity_sleep(&kfull[st], (i / kKlStages) & 1, 0xB42, abort_flag))) break;
                    tc_fence_after();
                    const uint8_t* kst = sK + st * kKlStageBytes;
                    const uint64_t ad[2] = {smem_desc_k128_sw128(kst), smem_desc_k128_sw128(kst + kKlHalfBytes)};
                    const uint8_t* qg = sQ + gg * NG * 256;
                    const uint64_t bd[2] = {smem_desc_k128_sw128(qg), smem_desc_k128_sw128(qg + NG * 128)};
#pragma unroll
                    for (int kk = 0; kk < kKlD / 16; ++kk)
                        umma_bf16(tmem + b * 256 + gg * NG, ad[kk >> 2] + 2 * (kk & 3), bd[kk >> 2] + 2 * (kk & 3),
                                  idesc, kk > 0 ? 1u : 0u);
                    umma_commit(&kempty[st]);
                }
                if (!ok) break;
                umma_commit(&afull[b]);
            }
        }
    } else if (warp >= 4) {
        // epilogue: warpgroup wg owns tokens wg*TPW .. wg*TPW + TPW - 1; lane row = key of the tile
        const int et = threadIdx.x - 128, wg = et >> 7, q4 = warp & 3;
        const int key = q4 * 32 + lane;
        const int tok0 = wg * TPW;  // first token of this warpgroup, within the block
        const uint32_t tbase = tmem + ((uint32_t)(q4 * 32) << 16);
        for (int i = et; i < TB * HQ; i += 512) {
            const int row = tb0 + i / HQ;
            l2s[i] = row < P.T ? P.lse2[(long long)row * HQ + i % HQ] : 0.f;
        }
        named_bar_sync(1, 512);
        float acc[TPW], mI[TPW], sI[TPW];
#pragma unroll
        for (int tt = 0; tt < TPW; ++tt) acc[tt] = 0.f, mI[tt] = -INFINITY, sI[tt] = 0.f;
        // TMEM columns of group gg for this warpgroup: gg*NG + tok0*G + c, c < CPG (token c / G,
        // head gg*G + c % G), loaded CH at a time
        constexpr int CH = CPG < 32 ? CPG : 32;
        bool ok = true;
        for (int kt = 0; kt < ntiles; ++kt) {
            const int b = kt & 1;
            ok = __all_sync(0xffffffffu, wait_parity_sleep(&afull[b], (kt >> 1) & 1, 0xB50, abort_flag));
            if (!ok) break;
            tc_fence_after();
            // this key's indexer scores for the warpgroup's tokens, loaded before the exponentials
            const long long s = (long long)kt * kKlKeys + key;
            float sc[TPW];
#pragma unroll
            for (int tt = 0; tt < TPW; ++tt) {
                const int row = tb0 + tok0 + tt;
                sc[tt] = (row < P.T && s <= P.q_pos0 + row) ? __ldg(P.scores + (long long)row * P.ld + s) : 0.f;
            }
            float pacc[TPW];
#pragma unroll
            for (int tt = 0; tt < TPW; ++tt) pacc[tt] = 0.f;
#pragma unroll
            for (int gg = 0; gg < HKV; ++gg) {
#pragma unroll
                for (int c0 = 0; c0 < CPG; c0 += CH) {
                    float z[CH];
                    const uint32_t ta = tbase + b * 256 + gg * NG + tok0 * G + c0;
                    if constexpr (CH == 32) tmem_ld_32x32b_x32(ta, *reinterpret_cast<float(*)[32]>(z));
                    else tmem_ld_32x32b_x16(ta, *reinterpret_cast<float(*)[16]>(z));
                    tmem_ld_wait();
                    if (gg == HKV - 1 && c0 + CH == CPG) {  // the last columns are in registers
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&aempty[b]);
                    }
#pragma unroll
                    for (int c = 0; c < CH; c += 2) {
                        // columns c, c+1: token (c0+c)/G, heads gg*G + (c0+c)%G and the next (G even)
                        const int tt = (c0 + c) / G, h = gg * G + (c0 + c) % G;
                        const float2 l = *reinterpret_cast<const float2*>(l2s + (tok0 + tt) * HQ + h);
                        pacc[tt] += ex2_approx(fmaf(z[c], P.scale_log2, -l.x)) +
                                    ex2_approx(fmaf(z[c + 1], P.scale_log2, -l.y));
                    }
                }
            }
#pragma unroll
            for (int tt = 0; tt < TPW; ++tt) {
                const int row = tb0 + tok0 + tt;
                if (row < P.T && s <= P.q_pos0 + row) {
                    const float p = pacc[tt] * (1.f / HQ);
                    if (p > 0.f) acc[tt] += p * (lg2_approx(p) * kLn2 - sc[tt]);
                    const float xs = sc[tt] * kLog2e;  // online log-sum-exp of the scores (log2 domain)
                    if (xs > mI[tt]) {
                        sI[tt] = sI[tt] * ex2_approx(mI[tt] - xs) + 1.f;
                        mI[tt] = xs;
                    } else {
                        sI[tt] += ex2_approx(xs - mI[tt]);
                    }
                }
            }
        }
        // reduce over the 128 keys: lanes by shuffles, then the 4 warps of the warpgroup
#pragma unroll
        for (int tt = 0; tt < TPW; ++tt) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                acc[tt] += __shfl_xor_sync(0xffffffffu, acc[tt], o);
                const float m2 = __shfl_xor_sync(0xffffffffu, mI[tt], o);
                const float s2 = __shfl_xor_sync(0xffffffffu, sI[tt], o);
                const float M = fmaxf(mI[tt], m2);
                sI[tt] = (mI[tt] == -INFINITY ? 0.f : sI[tt] * ex2_approx(mI[tt] - M)) +
                         (m2 == -INFINITY ? 0.f : s2 * ex2_approx(m2 - M));
                mI[tt] = M;
            }
            if (lane == 0) {
                float* rr = red + ((wg * 4 + q4) * 16 + tt) * 3;
                rr[0] = acc[tt];
                rr[1] = mI[tt];
                rr[2] = sI[tt];
            }
        }
        named_bar_sync(1, 512);
        if (ok && q4 == 0 && lane < TPW) {
            const int tt = lane, row = tb0 + tok0 + tt;
            float a = 0.f, M = -INFINITY;
            for (int w = 0; w < 4; ++w) M = fmaxf(M, red[((wg * 4 + w) * 16 + tt) * 3 + 1]);
            float S = 0.f;
            for (int w = 0; w < 4; ++w) {
                const float* rr = red + ((wg * 4 + w) * 16 + tt) * 3;
                a += rr[0];
                if (rr[1] != -INFINITY) S += rr[2] * ex2_approx(rr[1] - M);
            }
            if (row < P.T) P.kl[row] = a + (M + log2f(S)) * kLn2;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace dsa
