// Indexer warm-up target, forward only: for every query row t of a causal sequence
//   P_t(s) = (1/Hq) sum_h softmax_s(scale * q[t,h] . k[s,g(h)])     s = 0..t (dense attention)
//   Q_t(s) = softmax_s(score(t, s))                                  (the lightning indexer's scores)
//   KL_t   = sum_s P_t(s) * (log P_t(s) - log Q_t(s))
// (page "快手开源大模型Keye-VL-2.0：一个能“看懂“两小时视频AI", gsyq.cn, section 一: training stage 1
// fits the scout to the full attention distribution by minimising a KL divergence; the pages give
// no formula, this is the plainest reading of it).
//
// Unlike the sparse path this is dense: 2 x 2 x Hq x D flop per causal (t, s) pair over two passes,
// a tensor-core contraction.  One CTA takes 8 consecutive query tokens, warp w owning token w with
// all of its heads; the keys stream through a 3-stage shared-memory ring of 16-key tiles (all KV
// heads of a key are one contiguous Hkv*256-byte span, 16-byte cp.async, rows padded by 16 bytes
// for conflict-free ldmatrix), shared by the 8 tokens.  Per tile and KV group a warp computes
// S^T[16 keys x G heads] = K_g . Q_g^T on m16n8k16 bf16 MMAs (keys as M, the group's heads as N),
// so that a lane holds two keys x two heads and the sum over heads for P stays in registers until
// one two-step shuffle per tile.
//   pass 1: per head, the log-sum-exp of its logits over s <= t (lane-local online max/sum, then
//           a shuffle reduction); the log-sum-exp of the indexer row likewise;
//   pass 2: P_t(s) for the lane's two keys, then P (ln P - score + LSE_I) accumulated.
#pragma once

#include "ptx.cuh"

namespace dsa {

constexpr int kKlD = 128;
constexpr int kKlTokens = 8;    // query tokens per CTA (one warp each)
constexpr int kKlKeys = 16;     // keys per tile
constexpr int kKlStages = 3;
constexpr int kKlMaxHkv = 4;

struct KlParams {
    const __nv_bfloat16* q;   // [T, Hq, D]: this launch's query rows
    const __nv_bfloat16* k;   // [>= q_pos0 + T, Hkv, D]
    const float* scores;      // indexer scores of this launch's rows: row i at scores + i * ld, keys 0..q_pos0+i
    long long ld;
    int T;
    long long q_pos0;         // row i is query position q_pos0 + i
    int Hq, Hkv;
    float scale_log2;         // scale * log2(e)
    float* kl;                // [T]
};

__host__ __device__ constexpr int kl_row_bytes(int hkv) { return hkv * kKlD * 2 + 16; }
__host__ __device__ constexpr int kl_smem_bytes(int hkv) { return kKlStages * kKlKeys * kl_row_bytes(hkv); }

__global__ void __launch_bounds__(kKlTokens * 32, 2) indexer_kl_kernel(const KlParams P) {
    extern __shared__ __align__(1024) uint8_t smem[];
    constexpr float kLn2 = 0.69314718055994531f;
    constexpr float kLog2e = 1.4426950408889634f;
    const int Hkv = P.Hkv, G = P.Hq / P.Hkv;
    const int RB = kl_row_bytes(Hkv);
    const int STAGE = kKlKeys * RB;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // blocks in descending order of work: block 0 holds the last tokens
    const int nblk = (P.T + kKlTokens - 1) / kKlTokens;
    const int blk = nblk - 1 - (int)blockIdx.x;
    const int i0 = blk * kKlTokens;
    const int ntok = min(kKlTokens, P.T - i0);
    const int row = i0 + warp;                 // this warp's row in the launch
    const bool active = warp < ntok;
    const long long t = P.q_pos0 + row;        // its query position
    const long long t_last = P.q_pos0 + i0 + ntok - 1;
    const int ntiles = (int)(t_last / kKlKeys) + 1;
    const int my_tiles = active ? (int)(t / kKlKeys) + 1 : 0;

    // Q^T fragments per KV group (B operand: K = head dim, N = 8 heads): head lane/4, dims 2*(lane%4)+{0,1}(+8)
    uint32_t qf[kKlMaxHkv][8][2];
#pragma unroll
    for (int g = 0; g < kKlMaxHkv; ++g) {
        const int hl = lane >> 2;
        const bool hv = active && g < Hkv && hl < G;
        const __nv_bfloat16* qrow = P.q + ((long long)(active ? row : 0) * P.Hq + (hv ? g * G + hl : 0)) * kKlD;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const int d = kk * 16 + 2 * (lane & 3);
            qf[g][kk][0] = hv ? *reinterpret_cast<const uint32_t*>(qrow + d) : 0u;
            qf[g][kk][1] = hv ? *reinterpret_cast<const uint32_t*>(qrow + d + 8) : 0u;
        }
    }
    const float* srow = P.scores + (long long)(active ? row : 0) * P.ld;

    const int chunks_per_row = Hkv * kKlD * 2 / 16;
    auto load_tile = [&](int tile, int buf) {
        uint8_t* st = smem + buf * STAGE;
        for (int c = threadIdx.x; c < kKlKeys * chunks_per_row; c += blockDim.x) {
            const int key = c / chunks_per_row, ch = c % chunks_per_row;
            const long long s = (long long)tile * kKlKeys + key;
            const bool ok = s <= t_last;
            cp_async_16(st + key * RB + ch * 16, P.k + (ok ? s : 0) * (Hkv * kKlD) + ch * 8, ok);
        }
    };
    // S^T for the tile in stage buf and KV group g: sacc = keys lane/4 (c0, c1) and lane/4+8 (c2, c3),
    // heads 2*(lane%4) + {0, 1}
    auto logits = [&](const uint8_t* st, int g, float (&sacc)[4]) {
        float a2[4] = {0.f, 0.f, 0.f, 0.f};
        sacc[0] = sacc[1] = sacc[2] = sacc[3] = 0.f;
        const int mi = lane >> 3, ri = lane & 7;
        const uint8_t* arow = st + ((mi & 1) * 8 + ri) * RB + (g * kKlD + (mi >> 1) * 8) * 2;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            uint32_t a[4];
            ldmatrix_x4(a, arow + kk * 32);
            if (kk & 1) mma_16816(a2, a, qf[g][kk][0], qf[g][kk][1]);
            else mma_16816(sacc, a, qf[g][kk][0], qf[g][kk][1]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) sacc[i] += a2[i];
    };

    // the ring runs over all ntiles of the block twice: pass 1 (tiles 0..ntiles-1), pass 2 (again)
    const int total = 2 * ntiles;
#pragma unroll
    for (int s = 0; s < kKlStages - 1; ++s) {
        if (s < total) load_tile(s % ntiles, s);
        cp_async_commit();
    }
    // pass-1 state: per (group, head column j) lane-local max and sum (log2 domain), and the
    // indexer row's (natural-log domain, via exp2 of score * log2 e)
    float m1[kKlMaxHkv][2], l1[kKlMaxHkv][2];
#pragma unroll
    for (int g = 0; g < kKlMaxHkv; ++g) m1[g][0] = m1[g][1] = -INFINITY, l1[g][0] = l1[g][1] = 0.f;
    float mI = -INFINITY, lI = 0.f;
    float lse2[kKlMaxHkv][2];  // per head, log2 domain, after pass 1
    float lseI = 0.f;          // natural log
    float kl_acc = 0.f;
    const int key0 = lane >> 2;  // this lane's keys in a tile: key0 and key0 + 8
    const bool head_lane = (lane & 3) == 0;  // one lane of each key row accumulates the key's terms

    for (int it = 0; it < total; ++it) {
        cp_async_wait<kKlStages - 2>();
        __syncthreads();
        if (it + kKlStages - 1 < total) load_tile((it + kKlStages - 1) % ntiles, (it + kKlStages - 1) % kKlStages);
        cp_async_commit();
        const int tile = it % ntiles;
        const bool pass2 = it >= ntiles;
        if (pass2 && tile == 0 && active) {
            // end of pass 1: reduce the lane-local statistics over the 8 key rows of the warp
#pragma unroll
            for (int g = 0; g < kKlMaxHkv; ++g)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    float m = m1[g][j], l = l1[g][j];
#pragma unroll
                    for (int o = 4; o < 32; o <<= 1) {
                        const float m2 = __shfl_xor_sync(0xffffffffu, m, o), l2 = __shfl_xor_sync(0xffffffffu, l, o);
                        const float mn = fmaxf(m, m2);
                        l = (mn == -INFINITY) ? 0.f : l * exp2f(m - mn) + l2 * exp2f(m2 - mn);
                        m = mn;
                    }
                    lse2[g][j] = m + log2f(l);
                }
            float m = mI, l = lI;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float m2 = __shfl_xor_sync(0xffffffffu, m, o), l2 = __shfl_xor_sync(0xffffffffu, l, o);
                const float mn = fmaxf(m, m2);
                l = (mn == -INFINITY) ? 0.f : l * exp2f(m - mn) + l2 * exp2f(m2 - mn);
                m = mn;
            }
            lseI = (m + log2f(l)) * kLn2;
        }
        if (tile < my_tiles) {  // warp-uniform
            const uint8_t* st = smem + (it % kKlStages) * STAGE;
            const long long s0 = (long long)tile * kKlKeys + key0, s1 = s0 + 8;
            const bool v0 = s0 <= t, v1 = s1 <= t;
            const float I0 = v0 ? srow[s0] : 0.f, I1 = v1 ? srow[s1] : 0.f;
            if (!pass2) {
                if (head_lane) {  // the indexer row: each key once (lanes 0, 4, ..., 28 hold keys key0/key1)
                    const float z0 = v0 ? I0 * kLog2e : -INFINITY, z1 = v1 ? I1 * kLog2e : -INFINITY;
                    const float mn = fmaxf(mI, fmaxf(z0, z1));
                    if (mn != -INFINITY) {
                        lI = lI * exp2f(mI - mn) + exp2f(z0 - mn) + exp2f(z1 - mn);
                        mI = mn;
                    }
                }
#pragma unroll
                for (int g = 0; g < kKlMaxHkv; ++g) {
                    if (g >= Hkv) break;
                    float sacc[4];
                    logits(st, g, sacc);
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const float z0 = v0 ? sacc[j] * P.scale_log2 : -INFINITY;
                        const float z1 = v1 ? sacc[2 + j] * P.scale_log2 : -INFINITY;
                        const float mn = fmaxf(m1[g][j], fmaxf(z0, z1));
                        if (mn != -INFINITY) {
                            l1[g][j] = l1[g][j] * exp2f(m1[g][j] - mn) + exp2f(z0 - mn) + exp2f(z1 - mn);
                            m1[g][j] = mn;
                        }
                    }
                }
            } else {
                float p0 = 0.f, p1 = 0.f;  // sum over this lane's heads of the per-head probabilities
#pragma unroll
                for (int g = 0; g < kKlMaxHkv; ++g) {
                    if (g >= Hkv) break;
                    float sacc[4];
                    logits(st, g, sacc);
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int hl = 2 * (lane & 3) + j;
                        if (hl >= G) continue;
                        p0 += v0 ? exp2f(sacc[j] * P.scale_log2 - lse2[g][j]) : 0.f;
                        p1 += v1 ? exp2f(sacc[2 + j] * P.scale_log2 - lse2[g][j]) : 0.f;
                    }
                }
                // the other heads of the key row live in lanes lane^1, lane^2
                p0 += __shfl_xor_sync(0xffffffffu, p0, 1);
                p1 += __shfl_xor_sync(0xffffffffu, p1, 1);
                p0 += __shfl_xor_sync(0xffffffffu, p0, 2);
                p1 += __shfl_xor_sync(0xffffffffu, p1, 2);
                if (head_lane) {
                    const float inv_h = 1.f / (float)P.Hq;
                    const float P0 = p0 * inv_h, P1 = p1 * inv_h;
                    if (P0 > 0.f) kl_acc += P0 * (log2f(P0) * kLn2 - (I0 - lseI));
                    if (P1 > 0.f) kl_acc += P1 * (log2f(P1) * kLn2 - (I1 - lseI));
                }
            }
        }
    }
    cp_async_wait<0>();
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) kl_acc += __shfl_xor_sync(0xffffffffu, kl_acc, o);
    if (active && lane == 0) P.kl[row] = kl_acc;
}

}  // namespace dsa
