// Sparse scaled-dot-product attention over the selected keys, one index set per token shared by
// every GQA KV group:
//   out[t,h,:] = sum_{s in S_t} softmax_s(scale * q[t,h,:] . k[s,g,:]) v[s,g,:],  g = h / (Hq/Hkv)
// (page "从“看”到“想”多模态大模型推理能力的瓶颈与突破", wmrh.cn, section 2, step 3: standard
// scaled dot-product attention on the small selected candidate set; page "快手开源大模型
// Keye-VL-2.0：一个能“看懂“两小时视频AI", gsyq.cn, section 一: GQA adaptation of DSA).
//
// The work is a gather: per token, 2048 keys x Hkv x 128 x (K and V) x 2 bytes = 4 MiB at the
// 32/4/128 shape against 32 x 128 x 2048 x 4 flop, i.e. 8 flop per byte, far below the ridge
// of the tensor cores.  The kernel therefore spends its effort on the memory side:
//   - one CTA per (token, key split), two CTAs per SM for up to 8 heads per KV group; each
//     selected key's K and V rows for all KV heads are one contiguous Hkv*256-byte span, moved
//     with one bulk copy into a ring of 3 stages of 64/Hkv keys (rows padded by 16 bytes:
//     conflict-free ldmatrix).  The copies are issued by 3 producer warps, warp i owning ring
//     slot i: the rate at which one warp issues bulk copies, not the memory system, bounds a
//     single producer, so each SM runs six;
//   - an mbarrier per slot counts the bytes in, another the 4 consumer warps out.  Every waiter
//     waits for every phase of the barriers it uses (the consumers for every stage, producer i
//     for every refill of slot i): copies land out of order, and a parity wait that skipped a
//     phase could mistake an older completion for the one it wants;
//   - consumer warp w takes 16-key tile w % (4/Hkv) of every stage for KV group w / (4/Hkv) and
//     owns the group's G query heads (GQA head packing: the K/V tile it reads from shared
//     memory serves all G heads at once);
//   - S^T[keys x heads] = K . Q^T and O^T += V^T . P^T on warp-level bf16 MMAs
//     (m16n8k16, keys or head-dimension rows as M, 8 heads as N), so no MMA lane is wasted on
//     the small head count; P^T goes from the accumulator layout to the operand layout with
//     movmatrix; online softmax in fp32 (exp2 domain) against a reference maximum that moves only
//     when a logit exceeds it by more than 2^8 (one warp vote per tile instead of a shuffle
//     reduction; the probabilities stay below 2^8 and m + log2(l) is the same log-sum-exp);
//   - slots past the row's count and entries naming no key (index -1 or >= n_keys) copy a
//     zero row and get logit -inf.
// With nsplit > 1 every CTA writes unnormalised partial results (O, running max, running sum)
// for its slice of the index list; attn_combine_kernel merges them.
#pragma once

#include "ptx.cuh"

namespace dsa {

constexpr int kAttnD = 128;
constexpr int kAttnCW = 4;              // consumer warps, one 16-key tile of every stage each
constexpr int kAttnNS = 3;              // ring slots = producer warps
constexpr int kAttnThreads = (kAttnCW + kAttnNS) * 32;
constexpr int kAttnMaxKS = 64;          // keys per stage at Hkv = 1
constexpr int kAttnPartStride = kAttnD + 4;  // floats per split partial: O[128], m, l, 2 pad (16-byte rows)

// Rows of zeros that stand in for slots naming no key (Hkv * 256 bytes at most).
__device__ __align__(128) uint8_t g_attn_zero_row[4 * kAttnD * 2];

struct AttnParams {
    const __nv_bfloat16* q;   // [T, Hq, D]
    const __nv_bfloat16* k;   // [*, Hkv, D] per batch entry
    const __nv_bfloat16* v;
    long long kv_bstride;     // elements between batch entries of k/v (decode); 0 for prefill
    const int* idx;           // [T, topk]
    int topk;
    int T;                    // tokens in this launch
    long long q_pos0;         // prefill: token t sees min(topk, q_pos0 + t + 1) keys
    const int* ctx_len;       // decode: token t sees min(topk, ctx_len[t] + 1) keys, batch entry t
    long long n_keys;         // valid key rows per batch entry (bounds check on indices)
    int Hq, Hkv;
    float scale_log2;         // scale * log2(e)
    __nv_bfloat16* out;       // [T, Hq, D]
    float* lse;               // [T, Hq] natural-log LSE, may be null
    int nsplit;               // key splits per token
    float* part;              // nsplit > 1: [T, nsplit, Hq, kAttnPartStride]
    int* advance_ctx;         // decode with nsplit == 1, may be null: ctx_len[t] += 1 once token t is done
    long long window;         // > 0 (prefill): a row holds at most min(topk, window) keys
};

__host__ __device__ constexpr int attn_stage_keys(int hkv) { return 16 * (kAttnCW / hkv); }
__host__ __device__ constexpr int attn_row_bytes(int hkv) { return hkv * kAttnD * 2 + 16; }
__host__ __device__ constexpr int attn_stage_bytes(int hkv) { return attn_stage_keys(hkv) * attn_row_bytes(hkv) * 2; }
// per consumer warp after the loop: [NT][36][32] floats (O fragments, m, l) for the merge
__host__ __device__ constexpr int attn_xch_bytes(int nt) { return kAttnCW * nt * 36 * 32 * 4; }
__host__ __device__ constexpr int attn_ring_bytes(int hkv, int nt) {
    return kAttnNS * attn_stage_bytes(hkv) > attn_xch_bytes(nt) ? kAttnNS * attn_stage_bytes(hkv) : attn_xch_bytes(nt);
}
// ring (or merge area) | full[NS], empty[NS] mbarriers | abort flag | valid flags [NS][64]
__host__ __device__ constexpr int attn_smem_bytes(int hkv, int nt) {
    return attn_ring_bytes(hkv, nt) + kAttnNS * 16 + 16 + kAttnNS * kAttnMaxKS;
}

// NT: n-tiles of 8 query heads per KV group (G <= 8 * NT).
template <int NT>
__global__ void __launch_bounds__(kAttnThreads, NT == 1 ? 2 : 1) sparse_attn_kernel(const AttnParams P) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int Hkv = P.Hkv, G = P.Hq / P.Hkv;
    const int WPG = kAttnCW / Hkv;                  // consumer warps per KV group
    const int KS = attn_stage_keys(Hkv);            // keys per stage
    const int RB = attn_row_bytes(Hkv);             // padded row bytes (K or V of one key)
    const int STAGE = attn_stage_bytes(Hkv);        // K rows then V rows
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int grp = warp / WPG, wsub = warp % WPG;  // consumer warps only

    uint64_t* full = reinterpret_cast<uint64_t*>(smem + attn_ring_bytes(Hkv, NT));
    uint64_t* empty = full + kAttnNS;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kAttnNS);
    uint8_t* svalid = reinterpret_cast<uint8_t*>(empty + kAttnNS) + 16;

    const int t = blockIdx.x / P.nsplit;
    const int split = blockIdx.x % P.nsplit;
    long long n_ll;
    const __nv_bfloat16 *kb = P.k, *vb = P.v;
    if (P.ctx_len) {
        n_ll = (long long)P.ctx_len[t] + 1;
        n_ll = n_ll < 1 ? 1 : (n_ll > P.n_keys ? P.n_keys : n_ll);
        kb += (long long)t * P.kv_bstride;
        vb += (long long)t * P.kv_bstride;
    } else {
        n_ll = P.q_pos0 + t + 1;
        if (P.window > 0 && n_ll > P.window) n_ll = P.window;
    }
    const int n_sel = (int)min((long long)P.topk, n_ll);
    const int per_split = (n_sel + P.nsplit - 1) / P.nsplit;
    const int p_begin = split * per_split;
    const int p_end = min(n_sel, p_begin + per_split);
    const int* idx_row = P.idx + (long long)t * P.topk;
    const int nsteps = p_end > p_begin ? (p_end - p_begin + KS - 1) / KS : 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kAttnNS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kAttnCW);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    float o[NT][8][4];  // O^T: [d-tile][4] per n-tile; rows = head dims, cols = heads
    float m_run[NT][2], l_run[NT][2];  // per owned head (cols 2*(lane%4)+{0,1})
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int dt = 0; dt < 8; ++dt)
#pragma unroll
            for (int i = 0; i < 4; ++i) o[nt][dt][i] = 0.f;
        m_run[nt][0] = m_run[nt][1] = -INFINITY, l_run[nt][0] = l_run[nt][1] = 0.f;
    }

    if (warp >= kAttnCW) {
        // ------------------------------------------------------------ producer warp: ring slot `slot`
        // Copy c of a stage (c < 2*KS: K rows, then V rows) goes to lane c % 32; the stage's
        // indices are loaded one refill ahead.
        const int slot = warp - kAttnCW;
        const int rowb = Hkv * kAttnD * 2;
        const int ncp = (2 * KS) / 32;  // copies per lane: 1, 2 or 4
        auto ld_idx = [&](int step, int i) {
            const int key = (lane + 32 * i) % KS;
            const int p = p_begin + step * KS + key;
            return (step < nsteps && p < p_end) ? __ldg(idx_row + p) : -1;
        };
        int pre[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) pre[i] = i < ncp ? ld_idx(slot, i) : -1;
        int fills = 0;
        bool ok = true;
        for (int step = slot; step < nsteps; step += kAttnNS, ++fills) {
            // every lane waits (and so acquires); the warp leaves together if any lane gave up
            ok = __all_sync(0xffffffffu, wait_parity(&empty[slot], (fills & 1) ^ 1, 0x401, abort_flag));
            if (!ok) break;
            int cur[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                cur[i] = pre[i];
                pre[i] = i < ncp ? ld_idx(step + kAttnNS, i) : -1;
            }
            bool kv_ok[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int c = lane + 32 * i, key = c % KS;
                kv_ok[i] = i < ncp && p_begin + step * KS + key < p_end && cur[i] >= 0 && cur[i] < P.n_keys;
                if (i < ncp && c < KS) svalid[slot * kAttnMaxKS + key] = kv_ok[i] ? 1 : 0;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive_expect_tx(&full[slot], 2 * KS * rowb);
            __syncwarp();
            uint8_t* st = smem + slot * STAGE;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (i >= ncp) break;
                const int c = lane + 32 * i, key = c % KS;
                const bool is_v = c >= KS;
                const __nv_bfloat16* src = (is_v ? vb : kb) + (long long)(kv_ok[i] ? cur[i] : 0) * (Hkv * kAttnD);
                bulk_load(st + (is_v ? KS * RB : 0) + key * RB,
                          kv_ok[i] ? static_cast<const void*>(src) : static_cast<const void*>(g_attn_zero_row), rowb,
                          &full[slot]);
            }
        }
        if (!ok && fills > 0) {
            // let this slot's last copies land before the CTA leaves (bounded wait)
            wait_parity(&full[slot], (fills - 1) & 1, 0x402, nullptr);
        }
    } else {
        // ------------------------------------------------------------ consumer warps
        // ---- Q^T fragments (B operand, K = head dim, N = 8 heads): head lane/4, dims 2*(lane%4)+{0,1}(+8)
        uint32_t qf[NT][8][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int hl = nt * 8 + (lane >> 2);
            const bool hv = hl < G;
            const __nv_bfloat16* qrow = P.q + ((long long)t * P.Hq + grp * G + (hv ? hl : 0)) * kAttnD;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int d = kk * 16 + 2 * (lane & 3);
                qf[nt][kk][0] = hv ? *reinterpret_cast<const uint32_t*>(qrow + d) : 0u;
                qf[nt][kk][1] = hv ? *reinterpret_cast<const uint32_t*>(qrow + d + 8) : 0u;
            }
        }

        for (int step = 0; step < nsteps; ++step) {
            const int buf = step % kAttnNS;
            if (!__all_sync(0xffffffffu, wait_parity(&full[buf], (step / kAttnNS) & 1, 0x403, abort_flag))) break;
            const uint8_t* sk = smem + buf * STAGE + wsub * 16 * RB;  // this warp's 16-key tile
            const uint8_t* sv = sk + KS * RB;
            // S^T = K Q^T : 16 keys x 8 heads per n-tile, two independent accumulation chains
            float sacc[NT][4], sacc2[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) sacc[nt][i] = sacc2[nt][i] = 0.f;
            {
                const int mi = lane >> 3, ri = lane & 7;
                const uint8_t* arow = sk + ((mi & 1) * 8 + ri) * RB + (grp * kAttnD + (mi >> 1) * 8) * 2;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    uint32_t a[4];
                    ldmatrix_x4(a, arow + kk * 32);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        if (kk & 1) mma_16816(sacc2[nt], a, qf[nt][kk][0], qf[nt][kk][1]);
                        else mma_16816(sacc[nt], a, qf[nt][kk][0], qf[nt][kk][1]);
                    }
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) sacc[nt][i] += sacc2[nt][i];
            }
            // masked: slots past this CTA's range and entries that name no key (e.g. -1 padding);
            // rows: key lane/4 (c0,c1) and lane/4+8 (c2,c3)
            const uint8_t* vflag = svalid + buf * kAttnMaxKS + wsub * 16;
            const bool v0 = vflag[lane >> 2] != 0;
            const bool v1 = vflag[(lane >> 2) + 8] != 0;
            uint32_t pb[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                float z[4];
                z[0] = v0 ? sacc[nt][0] * P.scale_log2 : -INFINITY;
                z[1] = v0 ? sacc[nt][1] * P.scale_log2 : -INFINITY;
                z[2] = v1 ? sacc[nt][2] * P.scale_log2 : -INFINITY;
                z[3] = v1 ? sacc[nt][3] * P.scale_log2 : -INFINITY;
                float mx[2] = {fmaxf(z[0], z[2]), fmaxf(z[1], z[3])};
                float alpha[2] = {1.f, 1.f};
                // the reference maximum moves only when a logit exceeds it by more than 2^8
                if (__any_sync(0xffffffffu, mx[0] > m_run[nt][0] + 8.f || mx[1] > m_run[nt][1] + 8.f)) {
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], 4));
                        mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], 8));
                        mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], 16));
                        if (mx[j] > m_run[nt][j] + 8.f) {
                            alpha[j] = m_run[nt][j] == -INFINITY ? 0.f : ex2_approx(m_run[nt][j] - mx[j]);
                            m_run[nt][j] = mx[j];
                        }
                    }
                }
                const float base[2] = {m_run[nt][0] == -INFINITY ? 0.f : m_run[nt][0],
                                       m_run[nt][1] == -INFINITY ? 0.f : m_run[nt][1]};
                const float p0 = ex2_approx(z[0] - base[0]), p1 = ex2_approx(z[1] - base[1]);
                const float p2 = ex2_approx(z[2] - base[0]), p3 = ex2_approx(z[3] - base[1]);
                l_run[nt][0] = l_run[nt][0] * alpha[0] + p0 + p2;
                l_run[nt][1] = l_run[nt][1] * alpha[1] + p1 + p3;
                // rescale only when some reference maximum moved (alpha == 1 leaves O unchanged)
                if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
                    for (int dt = 0; dt < 8; ++dt) {
                        o[nt][dt][0] *= alpha[0];
                        o[nt][dt][1] *= alpha[1];
                        o[nt][dt][2] *= alpha[0];
                        o[nt][dt][3] *= alpha[1];
                    }
                }
                // P^T (keys x heads) -> B operand layout (keys as K, heads as N)
                pb[nt][0] = movmatrix_trans(pack_bf16x2(p0, p1));
                pb[nt][1] = movmatrix_trans(pack_bf16x2(p2, p3));
            }
            // O^T += V^T P^T : A = V^T (16 dims x 16 keys) via transposing ldmatrix
            {
                const int mi = lane >> 3, ri = lane & 7;
                const uint8_t* vrow = sv + ((mi >> 1) * 8 + ri) * RB + (grp * kAttnD + (mi & 1) * 8) * 2;
#pragma unroll
                for (int dt = 0; dt < 8; ++dt) {
                    uint32_t a[4];
                    ldmatrix_x4_trans(a, vrow + dt * 32);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_16816(o[nt][dt], a, pb[nt][0], pb[nt][1]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[buf]);
        }
    }

    // ---- finish: full row sums, merge the WPG consumer warps of a group through shared memory
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            float l = l_run[nt][j];
            l += __shfl_xor_sync(0xffffffffu, l, 4);
            l += __shfl_xor_sync(0xffffffffu, l, 8);
            l += __shfl_xor_sync(0xffffffffu, l, 16);
            l_run[nt][j] = l;
        }
    __syncthreads();  // every issued copy was consumed (or waited for): the ring is free now
    // per warp: [NT][8][4] O values per lane + m, l per owned head
    float* xch = reinterpret_cast<float*>(smem) + (size_t)warp * (NT * 36 * 32);
    if (warp < kAttnCW && wsub != 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int dt = 0; dt < 8; ++dt)
#pragma unroll
                for (int i = 0; i < 4; ++i) xch[((nt * 36) + dt * 4 + i) * 32 + lane] = o[nt][dt][i];
            xch[(nt * 36 + 32) * 32 + lane] = m_run[nt][0];
            xch[(nt * 36 + 33) * 32 + lane] = m_run[nt][1];
            xch[(nt * 36 + 34) * 32 + lane] = l_run[nt][0];
            xch[(nt * 36 + 35) * 32 + lane] = l_run[nt][1];
        }
    }
    __syncthreads();
    if (warp < kAttnCW && wsub == 0) {
#pragma unroll 1
        for (int w2 = 1; w2 < WPG; ++w2) {
            const float* x2 = reinterpret_cast<const float*>(smem) + (size_t)(warp + w2) * (NT * 36 * 32);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                float a1[2], a2[2];
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const float m2 = x2[(nt * 36 + 32 + j) * 32 + lane];
                    const float l2 = x2[(nt * 36 + 34 + j) * 32 + lane];
                    const float mn = fmaxf(m_run[nt][j], m2);
                    const float bs = mn == -INFINITY ? 0.f : mn;
                    a1[j] = exp2f(m_run[nt][j] - bs);
                    a2[j] = exp2f(m2 - bs);
                    l_run[nt][j] = l_run[nt][j] * a1[j] + l2 * a2[j];
                    m_run[nt][j] = mn;
                }
#pragma unroll
                for (int dt = 0; dt < 8; ++dt)
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        o[nt][dt][i] = o[nt][dt][i] * a1[i & 1] + x2[((nt * 36) + dt * 4 + i) * 32 + lane] * a2[i & 1];
            }
        }
        // write: fragment (dims dt*16 + lane/4 (+8), heads nt*8 + 2*(lane%4) + {0,1})
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int hl = nt * 8 + 2 * (lane & 3) + j;
                if (hl >= G) continue;
                const int h = grp * G + hl;
                if (P.nsplit == 1) {
                    const float inv = l_run[nt][j] > 0.f ? 1.f / l_run[nt][j] : 0.f;
                    __nv_bfloat16* orow = P.out + ((long long)t * P.Hq + h) * kAttnD;
#pragma unroll
                    for (int dt = 0; dt < 8; ++dt) {
                        orow[dt * 16 + (lane >> 2)] = __float2bfloat16_rn(o[nt][dt][j] * inv);
                        orow[dt * 16 + (lane >> 2) + 8] = __float2bfloat16_rn(o[nt][dt][2 + j] * inv);
                    }
                    if (P.lse && (lane >> 2) == 0)
                        P.lse[(long long)t * P.Hq + h] =
                            l_run[nt][j] > 0.f ? (m_run[nt][j] + log2f(l_run[nt][j])) * 0.69314718055994531f : -INFINITY;
                } else {
                    float* prow = P.part + (((long long)t * P.nsplit + split) * P.Hq + h) * kAttnPartStride;
#pragma unroll
                    for (int dt = 0; dt < 8; ++dt) {
                        prow[dt * 16 + (lane >> 2)] = o[nt][dt][j];
                        prow[dt * 16 + (lane >> 2) + 8] = o[nt][dt][2 + j];
                    }
                    if ((lane >> 2) == 0) {
                        prow[kAttnD] = m_run[nt][j];
                        prow[kAttnD + 1] = l_run[nt][j];
                    }
                }
            }
        }
    }
    // decode with one CTA per token: advance its context length here (every thread read
    // ctx_len[t] before the first barrier of the kernel); with splits the merge kernel does it
    if (P.nsplit == 1 && P.advance_ctx && threadIdx.x == 0 && P.advance_ctx[t] >= 0 && P.advance_ctx[t] < P.n_keys)
        P.advance_ctx[t] += 1;
}

// Merge split partials: one warp per (token, head).  Lane s < nsplit holds split s's running
// max and sum; every lane then accumulates its 4 output dims over all splits with independent
// 16-byte loads.  With advance_ctx (decode), block 0 also moves every sequence's context length
// one position on (nothing later in the step reads it).
__global__ void __launch_bounds__(128) attn_combine_kernel(const float* part, int T, int nsplit, int Hq,
                                                           __nv_bfloat16* out, float* lse, int* advance_ctx,
                                                           long long Lmax) {
    constexpr int kMaxSplits = 32;
    const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (advance_ctx && blockIdx.x == 0)
        for (int b = threadIdx.x; b < T; b += blockDim.x)
            if (advance_ctx[b] >= 0 && advance_ctx[b] < Lmax) advance_ctx[b] += 1;
    if (wid >= T * Hq || nsplit > kMaxSplits) return;
    const int t = wid / Hq, h = wid % Hq;
    const long long sstride = (long long)Hq * kAttnPartStride;
    const float* base = part + ((long long)t * nsplit * Hq + h) * kAttnPartStride;
    float m_s = -INFINITY, l_s = 0.f;
    if (lane < nsplit) {
        const float2 ml = *reinterpret_cast<const float2*>(base + lane * sstride + kAttnD);
        m_s = ml.x;
        l_s = ml.y;
    }
    float mx = m_s;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float bs = mx == -INFINITY ? 0.f : mx;
    const float a_s = lane < nsplit ? exp2f(m_s - bs) : 0.f;
    float l = l_s * a_s;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int s = 0; s < kMaxSplits; ++s) {
        const float w = __shfl_sync(0xffffffffu, a_s, s);
        if (s < nsplit) {
            const float4 v = *reinterpret_cast<const float4*>(base + s * sstride + lane * 4);
            acc.x += v.x * w;
            acc.y += v.y * w;
            acc.z += v.z * w;
            acc.w += v.w * w;
        }
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    __nv_bfloat162* orow = reinterpret_cast<__nv_bfloat162*>(out + ((long long)t * Hq + h) * kAttnD + lane * 4);
    orow[0] = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    orow[1] = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    if (lse && lane == 0) lse[(long long)t * Hq + h] = l > 0.f ? (mx + log2f(l)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace dsa
