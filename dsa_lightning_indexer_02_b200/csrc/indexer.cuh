// Lightning-indexer scores on the 5th-generation tensor cores.
//
//   score(t, s) = sum_h w[t,h] * max(0, qI[t,h,:] . kI[s,:])      for keys s <= t
//
// The pages describe a light "scout" with one MQA-shared key per position that scores every
// position for the current token (page "快手开源大模型Keye-VL-2.0：一个能“看懂“两小时视频AI",
// gsyq.cn, section 一); the formula above is the one this library adopts (the pages give none).
//
// Tiling.  One MMA tile is D[128 keys, BN columns] = kI_tile[128 x 64] . Qtile[BN x 64]^T where
// the BN columns are (token, head) pairs of TB = BN/HI consecutive query tokens.  The key tile
// is the M operand, so every TMEM lane holds one key and the head sum for a token is a plain
// in-thread reduction over that token's HI columns; the token weights stay in registers for the
// whole work unit and consecutive lanes write consecutive keys (coalesced 128-byte score stores).
//
// Roles (one CTA per SM, persistent):
//   warp 0        TMA producer: the unit's Q tile (once per unit) and a ring of kI tiles
//   warp 1        TMEM allocator + single-thread tcgen05.mma issuer
//   warps 2-3     idle (they complete the role warpgroup)
//   warps 4..     epilogue: tcgen05.ld, ReLU, weight FMA, head sum, score store;
//                 NWG warpgroups split the BN columns between them and keep the unit's weights
//                 for their columns in registers
// Two TMEM accumulators (2 x BN fp32 columns) let the MMA of tile j+1 overlap the epilogue of
// tile j.  Work units are (problem p, query block qb, key-tile range); prefill uses one problem
// and whole causal key ranges, decode uses one problem per sequence and splits its keys.
#pragma once

#include "ptx.cuh"

namespace dsa {

constexpr int kIdxBM = 128;  // keys per tile
constexpr int kIdxBK = 64;   // = d_I, one 128-byte swizzled row per key / per (token, head)

struct IndexerParams {
    int P;                      // problems: 1 (prefill) or B sequences (decode)
    int Lq;                     // query rows per problem
    long long q_pos0;           // prefill: absolute position of query row 0
    const int* ctx_len;         // decode: query position of problem p is ctx_len[p]; else null
    long long Lk;               // keys addressable per problem (TMA extent)
    const __nv_bfloat16* w;     // [P, Lq, HI]
    float* scores;              // row (p*Lq + i) at scores + row*ld
    long long ld;
    int num_qb;                 // query blocks per problem
    int nsplit;                 // key-range splits per (p, qb)
    int kt_per_split;           // key tiles per split (nsplit > 1)
    int num_units;              // P * num_qb * nsplit
    uint32_t q_box_bytes;       // bytes one Q TMA box brings
    uint32_t k_box_bytes;       // bytes one kI TMA box brings
    long long window;           // > 0 (prefill): keys s <= t - window are not needed (not scored)
    // decode: the new token of sequence p goes to row ctx_len[p] of the caches before any load of
    // that key tile (the CTA that owns the tile writes it); null when nothing is appended
    const uint4* new_k;         // [P, kv16] 16-byte units
    const uint4* new_v;
    const uint4* new_kI;        // [P, kI16]
    uint4* cache_k;             // [P, Lk, kv16]
    uint4* cache_v;
    uint4* cache_kI;            // [P, Lk, kI16]
    int kv16, kI16;
};

struct IndexerUnit {
    int p, qb, kt0, kt1;        // key tiles [kt0, kt1)
    long long tq0;              // absolute position of the block's first query row
    int rows;                   // valid query rows in the block
};

template <int TB>
__device__ __forceinline__ IndexerUnit indexer_unit(const IndexerParams& P, int u) {
    IndexerUnit r;
    const int per_p = P.num_qb * P.nsplit;
    r.p = u / per_p;
    const int rem = u - r.p * per_p;
    // prefill: the last query blocks carry the most keys, start with them
    r.qb = P.num_qb - 1 - rem / P.nsplit;
    const int split = rem % P.nsplit;
    long long base = P.q_pos0;
    if (P.ctx_len) {  // decode: clamp a bad context length to the cache (the append kernel reports it)
        base = P.ctx_len[r.p];
        base = base < 0 ? 0 : (base >= P.Lk ? P.Lk - 1 : base);
    }
    r.tq0 = base + (long long)r.qb * TB;
    const int first = r.qb * TB;
    r.rows = min(TB, P.Lq - first);
    const long long t_last = r.tq0 + r.rows - 1;
    const int nkt = (int)(t_last / kIdxBM) + 1;
    if (P.nsplit == 1) {
        // sliding window: the block's first token needs keys from tq0 - window + 1 on
        r.kt0 = P.window > 0 ? (int)(max(0LL, r.tq0 - P.window + 1) / kIdxBM) : 0;
        r.kt1 = nkt;
    } else {
        r.kt0 = split * P.kt_per_split;
        r.kt1 = min(nkt, r.kt0 + P.kt_per_split);
    }
    return r;
}

// Snake order over CTAs so that long and short units mix evenly.
__device__ __forceinline__ int indexer_unit_of(int round, int cta, int grid) {
    return round * grid + ((round & 1) ? (grid - 1 - cta) : cta);
}

// Decode (one query token per unit): a CTA's few work units, each with its sequence's context
// length and the token's head weights (up to 64 bf16), read into shared memory once -- one
// parallel round of global loads at the start instead of a dependent load (ctx_len, then the
// weights) in every role at every unit boundary.
constexpr int kIdxUnitTab = 8;  // rounds per CTA the table holds; more fall back to direct loads
struct IndexerUnitEntry {
    IndexerUnit U;
    long long pos;  // ctx_len[U.p] as given (the append's row; checked before use)
    int valid, pad;
    uint4 w[8];     // the unit's token weights, raw bf16
};

template <int CHUNK>
__device__ __forceinline__ void tmem_ld_chunk(uint32_t taddr, float (&v)[CHUNK]) {
    if constexpr (CHUNK == 32) tmem_ld_32x32b_x32(taddr, v);
    else if constexpr (CHUNK == 16) tmem_ld_32x32b_x16(taddr, v);
    else tmem_ld_32x32b_x8(taddr, v);
}

// c + a * b on packed fp32 pairs (one fma.rn.f32x2).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    uint64_t pa, pb, pc, pd;
    asm("mov.b64 %0, {%1, %2};" : "=l"(pa) : "f"(a.x), "f"(a.y));
    asm("mov.b64 %0, {%1, %2};" : "=l"(pb) : "f"(b.x), "f"(b.y));
    asm("mov.b64 %0, {%1, %2};" : "=l"(pc) : "f"(c.x), "f"(c.y));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(pd) : "l"(pa), "l"(pb), "l"(pc));
    float2 d;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(pd));
    return d;
}

// ReLU is split across two pipes.  Heads h with (h & 6) == 0 (a quarter of them) take max(x, 0)
// on the integer/ALU pipe; the others take x + |x| = 2 max(x, 0) on the floating-point pipe, one
// packed add per pair, and their weights are stored halved (exact: a power-of-two scale), so
// w * max(x, 0) is reproduced to the bit for every finite x.  Per element that is half an issue
// slot on the FP path against one on the ALU path; a quarter on the ALU path measured best (944
// TFLOP/s over a 128K sequence, against 913 with half and 938 with none).
__device__ __forceinline__ float2 relu_pair_alu(float a, float b) { return make_float2(fmaxf(a, 0.f), fmaxf(b, 0.f)); }
// x + |x| for a pair as one packed add (the absolute value rides on the operand; the same
// per-element rounding as two scalar adds, half the instructions).
__device__ __forceinline__ float2 relu2_pair_fma(float a, float b) {
    uint64_t px, pa, pd;
    asm("mov.b64 %0, {%1, %2};" : "=l"(px) : "f"(a), "f"(b));
    asm("mov.b64 %0, {%1, %2};" : "=l"(pa) : "f"(fabsf(a)), "f"(fabsf(b)));
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(pd) : "l"(px), "l"(pa));
    float2 d;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(pd));
    return d;
}
// Scale that the stored weight of head h carries (see above); heads come in groups of four only
// when the head count is a multiple of four.
template <int HI>
__device__ __forceinline__ float weight_store_scale(int h) { return (HI % 4 == 0 && (h & 6)) ? 0.5f : 1.f; }

// sum_h w[h] * max(v[h], 0) over N >= 1 heads, with independent partial sums (no long
// dependent FMA chain) on packed fp32 pairs.
template <int N>
__device__ __forceinline__ float head_sum(const float* v, const float* w) {
    if constexpr (N == 1) {
        return w[0] * fmaxf(v[0], 0.f);
    } else {
        constexpr int NP = N / 2;                 // pairs
        constexpr int NA = NP < 4 ? NP : 4;       // independent accumulators
        float2 acc[NA];
#pragma unroll
        for (int i = 0; i < NA; ++i) acc[i] = make_float2(0.f, 0.f);
        if constexpr (N % 4 == 0) {
#pragma unroll
            for (int q = 0; q < N / 4; ++q) {
                const float2 x0 = (q & 1) ? relu2_pair_fma(v[4 * q], v[4 * q + 1]) : relu_pair_alu(v[4 * q], v[4 * q + 1]);
                const float2 x1 = relu2_pair_fma(v[4 * q + 2], v[4 * q + 3]);
                acc[(2 * q) % NA] = ffma2(x0, make_float2(w[4 * q], w[4 * q + 1]), acc[(2 * q) % NA]);
                acc[(2 * q + 1) % NA] = ffma2(x1, make_float2(w[4 * q + 2], w[4 * q + 3]), acc[(2 * q + 1) % NA]);
            }
        } else {
#pragma unroll
            for (int p = 0; p < NP; ++p) {
                const float2 x = make_float2(fmaxf(v[2 * p], 0.f), fmaxf(v[2 * p + 1], 0.f));
                acc[p % NA] = ffma2(x, make_float2(w[2 * p], w[2 * p + 1]), acc[p % NA]);
            }
        }
        float r = 0.f;
#pragma unroll
        for (int i = 0; i < NA; ++i) r += acc[i].x + acc[i].y;
        return r;
    }
}

// carry[0..1] += packed partial sums of w[h] * max(v[h], 0) over one chunk of N heads.  `w` points
// into a register array (every index is a compile-time constant after unrolling).
template <int N>
__device__ __forceinline__ void head_sum_acc(const float* v, const float* w, float2 (&carry)[2]) {
#pragma unroll
    for (int q = 0; q < N / 4; ++q) {
        const float2 x0 = (q & 1) ? relu2_pair_fma(v[4 * q], v[4 * q + 1]) : relu_pair_alu(v[4 * q], v[4 * q + 1]);
        const float2 x1 = relu2_pair_fma(v[4 * q + 2], v[4 * q + 3]);
        carry[0] = ffma2(x0, make_float2(w[4 * q], w[4 * q + 1]), carry[0]);
        carry[1] = ffma2(x1, make_float2(w[4 * q + 2], w[4 * q + 3]), carry[1]);
    }
}

template <int HI, int BN, int STAGES>
struct IndexerCfg {
    static constexpr int TB = BN / HI;
    // epilogue warpgroups: each owns BN/NWG columns (whole tokens); more warps hide the latency
    // of the per-token reduction chains
    static constexpr int NWG = (BN >= 256 && BN / 4 >= HI) ? 4 : (BN >= 128 && BN / 2 >= HI) ? 2 : 1;
    static constexpr int COLS_WG = BN / NWG;
    // TMEM loads of 16 columns, one at a time (the other warps of the SM hide their latency): the
    // warpgroup's COLS_WG weights live in registers for a whole work unit, so the loads stay small.
    // Measured 3 % faster than double-buffered 8-column loads (half the load and wait instructions).
    // A single epilogue warpgroup (decode: one token per tile) has no other epilogue warps to hide
    // the load latency behind, so it reads 32 columns per load: one load-and-wait round trip per
    // tile for 32 heads, and the accumulator goes back to the MMA one round trip earlier.
    static constexpr int CHUNK = (NWG == 1 && COLS_WG % 32 == 0) ? 32 : 16;
    static constexpr int NCHUNK = COLS_WG / CHUNK;
    // warpgroup 0 holds the roles (warp 0 TMA, warp 1 MMA, warps 2-3 idle); warpgroups 1..NWG the
    // epilogue.  With four epilogue warpgroups the roles hand registers to the epilogue
    // (setmaxnreg): launched at 96 per thread (20 warps, 5 per SM sub-partition), the role
    // warpgroup drops to 32 and the epilogue rises to 112 -- 4*32*32 + 16*32*112 = 640*96, and
    // per sub-partition 32*(32 + 4*112) <= 16384 -- which keeps a unit's 64 weights in registers.
    static constexpr int THREADS = 128 + NWG * 128;
    static constexpr bool REGSPLIT = NWG == 4;
    static constexpr int ROLE_REGS = 32, EPI_REGS = 112;
    static constexpr int A_BYTES = kIdxBM * kIdxBK * 2;  // 16 KB
    static constexpr int B_BYTES = BN * kIdxBK * 2;
    static constexpr int TMEM_COLS = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128 : (2 * BN <= 256) ? 256 : 512;
    // shared memory layout (offsets from a 1024-aligned base)
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
    static constexpr int OFF_BAR = OFF_B + 2 * B_BYTES;
    static constexpr int NBAR = 2 * STAGES + 8;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr bool UNIT_TAB = TB == 1;  // decode: the unit table in shared memory
    static constexpr int OFF_UT = (OFF_MISC + 16 + 15) / 16 * 16;
    static constexpr int SMEM = OFF_UT + (UNIT_TAB ? kIdxUnitTab * (int)sizeof(IndexerUnitEntry) : 0) + 1024;  // + alignment slack
    static_assert(BN % HI == 0 && BN >= 16 && BN <= 256 && BN % 16 == 0, "bad BN");
    static_assert(HI <= COLS_WG, "a token's heads must stay inside one warpgroup");
    static_assert(HI <= CHUNK || HI % CHUNK == 0, "bad HI");
    static_assert(COLS_WG % 8 == 0 && COLS_WG <= 64, "weights: whole 16-byte groups, at most 64 registers");
};

template <int HI, int BN, int STAGES>
__global__ void __launch_bounds__(IndexerCfg<HI, BN, STAGES>::THREADS, 1) indexer_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                   const IndexerParams P) {
    using C = IndexerCfg<HI, BN, STAGES>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem + C::OFF_A;
    uint8_t* sB = smem + C::OFF_B;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* a_full = bars;
    uint64_t* a_empty = bars + STAGES;
    uint64_t* q_full = bars + 2 * STAGES;
    uint64_t* q_empty = q_full + 2;
    uint64_t* acc_full = q_full + 4;
    uint64_t* acc_empty = q_full + 6;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    IndexerUnitEntry* utab = reinterpret_cast<IndexerUnitEntry*>(smem + C::OFF_UT);
    // uniform: the decode table covers every round of this CTA
    const bool use_tab = C::UNIT_TAB && P.ctx_len && (P.num_units + (int)gridDim.x - 1) / (int)gridDim.x <= kIdxUnitTab;
    if (use_tab) {
        if (threadIdx.x < kIdxUnitTab) {
            const int rd = threadIdx.x;
            const int u = indexer_unit_of(rd, blockIdx.x, gridDim.x);
            IndexerUnitEntry& E = utab[rd];
            E.valid = u < P.num_units;
            if (E.valid) {
                E.U = indexer_unit<C::TB>(P, u);
                E.pos = P.ctx_len[E.U.p];
                const uint4* wsrc = reinterpret_cast<const uint4*>(P.w + (long long)E.U.p * P.Lq * HI);
#pragma unroll
                for (int i = 0; i < HI / 8; ++i) E.w[i] = __ldg(wsrc + i);
            }
        }
        __syncthreads();
    }
    auto unit_at = [&](int rd, int u) { return use_tab ? utab[rd].U : indexer_unit<C::TB>(P, u); };

    if (P.new_kI) {
        // append each sequence's new token in the CTA that owns the key tile holding it, ahead of
        // that tile's TMA load (generic-proxy stores, then a proxy fence and the barrier below)
        for (int rd = 0;; ++rd) {
            const int u = indexer_unit_of(rd, blockIdx.x, gridDim.x);
            if (u >= P.num_units) break;
            const IndexerUnit U = unit_at(rd, u);
            const long long pos = use_tab ? utab[rd].pos : P.ctx_len[U.p];
            if (pos < 0 || pos >= P.Lk) {  // reported once per sequence; the sequence is not appended
                if (U.kt0 == 0 && threadIdx.x == 0) record_error(DSA_DEV_ERR_BOUNDS, 0x501);
                continue;
            }
            const int kt = (int)(pos / kIdxBM);
            if (kt < U.kt0 || kt >= U.kt1) continue;
            const long long row = (long long)U.p * P.Lk + pos;
            for (int i = threadIdx.x; i < P.kv16; i += blockDim.x) {
                P.cache_k[row * P.kv16 + i] = P.new_k[(long long)U.p * P.kv16 + i];
                P.cache_v[row * P.kv16 + i] = P.new_v[(long long)U.p * P.kv16 + i];
            }
            for (int i = threadIdx.x; i < P.kI16; i += blockDim.x)
                P.cache_kI[row * P.kI16 + i] = P.new_kI[(long long)U.p * P.kI16 + i];
        }
        asm volatile("fence.proxy.async.global;" ::: "memory");
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&a_full[i], 1);
            mbar_init(&a_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&q_full[i], 1);
            mbar_init(&q_empty[i], 1);
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], C::NWG * 128);
        }
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&map_q);
        prefetch_tensormap(&map_k);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int grid = gridDim.x, cta = blockIdx.x;

    if (warp < 4) {
      if constexpr (C::REGSPLIT) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(C::ROLE_REGS));
      if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int st = 0;
            uint32_t a_ph = 0, q_ph = 0;
            int qbuf = 0;
            bool ok = true;
            for (int rd = 0; ok; ++rd) {
                const int u = indexer_unit_of(rd, cta, grid);
                if (u >= P.num_units) break;
                const IndexerUnit U = unit_at(rd, u);
                if (U.kt0 >= U.kt1) continue;
                ok = wait_parity(&q_empty[qbuf], q_ph ^ 1, 0x101, abort_flag);
                if (!ok) break;
                mbar_arrive_expect_tx(&q_full[qbuf], P.q_box_bytes);
                tma_load_3d(sB + qbuf * C::B_BYTES, &map_q, &q_full[qbuf], 0, U.qb * C::TB * HI, U.p);
                if (++qbuf == 2) { qbuf = 0; q_ph ^= 1; }
                for (int kt = U.kt0; kt < U.kt1; ++kt) {
                    ok = wait_parity(&a_empty[st], a_ph ^ 1, 0x102, abort_flag);
                    if (!ok) break;
                    mbar_arrive_expect_tx(&a_full[st], P.k_box_bytes);
                    tma_load_3d(sA + st * C::A_BYTES, &map_k, &a_full[st], 0, kt * kIdxBM, U.p);
                    if (++st == STAGES) { st = 0; a_ph ^= 1; }
                }
            }
            if (!ok) {
                // Let the copies already issued land before the CTA leaves (bounded waits).  The
                // last copy into stage i used phase a_ph if i < st, else a_ph ^ 1; waiting on a
                // phase that already completed returns at once.
                for (int i = 0; i < STAGES; ++i) wait_parity(&a_full[i], i < st ? a_ph : a_ph ^ 1, 0x103, nullptr);
                for (int i = 0; i < 2; ++i) wait_parity(&q_full[i], i < qbuf ? q_ph : q_ph ^ 1, 0x104, nullptr);
            }
        }
      } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32<kIdxBM, BN>();
            int st = 0, ab = 0, qbuf = 0;
            uint32_t a_ph = 0, acc_ph = 0, q_ph = 0;
            bool ok = true;
            for (int rd = 0; ok; ++rd) {
                const int u = indexer_unit_of(rd, cta, grid);
                if (u >= P.num_units) break;
                const IndexerUnit U = unit_at(rd, u);
                if (U.kt0 >= U.kt1) continue;
                ok = wait_parity(&q_full[qbuf], q_ph, 0x201, abort_flag);
                if (!ok) break;
                const uint64_t bdesc = smem_desc_k128_sw128(sB + qbuf * C::B_BYTES);
                for (int kt = U.kt0; kt < U.kt1; ++kt) {
                    ok = wait_parity(&a_full[st], a_ph, 0x202, abort_flag) &&
                         wait_parity(&acc_empty[ab], acc_ph ^ 1, 0x203, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    const uint64_t adesc = smem_desc_k128_sw128(sA + st * C::A_BYTES);
                    const uint32_t d_tmem = tmem_base + ab * BN;
#pragma unroll
                    for (int kk = 0; kk < kIdxBK / 16; ++kk)  // K = 16 per MMA, 32 bytes along the row
                        umma_bf16(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc, kk > 0 ? 1u : 0u);
                    umma_commit(&a_empty[st]);
                    umma_commit(&acc_full[ab]);
                    if (++st == STAGES) { st = 0; a_ph ^= 1; }
                    if (++ab == 2) { ab = 0; acc_ph ^= 1; }
                }
                if (!ok) break;
                umma_commit(&q_empty[qbuf]);
                if (++qbuf == 2) { qbuf = 0; q_ph ^= 1; }
            }
        }
      }
    } else {
        if constexpr (C::REGSPLIT) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(C::EPI_REGS));
        // ------------------------------------------------------------ epilogue warpgroups
        const int et = threadIdx.x - 128;           // 0 .. NWG*128-1
        const int wg = et >> 7;                     // column half
        const int quarter = warp & 3;               // TMEM lanes this warp may access
        const int key_in_tile = quarter * 32 + lane;
        int ab = 0;
        uint32_t acc_ph = 0;
        for (int rd = 0;; ++rd) {
            const int u = indexer_unit_of(rd, cta, grid);
            if (u >= P.num_units) break;
            const IndexerUnit U = unit_at(rd, u);
            if (U.kt0 >= U.kt1) continue;
            // This unit's weights for this warpgroup's columns (column c = token*HI + head), held in
            // registers for all of the unit's key tiles: columns [c, c+8) are 8 consecutive bf16 of
            // w (the unit's tokens are consecutive rows), one 16-byte load each; tokens past the
            // unit's rows get weight 0.
            float wr[C::COLS_WG];
            {
                const __nv_bfloat16* wu = P.w + ((long long)U.p * P.Lq + (long long)U.qb * C::TB) * HI;
#pragma unroll
                for (int cc = 0; cc < C::COLS_WG; cc += 8) {
                    const int c = wg * C::COLS_WG + cc;
                    if ((c + 7) / HI < U.rows) {
                        const uint4 raw = use_tab ? utab[rd].w[c / 8] : __ldg(reinterpret_cast<const uint4*>(wu + c));
                        const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const uint32_t bits = (e & 1) ? (wv[e >> 1] & 0xFFFF0000u) : (wv[e >> 1] << 16);
                            wr[cc + e] = __uint_as_float(bits) * weight_store_scale<HI>((c + e) % HI);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            wr[cc + e] = (c + e) / HI < U.rows
                                             ? __bfloat162float(wu[c + e]) * weight_store_scale<HI>((c + e) % HI)
                                             : 0.f;
                    }
                }
            }
            bool ok = true;
            for (int kt = U.kt0; kt < U.kt1; ++kt) {
                ok = wait_parity(&acc_full[ab], acc_ph, 0x301, abort_flag);
                __syncwarp();  // reconverge before the warp-collective tcgen05.ld
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after();
                // key positions fit in 32 bits (the entry points refuse Lk > INT32_MAX)
                const int s = kt * kIdxBM + key_in_tile;
                const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + ab * BN + wg * C::COLS_WG;
                // this lane's score of the unit's first token (row0) and key s; token j adds j*ld
                float* const srow = P.scores + ((long long)U.p * P.Lq + (long long)U.qb * C::TB) * P.ld + s;
                // s <= tq0 + tok also keeps s < Lk: a valid token's position is below Lk
                const int tq0 = (int)U.tq0;
                // the accumulator is released right after its last columns are in registers
                float cur[C::CHUNK];
                float2 carry[2];
#pragma unroll
                for (int i = 0; i < 2; ++i) carry[i] = make_float2(0.f, 0.f);
#pragma unroll
                for (int ch = 0; ch < C::NCHUNK; ++ch) {
                    tmem_ld_chunk<C::CHUNK>(taddr + ch * C::CHUNK, cur);
                    tmem_ld_wait();
                    if (ch + 1 == C::NCHUNK) {
                        tc_fence_before();
                        mbar_arrive(&acc_empty[ab]);
                    }
                    const int cw = ch * C::CHUNK;  // column offset inside this warpgroup
                    if constexpr (HI <= C::CHUNK) {
#pragma unroll
                        for (int j = 0; j < C::CHUNK / HI; ++j) {
                            const float a = head_sum<HI>(cur + j * HI, wr + cw + j * HI);
                            const int tok = (wg * C::COLS_WG + cw) / HI + j;
                            if (tok < U.rows && s <= tq0 + tok) srow[(long long)tok * P.ld] = a;
                        }
                    } else {
                        head_sum_acc<C::CHUNK>(cur, wr + cw, carry);
                        if ((wg * C::COLS_WG + cw + C::CHUNK) % HI == 0) {
                            const float a = (carry[0].x + carry[0].y) + (carry[1].x + carry[1].y);
                            const int tok = (wg * C::COLS_WG + cw) / HI;
                            if (tok < U.rows && s <= tq0 + tok) srow[(long long)tok * P.ld] = a;
#pragma unroll
                            for (int i = 0; i < 2; ++i) carry[i] = make_float2(0.f, 0.f);
                        }
                    }
                }
                if (++ab == 2) { ab = 0; acc_ph ^= 1; }
            }
            if (!ok) break;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace dsa
