// prefill_sm100.cuh -- fused soft-capped local/global GQA attention forward
// (prefill, dense and packed variable-length) for B200 / sm_100a.
//
// Operation: Gemma 2 card, "Method", per-layer attention pseudo-code
// (scale queries, grouped scores, 50*tanh(s/50) cap, causal mask and 4096
// window on local layers, softmax over keys, grouped mix of the values);
// cap formula from the "Gemma 2 Guide", section 1.
//
// Design (one persistent CTA per SM, 192 threads, warp-specialised):
//   warp 0      TMA producer: Q tile once per work unit, then K/V tiles into a
//               ring of shared-memory slots (128-byte swizzle).
//   warp 1      UMMA issuer (one thread): S = Q K^T into TMEM (two S buffers),
//               O += P V with P read from TMEM; owns the TMEM allocation.
//   warps 2..5  softmax + epilogue: thread r owns MMA row r (TMEM lane r).
// A work unit is (sequence, KV head g, 64 query positions); its 128 MMA rows
// are the two query heads 2g, 2g+1 that share KV head g (row = head_local*64 +
// position), so each K/V tile feeds both heads. Only KV tiles that intersect
// the causal band (and the window on local layers) are visited, and only
// tiles that cross a band edge evaluate the mask.
// Softmax: fp32, log2 domain. s2 = C*log2(e)*tanh(x/C) computed as
// C*log2(e)*(1 - 2/(1 + 2^(2*x*log2(e)/C))) with ex2/rcp, then a running max
// per row with lazy rescaling of O (only when the max grows by more than
// 2^8), p = 2^(s2 - m) rounded to bf16 for the PV product, row sum in fp32.
// lse = ln2 * (m + log2(l)).
#pragma once

#include "common.cuh"

namespace g2 {

constexpr int PF_THREADS = 192;
constexpr int PF_BM = 128;   // MMA rows per tile (64 positions x 2 heads)
constexpr int PF_QPOS = 64;  // query positions per tile
constexpr int PF_BN = 128;   // keys per KV tile
constexpr int PF_TMEM_COLS = 512;
constexpr int PF_S_COL0 = 256;  // S buffers at TMEM columns 256 and 384; O at 0
constexpr float PF_RESCALE_LOG2 = 8.0f;

template <int D>
struct PfCfg {
    static constexpr int SLOT_BYTES = (D == 64) ? 16384 : 32768;
    static constexpr int KCOLS = SLOT_BYTES / (PF_BN * 2);  // d-columns per K slot (64 or 128)
    static constexpr int KSL = D / KCOLS;                   // K slots per KV tile
    static constexpr int VROWS = SLOT_BYTES / (D * 2);      // keys per V slot
    static constexpr int VSL = PF_BN / VROWS;               // V slots per KV tile
    static constexpr int NSLOT = (D == 64) ? 8 : (D == 128 ? 5 : 4);
    static constexpr int Q_BYTES = PF_BM * D * 2;
    static constexpr int MAX_SEQ_TABLE = 1024;  // varlen: per-sequence unit prefix table
    static constexpr int SMEM_TILES = Q_BYTES + NSLOT * SLOT_BYTES;
    static constexpr int SMEM_BYTES = 1024 + SMEM_TILES + 1024 + 4 * (MAX_SEQ_TABLE + 1);
    static_assert(KCOLS % 64 == 0 && VROWS % 16 == 0, "tile shapes");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

struct PfParams {
    __nv_bfloat16* out;
    float* lse;
    const int* cu_q;  // varlen only
    const int* cu_k;  // varlen only
    int num_seqs;     // dense: B
    int T, S;         // dense sizes (varlen: unused)
    int H, Hkv;
    int q_offset;     // dense only
    int window;
    int varlen;
    int total_q;      // packed query rows (dense: B*T); lse head stride for varlen
    int num_units;
    int max_units_per_seq_tiles;  // dense: q tiles per sequence
    float k_exp;    // 2*alpha*log2(e)/C   (cap on)
    float cap_l2;   // C*log2(e)           (cap on)
    float scale_l2; // alpha*log2(e)       (cap off)
    int has_cap;
    unsigned long long timeout_ns;
};

struct PfUnit {
    int seq;     // sequence (dense: batch index)
    int g;       // KV head
    int t0;      // first query row of the tile within the sequence
    int tvalid;  // valid query rows in the tile (1..64)
    int qbase;   // packed row of the sequence's first query
    int kbase;   // packed row of the sequence's first key
    int qoff;    // position of query row 0 of the sequence
    int kt0;     // first KV tile (index of 128-key tile)
    int nkt;     // number of KV tiles
    int p_min, p_max;
};

// Work unit u of the launch. Dense: query tiles in descending order (longest
// rows first), then batch, then KV head. Varlen: sequences in order, each with
// its query tiles descending; `pre` holds the unit prefix per sequence.
__device__ __forceinline__ void pf_unit(const PfParams& P, const int* pre, int u, PfUnit& U) {
    int seq, lu, Tq, Sk, qbase, kbase;
    if (!P.varlen) {
        const int BG = P.num_seqs * P.Hkv;
        const int nq = P.max_units_per_seq_tiles;
        const int qt = nq - 1 - u / BG;
        const int rem = u % BG;
        seq = rem / P.Hkv;
        U.g = rem % P.Hkv;
        Tq = P.T;
        Sk = P.S;
        qbase = seq * P.T;
        kbase = seq * P.S;
        U.t0 = qt * PF_QPOS;
        U.qoff = P.q_offset;
    } else {
        int lo = 0, hi = P.num_seqs - 1;  // largest s with pre[s] <= u
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (pre[mid] <= u) lo = mid; else hi = mid - 1;
        }
        seq = lo;
        lu = u - pre[seq];
        qbase = P.cu_q[seq];
        kbase = P.cu_k[seq];
        Tq = P.cu_q[seq + 1] - qbase;
        Sk = P.cu_k[seq + 1] - kbase;
        const int nq = (Tq + PF_QPOS - 1) / PF_QPOS;
        const int qt = nq - 1 - lu / P.Hkv;
        U.g = lu % P.Hkv;
        U.t0 = qt * PF_QPOS;
        U.qoff = Sk - Tq;
    }
    U.seq = seq;
    U.qbase = qbase;
    U.kbase = kbase;
    U.tvalid = min(PF_QPOS, Tq - U.t0);
    U.p_min = U.t0 + U.qoff;
    U.p_max = U.t0 + U.tvalid - 1 + U.qoff;
    const int j_lo = P.window > 0 ? max(0, U.p_min - P.window + 1) : 0;
    const int j_hi = min(U.p_max, Sk - 1);
    U.kt0 = j_lo / PF_BN;
    U.nkt = j_hi / PF_BN - U.kt0 + 1;
}

// Static persistent schedule: round r gives CTA c unit r*G + c (even rounds)
// or r*G + G-1-c (odd rounds), so the longest units spread evenly.
__device__ __forceinline__ int pf_sched(int r, int c, int G) {
    return r * G + ((r & 1) ? (G - 1 - c) : c);
}

template <int D>
__global__ void __launch_bounds__(PF_THREADS, 1)
    prefill_fwd_sm100(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const PfParams P) {
    using C = PfCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t* sQ = base;
    uint8_t* sSlots = base + C::Q_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + C::SMEM_TILES);
    uint64_t* q_full = bars + 0;
    uint64_t* q_empty = bars + 1;
    uint64_t* s_full = bars + 2;   // [2]
    uint64_t* p_full = bars + 4;   // [2]
    uint64_t* o_done = bars + 6;   // [2]: PV(t) completes phase t/2 of o_done[t%2]
    uint64_t* o_free = bars + 8;
    uint64_t* drain = bars + 9;
    uint64_t* slot_full = bars + 10;              // [NSLOT]
    uint64_t* slot_empty = bars + 10 + C::NSLOT;  // [NSLOT]
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 10 + 2 * C::NSLOT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    int* pre = reinterpret_cast<int*>(base + C::SMEM_TILES + 1024);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 128);
            mbar_init(&o_done[i], 1);
        }
        mbar_init(o_free, 128);
        mbar_init(drain, 1);
        for (int i = 0; i < C::NSLOT; ++i) {
            mbar_init(&slot_full[i], 1);
            mbar_init(&slot_empty[i], 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (P.varlen) {  // unit prefix per sequence: Hkv * q-tiles of each sequence
        for (int s = threadIdx.x; s < P.num_seqs; s += blockDim.x) {
            const int t = max(0, P.cu_q[s + 1] - P.cu_q[s]);
            pre[s] = P.Hkv * ((t + PF_QPOS - 1) / PF_QPOS);
        }
        __syncthreads();
        if (warp == 0) {  // exclusive scan, 32 entries at a time
            int carry = 0;
            for (int s0 = 0; s0 < P.num_seqs; s0 += 32) {
                const int s = s0 + lane;
                const int x = (s < P.num_seqs) ? pre[s] : 0;
                int incl = x;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, incl, off);
                    if (lane >= off) incl += y;
                }
                if (s < P.num_seqs) pre[s] = carry + incl - x;
                carry += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (lane == 0) pre[P.num_seqs] = carry;
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, PF_TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const int G = gridDim.x;
    const int cta = blockIdx.x;
    const int num_units = P.varlen ? min(P.num_units, pre[P.num_seqs]) : P.num_units;
    const uint64_t lim = P.timeout_ns;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            uint32_t fill = 0;  // slot fills issued so far
            int unit_it = 0;
            int q_armed = 0;    // Q loads issued so far
            bool ok = true;
            for (int r = 0; ok && r * G < num_units; ++r) {
                const int u = pf_sched(r, cta, G);
                if (u >= num_units) continue;
                PfUnit U;
                pf_unit(P, pre, u, U);
                if (unit_it > 0) {
                    ok = mbar_wait(q_empty, (unit_it - 1) & 1, abort_flag, lim, SITE_PROD_Q_EMPTY);
                    if (!ok) break;
                }
                mbar_arrive_expect_tx(q_full, C::Q_BYTES);
                ++q_armed;
#pragma unroll
                for (int c = 0; c < D / 64; ++c)
                    tma_load_3d(sQ + c * 16384, &tmQ, q_full, c * 64, U.qbase + U.t0, 2 * U.g);
                // Consumption order of the MMA warp: K0, K1, V0, K2, V1, ..., V(n-1).
                auto load_k = [&](int jj) -> bool {
                    const int key0 = U.kbase + (U.kt0 + jj) * PF_BN;
#pragma unroll
                    for (int s = 0; s < C::KSL; ++s) {
                        const int slot = fill % C::NSLOT;
                        if (!mbar_wait(&slot_empty[slot], ((fill / C::NSLOT) & 1) ^ 1, abort_flag,
                                       lim, SITE_PROD_SLOT_EMPTY))
                            return false;
                        mbar_arrive_expect_tx(&slot_full[slot], C::SLOT_BYTES);
                        uint8_t* dst = sSlots + slot * C::SLOT_BYTES;
#pragma unroll
                        for (int b = 0; b < C::KCOLS / 64; ++b)
                            tma_load_3d(dst + b * (PF_BN * 128), &tmK, &slot_full[slot],
                                        s * C::KCOLS + b * 64, key0, U.g);
                        ++fill;
                    }
                    return true;
                };
                auto load_v = [&](int jj) -> bool {
                    const int key0 = U.kbase + (U.kt0 + jj) * PF_BN;
#pragma unroll
                    for (int s = 0; s < C::VSL; ++s) {
                        const int slot = fill % C::NSLOT;
                        if (!mbar_wait(&slot_empty[slot], ((fill / C::NSLOT) & 1) ^ 1, abort_flag,
                                       lim, SITE_PROD_SLOT_EMPTY))
                            return false;
                        mbar_arrive_expect_tx(&slot_full[slot], C::SLOT_BYTES);
                        uint8_t* dst = sSlots + slot * C::SLOT_BYTES;
#pragma unroll
                        for (int b = 0; b < D / 64; ++b)
                            tma_load_3d(dst + b * (C::VROWS * 128), &tmV, &slot_full[slot], b * 64,
                                        key0 + s * C::VROWS, U.g);
                        ++fill;
                    }
                    return true;
                };
                ok = load_k(0);
                for (int jj = 0; ok && jj < U.nkt; ++jj) {
                    if (jj + 1 < U.nkt) ok = load_k(jj + 1);
                    if (ok) ok = load_v(jj);
                }
                ++unit_it;
            }
            // Drain: every copy this thread issued lands before the CTA exits.
            const uint32_t last = fill < (uint32_t)C::NSLOT ? fill : (uint32_t)C::NSLOT;
            for (uint32_t i = 0; i < last; ++i) {
                const uint32_t f = fill - 1 - i;
                mbar_wait_drain(&slot_full[f % C::NSLOT], (f / C::NSLOT) & 1, lim);
            }
            if (q_armed > 0) mbar_wait_drain(q_full, (q_armed - 1) & 1, lim);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ UMMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC_S = idesc_bf16(PF_BM, PF_BN, false);
            constexpr uint32_t IDESC_O = idesc_bf16(PF_BM, D, true);
            const uint32_t sQ_addr = smem_u32(sQ);
            const uint32_t slots_addr = smem_u32(sSlots);
            uint32_t fill = 0;
            uint32_t tile = 0;  // KV tiles processed by this CTA (S/P/PV index)
            int unit_it = 0;
            bool ok = true;

            auto issue_s = [&](uint32_t gt) -> bool {
                const uint32_t buf = gt & 1;
                if (gt >= 2) {  // S buffer reuse: P(gt-2) consumed by PV(gt-2)
                    if (!mbar_wait(&o_done[buf], ((gt - 2) >> 1) & 1, abort_flag, lim,
                                   SITE_MMA_O_DONE))
                        return false;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem + PF_S_COL0 + buf * PF_BN;
#pragma unroll
                for (int s = 0; s < C::KSL; ++s) {
                    const int slot = fill % C::NSLOT;
                    if (!mbar_wait(&slot_full[slot], (fill / C::NSLOT) & 1, abort_flag, lim,
                                   SITE_MMA_SLOT_FULL))
                        return false;
                    tc_fence_after();
                    const uint32_t kb = slots_addr + slot * C::SLOT_BYTES;
#pragma unroll
                    for (int kk = 0; kk < C::KCOLS / 16; ++kk) {
                        const int dcol = s * C::KCOLS + kk * 16;  // Q column of this k-step
                        const uint64_t a = sdesc_sw128(
                            sQ_addr + (dcol / 64) * 16384 + ((dcol % 64) / 16) * 32, 16, 1024);
                        const uint64_t b = sdesc_sw128(
                            kb + ((kk * 16) / 64) * (PF_BN * 128) + (((kk * 16) % 64) / 16) * 32,
                            16, 1024);
                        umma_ss(d_tmem, a, b, IDESC_S, (s | kk) != 0);
                    }
                    umma_commit(&slot_empty[slot]);
                    ++fill;
                }
                umma_commit(&s_full[buf]);
                return true;
            };
            auto issue_pv = [&](uint32_t gt, bool first) -> bool {
                const uint32_t buf = gt & 1;
                const uint32_t p_tmem = tmem + PF_S_COL0 + buf * PF_BN;
#pragma unroll
                for (int s = 0; s < C::VSL; ++s) {
                    const int slot = fill % C::NSLOT;
                    if (!mbar_wait(&slot_full[slot], (fill / C::NSLOT) & 1, abort_flag, lim,
                                   SITE_MMA_SLOT_FULL))
                        return false;
                    tc_fence_after();
                    const uint32_t vb = slots_addr + slot * C::SLOT_BYTES;
#pragma unroll
                    for (int kk = 0; kk < C::VROWS / 16; ++kk) {
                        const uint64_t b = sdesc_sw128(vb + kk * 16 * 128, C::VROWS * 128, 1024);
                        const uint32_t a = p_tmem + (s * C::VROWS + kk * 16) / 2;
                        umma_ts(tmem, a, b, IDESC_O, (first && s == 0 && kk == 0) ? 0u : 1u);
                    }
                    umma_commit(&slot_empty[slot]);
                    ++fill;
                }
                umma_commit(&o_done[buf]);
                return true;
            };

            for (int r = 0; ok && r * G < num_units; ++r) {
                const int u = pf_sched(r, cta, G);
                if (u >= num_units) continue;
                PfUnit U;
                pf_unit(P, pre, u, U);
                ok = mbar_wait(q_full, unit_it & 1, abort_flag, lim, SITE_MMA_Q_FULL);
                if (!ok) break;
                ok = issue_s(tile);
                for (int jj = 0; ok && jj < U.nkt; ++jj) {
                    const uint32_t gt = tile + jj;
                    if (jj + 1 < U.nkt) {
                        ok = issue_s(gt + 1);
                        if (!ok) break;
                    } else {
                        umma_commit(q_empty);  // last S of the unit issued: Q reusable
                    }
                    ok = mbar_wait(&p_full[gt & 1], (gt >> 1) & 1, abort_flag, lim,
                                   SITE_MMA_P_FULL);
                    if (!ok) break;
                    if (jj == 0 && unit_it > 0) {
                        ok = mbar_wait(o_free, (unit_it - 1) & 1, abort_flag, lim,
                                       SITE_MMA_O_FREE);
                        if (!ok) break;
                    }
                    tc_fence_after();
                    ok = issue_pv(gt, jj == 0);
                }
                tile += U.nkt;
                ++unit_it;
            }
            // Drain: all issued UMMAs complete before TMEM is released.
            umma_commit(drain);
            mbar_wait_drain(drain, 0, lim);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        const int r = ((warp & 3) << 5) | lane;        // MMA row == TMEM lane
        const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const int hl = r >> 6;                          // head within the pair
        const int pr = r & 63;                          // position within the tile
        uint32_t tile = 0;
        int unit_it = 0;
        bool ok = true;
        for (int rr = 0; ok && rr * G < num_units; ++rr) {
            const int u = pf_sched(rr, cta, G);
            if (u >= num_units) continue;
            PfUnit U;
            pf_unit(P, pre, u, U);
            const int p = U.p_min + pr;  // absolute query position of this row
            float m_ref = -INFINITY;     // log2-domain reference max of the row
            float l = 0.f;               // sum of the fp32 weights (for lse)
            float lr = 0.f;              // sum of the bf16-rounded weights (normalises O)
            for (int jj = 0; jj < U.nkt; ++jj) {
                const uint32_t gt = tile + jj;
                const uint32_t buf = gt & 1;
                ok = mbar_wait(&s_full[buf], (gt >> 1) & 1, abort_flag, lim, SITE_SM_S_FULL);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after();
                const uint32_t s_addr = tmem + lane_addr + PF_S_COL0 + buf * PF_BN;
                float s[PF_BN];
#pragma unroll
                for (int c = 0; c < PF_BN / 32; ++c) {
                    uint32_t v[32];
                    tmem_ld32(s_addr + c * 32, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(v[i]);
                }
                // capped logit in log2 units
                if (P.has_cap) {
#pragma unroll
                    for (int i = 0; i < PF_BN; ++i) {
                        const float e = ex2_approx(s[i] * P.k_exp);
                        const float rc = rcp_approx(1.0f + e);
                        s[i] = fmaf(-2.0f * P.cap_l2, rc, P.cap_l2);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < PF_BN; ++i) s[i] *= P.scale_l2;
                }
                const int j0 = (U.kt0 + jj) * PF_BN;  // key position of column 0
                const bool boundary =
                    (j0 + PF_BN - 1 > U.p_min) || (P.window > 0 && j0 < U.p_max - P.window + 1);
                if (boundary) {
                    const int hi = p - j0;  // visible columns: [lo, hi]
                    const int lo = P.window > 0 ? p - P.window + 1 - j0 : -1;
#pragma unroll
                    for (int i = 0; i < PF_BN; ++i)
                        if (i > hi || i < lo) s[i] = -INFINITY;
                }
                float mt = s[0];
#pragma unroll
                for (int i = 1; i < PF_BN; ++i) mt = fmaxf(mt, s[i]);
                const float m_new = fmaxf(m_ref, mt);
                const bool need = (m_ref != -INFINITY) && (m_new > m_ref + PF_RESCALE_LOG2);
                if (__any_sync(0xffffffffu, need)) {
                    // O holds PV(0..gt-1) relative to m_ref: scale it to m_new.
                    ok = mbar_wait(&o_done[(gt - 1) & 1], ((gt - 1) >> 1) & 1, abort_flag, lim,
                                   SITE_SM_O_DONE);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    tc_fence_after();
                    const float f = need ? ex2_approx(m_ref - m_new) : 1.0f;
                    const uint32_t o_addr = tmem + lane_addr;
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t v[32];
                        tmem_ld32(o_addr + c * 32, v);
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            v[i] = __float_as_uint(__uint_as_float(v[i]) * f);
                        tmem_st32(o_addr + c * 32, v);
                    }
                    tmem_wait_st();
                    l *= f;
                    lr *= f;
                    if (need) m_ref = m_new;
                }
                if (m_ref == -INFINITY) m_ref = mt;
                const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
                // The PV product sees bf16(p); normalising O by the sum of the
                // same rounded weights makes them sum to one exactly, so their
                // rounding errors cancel against the row's mean value.
                float lsum = 0.f, lrsum = 0.f;
#pragma unroll
                for (int c = 0; c < PF_BN / 64; ++c) {
                    uint32_t pk[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float a = ex2_approx(s[c * 64 + 2 * i] - m_use);
                        const float b = ex2_approx(s[c * 64 + 2 * i + 1] - m_use);
                        lsum += a + b;
                        pk[i] = pack_bf16x2(a, b);
                        lrsum += __uint_as_float(pk[i] << 16) + __uint_as_float(pk[i] & 0xFFFF0000u);
                    }
                    tmem_st32(s_addr + c * 32, pk);
                }
                l += lsum;
                lr += lrsum;
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&p_full[buf]);
            }
            if (!ok) break;
            // ---- epilogue: O / l -> bf16, lse
            // PV(gl) completing implies every earlier UMMA of this CTA completed.
            const uint32_t gl = tile + U.nkt - 1;
            ok = mbar_wait(&o_done[gl & 1], (gl >> 1) & 1, abort_flag, lim, SITE_SM_O_DONE);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            const bool valid = pr < U.tvalid;
            const int h = 2 * U.g + hl;
            const float inv_l = 1.0f / lr;
            const size_t orow = static_cast<size_t>(U.qbase + U.t0 + pr) * P.H + h;
            __nv_bfloat16* optr = P.out + orow * D;
            const uint32_t o_addr = tmem + lane_addr;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t v[32];
                tmem_ld32(o_addr + c * 32, v);
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * inv_l,
                                        __uint_as_float(v[2 * i + 1]) * inv_l);
                if (valid) {
                    uint4* dst = reinterpret_cast<uint4*>(optr + c * 32);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                }
            }
            if (valid && P.lse != nullptr) {
                const float lse = (m_ref + log2f(l)) * 0.69314718055994531f;
                size_t li;
                if (P.varlen)
                    li = static_cast<size_t>(h) * P.total_q + U.qbase + U.t0 + pr;
                else
                    li = (static_cast<size_t>(U.seq) * P.H + h) * P.T + U.t0 + pr;
                P.lse[li] = lse;
            }
            tc_fence_before();
            mbar_arrive(o_free);
            tile += U.nkt;
            ++unit_it;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, PF_TMEM_COLS);
    }
}

}  // namespace g2
