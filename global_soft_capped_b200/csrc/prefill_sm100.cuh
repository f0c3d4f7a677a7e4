// prefill_sm100.cuh -- fused soft-capped local/global GQA attention forward
// (prefill, dense and packed variable-length) for B200 / sm_100a.
//
// Operation: Gemma 2 card, "Method", per-layer attention pseudo-code
// (scale queries, grouped scores, 50*tanh(s/50) cap, causal mask and 4096
// window on local layers, softmax over keys, grouped mix of the values);
// cap formula from the "Gemma 2 Guide", section 1.
//
// Design (one persistent CTA per SM, 512 threads, warp-specialised):
//   warps 0..7  softmax: warps w and w+4 share MMA rows 32*(w%4)..+31 (the
//               TMEM lanes of their sub-partition); part w/4 takes key columns
//               64*part..+63 of every S tile and O columns part*D/2..+D/2-1
//               when O is rescaled. With a running max the parts exchange
//               their partial row maxima through shared memory once per tile
//               (a bounded mbarrier wait), so both use the same one. At the end
//               of a unit they hand the row sums to the epilogue warps and go
//               on with the next unit.
//   warp 8      TMA producer: Q tile once per work unit, then K/V tiles into a
//               ring of shared-memory slots (128-byte swizzle).
//   warp 9      UMMA issuer (one thread): S = Q K^T into TMEM (two S buffers),
//               O += P V with P read from TMEM; owns the TMEM allocation.
//   warps 12..15 epilogue, one per TMEM lane quadrant: once a unit's last PV
//               has completed, O / l -> bf16 rows and the log-sum-exp, while
//               the softmax warps already work on the next unit; the next
//               unit's first PV waits until O has been read. (Warps 10 and 11
//               only keep the warpgroups aligned.)
// A work unit is (sequence, KV head g, 64 query positions); its 128 MMA rows
// are the two query heads 2g, 2g+1 that share KV head g (row = head_local*64 +
// position), so each K/V tile feeds both heads. Only KV tiles that intersect
// the causal band (and the window on local layers) are visited, and only
// tiles that cross a band edge evaluate the mask.
// Softmax: fp32, log2 domain. s2 = C*log2(e)*tanh(x/C): when |x/C| <= 1/4 over
// a warp's tile, by the Taylor series of tanh through x^7 on the FMA pipe;
// otherwise as C*log2(e)*(1 - 2/(1 + 2^(2*x*log2(e)/C))) with ex2/rcp. Then a running max
// per row with lazy rescaling of O (only when the max grows by more than
// 2^8), p = 2^(s2 - m) rounded to bf16 for the PV product, row sum in fp32.
// lse = ln2 * (m + log2(l)).
#pragma once

#include "common.cuh"

namespace g2 {

constexpr int PF_NSPLIT = 2;     // softmax warps per TMEM lane quadrant
constexpr int PF_SOFTMAX_THREADS = 128 * PF_NSPLIT;
constexpr int PF_WARP_PRODUCER = 4 * PF_NSPLIT;
constexpr int PF_WARP_MMA = PF_WARP_PRODUCER + 1;
constexpr int PF_WARP_EPI = PF_WARP_PRODUCER + 4;   // warps 12..15
constexpr int PF_EPI_WARPS = 4;
constexpr int PF_THREADS = PF_SOFTMAX_THREADS + 256;  // + producer, issuer, 2 idle, 4 epilogue
constexpr int PF_BM = 128;   // MMA rows per tile (64 positions x 2 heads)
constexpr int PF_QPOS = 64;  // query positions per tile
constexpr int PF_BN = 128;   // keys per KV tile
constexpr int PF_PHC = PF_BN / PF_NSPLIT;  // keys (S columns) per softmax column part
constexpr int PF_TMEM_COLS = 512;
constexpr int PF_S_COL0 = 256;  // S buffers at TMEM columns 256 and 384; O at 0
constexpr float PF_RESCALE_LOG2 = 8.0f;
// Taylor coefficients of tanh(u) = u (1 + c1 u^2 + c2 u^4 + c3 u^6 + ...):
// -1/3, 2/15, -17/315 (the series of tanh, from its Bernoulli-number form; the
// next coefficient, 62/2835, bounds the truncation for |u| <= 1/4).
constexpr float kTanhC1 = -1.0f / 3.0f;
constexpr float kTanhC2 = 2.0f / 15.0f;
constexpr float kTanhC3 = -17.0f / 315.0f;
constexpr float PF_POLY_U_MAX = 0.25f;  // |x / C| bound of the series path
// Largest C log2(e) for which the fixed softmax shift keeps every weight a
// normal float: 2^(-2 C log2(e) + 64) >= 2^-126.
constexpr float PF_FIXED_REF_MAX = 95.0f;
// softmax variants of the forward kernel (template parameter SM)
constexpr int PF_SM_FIXED = 0;  // cap on, fixed softmax shift
constexpr int PF_SM_CAP = 1;    // cap on, running max
constexpr int PF_SM_NOCAP = 2;  // no cap, running max

// CG = 1: one CTA per unit of 64 query positions. CG = 2 (d = 256 only): a CTA
// pair per unit of 128 positions, 64 per CTA; each CTA stages half of every
// K tile (64 of its 128 keys) and half of every V tile (128 of its 256
// d-columns), and the even CTA issues M = 256 UMMAs over both halves.
template <int D, int CG = 1>
struct PfCfg {
    static_assert(CG == 1 || (CG == 2 && D == 256), "CTA pairs are built for d = 256");
    static constexpr int SLOT_BYTES = (D == 64) ? 16384 : 32768;
    static constexpr int KROWS = PF_BN / CG;                // keys of a K tile staged by this CTA
    static constexpr int KCOLS = SLOT_BYTES / (KROWS * 2);  // d-columns per K slot
    static constexpr int KSL = D / KCOLS;                   // K slots per KV tile
    static constexpr int VCOLS = D / CG;                    // d-columns of V staged by this CTA
    static constexpr int VROWS = SLOT_BYTES / (VCOLS * 2);  // keys per V slot
    static constexpr int VSL = PF_BN / VROWS;               // V slots per KV tile
    static constexpr int NSLOT = (D == 64) ? 8 : (D == 128 ? 5 : 4);
    static constexpr int Q_BYTES = PF_BM * D * 2;
    static constexpr int MAX_SEQ_TABLE = 1024;  // varlen: sequences per launch
    static constexpr int VL_BYTES = 4 * (3 * MAX_SEQ_TABLE + 1);
    static constexpr int SMEM_TILES = Q_BYTES + NSLOT * SLOT_BYTES;
    // barriers, partial row maxima [2][NSPLIT][128], row statistics handed to
    // the epilogue by unit parity: sums [2][NSPLIT][128][2], maxima [2][128]
    static constexpr int CTRL_BYTES =
        1024 + 2 * PF_NSPLIT * 128 * 4 + 2 * PF_NSPLIT * 128 * 2 * 4 + 2 * 128 * 4;
    static constexpr int SMEM_BYTES = 1024 + SMEM_TILES + CTRL_BYTES + VL_BYTES;
    static_assert(KCOLS % 64 == 0 && KCOLS <= D && VROWS % 16 == 0 && VROWS <= PF_BN,
                  "tile shapes");
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
    // paged K/V (varlen queries only): blocks of 2^kv_block_shift >= 128 rows
    // located through kv_table[seq][block]; S_s = kv_lens[seq]
    const int* kv_table;
    const int* kv_lens;
    int kv_block_shift, kv_max_blocks, kv_num_blocks;
    int paged;
    int total_q;      // packed query rows (dense: B*T); lse head stride for varlen
    int total_k;      // packed key rows (varlen, packed K/V)
    int num_units;
    int max_units_per_seq_tiles;  // dense: q tiles per sequence
    float k_exp;    // 2*alpha*log2(e)/C   (cap on)
    float cap_l2;   // C*log2(e)           (cap on)
    float scale_l2; // alpha*log2(e)
    float u_scale;  // alpha/C             (cap on)
    float poly_acc_max;  // largest |q.k| for which |alpha q.k / C| <= PF_POLY_U_MAX
    int has_cap;
    // Fixed softmax shift (cap on, C log2(e) <= PF_FIXED_REF_MAX): every capped
    // logit lies in [-C log2(e), C log2(e)], so p = 2^(s2 - fixed_ref) with
    // fixed_ref = C log2(e) - 64 stays in [2^(-2 C log2(e) + 64), 2^64]: normal
    // in fp32 and bf16, and sums over up to 2^31 keys stay finite. The
    // softmax is invariant to the shift, so no running max is needed.
    int fixed_ref_on;
    float fixed_ref;
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

// Per-launch varlen schedule in shared memory: sequences ranked by their work
// (KV tiles over all their query tiles), heaviest first, so the light units
// land at the end of the static schedule; within a sequence, query tiles run
// longest first. Consecutive units stay within one sequence, which keeps that
// sequence's K/V resident in L2 while all SMs work on it.
struct VlTables {
    int* work;   // [num_seqs] KV tiles of the sequence (one KV head)
    int* order;  // [num_seqs] sequences ranked by work, descending
    int* cum;    // [num_seqs + 1] units before each ranked sequence; cum[num_seqs] = total
};

// Rows [*base, *base + *len) of sequence s in a packed tensor of `total` rows
// described by cu[]: clamped into [0, total), so that malformed offsets can
// give wrong results but never an access outside the tensor.
__device__ __forceinline__ void pf_seq_rows(const int* cu, int s, int total, int* base,
                                            int* len) {
    const int b0 = min(max(cu[s], 0), total);
    const int b1 = min(max(cu[s + 1], b0), total);
    *base = b0;
    *len = b1 - b0;
}

// KV tiles visited by query tile t0 of a sequence (T queries at the end of S keys).
__device__ __forceinline__ int pf_tiles(int t0, int T, int S, int window) {
    const int tvalid = min(PF_QPOS, T - t0);
    const int p_min = t0 + (S - T), p_max = p_min + tvalid - 1;
    const int j_lo = window > 0 ? max(0, p_min - window + 1) : 0;
    const int j_hi = min(p_max, S - 1);
    return j_hi / PF_BN - j_lo / PF_BN + 1;
}

// Work unit u of the launch. Dense: query tiles in descending order (longest
// rows first), then batch, then KV head. Varlen: sequences in rank order, each
// with its query tiles descending, then KV head. A unit covers 64 * CG query
// positions; the KV tile range is that of the whole unit, and CTA `rank` of a
// pair takes the rows of positions t0 + 64*rank .. + 63 (tvalid may be <= 0
// for the odd CTA at the end of a sequence: it then stores nothing).
template <int CG = 1>
__device__ __forceinline__ void pf_unit(const PfParams& P, const VlTables& V, int u, PfUnit& U,
                                        int rank = 0) {
    constexpr int QT = PF_QPOS * CG;
    int seq, Tq, Sk, qbase, kbase;
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
        U.t0 = qt * QT;
        U.qoff = P.q_offset;
    } else {
        int lo = 0, hi = P.num_seqs - 1;  // largest rank with cum[rank] <= u
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (V.cum[mid] <= u) lo = mid; else hi = mid - 1;
        }
        seq = V.order[lo];
        const int lu = u - V.cum[lo];
        pf_seq_rows(P.cu_q, seq, P.total_q, &qbase, &Tq);
        if (P.paged) {
            kbase = 0;
            Sk = max(Tq, min(P.kv_lens[seq], P.kv_max_blocks << P.kv_block_shift));
        } else {
            pf_seq_rows(P.cu_k, seq, P.total_k, &kbase, &Sk);
        }
        const int nq = (Tq + QT - 1) / QT;
        U.g = lu % P.Hkv;
        U.t0 = (nq - 1 - lu / P.Hkv) * QT;
        U.qoff = Sk - Tq;
    }
    U.seq = seq;
    U.qbase = qbase;
    U.kbase = kbase;
    {  // KV tiles of the whole unit
        const int tv = min(QT, Tq - U.t0);
        const int p_lo = U.t0 + U.qoff, p_hi = U.t0 + tv - 1 + U.qoff;
        const int j_lo = P.window > 0 ? max(0, p_lo - P.window + 1) : 0;
        const int j_hi = min(p_hi, Sk - 1);
        U.kt0 = j_lo / PF_BN;
        U.nkt = j_hi / PF_BN - U.kt0 + 1;
    }
    U.t0 += PF_QPOS * rank;  // this CTA's rows
    U.tvalid = min(PF_QPOS, Tq - U.t0);
    U.p_min = U.t0 + U.qoff;
    U.p_max = U.p_min + max(U.tvalid, 1) - 1;
}

// Row of key `key` (relative to the sequence start) in the K/V tensor maps. A
// paged cache keeps every 128-key tile inside one block (blocks >= 128 rows).
// The table column stays inside the sequence's row and the entry inside the
// cache, whatever the lengths and the table hold.
__device__ __forceinline__ int pf_key_row(const PfParams& P, const PfUnit& U, int key) {
    if (!P.paged) return U.kbase + key;
    const int col = min(key >> P.kv_block_shift, P.kv_max_blocks - 1);
    int b = P.kv_table[static_cast<size_t>(U.seq) * P.kv_max_blocks + col];
    b = max(0, min(b, P.kv_num_blocks - 1));
    return (b << P.kv_block_shift) + (key & ((1 << P.kv_block_shift) - 1));
}

// Output rows of one warp (32 rows, one per lane, EC bf16 columns each as
// EC/2 packed words) stored so that every store instruction writes whole row
// segments: the 16-byte chunks are transposed within groups of NCH = EC/8
// lanes by an XOR-shuffle butterfly (log2 NCH stages, half the chunks moving
// in each), after which lane g*NCH + c holds chunk c of rows g*NCH + i in slot
// i. row_ptr(i) gives the destination of warp row i, or nullptr to skip it.
template <int EC, typename RowPtr>
__device__ __forceinline__ void pf_store_rows(uint32_t (&w)[EC / 2], int lane, RowPtr row_ptr) {
    constexpr int NCH = EC / 8;
    static_assert(NCH == 4 || NCH == 8, "row segments of 64 or 128 bytes");
#pragma unroll
    for (int k = NCH / 2; k >= 1; k >>= 1) {
        const bool upper = (lane & k) != 0;
#pragma unroll
        for (int j = 0; j < NCH; ++j) {
            if (j & k) continue;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint32_t send = upper ? w[4 * j + e] : w[4 * (j | k) + e];
                const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, k);
                if (upper)
                    w[4 * j + e] = recv;
                else
                    w[4 * (j | k) + e] = recv;
            }
        }
    }
    const int grp = lane / NCH, ch = lane % NCH;
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
        __nv_bfloat16* dst = row_ptr(grp * NCH + i);
        if (dst != nullptr)
            *reinterpret_cast<uint4*>(dst + 8 * ch) =
                make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
    }
}

// Dynamic schedule of packed sequences: per-launch unit counters (next unit,
// CTAs finished) at slot %gridid mod PF_SCHED_SLOTS. The CTA pairs take units
// in order from `next` (list scheduling, heaviest sequences first); the last
// CTA of a launch to finish zeroes its slot, so the slot is clean for the
// launch that reuses it (launches in flight at once use distinct grid ids).
constexpr int PF_SCHED_SLOTS = 4096;
__device__ unsigned int g_pf_sched[PF_SCHED_SLOTS][2];

// The general path of the fixed-shift softmax for one warp's PF_PHC columns of
// an S tile: tiles on the band's edges (columns outside [lo, hi] are masked)
// or with logits past the series range (series false: the exact cap). Out of
// line, so that the fast tile loop of the same kernel is compiled without it:
// inline, this rarely taken code cost the fast loop several percent at the
// 128-register bound. It reads the columns at `cols` again from TMEM (P has
// not been written over them yet), writes the bf16 weights at the start of
// the same columns, and returns the sums of the fp32 weights (x, y) and of
// the bf16-rounded ones (z, w), pair lanes as in the fast loop. Called by
// whole warps (the tcgen05 loads and stores are warp-wide).
__device__ __noinline__ float4 pf_softmax_general_fixed(uint32_t cols, int lo, int hi,
                                                        bool series, float b0, float b1,
                                                        float b2, float b3, float k_exp,
                                                        float cap_l2, float m_use) {
    constexpr int HC = PF_PHC;
    float s[HC];
    {
        uint32_t v[HC / 32][32];
#pragma unroll
        for (int c = 0; c < HC / 32; ++c) tmem_ld32_async(cols + 32 * c, v[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < HC / 32; ++c) tmem_reg_fence(v[c]);
#pragma unroll
        for (int i = 0; i < HC; ++i) s[i] = __uint_as_float(v[i / 32][i % 32]);
    }
    // capped logits in log2 units, then the mask
    if (series) {
#pragma unroll
        for (int i = 0; i < HC; ++i) {
            const float x2 = s[i] * s[i];
            float q = fmaf(x2, b3, b2);
            q = fmaf(x2, q, b1);
            q = fmaf(x2, q, b0);
            s[i] = s[i] * q;
        }
    } else {
#pragma unroll
        for (int i = 0; i < HC; ++i) {
            const float e = ex2_approx(s[i] * k_exp);
            const float rc = rcp_approx(1.0f + e);
            s[i] = fmaf(-2.0f * cap_l2, rc, cap_l2);
        }
    }
#pragma unroll
    for (int i = 0; i < HC; ++i)
        if (i > hi || i < lo) s[i] = -INFINITY;
    const float2 mneg = make_float2(-m_use, -m_use);
    float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    float2 lrs[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    uint32_t pk[HC / 2];
#pragma unroll
    for (int i = 0; i < HC / 2; ++i) {
        const float2 x = add2(make_float2(s[2 * i], s[2 * i + 1]), mneg);
        const float2 e = make_float2(ex2_approx(x.x), ex2_approx(x.y));
        ls[i & 1] = add2(ls[i & 1], e);
        pk[i] = pack_bf16x2(e.x, e.y);
        lrs[i & 1] = add_bf16x2_f32(lrs[i & 1], pk[i]);
    }
#pragma unroll
    for (int c = 0; c < HC / 32; ++c) {
        uint32_t pc[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) pc[i] = pk[16 * c + i];
        tmem_st16(cols + 16 * c, pc);
    }
    const float2 lsum = add2(ls[0], ls[1]);
    const float2 lrsum = add2(lrs[0], lrs[1]);
    return make_float4(lsum.x, lsum.y, lrsum.x, lrsum.y);
}

// Static persistent schedule: round r gives CTA c unit r*G + c (even rounds)
// or r*G + G-1-c (odd rounds), so the longest units spread evenly.
__device__ __forceinline__ int pf_sched(int r, int c, int G) {
    return r * G + ((r & 1) ? (G - 1 - c) : c);
}

// SM, the softmax variant: PF_SM_FIXED (cap on, fixed shift:
// PfParams::fixed_ref_on), PF_SM_CAP (cap on, running max) or PF_SM_NOCAP
// (running max). The host launches the one the parameters call for, so that
// each softmax carries only its own loops: compiled in beside the fixed-shift
// loop, the running-max exchange and the uncapped loop cost it about 15% at
// the 128-register bound.
template <int D, int CG, int SM>
__global__ void __launch_bounds__(PF_THREADS, 1)
    prefill_fwd_sm100(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const PfParams P) {
    using C = PfCfg<D, CG>;
    constexpr bool PAIR = CG == 2;
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
    // the last PV of a unit completed (one phase per unit): the epilogue warps
    // wait on it first, so that their o_done wait is never more than one
    // phase behind (o_done completes a phase per tile)
    uint64_t* o_last = bars + 10;
    uint64_t* slot_full = bars + 11;              // [NSLOT]
    uint64_t* slot_empty = bars + 11 + C::NSLOT;  // [NSLOT]
    // softmax warp pairs: max exchange per tile parity [4][2]
    uint64_t* xbar = bars + 11 + 2 * C::NSLOT;
    // row statistics of a unit handed to the epilogue warps, by unit parity [2]
    uint64_t* stat_full = xbar + 8;
    // dynamic schedule (packed sequences): the even CTA's producer publishes
    // each unit it takes in a ring of four in both CTAs (sq_full, one arrival);
    // every other role of both CTAs releases the entry on the even CTA's
    // sq_empty
    uint64_t* sq_full = stat_full + 2;   // [4]
    uint64_t* sq_empty = sq_full + 4;    // [4]
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sq_empty + 4);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    volatile int* sq_ring = reinterpret_cast<volatile int*>(tmem_holder + 2);  // [4]
    // partial row maxima of the column parts, by tile parity: [2][NSPLIT][128]
    float* xmax = reinterpret_cast<float*>(base + C::SMEM_TILES + 1024);
    // partial (l, lr) row sums of the parts at the end of a unit, by unit
    // parity: [2][NSPLIT][128][2]; the row's reference max: [2][128]
    float* xsum = xmax + 2 * PF_NSPLIT * 128;
    float* xref = xsum + 2 * PF_NSPLIT * 128 * 2;
    VlTables vt;
    vt.work = reinterpret_cast<int*>(base + C::SMEM_TILES + C::CTRL_BYTES);
    vt.order = vt.work + C::MAX_SEQ_TABLE;
    vt.cum = vt.order + C::MAX_SEQ_TABLE;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], CG * PF_SOFTMAX_THREADS / 32);
            mbar_init(&o_done[i], 1);
        }
        // softmax- and epilogue-side barriers take one arrival per warp
        // (elected lane, after __syncwarp orders the whole warp's prior
        // writes before it); a pair counts the warps of both CTAs on the even
        // CTA's p_full and o_free
        mbar_init(o_free, CG * PF_EPI_WARPS);
        for (int i = 0; i < 8; ++i) mbar_init(&xbar[i], PF_NSPLIT);
        for (int i = 0; i < 2; ++i) mbar_init(&stat_full[i], PF_SOFTMAX_THREADS / 32);
        // readers per CTA: softmax and epilogue warps, and the issuer (even
        // CTA) or the producer (odd CTA)
        for (int i = 0; i < 4; ++i) {
            mbar_init(&sq_full[i], 1);
            mbar_init(&sq_empty[i], CG * (PF_SOFTMAX_THREADS / 32 + PF_EPI_WARPS + 1));
        }
        mbar_init(drain, 1);
        mbar_init(o_last, 1);
        for (int i = 0; i < C::NSLOT; ++i) {
            mbar_init(&slot_full[i], 1);
            mbar_init(&slot_empty[i], 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (P.varlen) {  // per-launch schedule (see VlTables)
        const int ns = P.num_seqs;
        for (int s = threadIdx.x; s < ns; s += blockDim.x) {
            int qb, t, kb = 0, skr = 0;
            pf_seq_rows(P.cu_q, s, P.total_q, &qb, &t);
            if (!P.paged) pf_seq_rows(P.cu_k, s, P.total_k, &kb, &skr);
            const int sk = max(t, P.paged ? min(P.kv_lens[s], P.kv_max_blocks << P.kv_block_shift)
                                          : skr);
            int w = 0;
            for (int t0 = 0; t0 < t; t0 += PF_QPOS) w += pf_tiles(t0, t, sk, P.window);
            vt.work[s] = w;
        }
        __syncthreads();
        for (int s = threadIdx.x; s < ns; s += blockDim.x) {
            const int ws = vt.work[s];
            int rank = 0;
            for (int s2 = 0; s2 < ns; ++s2) {
                const int w2 = vt.work[s2];
                rank += (w2 > ws) || (w2 == ws && s2 < s);
            }
            vt.order[rank] = s;
        }
        __syncthreads();
        for (int r = threadIdx.x; r < ns; r += blockDim.x) {
            const int s = vt.order[r];
            int qb, t;
            pf_seq_rows(P.cu_q, s, P.total_q, &qb, &t);
            vt.cum[r] = P.Hkv * ((t + CG * PF_QPOS - 1) / (CG * PF_QPOS));
        }
        __syncthreads();
        if (warp == 0) {  // exclusive scan, 32 entries at a time
            int carry = 0;
            for (int s0 = 0; s0 < ns; s0 += 32) {
                const int s = s0 + lane;
                const int x = (s < ns) ? vt.cum[s] : 0;
                int incl = x;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, incl, off);
                    if (lane >= off) incl += y;
                }
                if (s < ns) vt.cum[s] = carry + incl - x;
                carry += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (lane == 0) vt.cum[ns] = carry;
        }
    }
    if (warp == PF_WARP_MMA) {
        if constexpr (PAIR) {
            tmem_alloc_pair(tmem_holder, PF_TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(tmem_holder, PF_TMEM_COLS);
            tmem_relinquish();
        }
    }
    if (warp == PF_WARP_PRODUCER && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    tc_fence_before();
    // A pair: both CTAs' barriers are initialised before either CTA's copies,
    // arrivals or commits can reach the other.
    if constexpr (PAIR) {
        __syncwarp();
        cluster_sync_all();
    } else {
        __syncthreads();
    }
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    // G units run in parallel (CTAs, or CTA pairs); this CTA (pair) is `cta`.
    const int G = PAIR ? static_cast<int>(cluster_count_x()) : static_cast<int>(gridDim.x);
    const int cta = PAIR ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);
    const int rank = PAIR ? static_cast<int>(cluster_ctarank()) : 0;
    const bool leader = rank == 0;  // issues the UMMAs and owns the pair's shared barriers
    const int num_units = P.varlen ? min(P.num_units, vt.cum[P.num_seqs]) : P.num_units;
    const uint64_t lim = P.timeout_ns;
    // Cluster-window addresses of the even CTA's barriers that both CTAs of a
    // pair signal (data arrival, P ready, O read).
    const uint32_t l_q_full = PAIR ? mapa_shared(smem_u32(q_full), 0) : 0u;
    const uint32_t l_o_free = PAIR ? mapa_shared(smem_u32(o_free), 0) : 0u;
    // Units of this CTA (pair), round by round; -1 when there are no more.
    // Dense: the static zig-zag rounds. Packed sequences: the dynamic schedule
    // (the even CTA's producer takes each unit and publishes it; the other
    // roles of both CTAs read it from their ring in the same order).
    const bool dyn = P.varlen != 0;
    unsigned int* sched = g_pf_sched[grid_launch_id() % PF_SCHED_SLOTS];
    auto ring_addr = [&](int i) {
        return smem_u32(reinterpret_cast<const void*>(const_cast<const int*>(sq_ring + i)));
    };
    auto static_unit = [&](int r) -> int {
        if (r * G >= num_units) return -1;
        const int u = pf_sched(r, cta, G);
        return u < num_units ? u : -1;
    };
    auto take_unit = [&](int r, bool& ok) -> int {  // the even CTA's producer
        if (!dyn) return static_unit(r);
        const int i = r & 3;
        if (!mbar_wait(&sq_empty[i], ((r >> 2) & 1) ^ 1, abort_flag, lim, SITE_SCHED)) {
            ok = false;
            return -1;
        }
        const int u = static_cast<int>(atomicAdd(&sched[0], 1u));
        sq_ring[i] = u;
        if constexpr (PAIR) {
            st_shared_cluster_u32(mapa_shared(ring_addr(i), 1), static_cast<uint32_t>(u));
            mbar_arrive_release_cluster(mapa_shared(smem_u32(&sq_full[i]), 1));
        }
        mbar_arrive(&sq_full[i]);
        return u < num_units ? u : -1;
    };
    // `warp_wide`: every lane calls it, one arrival per warp
    auto read_unit = [&](int r, bool& ok, bool warp_wide) -> int {
        if (!dyn) return static_unit(r);
        const int i = r & 3;
        bool w = (PAIR && !leader)
                     ? mbar_wait_acquire_cluster(&sq_full[i], (r >> 2) & 1, abort_flag, lim,
                                                 SITE_SCHED)
                     : mbar_wait(&sq_full[i], (r >> 2) & 1, abort_flag, lim, SITE_SCHED);
        if (warp_wide) w = __all_sync(0xffffffffu, w);
        if (!w) {
            ok = false;
            return -1;
        }
        const int u = sq_ring[i];
        if (warp_wide) __syncwarp();
        if (!warp_wide || lane == 0) {
            if (PAIR && !leader)
                mbar_arrive_release_cluster(mapa_shared(smem_u32(&sq_empty[i]), 0));
            else
                mbar_arrive(&sq_empty[i]);
        }
        return u < num_units ? u : -1;
    };

    if (warp == PF_WARP_PRODUCER) {
        // ------------------------------------------------------------ producer
        // A pair: each CTA copies its own share into its own shared memory and
        // counts the bytes on the even CTA's barrier, which the even CTA's
        // producer arms for both shares. Empty barriers are local (the even
        // CTA's commits reach both CTAs).
        if (lane == 0) {
            uint32_t fill = 0;  // slot fills issued so far
            int unit_it = 0;
            int q_armed = 0;    // Q loads issued so far
            bool ok = true;
            for (int r = 0; ok; ++r) {
                const int u = leader ? take_unit(r, ok) : read_unit(r, ok, false);
                if (u < 0) break;
                PfUnit U;
                pf_unit<CG>(P, vt, u, U, rank);
                if (unit_it > 0) {
                    ok = mbar_wait(q_empty, (unit_it - 1) & 1, abort_flag, lim,
                                         SITE_PROD_Q_EMPTY);
                    if (!ok) break;
                }
                if (leader) mbar_arrive_expect_tx(q_full, CG * C::Q_BYTES);
                ++q_armed;
#pragma unroll
                for (int c = 0; c < D / 64; ++c) {
                    if constexpr (PAIR)
                        tma_load_3d_pair(sQ + c * 16384, &tmQ, l_q_full, c * 64, U.qbase + U.t0,
                                         2 * U.g);
                    else
                        tma_load_3d(sQ + c * 16384, &tmQ, q_full, c * 64, U.qbase + U.t0, 2 * U.g);
                }
                // Consumption order of the MMA warp: K0, K1, V0, K2, V1, ..., V(n-1).
                // Slot `slot` of a fill: wait until it is free, arm its barrier,
                // then copy `nbox` boxes of 64 d-columns.
                auto fill_slot = [&](const CUtensorMap* map, int nbox, int box_bytes, int col0,
                                     int row) -> bool {
                    const int slot = fill % C::NSLOT;
                    if (!mbar_wait(&slot_empty[slot], ((fill / C::NSLOT) & 1) ^ 1, abort_flag,
                                         lim, SITE_PROD_SLOT_EMPTY))
                        return false;
                    if (leader) mbar_arrive_expect_tx(&slot_full[slot], CG * C::SLOT_BYTES);
                    uint8_t* dst = sSlots + slot * C::SLOT_BYTES;
#pragma unroll
                    for (int b = 0; b < nbox; ++b) {
                        if constexpr (PAIR)
                            tma_load_3d_pair(dst + b * box_bytes, map,
                                             mapa_shared(smem_u32(&slot_full[slot]), 0),
                                             col0 + b * 64, row, U.g);
                        else
                            tma_load_3d(dst + b * box_bytes, map, &slot_full[slot], col0 + b * 64,
                                        row, U.g);
                    }
                    ++fill;
                    return true;
                };
                // K: this CTA's KROWS keys of the tile, KCOLS d-columns per slot
                auto load_k = [&](int key0) -> bool {
#pragma unroll
                    for (int s = 0; s < C::KSL; ++s)
                        if (!fill_slot(&tmK, C::KCOLS / 64, C::KROWS * 128, s * C::KCOLS,
                                       key0 + rank * C::KROWS))
                            return false;
                    return true;
                };
                // V: VROWS keys per slot, this CTA's VCOLS d-columns
                auto load_v = [&](int key0) -> bool {
#pragma unroll
                    for (int s = 0; s < C::VSL; ++s)
                        if (!fill_slot(&tmV, C::VCOLS / 64, C::VROWS * 128, rank * C::VCOLS,
                                       key0 + s * C::VROWS))
                            return false;
                    return true;
                };
                // Tile rows are looked up two tiles ahead (a paged cache reads
                // the block table), so the lookup overlaps the slot waits.
                int row0 = pf_key_row(P, U, U.kt0 * PF_BN);
                int row1 = (U.nkt > 1) ? pf_key_row(P, U, (U.kt0 + 1) * PF_BN) : 0;
                ok = load_k(row0);
                for (int jj = 0; ok && jj < U.nkt; ++jj) {
                    const int row2 =
                        (jj + 2 < U.nkt) ? pf_key_row(P, U, (U.kt0 + jj + 2) * PF_BN) : 0;
                    if (jj + 1 < U.nkt) ok = load_k(row1);
                    if (ok) ok = load_v(row0);
                    row0 = row1;
                    row1 = row2;
                }
                ++unit_it;
            }
            // Drain: every copy issued lands before the CTA exits. The full
            // barriers of a pair live in the even CTA and count both CTAs'
            // copies; the odd CTA's copies are drained there, before the
            // cluster barrier at the end of the kernel.
            if (leader) {
                const uint32_t last = fill < (uint32_t)C::NSLOT ? fill : (uint32_t)C::NSLOT;
                for (uint32_t i = 0; i < last; ++i) {
                    const uint32_t f = fill - 1 - i;
                    mbar_wait_drain(&slot_full[f % C::NSLOT], (f / C::NSLOT) & 1, lim);
                }
                if (q_armed > 0) mbar_wait_drain(q_full, (q_armed - 1) & 1, lim);
            }
            if constexpr (PAIR) {
                // The even CTA's commits reach this CTA's empty barriers: wait
                // for the last of them so none lands after the pair has left.
                const uint32_t last = fill < (uint32_t)C::NSLOT ? fill : (uint32_t)C::NSLOT;
                for (uint32_t i = 0; i < last; ++i) {
                    const uint32_t f = fill - 1 - i;
                    mbar_wait_drain(&slot_empty[f % C::NSLOT], (f / C::NSLOT) & 1, lim);
                }
                if (q_armed > 0) mbar_wait_drain(q_empty, (q_armed - 1) & 1, lim);
            }
        }
        __syncwarp();
    } else if (warp == PF_WARP_MMA) {
        // ------------------------------------------------------------ UMMA issuer
        // In a pair the even CTA issues for both (M = 256: its 128 rows, then
        // the odd CTA's); the odd CTA's issuer warp only holds the allocation.
        if (lane == 0 && leader) {
            constexpr uint32_t IDESC_S = idesc_bf16(PF_BM * CG, PF_BN, false);
            constexpr uint32_t IDESC_O = idesc_bf16(PF_BM * CG, D, true);
            constexpr uint32_t HI = sdesc_hi(1024);  // SBO 1024 B (8 rows x 128 B)
            // Q (A of S = Q K^T): K-major, 64-column chunks of 16 KB, k-step = 32 B
            const uint32_t q_lo = sdesc_lo(smem_u32(sQ), 16);
            // ring slot s: K-major K (LBO unused) or MN-major V (LBO = VROWS*128 B);
            // a pair's descriptors address the same offsets in both CTAs
            const uint32_t slot_lo0 = sdesc_lo(smem_u32(sSlots), 16);
            const uint32_t slot_lo0_v = sdesc_lo(smem_u32(sSlots), C::VROWS * 128);
            constexpr uint32_t SLOT_STEP = C::SLOT_BYTES >> 4;
            int slot = 0;          // ring position and phase (fills consumed so far)
            uint32_t phase = 0;
            uint32_t tile = 0;     // KV tiles processed by this CTA (S/P/PV index)
            int unit_it = 0;
            bool ok = true;

            // completion of the UMMAs issued so far (both CTAs' barriers for a pair)
            auto commit = [&](uint64_t* bar) {
                if constexpr (PAIR) umma_commit_pair(bar); else umma_commit(bar);
            };
            auto issue_s = [&](uint32_t gt) -> bool {
                const uint32_t buf = gt & 1;
                // S(gt) overwrites P(gt-2) in the same TMEM columns. PV(gt-2) was
                // issued earlier by this thread, and UMMAs issued by one thread
                // execute in issue order, so no completion wait is needed here.
                const uint32_t d_tmem = tmem + PF_S_COL0 + buf * PF_BN;
#pragma unroll
                for (int s = 0; s < C::KSL; ++s) {
                    if (!mbar_wait(&slot_full[slot], phase, abort_flag, lim,
                                         SITE_MMA_SLOT_FULL))
                        return false;
                    tc_fence_after();
                    const uint32_t k_lo = slot_lo0 + slot * SLOT_STEP;
#pragma unroll
                    for (int kk = 0; kk < C::KCOLS / 16; ++kk) {
                        const int dcol = s * C::KCOLS + kk * 16;  // Q column of this k-step
                        const uint32_t a_lo = q_lo + (dcol / 64) * (16384 >> 4) + ((dcol % 64) / 16) * 2;
                        const uint32_t b_lo = k_lo + (kk / 4) * ((C::KROWS * 128) >> 4) + (kk % 4) * 2;
                        if constexpr (PAIR)
                            umma_ss_lh_pair(d_tmem, a_lo, b_lo, HI, IDESC_S, (s | kk) != 0);
                        else
                            umma_ss_lh(d_tmem, a_lo, b_lo, HI, IDESC_S, (s | kk) != 0);
                    }
                    commit(&slot_empty[slot]);
                    if (++slot == C::NSLOT) { slot = 0; phase ^= 1u; }
                }
                commit(&s_full[buf]);
                return true;
            };
            auto issue_pv = [&](uint32_t gt, bool first) -> bool {
                const uint32_t buf = gt & 1;
                const uint32_t p_tmem = tmem + PF_S_COL0 + buf * PF_BN;
#pragma unroll
                for (int s = 0; s < C::VSL; ++s) {
                    if (!mbar_wait(&slot_full[slot], phase, abort_flag, lim,
                                         SITE_MMA_SLOT_FULL))
                        return false;
                    tc_fence_after();
                    const uint32_t v_lo = slot_lo0_v + slot * SLOT_STEP;
#pragma unroll
                    for (int kk = 0; kk < C::VROWS / 16; ++kk) {
                        // key kc of the tile: its P pair in the column part kc/HC,
                        // at column part*HC + (kc % HC)/2
                        const int kc = s * C::VROWS + kk * 16;
                        const uint32_t a = p_tmem + (kc / PF_PHC) * PF_PHC + (kc % PF_PHC) / 2;
                        const uint32_t acc = (first && s == 0 && kk == 0) ? 0u : 1u;
                        if constexpr (PAIR)
                            umma_ts_lh_pair(tmem, a, v_lo + kk * ((16 * 128) >> 4), HI, IDESC_O, acc);
                        else
                            umma_ts_lh(tmem, a, v_lo + kk * ((16 * 128) >> 4), HI, IDESC_O, acc);
                    }
                    commit(&slot_empty[slot]);
                    if (++slot == C::NSLOT) { slot = 0; phase ^= 1u; }
                }
                commit(&o_done[buf]);
                return true;
            };

            for (int r = 0; ok; ++r) {
                const int u = read_unit(r, ok, false);
                if (u < 0) break;
                PfUnit U;
                pf_unit<CG>(P, vt, u, U, rank);
                ok = mbar_wait(q_full, unit_it & 1, abort_flag, lim, SITE_MMA_Q_FULL);
                if (!ok) break;
                tc_fence_after();
                ok = issue_s(tile);
                for (int jj = 0; ok && jj < U.nkt; ++jj) {
                    const uint32_t gt = tile + jj;
                    if (jj + 1 < U.nkt) {
                        ok = issue_s(gt + 1);
                        if (!ok) break;
                    } else {
                        commit(q_empty);  // last S of the unit issued: Q reusable
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
                if (!ok) break;
                commit(o_last);  // the unit's last PV issued
                tile += U.nkt;
                ++unit_it;
            }
            // Drain: all issued UMMAs complete before TMEM is released (a
            // pair: signalled in this CTA only, never into the other CTA
            // after it may have left).
            if constexpr (PAIR) umma_commit_pair_local(drain); else umma_commit(drain);
            mbar_wait_drain(drain, 0, lim);
        }
        __syncwarp();
    } else if (warp < PF_WARP_PRODUCER) {
        // ------------------------------------------------------------ softmax
        constexpr int HC = PF_PHC;                      // key columns per part
        static_assert(HC % 32 == 0 && (D / PF_NSPLIT) % 16 == 0, "softmax split");
        constexpr int OC = D / PF_NSPLIT;               // O columns per part
        constexpr int EC = OC >= 64 ? 64 : OC;          // O columns per TMEM round trip
        static_assert(OC % EC == 0 && EC % 32 == 0, "O chunks");
        const int qd = warp & 3;                        // TMEM lane quadrant
        const int part = warp >> 2;                     // column part of this warp
        const int r = (qd << 5) | lane;                 // MMA row == TMEM lane
        const uint32_t lane_addr = static_cast<uint32_t>(qd * 32) << 16;
        const int pr = r & 63;                          // position within the tile
        const int col0 = part * HC;                     // first S column of this warp
        // s2 = x * (b0 + b1 x^2 + b2 x^4 + b3 x^6) with b_k = alpha*log2(e)*c_k*(alpha/C)^(2k):
        // the tanh series through u^7 in u = x*alpha/C (|u| <= 1/4: truncation
        // below 3.3e-7 relative), in powers of the raw accumulator x and scaled
        // into log2 units.
        const float us2 = P.u_scale * P.u_scale;
        const float b0 = P.scale_l2, b1 = P.scale_l2 * kTanhC1 * us2,
                    b2 = P.scale_l2 * kTanhC2 * us2 * us2, b3 = P.scale_l2 * kTanhC3 * us2 * us2 * us2;
        auto series_s2 = [&](float x) {
            const float x2 = x * x;
            float q = fmaf(x2, b3, b2);
            q = fmaf(x2, q, b1);
            q = fmaf(x2, q, b0);
            return x * q;
        };
        uint32_t tile = 0;
        int unit_it = 0;
        bool ok = true;
        for (int rr = 0; ok; ++rr) {
            const int u = read_unit(rr, ok, true);
            if (u < 0) break;
            PfUnit U;
            pf_unit<CG>(P, vt, u, U, rank);
            const int p = U.p_min + pr;  // absolute query position of this row
            float m_ref = -INFINITY;     // log2-domain reference max of the row
            float l = 0.f;               // this part's sum of fp32 weights (for lse)
            float lr = 0.f;              // this part's sum of bf16-rounded weights
            for (int jj = 0; jj < U.nkt; ++jj) {
                const uint32_t gt = tile + jj;
                const uint32_t buf = gt & 1;
                ok = mbar_wait(&s_full[buf], (gt >> 1) & 1, abort_flag, lim, SITE_SM_S_FULL);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after();
                const uint32_t s_addr = tmem + lane_addr + PF_S_COL0 + buf * PF_BN;
                float s[HC];
                {  // HC/32 TMEM loads in flight, one wait
                    uint32_t v[HC / 32][32];
#pragma unroll
                    for (int c = 0; c < HC / 32; ++c) tmem_ld32_async(s_addr + col0 + 32 * c, v[c]);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < HC / 32; ++c) tmem_reg_fence(v[c]);
#pragma unroll
                    for (int i = 0; i < HC; ++i) s[i] = __uint_as_float(v[i / 32][i % 32]);
                }
                const int j0 = (U.kt0 + jj) * PF_BN;  // key position of column 0
                const bool boundary =
                    (j0 + PF_BN - 1 > U.p_min) || (P.window > 0 && j0 < U.p_max - P.window + 1);
                // Raw accumulator range of this warp's columns (the running max
                // needs the tile max; with the fixed shift only max |x| is
                // needed, for the series check).
                constexpr bool FIX = SM == PF_SM_FIXED;
                constexpr bool cap = SM != PF_SM_NOCAP;
                float amx, amn;
                if constexpr (FIX) {
                    float ma[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) ma[k] = fabsf(s[k]);
#pragma unroll
                    for (int i = 4; i < HC; i += 2)
                        ma[(i >> 1) & 3] = fmax3f(ma[(i >> 1) & 3], fabsf(s[i]), fabsf(s[i + 1]));
                    amx = fmaxf(fmaxf(ma[0], ma[1]), fmaxf(ma[2], ma[3]));
                    amn = -amx;
                } else {
                    float mxa[4], mna[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) mxa[k] = mna[k] = s[k];
#pragma unroll
                    for (int i = 4; i < HC; i += 2) {
                        mxa[(i >> 1) & 3] = fmax3f(mxa[(i >> 1) & 3], s[i], s[i + 1]);
                        mna[(i >> 1) & 3] = fmin3f(mna[(i >> 1) & 3], s[i], s[i + 1]);
                    }
                    amx = fmaxf(fmaxf(mxa[0], mxa[1]), fmaxf(mxa[2], mxa[3]));
                    amn = fminf(fminf(mna[0], mna[1]), fminf(mna[2], mna[3]));
                }
                // Fast path: no mask in this tile, cap on, |x/C| <= 1/4 for the
                // whole warp. The capped map is monotonic in x, so the tile max
                // is the map of the extreme accumulators and s2 - m fuses into
                // one packed FMA below.
                // Without the cap the map is the plain scale: the same fused path.
                const bool fast = __all_sync(
                    0xffffffffu, !boundary && (!cap ||
                                               fmaxf(fabsf(amx), fabsf(amn)) <= P.poly_acc_max));
                float mt = 0.f;
                if (fast) {
                    if constexpr (!FIX)
                        mt = cap ? fmaxf(series_s2(amx), series_s2(amn))
                                 : fmaxf(amx * P.scale_l2, amn * P.scale_l2);
                } else if constexpr (!FIX) {
                    // general path: capped logits in log2 units, then the mask
                    // (the fixed shift's general path is out of line, below)
                    if constexpr (cap) {
                        if (__all_sync(0xffffffffu,
                                       fmaxf(fabsf(amx), fabsf(amn)) <= P.poly_acc_max)) {
#pragma unroll
                            for (int i = 0; i < HC; ++i) s[i] = series_s2(s[i]);
                        } else {
#pragma unroll
                            for (int i = 0; i < HC; ++i) {
                                const float e = ex2_approx(s[i] * P.k_exp);
                                const float rc = rcp_approx(1.0f + e);
                                s[i] = fmaf(-2.0f * P.cap_l2, rc, P.cap_l2);
                            }
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < HC; ++i) s[i] *= P.scale_l2;
                    }
                    if (boundary) {
                        const int hi = p - j0 - col0;  // visible local columns: [lo, hi]
                        const int lo = P.window > 0 ? p - P.window + 1 - j0 - col0 : -1;
#pragma unroll
                        for (int i = 0; i < HC; ++i)
                            if (i > hi || i < lo) s[i] = -INFINITY;
                    }
                    if constexpr (!FIX) {
                        float mx[4];
#pragma unroll
                        for (int k = 0; k < 4; ++k) mx[k] = s[k];
#pragma unroll
                        for (int i = 4; i < HC; i += 2)
                            mx[(i >> 1) & 3] = fmax3f(mx[(i >> 1) & 3], s[i], s[i + 1]);
                        mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
                    }
                }
                if constexpr (FIX) {
                    // fixed shift: no running max, no exchange, no rescaling
                    m_ref = P.fixed_ref;
                } else {
                    // row max over all parts
                    xmax[(buf * PF_NSPLIT + part) * 128 + r] = mt;
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&xbar[qd * 2 + buf]);  // release for the warp
                    ok = mbar_wait(&xbar[qd * 2 + buf], (gt >> 1) & 1, abort_flag, lim,
                                   SITE_SM_PAIR);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
#pragma unroll
                    for (int k = 0; k < PF_NSPLIT; ++k)
                        mt = fmaxf(mt, xmax[(buf * PF_NSPLIT + k) * 128 + r]);
                    const float m_new = fmaxf(m_ref, mt);
                    const bool need = (m_ref != -INFINITY) && (m_new > m_ref + PF_RESCALE_LOG2);
                    if (__any_sync(0xffffffffu, need)) {
                        // O holds PV(0..gt-1) relative to m_ref: scale this part to m_new.
                        ok = mbar_wait(&o_done[(gt - 1) & 1], ((gt - 1) >> 1) & 1, abort_flag,
                                             lim, SITE_SM_O_DONE);
                        ok = __all_sync(0xffffffffu, ok);
                        if (!ok) break;
                        tc_fence_after();
                        const float f = need ? ex2_approx(m_ref - m_new) : 1.0f;
                        const uint32_t o_addr = tmem + lane_addr + part * OC;
#pragma unroll 1
                        for (int c = 0; c < OC / 32; ++c) {  // 32 columns per TMEM round trip
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
                }  // running max
                const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
                // The PV product sees bf16(p); normalising O by the sum of the
                // same rounded weights makes them sum to one exactly, so their
                // rounding errors cancel against the row's mean value.
                const float2 mneg = make_float2(-m_use, -m_use);
                if (FIX && !fast) {
                    // the band's edges or logits past the series range
                    const int hi = boundary ? p - j0 - col0 : HC;  // visible local columns
                    const int lo = (boundary && P.window > 0) ? p - P.window + 1 - j0 - col0 : -1;
                    const bool series = __all_sync(
                        0xffffffffu, fmaxf(fabsf(amx), fabsf(amn)) <= P.poly_acc_max);
                    const float4 r4 = pf_softmax_general_fixed(s_addr + col0, lo, hi, series, b0,
                                                               b1, b2, b3, P.k_exp, P.cap_l2,
                                                               m_use);
                    l += r4.x + r4.y;
                    lr += r4.z + r4.w;
                } else {
                    float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                    float2 lrs[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                    uint32_t pk[HC / 2];
                    if (!cap && fast) {
                        const float2 B0 = make_float2(b0, b0);
#pragma unroll
                        for (int i = 0; i < HC / 2; ++i) {
                            const float2 x = fma2(make_float2(s[2 * i], s[2 * i + 1]), B0, mneg);
                            const float2 e = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                            ls[i & 1] = add2(ls[i & 1], e);
                            pk[i] = pack_bf16x2(e.x, e.y);
                            lrs[i & 1] = add_bf16x2_f32(lrs[i & 1], pk[i]);
                        }
                    } else if (fast) {
                        const float2 B0 = make_float2(b0, b0), B1 = make_float2(b1, b1);
                        const float2 B2 = make_float2(b2, b2), B3 = make_float2(b3, b3);
#pragma unroll
                        for (int i = 0; i < HC / 2; ++i) {
                            const float2 a = make_float2(s[2 * i], s[2 * i + 1]);
                            const float2 x2 = mul2(a, a);
                            float2 q = fma2(x2, B3, B2);
                            q = fma2(x2, q, B1);
                            q = fma2(x2, q, B0);
                            const float2 x = fma2(a, q, mneg);  // s2 - m
                            const float2 e = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                            ls[i & 1] = add2(ls[i & 1], e);
                            pk[i] = pack_bf16x2(e.x, e.y);
                            lrs[i & 1] = add_bf16x2_f32(lrs[i & 1], pk[i]);
                        }
                    } else if constexpr (!FIX) {
#pragma unroll
                        for (int i = 0; i < HC / 2; ++i) {
                            const float2 x = add2(make_float2(s[2 * i], s[2 * i + 1]), mneg);
                            const float2 e = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                            ls[i & 1] = add2(ls[i & 1], e);
                            pk[i] = pack_bf16x2(e.x, e.y);
                            lrs[i & 1] = add_bf16x2_f32(lrs[i & 1], pk[i]);
                        }
                    }
                    // P of this part's HC keys as bf16 pairs: HC/2 columns at the
                    // start of its own S columns, which it has already read (the
                    // other part's S columns may still be unread)
#pragma unroll
                    for (int c = 0; c < HC / 32; ++c) {
                        uint32_t pc[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) pc[i] = pk[16 * c + i];
                        tmem_st16(s_addr + part * HC + 16 * c, pc);
                    }
                    const float2 lsum = add2(ls[0], ls[1]);
                    const float2 lrsum = add2(lrs[0], lrs[1]);
                    l += lsum.x + lsum.y;
                    lr += lrsum.x + lrsum.y;
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if constexpr (PAIR)
                        mbar_arrive_cluster(mapa_shared(smem_u32(&p_full[buf]), 0));
                    else
                        mbar_arrive(&p_full[buf]);
                }
            }
            if (!ok) break;
            // ---- hand the row statistics to the epilogue warps
            const int sb = unit_it & 1;
            xsum[((sb * PF_NSPLIT + part) * 128 + r) * 2 + 0] = l;
            xsum[((sb * PF_NSPLIT + part) * 128 + r) * 2 + 1] = lr;
            if (part == 0) xref[sb * 128 + r] = m_ref;
            __syncwarp();
            if (lane == 0) mbar_arrive(&stat_full[sb]);
            tile += U.nkt;
            ++unit_it;
        }
    } else if (warp >= PF_WARP_EPI) {
        // ------------------------------------------------------------ epilogue
        // O / lr -> bf16 and lse of each unit, one row (TMEM lane) per thread,
        // all D columns. lr sums the bf16-rounded weights that PV used, so the
        // weights of a row sum to one exactly; l (fp32 weights) gives the lse.
        constexpr int EC = 64;                          // O columns per TMEM round trip
        static_assert(D % EC == 0, "epilogue chunks");
        const int qd = warp & 3;                        // TMEM lane quadrant
        const int r = (qd << 5) | lane;                 // MMA row == TMEM lane
        const uint32_t lane_addr = static_cast<uint32_t>(qd * 32) << 16;
        const int hl = r >> 6;                          // head within the pair
        const int pr = r & 63;                          // position within the tile
        uint32_t tile = 0;
        int unit_it = 0;
        bool ok = true;
        for (int rr = 0; ok; ++rr) {
            const int u = read_unit(rr, ok, true);
            if (u < 0) break;
            PfUnit U;
            pf_unit<CG>(P, vt, u, U, rank);
            // PV(gl) completing implies every earlier UMMA of this CTA completed.
            // o_last first (at most one unit ahead: the next unit's first PV
            // waits for this epilogue), then the unit's last o_done phase, so
            // that its arrival has landed before this CTA can leave.
            const uint32_t gl = tile + U.nkt - 1;
            const int sb = unit_it & 1;
            ok = mbar_wait(o_last, unit_it & 1, abort_flag, lim, SITE_EPI_O_DONE);
            if (ok)
                ok = mbar_wait(&o_done[gl & 1], (gl >> 1) & 1, abort_flag, lim,
                               SITE_EPI_O_DONE);
            if (ok)
                ok = mbar_wait(&stat_full[sb], (unit_it >> 1) & 1, abort_flag, lim,
                               SITE_EPI_STATS);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            float l = 0.f, lr = 0.f;
#pragma unroll
            for (int k = 0; k < PF_NSPLIT; ++k) {
                l += xsum[((sb * PF_NSPLIT + k) * 128 + r) * 2 + 0];
                lr += xsum[((sb * PF_NSPLIT + k) * 128 + r) * 2 + 1];
            }
            const float m_ref = xref[sb * 128 + r];
            const float inv_l = 1.0f / lr;
            const uint32_t o_addr = tmem + lane_addr;
            // destination of warp row rw (TMEM lane 32 qd + rw), O column col
            auto row_ptr = [&](int rw, int col) -> __nv_bfloat16* {
                const int rq = (qd << 5) | rw;
                const int prr = rq & 63;
                if (prr >= U.tvalid) return nullptr;
                return P.out + (static_cast<size_t>(U.qbase + U.t0 + prr) * P.H + 2 * U.g +
                                (rq >> 6)) * D + col;
            };
#pragma unroll 1
            for (int c = 0; c < D / EC; ++c) {
                uint32_t v[EC / 32][32];
#pragma unroll
                for (int j = 0; j < EC / 32; ++j) tmem_ld32_async(o_addr + c * EC + 32 * j, v[j]);
                tmem_wait_ld();
                uint32_t w[EC / 2];
#pragma unroll
                for (int j = 0; j < EC / 32; ++j) {
                    tmem_reg_fence(v[j]);
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        w[16 * j + i] = pack_bf16x2(__uint_as_float(v[j][2 * i]) * inv_l,
                                                    __uint_as_float(v[j][2 * i + 1]) * inv_l);
                }
                pf_store_rows<EC>(w, lane, [&](int rw) { return row_ptr(rw, c * EC); });
            }
            if (pr < U.tvalid && P.lse != nullptr) {
                const int h = 2 * U.g + hl;
                const float lse = (m_ref + log2f(l)) * 0.69314718055994531f;
                size_t li;
                if (P.varlen)
                    li = static_cast<size_t>(h) * P.total_q + U.qbase + U.t0 + pr;
                else
                    li = (static_cast<size_t>(U.seq) * P.H + h) * P.T + U.t0 + pr;
                P.lse[li] = lse;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if constexpr (PAIR) mbar_arrive_cluster(l_o_free); else mbar_arrive(o_free);
            }
            tile += U.nkt;
            ++unit_it;
        }
    }

    tc_fence_before();
    // A pair leaves together: no copy, arrival or UMMA of one CTA may still
    // reach the other's shared or tensor memory after this barrier.
    if constexpr (PAIR) {
        __syncwarp();
        cluster_sync_all();
    } else {
        __syncthreads();
    }
    if (warp == PF_WARP_MMA) {
        tc_fence_after();
        if constexpr (PAIR) tmem_dealloc_pair(tmem, PF_TMEM_COLS);
        else tmem_dealloc(tmem, PF_TMEM_COLS);
    }
    // dynamic schedule: every unit of this launch was taken (each even CTA's
    // producer took one past the last before the barrier above); the last CTA
    // to get here zeroes the slot
    if (dyn && threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(&sched[1], 1u) == gridDim.x - 1) {
            atomicExch(&sched[0], 0u);
            atomicExch(&sched[1], 0u);
        }
    }
}

}  // namespace g2
