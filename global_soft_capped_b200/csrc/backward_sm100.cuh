// backward_sm100.cuh -- gradients of the soft-capped local/global attention
// layer on sm_100a (tcgen05 UMMA + TMA), for head sizes d = 64, 128 and 256.
//
// Chain rule through the layer (Gemma 2 card, "Method", per-layer attention
// pseudo-code; derivative of the soft-cap from the "Gemma 2 Guide", Deep Dive
// item 1: d/dx C tanh(x/C) = 1 - tanh^2(x/C)). With x the scaled logit
// (query_scale q.k), s = C tanh(x/C) its capped value, P the softmax weights
// recomputed from the forward's log-sum-exp, and D_i = dout_i . out_i:
//   dP_ij = dout_i . v_j
//   dS_ij = P_ij (dP_ij - D_i) (1 - (s_ij / C)^2)         (no cap: the last factor is 1)
//   dv_j  = sum_i P_ij dout_i,  dk_j = query_scale sum_i dS_ij q_i,
//   dq_i  = query_scale sum_j dS_ij k_j
// summing dk, dv over the two query heads that share a KV head.
//
// Three launches:
//   bwd_prep      D_i and lse_i * log2(e), per (b, h, position), into the
//                 caller's workspace (positions padded to a multiple of 64)
//   bwd_sm100<D, BW_KV>  one unit = 128 keys of one KV head: K and V stay in
//                 shared memory, the query tiles (CQ positions of both heads
//                 of the group: 2 CQ rows) stream through. X = K Q^T (S^T) and
//                 Y = V dout^T (dP^T) land in TMEM with one key per lane, so
//                 P^T and dS^T are written back as bf16 and used directly as
//                 the A operand of dv += P^T dout and dk += dS^T q.
//   bwd_sm100<D, BW_Q>   one unit = 64 query positions x 2 heads: q and dout
//                 stay, the CK-key tiles stream; X = q K^T, Y = dout V^T,
//                 dq += dS K.
// Column tiles are 64 rows (BwCfg): 32 positions x 2 heads, or 64 keys.
// TMEM (512 columns), d <= 128: accumulators at 0..2d-1; X and Y double-
// buffered, buffer b at 256 + 128 b (X) and 320 + 128 b (Y), so that the X / Y
// of the next column tiles run while the elementwise warps work on this one.
// d = 256: one 256-column accumulator at 0, one resident operand held in TMEM
// at 256..383 (read by the UMMAs as their A operand, so its bytes never cross
// shared memory again), X at 384 and Y at 448. The dk/dv kernel then runs
// each key tile as two units, a dv unit (X only: K in TMEM; dv += P^T dout)
// and a dk unit (X with K in shared memory, Y with V in TMEM; dk += dS^T q);
// the dq kernel keeps q in TMEM and dout in shared memory.
#pragma once

#include "common.cuh"

namespace g2 {

constexpr int BW_KV = 0;
constexpr int BW_Q = 1;
// Elementwise warps: BW_NPART column parts x 4 TMEM lane quadrants. Their
// per-tile work is bound by instruction issue, not latency: four parts (16
// warps) measured 5% slower than two at d = 128 and d = 256.
constexpr int BW_NPART = 2;
constexpr int BW_EW_WARPS = 4 * BW_NPART;
constexpr int BW_EW_THREADS = 32 * BW_EW_WARPS;
constexpr int BW_WARP_PRODUCER = BW_EW_WARPS;
constexpr int BW_WARP_MMA = BW_EW_WARPS + 1;   // issuer 0: X and the accumulation reading X; TMEM owner
constexpr int BW_WARP_MMA2 = BW_EW_WARPS + 2;  // issuer 1: Y and the accumulation reading Y
constexpr int BW_THREADS = 32 * (BW_EW_WARPS + 3);  // elementwise warps, producer, 2 UMMA issuers
constexpr int BW_QPOS = 64;              // query positions per column/row tile (x 2 heads)
constexpr int BW_KEYS = 128;             // keys per tile
constexpr int BW_X_COL = 256;
constexpr int BW_Y_COL = 384;
constexpr uint32_t BW_TMEM_COLS = 512;

// Tile shapes per head size. The resident (row) tiles are always 128 rows:
// 128 keys (KV mode) or 64 positions x 2 heads (Q mode). The streamed column
// tiles are CR = 64 rows: CQ = 32 positions x 2 heads (KV) or CK = 64 keys
// (Q), split into BW_NPART parts of HW columns, one per column part of the
// elementwise warps. X and Y are whole-tile N = 64 UMMAs issued by two
// threads: one thread issues a tcgen05.mma only about every 67 cycles, which
// is more than the math of an M = 128, N = 64, K = 16 product (32 cycles).
// d <= 128: K and V (or q and dout) stay in shared memory, four slots of
// column tiles stream, and X / Y are double-buffered in TMEM. d = 256: one
// resident operand lives in TMEM (see the file header), two slots stream (dv
// units: three, the third in the resident region), and the dk/dv kernel
// splits each key tile into a dv and a dk unit (DSPLIT) so that its
// accumulator fits TMEM; only the dv units double-buffer X.
template <int D>
struct BwCfg {
    static_assert(D == 64 || D == 128 || D == 256, "backward kernels: d = 64, 128, 256");
    static constexpr bool A_TMEM = D == 256;
    static constexpr bool DB = !A_TMEM;                  // X / Y double-buffered for every unit
    static constexpr int CQ = 32;                        // KV column tile: positions per head
    static constexpr int CK = 64;                        // Q column tile: keys
    static constexpr int CR = 2 * CQ;                    // column tile rows (both modes)
    static_assert(CR == CK, "column tiles of both modes have CR rows");
    static constexpr int HW = CR / BW_NPART;             // columns per warp part
    static constexpr int CHUNK = HW < 32 ? HW : 32;      // columns per TMEM round trip
    static constexpr int DSPLIT_KV = D == 256 ? 2 : 1;   // dk/dv kernel: units per key tile
    static constexpr int RES_TILES = A_TMEM ? 1 : 2;     // resident tiles in shared memory
    static constexpr int ISSUERS = 2;                    // UMMA issuing threads
    static constexpr int NSLOT = A_TMEM ? 2 : 4;         // column-tile slots
    static constexpr int TILE_BYTES = 128 * D * 2;       // one 128-row resident tile
    static constexpr int CTILE_BYTES = CR * D * 2;       // one streamed column tile
    static constexpr int VEC_BYTES = 1024;               // -lse2, -D of the tile's query rows
    static constexpr int VEC_TX = 2 * CR * 4;            //   (bytes copied: CR rows, two arrays)
    static constexpr int SLOT_BYTES = 2 * CTILE_BYTES + VEC_BYTES;
    static_assert(SLOT_BYTES % 1024 == 0 && VEC_TX <= VEC_BYTES, "slot layout");
    // Layout, d <= 128: R1, R2, then the NSLOT slots. d = 256: the slots, then
    // the one resident tile in a slot-sized region, so that a dv unit (which
    // keeps nothing in shared memory) can stream through it as a third slot.
    static constexpr int RES_BYTES = A_TMEM ? SLOT_BYTES : RES_TILES * TILE_BYTES;
    static_assert(!A_TMEM || SLOT_BYTES >= TILE_BYTES, "resident region holds a slot");
    static constexpr int NRING_MAX = A_TMEM ? NSLOT + 1 : NSLOT;  // slots of the widest ring
    static_assert(NRING_MAX <= 4, "slot barriers");
    static constexpr int SMEM_TILES = NSLOT * SLOT_BYTES + RES_BYTES;
    // TMEM columns: accumulators at 0, the resident A operand (d = 256), X, Y
    static constexpr uint32_t A_COL = 256;
    static constexpr uint32_t X_COL = A_TMEM ? 384 : BW_X_COL;
    static constexpr uint32_t Y_COL = A_TMEM ? 448 : BW_Y_COL;
    // double buffers: X of buffer b at XB0 + XB_STEP b, Y (d <= 128) at YB0 + XB_STEP b
    // (d = 256 dv units: X alternates between the X and Y columns)
    static constexpr uint32_t XB0 = A_TMEM ? 384 : 256;
    static constexpr uint32_t YB0 = A_TMEM ? 448 : 320;
    static constexpr uint32_t XB_STEP = A_TMEM ? 64 : 128;
    static_assert(!A_TMEM || (X_COL + CR <= Y_COL && Y_COL + CR <= BW_TMEM_COLS), "TMEM columns");
    static_assert(A_TMEM || (2 * D <= XB0 && YB0 + XB_STEP + CR <= BW_TMEM_COLS),
                  "TMEM columns (double-buffered X / Y)");
    static constexpr int MAX_SEQ_TABLE = 1024;                  // varlen: sequences per launch
    // varlen: per-sequence work, sequences ranked by it, unit prefix in rank order
    static constexpr int VL_BYTES = 4 * (3 * MAX_SEQ_TABLE + 1);
    static constexpr int SMEM_BYTES = 1024 + SMEM_TILES + 1024 + VL_BYTES;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

struct BwParams {
    __nv_bfloat16* dq;
    __nv_bfloat16* dk;
    __nv_bfloat16* dv;
    // inputs, read directly by the elementwise warps when a resident tile
    // goes to TMEM (d = 256)
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    // -lse * log2(e) and -D = -(dout . out) per (head, query position), with
    // each sequence's positions padded to whole 64-position tiles (-inf / 0):
    // dense (B, H, Tp); varlen (H, Wmax), sequence s at columns wq[s] ..
    const float* nlse2;
    const float* ndvec;
    int B, T, S, H, Hkv, Tp;
    int q_offset, window;
    // varlen (packed sequences): T_s, S_s from cu_q / cu_k, q_offset_s = S_s - T_s
    const int* cu_q;
    const int* cu_k;
    const int* wq;  // [num_seqs + 1] padded prefix of T_s (workspace columns)
    int num_seqs, varlen, wmax;
    int total_q, total_k;  // packed extents: sequence rows are clamped into them
    int num_units;
    int row_tiles;      // KV: key tiles per (b, g); Q: query tiles per (b, g)
    float k_exp;        // 2 alpha log2(e) / C   (cap on)
    float cap_l2;       // C log2(e)             (cap on)
    float scale_l2;     // alpha log2(e)
    float query_scale;
    float u_scale;       // alpha / C              (cap on)
    float th_c[4];       // series of tanh(alpha x / C) in x: (alpha/C)^(2k+1) c_k (cap on)
    float poly_acc_max;  // largest |q.k| with |alpha q.k / C| <= 1/4 (0: series off)
    int has_cap;
    unsigned long long timeout_ns;
    // Unit counter of this launch in the caller's workspace, zeroed by the
    // pass that runs before it: the CTAs take units in order from it (a
    // dynamic list schedule, longest units first). nullptr: the static
    // zig-zag schedule.
    unsigned int* sched;
};

// tanh(u) for |u| <= 1/4: Taylor series through u^7 (coefficients -1/3, 2/15,
// -17/315; truncation below 3.3e-7 relative), on the FMA pipe.
__device__ __forceinline__ float bw_tanh_series(float u) {
    const float u2 = u * u;
    float q = fmaf(u2, -17.0f / 315.0f, 2.0f / 15.0f);
    q = fmaf(u2, q, -1.0f / 3.0f);
    q = fmaf(u2, q, 1.0f);
    return u * q;
}

template <bool B>
struct BwMask {
    static constexpr bool value = B;
};

struct BwUnit {
    int g;
    int dh;           // dk/dv kernel at d = 256: 0 = dv unit, 1 = dk unit; 0 otherwise
    int T, S, qoff;   // the sequence: queries, keys, position of query 0
    int qbase, kbase; // packed row of its first query / key
    long long wbase;  // workspace column of its position 0 for head 0 ...
    long long wstride;  // ... and the stride between heads
    int row0;     // KV: first key; Q: first query position (row index t within the sequence)
    int rvalid;   // KV: keys in the tile (<= 128); Q: positions in the tile (<= 64)
    int col0;     // first column tile index (KV: CQ-position tiles; Q: CK-key tiles)
    int ncols;    // column tiles (0: no visible pair; KV units then store zeros)
};

// Rows [*base, *base + *len) of sequence s in a packed tensor of `total` rows
// described by cu[]: clamped into [0, total), so that malformed offsets can
// give wrong results but never an access outside the tensors.
__device__ __forceinline__ void bw_seq_rows(const int* cu, int s, int total, int* base,
                                            int* len) {
    const int b0 = min(max(cu[s], 0), total);
    const int b1 = min(max(cu[s + 1], b0), total);
    *base = b0;
    *len = b1 - b0;
}

// Row tile rt (of `tiles`) of a sequence with U.T queries at the end of U.S
// keys: its rows and the column tiles that hold a visible pair. KV: key tiles
// ascending (the earliest keys see the most queries); Q: query tiles
// descending (the latest queries see the most keys).
template <int D, int MODE>
__device__ __forceinline__ void bw_tile_cols(int rt, int tiles, int window, BwUnit& U) {
    constexpr int CQ = BwCfg<D>::CQ, CK = BwCfg<D>::CK;
    if (MODE == BW_KV) {
        U.row0 = rt * BW_KEYS;
        U.rvalid = min(BW_KEYS, U.S - U.row0);
        // query rows t whose position t + qoff sees a key of the tile
        const int t_lo = max(0, U.row0 - U.qoff);
        const int t_hi = window > 0 ? min(U.T - 1, U.row0 + BW_KEYS - 1 + window - 1 - U.qoff)
                                    : U.T - 1;
        U.col0 = t_lo / CQ;
        U.ncols = (t_lo <= t_hi) ? t_hi / CQ - U.col0 + 1 : 0;
    } else {
        const int qt = tiles - 1 - rt;
        U.row0 = qt * BW_QPOS;
        U.rvalid = min(BW_QPOS, U.T - U.row0);
        const int p_min = U.row0 + U.qoff, p_max = p_min + U.rvalid - 1;
        const int j_lo = window > 0 ? max(0, p_min - window + 1) : 0;
        const int j_hi = min(p_max, U.S - 1);
        U.col0 = j_lo / CK;
        U.ncols = j_hi >= j_lo ? j_hi / CK - U.col0 + 1 : 0;
    }
}

template <int MODE>
__device__ __forceinline__ int bw_row_tiles(int T, int S) {
    return MODE == BW_KV ? (S + BW_KEYS - 1) / BW_KEYS : (T + BW_QPOS - 1) / BW_QPOS;
}

// Units. Dense: row tiles in the order of bw_tile_cols, then batch, then KV
// head. Varlen: sequence by sequence, heaviest first (`order`, with the unit
// prefix `cum` in that order), within a sequence as dense. The dv and dk
// units of a key tile (dk/dv kernel at d = 256) are consecutive units.
template <int D, int MODE>
__device__ __forceinline__ void bw_unit(const BwParams& P, const int* cum, const int* order,
                                        int u, BwUnit& U) {
    constexpr int DS = MODE == BW_KV ? BwCfg<D>::DSPLIT_KV : 1;
    U.dh = u % DS;
    u /= DS;
    int rt, tiles;
    if (!P.varlen) {
        const int BG = P.B * P.Hkv;
        rt = u / BG;
        const int rem = u % BG, b = rem / P.Hkv;
        U.g = rem % P.Hkv;
        U.T = P.T;
        U.S = P.S;
        U.qoff = P.q_offset;
        U.qbase = b * P.T;
        U.kbase = b * P.S;
        U.wbase = static_cast<long long>(b) * P.H * P.Tp;
        U.wstride = P.Tp;
        tiles = P.row_tiles;
    } else {
        int lo = 0, hi = P.num_seqs - 1;  // largest s with cum[s] <= u
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (cum[mid] <= u) lo = mid; else hi = mid - 1;
        }
        const int s = order[lo], lu = u - cum[lo];
        U.g = lu % P.Hkv;
        rt = lu / P.Hkv;
        bw_seq_rows(P.cu_q, s, P.total_q, &U.qbase, &U.T);
        bw_seq_rows(P.cu_k, s, P.total_k, &U.kbase, &U.S);
        U.qoff = U.S - U.T;
        U.wbase = P.wq[s];
        U.wstride = P.wmax;
        tiles = bw_row_tiles<MODE>(U.T, U.S);
    }
    bw_tile_cols<D, MODE>(rt, tiles, P.window, U);
}

// -D_i = -(dout_i . out_i) (fp32 sum of bf16 products) and -lse_i * log2(e),
// D/8 lanes of 16 bytes per (b, h, t); padding positions t in [T, Tp) get
// -lse2 = -inf (zero weight) and -D = 0. Both are stored negated so that the
// kernels add them with one packed FMA / ADD.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep(const __nv_bfloat16* __restrict__ out,
                                                const __nv_bfloat16* __restrict__ dout,
                                                const float* __restrict__ lse, float* nlse2,
                                                float* ndvec, int B, int T, int H, int Tp,
                                                unsigned int* sched) {
    // the gradient kernels' unit counters, for the launches that follow
    if (blockIdx.x == 0 && threadIdx.x < 2) sched[threadIdx.x] = 0u;
    constexpr int LPR = D / 8;  // lanes per row
    const long long row = (static_cast<long long>(blockIdx.x) * 256 + threadIdx.x) / LPR;
    const int sub = threadIdx.x % LPR;
    const long long nrows = static_cast<long long>(B) * H * Tp;
    const bool in_range = row < nrows;  // no early return: the whole warp shuffles below
    const int t = static_cast<int>(row % Tp);
    const long long bh = row / Tp;  // b * H + h
    const int h = static_cast<int>(bh % H);
    const long long b = bh / H;
    float acc = 0.f;
    if (in_range && t < T) {
        const size_t off = ((static_cast<size_t>(b) * T + t) * H + h) * D + sub * 8;
        const uint4 o = *reinterpret_cast<const uint4*>(out + off);
        const uint4 g = *reinterpret_cast<const uint4*>(dout + off);
        const uint32_t ow[4] = {o.x, o.y, o.z, o.w}, gw[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc = fmaf(__uint_as_float(ow[i] << 16), __uint_as_float(gw[i] << 16), acc);
            acc = fmaf(__uint_as_float(ow[i] & 0xFFFF0000u), __uint_as_float(gw[i] & 0xFFFF0000u),
                       acc);
        }
    }
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (in_range && sub == 0) {
        ndvec[row] = -acc;
        nlse2[row] = (t < T) ? lse[bh * T + t] * -1.4426950408889634f : -INFINITY;
    }
}

// Varlen: wq[s] = sum over s' < s of T_s' rounded up to 64 (the workspace
// column where sequence s starts), wq[num_seqs] = the total. One block.
__global__ void __launch_bounds__(32) bwd_wq_prefix(const int* __restrict__ cu_q, int num_seqs,
                                                    int total_q, int* wq, unsigned int* sched) {
    const int lane = threadIdx.x;
    // the gradient kernels' unit counters, for the launches that follow
    if (lane < 2) sched[lane] = 0u;
    int carry = 0;
    for (int s0 = 0; s0 < num_seqs; s0 += 32) {
        const int q = s0 + lane;
        int qb = 0, t = 0;
        if (q < num_seqs) bw_seq_rows(cu_q, q, total_q, &qb, &t);
        const int x = (t + 63) / 64 * 64;
        int incl = x;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        if (q < num_seqs) wq[q] = carry + incl - x;
        carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) wq[num_seqs] = carry;
}

// Varlen form of bwd_prep over workspace columns w in [0, wmax) of every head:
// sequence s owns columns wq[s] .. wq[s+1]-1 (its positions, then padding);
// lse is (H, total_q) packed. Columns past wq[num_seqs] are left untouched.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_varlen(
    const __nv_bfloat16* __restrict__ out, const __nv_bfloat16* __restrict__ dout,
    const float* __restrict__ lse, const int* __restrict__ cu_q, const int* __restrict__ wq,
    float* nlse2, float* ndvec, int num_seqs, int H, int total_q, int wmax) {
    constexpr int LPR = D / 8;  // lanes per row
    const long long row = (static_cast<long long>(blockIdx.x) * 256 + threadIdx.x) / LPR;
    const int sub = threadIdx.x % LPR;
    const long long nrows = static_cast<long long>(H) * wmax;
    const int w = static_cast<int>(row % wmax);
    const int h = static_cast<int>(row / wmax);
    const bool in_range = row < nrows && w < wq[num_seqs];  // whole warp shuffles below
    int s = 0;
    if (in_range) {  // largest s with wq[s] <= w
        int lo = 0, hi = num_seqs - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (wq[mid] <= w) lo = mid; else hi = mid - 1;
        }
        s = lo;
    }
    int qb = 0, tl = 0;
    if (in_range) bw_seq_rows(cu_q, s, total_q, &qb, &tl);
    const int t = in_range ? w - wq[s] : 0;
    const bool valid = in_range && t < tl;
    const long long prow = valid ? static_cast<long long>(qb) + t : 0;
    float acc = 0.f;
    if (valid) {
        const size_t off = (static_cast<size_t>(prow) * H + h) * D + sub * 8;
        const uint4 o = *reinterpret_cast<const uint4*>(out + off);
        const uint4 g = *reinterpret_cast<const uint4*>(dout + off);
        const uint32_t ow[4] = {o.x, o.y, o.z, o.w}, gw[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc = fmaf(__uint_as_float(ow[i] << 16), __uint_as_float(gw[i] << 16), acc);
            acc = fmaf(__uint_as_float(ow[i] & 0xFFFF0000u), __uint_as_float(gw[i] & 0xFFFF0000u),
                       acc);
        }
    }
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (in_range && sub == 0) {
        ndvec[row] = -acc;
        nlse2[row] = valid ? lse[static_cast<size_t>(h) * total_q + prow] * -1.4426950408889634f
                           : -INFINITY;
    }
}

// Slot ring of the column tiles; producer, issuers and elementwise warps keep
// identical copies. Fixed ring (VAR false): every unit uses the same NMAX
// slots, and tiles are numbered across units. Variable ring (d = 256: dv
// units stream through one more slot than dk units): every unit starts with
// all slots free (the producer waits for the previous unit's UMMAs to
// complete before its first load), so tile c of a unit goes to slot c % n,
// n the unit's ring size, and the barrier phases continue per slot.
template <int NMAX, bool VAR>
struct BwRing {
    static_assert(NMAX >= 1 && NMAX <= 4, "up to four slots");
    static_assert(VAR || (NMAX & (NMAX - 1)) == 0, "a fixed ring has a power-of-two size");
    static constexpr int SLOTS = NMAX;
    uint32_t base;            // fixed ring: tiles before the current unit
    uint32_t u0, u1, u2, u3;  // variable ring: fills of each slot before the unit
    int n;                    // variable ring: slots in the current unit's ring
    __device__ __forceinline__ void init() {
        base = u0 = u1 = u2 = u3 = 0;
        n = NMAX;
    }
    // c / n and c % n for n in {1, 2, 3, 4} without a general division
    __device__ __forceinline__ int quot(int c) const {
        return n == 3 ? c / 3 : (n == 4 ? c >> 2 : (n == 2 ? c >> 1 : c));
    }
    __device__ __forceinline__ uint32_t uses(int p) const {
        if constexpr (!VAR)
            return base > static_cast<uint32_t>(p) ? (base - 1 - p) / NMAX + 1 : 0u;
        else
            return p == 0 ? u0 : (p == 1 ? u1 : (p == 2 ? u2 : u3));
    }
    __device__ __forceinline__ int slot(int c) const {
        if constexpr (!VAR) return static_cast<int>((base + c) % NMAX);
        else return c - n * quot(c);
    }
    __device__ __forceinline__ uint32_t phase(int c) const {
        if constexpr (!VAR) return ((base + c) / NMAX) & 1u;
        else return (uses(slot(c)) + static_cast<uint32_t>(quot(c))) & 1u;
    }
    __device__ __forceinline__ void end_unit(int ncols) {
        if constexpr (!VAR) {
            base += static_cast<uint32_t>(ncols);
        } else {
            const int q = quot(ncols), rem = ncols - n * q;
            u0 += static_cast<uint32_t>(q + (0 < rem));
            if (n > 1) u1 += static_cast<uint32_t>(q + (1 < rem));
            if (n > 2) u2 += static_cast<uint32_t>(q + (2 < rem));
            if (n > 3) u3 += static_cast<uint32_t>(q + (3 < rem));
        }
    }
};

// Static persistent schedule (as the forward): round r gives CTA c unit
// r*G + c on even rounds and r*G + G-1-c on odd rounds.
__device__ __forceinline__ int bw_sched(int r, int c, int G) {
    return r * G + ((r & 1) ? (G - 1 - c) : c);
}

// A `rows`-row tile of a (rows, heads, d) tensor into shared memory: D/64
// boxes of 64 d-columns (128-byte swizzle), `rows` x 128 B apart. The tensor
// map's box gives the rows: query-side maps take rows/2 positions of heads 2g
// and 2g+1, key-side maps `rows` keys of head g.
template <int D>
__device__ __forceinline__ void bw_load_tile(uint8_t* dst, const CUtensorMap* map, uint64_t* bar,
                                             int row, int head, int rows = 128) {
#pragma unroll
    for (int c = 0; c < D / 64; ++c) tma_load_3d(dst + c * rows * 128, map, bar, c * 64, row, head);
}

// TMEM round trips of N columns (32 lanes x 32 bit): loads of 16 or 32
// columns (complete with tmem_wait_ld, then bw_fence before use) and stores of
// 8 or 16.
template <int N>
__device__ __forceinline__ void bw_ld_async(uint32_t taddr, uint32_t (&r)[N]);
template <int N>
__device__ __forceinline__ void bw_fence(uint32_t (&r)[N]);

// NC accumulator columns of this thread's row (a multiple of 16), times f, as
// bf16 to dst (when valid): all loads in flight before one wait.
template <int NC>
__device__ __forceinline__ void bw_store_acc(uint32_t taddr, __nv_bfloat16* dst, float f,
                                             bool valid) {
    constexpr int W = NC % 32 == 0 ? 32 : 16;  // columns per TMEM load
    static_assert(NC % W == 0, "accumulator chunks");
    uint32_t v[NC / W][W];
#pragma unroll
    for (int j = 0; j < NC / W; ++j) bw_ld_async<W>(taddr + W * j, v[j]);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < NC / W; ++j) {
        bw_fence<W>(v[j]);
        uint32_t pk[W / 2];
#pragma unroll
        for (int i = 0; i < W / 2; ++i)
            pk[i] = pack_bf16x2(__uint_as_float(v[j][2 * i]) * f, __uint_as_float(v[j][2 * i + 1]) * f);
        if (valid) {
            uint4* o = reinterpret_cast<uint4*>(dst + W * j);
#pragma unroll
            for (int q4 = 0; q4 < W / 8; ++q4)
                o[q4] = make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
        }
    }
}

template <int N>
__device__ __forceinline__ void bw_ld_async(uint32_t taddr, uint32_t (&r)[N]) {
    static_assert(N == 16 || N == 32, "TMEM load width");
    if constexpr (N == 32) {
        tmem_ld32_async(taddr, r);
    } else {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
            "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
              "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
              "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
            : "r"(taddr)
            : "memory");
    }
}

template <int N>
__device__ __forceinline__ void bw_fence(uint32_t (&r)[N]) {
    if constexpr (N == 32) {
        tmem_reg_fence(r);
    } else {
        static_assert(N == 16, "TMEM load width");
        asm volatile(""
                     : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                       "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                       "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
                     :
                     : "memory");
    }
}

template <int N>
__device__ __forceinline__ void bw_st(uint32_t taddr, const uint32_t (&r)[N]) {
    static_assert(N == 8 || N == 16, "TMEM store width");
    if constexpr (N == 16) {
        tmem_st16(taddr, r);
    } else {
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(
                taddr),
            "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
            : "memory");
    }
}

// CAP: the soft-cap is on (BwParams::has_cap). The host launches the
// instantiation that matches, so that the elementwise pass of either kind
// of layer carries only its own loops.
template <int D, int MODE, bool CAP>
__global__ void __launch_bounds__(BW_THREADS, 1)
    bwd_sm100(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
              const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
              const BwParams P) {
    using C = BwCfg<D>;
    constexpr bool KV = MODE == BW_KV;
    constexpr int DS = KV ? C::DSPLIT_KV : 1;  // units per row tile
    constexpr bool AT = C::A_TMEM;
    constexpr int ACC_N = D;                   // accumulator columns per product
    constexpr uint32_t X_COL = C::X_COL, Y_COL = C::Y_COL, A_COL = C::A_COL;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    // d <= 128: R1 = K (KV) or q (Q), R2 = V or dout. d = 256: R1 = K (KV, dk
    // units) or dout (Q); the other operand is in TMEM.
    // [NSLOT] x (C1, C2, lse2[CR], D[CR]); d = 256 dv units: + R1 as one more slot
    uint8_t* sSlot = AT ? base : base + C::RES_BYTES;
    uint8_t* sR1 = AT ? base + C::NSLOT * C::SLOT_BYTES : base;
    uint8_t* sR2 = sR1 + C::TILE_BYTES;
    constexpr int NS = C::NSLOT;
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + C::SMEM_TILES);
    uint64_t* r_full = bars + 0;
    uint64_t* r_empty = bars + 1;
    uint64_t* c_full = bars + 2;    // [NRING_MAX <= 4]
    uint64_t* c_empty = bars + 6;   // [NRING_MAX <= 4]
    // Single-buffered X / Y (d = 256 dk units and dq kernel), per column part
    // h (columns HW h .. HW h + HW - 1 of X and Y, the column parts of the
    // elementwise warps):
    uint64_t* xy_full = bars + 10;  // [NPART] X and Y of the current tile are in TMEM
    uint64_t* z_full = bars + 14;   // [NPART] P / dS of part h written back (4 warp arrivals)
    uint64_t* acc_done = bars + 18; // last accumulation of the unit completed
    uint64_t* acc_free = bars + 19; // epilogue read the accumulators (one arrival per warp)
    uint64_t* drain = bars + 20;
    uint64_t* ra_full = bars + 21;  // d = 256: the unit's TMEM-resident operand written
    // Double-buffered X / Y (every unit at d <= 128, dv units at d = 256), by
    // buffer b: xb_full[b] = X and Y of the buffer's next tile are in TMEM;
    // zb_full[NPART b + h] = its part h's P / dS written back (4 warp
    // arrivals). Each completes one phase per tile of its buffer, so that
    // neither side can run two phases ahead of a waiter.
    uint64_t* xb_full = bars + 22;  // [2]
    uint64_t* zb_full = bars + 24;  // [2 NPART]
    // dynamic schedule: the producer publishes each unit it takes in a ring of
    // four (sq_full: published; sq_empty: read by both issuers and every
    // elementwise warp)
    uint64_t* sq_full = bars + 24 + 2 * BW_NPART;   // [4]
    uint64_t* sq_empty = sq_full + 4;               // [4]
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sq_empty + 4);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    volatile int* sq_ring = reinterpret_cast<volatile int*>(tmem_holder + 4);  // [4], 16-byte aligned
    // varlen tables: cum[num_seqs + 1] (unit prefix in rank order), order[], work[]
    int* cum = reinterpret_cast<int*>(base + C::SMEM_TILES + 1024);
    int* order = cum + C::MAX_SEQ_TABLE + 1;
    int* work = order + C::MAX_SEQ_TABLE;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(r_full, 1);
        mbar_init(r_empty, C::ISSUERS);
        for (int i = 0; i < C::NRING_MAX; ++i) {
            mbar_init(&c_full[i], 1);
            mbar_init(&c_empty[i], C::ISSUERS);
        }
        for (int h = 0; h < BW_NPART; ++h) {
            mbar_init(&xy_full[h], C::ISSUERS);
            mbar_init(&z_full[h], 4);  // the part's warp in each lane quadrant
        }
        mbar_init(acc_done, C::ISSUERS);
        mbar_init(acc_free, BW_EW_THREADS / 32);
        mbar_init(drain, C::ISSUERS);
        mbar_init(ra_full, BW_EW_THREADS / 32);
        for (int b = 0; b < 2; ++b) mbar_init(&xb_full[b], C::ISSUERS);
        for (int i = 0; i < 2 * BW_NPART; ++i) mbar_init(&zb_full[i], 4);
        for (int i = 0; i < 4; ++i) {
            mbar_init(&sq_full[i], 1);
            mbar_init(&sq_empty[i], C::ISSUERS + BW_EW_THREADS / 32);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (P.varlen) {
        // work of each sequence (column tiles of all its row tiles, one KV
        // head), its rank (heaviest first, ties by index), then the units
        // (Hkv x row tiles) of the ranked sequences as an exclusive scan
        const int ns = P.num_seqs;
        for (int q = threadIdx.x; q < ns; q += blockDim.x) {
            BwUnit W;
            int qb, kb;
            bw_seq_rows(P.cu_q, q, P.total_q, &qb, &W.T);
            bw_seq_rows(P.cu_k, q, P.total_k, &kb, &W.S);
            W.qoff = W.S - W.T;
            const int tiles = W.T > 0 ? bw_row_tiles<MODE>(W.T, W.S) : 0;
            int w = 0;
            for (int rt = 0; rt < tiles; ++rt) {
                bw_tile_cols<D, MODE>(rt, tiles, P.window, W);
                w += max(W.ncols, 0);
            }
            work[q] = w;
        }
        __syncthreads();
        for (int q = threadIdx.x; q < ns; q += blockDim.x) {
            const int wq = work[q];
            int rank = 0;
            for (int q2 = 0; q2 < ns; ++q2) {
                const int w2 = work[q2];
                rank += (w2 > wq) || (w2 == wq && q2 < q);
            }
            order[rank] = q;
        }
        __syncthreads();
        for (int k = threadIdx.x; k < ns; k += blockDim.x) {
            int qb, t, kb, sk;
            bw_seq_rows(P.cu_q, order[k], P.total_q, &qb, &t);
            bw_seq_rows(P.cu_k, order[k], P.total_k, &kb, &sk);
            cum[k] = P.Hkv * bw_row_tiles<MODE>(t, sk);
        }
        __syncthreads();
        if (warp == 0) {
            int carry = 0;
            for (int s0 = 0; s0 < ns; s0 += 32) {
                const int q = s0 + lane;
                const int x = (q < ns) ? cum[q] : 0;
                int incl = x;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, incl, off);
                    if (lane >= off) incl += y;
                }
                if (q < ns) cum[q] = carry + incl - x;
                carry += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (lane == 0) cum[ns] = carry;
        }
    }
    if (warp == BW_WARP_MMA) {
        tmem_alloc(tmem_holder, BW_TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == BW_WARP_PRODUCER && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmO);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const int G = gridDim.x;
    const int cta = blockIdx.x;
    const uint64_t lim = P.timeout_ns;
    const int num_units = P.varlen ? min(P.num_units, cum[P.num_seqs] * DS) : P.num_units;
    // Unit of round r for this CTA, or -1 when it has no more. Static: the
    // zig-zag schedule. Dynamic: the producer takes the next unit from the
    // launch's counter and publishes it in sq_ring; the issuers and the
    // elementwise warps read it there in the same order. Every role sees the
    // same sequence of units, ending with one past num_units.
    auto take_unit = [&](int r, bool& ok) -> int {
        if (P.sched == nullptr) return r * G < num_units ? bw_sched(r, cta, G) : -1;
        const int i = r & 3;
        if (!mbar_wait(&sq_empty[i], ((r >> 2) & 1) ^ 1, abort_flag, lim, SITE_BW_PROD)) {
            ok = false;
            return -1;
        }
        const int u = static_cast<int>(atomicAdd(P.sched, 1u));
        sq_ring[i] = u;
        mbar_arrive(&sq_full[i]);  // release: the ring entry is visible to the waiters
        return u < num_units ? u : -1;
    };
    // a consumer's copy; `warp_wide`: every lane of the warp calls it and one
    // arrival is made for the warp
    auto read_unit = [&](int r, bool& ok, bool warp_wide) -> int {
        if (P.sched == nullptr) return r * G < num_units ? bw_sched(r, cta, G) : -1;
        const int i = r & 3;
        bool w = mbar_wait(&sq_full[i], (r >> 2) & 1, abort_flag, lim, SITE_BW_MMA);
        if (warp_wide) w = __all_sync(0xffffffffu, w);
        if (!w) {
            ok = false;
            return -1;
        }
        const int u = sq_ring[i];
        if (warp_wide) __syncwarp();
        if (!warp_wide || lane == 0) mbar_arrive(&sq_empty[i]);
        return u < num_units ? u : -1;
    };
    // slots in a unit's ring: d = 256 dv units also stream through R1
    auto ring_size = [](const BwUnit& U) { return (AT && KV && U.dh == 0) ? NS + 1 : NS; };
    using Ring = BwRing<(AT && KV) ? C::NRING_MAX : NS, AT && KV>;

    if (warp == BW_WARP_PRODUCER) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            Ring ring;
            ring.init();
            int uw = 0;       // units with work so far
            bool ok = true;
            for (int r = 0; ok; ++r) {
                const int u = take_unit(r, ok);
                if (u < 0) break;
                BwUnit U;
                bw_unit<D, MODE>(P, cum, order, u, U);
                if (U.ncols == 0) continue;
                if (uw > 0) {
                    ok = mbar_wait(r_empty, (uw - 1) & 1, abort_flag, lim, SITE_BW_PROD);
                    if (!ok) break;
                }
                if constexpr (AT) {
                    // one resident tile in shared memory: K for a dk unit,
                    // dout for the dq kernel; a dv unit has none
                    if (KV && U.dh == 0) {
                        mbar_arrive(r_full);
                    } else {
                        mbar_arrive_expect_tx(r_full, C::TILE_BYTES);
                        if (KV)
                            bw_load_tile<D>(sR1, &tmK, r_full, U.kbase + U.row0, U.g);
                        else
                            bw_load_tile<D>(sR1, &tmO, r_full, U.qbase + U.row0, 2 * U.g);
                    }
                } else {
                    mbar_arrive_expect_tx(r_full, 2 * C::TILE_BYTES);
                    if (KV) {
                        bw_load_tile<D>(sR1, &tmK, r_full, U.kbase + U.row0, U.g);
                        bw_load_tile<D>(sR2, &tmV, r_full, U.kbase + U.row0, U.g);
                    } else {
                        bw_load_tile<D>(sR1, &tmQ, r_full, U.qbase + U.row0, 2 * U.g);
                        bw_load_tile<D>(sR2, &tmO, r_full, U.qbase + U.row0, 2 * U.g);
                    }
                }
                ring.n = ring_size(U);
                for (int c = 0; c < U.ncols; ++c) {
                    const int sl = ring.slot(c);
                    ok = mbar_wait(&c_empty[sl], ring.phase(c) ^ 1, abort_flag, lim, SITE_BW_PROD);
                    if (!ok) break;
                    uint8_t* slot = sSlot + sl * C::SLOT_BYTES;
                    if (KV) {
                        const int t0 = (U.col0 + c) * C::CQ;
                        mbar_arrive_expect_tx(&c_full[sl], 2 * C::CTILE_BYTES + C::VEC_TX);
                        bw_load_tile<D>(slot, &tmQ, &c_full[sl], U.qbase + t0, 2 * U.g, C::CR);
                        bw_load_tile<D>(slot + C::CTILE_BYTES, &tmO, &c_full[sl], U.qbase + t0,
                                        2 * U.g, C::CR);
                        // -lse2 and -D of the tile's CR query rows (head 2g, then 2g+1)
                        float* vec = reinterpret_cast<float*>(slot + 2 * C::CTILE_BYTES);
#pragma unroll
                        for (int hl = 0; hl < 2; ++hl) {
                            const size_t off = static_cast<size_t>(U.wbase) +
                                               (2 * U.g + hl) * U.wstride + t0;
                            bulk_load(vec + hl * C::CQ, P.nlse2 + off, C::CQ * 4, &c_full[sl]);
                            bulk_load(vec + C::CR + hl * C::CQ, P.ndvec + off, C::CQ * 4,
                                      &c_full[sl]);
                        }
                    } else {
                        const int key0 = (U.col0 + c) * C::CK;
                        mbar_arrive_expect_tx(&c_full[sl], 2 * C::CTILE_BYTES);
                        bw_load_tile<D>(slot, &tmK, &c_full[sl], U.kbase + key0, U.g, C::CR);
                        bw_load_tile<D>(slot + C::CTILE_BYTES, &tmV, &c_full[sl], U.kbase + key0,
                                        U.g, C::CR);
                    }
                }
                if (!ok) break;
                ring.end_unit(U.ncols);
                ++uw;
            }
            // Drain: every copy issued lands before the CTA exits (the last
            // fill of each slot).
#pragma unroll
            for (int p = 0; p < Ring::SLOTS; ++p)
                if (ring.uses(p) > 0) mbar_wait_drain(&c_full[p], (ring.uses(p) - 1) & 1, lim);
            if (uw > 0) mbar_wait_drain(r_full, (uw - 1) & 1, lim);
        }
        __syncwarp();
    }
    else if (warp == BW_WARP_MMA || (C::ISSUERS == 2 && warp == BW_WARP_MMA2)) {
        // ------------------------------------------------------------ UMMA issuers
        // One thread issues a tcgen05.mma about every 67 cycles, less than the
        // math of the N = 64 UMMAs, so two threads in different warps share
        // the issue: issuer 0 X and the accumulation that reads X (dv, or dq),
        // issuer 1 Y and the accumulation that reads Y (dk). Neither writes
        // what the other's UMMAs read, and each keeps its own order (the X of
        // a buffer after the accumulation over that buffer's P, its Y after
        // the one over its dS). Both take every wait; the barriers their
        // commits complete count both.
        const int role = warp - BW_WARP_MMA;
        const bool do_x = role == 0;
        const bool do_y = C::ISSUERS == 2 ? role == 1 : role == 0;
        if (lane == 0) {
            constexpr int HW = C::HW;
            constexpr uint32_t IDESC_ACC = idesc_bf16(128, ACC_N, true);
            constexpr uint32_t HI = sdesc_hi(1024);  // SBO 1024 B (8 rows x 128 B)
            // K-major operands (contraction over d): 64-column blocks of rows x
            // 128 B (resident tiles: 128 rows; column tiles: CR rows), k-step of
            // 16 columns = 32 B inside a block
            const uint32_t r1_lo = sdesc_lo(smem_u32(sR1), 16);
            const uint32_t r2_lo = sdesc_lo(smem_u32(sR2), 16);
            const uint32_t slot_lo = sdesc_lo(smem_u32(sSlot), 16);
            // the same column tiles read MN-major (contraction over their CR
            // rows): LBO = CR rows x 128 B between 64-column blocks
            constexpr uint32_t CBLOCK = (C::CR * 128) >> 4;
            const uint32_t slot_lo_mn = sdesc_lo(smem_u32(sSlot), C::CR * 128);
            constexpr uint32_t SLOT_STEP = C::SLOT_BYTES >> 4;
            constexpr uint32_t CTILE_STEP = C::CTILE_BYTES >> 4;
            Ring ring;         // column-tile slots
            ring.init();
            uint32_t bt = 0;   // column tiles with double-buffered X / Y (xb_full, zb_full)
            uint32_t xt = 0;   // column tiles with single-buffered X / Y (xy_full, z_full)
            int uw = 0;
            bool ok = true;
            auto kstep = [](int kk) -> uint32_t {
                return ((kk * 16) / 64) * (16384 >> 4) + (((kk * 16) % 64) / 16) * 2;
            };
            auto kstep_c = [](int kk) -> uint32_t {
                return ((kk * 16) / 64) * CBLOCK + (((kk * 16) % 64) / 16) * 2;
            };
            // Single-buffered X / Y of the tile in slot sl (d = 256 dk units and
            // the dq kernel), each one N = CR UMMA per k-step. A operands: KV dk
            // unit X: K in R1, Y: V in TMEM; Q: X: q in TMEM, Y: dout in R1.
            auto issue_xy_tile = [&](int sl, int kind) {
                constexpr uint32_t IDESC_XYT = idesc_bf16(128, C::CR, false);
                const uint32_t c1 = slot_lo + sl * SLOT_STEP;
                const uint32_t c2 = c1 + CTILE_STEP;
                if constexpr (AT) {
                    const bool x_tmem = !KV || kind == 0;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        if (!do_x) break;
                        if (x_tmem)
                            umma_ts_lh(tmem + X_COL, tmem + A_COL + 8 * kk, c1 + kstep_c(kk), HI,
                                       IDESC_XYT, kk != 0);
                        else
                            umma_ss_lh(tmem + X_COL, r1_lo + kstep(kk), c1 + kstep_c(kk), HI,
                                       IDESC_XYT, kk != 0);
                    }
                    if (do_y && (!KV || kind == 1)) {
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            if (KV)
                                umma_ts_lh(tmem + Y_COL, tmem + A_COL + 8 * kk, c2 + kstep_c(kk),
                                           HI, IDESC_XYT, kk != 0);
                            else
                                umma_ss_lh(tmem + Y_COL, r1_lo + kstep(kk), c2 + kstep_c(kk), HI,
                                           IDESC_XYT, kk != 0);
                        }
                    }
                } else {
                    if (do_x) {
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk)
                            umma_ss_lh(tmem + X_COL, r1_lo + kstep(kk), c1 + kstep_c(kk), HI,
                                       IDESC_XYT, kk != 0);
                    }
                    if (do_y) {
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk)
                            umma_ss_lh(tmem + Y_COL, r2_lo + kstep(kk), c2 + kstep_c(kk), HI,
                                       IDESC_XYT, kk != 0);
                    }
                }
#pragma unroll
                for (int h = 0; h < BW_NPART; ++h) umma_commit(&xy_full[h]);
            };
            // accumulations over part h's HW rows (K indices HW h ..): A = the
            // bf16 operand the part's warps wrote at columns HW h + 8 k4; B =
            // the streamed tile read MN-major (all D columns)
            auto issue_acc = [&](int sl, int h, int kind, bool first) {
                const uint32_t c1_mn = slot_lo_mn + sl * SLOT_STEP;
                const uint32_t c2_mn = c1_mn + CTILE_STEP;
                constexpr int KS = HW / 16;  // K steps per part
#pragma unroll
                for (int k4 = 0; k4 < KS; ++k4) {
                    const int kk = KS * h + k4;
                    const uint32_t acc = (first && kk == 0) ? 0u : 1u;
                    const uint32_t bstep = kk * ((16 * 128) >> 4);
                    const uint32_t zc = HW * h + 8 * k4;
                    if (KV) {
                        // dv += P^T dout (P^T at X), dk += dS^T q (dS^T at Y); at
                        // d = 256 the dv unit does the first, the dk unit the second
                        if (do_x && (!AT || kind == 0))
                            umma_ts_lh(tmem + 0, tmem + X_COL + zc, c2_mn + bstep, HI, IDESC_ACC,
                                       acc);
                        if (do_y && (!AT || kind == 1))
                            umma_ts_lh(tmem + (AT ? 0 : ACC_N), tmem + Y_COL + zc, c1_mn + bstep,
                                       HI, IDESC_ACC, acc);
                    } else if (do_x) {
                        // dq += dS K (dS at X)
                        umma_ts_lh(tmem + 0, tmem + X_COL + zc, c1_mn + bstep, HI, IDESC_ACC,
                                   acc);
                    }
                }
            };
            // Single-buffered order per tile c: XY(c) | z_0 | ACC_0(c) | z_1 |
            // ACC_1(c) | ... XY(c+1): X / Y overwrite P / dS only after the
            // accumulation reading them was issued, and UMMAs of one thread
            // execute in issue order. Double-buffered: X / Y of tile c into
            // buffer b = c & 1, the accumulation over buffer b, then X / Y of
            // tile c+2 into it again, so that X / Y(c+1) run while the
            // elementwise warps work on tile c.
            // X / Y of the tile in slot sl into buffer b (d = 256 dv units: X
            // only, K in TMEM)
            auto issue_xy_buf = [&](int sl, uint32_t b) {
                constexpr uint32_t IDESC_XYT = idesc_bf16(128, C::CR, false);
                const uint32_t c1 = slot_lo + sl * SLOT_STEP;
                const uint32_t c2 = c1 + CTILE_STEP;
                const uint32_t xc = C::XB0 + C::XB_STEP * b, yc = C::YB0 + C::XB_STEP * b;
                if constexpr (AT) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        if (!do_x) break;
                        umma_ts_lh(tmem + xc, tmem + A_COL + 8 * kk, c1 + kstep_c(kk), HI,
                                   IDESC_XYT, kk != 0);
                    }
                } else {
                    if (do_x) {
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk)
                            umma_ss_lh(tmem + xc, r1_lo + kstep(kk), c1 + kstep_c(kk), HI,
                                       IDESC_XYT, kk != 0);
                    }
                    if (do_y) {
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk)
                            umma_ss_lh(tmem + yc, r2_lo + kstep(kk), c2 + kstep_c(kk), HI,
                                       IDESC_XYT, kk != 0);
                    }
                }
                umma_commit(&xb_full[b]);
            };
            // accumulations over part h of buffer b: dv (issuer 0, P^T at X) and
            // dk (issuer 1, dS^T at Y) in KV mode, dq (issuer 0, dS at X) in Q
            // mode; d = 256 dv units: dv only
            auto issue_acc_buf = [&](int sl, int h, uint32_t b, bool first) {
                const uint32_t c1_mn = slot_lo_mn + sl * SLOT_STEP;
                const uint32_t c2_mn = c1_mn + CTILE_STEP;
                const uint32_t xc = C::XB0 + C::XB_STEP * b, yc = C::YB0 + C::XB_STEP * b;
                constexpr int KS = HW / 16;
#pragma unroll
                for (int k4 = 0; k4 < KS; ++k4) {
                    const int kk = KS * h + k4;
                    const uint32_t acc = (first && kk == 0) ? 0u : 1u;
                    const uint32_t bstep = kk * ((16 * 128) >> 4);
                    const uint32_t zc = HW * h + 8 * k4;
                    if (KV) {
                        if (do_x)
                            umma_ts_lh(tmem + 0, tmem + xc + zc, c2_mn + bstep, HI, IDESC_ACC, acc);
                        if (do_y && !AT)
                            umma_ts_lh(tmem + ACC_N, tmem + yc + zc, c1_mn + bstep, HI, IDESC_ACC,
                                       acc);
                    } else if (do_x) {
                        umma_ts_lh(tmem + 0, tmem + xc + zc, c1_mn + bstep, HI, IDESC_ACC, acc);
                    }
                }
            };
            // X / Y of the unit's column tile c into buffer b
            auto load_xy_buf = [&](int c, uint32_t b) -> bool {
                if (!mbar_wait(&c_full[ring.slot(c)], ring.phase(c), abort_flag, lim, SITE_BW_MMA))
                    return false;
                tc_fence_after();
                issue_xy_buf(ring.slot(c), b);
                return true;
            };
            for (int r = 0; ok; ++r) {
                const int u = read_unit(r, ok, false);
                if (u < 0) break;
                BwUnit U;
                bw_unit<D, MODE>(P, cum, order, u, U);
                if (U.ncols == 0) continue;
                ok = mbar_wait(r_full, uw & 1, abort_flag, lim, SITE_BW_MMA);
                if (!ok) break;
                if constexpr (AT) {  // the elementwise warps wrote the TMEM-resident operand
                    ok = mbar_wait(ra_full, uw & 1, abort_flag, lim, SITE_BW_MMA);
                    if (!ok) break;
                }
                tc_fence_after();
                ring.n = ring_size(U);
                if (C::DB || (KV && U.dh == 0)) {
                    // double-buffered X / Y (d = 256: dv units, X only)
                    ok = load_xy_buf(0, bt & 1);
                    if (ok && U.ncols > 1) ok = load_xy_buf(1, (bt + 1) & 1);
                    if (!ok) break;
                    for (int c = 0; c < U.ncols; ++c) {
                        const int sl = ring.slot(c);
                        const uint32_t b = bt & 1;
                        if (c == 0 && uw > 0) {
                            ok = mbar_wait(acc_free, (uw - 1) & 1, abort_flag, lim,
                                           SITE_BW_MMA_ACC);
                            if (!ok) break;
                        }
#pragma unroll
                        for (int h = 0; h < BW_NPART; ++h) {
                            ok = mbar_wait(&zb_full[BW_NPART * b + h], (bt >> 1) & 1, abort_flag,
                                           lim, SITE_BW_MMA_Z);
                            if (!ok) break;
                            tc_fence_after();
                            issue_acc_buf(sl, h, b, c == 0);
                        }
                        if (!ok) break;
                        umma_commit(&c_empty[sl]);
                        if (c + 2 < U.ncols) {  // tile c+2 goes into buffer b again
                            ok = load_xy_buf(c + 2, b);
                            if (!ok) break;
                        }
                        ++bt;
                    }
                    if (!ok) break;
                    ring.end_unit(U.ncols);
                    umma_commit(acc_done);
                    umma_commit(r_empty);
                    ++uw;
                    continue;
                }
                if constexpr (!AT) continue;  // (every unit above)
                // single-buffered X / Y (d = 256 dk units and dq kernel)
                ok = mbar_wait(&c_full[ring.slot(0)], ring.phase(0), abort_flag, lim, SITE_BW_MMA);
                if (!ok) break;
                tc_fence_after();
                issue_xy_tile(ring.slot(0), U.dh);
                for (int c = 0; c < U.ncols; ++c) {
                    const int sl = ring.slot(c);
                    if (c == 0 && uw > 0) {
                        ok = mbar_wait(acc_free, (uw - 1) & 1, abort_flag, lim, SITE_BW_MMA_ACC);
                        if (!ok) break;
                    }
#pragma unroll
                    for (int h = 0; h < BW_NPART; ++h) {
                        ok = mbar_wait(&z_full[h], xt & 1, abort_flag, lim, SITE_BW_MMA_Z);
                        if (!ok) break;
                        tc_fence_after();
                        issue_acc(sl, h, U.dh, c == 0);
                    }
                    if (!ok) break;
                    umma_commit(&c_empty[sl]);
                    if (c + 1 < U.ncols) {
                        ok = mbar_wait(&c_full[ring.slot(c + 1)], ring.phase(c + 1), abort_flag,
                                       lim, SITE_BW_MMA);
                        if (!ok) break;
                        tc_fence_after();
                        issue_xy_tile(ring.slot(c + 1), U.dh);
                    }
                    ++xt;
                }
                if (!ok) break;
                ring.end_unit(U.ncols);
                umma_commit(acc_done);
                umma_commit(r_empty);
                ++uw;
            }
            // Drain: all issued UMMAs complete before TMEM is released.
            umma_commit(drain);
            mbar_wait_drain(drain, 0, lim);
        }
        __syncwarp();
    }
    else if (warp < BW_WARP_PRODUCER) {
        // ------------------------------------------------------------ elementwise + epilogue
        // Warps w, w+4, ... share TMEM lane quadrant w%4 (rows 32(w%4)..+31);
        // warp w takes the columns HW (w/4) .. HW (w/4) + HW - 1 of X and Y.
        // KV mode: row = key, column = query row (head 2g + column/CQ). Q mode:
        // row = query row (head 2g + row/64), column = key.
        constexpr int HW = C::HW, CQ = C::CQ, CHUNK = C::CHUNK;
        const int qd = warp & 3, part = warp >> 2;
        const int r = (qd << 5) | lane;
        const uint32_t lane_addr = static_cast<uint32_t>(qd * 32) << 16;
        const int col0 = part * HW;
        Ring ring;         // column-tile slots
        ring.init();
        uint32_t xt = 0;   // column tiles with single-buffered X / Y (xy_full, z_full)
        uint32_t bt = 0;   // column tiles with double-buffered X / Y (xb_full, zb_full)
        int uw = 0;
        bool ok = true;
        for (int rr = 0; ok; ++rr) {
            const int u = read_unit(rr, ok, true);
            if (u < 0) break;
            BwUnit U;
            bw_unit<D, MODE>(P, cum, order, u, U);
            if (U.ncols == 0) {
                // keys that no query sees: zero gradients (KV mode only; every
                // query sees at least its own key)
                if (KV && r < U.rvalid) {
                    const size_t row = (static_cast<size_t>(U.kbase) + U.row0 + r) * P.Hkv + U.g;
                    const size_t c0 = row * D + part * (D / BW_NPART);
#pragma unroll
                    for (int c = 0; c < D / BW_NPART; c += 8) {
                        if (!AT || U.dh == 0)
                            *reinterpret_cast<uint4*>(P.dv + c0 + c) = make_uint4(0u, 0u, 0u, 0u);
                        if (!AT || U.dh == 1)
                            *reinterpret_cast<uint4*>(P.dk + c0 + c) = make_uint4(0u, 0u, 0u, 0u);
                    }
                }
                continue;
            }
            // Q mode: this thread's query row, its -lse2 and -D
            const int hl_row = r >> 6, pr_row = r & 63;
            const int t_row = U.row0 + pr_row;  // Q mode
            float row_nl2 = -INFINITY, row_nd = 0.f;
            if (!KV && t_row < U.T) {
                const size_t off =
                    static_cast<size_t>(U.wbase) + (2 * U.g + hl_row) * U.wstride + t_row;
                row_nl2 = P.nlse2[off];
                row_nd = P.ndvec[off];
            }
            const int key_row = U.row0 + r;  // KV mode
            if constexpr (AT) {
                // This thread's row of the unit's TMEM-resident operand (KV dv
                // unit: K, dk unit: V; Q: q), its part's D / NPART of the d
                // columns as bf16 pairs at TMEM columns A_COL + (D / NPART / 2)
                // part ..; rows past
                // the sequence are zeros. The previous unit's UMMAs, which read
                // these columns, completed before its epilogue (acc_done).
                const __nv_bfloat16* src = nullptr;
                if (KV) {
                    if (key_row < U.S)
                        src = (U.dh == 0 ? P.k : P.v) +
                              ((static_cast<size_t>(U.kbase) + key_row) * P.Hkv + U.g) * D;
                } else if (t_row < U.T) {
                    src = P.q + ((static_cast<size_t>(U.qbase) + t_row) * P.H + 2 * U.g + hl_row) * D;
                }
                constexpr int PD = D / BW_NPART;  // d values of this part
                static_assert(PD % 64 == 0, "resident operand: 32 TMEM columns per store");
#pragma unroll
                for (int hc = 0; hc < PD / 64; ++hc) {  // 32 columns = 64 d values
                    uint32_t w[32];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        uint4 x = make_uint4(0u, 0u, 0u, 0u);
                        if (src)
                            x = __ldg(reinterpret_cast<const uint4*>(src + part * PD + 64 * hc) + i);
                        w[4 * i] = x.x;
                        w[4 * i + 1] = x.y;
                        w[4 * i + 2] = x.z;
                        w[4 * i + 3] = x.w;
                    }
                    tmem_st32(tmem + lane_addr + A_COL + (PD / 2) * part + 32 * hc, w);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(ra_full);
            }
            // double-buffered X / Y (d <= 128; d = 256 dv units: X only, in
            // the X and Y columns alternately)
            const bool xbuf = C::DB || (KV && U.dh == 0);
            ring.n = ring_size(U);
            for (int c = 0; c < U.ncols; ++c) {
                const int sl = ring.slot(c);
                const uint32_t b = bt & 1;
                const uint32_t x_col = xbuf ? C::XB0 + C::XB_STEP * b : X_COL;
                const uint32_t y_col = xbuf ? C::YB0 + C::XB_STEP * b : Y_COL;
                if (xbuf)
                    ok = mbar_wait(&xb_full[b], (bt >> 1) & 1, abort_flag, lim, SITE_BW_EW);
                else
                    ok = mbar_wait(&xy_full[part], xt & 1, abort_flag, lim, SITE_BW_EW);
                if (KV && ok)  // the column tile's lse2 / D, copied with its operands
                    ok = mbar_wait(&c_full[sl], ring.phase(c), abort_flag, lim, SITE_BW_EW);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after();
                const float* vec =
                    reinterpret_cast<const float*>(sSlot + sl * C::SLOT_BYTES + 2 * C::CTILE_BYTES);
                const int ccol0 = (U.col0 + c) * (KV ? CQ : C::CK);  // first t or key
                // Every pair of the tile visible? (then no per-element mask)
                bool interior;
                {
                    int j_lo, j_hi, t_lo, t_hi;
                    if (KV) {
                        j_lo = U.row0; j_hi = U.row0 + BW_KEYS - 1;
                        t_lo = ccol0;  t_hi = ccol0 + CQ - 1;
                    } else {
                        j_lo = ccol0;  j_hi = ccol0 + C::CK - 1;
                        t_lo = U.row0; t_hi = U.row0 + BW_QPOS - 1;
                    }
                    interior = j_hi <= t_lo + U.qoff && t_hi < U.T && j_hi < U.S &&
                               (P.window == 0 || t_hi + U.qoff - j_lo < P.window);
                }
                // This thread's visible column indices [vlo, vhi] (KV: query
                // rows t of its key; Q: keys j of its query row), as an offset
                // and unsigned span; an empty range never matches.
                int vlo;
                unsigned vspan;
                {
                    int lo, hi;
                    if (KV) {
                        lo = key_row - U.qoff;
                        hi = P.window > 0 ? min(U.T - 1, lo + P.window - 1) : U.T - 1;
                        if (key_row >= U.S) hi = lo - 1;
                    } else {
                        const int pos = t_row + U.qoff;
                        lo = P.window > 0 ? max(0, pos - P.window + 1) : 0;
                        hi = min(pos, U.S - 1);
                        if (t_row >= U.T) hi = lo - 1;
                    }
                    if (hi < lo) { lo = 1 << 30; hi = lo; }
                    vlo = lo;
                    vspan = static_cast<unsigned>(hi - lo);
                }
#pragma unroll
                for (int h2 = 0; h2 < HW / CHUNK; ++h2) {  // chunks of CHUNK columns
                    const int cb = col0 + CHUNK * h2;
                    uint32_t xv[CHUNK], yv[CHUNK];
                    // d = 256 dv unit: P only (no Y; dS is not formed)
                    const bool want_y = !(AT && KV && U.dh == 0);
                    bw_ld_async<CHUNK>(tmem + lane_addr + x_col + cb, xv);
                    if (want_y) {
                        bw_ld_async<CHUNK>(tmem + lane_addr + y_col + cb, yv);
                    } else {
#pragma unroll
                        for (int i = 0; i < CHUNK; ++i) yv[i] = 0u;
                    }
                    tmem_wait_ld();
                    bw_fence<CHUNK>(xv);
                    bw_fence<CHUNK>(yv);
                    // the cap's tanh by series when every |u| of this warp's chunk <= 1/4
                    bool poly = false;
                    if constexpr (CAP) {
                        float am[2] = {0.f, 0.f};
#pragma unroll
                        for (int i = 0; i < CHUNK; i += 2)
                            am[(i >> 1) & 1] =
                                fmax3f(am[(i >> 1) & 1], fabsf(__uint_as_float(xv[i])),
                                       fabsf(__uint_as_float(xv[i + 1])));
                        poly = __all_sync(0xffffffffu, fmaxf(am[0], am[1]) <= P.poly_acc_max);
                    }
                    uint32_t pp[CHUNK / 2], pd[CHUNK / 2];
                    // -lse2 / -D of the column pair i, i+1 (KV: per column, from
                    // the slot; Q: this row's)
                    auto vec_pair = [&](int i, float2& nl2, float2& nd) {
                        if (KV) {
                            nl2 = *reinterpret_cast<const float2*>(vec + cb + i);
                            nd = *reinterpret_cast<const float2*>(vec + C::CR + cb + i);
                        } else {
                            nl2 = make_float2(row_nl2, row_nl2);
                            nd = make_float2(row_nd, row_nd);
                        }
                    };
                    // -lse2 / -D of columns i .. i+3 (KV: one 16-byte shared load each)
                    auto vec_quad = [&](int i, float4& nl4, float4& nd4) {
                        if (KV) {
                            nl4 = *reinterpret_cast<const float4*>(vec + cb + i);
                            nd4 = *reinterpret_cast<const float4*>(vec + C::CR + cb + i);
                        } else {
                            nl4 = make_float4(row_nl2, row_nl2, row_nl2, row_nl2);
                            nd4 = make_float4(row_nd, row_nd, row_nd, row_nd);
                        }
                    };
                    // fast path, packed pairs: P = 2^(s2 - lse2), dS = P (dP - D) (1 - tanh^2);
                    // on tiles that cross the band's edges each weight outside
                    // [vlo, vhi] is replaced by 0 after its exp2. d = 256 dv units
                    // need P only (want_y false: no dS).
                    auto fast = [&](auto mask_tag, auto ds_tag) {
                        constexpr bool MASK = decltype(mask_tag)::value;
                        constexpr bool DS = decltype(ds_tag)::value;
                        auto keep = [&](int i, int e, float p) {
                            if constexpr (MASK) {
                                const int idx = (KV ? ((cb + i + e) & (CQ - 1)) : cb + i + e) + ccol0;
                                return static_cast<unsigned>(idx - vlo) <= vspan ? p : 0.0f;
                            } else {
                                return p;
                            }
                        };
                        const float2 one = make_float2(1.f, 1.f), mone = make_float2(-1.f, -1.f);
                        if constexpr (CAP) {
                            // tanh(alpha x / C) = x (t0 + t1 x^2 + t2 x^4 + t3 x^6): the
                            // series in u = alpha x / C with the powers of alpha / C
                            // folded into its coefficients
                            const float2 T0 = make_float2(P.th_c[0], P.th_c[0]);
                            const float2 T1 = make_float2(P.th_c[1], P.th_c[1]);
                            const float2 T2 = make_float2(P.th_c[2], P.th_c[2]);
                            const float2 T3 = make_float2(P.th_c[3], P.th_c[3]);
                            const float2 cl2 = make_float2(P.cap_l2, P.cap_l2);
#pragma unroll
                            for (int i = 0; i < CHUNK; i += 4) {
                                float4 nl4, nd4;
                                vec_quad(i, nl4, nd4);
#pragma unroll
                                for (int j = 0; j < 4; j += 2) {
                                    const int c = i + j;
                                    const float2 nl2 = j ? make_float2(nl4.z, nl4.w)
                                                         : make_float2(nl4.x, nl4.y);
                                    const float2 nd = j ? make_float2(nd4.z, nd4.w)
                                                        : make_float2(nd4.x, nd4.y);
                                    const float2 x = make_float2(__uint_as_float(xv[c]),
                                                                 __uint_as_float(xv[c + 1]));
                                    const float2 x2 = mul2(x, x);
                                    float2 q = fma2(x2, T3, T2);
                                    q = fma2(x2, q, T1);
                                    q = fma2(x2, q, T0);
                                    const float2 th = mul2(x, q);             // tanh(alpha x / C)
                                    const float2 e2 = fma2(th, cl2, nl2);      // s2 - lse2
                                    const float p0 = keep(c, 0, ex2_approx(e2.x));
                                    const float p1 = keep(c, 1, ex2_approx(e2.y));
                                    pp[c / 2] = pack_bf16x2(p0, p1);
                                    if constexpr (DS) {
                                        const float2 y = make_float2(__uint_as_float(yv[c]),
                                                                     __uint_as_float(yv[c + 1]));
                                        const float2 dcap = fma2(mul2(th, th), mone, one);
                                        const float2 ds =
                                            mul2(mul2(make_float2(p0, p1), add2(y, nd)), dcap);
                                        pd[c / 2] = pack_bf16x2(ds.x, ds.y);
                                    }
                                }
                            }
                        } else {
                            const float2 sl2 = make_float2(P.scale_l2, P.scale_l2);
#pragma unroll
                            for (int i = 0; i < CHUNK; i += 4) {
                                float4 nl4, nd4;
                                vec_quad(i, nl4, nd4);
#pragma unroll
                                for (int j = 0; j < 4; j += 2) {
                                    const int c = i + j;
                                    const float2 nl2 = j ? make_float2(nl4.z, nl4.w)
                                                         : make_float2(nl4.x, nl4.y);
                                    const float2 nd = j ? make_float2(nd4.z, nd4.w)
                                                        : make_float2(nd4.x, nd4.y);
                                    const float2 x = make_float2(__uint_as_float(xv[c]),
                                                                 __uint_as_float(xv[c + 1]));
                                    const float2 e2 = fma2(x, sl2, nl2);
                                    const float p0 = keep(c, 0, ex2_approx(e2.x));
                                    const float p1 = keep(c, 1, ex2_approx(e2.y));
                                    pp[c / 2] = pack_bf16x2(p0, p1);
                                    if constexpr (DS) {
                                        const float2 y = make_float2(__uint_as_float(yv[c]),
                                                                     __uint_as_float(yv[c + 1]));
                                        const float2 ds = mul2(make_float2(p0, p1), add2(y, nd));
                                        pd[c / 2] = pack_bf16x2(ds.x, ds.y);
                                    }
                                }
                            }
                        }
                    };
                    if (poly || !CAP) {
                        if (want_y) {
                            if (interior) fast(BwMask<false>{}, BwMask<true>{});
                            else fast(BwMask<true>{}, BwMask<true>{});
                        } else {
                            if (interior) fast(BwMask<false>{}, BwMask<false>{});
                            else fast(BwMask<true>{}, BwMask<false>{});
                        }
                    } else {
                        // general path: per-element mask, exact cap when |u| > 1/4
#pragma unroll
                        for (int i = 0; i < CHUNK; i += 2) {
                            float2 nl2v, ndv;
                            vec_pair(i, nl2v, ndv);
                            float pv[2], dsv[2];
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const int cc = cb + i + e;  // column 0..127
                                int t, j;
                                if (KV) {
                                    t = ccol0 + (cc & (CQ - 1));  // head 2g + cc/CQ
                                    j = key_row;
                                } else {
                                    t = t_row;
                                    j = ccol0 + cc;
                                }
                                const float nl2 = e ? nl2v.y : nl2v.x;
                                const float nd = e ? ndv.y : ndv.x;
                                const int pos = t + U.qoff;
                                const bool vis = (j <= pos) &&
                                                 (P.window == 0 || pos - j < P.window) &&
                                                 (t < U.T) && (j < U.S);
                                const float x = __uint_as_float(xv[i + e]);
                                float s2, dcap;
                                if constexpr (CAP) {
                                    float th;
                                    if (poly) {
                                        th = bw_tanh_series(x * P.u_scale);
                                    } else {
                                        // tanh(alpha x / C) = 1 - 2 / (1 + 2^(2 alpha log2(e) x / C))
                                        const float ex = ex2_approx(x * P.k_exp);
                                        th = fmaf(-2.0f, rcp_approx(1.0f + ex), 1.0f);
                                    }
                                    s2 = P.cap_l2 * th;
                                    dcap = fmaf(-th, th, 1.0f);
                                } else {
                                    s2 = x * P.scale_l2;
                                    dcap = 1.0f;
                                }
                                const float pw = vis ? ex2_approx(s2 + nl2) : 0.0f;
                                pv[e] = pw;
                                dsv[e] = pw * (__uint_as_float(yv[i + e]) + nd) * dcap;
                            }
                            pp[i / 2] = pack_bf16x2(pv[0], pv[1]);
                            pd[i / 2] = pack_bf16x2(dsv[0], dsv[1]);
                        }
                    }
                    // bf16 pairs of columns cb .. cb+CHUNK-1 go to TMEM columns
                    // col0 + (CHUNK/2) h2 ..: inside this warp's own X / Y
                    // columns, already read (chunk 0), never the other warp's
                    // (no ordering between the two warps of a quadrant is needed)
                    const uint32_t zc = col0 + (CHUNK / 2) * h2;
                    if (KV) {
                        // d = 256: the dv unit needs P^T only, the dk unit dS^T only
                        if (!AT || U.dh == 0)
                            bw_st<CHUNK / 2>(tmem + lane_addr + x_col + zc, pp);  // P^T
                        if (!AT || U.dh == 1)
                            bw_st<CHUNK / 2>(tmem + lane_addr + y_col + zc, pd);  // dS^T
                    } else {
                        bw_st<CHUNK / 2>(tmem + lane_addr + x_col + zc, pd);  // dS
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(xbuf ? &zb_full[BW_NPART * b + part] : &z_full[part]);
                if (xbuf) ++bt; else ++xt;
            }
            if (!ok) break;
            ring.end_unit(U.ncols);
            // ---- epilogue: accumulators -> bf16 gradients
            ok = mbar_wait(acc_done, uw & 1, abort_flag, lim, SITE_BW_EW_ACC);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            constexpr int PCOLS = ACC_N / BW_NPART;       // accumulator columns per warp
            constexpr int SEG = PCOLS < 32 ? PCOLS : 32;  // columns per TMEM round trip
            if (KV) {
                const bool valid = r < U.rvalid;
                const size_t row = (static_cast<size_t>(U.kbase) + key_row) * P.Hkv + U.g;
#pragma unroll
                for (int a = 0; a < 2; ++a) {  // a = 0: dv (columns 0..), a = 1: dk (ACC_N..)
                    // d = 256: one accumulator at column 0, dv or dk by unit
                    if (AT && a != U.dh) continue;
                    const float f = a ? P.query_scale : 1.0f;
                    const uint32_t acol = AT ? 0u : static_cast<uint32_t>(a * ACC_N);
                    __nv_bfloat16* dst = (a ? P.dk : P.dv) + row * D + part * PCOLS;
#pragma unroll
                    for (int sg = 0; sg < PCOLS / SEG; ++sg)
                        bw_store_acc<SEG>(tmem + lane_addr + acol + part * PCOLS + SEG * sg,
                                          dst + SEG * sg, f, valid);
                }
            } else {
                const bool valid = pr_row < U.rvalid;
                const size_t row = (static_cast<size_t>(U.qbase) + t_row) * P.H + 2 * U.g + hl_row;
                __nv_bfloat16* dst = P.dq + row * D + part * PCOLS;
#pragma unroll
                for (int sg = 0; sg < PCOLS / SEG; ++sg)
                    bw_store_acc<SEG>(tmem + lane_addr + part * PCOLS + SEG * sg, dst + SEG * sg,
                                      P.query_scale, valid);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_free);
            ++uw;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == BW_WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, BW_TMEM_COLS);
    }
}

}  // namespace g2
