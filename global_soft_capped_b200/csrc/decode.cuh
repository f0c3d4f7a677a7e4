// decode.cuh -- split-KV decode of soft-capped local/global GQA attention
// (one query per sequence) for B200 / sm_100a.
//
// Operation: the per-layer attention of the Gemma 2 card ("Method") for a
// single query at position L-1 of a sequence's KV cache; a local layer reads
// only the last `window` cached keys (the Guide's serving note that local
// layers only keep the last 4,096 tokens). The cap is the Guide's section-1
// formula, 50*tanh(s/50).
//
// Kernel 1 (decode_split): one CTA per (split of the visible key range, KV
// head g, sequence). Each K/V row is read once, with 16-byte coalesced loads,
// for both query heads 2g and 2g+1. Partial dot products are reduced with
// warp shuffles; the split's scores sit in shared memory; the CTA writes a
// partial result (max m, sum l in log2 units, unnormalised acc[d]) per head,
// or the final output directly when the sequence has a single split.
// Kernel 2 (decode_merge): one warp per (sequence, query head) combines the
// splits: M = max m_s, out = sum 2^(m_s-M) acc_s / sum 2^(m_s-M) l_s.
#pragma once

#include "common.cuh"

namespace g2 {

constexpr int DEC_THREADS = 128;
constexpr int DEC_MAX_CHUNK = 512;

// KV cache layouts of the decode path. Every layout stores rows of
// (Hkv, d) bf16; they differ in where position p of sequence s lives.
//   DEC_LINEAR  packed by cu_seqlens_k:      row = cu_k[s] + p
//   DEC_RING    ring of R slots per sequence: row = s*R + p mod R (R a power of
//               two; holds the last R positions, enough for a window <= R)
//   DEC_PAGED   blocks of bs rows:           row = block_table[s][p / bs]*bs + p mod bs
enum DecLayout : int { DEC_LINEAR = 0, DEC_RING = 1, DEC_PAGED = 2 };

struct DecParams {
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    const int* cu_k;         // DEC_LINEAR
    __nv_bfloat16* out;
    float* lse;
    float* ws_ml;   // [n][H][max_splits][2]  (m, l) log2 domain
    float* ws_acc;  // [n][H][max_splits][D]
    int num_seqs, total_k, H, Hkv, window, chunk, max_splits;
    float k_exp, cap_l2, scale_l2;
    int has_cap;
};

// Layout-specific parameters, a separate kernel argument (kept out of
// DecParams: a larger DecParams raised the linear kernel's registers and cost
// occupancy).
struct DecLayoutParams {
    const int* seq_lens;     // DEC_RING, DEC_PAGED: tokens seen per sequence
    const int* block_table;  // DEC_PAGED: [num_seqs][max_blocks]
    int ring_mask;           // DEC_RING: R - 1
    int ring_shift;          // DEC_RING: log2 R
    int block_shift;         // DEC_PAGED: log2 bs
    int max_blocks;          // DEC_PAGED: blocks per sequence in the table
    int num_blocks;          // DEC_PAGED: blocks in the cache
};

// Tokens seen by sequence s (the query sits at position L - 1).
template <int LAYOUT>
__device__ __forceinline__ int dec_len(const DecParams& P, const DecLayoutParams& LP, int s) {
    if (LAYOUT == DEC_LINEAR) {
        const int k0 = max(0, min(P.cu_k[s], P.total_k));  // never read outside the cache
        const int k1 = max(k0, min(P.cu_k[s + 1], P.total_k));
        return k1 - k0;
    } else if (LAYOUT == DEC_PAGED) {
        return max(0, min(LP.seq_lens[s], LP.max_blocks << LP.block_shift));
    } else {
        return max(0, LP.seq_lens[s]);
    }
}

// Cache row of position p of sequence s for the ring and paged layouts
// (always inside the cache arrays).
template <int LAYOUT>
__device__ __forceinline__ int dec_row(const DecLayoutParams& LP, int s, int p) {
    if constexpr (LAYOUT == DEC_RING) {
        return (s << LP.ring_shift) + (p & LP.ring_mask);
    } else {
        int b = LP.block_table[static_cast<size_t>(s) * LP.max_blocks + (p >> LP.block_shift)];
        b = max(0, min(b, LP.num_blocks - 1));
        return (b << LP.block_shift) + (p & ((1 << LP.block_shift) - 1));
    }
}

// Visible key range [lo, hi) of sequence s and its number of splits. A ring
// holds only its last R positions: the range is clipped to them.
template <int LAYOUT>
__device__ __forceinline__ void dec_range(const DecParams& P, const DecLayoutParams& LP, int s,
                                          int& lo, int& hi, int& nsplit) {
    const int L = dec_len<LAYOUT>(P, LP, s);
    lo = (P.window > 0) ? max(0, L - P.window) : 0;
    if (LAYOUT == DEC_RING) lo = max(lo, L - (LP.ring_mask + 1));
    hi = L;
    // more splits than planned only when the caller's max_cache_len undercounts:
    // drop the excess (wrong result, but never a read past the workspace) and
    // report the broken precondition in the sticky device word
    const int need = (hi - lo + P.chunk - 1) / P.chunk;
    nsplit = min(need, P.max_splits);
    if (need > P.max_splits && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0)
        atomicOr(&g_device_error, DEVERR_CACHE_LEN);
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

template <int D, int LAYOUT>
__global__ void __launch_bounds__(DEC_THREADS) decode_split(const DecParams P, const DecLayoutParams LP) {
    constexpr int TPR = D / 8;               // threads per key row (8 bf16 each)
    constexpr int RPW = 32 / TPR;            // rows per warp per load
    constexpr int RPC = RPW * (DEC_THREADS / 32);  // rows per CTA per load
    // loads in flight per thread: the linear layout steps one pointer by a
    // constant stride (offsets fold into the loads); the others read each
    // key's cache row from a per-CTA table and keep more loads in flight
    constexpr int UNR = (LAYOUT == DEC_LINEAR) ? 4 : 8;
    __shared__ float sc[2][DEC_MAX_CHUNK];
    __shared__ float red[RPC][2][D];
    __shared__ float wred[2][DEC_THREADS / 32];

    const int s = blockIdx.z, g = blockIdx.y, sp = blockIdx.x;
    int lo, hi, nsplit;
    dec_range<LAYOUT>(P, LP, s, lo, hi, nsplit);
    if (sp >= nsplit) return;
    const int kb = lo + sp * P.chunk;
    const int ke = min(hi, kb + P.chunk);
    const int n = ke - kb;
    size_t row0 = 0;  // linear layout: first cache row of the sequence
    if constexpr (LAYOUT == DEC_LINEAR) row0 = static_cast<size_t>(max(0, min(P.cu_k[s], P.total_k)));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rw = lane / TPR, cg = lane % TPR;
    const int rslot = warp * RPW + rw;  // 0..RPC-1

    // queries of heads 2g and 2g+1, this thread's 8 columns
    float q0[8], q1[8];
    {
        const __nv_bfloat16* qp = P.q + (static_cast<size_t>(s) * P.H + 2 * g) * D + cg * 8;
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(qp), q0);
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(qp + D), q1);
    }
    const size_t kstride = static_cast<size_t>(P.Hkv) * D;
    // linear layout: base pointers of this chunk, stepped by j rows below
    const __nv_bfloat16* klin = P.k + (row0 + kb) * kstride + static_cast<size_t>(g) * D + cg * 8;
    const __nv_bfloat16* vlin = P.v + (row0 + kb) * kstride + static_cast<size_t>(g) * D + cg * 8;
    const size_t gofs = static_cast<size_t>(g) * D + cg * 8;  // this thread's columns
    // other layouts: cache row of every key of the chunk (dynamic shared memory,
    // n <= chunk entries, sized at launch)
    extern __shared__ int rows_dyn[];
    if constexpr (LAYOUT != DEC_LINEAR) {
        for (int j = tid; j < n; j += DEC_THREADS) rows_dyn[j] = dec_row<LAYOUT>(LP, s, kb + j);
        __syncthreads();
    }

    // ---- phase 1: scores (log2 domain, capped)
    for (int base = 0; base < n; base += RPC * UNR) {
        uint4 kv[UNR];
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int j = base + u * RPC + rslot;
            const __nv_bfloat16* kp;
            if constexpr (LAYOUT == DEC_LINEAR)
                kp = klin + static_cast<size_t>(j) * kstride;
            else
                kp = P.k + static_cast<size_t>(rows_dyn[j < n ? j : 0]) * kstride + gofs;
            kv[u] = (j < n) ? ldg_stream(kp)
                            : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            float kf[8];
            bf16x8_to_f32(kv[u], kf);
            float d0 = 0.f, d1 = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                d0 = fmaf(q0[i], kf[i], d0);
                d1 = fmaf(q1[i], kf[i], d1);
            }
#pragma unroll
            for (int off = TPR / 2; off > 0; off >>= 1) {
                d0 += __shfl_xor_sync(0xffffffffu, d0, off);
                d1 += __shfl_xor_sync(0xffffffffu, d1, off);
            }
            const int j = base + u * RPC + rslot;
            if (cg == 0 && j < n) {
                float s0, s1;
                if (P.has_cap) {
                    s0 = fmaf(-2.0f * P.cap_l2, rcp_approx(1.0f + ex2_approx(d0 * P.k_exp)),
                              P.cap_l2);
                    s1 = fmaf(-2.0f * P.cap_l2, rcp_approx(1.0f + ex2_approx(d1 * P.k_exp)),
                              P.cap_l2);
                } else {
                    s0 = d0 * P.scale_l2;
                    s1 = d1 * P.scale_l2;
                }
                sc[0][j] = s0;
                sc[1][j] = s1;
            }
        }
    }
    __syncthreads();

    // ---- phase 2: max and exponentials per head
    float m0 = -INFINITY, m1 = -INFINITY;
    for (int j = tid; j < n; j += DEC_THREADS) {
        m0 = fmaxf(m0, sc[0][j]);
        m1 = fmaxf(m1, sc[1][j]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, off));
        m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, off));
    }
    if (lane == 0) {
        wred[0][warp] = m0;
        wred[1][warp] = m1;
    }
    __syncthreads();
    m0 = wred[0][0];
    m1 = wred[1][0];
#pragma unroll
    for (int w = 1; w < DEC_THREADS / 32; ++w) {
        m0 = fmaxf(m0, wred[0][w]);
        m1 = fmaxf(m1, wred[1][w]);
    }
    __syncthreads();  // everyone read wred before it is reused
    float l0 = 0.f, l1 = 0.f;
    for (int j = tid; j < n; j += DEC_THREADS) {
        const float p0 = ex2_approx(sc[0][j] - m0);
        const float p1 = ex2_approx(sc[1][j] - m1);
        sc[0][j] = p0;
        sc[1][j] = p1;
        l0 += p0;
        l1 += p1;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, off);
        l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
    if (lane == 0) {
        wred[0][warp] = l0;
        wred[1][warp] = l1;
    }
    __syncthreads();
    l0 = 0.f;
    l1 = 0.f;
#pragma unroll
    for (int w = 0; w < DEC_THREADS / 32; ++w) {
        l0 += wred[0][w];
        l1 += wred[1][w];
    }

    // ---- phase 3: acc = sum_j p_j v_j for both heads
    float a0[8], a1[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) a0[i] = a1[i] = 0.f;
    for (int base = 0; base < n; base += RPC * UNR) {
        uint4 vv[UNR];
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int j = base + u * RPC + rslot;
            const __nv_bfloat16* vp;
            if constexpr (LAYOUT == DEC_LINEAR)
                vp = vlin + static_cast<size_t>(j) * kstride;
            else
                vp = P.v + static_cast<size_t>(rows_dyn[j < n ? j : 0]) * kstride + gofs;
            vv[u] = (j < n) ? ldg_stream(vp)
                            : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int j = base + u * RPC + rslot;
            const float p0 = (j < n) ? sc[0][j] : 0.f;
            const float p1 = (j < n) ? sc[1][j] : 0.f;
            float vf[8];
            bf16x8_to_f32(vv[u], vf);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                a0[i] = fmaf(p0, vf[i], a0[i]);
                a1[i] = fmaf(p1, vf[i], a1[i]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        red[rslot][0][cg * 8 + i] = a0[i];
        red[rslot][1][cg * 8 + i] = a1[i];
    }
    __syncthreads();

    const int H = P.H;
    if (nsplit == 1) {
        // single split: final output straight away
        for (int e = tid; e < 2 * D; e += DEC_THREADS) {
            const int hh = e / D, c = e % D;
            float acc = 0.f;
#pragma unroll
            for (int r = 0; r < RPC; ++r) acc += red[r][hh][c];
            const float l = hh ? l1 : l0;
            P.out[(static_cast<size_t>(s) * H + 2 * g + hh) * D + c] = __float2bfloat16_rn(acc / l);
        }
        if (tid < 2 && P.lse != nullptr) {
            const float m = tid ? m1 : m0, l = tid ? l1 : l0;
            P.lse[static_cast<size_t>(s) * H + 2 * g + tid] =
                (m + log2f(l)) * 0.69314718055994531f;
        }
        return;
    }
    for (int e = tid; e < 2 * D; e += DEC_THREADS) {
        const int hh = e / D, c = e % D;
        float acc = 0.f;
#pragma unroll
        for (int r = 0; r < RPC; ++r) acc += red[r][hh][c];
        const size_t slot = (static_cast<size_t>(s) * H + 2 * g + hh) * P.max_splits + sp;
        P.ws_acc[slot * D + c] = acc;
    }
    if (tid < 2) {
        const size_t slot = (static_cast<size_t>(s) * H + 2 * g + tid) * P.max_splits + sp;
        P.ws_ml[slot * 2 + 0] = tid ? m1 : m0;
        P.ws_ml[slot * 2 + 1] = tid ? l1 : l0;
    }
}

template <int D, int LAYOUT>
__global__ void __launch_bounds__(128) decode_merge(const DecParams P, const DecLayoutParams LP) {
    const int wid = blockIdx.x * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (wid >= P.num_seqs * P.H) return;
    const int s = wid / P.H, h = wid % P.H;
    int lo, hi, nsplit;
    dec_range<LAYOUT>(P, LP, s, lo, hi, nsplit);
    if (nsplit <= 1) return;  // written by decode_split
    const size_t slot0 = (static_cast<size_t>(s) * P.H + h) * P.max_splits;
    float M = -INFINITY;
    for (int i = 0; i < nsplit; ++i) M = fmaxf(M, P.ws_ml[(slot0 + i) * 2]);
    constexpr int PER = D / 32;
    float acc[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = 0.f;
    float L = 0.f;
    for (int i = 0; i < nsplit; ++i) {
        const float w = ex2_approx(P.ws_ml[(slot0 + i) * 2] - M);
        L = fmaf(w, P.ws_ml[(slot0 + i) * 2 + 1], L);
        const float* a = P.ws_acc + (slot0 + i) * D;
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] = fmaf(w, a[e * 32 + lane], acc[e]);
    }
    const float inv = 1.0f / L;
    __nv_bfloat16* o = P.out + (static_cast<size_t>(s) * P.H + h) * D;
#pragma unroll
    for (int e = 0; e < PER; ++e) o[e * 32 + lane] = __float2bfloat16_rn(acc[e] * inv);
    if (lane == 0 && P.lse != nullptr)
        P.lse[static_cast<size_t>(s) * P.H + h] = (M + log2f(L)) * 0.69314718055994531f;
}

}  // namespace g2
