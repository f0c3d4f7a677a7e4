/*
 * g2ref.h -- fp64 CPU oracle for the Gemma 2 per-layer attention forward
 * and its gradients.
 *
 * TEST INFRASTRUCTURE. This is the slow, plain reference that the CUDA
 * library is checked against. Only the test suite, the package smoke check
 * and the benchmark's CPU-baseline leg may load it. It shares no source with
 * the CUDA library and the CUDA library never calls it.
 *
 * What it computes (Gemma 2 card, "Method", per-layer attention pseudo-code;
 * soft-cap formula from the "Gemma 2 Guide", section 1):
 *   for each batch b, query head h, query row i:
 *     g = h / (H / Hkv)                 -- the KV head that h shares
 *     p = i + q_offset                  -- absolute position of the query
 *     q' = query_scale * q[b,i,h,:]     -- queries are scaled first
 *     x_j = q' . k[b,j,g,:]             for every key j in [0, S)
 *     s_j = softcap * tanh(x_j / softcap)   (softcap > 0; softcap == 0: s_j = x_j)
 *     visible(j) = j <= p and (window == 0 or p - j < window)
 *     s_j = -inf where not visible      -- cap first, then mask
 *     w = softmax_j(s)
 *     out[b,i,h,:] = sum_j w_j v[b,j,g,:]
 *     lse[b,h,i]  = log sum_{visible j} exp(s_j)   (natural log)
 *
 * Inputs are bf16 bit patterns (uint16), widened exactly to double.
 * Layouts are row-major with the head dimension contiguous:
 *   q (B,T,H,d), k and v (B,S,Hkv,d), out (B,T,H,d) double, lse (B,H,T) double.
 * Return value: 0 on success, -1 on an argument error.
 */
#ifndef G2REF_H
#define G2REF_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

int g2ref_attn(const uint16_t* q, const uint16_t* k, const uint16_t* v,
               double* out, double* lse,
               int64_t B, int64_t T, int64_t S, int64_t H, int64_t Hkv, int64_t d,
               int64_t q_offset, double query_scale, double softcap, int64_t window);

/* Same definition for a chosen list of rows. rows holds n triples (b, i, h);
 * out is (n, d) and lse is (n). */
int g2ref_attn_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                    double* out, double* lse, const int64_t* rows, int64_t n,
                    int64_t B, int64_t T, int64_t S, int64_t H, int64_t Hkv, int64_t d,
                    int64_t q_offset, double query_scale, double softcap, int64_t window);

/* One row in full: the capped logits s (S values, -inf where masked) and the
 * softmax weights w (S values, 0 where masked). */
int g2ref_row_detail(const uint16_t* q, const uint16_t* k,
                     double* s, double* w, int64_t b, int64_t i, int64_t h,
                     int64_t B, int64_t T, int64_t S, int64_t H, int64_t Hkv, int64_t d,
                     int64_t q_offset, double query_scale, double softcap, int64_t window);

/* Gradients of the dense layer above for an upstream gradient dout (B,T,H,d),
 * the chain rule applied to the same definition step by step:
 *   dw_j  = dout[b,i,h,:] . v[b,j,g,:]          (out = sum_j w_j v_j)
 *   ds_j  = w_j (dw_j - sum_k w_k dw_k)          (softmax)
 *   dx_j  = ds_j (1 - tanh^2(x_j / softcap))     (cap; "Gemma 2 Guide", Deep Dive
 *                                                  item 1; dx_j = ds_j without cap)
 *   dq[b,i,h,:] += query_scale sum_j dx_j k[b,j,g,:]
 *   dk[b,j,g,:] += dx_j query_scale q[b,i,h,:]    (summed over the heads of g)
 *   dv[b,j,g,:] += w_j dout[b,i,h,:]              (summed over the heads of g)
 * Masked keys have w_j = 0 and contribute nothing. dout is bf16 bits; dq
 * (B,T,H,d), dk and dv (B,S,Hkv,d) are double and fully overwritten. */
int g2ref_attn_bwd(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                   const uint16_t* dout, double* dq, double* dk, double* dv,
                   int64_t B, int64_t T, int64_t S, int64_t H, int64_t Hkv, int64_t d,
                   int64_t q_offset, double query_scale, double softcap, int64_t window);

/* The same gradients at chosen places, for layers whose full gradients are
 * too costly in fp64: qrows holds nq triples (b, i, h) and keys nk triples
 * (b, j, g) (g a KV head). dq (nq, d) gets dq[b,i,h,:]; dk and dv (nk, d) get
 * dk[b,j,g,:] and dv[b,j,g,:], each summed over every row of the group's
 * heads that sees key j. The softmax statistics of those rows (lse and
 * D = sum_j w_j dw_j) are computed first, and each weight is then
 * w_j = exp(s_j - lse). Returns -1 on an argument error or an index outside
 * the tensors. */
int g2ref_attn_bwd_sampled(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                           const uint16_t* dout, const int64_t* qrows, int64_t nq,
                           const int64_t* keys, int64_t nk, double* dq, double* dk, double* dv,
                           int64_t B, int64_t T, int64_t S, int64_t H, int64_t Hkv, int64_t d,
                           int64_t q_offset, double query_scale, double softcap,
                           int64_t window);

/* Threads used by the OpenMP loops (0 leaves the runtime default). */
void g2ref_set_threads(int n);
int g2ref_max_threads(void);

#ifdef __cplusplus
}
#endif
#endif
