/*
 * g2attn.h -- libg2attn: Gemma 2 soft-capped local/global attention (forward,
 * decode and gradients) for NVIDIA B200 (sm_100a).
 *
 * The operation (Gemma 2 card, "Method", per-layer attention pseudo-code; the
 * soft-cap formula is the "Gemma 2 Guide", section 1): for every query row i
 * at absolute position p = i + q_offset and query head h, with KV head
 * g = h / 2 (two query heads share one KV head: the card's "num_groups = 2"):
 *
 *   x_j  = query_scale * (q[i,h,:] . k[j,g,:])
 *   s_j  = softcap * tanh(x_j / softcap)        (softcap == 0: s_j = x_j)
 *   key j is visible iff j <= p and (window == 0 or p - j < window)
 *   out[i,h,:] = sum_j softmax_j(s)_j * v[j,g,:]        over visible j
 *   lse[h,i]   = ln sum_{visible j} exp(s_j)
 *
 * window == 0 is a global layer (full causal span); window == W > 0 is a local
 * layer that keeps the W most recent keys, the query's own key included
 * (Gemma 2 uses W = 4096 on local layers and softcap = 50 on both).
 *
 * Common rules for every entry point:
 *  - Tensors q, k, v, out, caches are bf16, row-major, head dimension
 *    contiguous; lse is fp32. Every pointer is device memory owned by the
 *    caller; the library never allocates or frees device memory and keeps no
 *    pointer after the call returns. lse may be NULL (then it is not written).
 *  - d must be 64, 128 or 256; H must equal 2 * Hkv.
 *  - Tensor pointers must be 16-byte aligned.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream). Arguments are checked on the host before any launch; on an
 *    argument error nothing is launched and nothing is written.
 *  - The host never reads device memory; cu_seqlens arrays stay on the device.
 *  - Return value: a g2attn_status code.
 *  - Library state on the device: the sticky error word, the scratch array of
 *    g2attn_decode_noalloc, and the unit counters of the packed-sequence
 *    prefill launches (slot = the launch's grid id mod 4096; each launch's
 *    last CTA zeroes its slot, so concurrent launches only interfere if 4096
 *    of them are in flight at once).
 */
#ifndef G2ATTN_H
#define G2ATTN_H

#include <stddef.h>

#if defined(__GNUC__)
#define G2ATTN_API __attribute__((visibility("default")))
#else
#define G2ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* g2attn_stream_t; /* same type as cudaStream_t */

typedef enum {
    G2ATTN_OK = 0,
    G2ATTN_ERR_INVALID_ARG = 1,    /* a size, scale, cap or window is out of range */
    G2ATTN_ERR_UNSUPPORTED = 2,    /* d or H/Hkv outside what the kernels implement */
    G2ATTN_ERR_MISALIGNED = 3,     /* a tensor pointer is not 16-byte aligned */
    G2ATTN_ERR_CUDA = 4,           /* a CUDA runtime/driver call or launch failed */
    G2ATTN_ERR_DEVICE_TIMEOUT = 5, /* a kernel gave up waiting (see g2attn_get_device_error) */
    G2ATTN_ERR_WORKSPACE = 6,      /* a workspace NULL or smaller than required */
    G2ATTN_ERR_CACHE_LEN = 7       /* a decode sequence saw more keys than max_cache_len
                                      planned for (see g2attn_get_device_error) */
} g2attn_status;

/*
 * Dense prefill of one attention layer.
 *   q   (B, T, H, d)      queries of rows i = 0..T-1 at positions q_offset + i
 *   k,v (B, S, Hkv, d)    keys and values at positions 0..S-1
 *   out (B, T, H, d)      bf16 output
 *   lse (B, H, T)         fp32 natural-log log-sum-exp of the capped logits
 * Requires B, T, S >= 1, 0 <= q_offset, q_offset + T <= S, window >= 0,
 * finite query_scale, finite softcap >= 0.
 * Kernel choice (all three prefill calls): d = 256 launches clusters of two
 * CTAs sharing each K/V tile (tcgen05 .cta_group::2); the environment variable
 * G2ATTN_PREFILL_PAIR=0, read once per process, selects the single-CTA kernel
 * instead. d = 64 and 128 always use the single-CTA kernel. Both kernels
 * compute the same result.
 * Source: Gemma 2 card, "Method" (attention_layer pseudo-code: queries
 * (B,T,H,d), keys/values (B,S,K,d), K = H/2, cap 50, causal and 4096 window).
 */
G2ATTN_API int g2attn_prefill(const void* q, const void* k, const void* v, void* out, float* lse,
                   int B, int T, int S, int H, int Hkv, int d, int q_offset,
                   float query_scale, float softcap, int window, g2attn_stream_t stream);

/*
 * Packed variable-length prefill. Sequence s owns query rows
 * cu_seqlens_q[s] .. cu_seqlens_q[s+1]-1 and key rows cu_seqlens_k[s] ..
 * cu_seqlens_k[s+1]-1; with T_s and S_s its lengths, its queries sit at the
 * last T_s positions of its keys (q_offset_s = S_s - T_s; a chunked-prefill
 * tail has T_s < S_s). Each sequence is the dense layer above with B = 1.
 *   q   (total_q, H, d), k and v (total_k, Hkv, d), out like q,
 *   lse (H, total_q) fp32.
 *   cu_seqlens_q, cu_seqlens_k: device int32 arrays of num_seqs + 1 entries,
 *   non-decreasing, starting at 0, ending at total_q / total_k, with
 *   T_s <= S_s, T_s <= max_T and S_s <= max_S for every sequence (the kernel
 *   cannot check these; a violation gives undefined results, never an
 *   out-of-bounds access of q/k/v/out/lse, which are bounded by total_q/k).
 * total_q and total_k are the packed extents (the host does not read the
 * device arrays). Limit: num_seqs <= 1024 (the kernel ranks the sequences by
 * their work in a per-launch table in shared memory); more sequences return
 * G2ATTN_ERR_UNSUPPORTED.
 * Source: as g2attn_prefill; the packing is this library's.
 */
G2ATTN_API int g2attn_prefill_varlen(const void* q, const void* k, const void* v, void* out, float* lse,
                          const int* cu_seqlens_q, const int* cu_seqlens_k, int num_seqs,
                          int total_q, int total_k, int max_T, int max_S,
                          int H, int Hkv, int d, float query_scale, float softcap, int window,
                          g2attn_stream_t stream);

/*
 * Chunked prefill over a paged KV cache: queries packed as in
 * g2attn_prefill_varlen (cu_seqlens_q), keys and values read from fixed blocks
 * of block_size token rows through a per-sequence block table (the
 * block-managed caches of the serving runtimes the Guide names, "Deep Dive"
 * item 2). Sequence s has S_s = seq_lens_k[s] keys and T_s queries at its last
 * positions (q_offset_s = S_s - T_s).
 *   k_blocks, v_blocks (num_blocks, block_size, Hkv, d); block_table: device
 *   int32 [num_seqs][max_blocks_per_seq], entry b = cache block of key rows
 *   b*block_size .. b*block_size + block_size - 1; seq_lens_k: device int32
 *   [num_seqs] with T_s <= S_s <= max_S.
 *   Requires block_size a power of two >= 128 (every 128-key tile then lies in
 *   one block) and max_blocks_per_seq * block_size >= max_S. Rows of a sequence's
 *   last block beyond S_s must hold finite values (they meet zero weights).
 *   Table entries outside [0, num_blocks) are clamped and no table column past
 *   max_blocks_per_seq is read: malformed lengths or tables give undefined
 *   results, never an out-of-bounds access. out, lse, limits and errors as
 *   g2attn_prefill_varlen.
 */
G2ATTN_API int g2attn_prefill_paged(const void* q, const void* k_blocks, const void* v_blocks,
                         void* out, float* lse, const int* cu_seqlens_q,
                         const int* block_table, const int* seq_lens_k, int num_seqs,
                         int total_q, int num_blocks, int block_size, int max_blocks_per_seq,
                         int max_T, int max_S, int H, int Hkv, int d, float query_scale,
                         float softcap, int window, g2attn_stream_t stream);

/*
 * Bytes of device workspace g2attn_decode needs for these sizes (split-KV
 * partial results: per sequence, query head and split, a running max, a sum
 * and d accumulators, fp32). Depends only on the arguments.
 */
G2ATTN_API size_t g2attn_decode_workspace_size(int num_seqs, int H, int d, int max_cache_len);

/*
 * Decode: one new query per sequence over that sequence's KV cache.
 *   q (num_seqs, H, d); k_cache, v_cache (total_k, Hkv, d) packed by
 *   cu_seqlens_k (device int32, num_seqs + 1 entries, L_s = difference,
 *   1 <= L_s <= max_cache_len); the query of sequence s sits at position
 *   L_s - 1, so it sees keys max(0, L_s - window) .. L_s - 1 on a local
 *   layer and 0 .. L_s - 1 on a global one.
 *   out (num_seqs, H, d) bf16; lse (num_seqs, H) fp32.
 *   workspace: device memory of at least g2attn_decode_workspace_size(...)
 *   bytes, 16-byte aligned, owned by the caller; no initial contents needed.
 *   A sequence longer than max_cache_len (which the host cannot see) keeps
 *   only the splits the plan has room for: its output is wrong, nothing
 *   outside the buffers is touched, and g2attn_get_device_error reports
 *   G2ATTN_ERR_CACHE_LEN (all decode calls).
 * Source: the Guide's serving notes (local layers only need the last 4,096
 * cached tokens, "Interleaved Local Sliding Window and Global Attention").
 */
G2ATTN_API int g2attn_decode(const void* q, const void* k_cache, const void* v_cache,
                  const int* cu_seqlens_k, void* out, float* lse,
                  int num_seqs, int total_k, int max_cache_len, int H, int Hkv, int d,
                  float query_scale, float softcap, int window,
                  void* workspace, size_t workspace_bytes, g2attn_stream_t stream);

/*
 * Decode over a ring-buffer KV cache, for local layers: each sequence keeps only
 * its last ring_size cached tokens (the Guide's serving note: local layers
 * only store 4,096 tokens; the Hub page: the local layer's cache is bounded by
 * its window).
 *   q (num_seqs, H, d); k_ring, v_ring (num_seqs, ring_size, Hkv, d): position
 *   p of sequence s is in slot p mod ring_size of that sequence.
 *   seq_lens: device int32 [num_seqs], L_s >= 1 tokens seen so far; the query
 *   sits at position L_s - 1 and sees positions max(0, L_s - window) .. L_s - 1.
 *   Requires ring_size a power of two and 0 < window <= ring_size.
 *   max_cache_len: at least the keys any query sees (min(L_s, window)); it
 *   sizes the split plan and the workspace (g2attn_decode_workspace_size).
 *   out, lse, workspace and errors as g2attn_decode.
 */
G2ATTN_API int g2attn_decode_ring(const void* q, const void* k_ring, const void* v_ring,
                       const int* seq_lens, void* out, float* lse, int num_seqs, int ring_size,
                       int max_cache_len, int H, int Hkv, int d, float query_scale,
                       float softcap, int window, void* workspace, size_t workspace_bytes,
                       g2attn_stream_t stream);

/*
 * Decode over a paged KV cache: fixed blocks of block_size token rows, located
 * through a per-sequence block table (the block-managed caches of the serving
 * runtimes the Guide names, "Deep Dive" item 2).
 *   k_blocks, v_blocks (num_blocks, block_size, Hkv, d); block_table: device
 *   int32 [num_seqs][max_blocks_per_seq], entry b = cache block of positions
 *   b*block_size .. b*block_size + block_size - 1; seq_lens: device int32
 *   [num_seqs], L_s >= 1, L_s <= max_blocks_per_seq * block_size.
 *   Requires block_size a power of two. Table entries outside [0, num_blocks)
 *   are clamped (undefined results, never an out-of-bounds read).
 *   max_cache_len: at least the keys any query sees. Global (window 0) and
 *   local layers; out, lse, workspace and errors as g2attn_decode.
 */
G2ATTN_API int g2attn_decode_paged(const void* q, const void* k_blocks, const void* v_blocks,
                        const int* block_table, const int* seq_lens, void* out, float* lse,
                        int num_seqs, int num_blocks, int block_size, int max_blocks_per_seq,
                        int max_cache_len, int H, int Hkv, int d, float query_scale,
                        float softcap, int window, void* workspace, size_t workspace_bytes,
                        g2attn_stream_t stream);

/*
 * Decode without allocating: the same operation and arguments as
 * g2attn_decode, minus the workspace. For callers that cannot allocate device
 * memory at call time -- a serving loop whose device memory is planned up
 * front by another allocator, a plug-in that is handed only its input and
 * output pointers, or code that must not pay cudaMalloc's implicit device
 * synchronisation. The split-KV partial results go to a static scratch array
 * of 24 MiB inside the library, which every GPU that loads the library holds
 * until the process exits; this call never calls cudaMalloc, cudaFree or any
 * allocating routine. Inputs and outputs are still the caller's.
 *   - Rejects with G2ATTN_ERR_WORKSPACE (before any CUDA call) when
 *     g2attn_decode_workspace_size(num_seqs, H, d, max_cache_len) exceeds
 *     24 MiB (25165824 bytes).
 *   - The first call on each device looks up the scratch array's device
 *     address (cudaGetSymbolAddress) with that device current; make that
 *     first call before any stream capture. The address is cached per device
 *     and context: the first call after a cudaDeviceReset looks it up again
 *     (a reset gives the device a new context, in which the array may move).
 *   - Every call on a device shares the one scratch array and leaves its
 *     contents behind (nothing in it needs clearing: the kernels write every
 *     partial before reading it). Calls that overlap on the GPU -- on
 *     different streams, or from different host threads -- race on it and
 *     must be serialised by the caller.
 * The Gemma 2 pages have no counterpart to this entry point.
 */
G2ATTN_API int g2attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                          const int* cu_seqlens_k, void* out, float* lse,
                          int num_seqs, int total_k, int max_cache_len, int H, int Hkv, int d,
                          float query_scale, float softcap, int window, g2attn_stream_t stream);

/*
 * Bytes of device workspace g2attn_prefill_backward needs: two fp32 values
 * (lse in log2 units and D = dout . out) per (b, h, query position), the
 * positions rounded up to a multiple of 64. 0 for non-positive arguments.
 */
G2ATTN_API size_t g2attn_backward_workspace_size(int B, int T, int H);

/*
 * Gradients of g2attn_prefill (same q, k, v, sizes and parameters) for the
 * upstream gradient dout of its output. The chain rule runs through the value
 * mix, the softmax, the soft-cap (derivative 1 - tanh^2(x/C) of C tanh(x/C),
 * "Gemma 2 Guide", Deep Dive item 1; none when softcap = 0) and the scaled
 * dot product; dk and dv sum over the two query heads sharing a KV head.
 *   out (B,T,H,d) bf16 and lse (B,H,T) fp32: the forward's outputs for these
 *     inputs (the softmax weights are recomputed from lse, not stored).
 *   dout (B,T,H,d) bf16; dq (B,T,H,d), dk and dv (B,S,Hkv,d) bf16, written in
 *     full (keys that no query sees get zero gradients).
 *   workspace: device memory of at least
 *     g2attn_backward_workspace_size(B, T, H) bytes, 16-byte aligned, owned by
 *     the caller and overwritten: -lse*log2(e) and -D per (b, h, position),
 *     then the two gradient kernels' unit counters (the CTAs take their units
 *     in order from a counter, longest first; the first pass zeroes them).
 * Supported: d = 64, 128 and 256. At d = 256 one of the two resident tiles of
 * each gradient kernel is held in tensor memory (it is read by the UMMAs as
 * their A operand), the streamed tiles are 64 rows, and the dk/dv kernel runs
 * each 128-key tile as two units, one accumulating dv and one dk, so that an
 * accumulator fits the 512 TMEM columns of an SM next to X and Y.
 * Other limits and errors as g2attn_prefill; lse is required; a workspace that
 * is missing or too small returns G2ATTN_ERR_WORKSPACE. Three kernels run on
 * `stream`: a pass computing D and lse*log2(e), the dk/dv kernel (K, V tiles
 * resident, query tiles streamed) and the dq kernel (query tiles resident).
 * Source: the Gemma 2 card's "Method" pseudo-code (the forward being
 * differentiated) and the Guide's derivative of the cap.
 */
G2ATTN_API int g2attn_prefill_backward(const void* q, const void* k, const void* v,
                            const void* out, const float* lse, const void* dout, void* dq,
                            void* dk, void* dv, int B, int T, int S, int H, int Hkv, int d,
                            int q_offset, float query_scale, float softcap, int window,
                            void* workspace, size_t workspace_bytes, g2attn_stream_t stream);

/*
 * Bytes of device workspace g2attn_prefill_varlen_backward needs: -lse*log2(e)
 * and -D per (head, query position) with every sequence padded to a multiple
 * of 64 positions (bounded by total_q + 64*num_seqs per head), plus
 * num_seqs + 1 ints. 0 for non-positive arguments.
 */
G2ATTN_API size_t g2attn_varlen_backward_workspace_size(int num_seqs, int total_q, int H);

/*
 * Gradients of g2attn_prefill_varlen: the packed layout, cu_seqlens and limits
 * of that call, with out and lse its outputs (lse (H, total_q) fp32) and dout
 * packed like q.
 *   dq like q, dk and dv like k and v (bf16), written in full.
 *   workspace: at least g2attn_varlen_backward_workspace_size(num_seqs,
 *     total_q, H) bytes, 16-byte aligned, overwritten (per-row vectors, the
 *     padded prefix of the sequences, the unit counters).
 * Sequence rows derived from cu_seqlens are clamped into [0, total_q) and
 * [0, total_k): malformed offsets give undefined results but no access
 * outside the tensors. Supported: d = 64, 128 and 256; num_seqs <= 1024.
 * Other errors as g2attn_prefill_backward. Four kernels run on `stream`: the
 * padded-prefix and D passes, the dk/dv kernel and the dq kernel.
 * Source: as g2attn_prefill_backward; the packing is this library's.
 */
G2ATTN_API int g2attn_prefill_varlen_backward(const void* q, const void* k, const void* v,
                                   const void* out, const float* lse, const void* dout,
                                   void* dq, void* dk, void* dv, const int* cu_seqlens_q,
                                   const int* cu_seqlens_k, int num_seqs, int total_q,
                                   int total_k, int max_T, int max_S, int H, int Hkv, int d,
                                   float query_scale, float softcap, int window, void* workspace,
                                   size_t workspace_bytes, g2attn_stream_t stream);

/* Human-readable name of a status code (static storage). */
G2ATTN_API const char* g2attn_status_string(int status);

/*
 * Sticky device-side error word of the current device. It is set when a
 * kernel gave up on a bounded wait, and when a decode call (any cache layout)
 * met a sequence whose visible keys need more splits than its max_cache_len
 * planned for: that call still returned G2ATTN_OK and stayed inside its
 * buffers, but dropped the keys past the plan, so its output for that
 * sequence is wrong. Reading the word synchronizes the device and clears it.
 * Returns G2ATTN_OK when clear, G2ATTN_ERR_DEVICE_TIMEOUT when a wait gave up
 * (this takes precedence), G2ATTN_ERR_CACHE_LEN when only the decode
 * precondition was broken, G2ATTN_ERR_CUDA if the word cannot be read.
 */
G2ATTN_API int g2attn_get_device_error(void);

/*
 * Self-test of the bounded-wait machinery: launches one tiny kernel that waits
 * on a shared-memory barrier nothing will ever complete, with a limit of
 * timeout_us microseconds (1..1000000), then reads and clears the device
 * error word. Returns G2ATTN_ERR_DEVICE_TIMEOUT when the wait gave up as it
 * should (the GPU context stays usable), another code otherwise. No fault,
 * trap or hang is involved.
 */
G2ATTN_API int g2attn_selftest_wait_timeout(int timeout_us);

#ifdef __cplusplus
}
#endif
#endif /* G2ATTN_H */
