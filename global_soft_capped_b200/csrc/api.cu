// api.cu -- C ABI of libg2attn (declared in include/g2attn.h): argument
// checks, TMA descriptor encoding, launch configuration and the kernels
// (compiled as one translation unit so the device error word is unique).
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#include <algorithm>
#include <mutex>

#include "../../include/g2attn.h"
#include "common.cuh"
#include "decode.cuh"
#include "prefill_sm100.cuh"
#include "backward_sm100.cuh"

// Scratch of g2attn_decode_noalloc (see there): 24 MiB, reserved on every GPU
// that loads the library until the process exits.
constexpr size_t kNoAllocScratchBytes = 24u << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------
// Host-side helpers
// ---------------------------------------------------------------------------
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool finite_f(float x) { return isfinite(x) != 0; }

unsigned long long wait_limit_ns() {
    // Bounded waits inside the kernels give up after this long (default 4 s).
    static unsigned long long v = [] {
        const char* e = getenv("G2ATTN_WAIT_TIMEOUT_US");
        unsigned long long us = e ? strtoull(e, nullptr, 10) : 0ull;
        if (us == 0ull) us = 4000000ull;
        return us * 1000ull;
    }();
    return v;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 3-D bf16 tensor map over a packed (rows, heads, d) tensor, viewed as
// {d, rows, heads} so one box covers `box_rows` rows of `box_heads` heads.
bool make_map(CUtensorMap* map, const void* ptr, int d, long long rows, int heads, int box_rows,
              int box_heads) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows),
                          static_cast<cuuint64_t>(heads)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(heads) * d * 2,  // next row
                             static_cast<cuuint64_t>(d) * 2};         // next head
    cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(box_rows), static_cast<cuuint32_t>(box_heads)};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    return n;
}

void fill_cap(float query_scale, float softcap, float& k_exp, float& cap_l2, float& scale_l2,
              int& has_cap) {
    has_cap = softcap > 0.f;
    k_exp = has_cap ? 2.0f * query_scale * kLog2e / softcap : 0.f;
    cap_l2 = has_cap ? softcap * kLog2e : 0.f;
    scale_l2 = query_scale * kLog2e;
}

void fill_poly(float query_scale, float softcap, g2::PfParams& P) {
    // fixed softmax shift when the cap bounds every logit tightly enough
    P.fixed_ref_on = softcap > 0.f && softcap * kLog2e <= g2::PF_FIXED_REF_MAX;
    P.fixed_ref = P.fixed_ref_on ? softcap * kLog2e - 64.0f : 0.f;
    P.u_scale = softcap > 0.f ? query_scale / softcap : 0.f;
    const float a = fabsf(query_scale);
    P.poly_acc_max = (softcap > 0.f && a > 0.f) ? g2::PF_POLY_U_MAX * softcap / a : INFINITY;
    // The series path runs in powers of the raw accumulator with the factors
    // (alpha/C)^(2k) folded into its coefficients; use it only while the
    // smallest folded coefficient is a comfortably normal float.
    if (softcap > 0.f && a > 0.f) {
        const float us2 = P.u_scale * P.u_scale;
        const float b3 = fabsf(query_scale * kLog2e * (17.0f / 315.0f) * us2 * us2 * us2);
        if (!(b3 > 1e-30f) || !isfinite(b3) || !isfinite(P.poly_acc_max)) P.poly_acc_max = 0.f;
    }
}

// CG = 2 launches clusters of two CTAs (one unit of 128 query positions per
// pair); the grid holds as many pairs as can be resident at once.
template <int D, int CG, int SM>
int launch_prefill_kernel(const void* q, const void* k, const void* v, long long total_q,
                          long long total_k, g2::PfParams& P, cudaStream_t stream) {
    using C = g2::PfCfg<D, CG>;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, D, total_q, P.H, g2::PF_QPOS, 2) ||
        !make_map(&mk, k, D, total_k, P.Hkv, C::KROWS, 1) ||
        !make_map(&mv, v, D, total_k, P.Hkv, C::VROWS, 1))
        return G2ATTN_ERR_CUDA;
    const int sms = num_sms();
    if (sms <= 0) return G2ATTN_ERR_CUDA;
    auto kern = g2::prefill_fwd_sm100<D, CG, SM>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
        cudaSuccess)
        return G2ATTN_ERR_CUDA;
    if (CG == 1) {
        const int grid = P.num_units < sms ? P.num_units : sms;
        kern<<<grid, g2::PF_THREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, P);
        return cudaGetLastError() == cudaSuccess ? G2ATTN_OK : G2ATTN_ERR_CUDA;
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CG;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(g2::PF_THREADS, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    static int pairs_resident = -1;  // per process: one device type
    if (pairs_resident < 0) {
        cfg.gridDim = dim3(CG * (sms / CG), 1, 1);
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0)
            return G2ATTN_ERR_CUDA;
        pairs_resident = n;
    }
    const int pairs = P.num_units < pairs_resident ? P.num_units : pairs_resident;
    cfg.gridDim = dim3(CG * pairs, 1, 1);
    if (cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, P) != cudaSuccess) return G2ATTN_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? G2ATTN_OK : G2ATTN_ERR_CUDA;
}

// The softmax variant the parameters call for: the fixed shift whenever it
// is on (see PfParams::fixed_ref_on), else the running max with or without
// the cap.
template <int D, int CG>
int launch_prefill(const void* q, const void* k, const void* v, long long total_q,
                   long long total_k, g2::PfParams& P, cudaStream_t stream) {
    if (P.fixed_ref_on)
        return launch_prefill_kernel<D, CG, g2::PF_SM_FIXED>(q, k, v, total_q, total_k, P, stream);
    if (P.has_cap)
        return launch_prefill_kernel<D, CG, g2::PF_SM_CAP>(q, k, v, total_q, total_k, P, stream);
    return launch_prefill_kernel<D, CG, g2::PF_SM_NOCAP>(q, k, v, total_q, total_k, P, stream);
}

// d = 256 runs on CTA pairs unless G2ATTN_PREFILL_PAIR=0 selects the
// single-CTA kernel (read once per process).
bool use_pairs() {
    static bool v = [] {
        const char* e = getenv("G2ATTN_PREFILL_PAIR");
        return !(e != nullptr && e[0] == '0');
    }();
    return v;
}

int dispatch_prefill(int d, const void* q, const void* k, const void* v, long long tq,
                     long long tk, g2::PfParams& P, cudaStream_t st) {
    switch (d) {
        case 64: return launch_prefill<64, 1>(q, k, v, tq, tk, P, st);
        case 128: return launch_prefill<128, 1>(q, k, v, tq, tk, P, st);
        case 256:
            if (use_pairs()) {
                // units of 128 query positions (varlen: the kernel counts them
                // itself; the single-CTA count stays a valid upper bound)
                if (!P.varlen) {
                    P.max_units_per_seq_tiles = (P.T + 2 * g2::PF_QPOS - 1) / (2 * g2::PF_QPOS);
                    P.num_units = P.max_units_per_seq_tiles * P.num_seqs * P.Hkv;
                }
                return launch_prefill<256, 2>(q, k, v, tq, tk, P, st);
            }
            return launch_prefill<256, 1>(q, k, v, tq, tk, P, st);
        default: return G2ATTN_ERR_UNSUPPORTED;
    }
}

int check_common(int H, int Hkv, int d, float query_scale, float softcap, int window) {
    if (H <= 0 || Hkv <= 0) return G2ATTN_ERR_INVALID_ARG;
    if (!finite_f(query_scale) || !finite_f(softcap) || softcap < 0.f || window < 0)
        return G2ATTN_ERR_INVALID_ARG;
    if (H != 2 * Hkv) return G2ATTN_ERR_UNSUPPORTED;
    if (d != 64 && d != 128 && d != 256) return G2ATTN_ERR_UNSUPPORTED;
    return G2ATTN_OK;
}

// Decode split plan: chunk of keys per CTA. Depends only on the sizes, so the
// workspace size query and the launch agree without a device query.
int decode_chunk(int num_seqs, int H, int max_len) {
    int chunk = g2::DEC_MAX_CHUNK;
    const long long kv_heads = static_cast<long long>(num_seqs) * (H / 2 > 0 ? H / 2 : 1);
    while (chunk > 64 && kv_heads * ((max_len + chunk - 1) / chunk) < 1184) chunk >>= 1;
    return chunk;
}

size_t decode_ws_bytes(int num_seqs, int H, int d, int max_len, int chunk) {
    const size_t splits = static_cast<size_t>((max_len + chunk - 1) / chunk);
    const size_t slots = static_cast<size_t>(num_seqs) * H * splits;
    size_t ml = slots * 2 * sizeof(float);
    ml = (ml + 255) & ~static_cast<size_t>(255);
    return ml + slots * static_cast<size_t>(d) * sizeof(float);
}

template <int D, int LAYOUT>
int launch_decode(g2::DecParams& P, const g2::DecLayoutParams& LP, cudaStream_t stream) {
    dim3 grid(P.max_splits, P.Hkv, P.num_seqs);
    // ring / paged layouts: per-CTA table of the chunk's cache rows
    const size_t dyn = (LAYOUT == g2::DEC_LINEAR) ? 0 : static_cast<size_t>(P.chunk) * sizeof(int);
    g2::decode_split<D, LAYOUT><<<grid, g2::DEC_THREADS, dyn, stream>>>(P, LP);
    if (cudaGetLastError() != cudaSuccess) return G2ATTN_ERR_CUDA;
    const int warps = P.num_seqs * P.H;
    g2::decode_merge<D, LAYOUT><<<(warps + 3) / 4, 128, 0, stream>>>(P, LP);
    return cudaGetLastError() == cudaSuccess ? G2ATTN_OK : G2ATTN_ERR_CUDA;
}

bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

int log2i(int x) {
    int r = 0;
    while ((1 << r) < x) ++r;
    return r;
}

// Checks shared by every decode layout, then the split plan and workspace
// carving; launches the layout's kernels on success.
template <int LAYOUT>
int decode_common(g2::DecParams& P, const g2::DecLayoutParams& LP, const void* q, const void* k_cache, const void* v_cache,
                  void* out, float* lse, int num_seqs, int max_cache_len, int H, int Hkv, int d,
                  float query_scale, float softcap, int window, void* workspace,
                  size_t workspace_bytes, g2attn_stream_t stream) {
    if (!q || !k_cache || !v_cache || !out) return G2ATTN_ERR_INVALID_ARG;
    if (num_seqs <= 0 || max_cache_len <= 0) return G2ATTN_ERR_INVALID_ARG;
    int rc = check_common(H, Hkv, d, query_scale, softcap, window);
    if (rc) return rc;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        (lse && !aligned16(lse)) || (workspace && !aligned16(workspace)))
        return G2ATTN_ERR_MISALIGNED;
    const int chunk = decode_chunk(num_seqs, H, max_cache_len);
    const size_t need = decode_ws_bytes(num_seqs, H, d, max_cache_len, chunk);
    if (!workspace || workspace_bytes < need) return G2ATTN_ERR_WORKSPACE;
    P.q = static_cast<const __nv_bfloat16*>(q);
    P.k = static_cast<const __nv_bfloat16*>(k_cache);
    P.v = static_cast<const __nv_bfloat16*>(v_cache);
    P.out = static_cast<__nv_bfloat16*>(out);
    P.lse = lse;
    const int splits = (max_cache_len + chunk - 1) / chunk;
    size_t ml = static_cast<size_t>(num_seqs) * H * splits * 2 * sizeof(float);
    ml = (ml + 255) & ~static_cast<size_t>(255);
    P.ws_ml = static_cast<float*>(workspace);
    P.ws_acc = reinterpret_cast<float*>(static_cast<char*>(workspace) + ml);
    P.num_seqs = num_seqs;
    P.H = H;
    P.Hkv = Hkv;
    P.window = window;
    P.chunk = chunk;
    // a local layer sees at most `window` keys per sequence: no more splits than
    // that range needs (the workspace, sized for max_cache_len, stays large enough)
    P.max_splits = window > 0 ? std::min(splits, (window + chunk - 1) / chunk) : splits;
    fill_cap(query_scale, softcap, P.k_exp, P.cap_l2, P.scale_l2, P.has_cap);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    switch (d) {
        case 64: return launch_decode<64, LAYOUT>(P, LP, st);
        case 128: return launch_decode<128, LAYOUT>(P, LP, st);
        case 256: return launch_decode<256, LAYOUT>(P, LP, st);
        default: return G2ATTN_ERR_UNSUPPORTED;
    }
}

__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        g2::mbar_init(&bar, 1);
        abort_flag = 0;
        g2::fence_mbar_init();
    }
    __syncthreads();
    // Nothing ever arrives on `bar`: the wait must give up after limit_ns.
    if (threadIdx.x == 0)
        g2::mbar_wait(&bar, 0, &abort_flag, limit_ns, g2::SITE_SELFTEST);
    __syncthreads();
}

// ---------------------------------------------------------------------------
// Decode without any allocation: the split-KV partial results live in this
// file-scope device array instead of a caller-provided workspace. It is
// reserved on every GPU that loads the library, for the life of the process.
// ---------------------------------------------------------------------------
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};
unsigned long long g_noalloc_ctx[kMaxDevices] = {};  // context the address belongs to

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the current context (ids are never reused within a process),
// or 0 when there is no current context or the driver lacks the call.
unsigned long long current_ctx_id() {
    static CtxGetCurrentFn get_cur = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_cur || !get_id || get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
    if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of g_noalloc_scratch on the current device. The host-side
// name of the array is only a stand-in, so the address is looked up with the
// device current, once per device and context: after cudaDeviceReset the
// device gets a new context, the library's module is loaded again and the
// array may sit elsewhere, so a changed context id triggers a new lookup.
int noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return G2ATTN_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    const unsigned long long ctx = current_ctx_id();
    if (g_noalloc_ptr[dev] == nullptr || ctx == 0 || ctx != g_noalloc_ctx[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
            return G2ATTN_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
        // the lookup makes the device's context current if none was
        g_noalloc_ctx[dev] = ctx != 0 ? ctx : current_ctx_id();
    }
    *out = g_noalloc_ptr[dev];
    return G2ATTN_OK;
}

// The gradients' series for tanh(u), u = alpha x / C, |u| <= 1/4: the same
// window as the forward's fast path, with the coefficients of the Taylor
// series (1, -1/3, 2/15, -17/315) times (alpha/C)^(2k+1) so that the kernels
// evaluate it in powers of the raw accumulator x. Off when the smallest folded
// coefficient is not a comfortably normal float.
void fill_bwd_series(float query_scale, float softcap, g2::BwParams& P) {
    g2::PfParams F{};
    fill_poly(query_scale, softcap, F);
    P.u_scale = F.u_scale;
    P.poly_acc_max = F.poly_acc_max;
    const float us = F.u_scale, us2 = us * us;
    const float c[4] = {1.0f, -1.0f / 3.0f, 2.0f / 15.0f, -17.0f / 315.0f};
    float pw = us;
    for (int i = 0; i < 4; ++i) {
        P.th_c[i] = c[i] * pw;
        pw *= us2;
    }
    if (!(fabsf(P.th_c[3]) > 1e-30f) || !isfinite(P.th_c[3]) || !isfinite(P.th_c[0]))
        P.poly_acc_max = 0.f;
}

// Backward: query-side positions padded to whole 64-position tiles in the
// workspace (-lse*log2(e) and -D, fp32 each).
long long bwd_tp(int T) { return (static_cast<long long>(T) + 63) / 64 * 64; }

// Then a 256-byte block holding the unit counters of the two gradient kernels
// (zeroed by the pass that runs before them).
constexpr size_t kBwdSchedBytes = 256;

size_t bwd_ws_rows_bytes(int B, int T, int H) {
    return 2ull * static_cast<size_t>(B) * static_cast<size_t>(H) * bwd_tp(T) * sizeof(float);
}

size_t bwd_ws_bytes(int B, int T, int H) {
    const size_t rows = bwd_ws_rows_bytes(B, T, H);
    return rows == 0 ? 0 : rows + kBwdSchedBytes;
}

template <int D, int MODE, bool CAP>
int launch_bwd_kernel(const CUtensorMap& mq, const CUtensorMap& mo, const CUtensorMap& mk,
                      const CUtensorMap& mv, g2::BwParams P, int units, int sms, cudaStream_t st) {
    using C = g2::BwCfg<D>;
    auto kern = g2::bwd_sm100<D, MODE, CAP>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
        cudaSuccess)
        return G2ATTN_ERR_CUDA;
    P.num_units = units;
    const int grid = units < sms ? units : sms;
    kern<<<grid, g2::BW_THREADS, C::SMEM_BYTES, st>>>(mq, mo, mk, mv, P);
    return cudaGetLastError() == cudaSuccess ? G2ATTN_OK : G2ATTN_ERR_CUDA;
}

// The capped or the uncapped instantiation, as the parameters say.
template <int D, int MODE>
int launch_bwd(const CUtensorMap& mq, const CUtensorMap& mo, const CUtensorMap& mk,
               const CUtensorMap& mv, g2::BwParams P, int units, int sms, cudaStream_t st) {
    return P.has_cap ? launch_bwd_kernel<D, MODE, true>(mq, mo, mk, mv, P, units, sms, st)
                     : launch_bwd_kernel<D, MODE, false>(mq, mo, mk, mv, P, units, sms, st);
}

// Tensor maps of the two gradient kernels: the dk/dv kernel keeps 128-key K/V
// tiles and streams CQ-position q/dout tiles; the dq kernel keeps 64-position
// q/dout tiles and streams CK-key K/V tiles (both heads of a group per q box).
struct BwMaps {
    CUtensorMap q_kv, o_kv, k_kv, v_kv;  // dk/dv kernel
    CUtensorMap q_q, o_q, k_q, v_q;      // dq kernel
};

template <int D>
bool make_bw_maps(BwMaps& m, const void* q, const void* k, const void* v, const void* dout,
                  long long tq, long long tk, int H, int Hkv) {
    using C = g2::BwCfg<D>;
    return make_map(&m.q_kv, q, D, tq, H, C::CQ, 2) && make_map(&m.o_kv, dout, D, tq, H, C::CQ, 2) &&
           make_map(&m.k_kv, k, D, tk, Hkv, g2::BW_KEYS, 1) &&
           make_map(&m.v_kv, v, D, tk, Hkv, g2::BW_KEYS, 1) &&
           make_map(&m.q_q, q, D, tq, H, g2::BW_QPOS, 2) &&
           make_map(&m.o_q, dout, D, tq, H, g2::BW_QPOS, 2) &&
           make_map(&m.k_q, k, D, tk, Hkv, C::CK, 1) && make_map(&m.v_q, v, D, tk, Hkv, C::CK, 1);
}

template <int D>
int launch_backward(const void* q, const void* k, const void* v, const void* out,
                    const float* lse, const void* dout, g2::BwParams& P, cudaStream_t st) {
    BwMaps m;
    const long long tq = static_cast<long long>(P.B) * P.T, tk = static_cast<long long>(P.B) * P.S;
    if (!make_bw_maps<D>(m, q, k, v, dout, tq, tk, P.H, P.Hkv)) return G2ATTN_ERR_CUDA;
    const int sms = num_sms();
    if (sms <= 0) return G2ATTN_ERR_CUDA;
    // -D = -(dout . out) and -lse * log2(e) per (b, h, position)
    const long long rows = static_cast<long long>(P.B) * P.H * P.Tp;
    const long long threads = rows * (D / 8);
    // the unit counters follow the rows in the workspace
    unsigned int* sched = reinterpret_cast<unsigned int*>(
        reinterpret_cast<char*>(const_cast<float*>(P.nlse2)) + bwd_ws_rows_bytes(P.B, P.T, P.H));
    const long long blocks = (threads + 255) / 256;
    if (blocks > INT32_MAX) return G2ATTN_ERR_UNSUPPORTED;
    g2::bwd_prep<D><<<static_cast<int>(blocks), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(dout), lse,
        const_cast<float*>(P.nlse2), const_cast<float*>(P.ndvec), P.B, P.T, P.H, P.Tp, sched);
    if (cudaGetLastError() != cudaSuccess) return G2ATTN_ERR_CUDA;
    const int BG = P.B * P.Hkv;
    const int key_tiles = (P.S + g2::BW_KEYS - 1) / g2::BW_KEYS;
    const int q_tiles = (P.T + g2::BW_QPOS - 1) / g2::BW_QPOS;
    P.row_tiles = key_tiles;
    const long long kv_units = static_cast<long long>(key_tiles) * BG * g2::BwCfg<D>::DSPLIT_KV;
    if (kv_units > INT32_MAX) return G2ATTN_ERR_UNSUPPORTED;
    P.sched = sched;
    int rc = launch_bwd<D, g2::BW_KV>(m.q_kv, m.o_kv, m.k_kv, m.v_kv, P,
                                      static_cast<int>(kv_units), sms, st);
    if (rc) return rc;
    P.row_tiles = q_tiles;
    P.sched = sched + 1;
    return launch_bwd<D, g2::BW_Q>(m.q_q, m.o_q, m.k_q, m.v_q, P, q_tiles * BG, sms, st);
}

// Varlen backward workspace: -lse2 and -D as (H, wmax) fp32 each, then the
// int prefix wq[num_seqs + 1]. wmax bounds the padded query count.
long long bwd_vl_wmax(int num_seqs, int total_q) {
    return (static_cast<long long>(total_q) + 64ll * num_seqs + 63) / 64 * 64;
}

size_t bwd_vl_ws_head_bytes(int num_seqs, int total_q, int H) {
    const size_t b = 2ull * H * bwd_vl_wmax(num_seqs, total_q) * sizeof(float) +
                     (static_cast<size_t>(num_seqs) + 1) * sizeof(int);
    return (b + kBwdSchedBytes - 1) / kBwdSchedBytes * kBwdSchedBytes;
}

size_t bwd_vl_ws_bytes(int num_seqs, int total_q, int H) {
    return bwd_vl_ws_head_bytes(num_seqs, total_q, H) + kBwdSchedBytes;
}

template <int D>
int launch_backward_varlen(const void* q, const void* k, const void* v, const void* out,
                           const float* lse, const void* dout, int total_q, int total_k,
                           g2::BwParams& P, cudaStream_t st) {
    BwMaps m;
    if (!make_bw_maps<D>(m, q, k, v, dout, total_q, total_k, P.H, P.Hkv)) return G2ATTN_ERR_CUDA;
    const int sms = num_sms();
    if (sms <= 0) return G2ATTN_ERR_CUDA;
    unsigned int* sched = reinterpret_cast<unsigned int*>(
        reinterpret_cast<char*>(const_cast<float*>(P.nlse2)) +
        bwd_vl_ws_head_bytes(P.num_seqs, total_q, P.H));
    g2::bwd_wq_prefix<<<1, 32, 0, st>>>(P.cu_q, P.num_seqs, total_q, const_cast<int*>(P.wq),
                                       sched);
    if (cudaGetLastError() != cudaSuccess) return G2ATTN_ERR_CUDA;
    const long long threads = static_cast<long long>(P.H) * P.wmax * (D / 8);
    const long long blocks = (threads + 255) / 256;
    if (blocks > INT32_MAX) return G2ATTN_ERR_UNSUPPORTED;
    g2::bwd_prep_varlen<D><<<static_cast<int>(blocks), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(dout), lse,
        P.cu_q, P.wq, const_cast<float*>(P.nlse2), const_cast<float*>(P.ndvec), P.num_seqs, P.H,
        total_q, P.wmax);
    if (cudaGetLastError() != cudaSuccess) return G2ATTN_ERR_CUDA;
    // Units are counted on the device from cu_seqlens; the grids come from
    // upper bounds and surplus units are skipped by the kernels.
    const long long kv_ub = (static_cast<long long>(total_k) / g2::BW_KEYS + P.num_seqs) * P.Hkv *
                            g2::BwCfg<D>::DSPLIT_KV;
    const long long q_ub = (static_cast<long long>(total_q) / g2::BW_QPOS + P.num_seqs) * P.Hkv;
    if (kv_ub > INT32_MAX || q_ub > INT32_MAX) return G2ATTN_ERR_UNSUPPORTED;
    P.sched = sched;
    int rc = launch_bwd<D, g2::BW_KV>(m.q_kv, m.o_kv, m.k_kv, m.v_kv, P, static_cast<int>(kv_ub),
                                      sms, st);
    if (rc) return rc;
    P.sched = sched + 1;
    return launch_bwd<D, g2::BW_Q>(m.q_q, m.o_q, m.k_q, m.v_q, P, static_cast<int>(q_ub), sms, st);
}

}  // namespace

extern "C" {

size_t g2attn_varlen_backward_workspace_size(int num_seqs, int total_q, int H) {
    if (num_seqs <= 0 || total_q <= 0 || H <= 0) return 0;
    return bwd_vl_ws_bytes(num_seqs, total_q, H);
}

int g2attn_prefill_varlen_backward(const void* q, const void* k, const void* v, const void* out,
                                   const float* lse, const void* dout, void* dq, void* dk,
                                   void* dv, const int* cu_seqlens_q, const int* cu_seqlens_k,
                                   int num_seqs, int total_q, int total_k, int max_T, int max_S,
                                   int H, int Hkv, int d, float query_scale, float softcap,
                                   int window, void* workspace, size_t workspace_bytes,
                                   g2attn_stream_t stream) {
    if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv || !cu_seqlens_q ||
        !cu_seqlens_k)
        return G2ATTN_ERR_INVALID_ARG;
    if (num_seqs <= 0 || total_q <= 0 || total_k <= 0 || max_T <= 0 || max_S <= 0 ||
        max_T > max_S || max_T > total_q || max_S > total_k)
        return G2ATTN_ERR_INVALID_ARG;
    int rc = check_common(H, Hkv, d, query_scale, softcap, window);
    if (rc) return rc;
    if (num_seqs > g2::BwCfg<64>::MAX_SEQ_TABLE) return G2ATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse) ||
        !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
        (reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) ||
        (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u))
        return G2ATTN_ERR_MISALIGNED;
    if (static_cast<long long>(H) * bwd_vl_wmax(num_seqs, total_q) > INT32_MAX)
        return G2ATTN_ERR_UNSUPPORTED;
    if (!workspace || workspace_bytes < bwd_vl_ws_bytes(num_seqs, total_q, H))
        return G2ATTN_ERR_WORKSPACE;
    if (!aligned16(workspace)) return G2ATTN_ERR_MISALIGNED;
    g2::BwParams P{};
    P.dq = static_cast<__nv_bfloat16*>(dq);
    P.dk = static_cast<__nv_bfloat16*>(dk);
    P.dv = static_cast<__nv_bfloat16*>(dv);
    P.q = static_cast<const __nv_bfloat16*>(q);
    P.k = static_cast<const __nv_bfloat16*>(k);
    P.v = static_cast<const __nv_bfloat16*>(v);
    P.B = 1;
    P.T = max_T;
    P.S = max_S;
    P.H = H;
    P.Hkv = Hkv;
    P.window = window;
    P.varlen = 1;
    P.num_seqs = num_seqs;
    P.cu_q = cu_seqlens_q;
    P.cu_k = cu_seqlens_k;
    P.total_q = total_q;
    P.total_k = total_k;
    P.wmax = static_cast<int>(bwd_vl_wmax(num_seqs, total_q));
    float* ws = static_cast<float*>(workspace);
    P.nlse2 = ws;
    P.ndvec = ws + static_cast<size_t>(H) * P.wmax;
    P.wq = reinterpret_cast<const int*>(ws + 2 * static_cast<size_t>(H) * P.wmax);
    int has_cap = 0;
    fill_cap(query_scale, softcap, P.k_exp, P.cap_l2, P.scale_l2, has_cap);
    P.has_cap = has_cap;
    P.query_scale = query_scale;
    fill_bwd_series(query_scale, softcap, P);
    P.timeout_ns = wait_limit_ns();
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (d == 64)
        return launch_backward_varlen<64>(q, k, v, out, lse, dout, total_q, total_k, P, st);
    if (d == 128)
        return launch_backward_varlen<128>(q, k, v, out, lse, dout, total_q, total_k, P, st);
    return launch_backward_varlen<256>(q, k, v, out, lse, dout, total_q, total_k, P, st);
}

size_t g2attn_backward_workspace_size(int B, int T, int H) {
    if (B <= 0 || T <= 0 || H <= 0) return 0;
    return bwd_ws_bytes(B, T, H);
}

int g2attn_prefill_backward(const void* q, const void* k, const void* v, const void* out,
                            const float* lse, const void* dout, void* dq, void* dk, void* dv,
                            int B, int T, int S, int H, int Hkv, int d, int q_offset,
                            float query_scale, float softcap, int window, void* workspace,
                            size_t workspace_bytes, g2attn_stream_t stream) {
    if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv)
        return G2ATTN_ERR_INVALID_ARG;
    if (B <= 0 || T <= 0 || S <= 0 || q_offset < 0 ||
        static_cast<long long>(q_offset) + T > S)
        return G2ATTN_ERR_INVALID_ARG;
    int rc = check_common(H, Hkv, d, query_scale, softcap, window);
    if (rc) return rc;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse) ||
        !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return G2ATTN_ERR_MISALIGNED;
    const long long tq = static_cast<long long>(B) * T, tk = static_cast<long long>(B) * S;
    if (tq > INT32_MAX || tk > INT32_MAX || static_cast<long long>(B) * H * bwd_tp(T) > INT32_MAX)
        return G2ATTN_ERR_UNSUPPORTED;
    if (!workspace || workspace_bytes < bwd_ws_bytes(B, T, H)) return G2ATTN_ERR_WORKSPACE;
    if (!aligned16(workspace)) return G2ATTN_ERR_MISALIGNED;
    g2::BwParams P{};
    P.dq = static_cast<__nv_bfloat16*>(dq);
    P.dk = static_cast<__nv_bfloat16*>(dk);
    P.dv = static_cast<__nv_bfloat16*>(dv);
    P.q = static_cast<const __nv_bfloat16*>(q);
    P.k = static_cast<const __nv_bfloat16*>(k);
    P.v = static_cast<const __nv_bfloat16*>(v);
    P.B = B;
    P.T = T;
    P.S = S;
    P.H = H;
    P.Hkv = Hkv;
    P.Tp = static_cast<int>(bwd_tp(T));
    P.q_offset = q_offset;
    P.window = window;
    float* ws = static_cast<float*>(workspace);
    P.nlse2 = ws;
    P.ndvec = ws + static_cast<size_t>(B) * H * P.Tp;
    int has_cap = 0;
    fill_cap(query_scale, softcap, P.k_exp, P.cap_l2, P.scale_l2, has_cap);
    P.has_cap = has_cap;
    P.query_scale = query_scale;
    fill_bwd_series(query_scale, softcap, P);
    P.timeout_ns = wait_limit_ns();
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (d == 64) return launch_backward<64>(q, k, v, out, lse, dout, P, st);
    if (d == 128) return launch_backward<128>(q, k, v, out, lse, dout, P, st);
    return launch_backward<256>(q, k, v, out, lse, dout, P, st);
}

int g2attn_prefill(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                   int T, int S, int H, int Hkv, int d, int q_offset, float query_scale,
                   float softcap, int window, g2attn_stream_t stream) {
    if (!q || !k || !v || !out) return G2ATTN_ERR_INVALID_ARG;
    if (B <= 0 || T <= 0 || S <= 0 || q_offset < 0 ||
        static_cast<long long>(q_offset) + T > S)
        return G2ATTN_ERR_INVALID_ARG;
    int rc = check_common(H, Hkv, d, query_scale, softcap, window);
    if (rc) return rc;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        (lse && !aligned16(lse)))
        return G2ATTN_ERR_MISALIGNED;
    const long long tq = static_cast<long long>(B) * T, tk = static_cast<long long>(B) * S;
    if (tq > INT32_MAX || tk > INT32_MAX) return G2ATTN_ERR_UNSUPPORTED;
    g2::PfParams P{};
    P.out = static_cast<__nv_bfloat16*>(out);
    P.lse = lse;
    P.num_seqs = B;
    P.T = T;
    P.S = S;
    P.H = H;
    P.Hkv = Hkv;
    P.q_offset = q_offset;
    P.window = window;
    P.varlen = 0;
    P.total_q = static_cast<int>(tq);
    P.max_units_per_seq_tiles = (T + g2::PF_QPOS - 1) / g2::PF_QPOS;
    const long long units = static_cast<long long>(P.max_units_per_seq_tiles) * B * Hkv;
    if (units > INT32_MAX) return G2ATTN_ERR_UNSUPPORTED;
    P.num_units = static_cast<int>(units);
    fill_cap(query_scale, softcap, P.k_exp, P.cap_l2, P.scale_l2, P.has_cap);
    fill_poly(query_scale, softcap, P);
    P.timeout_ns = wait_limit_ns();
    return dispatch_prefill(d, q, k, v, tq, tk, P, reinterpret_cast<cudaStream_t>(stream));
}

int g2attn_prefill_varlen(const void* q, const void* k, const void* v, void* out, float* lse,
                          const int* cu_seqlens_q, const int* cu_seqlens_k, int num_seqs,
                          int total_q, int total_k, int max_T, int max_S, int H, int Hkv, int d,
                          float query_scale, float softcap, int window, g2attn_stream_t stream) {
    if (!q || !k || !v || !out || !cu_seqlens_q || !cu_seqlens_k) return G2ATTN_ERR_INVALID_ARG;
    if (num_seqs <= 0 || total_q <= 0 || total_k <= 0 || max_T <= 0 || max_S <= 0 ||
        max_T > max_S || max_T > total_q || max_S > total_k)
        return G2ATTN_ERR_INVALID_ARG;
    int rc = check_common(H, Hkv, d, query_scale, softcap, window);
    if (rc) return rc;
    if (num_seqs > g2::PfCfg<64>::MAX_SEQ_TABLE) return G2ATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        (lse && !aligned16(lse)) || (reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) ||
        (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u))
        return G2ATTN_ERR_MISALIGNED;
    g2::PfParams P{};
    P.out = static_cast<__nv_bfloat16*>(out);
    P.lse = lse;
    P.cu_q = cu_seqlens_q;
    P.cu_k = cu_seqlens_k;
    P.num_seqs = num_seqs;
    P.T = max_T;
    P.S = max_S;
    P.H = H;
    P.Hkv = Hkv;
    P.window = window;
    P.varlen = 1;
    P.total_q = total_q;
    P.total_k = total_k;
    // Units are enumerated on the device from cu_seqlens_q; the grid is sized
    // from an upper bound and surplus units are skipped by the kernel.
    const long long ub = (static_cast<long long>(total_q) / g2::PF_QPOS + num_seqs) * Hkv;
    if (ub > INT32_MAX) return G2ATTN_ERR_UNSUPPORTED;
    P.num_units = static_cast<int>(ub);
    P.max_units_per_seq_tiles = (max_T + g2::PF_QPOS - 1) / g2::PF_QPOS;
    fill_cap(query_scale, softcap, P.k_exp, P.cap_l2, P.scale_l2, P.has_cap);
    fill_poly(query_scale, softcap, P);
    P.timeout_ns = wait_limit_ns();
    return dispatch_prefill(d, q, k, v, total_q, total_k, P,
                            reinterpret_cast<cudaStream_t>(stream));
}

int g2attn_prefill_paged(const void* q, const void* k_blocks, const void* v_blocks, void* out,
                         float* lse, const int* cu_seqlens_q, const int* block_table,
                         const int* seq_lens_k, int num_seqs, int total_q, int num_blocks,
                         int block_size, int max_blocks_per_seq, int max_T, int max_S, int H,
                         int Hkv, int d, float query_scale, float softcap, int window,
                         g2attn_stream_t stream) {
    if (!q || !k_blocks || !v_blocks || !out || !cu_seqlens_q || !block_table || !seq_lens_k)
        return G2ATTN_ERR_INVALID_ARG;
    if (num_seqs <= 0 || total_q <= 0 || max_T <= 0 || max_S <= 0 || max_T > max_S ||
        max_T > total_q || num_blocks <= 0 || max_blocks_per_seq <= 0)
        return G2ATTN_ERR_INVALID_ARG;
    if (!pow2(block_size) || block_size < g2::PF_BN) return G2ATTN_ERR_INVALID_ARG;
    if (static_cast<long long>(max_blocks_per_seq) * block_size < max_S)
        return G2ATTN_ERR_INVALID_ARG;
    int rc = check_common(H, Hkv, d, query_scale, softcap, window);
    if (rc) return rc;
    if (num_seqs > g2::PfCfg<64>::MAX_SEQ_TABLE) return G2ATTN_ERR_UNSUPPORTED;
    const long long rows = static_cast<long long>(num_blocks) * block_size;
    if (rows > INT32_MAX || static_cast<long long>(max_blocks_per_seq) * block_size > INT32_MAX)
        return G2ATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k_blocks) || !aligned16(v_blocks) || !aligned16(out) ||
        (lse && !aligned16(lse)) || (reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) ||
        (reinterpret_cast<uintptr_t>(block_table) & 3u) ||
        (reinterpret_cast<uintptr_t>(seq_lens_k) & 3u))
        return G2ATTN_ERR_MISALIGNED;
    g2::PfParams P{};
    P.out = static_cast<__nv_bfloat16*>(out);
    P.lse = lse;
    P.cu_q = cu_seqlens_q;
    P.num_seqs = num_seqs;
    P.T = max_T;
    P.S = max_S;
    P.H = H;
    P.Hkv = Hkv;
    P.window = window;
    P.varlen = 1;
    P.paged = 1;
    P.kv_table = block_table;
    P.kv_lens = seq_lens_k;
    P.kv_block_shift = log2i(block_size);
    P.kv_max_blocks = max_blocks_per_seq;
    P.kv_num_blocks = num_blocks;
    P.total_q = total_q;
    const long long ub = (static_cast<long long>(total_q) / g2::PF_QPOS + num_seqs) * Hkv;
    if (ub > INT32_MAX) return G2ATTN_ERR_UNSUPPORTED;
    P.num_units = static_cast<int>(ub);
    P.max_units_per_seq_tiles = (max_T + g2::PF_QPOS - 1) / g2::PF_QPOS;
    fill_cap(query_scale, softcap, P.k_exp, P.cap_l2, P.scale_l2, P.has_cap);
    fill_poly(query_scale, softcap, P);
    P.timeout_ns = wait_limit_ns();
    return dispatch_prefill(d, q, k_blocks, v_blocks, total_q, rows, P,
                            reinterpret_cast<cudaStream_t>(stream));
}

size_t g2attn_decode_workspace_size(int num_seqs, int H, int d, int max_cache_len) {
    if (num_seqs <= 0 || H <= 0 || d <= 0 || max_cache_len <= 0) return 0;
    return decode_ws_bytes(num_seqs, H, d, max_cache_len, decode_chunk(num_seqs, H, max_cache_len));
}

int g2attn_decode(const void* q, const void* k_cache, const void* v_cache,
                  const int* cu_seqlens_k, void* out, float* lse, int num_seqs, int total_k,
                  int max_cache_len, int H, int Hkv, int d, float query_scale, float softcap,
                  int window, void* workspace, size_t workspace_bytes, g2attn_stream_t stream) {
    if (!cu_seqlens_k || total_k <= 0) return G2ATTN_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u) return G2ATTN_ERR_MISALIGNED;
    g2::DecParams P{};
    P.cu_k = cu_seqlens_k;
    P.total_k = total_k;
    const g2::DecLayoutParams LP{};
    return decode_common<g2::DEC_LINEAR>(P, LP, q, k_cache, v_cache, out, lse, num_seqs,
                                         max_cache_len, H, Hkv, d, query_scale, softcap, window,
                                         workspace, workspace_bytes, stream);
}

int g2attn_decode_ring(const void* q, const void* k_ring, const void* v_ring,
                       const int* seq_lens, void* out, float* lse, int num_seqs, int ring_size,
                       int max_cache_len, int H, int Hkv, int d, float query_scale,
                       float softcap, int window, void* workspace, size_t workspace_bytes,
                       g2attn_stream_t stream) {
    if (!seq_lens) return G2ATTN_ERR_INVALID_ARG;
    if (!pow2(ring_size) || window <= 0 || window > ring_size) return G2ATTN_ERR_INVALID_ARG;
    if (static_cast<long long>(num_seqs) * ring_size > INT32_MAX) return G2ATTN_ERR_UNSUPPORTED;
    if (reinterpret_cast<uintptr_t>(seq_lens) & 3u) return G2ATTN_ERR_MISALIGNED;
    g2::DecParams P{};
    g2::DecLayoutParams LP{};
    LP.seq_lens = seq_lens;
    LP.ring_mask = ring_size - 1;
    LP.ring_shift = log2i(ring_size);
    return decode_common<g2::DEC_RING>(P, LP, q, k_ring, v_ring, out, lse, num_seqs, max_cache_len,
                                       H, Hkv, d, query_scale, softcap, window, workspace,
                                       workspace_bytes, stream);
}

int g2attn_decode_paged(const void* q, const void* k_blocks, const void* v_blocks,
                        const int* block_table, const int* seq_lens, void* out, float* lse,
                        int num_seqs, int num_blocks, int block_size, int max_blocks_per_seq,
                        int max_cache_len, int H, int Hkv, int d, float query_scale,
                        float softcap, int window, void* workspace, size_t workspace_bytes,
                        g2attn_stream_t stream) {
    if (!block_table || !seq_lens) return G2ATTN_ERR_INVALID_ARG;
    if (!pow2(block_size) || num_blocks <= 0 || max_blocks_per_seq <= 0)
        return G2ATTN_ERR_INVALID_ARG;
    if (static_cast<long long>(num_blocks) * block_size > INT32_MAX ||
        static_cast<long long>(max_blocks_per_seq) * block_size > INT32_MAX)
        return G2ATTN_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(block_table) & 3u) ||
        (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
        return G2ATTN_ERR_MISALIGNED;
    g2::DecParams P{};
    g2::DecLayoutParams LP{};
    LP.seq_lens = seq_lens;
    LP.block_table = block_table;
    LP.block_shift = log2i(block_size);
    LP.max_blocks = max_blocks_per_seq;
    LP.num_blocks = num_blocks;
    return decode_common<g2::DEC_PAGED>(P, LP, q, k_blocks, v_blocks, out, lse, num_seqs,
                                        max_cache_len, H, Hkv, d, query_scale, softcap, window,
                                        workspace, workspace_bytes, stream);
}

int g2attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                          const int* cu_seqlens_k, void* out, float* lse, int num_seqs,
                          int total_k, int max_cache_len, int H, int Hkv, int d,
                          float query_scale, float softcap, int window,
                          g2attn_stream_t stream) {
    // Size check first (host arithmetic only), so an oversized request is
    // rejected before any CUDA call.
    if (num_seqs > 0 && H > 0 && max_cache_len > 0 && (d == 64 || d == 128 || d == 256) &&
        g2attn_decode_workspace_size(num_seqs, H, d, max_cache_len) > kNoAllocScratchBytes)
        return G2ATTN_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (!q || !k_cache || !v_cache || !cu_seqlens_k || !out || num_seqs <= 0 || total_k <= 0 ||
        max_cache_len <= 0)
        return G2ATTN_ERR_INVALID_ARG;
    int rc = check_common(H, Hkv, d, query_scale, softcap, window);
    if (rc) return rc;
    rc = noalloc_scratch(&scratch);
    if (rc) return rc;
    // The decode kernels write every partial they later read, so the scratch
    // needs no clearing between calls.
    return g2attn_decode(q, k_cache, v_cache, cu_seqlens_k, out, lse, num_seqs, total_k,
                         max_cache_len, H, Hkv, d, query_scale, softcap, window, scratch,
                         kNoAllocScratchBytes, stream);
}

const char* g2attn_status_string(int status) {
    switch (status) {
        case G2ATTN_OK: return "ok";
        case G2ATTN_ERR_INVALID_ARG: return "invalid argument";
        case G2ATTN_ERR_UNSUPPORTED: return "unsupported shape";
        case G2ATTN_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case G2ATTN_ERR_CUDA: return "CUDA call failed";
        case G2ATTN_ERR_DEVICE_TIMEOUT: return "device wait timed out";
        case G2ATTN_ERR_WORKSPACE: return "workspace missing or too small";
        case G2ATTN_ERR_CACHE_LEN: return "decode sequence longer than max_cache_len";
        default: return "unknown status";
    }
}

int g2attn_get_device_error(void) {
    unsigned int v = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return G2ATTN_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&v, g2::g_device_error, sizeof(v)) != cudaSuccess)
        return G2ATTN_ERR_CUDA;
    if (v == 0) return G2ATTN_OK;
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g2::g_device_error, &zero, sizeof(zero)) != cudaSuccess)
        return G2ATTN_ERR_CUDA;
    return (v & g2::DEVERR_TIMEOUT) ? G2ATTN_ERR_DEVICE_TIMEOUT : G2ATTN_ERR_CACHE_LEN;
}

int g2attn_selftest_wait_timeout(int timeout_us) {
    if (timeout_us < 1 || timeout_us > 1000000) return G2ATTN_ERR_INVALID_ARG;
    int pre = g2attn_get_device_error();  // start from a clear word
    if (pre == G2ATTN_ERR_CUDA) return pre;
    selftest_wait_kernel<<<1, 32>>>(static_cast<unsigned long long>(timeout_us) * 1000ull);
    if (cudaGetLastError() != cudaSuccess) return G2ATTN_ERR_CUDA;
    return g2attn_get_device_error();
}

}  // extern "C"
