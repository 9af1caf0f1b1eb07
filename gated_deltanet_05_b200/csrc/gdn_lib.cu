// gdn_lib.cu -- the C ABI of libgdn_b200.so (declared in include/gdn.h): argument
// validation, kernel selection and launch. The only translation unit of the library;
// the kernels live in the headers it includes.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

#include "gdn.h"
#include "gdn_backward_chunk.cuh"
#include "gdn_chunk_f32.cuh"
#include "gdn_chunk_sm100.cuh"
#include "gdn_common.cuh"
#include "gdn_decode.cuh"
#include "gdn_featurize.cuh"
#include "gdn_gate_norm.cuh"
#include "gdn_qsa.cuh"

#include <cmath>

namespace {

using gdn::chunk_f32_layout;

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool pow2_in(int x, int lo, int hi) { return x >= lo && x <= hi && (x & (x - 1)) == 0; }
cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

gdn_status launch_status()
{
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// ---- driver entry point for tensor-map encoding (no link-time libcuda dependency)
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode;
}

// 3-D map over a [n_tok][H][128] bf16 tensor, box {64, 1, 64}, 128-byte swizzle.
bool make_map(CUtensorMap *map, const void *base, int64_t n_tok, int H)
{
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {128, (cuuint64_t)H, (cuuint64_t)n_tok};
    cuuint64_t strides[2] = {128 * 2, (cuuint64_t)H * 128 * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 3-D map over the [n_tok][H][128] output y (fp32 or bf16), box {128, 1, 32}: one
// warpgroup's 32 token rows of one head, no swizzle (the staging tile is row-major).
bool make_y_map(CUtensorMap *map, void *base, int64_t n_tok, int H, bool f32)
{
    auto enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t es = f32 ? 4 : 2;
    cuuint64_t dims[3] = {128, (cuuint64_t)H, (cuuint64_t)n_tok};
    cuuint64_t strides[2] = {128 * es, (cuuint64_t)H * 128 * es};
    cuuint32_t box[3] = {128, 1, 32};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int g_smem_optin = -1;

int smem_optin()
{
    if (g_smem_optin < 0) {
        int dev = 0, v = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        g_smem_optin = v;
    }
    return g_smem_optin;
}

template <typename T, typename TY>
gdn_status launch_chunk_f32(const void *q, const void *k, const void *v, const float *la,
                            const float *beta, const float *S0, const int32_t *cu, int n_seq,
                            int H, int dk, int dv, int C, float scale, void *y, float *S_T,
                            cudaStream_t st)
{
    const int dvt = dv < 32 ? dv : 32;
    const size_t smem = (size_t)chunk_f32_layout(C, dk, dvt).total * sizeof(float);
    if ((int)smem > smem_optin()) return GDN_ERR_UNSUPPORTED;
    auto kern = gdn::chunk_fwd_f32_kernel<T, TY>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return GDN_ERR_CUDA;
    const unsigned grid = (unsigned)((int64_t)n_seq * H * (dv / dvt));
    kern<<<grid, gdn::kChunkF32Threads, smem, st>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), la, beta, S0,
        cu, H, dk, dv, C, dvt, scale, static_cast<TY *>(y), S_T);
    return launch_status();
}

// Number of SM ids of the current device. The tensor-core kernel's workspace has one
// region per SM id, and SM ids (%smid) run up to %nsmid - 1, which may exceed the SM count
// (ids need not be contiguous). %nsmid is read once per device by a one-thread kernel
// (followed by a synchronous copy, so the first query on a device synchronises it and
// must not happen inside a stream capture); the result is the larger of it and the SM
// count. 0 if the device cannot be queried.
__device__ unsigned int g_nsmid_word;

__global__ void nsmid_kernel()
{
    unsigned int n;
    asm volatile("mov.u32 %0, %%nsmid;" : "=r"(n));
    g_nsmid_word = n;
}

constexpr int kMaxDevices = 64;
int g_sm_ids[kMaxDevices] = {};
std::mutex g_sm_ids_mutex;

int device_sm_ids()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    if (dev < 0 || dev >= kMaxDevices) return 0;
    std::lock_guard<std::mutex> lock(g_sm_ids_mutex);
    if (g_sm_ids[dev] > 0) return g_sm_ids[dev];
    nsmid_kernel<<<1, 1>>>();
    unsigned int ids = 0;
    if (cudaGetLastError() != cudaSuccess ||
        cudaMemcpyFromSymbol(&ids, g_nsmid_word, sizeof(ids)) != cudaSuccess)
        return 0;
    g_sm_ids[dev] = (int)ids > n ? (int)ids : n;
    return g_sm_ids[dev];
}

// Device check of the kernels' bounded mbarrier wait (gdn_selftest_bounded_wait). Thread 0
// waits on a phase of a fresh barrier; mode 0: nothing completes it (the wait must give up
// after `limit` cycles and record a timeout); mode 1: thread 32 raises the abort flag after
// a short delay (the wait must return early without recording anything); mode 2: thread 32
// completes the phase (the wait must succeed). Only the timeout records an error.
__global__ void selftest_wait_kernel(long long limit, int mode)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        gdn::sm100::mbar_init(&bar, 1);
        abort_flag = 0;
        gdn::sm100::fence_mbarrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const bool ok = gdn::sm100::mbar_wait_bounded(&bar, 0, &abort_flag, limit);
        // a wait that returned the wrong answer for its mode is an internal-check failure
        if (ok != (mode == 2)) gdn::raise_error(gdn::kErrCheck);
    } else if (threadIdx.x == 32 && mode != 0) {
        const long long t0 = clock64();
        while (clock64() - t0 < 20000) {}
        if (mode == 1) {
            *reinterpret_cast<volatile int *>(&abort_flag) = 1;
        } else {
            gdn::sm100::mbar_arrive(&bar);
        }
    }
}

// Fixed scratch of gdn_chunk_fwd_noalloc: the tensor-core kernel's K ring for up to
// kNoAllocMaxSms SM ids, as a file-scope device array (one copy per device, created with
// the module; never allocated by a call).
constexpr int kNoAllocMaxSms = 160;
static __device__ __align__(256) uint8_t g_noalloc_ws[(size_t)kNoAllocMaxSms * gdn::sm100::kWsBytesPerSm];

template <typename TY>
gdn_status launch_chunk_sm100(const void *q, const void *k, const void *v, const float *la,
                              const float *beta, const float *S0, const int32_t *cu, int n_seq,
                              int64_t n_tok, int H, float scale, void *y, float *S_T, void *ws,
                              size_t ws_bytes, cudaStream_t st)
{
    const int n_ids = device_sm_ids();
    if (n_ids <= 0) return GDN_ERR_CUDA;
    if (!ws || !aligned(ws, 128) || ws_bytes < (size_t)n_ids * gdn::sm100::kWsBytesPerSm)
        return GDN_ERR_INVALID_ARG;
    if (2 * (int64_t)n_seq * H > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
    // every region the workspace holds may serve an SM id (the kernel checks its own id
    // against this count and records GDN_ERR_DEVICE_CHECK if it falls outside)
    const size_t slots = ws_bytes / gdn::sm100::kWsBytesPerSm;
    const int ws_slots = slots > 0x7fffffff ? 0x7fffffff : (int)slots;
    CUtensorMap mq, mk, mv, my;
    if (!make_map(&mq, q, n_tok, H) || !make_map(&mk, k, n_tok, H) || !make_map(&mv, v, n_tok, H) ||
        !make_y_map(&my, y, n_tok, H, sizeof(TY) == 4))
        return GDN_ERR_CUDA;
    const int smem = (int)gdn::sm100::SMEM_BYTES;
    if (smem > smem_optin()) return GDN_ERR_UNSUPPORTED;
    auto kern = gdn::sm100::chunk_fwd_bf16_kernel<TY>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return GDN_ERR_CUDA;
    // one cluster of two CTAs (solver, chain) per (sequence, head) chain
    const unsigned grid = (unsigned)(2 * (int64_t)n_seq * H);
    kern<<<grid, gdn::sm100::kThreads, smem, st>>>(mq, mk, mv, my, la, beta, S0, cu, n_seq, H, scale,
                                                   static_cast<TY *>(y), S_T,
                                                   static_cast<uint8_t *>(ws), ws_slots);
    return launch_status();
}

// ---- QSA indexer: host-side sizes (the same formulas as qsa_setup_kernel)
struct QsaSizes {
    int64_t n_tok = 0, n_blocks = 0, nb_max = 0, n_tiles = 0, n_ctas = 0;
};

QsaSizes qsa_sizes(const int32_t *cu, int n_seq, int r)
{
    QsaSizes z;
    z.n_tok = cu[n_seq];
    for (int s = 0; s < n_seq; ++s) {
        const int64_t len = (int64_t)cu[s + 1] - cu[s];
        z.n_blocks += len / r;
        if (len / r > z.nb_max) z.nb_max = len / r;
        const int64_t nt = (len + gdn::qsa::kTileT - 1) / gdn::qsa::kTileT;
        z.n_tiles += nt;
        for (int64_t i = 0; i < nt; ++i)
            z.n_ctas += (gdn::qsa::qsa_tile_steps(len, r, i) + gdn::qsa::kMaxSteps - 1) / gdn::qsa::kMaxSteps;
    }
    return z;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// workspace: blk0, tile0 [n_seq + 1], cta0 [n_tiles + 1] (int32), then the query and key
// vectors (bf16 or fp32)
size_t qsa_ws_layout(const QsaSizes &z, int n_seq, int Hq, size_t elem, size_t *off_q, size_t *off_k)
{
    const size_t ints = align256(sizeof(int32_t) * ((size_t)2 * (n_seq + 1) + (size_t)z.n_tiles + 1));
    *off_q = ints;
    *off_k = *off_q + align256((size_t)z.n_tok * Hq * gdn::qsa::kD * elem);
    return *off_k + align256((size_t)z.n_blocks * gdn::qsa::kD * elem);
}

// q vectors [n_tok][Hq][128] bf16 as a 3-D map, box {64, 1, 128}; key vectors [n_blocks][128]
// bf16 as a 2-D map, box {64, 128}; both 128-byte swizzled (the MMA operand layout)
bool make_qsa_maps(CUtensorMap *mq, CUtensorMap *mk, void *qv, void *kv, int64_t n_tok, int Hq, int64_t n_blocks)
{
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t qd[3] = {128, (cuuint64_t)Hq, (cuuint64_t)n_tok};
    cuuint64_t qs[2] = {256, (cuuint64_t)Hq * 256};
    cuuint32_t qb[3] = {64, 1, 128}, e3[3] = {1, 1, 1};
    if (enc(mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, qv, qd, qs, qb, e3, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
        return false;
    cuuint64_t kd[2] = {128, (cuuint64_t)n_blocks};
    cuuint64_t ks[1] = {256};
    cuuint32_t kbx[2] = {64, 128}, e2[2] = {1, 1};
    return enc(mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kv, kd, ks, kbx, e2, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

template <int HQ>
gdn_status launch_qsa_scores_tc(const CUtensorMap &mq, const CUtensorMap &mk, const int32_t *cu, const int32_t *blk0,
                                const int32_t *tile0, const int32_t *cta0, int n_seq, int r, int64_t nb_max,
                                int64_t n_ctas, float *I, cudaStream_t st)
{
    const int smem = (int)gdn::qsa::tc::smem_bytes(HQ);
    if (smem > smem_optin()) return GDN_ERR_UNSUPPORTED;
    auto kern = gdn::qsa::qsa_scores_tc_kernel<HQ>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return GDN_ERR_CUDA;
    kern<<<(unsigned)n_ctas, gdn::qsa::tc::kThreads, smem, st>>>(mq, mk, cu, blk0, tile0, cta0, n_seq, r,
                                                                 (int)nb_max, I);
    return launch_status();
}

}  // namespace

extern "C" {

const char *gdn_status_string(gdn_status s)
{
    switch (s) {
    case GDN_OK: return "GDN_OK";
    case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
    case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
    case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT";
    case GDN_ERR_DEVICE_CHECK: return "GDN_ERR_DEVICE_CHECK";
    }
    return "GDN_ERR_UNKNOWN";
}

int gdn_version(void) { return 100; }

size_t gdn_chunk_fwd_workspace_bytes(int n_seq, int64_t total_tokens, int H, int d_k, int d_v,
                                     int chunk)
{
    (void)n_seq; (void)total_tokens; (void)H;
    if (d_k != 128 || d_v != 128 || chunk != 64) return 0;
    return (size_t)device_sm_ids() * gdn::sm100::kWsBytesPerSm;
}

gdn_status gdn_chunk_fwd(const void *q, const void *k, const void *v, gdn_dtype in_dtype,
                         const float *log_alpha, const float *beta, const float *S0,
                         const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                         int n_seq, int H, int d_k, int d_v, int chunk, float scale, void *y,
                         gdn_dtype y_dtype, float *S_T, void *workspace, size_t workspace_bytes,
                         void *stream)
{
    if (n_seq < 0 || H <= 0 || !cu_seqlens_host || (n_seq > 0 && !cu_seqlens_dev))
        return GDN_ERR_INVALID_ARG;
    if (in_dtype != GDN_F32 && in_dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (y_dtype != GDN_F32 && y_dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (!pow2_in(d_k, 16, 128) || !pow2_in(d_v, 16, 128) || !pow2_in(chunk, 16, 64))
        return GDN_ERR_UNSUPPORTED;
    if (cu_seqlens_host[0] != 0) return GDN_ERR_INVALID_ARG;
    for (int i = 0; i < n_seq; ++i)
        if (cu_seqlens_host[i + 1] < cu_seqlens_host[i]) return GDN_ERR_INVALID_ARG;
    if (n_seq == 0) return GDN_OK;
    const int64_t n_tok = cu_seqlens_host[n_seq];
    if (n_tok > 0 && (!q || !k || !v || !log_alpha || !beta || !y)) return GDN_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(y, 16) ||
        !aligned(S0, 16) || !aligned(S_T, 16) || !aligned(log_alpha, 4) || !aligned(beta, 4) ||
        !aligned(cu_seqlens_dev, 4))
        return GDN_ERR_INVALID_ARG;
    if ((int64_t)n_seq * H * (d_v / (d_v < 32 ? d_v : 32)) > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
    cudaStream_t st = as_stream(stream);
    const bool y32 = y_dtype == GDN_F32;
    if (in_dtype == GDN_BF16 && d_k == 128 && d_v == 128 && chunk == 64 && n_tok > 0)
        return y32 ? launch_chunk_sm100<float>(q, k, v, log_alpha, beta, S0, cu_seqlens_dev, n_seq,
                                               n_tok, H, scale, y, S_T, workspace, workspace_bytes, st)
                   : launch_chunk_sm100<__nv_bfloat16>(q, k, v, log_alpha, beta, S0, cu_seqlens_dev,
                                                       n_seq, n_tok, H, scale, y, S_T, workspace,
                                                       workspace_bytes, st);
#define GDN_F32_PATH(T, TY)                                                                        \
    launch_chunk_f32<T, TY>(q, k, v, log_alpha, beta, S0, cu_seqlens_dev, n_seq, H, d_k, d_v, chunk, \
                            scale, y, S_T, st)
    if (in_dtype == GDN_BF16)
        return y32 ? GDN_F32_PATH(__nv_bfloat16, float) : GDN_F32_PATH(__nv_bfloat16, __nv_bfloat16);
    return y32 ? GDN_F32_PATH(float, float) : GDN_F32_PATH(float, __nv_bfloat16);
#undef GDN_F32_PATH
}

gdn_status gdn_chunk_fwd_gated(const void *q, const void *k, const void *v, gdn_dtype in_dtype,
                               const float *log_alpha, const float *beta, const float *S0,
                               const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                               int n_seq, int H, int d_k, int d_v, int chunk, float scale,
                               const void *z, const float *w, float eps, void *o, gdn_dtype o_dtype,
                               float *S_T, void *workspace, size_t workspace_bytes, void *stream)
{
    if (n_seq < 0 || H <= 0 || !cu_seqlens_host || (n_seq > 0 && !cu_seqlens_dev))
        return GDN_ERR_INVALID_ARG;
    if (in_dtype != GDN_F32 && in_dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (o_dtype != GDN_F32 && o_dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (!(eps >= 0.f)) return GDN_ERR_INVALID_ARG;
    if (in_dtype != GDN_BF16 || d_k != 128 || d_v != 128 || chunk != 64) return GDN_ERR_UNSUPPORTED;
    if (cu_seqlens_host[0] != 0) return GDN_ERR_INVALID_ARG;
    for (int i = 0; i < n_seq; ++i)
        if (cu_seqlens_host[i + 1] < cu_seqlens_host[i]) return GDN_ERR_INVALID_ARG;
    if (n_seq == 0) return GDN_OK;
    const int64_t n_tok = cu_seqlens_host[n_seq];
    if (n_tok > 0 && (!z || !w || !o)) return GDN_ERR_INVALID_ARG;
    if (n_tok > 0 && (!aligned(o, 16) || !aligned(z, 16) || !aligned(w, 4))) return GDN_ERR_INVALID_ARG;
    if (n_tok > 0) {                    // z is read after o is written: they must not overlap
        const uintptr_t z0 = (uintptr_t)z, o0 = (uintptr_t)o, n = (uintptr_t)n_tok * H * d_v;
        if (z0 < o0 + n * (o_dtype == GDN_F32 ? 4u : 2u) && o0 < z0 + n * 2u) return GDN_ERR_INVALID_ARG;
    }
    // y into o (in o's dtype), then the gate-norm in place on o: two launches on the stream.
    // (A gate-norm inside the prefill kernel's output stage sat on the chain CTA's per-chunk
    // path and measured 0.52 ms against 0.28 ms for these two launches on the prefill shape.)
    const gdn_status rc = gdn_chunk_fwd(q, k, v, in_dtype, log_alpha, beta, S0, cu_seqlens_dev,
                                        cu_seqlens_host, n_seq, H, d_k, d_v, chunk, scale, o, o_dtype,
                                        S_T, workspace, workspace_bytes, stream);
    if (rc != GDN_OK || n_tok == 0) return rc;
    return gdn_gate_norm(o, o_dtype, z, GDN_BF16, w, n_tok * H, d_v, eps, o, o_dtype, stream);
}

size_t gdn_backward_workspace_bytes(const int32_t *cu_seqlens_host, int n_seq, int H, int d_k, int d_v)
{
    if (!cu_seqlens_host || n_seq <= 0 || H <= 0 || d_k <= 0 || d_v <= 0) return 0;
    int64_t max_len = 0;
    for (int i = 0; i < n_seq; ++i) {
        const int64_t l = (int64_t)cu_seqlens_host[i + 1] - cu_seqlens_host[i];
        if (l > max_len) max_len = l;
    }
    const int64_t max_chunks = (max_len + gdn::bwdc::kC - 1) / gdn::bwdc::kC;
    const int n_vt = d_v / gdn::bwdc::slice_cols(d_v);
    // per (chain, chunk): the start state and the end-state adjoint [d_k][d_v], U~ and dU~
    // [C][d_v], the chunk's cache (T, A o Gamma, P, W), and one block of sums over v per
    // value slice
    const size_t per_chunk = 2 * (size_t)d_k * d_v + 2 * (size_t)gdn::bwdc::kC * d_v +
                             gdn::bwdc::cache_floats(d_k) + (size_t)n_vt * gdn::bwdc::part_floats(d_k);
    return (size_t)n_seq * H * (size_t)max_chunks * per_chunk * sizeof(float);
}

gdn_status gdn_backward(const void *q, const void *k, const void *v, gdn_dtype in_dtype,
                        const float *log_alpha, const float *beta, const float *S0,
                        const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host, int n_seq,
                        int H, int d_k, int d_v, float scale, const void *dy, const float *dS_T,
                        float *dq, float *dk, float *dv, float *dlog_alpha, float *dbeta, float *dS0,
                        void *workspace, size_t workspace_bytes, void *stream)
{
    using namespace gdn::bwdc;
    if (n_seq < 0 || H <= 0 || !cu_seqlens_host || (n_seq > 0 && !cu_seqlens_dev))
        return GDN_ERR_INVALID_ARG;
    if (in_dtype != GDN_F32 && in_dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (!pow2_in(d_k, 16, 128) || !pow2_in(d_v, 16, 128)) return GDN_ERR_UNSUPPORTED;
    if (cu_seqlens_host[0] != 0) return GDN_ERR_INVALID_ARG;
    for (int i = 0; i < n_seq; ++i)
        if (cu_seqlens_host[i + 1] < cu_seqlens_host[i]) return GDN_ERR_INVALID_ARG;
    if (n_seq == 0) return GDN_OK;
    const int64_t n_tok = cu_seqlens_host[n_seq];
    if (n_tok > 0 && (!q || !k || !v || !log_alpha || !beta || !dy || !dq || !dk || !dv ||
                      !dlog_alpha || !dbeta))
        return GDN_ERR_INVALID_ARG;
    const size_t need = gdn_backward_workspace_bytes(cu_seqlens_host, n_seq, H, d_k, d_v);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 16)) return GDN_ERR_INVALID_ARG;
    if (!aligned(S0, 4) || !aligned(dS_T, 4) || !aligned(dS0, 4)) return GDN_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(dy, 16) || !aligned(dq, 16) ||
        !aligned(dk, 16) || !aligned(dv, 16))
        return GDN_ERR_INVALID_ARG;
    int64_t max_len = 0;
    for (int i = 0; i < n_seq; ++i)
        if ((int64_t)cu_seqlens_host[i + 1] - cu_seqlens_host[i] > max_len)
            max_len = (int64_t)cu_seqlens_host[i + 1] - cu_seqlens_host[i];
    const int64_t n_chain = (int64_t)n_seq * H;
    const int64_t max_chunks = (max_len + kC - 1) / kC;
    const int dvt = slice_cols(d_v);
    const int n_vt = d_v / dvt;
    if (n_chain * n_vt > 0x7fffffffLL || max_chunks > 65535) return GDN_ERR_UNSUPPORTED;
    if (max_chunks == 0) {
        // no tokens: dS0 = dS_T (or 0)
        if (dS0) {
            cudaStream_t st0 = as_stream(stream);
            const size_t bytes = (size_t)n_chain * d_k * d_v * sizeof(float);
            const cudaError_t e = dS_T ? cudaMemcpyAsync(dS0, dS_T, bytes, cudaMemcpyDeviceToDevice, st0)
                                       : cudaMemsetAsync(dS0, 0, bytes, st0);
            if (e != cudaSuccess) return GDN_ERR_CUDA;
        }
        return GDN_OK;
    }
    cudaStream_t st = as_stream(stream);
    const size_t n_cc = (size_t)n_chain * max_chunks;
    float *S_chunks = static_cast<float *>(workspace);
    float *dS_chunks = S_chunks + n_cc * d_k * d_v;
    float *Ut_chunks = dS_chunks + n_cc * d_k * d_v;
    float *dUt_chunks = Ut_chunks + n_cc * kC * d_v;
    float *cache = dUt_chunks + n_cc * kC * d_v;
    float *parts = cache + n_cc * cache_floats(d_k);
    const int smem_p = (int)(prep_layout(d_k).total * sizeof(float));
    const int smem_f = (int)(fwd_layout(d_k, dvt, in_dtype == GDN_F32 ? 4 : 2).total * sizeof(float));
    const int smem_s = (int)(state_layout(d_k, dvt, in_dtype == GDN_BF16 ? 2 : 0).total * sizeof(float));
    const int smem_v = (int)(vpart_layout(d_k, dvt).total * sizeof(float));
    const int smem_k = (int)(kpart_layout(d_k).total * sizeof(float));
    const int optin = smem_optin();
    if (smem_p > optin || smem_f > optin || smem_s > optin || smem_v > optin || smem_k > optin)
        return GDN_ERR_UNSUPPORTED;
    const dim3 grid_c((unsigned)n_chain, (unsigned)max_chunks);
    const dim3 grid_v((unsigned)(n_chain * n_vt), (unsigned)max_chunks);
    const unsigned grid_s = (unsigned)(n_chain * n_vt);
#define GDN_BWD(T)                                                                                   \
    {                                                                                                \
        auto kp = chunk_bwd_prep_kernel<T>;                                                          \
        auto kf = chunk_bwd_fwd_kernel<T>;                                                           \
        auto ks = chunk_bwd_state_kernel<T>;                                                         \
        auto kv = chunk_bwd_vpart_kernel<T>;                                                         \
        auto kk = chunk_bwd_kpart_kernel<T>;                                                         \
        if (cudaFuncSetAttribute(kp, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_p) != cudaSuccess || \
            cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_f) != cudaSuccess || \
            cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_s) != cudaSuccess || \
            cudaFuncSetAttribute(kv, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_v) != cudaSuccess || \
            cudaFuncSetAttribute(kk, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_k) != cudaSuccess)   \
            return GDN_ERR_CUDA;                                                                     \
        kp<<<grid_c, kThreads, smem_p, st>>>((const T *)q, (const T *)k, log_alpha, beta, cu_seqlens_dev, H, d_k, \
                                             scale, (int)max_chunks, cache);                        \
        kf<<<grid_s, kThreadsWide, smem_f, st>>>((const T *)k, (const T *)v, log_alpha, beta, S0, cu_seqlens_dev, \
                                                 H, d_k, d_v, (int)max_chunks, cache, S_chunks, Ut_chunks); \
        ks<<<grid_s, kThreadsWide, smem_s, st>>>((const T *)q, (const T *)k, (const T *)dy, log_alpha, beta,     \
                                                 cu_seqlens_dev, H, d_k, d_v, scale, dS_T, (int)max_chunks,     \
                                                 cache, dS_chunks, dUt_chunks, dS0);                \
        kv<<<grid_v, kThreadsWide, smem_v, st>>>((const T *)v, (const T *)dy, beta, cu_seqlens_dev, H, d_k, d_v, \
                                                 (int)max_chunks, cache, S_chunks, dS_chunks, Ut_chunks,        \
                                                 dUt_chunks, parts, dv);                            \
        kk<<<grid_c, kThreadsWide, smem_k, st>>>((const T *)q, (const T *)k, log_alpha, beta, cu_seqlens_dev, H, d_k, \
                                             n_vt, scale, (int)max_chunks, cache, parts, dq, dk, dbeta,  \
                                             dlog_alpha);                                           \
    }
    if (in_dtype == GDN_F32)
        GDN_BWD(float)
    else
        GDN_BWD(__nv_bfloat16)
#undef GDN_BWD
    return launch_status();
}

gdn_status gdn_chunk_fwd_noalloc(const void *q, const void *k, const void *v, gdn_dtype in_dtype,
                                 const float *log_alpha, const float *beta, const float *S0,
                                 const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                                 int n_seq, int H, int d_k, int d_v, int chunk, float scale, void *y,
                                 gdn_dtype y_dtype, float *S_T, void *stream)
{
    // the fixed array covers kNoAllocMaxSms SM ids of the current device; all of it is
    // offered to the kernel
    size_t have = 0;
    if (d_k == 128 && d_v == 128 && chunk == 64) {
        const int n_ids = device_sm_ids();
        if (n_ids <= 0) return GDN_ERR_CUDA;
        if (n_ids > kNoAllocMaxSms) return GDN_ERR_UNSUPPORTED;
        have = sizeof(g_noalloc_ws);
    }
    void *ws = nullptr;
    if (have > 0 && cudaGetSymbolAddress(&ws, g_noalloc_ws) != cudaSuccess) return GDN_ERR_CUDA;
    return gdn_chunk_fwd(q, k, v, in_dtype, log_alpha, beta, S0, cu_seqlens_dev, cu_seqlens_host, n_seq, H,
                         d_k, d_v, chunk, scale, y, y_dtype, S_T, ws, have, stream);
}

gdn_status gdn_selftest_bounded_wait(int64_t limit_cycles, int mode, void *stream)
{
    if (limit_cycles < 1 || limit_cycles > 2000000000LL || mode < 0 || mode > 2) return GDN_ERR_INVALID_ARG;
    if (mode == 1 && limit_cycles < 1000000) return GDN_ERR_INVALID_ARG;   // the abort must come first
    selftest_wait_kernel<<<1, 64, 0, as_stream(stream)>>>((long long)limit_cycles, mode);
    return launch_status();
}

gdn_status gdn_decode_step(const void *q, const void *k, const void *v, gdn_dtype in_dtype,
                           const float *alpha, const float *beta, float *S, int n_seq, int H,
                           int d_k, int d_v, float scale, void *y, gdn_dtype y_dtype, void *stream)
{
    if (n_seq < 0 || H <= 0) return GDN_ERR_INVALID_ARG;
    if (in_dtype != GDN_F32 && in_dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (y_dtype != GDN_F32 && y_dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (!pow2_in(d_k, 16, 128) || !pow2_in(d_v, 16, 128)) return GDN_ERR_UNSUPPORTED;
    const int64_t n_chain = (int64_t)n_seq * H;
    if (n_chain == 0) return GDN_OK;
    if (n_chain > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
    if (!q || !k || !v || !alpha || !beta || !S || !y) return GDN_ERR_INVALID_ARG;
    const size_t vec = in_dtype == GDN_F32 ? 16 : 8;
    if (!aligned(q, vec) || !aligned(k, vec) || !aligned(S, 16) || !aligned(alpha, 4) ||
        !aligned(beta, 4) || !aligned(v, 4) || !aligned(y, 4))
        return GDN_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    const unsigned grid = (unsigned)n_chain;
#define GDN_DECODE_LAUNCH(DK, T, TY)                                                               \
    gdn::decode_step_kernel<DK, T, TY><<<grid, gdn::kDecodeThreads, 0, st>>>(                      \
        (const T *)q, (const T *)k, (const T *)v, alpha, beta, S, d_v, scale, (TY *)y)
#define GDN_DECODE_CASE(DK)                                                                        \
    case DK:                                                                                       \
        if (in_dtype == GDN_F32) {                                                                 \
            if (y_dtype == GDN_F32) GDN_DECODE_LAUNCH(DK, float, float);                           \
            else GDN_DECODE_LAUNCH(DK, float, __nv_bfloat16);                                      \
        } else {                                                                                   \
            if (y_dtype == GDN_F32) GDN_DECODE_LAUNCH(DK, __nv_bfloat16, float);                   \
            else GDN_DECODE_LAUNCH(DK, __nv_bfloat16, __nv_bfloat16);                              \
        }                                                                                          \
        break;
    switch (d_k) {
        GDN_DECODE_CASE(16)
        GDN_DECODE_CASE(32)
        GDN_DECODE_CASE(64)
        GDN_DECODE_CASE(128)
    default: return GDN_ERR_UNSUPPORTED;
    }
#undef GDN_DECODE_CASE
#undef GDN_DECODE_LAUNCH
    return launch_status();
}

gdn_status gdn_decode_tokens(const void *q, const void *k, const void *v, gdn_dtype in_dtype,
                             const float *alpha, const float *beta, float *S, int n_seq,
                             int n_tokens, int H, int d_k, int d_v, float scale, void *y,
                             gdn_dtype y_dtype, void *stream)
{
    if (n_seq < 0 || H <= 0 || n_tokens < 1 || n_tokens > gdn::kDecodeMaxTokens)
        return GDN_ERR_INVALID_ARG;
    if (in_dtype != GDN_F32 && in_dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (y_dtype != GDN_F32 && y_dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (!pow2_in(d_k, 16, 128) || !pow2_in(d_v, 16, 128)) return GDN_ERR_UNSUPPORTED;
    const int64_t n_chain = (int64_t)n_seq * H;
    if (n_chain == 0) return GDN_OK;
    if (n_chain > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
    if (!q || !k || !v || !alpha || !beta || !S || !y) return GDN_ERR_INVALID_ARG;
    const size_t vec = in_dtype == GDN_F32 ? 16 : 8;
    if (!aligned(q, vec) || !aligned(k, vec) || !aligned(S, 16) || !aligned(alpha, 4) ||
        !aligned(beta, 4) || !aligned(v, 4) || !aligned(y, 4))
        return GDN_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    if (d_k == 128 && d_v == 128 && aligned(v, 16)) {
        // pipelined kernel: two persistent CTAs per SM walk the chains
        int dev = 0, n_sm = 148;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return GDN_ERR_CUDA;
        const unsigned grid_p = (unsigned)(n_chain < 2LL * n_sm ? n_chain : 2LL * n_sm);
#define GDN_DECPIPE_LAUNCH(T, TY)                                                                  \
    {                                                                                              \
        auto kern = gdn::decode_tokens_pipe_kernel<T, TY>;                                         \
        constexpr int smem = (int)gdn::decode_pipe_smem_bytes<T>();                                \
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) \
            return GDN_ERR_CUDA;                                                                   \
        kern<<<grid_p, gdn::kDecPipeThreads, smem, st>>>((const T *)q, (const T *)k, (const T *)v, alpha, beta, S, \
                                                         n_tokens, H, (int)n_chain, scale, (TY *)y);  \
    }
        if (in_dtype == GDN_F32) {
            if (y_dtype == GDN_F32) GDN_DECPIPE_LAUNCH(float, float)
            else GDN_DECPIPE_LAUNCH(float, __nv_bfloat16)
        } else {
            if (y_dtype == GDN_F32) GDN_DECPIPE_LAUNCH(__nv_bfloat16, float)
            else GDN_DECPIPE_LAUNCH(__nv_bfloat16, __nv_bfloat16)
        }
#undef GDN_DECPIPE_LAUNCH
        return launch_status();
    }
    const unsigned grid = (unsigned)n_chain;
#define GDN_DECTOK_LAUNCH(DK, T, TY)                                                               \
    gdn::decode_tokens_kernel<DK, T, TY><<<grid, gdn::kDecodeTokThreads, 0, st>>>(                 \
        (const T *)q, (const T *)k, (const T *)v, alpha, beta, S, n_tokens, H, d_v, scale, (TY *)y)
#define GDN_DECTOK_CASE(DK)                                                                        \
    case DK:                                                                                       \
        if (in_dtype == GDN_F32) {                                                                 \
            if (y_dtype == GDN_F32) GDN_DECTOK_LAUNCH(DK, float, float);                           \
            else GDN_DECTOK_LAUNCH(DK, float, __nv_bfloat16);                                      \
        } else {                                                                                   \
            if (y_dtype == GDN_F32) GDN_DECTOK_LAUNCH(DK, __nv_bfloat16, float);                   \
            else GDN_DECTOK_LAUNCH(DK, __nv_bfloat16, __nv_bfloat16);                              \
        }                                                                                          \
        break;
    switch (d_k) {
        GDN_DECTOK_CASE(16)
        GDN_DECTOK_CASE(32)
        GDN_DECTOK_CASE(64)
        GDN_DECTOK_CASE(128)
    default: return GDN_ERR_UNSUPPORTED;
    }
#undef GDN_DECTOK_CASE
#undef GDN_DECTOK_LAUNCH
    return launch_status();
}

gdn_status gdn_gate_norm(const void *y, gdn_dtype y_dtype, const void *z, gdn_dtype z_dtype,
                         const float *w, int64_t n_rows, int d_v, float eps, void *o,
                         gdn_dtype o_dtype, void *stream)
{
    if (n_rows < 0) return GDN_ERR_INVALID_ARG;
    for (gdn_dtype dt : {y_dtype, z_dtype, o_dtype})
        if (dt != GDN_F32 && dt != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (!pow2_in(d_v, 16, 256)) return GDN_ERR_UNSUPPORTED;
    if (n_rows == 0) return GDN_OK;
    if (!y || !z || !w || !o) return GDN_ERR_INVALID_ARG;
    if (!aligned(y, 16) || !aligned(z, 16) || !aligned(o, 16) || !aligned(w, 4))
        return GDN_ERR_INVALID_ARG;
    // o may be y itself with the same dtype (in place); otherwise o overlaps neither y nor z
    {
        auto bytes = [&](gdn_dtype dt) { return (uintptr_t)n_rows * (uintptr_t)d_v * (dt == GDN_F32 ? 4u : 2u); };
        auto overlap = [](const void *a, uintptr_t na, const void *b, uintptr_t nb) {
            const uintptr_t a0 = (uintptr_t)a, b0 = (uintptr_t)b;
            return a0 < b0 + nb && b0 < a0 + na;
        };
        const uintptr_t ob = bytes(o_dtype);
        if (y == o ? y_dtype != o_dtype : overlap(y, bytes(y_dtype), o, ob)) return GDN_ERR_INVALID_ARG;
        if (overlap(z, bytes(z_dtype), o, ob)) return GDN_ERR_INVALID_ARG;
    }
    cudaStream_t st = as_stream(stream);
    int dev = 0, n_sm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);   // grid sizing only
    // rows per CTA pass = 8 warps x rows per warp pass (32 bytes of y per lane) x 4 (unroll);
    // at most 8 CTAs per SM
    const int epl = y_dtype == GDN_BF16 ? 16 : 8;
    const int lpr = d_v / epl > 0 ? d_v / epl : 1;
    const int64_t rows_per_cta = (int64_t)(gdn::kGateNormThreads / 32) * (32 / lpr) * 4;
    int64_t blocks = (n_rows + rows_per_cta - 1) / rows_per_cta;
    const int64_t cap = (int64_t)n_sm * 8;
    if (blocks > cap) blocks = cap;
    const int combo = (y_dtype == GDN_BF16) * 4 + (z_dtype == GDN_BF16) * 2 + (o_dtype == GDN_BF16);
    using f32 = float;
    using b16 = __nv_bfloat16;
#define GDN_GN(TY, TZ, TO, DV)                                                                     \
    gdn::gate_norm_kernel<TY, TZ, TO, DV><<<(unsigned)blocks, gdn::kGateNormThreads, 0, st>>>(     \
        (const TY *)y, (const TZ *)z, w, n_rows, eps, (TO *)o)
#define GDN_GN_DV(TY, TZ, TO)                                                                      \
    switch (d_v) {                                                                                 \
    case 16: GDN_GN(TY, TZ, TO, 16); break;                                                        \
    case 32: GDN_GN(TY, TZ, TO, 32); break;                                                        \
    case 64: GDN_GN(TY, TZ, TO, 64); break;                                                        \
    case 128: GDN_GN(TY, TZ, TO, 128); break;                                                      \
    default: GDN_GN(TY, TZ, TO, 256); break;                                                       \
    }
    switch (combo) {
    case 0: GDN_GN_DV(f32, f32, f32) break;
    case 1: GDN_GN_DV(f32, f32, b16) break;
    case 2: GDN_GN_DV(f32, b16, f32) break;
    case 3: GDN_GN_DV(f32, b16, b16) break;
    case 4: GDN_GN_DV(b16, f32, f32) break;
    case 5: GDN_GN_DV(b16, f32, b16) break;
    case 6: GDN_GN_DV(b16, b16, f32) break;
    default: GDN_GN_DV(b16, b16, b16) break;
    }
#undef GDN_GN_DV
#undef GDN_GN
    return launch_status();
}

gdn_status gdn_featurize(const void *xq, const void *xk, const void *xv, gdn_dtype dtype,
                         const float *conv_q, const float *conv_k, const float *conv_v, int W,
                         const float *beta_logit, const float *alpha_logit, const float *A,
                         const float *b_alpha, const int32_t *cu_seqlens_dev,
                         const int32_t *cu_seqlens_host, int n_seq, int64_t n_tok, int H, int d_k,
                         int d_v, float eps, void *q, void *k, void *v, float *beta,
                         float *log_alpha, void *stream)
{
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (n_tok < 0 || n_seq < 1 || H < 1 || W < 1 || W > gdn::kFeatMaxWidth || !(eps >= 0.f))
        return GDN_ERR_INVALID_ARG;
    if (!pow2_in(d_k, 16, 128) || !pow2_in(d_v, 16, 128)) return GDN_ERR_UNSUPPORTED;
    if (cu_seqlens_host) {
        if (cu_seqlens_host[0] != 0 || cu_seqlens_host[n_seq] != n_tok) return GDN_ERR_INVALID_ARG;
        for (int i = 0; i < n_seq; ++i)
            if (cu_seqlens_host[i + 1] < cu_seqlens_host[i]) return GDN_ERR_INVALID_ARG;
    }
    if (n_tok == 0) return GDN_OK;
    const void *ptrs[] = {xq, xk, xv, conv_q, conv_k, conv_v, beta_logit, alpha_logit, A, b_alpha,
                          cu_seqlens_dev, q, k, v, beta, log_alpha};
    for (const void *p : ptrs)
        if (!p) return GDN_ERR_INVALID_ARG;
    for (const void *p : {xq, xk, xv, (const void *)q, (const void *)k, (const void *)v})
        if (!aligned(p, 16)) return GDN_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    const int64_t n_runs = (n_tok + gdn::kFeatRun - 1) / gdn::kFeatRun;
    const int warps_per_block = gdn::kFeatThreads / 32;
    auto blocks_for = [&](int d, int n_streams, bool gates) -> unsigned {
        const int rpw = 32 / (d / 8);
        const int64_t n_hg = (H + rpw - 1) / rpw;
        const int64_t tasks = n_streams * n_runs * n_hg + (gates ? n_runs : 0);
        return (unsigned)((tasks + warps_per_block - 1) / warps_per_block);
    };
    using f32 = float;
    using b16 = __nv_bfloat16;
    // launch 1: q and k (L2-normalised); launch 2: v and the gates
#define GDN_FT(T, D, L2, X0, X1, W0, W1, O0, O1, NS, GATES)                                       \
    gdn::featurize_kernel<T, D, L2><<<blocks_for(D, NS, GATES), gdn::kFeatThreads, 0, st>>>(      \
        (const T *)(X0), (const T *)(X1), W0, W1, (T *)(O0), (T *)(O1), NS, W, cu_seqlens_dev, n_seq, \
        n_tok, H, eps, GATES ? beta_logit : nullptr, alpha_logit, A, b_alpha, beta, log_alpha)
#define GDN_FT_D(T, d, L2, X0, X1, W0, W1, O0, O1, NS, GATES)                                     \
    switch (d) {                                                                                 \
    case 16: GDN_FT(T, 16, L2, X0, X1, W0, W1, O0, O1, NS, GATES); break;                        \
    case 32: GDN_FT(T, 32, L2, X0, X1, W0, W1, O0, O1, NS, GATES); break;                        \
    case 64: GDN_FT(T, 64, L2, X0, X1, W0, W1, O0, O1, NS, GATES); break;                        \
    default: GDN_FT(T, 128, L2, X0, X1, W0, W1, O0, O1, NS, GATES); break;                       \
    }
    if (dtype == GDN_BF16) {
        GDN_FT_D(b16, d_k, true, xq, xk, conv_q, conv_k, q, k, 2, false)
        GDN_FT_D(b16, d_v, false, xv, nullptr, conv_v, nullptr, v, nullptr, 1, true)
    } else {
        GDN_FT_D(f32, d_k, true, xq, xk, conv_q, conv_k, q, k, 2, false)
        GDN_FT_D(f32, d_v, false, xv, nullptr, conv_v, nullptr, v, nullptr, 1, true)
    }
#undef GDN_FT_D
#undef GDN_FT
    return launch_status();
}

size_t gdn_qsa_workspace_bytes(const int32_t *cu_seqlens_host, int n_seq, int Hq, int d, int r, gdn_dtype dtype)
{
    if (!cu_seqlens_host || n_seq < 1 || Hq < 1 || d != gdn::qsa::kD || r < 1) return 0;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return 0;
    const QsaSizes z = qsa_sizes(cu_seqlens_host, n_seq, r);
    size_t oq, ok;
    return qsa_ws_layout(z, n_seq, Hq, dtype == GDN_BF16 ? 2 : 4, &oq, &ok);
}

gdn_status gdn_qsa_indexer(const void *qx, const void *kx, gdn_dtype dtype, const float *wq, const float *wk,
                           const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host, int n_seq, int Hq,
                           int d, int r, int K, int rot, float base, float eps, float *scores, int32_t *blocks,
                           void *workspace, size_t workspace_bytes, void *stream)
{
    using namespace gdn::qsa;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (!cu_seqlens_host || !cu_seqlens_dev || n_seq < 1 || Hq < 1 || r < 1 || K < 1) return GDN_ERR_INVALID_ARG;
    if (rot < 0 || rot > d || rot % 8 != 0 || !(base > 0.f) || !(eps >= 0.f)) return GDN_ERR_INVALID_ARG;
    if (d != kD) return GDN_ERR_UNSUPPORTED;
    if (dtype == GDN_BF16 ? (Hq != 1 && Hq != 2 && Hq != 4) : Hq > kMaxHeadsF32) return GDN_ERR_UNSUPPORTED;
    const int kb = (K + r - 1) / r;
    if (kb > kMaxKB) return GDN_ERR_UNSUPPORTED;
    if (cu_seqlens_host[0] != 0) return GDN_ERR_INVALID_ARG;
    for (int i = 0; i < n_seq; ++i)
        if (cu_seqlens_host[i + 1] < cu_seqlens_host[i]) return GDN_ERR_INVALID_ARG;
    const QsaSizes z = qsa_sizes(cu_seqlens_host, n_seq, r);
    if (z.n_tok == 0) return GDN_OK;
    if (!qx || !kx || !wq || !wk || !blocks || (z.nb_max > 0 && !scores)) return GDN_ERR_INVALID_ARG;
    if (!aligned(qx, 16) || !aligned(kx, 16) || !aligned(wq, 4) || !aligned(wk, 4) || !aligned(scores, 4) ||
        !aligned(blocks, 4) || !aligned(cu_seqlens_dev, 4))
        return GDN_ERR_INVALID_ARG;
    if (z.n_tok * Hq > 0x3fffffffLL || z.n_tok * z.nb_max > ((int64_t)1 << 40) || z.n_ctas > 0x7fffffffLL)
        return GDN_ERR_UNSUPPORTED;
    const size_t elem = dtype == GDN_BF16 ? 2 : 4;
    size_t off_q, off_k;
    const size_t need = qsa_ws_layout(z, n_seq, Hq, elem, &off_q, &off_k);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 16)) return GDN_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int32_t *blk0 = reinterpret_cast<int32_t *>(ws);
    int32_t *tile0 = blk0 + (n_seq + 1);
    int32_t *cta0 = tile0 + (n_seq + 1);
    RopeTable rope{};
    for (int j = 0; j < rot / 2; ++j) rope.inv_freq[j] = std::pow((double)base, -2.0 * j / (double)rot);

    qsa_setup_kernel<<<1, 32, 0, st>>>(cu_seqlens_dev, n_seq, r, blk0, tile0, cta0);
    const int64_t n_vec = z.n_tok * Hq + z.n_blocks;
    const unsigned vec_blocks = (unsigned)((n_vec * 32 + kVecThreads - 1) / kVecThreads);
    if (dtype == GDN_BF16)
        qsa_vectors_kernel<__nv_bfloat16, __nv_bfloat16><<<vec_blocks, kVecThreads, 0, st>>>(
            (const __nv_bfloat16 *)qx, (const __nv_bfloat16 *)kx, wq, wk, cu_seqlens_dev, blk0, n_seq, z.n_tok, Hq, r,
            rot, eps, rope, (__nv_bfloat16 *)(ws + off_q), (__nv_bfloat16 *)(ws + off_k));
    else
        qsa_vectors_kernel<float, float><<<vec_blocks, kVecThreads, 0, st>>>(
            (const float *)qx, (const float *)kx, wq, wk, cu_seqlens_dev, blk0, n_seq, z.n_tok, Hq, r, rot, eps,
            rope, (float *)(ws + off_q), (float *)(ws + off_k));
    if (launch_status() != GDN_OK) return GDN_ERR_CUDA;
    if (z.nb_max > 0) {
        if (dtype == GDN_BF16) {
            CUtensorMap mq, mk;
            if (!make_qsa_maps(&mq, &mk, ws + off_q, ws + off_k, z.n_tok, Hq, z.n_blocks)) return GDN_ERR_CUDA;
            gdn_status rc = Hq == 1 ? launch_qsa_scores_tc<1>(mq, mk, cu_seqlens_dev, blk0, tile0, cta0, n_seq, r,
                                                              z.nb_max, z.n_ctas, scores, st)
                          : Hq == 2 ? launch_qsa_scores_tc<2>(mq, mk, cu_seqlens_dev, blk0, tile0, cta0, n_seq, r,
                                                              z.nb_max, z.n_ctas, scores, st)
                                    : launch_qsa_scores_tc<4>(mq, mk, cu_seqlens_dev, blk0, tile0, cta0, n_seq, r,
                                                              z.nb_max, z.n_ctas, scores, st);
            if (rc != GDN_OK) return rc;
        } else {
            const int smem = kF32Tok * Hq * kD * (int)sizeof(float);
            dim3 grid((unsigned)((z.nb_max + kF32Blk - 1) / kF32Blk), (unsigned)((z.n_tok + kF32Tok - 1) / kF32Tok));
            if (cudaFuncSetAttribute(qsa_scores_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
                cudaSuccess)
                return GDN_ERR_CUDA;
            qsa_scores_f32_kernel<<<grid, 256, smem, st>>>((const float *)(ws + off_q), (const float *)(ws + off_k),
                                                           cu_seqlens_dev, blk0, n_seq, z.n_tok, Hq, (int)z.nb_max, r,
                                                           scores);
            if (launch_status() != GDN_OK) return GDN_ERR_CUDA;
        }
    }
    const int smem_sel = (int)topk_smem_bytes(kb);
    if (smem_sel > smem_optin()) return GDN_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(qsa_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_sel) != cudaSuccess)
        return GDN_ERR_CUDA;
    qsa_topk_kernel<<<(unsigned)((z.n_tok + kTopkWarps - 1) / kTopkWarps), kTopkWarps * 32, smem_sel, st>>>(
        scores, cu_seqlens_dev, n_seq, z.n_tok, (int)z.nb_max, r, kb, blocks);
    return launch_status();
}

gdn_status gdn_qsa_token_sets(const int32_t *blocks, const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                              int n_seq, int K_B, int r, int32_t *tokens, int32_t *count, void *stream)
{
    using namespace gdn::qsa;
    if (!cu_seqlens_host || !cu_seqlens_dev || n_seq < 1 || K_B < 1 || r < 1) return GDN_ERR_INVALID_ARG;
    if (K_B > kMaxKB) return GDN_ERR_UNSUPPORTED;
    if (cu_seqlens_host[0] != 0) return GDN_ERR_INVALID_ARG;
    for (int i = 0; i < n_seq; ++i)
        if (cu_seqlens_host[i + 1] < cu_seqlens_host[i]) return GDN_ERR_INVALID_ARG;
    const int64_t n_tok = cu_seqlens_host[n_seq];
    if (n_tok == 0) return GDN_OK;
    if (!blocks || !tokens || !count) return GDN_ERR_INVALID_ARG;
    if ((int64_t)K_B * r + r - 1 > 0x7fffffffLL || n_tok > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
    int kb2 = 1;
    while (kb2 < K_B) kb2 <<= 1;
    qsa_token_sets_kernel<<<(unsigned)n_tok, kTopkThreads, kb2 * sizeof(uint32_t), as_stream(stream)>>>(
        blocks, cu_seqlens_dev, n_seq, K_B, r, tokens, count);
    return launch_status();
}

gdn_status gdn_device_error(void *stream)
{
    if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return GDN_ERR_CUDA;
    unsigned int word = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&word, gdn::g_error_word, sizeof(word)) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (word && cudaMemcpyToSymbol(gdn::g_error_word, &zero, sizeof(zero)) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (word & gdn::kErrTimeout) return GDN_ERR_TIMEOUT;
    if (word & gdn::kErrCheck) return GDN_ERR_DEVICE_CHECK;
    return GDN_OK;
}

}  // extern "C"
