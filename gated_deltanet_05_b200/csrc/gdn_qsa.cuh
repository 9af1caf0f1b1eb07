// gdn_qsa.cuh -- the compressed lightweight indexer of Qwen Sparse Attention (QSA).
//
// Follows the indexer equations of the joezjh.github.io notes page "Qwen3.8-Flash-Next"
// (section on Qwen Sparse Attention): per query head h, q_i^h = PRoPE(RMSNorm(qx_i^h), i);
// keys compressed per non-overlapping block of r tokens, k_b = PRoPE(RMSNorm(mean_r kx), b r);
// importance I_ib = sum_h ReLU(<q_i^h, k_b>) over the blocks complete at token i
// (b r + r - 1 <= i); the K_B = ceil(K / r) best blocks per token, ties to the lower block;
// the token set = the selected blocks' tokens plus the incomplete tail block. Positions
// restart at every sequence of the packed batch. RMSNorm is zero-centred,
// x / sqrt(mean x^2 + eps) * (1 + w); PRoPE rotates dimension j with j + rot/2 (j < rot/2)
// by the angle pos * base^(-2j/rot), the angle formed in fp64 so that it stays exact at
// long positions.
//
// d = 128. Kernels:
//   qsa_setup_kernel    one thread: per-sequence block offsets, per-tile CTA offsets of the
//                       tensor-core score kernel
//   qsa_vectors_kernel  one warp per query (token, head) or compressed key block: the
//                       normalised, rotated vectors (bf16 for the tensor-core scores, fp32
//                       for the CUDA-core ones)
//   qsa_scores_tc_kernel  tcgen05: 128 query tokens x 128 key blocks per step, one M=128,
//                       N=128 accumulator per query head in TMEM, ReLU-summed over heads
//   qsa_scores_f32_kernel CUDA cores, fp32: one thread per (token, block)
//   qsa_topk_kernel     one warp per token: radix selection of the K_B largest scores, then
//                       a bitonic sort of the selection by (score desc, block asc)
//   qsa_token_sets_kernel one CTA per token: the selected blocks in ascending order,
//                       expanded to tokens, plus the tail
#pragma once
#include <cuda.h>

#include "gdn_common.cuh"
#include "sm100_ptx.cuh"

namespace gdn {
namespace qsa {

constexpr int kD = 128;
constexpr int kMaxHeadsF32 = 8;
constexpr int kTileT = 128;          // query tokens per tensor-core CTA (MMA M)
constexpr int kTileB = 128;          // key blocks per step (MMA N)
constexpr int kMaxSteps = 8;         // key tiles per CTA; longer rows are split over CTAs
constexpr int kVecThreads = 256;
constexpr int kTopkThreads = 256;
constexpr int kMaxKB = 4096;         // largest K_B the selection sorts in shared memory

// RoPE inverse frequencies base^(-2j/rot), j < rot/2, formed on the host in fp64.
struct RopeTable {
    double inv_freq[kD / 2];
};

// --------------------------------------------------------------------------- setup
// ws_int layout: blk0[n_seq + 1] (first compressed block of each sequence),
// tile0[n_seq + 1] (first query tile of each sequence), cta0[n_tiles + 1] (first
// tensor-core CTA of each query tile); a tile of queries [128 i, 128 i + 128) of a sequence
// needs ceil(nvis_last / 128) key steps, split into chunks of at most kMaxSteps.
__host__ __device__ inline int64_t qsa_tile_steps(int64_t len, int r, int64_t tile)
{
    const int64_t last = (tile + 1) * kTileT < len ? (tile + 1) * kTileT - 1 : len - 1;
    int64_t nvis = (last + 1) / r;
    const int64_t nb = len / r;
    if (nvis > nb) nvis = nb;
    return (nvis + kTileB - 1) / kTileB;
}

__global__ void qsa_setup_kernel(const int32_t *__restrict__ cu, int n_seq, int r, int32_t *__restrict__ blk0,
                                 int32_t *__restrict__ tile0, int32_t *__restrict__ cta0)
{
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    int32_t b = 0, t = 0, c = 0;
    for (int s = 0; s < n_seq; ++s) {
        blk0[s] = b;
        tile0[s] = t;
        const int64_t len = (int64_t)cu[s + 1] - cu[s];
        b += (int32_t)(len / r);
        const int64_t n_tiles = (len + kTileT - 1) / kTileT;
        for (int64_t i = 0; i < n_tiles; ++i) {
            cta0[t++] = c;
            c += (int32_t)((qsa_tile_steps(len, r, i) + kMaxSteps - 1) / kMaxSteps);
        }
    }
    blk0[n_seq] = b;
    tile0[n_seq] = t;
    cta0[t] = c;
}

// the last index i in [0, n) with a[i] <= x (a non-decreasing, a[0] <= x)
__device__ __forceinline__ int upper_index(const int32_t *a, int n, int64_t x)
{
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a[mid] <= x) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// --------------------------------------------------------------------------- vectors
template <typename TO> __device__ __forceinline__ void store_vec4(TO *p, const float (&x)[4]);
template <> __device__ __forceinline__ void store_vec4<float>(float *p, const float (&x)[4])
{
    *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
}
template <> __device__ __forceinline__ void store_vec4<__nv_bfloat16>(__nv_bfloat16 *p, const float (&x)[4])
{
    store4(p, make_float4(x[0], x[1], x[2], x[3]));
}

// One warp normalises and rotates one 128-vector; lane l owns dimensions 4l .. 4l + 3.
__device__ __forceinline__ void norm_rope(float (&x)[4], const float *__restrict__ w, float eps, int64_t pos,
                                          int rot, const RopeTable &rope, int lane)
{
    float ss = x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3];
    ss = group_sum<32>(ss);
    const float inv = rsqrtf(ss * (1.0f / kD) + eps);
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] = x[e] * inv * (1.0f + w[4 * lane + e]);
    // dimension j pairs with j + rot/2: lane l with lane l + rot/8 (rot is a multiple of 8)
    const int half = rot / 2, half_lanes = rot / 8;
    float p[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) p[e] = __shfl_xor_sync(0xffffffffu, x[e], half_lanes > 0 ? half_lanes : 0);
    const int dim0 = 4 * lane;
    if (dim0 < rot) {
        const bool lo = dim0 < half;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int j = (lo ? dim0 : dim0 - half) + e;
            // the angle in fp64, reduced to [-pi, pi] before the single-precision sin/cos
            double ang = (double)pos * rope.inv_freq[j];
            ang -= 6.283185307179586 * rint(ang * 0.15915494309189535);
            float s, c;
            sincosf((float)ang, &s, &c);
            x[e] = lo ? x[e] * c - p[e] * s : x[e] * c + p[e] * s;
        }
    }
}

// Warps [0, n_tok * Hq) make the queries qv [n_tok][Hq][128]; warps from n_tok * Hq on make
// the compressed keys kv [n_blocks][128] (sequence s's block b at row blk0[s] + b).
template <typename T, typename TO>
__global__ void __launch_bounds__(kVecThreads)
qsa_vectors_kernel(const T *__restrict__ qx, const T *__restrict__ kx, const float *__restrict__ wq,
                   const float *__restrict__ wk, const int32_t *__restrict__ cu, const int32_t *__restrict__ blk0,
                   int n_seq, int64_t n_tok, int Hq, int r, int rot, float eps, const __grid_constant__ RopeTable rope,
                   TO *__restrict__ qv, TO *__restrict__ kv)
{
    const int lane = threadIdx.x & 31;
    const int64_t wid = ((int64_t)blockIdx.x * kVecThreads + threadIdx.x) >> 5;
    const int64_t n_q = n_tok * Hq;
    const int64_t n_blocks = blk0[n_seq];
    if (wid >= n_q + n_blocks) return;
    float x[4];
    int64_t pos;
    TO *dst;
    const float *w;
    if (wid < n_q) {
        const int64_t t = wid / Hq;
        const int s = upper_index(cu, n_seq + 1, t);
        pos = t - cu[s];
        const float4 f = load4(qx + wid * kD + 4 * lane);
        x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
        w = wq;
        dst = qv + wid * kD;
    } else {
        const int64_t g = wid - n_q;
        const int s = upper_index(blk0, n_seq + 1, g);
        const int64_t b = g - blk0[s];
        const int64_t tok0 = cu[s] + b * r;
        x[0] = x[1] = x[2] = x[3] = 0.f;
        for (int j = 0; j < r; ++j) {
            const float4 f = load4(kx + (tok0 + j) * kD + 4 * lane);
            x[0] += f.x; x[1] += f.y; x[2] += f.z; x[3] += f.w;
        }
        const float inv_r = 1.0f / (float)r;
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] *= inv_r;
        pos = b * r;
        w = wk;
        dst = kv + g * kD;
    }
    norm_rope(x, w, eps, pos, rot, rope, lane);
    store_vec4<TO>(dst + 4 * lane, x);
}

// --------------------------------------------------------------------------- fp32 scores
// One thread per (token, key block); a CTA covers 16 tokens x 64 blocks with the tokens'
// queries staged in shared memory. Only visible blocks are written.
constexpr int kF32Tok = 16, kF32Blk = 64;

__global__ void __launch_bounds__(256)
qsa_scores_f32_kernel(const float *__restrict__ qv, const float *__restrict__ kv, const int32_t *__restrict__ cu,
                      const int32_t *__restrict__ blk0, int n_seq, int64_t n_tok, int Hq, int nb_max, int r,
                      float *__restrict__ I)
{
    extern __shared__ float qs[];               // [16][Hq][128]
    const int64_t t0 = (int64_t)blockIdx.y * kF32Tok;
    const int b = blockIdx.x * kF32Blk + (threadIdx.x & (kF32Blk - 1));
    for (int e = threadIdx.x; e < kF32Tok * Hq * kD; e += blockDim.x) {
        const int64_t t = t0 + e / (Hq * kD);
        qs[e] = t < n_tok ? qv[(size_t)t0 * Hq * kD + e] : 0.f;
    }
    __syncthreads();
    for (int tt = threadIdx.x >> 6; tt < kF32Tok; tt += 4) {
        const int64_t t = t0 + tt;
        if (t >= n_tok || b >= nb_max) continue;
        const int s = upper_index(cu, n_seq + 1, t);
        const int64_t pos = t - cu[s], len = (int64_t)cu[s + 1] - cu[s];
        int64_t nvis = (pos + 1) / r;
        if (nvis > len / r) nvis = len / r;
        if (b >= nvis) continue;
        const float *kb = kv + ((size_t)blk0[s] + b) * kD;
        float out = 0.f;
        for (int h = 0; h < Hq; ++h) {
            const float *qh = qs + (tt * Hq + h) * kD;
            float acc = 0.f;
            for (int c = 0; c < kD; c += 4) {
                const float4 kk = *reinterpret_cast<const float4 *>(kb + c);
                acc = fmaf(qh[c], kk.x, fmaf(qh[c + 1], kk.y, fmaf(qh[c + 2], kk.z, fmaf(qh[c + 3], kk.w, acc))));
            }
            out += fmaxf(acc, 0.f);
        }
        I[(size_t)t * nb_max + b] = out;
    }
}

// --------------------------------------------------------------------------- tensor-core scores
namespace tc {
constexpr int kThreads = 384;                // warp 0 TMA, warp 1 MMA, warps 4..11 epilogue
constexpr uint32_t HEAD_BYTES = 32768;       // one head's 128 tokens x 128 dims bf16: two 16 KB boxes
constexpr uint32_t KT_BYTES = 32768;         // one key tile: 128 blocks x 128 dims bf16, two boxes
constexpr int kKStages = 2;
constexpr long long kWaitLimit = 2000000000LL;
constexpr uint32_t STAGE_BYTES = 8 * 32 * 17 * 4;   // per epilogue warp: 32 rows x 16 columns (+1 pad)
constexpr uint32_t smem_bytes(int hq)
{
    return (uint32_t)hq * HEAD_BYTES + kKStages * KT_BYTES + STAGE_BYTES + 256 + 1024;
}
}  // namespace tc

// One CTA: query tile `tile` of sequence s (128 tokens from the sequence's token 128 i),
// key steps [step0, step1) of 128 blocks each. D_h = Q_h K^T (bf16, fp32 accumulate) for
// every head h into TMEM columns [128 h, 128 h + 128); the epilogue (8 warps: TMEM lane
// quadrant w % 4, column half (w - 4) / 4) sums ReLU(D_h) over heads and writes the
// visible scores. The per-head accumulators form a ring: head h's MMA of the next step
// starts once the epilogue has read head h of this one.
template <int HQ>
__global__ void __launch_bounds__(tc::kThreads, 1)
qsa_scores_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const int32_t *__restrict__ cu, const int32_t *__restrict__ blk0,
                     const int32_t *__restrict__ tile0, const int32_t *__restrict__ cta0, int n_seq, int r,
                     int nb_max, float *__restrict__ I)
{
    using namespace sm100;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);
    constexpr uint32_t OFF_K = HQ * tc::HEAD_BYTES;
    constexpr uint32_t OFF_STAGE = OFF_K + tc::kKStages * tc::KT_BYTES;
    constexpr uint32_t OFF_BAR = OFF_STAGE + tc::STAGE_BYTES;
    enum { B_Q = 0, B_KFULL = 1, B_KEMPTY = B_KFULL + tc::kKStages, B_AFULL = B_KEMPTY + tc::kKStages,
           B_AEMPTY = B_AFULL + HQ, B_DRAIN = B_AEMPTY + HQ, N_BAR };
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_BAR + N_BAR * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_BAR + N_BAR * 8 + 4);
    constexpr uint32_t TM_COLS = HQ * 128;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // this CTA's query tile and key steps
    const int n_tiles = tile0[n_seq];
    const int tile = upper_index(cta0, n_tiles + 1, blockIdx.x);
    const int s = upper_index(tile0, n_seq + 1, tile);
    const int64_t i_tile = tile - tile0[s];
    const int64_t bos = cu[s], len = (int64_t)cu[s + 1] - bos;
    const int64_t n_steps = qsa_tile_steps(len, r, i_tile);
    const int64_t step0 = (int64_t)(blockIdx.x - cta0[tile]) * kMaxSteps;
    const int64_t step1 = step0 + kMaxSteps < n_steps ? step0 + kMaxSteps : n_steps;
    const int n_my = (int)(step1 - step0);
    const int64_t t_first = i_tile * kTileT;                 // sequence position of row 0

    if (tid == 0) {
        for (int b = 0; b < N_BAR; ++b) mbar_init(&bar[b], (b >= B_AEMPTY && b < B_AEMPTY + HQ) ? 256 : 1);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    auto wait = [&](int b, int parity) -> bool {
        return mbar_test(&bar[b], (uint32_t)parity & 1u) ||
               mbar_wait_bounded(&bar[b], (uint32_t)parity & 1u, abort_flag, tc::kWaitLimit);
    };

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (n_my > 0) {
            const uint32_t lead = elect_one();
            const int tok = (int)(bos + t_first);
            mbar_arrive_expect_tx_lead(&bar[B_Q], HQ * tc::HEAD_BYTES, lead);
#pragma unroll 1
            for (int h = 0; h < HQ; ++h) {
                tma_load_3d_lead(smem + h * tc::HEAD_BYTES, &tm_q, &bar[B_Q], 0, h, tok, lead);
                tma_load_3d_lead(smem + h * tc::HEAD_BYTES + 16384, &tm_q, &bar[B_Q], 64, h, tok, lead);
            }
            int issued[tc::kKStages] = {};
#pragma unroll 1
            for (int j = 0; j < n_my; ++j) {
                const int st = j % tc::kKStages;
                if (j >= tc::kKStages && !__all_sync(0xffffffffu, wait(B_KEMPTY + st, j / tc::kKStages - 1))) break;
                const int row = (int)(blk0[s] + (step0 + j) * kTileB);
                uint8_t *dst = smem + OFF_K + st * tc::KT_BYTES;
                mbar_arrive_expect_tx_lead(&bar[B_KFULL + st], tc::KT_BYTES, lead);
                tma_load_2d_lead(dst, &tm_k, &bar[B_KFULL + st], 0, row, lead);
                tma_load_2d_lead(dst + 16384, &tm_k, &bar[B_KFULL + st], 64, row, lead);
                issued[st] = j + 1;
            }
            mbar_wait_drain(&bar[B_Q], 0, tc::kWaitLimit);
            for (int st = 0; st < tc::kKStages; ++st)
                if (issued[st] > 0) mbar_wait_drain(&bar[B_KFULL + st], ((issued[st] - 1) / tc::kKStages) & 1, tc::kWaitLimit);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (n_my > 0) {
            const uint32_t lead = elect_one();
            const uint32_t idesc = idesc_f32acc(kFmtBF16, 128, 128, 0, 0);
            const uint64_t dq0 = sdesc_sw128(sbase, 16, 1024);
            const uint64_t dk0 = sdesc_sw128(sbase + OFF_K, 16, 1024);
            bool ok = __all_sync(0xffffffffu, wait(B_Q, 0));
#pragma unroll 1
            for (int j = 0; ok && j < n_my; ++j) {
                const int st = j % tc::kKStages;
                if (!__all_sync(0xffffffffu, wait(B_KFULL + st, j / tc::kKStages))) break;
#pragma unroll 1
                for (int h = 0; h < HQ; ++h) {
                    if (j > 0 && !__all_sync(0xffffffffu, wait(B_AEMPTY + h, j - 1))) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t a = dq0 + ((uint64_t)(h * tc::HEAD_BYTES) >> 4);
                    const uint64_t b = dk0 + ((uint64_t)(st * tc::KT_BYTES) >> 4);
#pragma unroll 1
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint64_t off = (uint64_t)((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
                        mma_ss_lead(tmem + h * 128, a + off, b + off, idesc, kk > 0, lead);
                    }
                    mma_commit_lead(&bar[B_AFULL + h], lead);
                }
                mma_commit_lead(&bar[B_KEMPTY + st], lead);
            }
            mma_commit_lead(&bar[B_DRAIN], lead);
            mbar_wait_drain(&bar[B_DRAIN], 0, tc::kWaitLimit);
        }
    } else if (warp >= 4) {
        // ---------------------------------------------------------------- epilogue
        const int e = warp - 4, half = e >> 2;
        const uint32_t lane_base = (uint32_t)(warp & 3) * 32u << 16;
        bool ok = true;
#pragma unroll 1
        for (int j = 0; j < n_my && ok; ++j) {
            float acc[64];
#pragma unroll
            for (int i = 0; i < 64; ++i) acc[i] = 0.f;
#pragma unroll 1
            for (int h = 0; h < HQ; ++h) {
                bool got = true;
                if (lane == 0) got = wait(B_AFULL + h, j);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                tc_fence_after();
                uint32_t v[32];
#pragma unroll
                for (int c2 = 0; c2 < 2; ++c2) {
                    tmem_ld_x32(tmem + lane_base + h * 128 + 64 * half + 32 * c2, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) acc[32 * c2 + i] += fmaxf(__uint_as_float(v[i]), 0.f);
                }
                tc_fence_before();
                mbar_arrive(&bar[B_AEMPTY + h]);
            }
            if (!ok) break;
            // the warp's 32 rows x 64 scores go out through its staging slice, 16 columns at
            // a time: each store instruction writes two rows' 16 consecutive scores (lanes
            // 0..15 and 16..31), instead of 32 rows' single scores
            const int64_t b0 = (step0 + j) * kTileB + 64 * half;
            float *stg = reinterpret_cast<float *>(smem + OFF_STAGE) + e * 32 * 17;
            const int64_t t_row0 = t_first + 32 * (warp & 3);      // sequence position of row 0
#pragma unroll
            for (int c16 = 0; c16 < 4; ++c16) {
#pragma unroll
                for (int i = 0; i < 16; ++i) stg[lane * 17 + i] = acc[16 * c16 + i];
                __syncwarp();
#pragma unroll 4
                for (int rr = 0; rr < 32; rr += 2) {
                    const int row = rr + (lane >> 4), col = lane & 15;
                    const int64_t p_row = t_row0 + row;
                    int64_t nv_row = (p_row + 1) / r;
                    if (nv_row > len / r) nv_row = len / r;
                    const int64_t b = b0 + 16 * c16 + col;
                    if (p_row < len && b < nv_row) I[(size_t)(bos + p_row) * nb_max + b] = stg[row * 17 + col];
                }
                __syncwarp();
            }
        }
        // leaving early: release the issuer from any head it may still wait for
        if (!ok)
            for (int h = 0; h < HQ; ++h) mbar_arrive(&bar[B_AEMPTY + h]);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

// --------------------------------------------------------------------------- selection
// order-preserving key of a float: larger floats give larger unsigned integers
__device__ __forceinline__ uint32_t fkey(float x)
{
    const uint32_t u = __float_as_uint(x);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// One warp per token (kTopkWarps tokens per CTA): B_t = the kb largest scores of the visible
// blocks, ordered by (score descending, block ascending); -1 padded. Radix selection on the
// order-preserving keys (four 8-bit passes over the row, a 256-bin histogram per warp in
// shared memory) finds the kb-th largest key T; the keys above T and the lowest-index keys
// equal to T are gathered (ballots keep index order), then sorted by the warp (bitonic: in
// registers for selections of up to kTopkRegSort entries, else in its shared-memory slice).
// Rows with at most kb visible blocks take every block.
constexpr int kTopkWarps = 4;

__host__ __device__ inline int topk_pow2(int kb)
{
    int p = 1;
    while (p < kb) p <<= 1;
    return p;
}
__host__ __device__ inline size_t topk_smem_bytes(int kb)
{
    return (size_t)kTopkWarps * ((size_t)topk_pow2(kb) * sizeof(unsigned long long) + 256 * sizeof(int));
}

// Selections of 16..512 entries are sorted in registers: 16 keys per lane, entry i =
// 16 lane + e. Pairs (i, i ^ jj) with jj < 16 sit in one lane; with jj >= 16 they are
// exchanged by shuffles. kTopkRegSort entries in all (zeros pad the selection and sort last).
constexpr int kTopkRegSort = 512;
// where entry i of a register-sorted selection is kept in shared memory: rotated inside its
// 16-entry group, so that the 32 lanes loading entries 16 lane + e for one e hit distinct banks
__device__ __forceinline__ int topk_swz(int i) { return (i & ~15) | ((i + (i >> 4)) & 15); }

template <int JJ>
__device__ __forceinline__ void bitonic_in_lane(unsigned long long (&v)[16], int lane, int k)
{
#pragma unroll
    for (int e = 0; e < 16; ++e)
        if ((e & JJ) == 0) {
            const bool desc = ((lane * 16 + e) & k) == 0;
            const unsigned long long a = v[e], b = v[e | JJ];
            const bool sw = desc ? (a < b) : (a > b);
            v[e] = sw ? b : a;
            v[e | JJ] = sw ? a : b;
        }
}

__global__ void __launch_bounds__(kTopkWarps * 32)
qsa_topk_kernel(const float *__restrict__ I, const int32_t *__restrict__ cu, int n_seq, int64_t n_tok, int nb_max,
                int r, int kb, int32_t *__restrict__ B)
{
    extern __shared__ unsigned long long topk_sm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kb2 = topk_pow2(kb);
    unsigned long long *sel = topk_sm + (size_t)warp * kb2;
    int *hist = reinterpret_cast<int *>(topk_sm + (size_t)kTopkWarps * kb2) + warp * 256;
    const int64_t t = (int64_t)blockIdx.x * kTopkWarps + warp;
    if (t >= n_tok) return;
    const int s = upper_index(cu, n_seq + 1, t);
    const int64_t pos = t - cu[s], len = (int64_t)cu[s + 1] - cu[s];
    int64_t nv64 = (pos + 1) / r;
    if (nv64 > len / r) nv64 = len / r;
    const int nvis = (int)nv64;
    const float *row = I + (size_t)t * nb_max;
    const int take = nvis < kb ? nvis : kb;

    uint32_t prefix = 0, mask = 0;
    int need = take;                               // keys still to take at or below the prefix
    if (nvis > kb) {
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int i = lane; i < 256; i += 32) hist[i] = 0;
            __syncwarp();
            for (int b = lane; b < nvis; b += 32) {
                const uint32_t key = fkey(row[b]);
                if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
            }
            __syncwarp();
            // the digit d with (keys above d) < need <= (keys at or above d): lane l holds the
            // digits 255 - 8l .. 248 - 8l
            int cnt[8], tot = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                cnt[j] = hist[255 - 8 * lane - j];
                tot += cnt[j];
            }
            int incl = tot;                       // keys at or above this lane's lowest digit
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int nb = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += nb;
            }
            const int above_lane = incl - tot;     // keys above this lane's digits
            const bool hit = above_lane < need && incl >= need;
            const unsigned m = __ballot_sync(0xffffffffu, hit);
            const int src = __ffs(m) - 1;
            int digit = 0, above = 0;
            if (lane == src) {
                int acc = above_lane;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (acc + cnt[j] >= need) {
                        digit = 255 - 8 * lane - j;
                        above = acc;
                        break;
                    }
                    acc += cnt[j];
                }
            }
            digit = __shfl_sync(0xffffffffu, digit, src);
            above = __shfl_sync(0xffffffffu, above, src);
            prefix |= (uint32_t)digit << shift;
            mask |= 255u << shift;
            need -= above;
            __syncwarp();
        }
    }
    // gather in index order: the keys above T (every visible key when nvis <= kb), then the
    // `need` lowest-index keys equal to T
    const uint32_t T = prefix;
    const bool all = nvis <= kb;
    const bool reg_sort = kb2 >= 16 && kb2 <= kTopkRegSort;
    auto slot = [&](int i) { return reg_sort ? topk_swz(i) : i; };
    int n_gt = 0, n_eq = 0;
    for (int b0 = 0; b0 < nvis; b0 += 32) {
        const int b = b0 + lane;
        const uint32_t key = b < nvis ? fkey(row[b]) : 0u;
        const bool gt = b < nvis && (all || key > T);
        const bool eq = b < nvis && !all && key == T;
        const unsigned mg = __ballot_sync(0xffffffffu, gt), me = __ballot_sync(0xffffffffu, eq);
        const unsigned below = (1u << lane) - 1u;
        if (gt) sel[slot(n_gt + __popc(mg & below))] = ((unsigned long long)key << 32) | (0xffffffffu - (uint32_t)b);
        if (eq) {
            const int at = n_eq + __popc(me & below);
            if (at < need) sel[slot(kb - need + at)] = ((unsigned long long)key << 32) | (0xffffffffu - (uint32_t)b);
        }
        n_gt += __popc(mg);
        n_eq += __popc(me);
    }
    __syncwarp();
    int32_t *out = B + (size_t)t * kb;
    if (reg_sort) {
        // bitonic sort, descending, of kTopkRegSort entries in registers
        unsigned long long v[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int i = lane * 16 + e;
            v[e] = i < take ? sel[topk_swz(i)] : 0ull;
        }
        for (int k = 2; k <= kTopkRegSort; k <<= 1)
            for (int jj = k >> 1; jj > 0; jj >>= 1) {
                if (jj >= 16) {
                    const int lm = jj >> 4;
                    const bool upper = (lane & lm) != 0;      // this lane holds the higher index
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const bool desc = ((lane * 16 + e) & k) == 0;
                        const unsigned long long o = __shfl_xor_sync(0xffffffffu, v[e], lm);
                        const bool keep_max = desc != upper;
                        v[e] = keep_max ? (v[e] > o ? v[e] : o) : (v[e] < o ? v[e] : o);
                    }
                } else if (jj == 8) {
                    bitonic_in_lane<8>(v, lane, k);
                } else if (jj == 4) {
                    bitonic_in_lane<4>(v, lane, k);
                } else if (jj == 2) {
                    bitonic_in_lane<2>(v, lane, k);
                } else {
                    bitonic_in_lane<1>(v, lane, k);
                }
            }
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int i = lane * 16 + e;
            if (i < kb) out[i] = i < take ? (int32_t)(0xffffffffu - (uint32_t)(v[e] & 0xffffffffull)) : -1;
        }
        return;
    }
    for (int i = take + lane; i < kb2; i += 32) sel[i] = 0ull;
    __syncwarp();
    // bitonic sort, descending
    for (int k = 2; k <= kb2; k <<= 1)
        for (int jj = k >> 1; jj > 0; jj >>= 1) {
            for (int i = lane; i < kb2; i += 32) {
                const int ixj = i ^ jj;
                if (ixj > i) {
                    const bool desc = (i & k) == 0;
                    const unsigned long long a = sel[i], c = sel[ixj];
                    if (desc ? (a < c) : (a > c)) {
                        sel[i] = c;
                        sel[ixj] = a;
                    }
                }
            }
            __syncwarp();
        }
    for (int i = lane; i < kb; i += 32)
        out[i] = i < take ? (int32_t)(0xffffffffu - (uint32_t)(sel[i] & 0xffffffffull)) : -1;
}

// --------------------------------------------------------------------------- token sets
// One CTA per token: the selected blocks sorted ascending (-1 last), each expanded to its r
// tokens, then the tail r floor((pos + 1) / r) .. pos; positions within the sequence.
__global__ void __launch_bounds__(kTopkThreads)
qsa_token_sets_kernel(const int32_t *__restrict__ B, const int32_t *__restrict__ cu, int n_seq, int kb, int r,
                      int32_t *__restrict__ tokens, int32_t *__restrict__ count)
{
    extern __shared__ uint32_t blk[];                   // [kb_pow2]
    __shared__ int s_n;
    const int64_t t = blockIdx.x;
    const int s = upper_index(cu, n_seq + 1, t);
    const int64_t pos = t - cu[s];
    int kb2 = 1;
    while (kb2 < kb) kb2 <<= 1;
    if (threadIdx.x == 0) s_n = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < kb2; i += kTopkThreads) {
        const int32_t b = i < kb ? B[(size_t)t * kb + i] : -1;
        blk[i] = b >= 0 ? (uint32_t)b : 0xffffffffu;
        if (b >= 0) atomicAdd(&s_n, 1);
    }
    __syncthreads();
    for (int k = 2; k <= kb2; k <<= 1)
        for (int jj = k >> 1; jj > 0; jj >>= 1) {
            for (int i = threadIdx.x; i < kb2; i += kTopkThreads) {
                const int ixj = i ^ jj;
                if (ixj > i) {
                    const bool asc = (i & k) == 0;
                    const uint32_t a = blk[i], c = blk[ixj];
                    if (asc ? (a > c) : (a < c)) {
                        blk[i] = c;
                        blk[ixj] = a;
                    }
                }
            }
            __syncthreads();
        }
    const int n_sel = s_n;
    const int64_t tail0 = (int64_t)r * ((pos + 1) / r);
    const int n_tail = (int)(pos + 1 - tail0);
    const int width = kb * r + r - 1;
    int32_t *out = tokens + (size_t)t * width;
    for (int i = threadIdx.x; i < width; i += kTopkThreads) {
        int32_t v = -1;
        if (i < n_sel * r) v = (int32_t)(blk[i / r] * (uint32_t)r + (uint32_t)(i % r));
        else if (i < n_sel * r + n_tail) v = (int32_t)(tail0 + (i - n_sel * r));
        out[i] = v;
    }
    if (threadIdx.x == 0) count[t] = n_sel * r + n_tail;
}

}  // namespace qsa
}  // namespace gdn
