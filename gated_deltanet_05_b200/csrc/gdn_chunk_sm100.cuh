// gdn_chunk_sm100.cuh -- chunked prefill of the gated delta rule on sm_100a tensor cores.
//
// Computes the token update rule of the joezjh.github.io notes page "Qwen3.8-Flash-Next"
// (section "Gated DeltaNet 核心机制") for bf16 q/k/v with d_k = d_v = 128, in chunks of
// C = 64 tokens, through the chunked rewrite (exact up to rounding):
//   g_t = sum_{r<=t} log alpha_r, gamma_t = exp(g_t), Gamma_ts = exp(g_t - g_s), s <= t
//   L = strict_tril(diag(beta)(K K^T o Gamma)),  T = (I + L)^-1
//   W = T diag(beta gamma) K,  U = T diag(beta) V,  U~ = U - W S
//   Y = diag(gamma) Q S + tril(Q K^T o Gamma) U~
//   S <- gamma_C S + (diag(exp(g_C - g)) K)^T U~
// Every product is taken "value-major" so that the MMA M dimension is d_v = 128 (or
// d_k = 128) and all accumulators fill the 128 TMEM lanes:
//   G   = [K; Q] K^T                      M=128 (64 K rows, 64 Q rows), N=64, K=128
//   W^T = K^T (T diag(beta gamma))^T      M=128 (d_k), N=64, K=64       A MN-major
//   U^T = V^T (T diag(beta))^T            M=128 (d_v), N=64, K=64       A MN-major
//   U~^T = U^T - S^T W^T                  M=128 (d_v), N=64, K=128      B MN-major (-W^T)
//   Y^T  = S^T (diag(gamma) Q)^T + U~^T P^T   M=128, N=64, K=128 + 64
//   S^T <- gamma_C S^T + (U~^T diag(exp(g_C - g))) K   M=128, N=128, K=64, B MN-major
// The state S^T (value-major, the library's state layout) lives in TMEM in fp32 for the
// whole sequence; each chunk it is also written as an fp16 copy to shared memory as the
// MMA operand. Every exponent is <= 0.
//
// Operand precision: G = [K; Q] K^T runs on the bf16 inputs as loaded. Every other
// product runs on fp16 operands (kind::f16, fp32 accumulate): after G, the K, Q, V tiles
// are converted to fp16 in place (exact for |x| in [2^-14, 65504], which bf16 inputs of
// unit-norm keys/queries and O(1) values satisfy) and all derived operands (T diag(beta),
// T diag(beta gamma), P, -W^T, the S^T copy, U~^T) are rounded to fp16, whose 11-bit
// significand keeps the chunked form within the bf16-input accuracy bar where bf16
// (8-bit) operands do not. y is written in fp32 or bf16.
//
// One CTA owns one (sequence, head) chain. Warp roles (384 threads):
//   warp 0     TMA producer: K, Q, V tiles of each chunk (2-stage ring, 128B swizzle)
//   warp 1     TMEM allocator and single-thread tcgen05.mma issuer
//   warps 2-3  idle
//   warps 4-7  "solve" warpgroup: gates, L and P from G, the triangular solve (fp32,
//              blocked forward substitution in shared memory), T/P/Q/K/V fp16 operands,
//              and the -W^T operand from its TMEM accumulator
//   warps 8-11 "state" warpgroup: U~ -> fp16 operands, y = Y^T out, S carry
//              (scale by gamma_C, fp16 copy), S0 in and S_T out
// All mbarrier waits are bounded (~1 s); on a timeout the kernel records it in the
// device error word, every role leaves its loop, in-flight TMA and MMA work is drained
// (again with bounded waits) and TMEM is released before the CTA exits.
#pragma once
#include <cuda.h>

#include "gdn_common.cuh"
#include "sm100_ptx.cuh"

namespace gdn {
namespace sm100 {

constexpr int kC = 64;       // chunk length
constexpr int kD = 128;      // d_k = d_v
constexpr int kThreads = 384;
constexpr long long kWaitLimit = 2000000000LL;   // SM cycles (~1 s at 1.9 GHz)

// shared-memory layout (bytes from a 1024-aligned base)
constexpr uint32_t OFF_QK = 0;          // 2 stages x 32 KB: [K d0..63 | Q d0..63 | K d64.. | Q d64..]
constexpr uint32_t QK_STAGE = 32768;
constexpr uint32_t OFF_V = 65536;       // 2 stages x 16 KB: [V d0..63 | V d64..127]
constexpr uint32_t V_STAGE = 16384;
constexpr uint32_t OFF_SB = 98304;      // 32 KB fp16 S^T [128 v][128 k], K-major, two 16 KB halves
constexpr uint32_t OFF_UB = 131072;     // 16 KB fp16 U~^T [128 v][64 s]
constexpr uint32_t OFF_UD = 147456;     // 16 KB fp16 U~^T diag(exp(g_C - g))
constexpr uint32_t OFF_WB = 163840;     // 16 KB fp16 -W^T [128 k][64 t], MN-major
constexpr uint32_t OFF_P = 180224;      // 8 KB fp16 P [64 t][64 s]
constexpr uint32_t OFF_TBG = 188416;    // 8 KB fp16 T diag(beta gamma) [64 t][64 s]
constexpr uint32_t OFF_TB = 196608;     // 8 KB fp16 T diag(beta)
constexpr uint32_t OFF_LS = 204800;     // fp32 [64][65]: L, then T in place
constexpr int LS_LD = 65;
constexpr uint32_t OFF_RT = OFF_LS + 64 * LS_LD * 4;     // fp32 [16][48] block-row temp
constexpr uint32_t OFF_GATES = OFF_RT + 16 * 48 * 4;     // {g, gamma, beta}[64] fp32 of the solve's chunk
constexpr uint32_t OFF_BAR = OFF_GATES + 3 * 64 * 4;     // mbarriers
constexpr int N_BAR = 16;
constexpr uint32_t OFF_MISC = OFF_BAR + N_BAR * 8;       // tmem base, abort flag, chain's sequence
constexpr uint32_t SMEM_USED = OFF_MISC + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;        // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// TMEM columns (fp32, 128 lanes)
constexpr uint32_t TM_S = 0, TM_G = 128, TM_W = 192, TM_U = 256, TM_Y = 320, TM_COLS = 512;

// barrier indices
enum {
    B_FULL0 = 0, B_FULL1, B_EMPTY0, B_EMPTY1, B_GFULL, B_GEMPTY, B_TBG, B_WFULL, B_TB, B_WB,
    B_P, B_XFULL, B_UD, B_SFULL, B_SB, B_DRAIN
};

struct ChainInfo {
    int seq, h;
    int64_t bos, len;
};

// Inclusive scan of one chunk's log decays (zero past the sequence end), two tokens per
// lane: g_lo for tokens 0..31, g_hi for 32..63. Every warp that calls it gets
// bit-identical values.
__device__ __forceinline__ void chunk_log_decay_scan(const float *__restrict__ log_alpha, int64_t tok0,
                                                     int H, int h, int n_valid, int lane,
                                                     float &g_lo, float &g_hi)
{
    float x0 = lane < n_valid ? log_alpha[(size_t)(tok0 + lane) * H + h] : 0.f;
    float x1 = lane + 32 < n_valid ? log_alpha[(size_t)(tok0 + lane + 32) * H + h] : 0.f;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float o0 = __shfl_up_sync(0xffffffffu, x0, off);
        const float o1 = __shfl_up_sync(0xffffffffu, x1, off);
        if (lane >= off) {
            x0 += o0;
            x1 += o1;
        }
    }
    g_lo = x0;
    g_hi = x1 + __shfl_sync(0xffffffffu, x0, 31);
}

__device__ __forceinline__ float bf_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf_hi(uint32_t x) { return __uint_as_float(x & 0xFFFF0000u); }

template <typename TY>
__global__ void __launch_bounds__(kThreads, 1)
chunk_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ log_alpha,
                      const float *__restrict__ beta, const float *__restrict__ S0,
                      const int32_t *__restrict__ cu_seqlens, int n_seq, int H, float scale,
                      TY *__restrict__ y, float *__restrict__ S_T)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);

    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);
    float *Ls = reinterpret_cast<float *>(smem + OFF_LS);
    float *Rt = reinterpret_cast<float *>(smem + OFF_RT);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;

    // ---- which chain: sequences in order of decreasing length (ties by index), so the
    // longest chains start first; identity order beyond kThreads sequences
    const int rank = blockIdx.x / H;
    int *seq_slot = reinterpret_cast<int *>(smem + OFF_MISC + 8);
    if (n_seq > kThreads) {
        if (tid == 0) *seq_slot = rank;
    } else if (tid < n_seq) {
        const int ls = cu_seqlens[tid + 1] - cu_seqlens[tid];
        int rk = 0;
        for (int o = 0; o < n_seq; ++o) {
            const int lo = cu_seqlens[o + 1] - cu_seqlens[o];
            rk += (lo > ls) || (lo == ls && o < tid);
        }
        if (rk == rank) *seq_slot = tid;
    }

    // ---- setup
    if (tid == 0) {
        mbar_init(&bar[B_FULL0], 1);
        mbar_init(&bar[B_FULL1], 1);
        mbar_init(&bar[B_EMPTY0], 1);
        mbar_init(&bar[B_EMPTY1], 1);
        mbar_init(&bar[B_GFULL], 1);
        mbar_init(&bar[B_GEMPTY], 128);
        mbar_init(&bar[B_TBG], 128);
        mbar_init(&bar[B_WFULL], 1);
        mbar_init(&bar[B_TB], 128);
        mbar_init(&bar[B_WB], 128);
        mbar_init(&bar[B_P], 128);
        mbar_init(&bar[B_XFULL], 1);
        mbar_init(&bar[B_UD], 128);
        mbar_init(&bar[B_SFULL], 1);
        mbar_init(&bar[B_SB], 128);
        mbar_init(&bar[B_DRAIN], 1);
        *abort_flag = 0;
        fence_mbarrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    ChainInfo ci;
    ci.h = blockIdx.x % H;
    ci.seq = *seq_slot;
    ci.bos = cu_seqlens[ci.seq];
    ci.len = (int64_t)cu_seqlens[ci.seq + 1] - ci.bos;
    const int n_chunks = (int)((ci.len + kC - 1) / kC);
    const size_t state_off = ((size_t)ci.seq * H + ci.h) * (size_t)kD * kD;

    if (warp == 0) {
        // ================================================================ TMA producer
        if (lane == 0 && n_chunks > 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            int issued[2] = {0, 0};
            for (int c = 0; c < n_chunks; ++c) {
                const int st = c & 1;
                if (c >= 2 && !mbar_wait_bounded(&bar[B_EMPTY0 + st], ((c >> 1) - 1) & 1, abort_flag, kWaitLimit))
                    break;
                const int tok = (int)(ci.bos + (int64_t)c * kC);
                uint8_t *qk = smem + OFF_QK + st * QK_STAGE;
                uint8_t *vv = smem + OFF_V + st * V_STAGE;
                mbar_arrive_expect_tx(&bar[B_FULL0 + st], QK_STAGE + V_STAGE);
                tma_load_3d(qk + 0, &tm_k, &bar[B_FULL0 + st], 0, ci.h, tok);
                tma_load_3d(qk + 8192, &tm_q, &bar[B_FULL0 + st], 0, ci.h, tok);
                tma_load_3d(qk + 16384, &tm_k, &bar[B_FULL0 + st], 64, ci.h, tok);
                tma_load_3d(qk + 24576, &tm_q, &bar[B_FULL0 + st], 64, ci.h, tok);
                tma_load_3d(vv + 0, &tm_v, &bar[B_FULL0 + st], 0, ci.h, tok);
                tma_load_3d(vv + 8192, &tm_v, &bar[B_FULL0 + st], 64, ci.h, tok);
                issued[st] = c + 1;
            }
            // drain: no TMA write may land after the CTA exits
            for (int st = 0; st < 2; ++st)
                if (issued[st] > 0)
                    mbar_wait_drain(&bar[B_FULL0 + st], ((issued[st] - 1) >> 1) & 1, kWaitLimit);
        }
    } else if (warp == 1) {
        // ================================================================ MMA issuer
        if (lane == 0 && n_chunks > 0) {
            const uint32_t id_g = idesc_f32acc(kFmtBF16, 128, 64, 0, 0);
            const uint32_t id_wu = idesc_f32acc(kFmtF16, 128, 64, 1, 0);
            const uint32_t id_xw = idesc_f32acc(kFmtF16, 128, 64, 0, 1);
            const uint32_t id_yq = idesc_f32acc(kFmtF16, 128, 64, 0, 0);
            const uint32_t id_s = idesc_f32acc(kFmtF16, 128, 128, 0, 1);
            bool ok = true;
            auto issue_G = [&](int c) -> bool {
                const int st = c & 1;
                if (!mbar_wait_bounded(&bar[B_FULL0 + st], (c >> 1) & 1, abort_flag, kWaitLimit)) return false;
                if (c > 0 && !mbar_wait_bounded(&bar[B_GEMPTY], (c - 1) & 1, abort_flag, kWaitLimit)) return false;
                tc_fence_after();
                const uint32_t qk = sbase + OFF_QK + st * QK_STAGE;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t a = qk + (kk >> 2) * 16384 + (kk & 3) * 32;
                    mma_f16kind_ss(tmem + TM_G, sdesc_sw128(a, 16, 1024), sdesc_sw128(a, 16, 1024), id_g, kk > 0);
                }
                mma_commit(&bar[B_GFULL]);
                return true;
            };
            auto issue_W = [&](int c) -> bool {
                if (!mbar_wait_bounded(&bar[B_TBG], c & 1, abort_flag, kWaitLimit)) return false;
                tc_fence_after();
                const uint32_t kt = sbase + OFF_QK + (c & 1) * QK_STAGE;   // K^T: MN-major, LBO 16 KB
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f16kind_ss(tmem + TM_W, sdesc_sw128(kt + kk * 2048, 16384, 1024),
                                sdesc_sw128(sbase + OFF_TBG + kk * 32, 16, 1024), id_wu, kk > 0);
                mma_commit(&bar[B_WFULL]);
                return true;
            };
            auto issue_U = [&](int c) -> bool {
                if (!mbar_wait_bounded(&bar[B_TB], c & 1, abort_flag, kWaitLimit)) return false;
                tc_fence_after();
                const uint32_t vt = sbase + OFF_V + (c & 1) * V_STAGE;     // V^T: MN-major, LBO 8 KB
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f16kind_ss(tmem + TM_U, sdesc_sw128(vt + kk * 2048, 8192, 1024),
                                sdesc_sw128(sbase + OFF_TB + kk * 32, 16, 1024), id_wu, kk > 0);
                return true;
            };
            auto issue_X = [&](int c) -> bool {
                if (!mbar_wait_bounded(&bar[B_WB], c & 1, abort_flag, kWaitLimit)) return false;
                if (!mbar_wait_bounded(&bar[B_SB], c & 1, abort_flag, kWaitLimit)) return false;
                tc_fence_after();
                const uint32_t qk = sbase + OFF_QK + (c & 1) * QK_STAGE;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t a = sbase + OFF_SB + (kk >> 2) * 16384 + (kk & 3) * 32;
                    // U~^T += S^T (-W^T): B = -W^T stored [k][t], MN-major
                    mma_f16kind_ss(tmem + TM_U, sdesc_sw128(a, 16, 1024),
                                sdesc_sw128(sbase + OFF_WB + kk * 2048, 8192, 1024), id_xw, 1);
                    // Y^T = S^T (gamma Q)^T: B = Q rows (K-major), Q at +8 KB / +24 KB
                    mma_f16kind_ss(tmem + TM_Y, sdesc_sw128(a, 16, 1024),
                                sdesc_sw128(qk + 8192 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                                id_yq, kk > 0);
                }
                mma_commit(&bar[B_XFULL]);
                return true;
            };
            auto issue_S = [&](int c) -> bool {
                if (!mbar_wait_bounded(&bar[B_UD], c & 1, abort_flag, kWaitLimit)) return false;
                if (!mbar_wait_bounded(&bar[B_P], c & 1, abort_flag, kWaitLimit)) return false;
                tc_fence_after();
                const uint32_t kb = sbase + OFF_QK + (c & 1) * QK_STAGE;   // K as [s][k]: MN-major B
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    mma_f16kind_ss(tmem + TM_Y, sdesc_sw128(sbase + OFF_UB + kk * 32, 16, 1024),
                                sdesc_sw128(sbase + OFF_P + kk * 32, 16, 1024), id_yq, 1);
                    mma_f16kind_ss(tmem + TM_S, sdesc_sw128(sbase + OFF_UD + kk * 32, 16, 1024),
                                sdesc_sw128(kb + kk * 2048, 16384, 1024), id_s, 1);
                }
                mma_commit(&bar[B_SFULL]);
                mma_commit(&bar[B_EMPTY0 + (c & 1)]);
                return true;
            };
            ok = issue_G(0) && issue_W(0) && issue_U(0) && issue_X(0);
            for (int c = 0; ok && c < n_chunks; ++c) {
                if (c + 1 < n_chunks) ok = issue_G(c + 1);
                ok = ok && issue_S(c);
                if (ok && c + 1 < n_chunks) ok = issue_W(c + 1) && issue_U(c + 1) && issue_X(c + 1);
            }
            // drain the tensor pipe before TMEM is released
            mma_commit(&bar[B_DRAIN]);
            mbar_wait_drain(&bar[B_DRAIN], 0, kWaitLimit);
        }
    } else if (warp >= 4 && warp < 8) {
        // ================================================================ solve warpgroup
        const int r = tid - 128;              // TMEM lane / row
        const int t = r & 63;
        const uint32_t lane_base = (uint32_t)(warp & 3) * 32u << 16;
        for (int c = 0; c < n_chunks; ++c) {
            float *gs = reinterpret_cast<float *>(smem + OFF_GATES);
            float *gam = gs + 64, *bet = gs + 128;
            const int64_t tok0 = ci.bos + (int64_t)c * kC;
            const int n_valid = (int)(ci.len - (int64_t)c * kC < kC ? ci.len - (int64_t)c * kC : kC);
            if (warp == 4) {
                // gates of this chunk
                float g_lo, g_hi;
                chunk_log_decay_scan(log_alpha, tok0, H, ci.h, n_valid, lane, g_lo, g_hi);
                gs[lane] = g_lo;
                gs[lane + 32] = g_hi;
                gam[lane] = expf(g_lo);
                gam[lane + 32] = expf(g_hi);
                bet[lane] = lane < n_valid ? beta[(size_t)(tok0 + lane) * H + ci.h] : 0.f;
                bet[lane + 32] = lane + 32 < n_valid ? beta[(size_t)(tok0 + lane + 32) * H + ci.h] : 0.f;
            }
            // (a) G = [K K^T ; Q K^T] rows
            bool ok = true;
            if (r == 0) ok = mbar_wait_bounded(&bar[B_GFULL], c & 1, abort_flag, kWaitLimit);
            if (!named_bar_and(1, 128, ok)) break;
            tc_fence_after();
            uint32_t gv[64];
            {
                uint32_t (&g0)[32] = *reinterpret_cast<uint32_t (*)[32]>(&gv[0]);
                uint32_t (&g1)[32] = *reinterpret_cast<uint32_t (*)[32]>(&gv[32]);
                tmem_ld_x32(tmem + lane_base + TM_G, g0);
                tmem_ld_x32(tmem + lane_base + TM_G + 32, g1);
                tmem_wait_ld();
            }
            tc_fence_before();
            mbar_arrive(&bar[B_GEMPTY]);
            const float gt = gs[t];
            uint32_t pk[32];                  // P row (threads 64..127), fp16 pairs
            if (r < 64) {
                const float bt = bet[t];
#pragma unroll
                for (int s = 0; s < 64; ++s)
                    Ls[t * LS_LD + s] = (s < t) ? bt * __uint_as_float(gv[s]) * expf(gt - gs[s]) : 0.f;
            } else {
#pragma unroll
                for (int s = 0; s < 64; s += 2) {
                    const float p0 = (s <= t) ? scale * __uint_as_float(gv[s]) * expf(gt - gs[s]) : 0.f;
                    const float p1 = (s + 1 <= t) ? scale * __uint_as_float(gv[s + 1]) * expf(gt - gs[s + 1]) : 0.f;
                    pk[s >> 1] = pack_f16x2(p0, p1);
                }
            }
            named_bar_sync(1, 128);
            // (b) T = (I + L)^-1: 16x16 diagonal blocks, one column per thread in registers
            if (r < 64) {
                const int j = r, b0 = (j >> 4) << 4, jb = j & 15;
                float x[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float acc = (i == jb) ? 1.f : 0.f;
#pragma unroll
                    for (int s = 0; s < i; ++s)
                        if (s >= jb) acc = fmaf(-Ls[(b0 + i) * LS_LD + b0 + s], x[s], acc);
                    x[i] = (i < jb) ? 0.f : acc;
                }
                named_bar_sync(3, 64);        // the 64 column threads have read their L blocks
#pragma unroll
                for (int i = 0; i < 16; ++i) Ls[(b0 + i) * LS_LD + j] = x[i];
            }
            named_bar_sync(1, 128);
            // off-diagonal block rows: T_ij = -T_ii sum_{k=j}^{i-1} L_ik T_kj
            for (int ib = 1; ib < 4; ++ib) {
                const int w = 16 * ib, n_out = 16 * w;
                for (int o = r; o < n_out; o += 128) {
                    const int i = o / w, jj = o % w;
                    float acc = 0.f;
                    for (int s = (jj >> 4) << 4; s < w; ++s)
                        acc = fmaf(Ls[(w + i) * LS_LD + s], Ls[s * LS_LD + jj], acc);
                    Rt[i * 48 + jj] = acc;
                }
                named_bar_sync(1, 128);
                for (int o = r; o < n_out; o += 128) {
                    const int i = o / w, jj = o % w;
                    float acc = 0.f;
                    for (int m = 0; m <= i; ++m)
                        acc = fmaf(-Ls[(w + i) * LS_LD + w + m], Rt[m * 48 + jj], acc);
                    Ls[(w + i) * LS_LD + jj] = acc;
                }
                named_bar_sync(1, 128);
            }
            // (c) T diag(beta gamma) (rows by threads 0..63) and the input tiles in place
            const uint32_t qk_off = OFF_QK + (c & 1) * QK_STAGE;
            if (r < 64) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    uint4 v4;
                    uint32_t *vv = reinterpret_cast<uint32_t *>(&v4);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int s = ch * 8 + 2 * e;
                        vv[e] = pack_f16x2(Ls[t * LS_LD + s] * bet[s] * gam[s],
                                            Ls[t * LS_LD + s + 1] * bet[s + 1] * gam[s + 1]);
                    }
                    *reinterpret_cast<uint4 *>(smem + OFF_TBG + sw128_off(t, ch)) = v4;
                }
            }
            {
                // the stage's K, V tiles -> fp16 in place (exact); Q -> fp16(gamma_t * scale * q_t).
                // Thread r owns token row t of the d-half (r >> 6) of each tile; a whole
                // 128-byte row is rewritten, so the swizzle does not matter.
                const float sc = gam[t] * scale;
                uint8_t *rows[3] = {smem + qk_off + (r >> 6) * 16384 + t * 128,
                                    smem + qk_off + 8192 + (r >> 6) * 16384 + t * 128,
                                    smem + OFF_V + (c & 1) * V_STAGE + (r >> 6) * 8192 + t * 128};
#pragma unroll
                for (int which = 0; which < 3; ++which) {
                    const float f = which == 1 ? sc : 1.f;
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        uint4 v4 = *reinterpret_cast<uint4 *>(rows[which] + ch * 16);
                        uint32_t *vv = reinterpret_cast<uint32_t *>(&v4);
#pragma unroll
                        for (int e = 0; e < 4; ++e) vv[e] = pack_f16x2(bf_lo(vv[e]) * f, bf_hi(vv[e]) * f);
                        *reinterpret_cast<uint4 *>(rows[which] + ch * 16) = v4;
                    }
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&bar[B_TBG]);
            // (d) T diag(beta) once the previous chunk's U^T product is done (x_full(c-1))
            ok = true;
            if (c > 0 && r == 0) ok = mbar_wait_bounded(&bar[B_XFULL], (c - 1) & 1, abort_flag, kWaitLimit);
            if (!named_bar_and(1, 128, ok)) break;
            if (r >= 64) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    uint4 v4;
                    uint32_t *vv = reinterpret_cast<uint32_t *>(&v4);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int s = ch * 8 + 2 * e;
                        vv[e] = pack_f16x2(Ls[t * LS_LD + s] * bet[s], Ls[t * LS_LD + s + 1] * bet[s + 1]);
                    }
                    *reinterpret_cast<uint4 *>(smem + OFF_TB + sw128_off(t, ch)) = v4;
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&bar[B_TB]);
            // (e) P once the previous chunk's state products are done (s_full(c-1))
            ok = true;
            if (c > 0 && r == 0) ok = mbar_wait_bounded(&bar[B_SFULL], (c - 1) & 1, abort_flag, kWaitLimit);
            if (!named_bar_and(1, 128, ok)) break;
            if (r >= 64) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch)
                    *reinterpret_cast<uint4 *>(smem + OFF_P + sw128_off(t, ch)) =
                        make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
            }
            fence_proxy_async_smem();
            mbar_arrive(&bar[B_P]);
            // (f) -W^T from its accumulator into the MN-major operand [k][t]
            ok = true;
            if (r == 0) ok = mbar_wait_bounded(&bar[B_WFULL], c & 1, abort_flag, kWaitLimit);
            if (!named_bar_and(1, 128, ok)) break;
            tc_fence_after();
            {
                uint32_t (&w0)[32] = *reinterpret_cast<uint32_t (*)[32]>(&gv[0]);
                uint32_t (&w1)[32] = *reinterpret_cast<uint32_t (*)[32]>(&gv[32]);
                tmem_ld_x32(tmem + lane_base + TM_W, w0);
                tmem_ld_x32(tmem + lane_base + TM_W + 32, w1);
                tmem_wait_ld();
            }
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                uint4 v4;
                uint32_t *vv = reinterpret_cast<uint32_t *>(&v4);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    vv[e] = pack_f16x2(-__uint_as_float(gv[ch * 8 + 2 * e]), -__uint_as_float(gv[ch * 8 + 2 * e + 1]));
                *reinterpret_cast<uint4 *>(smem + OFF_WB + sw128_off(r, ch)) = v4;
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bar[B_WB]);
        }
    } else if (warp >= 8) {
        // ================================================================ state warpgroup
        const int r = tid - 256;              // TMEM lane = value index v
        const uint32_t lane_base = (uint32_t)(warp & 3) * 32u << 16;
        // every warp scans the log decays itself (bit-identical to the solve warpgroup's)
        auto scan = [&](int c, float &g_lo, float &g_hi) {
            const int64_t tok0 = ci.bos + (int64_t)c * kC;
            const int n_valid = (int)(ci.len - (int64_t)c * kC < kC ? ci.len - (int64_t)c * kC : kC);
            chunk_log_decay_scan(log_alpha, tok0, H, ci.h, n_valid, lane, g_lo, g_hi);
        };
        float g_lo = 0.f, g_hi = 0.f;
        if (n_chunks > 0) scan(0, g_lo, g_hi);
        // S0 -> TMEM (scaled by gamma_C of chunk 0) and its fp16 copy
        {
            const float gC = expf(__shfl_sync(0xffffffffu, g_hi, 31));
            const float *src = S0 ? S0 + state_off + (size_t)r * kD : nullptr;
            if (n_chunks == 0) {
                if (S_T) {
                    float *dst = S_T + state_off + (size_t)r * kD;
                    for (int i = 0; i < kD; i += 4)
                        store4(dst + i, src ? load4(src + i) : make_float4(0.f, 0.f, 0.f, 0.f));
                }
            } else {
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint32_t sv[32];
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        const float4 f = src ? load4(src + q4 * 32 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
                        sv[i] = __float_as_uint(f.x);
                        sv[i + 1] = __float_as_uint(f.y);
                        sv[i + 2] = __float_as_uint(f.z);
                        sv[i + 3] = __float_as_uint(f.w);
                    }
                    uint8_t *sb_half = smem + OFF_SB + (q4 >> 1) * 16384;
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        const int e0 = ch * 8;
                        *reinterpret_cast<uint4 *>(sb_half + sw128_off(r, (q4 & 1) * 4 + ch)) = make_uint4(
                            pack_f16x2(__uint_as_float(sv[e0]), __uint_as_float(sv[e0 + 1])),
                            pack_f16x2(__uint_as_float(sv[e0 + 2]), __uint_as_float(sv[e0 + 3])),
                            pack_f16x2(__uint_as_float(sv[e0 + 4]), __uint_as_float(sv[e0 + 5])),
                            pack_f16x2(__uint_as_float(sv[e0 + 6]), __uint_as_float(sv[e0 + 7])));
                    }
#pragma unroll
                    for (int i = 0; i < 32; ++i) sv[i] = __float_as_uint(__uint_as_float(sv[i]) * gC);
                    tmem_st_x32(tmem + lane_base + TM_S + q4 * 32, sv);
                }
                tmem_wait_st();
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(&bar[B_SB]);
            }
        }
        for (int c = 0; c < n_chunks; ++c) {
            const int64_t tok0 = ci.bos + (int64_t)c * kC;
            const int n_valid = (int)(ci.len - (int64_t)c * kC < kC ? ci.len - (int64_t)c * kC : kC);
            const bool last = (c + 1 == n_chunks);
            // exp(g_C - g_s) of this chunk, two per lane
            const float gC = __shfl_sync(0xffffffffu, g_hi, 31);
            const float dec_lo = expf(gC - g_lo), dec_hi = expf(gC - g_hi);
            // the next chunk's scan (its gamma_C scales the carried state below)
            float n_lo = 0.f, n_hi = 0.f;
            if (!last) scan(c + 1, n_lo, n_hi);
            const float gC_next = last ? 1.f : expf(__shfl_sync(0xffffffffu, n_hi, 31));
            // E2: U~^T -> fp16 operands (plain and decayed)
            bool ok = true;
            if (r == 0) ok = mbar_wait_bounded(&bar[B_XFULL], c & 1, abort_flag, kWaitLimit);
            if (!named_bar_and(2, 128, ok)) break;
            tc_fence_after();
            {
                uint32_t u[64];
                uint32_t (&u0)[32] = *reinterpret_cast<uint32_t (*)[32]>(&u[0]);
                uint32_t (&u1)[32] = *reinterpret_cast<uint32_t (*)[32]>(&u[32]);
                tmem_ld_x32(tmem + lane_base + TM_U, u0);
                tmem_ld_x32(tmem + lane_base + TM_U + 32, u1);
                tmem_wait_ld();
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    uint4 a4, d4;
                    uint32_t *aa = reinterpret_cast<uint32_t *>(&a4), *dd = reinterpret_cast<uint32_t *>(&d4);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int s = ch * 8 + 2 * e;
                        const float u0f = __uint_as_float(u[s]), u1f = __uint_as_float(u[s + 1]);
                        const float d0 = __shfl_sync(0xffffffffu, s < 32 ? dec_lo : dec_hi, s & 31);
                        const float d1 = __shfl_sync(0xffffffffu, s + 1 < 32 ? dec_lo : dec_hi, (s + 1) & 31);
                        aa[e] = pack_f16x2(u0f, u1f);
                        dd[e] = pack_f16x2(u0f * d0, u1f * d1);
                    }
                    *reinterpret_cast<uint4 *>(smem + OFF_UB + sw128_off(r, ch)) = a4;
                    *reinterpret_cast<uint4 *>(smem + OFF_UD + sw128_off(r, ch)) = d4;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bar[B_UD]);
            // E3: y out, S carry
            ok = true;
            if (r == 0) ok = mbar_wait_bounded(&bar[B_SFULL], c & 1, abort_flag, kWaitLimit);
            if (!named_bar_and(2, 128, ok)) break;
            tc_fence_after();
            {
                uint32_t yv[64];
                uint32_t (&y0)[32] = *reinterpret_cast<uint32_t (*)[32]>(&yv[0]);
                uint32_t (&y1)[32] = *reinterpret_cast<uint32_t (*)[32]>(&yv[32]);
                tmem_ld_x32(tmem + lane_base + TM_Y, y0);
                tmem_ld_x32(tmem + lane_base + TM_Y + 32, y1);
                tmem_wait_ld();
                TY *yp = y + ((size_t)tok0 * H + ci.h) * kD + r;
#pragma unroll 8
                for (int tt = 0; tt < 64; ++tt)
                    if (tt < n_valid) yp[(size_t)tt * H * kD] = from_f32<TY>(__uint_as_float(yv[tt]));
            }
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                uint32_t sv[32];
                tmem_ld_x32(tmem + lane_base + TM_S + q4 * 32, sv);
                tmem_wait_ld();
                if (last) {
                    if (S_T) {
                        float *dst = S_T + state_off + (size_t)r * kD + q4 * 32;
#pragma unroll
                        for (int i = 0; i < 32; i += 4)
                            store4(dst + i, make_float4(__uint_as_float(sv[i]), __uint_as_float(sv[i + 1]),
                                                        __uint_as_float(sv[i + 2]), __uint_as_float(sv[i + 3])));
                    }
                } else {
                    uint8_t *sb_half = smem + OFF_SB + (q4 >> 1) * 16384;
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        const int e0 = ch * 8;
                        *reinterpret_cast<uint4 *>(sb_half + sw128_off(r, (q4 & 1) * 4 + ch)) = make_uint4(
                            pack_f16x2(__uint_as_float(sv[e0]), __uint_as_float(sv[e0 + 1])),
                            pack_f16x2(__uint_as_float(sv[e0 + 2]), __uint_as_float(sv[e0 + 3])),
                            pack_f16x2(__uint_as_float(sv[e0 + 4]), __uint_as_float(sv[e0 + 5])),
                            pack_f16x2(__uint_as_float(sv[e0 + 6]), __uint_as_float(sv[e0 + 7])));
                    }
#pragma unroll
                    for (int i = 0; i < 32; ++i) sv[i] = __float_as_uint(__uint_as_float(sv[i]) * gC_next);
                    tmem_st_x32(tmem + lane_base + TM_S + q4 * 32, sv);
                }
            }
            if (!last) {
                tmem_wait_st();
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(&bar[B_SB]);
            }
            g_lo = n_lo;
            g_hi = n_hi;
        }
    }

    // ---- teardown: every role has left its loop and drained its own async work
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

}  // namespace sm100
}  // namespace gdn
