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
//   G    = [K; Q] K^T                      M=128 (64 K rows, 64 Q rows), N=64, K=128
//   W^T  = K^T (T diag(beta gamma))^T      M=128 (d_k), N=64, K=64       A MN-major
//   U^T  = V^T (T diag(beta))^T            M=128 (d_v), N=64, K=64       A MN-major
//   U~^T = U^T - S^T W^T                   M=128 (d_v), N=64, K=128      B MN-major (-W^T)
//   Y^T  = S^T (diag(gamma) Q)^T + U~^T P^T    M=128, N=64, K=128 + 64
//   S^T <- gamma_C S^T + (U~^T diag(exp(g_C - g))) K   M=128, N=128, K=64, B MN-major
// The state S^T (value-major, the library's state layout) lives in TMEM in fp32 for the
// whole sequence; each chunk it is also written as an fp16 copy to shared memory as the
// MMA operand. Every exponent is <= 0 (exponentials are taken base 2 on log2-scaled
// decays, with the SM's approximate exp2 instruction).
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
//   warp 0      TMA producer: K, Q, V tiles of each chunk (2-stage ring, 128B swizzle)
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//   warps 2-3   converters: the stage's K, V -> fp16 and Q -> fp16(gamma scale q), in place
//   warps 4-7   "solve" warpgroup: L and P from G, T = (I + L)^-1 (16x16 diagonal blocks
//               by fp32 forward substitution, then two levels of block merges on tf32
//               mma.sync tiles), the fp16 T/P operands and -W^T from its TMEM accumulator
//   warps 8-11  "state" warpgroup: U~ -> fp16 operands, the fp16 state copy, y out,
//               the state carry (scale by gamma_C), S0 in and S_T out
// The state warpgroup publishes the fp16 copy of S_{c+1} and the rescaled fp32 state
// before it writes y_c, which keeps the y stores off the chunk-to-chunk critical path;
// the Y^T accumulator is double-buffered for that reason, and y leaves through a
// shared-memory staging tile and one asynchronous bulk copy per token row. The MMA issuer polls its
// barriers and issues whichever product is ready (chain products first), so the next
// chunk's K K^T / Q K^T and solve overlap the current chunk's state chain.
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
constexpr float kLog2e = 1.4426950408889634f;

// shared-memory layout (bytes from a 1024-aligned base)
constexpr uint32_t OFF_QK = 0;          // 2 stages x 32 KB: [K d0..63 | Q d0..63 | K d64.. | Q d64..]
constexpr uint32_t QK_STAGE = 32768;
constexpr uint32_t OFF_V = 65536;       // 2 stages x 16 KB: [V d0..63 | V d64..127]
constexpr uint32_t V_STAGE = 16384;
constexpr uint32_t OFF_SB = 98304;      // 32 KB fp16 S^T [128 v][128 k], K-major, two 16 KB halves
constexpr uint32_t OFF_UB = 131072;     // 16 KB fp16 U~^T [128 v][64 s]
constexpr uint32_t OFF_UD = 147456;     // 16 KB fp16 U~^T diag(exp(g_C - g))
constexpr uint32_t OFF_WB = 163840;     // 16 KB fp16 -W^T [128 k][64 t], MN-major
constexpr uint32_t OFF_YST = OFF_UB;    // y staging [64 t][128 v] (32 KB over U~b and U~d, free in E3)
constexpr uint32_t OFF_SPARE = 180224;  // 8 KB unused
constexpr uint32_t OFF_TBG = 188416;    // 8 KB fp16 T diag(beta gamma) [64 t][64 s]
constexpr uint32_t OFF_TB = 196608;     // 8 KB fp16 T diag(beta)
constexpr uint32_t OFF_LS = 204800;     // fp32 [64][68]: L, then T in place
constexpr int LS_LD = 68;
constexpr uint32_t OFF_RT = OFF_LS + 64 * LS_LD * 4;     // fp32 merge temp: [32][8] per solve warp
constexpr int RT_LD = 36;                                // (region sized [32][36])
constexpr float kSpanMax = 240.f;       // log2 span of a chunk's decays for the factored Gamma
constexpr uint32_t OFF_GATES = OFF_RT + 32 * RT_LD * 4;  // {g2, gamma, beta, 2^(m - g2)}[64] fp32 of the solve's chunk
constexpr uint32_t OFF_DEC = OFF_GATES + 4 * 64 * 4;     // state warpgroup: exp(g_C - g)[64] per warp
constexpr uint32_t OFF_BAR = OFF_DEC + 4 * 64 * 4;       // mbarriers
constexpr int N_BAR = 19;
constexpr uint32_t OFF_MISC = OFF_BAR + N_BAR * 8;       // tmem base, abort flag, chain's sequence
constexpr uint32_t SMEM_USED = OFF_MISC + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;        // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// TMEM columns (fp32, 128 lanes); the Y^T accumulator is double-buffered
constexpr uint32_t TM_S = 0, TM_G = 128, TM_W = 192, TM_U = 256, TM_Y = 320, TM_COLS = 512;

// barrier indices
enum {
    B_FULL0 = 0, B_FULL1, B_EMPTY0, B_EMPTY1, B_GFULL, B_GEMPTY, B_CONV, B_TBG, B_WFULL, B_TB,
    B_WB, B_P, B_XFULL, B_UD, B_SFULL, B_SB, B_SACC, B_UFULL, B_DRAIN
};
static_assert(B_DRAIN + 1 == N_BAR, "barrier count");

// named barriers (0 is __syncthreads)
enum { NB_SOLVE = 1, NB_STATE = 2, NB_SOLVE_LO = 3, NB_CONV = 4 };

struct ChainInfo {
    int seq, h;
    int64_t bos, len;
};

// Inclusive scan of one chunk's log2-scaled decays (zero past the sequence end), two
// tokens per lane: g_lo for tokens 0..31, g_hi for 32..63. Every warp that calls it gets
// bit-identical values.
__device__ __forceinline__ void chunk_log2_decay_scan(const float *__restrict__ log_alpha, int64_t tok0,
                                                      int H, int h, int n_valid, int lane,
                                                      float &g_lo, float &g_hi)
{
    float x0 = lane < n_valid ? log_alpha[(size_t)(tok0 + lane) * H + h] * kLog2e : 0.f;
    float x1 = lane + 32 < n_valid ? log_alpha[(size_t)(tok0 + lane + 32) * H + h] * kLog2e : 0.f;
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

__device__ __forceinline__ uint4 lds128(const uint8_t *p) { return *reinterpret_cast<const uint4 *>(p); }
__device__ __forceinline__ void sts128(uint8_t *p, uint4 v) { *reinterpret_cast<uint4 *>(p) = v; }
__device__ __forceinline__ float4 ldsf4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ void stsf4(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }

// fp16 pairs of 8 consecutive floats
__device__ __forceinline__ uint4 pack8_f16(const float *x)
{
    return make_uint4(pack_f16x2(x[0], x[1]), pack_f16x2(x[2], x[3]), pack_f16x2(x[4], x[5]),
                      pack_f16x2(x[6], x[7]));
}

// One bf16 16-byte chunk -> fp16, each value multiplied by f.
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 v, float f)
{
    return make_uint4(pack_f16x2(bf_lo(v.x) * f, bf_hi(v.x) * f), pack_f16x2(bf_lo(v.y) * f, bf_hi(v.y) * f),
                      pack_f16x2(bf_lo(v.z) * f, bf_hi(v.z) * f), pack_f16x2(bf_lo(v.w) * f, bf_hi(v.w) * f));
}

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
    int *seq_slot = reinterpret_cast<int *>(smem + OFF_MISC + 8);
    float *Ls = reinterpret_cast<float *>(smem + OFF_LS);
    float *Rt = reinterpret_cast<float *>(smem + OFF_RT);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;

    // ---- which chain: sequences in order of decreasing length (ties by index), so the
    // longest chains start first; identity order beyond kThreads sequences
    const int rank = blockIdx.x / H;
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
        for (int b = 0; b < N_BAR; ++b) {
            uint32_t count = 1;
            if (b == B_GEMPTY || b == B_TBG || b == B_TB || b == B_WB || b == B_P || b == B_UD ||
                b == B_SB || b == B_SACC)
                count = 128;
            if (b == B_CONV) count = 64;
            mbar_init(&bar[b], count);
        }
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
    auto chunk_valid = [&](int c) -> int {
        const int64_t rem = ci.len - (int64_t)c * kC;
        return (int)(rem < kC ? rem : kC);
    };

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
            auto done = [&](int b, int parity) { return mbar_test(&bar[b], parity & 1); };
            // Base descriptors, computed once; a k-step adds a constant to the start address
            // field (addresses < 256 KB keep it inside its 14 bits).
            const uint64_t dqk0 = sdesc_sw128(sbase + OFF_QK, 16, 1024);
            const uint64_t dkt0 = sdesc_sw128(sbase + OFF_QK, 16384, 1024);     // K^T / K as MN-major
            const uint64_t dvt0 = sdesc_sw128(sbase + OFF_V, 8192, 1024);       // V^T MN-major
            const uint64_t dtbg = sdesc_sw128(sbase + OFF_TBG, 16, 1024);
            const uint64_t dtb = sdesc_sw128(sbase + OFF_TB, 16, 1024);
            const uint64_t dsb = sdesc_sw128(sbase + OFF_SB, 16, 1024);
            const uint64_t dwb = sdesc_sw128(sbase + OFF_WB, 8192, 1024);
            const uint64_t dub = sdesc_sw128(sbase + OFF_UB, 16, 1024);
            const uint64_t dud = sdesc_sw128(sbase + OFF_UD, 16, 1024);
            const uint64_t dv0 = sdesc_sw128(sbase + OFF_V, 16, 1024);          // P in the V stage
#define GDN_DOFF(bytes) ((uint64_t)((bytes) >> 4))
            auto do_G = [&](int c) {
                const uint64_t base = dqk0 + GDN_DOFF((c & 1) * QK_STAGE);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t d = base + GDN_DOFF((kk >> 2) * 16384 + (kk & 3) * 32);
                    mma_f16kind_ss(tmem + TM_G, d, d, id_g, kk > 0);
                }
                mma_commit(&bar[B_GFULL]);
            };
            auto do_W = [&](int c) {
                const uint64_t kt = dkt0 + GDN_DOFF((c & 1) * QK_STAGE);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f16kind_ss(tmem + TM_W, kt + GDN_DOFF(kk * 2048), dtbg + GDN_DOFF(kk * 32), id_wu, kk > 0);
                mma_commit(&bar[B_WFULL]);
            };
            auto do_U = [&](int c) {
                const uint64_t vt = dvt0 + GDN_DOFF((c & 1) * V_STAGE);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f16kind_ss(tmem + TM_U, vt + GDN_DOFF(kk * 2048), dtb + GDN_DOFF(kk * 32), id_wu, kk > 0);
                mma_commit(&bar[B_UFULL]);
            };
            auto do_X = [&](int c) {
                const uint64_t q0 = dqk0 + GDN_DOFF((c & 1) * QK_STAGE + 8192);
                const uint32_t ty = tmem + TM_Y + (c & 1) * 64;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t a = dsb + GDN_DOFF((kk >> 2) * 16384 + (kk & 3) * 32);
                    // U~^T += S^T (-W^T): B = -W^T stored [k][t], MN-major
                    mma_f16kind_ss(tmem + TM_U, a, dwb + GDN_DOFF(kk * 2048), id_xw, 1);
                    // Y^T = S^T (gamma scale Q)^T: B = Q rows (K-major), Q at +8 KB / +24 KB
                    mma_f16kind_ss(ty, a, q0 + GDN_DOFF((kk >> 2) * 16384 + (kk & 3) * 32), id_yq, kk > 0);
                }
                mma_commit(&bar[B_XFULL]);
            };
            auto do_S = [&](int c) {
                const uint64_t kb = dkt0 + GDN_DOFF((c & 1) * QK_STAGE);      // K as [s][k]: MN-major B
                const uint64_t pp = dv0 + GDN_DOFF((c & 1) * V_STAGE);        // P of chunk c
                const uint32_t ty = tmem + TM_Y + (c & 1) * 64;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    mma_f16kind_ss(ty, dub + GDN_DOFF(kk * 32), pp + GDN_DOFF(kk * 32), id_yq, 1);
                    mma_f16kind_ss(tmem + TM_S, dud + GDN_DOFF(kk * 32), kb + GDN_DOFF(kk * 2048), id_s, 1);
                }
                mma_commit(&bar[B_SFULL]);
                mma_commit(&bar[B_EMPTY0 + (c & 1)]);
            };
#undef GDN_DOFF
            // Issue whatever is ready, chain products first. Per operation the chunks go in
            // order; the preconditions also keep every TMEM accumulator single-writer:
            //   G(c): stage loaded, G(c-1) read by the solve group (TMEM G is single), and
            //         W(c-1) issued (so the converters, which start on G(c), never run two
            //         phases ahead of the CONV barrier polled for W)
            //   W(c): T diag(beta gamma) and the converted tiles of c
            //   U(c): T diag(beta) of c, and S(c-1) issued (it waited for U~(c-1) to be read)
            //   X(c): U(c) issued, -W^T(c) and the fp16 state copy of c written
            //   S(c): X(c) issued, U~ operands, P and the rescaled state of c ready
            // A barrier phase seen complete is remembered until its operation is issued, so
            // each pass re-tests only what is still pending.
            int nG = 0, nW = 0, nU = 0, nX = 0, nS = 0;
            uint32_t seen = 0;                // bit per (operation, barrier) seen complete
            enum : uint32_t { kS_UD = 1, kS_P = 2, kS_SACC = 4, kX_WB = 8, kX_SB = 16, kU_TB = 32,
                              kW_TBG = 64, kW_CONV = 128, kG_FULL = 256, kG_EMPTY = 512 };
            auto ready = [&](uint32_t bit, int b, int parity) {
                if (seen & bit) return true;
                if (done(b, parity)) { seen |= bit; return true; }
                return false;
            };
            long long idle_since = clock64();
            while (nS < n_chunks) {
                bool progressed = false;
                if (nS < nX && ready(kS_UD, B_UD, nS) && ready(kS_P, B_P, nS) && ready(kS_SACC, B_SACC, nS)) {
                    tc_fence_after();
                    do_S(nS++);
                    seen &= ~(kS_UD | kS_P | kS_SACC);
                    progressed = true;
                } else if (nX < nU && ready(kX_WB, B_WB, nX) && ready(kX_SB, B_SB, nX)) {
                    tc_fence_after();
                    do_X(nX++);
                    seen &= ~(kX_WB | kX_SB);
                    progressed = true;
                } else if (nW < nG && ready(kW_TBG, B_TBG, nW) && ready(kW_CONV, B_CONV, nW)) {
                    tc_fence_after();
                    do_W(nW++);
                    seen &= ~(kW_TBG | kW_CONV);
                    progressed = true;
                } else if (nU < nW && nU <= nS && ready(kU_TB, B_TB, nU)) {
                    tc_fence_after();
                    do_U(nU++);
                    seen &= ~kU_TB;
                    progressed = true;
                } else if (nG < n_chunks && nG <= nW && ready(kG_FULL, B_FULL0 + (nG & 1), nG >> 1) &&
                           (nG == 0 || ready(kG_EMPTY, B_GEMPTY, nG - 1))) {
                    tc_fence_after();
                    do_G(nG++);
                    seen &= ~(kG_FULL | kG_EMPTY);
                    progressed = true;
                }
                if (progressed) {
                    idle_since = clock64();
                    continue;
                }
                if (*abort_flag) break;
                if (clock64() - idle_since > kWaitLimit) {
                    *abort_flag = 1;
                    raise_error(kErrTimeout);
                    break;
                }
                __nanosleep(20);              // leave the issue slots to the warps doing the work
            }
            // drain the tensor pipe before TMEM is released
            mma_commit(&bar[B_DRAIN]);
            mbar_wait_drain(&bar[B_DRAIN], 0, kWaitLimit);
        }
    } else if (warp < 4) {
        // ================================================================ converters
        const int u = tid - 64;               // token row 0..63 of every tile
        for (int c = 0; c < n_chunks; ++c) {
            float g_lo, g_hi;
            chunk_log2_decay_scan(log_alpha, ci.bos + (int64_t)c * kC, H, ci.h, chunk_valid(c), lane, g_lo, g_hi);
            const float fq = fast_exp2(warp == 2 ? g_lo : g_hi) * scale;     // gamma_u * scale
            bool ok = true;
            if (u == 0) ok = mbar_wait_bounded(&bar[B_GFULL], c & 1, abort_flag, kWaitLimit);
            if (!named_bar_and(NB_CONV, 64, ok)) break;
            uint8_t *qk = smem + OFF_QK + (c & 1) * QK_STAGE;
            uint8_t *vv = smem + OFF_V + (c & 1) * V_STAGE;
            uint8_t *rows[6] = {qk + u * 128, qk + 16384 + u * 128, qk + 8192 + u * 128,
                                qk + 24576 + u * 128, vv + u * 128, vv + 8192 + u * 128};
            // A whole 128-byte row is rewritten, so the swizzle does not matter; the rotated
            // order keeps the eight threads of a row group on distinct banks. Three rows of
            // loads are issued before their first store.
#pragma unroll
            for (int grp = 0; grp < 6; grp += 3) {
                uint4 v[3][8];
#pragma unroll
                for (int w3 = 0; w3 < 3; ++w3)
#pragma unroll
                    for (int it = 0; it < 8; ++it) v[w3][it] = lds128(rows[grp + w3] + (((it + u) & 7) << 4));
#pragma unroll
                for (int w3 = 0; w3 < 3; ++w3) {
                    const int which = grp + w3;
                    const float f = (which == 2 || which == 3) ? fq : 1.f;
#pragma unroll
                    for (int it = 0; it < 8; ++it)
                        sts128(rows[which] + (((it + u) & 7) << 4), bf16x8_to_f16x8(v[w3][it], f));
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&bar[B_CONV]);
        }
    } else if (warp < 8) {
        // ================================================================ solve warpgroup
        const int r = tid - 128;              // TMEM lane / row
        const int t = r & 63;
        const uint32_t lane_base = (uint32_t)(warp & 3) * 32u << 16;
        float *g2s = reinterpret_cast<float *>(smem + OFF_GATES);
        float *gam = g2s + 64, *bet = g2s + 128, *bfac = g2s + 192;
        for (int c = 0; c < n_chunks; ++c) {
            const int64_t tok0 = ci.bos + (int64_t)c * kC;
            const int n_valid = chunk_valid(c);
            if (warp == 4) {
                float g_lo, g_hi;
                chunk_log2_decay_scan(log_alpha, tok0, H, ci.h, n_valid, lane, g_lo, g_hi);
                // Gamma_ts = 2^(g_t - g_s) = 2^(g_t - m) 2^(m - g_s) around the mid decay m
                const float mid = 0.5f * (__shfl_sync(0xffffffffu, g_lo, 0) + __shfl_sync(0xffffffffu, g_hi, 31));
                g2s[lane] = g_lo;
                g2s[lane + 32] = g_hi;
                gam[lane] = fast_exp2(g_lo);
                gam[lane + 32] = fast_exp2(g_hi);
                bet[lane] = lane < n_valid ? beta[(size_t)(tok0 + lane) * H + ci.h] : 0.f;
                bet[lane + 32] = lane + 32 < n_valid ? beta[(size_t)(tok0 + lane + 32) * H + ci.h] : 0.f;
                bfac[lane] = fast_exp2(mid - g_lo);
                bfac[lane + 32] = fast_exp2(mid - g_hi);
            }
            // (a) G rows: K K^T (lanes 0..63), Q K^T (lanes 64..127)
            bool ok = true;
            if (r == 0) ok = mbar_wait_bounded(&bar[B_GFULL], c & 1, abort_flag, kWaitLimit);
            if (!named_bar_and(NB_SOLVE, 128, ok)) break;
            tc_fence_after();
            uint32_t ga[32], gb[32];
            tmem_ld_x32(tmem + lane_base + TM_G, ga);
            tmem_ld_x32(tmem + lane_base + TM_G + 32, gb);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&bar[B_GEMPTY]);
            const float g2t = g2s[t];
            // one uniform choice per chunk: factored Gamma (both factors in the fp32 normal
            // range when the chunk's decay span is at most kSpanMax) or one exp2 per entry
            const float g2first = g2s[0], g2last = g2s[63];
            const bool factored = (g2first - g2last) <= kSpanMax;
            const float at = fast_exp2(g2t - 0.5f * (g2first + g2last));
            uint32_t pk[32];                  // P row (threads 64..127), fp16 pairs
            // the row's weight for column s: w_s = c * Gamma_ts, c = beta_t (L) or scale (P)
            const float cw = r < 64 ? bet[t] : scale;
            float wrow[64];
            if (factored) {
                const float cat = cw * at;
#pragma unroll
                for (int s4 = 0; s4 < 64; s4 += 4) {
                    const float4 b4 = ldsf4(bfac + s4);
                    wrow[s4] = cat * b4.x;
                    wrow[s4 + 1] = cat * b4.y;
                    wrow[s4 + 2] = cat * b4.z;
                    wrow[s4 + 3] = cat * b4.w;
                }
            } else {
#pragma unroll
                for (int s4 = 0; s4 < 64; s4 += 4) {
                    const float4 g4 = ldsf4(g2s + s4);
                    wrow[s4] = cw * fast_exp2(fminf(g2t - g4.x, 0.f));
                    wrow[s4 + 1] = cw * fast_exp2(fminf(g2t - g4.y, 0.f));
                    wrow[s4 + 2] = cw * fast_exp2(fminf(g2t - g4.z, 0.f));
                    wrow[s4 + 3] = cw * fast_exp2(fminf(g2t - g4.w, 0.f));
                }
            }
            if (r < 64) {
#pragma unroll
                for (int s4 = 0; s4 < 64; s4 += 4) {
                    float lv[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int s = s4 + e;
                        lv[e] = (s < t) ? wrow[s] * __uint_as_float(s < 32 ? ga[s] : gb[s - 32]) : 0.f;
                    }
                    stsf4(Ls + t * LS_LD + s4, make_float4(lv[0], lv[1], lv[2], lv[3]));
                }
            } else {
#pragma unroll
                for (int s2 = 0; s2 < 64; s2 += 2) {
                    const float p0 = (s2 <= t) ? wrow[s2] * __uint_as_float(s2 < 32 ? ga[s2] : gb[s2 - 32]) : 0.f;
                    const float p1 = (s2 + 1 <= t) ? wrow[s2 + 1] * __uint_as_float(s2 + 1 < 32 ? ga[s2 + 1] : gb[s2 - 31]) : 0.f;
                    pk[s2 >> 1] = pack_f16x2(p0, p1);
                }
            }
            named_bar_sync(NB_SOLVE, 128);
            // (b) T = (I + L)^-1
            // 16x16 diagonal blocks: one column per thread, right-looking substitution
            if (r < 64) {
                const int j = r, b0 = (j >> 4) << 4, jb = j & 15;
                float acc[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) acc[i] = (i == jb) ? 1.f : 0.f;
#pragma unroll
                for (int s = 0; s < 16; ++s) {
                    const float xs = acc[s];
#pragma unroll
                    for (int i = s + 1; i < 16; ++i) acc[i] = fmaf(-Ls[(b0 + i) * LS_LD + b0 + s], xs, acc[i]);
                }
                named_bar_sync(NB_SOLVE_LO, 64);   // every column thread has read its L block
#pragma unroll
                for (int i = 0; i < 16; ++i) Ls[(b0 + i) * LS_LD + j] = acc[i];
            }
            named_bar_sync(NB_SOLVE, 128);
            // Block merges on tf32 mma.sync tiles, one 8-column strip per warp, fp32 in
            // shared memory: M = L_ab T_b (strip), then X = -T_a M (strip) -> T's block (a, b).
            {
                const int w = warp - 4, g = lane >> 2, q = lane & 3;
                float *rt = Rt + w * 32 * 8;                 // this warp's [32][8] strip of M
                auto lda = [&](uint32_t (&a)[4], const float *base, int ld) {
                    a[0] = to_tf32(base[g * ld + q]);
                    a[1] = to_tf32(base[(g + 8) * ld + q]);
                    a[2] = to_tf32(base[g * ld + q + 4]);
                    a[3] = to_tf32(base[(g + 8) * ld + q + 4]);
                };
                auto ldb = [&](uint32_t (&b)[2], const float *base, int ld) {
                    b[0] = to_tf32(base[q * ld + g]);
                    b[1] = to_tf32(base[(q + 4) * ld + g]);
                };
                auto std_ = [&](float *base, int ld, const float (&d)[4], float sgn) {
                    base[g * ld + 2 * q] = sgn * d[0];
                    base[g * ld + 2 * q + 1] = sgn * d[1];
                    base[(g + 8) * ld + 2 * q] = sgn * d[2];
                    base[(g + 8) * ld + 2 * q + 1] = sgn * d[3];
                };
                // level 1: blocks (1,0) and (3,2), 16x16 each; warp w: pair w >> 1, strip w & 1
                {
                    const int pair = w >> 1, j = w & 1;
                    const int a0 = 16 + 32 * pair, b0 = 32 * pair;
                    float m[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int kk = 0; kk < 16; kk += 8) {
                        uint32_t a[4], b[2];
                        lda(a, Ls + a0 * LS_LD + b0 + kk, LS_LD);
                        ldb(b, Ls + (b0 + kk) * LS_LD + b0 + 8 * j, LS_LD);
                        mma_tf32_16x8x8(m, a, b);
                    }
                    std_(rt, 8, m, 1.f);
                    __syncwarp();
                    float x[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int kk = 0; kk < 16; kk += 8) {
                        uint32_t a[4], b[2];
                        lda(a, Ls + a0 * LS_LD + a0 + kk, LS_LD);
                        ldb(b, rt + kk * 8, 8);
                        mma_tf32_16x8x8(x, a, b);
                    }
                    // the sibling strip's warp may still read L_ab: store X after everyone
                    named_bar_sync(NB_SOLVE, 128);
                    std_(Ls + a0 * LS_LD + b0 + 8 * j, LS_LD, x, -1.f);
                }
                named_bar_sync(NB_SOLVE, 128);
                // level 2: rows 32..63 x cols 0..31; warp w owns strip w (cols 8w..8w+7)
                {
                    const int k_lo = w >= 2 ? 16 : 0;        // T_A is zero in rows 0..15 of cols 16..31
                    __syncwarp();
                    float m[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
                    for (int kk = 0; kk < 32; kk += 8) {
                        if (kk < k_lo) continue;
                        uint32_t b[2];
                        ldb(b, Ls + kk * LS_LD + 8 * w, LS_LD);
#pragma unroll
                        for (int mt = 0; mt < 2; ++mt) {
                            uint32_t a[4];
                            lda(a, Ls + (32 + 16 * mt) * LS_LD + kk, LS_LD);
                            mma_tf32_16x8x8(m[mt], a, b);
                        }
                    }
                    std_(rt, 8, m[0], 1.f);
                    std_(rt + 16 * 8, 8, m[1], 1.f);
                    __syncwarp();
                    float x[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
                    for (int kk = 0; kk < 32; kk += 8) {
                        uint32_t b[2];
                        ldb(b, rt + kk * 8, 8);
#pragma unroll
                        for (int mt = 0; mt < 2; ++mt) {
                            if (mt == 0 && kk >= 16) continue;   // T_B is zero above its diagonal blocks
                            uint32_t a[4];
                            lda(a, Ls + (32 + 16 * mt) * LS_LD + 32 + kk, LS_LD);
                            mma_tf32_16x8x8(x[mt], a, b);
                        }
                    }
                    named_bar_sync(NB_SOLVE, 128);      // every warp is done reading L_BA
                    std_(Ls + 32 * LS_LD + 8 * w, LS_LD, x[0], -1.f);
                    std_(Ls + 48 * LS_LD + 8 * w, LS_LD, x[1], -1.f);
                }
            }
            named_bar_sync(NB_SOLVE, 128);
            // (c) T diag(beta gamma), rows by threads 0..63. The row is computed into registers
            // first, then stored, so no load waits behind a store.
            float trow[64];
            {
#pragma unroll
                for (int s4 = 0; s4 < 64; s4 += 4) {
                    const float4 t4 = ldsf4(Ls + t * LS_LD + s4);
                    const float4 b4 = ldsf4(bet + s4);
                    const float4 c4 = r < 64 ? ldsf4(gam + s4) : make_float4(1.f, 1.f, 1.f, 1.f);
                    trow[s4] = t4.x * b4.x * c4.x;
                    trow[s4 + 1] = t4.y * b4.y * c4.y;
                    trow[s4 + 2] = t4.z * b4.z * c4.z;
                    trow[s4 + 3] = t4.w * b4.w * c4.w;
                }
            }
            if (r < 64) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) sts128(smem + OFF_TBG + sw128_off(t, ch), pack8_f16(trow + ch * 8));
            }
            fence_proxy_async_smem();
            mbar_arrive(&bar[B_TBG]);
            // (d) T diag(beta) (rows by threads 64..127) once the previous chunk's U^T product
            // is done (x_full(c-1))
            ok = true;
            if (c > 0 && r == 0) ok = mbar_wait_bounded(&bar[B_XFULL], (c - 1) & 1, abort_flag, kWaitLimit);
            if (!named_bar_and(NB_SOLVE, 128, ok)) break;
            if (r >= 64) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) sts128(smem + OFF_TB + sw128_off(t, ch), pack8_f16(trow + ch * 8));
            }
            fence_proxy_async_smem();
            mbar_arrive(&bar[B_TB]);
            // (f) -W^T from its accumulator into the MN-major operand [k][t]
            ok = true;
            if (r == 0) ok = mbar_wait_bounded(&bar[B_WFULL], c & 1, abort_flag, kWaitLimit);
            if (!named_bar_and(NB_SOLVE, 128, ok)) break;
            tc_fence_after();
            tmem_ld_x32(tmem + lane_base + TM_W, ga);
            tmem_ld_x32(tmem + lane_base + TM_W + 32, gb);
            tmem_wait_ld();
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                float v8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int s = ch * 8 + e;
                    v8[e] = -__uint_as_float(s < 32 ? ga[s] : gb[s - 32]);
                }
                sts128(smem + OFF_WB + sw128_off(r, ch), pack8_f16(v8));
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bar[B_WB]);
            // (e) P into the V stage of this chunk, free once U^T(c) is done (u_full(c));
            // S(c) reads it, and the stage is reloaded only after S(c) completes
            ok = true;
            if (r == 0) ok = mbar_wait_bounded(&bar[B_UFULL], c & 1, abort_flag, kWaitLimit);
            if (!named_bar_and(NB_SOLVE, 128, ok)) break;
            if (r >= 64) {
                uint8_t *pdst = smem + OFF_V + (c & 1) * V_STAGE;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch)
                    sts128(pdst + sw128_off(t, ch), make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]));
            }
            fence_proxy_async_smem();
            mbar_arrive(&bar[B_P]);
        }
    } else {
        // ================================================================ state warpgroup
        const int r = tid - 256;              // TMEM lane = value index v
        const uint32_t lane_base = (uint32_t)(warp & 3) * 32u << 16;
        float *decw = reinterpret_cast<float *>(smem + OFF_DEC) + (warp - 8) * 64;
        auto scan = [&](int c, float &g_lo, float &g_hi) {
            chunk_log2_decay_scan(log_alpha, ci.bos + (int64_t)c * kC, H, ci.h, chunk_valid(c), lane, g_lo, g_hi);
        };
        float g_lo = 0.f, g_hi = 0.f;
        if (n_chunks > 0) scan(0, g_lo, g_hi);
        // S0 -> TMEM (scaled by gamma_C of chunk 0) and its fp16 copy
        {
            const float gC = fast_exp2(__shfl_sync(0xffffffffu, g_hi, 31));
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
                    for (int cc = 0; cc < 4; ++cc) {
                        float v8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) v8[e] = __uint_as_float(sv[cc * 8 + e]);
                        sts128(sb_half + sw128_off(r, (q4 & 1) * 4 + cc), pack8_f16(v8));
                    }
#pragma unroll
                    for (int i = 0; i < 32; ++i) sv[i] = __float_as_uint(__uint_as_float(sv[i]) * gC);
                    tmem_st_x32(tmem + lane_base + TM_S + q4 * 32, sv);
                }
                tmem_wait_st();
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(&bar[B_SB]);
                mbar_arrive(&bar[B_SACC]);
            }
        }
        for (int c = 0; c < n_chunks; ++c) {
            const int64_t tok0 = ci.bos + (int64_t)c * kC;
            const int n_valid = chunk_valid(c);
            const bool last = (c + 1 == n_chunks);
            // exp(g_C - g_s) of this chunk into the warp's own slot (read back as broadcasts)
            const float g2C = __shfl_sync(0xffffffffu, g_hi, 31);
            __syncwarp();                     // the previous chunk's reads of decw are done
            decw[lane] = fast_exp2(g2C - g_lo);
            decw[lane + 32] = fast_exp2(g2C - g_hi);
            __syncwarp();
            // the next chunk's scan: its gamma_C rescales the carried state below
            float n_lo = 0.f, n_hi = 0.f;
            if (!last) scan(c + 1, n_lo, n_hi);
            const float gC_next = last ? 1.f : fast_exp2(__shfl_sync(0xffffffffu, n_hi, 31));
            // E2: U~^T -> fp16 operands (plain and decayed). The previous chunk's y copies
            // read the same buffers: every issuer waits for them before the barrier.
            bulk_wait_read();
            bool ok = true;
            if (r == 0) ok = mbar_wait_bounded(&bar[B_XFULL], c & 1, abort_flag, kWaitLimit);
            if (!named_bar_and(NB_STATE, 128, ok)) break;
            tc_fence_after();
            {
                uint32_t ua[32], ub[32];
                tmem_ld_x32(tmem + lane_base + TM_U, ua);
                tmem_ld_x32(tmem + lane_base + TM_U + 32, ub);
                tmem_wait_ld();
                float dd[64];
#pragma unroll
                for (int s4 = 0; s4 < 64; s4 += 4) {
                    const float4 d4 = ldsf4(decw + s4);
                    dd[s4] = d4.x;
                    dd[s4 + 1] = d4.y;
                    dd[s4 + 2] = d4.z;
                    dd[s4 + 3] = d4.w;
                }
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    float pl[8], dc[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int s = ch * 8 + e;
                        pl[e] = __uint_as_float(s < 32 ? ua[s] : ub[s - 32]);
                        dc[e] = pl[e] * dd[s];
                    }
                    sts128(smem + OFF_UB + sw128_off(r, ch), pack8_f16(pl));
                    sts128(smem + OFF_UD + sw128_off(r, ch), pack8_f16(dc));
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bar[B_UD]);
            // E3: the fp16 copy of S_{c+1} and the fp32 state rescaled by the next gamma_C
            // (both gate the next chunk), then y
            ok = true;
            if (r == 0) ok = mbar_wait_bounded(&bar[B_SFULL], c & 1, abort_flag, kWaitLimit);
            if (!named_bar_and(NB_STATE, 128, ok)) break;
            tc_fence_after();
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                // two 32-column loads in flight, then the fp16 copy (or S_T) and the rescale
                uint32_t sa[32], sb[32];
                tmem_ld_x32(tmem + lane_base + TM_S + h2 * 64, sa);
                tmem_ld_x32(tmem + lane_base + TM_S + h2 * 64 + 32, sb);
                tmem_wait_ld();
                if (last) {
                    if (S_T) {
                        float *dst = S_T + state_off + (size_t)r * kD + h2 * 64;
#pragma unroll
                        for (int i = 0; i < 64; i += 4) {
                            const uint32_t *sv = i < 32 ? sa + i : sb + (i - 32);
                            store4(dst + i, make_float4(__uint_as_float(sv[0]), __uint_as_float(sv[1]),
                                                        __uint_as_float(sv[2]), __uint_as_float(sv[3])));
                        }
                    }
                } else {
                    uint8_t *sb_half = smem + OFF_SB + h2 * 16384;
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) {
                        float v8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int i = cc * 8 + e;
                            v8[e] = __uint_as_float(i < 32 ? sa[i] : sb[i - 32]);
                        }
                        sts128(sb_half + sw128_off(r, cc), pack8_f16(v8));
                    }
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        sa[i] = __float_as_uint(__uint_as_float(sa[i]) * gC_next);
                        sb[i] = __float_as_uint(__uint_as_float(sb[i]) * gC_next);
                    }
                    tmem_st_x32(tmem + lane_base + TM_S + h2 * 64, sa);
                    tmem_st_x32(tmem + lane_base + TM_S + h2 * 64 + 32, sb);
                }
            }
            if (!last) {
                fence_proxy_async_smem();
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bar[B_SB]);
                mbar_arrive(&bar[B_SACC]);
            }
            {
                // y: Y^T column v of every token into the staging tile [t][v] (the U~ operand
                // buffers, idle until the next chunk's E2), then one bulk copy per token row
                uint32_t ya[32], yb[32];
                tmem_ld_x32(tmem + lane_base + TM_Y + (c & 1) * 64, ya);
                tmem_ld_x32(tmem + lane_base + TM_Y + (c & 1) * 64 + 32, yb);
                tmem_wait_ld();
                TY *ys = reinterpret_cast<TY *>(smem + OFF_YST);
#pragma unroll
                for (int tt = 0; tt < 64; ++tt)
                    ys[tt * kD + r] = from_f32<TY>(__uint_as_float(tt < 32 ? ya[tt] : yb[tt - 32]));
                fence_proxy_async_smem();
                named_bar_sync(NB_STATE, 128);
                const int tt = (warp - 8) * 16 + lane;
                if (lane < 16 && tt < n_valid) {
                    bulk_store_s2g(y + ((size_t)(tok0 + tt) * H + ci.h) * kD, ys + tt * kD, kD * sizeof(TY));
                    bulk_commit();
                }
            }
            g_lo = n_lo;
            g_hi = n_hi;
        }
        bulk_wait_all();                      // y copies complete before the CTA exits
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
