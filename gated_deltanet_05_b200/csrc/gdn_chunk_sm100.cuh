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
//   U~^T = U^T + S^T (-W^T)                M=128 (d_v), N=64, K=128      A in TMEM
//   Y^T  = S^T (diag(gamma) Q)^T + U~^T P^T    M=128, N=64, K=128 + 64   A in TMEM
//   S^T <- gamma_C S^T + (U~^T diag(exp(g_C - g))) K   M=128, N=128, K=64, A in TMEM
// The state S^T (value-major, the library's state layout) lives in TMEM in fp32 for the
// whole sequence. Every exponent is <= 0 (exponentials are taken base 2 on log2-scaled
// decays, with the SM's approximate exp2 instruction).
//
// Operand precision: G = [K; Q] K^T runs on the bf16 inputs as loaded. Every other
// product runs on fp16 operands (kind::f16, fp32 accumulate): the K, Q, V tiles are
// converted to fp16 (exact for |x| in [2^-14, 65504], which bf16 inputs of unit-norm
// keys/queries and O(1) values satisfy) and all derived operands (T diag(beta),
// T diag(beta gamma), P, -W^T, the S^T copy, U~^T) are rounded to fp16, whose 11-bit
// significand keeps the chunked form within the bf16-input accuracy bar where bf16
// (8-bit) operands do not. y is written in fp32 or bf16.
//
// One thread-block cluster of two CTAs owns one (sequence, head) chain; the two halves of
// the chunk algebra run on two SMs:
//   rank 0, "solver": everything that does not depend on the state -- G, the decay
//     factors, L and P, T = (I + L)^-1 (16x16 diagonal blocks by fp32 forward
//     substitution, then two levels of block merges on tf32 mma.sync tiles), the fp16
//     operands T diag(beta gamma), T diag(beta), P, and the fp16 K tile. Two solve
//     warpgroups take alternate chunks, so the solver runs ahead of the state chain.
//       warp 0 TMA (K, Q), warp 1 TMEM + G issuer, warps 2-3 convert K to fp16 and
//       publish it, warps 4-7 / 8-11 solve chunks c even / odd
//   rank 1, "chain": W, U, the state chain and the outputs.
//       warp 0 loads (Q and V by TMA, fp16 K), warp 1 TMEM + MMA issuer (the whole warp
//       runs the scheduler, one elected lane issues), warps 2-3 convert Q (scaled by gamma
//       and the attention scale) and V to fp16, warps 4-7 and
//       8-11 are two epilogue warpgroups that split every accumulator by columns: -W^T
//       into shared memory, U~^T and its decayed copy into TMEM (fp16), the fp16 copy of
//       the state into TMEM and the carry rescale by gamma_C, y (straight from TMEM to
//       global, coalesced across the value lanes) and S_T.
// Hand-off between the two CTAs, chosen by bandwidth: the 24 KB of solver operands per
// chunk go shared memory to shared memory (a bulk copy completing on the chain CTA's
// mbarrier, into one of three slots; no multicast); the 16 KB fp16 K tile goes through
// a small ring in global
// memory (L2-resident, one region per solver SM, indexed by %smid: at most one solver CTA
// runs on an SM, so concurrent launches sharing the workspace cannot collide), written by
// a bulk store and read back by a bulk load after a remote mbarrier signal.
// The chain's A operands (the fp16 state copy and the two U~^T copies) live in TMEM,
// which keeps the chunk-to-chunk critical path (U~ -> state update -> state copy ->
// next U~) off shared memory.
// All mbarrier waits are bounded (~1 s); on a timeout the kernel records it in the
// device error word, raises the abort flag of both CTAs, every role leaves its loop,
// in-flight TMA, bulk and MMA work is drained (again with bounded waits) and TMEM is
// released. Neither CTA exits while a copy into the other's shared memory is in flight.
#pragma once
#include <cuda.h>

#include "gdn_common.cuh"
#include "sm100_ptx.cuh"

namespace gdn {
namespace sm100 {

constexpr int kC = 64;       // chunk length
constexpr int kD = 128;      // d_k = d_v
constexpr int kThreads = 384;
constexpr int kStages = 3;   // K ring depth of the chain CTA
constexpr int kSvStages = 2; // K/Q TMA ring depth of the solver CTA
constexpr int kRing = 4;     // K/Q chunks in flight through global memory, per solver SM
constexpr int kRecv = 2;     // solver-operand slots in the chain CTA
constexpr int kQVStages = 2; // Q/V ring of the chain CTA
constexpr long long kWaitLimit = 2000000000LL;   // SM cycles (~1 s at 1.9 GHz)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kSpanMax = 240.f;       // log2 span of a chunk's decays for the factored Gamma
constexpr uint32_t TP_BYTES = 24576;    // one chunk's solver operands: [T diag(beta gamma) | T diag(beta) | P]
constexpr uint32_t K_BYTES = 16384;     // one chunk's fp16 K tile: [K d0..63 | K d64..127]
constexpr size_t kWsBytesPerSm = (size_t)kRing * K_BYTES;

// ---------------------------------------------------------------- solver CTA layout
namespace sv {
constexpr uint32_t OFF_QK = 0;          // kSvStages x 32 KB, bf16 as loaded, then fp16 in place
constexpr uint32_t QK_STAGE = 32768;
constexpr uint32_t OFF_SEND = OFF_QK + kSvStages * QK_STAGE; // per solve group: two chunks' operands
constexpr int LS_LD = 68;
constexpr uint32_t LS_BYTES = 64 * LS_LD * 4;                // fp32 [64][68]: L, then T in place
constexpr uint32_t OFF_LS = OFF_SEND + 4 * TP_BYTES;
constexpr uint32_t RT_BYTES = 4 * 32 * 8 * 4;                // merge temp: [32][8] fp32 per warp
constexpr uint32_t OFF_RT = OFF_LS + 2 * LS_BYTES;
constexpr uint32_t GATES_BYTES = 4 * 64 * 4;                 // {g2, gamma, beta, 2^(m - g2)}[64]
constexpr uint32_t OFF_GATES = OFF_RT + 2 * RT_BYTES;
constexpr uint32_t OFF_BAR = OFF_GATES + 2 * GATES_BYTES;
enum {
    B_FULL = 0, B_EMPTY = B_FULL + kSvStages, B_CREADY = B_EMPTY + kSvStages, B_GFULL = B_CREADY + kSvStages,
    // RECV_EMPTY: chain slot of chunk c free again, one barrier per c % (2 kRecv) so that
    // each has a single waiting solve group; LANDED: the send buffer of chunk c % 4 copied out
    B_GEMPTY = B_GFULL + 2, B_RECV_EMPTY = B_GEMPTY + 2, B_LANDED = B_RECV_EMPTY + 2 * kRecv,
    B_SCR_EMPTY = B_LANDED + 4, B_DRAIN = B_SCR_EMPTY + kRing, N_BAR
};
constexpr uint32_t OFF_MISC = OFF_BAR + N_BAR * 8;           // tmem base, abort flag, sequence, smid
constexpr uint32_t SMEM_USED = OFF_MISC + 16;
constexpr uint32_t TM_G = 0, TM_COLS = 128;                  // G double buffer
}  // namespace sv

// ---------------------------------------------------------------- chain CTA layout
namespace ch {
constexpr uint32_t OFF_K = 0;           // kStages x 16 KB fp16 K from the ring: [K d0..63 | K d64..]
constexpr uint32_t OFF_QV = OFF_K + kStages * K_BYTES;       // kQVStages x 32 KB: [Q d0..63 | Q d64.. | V d0..63 | V d64..]
constexpr uint32_t QV_STAGE = 32768;                         // bf16 as loaded, then fp16 (Q scaled by gamma and scale)
constexpr uint32_t OFF_RECV = OFF_QV + kQVStages * QV_STAGE; // kRecv slots of one chunk's solver operands
constexpr uint32_t OFF_WB = OFF_RECV + kRecv * TP_BYTES;     // fp16 -W^T [128 k][64 t], MN-major
constexpr uint32_t OFF_YST = OFF_WB + 16384;                 // y staging: [32 t][128 v] per epilogue warpgroup
constexpr uint32_t YST_HALF = 16384;
constexpr uint32_t OFF_DEC = OFF_YST + 2 * YST_HALF;         // exp(g_C - g)[64] per epilogue warp
constexpr uint32_t OFF_BAR = OFF_DEC + 8 * 64 * 4;
enum {
    B_K_FULL = 0, B_K_EMPTY = B_K_FULL + kStages, B_QV_FULL = B_K_EMPTY + kStages,
    B_QV_EMPTY = B_QV_FULL + kQVStages, B_CONV = B_QV_EMPTY + kQVStages, B_RECV = B_CONV + kQVStages,
    B_K_READY = B_RECV + kRecv, B_WFULL = B_K_READY + kRing, B_XFULL, B_SFULL, B_DRAIN, N_BAR
};
// named barriers: 1, 2 epilogue groups, 3 converters; the epilogue (256 threads, arrive)
// hands the two critical products to the issuer warp (32 threads, sync) through
constexpr int NB_S_TRIG = 4, NB_X_TRIG = 5, NB_TRIG_THREADS = 288;
constexpr uint32_t OFF_MISC = OFF_BAR + N_BAR * 8;           // tmem base, abort, sequence, operand copies sent[2][kRecv]
constexpr uint32_t SMEM_USED = OFF_MISC + 48;
// TMEM columns (128 lanes): fp32 state, Y^T double buffer, W^T, U~^T, and the fp16 A
// operands (two values per column): state copy, U~^T, U~^T diag(exp(g_C - g))
constexpr uint32_t TM_S = 0, TM_Y = 128, TM_W = 256, TM_U = 320, TM_SB = 384, TM_UB = 448, TM_UD = 480,
                   TM_COLS = 512;
}  // namespace ch

constexpr uint32_t SMEM_BYTES = (sv::SMEM_USED > ch::SMEM_USED ? sv::SMEM_USED : ch::SMEM_USED) + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
// At most one CTA of this kernel fits on an SM. The workspace (and the fixed array of the
// allocation-free entry point) gives each SM id one K-ring region, which is safe for
// overlapping launches only because no two solver CTAs can share an SM.
static_assert(2 * SMEM_BYTES > 232448, "one CTA per SM: the per-SM-id workspace regions rely on it");
static_assert(sv::OFF_SEND % 1024 == 0 && ch::OFF_QV % 1024 == 0 && ch::OFF_RECV % 1024 == 0 &&
                  ch::OFF_WB % 1024 == 0, "swizzle atoms");

// Inclusive scan of one chunk's log2-scaled decays, two tokens per lane: g_lo for tokens
// 0..31, g_hi for 32..63 (x0, x1 are lane's two log2 decays, zero past the sequence end).
// Every warp that calls it with the same values gets bit-identical results.
__device__ __forceinline__ void log2_decay_scan(float x0, float x1, int lane, float &g_lo, float &g_hi)
{
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

__device__ __forceinline__ void chunk_log2_decay_scan(const float *__restrict__ log_alpha, int64_t tok0,
                                                      int H, int h, int n_valid, int lane,
                                                      float &g_lo, float &g_hi)
{
    const float x0 = lane < n_valid ? log_alpha[(size_t)(tok0 + lane) * H + h] * kLog2e : 0.f;
    const float x1 = lane + 32 < n_valid ? log_alpha[(size_t)(tok0 + lane + 32) * H + h] * kLog2e : 0.f;
    log2_decay_scan(x0, x1, lane, g_lo, g_hi);
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

// Converts row u of n_tiles consecutive 8 KB tiles (64 rows of 128 bytes, bf16 as loaded)
// to fp16 in place, multiplying the values of the first n_scaled tiles by f; returns the
// running magnitude maximum of the converted fp16 values (f16x2_absmax). A whole row is
// rewritten, so the 128-byte swizzle does not matter; the rotated chunk order keeps the
// eight threads of a row group on distinct banks. Rolled two 16-byte chunks at a time:
// this code shares the instruction cache with the kernel's other roles.
__device__ __forceinline__ uint32_t convert_rows_bf16_f16(uint8_t *tiles, int n_tiles, int n_scaled, float f, int u,
                                                         uint32_t absmax)
{
#pragma unroll 1
    for (int i = 0; i < 8 * n_tiles; i += 2) {
        uint8_t *row = tiles + (i >> 3) * 8192 + u * 128;
        const float fi = (i >> 3) < n_scaled ? f : 1.f;
        const uint32_t o0 = (uint32_t)((((i & 7) + u) & 7) << 4), o1 = (uint32_t)((((i & 7) + 1 + u) & 7) << 4);
        const uint4 a = lds128(row + o0), b = lds128(row + o1);
        const uint4 ha = bf16x8_to_f16x8(a, fi), hb = bf16x8_to_f16x8(b, fi);
        absmax = f16x8_absmax(f16x8_absmax(absmax, ha), hb);
        sts128(row + o0, ha);
        sts128(row + o1, hb);
    }
    return absmax;
}

#define GDN_DOFF(bytes) ((uint64_t)((bytes) >> 4))

// ws: kWsBytesPerSm bytes per SM id below ws_slots (the K ring of the solver CTA on
// that SM). No other scratch.
template <typename TY>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
chunk_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_y,
                      const float *__restrict__ log_alpha,
                      const float *__restrict__ beta, const float *__restrict__ S0,
                      const int32_t *__restrict__ cu_seqlens, int n_seq, int H, float scale,
                      TY *__restrict__ y, float *__restrict__ S_T, uint8_t *__restrict__ ws, int ws_slots)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);

    const uint32_t crank = cluster_ctarank();       // 0 solver, 1 chain
    const bool is_solver = crank == 0;
    const uint32_t off_bar = is_solver ? sv::OFF_BAR : ch::OFF_BAR;
    const uint32_t off_misc = is_solver ? sv::OFF_MISC : ch::OFF_MISC;
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + off_bar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + off_misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + off_misc + 4);
    int *seq_slot = reinterpret_cast<int *>(smem + off_misc + 8);
    // the other CTA's abort flag: a timeout on either side stops both
    const uint32_t peer_abort = map_to_peer(sbase + (is_solver ? ch::OFF_MISC : sv::OFF_MISC) + 4, crank ^ 1u);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;

    // ---- which chain: sequences in order of decreasing length (ties by index), so the
    // longest chains start first; identity order beyond kThreads sequences
    const int chain = blockIdx.x >> 1;
    const int rank = chain / H;
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
        if (is_solver) {
            for (int b = 0; b < sv::N_BAR; ++b)
                mbar_init(&bar[b], (b == sv::B_GEMPTY || b == sv::B_GEMPTY + 1) ? 128 : 1);
            reinterpret_cast<uint32_t *>(smem + sv::OFF_MISC + 12)[0] = smid();
        } else {
            for (int b = 0; b < ch::N_BAR; ++b) {
                uint32_t count = 1;
                if (b >= ch::B_CONV && b < ch::B_CONV + kQVStages) count = 64;
                mbar_init(&bar[b], count);
            }
            for (int i = 0; i < 2 * kRecv; ++i) reinterpret_cast<int *>(smem + ch::OFF_MISC + 12)[i] = 0;
        }
        *abort_flag = 0;
        fence_mbarrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, is_solver ? sv::TM_COLS : ch::TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();                 // both CTAs' barriers exist before any remote use
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int head = chain % H;
    const int seq = *seq_slot;
    const int64_t bos = cu_seqlens[seq];
    const int64_t len = (int64_t)cu_seqlens[seq + 1] - bos;
    // the K ring of this cluster: the region of the solver CTA's SM
    const uint32_t solver_sm = is_solver ? reinterpret_cast<const uint32_t *>(smem + sv::OFF_MISC + 12)[0]
                                         : ld_cluster_u32(map_to_peer(sbase + sv::OFF_MISC + 12, 0));
    const bool ws_ok = ws != nullptr && solver_sm < (uint32_t)ws_slots;
    if (!ws_ok && tid == 0 && is_solver) raise_error(kErrCheck);
    uint8_t *ring = ws_ok ? ws + (size_t)solver_sm * kWsBytesPerSm : nullptr;
    const int n_chunks = ws_ok ? (int)((len + kC - 1) / kC) : 0;
    const size_t state_off = ((size_t)seq * H + head) * (size_t)kD * kD;
    auto chunk_valid = [&](int c) -> int {
        const int64_t rem = len - (int64_t)c * kC;
        return (int)(rem < kC ? rem : kC);
    };
    // Bounded waits. A non-blocking test goes first: a blocking try_wait on a phase that
    // has already completed still costs a few hundred cycles.
    auto wait = [&](int b, int parity) -> bool {
        return mbar_test(&bar[b], (uint32_t)parity & 1u) ||
               mbar_wait_or_abort(&bar[b], (uint32_t)parity & 1u, abort_flag, peer_abort, 0u, kWaitLimit);
    };
    auto wait_cl = [&](int b, int parity) -> bool {
        return mbar_test_cluster(&bar[b], (uint32_t)parity & 1u) ||
               mbar_wait_or_abort(&bar[b], (uint32_t)parity & 1u, abort_flag, peer_abort, 1u, kWaitLimit);
    };
    // the same, called by a whole warp: every lane gets the same answer
    auto wait_w = [&](int b, int parity) -> bool { return __all_sync(0xffffffffu, wait(b, parity)); };
    auto wait_cl_w = [&](int b, int parity) -> bool { return __all_sync(0xffffffffu, wait_cl(b, parity)); };

    if (is_solver) {
        using namespace sv;
        if (warp == 0) {
            // ============================================================ TMA producer (K, Q)
            // The whole warp runs the loop; one elected lane issues.
            if (n_chunks > 0) {
                const uint32_t lead = elect_one();
                if (lead) {
                    tma_prefetch_desc(&tm_q);
                    tma_prefetch_desc(&tm_k);
                }
                int issued[kSvStages] = {};
#pragma unroll 1
                for (int c = 0; c < n_chunks; ++c) {
                    const int st = c % kSvStages;
                    // the stage is free once its fp16 K tile has been copied out
                    if (c >= kSvStages && !wait_w(B_EMPTY + st, c / kSvStages - 1)) break;
                    const int tok = (int)(bos + (int64_t)c * kC);
                    uint8_t *qk = smem + OFF_QK + st * QK_STAGE;
                    mbar_arrive_expect_tx_lead(&bar[B_FULL + st], QK_STAGE, lead);
                    tma_load_3d_lead(qk + 0, &tm_k, &bar[B_FULL + st], 0, head, tok, lead);
                    tma_load_3d_lead(qk + 8192, &tm_q, &bar[B_FULL + st], 0, head, tok, lead);
                    tma_load_3d_lead(qk + 16384, &tm_k, &bar[B_FULL + st], 64, head, tok, lead);
                    tma_load_3d_lead(qk + 24576, &tm_q, &bar[B_FULL + st], 64, head, tok, lead);
                    issued[st] = c + 1;
                }
                for (int st = 0; st < kSvStages; ++st)
                    if (issued[st] > 0) mbar_wait_drain(&bar[B_FULL + st], ((issued[st] - 1) / kSvStages) & 1, kWaitLimit);
            }
        } else if (warp == 1) {
            // ============================================================ G = [K; Q] K^T issuer
            if (n_chunks > 0) {
                const uint32_t lead = elect_one();
                const uint32_t id_g = idesc_f32acc(kFmtBF16, 128, 64, 0, 0);
                const uint64_t dqk0 = sdesc_sw128(sbase + OFF_QK, 16, 1024);
#pragma unroll 1
                for (int c = 0; c < n_chunks; ++c) {
                    const int st = c % kSvStages;
                    if (!wait_w(B_FULL + st, c / kSvStages)) break;
                    if (c >= 2 && !wait_w(B_GEMPTY + (c & 1), (c >> 1) - 1)) break;
                    tc_fence_after();
                    const uint64_t base = dqk0 + GDN_DOFF(st * QK_STAGE);
#pragma unroll 1
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint64_t d = base + GDN_DOFF((kk >> 2) * 16384 + (kk & 3) * 32);
                        mma_ss_lead(tmem + TM_G + (c & 1) * 64, d, d, id_g, kk > 0, lead);
                    }
                    mma_commit_lead(&bar[B_GFULL + (c & 1)], lead);
                    mma_commit_lead(&bar[B_CREADY + st], lead);      // the bf16 tiles may now be converted
                }
                mma_commit_lead(&bar[B_DRAIN], lead);
                mbar_wait_drain(&bar[B_DRAIN], 0, kWaitLimit);
            }
        } else if (warp < 4) {
            // ============================================================ K converters
            // Convert K in place once G no longer reads it, then one thread stores the tile
            // to the ring in global memory and, once the store of the previous chunk has
            // completed, signals that chunk to the chain CTA (one chunk of slack keeps the
            // converters from waiting on L2).
            const int u = tid - 64;               // token row 0..63 of both K tiles
            const uint32_t k_ready0 = map_to_peer(sbase + ch::OFF_BAR + ch::B_K_READY * 8, 1);
            const uint32_t lead = elect_one();    // in warp 2: the lane that issues the ring stores
            int stored = 0;
            uint32_t ovf = 0;                     // magnitude maximum of the converted K values
            for (int c = 0; c < n_chunks; ++c) {
                const int st = c % kSvStages;
                bool ok = true;
                if (u == 0) ok = wait(B_CREADY + st, c / kSvStages);
                if (!named_bar_and(5, 64, ok)) break;
                uint8_t *qk = smem + OFF_QK + st * QK_STAGE;
                // the K tiles are [K d0..63 | Q d0..63 | K d64..127 | Q d64..]: tiles 0 and 2
                ovf = convert_rows_bf16_f16(qk, 1, 0, 1.f, u, ovf);
                ovf = convert_rows_bf16_f16(qk + 16384, 1, 0, 1.f, u, ovf);
                fence_proxy_async_smem();
                // the ring slot is free once the chain CTA has loaded chunk c - kRing
                ok = true;
                if (u == 0 && c >= kRing) ok = wait_cl(B_SCR_EMPTY + c % kRing, c / kRing - 1);
                if (!named_bar_and(5, 64, ok)) break;
                if (warp == 2) {                  // converged; lane `lead` issues
                    uint8_t *dst = ring + (size_t)(c % kRing) * K_BYTES;
                    bulk_store_s2g_lead(dst, qk, 8192, lead);
                    bulk_store_s2g_lead(dst + 8192, qk + 16384, 8192, lead);
                    bulk_commit();
                    bulk_wait_read();             // the stage has been read: TMA may refill it
                    mbar_arrive_lead(&bar[B_EMPTY + st], lead);
                    if (c > 0) {
                        bulk_wait_all_but_1();    // chunk c - 1 is in global memory
                        fence_proxy_async_global();
                        mbar_arrive_remote_lead(k_ready0 + (uint32_t)((c - 1) % kRing) * 8u, lead);
                    }
                }
                stored = c + 1;
            }
            if (f16x2_overflowed(ovf)) raise_error(kErrCheck);
            if (warp == 2 && stored > 0) {
                bulk_wait_all();
                fence_proxy_async_global();
                mbar_arrive_remote_lead(k_ready0 + (uint32_t)((stored - 1) % kRing) * 8u, lead);
            }
        } else {
            // ============================================================ solve warpgroups
            const int j = (warp - 4) >> 2;            // chunks c with c % 2 == j
            const int r = tid - 128 - 128 * j;        // TMEM lane / row
            const int t = r & 63;
            const uint32_t lane_base = (uint32_t)(warp & 3) * 32u << 16;
            const int nb = 1 + 2 * j, nb_lo = 2 + 2 * j;
            float *Ls = reinterpret_cast<float *>(smem + OFF_LS + j * LS_BYTES);
            float *Rt = reinterpret_cast<float *>(smem + OFF_RT + j * RT_BYTES);
            float *g2s = reinterpret_cast<float *>(smem + OFF_GATES + j * GATES_BYTES);
            float *gam = g2s + 64, *bet = g2s + 128, *bfac = g2s + 192;
            const bool gate_warp = (warp & 3) == 0;
            // log alpha and beta of this group's next chunk, loaded one chunk ahead
            float la0 = 0.f, la1 = 0.f, be0 = 0.f, be1 = 0.f;
            auto load_gates = [&](int c) {
                const int64_t tok0 = bos + (int64_t)c * kC;
                const int nv = chunk_valid(c);
                la0 = lane < nv ? log_alpha[(size_t)(tok0 + lane) * H + head] : 0.f;
                la1 = lane + 32 < nv ? log_alpha[(size_t)(tok0 + lane + 32) * H + head] : 0.f;
                be0 = lane < nv ? beta[(size_t)(tok0 + lane) * H + head] : 0.f;
                be1 = lane + 32 < nv ? beta[(size_t)(tok0 + lane + 32) * H + head] : 0.f;
            };
            if (gate_warp && j < n_chunks) load_gates(j);
            int n_sent[kRecv] = {};
            uint32_t ovf = 0;                         // magnitude maximum of the fp16 operands sent
            for (int c = j; c < n_chunks; c += 2) {
                if (gate_warp) {
                    float g_lo, g_hi;
                    log2_decay_scan(la0 * kLog2e, la1 * kLog2e, lane, g_lo, g_hi);
                    // Gamma_ts = 2^(g_t - g_s) = 2^(g_t - m) 2^(m - g_s) around the mid decay m
                    const float mid = 0.5f * (__shfl_sync(0xffffffffu, g_lo, 0) + __shfl_sync(0xffffffffu, g_hi, 31));
                    g2s[lane] = g_lo;
                    g2s[lane + 32] = g_hi;
                    gam[lane] = fast_exp2(g_lo);
                    gam[lane + 32] = fast_exp2(g_hi);
                    bet[lane] = be0;
                    bet[lane + 32] = be1;
                    bfac[lane] = fast_exp2(mid - g_lo);
                    bfac[lane + 32] = fast_exp2(mid - g_hi);
                    if (c + 2 < n_chunks) load_gates(c + 2);
                }
                // (a) the group's two send buffers alternate: this one is free once its previous
                // copy (chunk c - 4) has landed; G rows: K K^T (lanes 0..63), Q K^T (lanes 64..127)
                uint8_t *send = smem + OFF_SEND + (c & 3) * TP_BYTES;
                bool ok = true;
                if (r == 0) {
                    if (c >= 4) ok = wait_cl(B_LANDED + (c & 3), (c >> 2) - 1);
                    if (ok) ok = wait(B_GFULL + j, c >> 1);
                }
                if (!named_bar_and(nb, 128, ok)) break;
                tc_fence_after();
                // The raw row goes to shared memory first (K K^T rows into L's place, Q K^T rows
                // into the send buffer's T part, free until step (c)); the weighting below then
                // runs as a short rolled loop over the row. Each thread only reads back its own
                // row. Q K^T rows are [64][64] fp32 with 16-byte chunks XOR-swizzled by row.
                float *prow_raw = reinterpret_cast<float *>(send) + t * 64;
                auto praw = [&](int s4) -> float * { return prow_raw + (((s4 >> 2) ^ (t & 7)) << 2); };
                {
                    uint32_t ga[32], gb[32];
                    tmem_ld_x32(tmem + lane_base + TM_G + j * 64, ga);
                    tmem_ld_x32(tmem + lane_base + TM_G + j * 64 + 32, gb);
                    tmem_wait_ld();
                    tc_fence_before();
                    mbar_arrive(&bar[B_GEMPTY + j]);
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        const float4 lo = make_float4(__uint_as_float(ga[i]), __uint_as_float(ga[i + 1]),
                                                      __uint_as_float(ga[i + 2]), __uint_as_float(ga[i + 3]));
                        const float4 hi = make_float4(__uint_as_float(gb[i]), __uint_as_float(gb[i + 1]),
                                                      __uint_as_float(gb[i + 2]), __uint_as_float(gb[i + 3]));
                        stsf4(r < 64 ? Ls + t * LS_LD + i : praw(i), lo);
                        stsf4(r < 64 ? Ls + t * LS_LD + 32 + i : praw(32 + i), hi);
                    }
                }
                const float g2t = g2s[t];
                // one uniform choice per chunk: factored Gamma (both factors in the fp32 normal
                // range when the chunk's decay span is at most kSpanMax) or one exp2 per entry
                const float g2first = g2s[0], g2last = g2s[63];
                const bool factored = (g2first - g2last) <= kSpanMax;
                const float at = fast_exp2(g2t - 0.5f * (g2first + g2last));
                // the row's weight for column s: w_s = c * Gamma_ts, c = beta_t (L) or scale (P)
                const float cw = r < 64 ? bet[t] : scale;
                const float cat = cw * at;
                // L rows (strictly lower, fp32, in place) and P rows (lower incl. the diagonal,
                // fp16 into the send buffer's P part), eight columns per step
#pragma unroll 1
                for (int s8 = 0; s8 < 64; s8 += 8) {
                    float v[8], w[8];
                    const float4 x0 = ldsf4(r < 64 ? Ls + t * LS_LD + s8 : praw(s8));
                    const float4 x1 = ldsf4(r < 64 ? Ls + t * LS_LD + s8 + 4 : praw(s8 + 4));
                    v[0] = x0.x; v[1] = x0.y; v[2] = x0.z; v[3] = x0.w;
                    v[4] = x1.x; v[5] = x1.y; v[6] = x1.z; v[7] = x1.w;
                    if (factored) {
                        const float4 b0 = ldsf4(bfac + s8), b1 = ldsf4(bfac + s8 + 4);
                        w[0] = cat * b0.x; w[1] = cat * b0.y; w[2] = cat * b0.z; w[3] = cat * b0.w;
                        w[4] = cat * b1.x; w[5] = cat * b1.y; w[6] = cat * b1.z; w[7] = cat * b1.w;
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) w[e] = cw * fast_exp2(fminf(g2t - g2s[s8 + e], 0.f));
                    }
                    const int lim = r < 64 ? t : t + 1;       // columns s < lim are kept
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[e] = (s8 + e < lim) ? w[e] * v[e] : 0.f;
                    if (r < 64) {
                        stsf4(Ls + t * LS_LD + s8, make_float4(v[0], v[1], v[2], v[3]));
                        stsf4(Ls + t * LS_LD + s8 + 4, make_float4(v[4], v[5], v[6], v[7]));
                    } else {
                        const uint4 h = pack8_f16(v);
                        ovf = f16x8_absmax(ovf, h);
                        sts128(send + 16384 + sw128_off(t, s8 >> 3), h);
                    }
                }
                named_bar_sync(nb, 128);
                // (b) T = (I + L)^-1
                // 16x16 diagonal blocks: one column per thread, right-looking substitution
                if (r < 64) {
                    const int jc = r, b0 = (jc >> 4) << 4, jb = jc & 15;
                    float acc[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) acc[i] = (i == jb) ? 1.f : 0.f;
#pragma unroll
                    for (int s = 0; s < 16; ++s) {
                        const float xs = acc[s];
#pragma unroll
                        for (int i = s + 1; i < 16; ++i) acc[i] = fmaf(-Ls[(b0 + i) * LS_LD + b0 + s], xs, acc[i]);
                    }
                    named_bar_sync(nb_lo, 64);       // every column thread has read its L block
#pragma unroll
                    for (int i = 0; i < 16; ++i) Ls[(b0 + i) * LS_LD + jc] = acc[i];
                }
                named_bar_sync(nb, 128);
                // Block merges on tf32 mma.sync tiles, one 8-column strip per warp, fp32 in
                // shared memory: M = L_ab T_b (strip), then X = -T_a M (strip) -> T's block (a, b).
                {
                    const int w = warp & 3, g = lane >> 2, q = lane & 3;
                    float *rt = Rt + w * 32 * 8;             // this warp's [32][8] strip of M
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
                        const int pair = w >> 1, jj = w & 1;
                        const int a0 = 16 + 32 * pair, b0 = 32 * pair;
                        float m[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int kk = 0; kk < 16; kk += 8) {
                            uint32_t a[4], b[2];
                            lda(a, Ls + a0 * LS_LD + b0 + kk, LS_LD);
                            ldb(b, Ls + (b0 + kk) * LS_LD + b0 + 8 * jj, LS_LD);
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
                        named_bar_sync(nb, 128);
                        std_(Ls + a0 * LS_LD + b0 + 8 * jj, LS_LD, x, -1.f);
                    }
                    named_bar_sync(nb, 128);
                    // level 2: rows 32..63 x cols 0..31; warp w owns strip w (cols 8w..8w+7)
                    {
                        const int k_lo = w >= 2 ? 16 : 0;    // T_A is zero in rows 0..15 of cols 16..31
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
                        named_bar_sync(nb, 128);              // every warp is done reading L_BA
                        std_(Ls + 32 * LS_LD + 8 * w, LS_LD, x[0], -1.f);
                        std_(Ls + 48 * LS_LD + 8 * w, LS_LD, x[1], -1.f);
                    }
                }
                named_bar_sync(nb, 128);
                // (c) row t of T diag(beta gamma) (threads 0..63) or T diag(beta) (64..127), fp16,
                // into the send buffer (over the raw Q K^T rows, all read by now)
#pragma unroll 1
                for (int s8 = 0; s8 < 64; s8 += 8) {
                    const float4 t0 = ldsf4(Ls + t * LS_LD + s8), t1 = ldsf4(Ls + t * LS_LD + s8 + 4);
                    const float4 b0 = ldsf4(bet + s8), b1 = ldsf4(bet + s8 + 4);
                    const float4 c0 = r < 64 ? ldsf4(gam + s8) : make_float4(1.f, 1.f, 1.f, 1.f);
                    const float4 c1 = r < 64 ? ldsf4(gam + s8 + 4) : make_float4(1.f, 1.f, 1.f, 1.f);
                    const float v[8] = {t0.x * b0.x * c0.x, t0.y * b0.y * c0.y, t0.z * b0.z * c0.z, t0.w * b0.w * c0.w,
                                        t1.x * b1.x * c1.x, t1.y * b1.y * c1.y, t1.z * b1.z * c1.z, t1.w * b1.w * c1.w};
                    const uint4 h = pack8_f16(v);
                    ovf = f16x8_absmax(ovf, h);
                    sts128(send + (r < 64 ? 0 : 8192) + sw128_off(t, s8 >> 3), h);
                }
                fence_proxy_async_smem();
                // then one copy into the chain CTA's slot c % kRecv, once it has finished the
                // slot's previous chunk (c - kRecv)
                ok = true;
                if (c >= kRecv && r == 0) ok = wait_cl(B_RECV_EMPTY + (c - kRecv) % (2 * kRecv), (c - kRecv) / (2 * kRecv));
                if (!named_bar_and(nb, 128, ok)) break;
                const int slot = c % kRecv;
                if (r == 0) {
                    const uint32_t rbar = map_to_peer(sbase + ch::OFF_BAR + (ch::B_RECV + slot) * 8, 1);
                    const uint32_t rdst = map_to_peer(sbase + ch::OFF_RECV + slot * TP_BYTES, 1);
                    mbar_arrive_expect_tx_remote_relaxed(rbar, TP_BYTES);
                    bulk_copy_s2peer(rdst, send, TP_BYTES, rbar);
                }
                ++n_sent[slot];
            }
            if (f16x2_overflowed(ovf)) raise_error(kErrCheck);
            // the chain CTA drains this group's copies before either CTA exits
            if (r == 0)
                for (int sl = 0; sl < kRecv; ++sl)
                    st_cluster_u32(map_to_peer(sbase + ch::OFF_MISC + 12 + 4 * (kRecv * j + sl), 1), (uint32_t)n_sent[sl]);
        }
    } else {
        using namespace ch;
        if (warp == 0) {
            // ============================================================ loads: Q, V by TMA, fp16 K from the ring
            // The whole warp runs the loop; one elected lane issues.
            if (n_chunks > 0) {
                const uint32_t lead = elect_one();
                if (lead) {
                    tma_prefetch_desc(&tm_q);
                    tma_prefetch_desc(&tm_v);
                }
                int issued_qv[kQVStages] = {}, issued_k[kStages] = {};
#pragma unroll 1
                for (int c = 0; c < n_chunks; ++c) {
                    const int sq = c % kQVStages, sk = c % kStages;
                    // Q and V do not depend on the solver: they go first
                    if (c >= kQVStages && !wait_w(B_QV_EMPTY + sq, c / kQVStages - 1)) break;
                    const int tok = (int)(bos + (int64_t)c * kC);
                    uint8_t *qv = smem + OFF_QV + sq * QV_STAGE;
                    mbar_arrive_expect_tx_lead(&bar[B_QV_FULL + sq], QV_STAGE, lead);
                    tma_load_3d_lead(qv, &tm_q, &bar[B_QV_FULL + sq], 0, head, tok, lead);
                    tma_load_3d_lead(qv + 8192, &tm_q, &bar[B_QV_FULL + sq], 64, head, tok, lead);
                    tma_load_3d_lead(qv + 16384, &tm_v, &bar[B_QV_FULL + sq], 0, head, tok, lead);
                    tma_load_3d_lead(qv + 24576, &tm_v, &bar[B_QV_FULL + sq], 64, head, tok, lead);
                    issued_qv[sq] = c + 1;
                    if (c >= kStages && !wait_w(B_K_EMPTY + sk, c / kStages - 1)) break;
                    if (!wait_cl_w(B_K_READY + c % kRing, c / kRing)) break;
                    fence_proxy_async_global();
                    mbar_arrive_expect_tx_lead(&bar[B_K_FULL + sk], K_BYTES, lead);
                    bulk_load_g2s_lead(smem + OFF_K + sk * K_BYTES, ring + (size_t)(c % kRing) * K_BYTES, K_BYTES,
                                       &bar[B_K_FULL + sk], lead);
                    issued_k[sk] = c + 1;
                }
                for (int i = 0; i < kQVStages; ++i)
                    if (issued_qv[i] > 0) mbar_wait_drain(&bar[B_QV_FULL + i], ((issued_qv[i] - 1) / kQVStages) & 1, kWaitLimit);
                for (int i = 0; i < kStages; ++i)
                    if (issued_k[i] > 0) mbar_wait_drain(&bar[B_K_FULL + i], ((issued_k[i] - 1) / kStages) & 1, kWaitLimit);
            }
        } else if (warp == 1) {
            // ============================================================ MMA issuer
            // The whole warp runs the issuer (operands stay warp-uniform); one elected lane
            // issues every product, in the steady-state order
            //   X(c), W(c+1), S(c), U(c+1), X(c+1), ...
            // each after a blocking wait for its inputs (the solver runs ahead, so W(c+1)'s
            // inputs are normally there before X(c) completes, and W(c+1) runs on the tensor
            // pipe while the epilogue turns U~(c) into S(c)'s operands). The order also keeps
            // every TMEM accumulator single-writer:
            //   W(c+1): K and solver operands of c+1 arrived; -W^T(c) read out (before X(c))
            //   S(c):   U~ operands of c in TMEM, the state rescaled (S trigger)
            //   U(c+1): Q and V of c+1 converted; U~(c) read out (before S(c))
            //   X(c+1): -W^T(c+1) in shared memory, the state copy of c+1 in TMEM (X trigger)
            if (n_chunks > 0) {
                const uint32_t lead = elect_one();
                const uint32_t id_wu = idesc_f32acc(kFmtF16, 128, 64, 1, 0);
                const uint32_t id_xw = idesc_f32acc(kFmtF16, 128, 64, 0, 1);
                const uint32_t id_yq = idesc_f32acc(kFmtF16, 128, 64, 0, 0);
                const uint32_t id_s = idesc_f32acc(kFmtF16, 128, 128, 0, 1);
                // Base descriptors, computed once; a k-step adds a constant to the start
                // address field (addresses < 256 KB keep it inside its 14 bits).
                const uint64_t dkt0 = sdesc_sw128(sbase + OFF_K, 8192, 1024);           // K^T / K, MN-major
                const uint64_t dq0 = sdesc_sw128(sbase + OFF_QV, 16, 1024);             // Q rows, K-major
                const uint64_t dvt0 = sdesc_sw128(sbase + OFF_QV + 16384, 8192, 1024);  // V^T, MN-major
                const uint64_t dop0 = sdesc_sw128(sbase + OFF_RECV, 16, 1024);          // solver operands, K-major
                const uint64_t dwb = sdesc_sw128(sbase + OFF_WB, 8192, 1024);           // -W^T [k][t], MN-major
                // Signals to the solver CTA. They publish no data of this thread (the copies'
                // completion is what they report), so they are relaxed: a release would wait
                // for the thread's outstanding work.
                const uint32_t scr_empty0 = map_to_peer(sbase + sv::OFF_BAR + sv::B_SCR_EMPTY * 8, 0);
                const uint32_t landed0 = map_to_peer(sbase + sv::OFF_BAR + sv::B_LANDED * 8, 0);
                auto issue_W = [&](int c) -> bool {
                    if (!wait_w(B_K_FULL + c % kStages, c / kStages)) return false;
                    mbar_arrive_remote_relaxed_lead(scr_empty0 + (uint32_t)(c % kRing) * 8u, lead);   // ring slot reusable
                    if (!wait_cl_w(B_RECV + c % kRecv, c / kRecv)) return false;
                    mbar_arrive_remote_relaxed_lead(landed0 + (uint32_t)(c & 3) * 8u, lead);          // send buffer reusable
                    tc_fence_after();
                    const uint64_t kt = dkt0 + GDN_DOFF((c % kStages) * K_BYTES);
                    const uint64_t tbg = dop0 + GDN_DOFF((c % kRecv) * TP_BYTES);
#pragma unroll 1
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ss_lead(tmem + TM_W, kt + GDN_DOFF(kk * 2048), tbg + GDN_DOFF(kk * 32), id_wu, kk > 0, lead);
                    mma_commit_lead(&bar[B_WFULL], lead);
                    return true;
                };
                auto issue_U = [&](int c) -> bool {
                    if (!wait_w(B_CONV + c % kQVStages, c / kQVStages)) return false;
                    tc_fence_after();
                    const uint64_t vt = dvt0 + GDN_DOFF((c % kQVStages) * QV_STAGE);
                    const uint64_t tb = dop0 + GDN_DOFF((c % kRecv) * TP_BYTES + 8192);
#pragma unroll 1
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ss_lead(tmem + TM_U, vt + GDN_DOFF(kk * 2048), tb + GDN_DOFF(kk * 32), id_wu, kk > 0, lead);
                    return true;
                };
                // X(c) and S(c) start when the epilogue has stored their operands: a named
                // barrier (the epilogue arrives without waiting) wakes this warp faster than an
                // mbarrier wait. The epilogue always makes one last arrival on each trigger when
                // it leaves early, so these never wait for good; an abort is checked after each.
                auto trigger = [&](int nb_id) -> bool {
                    named_bar_sync(nb_id, NB_TRIG_THREADS);
                    return !__any_sync(0xffffffffu, *abort_flag != 0);
                };
                auto issue_X = [&](int c) -> bool {
                    if (!trigger(NB_X_TRIG)) return false;
                    tc_fence_after();
                    const uint64_t q0 = dq0 + GDN_DOFF((c % kQVStages) * QV_STAGE);
                    const uint32_t ty = tmem + TM_Y + (c & 1) * 64;
#pragma unroll 1
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t a = tmem + TM_SB + kk * 8;
                        // U~^T += S^T (-W^T): B = -W^T stored [k][t], MN-major
                        mma_ts_lead(tmem + TM_U, a, dwb + GDN_DOFF(kk * 2048), id_xw, 1, lead);
                        // Y^T = S^T (gamma scale Q)^T: B = Q rows (K-major), d 64..127 at +8 KB
                        mma_ts_lead(ty, a, q0 + GDN_DOFF((kk >> 2) * 8192 + (kk & 3) * 32), id_yq, kk > 0, lead);
                    }
                    mma_commit_lead(&bar[B_XFULL], lead);
                    mma_commit_lead(&bar[B_QV_EMPTY + c % kQVStages], lead);   // U(c) read V before, X(c) read Q
                    return true;
                };
                auto issue_S = [&](int c) -> bool {
                    if (!trigger(NB_S_TRIG)) return false;
                    tc_fence_after();
                    const uint64_t kb = dkt0 + GDN_DOFF((c % kStages) * K_BYTES);     // K as [s][k]: MN-major B
                    const uint64_t pp = dop0 + GDN_DOFF((c % kRecv) * TP_BYTES + 16384);
                    const uint32_t ty = tmem + TM_Y + (c & 1) * 64;
#pragma unroll 1
                    for (int kk = 0; kk < 4; ++kk) {
                        mma_ts_lead(ty, tmem + TM_UB + kk * 8, pp + GDN_DOFF(kk * 32), id_yq, 1, lead);
                        mma_ts_lead(tmem + TM_S, tmem + TM_UD + kk * 8, kb + GDN_DOFF(kk * 2048), id_s, 1, lead);
                    }
                    mma_commit_lead(&bar[B_SFULL], lead);
                    mma_commit_lead(&bar[B_K_EMPTY + c % kStages], lead);
                    return true;
                };
                // c = -1 issues W(0) and U(0); every step appears once in the code
#pragma unroll 1
                for (int c = -1; c < n_chunks; ++c) {
                    const bool more = c + 1 < n_chunks;
                    if (c >= 0 && !issue_X(c)) break;
                    if (more && !issue_W(c + 1)) break;
                    if (c >= 0 && !issue_S(c)) break;
                    if (more && !issue_U(c + 1)) break;
                }
                mma_commit_lead(&bar[B_DRAIN], lead);
                mbar_wait_drain(&bar[B_DRAIN], 0, kWaitLimit);
            }
        } else if (warp < 4) {
            // ============================================================ Q and V converters
            // Q is scaled by gamma_t (the chunk's cumulative decay at its row) and the
            // attention scale; the decays are loaded one chunk ahead.
            const int u = tid - 64;               // token row 0..63 of every tile
            float la0 = 0.f, la1 = 0.f;
            auto load_la = [&](int c) {
                const int64_t tok0 = bos + (int64_t)c * kC;
                const int nv = chunk_valid(c);
                la0 = lane < nv ? log_alpha[(size_t)(tok0 + lane) * H + head] : 0.f;
                la1 = lane + 32 < nv ? log_alpha[(size_t)(tok0 + lane + 32) * H + head] : 0.f;
            };
            if (n_chunks > 0) load_la(0);
            uint32_t ovf = 0;                     // magnitude maximum of the converted (scaled) Q, V values
            for (int c = 0; c < n_chunks; ++c) {
                const int st = c % kQVStages;
                float g_lo, g_hi;
                log2_decay_scan(la0 * kLog2e, la1 * kLog2e, lane, g_lo, g_hi);
                if (c + 1 < n_chunks) load_la(c + 1);
                const float fq = fast_exp2(warp == 2 ? g_lo : g_hi) * scale;     // gamma_u * scale
                bool ok = true;
                if (u == 0) ok = wait(B_QV_FULL + st, c / kQVStages);
                if (!named_bar_and(3, 64, ok)) break;
                uint8_t *qv = smem + OFF_QV + st * QV_STAGE;
                // [Q d0..63 | Q d64.. | V d0..63 | V d64..]: Q scaled by gamma_u * scale
                ovf = convert_rows_bf16_f16(qv, 4, 2, fq, u, ovf);
                fence_proxy_async_smem();
                mbar_arrive(&bar[B_CONV + st]);
            }
            if (f16x2_overflowed(ovf)) raise_error(kErrCheck);
        } else {
            // ============================================================ epilogue warpgroups
            const int hh = (warp - 4) >> 2;           // column half of every accumulator
            const int r = tid - 128 - 128 * hh;       // TMEM lane: value index v (row k of -W^T)
            const uint32_t lane_base = (uint32_t)(warp & 3) * 32u << 16;
            const int nb = 1 + hh;
            float *decw = reinterpret_cast<float *>(smem + OFF_DEC) + (warp - 4) * 64;
            // log alpha of the chunk after the current one, loaded one chunk ahead
            float la0 = 0.f, la1 = 0.f;
            auto load_la = [&](int c) {
                const int64_t tok0 = bos + (int64_t)c * kC;
                const int nv = chunk_valid(c);
                la0 = lane < nv ? log_alpha[(size_t)(tok0 + lane) * H + head] : 0.f;
                la1 = lane + 32 < nv ? log_alpha[(size_t)(tok0 + lane + 32) * H + head] : 0.f;
            };
            auto group_wait = [&](int b, int parity) -> bool {
                bool ok = true;
                if (r == 0) ok = wait(b, parity);
                return named_bar_and(nb, 128, ok);
            };
            // magnitude maxima of the values converted to fp16 operands here: -W^T and U~^T
            // (packed fp16, f16x2_absmax) and the state copy (fp32, NaN-propagating)
            uint32_t h16max = 0;
            float fmax16 = 0.f;
            // -W^T of chunk c: this half's 32 columns t of W^T into rows k = r of the operand
            // (off the recursion's critical path: rolled, eight columns at a time)
            auto do_wb = [&](int c) -> bool {
                if (!group_wait(B_WFULL, c)) return false;
                tc_fence_after();
#pragma unroll 1
                for (int c4 = 0; c4 < 4; ++c4) {
                    uint32_t wv[8];
                    tmem_ld_x8(tmem + lane_base + TM_W + 32 * hh + 8 * c4, wv);
                    tmem_wait_ld();
                    float v8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) v8[e] = -__uint_as_float(wv[e]);
                    const uint4 h = pack8_f16(v8);
                    h16max = f16x8_absmax(h16max, h);
                    sts128(smem + OFF_WB + sw128_off(r, 4 * hh + c4), h);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                return true;
            };
            float g_lo = 0.f, g_hi = 0.f;
            if (n_chunks > 0) {
                load_la(0);
                log2_decay_scan(la0 * kLog2e, la1 * kLog2e, lane, g_lo, g_hi);
                if (n_chunks > 1) load_la(1);
            }
            // S0 -> TMEM (scaled by gamma_C of chunk 0) and its fp16 copy, columns k in [64 hh, 64 hh + 64)
            {
                const float gC = fast_exp2(__shfl_sync(0xffffffffu, g_hi, 31));
                const float *src = S0 ? S0 + state_off + (size_t)r * kD + 64 * hh : nullptr;
                if (n_chunks == 0) {
                    if (S_T) {
                        float *dst = S_T + state_off + (size_t)r * kD + 64 * hh;
                        for (int i = 0; i < 64; i += 4)
                            store4(dst + i, src ? load4(src + i) : make_float4(0.f, 0.f, 0.f, 0.f));
                    }
                } else {
#pragma unroll
                    for (int q2 = 0; q2 < 2; ++q2) {
                        uint32_t sv[32], sp[16];
#pragma unroll
                        for (int i = 0; i < 32; i += 4) {
                            const float4 f = src ? load4(src + q2 * 32 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
                            sv[i] = __float_as_uint(f.x);
                            sv[i + 1] = __float_as_uint(f.y);
                            sv[i + 2] = __float_as_uint(f.z);
                            sv[i + 3] = __float_as_uint(f.w);
                        }
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            fmax16 = max_abs_nan(fmax16, __uint_as_float(sv[2 * i]));
                            fmax16 = max_abs_nan(fmax16, __uint_as_float(sv[2 * i + 1]));
                            sp[i] = pack_f16x2(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1]));
                        }
                        tmem_st_x16(tmem + lane_base + TM_SB + 32 * hh + 16 * q2, sp);
#pragma unroll
                        for (int i = 0; i < 32; ++i) sv[i] = __float_as_uint(__uint_as_float(sv[i]) * gC);
                        tmem_st_x32(tmem + lane_base + TM_S + 64 * hh + 32 * q2, sv);
                    }
                    tmem_wait_st();
                    tc_fence_before();
                }
            }
            // triggers given to the issuer (each is taken n_chunks times in a complete run)
            int n_strig = 0, n_xtrig = 0;
            bool alive = n_chunks > 0 && do_wb(0);
            if (alive) {                          // X(0): state copy of S0 and -W^T(0) in place
                named_bar_arrive(NB_X_TRIG, NB_TRIG_THREADS);
                ++n_xtrig;
            }
            for (int c = 0; alive && c < n_chunks; ++c) {
                const int64_t tok0 = bos + (int64_t)c * kC;
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
                if (!last) {
                    log2_decay_scan(la0 * kLog2e, la1 * kLog2e, lane, n_lo, n_hi);
                    if (c + 2 < n_chunks) load_la(c + 2);
                }
                const float gC_next = last ? 1.f : fast_exp2(__shfl_sync(0xffffffffu, n_hi, 31));
                // E2: U~^T -> fp16 A operands in TMEM (plain and decayed), 32 columns s per half
                if (!group_wait(B_XFULL, c)) break;
                tc_fence_after();
                {
                    uint32_t ua[32], pu[16], pd[16];
                    tmem_ld_x32(tmem + lane_base + TM_U + 32 * hh, ua);
                    tmem_wait_ld();
#pragma unroll
                    for (int i4 = 0; i4 < 8; ++i4) {
                        const float4 d4 = ldsf4(decw + 32 * hh + 4 * i4);
                        const float u0 = __uint_as_float(ua[4 * i4]), u1 = __uint_as_float(ua[4 * i4 + 1]);
                        const float u2 = __uint_as_float(ua[4 * i4 + 2]), u3 = __uint_as_float(ua[4 * i4 + 3]);
                        pu[2 * i4] = pack_f16x2(u0, u1);
                        pu[2 * i4 + 1] = pack_f16x2(u2, u3);
                        pd[2 * i4] = pack_f16x2(u0 * d4.x, u1 * d4.y);
                        pd[2 * i4 + 1] = pack_f16x2(u2 * d4.z, u3 * d4.w);
                    }
                    tmem_st_x16(tmem + lane_base + TM_UB + 16 * hh, pu);
                    tmem_st_x16(tmem + lane_base + TM_UD + 16 * hh, pd);
                    tmem_wait_st();
                    tc_fence_before();
                    named_bar_arrive(NB_S_TRIG, NB_TRIG_THREADS);   // S(c)
                    ++n_strig;
                    // range check of U~ (the decayed copy is no larger), after the trigger
#pragma unroll
                    for (int i = 0; i < 16; ++i) h16max = f16x2_absmax(h16max, pu[i]);
                }
                // -W^T of the next chunk while S(c) runs
                if (!last && !do_wb(c + 1)) break;
                // E3: the fp16 state copy of S_{c+1} and the fp32 state rescaled by the next
                // gamma_C (both gate the next chunk), or S_T after the last chunk
                if (!group_wait(B_SFULL, c)) break;
                tc_fence_after();
                {
                    uint32_t sa[32], sb[32];
                    tmem_ld_x32(tmem + lane_base + TM_S + 64 * hh, sa);
                    tmem_ld_x32(tmem + lane_base + TM_S + 64 * hh + 32, sb);
                    tmem_wait_ld();
                    if (last) {
                        if (hh == 0 && r == 0)
                            mbar_arrive_remote_relaxed(
                                map_to_peer(sbase + sv::OFF_BAR + (sv::B_RECV_EMPTY + c % (2 * kRecv)) * 8, 0));
                        if (S_T) {
                            float *dst = S_T + state_off + (size_t)r * kD + 64 * hh;
#pragma unroll
                            for (int i = 0; i < 64; i += 4) {
                                const uint32_t *sv = i < 32 ? sa + i : sb + (i - 32);
                                store4(dst + i, make_float4(__uint_as_float(sv[0]), __uint_as_float(sv[1]),
                                                            __uint_as_float(sv[2]), __uint_as_float(sv[3])));
                            }
                        }
                    } else {
                        // the state copy first (it gates X(c+1)), then the rescale (it gates S(c+1))
                        uint32_t pa[16], pb[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            pa[i] = pack_f16x2(__uint_as_float(sa[2 * i]), __uint_as_float(sa[2 * i + 1]));
                            pb[i] = pack_f16x2(__uint_as_float(sb[2 * i]), __uint_as_float(sb[2 * i + 1]));
                        }
                        tmem_st_x16(tmem + lane_base + TM_SB + 32 * hh, pa);
                        tmem_st_x16(tmem + lane_base + TM_SB + 32 * hh + 16, pb);
                        // S(c) has completed, so has every read of this chunk's operand slot: the
                        // solver may refill it (the signal publishes no data of this thread)
                        if (hh == 0 && r == 0)
                            mbar_arrive_remote_relaxed(
                                map_to_peer(sbase + sv::OFF_BAR + (sv::B_RECV_EMPTY + c % (2 * kRecv)) * 8, 0));
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            sa[i] = __float_as_uint(__uint_as_float(sa[i]) * gC_next);
                            sb[i] = __float_as_uint(__uint_as_float(sb[i]) * gC_next);
                        }
                        tmem_st_x32(tmem + lane_base + TM_S + 64 * hh, sa);
                        tmem_st_x32(tmem + lane_base + TM_S + 64 * hh + 32, sb);
                        tmem_wait_st();
                        tc_fence_before();
                        named_bar_arrive(NB_X_TRIG, NB_TRIG_THREADS);   // X(c+1)
                        ++n_xtrig;
                        // range check of the state copy, after the trigger
#pragma unroll
                        for (int i = 0; i < 16; ++i) h16max = f16x2_absmax(f16x2_absmax(h16max, pa[i]), pb[i]);
                    }
                }
                // y: tokens [32 hh, 32 hh + 32) of Y^T (lane v of each warp). A full chunk goes
                // through the group's staging tile [t][v] and one TMA store; the partial last
                // chunk of a sequence is written row by row with plain stores (a box store
                // would run into the next sequence's rows).
                {
                    // eight tokens at a time (off the critical path: rolled). A full chunk: the
                    // staging tile, once the previous chunk's store has read it (it had a whole
                    // chunk to do so), then one TMA store; a partial one: row by row.
                    const bool full = n_valid == kC;
                    if (full) {
                        if (r == 0) bulk_wait_read();
                        named_bar_sync(nb, 128);
                    }
                    const int nv = full ? 32 : n_valid - 32 * hh;
                    TY *ys = reinterpret_cast<TY *>(smem + OFF_YST + hh * YST_HALF);
                    TY *yp = y + ((size_t)(tok0 + 32 * hh) * H + head) * kD + r;
                    const size_t ystride = (size_t)H * kD;
#pragma unroll 1
                    for (int j8 = 0; j8 < 32; j8 += 8) {
                        uint32_t ya[8];
                        tmem_ld_x8(tmem + lane_base + TM_Y + (c & 1) * 64 + 32 * hh + j8, ya);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const TY v = from_f32<TY>(__uint_as_float(ya[e]));
                            if (full)
                                ys[(j8 + e) * kD + r] = v;
                            else if (j8 + e < nv)
                                yp[(size_t)(j8 + e) * ystride] = v;
                        }
                    }
                    if (full) {
                        fence_proxy_async_smem();
                        named_bar_sync(nb, 128);
                        if (r == 0) {
                            tma_store_3d(&tm_y, ys, 0, head, (int)(tok0 + 32 * hh));
                            bulk_commit();
                        }
                    }
                }
                g_lo = n_lo;
                g_hi = n_hi;
            }
            // leaving early (abort): one last arrival on each trigger the issuer may still be
            // waiting for
            if (n_strig < n_chunks) named_bar_arrive(NB_S_TRIG, NB_TRIG_THREADS);
            if (n_xtrig < n_chunks) named_bar_arrive(NB_X_TRIG, NB_TRIG_THREADS);
            if (!(fmax16 < kF16Limit) || f16x2_overflowed(h16max)) raise_error(kErrCheck);
            if (r == 0) bulk_wait_all();          // y stores complete before the CTA exits
        }
    }

    // ---- teardown: every role has left its loop and drained its own async work. The
    // chain CTA then waits for every operand copy that was sent to it to land, and only
    // after that may either CTA exit (a CTA's shared memory must outlive copies into or
    // out of it).
    tc_fence_before();
    __syncwarp();
    __syncthreads();
    cluster_sync_all();                   // copies-sent counts are visible
    if (!is_solver && tid == 0) {
        const int *sent = reinterpret_cast<const int *>(smem + ch::OFF_MISC + 12);
        for (int sl = 0; sl < kRecv; ++sl) {
            const int n = sent[sl] + sent[kRecv + sl];
            if (n <= 0) continue;
            const long long t0 = clock64();
            while (!mbar_try_wait_cluster(&bar[ch::B_RECV + sl], (uint32_t)(n - 1) & 1u))
                if (clock64() - t0 > kWaitLimit) {
                    raise_error(kErrTimeout);
                    break;
                }
        }
    }
    __syncwarp();
    cluster_sync_all();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, is_solver ? sv::TM_COLS : ch::TM_COLS);
    }
}

#undef GDN_DOFF

}  // namespace sm100
}  // namespace gdn
