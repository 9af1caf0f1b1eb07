// gdn_backward_chunk.cuh -- gradients of the gated delta rule through its chunked form,
// on CUDA cores in fp32.
//
// The reverse of the chunkwise forward (the four-line update of the joezjh.github.io notes
// page "Qwen3.8-Flash-Next", section "Gated DeltaNet 核心机制", rewritten chunk by chunk,
// exact up to rounding). Inside a chunk of C tokens with start state S (d_k x d_v, the
// pages' orientation), g = in-chunk cumulative log decay, gamma = exp(g),
// Gamma_ts = exp(g_t - g_s) (s <= t), D_s = exp(g_C - g_s):
//     A = K K^T,  L = strict_tril(diag(beta) (A o Gamma)),  T = (I + L)^-1
//     U = T diag(beta) V,  W = T diag(beta gamma) K,  U~ = U - W S
//     Y = diag(gamma) Q S + P U~  (P = tril(Q K^T o Gamma)),   S' = gamma_C S + (diag(D) K)^T U~
// Given dY and dS' = dL/dS', the chain rule gives
//     dU~ = P^T dY + diag(D) K dS',    dS = gamma_C dS' + (diag(gamma) Q)^T dY - W^T dU~
// and, with Z = diag(beta) V - diag(beta gamma) K S (so that T Z = U~),
//     dP = dY U~^T,  dT = dU~ Z^T,  dW = -dU~ S^T,  dK~ = U~ dS'^T,  dV = diag(beta) T^T dU~
//     dQ = diag(gamma) dY S^T + (dP o Gamma) K
//     dK = (dP o Gamma)^T Q + diag(beta gamma) T^T dW + (dA + dA^T) K + diag(D) dK~
//     dL = strict_tril(-T^T dT T^T),  dA = diag(beta) (dL o Gamma)
//     dbeta = rowsum(V o T^T dU~) + gamma o rowsum(K o T^T dW) + rowsum(dL o A o Gamma)
// and the decays gamma, Gamma, D fold into d g, then into d log alpha by a reverse
// cumulative sum inside the chunk. (The same algebra is restated in fp64 and pinned to the
// oracle's token-by-token adjoint in the tests.)
//
// Five launches:
//   chunk_bwd_prep_kernel   per (chain, chunk), all at once: T, A o Gamma, P and W of the
//                           chunk, kept in the workspace (all that does not depend on the state)
//   chunk_bwd_fwd_kernel    per (chain, d_v slice), chunks in order: the start state of every
//                           chunk (the forward's state chain)
//   chunk_bwd_state_kernel  per (chain, d_v slice), chunks in reverse: dS at every chunk end,
//                           and dS0
//   chunk_bwd_vpart_kernel  per (chain, chunk, d_v slice), all at once: dV, and the slice's
//                           sums over v that the rest needs (dP, dT, dW, dK~, dY S^T, ...), each
//                           slice into its own block (no atomics: the result is deterministic)
//   chunk_bwd_kpart_kernel  per (chain, chunk), all at once: dQ, dK, dbeta, dlog_alpha
// Every matrix product runs from shared memory with a register tile per thread (rows and
// columns interleaved across threads; odd row strides keep the lanes of a warp on distinct
// banks).
#pragma once
#include "gdn_common.cuh"

namespace gdn {
namespace bwdc {

constexpr int kC = 64;               // chunk length
constexpr int kDVT = 64;             // value columns per CTA in the sliced steps
constexpr int kThreads = 256;        // prep and kpart
constexpr int kThreadsWide = 512;    // fwd, state and vpart

__host__ __device__ inline int slice_cols(int DV) { return DV < kDVT ? DV : kDVT; }
// floats of the per-chunk sums block of one value slice: dP, dT [C][C]; dW, dK~, dY S^T
// [C][DK]; the row sums of V o T^T dU~ [C]; <dS', S> [1]
__host__ __device__ inline size_t part_floats(int DK) { return (size_t)kC * (2 * kC + 3 * DK + 1) + 1; }
// floats of the per-chunk cache: T, A o Gamma, P [C][C] and W [C][DK]
__host__ __device__ inline size_t cache_floats(int DK) { return (size_t)kC * (3 * kC + DK); }
constexpr int kCacheT = 0, kCacheAG = kC * kC, kCacheP = 2 * kC * kC, kCacheW = 3 * kC * kC;

// In-chunk decays of chunk [c0, c0 + n): g (cumulative log alpha, padded rows add 0),
// gamma = exp(g), beta (0 on padded rows), D = exp(g_C - g). Warp 0 only.
__device__ __forceinline__ void chunk_decays(const float *__restrict__ log_alpha, const float *__restrict__ beta,
                                             int64_t c0, int n, int H, int h, float *g, float *gam, float *bet,
                                             float *Dd)
{
    const int lane = threadIdx.x;
    float carry = 0.f;
    for (int base = 0; base < kC; base += 32) {
        const int t = base + lane;
        float x = t < n ? log_alpha[(size_t)(c0 + t) * H + h] : 0.f;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y_ = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y_;
        }
        x += carry;
        carry = __shfl_sync(0xffffffffu, x, 31);
        g[t] = x;
        gam[t] = expf(x);
        bet[t] = t < n ? beta[(size_t)(c0 + t) * H + h] : 0.f;
    }
    __syncwarp();
    const float gC = g[kC - 1];
    for (int t = lane; t < kC; t += 32) Dd[t] = expf(gC - g[t]);
}

// Rows of a chunk into shared memory [kC][ld] (zero past n), optionally scaled.
template <typename T>
__device__ __forceinline__ void load_rows(float *dst, int ld, const T *__restrict__ src, int64_t c0, int n, int H,
                                          int h, int D, int col0, int ncol, float f)
{
    for (int i = threadIdx.x; i < kC * ncol; i += blockDim.x) {
        const int t = i / ncol, a = i % ncol;
        dst[t * ld + a] = t < n ? f * to_f32(src[((size_t)(c0 + t) * H + h) * D + col0 + a]) : 0.f;
    }
}

// A row-major block of the cache into shared memory with a padded stride.
__device__ __forceinline__ void load_block(float *dst, int ld, const float *__restrict__ src, int rows, int cols)
{
    for (int i = threadIdx.x; i < rows * cols; i += blockDim.x) dst[(i / cols) * ld + i % cols] = src[i];
}

// acc[i][j] += sum_k a(m_i, k) b(k, n_j) over k < K, for one thread's tile: rows
// m_i = tm + i ntm, columns n_j = tn + j ntn.
template <int TM, int TN, class FA, class FB>
__device__ __forceinline__ void mm_acc(float (&acc)[TM][TN], int tm, int tn, int ntm, int ntn, int K, FA a, FB b)
{
#pragma unroll 4
    for (int kk = 0; kk < K; ++kk) {
        float av[TM], bv[TN];
#pragma unroll
        for (int i = 0; i < TM; ++i) av[i] = a(tm + i * ntm, kk);
#pragma unroll
        for (int j = 0; j < TN; ++j) bv[j] = b(kk, tn + j * ntn);
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
            for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
}

template <int TM, int TN>
__device__ __forceinline__ void zero(float (&acc)[TM][TN])
{
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;
}

// Sum over the `width` consecutive lanes that share a tile row (width a power of two <= 32;
// every lane of the warp takes part).
__device__ __forceinline__ float row_group_sum(float x, int width)
{
    for (int off = width >> 1; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

// Chunk geometry of (chain, chunk c): first token, valid rows; false past the sequence end.
__device__ __forceinline__ bool chunk_of(const int32_t *__restrict__ cu_seqlens, int seq, int c, int64_t &c0, int &n)
{
    const int64_t bos = cu_seqlens[seq], len = (int64_t)cu_seqlens[seq + 1] - bos;
    if ((int64_t)c * kC >= len) return false;
    c0 = bos + (int64_t)c * kC;
    n = (int)(len - (int64_t)c * kC < kC ? len - (int64_t)c * kC : kC);
    return true;
}

// --------------------------------------------------------------------------- prep
struct PrepSmem {
    int KQ, Ls, Ts, g, gam, bet, Dd, total;
};
__host__ __device__ inline PrepSmem prep_layout(int DK)
{
    PrepSmem L;
    int o = 0;
    const int kp = DK + 1, cp = kC + 1;
    L.KQ = o; o += 2 * kC * kp;
    L.Ls = o; o += kC * cp;
    L.Ts = o; o += kC * cp;
    L.g = o; o += kC;
    L.gam = o; o += kC;
    L.bet = o; o += kC;
    L.Dd = o; o += kC;
    L.total = o;
    return L;
}

// One CTA (kThreads) per (chain, chunk): [K; Q] K^T, then A o Gamma, P and L; T = (I + L)^-1
// row by row (four lanes per entry); W = T diag(beta gamma) K. All into the chunk's cache.
template <typename T>
__global__ void __launch_bounds__(kThreads)
chunk_bwd_prep_kernel(const T *__restrict__ q, const T *__restrict__ k, const float *__restrict__ log_alpha,
                      const float *__restrict__ beta, const int32_t *__restrict__ cu_seqlens, int H, int DK,
                      float scale, int max_chunks, float *__restrict__ cache)
{
    extern __shared__ float sm[];
    const PrepSmem Y = prep_layout(DK);
    float *KQ = sm + Y.KQ, *Ls = sm + Y.Ls, *Ts = sm + Y.Ts;
    float *g = sm + Y.g, *gam = sm + Y.gam, *bet = sm + Y.bet, *Dd = sm + Y.Dd;
    const int kp = DK + 1, cp = kC + 1;
    const int c = blockIdx.y, chain = blockIdx.x;
    const int seq = chain / H, h = chain % H;
    const int tid = threadIdx.x;
    int64_t c0;
    int n;
    if (!chunk_of(cu_seqlens, seq, c, c0, n)) return;
    float *cb = cache + ((size_t)chain * max_chunks + c) * cache_floats(DK);
    load_rows(KQ, kp, k, c0, n, H, h, DK, 0, DK, 1.f);
    load_rows(KQ + kC * kp, kp, q, c0, n, H, h, DK, 0, DK, scale);
    if (tid < 32) chunk_decays(log_alpha, beta, c0, n, H, h, g, gam, bet, Dd);
    for (int i = tid; i < kC * kC; i += blockDim.x) Ts[(i / kC) * cp + i % kC] = (i / kC == i % kC) ? 1.f : 0.f;
    __syncthreads();
    {
        constexpr int TM = 8, TN = 4;
        const int ntm = 2 * kC / TM, ntn = kC / TN;
        for (int gi = tid; gi < ntm * ntn; gi += blockDim.x) {
            const int tm = gi / ntn, tn = gi % ntn;
            float acc[TM][TN];
            zero(acc);
            mm_acc(acc, tm, tn, ntm, ntn, DK, [&](int m, int a) { return KQ[m * kp + a]; },
                   [&](int a, int s) { return KQ[s * kp + a]; });
#pragma unroll
            for (int i = 0; i < TM; ++i) {
                const int m = tm + i * ntm, t = m & (kC - 1);
#pragma unroll
                for (int j = 0; j < TN; ++j) {
                    const int s = tn + j * ntn;
                    const float x = s <= t ? acc[i][j] * expf(g[t] - g[s]) : 0.f;
                    if (m < kC) {
                        cb[kCacheAG + t * kC + s] = x;
                        Ls[t * cp + s] = s < t ? bet[t] * x : 0.f;
                    } else {
                        cb[kCacheP + t * kC + s] = x;
                    }
                }
            }
        }
    }
    __syncthreads();
    // T[t][j] = -sum_{j <= s < t} L[t][s] T[s][j] for j < t, one row after the other
    {
        const int j = tid >> 2, part = tid & 3;
        for (int t = 1; t < kC; ++t) {
            float x = 0.f;
            if (j < t)
                for (int s = j + part; s < t; s += 4) x = fmaf(Ls[t * cp + s], Ts[s * cp + j], x);
            x += __shfl_xor_sync(0xffffffffu, x, 1);
            x += __shfl_xor_sync(0xffffffffu, x, 2);
            if (part == 0 && j < t) Ts[t * cp + j] = -x;
            __syncthreads();
        }
    }
    for (int i = tid; i < kC * kC; i += blockDim.x) cb[kCacheT + i] = Ts[(i / kC) * cp + i % kC];
    for (int i = tid; i < kC * DK; i += blockDim.x) {
        const int s = i / DK;
        KQ[s * kp + i % DK] *= bet[s] * gam[s];
    }
    __syncthreads();
    {
        constexpr int TM = 8, TN = 4;
        const int ntm = kC / TM, ntn = DK / TN;
        for (int gi = tid; gi < ntm * ntn; gi += blockDim.x) {
            const int tm = gi / ntn, tn = gi % ntn;
            float acc[TM][TN];
            zero(acc);
            mm_acc(acc, tm, tn, ntm, ntn, kC, [&](int t, int s) { return Ts[t * cp + s]; },
                   [&](int s, int a) { return KQ[s * kp + a]; });
#pragma unroll
            for (int i = 0; i < TM; ++i)
#pragma unroll
                for (int j = 0; j < TN; ++j) cb[kCacheW + (tm + i * ntm) * DK + tn + j * ntn] = acc[i][j];
        }
    }
}

// --------------------------------------------------------------------------- fwd
struct FwdSmem {
    int Kd, Ws, Ts, Vb, Us, Ss, g, gam, bet, Dd, total;
};
__host__ __device__ inline FwdSmem fwd_layout(int DK, int DVT)
{
    FwdSmem L;
    int o = 0;
    const int kp = DK + 1, vp = DVT + 1, cp = kC + 1;
    L.Kd = o; o += kC * kp;
    L.Ws = o; o += kC * kp;
    L.Ts = o; o += kC * cp;
    L.Vb = o; o += kC * vp;
    L.Us = o; o += kC * vp;
    L.Ss = o; o += DK * vp;
    L.g = o; o += kC;
    L.gam = o; o += kC;
    L.bet = o; o += kC;
    L.Dd = o; o += kC;
    L.total = o;
    return L;
}

// One CTA (kThreadsWide) per (chain, d_v slice): the forward's state chain from S0
// (value-major [DV][DK] or NULL) with the cached T and W, keeping the start state of every
// chunk in S_chunks [chain][max_chunks][DK][DV] (the pages' orientation).
template <typename T>
__global__ void __launch_bounds__(kThreadsWide)
chunk_bwd_fwd_kernel(const T *__restrict__ k, const T *__restrict__ v, const float *__restrict__ log_alpha,
                     const float *__restrict__ beta, const float *__restrict__ S0,
                     const int32_t *__restrict__ cu_seqlens, int H, int DK, int DV, int max_chunks,
                     const float *__restrict__ cache, float *__restrict__ S_chunks)
{
    extern __shared__ float sm[];
    const int DVT = slice_cols(DV);
    const FwdSmem Y = fwd_layout(DK, DVT);
    float *Kd = sm + Y.Kd, *Ws = sm + Y.Ws, *Ts = sm + Y.Ts, *Vb = sm + Y.Vb, *Us = sm + Y.Us, *Ss = sm + Y.Ss;
    float *g = sm + Y.g, *gam = sm + Y.gam, *bet = sm + Y.bet, *Dd = sm + Y.Dd;
    const int kp = DK + 1, vp = DVT + 1, cp = kC + 1;
    const int n_vt = DV / DVT;
    const int chain = blockIdx.x / n_vt, v0 = (blockIdx.x % n_vt) * DVT;
    const int seq = chain / H, h = chain % H;
    const int tid = threadIdx.x;
    const int64_t len = (int64_t)cu_seqlens[seq + 1] - cu_seqlens[seq];
    const size_t st_off = (size_t)chain * DV * DK;
    for (int i = tid; i < DK * DVT; i += blockDim.x) {
        const int a = i % DK, b = i / DK;
        Ss[a * vp + b] = S0 ? S0[st_off + (size_t)(v0 + b) * DK + a] : 0.f;
    }
    const int n_chunks = (int)((len + kC - 1) / kC);
    for (int c = 0; c < n_chunks; ++c) {
        int64_t c0;
        int n;
        chunk_of(cu_seqlens, seq, c, c0, n);
        const float *cb = cache + ((size_t)chain * max_chunks + c) * cache_floats(DK);
        __syncthreads();
        {
            float *dst = S_chunks + ((size_t)chain * max_chunks + c) * DK * DV + v0;
            for (int i = tid; i < DK * DVT; i += blockDim.x) {
                const int a = i / DVT, b = i % DVT;
                dst[(size_t)a * DV + b] = Ss[a * vp + b];
            }
        }
        load_rows(Kd, kp, k, c0, n, H, h, DK, 0, DK, 1.f);
        load_rows(Vb, vp, v, c0, n, H, h, DV, v0, DVT, 1.f);
        load_block(Ts, cp, cb + kCacheT, kC, kC);
        load_block(Ws, kp, cb + kCacheW, kC, DK);
        if (tid < 32) chunk_decays(log_alpha, beta, c0, n, H, h, g, gam, bet, Dd);
        __syncthreads();
        for (int i = tid; i < kC * DK; i += blockDim.x) Kd[(i / DK) * kp + i % DK] *= Dd[i / DK];
        for (int i = tid; i < kC * DVT; i += blockDim.x) Vb[(i / DVT) * vp + i % DVT] *= bet[i / DVT];
        __syncthreads();
        // U~ = T diag(beta) V - W S
        {
            constexpr int TM = 4, TN = 2;
            const int ntm = kC / TM, ntn = DVT / TN;
            for (int gi = tid; gi < ntm * ntn; gi += blockDim.x) {
                const int tm = gi / ntn, tn = gi % ntn;
                float acc[TM][TN];
                zero(acc);
                mm_acc(acc, tm, tn, ntm, ntn, kC, [&](int t, int s) { return Ts[t * cp + s]; },
                       [&](int s, int b) { return Vb[s * vp + b]; });
                mm_acc(acc, tm, tn, ntm, ntn, DK, [&](int t, int a) { return -Ws[t * kp + a]; },
                       [&](int a, int b) { return Ss[a * vp + b]; });
#pragma unroll
                for (int i = 0; i < TM; ++i)
#pragma unroll
                    for (int j = 0; j < TN; ++j) Us[(tm + i * ntm) * vp + tn + j * ntn] = acc[i][j];
            }
        }
        __syncthreads();
        // S <- gamma_C S + (diag(D) K)^T U~ (each thread reads and writes only its own entries of S)
        {
            constexpr int TM = 4, TN = 4;
            const int ntm = DK / TM, ntn = DVT / TN;
            const float gamC = gam[kC - 1];
            for (int gi = tid; gi < ntm * ntn; gi += blockDim.x) {
                const int tm = gi / ntn, tn = gi % ntn;
                float acc[TM][TN];
#pragma unroll
                for (int i = 0; i < TM; ++i)
#pragma unroll
                    for (int j = 0; j < TN; ++j) acc[i][j] = gamC * Ss[(tm + i * ntm) * vp + tn + j * ntn];
                mm_acc(acc, tm, tn, ntm, ntn, kC, [&](int a, int s) { return Kd[s * kp + a]; },
                       [&](int s, int b) { return Us[s * vp + b]; });
#pragma unroll
                for (int i = 0; i < TM; ++i)
#pragma unroll
                    for (int j = 0; j < TN; ++j) Ss[(tm + i * ntm) * vp + tn + j * ntn] = acc[i][j];
            }
        }
    }
}

// --------------------------------------------------------------------------- state
struct StateSmem {
    int Kd, Qg, Ws, Ps, dYs, dUs, dSs, g, gam, bet, Dd, total;
};
__host__ __device__ inline StateSmem state_layout(int DK, int DVT)
{
    StateSmem L;
    int o = 0;
    const int kp = DK + 1, vp = DVT + 1, cp = kC + 1;
    L.Kd = o; o += kC * kp;
    L.Qg = o; o += kC * kp;
    L.Ws = o; o += kC * kp;
    L.Ps = o; o += kC * cp;
    L.dYs = o; o += kC * vp;
    L.dUs = o; o += kC * vp;
    L.dSs = o; o += DK * vp;
    L.g = o; o += kC;
    L.gam = o; o += kC;
    L.bet = o; o += kC;
    L.Dd = o; o += kC;
    L.total = o;
    return L;
}

// One CTA (kThreadsWide) per (chain, d_v slice): dS from dS_T back through the chunks with
// the cached W and P; dS at the end of every chunk goes to dS_chunks
// [chain][max_chunks][DK][DV], the final one to dS0 (value-major [DV][DK]).
template <typename T>
__global__ void __launch_bounds__(kThreadsWide)
chunk_bwd_state_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ dy,
                       const float *__restrict__ log_alpha, const float *__restrict__ beta,
                       const int32_t *__restrict__ cu_seqlens, int H, int DK, int DV, float scale,
                       const float *__restrict__ dS_T, int max_chunks, const float *__restrict__ cache,
                       float *__restrict__ dS_chunks, float *__restrict__ dS0)
{
    extern __shared__ float sm[];
    const int DVT = slice_cols(DV);
    const StateSmem Y = state_layout(DK, DVT);
    float *Kd = sm + Y.Kd, *Qg = sm + Y.Qg, *Ws = sm + Y.Ws, *Ps = sm + Y.Ps;
    float *dYs = sm + Y.dYs, *dUs = sm + Y.dUs, *dSs = sm + Y.dSs;
    float *g = sm + Y.g, *gam = sm + Y.gam, *bet = sm + Y.bet, *Dd = sm + Y.Dd;
    const int kp = DK + 1, vp = DVT + 1, cp = kC + 1;
    const int n_vt = DV / DVT;
    const int chain = blockIdx.x / n_vt, v0 = (blockIdx.x % n_vt) * DVT;
    const int seq = chain / H, h = chain % H;
    const int tid = threadIdx.x;
    const int64_t len = (int64_t)cu_seqlens[seq + 1] - cu_seqlens[seq];
    const size_t st_off = (size_t)chain * DV * DK;
    for (int i = tid; i < DK * DVT; i += blockDim.x) {
        const int a = i % DK, b = i / DK;
        dSs[a * vp + b] = dS_T ? dS_T[st_off + (size_t)(v0 + b) * DK + a] : 0.f;
    }
    const int n_chunks = (int)((len + kC - 1) / kC);
    for (int c = n_chunks - 1; c >= 0; --c) {
        int64_t c0;
        int n;
        chunk_of(cu_seqlens, seq, c, c0, n);
        const float *cb = cache + ((size_t)chain * max_chunks + c) * cache_floats(DK);
        __syncthreads();
        {
            float *dst = dS_chunks + ((size_t)chain * max_chunks + c) * DK * DV + v0;
            for (int i = tid; i < DK * DVT; i += blockDim.x) {
                const int a = i / DVT, b = i % DVT;
                dst[(size_t)a * DV + b] = dSs[a * vp + b];
            }
        }
        load_rows(Kd, kp, k, c0, n, H, h, DK, 0, DK, 1.f);
        load_rows(Qg, kp, q, c0, n, H, h, DK, 0, DK, scale);
        load_rows(dYs, vp, dy, c0, n, H, h, DV, v0, DVT, 1.f);
        load_block(Ws, kp, cb + kCacheW, kC, DK);
        load_block(Ps, cp, cb + kCacheP, kC, kC);
        if (tid < 32) chunk_decays(log_alpha, beta, c0, n, H, h, g, gam, bet, Dd);
        __syncthreads();
        for (int i = tid; i < kC * DK; i += blockDim.x) {
            const int t = i / DK, a = i % DK;
            Kd[t * kp + a] *= Dd[t];
            Qg[t * kp + a] *= gam[t];
        }
        __syncthreads();
        // dU~ = P^T dY + diag(D) K dS'
        {
            constexpr int TM = 4, TN = 2;
            const int ntm = kC / TM, ntn = DVT / TN;
            for (int gi = tid; gi < ntm * ntn; gi += blockDim.x) {
                const int tm = gi / ntn, tn = gi % ntn;
                float acc[TM][TN];
                zero(acc);
                mm_acc(acc, tm, tn, ntm, ntn, kC, [&](int s, int t) { return Ps[t * cp + s]; },
                       [&](int t, int b) { return dYs[t * vp + b]; });
                mm_acc(acc, tm, tn, ntm, ntn, DK, [&](int s, int a) { return Kd[s * kp + a]; },
                       [&](int a, int b) { return dSs[a * vp + b]; });
#pragma unroll
                for (int i = 0; i < TM; ++i)
#pragma unroll
                    for (int j = 0; j < TN; ++j) dUs[(tm + i * ntm) * vp + tn + j * ntn] = acc[i][j];
            }
        }
        __syncthreads();
        // dS = gamma_C dS' + (diag(gamma) Q)^T dY - W^T dU~ (own entries of dS only)
        {
            constexpr int TM = 4, TN = 4;
            const int ntm = DK / TM, ntn = DVT / TN;
            const float gamC = gam[kC - 1];
            for (int gi = tid; gi < ntm * ntn; gi += blockDim.x) {
                const int tm = gi / ntn, tn = gi % ntn;
                float acc[TM][TN];
#pragma unroll
                for (int i = 0; i < TM; ++i)
#pragma unroll
                    for (int j = 0; j < TN; ++j) acc[i][j] = gamC * dSs[(tm + i * ntm) * vp + tn + j * ntn];
                mm_acc(acc, tm, tn, ntm, ntn, kC, [&](int a, int t) { return Qg[t * kp + a]; },
                       [&](int t, int b) { return dYs[t * vp + b]; });
                mm_acc(acc, tm, tn, ntm, ntn, kC, [&](int a, int t) { return -Ws[t * kp + a]; },
                       [&](int t, int b) { return dUs[t * vp + b]; });
#pragma unroll
                for (int i = 0; i < TM; ++i)
#pragma unroll
                    for (int j = 0; j < TN; ++j) dSs[(tm + i * ntm) * vp + tn + j * ntn] = acc[i][j];
            }
        }
    }
    __syncthreads();
    if (dS0)
        for (int i = tid; i < DK * DVT; i += blockDim.x) {
            const int a = i % DK, b = i / DK;
            dS0[st_off + (size_t)(v0 + b) * DK + a] = dSs[a * vp + b];
        }
}

// --------------------------------------------------------------------------- vpart
struct VpartSmem {
    int Ks, Ts, Ps, Ss, dSs, Vs, dYs, Uts, dUs, Zs, g, gam, bet, Dd, red, total;
};
__host__ __device__ inline VpartSmem vpart_layout(int DK, int DVT)
{
    VpartSmem L;
    int o = 0;
    const int kp = DK + 1, vp = DVT + 1, cp = kC + 1;
    L.Ks = o; o += kC * kp;
    L.Ts = o; o += kC * cp;
    L.Ps = o; o += kC * cp;
    L.Ss = o; o += DK * vp;
    L.dSs = o; o += DK * vp;
    L.Vs = o; o += kC * vp;
    L.dYs = o; o += kC * vp;
    L.Uts = o; o += kC * vp;
    L.dUs = o; o += kC * vp;
    L.Zs = o; o += kC * vp;
    L.g = o; o += kC;
    L.gam = o; o += kC;
    L.bet = o; o += kC;
    L.Dd = o; o += kC;
    L.red = o; o += kThreadsWide / 32;
    L.total = o;
    return L;
}

// One CTA (kThreadsWide) per (chain, chunk, d_v slice): dV of the slice, and the slice's share
// of the sums over v, written to the slice's block of the sums buffer
// [chain][max_chunks][n_slices][part_floats].
template <typename T>
__global__ void __launch_bounds__(kThreadsWide)
chunk_bwd_vpart_kernel(const T *__restrict__ k, const T *__restrict__ v, const T *__restrict__ dy,
                       const float *__restrict__ log_alpha, const float *__restrict__ beta,
                       const int32_t *__restrict__ cu_seqlens, int H, int DK, int DV, int max_chunks,
                       const float *__restrict__ cache, const float *__restrict__ S_chunks,
                       const float *__restrict__ dS_chunks, float *__restrict__ parts, float *__restrict__ dv_out)
{
    extern __shared__ float sm[];
    const int DVT = slice_cols(DV);
    const VpartSmem Y = vpart_layout(DK, DVT);
    float *Ks = sm + Y.Ks, *Ts = sm + Y.Ts, *Ps = sm + Y.Ps, *Ss = sm + Y.Ss, *dSs = sm + Y.dSs;
    float *Vs = sm + Y.Vs, *dYs = sm + Y.dYs, *Uts = sm + Y.Uts, *dUs = sm + Y.dUs, *Zs = sm + Y.Zs;
    float *g = sm + Y.g, *gam = sm + Y.gam, *bet = sm + Y.bet, *Dd = sm + Y.Dd, *red = sm + Y.red;
    const int kp = DK + 1, vp = DVT + 1, cp = kC + 1;
    const int n_vt = DV / DVT;
    const int c = blockIdx.y;
    const int chain = blockIdx.x / n_vt, vt = blockIdx.x % n_vt, v0 = vt * DVT;
    const int seq = chain / H, h = chain % H;
    const int tid = threadIdx.x;
    int64_t c0;
    int n;
    if (!chunk_of(cu_seqlens, seq, c, c0, n)) return;
    const size_t cidx = (size_t)chain * max_chunks + c;
    const float *cb = cache + cidx * cache_floats(DK);
    const float *Sg = S_chunks + cidx * DK * DV + v0, *dSg = dS_chunks + cidx * DK * DV + v0;
    for (int i = tid; i < DK * DVT; i += blockDim.x) {
        const int a = i / DVT, b = i % DVT;
        Ss[a * vp + b] = Sg[(size_t)a * DV + b];
        dSs[a * vp + b] = dSg[(size_t)a * DV + b];
    }
    load_rows(Ks, kp, k, c0, n, H, h, DK, 0, DK, 1.f);
    load_rows(Vs, vp, v, c0, n, H, h, DV, v0, DVT, 1.f);
    load_rows(dYs, vp, dy, c0, n, H, h, DV, v0, DVT, 1.f);
    load_block(Ts, cp, cb + kCacheT, kC, kC);
    load_block(Ps, cp, cb + kCacheP, kC, kC);
    if (tid < 32) chunk_decays(log_alpha, beta, c0, n, H, h, g, gam, bet, Dd);
    __syncthreads();
    float *P = parts + (cidx * n_vt + vt) * part_floats(DK);
    float *PdP = P, *PdT = P + kC * kC, *PdW = P + 2 * kC * kC, *PdKd = PdW + kC * DK, *PdYS = PdKd + kC * DK;
    float *Pvs = PdYS + kC * DK, *PdgC = Pvs + kC;
    // Z = diag(beta) (V - diag(gamma) K S);  dU~ = P^T dY + diag(D) K dS'
    {
        constexpr int TM = 4, TN = 2;
        const int ntm = kC / TM, ntn = DVT / TN;
        for (int gi = tid; gi < ntm * ntn; gi += blockDim.x) {
            const int tm = gi / ntn, tn = gi % ntn;
            float ks[TM][TN], kd[TM][TN], pd[TM][TN];
            zero(ks);
            zero(kd);
            zero(pd);
#pragma unroll 4
            for (int a = 0; a < DK; ++a) {
                float av[TM], bs[TN], bd[TN];
#pragma unroll
                for (int i = 0; i < TM; ++i) av[i] = Ks[(tm + i * ntm) * kp + a];
#pragma unroll
                for (int j = 0; j < TN; ++j) {
                    bs[j] = Ss[a * vp + tn + j * ntn];
                    bd[j] = dSs[a * vp + tn + j * ntn];
                }
#pragma unroll
                for (int i = 0; i < TM; ++i)
#pragma unroll
                    for (int j = 0; j < TN; ++j) {
                        ks[i][j] = fmaf(av[i], bs[j], ks[i][j]);
                        kd[i][j] = fmaf(av[i], bd[j], kd[i][j]);
                    }
            }
            mm_acc(pd, tm, tn, ntm, ntn, kC, [&](int s, int t) { return Ps[t * cp + s]; },
                   [&](int t, int b) { return dYs[t * vp + b]; });
#pragma unroll
            for (int i = 0; i < TM; ++i) {
                const int t = tm + i * ntm;
#pragma unroll
                for (int j = 0; j < TN; ++j) {
                    const int b = tn + j * ntn;
                    Zs[t * vp + b] = bet[t] * (Vs[t * vp + b] - gam[t] * ks[i][j]);
                    dUs[t * vp + b] = fmaf(Dd[t], kd[i][j], pd[i][j]);
                }
            }
        }
    }
    __syncthreads();
    // U~ = T Z;  T^T dU~ -> dV = diag(beta) T^T dU~ and the row sums of V o T^T dU~.
    // ntm * ntn is a multiple of 32 and at most the block, so every lane of a warp that
    // enters has a tile and the row sums can use shuffles.
    {
        constexpr int TM = 4, TN = 2;
        const int ntm = kC / TM, ntn = DVT / TN;
        if (tid < ntm * ntn) {
            const int tm = tid / ntn, tn = tid % ntn;
            float u[TM][TN], w[TM][TN];
            zero(u);
            zero(w);
            mm_acc(u, tm, tn, ntm, ntn, kC, [&](int t, int s) { return Ts[t * cp + s]; },
                   [&](int s, int b) { return Zs[s * vp + b]; });
            mm_acc(w, tm, tn, ntm, ntn, kC, [&](int t, int s) { return Ts[s * cp + t]; },
                   [&](int s, int b) { return dUs[s * vp + b]; });
#pragma unroll
            for (int i = 0; i < TM; ++i) {
                const int t = tm + i * ntm;
                float rs = 0.f;
#pragma unroll
                for (int j = 0; j < TN; ++j) {
                    const int b = tn + j * ntn;
                    Uts[t * vp + b] = u[i][j];
                    if (t < n) dv_out[((size_t)(c0 + t) * H + h) * DV + v0 + b] = bet[t] * w[i][j];
                    rs = fmaf(Vs[t * vp + b], w[i][j], rs);
                }
                rs = row_group_sum(rs, ntn);
                if (tn == 0) Pvs[t] = rs;
            }
        }
    }
    __syncthreads();
    // this slice's dY U~^T and dU~ Z^T [C][C]
    {
        constexpr int TM = 4, TN = 2;
        const int ntm = kC / TM, ntn = kC / TN;
        for (int gi = tid; gi < ntm * ntn; gi += blockDim.x) {
            const int tm = gi / ntn, tn = gi % ntn;
            float p[TM][TN], tt[TM][TN];
            zero(p);
            zero(tt);
            mm_acc(p, tm, tn, ntm, ntn, DVT, [&](int t, int b) { return dYs[t * vp + b]; },
                   [&](int b, int s) { return Uts[s * vp + b]; });
            mm_acc(tt, tm, tn, ntm, ntn, DVT, [&](int t, int b) { return dUs[t * vp + b]; },
                   [&](int b, int s) { return Zs[s * vp + b]; });
#pragma unroll
            for (int i = 0; i < TM; ++i)
#pragma unroll
                for (int j = 0; j < TN; ++j) {
                    const int e = (tm + i * ntm) * kC + tn + j * ntn;
                    PdP[e] = p[i][j];
                    PdT[e] = tt[i][j];
                }
        }
    }
    // this slice's -dU~ S^T, U~ dS'^T and dY S^T [C][DK]
    {
        constexpr int TM = 4, TN = 4;
        const int ntm = kC / TM, ntn = DK / TN;
        for (int gi = tid; gi < ntm * ntn; gi += blockDim.x) {
            const int tm = gi / ntn, tn = gi % ntn;
            float w[TM][TN], kd[TM][TN], ys[TM][TN];
            zero(w);
            zero(kd);
            zero(ys);
#pragma unroll 2
            for (int b = 0; b < DVT; ++b) {
                float au[TM], at[TM], ay[TM], bs[TN], bd[TN];
#pragma unroll
                for (int i = 0; i < TM; ++i) {
                    const int t = tm + i * ntm;
                    au[i] = dUs[t * vp + b];
                    at[i] = Uts[t * vp + b];
                    ay[i] = dYs[t * vp + b];
                }
#pragma unroll
                for (int j = 0; j < TN; ++j) {
                    const int a = tn + j * ntn;
                    bs[j] = Ss[a * vp + b];
                    bd[j] = dSs[a * vp + b];
                }
#pragma unroll
                for (int i = 0; i < TM; ++i)
#pragma unroll
                    for (int j = 0; j < TN; ++j) {
                        w[i][j] = fmaf(au[i], bs[j], w[i][j]);
                        kd[i][j] = fmaf(at[i], bd[j], kd[i][j]);
                        ys[i][j] = fmaf(ay[i], bs[j], ys[i][j]);
                    }
            }
#pragma unroll
            for (int i = 0; i < TM; ++i)
#pragma unroll
                for (int j = 0; j < TN; ++j) {
                    const int e = (tm + i * ntm) * DK + tn + j * ntn;
                    PdW[e] = -w[i][j];
                    PdKd[e] = kd[i][j];
                    PdYS[e] = ys[i][j];
                }
        }
    }
    // <dS', S> over this slice
    float sd = 0.f;
    for (int i = tid; i < DK * DVT; i += blockDim.x) {
        const int a = i / DVT, b = i % DVT;
        sd = fmaf(dSs[a * vp + b], Ss[a * vp + b], sd);
    }
    sd = group_sum<32>(sd);
    if ((tid & 31) == 0) red[tid >> 5] = sd;
    __syncthreads();
    if (tid == 0) {
        float tot = 0.f;
        for (int w = 0; w < (int)(blockDim.x / 32); ++w) tot += red[w];
        PdgC[0] = tot;
    }
}

// --------------------------------------------------------------------------- kpart
struct KpartSmem {
    int Ks, Qs, PdWs, Ts, G1, Asym, dGs, Es, g, gam, bet, Dd, red, total;
};
__host__ __device__ inline KpartSmem kpart_layout(int DK)
{
    KpartSmem L;
    int o = 0;
    const int kp = DK + 1, cp = kC + 1;
    L.Ks = o; o += kC * kp;
    L.Qs = o; o += kC * kp;
    L.PdWs = o; o += kC * kp;
    L.Ts = o; o += kC * cp;
    L.G1 = o; o += kC * cp;
    L.Asym = o; o += kC * cp;
    L.dGs = o; o += kC * cp;
    L.Es = o; o += kC * cp;
    L.g = o; o += kC;
    L.gam = o; o += kC;
    L.bet = o; o += kC;
    L.Dd = o; o += kC;
    L.red = o; o += 5 * kC;
    L.total = o;
    return L;
}

// One CTA (kThreads) per (chain, chunk): dQ, dK, dbeta and dlog_alpha of the chunk from its
// cache block and its sums buffer (the value slices' blocks added here, in slice order).
template <typename T>
__global__ void __launch_bounds__(kThreads)
chunk_bwd_kpart_kernel(const T *__restrict__ q, const T *__restrict__ k, const float *__restrict__ log_alpha,
                       const float *__restrict__ beta, const int32_t *__restrict__ cu_seqlens, int H, int DK,
                       int n_vt, float scale, int max_chunks, const float *__restrict__ cache,
                       const float *__restrict__ parts, float *__restrict__ dq, float *__restrict__ dk,
                       float *__restrict__ dbeta, float *__restrict__ dlog_alpha)
{
    extern __shared__ float sm[];
    const KpartSmem Y = kpart_layout(DK);
    float *Ks = sm + Y.Ks, *Qs = sm + Y.Qs, *PdWs = sm + Y.PdWs, *Ts = sm + Y.Ts, *G1 = sm + Y.G1;
    float *Asym = sm + Y.Asym, *dGs = sm + Y.dGs, *Es = sm + Y.Es, *g = sm + Y.g;
    float *gam = sm + Y.gam, *bet = sm + Y.bet, *Dd = sm + Y.Dd, *red = sm + Y.red;
    const int kp = DK + 1, cp = kC + 1;
    const int c = blockIdx.y, chain = blockIdx.x;
    const int seq = chain / H, h = chain % H;
    const int tid = threadIdx.x;
    int64_t c0;
    int n;
    if (!chunk_of(cu_seqlens, seq, c, c0, n)) return;
    const size_t cidx = (size_t)chain * max_chunks + c;
    const float *cb = cache + cidx * cache_floats(DK);
    const size_t pf = part_floats(DK);
    const float *P0 = parts + cidx * n_vt * pf;
    // offsets inside one slice block
    const size_t oP = 0, oT = (size_t)kC * kC, oW = 2 * (size_t)kC * kC, oKd = oW + (size_t)kC * DK,
                 oYS = oKd + (size_t)kC * DK, oVs = oYS + (size_t)kC * DK, oGC = oVs + kC;
    auto sum_slices = [&](size_t off) -> float {
        float acc = 0.f;
        for (int j = 0; j < n_vt; ++j) acc += P0[j * pf + off];
        return acc;
    };

    load_rows(Ks, kp, k, c0, n, H, h, DK, 0, DK, 1.f);
    load_rows(Qs, kp, q, c0, n, H, h, DK, 0, DK, scale);
    load_block(Ts, cp, cb + kCacheT, kC, kC);
    if (tid < 32) chunk_decays(log_alpha, beta, c0, n, H, h, g, gam, bet, Dd);
    for (int i = tid; i < kC * DK; i += blockDim.x) PdWs[(i / DK) * kp + i % DK] = sum_slices(oW + i);
    // dT into dGs and dP into G1, summed over the slices
    for (int i = tid; i < kC * kC; i += blockDim.x) {
        const int t = i / kC, s = i % kC;
        dGs[t * cp + s] = sum_slices(oT + i);
        G1[t * cp + s] = sum_slices(oP + i);
    }
    __syncthreads();
    constexpr int SM = 4, SN = 4;            // tiles of the C x C products
    const int sntm = kC / SM, sntn = kC / SN;
    // M = dT T^T (into Asym)
    for (int gi = tid; gi < sntm * sntn; gi += blockDim.x) {
        const int tm = gi / sntn, tn = gi % sntn;
        float acc[SM][SN];
        zero(acc);
        mm_acc(acc, tm, tn, sntm, sntn, kC, [&](int t, int r) { return dGs[t * cp + r]; },
               [&](int r, int s) { return Ts[s * cp + r]; });
#pragma unroll
        for (int i = 0; i < SM; ++i)
#pragma unroll
            for (int j = 0; j < SN; ++j) Asym[(tm + i * sntm) * cp + tn + j * sntn] = acc[i][j];
    }
    __syncthreads();
    // dL = strict_tril(-T^T M), into dGs
    for (int gi = tid; gi < sntm * sntn; gi += blockDim.x) {
        const int tm = gi / sntn, tn = gi % sntn;
        float acc[SM][SN];
        zero(acc);
        mm_acc(acc, tm, tn, sntm, sntn, kC, [&](int t, int r) { return Ts[r * cp + t]; },
               [&](int r, int s) { return Asym[r * cp + s]; });
#pragma unroll
        for (int i = 0; i < SM; ++i)
#pragma unroll
            for (int j = 0; j < SN; ++j) {
                const int t = tm + i * sntm, s = tn + j * sntn;
                dGs[t * cp + s] = s < t ? -acc[i][j] : 0.f;
            }
    }
    __syncthreads();
    // dA + dA^T with dA = diag(beta) (dL o Gamma), into Asym
    for (int i = tid; i < kC * kC; i += blockDim.x) {
        const int t = i / kC, s = i % kC;
        const float da_ts = s < t ? bet[t] * dGs[t * cp + s] * expf(g[t] - g[s]) : 0.f;
        const float da_st = t < s ? bet[s] * dGs[s * cp + t] * expf(g[s] - g[t]) : 0.f;
        Asym[t * cp + s] = da_ts + da_st;
    }
    // T^T dW, kept in registers until PdWs may be overwritten (one tile per thread)
    constexpr int TM = 8, TN = 4;
    const int ntm = kC / TM, ntn = DK / TN;
    const bool has_tile = tid < ntm * ntn;
    const int tm = tid / ntn, tn = tid % ntn;
    float tdw[TM][TN];
    zero(tdw);
    if (has_tile)
        mm_acc(tdw, tm, tn, ntm, ntn, kC, [&](int t, int s) { return Ts[s * cp + t]; },
               [&](int s, int a) { return PdWs[s * kp + a]; });
    __syncthreads();
    // per entry (same thread reads and writes it): dGamma o Gamma into dGs, dL o A o Gamma into
    // Es, dP o Gamma into G1
    for (int i = tid; i < kC * kC; i += blockDim.x) {
        const int t = i / kC, s = i % kC;
        const float gts = s <= t ? expf(g[t] - g[s]) : 0.f;
        const float dl = dGs[t * cp + s], ag = cb[kCacheAG + i], dp = G1[t * cp + s];
        dGs[t * cp + s] = dp * cb[kCacheP + i] + bet[t] * dl * ag;
        Es[t * cp + s] = dl * ag;
        G1[t * cp + s] = dp * gts;
    }
    if (has_tile)
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
            for (int j = 0; j < TN; ++j) PdWs[(tm + i * ntm) * kp + tn + j * ntn] = tdw[i][j];
    __syncthreads();
    if (tid < kC) {
        float rs = 0.f, cs = 0.f, ab = 0.f;
        for (int s = 0; s < kC; ++s) {
            rs += dGs[tid * cp + s];
            cs += dGs[s * cp + tid];
            ab += Es[tid * cp + s];
        }
        red[tid] = rs - cs;          // row sum - column sum of dGamma o Gamma
        red[kC + tid] = ab;          // row sum of dL o A o Gamma
    }
    // dQ = diag(gamma) dY S^T + (dP o Gamma) K;
    // dK = (dP o Gamma)^T Q + (dA + dA^T) K + diag(beta gamma) T^T dW + diag(D) dK~.
    // ntm * ntn = 2 DK is a multiple of 32 and at most the block: shuffles are safe.
    if (has_tile) {
        float aq[TM][TN], ak[TM][TN];
        zero(aq);
        zero(ak);
#pragma unroll 2
        for (int s = 0; s < kC; ++s) {
            float g1[TM], g1t[TM], as[TM], bk[TN], bq[TN];
#pragma unroll
            for (int i = 0; i < TM; ++i) {
                const int t = tm + i * ntm;
                g1[i] = G1[t * cp + s];
                g1t[i] = G1[s * cp + t];
                as[i] = Asym[t * cp + s];
            }
#pragma unroll
            for (int j = 0; j < TN; ++j) {
                bk[j] = Ks[s * kp + tn + j * ntn];
                bq[j] = Qs[s * kp + tn + j * ntn];
            }
#pragma unroll
            for (int i = 0; i < TM; ++i)
#pragma unroll
                for (int j = 0; j < TN; ++j) {
                    aq[i][j] = fmaf(g1[i], bk[j], aq[i][j]);
                    ak[i][j] = fmaf(g1t[i], bq[j], fmaf(as[i], bk[j], ak[i][j]));
                }
        }
#pragma unroll
        for (int i = 0; i < TM; ++i) {
            const int t = tm + i * ntm;
            float rg = 0.f, rb = 0.f, rd = 0.f;
#pragma unroll
            for (int j = 0; j < TN; ++j) {
                const int a = tn + j * ntn;
                const size_t ta = (size_t)t * DK + a;
                const float pys = sum_slices(oYS + ta), pkd = sum_slices(oKd + ta);
                const float tw = PdWs[t * kp + a];
                const float kta = Ks[t * kp + a];
                rg = fmaf(Qs[t * kp + a], pys, rg);
                rb = fmaf(kta, tw, rb);
                rd = fmaf(kta, pkd, rd);
                if (t < n) {
                    dq[((size_t)(c0 + t) * H + h) * DK + a] = scale * (gam[t] * pys + aq[i][j]);
                    dk[((size_t)(c0 + t) * H + h) * DK + a] = ak[i][j] + bet[t] * gam[t] * tw + Dd[t] * pkd;
                }
            }
            rg = row_group_sum(rg, ntn);
            rb = row_group_sum(rb, ntn);
            rd = row_group_sum(rd, ntn);
            if (tn == 0) {
                red[2 * kC + t] = rg + bet[t] * rb;     // dgamma_t
                red[3 * kC + t] = rb;                   // sum_a K o T^T dW
                red[4 * kC + t] = rd;                   // dD_t
            }
        }
    }
    __syncthreads();
    if (tid < 32) {
        // dbeta_t = sum V o T^T dU~ + gamma_t sum K o T^T dW + sum dL o A o Gamma
        // dg_t = gamma_t dgamma_t + (row - column sums of dGamma o Gamma) - dD_t D_t, the
        // last row adding sum_s dD_s D_s + gamma_C <dS', S>; then the reverse cumsum
        float sumDD = red[4 * kC + tid] * Dd[tid] + red[4 * kC + tid + 32] * Dd[tid + 32];
        sumDD = group_sum<32>(sumDD);
        const float dgC = sum_slices(oGC);
        float dgv[2];
        for (int j = 0; j < 2; ++j) {
            const int t = tid + 32 * j;
            float dg = gam[t] * red[2 * kC + t] + red[t] - red[4 * kC + t] * Dd[t];
            if (t == kC - 1) dg += sumDD + gam[kC - 1] * dgC;
            dgv[j] = dg;
            const float db = sum_slices(oVs + t) + gam[t] * red[3 * kC + t] + red[kC + t];
            if (t < n) dbeta[(size_t)(c0 + t) * H + h] = db;
        }
        // reverse inclusive cumsum over t = 0..63 (lane l holds rows l and l + 32)
        float hi = dgv[1], lo = dgv[0];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float o = __shfl_down_sync(0xffffffffu, hi, off);
            if (tid + off < 32) hi += o;
        }
        const float hi_total = __shfl_sync(0xffffffffu, hi, 0);
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float o = __shfl_down_sync(0xffffffffu, lo, off);
            if (tid + off < 32) lo += o;
        }
        lo += hi_total;
        if (tid < n) dlog_alpha[(size_t)(c0 + tid) * H + h] = lo;
        if (tid + 32 < n) dlog_alpha[(size_t)(c0 + tid + 32) * H + h] = hi;
    }
}

}  // namespace bwdc
}  // namespace gdn
