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
// Three steps after a forward pass that keeps each chunk's start state (chunk_fwd_f32_kernel
// with S_chunks):
//   chunk_bwd_state_kernel  per (chain, d_v slice), chunks in reverse: dS at every chunk
//                           end and dS0; the serial part
//   chunk_bwd_vpart_kernel  per (chain, chunk, d_v slice): dV, and the slice's sums over v
//                           that the rest needs (dP, dT, dW, dK~, dY S^T, ...), each slice
//                           into its own block (no atomics: the result is deterministic)
//   chunk_bwd_kpart_kernel  per (chain, chunk): dQ, dK, dbeta, dlog_alpha
// Chunks of all chains run in parallel in the last two steps.
#pragma once
#include "gdn_common.cuh"

namespace gdn {
namespace bwdc {

constexpr int kThreads = 256;
constexpr int kC = 64;               // chunk length
constexpr int kDVT = 32;             // value columns per CTA in the sliced steps

// floats of the per-chunk sums buffer: dP, dT [C][C]; dW, dK~, dY S^T [C][DK]; the row sums
// of V o T^T dU~ [C]; <dS', S> [1]
__host__ __device__ inline size_t part_floats(int DK) { return (size_t)kC * (2 * kC + 3 * DK + 1) + 1; }

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

// A = K K^T (all t, s), L = strict_tril(beta A Gamma), P = tril(Q K^T Gamma) (when Ps), then
// T = (I + L)^-1 by forward substitution (one column per thread). Ends with a barrier.
__device__ __forceinline__ void chunk_solve(const float *Ks, const float *Qs, int kp, int DK, const float *g,
                                            const float *bet, float *As, float *Ls, float *Ps, float *Ts, int cp)
{
    for (int i = threadIdx.x; i < kC * kC; i += blockDim.x) {
        const int t = i / kC, s = i % kC;
        float ak = 0.f, aq = 0.f;
        for (int a = 0; a < DK; ++a) {
            const float ks = Ks[s * kp + a];
            ak = fmaf(Ks[t * kp + a], ks, ak);
            if (Ps) aq = fmaf(Qs[t * kp + a], ks, aq);
        }
        const float decay = s <= t ? expf(g[t] - g[s]) : 0.f;
        if (As) As[t * cp + s] = ak;
        Ls[t * cp + s] = s < t ? bet[t] * ak * decay : 0.f;
        if (Ps) Ps[t * cp + s] = s <= t ? aq * decay : 0.f;
    }
    __syncthreads();
    if (threadIdx.x < kC) {
        const int j = threadIdx.x;
        for (int t = 0; t < kC; ++t) {
            float x;
            if (t < j) {
                x = 0.f;
            } else if (t == j) {
                x = 1.f;
            } else {
                x = 0.f;
                for (int s = j; s < t; ++s) x = fmaf(-Ls[t * cp + s], Ts[s * cp + j], x);
            }
            Ts[t * cp + j] = x;
        }
    }
    __syncthreads();
}

// W = T diag(beta gamma) K  [kC][DK]. Ends with a barrier.
__device__ __forceinline__ void chunk_w(const float *Ts, int cp, const float *bet, const float *gam, const float *Ks,
                                        int kp, int DK, float *Ws)
{
    for (int i = threadIdx.x; i < kC * DK; i += blockDim.x) {
        const int t = i / DK, a = i % DK;
        float acc = 0.f;
        for (int s = 0; s <= t; ++s) acc = fmaf(Ts[t * cp + s] * bet[s] * gam[s], Ks[s * kp + a], acc);
        Ws[t * kp + a] = acc;
    }
    __syncthreads();
}

struct StateSmem {
    int Ks, Qs, dYs, dSs, Ws, dUs, Ls, Ts, Ps, g, gam, bet, Dd, total;
};
__host__ __device__ inline StateSmem state_layout(int DK)
{
    StateSmem L;
    int o = 0;
    const int kp = DK + 1, vp = kDVT + 1, cp = kC + 1;
    L.Ks = o; o += kC * kp;
    L.Qs = o; o += kC * kp;
    L.dYs = o; o += kC * vp;
    L.dSs = o; o += DK * vp;
    L.Ws = o; o += kC * kp;
    L.dUs = o; o += kC * vp;
    L.Ls = o; o += kC * cp;
    L.Ts = o; o += kC * cp;
    L.Ps = o; o += kC * cp;
    L.g = o; o += kC;
    L.gam = o; o += kC;
    L.bet = o; o += kC;
    L.Dd = o; o += kC;
    L.total = o;
    return L;
}

// One CTA per (chain, 32-column slice of d_v): dS from dS_T back through the chunks; dS at
// the end of every chunk goes to dS_chunks [chain][max_chunks][DK][DV], the final one to dS0
// (value-major [DV][DK], the library's state layout).
template <typename T>
__global__ void __launch_bounds__(kThreads)
chunk_bwd_state_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ dy,
                       const float *__restrict__ log_alpha, const float *__restrict__ beta,
                       const int32_t *__restrict__ cu_seqlens, int H, int DK, int DV, float scale,
                       const float *__restrict__ dS_T, float *__restrict__ dS_chunks, int max_chunks,
                       float *__restrict__ dS0)
{
    extern __shared__ float sm[];
    const StateSmem Y = state_layout(DK);
    float *Ks = sm + Y.Ks, *Qs = sm + Y.Qs, *dYs = sm + Y.dYs, *dSs = sm + Y.dSs, *Ws = sm + Y.Ws;
    float *dUs = sm + Y.dUs, *Ls = sm + Y.Ls, *Ts = sm + Y.Ts, *Ps = sm + Y.Ps;
    float *g = sm + Y.g, *gam = sm + Y.gam, *bet = sm + Y.bet, *Dd = sm + Y.Dd;
    const int kp = DK + 1, vp = kDVT + 1, cp = kC + 1;
    const int DVT = DV < kDVT ? DV : kDVT;
    const int n_vt = DV / DVT;
    const int chain = blockIdx.x / n_vt, v0 = (blockIdx.x % n_vt) * DVT;
    const int seq = chain / H, h = chain % H;
    const int tid = threadIdx.x;
    const int64_t bos = cu_seqlens[seq], len = (int64_t)cu_seqlens[seq + 1] - bos;
    const size_t st_off = (size_t)chain * DV * DK;
    for (int i = tid; i < DK * DVT; i += blockDim.x) {
        const int a = i / DVT, b = i % DVT;
        dSs[a * vp + b] = dS_T ? dS_T[st_off + (size_t)(v0 + b) * DK + a] : 0.f;
    }
    const int n_chunks = (int)((len + kC - 1) / kC);
    for (int c = n_chunks - 1; c >= 0; --c) {
        const int64_t c0 = bos + (int64_t)c * kC;
        const int n = (int)(len - (int64_t)c * kC < kC ? len - (int64_t)c * kC : kC);
        __syncthreads();
        {
            float *dst = dS_chunks + ((size_t)chain * max_chunks + c) * DK * DV + v0;
            for (int i = tid; i < DK * DVT; i += blockDim.x) {
                const int a = i / DVT, b = i % DVT;
                dst[(size_t)a * DV + b] = dSs[a * vp + b];
            }
        }
        load_rows(Ks, kp, k, c0, n, H, h, DK, 0, DK, 1.f);
        load_rows(Qs, kp, q, c0, n, H, h, DK, 0, DK, scale);
        load_rows(dYs, vp, dy, c0, n, H, h, DV, v0, DVT, 1.f);
        if (tid < 32) chunk_decays(log_alpha, beta, c0, n, H, h, g, gam, bet, Dd);
        __syncthreads();
        chunk_solve(Ks, Qs, kp, DK, g, bet, nullptr, Ls, Ps, Ts, cp);
        chunk_w(Ts, cp, bet, gam, Ks, kp, DK, Ws);
        // dU~ = P^T dY + diag(D) K dS'
        for (int i = tid; i < kC * DVT; i += blockDim.x) {
            const int s = i / DVT, b = i % DVT;
            float acc = 0.f;
            for (int t = s; t < kC; ++t) acc = fmaf(Ps[t * cp + s], dYs[t * vp + b], acc);
            float kd = 0.f;
            for (int a = 0; a < DK; ++a) kd = fmaf(Ks[s * kp + a], dSs[a * vp + b], kd);
            dUs[s * vp + b] = fmaf(Dd[s], kd, acc);
        }
        __syncthreads();
        // dS = gamma_C dS' + (diag(gamma) Q)^T dY - W^T dU~
        const float gamC = gam[kC - 1];
        for (int i = tid; i < DK * DVT; i += blockDim.x) {
            const int a = i / DVT, b = i % DVT;
            float acc = gamC * dSs[a * vp + b];
            for (int t = 0; t < kC; ++t)
                acc = fmaf(gam[t] * Qs[t * kp + a], dYs[t * vp + b], fmaf(-Ws[t * kp + a], dUs[t * vp + b], acc));
            dSs[a * vp + b] = acc;
        }
    }
    __syncthreads();
    if (dS0)
        for (int i = tid; i < DK * DVT; i += blockDim.x) {
            const int a = i % DK, b = i / DK;
            dS0[st_off + (size_t)(v0 + b) * DK + a] = dSs[a * vp + b];
        }
}

struct VpartSmem {
    int Ks, Qs, Ws, Ls, Ts, Ps, Ss, dSs, Vs, dYs, Uts, dUs, Zs, g, gam, bet, Dd, total;
};
__host__ __device__ inline VpartSmem vpart_layout(int DK)
{
    VpartSmem L;
    int o = 0;
    const int kp = DK + 1, vp = kDVT + 1, cp = kC + 1;
    L.Ks = o; o += kC * kp;
    L.Qs = o; o += kC * kp;
    L.Ws = o; o += kC * kp;
    L.Ls = o; o += kC * cp;
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
    L.total = o;
    return L;
}

// One CTA per (chain, chunk, 32-column slice of d_v): dV of the slice, and the slice's share
// of the sums over v, written to the slice's block of the chunk's sums buffer
// [chain][max_chunks][n_slices][part_floats].
template <typename T>
__global__ void __launch_bounds__(kThreads)
chunk_bwd_vpart_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                       const T *__restrict__ dy, const float *__restrict__ log_alpha,
                       const float *__restrict__ beta, const int32_t *__restrict__ cu_seqlens, int H, int DK,
                       int DV, float scale, const float *__restrict__ S_chunks, const float *__restrict__ dS_chunks,
                       int max_chunks, float *__restrict__ parts, float *__restrict__ dv_out)
{
    extern __shared__ float sm[];
    const VpartSmem Y = vpart_layout(DK);
    float *Ks = sm + Y.Ks, *Qs = sm + Y.Qs, *Ws = sm + Y.Ws, *Ls = sm + Y.Ls, *Ts = sm + Y.Ts, *Ps = sm + Y.Ps;
    float *Ss = sm + Y.Ss, *dSs = sm + Y.dSs, *Vs = sm + Y.Vs, *dYs = sm + Y.dYs, *Uts = sm + Y.Uts;
    float *dUs = sm + Y.dUs, *Zs = sm + Y.Zs, *g = sm + Y.g, *gam = sm + Y.gam, *bet = sm + Y.bet, *Dd = sm + Y.Dd;
    const int kp = DK + 1, vp = kDVT + 1, cp = kC + 1;
    const int DVT = DV < kDVT ? DV : kDVT;
    const int n_vt = DV / DVT;
    const int c = blockIdx.y;
    const int chain = blockIdx.x / n_vt, v0 = (blockIdx.x % n_vt) * DVT;
    const int seq = chain / H, h = chain % H;
    const int tid = threadIdx.x;
    const int64_t bos = cu_seqlens[seq], len = (int64_t)cu_seqlens[seq + 1] - bos;
    if ((int64_t)c * kC >= len) return;
    const int64_t c0 = bos + (int64_t)c * kC;
    const int n = (int)(len - (int64_t)c * kC < kC ? len - (int64_t)c * kC : kC);
    const size_t cidx = (size_t)chain * max_chunks + c;
    const float *Sg = S_chunks + cidx * DK * DV + v0, *dSg = dS_chunks + cidx * DK * DV + v0;
    for (int i = tid; i < DK * DVT; i += blockDim.x) {
        const int a = i / DVT, b = i % DVT;
        Ss[a * vp + b] = Sg[(size_t)a * DV + b];
        dSs[a * vp + b] = dSg[(size_t)a * DV + b];
    }
    load_rows(Ks, kp, k, c0, n, H, h, DK, 0, DK, 1.f);
    load_rows(Qs, kp, q, c0, n, H, h, DK, 0, DK, scale);
    load_rows(Vs, vp, v, c0, n, H, h, DV, v0, DVT, 1.f);
    load_rows(dYs, vp, dy, c0, n, H, h, DV, v0, DVT, 1.f);
    if (tid < 32) chunk_decays(log_alpha, beta, c0, n, H, h, g, gam, bet, Dd);
    __syncthreads();
    chunk_solve(Ks, Qs, kp, DK, g, bet, nullptr, Ls, Ps, Ts, cp);
    chunk_w(Ts, cp, bet, gam, Ks, kp, DK, Ws);
    // Z = diag(beta) V - diag(beta gamma) K S;  U~ = T Z;  dU~ = P^T dY + diag(D) K dS'
    for (int i = tid; i < kC * DVT; i += blockDim.x) {
        const int t = i / DVT, b = i % DVT;
        float ks = 0.f, kd = 0.f;
        for (int a = 0; a < DK; ++a) {
            ks = fmaf(Ks[t * kp + a], Ss[a * vp + b], ks);
            kd = fmaf(Ks[t * kp + a], dSs[a * vp + b], kd);
        }
        Zs[t * vp + b] = bet[t] * (Vs[t * vp + b] - gam[t] * ks);
        float acc = 0.f;
        for (int r = t; r < kC; ++r) acc = fmaf(Ps[r * cp + t], dYs[r * vp + b], acc);
        dUs[t * vp + b] = fmaf(Dd[t], kd, acc);
    }
    __syncthreads();
    float *P = parts + (cidx * n_vt + blockIdx.x % n_vt) * part_floats(DK);
    float *PdP = P, *PdT = P + kC * kC, *PdW = P + 2 * kC * kC, *PdKd = PdW + kC * DK, *PdYS = PdKd + kC * DK;
    float *Pvs = PdYS + kC * DK, *PdgC = Pvs + kC;
    for (int i = tid; i < kC * DVT; i += blockDim.x) {
        const int t = i / DVT, b = i % DVT;
        float u = 0.f, tdu = 0.f;
        for (int s = 0; s <= t; ++s) u = fmaf(Ts[t * cp + s], Zs[s * vp + b], u);
        for (int s = t; s < kC; ++s) tdu = fmaf(Ts[s * cp + t], dUs[s * vp + b], tdu);
        Uts[t * vp + b] = u;
        if (t < n) dv_out[((size_t)(c0 + t) * H + h) * DV + v0 + b] = bet[t] * tdu;
        Ls[t * cp + b] = Vs[t * vp + b] * tdu;    // L is no longer needed: V o T^T dU~ per column
    }
    __syncthreads();
    // this slice's sums over its v of: dY U~^T, dU~ Z^T [C][C]; -dU~ S^T, U~ dS'^T, dY S^T
    // [C][DK]; V o T^T dU~ [C]; <dS', S> -- written to the slice's own block
    for (int i = tid; i < kC * kC; i += blockDim.x) {
        const int t = i / kC, s = i % kC;
        float p = 0.f, tt = 0.f;
        for (int b = 0; b < DVT; ++b) {
            p = fmaf(dYs[t * vp + b], Uts[s * vp + b], p);
            tt = fmaf(dUs[t * vp + b], Zs[s * vp + b], tt);
        }
        PdP[i] = p;
        PdT[i] = tt;
    }
    for (int i = tid; i < kC * DK; i += blockDim.x) {
        const int t = i / DK, a = i % DK;
        float w = 0.f, kd = 0.f, ys = 0.f;
        for (int b = 0; b < DVT; ++b) {
            const float sab = Ss[a * vp + b];
            w = fmaf(-dUs[t * vp + b], sab, w);
            kd = fmaf(Uts[t * vp + b], dSs[a * vp + b], kd);
            ys = fmaf(dYs[t * vp + b], sab, ys);
        }
        PdW[i] = w;
        PdKd[i] = kd;
        PdYS[i] = ys;
    }
    if (tid < kC) {
        float acc = 0.f;
        for (int b = 0; b < DVT; ++b) acc += Ls[tid * cp + b];
        Pvs[tid] = acc;
    }
    float sd = 0.f;
    for (int i = tid; i < DK * DVT; i += blockDim.x) {
        const int a = i / DVT, b = i % DVT;
        sd = fmaf(dSs[a * vp + b], Ss[a * vp + b], sd);
    }
    sd = group_sum<32>(sd);
    __syncthreads();                                  // Zs is free: the warp totals go there
    if ((tid & 31) == 0) Zs[tid >> 5] = sd;
    __syncthreads();
    if (tid == 0) {
        float tot = 0.f;
        for (int w = 0; w < kThreads / 32; ++w) tot += Zs[w];
        PdgC[0] = tot;
    }
}

struct KpartSmem {
    int Ks, Qs, PdWs, As, QKs, Ts, G1, Asym, dGs, g, gam, bet, Dd, red, total;
};
__host__ __device__ inline KpartSmem kpart_layout(int DK)
{
    KpartSmem L;
    int o = 0;
    const int kp = DK + 1, cp = kC + 1;
    L.Ks = o; o += kC * kp;
    L.Qs = o; o += kC * kp;
    L.PdWs = o; o += kC * kp;
    L.As = o; o += kC * cp;
    L.QKs = o; o += kC * cp;
    L.Ts = o; o += kC * cp;
    L.G1 = o; o += kC * cp;
    L.Asym = o; o += kC * cp;
    L.dGs = o; o += kC * cp;
    L.g = o; o += kC;
    L.gam = o; o += kC;
    L.bet = o; o += kC;
    L.Dd = o; o += kC;
    L.red = o; o += 5 * kC;
    L.total = o;
    return L;
}

// One CTA per (chain, chunk): dQ, dK, dbeta and dlog_alpha of the chunk from its sums
// buffer (the value slices' blocks added here, in slice order).
template <typename T>
__global__ void __launch_bounds__(kThreads)
chunk_bwd_kpart_kernel(const T *__restrict__ q, const T *__restrict__ k, const float *__restrict__ log_alpha,
                       const float *__restrict__ beta, const int32_t *__restrict__ cu_seqlens, int H, int DK,
                       int n_vt, float scale, int max_chunks, const float *__restrict__ parts, float *__restrict__ dq,
                       float *__restrict__ dk, float *__restrict__ dbeta, float *__restrict__ dlog_alpha)
{
    extern __shared__ float sm[];
    const KpartSmem Y = kpart_layout(DK);
    float *Ks = sm + Y.Ks, *Qs = sm + Y.Qs, *PdWs = sm + Y.PdWs, *As = sm + Y.As, *QKs = sm + Y.QKs;
    float *Ts = sm + Y.Ts, *G1 = sm + Y.G1, *Asym = sm + Y.Asym, *dGs = sm + Y.dGs, *g = sm + Y.g;
    float *gam = sm + Y.gam, *bet = sm + Y.bet, *Dd = sm + Y.Dd, *red = sm + Y.red;
    const int kp = DK + 1, cp = kC + 1;
    const int c = blockIdx.y, chain = blockIdx.x;
    const int seq = chain / H, h = chain % H;
    const int tid = threadIdx.x;
    const int64_t bos = cu_seqlens[seq], len = (int64_t)cu_seqlens[seq + 1] - bos;
    if ((int64_t)c * kC >= len) return;
    const int64_t c0 = bos + (int64_t)c * kC;
    const int n = (int)(len - (int64_t)c * kC < kC ? len - (int64_t)c * kC : kC);
    const size_t pf = part_floats(DK);
    const float *P0 = parts + ((size_t)chain * max_chunks + c) * n_vt * pf;
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
    if (tid < 32) chunk_decays(log_alpha, beta, c0, n, H, h, g, gam, bet, Dd);
    for (int i = tid; i < kC * DK; i += blockDim.x) PdWs[(i / DK) * kp + i % DK] = sum_slices(oW + i);
    __syncthreads();
    // A = K K^T and Q K^T (all entries); L (in G1, for the solve) and T
    for (int i = tid; i < kC * kC; i += blockDim.x) {
        const int t = i / kC, s = i % kC;
        float ak = 0.f, aq = 0.f;
        for (int a = 0; a < DK; ++a) {
            const float ks = Ks[s * kp + a];
            ak = fmaf(Ks[t * kp + a], ks, ak);
            aq = fmaf(Qs[t * kp + a], ks, aq);
        }
        As[t * cp + s] = ak;
        QKs[t * cp + s] = aq;
        G1[t * cp + s] = s < t ? bet[t] * ak * expf(g[t] - g[s]) : 0.f;
    }
    __syncthreads();
    if (tid < kC) {
        const int j = tid;
        for (int t = 0; t < kC; ++t) {
            float x;
            if (t < j) {
                x = 0.f;
            } else if (t == j) {
                x = 1.f;
            } else {
                x = 0.f;
                for (int s = j; s < t; ++s) x = fmaf(-G1[t * cp + s], Ts[s * cp + j], x);
            }
            Ts[t * cp + j] = x;
        }
    }
    __syncthreads();
    // dT into dGs and dP into G1, summed over the slices
    for (int i = tid; i < kC * kC; i += blockDim.x) {
        const int t = i / kC, s = i % kC;
        dGs[t * cp + s] = sum_slices(oT + i);
        G1[t * cp + s] = sum_slices(oP + i);
    }
    __syncthreads();
    // M = dT T^T (into Asym)
    for (int i = tid; i < kC * kC; i += blockDim.x) {
        const int t = i / kC, s = i % kC;
        float acc = 0.f;
        for (int r = 0; r <= s; ++r) acc = fmaf(dGs[t * cp + r], Ts[s * cp + r], acc);
        Asym[t * cp + s] = acc;
    }
    __syncthreads();
    // dL = strict_tril(-T^T M), into dGs
    for (int i = tid; i < kC * kC; i += blockDim.x) {
        const int t = i / kC, s = i % kC;
        float dl = 0.f;
        if (s < t)
            for (int r = t; r < kC; ++r) dl = fmaf(-Ts[r * cp + t], Asym[r * cp + s], dl);
        dGs[t * cp + s] = dl;
    }
    __syncthreads();
    // dA + dA^T with dA = diag(beta) (dL o Gamma), into Asym
    for (int i = tid; i < kC * kC; i += blockDim.x) {
        const int t = i / kC, s = i % kC;
        const float da_ts = s < t ? bet[t] * dGs[t * cp + s] * expf(g[t] - g[s]) : 0.f;
        const float da_st = t < s ? bet[s] * dGs[s * cp + t] * expf(g[s] - g[t]) : 0.f;
        Asym[t * cp + s] = da_ts + da_st;
    }
    __syncthreads();
    // per entry (same thread reads and writes it): dGamma o Gamma into dGs, dL o A o Gamma into
    // As, dP o Gamma (lower triangle) into G1
    for (int i = tid; i < kC * kC; i += blockDim.x) {
        const int t = i / kC, s = i % kC;
        const float gts = s <= t ? expf(g[t] - g[s]) : 0.f;
        const float dl = dGs[t * cp + s], a = As[t * cp + s], dp = G1[t * cp + s];
        dGs[t * cp + s] = (dp * QKs[t * cp + s] + bet[t] * dl * a) * gts;
        As[t * cp + s] = dl * a * gts;
        G1[t * cp + s] = dp * gts;
    }
    __syncthreads();
    if (tid < kC) {
        float rs = 0.f, cs = 0.f, ab = 0.f;
        for (int s = 0; s < kC; ++s) {
            rs += dGs[tid * cp + s];
            cs += dGs[s * cp + tid];
            ab += As[tid * cp + s];
        }
        red[tid] = rs - cs;          // row sum - column sum of dGamma o Gamma
        red[kC + tid] = ab;          // row sum of dL o A o Gamma
    }
    // per (t, a): dQ, dK and the row sums; a warp per row t at a time, lanes over a
    const int warp = tid >> 5, lane = tid & 31;
    for (int t = warp; t < kC; t += kThreads / 32) {
        float rg = 0.f, rb = 0.f, rd = 0.f;
        for (int a = lane; a < DK; a += 32) {
            const size_t ta = (size_t)t * DK + a;
            float tdw = 0.f;
            for (int s = t; s < kC; ++s) tdw = fmaf(Ts[s * cp + t], PdWs[s * kp + a], tdw);
            float gq = 0.f, gk = 0.f, sk = 0.f;
            for (int s = 0; s < kC; ++s) {
                gq = fmaf(G1[t * cp + s], Ks[s * kp + a], gq);
                gk = fmaf(G1[s * cp + t], Qs[s * kp + a], gk);
                sk = fmaf(Asym[t * cp + s], Ks[s * kp + a], sk);
            }
            const float pys = sum_slices(oYS + ta), pkd = sum_slices(oKd + ta);
            const float dqv = gam[t] * pys + gq;
            const float dkv = gk + bet[t] * gam[t] * tdw + sk + Dd[t] * pkd;
            rg = fmaf(Qs[t * kp + a], pys, rg);
            rb = fmaf(Ks[t * kp + a], tdw, rb);
            rd = fmaf(Ks[t * kp + a], pkd, rd);
            if (t < n) {
                dq[((size_t)(c0 + t) * H + h) * DK + a] = scale * dqv;
                dk[((size_t)(c0 + t) * H + h) * DK + a] = dkv;
            }
        }
        rg = group_sum<32>(rg);
        rb = group_sum<32>(rb);
        rd = group_sum<32>(rd);
        if (lane == 0) {
            red[2 * kC + t] = rg + bet[t] * rb;     // dgamma_t
            red[3 * kC + t] = rb;                   // sum_a K o T^T dW
            red[4 * kC + t] = rd;                   // dD_t
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
