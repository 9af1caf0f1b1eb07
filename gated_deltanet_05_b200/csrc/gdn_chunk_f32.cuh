// gdn_chunk_f32.cuh -- chunkwise-parallel gated delta rule on CUDA cores, fp32 throughout.
//
// The general path: any supported (d_k, d_v, chunk) and fp32 or bf16 inputs (bf16 is
// widened to fp32 on load). It follows the token update rule of the joezjh.github.io
// notes page "Qwen3.8-Flash-Next" (section "Gated DeltaNet 核心机制") through its
// chunked rewrite, exact up to rounding. Inside a chunk of C tokens with start state
// S (d_k x d_v), u~_t = beta_t e_t, g_t = sum_{r<=t} log alpha_r, gamma_t = exp(g_t):
//     S_t = gamma_t S + sum_{s<=t} exp(g_t - g_s) k_s u~_s^T          (induction)
//     (I + L) U~ = diag(beta) V - diag(beta gamma) K S,
//         L_ts = beta_t exp(g_t - g_s) k_t.k_s for s < t
//     T = (I + L)^-1;  U = T diag(beta) V;  W = T diag(beta gamma) K;  U~ = U - W S
//     Y = diag(gamma) Q S + P U~,   P_ts = exp(g_t - g_s) q_t.k_s for s <= t (y reads S_t)
//     S <- gamma_C S + sum_s exp(g_C - g_s) k_s u~_s^T
// Every exponent is <= 0, so nothing overflows however strong the decay.
//
// One CTA owns one (sequence, head) chain and a DVT-wide slice of the value dimension
// (columns of S evolve independently); the v-independent work (K K^T, Q K^T, T, W) is
// recomputed per slice. Chunks of a chain run in order inside the CTA.
#pragma once
#include "gdn_common.cuh"

namespace gdn {

constexpr int kChunkF32Threads = 256;

struct ChunkF32Smem {
    // float offsets into dynamic shared memory
    int Ks, Qs, Vs, Ss, Ws, Us, Ls, Ts, Ps, g, gam, bet, total;
};

__host__ __device__ inline ChunkF32Smem chunk_f32_layout(int C, int DK, int DVT)
{
    ChunkF32Smem L;
    int o = 0;
    const int kp = DK + 1, vp = DVT + 1, cp = C + 1;
    L.Ks = o; o += C * kp;
    L.Qs = o; o += C * kp;
    L.Vs = o; o += C * vp;
    L.Ss = o; o += DK * vp;
    L.Ws = o; o += C * kp;
    L.Us = o; o += C * vp;
    L.Ls = o; o += C * cp;
    L.Ts = o; o += C * cp;
    L.Ps = o; o += C * cp;
    L.g = o; o += C;
    L.gam = o; o += C;
    L.bet = o; o += C;
    L.total = o;
    return L;
}

template <typename T, typename TY>
__global__ void __launch_bounds__(kChunkF32Threads)
chunk_fwd_f32_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                     const float *__restrict__ log_alpha, const float *__restrict__ beta,
                     const float *__restrict__ S0, const int32_t *__restrict__ cu_seqlens,
                     int H, int DK, int DV, int C, int DVT, float scale, TY *__restrict__ y,
                     float *__restrict__ S_T)
{
    extern __shared__ float sm[];
    const ChunkF32Smem L = chunk_f32_layout(C, DK, DVT);
    float *Ks = sm + L.Ks, *Qs = sm + L.Qs, *Vs = sm + L.Vs, *Ss = sm + L.Ss, *Ws = sm + L.Ws;
    float *Us = sm + L.Us, *Ls = sm + L.Ls, *Ts = sm + L.Ts, *Ps = sm + L.Ps;
    float *g = sm + L.g, *gam = sm + L.gam, *bet = sm + L.bet;
    const int kp = DK + 1, vp = DVT + 1, cp = C + 1;

    const int n_vt = DV / DVT;
    const int chain = blockIdx.x / n_vt;
    const int vt = blockIdx.x % n_vt;
    const int seq = chain / H, h = chain % H;
    const int v0 = vt * DVT;
    const int tid = threadIdx.x;
    const int64_t bos = cu_seqlens[seq], eos = cu_seqlens[seq + 1];

    // state slice S[a][b] (pages' orientation) for value columns v0 .. v0+DVT
    const size_t st_off = ((size_t)seq * H + h) * (size_t)DV * DK;
    for (int i = tid; i < DK * DVT; i += blockDim.x) {
        const int a = i % DK, b = i / DK;
        Ss[a * vp + b] = S0 ? S0[st_off + (size_t)(v0 + b) * DK + a] : 0.f;
    }

    for (int64_t c0 = bos; c0 < eos; c0 += C) {
        const int n = (int)((eos - c0) < C ? (eos - c0) : C);
        __syncthreads();
        // 1. load the chunk (rows past the sequence end are zero, with beta = log alpha = 0)
        for (int i = tid; i < C * DK; i += blockDim.x) {
            const int t = i / DK, a = i % DK;
            float kv = 0.f, qv = 0.f;
            if (t < n) {
                const size_t off = ((size_t)(c0 + t) * H + h) * DK + a;
                kv = to_f32(k[off]);
                qv = scale * to_f32(q[off]);
            }
            Ks[t * kp + a] = kv;
            Qs[t * kp + a] = qv;
        }
        for (int i = tid; i < C * DVT; i += blockDim.x) {
            const int t = i / DVT, b = i % DVT;
            Vs[t * vp + b] = t < n ? to_f32(v[((size_t)(c0 + t) * H + h) * DV + v0 + b]) : 0.f;
        }
        if (tid < 32) {
            // 2. in-chunk cumulative log decay by a warp scan (C <= 64: two values per lane)
            float carry = 0.f;
            for (int base = 0; base < C; base += 32) {
                const int t = base + tid;
                float x = (t < n) ? log_alpha[(size_t)(c0 + t) * H + h] : 0.f;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y_ = __shfl_up_sync(0xffffffffu, x, off);
                    if (tid >= off) x += y_;
                }
                x += carry;
                carry = __shfl_sync(0xffffffffu, x, 31);
                if (t < C) {
                    g[t] = x;
                    gam[t] = expf(x);
                    bet[t] = (t < n) ? beta[(size_t)(c0 + t) * H + h] : 0.f;
                }
            }
        }
        __syncthreads();
        // 3. L (strictly lower, with beta_t and the decay) and P (lower, diagonal kept)
        for (int i = tid; i < C * C; i += blockDim.x) {
            const int t = i / C, s = i % C;
            float lk = 0.f, pq = 0.f;
            if (s <= t) {
                float dk_ = 0.f, dq = 0.f;
                for (int a = 0; a < DK; ++a) {
                    dk_ = fmaf(Ks[t * kp + a], Ks[s * kp + a], dk_);
                    dq = fmaf(Qs[t * kp + a], Ks[s * kp + a], dq);
                }
                const float decay = expf(g[t] - g[s]);
                pq = dq * decay;
                lk = (s < t) ? bet[t] * dk_ * decay : 0.f;
            }
            Ls[t * cp + s] = lk;
            Ps[t * cp + s] = pq;
        }
        __syncthreads();
        // 4. T = (I + L)^-1 by forward substitution, one column per thread
        if (tid < C) {
            const int j = tid;
            for (int t = 0; t < C; ++t) {
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
        // 5. W = T diag(beta gamma) K (C x DK) ; U = T diag(beta) V (C x DVT)
        for (int i = tid; i < C * DK; i += blockDim.x) {
            const int t = i / DK, a = i % DK;
            float acc = 0.f;
            for (int s = 0; s <= t; ++s) acc = fmaf(Ts[t * cp + s] * bet[s] * gam[s], Ks[s * kp + a], acc);
            Ws[t * kp + a] = acc;
        }
        for (int i = tid; i < C * DVT; i += blockDim.x) {
            const int t = i / DVT, b = i % DVT;
            float acc = 0.f;
            for (int s = 0; s <= t; ++s) acc = fmaf(Ts[t * cp + s] * bet[s], Vs[s * vp + b], acc);
            Us[t * vp + b] = acc;
        }
        __syncthreads();
        // 6. U~ = U - W S
        for (int i = tid; i < C * DVT; i += blockDim.x) {
            const int t = i / DVT, b = i % DVT;
            float acc = Us[t * vp + b];
            for (int a = 0; a < DK; ++a) acc = fmaf(-Ws[t * kp + a], Ss[a * vp + b], acc);
            Us[t * vp + b] = acc;
        }
        __syncthreads();
        // 7. Y = diag(gamma) Q S + P U~  (rows past the end are not stored)
        for (int i = tid; i < C * DVT; i += blockDim.x) {
            const int t = i / DVT, b = i % DVT;
            if (t >= n) continue;
            float qs = 0.f;
            for (int a = 0; a < DK; ++a) qs = fmaf(Qs[t * kp + a], Ss[a * vp + b], qs);
            float acc = gam[t] * qs;
            for (int s = 0; s <= t; ++s) acc = fmaf(Ps[t * cp + s], Us[s * vp + b], acc);
            y[((size_t)(c0 + t) * H + h) * DV + v0 + b] = from_f32<TY>(acc);
        }
        __syncthreads();
        // 8. S <- gamma_C S + sum_s exp(g_C - g_s) k_s u~_s^T
        const float gC = g[C - 1];
        const float gamC = gam[C - 1];
        for (int i = tid; i < DK * DVT; i += blockDim.x) {
            const int a = i / DVT, b = i % DVT;
            float acc = gamC * Ss[a * vp + b];
            for (int s = 0; s < n; ++s) acc = fmaf(expf(gC - g[s]) * Ks[s * kp + a], Us[s * vp + b], acc);
            Ss[a * vp + b] = acc;
        }
    }
    __syncthreads();
    if (S_T) {
        for (int i = tid; i < DK * DVT; i += blockDim.x) {
            const int a = i % DK, b = i / DK;
            S_T[st_off + (size_t)(v0 + b) * DK + a] = Ss[a * vp + b];
        }
    }
}

}  // namespace gdn
