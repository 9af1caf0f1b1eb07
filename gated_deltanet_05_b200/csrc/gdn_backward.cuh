// gdn_backward.cuh -- gradients of the gated delta rule, token by token, on CUDA cores.
//
// The reverse-mode adjoint of the four-line update of the joezjh.github.io notes page
// "Qwen3.8-Flash-Next" (section "Gated DeltaNet 核心机制"), for the loss
// L = sum_t <dy_t, y_t> + <dS_T, S_T>. In the library's value-major layout (row b of S^T is
// column b of the pages' S), with G = dL/dS carried backwards from dS_T:
//     y_t = S_t^T (scale q_t):      dq_t = scale S_t dy_t;        G += scale q_t dy_t^T
//     e_t = v_t - alpha_t S_{t-1}^T k_t
//     S_t = alpha_t S_{t-1} + beta_t k_t e_t^T:
//         dbeta_t = k_t^T G e_t;  dk_t = beta_t G e_t;  de_t = beta_t G^T k_t;  dv_t = de_t
//         G~ = G - k_t de_t^T;    dk_t -= alpha_t S_{t-1} de_t
//         dlog_alpha_t = alpha_t <G~, S_{t-1}>;   G <- alpha_t G~
// dS0 = G after the first token. The states S_{t-1}, S_t come from a forward pass that
// keeps a copy every kBwdSeg tokens and, per segment from the last, recomputes the
// segment's states into the workspace.
//
// One CTA per (sequence, head) chain; S and G live in shared memory (rows padded by one
// float so that column walks do not conflict). fp32 throughout; a correctness-first
// kernel, not a throughput one.
#pragma once
#include "gdn_common.cuh"

namespace gdn {

constexpr int kBwdThreads = 256;
constexpr int kBwdSeg = 64;

// Workspace floats per chain: checkpoints (max_len / kBwdSeg + 1) and one segment of
// kBwdSeg + 1 states, each dk * dv.
__host__ __device__ inline size_t bwd_ws_floats_per_chain(int64_t max_len, int dk, int dv)
{
    return (size_t)(max_len / kBwdSeg + 1 + kBwdSeg + 1) * (size_t)dk * dv;
}

__device__ __forceinline__ float block_sum_bwd(float x, float *red)
{
    x = group_sum<32>(x);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();                        // red is free (previous use finished)
    if (lane == 0) red[warp] = x;
    __syncthreads();
    float t = 0.f;
    for (int w = 0; w < kBwdThreads / 32; ++w) t += red[w];
    return t;
}

template <typename T>
__global__ void __launch_bounds__(kBwdThreads)
gdn_backward_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                    const float *__restrict__ log_alpha, const float *__restrict__ beta,
                    const float *__restrict__ S0, const int32_t *__restrict__ cu_seqlens, int H,
                    int DK, int DV, float scale, const T *__restrict__ dy, const float *__restrict__ dS_T,
                    float *__restrict__ dq, float *__restrict__ dk_out, float *__restrict__ dv_out,
                    float *__restrict__ dlog_alpha, float *__restrict__ dbeta, float *__restrict__ dS0,
                    float *__restrict__ ws, int64_t max_len)
{
    extern __shared__ float bsm[];
    const int P = DK + 1;                   // padded row stride of S and G in shared memory
    float *SL = bsm;                        // [DV][P]
    float *GL = SL + (size_t)DV * P;        // [DV][P]
    float *kv = GL + (size_t)DV * P;        // k_t [DK]
    float *qv = kv + DK;                    // q_t [DK]
    float *vv = qv + DK;                    // v_t [DV]
    float *dyv = vv + DV;                   // dy_t [DV]
    float *ev = dyv + DV;                   // e_t [DV]
    float *dev_ = ev + DV;                  // de_t [DV]
    float *red = dev_ + DV;                 // [kBwdThreads / 32]

    const int chain = blockIdx.x, seq = chain / H, head = chain % H;
    const int tid = threadIdx.x;
    const int64_t bos = cu_seqlens[seq], len = (int64_t)cu_seqlens[seq + 1] - bos;
    const size_t SZ = (size_t)DK * DV;
    float *ck = ws + (size_t)chain * bwd_ws_floats_per_chain(max_len, DK, DV);
    float *segb = ck + (size_t)(max_len / kBwdSeg + 1) * SZ;
    const size_t soff = (size_t)chain * SZ;
    auto row = [&](int64_t t) -> size_t { return (size_t)(bos + t) * H + head; };

    // S (shared, padded) <-> a dense [DV][DK] state in global memory
    auto load_state = [&](float *dst, const float *src) {
        for (int i = tid; i < (int)SZ; i += kBwdThreads) dst[(i / DK) * P + i % DK] = src ? src[i] : 0.f;
    };
    auto store_state = [&](float *dst, const float *src) {
        for (int i = tid; i < (int)SZ; i += kBwdThreads) dst[i] = src[(i / DK) * P + i % DK];
    };
    auto load_kv = [&](int64_t t) {
        const size_t r = row(t);
        for (int a = tid; a < DK; a += kBwdThreads) kv[a] = to_f32(k[r * DK + a]);
        for (int b = tid; b < DV; b += kBwdThreads) vv[b] = to_f32(v[r * DV + b]);
    };
    // one forward token on SL (k_t, v_t already in shared memory)
    auto forward_token = [&](float alpha, float bt) {
        for (int i = tid; i < (int)SZ; i += kBwdThreads) SL[(i / DK) * P + i % DK] *= alpha;
        __syncthreads();
        for (int b = tid; b < DV; b += kBwdThreads) {
            float acc = 0.f;
            for (int a = 0; a < DK; ++a) acc = fmaf(SL[b * P + a], kv[a], acc);
            ev[b] = vv[b] - acc;
        }
        __syncthreads();
        for (int i = tid; i < (int)SZ; i += kBwdThreads) {
            const int b = i / DK, a = i % DK;
            SL[b * P + a] = fmaf(bt * ev[b], kv[a], SL[b * P + a]);
        }
        __syncthreads();
    };

    // ---- forward: a copy of the state every kBwdSeg tokens
    load_state(SL, S0 ? S0 + soff : nullptr);
    __syncthreads();
    store_state(ck, SL);
    for (int64_t t = 0; t < len; ++t) {
        load_kv(t);
        __syncthreads();
        forward_token(expf(log_alpha[row(t)]), beta[row(t)]);
        if ((t + 1) % kBwdSeg == 0) store_state(ck + (size_t)((t + 1) / kBwdSeg) * SZ, SL);
    }

    // ---- backward, one segment at a time from the last
    load_state(GL, dS_T ? dS_T + soff : nullptr);
    __syncthreads();
    for (int64_t s0 = len > 0 ? (len - 1) / kBwdSeg * kBwdSeg : -1; s0 >= 0; s0 -= kBwdSeg) {
        const int64_t s1 = s0 + kBwdSeg < len ? s0 + kBwdSeg : len;
        __syncthreads();
        load_state(SL, ck + (size_t)(s0 / kBwdSeg) * SZ);
        __syncthreads();
        store_state(segb, SL);
        for (int64_t t = s0; t < s1; ++t) {
            load_kv(t);
            __syncthreads();
            forward_token(expf(log_alpha[row(t)]), beta[row(t)]);
            store_state(segb + (size_t)(t - s0 + 1) * SZ, SL);
        }
        __threadfence_block();
        __syncthreads();
        for (int64_t t = s1 - 1; t >= s0; --t) {
            const size_t r = row(t);
            const float *St = segb + (size_t)(t - s0 + 1) * SZ;   // [DV][DK] dense
            const float *Sp = segb + (size_t)(t - s0) * SZ;
            const float alpha = expf(log_alpha[r]), bt = beta[r];
            for (int a = tid; a < DK; a += kBwdThreads) {
                kv[a] = to_f32(k[r * DK + a]);
                qv[a] = to_f32(q[r * DK + a]);
            }
            for (int b = tid; b < DV; b += kBwdThreads) {
                vv[b] = to_f32(v[r * DV + b]);
                dyv[b] = to_f32(dy[r * DV + b]);
            }
            __syncthreads();
            // dq = scale S_t dy;  e = v - alpha S_{t-1}^T k
            for (int a = tid; a < DK; a += kBwdThreads) {
                float acc = 0.f;
                for (int b = 0; b < DV; ++b) acc = fmaf(St[(size_t)b * DK + a], dyv[b], acc);
                dq[r * DK + a] = scale * acc;
            }
            for (int b = tid; b < DV; b += kBwdThreads) {
                float acc = 0.f;
                for (int a = 0; a < DK; ++a) acc = fmaf(alpha * Sp[(size_t)b * DK + a], kv[a], acc);
                ev[b] = vv[b] - acc;
            }
            // G += scale q dy^T
            for (int i = tid; i < (int)SZ; i += kBwdThreads) {
                const int b = i / DK, a = i % DK;
                GL[b * P + a] = fmaf(scale * qv[a], dyv[b], GL[b * P + a]);
            }
            __syncthreads();
            // de = beta G^T k (per value row);  (G e)_a per key column
            for (int b = tid; b < DV; b += kBwdThreads) {
                float acc = 0.f;
                for (int a = 0; a < DK; ++a) acc = fmaf(GL[b * P + a], kv[a], acc);
                dev_[b] = bt * acc;
                dv_out[r * DV + b] = bt * acc;
            }
            float ge = 0.f;                  // (G e)_a of this thread's column (tid < DK)
            if (tid < DK)
                for (int b = 0; b < DV; ++b) ge = fmaf(GL[b * P + tid], ev[b], ge);
            const float db = block_sum_bwd(tid < DK ? kv[tid] * ge : 0.f, red);
            if (tid == 0) dbeta[r] = db;
            // G~ = G - k de^T   (block_sum_bwd's barriers ordered the de writes before this)
            for (int i = tid; i < (int)SZ; i += kBwdThreads) {
                const int b = i / DK, a = i % DK;
                GL[b * P + a] = fmaf(-kv[a], dev_[b], GL[b * P + a]);
            }
            // dk = beta (G e) - alpha S_{t-1} de
            if (tid < DK) {
                float sd = 0.f;
                for (int b = 0; b < DV; ++b) sd = fmaf(alpha * Sp[(size_t)b * DK + tid], dev_[b], sd);
                dk_out[r * DK + tid] = bt * ge - sd;
            }
            __syncthreads();
            // dlog_alpha = alpha <G~, S_{t-1}>;  G = alpha G~
            float part = 0.f;
            for (int i = tid; i < (int)SZ; i += kBwdThreads) {
                const int b = i / DK, a = i % DK;
                part = fmaf(GL[b * P + a], Sp[i], part);
                GL[b * P + a] *= alpha;
            }
            const float dal = block_sum_bwd(part, red);
            if (tid == 0) dlog_alpha[r] = alpha * dal;
            __syncthreads();
        }
    }
    __syncthreads();
    if (dS0) store_state(dS0 + soff, GL);
}

}  // namespace gdn
