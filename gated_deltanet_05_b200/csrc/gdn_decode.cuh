// gdn_decode.cuh -- single-token decode step of the gated delta rule, one pass over S.
//
// Follows the four-line update rule of the joezjh.github.io notes page
// "Qwen3.8-Flash-Next" (section "Gated DeltaNet 核心机制") for one token per chain.
// The state is stored value-major (row j of S^T holds column j of the pages' S, the
// key dimension contiguous), so every quantity the update needs is a dot product
// along a row:  u_j = S[:,j].k,  r_j = S[:,j].q  (old state). Then
//     e_j = v_j - alpha u_j
//     y_j = scale (alpha r_j + beta (k.q) e_j)        (= S_new[:,j] . (scale q))
//     S[:,j] <- alpha S[:,j] + beta e_j k
// Each row is read once and written once: the kernel is HBM-bound at
// 2 * d_k * d_v * 4 bytes of state traffic per chain per step.
//
// Mapping: LPR = d_k / 4 lanes share one row (one float4 per lane); a warp covers
// 32 / LPR rows per pass and issues ROWS_IN_FLIGHT passes of loads before it reduces,
// so several 512-byte rows per warp are in flight. One CTA of 8 warps owns a chain.
#pragma once
#include "gdn_common.cuh"

namespace gdn {

constexpr int kDecodeThreads = 256;

template <int DK, typename T>
__global__ void __launch_bounds__(kDecodeThreads)
decode_step_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                   const float *__restrict__ alpha, const float *__restrict__ beta,
                   float *__restrict__ S, int dv, float scale, T *__restrict__ y)
{
    constexpr int LPR = DK / 4;              // lanes per row
    constexpr int RPW = 32 / LPR;            // rows per warp pass
    constexpr int WARPS = kDecodeThreads / 32;
    constexpr int ROWS_IN_FLIGHT = 4;        // passes whose loads are issued together

    const int chain = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int part = lane % LPR;             // which float4 of the row
    const int sub = lane / LPR;              // which row of the warp pass

    const float4 kv = load4(k + (size_t)chain * DK + 4 * part);
    float4 qv = load4(q + (size_t)chain * DK + 4 * part);
    qv.x *= scale; qv.y *= scale; qv.z *= scale; qv.w *= scale;
    const float a = alpha[chain], b = beta[chain];
    const float kq = group_sum<LPR>(kv.x * qv.x + kv.y * qv.y + kv.z * qv.z + kv.w * qv.w);

    float *Sc = S + (size_t)chain * dv * DK;
    const T *vc = v + (size_t)chain * dv;
    T *yc = y + (size_t)chain * dv;

    const int rows_per_round = WARPS * RPW * ROWS_IN_FLIGHT;
    for (int base = 0; base < dv; base += rows_per_round) {
        float4 s[ROWS_IN_FLIGHT];
        float vj[ROWS_IN_FLIGHT];
        int row[ROWS_IN_FLIGHT];
#pragma unroll
        for (int i = 0; i < ROWS_IN_FLIGHT; ++i) {
            row[i] = base + (i * WARPS + warp) * RPW + sub;
            if (row[i] < dv) {
                s[i] = load4(Sc + (size_t)row[i] * DK + 4 * part);
                vj[i] = to_f32(vc[row[i]]);
            } else {
                s[i] = make_float4(0.f, 0.f, 0.f, 0.f);
                vj[i] = 0.f;
            }
        }
#pragma unroll
        for (int i = 0; i < ROWS_IN_FLIGHT; ++i) {
            const float u = group_sum<LPR>(s[i].x * kv.x + s[i].y * kv.y + s[i].z * kv.z +
                                           s[i].w * kv.w);
            const float r = group_sum<LPR>(s[i].x * qv.x + s[i].y * qv.y + s[i].z * qv.z +
                                           s[i].w * qv.w);
            const float e = vj[i] - a * u;
            const float be = b * e;
            if (row[i] < dv) {
                float4 sn;
                sn.x = fmaf(a, s[i].x, be * kv.x);
                sn.y = fmaf(a, s[i].y, be * kv.y);
                sn.z = fmaf(a, s[i].z, be * kv.z);
                sn.w = fmaf(a, s[i].w, be * kv.w);
                store4(Sc + (size_t)row[i] * DK + 4 * part, sn);
                if (part == 0)
                    yc[row[i]] = from_f32<T>(fmaf(a, r, be * kq));
            }
        }
    }
}

}  // namespace gdn
