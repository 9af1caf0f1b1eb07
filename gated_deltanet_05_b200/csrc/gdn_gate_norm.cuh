// gdn_gate_norm.cuh -- fused output epilogue o = sigmoid(z) * RMSNorm(y) * (1 + w).
//
// The output-gate equation of the joezjh.github.io notes page "Qwen3.8-Flash-Next"
// (section "GDN 参数化细节") without its projections, with the zero-centred RMSNorm of
// the pwwt.cn translation (section 2.1.1): the stored weight w multiplies as (1 + w)
// and y is not mean-subtracted. One row per (token, head), over its d_v elements;
// fp32 arithmetic, one read of y and z and one write of o (HBM-bound).
//
// Mapping: each lane owns 8 consecutive elements of a row (y, z and o may each be fp32 or
// bf16); LPR = d_v / 8 lanes cover one row, a warp takes RPW = 32 / LPR rows per pass
// and UNROLL passes at once, in a grid-stride loop over rows.
#pragma once
#include "gdn_common.cuh"

namespace gdn {

constexpr int kGateNormThreads = 256;

// 8 consecutive elements <-> 8 floats (two 16-byte accesses for fp32, one for bf16).
__device__ __forceinline__ void load8(const float *p, float *x)
{
    const float4 a = *reinterpret_cast<const float4 *>(p), b = *reinterpret_cast<const float4 *>(p + 4);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float *x)
{
    const uint4 raw = *reinterpret_cast<const uint4 *>(p);
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ void store8(float *p, const float *x)
{
    *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
    *reinterpret_cast<float4 *>(p + 4) = make_float4(x[4], x[5], x[6], x[7]);
}
__device__ __forceinline__ void store8(__nv_bfloat16 *p, const float *x)
{
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t *>(&h);
    }
    *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

template <typename TY, typename TZ, typename TO, int DV>
__global__ void __launch_bounds__(kGateNormThreads)
gate_norm_kernel(const TY *__restrict__ y, const TZ *__restrict__ z, const float *__restrict__ w,
                 int64_t n_rows, float eps, TO *__restrict__ o)
{
    constexpr int LPR = DV / 8;                     // lanes per row, 8 elements each
    static_assert(LPR >= 1 && LPR <= 32, "d_v in 8..256");
    constexpr int RPW = 32 / LPR;                   // rows per warp pass
    constexpr int UNROLL = 2;

    const int lane = threadIdx.x & 31;
    const int part = lane % LPR, sub = lane / LPR;
    const int64_t warp_global = ((int64_t)blockIdx.x * kGateNormThreads + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * kGateNormThreads) >> 5;

    float wp[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) wp[e] = 1.0f + w[part * 8 + e];

    for (int64_t r0 = warp_global * RPW * UNROLL; r0 < n_rows; r0 += n_warps * RPW * UNROLL) {
        float yv[UNROLL][8], zv[UNROLL][8];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int64_t row = r0 + u * RPW + sub;
            if (row < n_rows) {
                load8(y + row * DV + part * 8, yv[u]);
                load8(z + row * DV + part * 8, zv[u]);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) yv[u][e] = zv[u][e] = 0.f;
            }
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int64_t row = r0 + u * RPW + sub;
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) ss = fmaf(yv[u][e], yv[u][e], ss);
            ss = group_sum<LPR>(ss);
            const float inv_rms = rsqrtf(ss * (1.0f / DV) + eps);
            if (row < n_rows) {
                float ov[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float gate = 1.0f / (1.0f + expf(-zv[u][e]));
                    ov[e] = gate * (yv[u][e] * inv_rms) * wp[e];
                }
                store8(o + row * DV + part * 8, ov);
            }
        }
    }
}

}  // namespace gdn
