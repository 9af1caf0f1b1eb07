// gdn_gate_norm.cuh -- fused output epilogue o = sigmoid(z) * RMSNorm(y) * (1 + w).
//
// The output-gate equation of the joezjh.github.io notes page "Qwen3.8-Flash-Next"
// (section "GDN 参数化细节") without its projections, with the zero-centred RMSNorm of
// the pwwt.cn translation (section 2.1.1): the stored weight w multiplies as (1 + w)
// and y is not mean-subtracted. One row per (token, head), over its d_v elements;
// fp32 arithmetic, one read of y and z and one write of o (HBM-bound).
//
// Mapping: each lane owns 32 bytes of y of a row (8 fp32 or 16 bf16 elements; z and o may
// each be fp32 or bf16); LPR lanes cover one row, a warp takes RPW = 32 / LPR rows per pass
// and UNROLL passes at once (their loads all in flight), in a grid-stride loop over rows.
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

// Raw 16-byte words <-> floats: element i of a lane's run, for fp32 or bf16 storage.
__device__ __forceinline__ float raw_elem(const uint4 *w, int i, float)
{
    const uint4 v = w[i >> 2];
    const uint32_t x = (i & 3) == 0 ? v.x : (i & 3) == 1 ? v.y : (i & 3) == 2 ? v.z : v.w;
    return __uint_as_float(x);
}
__device__ __forceinline__ float raw_elem(const uint4 *w, int i, __nv_bfloat16)
{
    const uint4 v = w[i >> 3];
    const int j = (i & 7) >> 1;
    const uint32_t x = j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
    return __uint_as_float((i & 1) ? (x & 0xffff0000u) : (x << 16));
}

// sigmoid(z) with the SM's approximate exponential and division (a few ulp of fp32)
__device__ __forceinline__ float fast_sigmoid(float z) { return __fdividef(1.0f, 1.0f + __expf(-z)); }

// y and o may be the same buffer (TY = TO): a row is written only by the lanes that read it,
// after all of its values are in registers (its sum of squares needs them all).
template <typename TY, typename TZ, typename TO, int DV>
__global__ void __launch_bounds__(kGateNormThreads)
gate_norm_kernel(const TY *y, const TZ *__restrict__ z, const float *__restrict__ w,
                 int64_t n_rows, float eps, TO *o)
{
    // each lane reads 32 bytes of y per row (8 fp32 or 16 bf16 elements), kept as raw words
    // until used, so that UNROLL rows per lane are in flight at a modest register cost
    constexpr int EPL_W = 32 / (int)sizeof(TY);
    constexpr int EPL = DV < EPL_W ? DV : EPL_W;    // elements per lane
    constexpr int LPR = DV / EPL;                   // lanes per row
    static_assert(LPR >= 1 && LPR <= 32, "d_v in 16..256");
    constexpr int RPW = 32 / LPR;                   // rows per warp pass
    constexpr int UNROLL = 4;
    constexpr int NY = EPL * (int)sizeof(TY) / 16, NZ = EPL * (int)sizeof(TZ) / 16;
    static_assert(NY >= 1 && NZ >= 1, "16-byte accesses");

    const int lane = threadIdx.x & 31;
    const int part = lane % LPR, sub = lane / LPR;
    const int64_t warp_global = ((int64_t)blockIdx.x * kGateNormThreads + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * kGateNormThreads) >> 5;

    float wp[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) wp[e] = 1.0f + w[part * EPL + e];

    for (int64_t r0 = warp_global * RPW * UNROLL; r0 < n_rows; r0 += n_warps * RPW * UNROLL) {
        uint4 yr[UNROLL][NY], zr[UNROLL][NZ];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int64_t row = r0 + u * RPW + sub;
            const uint4 *yp = reinterpret_cast<const uint4 *>(y + row * DV + part * EPL);
            const uint4 *zp = reinterpret_cast<const uint4 *>(z + row * DV + part * EPL);
#pragma unroll
            for (int i = 0; i < NY; ++i) yr[u][i] = row < n_rows ? yp[i] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int i = 0; i < NZ; ++i) zr[u][i] = row < n_rows ? zp[i] : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int64_t row = r0 + u * RPW + sub;
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) {
                const float v = raw_elem(yr[u], e, TY());
                ss = fmaf(v, v, ss);
            }
            ss = group_sum<LPR>(ss);
            const float inv_rms = rsqrtf(ss * (1.0f / DV) + eps);
            if (row < n_rows) {
                float ov[EPL];
#pragma unroll
                for (int e = 0; e < EPL; ++e)
                    ov[e] = fast_sigmoid(raw_elem(zr[u], e, TZ())) * (raw_elem(yr[u], e, TY()) * inv_rms) * wp[e];
#pragma unroll
                for (int e = 0; e < EPL; e += 8) store8(o + row * DV + part * EPL + e, ov + e);
            }
        }
    }
}

}  // namespace gdn
