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

template <int DK, typename T, typename TY>
__global__ void __launch_bounds__(kDecodeThreads)
decode_step_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                   const float *__restrict__ alpha, const float *__restrict__ beta,
                   float *__restrict__ S, int dv, float scale, TY *__restrict__ y)
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
    TY *yc = y + (size_t)chain * dv;

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
                    yc[row[i]] = from_f32<TY>(fmaf(a, r, be * kq));
            }
        }
    }
}

}  // namespace gdn

namespace gdn {

// ---------------------------------------------------------------- several tokens per call
//
// n (<= kDecodeMaxTokens) consecutive tokens of every chain in one pass over S: the same
// update as decode_step_kernel, applied token after token to each row while the row stays
// in registers, so the state is read and written once per call instead of once per
// token. (d_k = d_v = 128 uses decode_tokens_pipe_kernel below; this one serves the
// other sizes.) A lane holds 16 consecutive elements of a row (LPR = d_k / 16 lanes per row), so
// each of the two dot products per row and token costs log2(LPR) shuffles. The tokens'
// k, scale q, v, alpha, beta and k.(scale q) are staged in shared memory first.
constexpr int kDecodeMaxTokens = 8;
constexpr int kDecodeTokThreads = 256;

template <int DK, typename T, typename TY>
__global__ void __launch_bounds__(kDecodeTokThreads)
decode_tokens_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                     const float *__restrict__ alpha, const float *__restrict__ beta,
                     float *__restrict__ S, int n, int H, int dv, float scale, TY *__restrict__ y)
{
    constexpr int LPR = DK / 16;             // lanes per row, 16 elements each
    constexpr int RPW = 32 / LPR;            // rows per warp pass
    constexpr int WARPS = kDecodeTokThreads / 32;
    constexpr int ROWS_IN_FLIGHT = 4;        // 128 rows of d_k = 128 in one round
    __shared__ float4 sk[kDecodeMaxTokens][DK / 4], sq[kDecodeMaxTokens][DK / 4];
    __shared__ float sv[kDecodeMaxTokens][128];
    __shared__ float sa[kDecodeMaxTokens], sb[kDecodeMaxTokens], skq[kDecodeMaxTokens];

    const int chain = blockIdx.x;            // seq * H + head
    const int seq = chain / H, head = chain % H;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // token i of this chain sits at row (seq * n + i) * H + head of the [n_seq * n, H, .] inputs
    auto tok_row = [&](int i) -> size_t { return ((size_t)seq * n + i) * H + head; };

    for (int e = threadIdx.x; e < n * (DK / 4); e += kDecodeTokThreads) {
        const int i = e / (DK / 4), c4 = e % (DK / 4);
        sk[i][c4] = load4(k + tok_row(i) * DK + 4 * c4);
        float4 qq = load4(q + tok_row(i) * DK + 4 * c4);
        qq.x *= scale; qq.y *= scale; qq.z *= scale; qq.w *= scale;
        sq[i][c4] = qq;
    }
    for (int e = threadIdx.x; e < n * dv; e += kDecodeTokThreads) {
        const int i = e / dv, j = e % dv;
        sv[i][j] = to_f32(v[tok_row(i) * dv + j]);
    }
    if (threadIdx.x < n) {
        sa[threadIdx.x] = alpha[tok_row(threadIdx.x)];
        sb[threadIdx.x] = beta[tok_row(threadIdx.x)];
    }
    __syncthreads();
    if (warp < n) {                           // k_i . (scale q_i), one warp per token
        float acc = 0.f;
        for (int c4 = lane; c4 < DK / 4; c4 += 32) {
            const float4 a = sk[warp][c4], b = sq[warp][c4];
            acc += a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
        }
        acc = group_sum<32>(acc);
        if (lane == 0) skq[warp] = acc;
    }
    __syncthreads();

    const int part = lane % LPR, sub = lane / LPR;
    float *Sc = S + (size_t)chain * dv * DK;
    const int rows_per_round = WARPS * RPW * ROWS_IN_FLIGHT;
    for (int base = 0; base < dv; base += rows_per_round) {
        float s[ROWS_IN_FLIGHT][16];
        int row[ROWS_IN_FLIGHT];
#pragma unroll
        for (int f = 0; f < ROWS_IN_FLIGHT; ++f) {
            row[f] = base + (f * WARPS + warp) * RPW + sub;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float4 x = row[f] < dv ? load4(Sc + (size_t)row[f] * DK + 16 * part + 4 * c)
                                             : make_float4(0.f, 0.f, 0.f, 0.f);
                s[f][4 * c] = x.x; s[f][4 * c + 1] = x.y; s[f][4 * c + 2] = x.z; s[f][4 * c + 3] = x.w;
            }
        }
#pragma unroll 1
        for (int i = 0; i < n; ++i) {
            float kv[16], qv[16];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float4 a = sk[i][4 * part + c], b = sq[i][4 * part + c];
                kv[4 * c] = a.x; kv[4 * c + 1] = a.y; kv[4 * c + 2] = a.z; kv[4 * c + 3] = a.w;
                qv[4 * c] = b.x; qv[4 * c + 1] = b.y; qv[4 * c + 2] = b.z; qv[4 * c + 3] = b.w;
            }
            const float a = sa[i], b = sb[i], kq = skq[i];
#pragma unroll
            for (int f = 0; f < ROWS_IN_FLIGHT; ++f) {
                float u = 0.f, r = 0.f;
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    u = fmaf(s[f][e], kv[e], u);
                    r = fmaf(s[f][e], qv[e], r);
                }
                u = group_sum<LPR>(u);
                r = group_sum<LPR>(r);
                const bool valid = row[f] < dv;
                const float ev = (valid ? sv[i][row[f]] : 0.f) - a * u;
                const float be = b * ev;
#pragma unroll
                for (int e = 0; e < 16; ++e) s[f][e] = fmaf(a, s[f][e], be * kv[e]);
                if (valid && part == 0) y[tok_row(i) * dv + row[f]] = from_f32<TY>(fmaf(a, r, be * kq));
            }
        }
#pragma unroll
        for (int f = 0; f < ROWS_IN_FLIGHT; ++f)
            if (row[f] < dv)
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    store4(Sc + (size_t)row[f] * DK + 16 * part + 4 * c,
                           make_float4(s[f][4 * c], s[f][4 * c + 1], s[f][4 * c + 2], s[f][4 * c + 3]));
    }
}

}  // namespace gdn

namespace gdn {

// ------------------------------------------------- several tokens per call, pipelined (d = 128)
//
// The same update as decode_tokens_kernel for d_k = d_v = 128, with the memory traffic of one
// chain overlapped with the arithmetic of the previous one. A CTA walks the chains
// blockIdx.x, blockIdx.x + gridDim.x, ...; each chain's state arrives in two halves of 64 rows
// by cp.async into two shared-memory stages, its tokens (k, q, v, alpha, beta, raw) with the
// first half into one of two token buffers. While half h of chain c is computed, half 1 - h
// (or half 0 of the next chain) is in flight. A lane's 16 elements of a row are the float4
// chunks at columns 32 j + 4 p (j = 0..3, p = lane % 8), so the 8 lanes of a row read 128
// contiguous bytes; each lane copies exactly the state it later reads. The updated rows go
// straight from registers to global memory.
constexpr int kDecPipeThreads = 256;
constexpr int kDecPipeHalf = 64;


template <typename T>
__host__ __device__ constexpr size_t decode_pipe_smem_bytes()
{
    return 2 * (size_t)kDecPipeHalf * 128 * sizeof(float) + 2 * 3 * (size_t)kDecodeMaxTokens * 128 * sizeof(T) +
           2 * 2 * (size_t)kDecodeMaxTokens * sizeof(float);
}

template <typename T, typename TY>
__global__ void __launch_bounds__(kDecPipeThreads, 2)
decode_tokens_pipe_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                          const float *__restrict__ alpha, const float *__restrict__ beta, float *__restrict__ S,
                          int n, int H, int n_chain, float scale, TY *__restrict__ y)
{
    constexpr int DK = 128, DV = 128, LPR = 8, RPW = 4, WARPS = kDecPipeThreads / 32, HALF = kDecPipeHalf;
    constexpr int TOK = kDecodeMaxTokens, EPC = 16 / (int)sizeof(T);   // elements per 16-byte chunk
    static_assert(2 * WARPS * RPW == HALF, "two passes of the warps cover a half");
    extern __shared__ __align__(16) unsigned char dec_sm[];
    float *stage = reinterpret_cast<float *>(dec_sm);                     // [2][HALF][DK]
    T *tk = reinterpret_cast<T *>(stage + 2 * HALF * DK);                 // [2][TOK][DK]
    T *tq = tk + 2 * TOK * DK;                                            // [2][TOK][DK]
    T *tv = tq + 2 * TOK * DK;                                            // [2][TOK][DV]
    float *tab = reinterpret_cast<float *>(tv + 2 * TOK * DV);            // [2][alpha, beta][TOK]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int p = lane % LPR, sub = lane / LPR;
    auto row_of = [&](int f) { return (f * WARPS + warp) * RPW + sub; };  // row within a half
    auto tok_row = [&](int chain, int i) -> size_t { return ((size_t)(chain / H) * n + i) * H + chain % H; };

    // one commit group: half h of `chain`'s state, with h == 0 also its tokens into buffer tb
    // (an empty group past the last chain keeps the group count uniform)
    auto issue = [&](int chain, int h, int tb) {
        if (chain < n_chain) {
            const float *src = S + ((size_t)chain * DV + (size_t)h * HALF) * DK;
            float *dst = stage + h * HALF * DK;
#pragma unroll
            for (int f = 0; f < 2; ++f) {
                const int r = row_of(f);
#pragma unroll
                for (int j = 0; j < 4; ++j) cp_async16(dst + r * DK + 32 * j + 4 * p, src + (size_t)r * DK + 32 * j + 4 * p);
            }
            if (h == 0) {
                constexpr int CK = DK / EPC, CV = DV / EPC;              // 16-byte chunks per row
                for (int e = tid; e < n * (2 * CK + CV); e += blockDim.x) {
                    const int i = e / (2 * CK + CV), w = e % (2 * CK + CV);
                    const size_t tr = tok_row(chain, i);
                    if (w < CK)
                        cp_async16(tk + (tb * TOK + i) * DK + w * EPC, k + tr * DK + w * EPC);
                    else if (w < 2 * CK)
                        cp_async16(tq + (tb * TOK + i) * DK + (w - CK) * EPC, q + tr * DK + (w - CK) * EPC);
                    else
                        cp_async16(tv + (tb * TOK + i) * DV + (w - 2 * CK) * EPC, v + tr * DV + (w - 2 * CK) * EPC);
                }
                if (tid < 2 * n) {
                    const int i = tid % n, which = tid / n;
                    cp_async4(tab + (tb * 2 + which) * TOK + i, (which == 0 ? alpha : beta) + tok_row(chain, i));
                }
            }
        }
        cp_async_commit();
    };

    int it = 0;
    issue(blockIdx.x, 0, 0);
    issue(blockIdx.x, 1, 0);
    for (int c = blockIdx.x; c < n_chain; c += gridDim.x, ++it) {
        const int tb = it & 1;
        float *Sc = S + (size_t)c * DV * DK;
        for (int h = 0; h < 2; ++h) {
            cp_async_wait1();               // this half (and its tokens) has landed, for this thread
            __syncthreads();                // ... and for every thread
            const float *src = stage + h * HALF * DK;
            float s[2][16];
#pragma unroll
            for (int f = 0; f < 2; ++f)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float4 x = *reinterpret_cast<const float4 *>(src + row_of(f) * DK + 32 * j + 4 * p);
                    s[f][4 * j] = x.x; s[f][4 * j + 1] = x.y; s[f][4 * j + 2] = x.z; s[f][4 * j + 3] = x.w;
                }
#pragma unroll 1
            for (int i = 0; i < n; ++i) {
                float kv[16], qv[16];
                float kq = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float4 a4 = load4(tk + (tb * TOK + i) * DK + 32 * j + 4 * p);
                    const float4 b4 = load4(tq + (tb * TOK + i) * DK + 32 * j + 4 * p);
                    kv[4 * j] = a4.x; kv[4 * j + 1] = a4.y; kv[4 * j + 2] = a4.z; kv[4 * j + 3] = a4.w;
                    qv[4 * j] = scale * b4.x; qv[4 * j + 1] = scale * b4.y;
                    qv[4 * j + 2] = scale * b4.z; qv[4 * j + 3] = scale * b4.w;
                }
#pragma unroll
                for (int e = 0; e < 16; ++e) kq = fmaf(kv[e], qv[e], kq);
                kq = group_sum<LPR>(kq);
                const float a = tab[(tb * 2) * TOK + i], b = tab[(tb * 2 + 1) * TOK + i];
                const size_t tr = tok_row(c, i);
#pragma unroll
                for (int f = 0; f < 2; ++f) {
                    float u = 0.f, r = 0.f;
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        u = fmaf(s[f][e], kv[e], u);
                        r = fmaf(s[f][e], qv[e], r);
                    }
                    u = group_sum<LPR>(u);
                    r = group_sum<LPR>(r);
                    const int row = h * HALF + row_of(f);
                    const float ev = to_f32(tv[(tb * TOK + i) * DV + row]) - a * u;
                    const float be = b * ev;
#pragma unroll
                    for (int e = 0; e < 16; ++e) s[f][e] = fmaf(a, s[f][e], be * kv[e]);
                    if (p == 0) y[tr * DV + row] = from_f32<TY>(fmaf(a, r, be * kq));
                }
            }
#pragma unroll
            for (int f = 0; f < 2; ++f) {
                const int row = h * HALF + row_of(f);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    store4(Sc + (size_t)row * DK + 32 * j + 4 * p,
                           make_float4(s[f][4 * j], s[f][4 * j + 1], s[f][4 * j + 2], s[f][4 * j + 3]));
            }
            __syncthreads();                // every thread is done with this stage (and, at h = 1,
                                            // with this chain's tokens)
            issue(c + gridDim.x, h, tb ^ 1);
        }
    }
    cp_async_wait_all();
}

}  // namespace gdn
