// gdn_featurize.cuh -- the feature and gate step in front of the recurrence.
//
// The q/k/v equations of the joezjh.github.io notes page "Qwen3.8-Flash-Next" (section
// "GDN 参数化细节") and its gate equations, with the projections W x taken as inputs:
//   f_t = SiLU(sum_j w[ch][j] x_{t-(W-1)+j})   short causal convolution per channel, no
//                                             token of an earlier sequence in the window
//   q_t, k_t = f_t / sqrt(|f_t|^2 + eps)      per (token, head) over d (pwwt.cn
//                                             translation, section 2.1.1: q and k only)
//   v_t = f_t
//   beta_t = sigmoid(logit),  log alpha_t = -exp(A_h) softplus(logit + b_alpha_h)
// fp32 arithmetic; one read of every input row and one write of every output row
// (HBM-bound: 2 x 2 d bytes per row for bf16, plus 16 bytes of gates per token-head).
//
// Mapping: a lane owns 4 consecutive channels of a row, LPR = D / 4 lanes cover a row and
// a warp takes RPW = 32 / LPR heads of one stream over a run of kFeatRun consecutive
// tokens. The convolution window (the previous W - 1 <= 3 rows) stays in registers as the
// warp walks its run. Rows are loaded kFeatBatch at a time, as raw words (bf16 stays
// packed until it is used), and the next batch is in flight while the current one is
// computed. Warps of the gate task handle the [n_tok][H] gate arrays of one run, which are
// contiguous.
#pragma once
#include "gdn_common.cuh"

namespace gdn {

constexpr int kFeatThreads = 128;
constexpr int kFeatRun = 32;      // tokens per warp task
constexpr int kFeatBatch = 2;     // rows loaded ahead
constexpr int kFeatMaxWidth = 4;  // convolution taps

// SiLU with the fast exponential and division intrinsics (relative error ~1e-6, well inside
// the step's 1e-4 bar); for x below about -87 the denominator is +inf and the result -0.
__device__ __forceinline__ float silu_f32(float x) { return __fdividef(x, 1.0f + __expf(-x)); }
__device__ __forceinline__ float softplus_f32(float x)
{
    return x > 0.f ? x + log1pf(expf(-x)) : log1pf(expf(x));
}

// Eight consecutive elements as loaded: two float4 (fp32) or four packed bf16 pairs.
struct F8 { float4 a, b; };
template <typename T> struct RawRow;
template <> struct RawRow<float> { using type = F8; };
template <> struct RawRow<__nv_bfloat16> { using type = uint4; };
__device__ __forceinline__ void raw_to_f32(const F8 &r, float (&x)[8])
{
    x[0] = r.a.x; x[1] = r.a.y; x[2] = r.a.z; x[3] = r.a.w;
    x[4] = r.b.x; x[5] = r.b.y; x[6] = r.b.z; x[7] = r.b.w;
}
__device__ __forceinline__ void raw_to_f32(const uint4 &r, float (&x)[8])
{
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ void store8f(float *p, const float (&x)[8])
{
    *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
    *reinterpret_cast<float4 *>(p + 4) = make_float4(x[4], x[5], x[6], x[7]);
}
__device__ __forceinline__ void store8f(__nv_bfloat16 *p, const float (&x)[8])
{
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t *>(&h);
    }
    *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

// One launch covers n_streams streams of width D (q and k with L2 = true; v with
// L2 = false) and, when beta_logit is given, the gates.
template <typename T, int D, bool L2>
__global__ void __launch_bounds__(kFeatThreads, 4)
featurize_kernel(const T *__restrict__ x0, const T *__restrict__ x1, const float *__restrict__ w0,
                 const float *__restrict__ w1, T *__restrict__ o0, T *__restrict__ o1, int n_streams,
                 int W, const int32_t *__restrict__ cu, int n_seq, int64_t n_tok, int H, float eps,
                 const float *__restrict__ beta_logit, const float *__restrict__ alpha_logit,
                 const float *__restrict__ A, const float *__restrict__ b_alpha, float *__restrict__ beta,
                 float *__restrict__ log_alpha)
{
    constexpr int CPL = 8;                  // channels per lane
    constexpr int LPR = D / CPL;
    static_assert(LPR >= 2 && LPR <= 16, "D in 16..128");
    constexpr int RPW = 32 / LPR;
    const int lane = threadIdx.x & 31;
    const int64_t task = ((int64_t)blockIdx.x * kFeatThreads + threadIdx.x) >> 5;
    const int64_t n_runs = (n_tok + kFeatRun - 1) / kFeatRun;
    const int n_hg = (H + RPW - 1) / RPW;
    const int64_t stream_tasks = (int64_t)n_streams * n_runs * n_hg;

    if (task >= stream_tasks) {
        // ---- gates of one run: [t0 H, t_end H) is contiguous
        const int64_t run = task - stream_tasks;
        if (!beta_logit || run >= n_runs) return;
        const int64_t t0 = run * kFeatRun;
        const int64_t t_end = t0 + kFeatRun < n_tok ? t0 + kFeatRun : n_tok;
        int h = (int)((t0 * H + lane) % H);
        for (int64_t e = t0 * H + lane; e < t_end * H; e += 32, h = (h + 32) % H) {
            beta[e] = 1.0f / (1.0f + expf(-beta_logit[e]));
            log_alpha[e] = -expf(A[h]) * softplus_f32(alpha_logit[e] + b_alpha[h]);
        }
        return;
    }

    const int s = (int)(task / (n_runs * n_hg));
    const int64_t rem = task % (n_runs * n_hg);
    const int64_t run = rem / n_hg;
    const int h = (int)(rem % n_hg) * RPW + lane / LPR;
    const bool active = h < H;
    const int ch0 = (lane % LPR) * CPL;
    const T *x = s == 0 ? x0 : x1;
    const float *wt = s == 0 ? w0 : w1;
    T *o = s == 0 ? o0 : o1;

    // taps padded to four: tap kFeatMaxWidth - W + j multiplies the row W - 1 - j back
    float w4[CPL][kFeatMaxWidth];
    if (W == kFeatMaxWidth && (reinterpret_cast<uintptr_t>(wt) & 15) == 0) {
        // the lane's 8 x 4 taps are 32 consecutive floats: eight 16-byte loads
        const float4 *wp = reinterpret_cast<const float4 *>(wt + ((size_t)h * D + ch0) * kFeatMaxWidth);
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            const float4 t = active ? wp[c] : make_float4(0.f, 0.f, 0.f, 0.f);
            w4[c][0] = t.x;
            w4[c][1] = t.y;
            w4[c][2] = t.z;
            w4[c][3] = t.w;
        }
    } else {
#pragma unroll
        for (int c = 0; c < CPL; ++c)
#pragma unroll
            for (int j = 0; j < kFeatMaxWidth; ++j) {
                const int jj = j - (kFeatMaxWidth - W);
                w4[c][j] = (active && jj >= 0) ? wt[((size_t)h * D + ch0 + c) * W + jj] : 0.f;
            }
    }

    const int64_t t0 = run * kFeatRun;
    const int64_t t_end = t0 + kFeatRun < n_tok ? t0 + kFeatRun : n_tok;
    // the sequence holding t0: the last i < n_seq with cu[i] <= t0 (cu is non-decreasing)
    int lo = 0, hi = n_seq - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cu[mid] <= t0) lo = mid; else hi = mid - 1;
    }
    int seq = lo;
    int64_t bos = cu[seq], next = cu[seq + 1];
    while (next <= t0 && seq < n_seq - 1) {     // skip empty sequences
        ++seq;
        bos = next;
        next = cu[seq + 1];
    }
    if (t0 < bos || t0 >= next) {               // cu_seqlens does not cover this token
        if (lane == 0) raise_error(kErrCheck);
        return;
    }
    const size_t row_stride = (size_t)H * D;
    const T *xh = x + (size_t)h * D + ch0;
    T *oh = o + (size_t)h * D + ch0;

    // window: rows t-3, t-2, t-1 (zero before the sequence's first token)
    using Raw = typename RawRow<T>::type;
    float win[3][CPL];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const int64_t tt = t0 - 3 + j;
        const Raw rw = (active && tt >= bos) ? *reinterpret_cast<const Raw *>(xh + tt * row_stride) : Raw{};
        raw_to_f32(rw, win[j]);
    }
    auto load_batch = [&](Raw (&raw)[kFeatBatch], int64_t tb) {
#pragma unroll
        for (int u = 0; u < kFeatBatch; ++u) {
            const int64_t tt = tb + u;
            raw[u] = (active && tt < t_end) ? *reinterpret_cast<const Raw *>(xh + tt * row_stride) : Raw{};
        }
    };
    Raw nxt[kFeatBatch];
    load_batch(nxt, t0);
    for (int64_t tb = t0; tb < t_end; tb += kFeatBatch) {
        Raw cur[kFeatBatch];
#pragma unroll
        for (int u = 0; u < kFeatBatch; ++u) cur[u] = nxt[u];
        if (tb + kFeatBatch < t_end) load_batch(nxt, tb + kFeatBatch);
#pragma unroll
        for (int u = 0; u < kFeatBatch; ++u) {
            const int64_t tt = tb + u;
            if (tt >= t_end) break;                 // warp-uniform
            float xr[CPL];
            raw_to_f32(cur[u], xr);
            if (tt == next) {                       // a new sequence starts here
                while (next <= tt && seq < n_seq - 1) {
                    ++seq;
                    next = cu[seq + 1];
                }
                if (next <= tt) {                   // tokens past the last sequence
                    if (lane == 0) raise_error(kErrCheck);
                    return;
                }
#pragma unroll
                for (int j = 0; j < 3; ++j)
#pragma unroll
                    for (int c = 0; c < CPL; ++c) win[j][c] = 0.f;
            }
            float f[CPL];
            float ss = 0.f;
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                float acc = w4[c][3] * xr[c];
                acc = fmaf(w4[c][2], win[2][c], acc);
                acc = fmaf(w4[c][1], win[1][c], acc);
                acc = fmaf(w4[c][0], win[0][c], acc);
                f[c] = silu_f32(acc);
                ss = fmaf(f[c], f[c], ss);
            }
            if constexpr (L2) {
                ss = group_sum<LPR>(ss);
                const float inv = rsqrtf(ss + eps);
#pragma unroll
                for (int c = 0; c < CPL; ++c) f[c] *= inv;
            }
            if (active) store8f(oh + tt * row_stride, f);
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                win[0][c] = win[1][c];
                win[1][c] = win[2][c];
                win[2][c] = xr[c];
            }
        }
    }
}

}  // namespace gdn
