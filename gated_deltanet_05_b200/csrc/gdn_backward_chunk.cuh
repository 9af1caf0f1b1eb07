// gdn_backward_chunk.cuh -- gradients of the gated delta rule through its chunked form,
// fp32-accurate, with the matrix products on the tensor cores.
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
//     dL = strict_tril(-T^T dT T^T) = strict_tril(-(T^T dU~) U~^T)  (as T Z = U~),
//     dA = diag(beta) (dL o Gamma)
//     dbeta = rowsum(V o T^T dU~) + gamma o rowsum(K o T^T dW) + rowsum(dL o A o Gamma)
// and the decays gamma, Gamma, D fold into d g, then into d log alpha by a reverse
// cumulative sum inside the chunk. (The same algebra is restated in fp64 and pinned to the
// oracle's token-by-token adjoint in the tests.)
//
// Five launches:
//   chunk_bwd_prep_kernel   per (chain, chunk), all at once: T, A o Gamma, P and W of the
//                           chunk, kept in the workspace (all that does not depend on the state)
//   chunk_bwd_fwd_kernel    per (chain, d_v slice), chunks in order: the start state and U~ of
//                           every chunk (the forward's state chain)
//   chunk_bwd_state_kernel  per (chain, d_v slice), chunks in reverse: dS at every chunk end and
//                           dU~ of every chunk, and dS0
//   chunk_bwd_vpart_kernel  per (chain, chunk, d_v slice), all at once: dV, and the slice's
//                           sums over v that the rest needs (dP, T^T dT T^T, dW, dK~, dY S^T,
//                           ...), each slice into its own block (no atomics: the result is
//                           deterministic)
//   chunk_bwd_kpart_kernel  per (chain, chunk), all at once: dQ, dK, dbeta, dlog_alpha
// Every matrix product runs from shared memory on the tensor cores (mma.sync m16n8k8, tf32)
// with each operand split into two tf32 parts, which keeps fp32 accuracy; an operand that is
// an unscaled bf16 input (K, Q, V, dY) is a tf32 value already and is not split, so the
// kernels move the scale factors (beta, gamma, D, the q scale) onto the other operand or onto
// the result. A warp owns a 16 x 16 block of the result. Rows in shared memory are padded to
// a multiple of 4 plus 4 floats (16-byte aligned rows; distinct banks for the fragment loads).
#pragma once
#include "gdn_common.cuh"
#include "sm100_ptx.cuh"
#include <type_traits>

namespace gdn {
namespace bwdc {

constexpr int kC = 64;               // chunk length
constexpr int kDVT = 64;             // value columns per CTA in the sliced steps
constexpr int kThreads = 256;        // prep
constexpr int kThreadsWide = 512;    // fwd, state, vpart and kpart

__host__ __device__ inline int slice_cols(int DV) { return DV < kDVT ? DV : kDVT; }
// bf16 inputs converted to fp32 without scaling are tf32 values (8 significant bits <= 11):
// products with such an operand need no split of it
template <typename T>
__host__ __device__ constexpr bool exact_tf32() { return sizeof(T) == 2; }
// shared-memory row stride for rows of D floats (D a multiple of 16): 16-byte aligned rows,
// and rows g = 0..7 of a fragment load start on distinct banks
__host__ __device__ inline int ldp(int D) { return D + 4; }
// floats of the per-chunk sums block of one value slice: dP, T^T dT T^T [C][C]; dW, dK~, dY S^T
// [C][DK]; the row sums of V o T^T dU~ [C]; <dS', S> [1]; rounded up to a multiple of 4
__host__ __device__ inline size_t part_floats(int DK)
{
    return ((size_t)kC * (2 * kC + 3 * DK + 1) + 1 + 3) & ~(size_t)3;
}
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
    // the four loads first, so that they are in flight together
    float la[kC / 32], be[kC / 32];
#pragma unroll
    for (int j = 0; j < kC / 32; ++j) {
        const int t = 32 * j + lane;
        la[j] = t < n ? log_alpha[(size_t)(c0 + t) * H + h] : 0.f;
        be[j] = t < n ? beta[(size_t)(c0 + t) * H + h] : 0.f;
    }
    float carry = 0.f;
#pragma unroll
    for (int j = 0; j < kC / 32; ++j) {
        const int t = 32 * j + lane;
        float x = la[j];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y_ = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y_;
        }
        x += carry;
        carry = __shfl_sync(0xffffffffu, x, 31);
        g[t] = x;
        gam[t] = expf(x);
        bet[t] = be[j];
    }
    __syncwarp();
    const float gC = g[kC - 1];
    for (int t = lane; t < kC; t += 32) Dd[t] = expf(gC - g[t]);
}

__device__ __forceinline__ float4 f4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ void st4(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
__device__ __forceinline__ void st2(float *p, float a, float b) { *reinterpret_cast<float2 *>(p) = make_float2(a, b); }
__device__ __forceinline__ float4 scale4(float4 v, float f) { return make_float4(v.x * f, v.y * f, v.z * f, v.w * f); }
__device__ __forceinline__ float4 add4(float4 a, float4 b) { return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w); }

// The same from the chunk's log alpha and beta already in shared memory (la, be; n valid).
__device__ __forceinline__ void chunk_decays_smem(const float *la_s, const float *be_s, int n, float *g, float *gam,
                                                  float *bet, float *Dd)
{
    const int lane = threadIdx.x;
    float carry = 0.f;
#pragma unroll
    for (int j = 0; j < kC / 32; ++j) {
        const int t = 32 * j + lane;
        float x = t < n ? la_s[t] : 0.f;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y_ = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y_;
        }
        x += carry;
        carry = __shfl_sync(0xffffffffu, x, 31);
        g[t] = x;
        gam[t] = expf(x);
        bet[t] = t < n ? be_s[t] : 0.f;
    }
    __syncwarp();
    const float gC = g[kC - 1];
    for (int t = lane; t < kC; t += 32) Dd[t] = expf(gC - g[t]);
}

// Columns [col0, col0 + ncol) of a chunk's rows of a token-major [.., H, D] tensor into shared
// memory [kC][ld] (zero past n), times f. ncol, col0 and D multiples of 4.
template <typename T>
__device__ __forceinline__ void load_rows(float *dst, int ld, const T *__restrict__ src, int64_t c0, int n, int H,
                                          int h, int D, int col0, int ncol, float f)
{
    const int nq = ncol >> 2;
#pragma unroll 4
    for (int i = threadIdx.x; i < kC * nq; i += blockDim.x) {
        const int t = i / nq, a = (i % nq) * 4;
        const float4 x = t < n ? scale4(load4(src + ((size_t)(c0 + t) * H + h) * D + col0 + a), f)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
        st4(dst + t * ld + a, x);
    }
}

// The first ncol columns of the same rows stored transposed, dst[a][t] = src[t][a] ([ncol][ld]).
// A warp covers 8 rows x 16 columns, so its global loads fill whole sectors and its
// shared-memory stores meet at most two to a bank.
template <typename T>
__device__ __forceinline__ void load_rows_t(float *dst, int ld, const T *__restrict__ src, int64_t c0, int n, int H,
                                            int h, int D, int ncol)
{
    const int nq = ncol >> 2;
#pragma unroll 4
    for (int i = threadIdx.x; i < kC * nq; i += blockDim.x) {
        const int rest = i >> 3, a = (rest % nq) * 4, t = (rest / nq) * 8 + (i & 7);
        const float4 x = t < n ? load4(src + ((size_t)(c0 + t) * H + h) * D + a) : make_float4(0.f, 0.f, 0.f, 0.f);
        dst[(a + 0) * ld + t] = x.x;
        dst[(a + 1) * ld + t] = x.y;
        dst[(a + 2) * ld + t] = x.z;
        dst[(a + 3) * ld + t] = x.w;
    }
}

// Up to R float4 row pieces of a chunk's rows per thread, loaded into registers before any is
// stored (so all of a thread's loads are in flight together), then stored to shared memory
// [kC][ld], or transposed ([ncol][ld]) when TRANS. Piece i = tid + r blockDim covers four
// columns of one row: row i / nq, columns 4 (i % nq) .. (nq = ncol / 4); for TRANS a warp
// takes 8 rows x 16 columns instead, so that its transposed stores meet at most two to a bank
// while each row's 16 columns still fill whole sectors. Zero past n.
template <bool TRANS>
__device__ __forceinline__ void piece_at(int i, int nq, int &t, int &a)
{
    if (TRANS) {
        const int rest = i >> 3;
        a = (rest % nq) * 4;
        t = (rest / nq) * 8 + (i & 7);
    } else {
        t = i / nq;
        a = (i % nq) * 4;
    }
}
template <bool TRANS, int R, typename T>
__device__ __forceinline__ void fetch_rows(float4 (&x)[R], const T *__restrict__ src, int64_t c0, int n, int H,
                                           int h, int D, int col0, int ncol)
{
    const int nq = ncol >> 2;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int i = threadIdx.x + r * blockDim.x;
        int t, a;
        piece_at<TRANS>(i, nq, t, a);
        x[r] = (i < kC * nq && t < n) ? load4(src + ((size_t)(c0 + t) * H + h) * D + col0 + a)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
}
template <bool TRANS, int R>
__device__ __forceinline__ void put_rows(float *dst, int ld, const float4 (&x)[R], int ncol)
{
    const int nq = ncol >> 2;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int i = threadIdx.x + r * blockDim.x;
        if (i >= kC * nq) continue;
        int t, a;
        piece_at<TRANS>(i, nq, t, a);
        if (TRANS) {
            dst[(a + 0) * ld + t] = x[r].x;
            dst[(a + 1) * ld + t] = x[r].y;
            dst[(a + 2) * ld + t] = x[r].z;
            dst[(a + 3) * ld + t] = x[r].w;
        } else {
            st4(dst + t * ld + a, x[r]);
        }
    }
}
// A row-major [rows][cols] fp32 block of the cache by cp.async into shared memory [rows][ld]
// (one commit group is left to the caller)
__device__ __forceinline__ void copy_block_async(float *dst, int ld, const float *__restrict__ src, int rows, int cols)
{
    const int nq = cols >> 2;
    for (int i = threadIdx.x; i < rows * nq; i += blockDim.x) cp_async16(dst + (i / nq) * ld + (i % nq) * 4, src + 4 * (size_t)i);
}

// A row-major [rows][cols] fp32 block (global, 16-byte aligned) into shared memory [rows][ld],
// times f.
__device__ __forceinline__ void load_block(float *dst, int ld, const float *__restrict__ src, int rows, int cols,
                                           float f)
{
    const int nq = cols >> 2;
#pragma unroll 4
    for (int i = threadIdx.x; i < rows * nq; i += blockDim.x) {
        const int r = i / nq, c = (i % nq) * 4;
        st4(dst + r * ld + c, scale4(f4(src + (size_t)r * cols + c), f));
    }
}

// ---- tensor-core products from shared memory --------------------------------------------
// C[M][N] += A[M][K] B[K][N] on mma.sync m16n8k8 tiles in tf32. Each operand is split as
// x = hi + lo with hi = x with its 13 low mantissa bits cleared (a tf32 value) and lo = x - hi
// (exact in fp32; the tensor core reads only its top 19 bits), and A B is taken as
// lo_A hi_B + hi_A lo_B + hi_A hi_B. |lo| < 2^-10 |x|, so the dropped lo_A lo_B and the bits of
// lo the tensor core does not read leave an error below about 3 * 2^-20 |A| |B| per term:
// fp32-level products, with fp32 accumulation.
// A(m, k) = AMK ? A[m lda + k] : A[k lda + m];  B(k, n) = BKN ? B[k ldb + n] : B[n ldb + k].
// A warp owns the 16 x 16 block `tile` of C (tiles numbered row-major over N / 16 columns):
// with g = lane / 4, q = lane % 4, its elements (f, e) (fragment f = 0, 1; e = 0..3) sit at
// row m0 + g + 8 (e / 2), column n0 + 8 f + 2 q + e % 2. M, N multiples of 16, K of 8.
__device__ __forceinline__ void split_tf32(float x, uint32_t &hi, uint32_t &lo)
{
    hi = __float_as_uint(x) & 0xffffe000u;
    lo = __float_as_uint(x - __uint_as_float(hi));
}

__device__ __forceinline__ void mma8(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <bool AMK, bool BKN>
struct WTile {
    int m0, n0, g, q;
    float c[2][4];
    __device__ __forceinline__ WTile(int tile, int N)
    {
        const int lane = threadIdx.x & 31, ntn = N >> 4;
        m0 = (tile / ntn) << 4;
        n0 = (tile % ntn) << 4;
        g = lane >> 2;
        q = lane & 3;
#pragma unroll
        for (int f = 0; f < 2; ++f)
#pragma unroll
            for (int e = 0; e < 4; ++e) c[f][e] = 0.f;
    }
    __device__ __forceinline__ int row(int h) const { return m0 + g + 8 * h; }          // h = e / 2
    __device__ __forceinline__ int col(int f) const { return n0 + 8 * f + 2 * q; }      // e % 2 = 0
    // fn(row, col, C[row][col], C[row][col + 1]) for the four pairs of this lane
    template <class F>
    __device__ __forceinline__ void each(F fn) const
    {
#pragma unroll
        for (int f = 0; f < 2; ++f)
#pragma unroll
            for (int h = 0; h < 2; ++h) fn(row(h), col(f), c[f][2 * h], c[f][2 * h + 1]);
    }
    // C[row][col], C[row][col + 1] = fn(row, col) (a float2)
    template <class F>
    __device__ __forceinline__ void init(F fn)
    {
#pragma unroll
        for (int f = 0; f < 2; ++f)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float2 v = fn(row(h), col(f));
                c[f][2 * h] = v.x;
                c[f][2 * h + 1] = v.y;
            }
    }
    // EXA / EXB: every entry of A / B is a tf32 value already (its lo part is zero: bf16
    // inputs converted to fp32 unscaled), so that operand is not split and its lo product is
    // skipped
    template <bool EXA = false, bool EXB = false>
    __device__ __forceinline__ void run(int K, const float *__restrict__ A, int lda, const float *__restrict__ B,
                                        int ldb)
    {
#pragma unroll 2
        for (int k = 0; k < K; k += 8) {
            uint32_t ah[4], al[4], bh[2][2], bl[2][2];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int m = m0 + g + 8 * (e & 1), kk = k + q + 4 * (e >> 1);
                const float x = AMK ? A[m * lda + kk] : A[kk * lda + m];
                if (EXA)
                    ah[e] = __float_as_uint(x);
                else
                    split_tf32(x, ah[e], al[e]);
            }
#pragma unroll
            for (int f = 0; f < 2; ++f)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int kk = k + q + 4 * e, nn = n0 + 8 * f + g;
                    const float x = BKN ? B[kk * ldb + nn] : B[nn * ldb + kk];
                    if (EXB)
                        bh[f][e] = __float_as_uint(x);
                    else
                        split_tf32(x, bh[f][e], bl[f][e]);
                }
#pragma unroll
            for (int f = 0; f < 2; ++f) {
                if (!EXA) mma8(c[f], al, bh[f][0], bh[f][1]);
                if (!EXB) mma8(c[f], ah, bl[f][0], bl[f][1]);
                mma8(c[f], ah, bh[f][0], bh[f][1]);
            }
        }
    }
};

// Two products with one B and the same tile, C1 += A1 B and C2 += A2 B: B's fragments are
// loaded and split once per k step for both.
template <bool EXA1, bool EXA2, bool EXB, bool AMK, bool BKN>
__device__ __forceinline__ void run2(WTile<AMK, BKN> &w1, WTile<AMK, BKN> &w2, int K, const float *__restrict__ A1,
                                     const float *__restrict__ A2, int lda, const float *__restrict__ B, int ldb)
{
    const int m0 = w1.m0, n0 = w1.n0, g = w1.g, q = w1.q;
#pragma unroll 2
    for (int k = 0; k < K; k += 8) {
        uint32_t bh[2][2], bl[2][2];
#pragma unroll
        for (int f = 0; f < 2; ++f)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int kk = k + q + 4 * e, nn = n0 + 8 * f + g;
                const float x = BKN ? B[kk * ldb + nn] : B[nn * ldb + kk];
                if (EXB)
                    bh[f][e] = __float_as_uint(x);
                else
                    split_tf32(x, bh[f][e], bl[f][e]);
            }
        auto one = [&](WTile<AMK, BKN> &w, const float *__restrict__ A, auto exa) {
            constexpr bool EXA = decltype(exa)::value;
            uint32_t ah[4], al[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int m = m0 + g + 8 * (e & 1), kk = k + q + 4 * (e >> 1);
                const float x = AMK ? A[m * lda + kk] : A[kk * lda + m];
                if (EXA)
                    ah[e] = __float_as_uint(x);
                else
                    split_tf32(x, ah[e], al[e]);
            }
#pragma unroll
            for (int f = 0; f < 2; ++f) {
                if (!EXA) mma8(w.c[f], al, bh[f][0], bh[f][1]);
                if (!EXB) mma8(w.c[f], ah, bl[f][0], bl[f][1]);
                mma8(w.c[f], ah, bh[f][0], bh[f][1]);
            }
        };
        one(w1, A1, std::integral_constant<bool, EXA1>());
        one(w2, A2, std::integral_constant<bool, EXA2>());
    }
}

// Chunk geometry of (sequence seq, chunk c): first token and valid rows; false past the end.
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
    int KQ, Ls, Ts, Ms, g, gam, bet, Dd, total;
};
__host__ __device__ inline PrepSmem prep_layout(int DK)
{
    PrepSmem L;
    int o = 0;
    const int kq = ldp(DK), cp = ldp(kC);
    L.KQ = o; o += 2 * kC * kq;
    L.Ls = o; o += kC * cp;
    L.Ts = o; o += kC * cp;
    L.Ms = o; o += 3 * 16 * 16;
    L.g = o; o += kC;
    L.gam = o; o += kC;
    L.bet = o; o += kC;
    L.Dd = o; o += kC;
    L.total = o;
    return L;
}

// One CTA (kThreads) per (chain, chunk): [K; Q] K^T, then A o Gamma, P and L; T = (I + L)^-1
// by 16 x 16 blocks (diagonal blocks by forward substitution, one column per thread; then
// T_ba = -T_bb sum_{a <= k < b} L_bk T_ka, one block diagonal at a time);
// W = T diag(beta gamma) K. All into the chunk's cache.
template <typename T>
__global__ void __launch_bounds__(kThreads)
chunk_bwd_prep_kernel(const T *__restrict__ q, const T *__restrict__ k, const float *__restrict__ log_alpha,
                      const float *__restrict__ beta, const int32_t *__restrict__ cu_seqlens, int H, int DK,
                      float scale, int max_chunks, float *__restrict__ cache)
{
    extern __shared__ __align__(16) float sm[];
    const PrepSmem Y = prep_layout(DK);
    float *KQ = sm + Y.KQ, *Ls = sm + Y.Ls, *Ts = sm + Y.Ts;
    float *g = sm + Y.g, *gam = sm + Y.gam, *bet = sm + Y.bet, *Dd = sm + Y.Dd;
    const int kq = ldp(DK), cp = ldp(kC);
    const int c = blockIdx.y, chain = blockIdx.x;
    const int seq = chain / H, h = chain % H;
    const int tid = threadIdx.x, warp = tid >> 5, n_warps = blockDim.x >> 5;
    int64_t c0;
    int n;
    if (!chunk_of(cu_seqlens, seq, c, c0, n)) return;
    float *cb = cache + ((size_t)chain * max_chunks + c) * cache_floats(DK);
    {
        // the K and Q rows in flight together, stored once the identity and the decays are done
        float4 kr[kC * 128 / 4 / kThreads], qr[kC * 128 / 4 / kThreads];
        fetch_rows<false>(kr, k, c0, n, H, h, DK, 0, DK);
        fetch_rows<false>(qr, q, c0, n, H, h, DK, 0, DK);
        for (int i = tid; i < kC * kC; i += blockDim.x) Ts[(i / kC) * cp + i % kC] = (i / kC == i % kC) ? 1.f : 0.f;
        if (tid < 32) chunk_decays(log_alpha, beta, c0, n, H, h, g, gam, bet, Dd);
        put_rows<false>(KQ, kq, kr, DK);
        put_rows<false>(KQ + kC * kq, kq, qr, DK);
    }
    __syncthreads();
    // [K; Q] K^T: A = KQ [m][a], B(a, s) = K[s][a] stored [n][k]; Q is unscaled here (the
    // scale goes to the Q rows of the result)
    for (int tile = warp; tile < (2 * kC / 16) * (kC / 16); tile += n_warps) {
        WTile<true, false> w(tile, kC);
        w.template run<exact_tf32<T>(), exact_tf32<T>()>(DK, KQ, kq, KQ, kq);
        w.each([&](int m, int s, float v0, float v1) {
            const int t = m & (kC - 1);
            const float f = m < kC ? 1.f : scale;
            const float x0 = s <= t ? f * v0 * expf(g[t] - g[s]) : 0.f;
            const float x1 = s + 1 <= t ? f * v1 * expf(g[t] - g[s + 1]) : 0.f;
            if (m < kC) {
                st2(cb + kCacheAG + t * kC + s, x0, x1);
                Ls[t * cp + s] = s < t ? bet[t] * x0 : 0.f;
                Ls[t * cp + s + 1] = s + 1 < t ? bet[t] * x1 : 0.f;
            } else {
                st2(cb + kCacheP + t * kC + s, x0, x1);
            }
        });
    }
    __syncthreads();
    // diagonal blocks: column j of block b, T[t][j] = -sum_{j <= s < t} L[t][s] T[s][j] for
    // j < t inside the block (the thread writes and reads back only its own column)
    if (tid < kC) {
        const int b16 = (tid >> 4) * 16, j = b16 + (tid & 15);
        for (int t = j + 1; t < b16 + 16; ++t) {
            float x = 0.f;
            for (int sd = j; sd < t; ++sd) x = fmaf(Ls[t * cp + sd], Ts[sd * cp + j], x);
            Ts[t * cp + j] = -x;
        }
    }
    __syncthreads();
    // off-diagonal blocks, distance d = b - a = 1, 2, 3: M = sum_{a <= k < b} L_bk T_ka, then
    // T_ba = -T_bb M (the blocks of one distance are independent)
    float *Ms = sm + Y.Ms;
    for (int d = 1; d < 4; ++d) {
        const int nblk = 4 - d;
        for (int i = tid; i < nblk * 256; i += blockDim.x) {
            const int a = i >> 8, t = (i >> 4) & 15, j = i & 15, b = a + d;
            float x = 0.f;
            for (int sd = 16 * a; sd < 16 * b; ++sd) x = fmaf(Ls[(16 * b + t) * cp + sd], Ts[sd * cp + 16 * a + j], x);
            Ms[i] = x;
        }
        __syncthreads();
        for (int i = tid; i < nblk * 256; i += blockDim.x) {
            const int a = i >> 8, t = (i >> 4) & 15, j = i & 15, b = a + d;
            float x = 0.f;
            for (int sd = 0; sd <= t; ++sd) x = fmaf(Ts[(16 * b + t) * cp + 16 * b + sd], Ms[(a << 8) + sd * 16 + j], x);
            Ts[(16 * b + t) * cp + 16 * a + j] = -x;
        }
        __syncthreads();
    }
    // T to the cache, then T diag(beta gamma) in place (K stays unscaled: an exact operand
    // for bf16 inputs)
    for (int i = tid; i < kC * kC / 4; i += blockDim.x) {
        const int r = i / (kC / 4), c4 = (i % (kC / 4)) * 4;
        const float4 x = f4(Ts + r * cp + c4);
        st4(cb + kCacheT + r * kC + c4, x);
        st4(Ts + r * cp + c4, make_float4(x.x * bet[c4] * gam[c4], x.y * bet[c4 + 1] * gam[c4 + 1],
                                          x.z * bet[c4 + 2] * gam[c4 + 2], x.w * bet[c4 + 3] * gam[c4 + 3]));
    }
    __syncthreads();
    // W = (T diag(beta gamma)) K: A = [t][s], B = K [s][a]
    for (int tile = warp; tile < (kC / 16) * (DK / 16); tile += n_warps) {
        WTile<true, true> w(tile, DK);
        w.template run<false, exact_tf32<T>()>(kC, Ts, cp, KQ, kq);
        w.each([&](int t, int a, float v0, float v1) { st2(cb + kCacheW + t * DK + a, v0, v1); });
    }
}

// --------------------------------------------------------------------------- fwd
struct FwdSmem {
    int Kd, Ws, Ts, Vb, Us, Ss, Kraw, Vraw, las, bes, g, gam, bet, Dd, total;
};
// esize: bytes per input element (the raw K and V rows of the next chunk wait in Kraw, Vraw)
__host__ __device__ inline FwdSmem fwd_layout(int DK, int DVT, int esize)
{
    FwdSmem L;
    int o = 0;
    const int kq = ldp(DK), vq = ldp(DVT), cp = ldp(kC);
    L.Kd = o; o += kC * kq;
    L.Ws = o; o += kC * kq;
    L.Ts = o; o += kC * cp;
    L.Vb = o; o += kC * vq;
    L.Us = o; o += kC * vq;
    L.Ss = o; o += DK * vq;
    L.Kraw = o; o += kC * DK * esize / 4;
    L.Vraw = o; o += kC * DVT * esize / 4;
    L.las = o; o += kC;
    L.bes = o; o += kC;
    L.g = o; o += kC;
    L.gam = o; o += kC;
    L.bet = o; o += kC;
    L.Dd = o; o += kC;
    L.total = o;
    return L;
}

// One CTA (kThreadsWide) per (chain, d_v slice): the forward's state chain from S0
// (value-major [DV][DK] or NULL) with the cached T and W, keeping the start state of every
// chunk in S_chunks [chain][max_chunks][DK][DV] (the pages' orientation) and every chunk's
// U~ in Ut_chunks [chain][max_chunks][C][DV]. Every input of chunk
// c + 1 is requested by cp.async while chunk c is computed: its raw K and V rows and gates
// once chunk c's have been converted, its T and W once chunk c's U~ product is done.
template <typename T>
__global__ void __launch_bounds__(kThreadsWide)
chunk_bwd_fwd_kernel(const T *__restrict__ k, const T *__restrict__ v, const float *__restrict__ log_alpha,
                     const float *__restrict__ beta, const float *__restrict__ S0,
                     const int32_t *__restrict__ cu_seqlens, int H, int DK, int DV, int max_chunks,
                     const float *__restrict__ cache, float *__restrict__ S_chunks, float *__restrict__ Ut_chunks)
{
    extern __shared__ __align__(16) float sm[];
    const int DVT = slice_cols(DV);
    const FwdSmem Y = fwd_layout(DK, DVT, (int)sizeof(T));
    float *Kd = sm + Y.Kd, *Ws = sm + Y.Ws, *Ts = sm + Y.Ts, *Vb = sm + Y.Vb, *Us = sm + Y.Us, *Ss = sm + Y.Ss;
    T *Kraw = reinterpret_cast<T *>(sm + Y.Kraw), *Vraw = reinterpret_cast<T *>(sm + Y.Vraw);
    float *las = sm + Y.las, *bes = sm + Y.bes;
    float *g = sm + Y.g, *gam = sm + Y.gam, *bet = sm + Y.bet, *Dd = sm + Y.Dd;
    const int kq = ldp(DK), vq = ldp(DVT), cp = ldp(kC);
    constexpr int EPC = 16 / (int)sizeof(T);          // elements per 16-byte piece
    const int n_vt = DV / DVT;
    const int chain = blockIdx.x / n_vt, v0 = (blockIdx.x % n_vt) * DVT;
    const int seq = chain / H, h = chain % H;
    const int tid = threadIdx.x, warp = tid >> 5, n_warps = blockDim.x >> 5;
    const int64_t len = (int64_t)cu_seqlens[seq + 1] - cu_seqlens[seq];
    const size_t st_off = (size_t)chain * DV * DK;
    for (int i = tid; i < DK * DVT; i += blockDim.x) {
        const int a = i % DK, b = i / DK;
        Ss[a * vq + b] = S0 ? S0[st_off + (size_t)(v0 + b) * DK + a] : 0.f;
    }
    const int n_chunks = (int)((len + kC - 1) / kC);
    const int nvq = DVT / 4;
    auto request_tw = [&](int c) {
        const float *cb = cache + ((size_t)chain * max_chunks + c) * cache_floats(DK);
        copy_block_async(Ts, cp, cb + kCacheT, kC, kC);
        copy_block_async(Ws, kq, cb + kCacheW, kC, DK);
        cp_async_commit();
    };
    auto request_rows = [&](int c) {                  // rows past the sequence end are not copied
        int64_t cc0;
        int nn;
        chunk_of(cu_seqlens, seq, c, cc0, nn);
        const int pk = DK / EPC, pv = DVT / EPC;
        for (int i = tid; i < nn * pk; i += blockDim.x) {
            const int t = i / pk, w = i % pk;
            cp_async16(Kraw + t * DK + w * EPC, k + ((size_t)(cc0 + t) * H + h) * DK + w * EPC);
        }
        for (int i = tid; i < nn * pv; i += blockDim.x) {
            const int t = i / pv, w = i % pv;
            cp_async16(Vraw + t * DVT + w * EPC, v + ((size_t)(cc0 + t) * H + h) * DV + v0 + w * EPC);
        }
        for (int i = tid; i < 2 * nn; i += blockDim.x) {
            const int t = i >> 1;
            cp_async4((i & 1) ? bes + t : las + t, ((i & 1) ? beta : log_alpha) + (size_t)(cc0 + t) * H + h);
        }
        cp_async_commit();
    };
    if (n_chunks > 0) {
        request_tw(0);
        request_rows(0);
    }
    for (int c = 0; c < n_chunks; ++c) {
        int64_t c0;
        int n;
        chunk_of(cu_seqlens, seq, c, c0, n);
        __syncthreads();
        {
            float *dst = S_chunks + ((size_t)chain * max_chunks + c) * DK * DV + v0;
            for (int i = tid; i < DK * nvq; i += blockDim.x) {
                const int a = i / nvq, b = (i % nvq) * 4;
                st4(dst + (size_t)a * DV + b, f4(Ss + a * vq + b));
            }
        }
        cp_async_wait_all();                           // this chunk's inputs have landed
        __syncthreads();
        if (tid < 32) chunk_decays_smem(las, bes, n, g, gam, bet, Dd);
        __syncthreads();
        // K and V in fp32, unscaled (zero past n), so that bf16 inputs stay exact tf32
        // operands; T diag(beta) in place (its columns scaled)
        for (int i = tid; i < kC * DK / 4; i += blockDim.x) {
            const int t = i / (DK / 4), a = (i % (DK / 4)) * 4;
            st4(Kd + t * kq + a, t < n ? load4(Kraw + t * DK + a) : make_float4(0.f, 0.f, 0.f, 0.f));
        }
        for (int i = tid; i < kC * nvq; i += blockDim.x) {
            const int t = i / nvq, b = (i % nvq) * 4;
            st4(Vb + t * vq + b, t < n ? load4(Vraw + t * DVT + b) : make_float4(0.f, 0.f, 0.f, 0.f));
        }
        for (int i = tid; i < kC * kC / 4; i += blockDim.x) {
            const int t = i / (kC / 4), s4 = (i % (kC / 4)) * 4;
            const float4 x = f4(Ts + t * cp + s4);
            st4(Ts + t * cp + s4, make_float4(x.x * bet[s4], x.y * bet[s4 + 1], x.z * bet[s4 + 2], x.w * bet[s4 + 3]));
        }
        __syncthreads();
        if (c + 1 < n_chunks) request_rows(c + 1);    // the raw rows and gates are free
        // U~ = (T diag(beta)) V - W S, to Ut_chunks; diag(D) U~ into Us for the state update
        {
            float *dst = Ut_chunks + ((size_t)chain * max_chunks + c) * kC * DV + v0;
            for (int tile = warp; tile < (kC / 16) * (DVT / 16); tile += n_warps) {
                WTile<true, true> w(tile, DVT), ws(tile, DVT);
                w.template run<false, exact_tf32<T>()>(kC, Ts, cp, Vb, vq);
                ws.run(DK, Ws, kq, Ss, vq);
#pragma unroll
                for (int f = 0; f < 2; ++f)
#pragma unroll
                    for (int e = 0; e < 4; ++e) w.c[f][e] -= ws.c[f][e];
                w.each([&](int t, int b, float v0_, float v1_) {
                    st2(dst + (size_t)t * DV + b, v0_, v1_);
                    st2(Us + t * vq + b, Dd[t] * v0_, Dd[t] * v1_);
                });
            }
        }
        __syncthreads();
        if (c + 1 < n_chunks) request_tw(c + 1);     // T and W are free: the next chunk's
        // S <- gamma_C S + K^T (diag(D) U~): A(a, s) = K[s][a] stored [k][m]; each warp reads
        // and writes only its own entries of S
        const float gamC = gam[kC - 1];
        for (int tile = warp; tile < (DK / 16) * (DVT / 16); tile += n_warps) {
            WTile<false, true> w(tile, DVT);
            w.init([&](int a, int b) {
                const float2 x = *reinterpret_cast<const float2 *>(Ss + a * vq + b);
                return make_float2(gamC * x.x, gamC * x.y);
            });
            w.template run<exact_tf32<T>(), false>(kC, Kd, kq, Us, vq);
            w.each([&](int a, int b, float v0_, float v1_) { st2(Ss + a * vq + b, v0_, v1_); });
        }
    }
    cp_async_wait_all();
}

// --------------------------------------------------------------------------- state
struct StateSmem {
    int Ks, Qg, Ws, Ps, dYs, dUs, dSs, Kraw, Qraw, Yraw, las, bes, g, gam, bet, Dd, total;
};
// esize: bytes per input element of the raw K, Q and dY rows of the next chunk (bf16 inputs,
// requested while the current chunk computes); 0 for fp32 inputs, whose rows are loaded at the
// start of their own chunk (a second fp32 copy does not fit)
__host__ __device__ inline StateSmem state_layout(int DK, int DVT, int esize)
{
    StateSmem L;
    int o = 0;
    const int kq = ldp(DK), vq = ldp(DVT), cp = ldp(kC);
    L.Ks = o; o += kC * kq;
    L.Qg = o; o += kC * kq;
    L.Ws = o; o += kC * kq;
    L.Ps = o; o += kC * cp;
    L.dYs = o; o += kC * vq;
    L.dUs = o; o += kC * vq;
    L.dSs = o; o += DK * vq;
    L.Kraw = o; o += kC * DK * esize / 4;
    L.Qraw = o; o += kC * DK * esize / 4;
    L.Yraw = o; o += kC * DVT * esize / 4;
    L.las = o; o += kC;
    L.bes = o; o += kC;
    L.g = o; o += kC;
    L.gam = o; o += kC;
    L.bet = o; o += kC;
    L.Dd = o; o += kC;
    L.total = o;
    return L;
}
template <typename T>
__host__ __device__ constexpr bool state_prefetch() { return sizeof(T) == 2; }

// One CTA (kThreadsWide) per (chain, d_v slice): dS from dS_T back through the chunks with
// the cached W and P; dS at the end of every chunk goes to dS_chunks
// [chain][max_chunks][DK][DV] and every chunk's dU~ to dUt_chunks [chain][max_chunks][C][DV],
// the final dS to dS0 (value-major [DV][DK]). Three cp.async groups per chunk c, in this
// order: W_c (at its start), the raw rows and gates of chunk c - 1 (bf16 inputs; empty
// otherwise) once chunk c's are converted, and P_{c-1} once chunk c's dU~ product is done.
template <typename T>
__global__ void __launch_bounds__(kThreadsWide, 1)
chunk_bwd_state_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ dy,
                       const float *__restrict__ log_alpha, const float *__restrict__ beta,
                       const int32_t *__restrict__ cu_seqlens, int H, int DK, int DV, float scale,
                       const float *__restrict__ dS_T, int max_chunks, const float *__restrict__ cache,
                       float *__restrict__ dS_chunks, float *__restrict__ dUt_chunks, float *__restrict__ dS0)
{
    constexpr bool kPre = state_prefetch<T>();
    extern __shared__ __align__(16) float sm[];
    const int DVT = slice_cols(DV);
    const StateSmem Y = state_layout(DK, DVT, kPre ? (int)sizeof(T) : 0);
    float *Ks = sm + Y.Ks, *Qg = sm + Y.Qg, *Ws = sm + Y.Ws, *Ps = sm + Y.Ps;
    float *dYs = sm + Y.dYs, *dUs = sm + Y.dUs, *dSs = sm + Y.dSs;
    T *Kraw = reinterpret_cast<T *>(sm + Y.Kraw), *Qraw = reinterpret_cast<T *>(sm + Y.Qraw);
    T *Yraw = reinterpret_cast<T *>(sm + Y.Yraw);
    float *las = sm + Y.las, *bes = sm + Y.bes;
    float *g = sm + Y.g, *gam = sm + Y.gam, *bet = sm + Y.bet, *Dd = sm + Y.Dd;
    const int kq = ldp(DK), vq = ldp(DVT), cp = ldp(kC);
    constexpr int EPC = 16 / (int)sizeof(T);          // elements per 16-byte piece
    const int n_vt = DV / DVT;
    const int chain = blockIdx.x / n_vt, v0 = (blockIdx.x % n_vt) * DVT;
    const int seq = chain / H, h = chain % H;
    const int tid = threadIdx.x, warp = tid >> 5, n_warps = blockDim.x >> 5;
    const int64_t len = (int64_t)cu_seqlens[seq + 1] - cu_seqlens[seq];
    const size_t st_off = (size_t)chain * DV * DK;
    for (int i = tid; i < DK * DVT; i += blockDim.x) {
        const int a = i % DK, b = i / DK;
        dSs[a * vq + b] = dS_T ? dS_T[st_off + (size_t)(v0 + b) * DK + a] : 0.f;
    }
    const int n_chunks = (int)((len + kC - 1) / kC);
    const int nvq = DVT / 4;
    auto cache_of = [&](int c) { return cache + ((size_t)chain * max_chunks + c) * cache_floats(DK); };
    auto request_rows = [&](int c) {                  // rows past the sequence end are not copied
        int64_t cc0;
        int nn;
        chunk_of(cu_seqlens, seq, c, cc0, nn);
        const int pk = DK / EPC, py = DVT / EPC;
        for (int i = tid; i < nn * pk; i += blockDim.x) {
            const int t = i / pk, w = i % pk;
            const size_t off = ((size_t)(cc0 + t) * H + h) * DK + w * EPC;
            cp_async16(Kraw + t * DK + w * EPC, k + off);
            cp_async16(Qraw + t * DK + w * EPC, q + off);
        }
        for (int i = tid; i < nn * py; i += blockDim.x) {
            const int t = i / py, w = i % py;
            cp_async16(Yraw + t * DVT + w * EPC, dy + ((size_t)(cc0 + t) * H + h) * DV + v0 + w * EPC);
        }
        for (int i = tid; i < 2 * nn; i += blockDim.x) {
            const int t = i >> 1;
            cp_async4((i & 1) ? bes + t : las + t, ((i & 1) ? beta : log_alpha) + (size_t)(cc0 + t) * H + h);
        }
    };
    if (n_chunks > 0) {
        if constexpr (kPre) request_rows(n_chunks - 1);
        cp_async_commit();
        copy_block_async(Ps, cp, cache_of(n_chunks - 1) + kCacheP, kC, kC);
        cp_async_commit();
    }
    for (int c = n_chunks - 1; c >= 0; --c) {
        int64_t c0;
        int n;
        chunk_of(cu_seqlens, seq, c, c0, n);
        __syncthreads();                               // chunk c + 1's products are done
        copy_block_async(Ws, kq, cache_of(c) + kCacheW, kC, DK);
        cp_async_commit();
        {
            float *dst = dS_chunks + ((size_t)chain * max_chunks + c) * DK * DV + v0;
            for (int i = tid; i < DK * nvq; i += blockDim.x) {
                const int a = i / nvq, b = (i % nvq) * 4;
                st4(dst + (size_t)a * DV + b, f4(dSs + a * vq + b));
            }
        }
        if constexpr (kPre) {
            cp_async_wait1();                          // chunk c's rows, gates and P have landed
            __syncthreads();
            if (tid < 32) chunk_decays_smem(las, bes, n, g, gam, bet, Dd);
            __syncthreads();
            // K, dY unscaled and diag(gamma) scale Q in fp32 (zero past n)
            for (int i = tid; i < kC * DK / 4; i += blockDim.x) {
                const int t = i / (DK / 4), a = (i % (DK / 4)) * 4;
                const bool in = t < n;
                st4(Ks + t * kq + a, in ? load4(Kraw + t * DK + a) : make_float4(0.f, 0.f, 0.f, 0.f));
                st4(Qg + t * kq + a, in ? scale4(load4(Qraw + t * DK + a), scale * gam[t]) : make_float4(0.f, 0.f, 0.f, 0.f));
            }
            for (int i = tid; i < kC * nvq; i += blockDim.x) {
                const int t = i / nvq, b = (i % nvq) * 4;
                st4(dYs + t * vq + b, t < n ? load4(Yraw + t * DVT + b) : make_float4(0.f, 0.f, 0.f, 0.f));
            }
            __syncthreads();
            if (c > 0) request_rows(c - 1);            // the raw rows and gates are free
        } else {
            // the chunk's K, Q and dY rows into registers, all loads in flight together, and
            // the decays on warp 0
            {
                float4 kr[kC * 128 / 4 / kThreadsWide], qr[kC * 128 / 4 / kThreadsWide];
                float4 yr[kC * kDVT / 4 / kThreadsWide];
                fetch_rows<false>(kr, k, c0, n, H, h, DK, 0, DK);
                fetch_rows<false>(qr, q, c0, n, H, h, DK, 0, DK);
                fetch_rows<false>(yr, dy, c0, n, H, h, DV, v0, DVT);
                if (tid < 32) chunk_decays(log_alpha, beta, c0, n, H, h, g, gam, bet, Dd);
                put_rows<false>(Ks, kq, kr, DK);
                put_rows<false>(Qg, kq, qr, DK);
                put_rows<false>(dYs, vq, yr, DVT);
            }
            cp_async_wait1();                          // P has landed
            __syncthreads();
            for (int i = tid; i < kC * DK / 4; i += blockDim.x) {
                const int t = i / (DK / 4), a = (i % (DK / 4)) * 4;
                st4(Qg + t * kq + a, scale4(f4(Qg + t * kq + a), scale * gam[t]));
            }
            __syncthreads();
        }
        cp_async_commit();                             // (empty without a prefetch)
        // dU~ = P^T dY + diag(D) K dS': A(s, t) = P[t][s] stored [k][m], A(s, a) = K[s][a]
        // (K and dY unscaled, so that bf16 inputs stay exact tf32 operands)
        for (int tile = warp; tile < (kC / 16) * (DVT / 16); tile += n_warps) {
            WTile<false, true> w(tile, DVT);
            WTile<true, true> kd(tile, DVT);
            w.template run<false, exact_tf32<T>()>(kC, Ps, cp, dYs, vq);
            kd.template run<exact_tf32<T>(), false>(DK, Ks, kq, dSs, vq);
#pragma unroll
            for (int f = 0; f < 2; ++f)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int s_ = w.row(hh), b = w.col(f);
                    st2(dUs + s_ * vq + b, fmaf(Dd[s_], kd.c[f][2 * hh], w.c[f][2 * hh]),
                        fmaf(Dd[s_], kd.c[f][2 * hh + 1], w.c[f][2 * hh + 1]));
                }
        }
        cp_async_wait1();                              // W_c has landed
        __syncthreads();
        if (c > 0) copy_block_async(Ps, cp, cache_of(c - 1) + kCacheP, kC, kC);   // P is free
        cp_async_commit();
        // dS = gamma_C dS' + (diag(gamma) Q)^T dY - W^T dU~ (each warp: its own entries of dS)
        const float gamC = gam[kC - 1];
        for (int tile = warp; tile < (DK / 16) * (DVT / 16); tile += n_warps) {
            WTile<false, true> w(tile, DVT);
            w.init([&](int a, int b) {
                const float2 x = *reinterpret_cast<const float2 *>(dSs + a * vq + b);
                return make_float2(gamC * x.x, gamC * x.y);
            });
            WTile<false, true> wd(tile, DVT);
            w.template run<false, exact_tf32<T>()>(kC, Qg, kq, dYs, vq);
            wd.run(kC, Ws, kq, dUs, vq);
#pragma unroll
            for (int f = 0; f < 2; ++f)
#pragma unroll
                for (int e = 0; e < 4; ++e) w.c[f][e] -= wd.c[f][e];
            w.each([&](int a, int b, float v0_, float v1_) { st2(dSs + a * vq + b, v0_, v1_); });
        }
        {
            float *dst = dUt_chunks + ((size_t)chain * max_chunks + c) * kC * DV + v0;
            for (int i = tid; i < kC * nvq; i += blockDim.x) {
                const int t = i / nvq, b = (i % nvq) * 4;
                st4(dst + (size_t)t * DV + b, f4(dUs + t * vq + b));
            }
        }
    }
    cp_async_wait_all();
    __syncthreads();
    if (dS0)
        for (int i = tid; i < DK * DVT; i += blockDim.x) {
            const int a = i % DK, b = i / DK;
            dS0[st_off + (size_t)(v0 + b) * DK + a] = dSs[a * vq + b];
        }
}

// --------------------------------------------------------------------------- vpart
struct VpartSmem {
    int Ts, Ss, dSs, Vs, dYs, Uts, dUs, Xs, bet, red, total;
};
__host__ __device__ inline VpartSmem vpart_layout(int DK, int DVT)
{
    VpartSmem L;
    int o = 0;
    const int vq = ldp(DVT), cp = ldp(kC);
    L.Ts = o; o += kC * cp;
    L.Ss = o; o += DK * vq;
    L.dSs = o; o += DK * vq;
    L.Vs = o; o += kC * vq;
    L.dYs = o; o += kC * vq;
    L.Uts = o; o += kC * vq;
    L.dUs = o; o += kC * vq;
    L.Xs = o; o += kC * vq;
    L.bet = o; o += kC;
    L.red = o; o += kThreadsWide / 32;
    L.total = o;
    return L;
}

// One CTA (kThreadsWide) per (chain, chunk, d_v slice): dV of the slice, and the slice's share
// of the sums over v, written to the slice's block of the sums buffer
// [chain][max_chunks][n_slices][part_floats]. U~ and dU~ come from the state chains
// (Ut_chunks, dUt_chunks [chain][max_chunks][C][DV]); with X = T^T dU~ the slice's terms are
// dV = diag(beta) X, rowsum(V o X), dY U~^T, X U~^T, -dU~ S^T, U~ dS'^T, dY S^T and <dS', S>.
template <typename T>
__global__ void __launch_bounds__(kThreadsWide, 1)
chunk_bwd_vpart_kernel(const T *__restrict__ v, const T *__restrict__ dy, const float *__restrict__ beta,
                       const int32_t *__restrict__ cu_seqlens, int H, int DK, int DV, int max_chunks,
                       const float *__restrict__ cache, const float *__restrict__ S_chunks,
                       const float *__restrict__ dS_chunks, const float *__restrict__ Ut_chunks,
                       const float *__restrict__ dUt_chunks, float *__restrict__ parts, float *__restrict__ dv_out)
{
    extern __shared__ __align__(16) float sm[];
    const int DVT = slice_cols(DV);
    const VpartSmem Y = vpart_layout(DK, DVT);
    float *Ts = sm + Y.Ts, *Ss = sm + Y.Ss, *dSs = sm + Y.dSs, *Vs = sm + Y.Vs, *dYs = sm + Y.dYs;
    float *Uts = sm + Y.Uts, *dUs = sm + Y.dUs, *Xs = sm + Y.Xs, *bet = sm + Y.bet, *red = sm + Y.red;
    const int vq = ldp(DVT), cp = ldp(kC);
    const int n_vt = DV / DVT;
    const int c = blockIdx.y;
    const int chain = blockIdx.x / n_vt, vt = blockIdx.x % n_vt, v0 = vt * DVT;
    const int seq = chain / H, h = chain % H;
    const int tid = threadIdx.x, warp = tid >> 5, n_warps = blockDim.x >> 5;
    int64_t c0;
    int n;
    if (!chunk_of(cu_seqlens, seq, c, c0, n)) return;
    const size_t cidx = (size_t)chain * max_chunks + c;
    const float *cb = cache + cidx * cache_floats(DK);
    const float *Sg = S_chunks + cidx * DK * DV + v0, *dSg = dS_chunks + cidx * DK * DV + v0;
    const float *Ug = Ut_chunks + cidx * kC * DV + v0, *dUg = dUt_chunks + cidx * kC * DV + v0;
    const int nvq = DVT / 4;
    // every load in flight together: the states, U~, dU~ and T by cp.async, the V and dY rows
    // into registers
    for (int i = tid; i < DK * nvq; i += blockDim.x) {
        const int a = i / nvq, b = (i % nvq) * 4;
        cp_async16(Ss + a * vq + b, Sg + (size_t)a * DV + b);
        cp_async16(dSs + a * vq + b, dSg + (size_t)a * DV + b);
    }
    for (int i = tid; i < kC * nvq; i += blockDim.x) {
        const int t = i / nvq, b = (i % nvq) * 4;
        cp_async16(Uts + t * vq + b, Ug + (size_t)t * DV + b);
        cp_async16(dUs + t * vq + b, dUg + (size_t)t * DV + b);
    }
    copy_block_async(Ts, cp, cb + kCacheT, kC, kC);
    cp_async_commit();
    {
        float4 vr[kC * kDVT / 4 / kThreadsWide], yr[kC * kDVT / 4 / kThreadsWide];
        fetch_rows<false>(vr, v, c0, n, H, h, DV, v0, DVT);
        fetch_rows<false>(yr, dy, c0, n, H, h, DV, v0, DVT);
        if (tid < kC) bet[tid] = tid < n ? beta[(size_t)(c0 + tid) * H + h] : 0.f;
        put_rows<false>(Vs, vq, vr, DVT);
        put_rows<false>(dYs, vq, yr, DVT);
    }
    cp_async_wait_all();
    __syncthreads();
    float *P = parts + (cidx * n_vt + vt) * part_floats(DK);
    float *PdP = P, *PdT = P + kC * kC, *PdW = P + 2 * kC * kC, *PdKd = PdW + kC * DK, *PdYS = PdKd + kC * DK;
    float *Pvs = PdYS + kC * DK, *PdgC = Pvs + kC;
    const int n_tv = (kC / 16) * (DVT / 16);
    // X = T^T dU~ (A(t, s) = T[s][t], stored [k][m]) into Xs; dV = diag(beta) X
    for (int tile = warp; tile < n_tv; tile += n_warps) {
        WTile<false, true> w(tile, DVT);
        w.run(kC, Ts, cp, dUs, vq);
        w.each([&](int t, int b, float w0, float w1) {
            if (t < n) st2(dv_out + ((size_t)(c0 + t) * H + h) * DV + v0 + b, bet[t] * w0, bet[t] * w1);
            st2(Xs + t * vq + b, w0, w1);
        });
    }
    __syncthreads();
    // row sums of V o X: eight lanes per row
    for (int r = tid; r < kC * 8; r += blockDim.x) {
        const int t = r >> 3, part = r & 7;
        float acc = 0.f;
        for (int b = part; b < DVT; b += 8) acc = fmaf(Vs[t * vq + b], Xs[t * vq + b], acc);
        acc = group_sum<8>(acc);
        if (part == 0) Pvs[t] = acc;
    }
    // this slice's dY U~^T and X U~^T [C][C] (B(b, s) = U~[s][b]: stored [n][k])
    for (int tile = warp; tile < (kC / 16) * (kC / 16); tile += n_warps) {
        WTile<true, false> p(tile, kC), tt(tile, kC);
        run2<exact_tf32<T>(), false, false>(p, tt, DVT, dYs, Xs, vq, Uts, vq);
        p.each([&](int t, int s, float v0_, float v1_) { st2(PdP + t * kC + s, v0_, v1_); });
        tt.each([&](int t, int s, float v0_, float v1_) { st2(PdT + t * kC + s, v0_, v1_); });
    }
    // this slice's -dU~ S^T, U~ dS'^T and dY S^T [C][DK] (B(b, a) = S[a][b]: stored [n][k])
    for (int tile = warp; tile < (kC / 16) * (DK / 16); tile += n_warps) {
        WTile<true, false> w(tile, DK), kd(tile, DK), ys(tile, DK);
        run2<false, exact_tf32<T>(), false>(w, ys, DVT, dUs, dYs, vq, Ss, vq);
        kd.run(DVT, Uts, vq, dSs, vq);
        w.each([&](int t, int a, float v0_, float v1_) { st2(PdW + t * DK + a, -v0_, -v1_); });
        kd.each([&](int t, int a, float v0_, float v1_) { st2(PdKd + t * DK + a, v0_, v1_); });
        ys.each([&](int t, int a, float v0_, float v1_) { st2(PdYS + t * DK + a, v0_, v1_); });
    }
    // <dS', S> over this slice (four columns per step)
    float sd = 0.f;
    for (int i = tid; i < DK * nvq; i += blockDim.x) {
        const int a = i / nvq, b = (i % nvq) * 4;
        const float4 x = f4(dSs + a * vq + b), y = f4(Ss + a * vq + b);
        sd = fmaf(x.x, y.x, fmaf(x.y, y.y, fmaf(x.z, y.z, fmaf(x.w, y.w, sd))));
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
    int Ks, Qs, PdWs, Ts, G1, G1T, Asym, dGs, Es, g, gam, bet, Dd, red, total;
};
__host__ __device__ inline KpartSmem kpart_layout(int DK)
{
    KpartSmem L;
    int o = 0;
    const int kq = ldp(DK), cp = ldp(kC);
    L.Ks = o; o += kC * kq;
    L.Qs = o; o += kC * kq;
    L.PdWs = o; o += kC * kq;
    // Ts .. Es are contiguous: after the last products they hold dQ's and dK's sums
    L.Ts = o; o += kC * cp;
    L.G1 = o; o += kC * cp;
    L.G1T = o; o += kC * cp;
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

// One CTA (kThreadsWide) per (chain, chunk): dQ, dK, dbeta and dlog_alpha of the chunk from
// its cache block and its sums buffer (the value slices' blocks added here, in slice order).
template <typename T>
__global__ void __launch_bounds__(kThreadsWide)
chunk_bwd_kpart_kernel(const T *__restrict__ q, const T *__restrict__ k, const float *__restrict__ log_alpha,
                       const float *__restrict__ beta, const int32_t *__restrict__ cu_seqlens, int H, int DK,
                       int n_vt, float scale, int max_chunks, const float *__restrict__ cache,
                       const float *__restrict__ parts, float *__restrict__ dq, float *__restrict__ dk,
                       float *__restrict__ dbeta, float *__restrict__ dlog_alpha)
{
    extern __shared__ __align__(16) float sm[];
    const KpartSmem Y = kpart_layout(DK);
    float *Ks = sm + Y.Ks, *Qs = sm + Y.Qs, *PdWs = sm + Y.PdWs, *Ts = sm + Y.Ts, *G1 = sm + Y.G1;
    float *G1T = sm + Y.G1T, *Asym = sm + Y.Asym, *dGs = sm + Y.dGs, *Es = sm + Y.Es, *g = sm + Y.g;
    float *gam = sm + Y.gam, *bet = sm + Y.bet, *Dd = sm + Y.Dd, *red = sm + Y.red;
    const int kq = ldp(DK), cp = ldp(kC);
    const int c = blockIdx.y, chain = blockIdx.x;
    const int seq = chain / H, h = chain % H;
    const int tid = threadIdx.x, warp = tid >> 5, n_warps = blockDim.x >> 5;
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
    auto sum_slices4 = [&](size_t off) -> float4 {
        float4 acc = f4(P0 + off);
        for (int j = 1; j < n_vt; ++j) acc = add4(acc, f4(P0 + j * pf + off));
        return acc;
    };

    // every load in flight together: T by cp.async; the K and Q rows and the slice sums
    // (P dW, and T^T dT T^T, as dL, into dGs and dP into G1) in registers; the decays on warp 0
    copy_block_async(Ts, cp, cb + kCacheT, kC, kC);
    cp_async_commit();
    {
        constexpr int RR = kC * 128 / 4 / kThreadsWide, RW = kC * 128 / 4 / kThreadsWide, RT = kC * kC / 4 / kThreadsWide;
        float4 kr[RR], qr[RR], wr[RW], tr[RT], pr[RT];
        fetch_rows<false>(kr, k, c0, n, H, h, DK, 0, DK);
        fetch_rows<false>(qr, q, c0, n, H, h, DK, 0, DK);
        const int nwq = kC * DK / 4;
#pragma unroll
        for (int r = 0; r < RW; ++r) {
            const int i = tid + r * kThreadsWide;
            const size_t off = oW + (size_t)(i / (DK / 4)) * DK + (i % (DK / 4)) * 4;
            wr[r] = i < nwq ? f4(P0 + off) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int r = 0; r < RT; ++r) {
            const int i = tid + r * kThreadsWide;
            tr[r] = f4(P0 + oT + 4 * (size_t)i);
            pr[r] = f4(P0 + oP + 4 * (size_t)i);
        }
        for (int j = 1; j < n_vt; ++j) {
            const float *Pj = P0 + j * pf;
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                const int i = tid + r * kThreadsWide;
                if (i < nwq) wr[r] = add4(wr[r], f4(Pj + oW + (size_t)(i / (DK / 4)) * DK + (i % (DK / 4)) * 4));
            }
#pragma unroll
            for (int r = 0; r < RT; ++r) {
                const int i = tid + r * kThreadsWide;
                tr[r] = add4(tr[r], f4(Pj + oT + 4 * (size_t)i));
                pr[r] = add4(pr[r], f4(Pj + oP + 4 * (size_t)i));
            }
        }
        if (tid < 32) chunk_decays(log_alpha, beta, c0, n, H, h, g, gam, bet, Dd);
        put_rows<false>(Ks, kq, kr, DK);
        put_rows<false>(Qs, kq, qr, DK);
#pragma unroll
        for (int r = 0; r < RW; ++r) {
            const int i = tid + r * kThreadsWide;
            if (i < nwq) st4(PdWs + (i / (DK / 4)) * kq + (i % (DK / 4)) * 4, wr[r]);
        }
#pragma unroll
        for (int r = 0; r < RT; ++r) {
            // dL = strict_tril(-T^T dT T^T), the slices' sums of X U~^T
            const int i = tid + r * kThreadsWide, t = i / (kC / 4), s = (i % (kC / 4)) * 4;
            st4(dGs + t * cp + s, make_float4(s < t ? -tr[r].x : 0.f, s + 1 < t ? -tr[r].y : 0.f,
                                              s + 2 < t ? -tr[r].z : 0.f, s + 3 < t ? -tr[r].w : 0.f));
            st4(G1 + t * cp + s, pr[r]);
        }
    }
    cp_async_wait_all();
    __syncthreads();
    // dA + dA^T with dA = diag(beta) (dL o Gamma), into Asym (symmetric)
    for (int i = tid; i < kC * kC; i += blockDim.x) {
        const int t = i / kC, s = i % kC;
        const float da_ts = s < t ? bet[t] * dGs[t * cp + s] * expf(g[t] - g[s]) : 0.f;
        const float da_st = t < s ? bet[s] * dGs[s * cp + t] * expf(g[s] - g[t]) : 0.f;
        Asym[t * cp + s] = da_ts + da_st;
    }
    // T^T dW (A(t, s) = T[s][t]), kept in registers until PdWs may be overwritten
    constexpr int kMaxWT = (kC / 16) * (128 / 16) / (kThreadsWide / 32);   // 2 at DK = 128
    static_assert(kMaxWT == 2, "the tile arrays below are initialised for two tiles per warp");
    const int n_ck = (kC / 16) * (DK / 16);
    WTile<false, true> tdw[kMaxWT] = {WTile<false, true>(warp, DK), WTile<false, true>(warp + n_warps, DK)};
#pragma unroll
    for (int r = 0; r < kMaxWT; ++r)
        if (warp + r * n_warps < n_ck) tdw[r].run(kC, Ts, cp, PdWs, kq);
    __syncthreads();
    // per entry (same thread reads and writes it): dGamma o Gamma into dGs, dL o A o Gamma into
    // Es, scale (dP o Gamma) into G1 and the unscaled transpose into G1T
#pragma unroll 2
    for (int i = tid; i < kC * kC / 4; i += blockDim.x) {
        const int t = i / (kC / 4), s0 = (i % (kC / 4)) * 4;
        const float4 ag4 = f4(cb + kCacheAG + t * kC + s0), p4 = f4(cb + kCacheP + t * kC + s0);
        const float4 dl4 = f4(dGs + t * cp + s0), dp4 = f4(G1 + t * cp + s0);
        const float ag[4] = {ag4.x, ag4.y, ag4.z, ag4.w}, pp[4] = {p4.x, p4.y, p4.z, p4.w};
        const float dl[4] = {dl4.x, dl4.y, dl4.z, dl4.w}, dp[4] = {dp4.x, dp4.y, dp4.z, dp4.w};
        float dgm[4], e[4], g1[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int s = s0 + u;
            const float gts = s <= t ? expf(g[t] - g[s]) : 0.f;
            dgm[u] = dp[u] * pp[u] + bet[t] * dl[u] * ag[u];
            e[u] = dl[u] * ag[u];
            g1[u] = dp[u] * gts;
            G1T[s * cp + t] = g1[u];
        }
        st4(dGs + t * cp + s0, make_float4(dgm[0], dgm[1], dgm[2], dgm[3]));
        st4(Es + t * cp + s0, make_float4(e[0], e[1], e[2], e[3]));
        // scale (dP o Gamma) for the product with the unscaled Q
        st4(G1 + t * cp + s0, make_float4(scale * g1[0], scale * g1[1], scale * g1[2], scale * g1[3]));
    }
#pragma unroll
    for (int r = 0; r < kMaxWT; ++r)
        if (warp + r * n_warps < n_ck)
            tdw[r].each([&](int t, int a, float v0, float v1) { st2(PdWs + t * kq + a, v0, v1); });
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
    // (dP o Gamma) K and (dP o Gamma)^T (scale Q) + (dA + dA^T) K, in registers until the region
    // Ts .. Es is free (A(t, s) = G1[t][s] = G1T[s][t], G1[s][t] and Asym[s][t]: all [k][m])
    WTile<false, true> aq[kMaxWT] = {WTile<false, true>(warp, DK), WTile<false, true>(warp + n_warps, DK)};
    WTile<false, true> ak[kMaxWT] = {WTile<false, true>(warp, DK), WTile<false, true>(warp + n_warps, DK)};
#pragma unroll
    for (int r = 0; r < kMaxWT; ++r)
        if (warp + r * n_warps < n_ck) {
            run2<false, false, exact_tf32<T>()>(aq[r], ak[r], kC, G1T, Asym, cp, Ks, kq);
            ak[r].template run<false, exact_tf32<T>()>(kC, G1, cp, Qs, kq);
        }
    __syncthreads();
    float *GQ = Ts, *GK = Ts + kC * kq;
#pragma unroll
    for (int r = 0; r < kMaxWT; ++r)
        if (warp + r * n_warps < n_ck) {
            aq[r].each([&](int t, int a, float v0, float v1) { st2(GQ + t * kq + a, v0, v1); });
            ak[r].each([&](int t, int a, float v0, float v1) { st2(GK + t * kq + a, v0, v1); });
        }
    __syncthreads();
    // dQ = diag(gamma) dY S^T + (dP o Gamma) K;
    // dK = (dP o Gamma)^T Q + (dA + dA^T) K + diag(beta gamma) T^T dW + diag(D) dK~;
    // a warp per row t, four consecutive a per lane, with the row sums for dbeta and
    // dlog_alpha; the warp's four rows at once so that all their loads are in flight together
    const int lane = tid & 31;
#pragma unroll 4
    for (int t = warp; t < kC; t += n_warps) {
        float rg = 0.f, rb = 0.f, rd = 0.f;
        for (int a = 4 * lane; a < DK; a += 128) {
            const size_t ta = (size_t)t * DK + a;
            const float4 pys = sum_slices4(oYS + ta), pkd = sum_slices4(oKd + ta);
            const float4 tw = f4(PdWs + t * kq + a), kt = f4(Ks + t * kq + a), qt = f4(Qs + t * kq + a);
            const float4 gq = f4(GQ + t * kq + a), gk = f4(GK + t * kq + a);
            rg += qt.x * pys.x + qt.y * pys.y + qt.z * pys.z + qt.w * pys.w;
            rb += kt.x * tw.x + kt.y * tw.y + kt.z * tw.z + kt.w * tw.w;
            rd += kt.x * pkd.x + kt.y * pkd.y + kt.z * pkd.z + kt.w * pkd.w;
            if (t < n) {
                const float gt = gam[t], bg = bet[t] * gam[t], dt = Dd[t];
                st4(dq + ((size_t)(c0 + t) * H + h) * DK + a,
                    make_float4(scale * (gt * pys.x + gq.x), scale * (gt * pys.y + gq.y),
                                scale * (gt * pys.z + gq.z), scale * (gt * pys.w + gq.w)));
                st4(dk + ((size_t)(c0 + t) * H + h) * DK + a,
                    make_float4(gk.x + bg * tw.x + dt * pkd.x, gk.y + bg * tw.y + dt * pkd.y,
                                gk.z + bg * tw.z + dt * pkd.z, gk.w + bg * tw.w + dt * pkd.w));
            }
        }
        rg = group_sum<32>(rg);
        rb = group_sum<32>(rb);
        rd = group_sum<32>(rd);
        if (lane == 0) {
            red[2 * kC + t] = scale * rg + bet[t] * rb;     // dgamma_t (Q unscaled in rg)
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
