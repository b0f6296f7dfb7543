// FP32-pipe (FFMA) kernels for the three steps of the split-N forward.
//
// KS  partial state  P[b,h,c] = sum_{n in chunk c} phi(K_n)^T [V_n | 1]
// KR  reduce         S[b,h]   = sum_{c = 0..C-1} P[b,h,c], ascending c
// KA  apply          O_n      = (phi(Q_n) S[:, :d]) / (phi(Q_n) S[:, d] + eps)
//
// These run every multiply-add on the FP32 pipe: 2 d (d+1) flops per token-head
// for KS and again for KA. At d = 32 that work takes longer on the FFMA pipe than
// moving the bytes takes on HBM, which is why the tensor-core kernels exist.
#pragma once

#include "common.cuh"

namespace sana {
namespace simt {

constexpr int kThreads = 128;
constexpr int kTileTokens = 64;     // tokens staged in shared memory per step (KS)
constexpr int kApplyTokens = 128;   // tokens per CTA (KA): one per thread

// ---------------------------------------------------------------- KS ------
// One CTA per unit (b, h, chunk c). Thread t owns state row i = t / TPR and
// columns [cg * COLS, cg * COLS + COLS) with cg = t % TPR; threads with cg == 0
// also own the normaliser column d.
template <int D>
__global__ void __launch_bounds__(kThreads)
ks_partial(const __nv_bfloat16* __restrict__ K, const __nv_bfloat16* __restrict__ V,
           int N, int H, int C, int chunk, float* __restrict__ partial)
{
    constexpr int TPR = kThreads / D;        // threads per state row: 4 (d=32) or 2 (d=64)
    constexpr int COLS = D / TPR;            // 8 or 32 columns per thread
    constexpr int VEC = 8;                   // bf16 per 16-byte load
    constexpr int CHUNKS_PER_ROW = D / VEC;
    __shared__ __align__(16) float Ks[kTileTokens][D];
    __shared__ __align__(16) float Vs[kTileTokens][D];

    const long long u = blockIdx.x;
    const int c = (int)(u % C);
    const int h = (int)((u / C) % H);
    const int b = (int)(u / ((long long)C * H));
    const int t = threadIdx.x;
    const int i = t / TPR;
    const int col0 = (t % TPR) * COLS;

    const long long n_begin = (long long)c * chunk;
    const long long n_end = min((long long)N, n_begin + chunk);

    float acc[COLS];
#pragma unroll
    for (int j = 0; j < COLS; ++j) acc[j] = 0.0f;
    float acc_norm = 0.0f;

    for (long long tok0 = n_begin; tok0 < n_end; tok0 += kTileTokens) {
        // stage phi(K) and V for tokens [tok0, tok0 + kTileTokens) as fp32
        for (int q = t; q < kTileTokens * CHUNKS_PER_ROW; q += kThreads) {
            const int r = q / CHUNKS_PER_ROW;
            const int cc = q % CHUNKS_PER_ROW;
            const long long n = tok0 + r;
            uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
            if (n < n_end) {
                const long long off = (((long long)b * N + n) * H + h) * D + cc * VEC;
                kv = ldg_stream(K + off);
                vv = ldg_stream(V + off);
            }
            const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w};
            const uint32_t vw[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float2 kf = bf16x2_to_float2(relu_bf16x2(kw[e]));
                float2 vf = bf16x2_to_float2(vw[e]);
                Ks[r][cc * VEC + 2 * e] = kf.x;
                Ks[r][cc * VEC + 2 * e + 1] = kf.y;
                Vs[r][cc * VEC + 2 * e] = vf.x;
                Vs[r][cc * VEC + 2 * e + 1] = vf.y;
            }
        }
        __syncthreads();
        const int rows = (int)min((long long)kTileTokens, n_end - tok0);
        for (int r = 0; r < rows; ++r) {
            const float k = Ks[r][i];
#pragma unroll
            for (int j = 0; j < COLS; j += 4) {
                const float4 v = *reinterpret_cast<const float4*>(&Vs[r][col0 + j]);
                acc[j + 0] = fmaf(k, v.x, acc[j + 0]);
                acc[j + 1] = fmaf(k, v.y, acc[j + 1]);
                acc[j + 2] = fmaf(k, v.z, acc[j + 2]);
                acc[j + 3] = fmaf(k, v.w, acc[j + 3]);
            }
            acc_norm += k;
        }
        __syncthreads();
    }

    float* P = partial + u * (long long)(D * (D + 1)) + i * (D + 1);
#pragma unroll
    for (int j = 0; j < COLS; ++j) P[col0 + j] = acc[j];
    if (col0 == 0) P[D] = acc_norm;
}

// ---------------------------------------------------------------- KR ------
// One CTA per (b, h): S = sum over chunks in ascending order (deterministic).
template <int D>
__global__ void __launch_bounds__(256)
kr_reduce(const float* __restrict__ partial, int C, float* __restrict__ state)
{
    constexpr int DD = D * (D + 1);
    const long long bh = blockIdx.x;
    const float* P = partial + bh * C * (long long)DD;
    for (int e = threadIdx.x; e < DD; e += blockDim.x) {
        float s = 0.0f;
        for (int c = 0; c < C; ++c) s += P[(long long)c * DD + e];
        state[bh * DD + e] = s;
    }
}

// ---------------------------------------------------------------- KA ------
// One CTA per (b, h, tile of 128 tokens); one thread per token.
template <int D, bool OUT_BF16>
__global__ void __launch_bounds__(kThreads)
ka_apply(const __nv_bfloat16* __restrict__ Q, const float* __restrict__ state,
         int N, int H, int tiles, float eps, void* __restrict__ O)
{
    constexpr int SROW = D + 4;   // padded row so each row starts 16-byte aligned
    __shared__ __align__(16) float Ss[D][SROW];

    const long long u = blockIdx.x;
    const int tile = (int)(u % tiles);
    const int h = (int)((u / tiles) % H);
    const int b = (int)(u / ((long long)tiles * H));
    const float* S = state + ((long long)b * H + h) * D * (D + 1);
    for (int e = threadIdx.x; e < D * (D + 1); e += kThreads) Ss[e / (D + 1)][e % (D + 1)] = S[e];
    __syncthreads();

    const long long n = (long long)tile * kApplyTokens + threadIdx.x;
    if (n >= N) return;
    const long long off = (((long long)b * N + n) * H + h) * D;

    float q[D];
#pragma unroll
    for (int cc = 0; cc < D / 8; ++cc) {
        const uint4 w = ldg_stream(Q + off + cc * 8);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float2 f = bf16x2_to_float2(relu_bf16x2(ws[e]));
            q[cc * 8 + 2 * e] = f.x;
            q[cc * 8 + 2 * e + 1] = f.y;
        }
    }
    float acc[D + 1];
#pragma unroll
    for (int j = 0; j <= D; ++j) acc[j] = 0.0f;
#pragma unroll
    for (int i = 0; i < D; ++i) {
#pragma unroll
        for (int j = 0; j < D; j += 4) {
            const float4 s = *reinterpret_cast<const float4*>(&Ss[i][j]);
            acc[j + 0] = fmaf(q[i], s.x, acc[j + 0]);
            acc[j + 1] = fmaf(q[i], s.y, acc[j + 1]);
            acc[j + 2] = fmaf(q[i], s.z, acc[j + 2]);
            acc[j + 3] = fmaf(q[i], s.w, acc[j + 3]);
        }
        acc[D] = fmaf(q[i], Ss[i][D], acc[D]);
    }
    const float den = acc[D] + eps;
    if (OUT_BF16) {
        __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(O) + off;
#pragma unroll
        for (int j = 0; j < D; j += 8) {
            uint4 w;
            w.x = float2_to_bf16x2(acc[j + 0] / den, acc[j + 1] / den);
            w.y = float2_to_bf16x2(acc[j + 2] / den, acc[j + 3] / den);
            w.z = float2_to_bf16x2(acc[j + 4] / den, acc[j + 5] / den);
            w.w = float2_to_bf16x2(acc[j + 6] / den, acc[j + 7] / den);
            stg_stream(o + j, w);
        }
    } else {
        float* o = reinterpret_cast<float*>(O) + off;
#pragma unroll
        for (int j = 0; j < D; j += 4) {
            uint4 w;
            w.x = __float_as_uint(acc[j + 0] / den);
            w.y = __float_as_uint(acc[j + 1] / den);
            w.z = __float_as_uint(acc[j + 2] / den);
            w.w = __float_as_uint(acc[j + 3] / den);
            stg_stream(o + j, w);
        }
    }
}

}  // namespace simt
}  // namespace sana
