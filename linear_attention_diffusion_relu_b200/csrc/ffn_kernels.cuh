// Mix-FFN kernels for sm_100a: the step after the linear attention in a Sana
// block ("SANA: Efficient High-Resolution Image Synthesis with Linear Diffusion
// Transformers", section 2.2 "선형 어텐션 블럭": an inverted residual block with
// a 3x3 depthwise convolution and a GLU; section 4: the GLU fused into the
// Mix-FFN kernel).
//
//   gemm_bf16_tc     C = A B^T (bf16 in, fp32 accumulate on UMMA, bf16 out):
//                    the 1x1 expand and the 1x1 project
//   dwconv_glu       3x3 depthwise convolution over the token grid of both
//                    channel halves, then Z = a * sigmoid(g), in one pass
#pragma once

#include "tc_kernels.cuh"

namespace sana {
namespace tc {

// ================================================================= GEMM ===
// Persistent CTAs; tile = 128 rows of A x 256 rows of B (M = 128, N = 256 on
// UMMA), k-blocks of 64 (one 128-byte swizzle span). Tile t of CTA c is
// c + k * grid, row-major over (m, n) tiles, so the CTAs running together
// share A tiles in L2. Two TMEM accumulators: the epilogue of one tile (TMEM
// -> registers -> bf16 -> global) overlaps the next tile's UMMAs.
struct GemmParams {
    int M, N, K;          // C is M x N; A is M x K; B is N x K (both K-major)
    int ldc;              // row stride of C in elements
    int kblocks, mtiles, ntiles;
};

constexpr int GM_TILE_M = 128;
constexpr int GM_TILE_N = 256;
constexpr int GM_A_BYTES = GM_TILE_M * kBoxBytesRow;        // 16 KB
constexpr int GM_B_BYTES = GM_TILE_N * kBoxBytesRow;        // 32 KB
constexpr int GM_STAGE_BYTES = GM_A_BYTES + GM_B_BYTES;
constexpr int GM_STAGES = 4;
constexpr int GM_DATA_BYTES = GM_STAGES * GM_STAGE_BYTES;
using GemmMap = SmemMap<GM_DATA_BYTES>;

struct GemmBars {
    uint64_t* full;        // [GM_STAGES]
    uint64_t* empty;       // [GM_STAGES]
    uint64_t* acc_full;    // [2] a tile's accumulator complete
    uint64_t* acc_empty;   // [2] read by every worker warp
    uint64_t* mma_done;
    __device__ void init() const {
        for (int s = 0; s < GM_STAGES; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        for (int j = 0; j < 2; ++j) {
            ptx::mbar_init(&acc_full[j], 1);
            ptx::mbar_init(&acc_empty[j], kWorkerWarps);
        }
        ptx::mbar_init(mma_done, 1);
    }
};

__device__ __forceinline__ GemmBars gemm_bars(uint64_t* b) {
    uint64_t* a = b + 2 * GM_STAGES;
    return GemmBars{b, b + GM_STAGES, a, a + 2, a + 4};
}

__global__ void __launch_bounds__(kThreads, 1)
gemm_bf16_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
             const GemmParams p, __nv_bfloat16* __restrict__ C)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    const GemmBars bar = gemm_bars(reinterpret_cast<uint64_t*>(smem + GemmMap::BAR_OFF));
    SharedCtl* ctl = reinterpret_cast<SharedCtl*>(smem + GemmMap::CTL_OFF);
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    volatile int* abort = &ctl->abort;
    uint32_t* err = &g_device_error;
    if (tid == 0) {
        bar.init();
        ptx::fence_mbar_init();
    }
    kernel_prologue(ctl, tid);
    if (tid == kProducerWarp * 32) {
        ptx::prefetch_tmap(&tmA);
        ptx::prefetch_tmap(&tmB);
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = ctl->tmem_base;
    const int tiles = p.mtiles * p.ntiles;
    const int ntl = (int)blockIdx.x < tiles ? (tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
    auto tile_of = [&](int i, int& m0, int& n0) {
        const int t = (int)blockIdx.x + i * (int)gridDim.x;
        m0 = (t / p.ntiles) * GM_TILE_M;
        n0 = (t % p.ntiles) * GM_TILE_N;
    };
    auto stage_ptr = [&](int s) { return smem + (size_t)s * GM_STAGE_BYTES; };

    if (warp == kProducerWarp) {
        if (lane == 0) {
            int k = 0, issued = 0;
            bool ok = true;
            for (int i = 0; i < ntl && ok; ++i) {
                int m0, n0;
                tile_of(i, m0, n0);
                for (int kb = 0; kb < p.kblocks; ++kb, ++k) {
                    const int s = k % GM_STAGES;
                    if (!ptx::mbar_wait(&bar.empty[s], ((k / GM_STAGES) & 1) ^ 1, abort, err)) { ok = false; break; }
                    uint8_t* st = stage_ptr(s);
                    ptx::mbar_arrive_expect_tx(&bar.full[s], GM_STAGE_BYTES);
                    ptx::tma_load_3d(st, &tmA, &bar.full[s], kb * 64, m0, 0);
                    ptx::tma_load_3d(st + GM_A_BYTES, &tmB, &bar.full[s], kb * 64, n0, 0);
                    issued = k + 1;
                }
            }
            for (int j = (issued > GM_STAGES ? issued - GM_STAGES : 0); j < issued; ++j)
                ptx::mbar_wait(&bar.full[j % GM_STAGES], (j / GM_STAGES) & 1, nullptr, err);
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_bf16_f32(GM_TILE_M, GM_TILE_N, 0, 0);
            int k = 0;
            bool ok = true;
            for (int i = 0; i < ntl && ok; ++i) {
                const int buf = i & 1;
                if (!ptx::mbar_wait(&bar.acc_empty[buf], ((i >> 1) & 1) ^ 1, abort, err)) break;
                ptx::tc_fence_after_sync();
                const uint32_t d_tmem = tmem + (uint32_t)(buf * GM_TILE_N);
                for (int kb = 0; kb < p.kblocks; ++kb, ++k) {
                    const int s = k % GM_STAGES;
                    if (!ptx::mbar_wait(&bar.full[s], (k / GM_STAGES) & 1, abort, err)) { ok = false; break; }
                    ptx::tc_fence_after_sync();
                    const uint32_t a0 = ptx::smem_u32(stage_ptr(s));
                    const uint32_t b0 = a0 + GM_A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        // K-major, 128-byte swizzle: 16 elements = 32 bytes along the row
                        const uint64_t a = ptx::smem_desc(a0 + kk * 32, 16, 1024, ptx::kLayoutSW128);
                        const uint64_t b = ptx::smem_desc(b0 + kk * 32, 16, 1024, ptx::kLayoutSW128);
                        ptx::umma_f16_ss(d_tmem, a, b, idesc, (kb | kk) != 0);
                    }
                    ptx::umma_commit(&bar.empty[s]);
                }
                if (ok) ptx::umma_commit(&bar.acc_full[buf]);
            }
            ptx::umma_commit(bar.mma_done);
            ptx::mbar_wait(bar.mma_done, 0, nullptr, err);
        }
    } else {
        // workers: warp w reads TMEM lanes 32*(w%4).. (its 32 rows) and columns
        // 128*(w/4).. of the tile, converts to bf16 and stores its row piece
        const int r = (warp & 3) * 32 + lane;
        const int half = warp >> 2;
        const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        for (int i = 0; i < ntl; ++i) {
            const int buf = i & 1;
            if (!warp_wait(&bar.acc_full[buf], (i >> 1) & 1, abort, err)) break;
            ptx::tc_fence_after_sync();
            float v[128];
            __syncwarp();
#pragma unroll
            for (int c = 0; c < 4; ++c)
                ptx::tmem_ld32(lane_base + (uint32_t)(buf * GM_TILE_N + half * 128 + c * 32), v + c * 32);
            ptx::tc_fence_before_sync();
            warp_arrive(&bar.acc_empty[buf]);
            int m0, n0;
            tile_of(i, m0, n0);
            const int m = m0 + r;
            if (m < p.M) {
                __nv_bfloat16* row = C + (size_t)m * p.ldc;
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int n = n0 + half * 128 + q * 8;
                    if (n < p.N) {
                        const float* x = v + q * 8;
                        uint4 w;
                        w.x = float2_to_bf16x2(x[0], x[1]);
                        w.y = float2_to_bf16x2(x[2], x[3]);
                        w.z = float2_to_bf16x2(x[4], x[5]);
                        w.w = float2_to_bf16x2(x[6], x[7]);
                        *reinterpret_cast<uint4*>(row + n) = w;
                    }
                }
            }
        }
    }
    kernel_epilogue(ctl, tid);
}

// ====================================================== depthwise + GLU ===
// A CTA is 32 channel chunks (8 channels each, both halves) x 8 token lanes.
// Each thread keeps its chunk's 2 x 8 x 9 taps in registers and walks the
// tokens t0 + lane_y, t0 + lane_y + 8, ... of its CTA's token range: for each
// of the 9 taps it reads 8 channels of the value half a and of the gate half g
// of U (16 bytes each; the 32 chunk lanes of a token read 512 contiguous
// bytes), accumulates in fp32 in tap order (dy, dx) and writes
// Z = a * sigmoid(g) as 8 bf16. Neighbour tokens come through L1/L2.
// U: (B, Hg*Wg, 2*Ch) bf16; Kdw: (2*Ch, 3, 3) fp32; Z: (B, Hg*Wg, Ch) bf16.
constexpr int DW_CHUNKS = 32;      // channel chunks per CTA
constexpr int DW_LANES = 8;        // token lanes per CTA
constexpr int DW_TOKENS = 64;      // tokens per CTA

__global__ void __launch_bounds__(DW_CHUNKS * DW_LANES)
dwconv_glu(const __nv_bfloat16* __restrict__ U, const float* __restrict__ Kdw, int B, int Hg, int Wg, int Ch,
           __nv_bfloat16* __restrict__ Z)
{
    const int chunks = Ch / 8;
    const int ck = blockIdx.x * DW_CHUNKS + (threadIdx.x % DW_CHUNKS);
    const int ly = threadIdx.x / DW_CHUNKS;
    if (ck >= chunks) return;
    const int c0 = ck * 8;
    float ka[8][9], kg[8][9];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
        for (int t = 0; t < 9; ++t) {
            ka[j][t] = Kdw[(c0 + j) * 9 + t];
            kg[j][t] = Kdw[(Ch + c0 + j) * 9 + t];
        }
    }
    const long long ntok = (long long)B * Hg * Wg;
    const long long t_begin = (long long)blockIdx.y * DW_TOKENS;
    for (long long tok = t_begin + ly; tok < ntok && tok < t_begin + DW_TOKENS; tok += DW_LANES) {
        const int x = (int)(tok % Wg);
        const int y = (int)((tok / Wg) % Hg);
        const long long base = tok - (long long)y * Wg - x;    // first token of this batch's grid
        float a[8], g[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) a[j] = g[j] = 0.0f;
#pragma unroll
        for (int dy = 0; dy < 3; ++dy) {
            const int yy = y + dy - 1;
#pragma unroll
            for (int dx = 0; dx < 3; ++dx) {
                const int xx = x + dx - 1;
                if (yy < 0 || yy >= Hg || xx < 0 || xx >= Wg) continue;
                const __nv_bfloat16* u = U + (base + (long long)yy * Wg + xx) * (2LL * Ch);
                const uint4 va = *reinterpret_cast<const uint4*>(u + c0);
                const uint4 vg = *reinterpret_cast<const uint4*>(u + Ch + c0);
                const uint32_t wa[4] = {va.x, va.y, va.z, va.w};
                const uint32_t wg[4] = {vg.x, vg.y, vg.z, vg.w};
                const int t = dy * 3 + dx;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 fa = bf16x2_to_float2(wa[j]);
                    const float2 fg = bf16x2_to_float2(wg[j]);
                    a[2 * j] = fmaf(fa.x, ka[2 * j][t], a[2 * j]);
                    a[2 * j + 1] = fmaf(fa.y, ka[2 * j + 1][t], a[2 * j + 1]);
                    g[2 * j] = fmaf(fg.x, kg[2 * j][t], g[2 * j]);
                    g[2 * j + 1] = fmaf(fg.y, kg[2 * j + 1][t], g[2 * j + 1]);
                }
            }
        }
        float z[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) z[j] = a[j] / (1.0f + __expf(-g[j]));   // a * sigmoid(g)
        uint4 out;
        out.x = float2_to_bf16x2(z[0], z[1]);
        out.y = float2_to_bf16x2(z[2], z[3]);
        out.z = float2_to_bf16x2(z[4], z[5]);
        out.w = float2_to_bf16x2(z[6], z[7]);
        *reinterpret_cast<uint4*>(Z + tok * Ch + c0) = out;
    }
}

}  // namespace tc
}  // namespace sana
