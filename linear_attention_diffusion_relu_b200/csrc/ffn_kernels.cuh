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
// A CTA takes one batch image's tile of DW_TY grid rows x DW_TX columns and 64
// channels of each half (value a: c0 .. c0+63, gate g: Ch+c0 .. Ch+c0+63). Two
// TMA loads bring the tile plus a one-token halo of each half into shared
// memory ([row][column][64 channels], zeros outside the grid: the load starts
// at column x0-1 and row y0-1); the 128 channels' taps go beside them. Each
// thread then computes 8 outputs of one 8-channel chunk: for each of the 9
// taps (order dy, dx) it reads 16 bytes of a and of g of the neighbour and
// accumulates in fp32; Z = a * sigmoid(g) is stored as 8 bf16 (8 lanes = one
// token's 128 bytes).
// U (tensor map): (B, Hg, Wg, 2*Ch) bf16; Kdw: (2*Ch, 3, 3) fp32; Z: (B, Hg*Wg, Ch) bf16.
constexpr int DW_TY = 4;                        // grid rows per CTA
constexpr int DW_TX = 64;                       // grid columns per CTA
constexpr int DW_CH = 64;                       // channels of each half per CTA
constexpr int DW_THREADS = 256;
constexpr int DW_HALF_BYTES = (DW_TY + 2) * (DW_TX + 2) * DW_CH * 2;   // one half's box: 50,688 B
constexpr int DW_TAPS_OFF = 2 * DW_HALF_BYTES;
constexpr int DW_BAR_OFF = DW_TAPS_OFF + 2 * DW_CH * 9 * 4;
constexpr int DW_SMEM = DW_BAR_OFF + 16 + 128;  // barrier, flag, alignment slack

__global__ void __launch_bounds__(DW_THREADS)
dwconv_glu(const __grid_constant__ CUtensorMap tmU, const float* __restrict__ Kdw, int B, int Hg, int Wg, int Ch,
           __nv_bfloat16* __restrict__ Z)
{
    extern __shared__ uint8_t dsm_raw[];
    uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 127) & ~uintptr_t(127));
    float* taps = reinterpret_cast<float*>(dsm + DW_TAPS_OFF);     // [tap][128 ch]
    uint64_t* bar = reinterpret_cast<uint64_t*>(dsm + DW_BAR_OFF);
    int* loaded = reinterpret_cast<int*>(dsm + DW_BAR_OFF + 8);
    const int tid = threadIdx.x;
    const int tiles_x = (Wg + DW_TX - 1) / DW_TX;
    const int tiles_y = (Hg + DW_TY - 1) / DW_TY;
    const int c0 = blockIdx.x * DW_CH;                       // first channel of the group (each half)
    const int b = blockIdx.y / (tiles_y * tiles_x);
    const int ty = (blockIdx.y / tiles_x) % tiles_y;
    const int tx = blockIdx.y % tiles_x;
    const int y0 = ty * DW_TY, x0 = tx * DW_TX;
    const int nch = min(DW_CH, Ch - c0);                     // channels of this group (multiple of 8)
    if (tid == 0) {
        ptx::mbar_init(bar, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        ptx::mbar_arrive_expect_tx(bar, 2 * DW_HALF_BYTES);
        ptx::tma_load_4d(dsm, &tmU, bar, c0, x0 - 1, y0 - 1, b);
        ptx::tma_load_4d(dsm + DW_HALF_BYTES, &tmU, bar, Ch + c0, x0 - 1, y0 - 1, b);
    }
    // taps: entry t * 128 + j, j < 64 the value half, j >= 64 the gate half
    for (int e = tid; e < 2 * DW_CH * 9; e += DW_THREADS) {
        const int t = e / (2 * DW_CH), j = e % (2 * DW_CH);
        const int c = j < DW_CH ? c0 + j : Ch + c0 + (j - DW_CH);
        taps[e] = (j % DW_CH) < nch ? Kdw[(size_t)c * 9 + t] : 0.0f;
    }
    // thread 0 waits for the tile (bounded) and tells the others, so the
    // decision to go on is the same for every thread
    if (tid == 0) {
        const bool ok = ptx::mbar_wait(bar, 0, nullptr, &g_device_error);
        if (!ok) ptx::mbar_wait(bar, 0, nullptr, &g_device_error);   // let the copies land before leaving
        *loaded = ok ? 1 : 0;
    }
    __syncthreads();
    if (!*loaded) return;
    // outputs: DW_TY * DW_TX tokens x 8 chunks; thread -> chunk tid % 8 and the
    // tokens tid / 8 + 32 k, taken two at a time so that each tap's 16 weights
    // (four 16-byte loads) serve two tokens
    const int ck = tid % 8;
    if (ck * 8 >= nch) return;
    const long long img = (long long)b * Hg * Wg;
    for (int o0 = tid / 8; o0 < DW_TY * DW_TX; o0 += 2 * (DW_THREADS / 8)) {
        int ly[2], lx[2];
        bool live[2];
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const int o = o0 + p * (DW_THREADS / 8);
            ly[p] = o / DW_TX;
            lx[p] = o % DW_TX;
            live[p] = o < DW_TY * DW_TX && y0 + ly[p] < Hg && x0 + lx[p] < Wg;
        }
        float a[2][8], g[2][8];
#pragma unroll
        for (int p = 0; p < 2; ++p)
#pragma unroll
            for (int j = 0; j < 8; ++j) a[p][j] = g[p][j] = 0.0f;
#pragma unroll 1
        for (int dy = 0; dy < 3; ++dy) {
#pragma unroll
            for (int dx = 0; dx < 3; ++dx) {
                const float4* tp = reinterpret_cast<const float4*>(taps + (dy * 3 + dx) * (2 * DW_CH) + ck * 8);
                const float4 ta0 = tp[0], ta1 = tp[1];                  // value channels
                const float4 tg0 = tp[DW_CH / 4], tg1 = tp[DW_CH / 4 + 1];   // gate channels
                const float ta[8] = {ta0.x, ta0.y, ta0.z, ta0.w, ta1.x, ta1.y, ta1.z, ta1.w};
                const float tg[8] = {tg0.x, tg0.y, tg0.z, tg0.w, tg1.x, tg1.y, tg1.z, tg1.w};
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    const size_t off = (size_t)((min(ly[p], DW_TY - 1) + dy) * (DW_TX + 2) + (lx[p] + dx)) *
                                       (DW_CH * 2) + ck * 16;
                    const uint4 va = *reinterpret_cast<const uint4*>(dsm + off);
                    const uint4 vg = *reinterpret_cast<const uint4*>(dsm + DW_HALF_BYTES + off);
                    const uint32_t wa[4] = {va.x, va.y, va.z, va.w};
                    const uint32_t wg[4] = {vg.x, vg.y, vg.z, vg.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float2 fa = bf16x2_to_float2(wa[j]);
                        const float2 fg = bf16x2_to_float2(wg[j]);
                        a[p][2 * j] = fmaf(fa.x, ta[2 * j], a[p][2 * j]);
                        a[p][2 * j + 1] = fmaf(fa.y, ta[2 * j + 1], a[p][2 * j + 1]);
                        g[p][2 * j] = fmaf(fg.x, tg[2 * j], g[p][2 * j]);
                        g[p][2 * j + 1] = fmaf(fg.y, tg[2 * j + 1], g[p][2 * j + 1]);
                    }
                }
            }
        }
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            if (!live[p]) continue;
            float z[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) z[j] = a[p][j] / (1.0f + __expf(-g[p][j]));   // a * sigmoid(g)
            uint4 out;
            out.x = float2_to_bf16x2(z[0], z[1]);
            out.y = float2_to_bf16x2(z[2], z[3]);
            out.z = float2_to_bf16x2(z[4], z[5]);
            out.w = float2_to_bf16x2(z[6], z[7]);
            *reinterpret_cast<uint4*>(Z + (img + (long long)(y0 + ly[p]) * Wg + (x0 + lx[p])) * Ch + c0 + ck * 8) = out;
        }
    }
}

}  // namespace tc
}  // namespace sana
