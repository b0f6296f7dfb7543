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

// ======================================================= GEMM, CTA pairs ===
// The same product on a cluster of two CTAs (the two SMs of a TPC): a tile is
// 256 rows of A x 256 rows of B; CTA r of the pair loads A rows 128r .. and B
// rows 128r .. of it into its own shared memory, and the even CTA issues
// tcgen05.mma.cta_group::2 with M = 256, which reads both CTAs' operands and
// leaves rows 128r .. of the product in CTA r's TMEM. Per CTA that halves the
// B bytes staged and read per flop against the one-CTA kernel.
// Both CTAs' loads complete on the even CTA's full barrier (it expects the
// pair's bytes); its UMMA commits arrive on the empty and accumulator barriers
// of both CTAs; the odd CTA's epilogue warps release the accumulator on the
// even CTA's barrier. The pair ends with a bounded handshake before TMEM is
// freed, so neither CTA leaves while the other may still use its memory.
constexpr int G2_TILE_M = 256;
constexpr int G2_TILE_N = 256;
constexpr int G2_HALF_BYTES = 128 * kBoxBytesRow;          // 128 rows x 64 bf16
constexpr int G2_STAGE_BYTES = 2 * G2_HALF_BYTES;          // this CTA's A half + B half
constexpr int G2_STAGES = 6;
using Gemm2Map = SmemMap<G2_STAGES * G2_STAGE_BYTES>;

struct Gemm2Bars {
    uint64_t* full;        // [G2_STAGES] both CTAs' tiles landed (even CTA's copy used)
    uint64_t* empty;       // [G2_STAGES] the pair's UMMAs have read the stage
    uint64_t* acc_full;    // [2] a tile's accumulator complete
    uint64_t* acc_empty;   // [2] read by the worker warps of both CTAs (even CTA's copy used)
    uint64_t* mma_done;
    uint64_t* pair_done;   // the other CTA of the pair has finished
    __device__ void init() const {
        for (int s = 0; s < G2_STAGES; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        for (int j = 0; j < 2; ++j) {
            ptx::mbar_init(&acc_full[j], 1);
            ptx::mbar_init(&acc_empty[j], 2 * kWorkerWarps);
        }
        ptx::mbar_init(mma_done, 1);
        ptx::mbar_init(pair_done, 1);
    }
};

__device__ __forceinline__ Gemm2Bars gemm2_bars(uint64_t* b) {
    uint64_t* a = b + 2 * G2_STAGES;
    return Gemm2Bars{b, b + G2_STAGES, a, a + 2, a + 4, a + 5};
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
gemm_bf16_tc2(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const GemmParams p, __nv_bfloat16* __restrict__ C)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    const Gemm2Bars bar = gemm2_bars(reinterpret_cast<uint64_t*>(smem + Gemm2Map::BAR_OFF));
    SharedCtl* ctl = reinterpret_cast<SharedCtl*>(smem + Gemm2Map::CTL_OFF);
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const uint32_t rank = ptx::cluster_ctarank();
    const bool leader = rank == 0;
    volatile int* abort = &ctl->abort;
    uint32_t* err = &g_device_error;
    if (tid == 0) {
        ctl->abort = 0;
        bar.init();
        ptx::fence_mbar_init();
    }
    if (warp == 0) {
        ptx::tmem_alloc_pair(&ctl->tmem_base, kTmemCols);
        ptx::tmem_relinquish_pair();
    }
    if (tid == kProducerWarp * 32) {
        ptx::prefetch_tmap(&tmA);
        ptx::prefetch_tmap(&tmB);
    }
    // both CTAs' barriers initialised and TMEM allocated before either uses
    // the other's
    ptx::tc_fence_before_sync();
    ptx::cluster_sync();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = ctl->tmem_base;
    const int pair = (int)blockIdx.x / 2;
    const int npairs = (int)gridDim.x / 2;
    const int tiles = p.mtiles * p.ntiles;
    const int ntl = pair < tiles ? (tiles - pair + npairs - 1) / npairs : 0;
    auto tile_of = [&](int i, int& m0, int& n0) {
        const int t = pair + i * npairs;
        m0 = (t / p.ntiles) * G2_TILE_M;
        n0 = (t % p.ntiles) * G2_TILE_N;
    };
    auto stage_ptr = [&](int s) { return smem + (size_t)s * G2_STAGE_BYTES; };

    if (warp == kProducerWarp) {
        if (lane == 0) {
            const uint32_t full0 = ptx::mapa_shared(&bar.full[0], 0);    // the even CTA's full[0]
            int k = 0, issued = 0;
            bool ok = true;
            for (int i = 0; i < ntl && ok; ++i) {
                int m0, n0;
                tile_of(i, m0, n0);
                for (int kb = 0; kb < p.kblocks; ++kb, ++k) {
                    const int s = k % G2_STAGES;
                    if (!ptx::mbar_wait(&bar.empty[s], ((k / G2_STAGES) & 1) ^ 1, abort, err)) { ok = false; break; }
                    if (leader) ptx::mbar_arrive_expect_tx(&bar.full[s], 2 * G2_STAGE_BYTES);
                    uint8_t* st = stage_ptr(s);
                    const uint32_t fb = full0 + (uint32_t)(s * sizeof(uint64_t));
                    ptx::tma_load_3d_pair(st, &tmA, fb, kb * 64, m0 + (int)rank * 128, 0);
                    ptx::tma_load_3d_pair(st + G2_HALF_BYTES, &tmB, fb, kb * 64, n0 + (int)rank * 128, 0);
                    issued = k + 1;
                }
            }
            // every issued load must land before the CTA may leave: the even
            // CTA sees them on its full barriers; the odd CTA's stages are
            // released (empty) only after the pair's UMMAs have read them
            for (int j = (issued > G2_STAGES ? issued - G2_STAGES : 0); j < issued; ++j) {
                if (leader) ptx::mbar_wait(&bar.full[j % G2_STAGES], (j / G2_STAGES) & 1, nullptr, err);
                else ptx::mbar_wait(&bar.empty[j % G2_STAGES], (j / G2_STAGES) & 1, nullptr, err);
            }
        }
    } else if (warp == kMmaWarp) {
        if (leader && lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_bf16_f32(G2_TILE_M, G2_TILE_N, 0, 0);
            int k = 0;
            bool ok = true;
            for (int i = 0; i < ntl && ok; ++i) {
                const int buf = i & 1;
                if (!ptx::mbar_wait(&bar.acc_empty[buf], ((i >> 1) & 1) ^ 1, abort, err)) break;
                ptx::tc_fence_after_sync();
                const uint32_t d_tmem = tmem + (uint32_t)(buf * G2_TILE_N);
                for (int kb = 0; kb < p.kblocks; ++kb, ++k) {
                    const int s = k % G2_STAGES;
                    if (!ptx::mbar_wait(&bar.full[s], (k / G2_STAGES) & 1, abort, err)) { ok = false; break; }
                    ptx::tc_fence_after_sync();
                    const uint32_t a0 = ptx::smem_u32(stage_ptr(s));
                    const uint32_t b0 = a0 + G2_HALF_BYTES;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t a = ptx::smem_desc(a0 + kk * 32, 16, 1024, ptx::kLayoutSW128);
                        const uint64_t b = ptx::smem_desc(b0 + kk * 32, 16, 1024, ptx::kLayoutSW128);
                        ptx::umma_f16_ss_pair(d_tmem, a, b, idesc, (kb | kk) != 0);
                    }
                    ptx::umma_commit_pair(&bar.empty[s], 0x3);
                }
                if (ok) ptx::umma_commit_pair(&bar.acc_full[buf], 0x3);
            }
            ptx::umma_commit_pair(bar.mma_done, 0x1);
            ptx::mbar_wait(bar.mma_done, 0, nullptr, err);
        }
    } else {
        // workers: warp w reads TMEM lanes 32*(w%4).. (its 32 rows of this
        // CTA's 128) and columns 128*(w/4).. of the tile
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
                ptx::tmem_ld32(lane_base + (uint32_t)(buf * G2_TILE_N + half * 128 + c * 32), v + c * 32);
            ptx::tc_fence_before_sync();
            if (leader) {
                warp_arrive(&bar.acc_empty[buf]);
            } else {
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive_cluster(ptx::mapa_shared(&bar.acc_empty[buf], 0));
            }
            int m0, n0;
            tile_of(i, m0, n0);
            const int m = m0 + (int)rank * 128 + r;
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
    // the pair: each CTA tells the other it is done (bounded wait), then both
    // free the shared TMEM allocation
    ptx::tc_fence_before_sync();
    __syncthreads();
    if (tid == 0) {
        ptx::mbar_arrive_cluster(ptx::mapa_shared(bar.pair_done, rank ^ 1u));
        ptx::mbar_wait(bar.pair_done, 0, nullptr, err);
    }
    __syncthreads();
    if (warp == 0) {
        __syncwarp();
        ptx::tc_fence_after_sync();
        ptx::tmem_dealloc_pair(tmem, kTmemCols);
    }
}

// ====================================================== depthwise + GLU ===
// A CTA takes one batch image's tile of TY grid rows x TX columns and 64
// channels of each half (value a: c0 .. c0+63, gate g: Ch+c0 .. Ch+c0+63). Two
// TMA loads bring the tile plus a one-token halo of each half into shared
// memory ([row][column][64 channels], zeros outside the grid: the load starts
// at column x0-1 and row y0-1). Lane l owns channels 2l and 2l+1 of both
// halves, with their 2 x 2 x 9 fp32 taps in registers; warp w owns RPW output
// rows and a strip of SX columns. It walks the strip's SX + 2 halo columns
// once: each step loads one column (RPW + 2 rows x 2 halves, 4 bytes per
// lane, one 128-byte line per warp), unpacks it to fp32 and adds its products
// with the taps (packed fp32x2 FMAs) into the accumulators of the three
// outputs of each row that use it (tap column dx for the output dx columns to
// its left). An accumulator thus receives its nine products one column at a
// time, a whole step apart, instead of in one dependent chain, and an output
// is done once its last column has been added: Z = a * sigmoid(g) as bf16x2,
// kept in registers until every warp is done with the input tile, written
// over it ([row][column][64 channels]) and stored with one TMA store, which
// leaves out what lies outside the grid or past the last channel.
// U (tensor map): (B, Hg, Wg, 2*Ch) bf16; Kdw: (2*Ch, 3, 3) fp32; Z (tensor
// map): (B, Hg, Wg, Ch) bf16.
constexpr int DW_CH = 64;                       // channels of each half per CTA

template <int TY_, int TX_, int SX_, int RPW_, int MINB_>
struct DwCfg {
    static constexpr int TY = TY_;              // grid rows per CTA
    static constexpr int TX = TX_;              // grid columns per CTA
    static constexpr int SX = SX_;              // columns per warp strip
    static constexpr int RPW = RPW_;            // output rows per warp
    static constexpr int MINB = MINB_;          // CTAs per SM the registers are sized for
    static constexpr int WARPS = (TY / RPW) * (TX / SX);
    static constexpr int THREADS = WARPS * 32;
    static constexpr int ROW_BYTES = (TX + 2) * DW_CH * 2;          // one halo row of one half
    static constexpr int HALF_BYTES = (TY + 2) * ROW_BYTES;         // one half's box
    static constexpr int TAPS_OFF = 2 * HALF_BYTES;                 // fp32 [half][tap][64 channels]
    static constexpr int BAR_OFF = TAPS_OFF + 2 * 9 * DW_CH * 4;
    static constexpr int SMEM = BAR_OFF + 16 + 128;                 // barrier, flag, alignment slack
    static_assert(TY % RPW == 0 && TX % SX == 0, "whole strips");
    static_assert(TY * TX * DW_CH * 2 <= HALF_BYTES, "the output tile fits over the value half");
};
// 4 x 32 tiles, 4 warps of 2 rows x 16 columns, 4 CTAs per SM (measured on
// B200 at the 4096px shape: 268 us, against 283 for 8 x 32 tiles with 8 warps
// and 2 CTAs per SM, 299 for 4 x 64 tiles of 1-row warps; summing each output's
// nine products in one dependent chain per half instead: 290-305 us)
using DwConfig = DwCfg<4, 32, 16, 2, 4>;

__device__ __forceinline__ float2 bf16x2_unpack(uint32_t v) {
    return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xFFFF0000u));
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, Cfg::MINB)
dwconv_glu(const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmZ,
           const float* __restrict__ Kdw, int Hg, int Wg, int Ch)
{
    constexpr int TY = Cfg::TY, TX = Cfg::TX, SX = Cfg::SX, RPW = Cfg::RPW;
    constexpr int ROW_BYTES = Cfg::ROW_BYTES, HALF_BYTES = Cfg::HALF_BYTES;
    extern __shared__ uint8_t dsm_raw[];
    uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 127) & ~uintptr_t(127));
    uint64_t* bar = reinterpret_cast<uint64_t*>(dsm + Cfg::BAR_OFF);
    int* loaded = reinterpret_cast<int*>(dsm + Cfg::BAR_OFF + 8);
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int tiles_x = (Wg + TX - 1) / TX;
    const int tiles_y = (Hg + TY - 1) / TY;
    // CTA = tile * groups + group: the CTAs running at the same time take every
    // group of a few tiles, i.e. whole token rows of U
    const int ngroups = (Ch + DW_CH - 1) / DW_CH;
    const int c0 = (int)(blockIdx.x % ngroups) * DW_CH;      // first channel of the group (each half)
    const int tile = (int)(blockIdx.x / ngroups);
    const int b = tile / (tiles_y * tiles_x);
    const int ty = (tile / tiles_x) % tiles_y;
    const int tx = tile % tiles_x;
    const int y0 = ty * TY, x0 = tx * TX;
    const int nch = min(DW_CH, Ch - c0);                     // channels of this group (multiple of 8)
    if (tid == 0) {
        ptx::mbar_init(bar, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        ptx::mbar_arrive_expect_tx(bar, 2 * HALF_BYTES);
        ptx::tma_load_4d(dsm, &tmU, bar, c0, x0 - 1, y0 - 1, b);
        ptx::tma_load_4d(dsm + HALF_BYTES, &tmU, bar, Ch + c0, x0 - 1, y0 - 1, b);
    }
    // the group's taps, read in address order (each half's 64 x 9 block is
    // contiguous) into [half][tap][channel]; zeros past the group's channels
    float* taps = reinterpret_cast<float*>(dsm + Cfg::TAPS_OFF);
    for (int e = tid; e < 2 * DW_CH * 9; e += Cfg::THREADS) {
        const int half = e / (DW_CH * 9), j = e % (DW_CH * 9);
        const int ch = j / 9, t = j % 9;
        taps[(half * 9 + t) * DW_CH + ch] =
            ch < nch ? __ldg(Kdw + (size_t)(half * Ch + c0) * 9 + j) : 0.0f;
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
    // this lane's channel pair and its taps (tap t = 3 dy + dx), both halves;
    // lanes past the group's channels compute zeros that the store leaves out
    const int cp = 2 * lane;
    float2 wa[9], wg[9];
#pragma unroll
    for (int t = 0; t < 9; ++t) {
        wa[t] = *reinterpret_cast<const float2*>(taps + t * DW_CH + cp);
        wg[t] = *reinterpret_cast<const float2*>(taps + (9 + t) * DW_CH + cp);
    }
    constexpr int STRIPS = TX / SX;
    const int ly = (warp / STRIPS) * RPW;                   // output rows y0 + ly .. = halo rows ly + 1 ..
    const int sx = (warp % STRIPS) * SX;                    // first output column of the strip
    // halo row ly + r, halo column sx + j holds grid (y0 + ly - 1 + r, x0 + sx - 1 + j);
    // output x of the strip (halo column sx + x + 1) takes halo columns
    // sx + x .. sx + x + 2 with tap columns dx = 0, 1, 2
    const uint8_t* base = dsm + (size_t)ly * ROW_BYTES + (size_t)sx * (DW_CH * 2) + lane * 4;
    constexpr float kLog2e = 1.4426950408889634f;
    float2 acc[2][RPW][3];                                  // [half][row][output x % 3]
    uint32_t zo[RPW][SX];
#pragma unroll
    for (int j = 0; j < SX + 2; ++j) {
        float2 v[2][RPW + 2];
#pragma unroll
        for (int r = 0; r < RPW + 2; ++r) {
            const uint8_t* q = base + r * ROW_BYTES + j * (DW_CH * 2);
            v[0][r] = bf16x2_unpack(*reinterpret_cast<const uint32_t*>(q));
            v[1][r] = bf16x2_unpack(*reinterpret_cast<const uint32_t*>(q + HALF_BYTES));
        }
#pragma unroll
        for (int dx = 0; dx < 3; ++dx) {
            const int x = j - dx;                           // the output this column feeds with tap column dx
            if (x < 0 || x >= SX) continue;
#pragma unroll
            for (int r = 0; r < RPW; ++r) {
#pragma unroll
                for (int dy = 0; dy < 3; ++dy) {
                    const int t = dy * 3 + dx;
                    if (dx == 0 && dy == 0) {
                        acc[0][r][x % 3] = __fmul2_rn(v[0][r], wa[t]);
                        acc[1][r][x % 3] = __fmul2_rn(v[1][r], wg[t]);
                    } else {
                        acc[0][r][x % 3] = __ffma2_rn(v[0][r + dy], wa[t], acc[0][r][x % 3]);
                        acc[1][r][x % 3] = __ffma2_rn(v[1][r + dy], wg[t], acc[1][r][x % 3]);
                    }
                }
            }
        }
        const int xd = j - 2;                               // the output completed by this column
        if (xd >= 0) {
#pragma unroll
            for (int r = 0; r < RPW; ++r) {
                const float2 a = acc[0][r][xd % 3], g = acc[1][r][xd % 3];
                // sigmoid(g) = 1 / (1 + 2^(-g log2 e))
                const float2 t = __fmul2_rn(g, make_float2(-kLog2e, -kLog2e));
                const float2 d = __fadd2_rn(make_float2(ptx::ex2_approx(t.x), ptx::ex2_approx(t.y)),
                                            make_float2(1.0f, 1.0f));
                const float2 z = __fmul2_rn(a, make_float2(ptx::rcp_approx(d.x), ptx::rcp_approx(d.y)));
                zo[r][xd] = float2_to_bf16x2(z.x, z.y);
            }
        }
    }
    __syncthreads();                                        // every warp is done with the input tile
    // output tile [row][column][64 channels] over the value half
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
        uint8_t* zt = dsm + ((size_t)(ly + r) * TX + sx) * (DW_CH * 2) + lane * 4;
#pragma unroll
        for (int x = 0; x < SX; ++x) *reinterpret_cast<uint32_t*>(zt + x * (DW_CH * 2)) = zo[r][x];
    }
    ptx::fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
        ptx::tma_store_4d(&tmZ, dsm, c0, x0, y0, b);
        ptx::bulk_commit_group();
        ptx::bulk_wait_group<0>();                          // written before the CTA retires
    }
}

}  // namespace tc
}  // namespace sana
