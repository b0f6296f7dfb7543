// Tensor-core (tcgen05) kernels of the split-N forward for sm_100a.
//
// KS  ks_state_tc   partial states  phi(K)^T [V | 1]  on UMMA, fp32 in TMEM
// KR  kr_reduce_tc  fixed-order sum of the partials of each (b, h)
// KA  ka_apply_tc   phi(Q) S on UMMA (S split into bf16 hi + lo), then
//                   O = num / (den + eps) in the epilogue
//
// The two contractions ("08_sana高效高分辨率生成", "Linear Attention 的原理":
// KV = phi(K)^T V, A = phi(Q) KV; the normaliser of the normalised form in
// "linear-diffusion-transformer-4k-efficient-generation", "核心架构") are dense
// products, so they run on the tensor cores; everything else rides along:
// phi is applied to the staged tiles in shared memory, the ones column of
// [V | 1] is a constant ones operand, and the division happens once per
// token-head in the epilogue (the fusions listed in the Sana walk-through's
// section "Triton을 통한 학습/추론 가속화", done here for sm_100a).
//
// Layout of a group: G = 128 / d heads, i.e. 128 consecutive elements (256 B)
// of a token row. TMA moves one group row of a tile as two 128-byte-wide boxes
// with the 128-byte swizzle.
//
// Warp roles (192 threads, one CTA per SM):
//   warps 0-3  workers: phi on the staged tile, state staging (KA), epilogue
//   warp  4    TMA producer (one lane)
//   warp  5    UMMA issuer (one lane)
// Every mbarrier wait is bounded; a wait that runs out sets an error code and
// the whole CTA winds down (drains its TMA loads and UMMAs, frees TMEM).
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"

namespace sana {
namespace tc {

constexpr int kWorkerThreads = 128;
constexpr int kThreads = kWorkerThreads + 64;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr uint32_t kTmemCols = 512;
constexpr int kBoxBytesRow = 128;            // one swizzled row of a box

__device__ uint32_t g_device_error;          // first error code seen by any kernel

struct SharedCtl {
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// phi on n16 16-byte chunks starting at base; thread t takes chunks t, t+128, ...
__device__ __forceinline__ void relu_smem(uint8_t* base, int n16, int tid) {
    for (int c = tid; c < n16; c += kWorkerThreads) {
        uint4* p = reinterpret_cast<uint4*>(base + (size_t)c * 16);
        uint4 v = *p;
        v.x = relu_bf16x2(v.x);
        v.y = relu_bf16x2(v.y);
        v.z = relu_bf16x2(v.z);
        v.w = relu_bf16x2(v.w);
        *p = v;
    }
}

// ===================================================================== KS ===
//
// Work split: the (b, group) slabs are cut into 64-token tiles, numbered
// t = bg * tiles_per_bg + tile. CTA c takes tiles [c*T/grid, (c+1)*T/grid);
// each run of its tiles that belongs to one bg is a "segment" and yields one
// partial state per head, at slot (c * max_seg + k) with k = bg - first bg of c.
// The reduction kernel sums a bg's segments in ascending c, i.e. token order.
struct KsParams {
    int N, H, groups, tiles_per_bg, grid, max_seg;
    long long total_tiles;
};

__host__ __device__ __forceinline__ long long ks_tile_begin(long long c, const KsParams& p) {
    return c * p.total_tiles / p.grid;
}

// the CTA whose range holds tile t
__host__ __device__ __forceinline__ long long ks_cta_of(long long t, const KsParams& p) {
    return ((t + 1) * p.grid - 1) / p.total_tiles;
}

constexpr int KS_TILE = 64;                                // tokens per stage
constexpr int KS_STAGES = 5;
constexpr int KS_BOX_BYTES = KS_TILE * kBoxBytesRow;       // 8 KB
constexpr int KS_STAGE_BYTES = 4 * KS_BOX_BYTES;           // K0 K1 V0 V1
constexpr int KS_ONES_OFF = KS_STAGES * KS_STAGE_BYTES;
constexpr int KS_BAR_OFF = KS_ONES_OFF + 1024;
constexpr int KS_NUM_BARS = 3 * KS_STAGES + 5;
constexpr int KS_CTL_OFF = KS_BAR_OFF + KS_NUM_BARS * 8;
constexpr int KS_SMEM_BYTES = KS_CTL_OFF + 64 + 1024;      // + alignment slack

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
ks_state_tc(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
            const KsParams p, float* __restrict__ partial)
{
    constexpr int G = 128 / D;
    constexpr int DD = D * (D + 1);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + KS_BAR_OFF);
    uint64_t* full = bars;
    uint64_t* empty = bars + KS_STAGES;
    uint64_t* relu_done = bars + 2 * KS_STAGES;
    uint64_t* acc_full = bars + 3 * KS_STAGES;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* mma_done = acc_full + 4;
    SharedCtl* ctl = reinterpret_cast<SharedCtl*>(smem + KS_CTL_OFF);
    volatile int* abort = &ctl->abort;
    uint32_t* err = &g_device_error;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const long long t_begin = ks_tile_begin(blockIdx.x, p);
    const int ntiles = (int)(ks_tile_begin(blockIdx.x + 1, p) - t_begin);
    const long long bg_first = t_begin / p.tiles_per_bg;

    if (tid == 0) {
        for (int s = 0; s < KS_STAGES; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
            ptx::mbar_init(&relu_done[s], kWorkerThreads);
        }
        for (int a = 0; a < 2; ++a) {
            ptx::mbar_init(&acc_full[a], 1);
            ptx::mbar_init(&acc_empty[a], kWorkerThreads);
        }
        ptx::mbar_init(mma_done, 1);
        ctl->abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0) {
        ptx::tmem_alloc(&ctl->tmem_base, kTmemCols);
        ptx::tmem_relinquish();
    }
    if (warp == kProducerWarp && lane == 0) {
        ptx::prefetch_tmap(&tmK);
        ptx::prefetch_tmap(&tmV);
    }
    // constant all-ones bf16 operand (16 tokens x 16 columns) for the normaliser column
    if (tid < 32) {
        uint4 ones = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
        reinterpret_cast<uint4*>(smem + KS_ONES_OFF)[tid] = ones;
        ptx::fence_proxy_async_smem();
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = ctl->tmem_base;

    auto stage_ptr = [&](int s) { return smem + (size_t)s * KS_STAGE_BYTES; };

    if (warp == kProducerWarp) {
        // ------------------------------------------------ TMA producer ----
        if (lane == 0) {
            int issued = 0;
            for (int i = 0; i < ntiles; ++i) {
                const int s = i % KS_STAGES;
                if (!ptx::mbar_wait(&empty[s], ((i / KS_STAGES) & 1) ^ 1, abort, err)) break;
                const long long t = t_begin + i;
                const long long bg = t / p.tiles_per_bg;
                const int tile = (int)(t % p.tiles_per_bg);
                const int b = (int)(bg / p.groups);
                const int g = (int)(bg % p.groups);
                const int x0 = g * 128;
                const int y = tile * KS_TILE;
                uint8_t* st = stage_ptr(s);
                ptx::mbar_arrive_expect_tx(&full[s], KS_STAGE_BYTES);
                ptx::tma_load_3d(st + 0 * KS_BOX_BYTES, &tmK, &full[s], x0, y, b);
                ptx::tma_load_3d(st + 1 * KS_BOX_BYTES, &tmK, &full[s], x0 + 64, y, b);
                ptx::tma_load_3d(st + 2 * KS_BOX_BYTES, &tmV, &full[s], x0, y, b);
                ptx::tma_load_3d(st + 3 * KS_BOX_BYTES, &tmV, &full[s], x0 + 64, y, b);
                issued = i + 1;
            }
            // drain: every issued load must land before the CTA may exit
            for (int i = (issued > KS_STAGES ? issued - KS_STAGES : 0); i < issued; ++i)
                ptx::mbar_wait(&full[i % KS_STAGES], (i / KS_STAGES) & 1, nullptr, err);
        }
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------- UMMA issuer ----
        if (lane == 0) {
            constexpr uint32_t idesc_v = ptx::idesc_bf16_f32(128, 128, 1, 1);
            constexpr uint32_t idesc_1 = ptx::idesc_bf16_f32(128, 16, 1, 1);
            const uint64_t ones_desc =
                ptx::smem_desc(ptx::smem_u32(smem + KS_ONES_OFF), 256, 128, ptx::kLayoutNone);
            int seg = -1;
            bool first = true;
            bool ok = true;
            for (int i = 0; i < ntiles && ok; ++i) {
                const long long t = t_begin + i;
                const long long bg = t / p.tiles_per_bg;
                const bool seg_start = (i == 0) || ((t - 1) / p.tiles_per_bg != bg);
                const bool seg_end = (i == ntiles - 1) || ((t + 1) / p.tiles_per_bg != bg);
                if (seg_start) {
                    ++seg;
                    if (!ptx::mbar_wait(&acc_empty[seg & 1], ((seg >> 1) & 1) ^ 1, abort, err)) break;
                    ptx::tc_fence_after_sync();
                    first = true;
                }
                const int s = i % KS_STAGES;
                if (!ptx::mbar_wait(&relu_done[s], (i / KS_STAGES) & 1, abort, err)) break;
                ptx::tc_fence_after_sync();
                const uint32_t d_tmem = tmem + (uint32_t)(seg & 1) * 256u;
                const uint32_t k_addr = ptx::smem_u32(stage_ptr(s));
                const uint32_t v_addr = k_addr + 2 * KS_BOX_BYTES;
#pragma unroll
                for (int ks = 0; ks < KS_TILE / 16; ++ks) {
                    // 16 tokens = two 8-row groups of 1024 B in the swizzled tile
                    const uint64_t a = ptx::smem_desc(k_addr + ks * 2048, KS_BOX_BYTES, 1024,
                                                      ptx::kLayoutSW128);
                    const uint64_t bv = ptx::smem_desc(v_addr + ks * 2048, KS_BOX_BYTES, 1024,
                                                       ptx::kLayoutSW128);
                    const bool acc = !(first && ks == 0);
                    ptx::umma_f16_ss(d_tmem, a, bv, idesc_v, acc);
                    ptx::umma_f16_ss(d_tmem + 128, a, ones_desc, idesc_1, acc);
                }
                first = false;
                ptx::umma_commit(&empty[s]);
                if (seg_end) ptx::umma_commit(&acc_full[seg & 1]);
            }
            ptx::umma_commit(mma_done);
            ptx::mbar_wait(mma_done, 0, nullptr, err);
        }
    } else {
        // --------------------------------------------------------- workers ----
        int seg = -1;
        for (int i = 0; i < ntiles; ++i) {
            const long long t = t_begin + i;
            const long long bg = t / p.tiles_per_bg;
            const bool seg_end = (i == ntiles - 1) || ((t + 1) / p.tiles_per_bg != bg);
            if (i == 0 || (t - 1) / p.tiles_per_bg != bg) ++seg;
            const int s = i % KS_STAGES;
            if (!ptx::mbar_wait(&full[s], (i / KS_STAGES) & 1, abort, err)) break;
            relu_smem(stage_ptr(s), 2 * KS_BOX_BYTES / 16, tid);      // phi on the K boxes only
            ptx::fence_proxy_async_smem();
            ptx::mbar_arrive(&relu_done[s]);
            if (seg_end) {
                // epilogue: this segment's partial states, TMEM -> workspace
                const int buf = seg & 1;
                if (!ptx::mbar_wait(&acc_full[buf], (seg >> 1) & 1, abort, err)) break;
                ptx::tc_fence_after_sync();
                const int hh = warp / (D / 32);                  // head within the group
                const int row = (warp % (D / 32)) * 32 + lane;   // state row i of that head
                const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)buf * 256u;
                float v[D], nrm;
                __syncwarp();
                ptx::tmem_ld_row<D>(lane_addr + hh * D, lane_addr + 128, v, &nrm);
                ptx::tc_fence_before_sync();
                ptx::mbar_arrive(&acc_empty[buf]);
                const int g = (int)(bg % p.groups);
                const int h = g * G + hh;
                if (h < p.H) {
                    const long long slot = ((long long)blockIdx.x * p.max_seg + (bg - bg_first)) * G + hh;
                    float* P = partial + slot * DD + (long long)row * (D + 1);
#pragma unroll
                    for (int j = 0; j < D; ++j) P[j] = v[j];
                    P[D] = nrm;
                }
            }
        }
    }

    ptx::tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        __syncwarp();
        ptx::tc_fence_after_sync();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

// ===================================================================== KR ===
template <int D>
__global__ void __launch_bounds__(256)
kr_reduce_tc(const float* __restrict__ partial, const KsParams p, float* __restrict__ state)
{
    constexpr int G = 128 / D;
    constexpr int DD = D * (D + 1);
    const long long bh = blockIdx.x;
    const int b = (int)(bh / p.H);
    const int h = (int)(bh % p.H);
    const int hh = h % G;
    const long long bg = (long long)b * p.groups + h / G;
    const long long c_lo = ks_cta_of(bg * p.tiles_per_bg, p);
    const long long c_hi = ks_cta_of(bg * p.tiles_per_bg + p.tiles_per_bg - 1, p);
    for (int e = threadIdx.x; e < DD; e += blockDim.x) {
        float s = 0.0f;
        for (long long c = c_lo; c <= c_hi; ++c) {
            const long long k = bg - ks_tile_begin(c, p) / p.tiles_per_bg;
            s += partial[((c * p.max_seg + k) * G + hh) * DD + e];
        }
        state[bh * DD + e] = s;
    }
}

// ===================================================================== KA ===
//
// Unit = (b, group, 128-token tile), numbered u = bg * tiles_per_bg + tile;
// CTA c takes units [c*U/grid, (c+1)*U/grid).
struct KaParams {
    int N, H, groups, tiles_per_bg, grid;
    long long total_units;
    float eps;
};

constexpr int KA_TILE = 128;                               // tokens = UMMA M
constexpr int KA_STAGES = 4;
constexpr int KA_BOX_BYTES = KA_TILE * kBoxBytesRow;       // 16 KB
constexpr int KA_STAGE_BYTES = 2 * KA_BOX_BYTES;           // one group row of 128 tokens

template <int D>
struct KaLayout {
    static constexpr int G = 128 / D;
    static constexpr int NA = D + 16;                      // UMMA N: d numerator cols + normaliser + pad
    static constexpr int SBO = (D / 8) * 128;              // 8-row group stride of the K-major state
    static constexpr int MAT_BYTES = (NA / 8) * SBO;       // one bf16 NA x D matrix
    static constexpr int STATE_BUF_BYTES = G * 2 * MAT_BYTES;   // hi and lo for every head
    static constexpr int STATE_OFF = KA_STAGES * KA_STAGE_BYTES;
    static constexpr int BAR_OFF = STATE_OFF + 2 * STATE_BUF_BYTES;
    static constexpr int NUM_BARS = 3 * KA_STAGES + 5;
    static constexpr int CTL_OFF = BAR_OFF + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = CTL_OFF + 64 + 1024;
    static constexpr int ACC_COLS = 256 / G;               // TMEM columns per head
};

// element (n, k) of a K-major, unswizzled bf16 matrix made of 8x8 core matrices
template <int D>
__device__ __forceinline__ int state_off(int n, int k) {
    return (n >> 3) * KaLayout<D>::SBO + (k >> 3) * 128 + (n & 7) * 16 + (k & 7) * 2;
}

template <int D, bool OUT_BF16>
__global__ void __launch_bounds__(kThreads, 1)
ka_apply_tc(const __grid_constant__ CUtensorMap tmQ, const KaParams p,
            const float* __restrict__ state, void* __restrict__ O)
{
    using L = KaLayout<D>;
    constexpr int G = L::G;
    constexpr int DD = D * (D + 1);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
    uint64_t* full = bars;
    uint64_t* empty = bars + KA_STAGES;
    uint64_t* relu_done = bars + 2 * KA_STAGES;
    uint64_t* acc_full = bars + 3 * KA_STAGES;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* mma_done = acc_full + 4;
    SharedCtl* ctl = reinterpret_cast<SharedCtl*>(smem + L::CTL_OFF);
    volatile int* abort = &ctl->abort;
    uint32_t* err = &g_device_error;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const long long u_begin = (long long)blockIdx.x * p.total_units / p.grid;
    const int nunits = (int)((long long)(blockIdx.x + 1) * p.total_units / p.grid - u_begin);

    if (tid == 0) {
        for (int s = 0; s < KA_STAGES; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
            ptx::mbar_init(&relu_done[s], kWorkerThreads);
        }
        for (int a = 0; a < 2; ++a) {
            ptx::mbar_init(&acc_full[a], 1);
            ptx::mbar_init(&acc_empty[a], kWorkerThreads);
        }
        ptx::mbar_init(mma_done, 1);
        ctl->abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0) {
        ptx::tmem_alloc(&ctl->tmem_base, kTmemCols);
        ptx::tmem_relinquish();
    }
    if (warp == kProducerWarp && lane == 0) ptx::prefetch_tmap(&tmQ);
    // padding columns n in (d, NA) of both state buffers are zero for good
    if (tid < kWorkerThreads) {
        for (int e = tid; e < 2 * G * 2 * (L::NA - D - 1) * D; e += kWorkerThreads) {
            const int k = e % D;
            const int n = D + 1 + (e / D) % (L::NA - D - 1);
            const int mat = e / (D * (L::NA - D - 1));
            *reinterpret_cast<__nv_bfloat16*>(smem + L::STATE_OFF + mat * L::MAT_BYTES +
                                              state_off<D>(n, k)) = __float2bfloat16_rn(0.0f);
        }
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = ctl->tmem_base;

    auto stage_ptr = [&](int s) { return smem + (size_t)s * KA_STAGE_BYTES; };
    auto state_buf = [&](int sb) { return smem + L::STATE_OFF + sb * L::STATE_BUF_BYTES; };

    if (warp == kProducerWarp) {
        // ------------------------------------------------ TMA producer ----
        if (lane == 0) {
            int issued = 0;
            for (int i = 0; i < nunits; ++i) {
                const int s = i % KA_STAGES;
                if (!ptx::mbar_wait(&empty[s], ((i / KA_STAGES) & 1) ^ 1, abort, err)) break;
                const long long u = u_begin + i;
                const long long bg = u / p.tiles_per_bg;
                const int tile = (int)(u % p.tiles_per_bg);
                const int b = (int)(bg / p.groups);
                const int x0 = (int)(bg % p.groups) * 128;
                ptx::mbar_arrive_expect_tx(&full[s], KA_STAGE_BYTES);
                ptx::tma_load_3d(stage_ptr(s), &tmQ, &full[s], x0, tile * KA_TILE, b);
                ptx::tma_load_3d(stage_ptr(s) + KA_BOX_BYTES, &tmQ, &full[s], x0 + 64, tile * KA_TILE, b);
                issued = i + 1;
            }
            for (int i = (issued > KA_STAGES ? issued - KA_STAGES : 0); i < issued; ++i)
                ptx::mbar_wait(&full[i % KA_STAGES], (i / KA_STAGES) & 1, nullptr, err);
        }
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------- UMMA issuer ----
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_bf16_f32(128, L::NA, 0, 0);
            int sb = -1;
            for (int i = 0; i < nunits; ++i) {
                const long long u = u_begin + i;
                const long long bg = u / p.tiles_per_bg;
                if (i == 0 || (u - 1) / p.tiles_per_bg != bg) ++sb;
                const int s = i % KA_STAGES;
                const int buf = i & 1;
                if (!ptx::mbar_wait(&relu_done[s], (i / KA_STAGES) & 1, abort, err)) break;
                if (!ptx::mbar_wait(&acc_empty[buf], ((i >> 1) & 1) ^ 1, abort, err)) break;
                ptx::tc_fence_after_sync();
                const uint32_t a_base = ptx::smem_u32(stage_ptr(s));
                const uint32_t s_base = ptx::smem_u32(state_buf(sb & 1));
#pragma unroll
                for (int hh = 0; hh < G; ++hh) {
                    const uint32_t d_tmem = tmem + (uint32_t)buf * 256u + (uint32_t)(hh * L::ACC_COLS);
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const int f = hh * D * 2 + ks * 32;       // byte offset in the group row
                        const uint64_t a = ptx::smem_desc(a_base + (f / 128) * KA_BOX_BYTES + (f % 128),
                                                          16, 1024, ptx::kLayoutSW128);
                        const uint32_t hi = s_base + (hh * 2 + 0) * L::MAT_BYTES + ks * 256;
                        const uint32_t lo = s_base + (hh * 2 + 1) * L::MAT_BYTES + ks * 256;
                        ptx::umma_f16_ss(d_tmem, a, ptx::smem_desc(hi, 128, L::SBO, ptx::kLayoutNone),
                                         idesc, ks > 0);
                        ptx::umma_f16_ss(d_tmem, a, ptx::smem_desc(lo, 128, L::SBO, ptx::kLayoutNone),
                                         idesc, true);
                    }
                }
                ptx::umma_commit(&empty[s]);
                ptx::umma_commit(&acc_full[buf]);
            }
            ptx::umma_commit(mma_done);
            ptx::mbar_wait(mma_done, 0, nullptr, err);
        }
    } else {
        // --------------------------------------------------------- workers ----
        int sb = -1;
        // stage unit i: (new state group ->) state hi/lo staging, then phi on the Q tile
        auto prep = [&](int i) -> bool {
            const long long u = u_begin + i;
            const long long bg = u / p.tiles_per_bg;
            if (i == 0 || (u - 1) / p.tiles_per_bg != bg) {
                ++sb;
                uint8_t* dst = state_buf(sb & 1);
                const int b = (int)(bg / p.groups);
                const int g = (int)(bg % p.groups);
                for (int hh = 0; hh < G; ++hh) {
                    const int h = g * G + hh;
                    const float* src = state + ((long long)b * p.H + h) * DD;
                    uint8_t* mhi = dst + (hh * 2 + 0) * L::MAT_BYTES;
                    uint8_t* mlo = dst + (hh * 2 + 1) * L::MAT_BYTES;
                    for (int e = tid; e < DD; e += kWorkerThreads) {
                        const int k = e / (D + 1);       // state row i = UMMA K index
                        const int n = e % (D + 1);       // state column j = UMMA N index
                        const float v = (h < p.H) ? src[e] : 0.0f;
                        const __nv_bfloat16 vh = __float2bfloat16_rn(v);
                        const __nv_bfloat16 vl = __float2bfloat16_rn(v - __bfloat162float(vh));
                        *reinterpret_cast<__nv_bfloat16*>(mhi + state_off<D>(n, k)) = vh;
                        *reinterpret_cast<__nv_bfloat16*>(mlo + state_off<D>(n, k)) = vl;
                    }
                }
            }
            const int s = i % KA_STAGES;
            if (!ptx::mbar_wait(&full[s], (i / KA_STAGES) & 1, abort, err)) return false;
            relu_smem(stage_ptr(s), KA_STAGE_BYTES / 16, tid);
            ptx::fence_proxy_async_smem();
            ptx::mbar_arrive(&relu_done[s]);
            return true;
        };
        bool ok = nunits > 0 ? prep(0) : true;
        for (int i = 0; i < nunits && ok; ++i) {
            if (i + 1 < nunits && !prep(i + 1)) break;
            // epilogue of unit i
            const int buf = i & 1;
            if (!ptx::mbar_wait(&acc_full[buf], (i >> 1) & 1, abort, err)) break;
            ptx::tc_fence_after_sync();
            const long long u = u_begin + i;
            const long long bg = u / p.tiles_per_bg;
            const int tile = (int)(u % p.tiles_per_bg);
            const int b = (int)(bg / p.groups);
            const int g = (int)(bg % p.groups);
            const long long n = (long long)tile * KA_TILE + warp * 32 + lane;
            const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)buf * 256u;
#pragma unroll 1
            for (int hh = 0; hh < G; ++hh) {
                float num[D], den;
                __syncwarp();
                ptx::tmem_ld_row<D>(lane_addr + hh * L::ACC_COLS, lane_addr + hh * L::ACC_COLS + D,
                                    num, &den);
                const int h = g * G + hh;
                if (n < p.N && h < p.H) {
                    const float r = 1.0f / (den + p.eps);
                    const long long off = (((long long)b * p.N + n) * p.H + h) * D;
                    if (OUT_BF16) {
                        __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(O) + off;
#pragma unroll
                        for (int j = 0; j < D; j += 8) {
                            uint4 w;
                            w.x = float2_to_bf16x2(num[j + 0] * r, num[j + 1] * r);
                            w.y = float2_to_bf16x2(num[j + 2] * r, num[j + 3] * r);
                            w.z = float2_to_bf16x2(num[j + 4] * r, num[j + 5] * r);
                            w.w = float2_to_bf16x2(num[j + 6] * r, num[j + 7] * r);
                            stg_stream(o + j, w);
                        }
                    } else {
                        float* o = reinterpret_cast<float*>(O) + off;
#pragma unroll
                        for (int j = 0; j < D; j += 4) {
                            uint4 w;
                            w.x = __float_as_uint(num[j + 0] * r);
                            w.y = __float_as_uint(num[j + 1] * r);
                            w.z = __float_as_uint(num[j + 2] * r);
                            w.w = __float_as_uint(num[j + 3] * r);
                            stg_stream(o + j, w);
                        }
                    }
                }
            }
            ptx::tc_fence_before_sync();
            ptx::mbar_arrive(&acc_empty[buf]);
        }
    }

    ptx::tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        __syncwarp();
        ptx::tc_fence_after_sync();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace tc
}  // namespace sana
