// Key-value projection with the state in its epilogue, for sm_100a.
//
// "SANA: Efficient High-Resolution Image Synthesis with Linear Diffusion
// Transformers" (phd-frog.tistory.com/40), section 4 "On-Device Deployment":
// the ReLU(K)^T V product of the linear attention is fused into the QKV
// projection, and the key-value projection stays in full precision. Here:
//   K = X Wk^T, V = X Wv^T  (bf16 in, fp32 accumulate on UMMA),
// rounded to bf16 (the values a stored K and V would hold), and
//   P = phi(K)^T [V | 1]   (the state kernel's product, on UMMA)
// accumulated per CTA, without writing K or V to memory. The partial states
// have the state kernel's layout, so kr_reduce_tc turns them into the state.
//
// Unit = one 128-token tile of a (b, group) slab, dealt out by the lockstep
// schedule of tc_kernels.cuh. Per unit:
//   producer  TMA: per 64-feature k-block, the X tile (128 tokens) and the
//             group's 128 rows of Wk and of Wv (K-major, 128-byte swizzle)
//   UMMA      GEMM D[128 x 256] = X [Wk_g; Wv_g]^T into TMEM columns 0-255
//   workers   D -> registers, bf16(K) -> phi, bf16(V), into staging tiles
//             laid out like the state kernel's TMA tiles (tokens as rows), one
//             64-token half after the other through the same 32 KB (so the
//             GEMM keeps 4 pipeline stages)
//   UMMA      state += phi(K)^T V and phi(K)^T 1 (TMEM columns 256-399) per
//             half, issued between the next unit's k-blocks
// At the end of a segment warps 0-3 write the partial states.
#pragma once

#include "tc_kernels.cuh"

namespace sana {
namespace tc {

struct KpParams {
    int N, H, groups;
    int C;            // input features
    int kblocks;      // ceil(C / 64)
    Sched q;          // slabs (b, group) x 128-token tiles
};

constexpr int KP_TILE = 128;                                // tokens per unit = GEMM M
constexpr int KP_BOX_BYTES = 128 * kBoxBytesRow;            // 128 rows x 128 bytes = 16 KB
constexpr int KP_STAGE_BYTES = 3 * KP_BOX_BYTES;            // X, Wk rows, Wv rows
constexpr int KP_STAGES = 4;
constexpr int KP_HALF = KP_TILE / 2;                        // tokens per staging half
constexpr int KP_HBOX_BYTES = KP_HALF * kBoxBytesRow;       // 64 token rows x 128 bytes = 8 KB
constexpr int KP_STG_OFF = KP_STAGES * KP_STAGE_BYTES;      // staging: phi(K) boxes 0/1, V boxes 0/1
constexpr int KP_ONES_OFF = KP_STG_OFF + 4 * KP_HBOX_BYTES;
constexpr int KP_DATA_BYTES = KP_ONES_OFF + 1024;
constexpr uint32_t KP_STATE_COL = 256;                      // state accumulator columns 256-399
// shared memory: data, 256 bytes of barriers, the control block, 1 KB of
// alignment slack (tighter than SmemMap to fit 4 stages)
struct KpMap {
    static constexpr int BAR_OFF = KP_DATA_BYTES;
    static constexpr int CTL_OFF = BAR_OFF + 256;
    static constexpr int BYTES = CTL_OFF + 64 + 1024;
    static_assert(BYTES <= kSmemLimit, "shared memory");
};

struct KpBars {
    uint64_t* full;        // [KP_STAGES] X and weight boxes landed
    uint64_t* empty;       // [KP_STAGES] read by the GEMM UMMAs
    uint64_t* acc_full;    // a unit's GEMM accumulator complete
    uint64_t* acc_empty;   // GEMM accumulator read by every worker warp
    uint64_t* staged;      // [2 halves] a half's phi(K) and V written by its 4 warps
    uint64_t* stg_free;    // [2 halves] the state UMMAs of a half have read the staging
    uint64_t* state_full;  // a segment's state accumulator complete
    uint64_t* state_empty; // state accumulator read by warps 0-3
    uint64_t* mma_done;
    __device__ void init() const {
        for (int s = 0; s < KP_STAGES; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        ptx::mbar_init(acc_full, 1);
        ptx::mbar_init(acc_empty, kWorkerWarps);
        for (int h = 0; h < 2; ++h) {
            ptx::mbar_init(&staged[h], kWorkerWarps / 2);
            ptx::mbar_init(&stg_free[h], 1);
        }
        ptx::mbar_init(state_full, 1);
        ptx::mbar_init(state_empty, 4);
        ptx::mbar_init(mma_done, 1);
    }
};

__device__ __forceinline__ KpBars kp_bars(uint64_t* b) {
    uint64_t* a = b + 2 * KP_STAGES;
    return KpBars{b, b + KP_STAGES, a, a + 1, a + 2, a + 4, a + 6, a + 7, a + 8};
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
kvproj_state_tc(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmWk,
                const __grid_constant__ CUtensorMap tmWv, const KpParams p, float* __restrict__ partial)
{
    constexpr int G = 128 / D;
    constexpr int DD = D * (D + 1);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    const KpBars bar = kp_bars(reinterpret_cast<uint64_t*>(smem + KpMap::BAR_OFF));
    SharedCtl* ctl = reinterpret_cast<SharedCtl*>(smem + KpMap::CTL_OFF);
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int cta = blockIdx.x;
    volatile int* abort = &ctl->abort;
    uint32_t* err = &g_device_error;
    if (tid == 0) {
        bar.init();
        ptx::fence_mbar_init();
    }
    kernel_prologue(ctl, tid);
    if (tid == kProducerWarp * 32) {
        ptx::prefetch_tmap(&tmX);
        ptx::prefetch_tmap(&tmWk);
        ptx::prefetch_tmap(&tmWv);
    }
    if (tid < 32) {
        // constant all-ones bf16 operand (16 tokens x 16 columns) for the normaliser column
        const uint4 ones = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
        reinterpret_cast<uint4*>(smem + KP_ONES_OFF)[tid] = ones;
        ptx::fence_proxy_async_smem();
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = ctl->tmem_base;

    const bool active = cta < p.q.grid;
    const int tps = active ? sched_tps(cta, p.q) : 0;
    const int nunits = active ? tps * sched_nseg(cta, p.q) : 0;
    auto stage_ptr = [&](int s) { return smem + (size_t)s * KP_STAGE_BYTES; };
    uint8_t* stg = smem + KP_STG_OFF;

    if (warp == kProducerWarp) {
        // ------------------------------------------------ TMA producer ----
        if (lane == 0) {
            int k = 0, issued = 0;
            for (int i = 0; i < nunits; ++i) {
                int slab, tile, seg;
                sched_item(cta, i, tps, p.q, slab, tile, seg);
                const int b = slab / p.groups;
                const int y_w = (slab % p.groups) * 128;
                bool ok = true;
                for (int kb = 0; kb < p.kblocks; ++kb, ++k) {
                    const int s = k % KP_STAGES;
                    if (!ptx::mbar_wait(&bar.empty[s], ((k / KP_STAGES) & 1) ^ 1, abort, err)) { ok = false; break; }
                    uint8_t* st = stage_ptr(s);
                    ptx::mbar_arrive_expect_tx(&bar.full[s], KP_STAGE_BYTES);
                    ptx::tma_load_3d(st, &tmX, &bar.full[s], kb * 64, tile * KP_TILE, b);
                    ptx::tma_load_3d(st + KP_BOX_BYTES, &tmWk, &bar.full[s], kb * 64, y_w, 0);
                    ptx::tma_load_3d(st + 2 * KP_BOX_BYTES, &tmWv, &bar.full[s], kb * 64, y_w, 0);
                    issued = k + 1;
                }
                if (!ok) break;
            }
            // drain: every issued load must land before the CTA may exit
            for (int j = (issued > KP_STAGES ? issued - KP_STAGES : 0); j < issued; ++j)
                ptx::mbar_wait(&bar.full[j % KP_STAGES], (j / KP_STAGES) & 1, nullptr, err);
        }
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------- UMMA issuer ----
        if (lane == 0) {
            constexpr uint32_t idesc_gemm = ptx::idesc_bf16_f32(128, 256, 0, 0);
            constexpr uint32_t idesc_v = ptx::idesc_bf16_f32(128, 128, 1, 1);
            constexpr uint32_t idesc_1 = ptx::idesc_bf16_f32(128, 16, 1, 1);
            const uint64_t ones_desc =
                ptx::smem_desc(ptx::smem_u32(smem + KP_ONES_OFF), 256, 128, ptx::kLayoutNone);
            const uint32_t kstg = ptx::smem_u32(stg);
            const uint32_t vstg = kstg + 2 * KP_HBOX_BYTES;
            // state UMMAs of half h of unit u: phi(K)^T [V | 1] over its 64 tokens
            auto issue_state = [&](int u, int h) -> bool {
                const int seg = u / tps;
                const bool first = (u % tps) == 0 && h == 0;
                if (first && seg > 0) {
                    // warps 0-3 have read the previous segment's state
                    if (!ptx::mbar_wait(bar.state_empty, (seg & 1) ^ 1, abort, err)) return false;
                }
                ptx::tc_fence_after_sync();
#pragma unroll
                for (int ks = 0; ks < KP_HALF / 16; ++ks) {
                    // 16 tokens = two 8-row groups of 1024 B in the swizzled tiles
                    const uint64_t a = ptx::smem_desc(kstg + ks * 2048, KP_HBOX_BYTES, 1024, ptx::kLayoutSW128);
                    const uint64_t bv = ptx::smem_desc(vstg + ks * 2048, KP_HBOX_BYTES, 1024, ptx::kLayoutSW128);
                    const bool acc = !(first && ks == 0);
                    ptx::umma_f16_ss(tmem + KP_STATE_COL, a, bv, idesc_v, acc);
                    ptx::umma_f16_ss(tmem + KP_STATE_COL + 128, a, ones_desc, idesc_1, acc);
                }
                ptx::umma_commit(&bar.stg_free[h]);
                if (h == 1 && (u % tps) == tps - 1) ptx::umma_commit(bar.state_full);
                return true;
            };
            int k = 0;
            int pending = -1;              // unit whose state halves are still to issue
            int pending_h = 0;             // its next half
            bool ok = true;
            for (int i = 0; i < nunits && ok; ++i) {
                // the workers have read the previous unit's accumulator
                if (!ptx::mbar_wait(bar.acc_empty, (i & 1) ^ 1, abort, err)) { ok = false; break; }
                ptx::tc_fence_after_sync();
                for (int kb = 0; kb < p.kblocks; ++kb, ++k) {
                    const int s = k % KP_STAGES;
                    if (!ptx::mbar_wait(&bar.full[s], (k / KP_STAGES) & 1, abort, err)) { ok = false; break; }
                    ptx::tc_fence_after_sync();
                    const uint32_t a0 = ptx::smem_u32(stage_ptr(s));
                    const uint32_t b0 = a0 + KP_BOX_BYTES;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        // K-major, 128-byte swizzle: 16 features = 32 bytes along the row
                        const uint64_t a = ptx::smem_desc(a0 + kk * 32, 16, 1024, ptx::kLayoutSW128);
                        const uint64_t bw = ptx::smem_desc(b0 + kk * 32, 16, 1024, ptx::kLayoutSW128);
                        ptx::umma_f16_ss(tmem, a, bw, idesc_gemm, (kb | kk) != 0);
                    }
                    ptx::umma_commit(&bar.empty[s]);
                    if (pending >= 0 && ptx::mbar_test_wait(&bar.staged[pending_h], pending & 1)) {
                        if (!issue_state(pending, pending_h)) { ok = false; break; }
                        if (++pending_h == 2) { pending = -1; pending_h = 0; }
                    }
                }
                if (!ok) break;
                ptx::umma_commit(bar.acc_full);
                while (ok && pending >= 0) {
                    if (!ptx::mbar_wait(&bar.staged[pending_h], pending & 1, abort, err) ||
                        !issue_state(pending, pending_h)) {
                        ok = false;
                        break;
                    }
                    if (++pending_h == 2) { pending = -1; pending_h = 0; }
                }
                if (!ok) break;
                pending = i;
                pending_h = 0;
            }
            while (ok && pending >= 0) {
                if (!ptx::mbar_wait(&bar.staged[pending_h], pending & 1, abort, err) ||
                    !issue_state(pending, pending_h))
                    break;
                if (++pending_h == 2) pending = -1;
            }
            ptx::umma_commit(bar.mma_done);
            ptx::mbar_wait(bar.mma_done, 0, nullptr, err);
        }
    } else {
        // --------------------------------------------------------- workers ----
        // Warp w reads TMEM lanes 32*(w%4).. (its 32 tokens) and half w/4 of the
        // accumulator: columns 0-127 (K) or 128-255 (V).
        const int t = (warp & 3) * 32 + lane;           // token row of the tile
        const int half = warp >> 2;                     // 0: K columns, 1: V columns
        const int th = (warp & 3) >> 1;                 // token half of this warp
        const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        for (int i = 0; i < nunits; ++i) {
            if (!warp_wait(bar.acc_full, i & 1, abort, err)) break;
            ptx::tc_fence_after_sync();
            float v[128];
            __syncwarp();
#pragma unroll
            for (int c = 0; c < 4; ++c) ptx::tmem_ld32(lane_base + (uint32_t)(half * 128 + c * 32), v + c * 32);
            ptx::tc_fence_before_sync();
            warp_arrive(bar.acc_empty);
            // the staging's previous contents must have been read by the state
            // UMMAs: the other token half of the previous unit for half 0, half
            // 0 of this unit for half 1
            const bool free_ok = th == 0 ? warp_wait(&bar.stg_free[1], (i & 1) ^ 1, abort, err)
                                         : warp_wait(&bar.stg_free[0], i & 1, abort, err);
            if (!free_ok) break;
            // bf16 as a stored projection would hold it; phi = ReLU on K (it
            // commutes with the rounding)
            const int row = t & (KP_HALF - 1);
            uint8_t* base = stg + half * 2 * KP_HBOX_BYTES + row * kBoxBytesRow;
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const float* x = v + q * 8;
                uint4 w;
                if (half == 0) {
                    w.x = relu_bf16x2(float2_to_bf16x2(x[0], x[1]));
                    w.y = relu_bf16x2(float2_to_bf16x2(x[2], x[3]));
                    w.z = relu_bf16x2(float2_to_bf16x2(x[4], x[5]));
                    w.w = relu_bf16x2(float2_to_bf16x2(x[6], x[7]));
                } else {
                    w.x = float2_to_bf16x2(x[0], x[1]);
                    w.y = float2_to_bf16x2(x[2], x[3]);
                    w.z = float2_to_bf16x2(x[4], x[5]);
                    w.w = float2_to_bf16x2(x[6], x[7]);
                }
                // features 64*(q/8).. in box q/8; 16-byte chunk q%8 of the row at (q%8) ^ (row%8)
                *reinterpret_cast<uint4*>(base + (q >> 3) * KP_HBOX_BYTES + (((q & 7) ^ (row & 7)) * 16)) = w;
            }
            ptx::fence_proxy_async_smem();
            warp_arrive(&bar.staged[th]);
            if ((i % tps) == tps - 1 && warp < 4) {
                // end of a segment: the partial states, TMEM -> workspace
                const int seg = i / tps;
                if (!warp_wait(bar.state_full, seg & 1, abort, err)) break;
                ptx::tc_fence_after_sync();
                const int hh = warp / (D / 32);                  // head within the group
                const int row = (warp % (D / 32)) * 32 + lane;   // state row of that head
                const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16) + KP_STATE_COL;
                float sv[D], nrm;
                __syncwarp();
                ptx::tmem_ld_row<D>(lane_addr + hh * D, lane_addr + 128, sv, &nrm);
                ptx::tc_fence_before_sync();
                warp_arrive(bar.state_empty);
                int slab, tile, sg;
                sched_item(cta, i, tps, p.q, slab, tile, sg);
                const int h = (slab % p.groups) * G + hh;
                if (h < p.H) {
                    // the state kernel's layout: by columns, column j at j * D
                    const long long slot = ((long long)cta * p.q.max_seg + seg) * G + hh;
                    float* P = partial + slot * DD + row;
#pragma unroll
                    for (int j = 0; j < D; ++j) P[j * D] = sv[j];
                    P[D * D] = nrm;
                }
            }
        }
    }
    kernel_epilogue(ctl, tid);
}

}  // namespace tc
}  // namespace sana
