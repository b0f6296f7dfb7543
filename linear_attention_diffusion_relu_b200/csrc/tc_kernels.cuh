// Tensor-core (tcgen05) kernels of the split-N forward for sm_100a.
//
// KS  ks_state_tc   partial states  phi(K)^T [V | 1]  on UMMA, fp32 in TMEM
// KR  kr_reduce_tc  fixed-order sum of the partials of each (b, h)
//     kr_prefix_tc  block-causal: fixed-order prefix sums over token blocks
// KA  ka_apply_tc   phi(Q) S on UMMA (S split into bf16 hi + lo), then
//                   O = num / (den + eps) in the epilogue, stored by TMA
// KF  fwd_fused_tc  KS, per-slab readiness flags and KA in one cooperative launch
//
// The feature map phi is a template parameter (ReLU, ELU+1, cos; the latter
// two carried as bf16 hi + lo pairs); the block-causal form is a runtime
// property of the schedule (see below).
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
// Warp roles (320 threads, one CTA per SM):
//   warps 0-7  workers: phi on the staged tile, state staging (KA), epilogue;
//              warps w and w+4 share TMEM lanes 32*(w%4).. and split the heads
//   warp  8    TMA producer (one lane)
//   warp  9    UMMA issuer (one lane)
//
// Schedule ("lockstep"): the B*groups (b, group) slabs are dealt out so that
// the CTAs running at the same time read the same token rows of every group,
// i.e. whole contiguous rows of Q, K and V, instead of 256-byte pieces of
// unrelated rows; on B200 that raised the HBM throughput of both kernels by
// 25-50 %. With S slabs and one CTA per SM (`sms` of them) there are P
// positions; CTA c works on the slabs c % P, c % P + P, ...:
//   S <= sms: P = S and R = min(sms / S, tiles) CTAs share a slab; CTA c takes
//             slab c % S and its tiles r, r + R, r + 2R, ... with r = c / S.
//   S >  sms: P = sms, R = 1: CTA c takes slabs c, c + sms, ... whole.
// Each (CTA, slab) pair is one "segment"; KS writes one partial state per
// segment and KR adds a slab's segments in ascending CTA order. (Taking the
// slabs in two sets, one batch after the other with twice the CTAs per slab,
// so that one set's reduction could overlap the other's loads, made the state
// phase's reads 15 % slower on B200: 54 vs 47 us for the 4096px keys and
// values in a load-only probe, more than the overlap saved.)
//
// Block-causal form (blocks of L tokens, L a multiple of 128): the tiles of a
// slab are padded to whole blocks, and its R = Rb * Rt CTAs split the blocks
// first: CTA r takes blocks r % Rb, r % Rb + Rb, ... and, of each, the tiles
// r / Rb, r / Rb + Rt, ... (Rt divides the tiles per block, so every CTA takes
// tpb of them; tiles past N read as zeros and are not stored). A segment is
// then one (slab, block) pair: KS writes one partial per (CTA, slab, block),
// KR turns them into prefix states (ascending blocks, within a block the Rt
// partials in ascending r), and KA stages the prefix state of a segment's
// block once for its tpb tiles.
// Every mbarrier wait is bounded; a wait that runs out sets an error code and
// the whole CTA winds down (drains its TMA loads and UMMAs, frees TMEM).
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"

namespace sana {
namespace tc {

constexpr int kWorkerThreads = 256;
constexpr int kWorkerWarps = kWorkerThreads / 32;
constexpr int kThreads = kWorkerThreads + 64;
constexpr int kProducerWarp = kWorkerWarps;
constexpr int kMmaWarp = kWorkerWarps + 1;
constexpr uint32_t kTmemCols = 512;
constexpr int kBoxBytesRow = 128;            // one swizzled row of a box
constexpr int kSmemLimit = 232448;           // dynamic shared memory per CTA on sm_100

__device__ uint32_t g_device_error;          // first error code seen by any kernel

struct SharedCtl {
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// phi on N16 16-byte chunks at base; worker t takes chunks t, t+128, ...
// All loads are issued before the stores so they overlap.
template <int N16>
__device__ __forceinline__ void relu_smem(uint8_t* base, int tid) {
    constexpr int PER = N16 / kWorkerThreads;
    static_assert(N16 % kWorkerThreads == 0, "whole chunks per worker");
    uint4 v[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) v[j] = *reinterpret_cast<const uint4*>(base + (size_t)(tid + j * kWorkerThreads) * 16);
#pragma unroll
    for (int j = 0; j < PER; ++j) {
        v[j].x = relu_bf16x2(v[j].x);
        v[j].y = relu_bf16x2(v[j].y);
        v[j].z = relu_bf16x2(v[j].z);
        v[j].w = relu_bf16x2(v[j].w);
        *reinterpret_cast<uint4*>(base + (size_t)(tid + j * kWorkerThreads) * 16) = v[j];
    }
}

// phi on the K boxes of a state-phase stage (N16 16-byte chunks of 128-byte
// rows, one token per row), split: hi in place, lo to the same offsets at
// lo_base. Rows at or past `valid_rows` are tokens past N, which TMA filled
// with zeros; phi(0) is not 0 for these feature maps, so they are written as
// zeros. Worker t takes chunks t, t+256, ...
template <int FM, int N16, int BOX_ROWS>
__device__ __forceinline__ void feature_split_smem(uint8_t* base, uint8_t* lo_base, int valid_rows, int tid) {
    constexpr int PER = N16 / kWorkerThreads;
    static_assert(N16 % kWorkerThreads == 0, "whole chunks per worker");
    uint4 v[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) v[j] = *reinterpret_cast<const uint4*>(base + (size_t)(tid + j * kWorkerThreads) * 16);
#pragma unroll
    for (int j = 0; j < PER; ++j) {
        const int c = tid + j * kWorkerThreads;
        const int row = (c % (BOX_ROWS * 8)) / 8;     // 8 chunks per 128-byte row, one box after the other
        uint4 h = make_uint4(0u, 0u, 0u, 0u), l = make_uint4(0u, 0u, 0u, 0u);
        if (row < valid_rows) {
            feature_split_bf16x2<FM>(v[j].x, h.x, l.x);
            feature_split_bf16x2<FM>(v[j].y, h.y, l.y);
            feature_split_bf16x2<FM>(v[j].z, h.z, l.z);
            feature_split_bf16x2<FM>(v[j].w, h.w, l.w);
        }
        *reinterpret_cast<uint4*>(base + (size_t)c * 16) = h;
        *reinterpret_cast<uint4*>(lo_base + (size_t)c * 16) = l;
    }
}

// Bounded wait whose outcome is the same for every lane of the warp: if any
// lane gives up, all do. Worker code paths stay warp-uniform this way, so a
// wind-down never leaves part of a warp at a warp-synchronous instruction.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          uint32_t* err) {
    const bool ok = ptx::mbar_wait(bar, parity, abort, err);
    return __all_sync(0xffffffffu, ok);
}

// One arrival per worker warp (barriers are initialised with kWorkerWarps).
// Each lane has already fenced its own writes; __syncwarp orders them before
// lane 0's arrive, which releases them to the waiting thread.
__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) ptx::mbar_arrive(bar);
}

// =============================================================== schedule ===
struct Sched {
    int S;          // (b, group) slabs = B * groups
    int P;          // positions: CTA c works on slabs c % P + j P, j = 0, 1, ...
    int T;          // tiles per slab (block-causal: padded to whole blocks)
    int R;          // CTAs sharing one position
    int grid;       // CTAs = P * R
    int max_seg;    // most segments one CTA visits
    int nblk;       // token blocks per slab (1 = not block-causal)
    int tpb;        // block-causal: tiles of one block per CTA (0 otherwise)
    int rb;         // block-causal: CTAs of a slab that split its blocks (R / rb split each block)
};

// tiles per segment of CTA c
__host__ __device__ __forceinline__ int sched_tps(int c, const Sched& q) {
    if (q.tpb > 0) return q.tpb;
    const int r = c / q.P;
    return (q.T - r + q.R - 1) / q.R;
}
// blocks of one slab that CTA c visits (1 unless block-causal)
__host__ __device__ __forceinline__ int sched_nb(int c, const Sched& q) {
    if (q.rb == 1) return q.nblk;
    const int rb = (c / q.P) % q.rb;
    return (q.nblk - rb + q.rb - 1) / q.rb;
}
// slabs (sets) of CTA c
__host__ __device__ __forceinline__ int sched_nslab(int c, const Sched& q) {
    return (q.S - c % q.P + q.P - 1) / q.P;
}
// segments of CTA c: its slabs times the blocks it visits in each
__host__ __device__ __forceinline__ int sched_nseg(int c, const Sched& q) {
    return sched_nslab(c, q) * sched_nb(c, q);
}
// token block of segment `seg` of CTA c
__host__ __device__ __forceinline__ int sched_block(int c, int seg, const Sched& q) {
    if (q.rb == 1) return seg % q.nblk;
    return (c / q.P) % q.rb + (seg % sched_nb(c, q)) * q.rb;
}
// i-th tile of CTA c -> (slab, tile, segment index). In round k the R CTAs of
// a slab take tiles kR .. kR + R - 1, CTA r always position r.
// (Rotating the positions from round to round made every CTA finish the state
// phase together, but all of them at the time the last position finished
// before: slower overall, measured on B200.) Block-causal: see the comment at
// the top.
__host__ __device__ __forceinline__ void sched_item(int c, int i, int tps, const Sched& q,
                                                    int& slab, int& tile, int& seg) {
    seg = i / tps;
    const int r = c / q.P;
    if (q.rb == 1) {
        // every CTA of the slab in every block (and the plain forward): the
        // general form below with rb = 1, in fewer divisions
        slab = c % q.P + seg / q.nblk * q.P;
        tile = r + ((seg % q.nblk) * tps + i % tps) * q.R;
        return;
    }
    slab = c % q.P + seg / sched_nb(c, q) * q.P;
    tile = sched_block(c, seg, q) * (q.T / q.nblk) + r / q.rb + (i % tps) * (q.R / q.rb);
}

// ===================================================================== KS ===
struct KsParams {
    int N, H, groups;
    Sched q;
};

// A partial state (one per CTA segment and head) is stored by columns: entry
// (i, j) of phi(K)^T [V | 1] (state row i, column j; j = d the normaliser) at
// j * d + i. A warp that holds 32 rows of one column in its lanes (the TMEM
// read-out) then stores 128 contiguous bytes per instruction, where the
// state's row-major layout made every lane write its own cache line.

constexpr int KS_TILE = 64;                                // tokens per stage
constexpr int KS_STAGES = 6;                               // stages with phi = ReLU
constexpr int KS_BOX_BYTES = KS_TILE * kBoxBytesRow;       // 8 KB
constexpr int KS_STAGE_BYTES = 4 * KS_BOX_BYTES;           // K0 K1 V0 V1
constexpr int KS_ONES_OFF = KS_STAGES * KS_STAGE_BYTES;
constexpr int KS_DATA_BYTES = KS_ONES_OFF + 1024;          // stages + the ones tile
constexpr int KS_NUM_BARS = 3 * KS_STAGES + 5;
// Other feature maps need phi(K) as bf16 hi + lo: 4 stages, and after them a
// lo copy of each stage's two K boxes (same swizzled layout), in the same bytes.
constexpr int KS_STAGES_SPLIT = 4;
constexpr int KS_LO_OFF = KS_STAGES_SPLIT * KS_STAGE_BYTES;
constexpr int KS_LO_BYTES = 2 * KS_BOX_BYTES;
static_assert(KS_LO_OFF + KS_STAGES_SPLIT * KS_LO_BYTES == KS_ONES_OFF, "split layout fits the ReLU one");

template <int FM>
__host__ __device__ constexpr int ks_stages() { return FM == kFeatureRelu ? KS_STAGES : KS_STAGES_SPLIT; }

struct KsBars {
    uint64_t* full;        // [KS_STAGES] K and V tiles landed
    uint64_t* empty;       // [KS_STAGES] tiles read by the UMMAs
    uint64_t* relu_done;   // [KS_STAGES] phi applied to the K tile
    uint64_t* acc_full;    // [2] a segment's accumulator complete
    uint64_t* acc_empty;   // [2] accumulator read by the epilogue warps 0-3
    uint64_t* mma_done;
    __device__ void init() const {
        for (int s = 0; s < KS_STAGES; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
            ptx::mbar_init(&relu_done[s], kWorkerWarps);
        }
        for (int a = 0; a < 2; ++a) {
            ptx::mbar_init(&acc_full[a], 1);
            ptx::mbar_init(&acc_empty[a], 4);
        }
        ptx::mbar_init(mma_done, 1);
    }
};

__device__ __forceinline__ KsBars ks_bars(uint64_t* b) {
    return KsBars{b, b + KS_STAGES, b + 2 * KS_STAGES, b + 3 * KS_STAGES, b + 3 * KS_STAGES + 2,
                  b + 3 * KS_STAGES + 4};
}

__device__ __forceinline__ void ks_fill_ones(uint8_t* smem, int tid) {
    // constant all-ones bf16 operand (16 tokens x 16 columns) for the normaliser column
    if (tid < 32) {
        uint4 ones = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
        reinterpret_cast<uint4*>(smem + KS_ONES_OFF)[tid] = ones;
        ptx::fence_proxy_async_smem();
    }
}

// TMA loads of the state phase's tile i of CTA `cta` (K and V boxes of its
// group row) into stage `s`, completing on full[s].
__device__ __forceinline__ void ks_load_tile(const CUtensorMap* tmK, const CUtensorMap* tmV, const KsParams& p,
                                             int cta, int i, int tps, uint8_t* st, uint64_t* full,
                                             bool evict_first) {
    int slab, tile, seg;
    sched_item(cta, i, tps, p.q, slab, tile, seg);
    const int b = slab / p.groups;
    const int x0 = (slab % p.groups) * 128;
    const int y = tile * KS_TILE;
    ptx::mbar_arrive_expect_tx(full, KS_STAGE_BYTES);
    if (evict_first) {
        const uint64_t pol = ptx::l2_policy_evict_first();
        ptx::tma_load_3d_hint(st + 0 * KS_BOX_BYTES, tmK, full, x0, y, b, pol);
        ptx::tma_load_3d_hint(st + 1 * KS_BOX_BYTES, tmK, full, x0 + 64, y, b, pol);
        ptx::tma_load_3d_hint(st + 2 * KS_BOX_BYTES, tmV, full, x0, y, b, pol);
        ptx::tma_load_3d_hint(st + 3 * KS_BOX_BYTES, tmV, full, x0 + 64, y, b, pol);
    } else {
        ptx::tma_load_3d(st + 0 * KS_BOX_BYTES, tmK, full, x0, y, b);
        ptx::tma_load_3d(st + 1 * KS_BOX_BYTES, tmK, full, x0 + 64, y, b);
        ptx::tma_load_3d(st + 2 * KS_BOX_BYTES, tmV, full, x0, y, b);
        ptx::tma_load_3d(st + 3 * KS_BOX_BYTES, tmV, full, x0 + 64, y, b);
    }
}

// The state phase for CTA `cta`: partial states phi(K)^T [V | 1] of its
// segments into `partial`. Every role returns once its part is done. Stage s
// of this phase is free again once bar.empty[s] has completed the phase of the
// last tile that used it (the single-launch kernel's apply phase waits for
// that before it loads into the same bytes).
template <int D, int FM>
__device__ __forceinline__ void ks_phase(const CUtensorMap* tmK, const CUtensorMap* tmV, const KsParams& p,
                                         int cta, float* __restrict__ partial, uint8_t* smem,
                                         const KsBars& bar, uint32_t tmem, volatile int* abort,
                                         uint32_t* err, bool evict_first = false, int pre_issued = 0)
{
    constexpr int G = 128 / D;
    constexpr int DD = D * (D + 1);
    constexpr int NS = ks_stages<FM>();
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    if (cta >= p.q.grid) return;
    const int tps = sched_tps(cta, p.q);
    const int ntiles = tps * sched_nseg(cta, p.q);
    auto stage_ptr = [&](int s) { return smem + (size_t)s * KS_STAGE_BYTES; };
    auto lo_ptr = [&](int s) { return smem + KS_LO_OFF + (size_t)s * KS_LO_BYTES; };

    if (warp == kProducerWarp) {
        // ------------------------------------------------ TMA producer ----
        if (lane == 0) {
            // (tiles [0, pre_issued) were loaded by the caller, before its
            // CTA-wide sync, into their stages; pre_issued <= NS)
            int issued = min(pre_issued, ntiles);
            for (int i = issued; i < ntiles; ++i) {
                const int s = i % NS;
                if (!ptx::mbar_wait(&bar.empty[s], ((i / NS) & 1) ^ 1, abort, err)) break;
                ks_load_tile(tmK, tmV, p, cta, i, tps, stage_ptr(s), &bar.full[s], evict_first);
                issued = i + 1;
            }
            // drain: every issued load must land before the CTA may exit
            for (int i = (issued > NS ? issued - NS : 0); i < issued; ++i)
                ptx::mbar_wait(&bar.full[i % NS], (i / NS) & 1, nullptr, err);
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
            for (int i = 0; i < ntiles; ++i) {
                const bool seg_start = (i % tps) == 0;
                const bool seg_end = (i % tps) == tps - 1;
                if (seg_start) {
                    ++seg;
                    if (!ptx::mbar_wait(&bar.acc_empty[seg & 1], ((seg >> 1) & 1) ^ 1, abort, err)) break;
                    ptx::tc_fence_after_sync();
                    first = true;
                }
                const int s = i % NS;
                if (!ptx::mbar_wait(&bar.relu_done[s], (i / NS) & 1, abort, err)) break;
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
                    if constexpr (FM != kFeatureRelu) {
                        // the lo part of phi(K): phi(K)^T [V | 1] = hi^T [V | 1] + lo^T [V | 1]
                        const uint64_t al = ptx::smem_desc(ptx::smem_u32(lo_ptr(s)) + ks * 2048, KS_BOX_BYTES,
                                                           1024, ptx::kLayoutSW128);
                        ptx::umma_f16_ss(d_tmem, al, bv, idesc_v, true);
                        ptx::umma_f16_ss(d_tmem + 128, al, ones_desc, idesc_1, true);
                    }
                }
                first = false;
                ptx::umma_commit(&bar.empty[s]);
                if (seg_end) ptx::umma_commit(&bar.acc_full[seg & 1]);
            }
            ptx::umma_commit(bar.mma_done);
            ptx::mbar_wait(bar.mma_done, 0, nullptr, err);
        }
    } else {
        // --------------------------------------------------------- workers ----
        for (int i = 0; i < ntiles; ++i) {
            const bool seg_end = (i % tps) == tps - 1;
            const int seg = i / tps;
            const int s = i % NS;
            if (!warp_wait(&bar.full[s], (i / NS) & 1, abort, err)) break;
            if constexpr (FM == kFeatureRelu) {
                relu_smem<2 * KS_BOX_BYTES / 16>(stage_ptr(s), tid);     // phi on the K boxes only
            } else {
                int slab, tile, sg;
                sched_item(cta, i, tps, p.q, slab, tile, sg);
                feature_split_smem<FM, 2 * KS_BOX_BYTES / 16, KS_TILE>(stage_ptr(s), lo_ptr(s),
                                                                      p.N - tile * KS_TILE, tid);
            }
            ptx::fence_proxy_async_smem();
            warp_arrive(&bar.relu_done[s]);
            if (seg_end && warp < 4) {
                // epilogue (warps 0-3, one per TMEM lane quarter): this segment's
                // partial states, TMEM -> workspace
                const int buf = seg & 1;
                if (!warp_wait(&bar.acc_full[buf], (seg >> 1) & 1, abort, err)) break;
                ptx::tc_fence_after_sync();
                const int hh = warp / (D / 32);                  // head within the group
                const int row = (warp % (D / 32)) * 32 + lane;   // state row i of that head
                const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)buf * 256u;
                float v[D], nrm;
                __syncwarp();
                ptx::tmem_ld_row<D>(lane_addr + hh * D, lane_addr + 128, v, &nrm);
                ptx::tc_fence_before_sync();
                warp_arrive(&bar.acc_empty[buf]);
                int slab, tile, sg;
                sched_item(cta, i, tps, p.q, slab, tile, sg);
                const int h = (slab % p.groups) * G + hh;
                if (h < p.H) {
                    const long long slot = ((long long)cta * p.q.max_seg + seg) * G + hh;
                    float* P = partial + slot * DD + row;               // column j at j * D
#pragma unroll
                    for (int j = 0; j < D; ++j) P[j * D] = v[j];
                    P[D * D] = nrm;
                }
            }
        }
    }
}

// Partial-state slot of segment `seg` of CTA `c` for head hh of the group.
__device__ __forceinline__ long long ks_slot(long long c, int seg, int hh, int G, const KsParams& p) {
    return (c * p.q.max_seg + seg) * G + hh;
}
// Slot of the first of the R / rb partials of block `blk` of `slab` (those of
// CTAs (slab % P) + (blk % rb + t rb) P, t = 0, 1, ...; they are always added
// in ascending t, ks_block_step slots apart).
__device__ __forceinline__ long long ks_block_slot(int slab, int blk, int hh, int G, const KsParams& p) {
    const int rbi = blk % p.q.rb;
    const long long c = slab % p.q.P + (long long)rbi * p.q.P;
    const int nb = (p.q.nblk - rbi + p.q.rb - 1) / p.q.rb;
    return ks_slot(c, slab / p.q.P * nb + blk / p.q.rb, hh, G, p);
}
__device__ __forceinline__ long long ks_block_step(int G, const KsParams& p) {
    return (long long)p.q.rb * p.q.P * p.q.max_seg * G;
}

// ===================================================================== KR ===
// One thread per state entry (grid: (b, h) x entry blocks), so every load is
// independent and the kernel costs about one L2 round trip; consecutive
// threads read consecutive partial entries.
constexpr int KR_THREADS = 128;

template <int D>
__global__ void __launch_bounds__(KR_THREADS)
kr_reduce_tc(const float* __restrict__ partial, const KsParams p, float* __restrict__ state)
{
    constexpr int G = 128 / D;
    constexpr int DD = D * (D + 1);
    // The apply kernel of a two-call forward may be scheduled now: its Q loads
    // only need ks_state_tc to have started, and it waits for this grid before
    // reading the state.
    ptx::launch_dependents();
    ptx::wait_prerequisite_grid();              // the partial states of ks_state_tc
    const int pe = blockIdx.y * KR_THREADS + threadIdx.x;     // entry in the partials' column order
    if (pe >= DD) return;
    const int e = (pe % D) * (D + 1) + pe / D;                // the same entry, row-major in the state
    const long long bh = blockIdx.x;
    const int b = (int)(bh / p.H);
    const int h = (int)(bh % p.H);
    const int slab = b * p.groups + h / G;
    const long long step = ks_block_step(G, p) * DD;
    const int nr = p.q.R / p.q.rb;                  // partials per block
    // one block: the sum of the slab's partials; block-causal: the running
    // sum over blocks, i.e. the inclusive prefix state of every block
    float s = 0.0f;
    for (int j = 0; j < p.q.nblk; ++j) {
        const float* src = partial + ks_block_slot(slab, j, h % G, G, p) * DD + pe;
        // eight loads in flight, then their additions in ascending order
        for (int r0 = 0; r0 < nr; r0 += 8) {
            float t[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) t[u] = r0 + u < nr ? src[(r0 + u) * step] : 0.0f;
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (r0 + u < nr) s += t[u];
        }
        state[(bh * p.q.nblk + j) * DD + e] = s;
    }
}

// Block-causal prefix states. A CTA takes 32 consecutive partial-state entries
// (so every load instruction reads 128 contiguous bytes) times 8 block lanes:
// lane jl sums the partials (ascending CTA) of blocks jl, jl+8, ... of a
// 64-block chunk into shared memory, then one thread per entry walks the
// chunk in block order: prefix_j = prefix_{j-1} + blocksum_j. The same
// additions in the same order on every run.
constexpr int KP_ENTRIES = 32;
constexpr int KP_LANES = 8;
constexpr int KP_CHUNK = 64;

template <int D>
__global__ void __launch_bounds__(KP_ENTRIES * KP_LANES)
kr_prefix_tc(const float* __restrict__ partial, const KsParams p, float* __restrict__ states)
{
    constexpr int G = 128 / D;
    constexpr int DD = D * (D + 1);
    __shared__ float bsum[KP_CHUNK][KP_ENTRIES];
    ptx::launch_dependents();
    ptx::wait_prerequisite_grid();              // the partial states of ks_state_tc
    const int el = threadIdx.x % KP_ENTRIES;
    const int jl = threadIdx.x / KP_ENTRIES;
    const int pe = blockIdx.y * KP_ENTRIES + el;              // entry in the partials' column order
    const bool live = pe < DD;
    const int e = (pe % D) * (D + 1) + pe / D;                // the same entry, row-major in the state
    const long long bh = blockIdx.x;
    const int b = (int)(bh / p.H);
    const int h = (int)(bh % p.H);
    const int slab = b * p.groups + h / G;
    const long long step = ks_block_step(G, p) * DD;
    const int nr = p.q.R / p.q.rb;                  // partials per block
    float carry = 0.0f;
    for (int j0 = 0; j0 < p.q.nblk; j0 += KP_CHUNK) {
        for (int jj = jl; jj < KP_CHUNK && j0 + jj < p.q.nblk; jj += KP_LANES) {
            float x = 0.0f;
            if (live) {
                const float* src = partial + ks_block_slot(slab, j0 + jj, h % G, G, p) * DD + pe;
                for (int r0 = 0; r0 < nr; r0 += 8) {
                    float t[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) t[u] = r0 + u < nr ? src[(r0 + u) * step] : 0.0f;
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        if (r0 + u < nr) x += t[u];
                }
            }
            bsum[jj][el] = x;
        }
        __syncthreads();
        if (jl == 0 && live) {
            for (int jj = 0; jj < KP_CHUNK && j0 + jj < p.q.nblk; ++jj) {
                carry = carry + bsum[jj][el];
                states[(bh * p.q.nblk + j0 + jj) * DD + e] = carry;
            }
        }
        __syncthreads();
    }
}

// ===================================================================== KA ===
//
// Unit = one 128-token tile of a (b, group) slab, dealt out by the lockstep
// schedule above. Per unit:
//   producer  TMA: the Q tile (128 tokens x one group row) into a stage
//   workers   read their token row from the stage, apply phi in registers and
//             store it into TMEM as the UMMA A operand (the stage is free
//             again as soon as it is read)
//   UMMA      per head: D = phi(Q) S_hi + phi(Q) S_lo (A from TMEM, the
//             state in shared memory as bf16 hi and lo parts)
//   workers   D -> registers, O = num / (den + eps), into a swizzled staging
//             tile, written to global memory by a TMA store (each half of the
//             worker warps stores its own heads' boxes)
// TMEM: the accumulator at columns [0, 256) (head h at h * 256/G) and two A
// buffers of 64 columns at 256 and 320.
struct KaParams {
    int N, H, groups;
    Sched q;
    float eps;
    // the state of block blk of (b, h) is at ((b H + h) state_nblk + blk0 + blk):
    // state_nblk = q.nblk and blk0 = 0, except for a call that applies a run of
    // whole blocks of a longer sequence (the host-buffer block-causal forward)
    int state_nblk, blk0;
};

constexpr int KA_TILE = 128;                               // tokens = UMMA M
constexpr int KA_BOX_BYTES = KA_TILE * kBoxBytesRow;       // 16 KB
constexpr int KA_STAGE_BYTES = 2 * KA_BOX_BYTES;           // one group row of 128 tokens
constexpr uint32_t KA_A_COL = 256;                         // first A buffer column
constexpr uint32_t KA_A_LO_COL = 384;                      // lo parts of phi(Q) (feature maps other than ReLU)
constexpr int kBarRegion = 4096;                           // barriers + control block + slack

template <int D, bool OUT_BF16>
struct KaLayout {
    static constexpr int G = 128 / D;
    static constexpr int NA = D + 16;                      // UMMA N: d numerator cols + normaliser + pad
    static constexpr int SBO = (D / 8) * 128;              // 8-row group stride of the K-major state
    static constexpr int MAT_BYTES = (NA / 8) * SBO;       // one bf16 NA x D matrix
    static constexpr int STATE_BYTES = G * 2 * MAT_BYTES;  // hi and lo for every head
    static constexpr int OUT_BYTES = OUT_BF16 ? 2 : 4;
    static constexpr int OUT_BOXES = 128 * OUT_BYTES / kBoxBytesRow;   // boxes per output group row
    static constexpr int OUT_BOX_ELEMS = kBoxBytesRow / OUT_BYTES;
    static constexpr int STG_BYTES = OUT_BOXES * KA_BOX_BYTES;
    static constexpr int AVAIL = kSmemLimit - 1024 - kBarRegion - STATE_BYTES;
    // two staging tiles if that still leaves four Q stages, else one (an
    // epilogue that waits for the previous unit's store to read a single tile
    // made the 4096px apply a quarter slower on B200, and three Q stages
    // instead of four 6 % slower)
    static constexpr int STG_BUFS = (AVAIL - 2 * STG_BYTES) / KA_STAGE_BYTES >= 4 ? 2 : 1;
    static constexpr int STAGES_FIT = (AVAIL - STG_BUFS * STG_BYTES) / KA_STAGE_BYTES;
    static constexpr int STAGES = STAGES_FIT > 6 ? 6 : STAGES_FIT;
    static constexpr int STATE_OFF = STAGES * KA_STAGE_BYTES;
    static constexpr int STG_OFF = STATE_OFF + STATE_BYTES;
    static constexpr int DATA_BYTES = STG_OFF + STG_BUFS * STG_BYTES;
    static constexpr int NUM_BARS = 2 * STAGES + 14;
    static constexpr int ACC_COLS = 256 / G;               // TMEM columns per head
    static_assert(STAGES >= 3, "KA needs at least three Q stages");
};

// element (n, k) of a K-major, unswizzled bf16 matrix made of 8x8 core matrices
template <int SBO>
__host__ __device__ __forceinline__ int state_off(int n, int k) {
    return (n >> 3) * SBO + (k >> 3) * 128 + (n & 7) * 16 + (k & 7) * 2;
}

template <int D, bool OUT_BF16>
struct KaBars {
    using L = KaLayout<D, OUT_BF16>;
    uint64_t* full;        // [STAGES] Q tile landed
    uint64_t* empty;       // [STAGES] Q tile read by every worker warp
    uint64_t* a_full;      // [2] A operand in TMEM (and the state staged)
    uint64_t* acc_full;    // UMMAs of a unit done
    uint64_t* acc_empty;   // accumulator read by every worker warp
    uint64_t* stg_free;    // [2 halves] this half's staging boxes may be written
    uint64_t* stg_full;    // [2 halves][2] this half's staging boxes written
    uint64_t* mma_done;
    uint64_t* p1_written;  // (single launch) partial states written (warps 0-3), state padding zeroed (4-7)
    uint64_t* bs_done;     // (block-causal single launch) this CTA's block sums are written
    __device__ void init() const {
        for (int s = 0; s < L::STAGES; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], kWorkerWarps);
        }
        ptx::mbar_init(&a_full[0], kWorkerWarps);
        ptx::mbar_init(&a_full[1], kWorkerWarps);
        ptx::mbar_init(acc_full, 1);
        ptx::mbar_init(acc_empty, kWorkerWarps);
        for (int h = 0; h < 2; ++h) {
            ptx::mbar_init(&stg_free[h], 1);
            ptx::mbar_init(&stg_full[2 * h + 0], kWorkerWarps / 2);
            ptx::mbar_init(&stg_full[2 * h + 1], kWorkerWarps / 2);
        }
        ptx::mbar_init(mma_done, 1);
        ptx::mbar_init(p1_written, kWorkerWarps);
        ptx::mbar_init(bs_done, kWorkerWarps);
    }
};

template <int D, bool OUT_BF16>
__device__ __forceinline__ KaBars<D, OUT_BF16> ka_bars(uint64_t* b) {
    constexpr int S = KaLayout<D, OUT_BF16>::STAGES;
    uint64_t* a = b + 2 * S;
    return KaBars<D, OUT_BF16>{b, b + S, a, a + 2, a + 3, a + 4, a + 6, a + 10, a + 11, a + 12};
}

// zero the padding columns n in (d, NA) of the staged state (threads [0, nthreads))
template <int D, bool OUT_BF16>
__device__ __forceinline__ void ka_zero_state_padding(uint8_t* smem, int tid, int nthreads = kWorkerThreads) {
    using L = KaLayout<D, OUT_BF16>;
    if (tid < nthreads) {
        constexpr int PAD = L::NA - D - 1;
        for (int e = tid; e < L::G * 2 * PAD * D; e += nthreads) {
            const int k = e % D;
            const int n = D + 1 + (e / D) % PAD;
            const int mat = e / (D * PAD);
            *reinterpret_cast<__nv_bfloat16*>(smem + L::STATE_OFF + mat * L::MAT_BYTES +
                                              state_off<L::SBO>(n, k)) = __float2bfloat16_rn(0.0f);
        }
    }
}

// Where the apply phase gets the state of a slab from:
//   state != nullptr   the reduced fp32 state (B, H, d, d+1) of the reduction kernel
//   otherwise          the partial states of the state phase (same launch), summed
//                      here in the reduction kernel's order, once the arrival
//                      flags of the CTAs that wrote them hold this launch's epoch
struct KaStateSrc {
    const float* state;
    const float* partial;
    KsParams ks;
    const unsigned long long* flags;   // one arrival flag per CTA of the grid
    unsigned long long epoch;          // unique to this launch (set by the host)
    float* carry;                      // block-causal: one state-sized scratch per CTA
    float* bsums;                      // block-causal, R > 1: the slabs' block sums (one state each)
    unsigned long long* flags2;        // block-causal, R > 1: a CTA's block sums are stored
};

// Readiness flags of the single-launch forward. CTA c announces that all its
// partial states are in memory by storing the launch's epoch into flags[c]
// with release semantics. The writers fenced their own stores and arrived on a
// CTA barrier that this thread waited on, so the release store orders them
// too (release is cumulative); a second fence here only added latency (0-1 us
// per forward at the mid-size shapes, measured on B200). Before staging a
// slab's state, a CTA reads only the flags of the CTAs that wrote that slab's
// partials (its R siblings), not those of the whole grid, and adds each
// partial as soon as it and the ones before it are in. The host draws a new
// 64-bit epoch for every launch, so flags left by earlier launches (or any
// other bytes) never pass for this one and the flag array needs no reset
// between launches.
__device__ __forceinline__ void grid_arrive(unsigned long long* flag, unsigned long long epoch) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" :: "l"(flag), "l"(epoch) : "memory");
}

// The apply phase for CTA `cta`.
// `prev_empty`/`prev_tiles` (single launch): the state phase's stage barriers
// and how many tiles it loaded; Q stage s (< 6) reuses its stage s, so the
// first load into each waits until the state phase released that stage.
constexpr int kQAhead = 2;

template <int D, bool OUT_BF16, int FM, bool BC = false>
__device__ __forceinline__ void ka_phase(const CUtensorMap* tmQ, const CUtensorMap* tmO, const KaParams& p,
                                         int cta, const KaStateSrc& src, uint8_t* smem,
                                         const KaBars<D, OUT_BF16>& bar, uint32_t tmem,
                                         volatile int* abort, uint32_t* err,
                                         uint64_t* prev_empty = nullptr, int prev_tiles = 0,
                                         bool evict_first = false)
{
    using L = KaLayout<D, OUT_BF16>;
    constexpr int G = L::G;
    constexpr int DD = D * (D + 1);
    constexpr int S = L::STAGES;
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    if (cta >= p.q.grid) return;
    uint8_t* sstate = smem + L::STATE_OFF;
    const int tps = sched_tps(cta, p.q);
    const int nunits = tps * sched_nseg(cta, p.q);
    auto stage_ptr = [&](int s) { return smem + (size_t)s * KA_STAGE_BYTES; };

    if (warp == kProducerWarp) {
        // ------------------------------------------------ TMA producer ----
        if (lane == 0) {
            int issued = 0;
            constexpr int PS = ks_stages<FM>();       // the state phase's stages (single launch)
            static_assert(L::STAGES <= PS && KA_STAGE_BYTES == KS_STAGE_BYTES, "stage reuse");
            for (int i = 0; i < nunits; ++i) {
                const int s = i % S;
                if (!ptx::mbar_wait(&bar.empty[s], ((i / S) & 1) ^ 1, abort, err)) break;
                if (prev_empty != nullptr && i < S) {
                    // the state phase's next (never issued) use of stage s
                    const int j = prev_tiles + ((s - prev_tiles) % PS + PS) % PS;
                    if (!ptx::mbar_wait(&prev_empty[s], ((j / PS) & 1) ^ 1, abort, err)) break;
                    // The first Q load waits until this CTA's partial states are
                    // written and fenced, and only kQAhead Q tiles are loaded before
                    // the first unit's tile has been read (the state is staged by
                    // then): the fence and the partial states the workers read
                    // meanwhile are not queued behind Q loads. Measured on B200
                    // against four tiles ahead from the state phase's end: 2 us
                    // faster at 2048px, d = 64 and N = 16,384, the same at 4096 px.
                    if (i == 0 && !ptx::mbar_wait(bar.p1_written, 0, abort, err)) break;
                    if (i >= kQAhead && !ptx::mbar_wait(&bar.empty[0], 0, abort, err)) break;
                }
                int slab, tile, seg;
                sched_item(cta, i, tps, p.q, slab, tile, seg);
                const int b = slab / p.groups;
                const int x0 = (slab % p.groups) * 128;
                ptx::mbar_arrive_expect_tx(&bar.full[s], KA_STAGE_BYTES);
                if (evict_first) {
                    const uint64_t pol = ptx::l2_policy_evict_first();
                    ptx::tma_load_3d_hint(stage_ptr(s), tmQ, &bar.full[s], x0, tile * KA_TILE, b, pol);
                    ptx::tma_load_3d_hint(stage_ptr(s) + KA_BOX_BYTES, tmQ, &bar.full[s], x0 + 64,
                                          tile * KA_TILE, b, pol);
                } else {
                    ptx::tma_load_3d(stage_ptr(s), tmQ, &bar.full[s], x0, tile * KA_TILE, b);
                    ptx::tma_load_3d(stage_ptr(s) + KA_BOX_BYTES, tmQ, &bar.full[s], x0 + 64, tile * KA_TILE, b);
                }
                issued = i + 1;
            }
            for (int i = (issued > S ? issued - S : 0); i < issued; ++i)
                ptx::mbar_wait(&bar.full[i % S], (i / S) & 1, nullptr, err);
        }
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------- UMMA issuer ----
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_bf16_f32(128, L::NA, 0, 0);
            const uint32_t s_base = ptx::smem_u32(sstate);
            for (int i = 0; i < nunits; ++i) {
                if (!ptx::mbar_wait(&bar.a_full[i & 1], (i >> 1) & 1, abort, err)) break;
                if (!ptx::mbar_wait(bar.acc_empty, (i & 1) ^ 1, abort, err)) break;
                ptx::tc_fence_after_sync();
                const uint32_t a_base = tmem + KA_A_COL + (uint32_t)(i & 1) * 64u;
                const uint32_t a_lo_base = tmem + KA_A_LO_COL + (uint32_t)(i & 1) * 64u;
#pragma unroll
                for (int hh = 0; hh < G; ++hh) {
                    const uint32_t d_tmem = tmem + (uint32_t)(hh * L::ACC_COLS);
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t a = a_base + (uint32_t)(hh * D / 2 + ks * 8);
                        const uint32_t hi = s_base + (hh * 2 + 0) * L::MAT_BYTES + ks * 256;
                        const uint32_t lo = s_base + (hh * 2 + 1) * L::MAT_BYTES + ks * 256;
                        ptx::umma_f16_ts(d_tmem, a, ptx::smem_desc(hi, 128, L::SBO, ptx::kLayoutNone),
                                         idesc, ks > 0);
                        ptx::umma_f16_ts(d_tmem, a, ptx::smem_desc(lo, 128, L::SBO, ptx::kLayoutNone),
                                         idesc, true);
                        if constexpr (FM != kFeatureRelu) {
                            // phi(Q) lo x S hi (lo x lo is below fp32 rounding)
                            const uint32_t al = a_lo_base + (uint32_t)(hh * D / 2 + ks * 8);
                            ptx::umma_f16_ts(d_tmem, al, ptx::smem_desc(hi, 128, L::SBO, ptx::kLayoutNone),
                                             idesc, true);
                        }
                    }
                }
                ptx::umma_commit(bar.acc_full);
            }
            ptx::umma_commit(bar.mma_done);
            ptx::mbar_wait(bar.mma_done, 0, nullptr, err);
        }
    } else {
        // --------------------------------------------------------- workers ----
        // Warps w and w+4 own token rows m = 32*(w%4) + lane (their TMEM lanes);
        // warp w < 4 takes box 0 of the group row and heads [0, G/2), warp w >= 4
        // box 1 and heads [G/2, G).
        const int m = (warp & 3) * 32 + lane;
        const int half = warp >> 2;
        constexpr int HPW = G / 2;
        const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        // Each half stores its own output boxes (its heads' bytes of the row):
        // the leader (lane 0 of warp 0 / warp 4) issues and tracks those stores.
        const bool leader = (warp & 3) == 0 && lane == 0;
        constexpr int HALF_BOXES = L::OUT_BOXES / 2;
        if (leader) ptx::mbar_arrive(&bar.stg_free[half]);      // staging is free for unit 0
        // With the reduced state from a preceding kernel: this kernel may have
        // started before that kernel finished (programmatic launch); the Q loads
        // do not depend on it, the state does.
        if (src.state != nullptr) ptx::wait_prerequisite_grid();

        // Chunks of four entries of one column (rows k0 .. k0 + 3 of column n
        // of head hh): chunk c of the group is the c-th float4 of the heads'
        // partial states (stored by columns); this thread takes chunks tid,
        // tid + 256, ...
        constexpr int NC = G * DD / 4;
        constexpr int NCT = (NC + kWorkerThreads - 1) / kWorkerThreads;
        // single launch, block-causal: the slab this CTA staged last and its
        // last block; the running prefix itself waits in src.carry between
        // segments (registers would have to hold it through the apply loop)
        int carry_slab = -1, carry_blk = -1;
        // single launch: wait (bounded) until the flags of CTAs slab % P + r P,
        // r in [r0, r0 + k), hold this launch's epoch; k = 0: wait for none.
        // Returns the length of the ready prefix (at least 1 if any remain),
        // or -1 if the wait gave up.
        auto ready_prefix = [&](const unsigned long long* flags, int slab, int r, bool all) -> int {
            const unsigned long long* fl = flags + slab % src.ks.q.P;
            const int R = src.ks.q.R;
            const uint64_t t0 = ptx::globaltimer_ns();
            for (;;) {
                bool ready = true;
                if (r + lane < R) {
                    unsigned long long f;
                    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];"
                                 : "=l"(f) : "l"(fl + (long long)(r + lane) * src.ks.q.P) : "memory");
                    ready = f == src.epoch;
                }
                const unsigned waiting = __ballot_sync(0xffffffffu, !ready);
                const int k = min(waiting ? __ffs(waiting) - 1 : 32, R - r);   // ready prefix from r
                if (k > 0 && (!all || k == min(32, R - r))) {
                    __syncwarp();          // every lane's reads after every lane's flag
                    return k;
                }
                bool give_up = *abort != 0;
                if (!give_up && ptx::globaltimer_ns() - t0 > 2000000000ull) {
                    if (lane == 0) {
                        atomicCAS(err, ptx::kErrNone, ptx::kErrWaitTimeout);
                        *abort = 1;
                    }
                    give_up = true;
                }
                if (__any_sync(0xffffffffu, give_up)) return -1;
                __nanosleep(64);
            }
        };

        // stage the state of `slab` in shared memory as bf16 hi + lo parts
        auto stage_state = [&](int slab, int blk) -> bool {
            const int b = slab / p.groups;
            const int g = slab % p.groups;
            float4 v[NCT];
#pragma unroll
            for (int j = 0; j < NCT; ++j) v[j] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            if (src.state != nullptr) {
                // the reduced state (row-major per head): four loads per chunk
#pragma unroll
                for (int j = 0; j < NCT; ++j) {
                    const int c = tid + j * kWorkerThreads;
                    const int hh = c / (DD / 4);
                    const int w = c % (DD / 4);
                    const int n = w / (D / 4);
                    const int k0 = (w % (D / 4)) * 4;
                    if (c < NC && g * G + hh < p.H) {
                        const float* st = src.state +
                            (((long long)b * p.H + g * G + hh) * p.state_nblk + p.blk0 + blk) * DD + n;
                        v[j] = make_float4(st[(k0 + 0) * (D + 1)], st[(k0 + 1) * (D + 1)],
                                           st[(k0 + 2) * (D + 1)], st[(k0 + 3) * (D + 1)]);
                    }
                }
            } else if constexpr (BC) {
                // Block-causal: the inclusive prefix over the slab's blocks
                // 0 .. blk, carried on from this CTA's previous segment of the
                // slab, with the additions of kr_prefix_tc in its order: each
                // block's partials summed in ascending order, then that sum
                // added to the running prefix. The partials of every block
                // come from the slab's R CTAs, so all their flags are waited for.
                // With several partials per block (nr > 1), the slab's R CTAs
                // share the block sums: CTA r of the slab sums the partials of
                // blocks r, r + R, ... once (ascending, from zero) into
                // src.bsums and raises its second flag; each CTA then adds
                // block sums instead of partials.
                float4* cs = reinterpret_cast<float4*>(src.carry) + (long long)cta * NC;   // this CTA's prefix
                const long long kstep = ks_block_step(G, src.ks) * DD;
                const int R = src.ks.q.R;
                const int P = src.ks.q.P;
                const int nr = R / src.ks.q.rb;
                const bool shared = nr > 1;                 // (then R > 1: one slab per CTA)
                float4* bsum = shared ? reinterpret_cast<float4*>(src.bsums) + (long long)slab * src.ks.q.nblk * NC
                                      : nullptr;
                if (slab != carry_slab) {
                    for (int r = 0; r < R; r += 32)
                        if (ready_prefix(src.flags, slab, r, true) < 0) return false;
                    if (shared) {
                        for (int jb = cta / P; jb < src.ks.q.nblk; jb += R) {
                            const float* base = src.partial + ks_block_slot(slab, jb, 0, G, src.ks) * DD;
                            for (int c = tid; c < NC; c += kWorkerThreads) {
                                float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                                for (int t0 = 0; t0 < nr; t0 += 8) {
                                    float4 x[8];
#pragma unroll
                                    for (int u = 0; u < 8; ++u)
                                        x[u] = t0 + u < nr
                                            ? __ldcg(reinterpret_cast<const float4*>(base + (t0 + u) * kstep) + c)
                                            : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
                                    for (int u = 0; u < 8; ++u) {
                                        if (t0 + u < nr) {
                                            acc.x += x[u].x;
                                            acc.y += x[u].y;
                                            acc.z += x[u].z;
                                            acc.w += x[u].w;
                                        }
                                    }
                                }
                                __stcg(bsum + (long long)jb * NC + c, acc);
                            }
                        }
                        __threadfence();
                        warp_arrive(bar.bs_done);
                        if (warp == 0) {
                            if (!warp_wait(bar.bs_done, 0, abort, err)) return false;
                            if (lane == 0) grid_arrive(src.flags2 + cta, src.epoch);
                        }
                        // every block sum of the slab, so later segments need no flags
                        for (int r = 0; r < R; r += 32)
                            if (ready_prefix(src.flags2, slab, r, true) < 0) return false;
                    }
                    carry_slab = slab;
                    carry_blk = -1;
                } else {
#pragma unroll
                    for (int j = 0; j < NCT; ++j) {
                        const int c = tid + j * kWorkerThreads;
                        if (c < NC) v[j] = __ldcg(cs + c);      // written by this thread
                    }
                }
                float4 bs[NCT];
                if (shared) {
                    // block sums of blocks carry_blk + 1 .. blk, in that order
                    // (all in memory: their flags were seen at the slab's first segment)
                    for (int jb = carry_blk + 1; jb <= blk; ++jb) {
#pragma unroll
                        for (int j = 0; j < NCT; ++j) {
                            const int c = tid + j * kWorkerThreads;
                            bs[j] = c < NC ? __ldcg(bsum + (long long)jb * NC + c) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                        }
#pragma unroll
                        for (int j = 0; j < NCT; ++j) {
                            v[j].x += bs[j].x;
                            v[j].y += bs[j].y;
                            v[j].z += bs[j].z;
                            v[j].w += bs[j].w;
                        }
                    }
                } else if constexpr (D == 32) {
                    constexpr int RB = 4;
                    const int total = (blk - carry_blk) * nr;
                    for (int q0 = 0; q0 < total; q0 += RB) {
                        float4 t[RB][NCT];
#pragma unroll
                        for (int u = 0; u < RB; ++u) {
                            const int q = q0 + u;
                            const float* base = q < total
                                ? src.partial + ks_block_slot(slab, carry_blk + 1 + q / nr, 0, G, src.ks) * DD
                                              + (q % nr) * kstep
                                : nullptr;
#pragma unroll
                            for (int j = 0; j < NCT; ++j) {
                                const int c = tid + j * kWorkerThreads;
                                t[u][j] = (c < NC && q < total) ? __ldcg(reinterpret_cast<const float4*>(base) + c)
                                                                : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                            }
                        }
#pragma unroll
                        for (int u = 0; u < RB; ++u) {
                            const int q = q0 + u;
                            if (q < total) {
                                const int tt = q % nr;
#pragma unroll
                                for (int j = 0; j < NCT; ++j) {
                                    if (tt == 0) bs[j] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                                    bs[j].x += t[u][j].x;
                                    bs[j].y += t[u][j].y;
                                    bs[j].z += t[u][j].z;
                                    bs[j].w += t[u][j].w;
                                    if (tt == nr - 1) {
                                        v[j].x += bs[j].x;
                                        v[j].y += bs[j].y;
                                        v[j].z += bs[j].z;
                                        v[j].w += bs[j].w;
                                    }
                                }
                            }
                        }
                    }
                } else {
                    for (int jb = carry_blk + 1; jb <= blk; ++jb) {
                        const float* base = src.partial + ks_block_slot(slab, jb, 0, G, src.ks) * DD;
#pragma unroll
                        for (int j = 0; j < NCT; ++j) bs[j] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                        for (int t = 0; t < nr; ++t) {
#pragma unroll
                            for (int j = 0; j < NCT; ++j) {
                                const int c = tid + j * kWorkerThreads;
                                if (c < NC) {
                                    const float4 x = __ldcg(reinterpret_cast<const float4*>(base + t * kstep) + c);
                                    bs[j].x += x.x;
                                    bs[j].y += x.y;
                                    bs[j].z += x.z;
                                    bs[j].w += x.w;
                                }
                            }
                        }
#pragma unroll
                        for (int j = 0; j < NCT; ++j) {
                            v[j].x += bs[j].x;
                            v[j].y += bs[j].y;
                            v[j].z += bs[j].z;
                            v[j].w += bs[j].w;
                        }
                    }
                }
                carry_blk = blk;
#pragma unroll
                for (int j = 0; j < NCT; ++j) {
                    const int c = tid + j * kWorkerThreads;
                    if (c < NC) __stcg(cs + c, v[j]);
                }
            } else {
                // The same additions, in the same order, as kr_reduce_tc: the R
                // partials of the slab in ascending r. Partial r is in memory
                // once flags[slab % P + r P] holds this launch's epoch (its CTA
                // stored it after its partials). Each warp polls the flags itself
                // and adds the partials of the ready prefix while it waits for
                // the rest, RB partials' loads in flight together, one float4
                // per chunk; only the last ones are loaded after the slowest CTA
                // of the slab is done.
                const long long kstep = ks_block_step(G, src.ks) * DD;
                const float* base = src.partial + ks_slot(slab % src.ks.q.P, slab / src.ks.q.P, 0, G, src.ks) * DD;
                const unsigned long long* fl = src.flags + slab % src.ks.q.P;
                const int R = src.ks.q.R;
                constexpr int RB = D == 32 ? 4 : 2;
                const uint64_t t0 = ptx::globaltimer_ns();
                for (int r = 0; r < R;) {
                    bool ready = true;
                    if (r + lane < R) {
                        unsigned long long f;
                        asm volatile("ld.acquire.gpu.global.u64 %0, [%1];"
                                     : "=l"(f) : "l"(fl + (long long)(r + lane) * src.ks.q.P) : "memory");
                        ready = f == src.epoch;
                    }
                    const unsigned waiting = __ballot_sync(0xffffffffu, !ready);
                    const int k = min(waiting ? __ffs(waiting) - 1 : 32, R - r);   // ready prefix from r
                    if (k == 0) {
                        bool give_up = *abort != 0;
                        if (!give_up && ptx::globaltimer_ns() - t0 > 2000000000ull) {
                            if (lane == 0) {
                                atomicCAS(err, ptx::kErrNone, ptx::kErrWaitTimeout);
                                *abort = 1;
                            }
                            give_up = true;
                        }
                        if (__any_sync(0xffffffffu, give_up)) return false;
                        __nanosleep(64);
                        continue;
                    }
                    __syncwarp();          // every lane's reads after every lane's flag
                    for (int r0 = r; r0 < r + k; r0 += RB) {
                        float4 t[RB][NCT];
#pragma unroll
                        for (int rb = 0; rb < RB; ++rb) {
#pragma unroll
                            for (int j = 0; j < NCT; ++j) {
                                const int c = tid + j * kWorkerThreads;
                                t[rb][j] = (c < NC && r0 + rb < r + k)
                                    ? __ldcg(reinterpret_cast<const float4*>(base + (r0 + rb) * kstep) + c)
                                    : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                            }
                        }
#pragma unroll
                        for (int rb = 0; rb < RB; ++rb) {
                            if (r0 + rb < r + k) {
#pragma unroll
                                for (int j = 0; j < NCT; ++j) {
                                    v[j].x += t[rb][j].x;
                                    v[j].y += t[rb][j].y;
                                    v[j].z += t[rb][j].z;
                                    v[j].w += t[rb][j].w;
                                }
                            }
                        }
                    }
                    r += k;
                }
            }
#pragma unroll
            for (int j = 0; j < NCT; ++j) {
                const int c = tid + j * kWorkerThreads;
                if (c < NC) {
                    const int hh = c / (DD / 4);
                    const int w = c % (DD / 4);
                    const int n = w / (D / 4);               // state column j = UMMA N index
                    const int k0 = (w % (D / 4)) * 4;        // state rows k0.. = UMMA K indices
                    const bool live = g * G + hh < p.H;
                    const float x[4] = {live ? v[j].x : 0.0f, live ? v[j].y : 0.0f,
                                        live ? v[j].z : 0.0f, live ? v[j].w : 0.0f};
                    uint32_t hw[2], lw[2];
#pragma unroll
                    for (int u = 0; u < 4; u += 2) {
                        const __nv_bfloat16 h0 = __float2bfloat16_rn(x[u]);
                        const __nv_bfloat16 h1 = __float2bfloat16_rn(x[u + 1]);
                        const __nv_bfloat16 l0 = __float2bfloat16_rn(x[u] - __bfloat162float(h0));
                        const __nv_bfloat16 l1 = __float2bfloat16_rn(x[u + 1] - __bfloat162float(h1));
                        hw[u / 2] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
                        lw[u / 2] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
                    }
                    // four consecutive K of one column: 8 contiguous bytes of a core matrix
                    const int off = state_off<L::SBO>(n, k0);
                    *reinterpret_cast<uint2*>(sstate + (hh * 2 + 0) * L::MAT_BYTES + off) = make_uint2(hw[0], hw[1]);
                    *reinterpret_cast<uint2*>(sstate + (hh * 2 + 1) * L::MAT_BYTES + off) = make_uint2(lw[0], lw[1]);
                }
            }
            ptx::fence_proxy_async_smem();
            return true;
        };

        // A operand of unit i: phi(Q) row m, this warp's half, into A buffer
        // i & 1; at the first unit of a segment also the state of its slab.
        auto prep = [&](int i) -> bool {
            if (i % tps == 0) {
                if (i > 0) {
                    // the previous unit's UMMAs must be done reading the state
                    if (!warp_wait(bar.acc_full, (i - 1) & 1, abort, err)) return false;
                }
                int slab, tile, seg;
                sched_item(cta, i, tps, p.q, slab, tile, seg);
                if (!stage_state(slab, sched_block(cta, seg, p.q))) return false;
            }
            const int s = i % S;
            if (!warp_wait(&bar.full[s], (i / S) & 1, abort, err)) return false;
            // row m of box `half`: logical 16-byte chunk q sits at q ^ (m % 8)
            const uint8_t* row = stage_ptr(s) + half * KA_BOX_BYTES + m * kBoxBytesRow;
            uint32_t r[32];
            if constexpr (FM == kFeatureRelu) {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const uint4 v = *reinterpret_cast<const uint4*>(row + ((q ^ (m & 7)) * 16));
                    r[4 * q + 0] = relu_bf16x2(v.x);
                    r[4 * q + 1] = relu_bf16x2(v.y);
                    r[4 * q + 2] = relu_bf16x2(v.z);
                    r[4 * q + 3] = relu_bf16x2(v.w);
                }
                warp_arrive(&bar.empty[s]);
                __syncwarp();
            } else {
                uint32_t rl[32];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const uint4 v = *reinterpret_cast<const uint4*>(row + ((q ^ (m & 7)) * 16));
                    feature_split_bf16x2<FM>(v.x, r[4 * q + 0], rl[4 * q + 0]);
                    feature_split_bf16x2<FM>(v.y, r[4 * q + 1], rl[4 * q + 1]);
                    feature_split_bf16x2<FM>(v.z, r[4 * q + 2], rl[4 * q + 2]);
                    feature_split_bf16x2<FM>(v.w, r[4 * q + 3], rl[4 * q + 3]);
                }
                warp_arrive(&bar.empty[s]);
                __syncwarp();
                ptx::tmem_st32_wait(lane_base + KA_A_LO_COL + (uint32_t)(i & 1) * 64u + (uint32_t)half * 32u, rl);
            }
            ptx::tmem_st32_wait(lane_base + KA_A_COL + (uint32_t)(i & 1) * 64u + (uint32_t)half * 32u, r);
            ptx::tc_fence_before_sync();
            warp_arrive(&bar.a_full[i & 1]);
            return true;
        };

        bool ok = nunits > 0 ? prep(0) : true;
        for (int i = 0; i < nunits && ok; ++i) {
            if (i + 1 < nunits && !prep(i + 1)) break;
            // ---- epilogue of unit i
            if (!warp_wait(bar.acc_full, i & 1, abort, err)) break;
            ptx::tc_fence_after_sync();
            float num[HPW][D], den[HPW];
            __syncwarp();
#pragma unroll
            for (int j = 0; j < HPW; ++j) {
                const uint32_t col = (uint32_t)((half * HPW + j) * L::ACC_COLS);
                ptx::tmem_ld_row<D>(lane_base + col, lane_base + col + D, num[j], &den[j]);
            }
            ptx::tc_fence_before_sync();
            warp_arrive(bar.acc_empty);
            int slab, tile, seg;
            sched_item(cta, i, tps, p.q, slab, tile, seg);
            const int b = slab / p.groups;
            const int g = slab % p.groups;
            uint8_t* staging = smem + L::STG_OFF + (i % L::STG_BUFS) * L::STG_BYTES;
            // this half's boxes of the staging tile must be free (the leader
            // released them after the store that last read them)
            if (!warp_wait(&bar.stg_free[half], i & 1, abort, err)) break;
#pragma unroll
            for (int j = 0; j < HPW; ++j) {
                const int hh = half * HPW + j;
                const float rcp = 1.0f / (den[j] + p.eps);
                // row m of the staging tile, 128-byte swizzle: chunk q lands at q ^ (m % 8)
#pragma unroll
                for (int e = 0; e < D; e += 16 / L::OUT_BYTES) {
                    const int f = (hh * D + e) * L::OUT_BYTES;        // byte offset in the group row
                    uint4 w;
                    if (OUT_BF16) {
                        w.x = float2_to_bf16x2(num[j][e + 0] * rcp, num[j][e + 1] * rcp);
                        w.y = float2_to_bf16x2(num[j][e + 2] * rcp, num[j][e + 3] * rcp);
                        w.z = float2_to_bf16x2(num[j][e + 4] * rcp, num[j][e + 5] * rcp);
                        w.w = float2_to_bf16x2(num[j][e + 6] * rcp, num[j][e + 7] * rcp);
                    } else {
                        w.x = __float_as_uint(num[j][e + 0] * rcp);
                        w.y = __float_as_uint(num[j][e + 1] * rcp);
                        w.z = __float_as_uint(num[j][e + 2] * rcp);
                        w.w = __float_as_uint(num[j][e + 3] * rcp);
                    }
                    const int box = f / kBoxBytesRow;
                    const int q = (f % kBoxBytesRow) / 16;
                    *reinterpret_cast<uint4*>(staging + box * KA_BOX_BYTES + m * kBoxBytesRow +
                                              ((q ^ (m & 7)) * 16)) = w;
                }
            }
            ptx::fence_proxy_async_smem();
            warp_arrive(&bar.stg_full[2 * half + (i & 1)]);
            if ((warp & 3) == 0) {
                if (!warp_wait(&bar.stg_full[2 * half + (i & 1)], (i >> 1) & 1, abort, err)) break;
                if (lane == 0) {
                    const int x0 = g * 128;
                    const int y = tile * KA_TILE;
#pragma unroll
                    for (int k = 0; k < HALF_BOXES; ++k) {
                        const int bx = half * HALF_BOXES + k;
                        const int x = x0 + bx * L::OUT_BOX_ELEMS;
                        if (x < p.H * D && y < p.N)    // (block-causal padding tiles are not stored)
                            ptx::tma_store_3d(tmO, staging + bx * KA_BOX_BYTES, x, y, b);
                    }
                    ptx::bulk_commit_group();
                    // release the staging boxes for unit i + 1: the store that last
                    // used them (unit i + 1 - STG_BUFS) must be done reading
                    if (L::STG_BUFS == 2) ptx::bulk_wait_group_read<1>();
                    else ptx::bulk_wait_group_read<0>();
                    ptx::mbar_arrive(&bar.stg_free[half]);
                }
            }
        }
        if (leader) ptx::bulk_wait_group<0>();
    }
}

// ============================================================ the kernels ===
// Shared memory of every kernel: a data region (the largest phase it runs;
// the phases of the single-launch kernel reuse it one after the other), then
// the mbarriers of its phases, then the control block.
template <int DATA>
struct SmemMap {
    static constexpr int BAR_OFF = DATA;
    static constexpr int CTL_OFF = BAR_OFF + 2048;
    static constexpr int BYTES = CTL_OFF + 64 + 1024;      // + 1 KB alignment slack
    static_assert(BYTES <= kSmemLimit, "shared memory");
};

__device__ __forceinline__ void kernel_prologue(SharedCtl* ctl, int tid) {
    if (tid == 0) ctl->abort = 0;
    if ((tid >> 5) == 0) {
        ptx::tmem_alloc(&ctl->tmem_base, kTmemCols);
        ptx::tmem_relinquish();
    }
}

__device__ __forceinline__ void kernel_epilogue(SharedCtl* ctl, int tid) {
    ptx::tc_fence_before_sync();
    __syncthreads();
    if ((tid >> 5) == 0) {
        __syncwarp();
        ptx::tc_fence_after_sync();
        ptx::tmem_dealloc(ctl->tmem_base, kTmemCols);
    }
}

using KsMap = SmemMap<KS_DATA_BYTES>;
template <int D, bool OUT_BF16>
using KaMap = SmemMap<KaLayout<D, OUT_BF16>::DATA_BYTES>;
template <int D, bool OUT_BF16>
using FwdMap = SmemMap<(KaLayout<D, OUT_BF16>::DATA_BYTES > KS_DATA_BYTES ? KaLayout<D, OUT_BF16>::DATA_BYTES
                                                                          : KS_DATA_BYTES)>;

template <int D, int FM>
__global__ void __launch_bounds__(kThreads, 1)
ks_state_tc(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
            const KsParams p, float* __restrict__ partial)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    const KsBars bar = ks_bars(reinterpret_cast<uint64_t*>(smem + KsMap::BAR_OFF));
    SharedCtl* ctl = reinterpret_cast<SharedCtl*>(smem + KsMap::CTL_OFF);
    const int tid = threadIdx.x;
    if (tid == 0) {
        bar.init();
        ptx::fence_mbar_init();
    }
    kernel_prologue(ctl, tid);
    if (tid == kProducerWarp * 32) {
        ptx::prefetch_tmap(&tmK);
        ptx::prefetch_tmap(&tmV);
    }
    ks_fill_ones(smem, tid);
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    // the reduction kernel may be scheduled now; it waits for this grid's results
    if (tid == 0) ptx::launch_dependents();
    ks_phase<D, FM>(&tmK, &tmV, p, blockIdx.x, partial, smem, bar, ctl->tmem_base, &ctl->abort, &g_device_error);
    kernel_epilogue(ctl, tid);
}

template <int D, bool OUT_BF16, int FM>
__global__ void __launch_bounds__(kThreads, 1)
ka_apply_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
            const KaParams p, const float* __restrict__ state)
{
    using Map = KaMap<D, OUT_BF16>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    const auto bar = ka_bars<D, OUT_BF16>(reinterpret_cast<uint64_t*>(smem + Map::BAR_OFF));
    SharedCtl* ctl = reinterpret_cast<SharedCtl*>(smem + Map::CTL_OFF);
    const int tid = threadIdx.x;
    if (tid == 0) {
        bar.init();
        ptx::fence_mbar_init();
    }
    kernel_prologue(ctl, tid);
    if (tid == kProducerWarp * 32) {
        ptx::prefetch_tmap(&tmQ);
        ptx::prefetch_tmap(&tmO);
    }
    ka_zero_state_padding<D, OUT_BF16>(smem, tid);
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    KaStateSrc src{state, nullptr, KsParams{}, nullptr, 0ull, nullptr, nullptr, nullptr};
    ka_phase<D, OUT_BF16, FM>(&tmQ, &tmO, p, blockIdx.x, src, smem, bar, ctl->tmem_base, &ctl->abort,
                          &g_device_error);
    kernel_epilogue(ctl, tid);
}

// The whole forward in one cooperative launch (all CTAs resident, so a CTA
// may wait for another): the state phase; a readiness flag per CTA; then the
// apply phase, which waits (bounded) for the flags of the CTAs that wrote its
// slab's partial states and sums them itself in the reduction kernel's order
// (BC, block-causal: the prefix kernel's, carried from block to block in
// `carry`, one state-sized scratch per CTA; a separate instance, so that the
// plain forward's code is not touched by it).
// The apply phase's Q loads start as soon as the state phase has released its
// shared memory, so they overlap that wait. `flags` has one slot per CTA;
// `epoch` is unique to the launch.
template <int D, bool OUT_BF16, int FM, bool BC>
__global__ void __launch_bounds__(kThreads, 1)
fwd_fused_tc(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
             const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
             const KsParams ks, const KaParams ka, float* __restrict__ partial,
             unsigned long long* flags, const unsigned long long epoch, const int evict_first,
             float* __restrict__ carry)
{
    using Map = FwdMap<D, OUT_BF16>;
    if constexpr (!BC) {
        // prefix states over token blocks take the BC instance
        if (ks.q.nblk != 1 || ka.q.nblk != 1) {
            if (threadIdx.x == 0) atomicCAS(&g_device_error, ptx::kErrNone, ptx::kErrUnsupported);
            return;
        }
    }
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Map::BAR_OFF);
    const KsBars kbar = ks_bars(bars);
    const auto abar = ka_bars<D, OUT_BF16>(bars + KS_NUM_BARS);
    SharedCtl* ctl = reinterpret_cast<SharedCtl*>(smem + Map::CTL_OFF);
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    // The producer thread initialises the state phase's barriers and issues
    // its first tiles' loads at once, ahead of the TMEM allocation and the
    // CTA-wide sync below (the other threads touch those barriers only after
    // that sync, and the loads' stages are not written before it).
    int pre_issued = 0;
    if (tid == kProducerWarp * 32) {
        kbar.init();
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tmK);
        ptx::prefetch_tmap(&tmV);
        if ((int)blockIdx.x < ks.q.grid) {
            const int tps = sched_tps(blockIdx.x, ks.q);
            pre_issued = min(ks_stages<FM>(), tps * sched_nseg(blockIdx.x, ks.q));
            for (int i = 0; i < pre_issued; ++i)
                ks_load_tile(&tmK, &tmV, ks, blockIdx.x, i, tps, smem + (size_t)i * KS_STAGE_BYTES, &kbar.full[i],
                             evict_first != 0);
        }
        ptx::prefetch_tmap(&tmQ);
        ptx::prefetch_tmap(&tmO);
    }
    if (tid == 0) {
        abar.init();
        ptx::fence_mbar_init();
    }
    kernel_prologue(ctl, tid);
    ks_fill_ones(smem, tid);
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = ctl->tmem_base;

    // with evict_first, K, V and Q (read once) are marked first to go when L2
    // needs room
    ks_phase<D, FM>(&tmK, &tmV, ks, blockIdx.x, partial, smem, kbar, tmem, &ctl->abort, &g_device_error,
                    evict_first != 0, pre_issued);

    // Warps 0-3 have written this CTA's partial states (after the last
    // accumulator was complete, i.e. after every state-phase UMMA): make them
    // visible and arrive. Warps 4-7 meanwhile zero the staged state's padding
    // columns, once every state-phase UMMA is done with those bytes (they were
    // a K/V stage); off the path from the last partial to the flag and the
    // first poll, where it cost ~0.8 us. Every worker waits for both before
    // it touches the apply phase's shared memory or TMEM, which reuse the
    // state phase's.
    if (warp < 4) {
        __threadfence();
        warp_arrive(abar.p1_written);
    } else if (warp < kWorkerWarps) {
        // (a CTA without state-phase tiles issued no UMMAs and commits none)
        if ((int)blockIdx.x < ks.q.grid) warp_wait(kbar.mma_done, 0, &ctl->abort, &g_device_error);
        ka_zero_state_padding<D, OUT_BF16>(smem, tid - 4 * 32, kWorkerThreads / 2);
        ptx::fence_proxy_async_smem();
        warp_arrive(abar.p1_written);
    }
    if (warp < kWorkerWarps) {
        warp_wait(abar.p1_written, 0, &ctl->abort, &g_device_error);
        // every CTA raises its readiness flag, with or without apply work
        if (tid == 0) grid_arrive(flags + blockIdx.x, epoch);
    }
    // block-causal: after the per-CTA prefixes, the slabs' block sums
    float* bsums = carry == nullptr ? nullptr
        : carry + (size_t)gridDim.x * (128 / D) * (D * (D + 1));
    KaStateSrc src{nullptr, partial, ks, flags, epoch, carry, bsums, flags + gridDim.x};
    const int ks_tiles = (int)blockIdx.x < ks.q.grid
        ? sched_tps(blockIdx.x, ks.q) * sched_nseg(blockIdx.x, ks.q) : 0;
    ka_phase<D, OUT_BF16, FM, BC>(&tmQ, &tmO, ka, blockIdx.x, src, smem, abar, tmem, &ctl->abort, &g_device_error,
                          kbar.empty, ks_tiles, evict_first != 0);
    kernel_epilogue(ctl, tid);
}

// Self-test of the bounded wait: one thread waits on an mbarrier that nothing
// arrives at, with the given limit; the wait gives up, records
// kErrWaitTimeout in g_device_error and the kernel returns normally.
__global__ void wait_timeout_selftest(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort;
    if (threadIdx.x == 0) {
        abort = 0;
        ptx::mbar_init(&bar, 1);
        ptx::fence_mbar_init();
        ptx::mbar_wait(&bar, 0, &abort, &g_device_error, limit_ns);
    }
}

}  // namespace tc
}  // namespace sana
