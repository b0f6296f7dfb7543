// C ABI of the ReLU linear-attention forward: argument checks, the work
// plans, TMA tensor maps, and kernel launches on the caller's stream. See
// include/sana_linattn.h for the contract.
#include <algorithm>
#include <atomic>
#include <chrono>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <random>
#include <utility>

#include <cudaTypedefs.h>

#include "../../include/sana_linattn.h"
#include "common.cuh"
#include "tc_kernels.cuh"
#include "kvproj_kernel.cuh"
#include "ffn_kernels.cuh"

namespace {

thread_local char g_last_error[256] = "";

void set_last_error(const char* where, cudaError_t e) {
    std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", where,
                  cudaGetErrorName(e), cudaGetErrorString(e));
}

constexpr int kDefaultSMs = 148;      // B200; the plans' CTA count when no device can be asked
constexpr int kMaxDevicesCached = 64; // per-device caches of launch properties

// Streaming multiprocessors of the current device (one persistent CTA runs on
// each), asked once per device; kDefaultSMs when no device answers (the size
// queries work on a host without a GPU). The work plans, and so the workspace
// size and the order of the partial sums, follow this count: results are
// bit-reproducible on devices with the same number of SMs.
int device_sms() {
    static std::atomic<int> cache[kMaxDevicesCached];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return kDefaultSMs;
    }
    if (dev >= 0 && dev < kMaxDevicesCached) {
        const int v = cache[dev].load(std::memory_order_acquire);
        if (v > 0) return v;
    }
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
        cudaGetLastError();
        return kDefaultSMs;
    }
    if (dev >= 0 && dev < kMaxDevicesCached) cache[dev].store(sms, std::memory_order_release);
    return sms;
}

// A unique id of the calling thread's current CUDA context (cuCtxGetId), or
// 0 when there is none or the driver cannot be asked. The per-device caches
// below (function attributes, copy streams and events, the scratch address)
// remember the context they were made in and are made again when it changed,
// e.g. after cudaDeviceReset destroyed the primary context.
unsigned long long current_context_id() {
    using GetCurrent = CUresult (*)(CUcontext*);
    using GetId = CUresult (*)(CUcontext, unsigned long long*);
    static std::once_flag once;
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrent>(p);
        p = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetId>(p);
    });
    CUcontext ctx = nullptr;
    if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr)
        return 0;
    unsigned long long id = 0;
    return get_id(ctx, &id) == CUDA_SUCCESS ? id : 0;
}
constexpr long long kMaxElems = 1LL << 62;
constexpr long long kMaxGrid = 0x7fffffffLL;

inline long long cdiv(long long a, long long b) { return (a + b - 1) / b; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Work plans of the kernels. A pure function of the sizes: the workspace
// size and the order in which partial states are summed never depend on the
// device or on timing.
struct Plan {
    sana::tc::KsParams ks;
    sana::tc::KaParams ka;
    size_t partial_bytes;   // fp32 partial states, one per (CTA segment, head)
    size_t state_bytes;     // fp32 (B, H, d, d+1); block-causal (B, H, nblk, d, d+1)
    size_t carry_bytes;     // block-causal single launch: one group's state per CTA and per slab block
    size_t flag_bytes;      // readiness flags of the single-launch forward (one per CTA)
};

// Lockstep schedule of S slabs of T tiles over at most `sms` CTAs (see the
// comment at the top of tc_kernels.cuh).
sana::tc::Sched make_sched(long long S, long long T, int sms) {
    sana::tc::Sched q{};
    q.S = (int)S;
    q.T = (int)T;
    if (S <= sms) {
        q.P = (int)S;
        q.R = (int)std::min<long long>(sms / S, T);
        q.max_seg = 1;
    } else {
        q.P = sms;
        q.R = 1;
        q.max_seg = (int)cdiv(S, sms);
    }
    q.grid = q.P * q.R;
    q.nblk = 1;
    q.tpb = 0;
    q.rb = 1;
    return q;
}

// Block-causal schedule: S slabs of nblk blocks of bt tiles; a slab's
// rb * rt CTAs split its blocks rb ways and each block's tiles rt ways (rt
// divides bt).
sana::tc::Sched make_block_sched(long long S, long long nblk, long long bt, int rb, int rt, int sms) {
    sana::tc::Sched q{};
    q.S = (int)S;
    q.T = (int)(nblk * bt);
    q.R = rb * rt;
    q.P = S <= sms ? (int)S : sms;
    q.grid = S <= sms ? (int)(S * q.R) : sms;
    q.nblk = (int)nblk;
    q.tpb = (int)(bt / rt);
    q.rb = rb;
    q.max_seg = (int)(cdiv(S, q.grid) * cdiv(nblk, rb));
    return q;
}

// How the CTAs of a slab split a block-causal slab (S slabs, nblk blocks of
// tiles128 128-token tiles; at most `sms` CTAs): the split (rb, rt), rb * rt <=
// sms / S and rt dividing tiles128, that minimises the tiles of the busiest
// CTA plus three tiles' worth for each state it stages (one per block it
// visits), times 1.15 when rb > 1; ties go to fewer partial states per block
// (smaller rt). The factor stands for what reading rb token regions at once
// instead of one cost on B200, fitted to two measurements with 9 slabs of 16
// blocks: 512 tiles per block, rb = 16, rt = 1 took 1796-1817 us against
// 1703 us for rb = 1, rt = 16; 32 tiles per block, rb = 16, rt = 1 took 138 us
// against 198 us for rb = 1, rt = 16.
struct BlockSplit {
    int rb, rt;
};
BlockSplit block_split(long long S, long long nblk, long long tiles128, int sms) {
    if (S > sms) return BlockSplit{1, 1};
    const long long rmax = sms / S;
    BlockSplit best{1, 1};
    long long best_cost = -1;
    for (long long rt = 1; rt <= std::min(rmax, tiles128); ++rt) {
        if (tiles128 % rt != 0) continue;
        const long long rb = std::min(nblk, rmax / rt);
        const long long cost = cdiv(nblk, rb) * (tiles128 / rt + 3) * (rb > 1 ? 115 : 100);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = BlockSplit{(int)rb, (int)rt};
        }
    }
    return best;
}

// L = 0: the plain forward; L > 0 (a multiple of 128): block-causal with
// blocks of L tokens.
Plan make_plan(int B, int N, int H, int d, int L = 0, int sms = device_sms()) {
    const int G = 128 / d;                        // heads per 128-row group
    const long long groups = cdiv(H, G);
    const long long S = (long long)B * groups;
    Plan p{};
    p.ks.N = N;
    p.ks.H = H;
    p.ks.groups = (int)groups;
    p.ka.N = N;
    p.ka.H = H;
    p.ka.groups = (int)groups;
    long long nblk = 1;
    if (L > 0) {
        nblk = cdiv(N, L);
        const long long tiles128 = L / sana::tc::KA_TILE;
        const BlockSplit sp = block_split(S, nblk, tiles128, sms);
        p.ks.q = make_block_sched(S, nblk, L / sana::tc::KS_TILE, sp.rb, sp.rt, sms);
        p.ka.q = make_block_sched(S, nblk, tiles128, sp.rb, sp.rt, sms);
    } else {
        p.ks.q = make_sched(S, cdiv(N, sana::tc::KS_TILE), sms);
        p.ka.q = make_sched(S, cdiv(N, sana::tc::KA_TILE), sms);
    }
    p.ka.eps = 0.0f;
    p.ka.state_nblk = (int)nblk;
    p.ka.blk0 = 0;
    const size_t dd = (size_t)d * (d + 1) * sizeof(float);
    p.partial_bytes = align256((size_t)p.ks.q.grid * p.ks.q.max_seg * G * dd);
    p.state_bytes = align256((size_t)B * H * nblk * dd);
    // two flags per CTA (partial states written; block-causal one-launch form:
    // its block sums written)
    p.flag_bytes = align256(2 * sizeof(unsigned long long) * (size_t)std::max(p.ks.q.grid, p.ka.q.grid));
    // block-causal one-launch form: one running prefix per CTA, then one block
    // sum per slab and block
    p.carry_bytes = L > 0 ? align256(((size_t)std::max(p.ks.q.grid, p.ka.q.grid) + (size_t)S * nblk) * G * dd) : 0;
    return p;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

sana_la_status check_sizes(int B, int N, int H, int d) {
    if (B < 1 || N < 1 || H < 1) return SANA_LA_ERR_INVALID_ARG;
    if (d != 32 && d != 64) return SANA_LA_ERR_UNSUPPORTED;
    const long long elems = (long long)B * N;
    if (elems > kMaxElems / ((long long)H * d)) return SANA_LA_ERR_INVALID_ARG;
    // one batch of one tensor must stay under the 2^40-byte TMA stride limit
    if ((long long)N * H * d * 2 >= (1LL << 40)) return SANA_LA_ERR_UNSUPPORTED;
    if ((long long)B * H > kMaxGrid) return SANA_LA_ERR_UNSUPPORTED;
    return SANA_LA_OK;
}

// Block length of the block-causal form: a multiple of 128 tokens, and the
// partial states (one per CTA, slab and block) within 4 GiB.
constexpr size_t kMaxBlockPartialBytes = size_t(4) << 30;

sana_la_status check_block(int B, int N, int H, int d, int L, int sms = device_sms()) {
    if (L < 1) return SANA_LA_ERR_INVALID_ARG;
    if (L % sana::tc::KA_TILE != 0) return SANA_LA_ERR_UNSUPPORTED;
    // the sizes of make_plan(B, N, H, d, L), in 64-bit arithmetic first
    const long long G = 128 / d;
    const long long S = (long long)B * cdiv(H, G);
    const long long nblk = cdiv(N, L);
    const BlockSplit sp = block_split(S, nblk, L / sana::tc::KA_TILE, sms);
    const long long grid = S <= sms ? S * sp.rb * sp.rt : sms;
    const long long segs = cdiv(S, grid) * cdiv(nblk, sp.rb);   // per CTA
    const long long per_seg = G * d * (d + 1) * (long long)sizeof(float);
    if (segs > (long long)(kMaxBlockPartialBytes / per_seg) / grid) return SANA_LA_ERR_UNSUPPORTED;
    if (nblk * L > 0x7fffffffLL) return SANA_LA_ERR_UNSUPPORTED;    // padded token coordinates
    return SANA_LA_OK;
}

sana_la_status check_eps(float eps) {
    return (std::isfinite(eps) && eps >= 0.0f) ? SANA_LA_OK : SANA_LA_ERR_INVALID_ARG;
}

sana_la_status launch_status(const char* where) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        set_last_error(where, e);
        return SANA_LA_ERR_CUDA;
    }
    return SANA_LA_OK;
}

// ------------------------------------------------------------- TMA maps ----
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// (B, N, H*d) tensor viewed as 3-D {H*d, N, B}; boxes of 128 bytes (one
// swizzle span: 64 bf16 or 32 fp32 elements) by `rows` tokens, 128-byte
// swizzle. Loads read zeros outside the tensor (tokens >= N, heads >= H);
// stores skip those parts.
sana_la_status make_tmap(CUtensorMap* m, const void* base, int B, int N, int H, int d, int rows,
                         bool fp32 = false) {
    auto encode = tensor_map_encoder();
    if (encode == nullptr) {
        std::snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled unavailable");
        return SANA_LA_ERR_CUDA;
    }
    const cuuint64_t esize = fp32 ? 4 : 2;
    const cuuint64_t row_elems = (cuuint64_t)H * d;
    cuuint64_t dims[3] = {row_elems, (cuuint64_t)N, (cuuint64_t)B};
    cuuint64_t strides[2] = {row_elems * esize, row_elems * esize * (cuuint64_t)N};
    cuuint32_t box[3] = {(cuuint32_t)(128 / esize), (cuuint32_t)rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = encode(m, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                        const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        std::snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled failed (%d)", (int)r);
        return SANA_LA_ERR_CUDA;
    }
    return SANA_LA_OK;
}

// Launch on `s`; with `overlap` the kernel may start before the preceding
// kernel of the stream has finished (programmatic stream serialization). Only
// kernels that wait with griddepcontrol.wait before reading that kernel's
// results, and whose other inputs were ready before it started, use it.
template <typename... KArgs, typename... Args>
sana_la_status launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                      bool overlap, const char* name, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = overlap ? 1 : 0;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    if (e != cudaSuccess) {
        set_last_error(name, e);
        return SANA_LA_ERR_CUDA;
    }
    return launch_status(name);
}

// Opt a kernel into its dynamic shared memory size, once per device and
// context (the attribute lives in the context).
template <typename Kernel>
sana_la_status ensure_smem(Kernel kernel, int bytes, std::atomic<unsigned long long> (&done)[kMaxDevicesCached]) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        set_last_error("cudaGetDevice", e);
        return SANA_LA_ERR_CUDA;
    }
    const bool cached = dev >= 0 && dev < kMaxDevicesCached;
    const unsigned long long ctx = current_context_id();
    if (cached && ctx != 0 && done[dev].load(std::memory_order_acquire) == ctx) return SANA_LA_OK;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) {
        set_last_error("cudaFuncSetAttribute", e);
        return SANA_LA_ERR_CUDA;
    }
    if (cached) done[dev].store(current_context_id(), std::memory_order_release);
    return SANA_LA_OK;
}

// ------------------------------------------------------------- launches ----
template <int D, int FM>
sana_la_status run_kv_state(const void* K, const void* V, int B, int N, int H, const Plan& p,
                            float* partial, float* state, cudaStream_t s) {
    static std::atomic<unsigned long long> smem_set[kMaxDevicesCached];
    CUtensorMap tmK, tmV;
    sana_la_status st;
    if ((st = make_tmap(&tmK, K, B, N, H, D, sana::tc::KS_TILE)) != SANA_LA_OK) return st;
    if ((st = make_tmap(&tmV, V, B, N, H, D, sana::tc::KS_TILE)) != SANA_LA_OK) return st;
    if ((st = ensure_smem(sana::tc::ks_state_tc<D, FM>, sana::tc::KsMap::BYTES, smem_set)) != SANA_LA_OK)
        return st;
    if ((st = launch(sana::tc::ks_state_tc<D, FM>, dim3(p.ks.q.grid), dim3(sana::tc::kThreads),
                     sana::tc::KsMap::BYTES, s, false, "ks_state_tc", tmK, tmV, p.ks, partial)) != SANA_LA_OK)
        return st;
    // the reduction overlaps the state kernel's tail; it waits for its results
    if (p.ks.q.nblk > 1) {
        // block-causal: prefix states over the blocks
        const dim3 kp_grid((unsigned)((long long)B * H),
                           (D * (D + 1) + sana::tc::KP_ENTRIES - 1) / sana::tc::KP_ENTRIES);
        return launch(sana::tc::kr_prefix_tc<D>, kp_grid, dim3(sana::tc::KP_ENTRIES * sana::tc::KP_LANES), 0, s,
                      true, "kr_prefix_tc", (const float*)partial, p.ks, state);
    }
    const dim3 kr_grid((unsigned)((long long)B * H), (D * (D + 1) + sana::tc::KR_THREADS - 1) / sana::tc::KR_THREADS);
    return launch(sana::tc::kr_reduce_tc<D>, kr_grid, dim3(sana::tc::KR_THREADS), 0, s, true, "kr_reduce_tc",
                  (const float*)partial, p.ks, state);
}

template <int D, bool OUT_BF16, int FM>
sana_la_status launch_apply(const CUtensorMap& tmQ, const void* O, int B, int N, int H,
                            const Plan& p, const float* state, cudaStream_t s, bool overlap) {
    static std::atomic<unsigned long long> smem_set[kMaxDevicesCached];
    CUtensorMap tmO;
    sana_la_status st;
    if ((st = make_tmap(&tmO, O, B, N, H, D, sana::tc::KA_TILE, !OUT_BF16)) != SANA_LA_OK) return st;
    constexpr int smem = sana::tc::KaMap<D, OUT_BF16>::BYTES;
    if ((st = ensure_smem(sana::tc::ka_apply_tc<D, OUT_BF16, FM>, smem, smem_set)) != SANA_LA_OK) return st;
    return launch(sana::tc::ka_apply_tc<D, OUT_BF16, FM>, dim3(p.ka.q.grid), dim3(sana::tc::kThreads), smem, s,
                  overlap, "ka_apply_tc", tmQ, tmO, p.ka, state);
}

// `overlap`: called right after this library's own state kernels on the same
// stream (forward), so Q was ready before they started and the apply kernel
// may start early; a standalone apply waits for everything before it.
template <int D, int FM>
sana_la_status run_apply(const void* Q, const float* state, int B, int N, int H, int L, void* O,
                         sana_la_out_dtype od, float eps, cudaStream_t s, bool overlap, int state_nblk,
                         int blk0) {
    Plan p = make_plan(B, N, H, D, L);
    p.ka.eps = eps;
    if (state_nblk > 0) {
        p.ka.state_nblk = state_nblk;
        p.ka.blk0 = blk0;
    }
    CUtensorMap tmQ;
    sana_la_status st;
    if ((st = make_tmap(&tmQ, Q, B, N, H, D, sana::tc::KA_TILE)) != SANA_LA_OK) return st;
    return od == SANA_LA_OUT_BF16 ? launch_apply<D, true, FM>(tmQ, O, B, N, H, p, state, s, overlap)
                                  : launch_apply<D, false, FM>(tmQ, O, B, N, H, p, state, s, overlap);
}

// The whole forward as one cooperative launch (fwd_fused_tc). Returns
// SANA_LA_ERR_UNSUPPORTED, with nothing enqueued, when the device refuses a
// cooperative launch of this size, so the caller can use the three kernels.
// Epochs of the single-launch forward's grid barrier: unique per launch within
// the process, and started at a random point so that flags another process
// left in reused memory do not match either.
unsigned long long next_epoch() {
    static std::atomic<unsigned long long> counter{[] {
        std::random_device rd;
        return ((unsigned long long)rd() << 32 ^ (unsigned long long)rd() ^
                (unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count()) | 1ull;
    }()};
    unsigned long long e = counter.fetch_add(1, std::memory_order_relaxed);
    return e != 0 ? e : counter.fetch_add(1, std::memory_order_relaxed);
}

// Blocks of `kernel` one SM holds at once, asked once per device.
template <typename Kernel>
int blocks_per_sm(Kernel kernel, int threads, int smem, std::atomic<int> (&cache)[kMaxDevicesCached], int dev) {
    if (dev < 0 || dev >= kMaxDevicesCached) return -1;
    int v = cache[dev].load(std::memory_order_acquire);
    if (v > 0) return v;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, kernel, threads, smem) != cudaSuccess) return -1;
    cache[dev].store(v, std::memory_order_release);
    return v;
}

template <int D, bool OUT_BF16, int FM, bool BC>
sana_la_status launch_forward_fused(const void* Q, const void* K, const void* V, void* O, int B, int N,
                                    int H, const Plan& p, float* partial, unsigned long long* flags,
                                    float* carry, cudaStream_t s) {
    static std::atomic<unsigned long long> smem_set[kMaxDevicesCached];
    static std::atomic<int> per_sm_cache[kMaxDevicesCached];
    CUtensorMap tmK, tmV, tmQ, tmO;
    sana_la_status st;
    if ((st = make_tmap(&tmK, K, B, N, H, D, sana::tc::KS_TILE)) != SANA_LA_OK) return st;
    if ((st = make_tmap(&tmV, V, B, N, H, D, sana::tc::KS_TILE)) != SANA_LA_OK) return st;
    if ((st = make_tmap(&tmQ, Q, B, N, H, D, sana::tc::KA_TILE)) != SANA_LA_OK) return st;
    if ((st = make_tmap(&tmO, O, B, N, H, D, sana::tc::KA_TILE, !OUT_BF16)) != SANA_LA_OK) return st;
    constexpr int smem = sana::tc::FwdMap<D, OUT_BF16>::BYTES;
    auto kernel = sana::tc::fwd_fused_tc<D, OUT_BF16, FM, BC>;
    if ((st = ensure_smem(kernel, smem, smem_set)) != SANA_LA_OK) return st;
    const int grid = std::max(p.ks.q.grid, p.ka.q.grid);
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return SANA_LA_ERR_UNSUPPORTED;
    }
    const int per_sm = blocks_per_sm(kernel, sana::tc::kThreads, smem, per_sm_cache, dev);
    if (per_sm <= 0 || (long long)sms * per_sm < grid) {
        cudaGetLastError();
        return SANA_LA_ERR_UNSUPPORTED;
    }
    const unsigned long long epoch = next_epoch();
    // A captured graph replays the same epoch: there the flags are cleared by
    // a memset node before each launch instead.
    cudaStreamCaptureStatus capture = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(s, &capture);
    if (e != cudaSuccess) {
        set_last_error("cudaStreamIsCapturing", e);
        return SANA_LA_ERR_CUDA;
    }
    if (capture != cudaStreamCaptureStatusNone) {
        e = cudaMemsetAsync(flags, 0, 2 * sizeof(unsigned long long) * (size_t)grid, s);
        if (e != cudaSuccess) {
            set_last_error("cudaMemsetAsync(grid barrier flags)", e);
            return SANA_LA_ERR_CUDA;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(sana::tc::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // Evict-first L2 policy on the input loads. Measured back to back on B200
    // (same process, A/B): 111.9 vs 119.3 us at 4096px (0.44 GB of inputs),
    // 400.7 vs 404.3 us at N = 262,144 and 1598 vs 1608 us at N = 1,048,576.
    const int evict_first = 1;
    e = cudaLaunchKernelEx(&cfg, kernel, tmK, tmV, tmQ, tmO, p.ks, p.ka, partial, flags, epoch, evict_first,
                           carry);
    if (e != cudaSuccess) {
        set_last_error("fwd_fused_tc", e);
        return SANA_LA_ERR_CUDA;
    }
    return launch_status("fwd_fused_tc");
}

sana_la_status kv_state_impl(const void* K, const void* V, int B, int N, int H, int d, int L,
                             float* state, void* ws, size_t ws_bytes, cudaStream_t s,
                             bool need_state_area, int fm = sana::kFeatureRelu) {
    const Plan p = make_plan(B, N, H, d, L);
    const size_t need = p.partial_bytes + (need_state_area ? p.state_bytes : 0);
    if (ws_bytes < need) return SANA_LA_ERR_WORKSPACE;
    float* partial = static_cast<float*>(ws);
    switch (d * 4 + fm) {
        case 32 * 4 + sana::kFeatureRelu: return run_kv_state<32, sana::kFeatureRelu>(K, V, B, N, H, p, partial, state, s);
        case 32 * 4 + sana::kFeatureElu1: return run_kv_state<32, sana::kFeatureElu1>(K, V, B, N, H, p, partial, state, s);
        case 32 * 4 + sana::kFeatureCos:  return run_kv_state<32, sana::kFeatureCos>(K, V, B, N, H, p, partial, state, s);
        case 64 * 4 + sana::kFeatureRelu: return run_kv_state<64, sana::kFeatureRelu>(K, V, B, N, H, p, partial, state, s);
        case 64 * 4 + sana::kFeatureElu1: return run_kv_state<64, sana::kFeatureElu1>(K, V, B, N, H, p, partial, state, s);
        case 64 * 4 + sana::kFeatureCos:  return run_kv_state<64, sana::kFeatureCos>(K, V, B, N, H, p, partial, state, s);
    }
    return SANA_LA_ERR_INVALID_ARG;
}

// state_nblk > 0: the states are (B, H, state_nblk, d, d+1) and this call
// applies blocks blk0, blk0 + 1, ... of them (block-causal host-buffer chunks)
sana_la_status apply_impl(const void* Q, const float* state, int B, int N, int H, int d, int L,
                          void* O, sana_la_out_dtype od, float eps, cudaStream_t s, bool overlap,
                          int fm = sana::kFeatureRelu, int state_nblk = 0, int blk0 = 0) {
    const int sn = state_nblk, b0 = blk0;
    switch (d * 4 + fm) {
        case 32 * 4 + sana::kFeatureRelu: return run_apply<32, sana::kFeatureRelu>(Q, state, B, N, H, L, O, od, eps, s, overlap, sn, b0);
        case 32 * 4 + sana::kFeatureElu1: return run_apply<32, sana::kFeatureElu1>(Q, state, B, N, H, L, O, od, eps, s, overlap, sn, b0);
        case 32 * 4 + sana::kFeatureCos:  return run_apply<32, sana::kFeatureCos>(Q, state, B, N, H, L, O, od, eps, s, overlap, sn, b0);
        case 64 * 4 + sana::kFeatureRelu: return run_apply<64, sana::kFeatureRelu>(Q, state, B, N, H, L, O, od, eps, s, overlap, sn, b0);
        case 64 * 4 + sana::kFeatureElu1: return run_apply<64, sana::kFeatureElu1>(Q, state, B, N, H, L, O, od, eps, s, overlap, sn, b0);
        case 64 * 4 + sana::kFeatureCos:  return run_apply<64, sana::kFeatureCos>(Q, state, B, N, H, L, O, od, eps, s, overlap, sn, b0);
    }
    return SANA_LA_ERR_INVALID_ARG;
}

// BC: the block-causal instance (running prefix states in `carry`)
template <int FM, bool BC = false>
sana_la_status forward_fused_dispatch(const void* Q, const void* K, const void* V, void* O, int B, int N,
                                      int H, int d, bool bf16, const Plan& p, float* partial,
                                      unsigned long long* flags, cudaStream_t s, float* carry = nullptr) {
    return d == 32
        ? (bf16 ? launch_forward_fused<32, true, FM, BC>(Q, K, V, O, B, N, H, p, partial, flags, carry, s)
                : launch_forward_fused<32, false, FM, BC>(Q, K, V, O, B, N, H, p, partial, flags, carry, s))
        : (bf16 ? launch_forward_fused<64, true, FM, BC>(Q, K, V, O, B, N, H, p, partial, flags, carry, s)
                : launch_forward_fused<64, false, FM, BC>(Q, K, V, O, B, N, H, p, partial, flags, carry, s));
}

bool valid_feature(int fm) {
    return fm == sana::kFeatureRelu || fm == sana::kFeatureElu1 || fm == sana::kFeatureCos;
}

// ------------------------------------------- key-value projection + state ----
struct KpPlan {
    sana::tc::KpParams kp;
    size_t partial_bytes;
};

KpPlan make_kp_plan(int B, int N, int C, int H, int d) {
    const int G = 128 / d;
    const long long groups = cdiv(H, G);
    KpPlan p{};
    p.kp.N = N;
    p.kp.H = H;
    p.kp.groups = (int)groups;
    p.kp.C = C;
    p.kp.kblocks = (int)cdiv(C, 64);
    p.kp.q = make_sched((long long)B * groups, cdiv(N, sana::tc::KP_TILE), device_sms());
    const size_t dd = (size_t)d * (d + 1) * sizeof(float);
    p.partial_bytes = align256((size_t)p.kp.q.grid * p.kp.q.max_seg * G * dd);
    return p;
}

sana_la_status check_projection(int B, int N, int C, int H, int d) {
    sana_la_status st = check_sizes(B, N, H, d);
    if (st != SANA_LA_OK) return st;
    if (C < 1) return SANA_LA_ERR_INVALID_ARG;
    if (C % 8 != 0) return SANA_LA_ERR_UNSUPPORTED;          // TMA row strides are multiples of 16 bytes
    if ((long long)B * N > kMaxElems / C) return SANA_LA_ERR_INVALID_ARG;
    if ((long long)N * C * 2 >= (1LL << 40) || (long long)H * d * C * 2 >= (1LL << 40))
        return SANA_LA_ERR_UNSUPPORTED;
    return SANA_LA_OK;
}

template <int D>
sana_la_status run_kvproj_state(const void* X, const void* Wk, const void* Wv, int B, int N, int C, int H,
                                const KpPlan& p, float* partial, float* state, cudaStream_t s) {
    static std::atomic<unsigned long long> smem_set[kMaxDevicesCached];
    CUtensorMap tmX, tmWk, tmWv;
    sana_la_status st;
    // X as {C, N, B}; the weights as {C, H*d, 1}: 64 features x 128 rows per box
    if ((st = make_tmap(&tmX, X, B, N, 1, C, sana::tc::KP_TILE)) != SANA_LA_OK) return st;
    if ((st = make_tmap(&tmWk, Wk, 1, H * D, 1, C, 128)) != SANA_LA_OK) return st;
    if ((st = make_tmap(&tmWv, Wv, 1, H * D, 1, C, 128)) != SANA_LA_OK) return st;
    if ((st = ensure_smem(sana::tc::kvproj_state_tc<D>, sana::tc::KpMap::BYTES, smem_set)) != SANA_LA_OK)
        return st;
    if ((st = launch(sana::tc::kvproj_state_tc<D>, dim3(p.kp.q.grid), dim3(sana::tc::kThreads),
                     sana::tc::KpMap::BYTES, s, false, "kvproj_state_tc", tmX, tmWk, tmWv, p.kp,
                     partial)) != SANA_LA_OK)
        return st;
    sana::tc::KsParams ksp{};
    ksp.N = N;
    ksp.H = H;
    ksp.groups = p.kp.groups;
    ksp.q = p.kp.q;
    const dim3 kr_grid((unsigned)((long long)B * H), (D * (D + 1) + sana::tc::KR_THREADS - 1) / sana::tc::KR_THREADS);
    return launch(sana::tc::kr_reduce_tc<D>, kr_grid, dim3(sana::tc::KR_THREADS), 0, s, true, "kr_reduce_tc",
                  (const float*)partial, ksp, state);
}

// ------------------------------------------------------------- Mix-FFN ----
struct FfnPlan {
    size_t u_bytes, z_bytes;
};

FfnPlan make_ffn_plan(int B, int Hg, int Wg, int Ch) {
    const size_t tokens = (size_t)B * Hg * Wg;
    return FfnPlan{align256(tokens * 2 * Ch * 2), align256(tokens * Ch * 2)};
}

sana_la_status check_ffn(int B, int Hg, int Wg, int C, int Ch) {
    if (B < 1 || Hg < 1 || Wg < 1 || C < 1 || Ch < 1) return SANA_LA_ERR_INVALID_ARG;
    if (C % 8 != 0 || Ch % 8 != 0) return SANA_LA_ERR_UNSUPPORTED;   // 16-byte rows and vectors
    const long long tokens = (long long)B * Hg * Wg;
    if (tokens > 0x7fffffffLL) return SANA_LA_ERR_UNSUPPORTED;
    if (tokens > kMaxElems / (2LL * Ch) || tokens > kMaxElems / C) return SANA_LA_ERR_INVALID_ARG;
    if (tokens * 2LL * Ch * 2 >= (1LL << 40) || tokens * (long long)C * 2 >= (1LL << 40))
        return SANA_LA_ERR_UNSUPPORTED;
    return SANA_LA_OK;
}

// C (M x N, row stride ldc) = A (M x K) B^T (B is N x K), bf16 in and out
// C = A B^T on CTA pairs (256 x 256 tiles, tcgen05.mma.cta_group::2) or, with
// kGemmPairs = false, on single CTAs (128 x 256 tiles).
constexpr bool kGemmPairs = true;

sana_la_status launch_gemm_pairs(const void* A, const void* Bm, void* C, int M, int N, int K, int ldc,
                                 cudaStream_t s) {
    static std::atomic<unsigned long long> smem_set[kMaxDevicesCached];
    CUtensorMap tmA, tmB;
    sana_la_status st;
    if ((st = make_tmap(&tmA, A, 1, M, 1, K, 128)) != SANA_LA_OK) return st;
    if ((st = make_tmap(&tmB, Bm, 1, N, 1, K, 128)) != SANA_LA_OK) return st;
    if ((st = ensure_smem(sana::tc::gemm_bf16_tc2, sana::tc::Gemm2Map::BYTES, smem_set)) != SANA_LA_OK) return st;
    sana::tc::GemmParams gp{};
    gp.M = M;
    gp.N = N;
    gp.K = K;
    gp.ldc = ldc;
    gp.kblocks = (int)cdiv(K, 64);
    gp.mtiles = (int)cdiv(M, sana::tc::G2_TILE_M);
    gp.ntiles = (int)cdiv(N, sana::tc::G2_TILE_N);
    const long long tiles = (long long)gp.mtiles * gp.ntiles;
    const int pairs = (int)std::min<long long>(tiles, device_sms() / 2);
    return launch(sana::tc::gemm_bf16_tc2, dim3(2 * pairs), dim3(sana::tc::kThreads), sana::tc::Gemm2Map::BYTES, s,
                  false, "gemm_bf16_tc2", tmA, tmB, gp, static_cast<__nv_bfloat16*>(C));
}

sana_la_status launch_gemm(const void* A, const void* Bm, void* C, int M, int N, int K, int ldc, cudaStream_t s) {
    if (kGemmPairs) return launch_gemm_pairs(A, Bm, C, M, N, K, ldc, s);
    static std::atomic<unsigned long long> smem_set[kMaxDevicesCached];
    CUtensorMap tmA, tmB;
    sana_la_status st;
    if ((st = make_tmap(&tmA, A, 1, M, 1, K, sana::tc::GM_TILE_M)) != SANA_LA_OK) return st;
    if ((st = make_tmap(&tmB, Bm, 1, N, 1, K, sana::tc::GM_TILE_N)) != SANA_LA_OK) return st;
    if ((st = ensure_smem(sana::tc::gemm_bf16_tc, sana::tc::GemmMap::BYTES, smem_set)) != SANA_LA_OK) return st;
    sana::tc::GemmParams gp{};
    gp.M = M;
    gp.N = N;
    gp.K = K;
    gp.ldc = ldc;
    gp.kblocks = (int)cdiv(K, 64);
    gp.mtiles = (int)cdiv(M, sana::tc::GM_TILE_M);
    gp.ntiles = (int)cdiv(N, sana::tc::GM_TILE_N);
    const long long tiles = (long long)gp.mtiles * gp.ntiles;
    const int grid = (int)std::min<long long>(tiles, device_sms());
    return launch(sana::tc::gemm_bf16_tc, dim3(grid), dim3(sana::tc::kThreads), sana::tc::GemmMap::BYTES, s,
                  false, "gemm_bf16_tc", tmA, tmB, gp, static_cast<__nv_bfloat16*>(C));
}

sana_la_status kv_state_entry(const void* K, const void* V, int B, int N, int H, int d, int fm,
                              float* state, void* workspace, size_t workspace_bytes,
                              sana_la_stream_t stream) {
    g_last_error[0] = '\0';
    if (!K || !V || !state || !workspace || !valid_feature(fm)) return SANA_LA_ERR_INVALID_ARG;
    sana_la_status st = check_sizes(B, N, H, d);
    if (st != SANA_LA_OK) return st;
    if (!aligned16(K) || !aligned16(V) || !aligned16(state) || !aligned16(workspace))
        return SANA_LA_ERR_INVALID_ARG;
    return kv_state_impl(K, V, B, N, H, d, 0, state, workspace, workspace_bytes,
                         reinterpret_cast<cudaStream_t>(stream), false, fm);
}

sana_la_status apply_entry(const void* Q, const float* state, int B, int N, int H, int d, int fm,
                           void* O, sana_la_out_dtype out_dtype, float eps, sana_la_stream_t stream) {
    g_last_error[0] = '\0';
    if (!Q || !state || !O || !valid_feature(fm)) return SANA_LA_ERR_INVALID_ARG;
    sana_la_status st = check_sizes(B, N, H, d);
    if (st != SANA_LA_OK) return st;
    if (out_dtype != SANA_LA_OUT_F32 && out_dtype != SANA_LA_OUT_BF16) return SANA_LA_ERR_INVALID_ARG;
    if ((st = check_eps(eps)) != SANA_LA_OK) return st;
    if (!aligned16(Q) || !aligned16(state) || !aligned16(O)) return SANA_LA_ERR_INVALID_ARG;
    return apply_impl(Q, state, B, N, H, d, 0, O, out_dtype, eps,
                      reinterpret_cast<cudaStream_t>(stream), false, fm);
}

sana_la_status forward_entry(const void* Q, const void* K, const void* V, int B, int N, int H, int d, int fm,
                             void* O, sana_la_out_dtype out_dtype, float eps, void* workspace,
                             size_t workspace_bytes, sana_la_stream_t stream) {
    g_last_error[0] = '\0';
    if (!Q || !K || !V || !O || !workspace || !valid_feature(fm)) return SANA_LA_ERR_INVALID_ARG;
    sana_la_status st = check_sizes(B, N, H, d);
    if (st != SANA_LA_OK) return st;
    if (out_dtype != SANA_LA_OUT_F32 && out_dtype != SANA_LA_OUT_BF16) return SANA_LA_ERR_INVALID_ARG;
    if ((st = check_eps(eps)) != SANA_LA_OK) return st;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(workspace))
        return SANA_LA_ERR_INVALID_ARG;
    Plan p = make_plan(B, N, H, d);
    if (workspace_bytes < p.partial_bytes + p.state_bytes + p.flag_bytes) return SANA_LA_ERR_WORKSPACE;
    char* ws = static_cast<char*>(workspace);
    float* partial = reinterpret_cast<float*>(ws);
    float* state = reinterpret_cast<float*>(ws + p.partial_bytes);
    auto* flags = reinterpret_cast<unsigned long long*>(ws + p.partial_bytes + p.state_bytes);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // one cooperative launch: state phase, per-slab readiness flags, apply phase
    p.ka.eps = eps;
    const bool bf16 = out_dtype == SANA_LA_OUT_BF16;
    switch (fm) {
        case sana::kFeatureElu1:
            st = forward_fused_dispatch<sana::kFeatureElu1>(Q, K, V, O, B, N, H, d, bf16, p, partial, flags, s);
            break;
        case sana::kFeatureCos:
            st = forward_fused_dispatch<sana::kFeatureCos>(Q, K, V, O, B, N, H, d, bf16, p, partial, flags, s);
            break;
        default:
            st = forward_fused_dispatch<sana::kFeatureRelu>(Q, K, V, O, B, N, H, d, bf16, p, partial, flags, s);
    }
    if (st != SANA_LA_ERR_UNSUPPORTED) return st;
    // the device cannot hold the whole grid at once: the same kernels as
    // kv_state + apply, overlapped by programmatic launch
    st = kv_state_impl(K, V, B, N, H, d, 0, state, workspace, p.partial_bytes, s, false, fm);
    if (st != SANA_LA_OK) return st;
    return apply_impl(Q, state, B, N, H, d, 0, O, out_dtype, eps, s, true, fm);
}

// ------------------------------------------------- host-buffer forward ----
// Device layout of the host-buffer forward's workspace: Q, K, V and O staging,
// the state, and the state kernels' partials, each 256-byte aligned.
struct HostPlan {
    size_t q, kv, o, state, partial, total;
};

// L > 0: the block-causal form (prefix states of blocks of L tokens)
HostPlan make_host_plan(int B, int N, int H, int d, sana_la_out_dtype od, int L = 0) {
    const Plan p = make_plan(B, N, H, d, L);
    const size_t elems = (size_t)B * N * H * d;
    const size_t nblk = L > 0 ? (size_t)cdiv(N, L) : 1;
    HostPlan h{};
    h.q = align256(elems * 2);
    h.kv = align256(elems * 2);
    h.o = align256(elems * (od == SANA_LA_OUT_F32 ? 4 : 2));
    h.state = align256((size_t)B * H * nblk * d * (d + 1) * sizeof(float));
    h.partial = p.partial_bytes;
    h.total = h.q + 2 * h.kv + h.o + h.state + h.partial;
    return h;
}

// Q is streamed in chunks of about 1/16 of the tokens (at least 1024): chunks
// of whole batches when a batch is shorter, else pieces of one batch.
struct HostChunks {
    long long tokens;   // tokens per chunk within a batch (N when chunks are whole batches)
    int batches;        // batches per chunk (1 when a batch is split)
    int count;
};

HostChunks host_chunks(int B, int N, int L = 0) {
    const long long target = std::max<long long>(1024, cdiv((long long)B * N, 16));
    HostChunks c{};
    if (L > 0) {
        // block-causal: whole blocks of one batch (each block's queries use
        // that block's prefix state), about `target` tokens per chunk
        const long long nblk = cdiv(N, L);
        const long long bpc = std::min<long long>(nblk, std::max<long long>(1, target / L));
        c.tokens = bpc * L;
        c.batches = 1;
        c.count = (int)(B * cdiv(nblk, bpc));
        return c;
    }
    if (N >= target) {
        c.tokens = cdiv(target, 128) * 128;
        c.batches = 1;
        c.count = (int)(B * cdiv(N, c.tokens));
    } else {
        c.tokens = N;
        c.batches = (int)std::max<long long>(1, target / N);
        c.count = (int)cdiv(B, c.batches);
    }
    return c;
}

// The library's copy streams (host to device, device to host) and rings of
// events, per device, made on first use. A ring entry is recorded and waited
// for right away, so reusing it later (a newer record) is safe.
constexpr int kHostEvents = 32;
struct CopyCtx {
    cudaStream_t h2d = nullptr;
    cudaStream_t d2h = nullptr;
    cudaEvent_t in[kHostEvents] = {};       // a chunk of Q (or K and V) is on the device
    cudaEvent_t out[kHostEvents] = {};      // a chunk's O is ready to be copied back
    cudaEvent_t start = nullptr;            // the caller's earlier work on its stream is done
    cudaEvent_t join = nullptr;             // the last copy back is done
    bool ready = false;
    unsigned long long context = 0;         // the context the streams and events belong to
    // Held while a call enqueues: an event must be waited for before another
    // call records it again from a different stream.
    std::mutex enqueue;
};
CopyCtx g_copy_ctx[kMaxDevicesCached];
std::mutex g_copy_ctx_mutex;

sana_la_status copy_ctx(CopyCtx** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        set_last_error("cudaGetDevice", e);
        return SANA_LA_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevicesCached) return SANA_LA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_copy_ctx_mutex);
    CopyCtx& c = g_copy_ctx[dev];
    const unsigned long long context = current_context_id();
    if (c.ready && context != 0 && context != c.context) {
        // made in a context that has since been destroyed: its handles went
        // with it (they are not destroyed here); make new ones in this context
        c.h2d = c.d2h = nullptr;
        for (int i = 0; i < kHostEvents; ++i) c.in[i] = c.out[i] = nullptr;
        c.start = c.join = nullptr;
        c.ready = false;
    }
    if (!c.ready) {
        e = cudaStreamCreateWithFlags(&c.h2d, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&c.d2h, cudaStreamNonBlocking);
        for (int i = 0; i < kHostEvents && e == cudaSuccess; ++i) {
            e = cudaEventCreateWithFlags(&c.in[i], cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c.out[i], cudaEventDisableTiming);
        }
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c.start, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c.join, cudaEventDisableTiming);
        if (e != cudaSuccess) {
            set_last_error("copy stream and events", e);
            // free what was made, so that a later call starts over cleanly
            auto drop_event = [](cudaEvent_t& ev) {
                if (ev != nullptr) cudaEventDestroy(ev);
                ev = nullptr;
            };
            auto drop_stream = [](cudaStream_t& st) {
                if (st != nullptr) cudaStreamDestroy(st);
                st = nullptr;
            };
            drop_event(c.start);
            drop_event(c.join);
            for (int i = 0; i < kHostEvents; ++i) {
                drop_event(c.in[i]);
                drop_event(c.out[i]);
            }
            drop_stream(c.h2d);
            drop_stream(c.d2h);
            return SANA_LA_ERR_CUDA;
        }
        c.ready = true;
        c.context = current_context_id();
    }
    *out = &c;
    return SANA_LA_OK;
}

// `waiter` waits for the work enqueued on `signaler` so far (through `ev`).
sana_la_status stream_after(cudaStream_t waiter, cudaStream_t signaler, cudaEvent_t ev, const char* what) {
    cudaError_t e = cudaEventRecord(ev, signaler);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(waiter, ev, 0);
    if (e != cudaSuccess) {
        set_last_error(what, e);
        return SANA_LA_ERR_CUDA;
    }
    return SANA_LA_OK;
}

sana_la_status copy_async(void* dst, const void* src, size_t bytes, cudaMemcpyKind kind, cudaStream_t s) {
    cudaError_t e = cudaMemcpyAsync(dst, src, bytes, kind, s);
    if (e != cudaSuccess) {
        set_last_error(kind == cudaMemcpyHostToDevice ? "cudaMemcpyAsync (to device)" : "cudaMemcpyAsync (to host)", e);
        return SANA_LA_ERR_CUDA;
    }
    return SANA_LA_OK;
}

// L > 0: the block-causal form (phi = ReLU)
sana_la_status forward_host_entry(const void* hQ, const void* hK, const void* hV, int B, int N, int H, int d,
                                  int fm, void* hO, sana_la_out_dtype out_dtype, float eps, void* workspace,
                                  size_t workspace_bytes, sana_la_stream_t stream, int L = 0) {
    g_last_error[0] = '\0';
    if (!hQ || !hK || !hV || !hO || !workspace || !valid_feature(fm)) return SANA_LA_ERR_INVALID_ARG;
    sana_la_status st = check_sizes(B, N, H, d);
    if (st != SANA_LA_OK) return st;
    if (L != 0 && (st = check_block(B, N, H, d, L)) != SANA_LA_OK) return st;
    if (out_dtype != SANA_LA_OUT_F32 && out_dtype != SANA_LA_OUT_BF16) return SANA_LA_ERR_INVALID_ARG;
    if ((st = check_eps(eps)) != SANA_LA_OK) return st;
    if (!aligned16(workspace)) return SANA_LA_ERR_INVALID_ARG;
    const HostPlan hp = make_host_plan(B, N, H, d, out_dtype, L);
    if (workspace_bytes < hp.total) return SANA_LA_ERR_WORKSPACE;
    CopyCtx* cc = nullptr;
    if ((st = copy_ctx(&cc)) != SANA_LA_OK) return st;
    std::lock_guard<std::mutex> enqueue_lock(cc->enqueue);
    char* ws = static_cast<char*>(workspace);
    char* dQ = ws;
    char* dK = dQ + hp.q;
    char* dV = dK + hp.kv;
    char* dO = dV + hp.kv;
    float* state = reinterpret_cast<float*>(dO + hp.o);
    void* partial = dO + hp.o + hp.state;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t row_in = (size_t)H * d * 2;                                  // bytes per token
    const size_t row_out = (size_t)H * d * (out_dtype == SANA_LA_OUT_F32 ? 4 : 2);
    const size_t tokens = (size_t)B * N;
    // Three queues: host-to-device copies on the library's h2d stream, the
    // kernels on `s`, device-to-host copies on its d2h stream. The copies in
    // start after the caller's earlier work on `s` (which may still use the
    // workspace); K and V go first, then every chunk of Q back to back, so
    // the host-to-device direction never waits for a kernel.
    if ((st = stream_after(cc->h2d, s, cc->start, "start event")) != SANA_LA_OK) return st;
    if ((st = copy_async(dK, hK, tokens * row_in, cudaMemcpyHostToDevice, cc->h2d)) != SANA_LA_OK) return st;
    if ((st = copy_async(dV, hV, tokens * row_in, cudaMemcpyHostToDevice, cc->h2d)) != SANA_LA_OK) return st;
    if ((st = stream_after(s, cc->h2d, cc->in[0], "K, V event")) != SANA_LA_OK) return st;
    if ((st = kv_state_impl(dK, dV, B, N, H, d, L, state, partial, hp.partial, s, false, fm)) != SANA_LA_OK)
        return st;
    const HostChunks hc = host_chunks(B, N, L);
    const long long per_batch = cdiv(N, hc.tokens);
    const int nblk = L > 0 ? (int)cdiv(N, L) : 1;
    const size_t state_stride = (size_t)H * nblk * d * (d + 1);     // one batch's states
    auto chunk = [&](int c, int& b0, int& nb, int& t0, int& nt) {
        if (hc.batches > 1 || hc.tokens >= N) {
            b0 = c * hc.batches;
            nb = std::min(hc.batches, B - b0);
            t0 = 0;
            nt = N;
        } else {
            b0 = (int)(c / per_batch);
            nb = 1;
            t0 = (int)((c % per_batch) * hc.tokens);
            nt = (int)std::min<long long>(hc.tokens, N - t0);
        }
    };
    for (int c = 0; c < hc.count; ++c) {
        int b0, nb, t0, nt;
        chunk(c, b0, nb, t0, nt);
        const size_t first = (size_t)b0 * N + t0;                       // first token of the chunk
        const size_t rows = (size_t)nb * nt;                             // tokens in the chunk
        // Q of the chunk in (h2d), its apply (s), its O back (d2h)
        if ((st = copy_async(dQ + first * row_in, static_cast<const char*>(hQ) + first * row_in, rows * row_in,
                             cudaMemcpyHostToDevice, cc->h2d)) != SANA_LA_OK)
            return st;
        if ((st = stream_after(s, cc->h2d, cc->in[(c + 1) % kHostEvents], "chunk in event")) != SANA_LA_OK)
            return st;
        // block-causal: the chunk is blocks t0 / L, ... of batch b0, applied
        // against that batch's prefix states (nblk of them, from block t0 / L)
        if ((st = apply_impl(dQ + first * row_in, state + (size_t)b0 * state_stride, nb, nt, H, d, L,
                             dO + first * row_out, out_dtype, eps, s, false, fm, L > 0 ? nblk : 0,
                             L > 0 ? t0 / L : 0)) != SANA_LA_OK)
            return st;
        if ((st = stream_after(cc->d2h, s, cc->out[c % kHostEvents], "chunk out event")) != SANA_LA_OK)
            return st;
        if ((st = copy_async(static_cast<char*>(hO) + first * row_out, dO + first * row_out, rows * row_out,
                             cudaMemcpyDeviceToHost, cc->d2h)) != SANA_LA_OK)
            return st;
    }
    // `s` ends after the last copy back
    if ((st = stream_after(s, cc->d2h, cc->join, "join event")) != SANA_LA_OK) return st;
    return SANA_LA_OK;
}

}  // namespace

extern "C" {

size_t sana_linattn_workspace_bytes(int B, int N, int H, int d) {
    if (check_sizes(B, N, H, d) != SANA_LA_OK) return 0;
    const Plan p = make_plan(B, N, H, d);
    return p.partial_bytes + p.state_bytes + p.flag_bytes;
}

sana_la_status sana_linattn_kv_state(const void* K, const void* V, int B, int N, int H, int d,
                                     float* state, void* workspace, size_t workspace_bytes,
                                     sana_la_stream_t stream) {
    return kv_state_entry(K, V, B, N, H, d, sana::kFeatureRelu, state, workspace, workspace_bytes, stream);
}

sana_la_status sana_linattn_apply(const void* Q, const float* state, int B, int N, int H, int d,
                                  void* O, sana_la_out_dtype out_dtype, float eps,
                                  sana_la_stream_t stream) {
    return apply_entry(Q, state, B, N, H, d, sana::kFeatureRelu, O, out_dtype, eps, stream);
}

sana_la_status sana_linattn_forward(const void* Q, const void* K, const void* V,
                                    int B, int N, int H, int d,
                                    void* O, sana_la_out_dtype out_dtype, float eps,
                                    void* workspace, size_t workspace_bytes,
                                    sana_la_stream_t stream) {
    return forward_entry(Q, K, V, B, N, H, d, sana::kFeatureRelu, O, out_dtype, eps, workspace,
                         workspace_bytes, stream);
}

// ------------------------------------------------------- feature maps ----
sana_la_status sana_linattn_kv_state_fm(const void* K, const void* V, int B, int N, int H, int d,
                                        sana_la_feature_map feature_map, float* state, void* workspace,
                                        size_t workspace_bytes, sana_la_stream_t stream) {
    return kv_state_entry(K, V, B, N, H, d, (int)feature_map, state, workspace, workspace_bytes, stream);
}

sana_la_status sana_linattn_apply_fm(const void* Q, const float* state, int B, int N, int H, int d,
                                     sana_la_feature_map feature_map, void* O, sana_la_out_dtype out_dtype,
                                     float eps, sana_la_stream_t stream) {
    return apply_entry(Q, state, B, N, H, d, (int)feature_map, O, out_dtype, eps, stream);
}

sana_la_status sana_linattn_forward_fm(const void* Q, const void* K, const void* V,
                                       int B, int N, int H, int d, sana_la_feature_map feature_map,
                                       void* O, sana_la_out_dtype out_dtype, float eps,
                                       void* workspace, size_t workspace_bytes,
                                       sana_la_stream_t stream) {
    return forward_entry(Q, K, V, B, N, H, d, (int)feature_map, O, out_dtype, eps, workspace,
                         workspace_bytes, stream);
}

// ------------------------------------------- key-value projection + state ----
size_t sana_linattn_kv_projection_workspace_bytes(int B, int N, int C, int H, int d) {
    if (check_projection(B, N, C, H, d) != SANA_LA_OK) return 0;
    return make_kp_plan(B, N, C, H, d).partial_bytes;
}

sana_la_status sana_linattn_kv_projection_state(const void* X, const void* Wk, const void* Wv,
                                                int B, int N, int C, int H, int d, float* state,
                                                void* workspace, size_t workspace_bytes,
                                                sana_la_stream_t stream) {
    g_last_error[0] = '\0';
    if (!X || !Wk || !Wv || !state || !workspace) return SANA_LA_ERR_INVALID_ARG;
    sana_la_status st = check_projection(B, N, C, H, d);
    if (st != SANA_LA_OK) return st;
    if (!aligned16(X) || !aligned16(Wk) || !aligned16(Wv) || !aligned16(state) || !aligned16(workspace))
        return SANA_LA_ERR_INVALID_ARG;
    const KpPlan p = make_kp_plan(B, N, C, H, d);
    if (workspace_bytes < p.partial_bytes) return SANA_LA_ERR_WORKSPACE;
    float* partial = static_cast<float*>(workspace);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return d == 32 ? run_kvproj_state<32>(X, Wk, Wv, B, N, C, H, p, partial, state, s)
                   : run_kvproj_state<64>(X, Wk, Wv, B, N, C, H, p, partial, state, s);
}

int sana_linattn_kv_projection_state_launches(int B, int N, int C, int H, int d) {
    return check_projection(B, N, C, H, d) == SANA_LA_OK ? 2 : 0;   // kvproj_state_tc, kr_reduce_tc
}

// ------------------------------------------------------------- Mix-FFN ----
size_t sana_linattn_mix_ffn_workspace_bytes(int B, int Hg, int Wg, int C, int Ch) {
    if (check_ffn(B, Hg, Wg, C, Ch) != SANA_LA_OK) return 0;
    const FfnPlan p = make_ffn_plan(B, Hg, Wg, Ch);
    return p.u_bytes + p.z_bytes;
}

sana_la_status sana_linattn_mix_ffn(const void* X, const void* W1, const float* Kdw, const void* W2,
                                    int B, int Hg, int Wg, int C, int Ch, void* Y,
                                    void* workspace, size_t workspace_bytes, sana_la_stream_t stream) {
    g_last_error[0] = '\0';
    if (!X || !W1 || !Kdw || !W2 || !Y || !workspace) return SANA_LA_ERR_INVALID_ARG;
    sana_la_status st = check_ffn(B, Hg, Wg, C, Ch);
    if (st != SANA_LA_OK) return st;
    if (!aligned16(X) || !aligned16(W1) || !aligned16(W2) || !aligned16(Y) || !aligned16(workspace) ||
        (reinterpret_cast<uintptr_t>(Kdw) & 3) != 0)
        return SANA_LA_ERR_INVALID_ARG;
    const FfnPlan p = make_ffn_plan(B, Hg, Wg, Ch);
    if (workspace_bytes < p.u_bytes + p.z_bytes) return SANA_LA_ERR_WORKSPACE;
    char* ws = static_cast<char*>(workspace);
    void* U = ws;
    void* Z = ws + p.u_bytes;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int M = B * Hg * Wg;
    // 1x1 expand: U = X W1^T (2 Ch channels)
    if ((st = launch_gemm(X, W1, U, M, 2 * Ch, C, 2 * Ch, s)) != SANA_LA_OK) return st;
    // 3x3 depthwise over the grid and the GLU, fused
    using DwC = sana::tc::DwConfig;
    static std::atomic<unsigned long long> dw_smem_set[kMaxDevicesCached];
    if ((st = ensure_smem(sana::tc::dwconv_glu<DwC>, DwC::SMEM, dw_smem_set)) != SANA_LA_OK) return st;
    // U as {2 Ch, Wg, Hg, B}: a load box is 64 channels x (TX + 2) columns x
    // (TY + 2) rows; Z as {Ch, Wg, Hg, B}: a store box is 64 x TX x TY
    CUtensorMap tmU, tmZ;
    {
        auto encode = tensor_map_encoder();
        if (encode == nullptr) return SANA_LA_ERR_CUDA;
        cuuint32_t estr[4] = {1, 1, 1, 1};
        for (int which = 0; which < 2; ++which) {
            const cuuint64_t ch = which == 0 ? (cuuint64_t)2 * Ch : (cuuint64_t)Ch;
            cuuint64_t dims[4] = {ch, (cuuint64_t)Wg, (cuuint64_t)Hg, (cuuint64_t)B};
            cuuint64_t strides[3] = {ch * 2, ch * 2 * Wg, ch * 2 * Wg * Hg};
            const int halo = which == 0 ? 2 : 0;
            cuuint32_t box[4] = {(cuuint32_t)sana::tc::DW_CH, (cuuint32_t)(DwC::TX + halo),
                                 (cuuint32_t)(DwC::TY + halo), 1};
            CUresult r = encode(which == 0 ? &tmU : &tmZ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                                which == 0 ? U : Z, dims, strides, box, estr,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
            if (r != CUDA_SUCCESS) {
                std::snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled failed (%d)", (int)r);
                return SANA_LA_ERR_CUDA;
            }
        }
    }
    const long long dw_ctas = (long long)B * cdiv(Hg, DwC::TY) * cdiv(Wg, DwC::TX) * cdiv(Ch, sana::tc::DW_CH);
    if (dw_ctas > 0x7fffffffLL) return SANA_LA_ERR_UNSUPPORTED;
    const dim3 dw_grid((unsigned)dw_ctas);
    if ((st = launch(sana::tc::dwconv_glu<DwC>, dw_grid, dim3(DwC::THREADS), DwC::SMEM, s,
                     false, "dwconv_glu", tmU, tmZ, Kdw, Hg, Wg, Ch)) != SANA_LA_OK)
        return st;
    // 1x1 project: Y = Z W2^T
    return launch_gemm(Z, W2, Y, M, C, Ch, C, s);
}

int sana_linattn_mix_ffn_launches(int B, int Hg, int Wg, int C, int Ch) {
    return check_ffn(B, Hg, Wg, C, Ch) == SANA_LA_OK ? 3 : 0;   // gemm, dwconv_glu, gemm
}

// ------------------------------------------------------- block-causal ----
// Block-causal workspace: the partial states, then either the prefix states
// (three-kernel form) or the single launch's flags and per-CTA running prefixes.
size_t block_causal_ws_bytes(const Plan& p) {
    return p.partial_bytes + std::max(p.state_bytes, p.flag_bytes + p.carry_bytes);
}

size_t sana_linattn_block_causal_workspace_bytes(int B, int N, int H, int d, int L) {
    if (check_sizes(B, N, H, d) != SANA_LA_OK || check_block(B, N, H, d, L) != SANA_LA_OK) return 0;
    return block_causal_ws_bytes(make_plan(B, N, H, d, L));
}

sana_la_status sana_linattn_block_causal_kv_state(const void* K, const void* V, int B, int N, int H,
                                                  int d, int L, float* states, void* workspace,
                                                  size_t workspace_bytes, sana_la_stream_t stream) {
    g_last_error[0] = '\0';
    if (!K || !V || !states || !workspace) return SANA_LA_ERR_INVALID_ARG;
    sana_la_status st = check_sizes(B, N, H, d);
    if (st != SANA_LA_OK) return st;
    if ((st = check_block(B, N, H, d, L)) != SANA_LA_OK) return st;
    if (!aligned16(K) || !aligned16(V) || !aligned16(states) || !aligned16(workspace))
        return SANA_LA_ERR_INVALID_ARG;
    return kv_state_impl(K, V, B, N, H, d, L, states, workspace, workspace_bytes,
                         reinterpret_cast<cudaStream_t>(stream), false);
}

sana_la_status sana_linattn_block_causal_apply(const void* Q, const float* states, int B, int N,
                                               int H, int d, int L, void* O,
                                               sana_la_out_dtype out_dtype, float eps,
                                               sana_la_stream_t stream) {
    g_last_error[0] = '\0';
    if (!Q || !states || !O) return SANA_LA_ERR_INVALID_ARG;
    sana_la_status st = check_sizes(B, N, H, d);
    if (st != SANA_LA_OK) return st;
    if ((st = check_block(B, N, H, d, L)) != SANA_LA_OK) return st;
    if (out_dtype != SANA_LA_OUT_F32 && out_dtype != SANA_LA_OUT_BF16) return SANA_LA_ERR_INVALID_ARG;
    if ((st = check_eps(eps)) != SANA_LA_OK) return st;
    if (!aligned16(Q) || !aligned16(states) || !aligned16(O)) return SANA_LA_ERR_INVALID_ARG;
    return apply_impl(Q, states, B, N, H, d, L, O, out_dtype, eps,
                      reinterpret_cast<cudaStream_t>(stream), false);
}

// single: one cooperative launch with running prefix states (fwd_fused_tc,
// block-causal instance); otherwise, and whenever the device cannot hold that
// grid at once, the state kernel and the prefix reduction, then the apply
// kernel (programmatic launch). Bit-identical either way.
static sana_la_status block_causal_forward_entry(const void* Q, const void* K, const void* V, int B, int N,
                                                 int H, int d, int L, void* O, sana_la_out_dtype out_dtype,
                                                 float eps, void* workspace, size_t workspace_bytes,
                                                 sana_la_stream_t stream, bool single) {
    g_last_error[0] = '\0';
    if (!Q || !K || !V || !O || !workspace) return SANA_LA_ERR_INVALID_ARG;
    sana_la_status st = check_sizes(B, N, H, d);
    if (st != SANA_LA_OK) return st;
    if ((st = check_block(B, N, H, d, L)) != SANA_LA_OK) return st;
    if (out_dtype != SANA_LA_OUT_F32 && out_dtype != SANA_LA_OUT_BF16) return SANA_LA_ERR_INVALID_ARG;
    if ((st = check_eps(eps)) != SANA_LA_OK) return st;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(workspace))
        return SANA_LA_ERR_INVALID_ARG;
    Plan p = make_plan(B, N, H, d, L);
    if (workspace_bytes < block_causal_ws_bytes(p)) return SANA_LA_ERR_WORKSPACE;
    char* ws = static_cast<char*>(workspace);
    float* partial = reinterpret_cast<float*>(ws);
    float* states = reinterpret_cast<float*>(ws + p.partial_bytes);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (single) {
        // flags and per-CTA prefixes where the three-kernel form keeps the
        // prefix states
        p.ka.eps = eps;
        auto* flags = reinterpret_cast<unsigned long long*>(ws + p.partial_bytes);
        float* carry = reinterpret_cast<float*>(ws + p.partial_bytes + p.flag_bytes);
        st = forward_fused_dispatch<sana::kFeatureRelu, true>(Q, K, V, O, B, N, H, d,
                                                              out_dtype == SANA_LA_OUT_BF16, p, partial, flags, s,
                                                              carry);
        if (st != SANA_LA_ERR_UNSUPPORTED) return st;
    }
    st = kv_state_impl(K, V, B, N, H, d, L, states, workspace, workspace_bytes, s, true);
    if (st != SANA_LA_OK) return st;
    return apply_impl(Q, states, B, N, H, d, L, O, out_dtype, eps, s, true);
}

sana_la_status sana_linattn_block_causal_forward(const void* Q, const void* K, const void* V,
                                                 int B, int N, int H, int d, int L,
                                                 void* O, sana_la_out_dtype out_dtype, float eps,
                                                 void* workspace, size_t workspace_bytes,
                                                 sana_la_stream_t stream) {
    return block_causal_forward_entry(Q, K, V, B, N, H, d, L, O, out_dtype, eps, workspace, workspace_bytes,
                                      stream, false);
}

int sana_linattn_block_causal_forward_launches(int B, int N, int H, int d, int L) {
    if (check_sizes(B, N, H, d) != SANA_LA_OK || check_block(B, N, H, d, L) != SANA_LA_OK) return 0;
    return 3;   // ks_state_tc, kr_prefix_tc (prefix states), ka_apply_tc
}

sana_la_status sana_linattn_block_causal_forward_single(const void* Q, const void* K, const void* V,
                                                        int B, int N, int H, int d, int L,
                                                        void* O, sana_la_out_dtype out_dtype, float eps,
                                                        void* workspace, size_t workspace_bytes,
                                                        sana_la_stream_t stream) {
    return block_causal_forward_entry(Q, K, V, B, N, H, d, L, O, out_dtype, eps, workspace, workspace_bytes,
                                      stream, true);
}

int sana_linattn_block_causal_forward_single_launches(int B, int N, int H, int d, int L) {
    if (check_sizes(B, N, H, d) != SANA_LA_OK || check_block(B, N, H, d, L) != SANA_LA_OK) return 0;
    return 1;   // fwd_fused_tc (plus a memset of its barrier flags when captured in a graph)
}

size_t sana_linattn_block_causal_forward_host_workspace_bytes(int B, int N, int H, int d, int L,
                                                              sana_la_out_dtype out_dtype) {
    if (check_sizes(B, N, H, d) != SANA_LA_OK || check_block(B, N, H, d, L) != SANA_LA_OK) return 0;
    if (out_dtype != SANA_LA_OUT_F32 && out_dtype != SANA_LA_OUT_BF16) return 0;
    return make_host_plan(B, N, H, d, out_dtype, L).total;
}

sana_la_status sana_linattn_block_causal_forward_host(const void* Q, const void* K, const void* V, int B, int N,
                                                      int H, int d, int L, void* O, sana_la_out_dtype out_dtype,
                                                      float eps, void* workspace, size_t workspace_bytes,
                                                      sana_la_stream_t stream) {
    if (L < 1) {
        g_last_error[0] = '\0';
        return SANA_LA_ERR_INVALID_ARG;
    }
    return forward_host_entry(Q, K, V, B, N, H, d, sana::kFeatureRelu, O, out_dtype, eps, workspace,
                              workspace_bytes, stream, L);
}

int sana_linattn_block_causal_forward_host_launches(int B, int N, int H, int d, int L) {
    if (check_sizes(B, N, H, d) != SANA_LA_OK || check_block(B, N, H, d, L) != SANA_LA_OK) return 0;
    return 2 + host_chunks(B, N, L).count;       // state, prefix states, one apply per chunk
}

size_t sana_linattn_forward_host_workspace_bytes(int B, int N, int H, int d, sana_la_out_dtype out_dtype) {
    if (check_sizes(B, N, H, d) != SANA_LA_OK) return 0;
    if (out_dtype != SANA_LA_OUT_F32 && out_dtype != SANA_LA_OUT_BF16) return 0;
    return make_host_plan(B, N, H, d, out_dtype).total;
}

sana_la_status sana_linattn_forward_host(const void* Q, const void* K, const void* V, int B, int N, int H, int d,
                                         sana_la_feature_map feature_map, void* O, sana_la_out_dtype out_dtype,
                                         float eps, void* workspace, size_t workspace_bytes,
                                         sana_la_stream_t stream) {
    return forward_host_entry(Q, K, V, B, N, H, d, (int)feature_map, O, out_dtype, eps, workspace,
                              workspace_bytes, stream);
}

int sana_linattn_forward_host_launches(int B, int N, int H, int d) {
    if (check_sizes(B, N, H, d) != SANA_LA_OK) return 0;
    return 2 + host_chunks(B, N).count;          // state, reduction, one apply per chunk
}

int sana_linattn_forward_launches(int B, int N, int H, int d) {
    if (check_sizes(B, N, H, d) != SANA_LA_OK) return 0;
    return 1;   // fwd_fused_tc (plus a memset of its barrier flags when captured in a graph)
}

const char* sana_linattn_build_info(void) { return "impl=tcgen05-tma;bound=hbm"; }

sana_la_status sana_linattn_device_error(unsigned int* code, int clear) {
    g_last_error[0] = '\0';
    if (!code) return SANA_LA_ERR_INVALID_ARG;
    uint32_t v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, sana::tc::g_device_error, sizeof(v));
    if (e != cudaSuccess) {
        set_last_error("cudaMemcpyFromSymbol", e);
        return SANA_LA_ERR_CUDA;
    }
    if (clear && v != 0) {
        const uint32_t zero = 0;
        e = cudaMemcpyToSymbol(sana::tc::g_device_error, &zero, sizeof(zero));
        if (e != cudaSuccess) {
            set_last_error("cudaMemcpyToSymbol", e);
            return SANA_LA_ERR_CUDA;
        }
    }
    *code = v;
    return SANA_LA_OK;
}

sana_la_status sana_linattn_selftest_wait_timeout(unsigned int limit_us, sana_la_stream_t stream) {
    g_last_error[0] = '\0';
    if (limit_us == 0 || limit_us > 10000000u) return SANA_LA_ERR_INVALID_ARG;
    sana::tc::wait_timeout_selftest<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        (uint64_t)limit_us * 1000ull);
    return launch_status("wait_timeout_selftest");
}

const char* sana_linattn_status_string(sana_la_status status) {
    switch (status) {
        case SANA_LA_OK: return "ok";
        case SANA_LA_ERR_INVALID_ARG: return "invalid argument";
        case SANA_LA_ERR_UNSUPPORTED:
            return "unsupported sizes (d must be 32 or 64; the other limits are in the header)";
        case SANA_LA_ERR_WORKSPACE: return "workspace too small";
        case SANA_LA_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

const char* sana_linattn_last_error(void) { return g_last_error; }

}  // extern "C"

// ----------------------------------------------------------------------------
// Forward without caller-provided scratch.
//
// The scratch that sana_linattn_forward takes as `workspace` lives here in a
// fixed device array instead. Loading this library reserves it on every GPU
// that uses the library, until the process exits. Every call on a device
// shares the one array: calls whose kernels overlap on that device (different
// streams, no ordering between them) race on it. Nothing in it has to start at
// zero: each call writes every byte it later reads.
namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;   // 16 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_static_scratch_mutex;
void* g_static_scratch_ptr[kMaxDevices] = {};
unsigned long long g_static_scratch_context[kMaxDevices] = {};

// Device address of g_static_scratch on the current device. The host-side
// name is only a stand-in; the address comes from cudaGetSymbolAddress, asked
// once per device (with that device current) and cached with the context it
// belongs to, and asked again when the device's context changed (a context
// destroyed and made anew, e.g. by cudaDeviceReset, reloads the module).
sana_la_status static_scratch_address(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        set_last_error("cudaGetDevice", e);
        return SANA_LA_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) {
        std::snprintf(g_last_error, sizeof(g_last_error),
                      "device ordinal %d is beyond the %d devices the static scratch address table holds",
                      dev, kMaxDevices);
        return SANA_LA_ERR_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> lock(g_static_scratch_mutex);
    const unsigned long long context = current_context_id();
    if (g_static_scratch_ptr[dev] == nullptr ||
        (context != 0 && context != g_static_scratch_context[dev])) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess || p == nullptr) {
            set_last_error("cudaGetSymbolAddress(g_static_scratch)", e);
            return SANA_LA_ERR_CUDA;
        }
        g_static_scratch_ptr[dev] = p;
        g_static_scratch_context[dev] = current_context_id();
    }
    *out = g_static_scratch_ptr[dev];
    return SANA_LA_OK;
}

}  // namespace

extern "C" sana_la_status sana_linattn_forward_noalloc(const void* Q, const void* K, const void* V,
                                                       int B, int N, int H, int d,
                                                       void* O, sana_la_out_dtype out_dtype,
                                                       float eps, sana_la_stream_t stream) {
    g_last_error[0] = '\0';
    if (!Q || !K || !V || !O) return SANA_LA_ERR_INVALID_ARG;
    sana_la_status st = check_sizes(B, N, H, d);
    if (st != SANA_LA_OK) return st;
    const size_t need = sana_linattn_workspace_bytes(B, N, H, d);
    if (need > kStaticScratchBytes) {
        std::snprintf(g_last_error, sizeof(g_last_error),
                      "these sizes need %zu bytes of scratch; the static scratch holds %zu",
                      need, kStaticScratchBytes);
        return SANA_LA_ERR_WORKSPACE;
    }
    void* scratch = nullptr;
    if ((st = static_scratch_address(&scratch)) != SANA_LA_OK) return st;
    return sana_linattn_forward(Q, K, V, B, N, H, d, O, out_dtype, eps, scratch,
                                kStaticScratchBytes, stream);
}
