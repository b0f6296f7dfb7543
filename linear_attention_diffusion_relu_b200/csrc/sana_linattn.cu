// C ABI of the ReLU linear-attention forward: argument checks, the split-N
// plan, and kernel launches on the caller's stream. See include/sana_linattn.h
// for the contract.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/sana_linattn.h"
#include "common.cuh"
#include "simt_kernels.cuh"

namespace {

thread_local char g_last_error[256] = "";

void set_last_error(const char* where, cudaError_t e) {
    std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", where,
                  cudaGetErrorName(e), cudaGetErrorString(e));
}

constexpr int kSMs = 148;             // B200
constexpr int kTargetUnits = 4 * kSMs;
constexpr int kMinChunk = 256;        // fewest tokens a chunk may hold
constexpr int kChunkAlign = 64;
constexpr long long kMaxElems = 1LL << 62;

inline long long cdiv(long long a, long long b) { return (a + b - 1) / b; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Split of the token range into C chunks of `chunk` tokens (the last may be
// short). A pure function of the sizes, so workspace size and reduction order
// never depend on the device or on timing.
struct Plan {
    int C;
    int chunk;
    size_t partial_bytes;   // fp32 (B, H, C, d, d+1)
    size_t state_bytes;     // fp32 (B, H, d, d+1)
};

Plan make_plan(int B, int N, int H, int d) {
    const int heads_per_group = (d == 32) ? 4 : 2;   // 128 state rows per group
    const long long groups = cdiv(H, heads_per_group);
    const long long per_chunk_units = (long long)B * groups;
    long long C = cdiv(kTargetUnits, per_chunk_units);
    C = std::max(1LL, std::min(C, cdiv(N, kMinChunk)));
    long long chunk = cdiv(cdiv(N, C), kChunkAlign) * kChunkAlign;
    C = cdiv(N, chunk);
    Plan p;
    p.C = (int)C;
    p.chunk = (int)chunk;
    const size_t dd = (size_t)d * (d + 1) * sizeof(float);
    p.partial_bytes = align256((size_t)B * H * C * dd);
    p.state_bytes = align256((size_t)B * H * dd);
    return p;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

sana_la_status check_sizes(int B, int N, int H, int d) {
    if (B < 1 || N < 1 || H < 1) return SANA_LA_ERR_INVALID_ARG;
    if (d != 32 && d != 64) return SANA_LA_ERR_UNSUPPORTED;
    const long long elems = (long long)B * N;
    if (elems > kMaxElems / ((long long)H * d)) return SANA_LA_ERR_INVALID_ARG;
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

constexpr long long kMaxGrid = 0x7fffffffLL;

template <int D>
sana_la_status run_kv_state(const __nv_bfloat16* K, const __nv_bfloat16* V, int B, int N, int H,
                            const Plan& p, float* partial, float* state, cudaStream_t s) {
    const long long units = (long long)B * H * p.C;
    if (units > kMaxGrid) return SANA_LA_ERR_UNSUPPORTED;
    sana::simt::ks_partial<D><<<(unsigned)units, sana::simt::kThreads, 0, s>>>(
        K, V, N, H, p.C, p.chunk, partial);
    sana_la_status st = launch_status("ks_partial");
    if (st != SANA_LA_OK) return st;
    sana::simt::kr_reduce<D><<<(unsigned)((long long)B * H), 256, 0, s>>>(partial, p.C, state);
    return launch_status("kr_reduce");
}

template <int D>
sana_la_status run_apply(const __nv_bfloat16* Q, const float* state, int B, int N, int H,
                         void* O, sana_la_out_dtype od, float eps, cudaStream_t s) {
    const long long tiles = cdiv(N, sana::simt::kApplyTokens);
    const long long units = (long long)B * H * tiles;
    if (units > kMaxGrid) return SANA_LA_ERR_UNSUPPORTED;
    if (od == SANA_LA_OUT_BF16)
        sana::simt::ka_apply<D, true><<<(unsigned)units, sana::simt::kThreads, 0, s>>>(
            Q, state, N, H, (int)tiles, eps, O);
    else
        sana::simt::ka_apply<D, false><<<(unsigned)units, sana::simt::kThreads, 0, s>>>(
            Q, state, N, H, (int)tiles, eps, O);
    return launch_status("ka_apply");
}

sana_la_status kv_state_impl(const void* K, const void* V, int B, int N, int H, int d,
                             float* state, void* ws, size_t ws_bytes, cudaStream_t s,
                             bool need_state_area) {
    const Plan p = make_plan(B, N, H, d);
    const size_t need = p.partial_bytes + (need_state_area ? p.state_bytes : 0);
    if (ws_bytes < need) return SANA_LA_ERR_WORKSPACE;
    float* partial = static_cast<float*>(ws);
    auto k = static_cast<const __nv_bfloat16*>(K);
    auto v = static_cast<const __nv_bfloat16*>(V);
    return d == 32 ? run_kv_state<32>(k, v, B, N, H, p, partial, state, s)
                   : run_kv_state<64>(k, v, B, N, H, p, partial, state, s);
}

sana_la_status apply_impl(const void* Q, const float* state, int B, int N, int H, int d,
                          void* O, sana_la_out_dtype od, float eps, cudaStream_t s) {
    auto q = static_cast<const __nv_bfloat16*>(Q);
    return d == 32 ? run_apply<32>(q, state, B, N, H, O, od, eps, s)
                   : run_apply<64>(q, state, B, N, H, O, od, eps, s);
}

}  // namespace

extern "C" {

size_t sana_linattn_workspace_bytes(int B, int N, int H, int d) {
    if (check_sizes(B, N, H, d) != SANA_LA_OK) return 0;
    const Plan p = make_plan(B, N, H, d);
    return p.partial_bytes + p.state_bytes;
}

sana_la_status sana_linattn_kv_state(const void* K, const void* V, int B, int N, int H, int d,
                                     float* state, void* workspace, size_t workspace_bytes,
                                     sana_la_stream_t stream) {
    g_last_error[0] = '\0';
    if (!K || !V || !state || !workspace) return SANA_LA_ERR_INVALID_ARG;
    sana_la_status st = check_sizes(B, N, H, d);
    if (st != SANA_LA_OK) return st;
    if (!aligned16(K) || !aligned16(V) || !aligned16(state) || !aligned16(workspace))
        return SANA_LA_ERR_INVALID_ARG;
    return kv_state_impl(K, V, B, N, H, d, state, workspace, workspace_bytes,
                         reinterpret_cast<cudaStream_t>(stream), false);
}

sana_la_status sana_linattn_apply(const void* Q, const float* state, int B, int N, int H, int d,
                                  void* O, sana_la_out_dtype out_dtype, float eps,
                                  sana_la_stream_t stream) {
    g_last_error[0] = '\0';
    if (!Q || !state || !O) return SANA_LA_ERR_INVALID_ARG;
    sana_la_status st = check_sizes(B, N, H, d);
    if (st != SANA_LA_OK) return st;
    if (out_dtype != SANA_LA_OUT_F32 && out_dtype != SANA_LA_OUT_BF16) return SANA_LA_ERR_INVALID_ARG;
    if ((st = check_eps(eps)) != SANA_LA_OK) return st;
    if (!aligned16(Q) || !aligned16(state) || !aligned16(O)) return SANA_LA_ERR_INVALID_ARG;
    return apply_impl(Q, state, B, N, H, d, O, out_dtype, eps,
                      reinterpret_cast<cudaStream_t>(stream));
}

sana_la_status sana_linattn_forward(const void* Q, const void* K, const void* V,
                                    int B, int N, int H, int d,
                                    void* O, sana_la_out_dtype out_dtype, float eps,
                                    void* workspace, size_t workspace_bytes,
                                    sana_la_stream_t stream) {
    g_last_error[0] = '\0';
    if (!Q || !K || !V || !O || !workspace) return SANA_LA_ERR_INVALID_ARG;
    sana_la_status st = check_sizes(B, N, H, d);
    if (st != SANA_LA_OK) return st;
    if (out_dtype != SANA_LA_OUT_F32 && out_dtype != SANA_LA_OUT_BF16) return SANA_LA_ERR_INVALID_ARG;
    if ((st = check_eps(eps)) != SANA_LA_OK) return st;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(workspace))
        return SANA_LA_ERR_INVALID_ARG;
    const Plan p = make_plan(B, N, H, d);
    if (workspace_bytes < p.partial_bytes + p.state_bytes) return SANA_LA_ERR_WORKSPACE;
    float* state = reinterpret_cast<float*>(static_cast<char*>(workspace) + p.partial_bytes);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    st = kv_state_impl(K, V, B, N, H, d, state, workspace, workspace_bytes, s, true);
    if (st != SANA_LA_OK) return st;
    return apply_impl(Q, state, B, N, H, d, O, out_dtype, eps, s);
}

int sana_linattn_forward_launches(int B, int N, int H, int d) {
    if (check_sizes(B, N, H, d) != SANA_LA_OK) return 0;
    return 3;   // KS, KR, KA
}

const char* sana_linattn_build_info(void) { return "impl=simt-ffma;bound=alu"; }

const char* sana_linattn_status_string(sana_la_status status) {
    switch (status) {
        case SANA_LA_OK: return "ok";
        case SANA_LA_ERR_INVALID_ARG: return "invalid argument";
        case SANA_LA_ERR_UNSUPPORTED: return "unsupported head size (d must be 32 or 64)";
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

// Device address of g_static_scratch on the current device. The host-side
// name is only a stand-in; the address comes from cudaGetSymbolAddress, asked
// once per device (with that device current) and cached.
sana_la_status static_scratch_address(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        set_last_error("cudaGetDevice", e);
        return SANA_LA_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return SANA_LA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_static_scratch_mutex);
    if (g_static_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess || p == nullptr) {
            set_last_error("cudaGetSymbolAddress(g_static_scratch)", e);
            return SANA_LA_ERR_CUDA;
        }
        g_static_scratch_ptr[dev] = p;
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

extern "C" {

}  // extern "C"
