/*
 * sana_linattn.h - C ABI of the B200 (sm_100a) multi-head ReLU linear
 * self-attention forward used by Sana's Linear DiT.
 *
 * The operation, per batch b and head h, with phi = ReLU:
 *
 *     S     = phi(K)^T [V | 1]                       d x (d+1), fp32
 *     O_n   = (phi(Q_n) S[:, 0:d]) / (phi(Q_n) S[:, d] + eps)
 *
 * Sources (page title, section):
 *   - "08_sana高效高分辨率生成" (papers-3lj.pages.dev), "Linear Attention 的原理":
 *     phi = ReLU, KV = phi(K)^T V is d x d whatever the token count, and
 *     A = phi(Q) KV.
 *   - "linear-diffusion-transformer-4k-efficient-generation" (blog.hotdry.top),
 *     "核心架构：Linear Attention 与 DC-AE 的协同设计": the normalised form
 *     phi(Q)(phi(K)^T V) / (phi(Q) phi(K)^T 1).
 *   - "SANA: Efficient High-Resolution Image Synthesis with Linear Diffusion
 *     Transformers" (phd-frog.tistory.com/40), section 2.2 "선형 어텐션 블럭":
 *     the two shared terms (phi(K)^T V and phi(K)^T 1) are computed once and
 *     reused by every query; section "Triton을 통한 학습/추론 가속화": the
 *     activation, precision conversion, padding and division are fused into the
 *     matrix products (here: the ones column of [V | 1] is that padding, and the
 *     division happens in the apply kernel's epilogue).
 *   eps is added to the normaliser only; the pages write the formula without it.
 *
 * Layout
 *   Q, K, V, O : (B, N, H, d) row-major. Element (b, n, h, i) is at
 *                ((b*N + n)*H + h)*d + i. Q, K, V are bfloat16.
 *                O is float32 or bfloat16 (round to nearest even).
 *   state      : (B, H, d, d+1) row-major float32. Entry (b, h, i, j) is at
 *                ((b*H + h)*d + i)*(d+1) + j. Column j = d is the normaliser
 *                sum_n phi(K[b,n,h,i]).
 *
 * Ownership and execution
 *   Every pointer is a DEVICE pointer owned by the caller; the library never
 *   allocates, frees or synchronises. All work is enqueued on `stream`
 *   (NULL = the legacy default stream) and the calls return as soon as it is
 *   enqueued. Inputs must not alias outputs. The result is deterministic: the
 *   same inputs and sizes give bit-identical outputs on every run (on devices
 *   with the same number of SMs: the work is split into one persistent CTA
 *   per SM), and sana_linattn_forward gives exactly the bits of
 *   sana_linattn_kv_state followed by sana_linattn_apply.
 *
 * Errors
 *   Arguments are checked on the host before anything is launched; on any
 *   error nothing is enqueued and the status says why:
 *     SANA_LA_ERR_INVALID_ARG  null pointer, B, N or H < 1, a pointer not 16-byte
 *                              aligned, eps negative or not finite, an unknown
 *                              output dtype, or sizes whose element count
 *                              overflows 63 bits;
 *     SANA_LA_ERR_UNSUPPORTED  d not 32 or 64 (the calls below state their
 *                              other limits);
 *     SANA_LA_ERR_WORKSPACE    workspace smaller than sana_linattn_workspace_bytes;
 *     SANA_LA_ERR_CUDA         a CUDA call or launch failed (details from
 *                              sana_linattn_last_error()).
 *   Faults inside a kernel surface at the caller's next synchronisation, as
 *   with any CUDA library. NaN or Inf inputs are outside the contract.
 *   The functions are thread-safe; sana_linattn_last_error is per thread.
 */
#ifndef SANA_LINATTN_H
#define SANA_LINATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The same handle type as cudaStream_t, declared here without CUDA headers. */
typedef struct CUstream_st* sana_la_stream_t;

typedef enum {
    SANA_LA_OK = 0,
    SANA_LA_ERR_INVALID_ARG = 1,
    SANA_LA_ERR_UNSUPPORTED = 2,
    SANA_LA_ERR_WORKSPACE = 3,
    SANA_LA_ERR_CUDA = 4
} sana_la_status;

typedef enum {
    SANA_LA_OUT_F32 = 0,
    SANA_LA_OUT_BF16 = 1
} sana_la_out_dtype;

/* Feature map phi ("08_sana高效高分辨率生成", "Linear Attention 的原理": ReLU, with
 * ELU+1 and cos named as alternatives). ELU is taken with alpha = 1:
 * phi(x) = x + 1 for x > 0, exp(x) otherwise. */
typedef enum {
    SANA_LA_FEATURE_RELU = 0,
    SANA_LA_FEATURE_ELU1 = 1,
    SANA_LA_FEATURE_COS = 2
} sana_la_feature_map;

/*
 * Bytes of device workspace that sana_linattn_kv_state and
 * sana_linattn_forward need for these sizes on the current device (a function
 * of the sizes and of the device's SM count; with no device to ask, the
 * B200's 148). The workspace holds the fp32 partial states of the token
 * chunks, and for sana_linattn_forward also the reduced state and one
 * readiness flag per CTA. Returns 0 for invalid or unsupported sizes. Any
 * content is acceptable on entry; it is scratch.
 */
size_t sana_linattn_workspace_bytes(int B, int N, int H, int d);

/*
 * The shared terms: state = phi(K)^T [V | 1] for every (b, h)
 * ("08_sana高效高分辨率生成", "Linear Attention 的原理"; the Sana walk-through,
 * section 2.2, Eq. 1 prose; the ones column is the "padding" of its Triton
 * section).
 *   K, V      bf16 (B, N, H, d), device.
 *   state     fp32 (B, H, d, d+1), device, written in full.
 *   workspace device scratch of at least sana_linattn_workspace_bytes(B,N,H,d).
 * The token range is split into fixed chunks whose partial states are summed in
 * ascending chunk order, so the result does not depend on scheduling.
 */
sana_la_status sana_linattn_kv_state(const void* K, const void* V,
                                     int B, int N, int H, int d,
                                     float* state,
                                     void* workspace, size_t workspace_bytes,
                                     sana_la_stream_t stream);

/*
 * The per-query product and normalisation:
 *   O[b,n,h,:] = (phi(Q[b,n,h,:]) state[b,h,:,0:d]) / (phi(Q[b,n,h,:]) state[b,h,:,d] + eps)
 * ("linear-diffusion-transformer-4k-efficient-generation", normalised form;
 * "08_sana高效高分辨率生成", A = phi(Q) KV).
 *   Q         bf16 (B, N, H, d), device.
 *   state     fp32 (B, H, d, d+1), device (e.g. from sana_linattn_kv_state).
 *   O         (B, N, H, d) device, fp32 or bf16 per out_dtype, written in full.
 *   eps       finite, >= 0; a row with phi(Q) = 0 gives exactly 0.
 */
sana_la_status sana_linattn_apply(const void* Q, const float* state,
                                  int B, int N, int H, int d,
                                  void* O, sana_la_out_dtype out_dtype, float eps,
                                  sana_la_stream_t stream);

/*
 * The whole forward: sana_linattn_kv_state into the workspace, then
 * sana_linattn_apply. Same arguments and rules as the two calls above; the
 * result is bit-identical to calling them in sequence.
 * It runs as one cooperative kernel launch: the state phase; a readiness flag
 * per CTA; the apply phase, in which each CTA waits for the flags of the CTAs
 * that made its (b, head group)'s partial states and sums them itself, in the
 * order sana_linattn_kv_state sums them. The flags are tagged with a number
 * unique to the call, so the workspace needs no initialisation. Under stream
 * capture the call also records a memset of those flags before the kernel,
 * because a replayed graph reuses the captured number. Where the device cannot
 * hold the whole grid at once, the call falls back to the kernels of the two
 * calls above.
 */
sana_la_status sana_linattn_forward(const void* Q, const void* K, const void* V,
                                    int B, int N, int H, int d,
                                    void* O, sana_la_out_dtype out_dtype, float eps,
                                    void* workspace, size_t workspace_bytes,
                                    sana_la_stream_t stream);

/*
 * The three calls above with another feature map phi. SANA_LA_FEATURE_RELU
 * gives exactly the calls above. For ELU+1 and cos, phi is evaluated in fp32
 * from the bf16 inputs (the hardware exponential; for cos a Cody-Waite
 * reduction to [-pi, pi] and the hardware cosine) and carried into the
 * tensor-core products as a bf16 hi + lo pair (~2^-17 relative), so the
 * output meets the ReLU path's tolerance; the state kernel runs with 4 instead of 6 pipeline stages and the
 * apply kernel issues one more product per head. With cos the normaliser
 * phi(Q) state[:, d] can be zero or negative; O = num / (den + eps) is returned
 * as it stands. A feature_map outside the enum is SANA_LA_ERR_INVALID_ARG. The
 * workspace size is sana_linattn_workspace_bytes; states from
 * sana_linattn_kv_state_fm must be applied with the same feature map.
 */
sana_la_status sana_linattn_kv_state_fm(const void* K, const void* V,
                                        int B, int N, int H, int d, sana_la_feature_map feature_map,
                                        float* state,
                                        void* workspace, size_t workspace_bytes,
                                        sana_la_stream_t stream);

sana_la_status sana_linattn_apply_fm(const void* Q, const float* state,
                                     int B, int N, int H, int d, sana_la_feature_map feature_map,
                                     void* O, sana_la_out_dtype out_dtype, float eps,
                                     sana_la_stream_t stream);

sana_la_status sana_linattn_forward_fm(const void* Q, const void* K, const void* V,
                                       int B, int N, int H, int d, sana_la_feature_map feature_map,
                                       void* O, sana_la_out_dtype out_dtype, float eps,
                                       void* workspace, size_t workspace_bytes,
                                       sana_la_stream_t stream);

/*
 * The state built inside the key-value projection ("SANA: Efficient
 * High-Resolution Image Synthesis with Linear Diffusion Transformers", section 4
 * "On-Device Deployment": the ReLU(K)^T V product is fused into the QKV
 * projection, which stays in full precision):
 *   K = X Wk^T, V = X Wv^T   (bf16 inputs, fp32 accumulation on the tensor cores,
 *                            then rounded to bf16 as a stored K and V would be)
 *   state = phi(K)^T [V | 1] per (b, h), as sana_linattn_kv_state would give
 *                            for those K and V (up to the summation order)
 * K and V are never written to memory. No bias. phi = ReLU.
 *   X         bf16 (B, N, C) row-major (token-major activations), device.
 *   Wk, Wv    bf16 (H*d, C) row-major (the layout of a linear layer's weight:
 *             output feature h*d + i is row h*d + i), device.
 *   state     fp32 (B, H, d, d+1), device, written in full.
 *   workspace at least sana_linattn_kv_projection_workspace_bytes(...) bytes.
 * C must be a multiple of 8 (SANA_LA_ERR_UNSUPPORTED otherwise). The queries
 * are a plain projection (Q = X Wq^T, any GEMM); sana_linattn_apply then gives O.
 */
size_t sana_linattn_kv_projection_workspace_bytes(int B, int N, int C, int H, int d);

sana_la_status sana_linattn_kv_projection_state(const void* X, const void* Wk, const void* Wv,
                                                int B, int N, int C, int H, int d,
                                                float* state,
                                                void* workspace, size_t workspace_bytes,
                                                sana_la_stream_t stream);

/* Kernel launches one sana_linattn_kv_projection_state call enqueues (0 if invalid). */
int sana_linattn_kv_projection_state_launches(int B, int N, int C, int H, int d);

/*
 * Mix-FFN, the step after the attention in a Sana block ("SANA: Efficient
 * High-Resolution Image Synthesis with Linear Diffusion Transformers", section
 * 2.2 "선형 어텐션 블럭": an inverted residual block with a 3x3 depthwise
 * convolution and a GLU; section 4: the GLU fused into the Mix-FFN kernel):
 *   U = X W1^T                      1x1 expand to 2*Ch channels (bf16 out)
 *   D = depthwise3x3(U)             per channel over the Hg x Wg token grid
 *                                   (token n = y*Wg + x), zero padding
 *   Z = D[:, :Ch] * sigmoid(D[:, Ch:])   GLU, fused with the convolution (bf16 out)
 *   Y = Z W2^T                      1x1 project back to C channels (bf16 out)
 * No biases, no other activation, no residual inside the block.
 *   X    bf16 (B, Hg*Wg, C) row-major, device.
 *   W1   bf16 (2*Ch, C) row-major (a linear layer's weight), device.
 *   Kdw  fp32 (2*Ch, 3, 3): tap (dy, dx) of channel c at c*9 + dy*3 + dx, device.
 *   W2   bf16 (C, Ch) row-major, device.
 *   Y    bf16 (B, Hg*Wg, C), device, written in full.
 *   workspace at least sana_linattn_mix_ffn_workspace_bytes(...) bytes; after
 *        the call it holds U (B*Hg*Wg x 2*Ch bf16) at offset 0 and Z (B*Hg*Wg x
 *        Ch bf16) at the next 256-byte boundary.
 * C and Ch must be multiples of 8 (SANA_LA_ERR_UNSUPPORTED otherwise). Three
 * launches: tcgen05 GEMM, fused depthwise + GLU, tcgen05 GEMM.
 */
size_t sana_linattn_mix_ffn_workspace_bytes(int B, int Hg, int Wg, int C, int Ch);

sana_la_status sana_linattn_mix_ffn(const void* X, const void* W1, const float* Kdw, const void* W2,
                                    int B, int Hg, int Wg, int C, int Ch, void* Y,
                                    void* workspace, size_t workspace_bytes, sana_la_stream_t stream);

/* Kernel launches one sana_linattn_mix_ffn call enqueues (0 if invalid). */
int sana_linattn_mix_ffn_launches(int B, int Hg, int Wg, int C, int Ch);

/*
 * Block-causal form ("linear-diffusion-transformer-4k-efficient-generation",
 * section "技术演进：从图像到视频与世界模型": SANA-Video's block causal linear
 * attention; the pages give no formula). The tokens form blocks of L
 * consecutive tokens (block j = tokens j*L .. min((j+1)*L, N) - 1, e.g. one
 * latent video frame each); a query of block j attends to the keys of blocks
 * 0 .. j, i.e. it uses the inclusive prefix state
 *   P[b,h,j] = sum over tokens n < min((j+1)*L, N) of phi(K_n)^T [V_n | 1]
 * in place of the state of sana_linattn_apply. nblk = ceil(N / L).
 *
 * L must be a positive multiple of 128 (SANA_LA_ERR_UNSUPPORTED otherwise; 0
 * or negative is SANA_LA_ERR_INVALID_ARG); sizes whose per-block partial states
 * would exceed 4 GiB of workspace are SANA_LA_ERR_UNSUPPORTED. N need not be a
 * multiple of L. Work is spread over ceil(B*H/(128/d)) slabs times R = rb*rt
 * CTAs (at most 148 in all): the CTAs of a slab split its blocks rb ways and
 * each block's 128-token tiles rt ways (rt divides L/128), chosen on the host
 * from the tiles of the busiest CTA and the states it stages. Few blocks with
 * an L/128 of few divisors (e.g. one block of L = 128) still run on few SMs.
 * Other arguments, layouts and errors are as for the calls above.
 */

/* Workspace bytes of the block-causal calls (0 for invalid or unsupported sizes). */
size_t sana_linattn_block_causal_workspace_bytes(int B, int N, int H, int d, int L);

/*
 * Prefix states: `states` fp32 (B, H, nblk, d, d+1), device, written in full;
 * entry (b, h, j, i, c) at (((b*H + h)*nblk + j)*d + i)*(d+1) + c. The blocks'
 * partial sums are added in ascending block order (and within a block in a
 * fixed order), so the result does not depend on scheduling.
 */
sana_la_status sana_linattn_block_causal_kv_state(const void* K, const void* V,
                                                  int B, int N, int H, int d, int L,
                                                  float* states,
                                                  void* workspace, size_t workspace_bytes,
                                                  sana_la_stream_t stream);

/* O from the prefix states: query row (b, n, h) uses states[b, h, n / L]. */
sana_la_status sana_linattn_block_causal_apply(const void* Q, const float* states,
                                               int B, int N, int H, int d, int L,
                                               void* O, sana_la_out_dtype out_dtype, float eps,
                                               sana_la_stream_t stream);

/*
 * The whole block-causal forward (three launches: state kernel, prefix
 * reduction, apply kernel); bit-identical to sana_linattn_block_causal_kv_state
 * followed by sana_linattn_block_causal_apply.
 */
sana_la_status sana_linattn_block_causal_forward(const void* Q, const void* K, const void* V,
                                                 int B, int N, int H, int d, int L,
                                                 void* O, sana_la_out_dtype out_dtype, float eps,
                                                 void* workspace, size_t workspace_bytes,
                                                 sana_la_stream_t stream);

/* Kernel launches one sana_linattn_block_causal_forward call enqueues (0 if invalid). */
int sana_linattn_block_causal_forward_launches(int B, int N, int H, int d, int L);

/*
 * The same forward in one cooperative launch: the state phase writes the
 * per-block partial states; each CTA of the apply phase, once the CTAs of its
 * slab have raised their readiness flags, adds the partials of every block up
 * to the one it applies onto a running prefix (kept between its segments in
 * the workspace), with the prefix reduction's additions in its order. Same
 * arguments, workspace and errors as sana_linattn_block_causal_forward, and
 * bit-identical to it. If the device cannot hold the whole grid at once, the
 * three kernels run instead. (Measured on B200 it is not faster: 143 against
 * 133 us for 16 frames of 4,096 tokens, 1.79 against 1.67 ms for 16 frames of
 * 65,536, 36 heads of 32: each CTA adds every earlier block's (shared) block
 * sum itself, where the prefix reduction forms each prefix once.)
 */
sana_la_status sana_linattn_block_causal_forward_single(const void* Q, const void* K, const void* V,
                                                        int B, int N, int H, int d, int L,
                                                        void* O, sana_la_out_dtype out_dtype, float eps,
                                                        void* workspace, size_t workspace_bytes,
                                                        sana_la_stream_t stream);

/* Kernel launches one sana_linattn_block_causal_forward_single call enqueues (0 if invalid). */
int sana_linattn_block_causal_forward_single_launches(int B, int N, int H, int d, int L);

/*
 * sana_linattn_block_causal_forward from and to HOST memory, with the copies
 * overlapped by the library as in sana_linattn_forward_host (below): K and V
 * are copied in and the prefix states computed over all blocks; then Q is
 * streamed in chunks of whole blocks of one batch (about a sixteenth of the
 * tokens, at least one block), each chunk applied against its blocks' prefix
 * states as soon as it is in, its O copied out on the library's
 * device-to-host stream while later chunks come in.
 *   Q, K, V   host, (B, N, H, d) bf16 row-major
 *   O         host, (B, N, H, d) fp32 or bf16 by out_dtype
 *   workspace device, sana_linattn_block_causal_forward_host_workspace_bytes
 *             (B, N, H, d, L, out_dtype) bytes, 16-byte aligned: device
 *             copies of Q, K, V and O, the prefix states and the partials
 * O is bit-identical to sana_linattn_block_causal_forward's on the same
 * inputs (the apply of a token depends only on its block's prefix state).
 * Page-locked host buffers make the copies asynchronous; ownership, streams
 * and errors as for sana_linattn_forward_host; L as for the block-causal
 * calls above (L < 1: SANA_LA_ERR_INVALID_ARG; not a multiple of 128:
 * SANA_LA_ERR_UNSUPPORTED).
 */
size_t sana_linattn_block_causal_forward_host_workspace_bytes(int B, int N, int H, int d, int L,
                                                              sana_la_out_dtype out_dtype);

sana_la_status sana_linattn_block_causal_forward_host(const void* Q, const void* K, const void* V,
                                                      int B, int N, int H, int d, int L,
                                                      void* O, sana_la_out_dtype out_dtype, float eps,
                                                      void* workspace, size_t workspace_bytes,
                                                      sana_la_stream_t stream);

/* Kernel launches one sana_linattn_block_causal_forward_host call enqueues (0 if invalid). */
int sana_linattn_block_causal_forward_host_launches(int B, int N, int H, int d, int L);

/*
 * sana_linattn_forward without a workspace argument, for callers that cannot
 * allocate device memory: code that runs under an allocator it does not own
 * (a host application or framework that hands out all device memory itself),
 * serving loops that must not allocate once started, and callers bound to an
 * interface that passes only inputs and outputs (no scratch buffer).
 * The paper has no counterpart to this call; it exists for those callers.
 *
 * The scratch sits in a fixed 16 MiB device array inside this library, which
 * every GPU that loads the library keeps until the process exits. Sizes whose
 * sana_linattn_workspace_bytes exceeds 16 MiB are rejected with
 * SANA_LA_ERR_WORKSPACE (sana_linattn_last_error says how much they need); the
 * 4096px shape (B=2, N=16384, H=70, d=32) fits. The call allocates nothing.
 *
 * Its first call on a device looks up the array's device address (with the
 * calling thread's current device, which must be the device of Q, K, V, O and
 * `stream`); make that first call before any stream capture. All calls on a
 * device share the array: calls whose work can overlap on the GPU (e.g. on
 * unordered streams) race and give wrong results; order them on one stream.
 * The array needs no clearing between calls. Results are bit-identical to
 * sana_linattn_forward with a caller workspace. Arguments and other errors are
 * as for sana_linattn_forward.
 */
sana_la_status sana_linattn_forward_noalloc(const void* Q, const void* K, const void* V,
                                            int B, int N, int H, int d,
                                            void* O, sana_la_out_dtype out_dtype, float eps,
                                            sana_la_stream_t stream);

/*
 * The forward of sana_linattn_forward_fm from and to HOST memory ("08_sana
 * 高效高分辨率生成", "Linear Attention 的原理": the state sum over all tokens,
 * then each token's row against it).
 *   Q, K, V   host, (B, N, H, d) bf16 row-major (as for sana_linattn_forward)
 *   O         host, (B, N, H, d) fp32 or bf16 by out_dtype
 *   workspace device, sana_linattn_forward_host_workspace_bytes(B, N, H, d,
 *             out_dtype) bytes, 16-byte aligned; holds device copies of Q, K,
 *             V and O, the state and the state kernels' partials
 * K and V are copied in and the state is computed over all tokens; then Q is
 * streamed in chunks of about a sixteenth of the tokens (at least 1024 tokens,
 * whole batches when a batch is shorter). The copies in run back to back on a
 * host-to-device stream of this library's, each chunk is applied on `stream`
 * as soon as it is in, and its O is copied out on a device-to-host stream of
 * this library's while later chunks are copied in, so the two copy directions
 * overlap (both streams and a few events per device are made on first use;
 * the copies in wait for the work enqueued on `stream` before this call). `stream` waits for the last copy out before anything
 * enqueued after this call: once `stream` is done, O is in host memory. O is
 * bit-identical to sana_linattn_forward_fm's on the same inputs (the apply of
 * a token does not depend on the chunk it is in). For the copies to be
 * asynchronous and to overlap, the host buffers must be page-locked
 * (cudaHostAlloc, cudaHostRegister); with pageable memory the copies still
 * happen, but CUDA completes them before the copy calls return. Host buffers
 * stay owned by the caller and must stay valid until `stream` has finished.
 * Calls from several host threads on one device are safe; they take turns to
 * enqueue their work and share the two copy streams.
 * Errors as for sana_linattn_forward (null pointers, bad sizes, an unaligned
 * workspace: SANA_LA_ERR_INVALID_ARG; a short workspace:
 * SANA_LA_ERR_WORKSPACE; a failed CUDA call: SANA_LA_ERR_CUDA).
 */
size_t sana_linattn_forward_host_workspace_bytes(int B, int N, int H, int d, sana_la_out_dtype out_dtype);

sana_la_status sana_linattn_forward_host(const void* Q, const void* K, const void* V,
                                         int B, int N, int H, int d, sana_la_feature_map feature_map,
                                         void* O, sana_la_out_dtype out_dtype, float eps,
                                         void* workspace, size_t workspace_bytes,
                                         sana_la_stream_t stream);

/* Kernel launches of one sana_linattn_forward_host call (0 for invalid sizes):
 * the state, its reduction, and one apply per chunk of Q. */
int sana_linattn_forward_host_launches(int B, int N, int H, int d);

/*
 * Number of kernel launches one sana_linattn_forward call enqueues for these
 * sizes (0 for invalid or unsupported sizes): 1 (the single cooperative
 * launch; a captured call adds one memset node). Useful for counting launches
 * in a profile.
 */
int sana_linattn_forward_launches(int B, int N, int H, int d);

/*
 * Static text naming the kernel set compiled into this library and the
 * resource that bounds its dominant kernel, as "impl=<name>;bound=<hbm|alu>".
 */
const char* sana_linattn_build_info(void);

/*
 * Diagnostic: the first error code a kernel of this library recorded on the
 * current device (0 = none; 1 = a pipeline wait inside a kernel ran past its
 * ~2 s limit, after which that kernel stopped early and its outputs are not
 * valid; 2 = a kernel was launched with parameters it does not handle, and did
 * nothing). With clear != 0 the code is reset to 0. This call synchronises with
 * the device; call it after the work it should cover has completed (e.g.
 * after cudaDeviceSynchronize), not in a hot loop.
 */
sana_la_status sana_linattn_device_error(unsigned int* code, int clear);

/*
 * Self-test of the failure detection (no counterpart in the paper): launches
 * one small kernel that waits on an in-kernel barrier nothing ever arrives at,
 * with a limit of `limit_us` microseconds (1 .. 10,000,000). The wait gives up,
 * records error code 1 for sana_linattn_device_error and the kernel returns;
 * the device stays usable. Returns SANA_LA_ERR_INVALID_ARG for a limit out of
 * range. Asynchronous on `stream`.
 */
sana_la_status sana_linattn_selftest_wait_timeout(unsigned int limit_us, sana_la_stream_t stream);

/* Static English text for a status code. */
const char* sana_linattn_status_string(sana_la_status status);

/* Text of the last CUDA error seen by a call on this thread ("" if none). */
const char* sana_linattn_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* SANA_LINATTN_H */
