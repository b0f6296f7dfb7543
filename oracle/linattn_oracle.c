/*
 * fp64 CPU oracle for multi-head ReLU linear self-attention (forward).
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the bench's CPU
 * baseline leg load this file's library. It shares no code, header, table or
 * helper with the CUDA library and never runs on the product path.
 *
 * What it computes, and where the pages define it:
 *
 *  - Feature map phi = ReLU, phi(x) = max(x, 0).
 *      "08_sana高效高分辨率生成" (papers-3lj.pages.dev), section
 *      "Linear Attention 的原理": phi = ReLU; KV = phi(K)^T V is d x d and does
 *      not depend on n; A = phi(Q) KV.
 *  - Normalised form  phi(Q)(phi(K)^T V) / (phi(Q) phi(K)^T 1).
 *      "linear-diffusion-transformer-4k-efficient-generation"
 *      (blog.hotdry.top), section "核心架构：Linear Attention 与 DC-AE 的协同设计".
 *  - The two shared terms sum_n phi(K_n)^T V_n and sum_n phi(K_n)^T are formed
 *    once and reused by every query (O(N) work).
 *      "SANA: Efficient High-Resolution Image Synthesis with Linear Diffusion
 *      Transformers" (phd-frog.tistory.com/40), section 2.2, "선형 어텐션 블럭"
 *      (the prose around Eq. 1; the equation itself is lost from the page).
 *  - Both shared terms as one d x (d+1) product phi(K)^T [V | 1]: the "padding"
 *    that the same walk-through's section "Triton을 통한 학습/추론 가속화" lists
 *    among the element-wise steps fused into the matmul, read here as a ones
 *    column appended to V.
 *
 * Readings where the pages are silent (each one is also listed in the design
 * notes): eps is added to the normaliser only, O = num / (den + eps); heads are
 * independent with head size d; no 1/sqrt(d) or 1/N scale; a row whose
 * normaliser is 0 gives 0 / eps = 0.
 *
 * Layout (the same one the library documents): Q, K, V, O are (B, N, H, d)
 * row-major, element (b, n, h, i) at ((b*N + n)*H + h)*d + i. The state S is
 * (B, H, d, d+1) row-major, entry (b, h, i, j) at ((b*H + h)*d + i)*(d+1) + j,
 * with column j = d holding the normaliser sum_n phi(K_{n,i}).
 *
 * Block-causal form ("linear-diffusion-transformer-4k-efficient-generation",
 * section "技术演进：从图像到视频与世界模型": SANA-Video turns the linear
 * attention into block causal linear attention; the pages give no formula).
 * Reading: the tokens form blocks of L consecutive tokens (block j holds tokens
 * j*L .. min((j+1)*L, N) - 1, e.g. one latent video frame per block; the
 * video row of the token table in "08_sana高效高分辨率生成", section
 * "Linear Attention 的原理", has 16 frames of 65,536 tokens); a query of
 * block j attends to every key of blocks 0 .. j, so it uses the prefix state
 *   P[b,h,j] = sum over tokens n < min((j+1)*L, N) of phi(K_n)^T [V_n | 1]
 * in place of S. The prefix states are (B, H, nblk, d, d+1), nblk = ceil(N/L).
 *
 * Other feature maps ("08_sana高效高分辨率生成", section "Linear Attention 的原理"
 * names ELU+1 and cos as alternatives to ReLU). Reading: ELU with alpha = 1,
 * plus one, i.e. phi(x) = x + 1 for x > 0 and exp(x) otherwise; cos is
 * phi(x) = cos(x) elementwise. Everything else (state, normaliser, eps) is the
 * same; with cos the normaliser can be zero or negative and O = num/(den+eps)
 * is taken as it stands.
 *
 * All arithmetic is IEEE double. Sums run in token order n = 0 .. N-1 and
 * feature order i = 0 .. d-1, nothing is blocked or reordered. OpenMP only
 * spreads independent (b, h) pairs or independent query rows over threads, which
 * does not change any sum.
 */
#include <stddef.h>
#include <math.h>
#include <stdlib.h>
#include <omp.h>

static double relu(double x) { return x > 0.0 ? x : 0.0; }

/* offset of element (b, n, h, i) in a (B, N, H, d) row-major tensor */
static size_t at_bnhd(long b, long n, long h, long i, long N, long H, long d)
{
    return (((size_t)b * N + n) * H + h) * d + i;
}

/* offset of entry (b, h, i, j) in a (B, H, d, d+1) row-major state */
static size_t at_state(long b, long h, long i, long j, long H, long d)
{
    return (((size_t)b * H + h) * d + i) * (d + 1) + j;
}

int oracle_num_threads(void) { return omp_get_max_threads(); }

/*
 * S[b,h] = sum over n of phi(K[b,n,h,:])^T [V[b,n,h,:] | 1].
 * S[b,h,i,j] = sum_n relu(K[b,n,h,i]) * V[b,n,h,j]   for j < d
 * S[b,h,i,d] = sum_n relu(K[b,n,h,i]) * 1
 */
void oracle_state(const double* K, const double* V, long B, long N, long H, long d,
                  double* S)
{
    #pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (long b = 0; b < B; ++b) {
        for (long h = 0; h < H; ++h) {
            for (long i = 0; i < d; ++i)
                for (long j = 0; j <= d; ++j)
                    S[at_state(b, h, i, j, H, d)] = 0.0;
            for (long n = 0; n < N; ++n) {
                for (long i = 0; i < d; ++i) {
                    double k = relu(K[at_bnhd(b, n, h, i, N, H, d)]);
                    for (long j = 0; j < d; ++j)
                        S[at_state(b, h, i, j, H, d)] += k * V[at_bnhd(b, n, h, j, N, H, d)];
                    S[at_state(b, h, i, d, H, d)] += k * 1.0;
                }
            }
        }
    }
}

/*
 * For each query row (b, n, h):
 *   num_j = sum_i relu(Q[b,n,h,i]) * S[b,h,i,j]   (j < d)
 *   den   = sum_i relu(Q[b,n,h,i]) * S[b,h,i,d]
 *   O[b,n,h,j] = num_j / (den + eps)
 * If den_out is not NULL it receives den for every (b, n, h).
 */
void oracle_apply(const double* Q, const double* S, long B, long N, long H, long d,
                  double eps, double* O, double* den_out)
{
    #pragma omp parallel for collapse(2) schedule(static)
    for (long b = 0; b < B; ++b) {
        for (long n = 0; n < N; ++n) {
            for (long h = 0; h < H; ++h) {
                double den = 0.0;
                for (long i = 0; i < d; ++i)
                    den += relu(Q[at_bnhd(b, n, h, i, N, H, d)]) * S[at_state(b, h, i, d, H, d)];
                for (long j = 0; j < d; ++j) {
                    double num = 0.0;
                    for (long i = 0; i < d; ++i)
                        num += relu(Q[at_bnhd(b, n, h, i, N, H, d)]) * S[at_state(b, h, i, j, H, d)];
                    O[at_bnhd(b, n, h, j, N, H, d)] = num / (den + eps);
                }
                if (den_out)
                    den_out[((size_t)b * N + n) * H + h] = den;
            }
        }
    }
}

/* forward = state, then apply (the scratch state is caller-provided) */
void oracle_forward(const double* Q, const double* K, const double* V,
                    long B, long N, long H, long d, double eps,
                    double* S, double* O)
{
    oracle_state(K, V, B, N, H, d, S);
    oracle_apply(Q, S, B, N, H, d, eps, O, NULL);
}

/* offset of entry (b, h, j, i, c) in (B, H, nblk, d, d+1) prefix states */
static size_t at_prefix(long b, long h, long j, long i, long c, long H, long nblk, long d)
{
    return ((((size_t)b * H + h) * nblk + j) * d + i) * (d + 1) + c;
}

/*
 * Block-causal prefix states: for every (b, h) a running sum over tokens in
 * order; after the last token of block j the running sum is P[b,h,j].
 */
void oracle_block_causal_state(const double* K, const double* V, long B, long N, long H, long d,
                               long L, double* P)
{
    const long nblk = (N + L - 1) / L;
    #pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (long b = 0; b < B; ++b) {
        for (long h = 0; h < H; ++h) {
            double* run = (double*)malloc(sizeof(double) * (size_t)d * (d + 1));
            for (long e = 0; e < d * (d + 1); ++e)
                run[e] = 0.0;
            for (long j = 0; j < nblk; ++j) {
                const long end = (j + 1) * L < N ? (j + 1) * L : N;
                for (long n = j * L; n < end; ++n) {
                    for (long i = 0; i < d; ++i) {
                        double k = relu(K[at_bnhd(b, n, h, i, N, H, d)]);
                        for (long c = 0; c < d; ++c)
                            run[i * (d + 1) + c] += k * V[at_bnhd(b, n, h, c, N, H, d)];
                        run[i * (d + 1) + d] += k * 1.0;
                    }
                }
                for (long i = 0; i < d; ++i)
                    for (long c = 0; c <= d; ++c)
                        P[at_prefix(b, h, j, i, c, H, nblk, d)] = run[i * (d + 1) + c];
            }
            free(run);
        }
    }
}

/*
 * Block-causal apply: query row (b, n, h) of block j = n / L uses P[b,h,j]:
 *   O[b,n,h,c] = (sum_i relu(Q_i) P[b,h,j,i,c]) / (sum_i relu(Q_i) P[b,h,j,i,d] + eps)
 */
void oracle_block_causal_apply(const double* Q, const double* P, long B, long N, long H, long d,
                               long L, double eps, double* O)
{
    const long nblk = (N + L - 1) / L;
    #pragma omp parallel for collapse(2) schedule(static)
    for (long b = 0; b < B; ++b) {
        for (long n = 0; n < N; ++n) {
            const long j = n / L;
            for (long h = 0; h < H; ++h) {
                double den = 0.0;
                for (long i = 0; i < d; ++i)
                    den += relu(Q[at_bnhd(b, n, h, i, N, H, d)]) * P[at_prefix(b, h, j, i, d, H, nblk, d)];
                for (long c = 0; c < d; ++c) {
                    double num = 0.0;
                    for (long i = 0; i < d; ++i)
                        num += relu(Q[at_bnhd(b, n, h, i, N, H, d)]) * P[at_prefix(b, h, j, i, c, H, nblk, d)];
                    O[at_bnhd(b, n, h, c, N, H, d)] = num / (den + eps);
                }
            }
        }
    }
}

/* feature map: 0 = ReLU, 1 = ELU + 1, 2 = cos */
static double feature(double x, int fm)
{
    if (fm == 1)
        return x > 0.0 ? x + 1.0 : exp(x);
    if (fm == 2)
        return cos(x);
    return x > 0.0 ? x : 0.0;
}

/* the state with feature map fm: S[b,h,i,j] = sum_n phi(K[b,n,h,i]) * [V | 1][b,n,h,j] */
void oracle_state_fm(const double* K, const double* V, long B, long N, long H, long d, int fm,
                     double* S)
{
    #pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (long b = 0; b < B; ++b) {
        for (long h = 0; h < H; ++h) {
            for (long i = 0; i < d; ++i)
                for (long j = 0; j <= d; ++j)
                    S[at_state(b, h, i, j, H, d)] = 0.0;
            for (long n = 0; n < N; ++n) {
                for (long i = 0; i < d; ++i) {
                    double k = feature(K[at_bnhd(b, n, h, i, N, H, d)], fm);
                    for (long j = 0; j < d; ++j)
                        S[at_state(b, h, i, j, H, d)] += k * V[at_bnhd(b, n, h, j, N, H, d)];
                    S[at_state(b, h, i, d, H, d)] += k * 1.0;
                }
            }
        }
    }
}

/* apply with feature map fm: O = (phi(Q) S[:, 0:d]) / (phi(Q) S[:, d] + eps) */
void oracle_apply_fm(const double* Q, const double* S, long B, long N, long H, long d, int fm,
                     double eps, double* O, double* den_out)
{
    #pragma omp parallel for collapse(2) schedule(static)
    for (long b = 0; b < B; ++b) {
        for (long n = 0; n < N; ++n) {
            for (long h = 0; h < H; ++h) {
                double den = 0.0;
                for (long i = 0; i < d; ++i)
                    den += feature(Q[at_bnhd(b, n, h, i, N, H, d)], fm) * S[at_state(b, h, i, d, H, d)];
                for (long j = 0; j < d; ++j) {
                    double num = 0.0;
                    for (long i = 0; i < d; ++i)
                        num += feature(Q[at_bnhd(b, n, h, i, N, H, d)], fm) * S[at_state(b, h, i, j, H, d)];
                    O[at_bnhd(b, n, h, j, N, H, d)] = num / (den + eps);
                }
                if (den_out)
                    den_out[((size_t)b * N + n) * H + h] = den;
            }
        }
    }
}
