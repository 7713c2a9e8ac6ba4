/*
 * KDA oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, fp64 CPU statement of what the KDA forward pass computes.
 * Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may
 * load this library.  It shares no code, header, constant or helper with the
 * CUDA path in gated_delta_rule_138_b200/csrc, and the CUDA path never calls
 * it.
 *
 * What it follows.  The worldcybernews article "Kimi K3 Open Model Surpasses
 * Closed GPT and Anthropic Systems on Independent Benchmarks", paragraph 2:
 * a fixed-size state matrix S replaces the KV cache and is updated by the
 * delta rule; beta sets the write strength, alpha the forgetting, and alpha is
 * held between e^-5 and 1 so that BF16 arithmetic neither underflows nor
 * overflows.  The page prints no equation; the reading taken here is the
 * gated delta rule with a per-key-channel alpha, decay first, then the delta
 * write, and the output read from the updated state:
 *
 *     a_t   = clamp(alpha_t, e^-5, 1)                    (d_k values)
 *     S_t   = (I - beta_t k_t k_t^T) Diag(a_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t   = S_t^T q_t
 *
 * S is d_k x d_v.  The same article's paragraph 3 says the kernel computes
 * this chunk-parallel and then "reconstructs correct sequential states"; the
 * oracle is that sequential result, token by token, with no chunking.
 *
 * Parity pins: tests/test_oracle_pins.py (identity, write exactness,
 * closed-form decay, orthonormal-key delta rule, clamp, linearity,
 * stability bound, resume, varlen, hand-worked golden values, and a
 * brute-force product of explicit update matrices).
 *
 * Precision.  Inputs arrive as fp32 arrays holding exactly the values the
 * GPU receives (bf16 inputs are widened to fp32 by the caller, which is
 * exact).  Every operation below is done in fp64.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* e^-5 rounded to the nearest fp32 (0x1.b993fep-8); the clamp is applied to
 * the fp32-widened input, then the value is widened to fp64. */
static const float ORACLE_ALPHA_MIN_F32 = 0x1.b993fep-8f;

double kda_oracle_alpha_min(void) { return (double)ORACLE_ALPHA_MIN_F32; }

/* clamp(x, e^-5, 1) taken on the fp32 value, then widened to fp64 */
static double clamp_alpha(float x) {
    float y = x;
    if (y < ORACLE_ALPHA_MIN_F32) y = ORACLE_ALPHA_MIN_F32;
    if (y > 1.0f) y = 1.0f;
    return (double)y;
}

/*
 * One (sequence, head) and one block of value columns [j0, j1).  The columns
 * of S evolve independently of one another (every step acts on S from the
 * left or adds a rank-1 term whose column j only involves v_t[j]), so
 * splitting them over threads changes no arithmetic.
 *
 * Pointers are already offset to the first token of the sequence and to the
 * head; the token stride (elements) is tok_stride_{k,v,b}.
 */
static void recur_block(const float* q, const float* k, const float* v,
                        const float* alpha, const float* beta,
                        int64_t ntok, int64_t tok_stride_k, int64_t tok_stride_v,
                        int64_t tok_stride_b, int dk, int dv, int j0, int j1,
                        const float* S0 /* [dk,dv] or NULL */,
                        double* out /* token stride tok_stride_v */,
                        double* S_final /* [dk,dv] or NULL */)
{
    const int w = j1 - j0;
    double* S = (double*)malloc(sizeof(double) * (size_t)dk * (size_t)w);
    double* a = (double*)malloc(sizeof(double) * (size_t)dk);
    double* kd = (double*)malloc(sizeof(double) * (size_t)dk);
    double* proj = (double*)malloc(sizeof(double) * (size_t)w);
    for (int c = 0; c < dk; ++c)
        for (int j = 0; j < w; ++j)
            S[(size_t)c * w + j] = S0 ? (double)S0[(size_t)c * dv + j0 + j] : 0.0;

    for (int64_t t = 0; t < ntok; ++t) {
        const float* qt = q + t * tok_stride_k;
        const float* kt = k + t * tok_stride_k;
        const float* at = alpha + t * tok_stride_k;
        const float* vt = v + t * tok_stride_v;
        const double bt = (double)beta[t * tok_stride_b];
        for (int c = 0; c < dk; ++c) { a[c] = clamp_alpha(at[c]); kd[c] = (double)kt[c]; }

        /* S <- Diag(a) S   (row c is key channel c) */
        for (int c = 0; c < dk; ++c)
            for (int j = 0; j < w; ++j) S[(size_t)c * w + j] *= a[c];

        /* S <- (I - beta k k^T) S  =  S - beta k (k^T S) */
        for (int j = 0; j < w; ++j) {
            double s = 0.0;
            for (int c = 0; c < dk; ++c) s += kd[c] * S[(size_t)c * w + j];
            proj[j] = s;
        }
        for (int c = 0; c < dk; ++c)
            for (int j = 0; j < w; ++j) S[(size_t)c * w + j] -= bt * kd[c] * proj[j];

        /* S <- S + beta k v^T */
        for (int c = 0; c < dk; ++c)
            for (int j = 0; j < w; ++j) S[(size_t)c * w + j] += bt * kd[c] * (double)vt[j0 + j];

        /* o_t = S_t^T q_t */
        double* ot = out + t * tok_stride_v;
        for (int j = 0; j < w; ++j) {
            double s = 0.0;
            for (int c = 0; c < dk; ++c) s += S[(size_t)c * w + j] * (double)qt[c];
            ot[j0 + j] = s;
        }
    }
    if (S_final)
        for (int c = 0; c < dk; ++c)
            for (int j = 0; j < w; ++j) S_final[(size_t)c * dv + j0 + j] = S[(size_t)c * w + j];
    free(S); free(a); free(kd); free(proj);
}

/*
 * Forward over a dense batch (cu_seqlens == NULL: B sequences of T tokens) or
 * a packed batch (cu_seqlens != NULL: B == 1, num_seqs sequences, sequence n
 * holding tokens [cu_seqlens[n], cu_seqlens[n+1]) of the T packed tokens).
 *
 * Layouts (row-major, fp32): q, k, alpha [B, T, H, dk]; v [B, T, H, dv];
 * beta [B, T, H].  S0 (NULL = zero state) and S_final (NULL = not wanted):
 * [num_seqs or B, H, dk, dv].  out: fp64 [B, T, H, dv].
 *
 * nthreads <= 0 uses the OpenMP default.  Returns 0, or -1 on bad sizes.
 */
int kda_oracle_forward(const float* q, const float* k, const float* v,
                       const float* alpha, const float* beta, const float* S0,
                       const int32_t* cu_seqlens, int32_t num_seqs,
                       int32_t B, int64_t T, int32_t H, int32_t dk, int32_t dv,
                       double* out, double* S_final, int32_t nthreads)
{
    if (B < 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    if (cu_seqlens && B != 1) return -1;
    const int64_t nseq = cu_seqlens ? (int64_t)num_seqs : (int64_t)B;
    if (cu_seqlens) {
        if (num_seqs < 0 || cu_seqlens[0] != 0 || (int64_t)cu_seqlens[num_seqs] != T) return -1;
        for (int32_t n = 0; n < num_seqs; ++n)
            if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    }
    const int64_t sk = (int64_t)H * dk, sv = (int64_t)H * dv, sb = H;
    /* column blocks: enough work items to keep the cores busy when there are
     * few (sequence, head) pairs, as in a single 1M-token head */
    int maxthr = 1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
    maxthr = omp_get_max_threads();
#else
    (void)nthreads;
#endif
    int ncb = 1;
    while (ncb < 32 && dv % (ncb * 2) == 0 && nseq * H * ncb < 2 * (int64_t)maxthr) ncb *= 2;
    const int64_t units = nseq * H * ncb;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t u = 0; u < units; ++u) {
        const int64_t n = u / ((int64_t)H * ncb);
        const int h = (int)((u / ncb) % H);
        const int cb = (int)(u % ncb);
        const int j0 = cb * (dv / ncb), j1 = j0 + dv / ncb;
        int64_t t0, ntok;
        if (cu_seqlens) { t0 = cu_seqlens[n]; ntok = (int64_t)cu_seqlens[n + 1] - cu_seqlens[n]; }
        else { t0 = n * T; ntok = T; }
        recur_block(q + t0 * sk + (int64_t)h * dk, k + t0 * sk + (int64_t)h * dk,
                    v + t0 * sv + (int64_t)h * dv, alpha + t0 * sk + (int64_t)h * dk,
                    beta + t0 * sb + h, ntok, sk, sv, sb, dk, dv, j0, j1,
                    S0 ? S0 + ((size_t)n * H + h) * (size_t)dk * dv : NULL,
                    out + t0 * sv + (int64_t)h * dv,
                    S_final ? S_final + ((size_t)n * H + h) * (size_t)dk * dv : NULL);
    }
    return 0;
}
