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

/*
 * Reverse mode of the same recurrence (the backward pass), fp64.  Written from
 * the forward above, one token at a time, in the order
 *
 *     S'_t = Diag(a_t) S_{t-1};   x_t = S'_t^T k_t;   u_t = b_t (v_t - x_t);
 *     S_t  = S'_t + k_t u_t^T;    o_t = S_t^T q_t,
 *
 * which is the forward's update expanded (S_t = S' - b k k^T S' + b k v^T).
 * Given dL/do_t for every token and dL/dS_final (NULL = 0), with G = dL/dS_t
 * carried backwards from the last token:
 *
 *     dq_t  = S_t do_t;              G += q_t do_t^T
 *     du    = G^T k_t;               dk_t = G u_t
 *     db_t  = du . (v_t - x_t);      dv_t = b_t du;     dx = -b_t du
 *     dS'   = G + k_t dx^T;          dk_t += S'_t dx
 *     da_c  = sum_n dS'[c,n] S_{t-1}[c,n];   dalpha_t[c] = da_c if e^-5 <= alpha <= 1, else 0
 *     G     = Diag(a_t) dS'          (dL/dS_{t-1});   dS0 = G after the first token.
 *
 * The clamp passes the gradient where alpha lies in [e^-5, 1], bounds
 * included, and blocks it outside.  Every state S_0..S_T of the sequence is
 * kept (T+1 matrices of dk x dv doubles): plain and slow, for test sizes.
 */
static void backward_one(const float* q, const float* k, const float* v,
                         const float* alpha, const float* beta, const float* dout,
                         int64_t ntok, int64_t sk, int64_t sv, int64_t sb, int dk, int dv,
                         const float* S0, const float* dSf,
                         double* dq, double* dkk, double* dvv, double* dal, double* dbe,
                         double* dS0)
{
    const size_t m = (size_t)dk * (size_t)dv;
    double* St = (double*)malloc(sizeof(double) * m * (size_t)(ntok + 1));
    double* G = (double*)malloc(sizeof(double) * m);
    double* Sp = (double*)malloc(sizeof(double) * m);
    double* dSp = (double*)malloc(sizeof(double) * m);
    double* a = (double*)malloc(sizeof(double) * (size_t)dk);
    double* x = (double*)malloc(sizeof(double) * (size_t)dv);
    double* u = (double*)malloc(sizeof(double) * (size_t)dv);
    double* du = (double*)malloc(sizeof(double) * (size_t)dv);
    double* dx = (double*)malloc(sizeof(double) * (size_t)dv);
    for (size_t i = 0; i < m; ++i) St[i] = S0 ? (double)S0[i] : 0.0;

    /* forward, keeping S_t for every t (S_0 first) */
    for (int64_t t = 0; t < ntok; ++t) {
        const double* Sprev = St + m * (size_t)t;
        double* Snew = St + m * (size_t)(t + 1);
        const float* kt = k + t * sk;
        const double bt = (double)beta[t * sb];
        for (int c = 0; c < dk; ++c) a[c] = clamp_alpha(alpha[t * sk + c]);
        for (int c = 0; c < dk; ++c)
            for (int n = 0; n < dv; ++n) Sp[(size_t)c * dv + n] = a[c] * Sprev[(size_t)c * dv + n];
        for (int n = 0; n < dv; ++n) {
            double s = 0.0;
            for (int c = 0; c < dk; ++c) s += Sp[(size_t)c * dv + n] * (double)kt[c];
            x[n] = s;
            u[n] = bt * ((double)v[t * sv + n] - s);
        }
        for (int c = 0; c < dk; ++c)
            for (int n = 0; n < dv; ++n)
                Snew[(size_t)c * dv + n] = Sp[(size_t)c * dv + n] + (double)kt[c] * u[n];
    }

    for (size_t i = 0; i < m; ++i) G[i] = dSf ? (double)dSf[i] : 0.0;
    for (int64_t t = ntok - 1; t >= 0; --t) {
        const double* Sprev = St + m * (size_t)t;
        const double* Scur = St + m * (size_t)(t + 1);
        const float* qt = q + t * sk;
        const float* kt = k + t * sk;
        const float* at = alpha + t * sk;
        const float* vt = v + t * sv;
        const float* dot = dout + t * sv;
        const double bt = (double)beta[t * sb];
        const double amin = (double)ORACLE_ALPHA_MIN_F32;
        for (int c = 0; c < dk; ++c) a[c] = clamp_alpha(at[c]);
        /* recompute S', x, u of this token */
        for (int c = 0; c < dk; ++c)
            for (int n = 0; n < dv; ++n) Sp[(size_t)c * dv + n] = a[c] * Sprev[(size_t)c * dv + n];
        for (int n = 0; n < dv; ++n) {
            double s = 0.0;
            for (int c = 0; c < dk; ++c) s += Sp[(size_t)c * dv + n] * (double)kt[c];
            x[n] = s;
            u[n] = bt * ((double)vt[n] - s);
        }
        /* through o_t = S_t^T q_t */
        for (int c = 0; c < dk; ++c) {
            double s = 0.0;
            for (int n = 0; n < dv; ++n) s += Scur[(size_t)c * dv + n] * (double)dot[n];
            dq[t * sk + c] = s;
        }
        for (int c = 0; c < dk; ++c)
            for (int n = 0; n < dv; ++n) G[(size_t)c * dv + n] += (double)qt[c] * (double)dot[n];
        /* S_t = S'_t + k_t u_t^T */
        for (int c = 0; c < dk; ++c) {
            double s = 0.0;
            for (int n = 0; n < dv; ++n) s += G[(size_t)c * dv + n] * u[n];
            dkk[t * sk + c] = s;
        }
        double db = 0.0;
        for (int n = 0; n < dv; ++n) {
            double s = 0.0;
            for (int c = 0; c < dk; ++c) s += G[(size_t)c * dv + n] * (double)kt[c];
            du[n] = s;
            /* u_t = b_t (v_t - x_t) */
            db += s * ((double)vt[n] - x[n]);
            dvv[t * sv + n] = bt * s;
            dx[n] = -bt * s;
        }
        dbe[t * sb] = db;
        /* x_t = S'_t^T k_t */
        for (int c = 0; c < dk; ++c) {
            double s = 0.0;
            for (int n = 0; n < dv; ++n) {
                dSp[(size_t)c * dv + n] = G[(size_t)c * dv + n] + (double)kt[c] * dx[n];
                s += Sp[(size_t)c * dv + n] * dx[n];
            }
            dkk[t * sk + c] += s;
        }
        /* S'_t = Diag(a_t) S_{t-1} */
        for (int c = 0; c < dk; ++c) {
            double s = 0.0;
            for (int n = 0; n < dv; ++n) s += dSp[(size_t)c * dv + n] * Sprev[(size_t)c * dv + n];
            const double araw = (double)at[c];
            dal[t * sk + c] = (araw >= amin && araw <= 1.0) ? s : 0.0;
            for (int n = 0; n < dv; ++n) G[(size_t)c * dv + n] = a[c] * dSp[(size_t)c * dv + n];
        }
    }
    if (dS0)
        for (size_t i = 0; i < m; ++i) dS0[i] = G[i];
    free(St); free(G); free(Sp); free(dSp); free(a); free(x); free(u); free(du); free(dx);
}

/*
 * Backward over a dense or packed batch, layouts as kda_oracle_forward; dout
 * like v (fp32), dS_final like S0 (NULL = 0).  Gradients are fp64 with the
 * layouts of their inputs: dq, dk, dalpha [B, T, H, dk]; dv [B, T, H, dv];
 * dbeta [B, T, H]; dS0 [num_seqs or B, H, dk, dv] (NULL = not wanted).
 * Returns 0, -1 on bad sizes, -2 when the kept states would pass 4 GB.
 */
int kda_oracle_backward(const float* q, const float* k, const float* v,
                        const float* alpha, const float* beta, const float* S0,
                        const float* dout, const float* dS_final,
                        const int32_t* cu_seqlens, int32_t num_seqs,
                        int32_t B, int64_t T, int32_t H, int32_t dk, int32_t dv,
                        double* dq, double* dk_out, double* dv_out, double* dalpha,
                        double* dbeta, double* dS0, int32_t nthreads)
{
    if (B < 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    if (cu_seqlens && B != 1) return -1;
    const int64_t nseq = cu_seqlens ? (int64_t)num_seqs : (int64_t)B;
    int64_t longest = cu_seqlens ? 0 : T;
    if (cu_seqlens) {
        if (num_seqs < 0 || cu_seqlens[0] != 0 || (int64_t)cu_seqlens[num_seqs] != T) return -1;
        for (int32_t n = 0; n < num_seqs; ++n) {
            if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
            if (cu_seqlens[n + 1] - cu_seqlens[n] > longest) longest = cu_seqlens[n + 1] - cu_seqlens[n];
        }
    }
    if ((double)(longest + 1) * dk * dv * 8.0 > 4e9) return -2;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    const int64_t sk = (int64_t)H * dk, sv = (int64_t)H * dv, sb = H;
    const int64_t units = nseq * H;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t uidx = 0; uidx < units; ++uidx) {
        const int64_t n = uidx / H;
        const int h = (int)(uidx % H);
        int64_t t0, ntok;
        if (cu_seqlens) { t0 = cu_seqlens[n]; ntok = (int64_t)cu_seqlens[n + 1] - cu_seqlens[n]; }
        else { t0 = n * T; ntok = T; }
        const size_t so = ((size_t)n * H + h) * (size_t)dk * dv;
        backward_one(q + t0 * sk + (int64_t)h * dk, k + t0 * sk + (int64_t)h * dk,
                     v + t0 * sv + (int64_t)dv * h, alpha + t0 * sk + (int64_t)h * dk,
                     beta + t0 * sb + h, dout + t0 * sv + (int64_t)dv * h, ntok, sk, sv, sb,
                     dk, dv, S0 ? S0 + so : NULL, dS_final ? dS_final + so : NULL,
                     dq + t0 * sk + (int64_t)h * dk, dk_out + t0 * sk + (int64_t)h * dk,
                     dv_out + t0 * sv + (int64_t)dv * h, dalpha + t0 * sk + (int64_t)h * dk,
                     dbeta + t0 * sb + h, dS0 ? dS0 + so : NULL);
    }
    return 0;
}
