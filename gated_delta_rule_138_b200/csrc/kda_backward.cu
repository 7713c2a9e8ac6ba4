// KDA backward pass: reverse mode of the token recurrence, on CUDA cores.
//
// The recurrence is the one the forward kernels compute (the worldcybernews
// article "Kimi K3 Open Model Surpasses Closed GPT and Anthropic Systems on
// Independent Benchmarks", paragraph 2), written per token as
//
//   S'_t = Diag(a_t) S_{t-1},  x_t = S'_t^T k_t,  u_t = b_t (v_t - x_t),
//   S_t  = S'_t + k_t u_t^T,   o_t = S_t^T q_t,          a_t = clamp(alpha_t, e^-5, 1).
//
// Given dL/do_t and dL/dS_final, with G = dL/dS_t carried from the last token
// backwards:
//
//   dq_t = S_t do_t;   G += q_t do_t^T;   du = G^T k_t;   db_t = du . (v_t - x_t)
//   dv_t = b_t du;     dx = -b_t du;      dk_t = G u_t + S'_t dx
//   dS' = G + k_t dx^T;  dalpha_t[c] = sum_n dS'[c,n] S_{t-1}[c,n] (0 outside [e^-5, 1])
//   G = Diag(a_t) dS'   (dL/dS_{t-1});    dS0 = G after the first token.
//
// One CTA of 256 threads owns one (sequence, head) and holds S and G in
// registers, d_k x d_v split as in the decode kernel (thread (tx, ty): rows
// ty + TY i, columns 4 tx .. 4 tx + 3).  The reverse sweep needs S_{t-1} for t
// descending, and the step is not invertible in floating point, so states are
// recomputed: a forward sweep stores the state at every 8-token chunk start
// (checkpoints); then, chunk by chunk from the last, the chunk's 8 states are
// recomputed from its checkpoint into a scratch slab (512 KB per CTA at d = 128:
// the slabs of all resident CTAs fit in L2) and read back in reverse.  Each thread reads back
// only what it wrote, so the slabs need no barriers.  The token rows of the
// next chunk to be worked on are prefetched into L2 one chunk ahead.
#include "kda_common.cuh"

namespace kda {
namespace bwd {

constexpr int NT = 256;
constexpr int CK = 8;    // tokens between checkpoints

template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(NT, 1)
kda_backward_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                    const Tin* __restrict__ alpha, const Tin* __restrict__ beta,
                    const float* __restrict__ S0, const Tin* __restrict__ dout,
                    const float* __restrict__ dSf, const int32_t* __restrict__ cu_seqlens,
                    int64_t T, int H, int64_t ck_per_seq, float* __restrict__ dq,
                    float* __restrict__ dk, float* __restrict__ dv, float* __restrict__ dalpha,
                    float* __restrict__ dbeta, float* __restrict__ dS0,
                    float* __restrict__ ckpt, float* __restrict__ scratch) {
    constexpr int TX = DV / 4;      // threads across a row (float4 each)
    constexpr int TY = NT / TX;     // rows per pass
    constexpr int RPT = DK / TY;    // rows per thread
    static_assert(DV % 4 == 0 && NT % TX == 0 && DK % TY == 0 && TX <= 32, "tile");
    // (arrays read or written as float4 are declared 16-byte aligned)
    __shared__ float ga[DK], ka[DK], kk[DK], qq[DK], okm[DK];
    __shared__ float vv[DV], xs[DV];
    __shared__ __align__(16) float dov[DV];
    __shared__ __align__(16) float us[DV];
    __shared__ __align__(16) float dxs[DV];
    __shared__ __align__(16) float red[TY][DV];
    // per-row partials over the TX threads of a row (dq; later dk and dalpha),
    // padded so that a thread summing one row reads its own bank sequence
    __shared__ float rowp[2][DK][TX + 1];
    __shared__ float dbp[NT / 32];
    __shared__ float sb;

    const int tid = threadIdx.x, tx = tid % TX, ty = tid / TX;
    const int64_t unit = blockIdx.x;
    const int n = (int)(unit / H), h = (int)(unit % H);
    int64_t bos, len;
    seq_range(cu_seqlens, n, T, bos, len);
    const size_t mat = (size_t)DK * DV;
    // this sequence's first checkpoint: dense, ck_per_seq per sequence; packed,
    // floor(bos / CK) + n (room for ceil(len / CK) before the next sequence's)
    const int64_t ck0 = cu_seqlens ? bos / CK + n : (int64_t)n * ck_per_seq;
    float4* scr = reinterpret_cast<float4*>(scratch + (size_t)unit * CK * mat);
    auto slab = [&](float4* base, int i) -> float4& { return base[(size_t)(ty + TY * i) * TX + tx]; };
    auto ck_at = [&](int64_t ci) {
        return reinterpret_cast<float4*>(ckpt + ((size_t)(ck0 + ci) * H + h) * mat);
    };
    auto tok = [&](int64_t t) { return (bos + t) * H + h; };   // (token, head) row
    // L2 prefetch of the rows of chunk ci (k, alpha, v, beta; with q and dout when
    // `grads`): one thread per 128-byte line, no registers held
    constexpr int LK = (DK * (int)sizeof(Tin) + 127) / 128, LV = (DV * (int)sizeof(Tin) + 127) / 128;
    constexpr int LINES = 3 * LK + 2 * LV + 1;
    auto prefetch_chunk = [&](int64_t ci, bool grads) {
        if (ci < 0 || ci * CK >= len) return;
        const int64_t t0 = ci * CK;
        const int L = (int)(min(len, t0 + CK) - t0);
        for (int e = tid; e < L * LINES; e += NT) {
            const int j = e / LINES, l = e % LINES;
            const int64_t r = tok(t0 + j);
            const char* line = nullptr;
            if (l < LK) line = reinterpret_cast<const char*>(k + r * DK) + 128 * l;
            else if (l < 2 * LK) line = reinterpret_cast<const char*>(alpha + r * DK) + 128 * (l - LK);
            else if (l < 3 * LK) {
                if (grads) line = reinterpret_cast<const char*>(q + r * DK) + 128 * (l - 2 * LK);
            } else if (l < 3 * LK + LV) line = reinterpret_cast<const char*>(v + r * DV) + 128 * (l - 3 * LK);
            else if (l < 3 * LK + 2 * LV) {
                if (grads) line = reinterpret_cast<const char*>(dout + r * DV) + 128 * (l - 3 * LK - LV);
            } else line = reinterpret_cast<const char*>(beta + r);
            if (line) asm volatile("prefetch.global.L2 [%0];" :: "l"(line));
        }
    };

    float4 s[RPT];
    {
        const float4* src = S0 ? reinterpret_cast<const float4*>(S0 + (size_t)unit * mat) : nullptr;
#pragma unroll
        for (int i = 0; i < RPT; ++i)
            s[i] = src ? src[(size_t)(ty + TY * i) * TX + tx] : make_float4(0.f, 0.f, 0.f, 0.f);
    }

    // x_t = S'^T k_t over this thread's rows, reduced over the rows of the block:
    // returns with xs and us (u_t) filled
    auto project = [&]() {
        float4 px = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const float w = ka[ty + TY * i];
            px.x = fmaf(s[i].x, w, px.x); px.y = fmaf(s[i].y, w, px.y);
            px.z = fmaf(s[i].z, w, px.z); px.w = fmaf(s[i].w, w, px.w);
        }
        *reinterpret_cast<float4*>(&red[ty][4 * tx]) = px;
        __syncthreads();
        if (tid < DV) {
            float x = 0.0f;
#pragma unroll
            for (int j = 0; j < TY; ++j) x += red[j][tid];
            xs[tid] = x;
            us[tid] = sb * (vv[tid] - x);
        }
        __syncthreads();
    };
    auto load_token = [&](int64_t t, bool grads) {
        const int64_t r = tok(t);
        if (tid < DK) {
            const float araw = to_f32(alpha[r * DK + tid]);
            const float a = clamp_gate(araw), kv = to_f32(k[r * DK + tid]);
            ga[tid] = a;
            ka[tid] = a * kv;
            kk[tid] = kv;
            if (grads) {
                qq[tid] = to_f32(q[r * DK + tid]);
                okm[tid] = (araw >= kAlphaMin && araw <= 1.0f) ? 1.0f : 0.0f;
            }
        }
        if (tid < DV) {
            vv[tid] = to_f32(v[r * DV + tid]);
            if (grads) dov[tid] = to_f32(dout[r * DV + tid]);
        }
        if (tid == 0) sb = to_f32(beta[r]);
        __syncthreads();
    };
    // one forward token: S <- Diag(a) S + k u^T
    auto forward_token = [&](int64_t t) {
        __syncthreads();   // the previous step has finished with the shared vectors
        load_token(t, false);
        project();
        const float4 u4 = *reinterpret_cast<const float4*>(&us[4 * tx]);
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const int c = ty + TY * i;
            const float a = ga[c], kc = kk[c];
            s[i].x = fmaf(a, s[i].x, kc * u4.x); s[i].y = fmaf(a, s[i].y, kc * u4.y);
            s[i].z = fmaf(a, s[i].z, kc * u4.z); s[i].w = fmaf(a, s[i].w, kc * u4.w);
        }
    };

    // ---- forward sweep: a checkpoint at every chunk start
    const int64_t nck = (len + CK - 1) / CK;
    prefetch_chunk(0, false);
    for (int64_t ci = 0; ci < nck; ++ci) {
        prefetch_chunk(ci + 1, false);
        float4* ck = ck_at(ci);
#pragma unroll
        for (int i = 0; i < RPT; ++i) slab(ck, i) = s[i];
        const int64_t t1 = min(len, (ci + 1) * CK);
        for (int64_t t = ci * CK; t < t1; ++t) forward_token(t);
    }

    float4 g[RPT];
    {
        const float4* src = dSf ? reinterpret_cast<const float4*>(dSf + (size_t)unit * mat) : nullptr;
#pragma unroll
        for (int i = 0; i < RPT; ++i)
            g[i] = src ? src[(size_t)(ty + TY * i) * TX + tx] : make_float4(0.f, 0.f, 0.f, 0.f);
    }

    // row c of slot `slot` summed over its TX partials
    auto row_sum = [&](int slot, int c) {
        const float* p = rowp[slot][c];
        float sum = 0.0f;
#pragma unroll
        for (int j = 0; j < TX; ++j) sum += p[j];
        return sum;
    };

    // ---- reverse sweep, chunk by chunk from the last
    prefetch_chunk(nck - 1, true);
    for (int64_t ci = nck - 1; ci >= 0; --ci) {
        prefetch_chunk(ci - 1, true);
        const float4* ck = ck_at(ci);
#pragma unroll
        for (int i = 0; i < RPT; ++i) s[i] = ck[(size_t)(ty + TY * i) * TX + tx];
        const int64_t t0 = ci * CK;
        const int L = (int)(min(len, t0 + CK) - t0);
        for (int j = 0; j < L; ++j) {   // S_{t-1} of every token of the chunk
#pragma unroll
            for (int i = 0; i < RPT; ++i) slab(scr + (size_t)j * (mat / 4), i) = s[i];
            forward_token(t0 + j);
        }
        for (int j = L - 1; j >= 0; --j) {
            const int64_t t = t0 + j, r = tok(t);
#pragma unroll
            for (int i = 0; i < RPT; ++i) s[i] = slab(scr + (size_t)j * (mat / 4), i);   // S_{t-1}
            __syncthreads();
            load_token(t, true);
            project();
            const float4 u4 = *reinterpret_cast<const float4*>(&us[4 * tx]);
            const float4 do4 = *reinterpret_cast<const float4*>(&dov[4 * tx]);
            // through o_t = S_t^T q_t: dq_t, then G += q_t do_t^T; du = G^T k_t (partial)
            float4 pdu = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int i = 0; i < RPT; ++i) {
                const int c = ty + TY * i;
                const float a = ga[c], kc = kk[c], qc = qq[c];
                float4 st;
                st.x = fmaf(a, s[i].x, kc * u4.x); st.y = fmaf(a, s[i].y, kc * u4.y);
                st.z = fmaf(a, s[i].z, kc * u4.z); st.w = fmaf(a, s[i].w, kc * u4.w);
                rowp[0][c][tx] = st.x * do4.x + st.y * do4.y + st.z * do4.z + st.w * do4.w;
                g[i].x = fmaf(qc, do4.x, g[i].x); g[i].y = fmaf(qc, do4.y, g[i].y);
                g[i].z = fmaf(qc, do4.z, g[i].z); g[i].w = fmaf(qc, do4.w, g[i].w);
                pdu.x = fmaf(g[i].x, kc, pdu.x); pdu.y = fmaf(g[i].y, kc, pdu.y);
                pdu.z = fmaf(g[i].z, kc, pdu.z); pdu.w = fmaf(g[i].w, kc, pdu.w);
            }
            *reinterpret_cast<float4*>(&red[ty][4 * tx]) = pdu;
            __syncthreads();
            for (int c = tid; c < DK; c += NT) dq[r * DK + c] = row_sum(0, c);
            // through u_t = b_t (v_t - x_t): dv_t, dx, db_t
            float db = 0.0f;
            if (tid < DV) {
                float du = 0.0f;
#pragma unroll
                for (int jy = 0; jy < TY; ++jy) du += red[jy][tid];
                dv[r * DV + tid] = sb * du;
                dxs[tid] = -sb * du;
                db = du * (vv[tid] - xs[tid]);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) db += __shfl_xor_sync(0xffffffffu, db, o);
            if ((tid & 31) == 0) dbp[tid >> 5] = db;
            __syncthreads();
            if (tid == 0) {
                float sum = 0.0f;
#pragma unroll
                for (int w = 0; w < NT / 32; ++w) sum += dbp[w];
                dbeta[r] = sum;
            }
            const float4 dx4 = *reinterpret_cast<const float4*>(&dxs[4 * tx]);
            // through x_t = S'^T k_t and S'_t = Diag(a_t) S_{t-1}: dk_t, dalpha_t, G <- dS_{t-1}
#pragma unroll
            for (int i = 0; i < RPT; ++i) {
                const int c = ty + TY * i;
                const float a = ga[c], kc = kk[c];
                const float4 sp = make_float4(a * s[i].x, a * s[i].y, a * s[i].z, a * s[i].w);
                rowp[0][c][tx] = g[i].x * u4.x + g[i].y * u4.y + g[i].z * u4.z + g[i].w * u4.w +
                                 sp.x * dx4.x + sp.y * dx4.y + sp.z * dx4.z + sp.w * dx4.w;
                float4 dsp;
                dsp.x = fmaf(kc, dx4.x, g[i].x); dsp.y = fmaf(kc, dx4.y, g[i].y);
                dsp.z = fmaf(kc, dx4.z, g[i].z); dsp.w = fmaf(kc, dx4.w, g[i].w);
                rowp[1][c][tx] = dsp.x * s[i].x + dsp.y * s[i].y + dsp.z * s[i].z + dsp.w * s[i].w;
                g[i] = make_float4(a * dsp.x, a * dsp.y, a * dsp.z, a * dsp.w);
            }
            __syncthreads();
            // (slot 0 was last read for dq before the barrier of the db reduction)
            for (int e = tid; e < 2 * DK; e += NT) {
                const int c = e % DK;
                if (e < DK) dk[r * DK + c] = row_sum(0, c);
                else dalpha[r * DK + c] = okm[c] * row_sum(1, c);
            }
        }
    }
    if (dS0) {
        float4* dst = reinterpret_cast<float4*>(dS0 + (size_t)unit * mat);
#pragma unroll
        for (int i = 0; i < RPT; ++i) dst[(size_t)(ty + TY * i) * TX + tx] = g[i];
    }
}

template <typename Tin, int DK, int DV>
static cudaError_t launch_t(const void* q, const void* k, const void* v, const void* alpha,
                            const void* beta, const float* S0, const void* dout, const float* dSf,
                            const int32_t* cu, int64_t units, int64_t T, int H, int64_t ck_per_seq,
                            float* dq, float* dk, float* dv, float* dalpha, float* dbeta,
                            float* dS0, float* ckpt, float* scratch, cudaStream_t s) {
    kda_backward_kernel<Tin, DK, DV><<<(unsigned)units, NT, 0, s>>>(
        (const Tin*)q, (const Tin*)k, (const Tin*)v, (const Tin*)alpha, (const Tin*)beta, S0,
        (const Tin*)dout, dSf, cu, T, H, ck_per_seq, dq, dk, dv, dalpha, dbeta, dS0, ckpt, scratch);
    return cudaGetLastError();
}

}  // namespace bwd

// Floats of workspace the backward needs: checkpoints (dense: nseq * ceil(T / 8)
// per head; packed: floor(T / 8) + nseq per head) and one 8-state scratch slab
// per (sequence, head).
size_t backward_workspace_floats(bool packed, int64_t nseq, int64_t T, int H, int DK, int DV) {
    const int64_t cks = packed ? T / bwd::CK + nseq : nseq * ((T + bwd::CK - 1) / bwd::CK);
    return ((size_t)cks * H + (size_t)nseq * H * bwd::CK) * (size_t)DK * DV;
}

cudaError_t launch_backward(int in_bf16, const void* q, const void* k, const void* v,
                            const void* alpha, const void* beta, const float* S0, const void* dout,
                            const float* dSf, const int32_t* cu, int64_t nseq, int64_t T, int H,
                            int DK, int DV, float* dq, float* dk, float* dv, float* dalpha,
                            float* dbeta, float* dS0, float* workspace, cudaStream_t s) {
    const int64_t units = nseq * H;
    const int64_t ck_per_seq = cu ? 0 : (T + bwd::CK - 1) / bwd::CK;
    const int64_t cks = cu ? T / bwd::CK + nseq : nseq * ck_per_seq;
    float* ckpt = workspace;
    float* scratch = workspace + (size_t)cks * H * DK * DV;
#define KDA_BWD_CASE(TI, A, B)                                                                   \
    if (DK == A && DV == B)                                                                      \
        return bwd::launch_t<TI, A, B>(q, k, v, alpha, beta, S0, dout, dSf, cu, units, T, H,      \
                                       ck_per_seq, dq, dk, dv, dalpha, dbeta, dS0, ckpt, scratch, s);
    if (in_bf16) {
        KDA_BWD_CASE(__nv_bfloat16, 64, 64) KDA_BWD_CASE(__nv_bfloat16, 64, 128)
        KDA_BWD_CASE(__nv_bfloat16, 128, 64) KDA_BWD_CASE(__nv_bfloat16, 128, 128)
    } else {
        KDA_BWD_CASE(float, 64, 64) KDA_BWD_CASE(float, 64, 128)
        KDA_BWD_CASE(float, 128, 64) KDA_BWD_CASE(float, 128, 128)
    }
#undef KDA_BWD_CASE
    return cudaErrorInvalidValue;
}

}  // namespace kda
