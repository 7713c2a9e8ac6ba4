// KDA single-token decode step: the fixed-size state replaces the KV cache
// (worldcybernews article "Kimi K3 Open Model Surpasses Closed GPT and
// Anthropic Systems on Independent Benchmarks", paragraph 2).
//
// For each (sequence, head), with a = clamp(alpha, e^-5, 1):
//   S_t = (I - beta k k^T) Diag(a) S + beta k v^T,   o = S_t^T q
// is computed in ONE pass over S (read once, written once):
//   x = S^T (a*k),  y = S^T (a*q)           (column sums over key channels)
//   u = beta (v - x)
//   o = y + u (k . q)
//   S <- Diag(a) S + k u^T
// which expands to the same S_t (Diag(a)S - beta k (k^T Diag(a) S) + beta k v^T)
// and o_t = S_t^T q = (Diag(a) S)^T q + u (k^T q).
//
// The state is fp32 and HBM-bound: one CTA per (sequence, head) streams its
// d_k x d_v slab with 16-byte loads and stores, keeping it in registers between
// the reduction and the update.  A multi-token step (T tokens per sequence,
// inputs [N, T, H, d]) keeps the state in registers across its T tokens: the
// state is read and written once per step, not once per token.  The token rows
// (q, k, alpha, v, beta) of up to kStageTokens tokens are staged in shared memory
// with 16-byte loads issued right behind the state loads, so that the token loop
// waits on no global load.
#include "kda_common.cuh"

namespace kda {

constexpr int kStageTokens = 8;    // token rows staged (and prepared) in shared memory at a time

// kFused: alpha and beta arrive as logits and q, k unnormalised (a compile-time
// variant, so that the plain step carries none of the transforms' code).
// kMulti: steps of T > 1 tokens (staged and prepared in batches); without it, T = 1.
template <typename Tin, typename Tout, int DK, int DV, bool kFused, bool kMulti>
// (a single-token step keeps three CTAs per SM for loads in flight; a multi-token step
// runs two, with the registers its batch work needs: 0.234 -> 0.227 ms per 4-token step)
__global__ void __launch_bounds__(256, kMulti ? 2 : 3)
kda_decode_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                  const Tin* __restrict__ v, const Tin* __restrict__ alpha,
                  const Tin* __restrict__ beta, float* __restrict__ S, Tout* __restrict__ out,
                  const int32_t* __restrict__ slots, int num_slots, int H, int T) {
    constexpr bool fused = kFused;
    constexpr int NT = 256;
    constexpr int TX = DV / 4;       // threads across a row (float4 each)
    constexpr int TY = NT / TX;      // rows per pass
    constexpr int RPT = DK / TY;     // rows per thread
    static_assert(DV % 4 == 0 && NT % TX == 0 && DK % TY == 0, "tile");
    __shared__ float ka[DK], qa[DK], kk[DK], ga[DK];
    // (arrays read or written as float4 are declared 16-byte aligned)
    __shared__ __align__(16) float red_x[TY][DV];
    __shared__ __align__(16) float red_y[TY][DV];
    __shared__ __align__(16) float us[DV];
    __shared__ float kq_part[NT / 32], nk_part[NT / 32], nq_part[NT / 32];
    constexpr int VE = 16 / (int)sizeof(Tin);            // elements per 16-byte load
    // multi-token steps: the staged token rows (q, k, alpha [NS][DK], v [NS][DV], beta),
    // then every staged token's a, a*k, a*q, k and k.q (one element in the single-token
    // variant)
    constexpr int NS = kMulti ? kStageTokens : 1;
    __shared__ __align__(16) Tin tin[NS * (3 * DK + DV)];
    __shared__ Tin tbeta[NS];
    // (a*k, a*q, a, k) of key channel c in one 16-byte element: one load per row and pass
    __shared__ __align__(16) float4 bcf[NS][DK];
    __shared__ float bkq[NS];

    const int tid = threadIdx.x, tx = tid % TX, ty = tid / TX;
    const size_t nh = blockIdx.x;                 // (sequence, head) flattened
    // state slot (slots null: the sequence's own index); an invalid slot decodes
    // from a zero state and writes no state
    const int64_t n = (int64_t)(nh / H), hh = (int64_t)(nh % H);
    const int64_t slot = slots ? (int64_t)slots[n] : n;
    const bool slot_ok = !slots || (slot >= 0 && slot < num_slots);
    float4* Sv = reinterpret_cast<float4*>(S + ((size_t)(slot_ok ? slot : 0) * H + hh) * (size_t)DK * DV);

    // issue the state loads first: they are the HBM traffic
    float4 s[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i)
        s[i] = slot_ok ? Sv[(size_t)(ty + TY * i) * TX + tx] : make_float4(0.f, 0.f, 0.f, 0.f);

    // a single-token step reads its rows straight from global memory (no staging,
    // no extra barrier); longer steps stage a batch of token rows and prepare every
    // token's gated vectors for the whole batch at once, so that a token then takes two
    // barriers (reduction partials, u) instead of four
    constexpr bool direct = !kMulti;
    for (int t = 0; t < T; ++t) {
    const size_t tok = ((size_t)n * T + t) * H + hh;   // (sequence, token, head)
    const size_t vb = tok * DV;
    const int ts = t % kStageTokens;                     // staged slot of this token
    if constexpr (kMulti) if (ts == 0) {
        // stage the token rows of tokens t .. t + nt - 1 with 16-byte loads (the barrier
        // before: every thread is done with the previous batch)
        if (t > 0) __syncthreads();
        const int nt = T - t < kStageTokens ? T - t : kStageTokens;
        constexpr int RK = DK / VE, RV = DV / VE, RT = 3 * RK + RV;   // 16-byte pieces per token
        for (int e = tid; e < nt * RT; e += NT) {
            const int tt = e / RT, w = e % RT;
            const size_t tk = ((size_t)n * T + t + tt) * H + hh;
            const Tin* src;
            Tin* dst;
            if (w < RK) { src = q + tk * DK + w * VE; dst = tin + tt * DK + w * VE; }
            else if (w < 2 * RK) { src = k + tk * DK + (w - RK) * VE; dst = tin + (NS + tt) * DK + (w - RK) * VE; }
            else if (w < 3 * RK) { src = alpha + tk * DK + (w - 2 * RK) * VE; dst = tin + (2 * NS + tt) * DK + (w - 2 * RK) * VE; }
            else { src = v + tk * DV + (w - 3 * RK) * VE; dst = tin + 3 * NS * DK + tt * DV + (w - 3 * RK) * VE; }
            *reinterpret_cast<uint4*>(dst) = __ldg(reinterpret_cast<const uint4*>(src));
        }
        if (tid < nt) tbeta[tid] = beta[((size_t)n * T + t + tid) * H + hh];
        __syncthreads();
        // per staged token: gate a, a*k, a*q, k (normalised in the fused variant) and k.q;
        // warp w takes tokens w and w + 8, lane l channels l, l + 32, ...
        for (int tt = tid >> 5; tt < nt; tt += NT / 32) {
            const int l = tid & 31;
            const Tin* rq = tin + tt * DK;
            const Tin* rk = tin + (NS + tt) * DK;
            const Tin* ra = tin + (2 * NS + tt) * DK;
            float kv[DK / 32], qv[DK / 32];
            float pk = 0.0f, pq = 0.0f;
#pragma unroll
            for (int j = 0; j < DK / 32; ++j) {
                kv[j] = to_f32(rk[l + 32 * j]);
                qv[j] = to_f32(rq[l + 32 * j]);
                pk = fmaf(kv[j], kv[j], pk);
                pq = fmaf(qv[j], qv[j], pq);
            }
            float ikn = 1.0f, iqn = 1.0f;
            if constexpr (fused) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    pk += __shfl_xor_sync(0xffffffffu, pk, o);
                    pq += __shfl_xor_sync(0xffffffffu, pq, o);
                }
                ikn = rsqrtf(fmaxf(pk, 1e-12f));
                iqn = rsqrtf(fmaxf(pq, 1e-12f));
            }
            float kqp = 0.0f;
#pragma unroll
            for (int j = 0; j < DK / 32; ++j) {
                const int c = l + 32 * j;
                const float ax = to_f32(ra[c]);
                const float a = clamp_gate(fused ? gate_from_logit(ax) : ax);
                const float kc = kv[j] * ikn, qc = qv[j] * iqn;
                bcf[tt][c] = make_float4(a * kc, a * qc, a, kc);
                kqp = fmaf(kc, qc, kqp);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) kqp += __shfl_xor_sync(0xffffffffu, kqp, o);
            if (l == 0) bkq[tt] = kqp;
        }
        __syncthreads();
    }
    const Tin* sq = direct ? q + tok * DK : nullptr;
    const Tin* sk = direct ? k + tok * DK : nullptr;
    const Tin* sa = direct ? alpha + tok * DK : nullptr;
    const Tin* sv = direct ? v + vb : tin + 3 * NS * DK + ts * DV;
    if constexpr (direct) {
        // fused inputs: alpha and beta are logits, q and k are L2-normalised here
        float ikn = 1.0f, iqn = 1.0f;
        if constexpr (fused) {
            float pk = 0.0f, pq = 0.0f;
            if (tid < DK) {
                const float kv = to_f32(sk[tid]), qv = to_f32(sq[tid]);
                pk = kv * kv;
                pq = qv * qv;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                pk += __shfl_xor_sync(0xffffffffu, pk, o);
                pq += __shfl_xor_sync(0xffffffffu, pq, o);
            }
            if ((tid & 31) == 0) { nk_part[tid >> 5] = pk; nq_part[tid >> 5] = pq; }
            __syncthreads();
            float sk2 = 0.0f, sq2 = 0.0f;
#pragma unroll
            for (int i = 0; i < NT / 32; ++i) { sk2 += nk_part[i]; sq2 += nq_part[i]; }
            ikn = rsqrtf(fmaxf(sk2, 1e-12f));
            iqn = rsqrtf(fmaxf(sq2, 1e-12f));
        }
        float kqp = 0.0f;
        if (tid < DK) {
            const float ax = to_f32(sa[tid]);
            const float a = clamp_gate(fused ? gate_from_logit(ax) : ax);
            const float kv = to_f32(sk[tid]) * ikn, qv = to_f32(sq[tid]) * iqn;
            ga[tid] = a;
            ka[tid] = a * kv;
            qa[tid] = a * qv;
            kk[tid] = kv;
            kqp = kv * qv;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) kqp += __shfl_xor_sync(0xffffffffu, kqp, o);
        if ((tid & 31) == 0) kq_part[tid >> 5] = kqp;
        __syncthreads();
    }

    float4 px = make_float4(0.f, 0.f, 0.f, 0.f), py = px;
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int c = ty + TY * i;
        float wk, wq;
        if constexpr (direct) {
            wk = ka[c];
            wq = qa[c];
        } else {
            const float4 cf = bcf[ts][c];
            wk = cf.x;
            wq = cf.y;
        }
        px.x = fmaf(s[i].x, wk, px.x); px.y = fmaf(s[i].y, wk, px.y);
        px.z = fmaf(s[i].z, wk, px.z); px.w = fmaf(s[i].w, wk, px.w);
        py.x = fmaf(s[i].x, wq, py.x); py.y = fmaf(s[i].y, wq, py.y);
        py.z = fmaf(s[i].z, wq, py.z); py.w = fmaf(s[i].w, wq, py.w);
    }
    *reinterpret_cast<float4*>(&red_x[ty][4 * tx]) = px;
    *reinterpret_cast<float4*>(&red_y[ty][4 * tx]) = py;
    __syncthreads();

    if (tid < DV) {
        float x = 0.0f, y = 0.0f;
#pragma unroll
        for (int i = 0; i < TY; ++i) { x += red_x[i][tid]; y += red_y[i][tid]; }
        float kq = 0.0f;
        if constexpr (direct) {
#pragma unroll
            for (int i = 0; i < NT / 32; ++i) kq += kq_part[i];
        } else {
            kq = bkq[ts];
        }
        const float bx = to_f32(direct ? beta[tok] : tbeta[ts]);
        const float b = fused ? sigmoid_f(bx) : bx;
        const float u = b * (to_f32(sv[tid]) - x);
        us[tid] = u;
        out[vb + tid] = from_f32<Tout>(fmaf(u, kq, y));
    }
    __syncthreads();

    const float4 u4 = *reinterpret_cast<const float4*>(&us[4 * tx]);
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int c = ty + TY * i;
        float a, kc;
        if constexpr (direct) {
            a = ga[c];
            kc = kk[c];
        } else {
            const float4 cf = bcf[ts][c];
            a = cf.z;
            kc = cf.w;
        }
        float4 r;
        r.x = fmaf(a, s[i].x, kc * u4.x);
        r.y = fmaf(a, s[i].y, kc * u4.y);
        r.z = fmaf(a, s[i].z, kc * u4.z);
        r.w = fmaf(a, s[i].w, kc * u4.w);
        s[i] = r;
    }
    }
    if (slot_ok) {
#pragma unroll
        for (int i = 0; i < RPT; ++i) Sv[(size_t)(ty + TY * i) * TX + tx] = s[i];
    }
}

template <typename Tin, typename Tout, int DK, int DV>
static cudaError_t launch_decode_t(const void* q, const void* k, const void* v, const void* alpha,
                                   const void* beta, float* S, void* out, int64_t NH,
                                   cudaStream_t stream, const int32_t* slots, int num_slots, int H,
                                   int T, int fused) {
#define KDA_DECODE_LAUNCH(F, M)                                                                   \
    kda_decode_kernel<Tin, Tout, DK, DV, F, M><<<(unsigned)NH, 256, 0, stream>>>(                 \
        (const Tin*)q, (const Tin*)k, (const Tin*)v, (const Tin*)alpha, (const Tin*)beta, S,      \
        (Tout*)out, slots, num_slots, H, T)
    if (T > 1) {
        if (fused) KDA_DECODE_LAUNCH(true, true);
        else KDA_DECODE_LAUNCH(false, true);
    } else {
        if (fused) KDA_DECODE_LAUNCH(true, false);
        else KDA_DECODE_LAUNCH(false, false);
    }
#undef KDA_DECODE_LAUNCH
    return cudaGetLastError();
}

template <typename Tin, typename Tout>
static cudaError_t launch_decode_d(int DK, int DV, const void* q, const void* k, const void* v,
                                   const void* alpha, const void* beta, float* S, void* out,
                                   int64_t NH, cudaStream_t s, const int32_t* slots, int num_slots,
                                   int H, int T, int fused) {
    if (DK == 64 && DV == 64) return launch_decode_t<Tin, Tout, 64, 64>(q, k, v, alpha, beta, S, out, NH, s, slots, num_slots, H, T, fused);
    if (DK == 64 && DV == 128) return launch_decode_t<Tin, Tout, 64, 128>(q, k, v, alpha, beta, S, out, NH, s, slots, num_slots, H, T, fused);
    if (DK == 128 && DV == 64) return launch_decode_t<Tin, Tout, 128, 64>(q, k, v, alpha, beta, S, out, NH, s, slots, num_slots, H, T, fused);
    return launch_decode_t<Tin, Tout, 128, 128>(q, k, v, alpha, beta, S, out, NH, s, slots, num_slots, H, T, fused);
}

cudaError_t launch_decode(int in_bf16, int out_bf16, const void* q, const void* k, const void* v,
                          const void* alpha, const void* beta, float* S, void* out, int64_t NH,
                          int DK, int DV, cudaStream_t s, const int32_t* slots, int num_slots,
                          int H, int T, int fused) {
    if (!in_bf16 && !out_bf16) return launch_decode_d<float, float>(DK, DV, q, k, v, alpha, beta, S, out, NH, s, slots, num_slots, H, T, fused);
    if (!in_bf16 && out_bf16) return launch_decode_d<float, __nv_bfloat16>(DK, DV, q, k, v, alpha, beta, S, out, NH, s, slots, num_slots, H, T, fused);
    if (in_bf16 && !out_bf16) return launch_decode_d<__nv_bfloat16, float>(DK, DV, q, k, v, alpha, beta, S, out, NH, s, slots, num_slots, H, T, fused);
    return launch_decode_d<__nv_bfloat16, __nv_bfloat16>(DK, DV, q, k, v, alpha, beta, S, out, NH, s, slots, num_slots, H, T, fused);
}

}  // namespace kda
