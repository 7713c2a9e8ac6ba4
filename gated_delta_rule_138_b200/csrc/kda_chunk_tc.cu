// KDA chunked forward on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
// bf16 q, k, v, alpha, beta; fp32 state; d_k = d_v = 128; chunk C = 64.
//
// The worldcybernews article "Kimi K3 Open Model Surpasses Closed GPT and
// Anthropic Systems on Independent Benchmarks": paragraph 2 gives the state
// S (d_k x d_v), the delta-rule update with write strength beta and forget
// gate alpha in [e^-5, 1]; paragraph 3 processes the tokens of a chunk in
// parallel and carries the sequential state across chunks.  Per chunk, with
// start state S and a = clamp(alpha):
//
//   A[r,j] = beta_r sum_c k_rc k_jc D(r,j)_c  (j < r),  P[r,j] = sum_c q_rc k_jc D(r,j)_c  (j <= r)
//   D(r,j) = prod_{s=j+1..r} a_s,   Tinv = (I + A)^-1,   Tb = Tinv diag(beta)
//   [-W ; Q'] = [0 ; q*gamma] - [Tb ; P Tb] (k*gamma)          (gamma_r = prod_{s<=r} a_s)
//   [ U ; O ] = [-W ; Q'] S + [Tb ; P Tb] V
//   S        <- Diag(gamma_C) S + (k*eta)^T U                   (eta_j = prod_{s>j} a_s)
//
// D(r,j) is split at 16-token sub-chunk boundaries so that every factor stays
// inside the fp32/bf16 exponent range (a product of 64 gates >= e^-5 can reach
// e^-320, but a 16-token product stays >= e^-80):
//   phi_r = prod_{s=start(I)..r} a_s,  psi_j = prod_{s=j+1..end(J)} a_s,
//   pi_I = prod over sub-chunk I,      Dp_{I,J} = prod_{J<M<I} pi_M (I > J), 1/pi_I (I = J)
//   D(r, j) = (phi_r) (psi_j Dp_{I(r),J(j)})
// so the 16-row block I of [A/beta | P] is  [k phi ; q phi]_I  times  R^(I)^T with
// R^(I)_j = k_j psi_j Dp_{I,J(j)} for j < end(I): one M=64 tcgen05 MMA per I.
//
// One CTA (256 threads) owns one (sequence, head) and walks its chunks in
// order.  Thread 0 issues the TMA loads and the MMAs; all eight warps do the
// element-wise work.  TMEM (512 columns): S fp32 [0,128), U|O accumulator
// [128,256), scratch accumulators [256,384).
#include <cuda.h>

#include "kda_common.cuh"
#include "kda_sm100.cuh"

// Optional phase-boundary hook for profiling builds (no-op in the library).
#ifndef KDA_TC_PHASE
#define KDA_TC_PHASE(i)
#endif

namespace kda {
using namespace sm100;

namespace tc {

constexpr int C = 64;         // tokens per chunk
constexpr int DK = 128;       // key channels
constexpr int DV = 128;       // value channels
constexpr int NT = 256;       // threads
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s per wait, then report a timeout

// shared-memory map (bytes from the 1024-aligned base)
constexpr uint32_t OFF_Q = 0;            // q tile [64][128] sw128, becomes q*gamma in place
constexpr uint32_t OFF_K = 16384;        // k tile
constexpr uint32_t OFF_AL = 32768;       // alpha tile, becomes [Tb ; P Tb] (K-major [128][64])
constexpr uint32_t OFF_V = 49152;        // v tile: MN-major B, two 64-column atoms of [64][64]
constexpr uint32_t OFF_X = 65536;        // 72 KB work region, see below
constexpr uint32_t OFF_KT = OFF_X + 73728;   // (k*gamma)^T  K-major B [128 c][64 j]
constexpr uint32_t OFF_KH = OFF_KT + 16384;  // (k*eta)^T    K-major A [128 c][64 j]
constexpr uint32_t OFF_IP = OFF_KH + 16384;  // [I ; P]      K-major A [128][64]
constexpr uint32_t OFF_S = OFF_IP + 16384;   // S bf16       MN-major B [128 c][128 n], two atoms
constexpr uint32_t OFF_MISC = OFF_S + 32768;
constexpr uint32_t MISC_PI = 0;          // float [4][128]
constexpr uint32_t MISC_GC = 2048;       // float [128] gamma_C
constexpr uint32_t MISC_BETA = 2560;     // float [64]
constexpr uint32_t MISC_BAR = 2816;      // 2 x uint64 mbarriers
constexpr uint32_t MISC_TMEM = 2832;     // uint32 TMEM base
constexpr uint32_t MISC_FLAG = 2836;     // int timeout seen
constexpr uint32_t SMEM_BYTES = OFF_MISC + 2848 + 1024;  // + alignment slack

// work region X, by phase
constexpr uint32_t X_R = 0;              // R rows [160][128] sw128 (2 atoms of 160 rows)
constexpr uint32_t X_L = 40960;          // L rows [128][128] sw128 (2 atoms of 128 rows)
constexpr uint32_t X_AM = 0;             // float A [64][65]
constexpr uint32_t X_PM = 16640;         // float P [64][65]
constexpr uint32_t X_TM = 33280;         // float Tinv [64][65]
constexpr uint32_t X_TB = 50176;         // Tb MN-major B [64 j][64 m]
constexpr uint32_t X_SCR = 58368;        // float scratch 3 x [16][16]
constexpr uint32_t X_WQ = 0;             // [-W ; Q'] K-major A [128][128] (2 atoms)
constexpr uint32_t X_U = 32768;          // U MN-major B [64 j][128 n] (2 atoms of [64][64])

constexpr uint32_t TM_S = 0, TM_UO = 128, TM_WK = 256;

// row offsets of R^(I) in the R buffer; the M=64 window of R^(I) starts there
__device__ __constant__ int kROff[4] = {0, 16, 48, 96};

__device__ __forceinline__ uint32_t swz(uint32_t row, uint32_t chunk) {
    return row * 128u + (((chunk ^ row) & 7u) << 4);
}
// byte offset of the bf16 pair (row, c..c+1), c even, in a tile with `rows`
// rows per 64-column atom
__device__ __forceinline__ uint32_t pair_off(uint32_t row, uint32_t c, uint32_t rows) {
    return (c >> 6) * rows * 128u + swz(row, (c & 63u) >> 3) + ((c & 7u) << 1);
}
__device__ __forceinline__ float2 ld_bf2(const uint8_t* p) {
    const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(p);
    return __bfloat1622float2(v);
}
__device__ __forceinline__ void st_bf2(uint8_t* p, float a, float b) {
    *reinterpret_cast<uint32_t*>(p) = pack_bf16x2(a, b);
}

// M=64 accumulator: row m lives in TMEM lane 32*(m/16) + m%16
// M=128 accumulator: row m lives in lane m.

// kCtaStatus = false: a timed-out wait sets the shared word *status to 1.
// kCtaStatus = true:  every CTA writes its own word status[n * H + h] (0 or 1).
template <bool kCtaStatus>
__global__ void __launch_bounds__(NT, 1)
kda_chunk_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmV,
                    const __nv_bfloat16* __restrict__ beta, const float* S0,
                    const int32_t* __restrict__ cu_seqlens, __nv_bfloat16* __restrict__ out,
                    float* S_final, int64_t T, int H, int* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    uint8_t* sQ = sm + OFF_Q;
    uint8_t* sK = sm + OFF_K;
    uint8_t* sAl = sm + OFF_AL;
    uint8_t* sV = sm + OFF_V;
    uint8_t* sX = sm + OFF_X;
    uint8_t* sKT = sm + OFF_KT;
    uint8_t* sKH = sm + OFF_KH;
    uint8_t* sIP = sm + OFF_IP;
    uint8_t* sS = sm + OFF_S;
    float* sPi = reinterpret_cast<float*>(sm + OFF_MISC + MISC_PI);
    float* sGC = reinterpret_cast<float*>(sm + OFF_MISC + MISC_GC);
    float* sBeta = reinterpret_cast<float*>(sm + OFF_MISC + MISC_BETA);
    uint64_t* barT = reinterpret_cast<uint64_t*>(sm + OFF_MISC + MISC_BAR);
    uint64_t* barM = barT + 1;
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + OFF_MISC + MISC_TMEM);
    int* sFlag = reinterpret_cast<int*>(sm + OFF_MISC + MISC_FLAG);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q4 = warp & 3;            // TMEM lane quarter this warp may touch
    const int hf = warp >> 2;           // which half of the columns this warp handles
    const int h = blockIdx.y, n = blockIdx.z;
    int64_t bos, len;
    seq_range(cu_seqlens, n, T, bos, len);
    const int nchunks = (int)((len + C - 1) / C);

    if (tid == 0) {
        mbar_init(barT, 1);
        mbar_init(barM, 1);
        mbar_fence_init();
        *sFlag = 0;
    }
    if (warp == 0) tmem_alloc(sTmem, 512);
    // identity rows of [I ; P]
    for (int i = tid; i < 64 * 8; i += NT) {
        const int r = i >> 3, ch = i & 7;
        uint32_t w[4] = {0, 0, 0, 0};
        if ((r >> 3) == ch) {
            const int e = r & 7;  // element within the 8-wide chunk
            w[e >> 1] = (e & 1) ? 0x3F800000u : 0x00003F80u;  // bf16 1.0 in the hi/lo half
        }
        *reinterpret_cast<uint4*>(sIP + swz(r, ch)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *sTmem;
    const uint32_t tlane = (uint32_t)(32 * q4) << 16;

    // ---- initial state: TMEM S (fp32) and its bf16 copy (MN-major B operand)
    {
        const int c = 32 * q4 + lane;
        const float* src = S0 ? S0 + (((size_t)n * H + h) * DK + c) * DV + 64 * hf : nullptr;
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; i += 4) {
                float4 f = src ? *reinterpret_cast<const float4*>(src + 16 * blk + i)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
                v[i] = f.x; v[i + 1] = f.y; v[i + 2] = f.z; v[i + 3] = f.w;
            }
            tmem_st16(tmem + tlane + TM_S + 64 * hf + 16 * blk, v);
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint4 w;
                w.x = pack_bf16x2(v[8 * ch + 0], v[8 * ch + 1]);
                w.y = pack_bf16x2(v[8 * ch + 2], v[8 * ch + 3]);
                w.z = pack_bf16x2(v[8 * ch + 4], v[8 * ch + 5]);
                w.w = pack_bf16x2(v[8 * ch + 6], v[8 * ch + 7]);
                *reinterpret_cast<uint4*>(sS + hf * 16384 + swz(c, 2 * blk + ch)) = w;
            }
        }
        tmem_wait_st();
    }

    auto issue_tma = [&](int64_t row0) {
        mbar_arrive_expect_tx(barT, 4 * 16384);
        const int y = (int)row0;
#pragma unroll
        for (int a = 0; a < 2; ++a) {
            const int x = h * DK + 64 * a;
            tma_load_2d(sQ + a * 8192, &tmQ, barT, x, y);
            tma_load_2d(sK + a * 8192, &tmK, barT, x, y);
            tma_load_2d(sAl + a * 8192, &tmA, barT, x, y);
            tma_load_2d(sV + a * 8192, &tmV, barT, h * DV + 64 * a, y);
        }
    };
    if (tid == 0 && nchunks > 0) issue_tma(bos);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    uint32_t phT = 0, phM = 0;
    bool ok = true;   // this thread has seen every wait complete
    auto wait_mma = [&]() {
        if (ok && !mbar_wait_ns(barM, phM, kWaitNs)) ok = false;
        phM ^= 1u;
        tc_fence_after();
    };

    for (int chunk = 0; chunk < nchunks; ++chunk) {
        const int64_t row0 = bos + (int64_t)chunk * C;
        const int Lc = (int)((len - (int64_t)chunk * C) < C ? (len - (int64_t)chunk * C) : C);
        if (tid < C)
            sBeta[tid] = tid < Lc ? __bfloat162float(beta[(size_t)(row0 + tid) * H + h]) : 0.0f;
        if (ok && !mbar_wait_ns(barT, phT, kWaitNs)) ok = false;
        phT ^= 1u;
        KDA_TC_PHASE(0);

        // ================= gate products and bf16 operands (all threads)
        {
            const int cp = tid & 63, I = tid >> 6, c0 = 2 * cp;
            float phi0[16], phi1[16], psi0[16], psi1[16];
            {
                float a0[16], a1[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int r = 16 * I + i;
                    float2 al = ld_bf2(sAl + pair_off(r, c0, 64));
                    a0[i] = r < Lc ? clamp_gate(al.x) : 1.0f;
                    a1[i] = r < Lc ? clamp_gate(al.y) : 1.0f;
                }
                float p0 = 1.f, p1 = 1.f;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    p0 *= a0[i]; p1 *= a1[i];
                    phi0[i] = p0; phi1[i] = p1;
                }
                float s0 = 1.f, s1 = 1.f;
#pragma unroll
                for (int i = 15; i >= 0; --i) {
                    psi0[i] = s0; psi1[i] = s1;
                    s0 *= a0[i]; s1 *= a1[i];
                }
                sPi[I * DK + c0] = p0;
                sPi[I * DK + c0 + 1] = p1;
            }
            __syncthreads();
            float pi0[4], pi1[4];
#pragma unroll
            for (int M = 0; M < 4; ++M) { pi0[M] = sPi[M * DK + c0]; pi1[M] = sPi[M * DK + c0 + 1]; }
            float bef0 = 1.f, bef1 = 1.f, aft0 = 1.f, aft1 = 1.f;
#pragma unroll
            for (int M = 0; M < 4; ++M) {
                if (M < I) { bef0 *= pi0[M]; bef1 *= pi1[M]; }
                if (M > I) { aft0 *= pi0[M]; aft1 *= pi1[M]; }
            }
            if (I == 0) {
                sGC[c0] = pi0[0] * pi0[1] * pi0[2] * pi0[3];
                sGC[c0 + 1] = pi1[0] * pi1[1] * pi1[2] * pi1[3];
            }
            // Dp_{I', I} for I' >= I
            float dp0[4], dp1[4];
#pragma unroll
            for (int Ip = 0; Ip < 4; ++Ip) {
                float x0 = 1.f, x1 = 1.f;
#pragma unroll
                for (int M = 0; M < 4; ++M)
                    if (M > I && M < Ip) { x0 *= pi0[M]; x1 *= pi1[M]; }
                if (Ip == I) { x0 = 1.0f / pi0[I]; x1 = 1.0f / pi1[I]; }
                dp0[Ip] = x0; dp1[Ip] = x1;
            }
            uint8_t* sR = sX + X_R;
            uint8_t* sL = sX + X_L;
            float kt0[16], kt1[16], kh0[16], kh1[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = 16 * I + i;
                float2 kk = ld_bf2(sK + pair_off(r, c0, 64));
                float2 qq = ld_bf2(sQ + pair_off(r, c0, 64));
                if (r >= Lc) { kk = make_float2(0.f, 0.f); qq = kk; }
                const float kp0 = kk.x * phi0[i], kp1 = kk.y * phi1[i];
                const float qp0 = qq.x * phi0[i], qp1 = qq.y * phi1[i];
                const float ks0 = kk.x * psi0[i], ks1 = kk.y * psi1[i];
                st_bf2(sL + pair_off(32 * I + i, c0, 128), kp0, kp1);
                st_bf2(sL + pair_off(32 * I + 16 + i, c0, 128), qp0, qp1);
#pragma unroll
                for (int Ip = 0; Ip < 4; ++Ip)
                    if (Ip >= I) st_bf2(sR + pair_off(kROff[Ip] + r, c0, 160), ks0 * dp0[Ip], ks1 * dp1[Ip]);
                st_bf2(sQ + pair_off(r, c0, 64), qp0 * bef0, qp1 * bef1);   // q*gamma in place
                kt0[i] = kp0 * bef0; kt1[i] = kp1 * bef1;                    // k*gamma
                kh0[i] = ks0 * aft0; kh1[i] = ks1 * aft1;                    // k*eta
            }
            // transposed tiles [c][j]: tokens 16I..16I+15 are chunks 2I, 2I+1 of rows c0, c0+1
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int ch = 2 * I + half;
                const int b = 8 * half;
                uint4 w;
                w = make_uint4(pack_bf16x2(kt0[b], kt0[b + 1]), pack_bf16x2(kt0[b + 2], kt0[b + 3]),
                               pack_bf16x2(kt0[b + 4], kt0[b + 5]), pack_bf16x2(kt0[b + 6], kt0[b + 7]));
                *reinterpret_cast<uint4*>(sKT + swz(c0, ch)) = w;
                w = make_uint4(pack_bf16x2(kt1[b], kt1[b + 1]), pack_bf16x2(kt1[b + 2], kt1[b + 3]),
                               pack_bf16x2(kt1[b + 4], kt1[b + 5]), pack_bf16x2(kt1[b + 6], kt1[b + 7]));
                *reinterpret_cast<uint4*>(sKT + swz(c0 + 1, ch)) = w;
                w = make_uint4(pack_bf16x2(kh0[b], kh0[b + 1]), pack_bf16x2(kh0[b + 2], kh0[b + 3]),
                               pack_bf16x2(kh0[b + 4], kh0[b + 5]), pack_bf16x2(kh0[b + 6], kh0[b + 7]));
                *reinterpret_cast<uint4*>(sKH + swz(c0, ch)) = w;
                w = make_uint4(pack_bf16x2(kh1[b], kh1[b + 1]), pack_bf16x2(kh1[b + 2], kh1[b + 3]),
                               pack_bf16x2(kh1[b + 4], kh1[b + 5]), pack_bf16x2(kh1[b + 6], kh1[b + 7]));
                *reinterpret_cast<uint4*>(sKH + swz(c0 + 1, ch)) = w;
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        KDA_TC_PHASE(1);
        // ================= [A/beta | P] row blocks: four M=64, N=32 MMAs
        if (tid == 0) {
            const uint32_t r0 = smem_u32(sX + X_R), l0 = smem_u32(sX + X_L);
            constexpr uint32_t idesc = idesc_bf16(64, 32);
#pragma unroll
            for (int I = 0; I < 4; ++I) {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t atom = ks >> 2, within = (ks & 3) * 32;
                    const uint32_t a = r0 + atom * (160 * 128) + kROff[I] * 128 + within;
                    const uint32_t b = l0 + atom * (128 * 128) + (32 * I) * 128 + within;
                    mma_bf16(tmem + TM_WK + 32 * I, sdesc_sw128(a), sdesc_sw128(b), idesc, ks > 0);
                }
            }
            mma_commit(barM);
        }
        wait_mma();

        KDA_TC_PHASE(2);
        // ================= A and P to fp32 shared memory (masked), P to the [I ; P] operand
        {
            float* Am = reinterpret_cast<float*>(sX + X_AM);
            float* Pm = reinterpret_cast<float*>(sX + X_PM);
            const int j = 16 * q4 + (lane & 15);   // key token of this lane (lanes 0-15)
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const int I = 2 * hf + t;
                float va[16], vp[16];
                tmem_ld16(tmem + tlane + TM_WK + 32 * I, va);
                tmem_ld16(tmem + tlane + TM_WK + 32 * I + 16, vp);
                tmem_wait_ld();
                if (lane < 16) {
#pragma unroll
                    for (int rr = 0; rr < 16; ++rr) {
                        const int r = 16 * I + rr;
                        Am[r * 65 + j] = (j < r) ? sBeta[r] * va[rr] : 0.0f;
                        const float p = (j <= r) ? vp[rr] : 0.0f;
                        Pm[r * 65 + j] = p;
                        *reinterpret_cast<__nv_bfloat16*>(sIP + swz(64 + r, j >> 3) + ((j & 7) << 1)) =
                            __float2bfloat16_rn(p);
                    }
                }
            }
        }
        tc_fence_before();
        __syncthreads();

        KDA_TC_PHASE(3);
        // ================= Tinv = (I + A)^-1: diagonal 16x16 blocks by forward substitution
        {
            const float* Am = reinterpret_cast<const float*>(sX + X_AM);
            float* Tm = reinterpret_cast<float*>(sX + X_TM);
            if (tid < 64) {
                const int I = tid >> 4, m = tid & 15, o = 16 * I;
                float col[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    float s = 0.0f;
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj)
                        if (jj < r) s = fmaf(Am[(o + r) * 65 + o + jj], col[jj], s);
                    col[r] = r < m ? 0.0f : (r == m ? 1.0f : -s);
                    Tm[(o + r) * 65 + o + m] = col[r];
                }
            }
            __syncthreads();
            // off-diagonal blocks, by distance d = I - J
            float* scr = reinterpret_cast<float*>(sX + X_SCR);
#pragma unroll 1
            for (int d = 1; d < 4; ++d) {
                const int nblk = 4 - d;
                for (int e = tid; e < nblk * 256; e += NT) {
                    const int J = e >> 8, I = J + d, r = (e >> 4) & 15, m = e & 15;
                    float s = 0.0f;
                    for (int M = J; M < I; ++M)
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj)
                            s = fmaf(Am[(16 * I + r) * 65 + 16 * M + jj], Tm[(16 * M + jj) * 65 + 16 * J + m], s);
                    scr[e] = s;
                }
                __syncthreads();
                for (int e = tid; e < nblk * 256; e += NT) {
                    const int J = e >> 8, I = J + d, r = (e >> 4) & 15, m = e & 15;
                    float s = 0.0f;
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj)
                        if (jj <= r) s = fmaf(Tm[(16 * I + r) * 65 + 16 * I + jj], scr[(J << 8) + jj * 16 + m], s);
                    Tm[(16 * I + r) * 65 + 16 * J + m] = -s;
                }
                __syncthreads();
            }
            // Tb = Tinv diag(beta) as MN-major B: row j, column m; zero above the diagonal
            uint8_t* sTB = sX + X_TB;
            for (int e = tid; e < 64 * 8; e += NT) {
                const int jr = e >> 3, ch = e & 7;
                float v[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int m = 8 * ch + i;
                    v[i] = (jr >= m) ? Tm[jr * 65 + m] * sBeta[m] : 0.0f;
                }
                *reinterpret_cast<uint4*>(sTB + swz(jr, ch)) =
                    make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                               pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        KDA_TC_PHASE(4);
        // ================= [Tb ; P Tb] = [I ; P] Tb   (M=128, N=64, K=64)
        if (tid == 0) {
            const uint32_t a0 = smem_u32(sIP), b0 = smem_u32(sX + X_TB);
            constexpr uint32_t idesc = idesc_bf16(128, 64, false, true);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tmem + TM_WK, sdesc_sw128(a0 + ks * 32), sdesc_sw128(b0 + ks * 2048), idesc,
                         ks > 0);
            mma_commit(barM);
        }
        wait_mma();
        {
            const int row = 32 * q4 + lane;
#pragma unroll
            for (int blk = 0; blk < 2; ++blk) {
                float v[16];
                tmem_ld16(tmem + tlane + TM_WK + 32 * hf + 16 * blk, v);
                tmem_wait_ld();
#pragma unroll
                for (int ch = 0; ch < 2; ++ch)
                    *reinterpret_cast<uint4*>(sAl + swz(row, 4 * hf + 2 * blk + ch)) =
                        make_uint4(pack_bf16x2(v[8 * ch], v[8 * ch + 1]), pack_bf16x2(v[8 * ch + 2], v[8 * ch + 3]),
                                   pack_bf16x2(v[8 * ch + 4], v[8 * ch + 5]), pack_bf16x2(v[8 * ch + 6], v[8 * ch + 7]));
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        KDA_TC_PHASE(5);
        // ================= [W ; P W] = [Tb ; P Tb] (k*gamma)   (M=128, N=128, K=64)
        if (tid == 0) {
            const uint32_t a0 = smem_u32(sAl), b0 = smem_u32(sKT);
            constexpr uint32_t idesc = idesc_bf16(128, 128);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tmem + TM_WK, sdesc_sw128(a0 + ks * 32), sdesc_sw128(b0 + ks * 32), idesc, ks > 0);
            mma_commit(barM);
        }
        wait_mma();
        {
            // [-W ; q*gamma - P W] as the K-major A operand of the state MMA
            const int row = 32 * q4 + lane;
            uint8_t* sWQ = sX + X_WQ;
#pragma unroll
            for (int blk = 0; blk < 4; ++blk) {
                float v[16];
                tmem_ld16(tmem + tlane + TM_WK + 64 * hf + 16 * blk, v);
                tmem_wait_ld();
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) {
                    const int chunk = 2 * blk + ch;           // 8-column chunk within the atom
                    float w8[8];
                    if (row < 64) {
#pragma unroll
                        for (int i = 0; i < 8; ++i) w8[i] = -v[8 * ch + i];
                    } else {
                        const uint4 qg = *reinterpret_cast<const uint4*>(
                            sQ + hf * 8192 + swz(row - 64, chunk));
                        const uint32_t qw[4] = {qg.x, qg.y, qg.z, qg.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qw[i]));
                            w8[2 * i] = f.x - v[8 * ch + 2 * i];
                            w8[2 * i + 1] = f.y - v[8 * ch + 2 * i + 1];
                        }
                    }
                    *reinterpret_cast<uint4*>(sWQ + hf * 16384 + swz(row, chunk)) =
                        make_uint4(pack_bf16x2(w8[0], w8[1]), pack_bf16x2(w8[2], w8[3]),
                                   pack_bf16x2(w8[4], w8[5]), pack_bf16x2(w8[6], w8[7]));
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        KDA_TC_PHASE(6);
        // ================= [U ; O] = [-W ; Q'] S + [Tb ; P Tb] V   (two N=64 halves, K=128+64)
        if (tid == 0) {
            const uint32_t wq = smem_u32(sX + X_WQ), s0 = smem_u32(sS), tb = smem_u32(sAl),
                           v0 = smem_u32(sV);
            constexpr uint32_t idesc = idesc_bf16(128, 64, false, true);
#pragma unroll
            for (int nh = 0; nh < 2; ++nh) {
                const uint32_t d = tmem + TM_UO + 64 * nh;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16(d, sdesc_sw128(wq + (ks >> 2) * 16384 + (ks & 3) * 32),
                             sdesc_sw128(s0 + nh * 16384 + ks * 2048), idesc, ks > 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(d, sdesc_sw128(tb + ks * 32), sdesc_sw128(v0 + nh * 8192 + ks * 2048), idesc, 1);
            }
            mma_commit(barM);
        }
        // meanwhile: S <- Diag(gamma_C) S in TMEM (the MMA reads the bf16 copy)
        {
            const int c = 32 * q4 + lane;
            const float g = sGC[c];
#pragma unroll
            for (int blk = 0; blk < 4; ++blk) {
                float v[16];
                const uint32_t ta = tmem + tlane + TM_S + 64 * hf + 16 * blk;
                tmem_ld16(ta, v);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] *= g;
                tmem_st16(ta, v);
            }
            tmem_wait_st();
        }
        wait_mma();
        // all of q, k, alpha, v are consumed: prefetch the next chunk
        if (tid == 0 && chunk + 1 < nchunks) issue_tma(row0 + C);
        {
            const int row = 32 * q4 + lane;
            uint8_t* sU = sX + X_U;
#pragma unroll
            for (int blk = 0; blk < 4; ++blk) {
                float v[16];
                tmem_ld16(tmem + tlane + TM_UO + 64 * hf + 16 * blk, v);
                tmem_wait_ld();
                uint4 w[2];
#pragma unroll
                for (int ch = 0; ch < 2; ++ch)
                    w[ch] = make_uint4(pack_bf16x2(v[8 * ch], v[8 * ch + 1]), pack_bf16x2(v[8 * ch + 2], v[8 * ch + 3]),
                                       pack_bf16x2(v[8 * ch + 4], v[8 * ch + 5]), pack_bf16x2(v[8 * ch + 6], v[8 * ch + 7]));
                if (row < 64) {
#pragma unroll
                    for (int ch = 0; ch < 2; ++ch)
                        *reinterpret_cast<uint4*>(sU + hf * 8192 + swz(row, 2 * blk + ch)) = w[ch];
                } else if (row - 64 < Lc) {
                    __nv_bfloat16* dst = out + ((size_t)(row0 + row - 64) * H + h) * DV + 64 * hf + 16 * blk;
                    reinterpret_cast<uint4*>(dst)[0] = w[0];
                    reinterpret_cast<uint4*>(dst)[1] = w[1];
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        KDA_TC_PHASE(7);
        // ================= S += (k*eta)^T U   (M=128, two N=64 halves, K=64)
        if (tid == 0) {
            const uint32_t a0 = smem_u32(sKH), u0 = smem_u32(sX + X_U);
            constexpr uint32_t idesc = idesc_bf16(128, 64, false, true);
#pragma unroll
            for (int nh = 0; nh < 2; ++nh)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + TM_S + 64 * nh, sdesc_sw128(a0 + ks * 32),
                             sdesc_sw128(u0 + nh * 8192 + ks * 2048), idesc, 1);
            mma_commit(barM);
        }
        wait_mma();
        {
            const int c = 32 * q4 + lane;
#pragma unroll
            for (int blk = 0; blk < 4; ++blk) {
                float v[16];
                tmem_ld16(tmem + tlane + TM_S + 64 * hf + 16 * blk, v);
                tmem_wait_ld();
#pragma unroll
                for (int ch = 0; ch < 2; ++ch)
                    *reinterpret_cast<uint4*>(sS + hf * 16384 + swz(c, 2 * blk + ch)) =
                        make_uint4(pack_bf16x2(v[8 * ch], v[8 * ch + 1]), pack_bf16x2(v[8 * ch + 2], v[8 * ch + 3]),
                                   pack_bf16x2(v[8 * ch + 4], v[8 * ch + 5]), pack_bf16x2(v[8 * ch + 6], v[8 * ch + 7]));
            }
        }
        fence_async_smem();
        tc_fence_before();
        const int any_timeout = __syncthreads_or(!ok);   // uniform: every thread leaves together
        tc_fence_after();
        KDA_TC_PHASE(8);
        if (any_timeout) break;
    }

    if (!ok) atomicExch(sFlag, 1);
    __syncthreads();
    if (kCtaStatus && tid == 0) status[(size_t)n * H + h] = *sFlag;
    if (*sFlag) {
        if (!kCtaStatus && tid == 0) atomicExch(status, 1);
    } else if (S_final) {
        const int c = 32 * q4 + lane;
        float* dst = S_final + (((size_t)n * H + h) * DK + c) * DV + 64 * hf;
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
            float v[16];
            tmem_ld16(tmem + tlane + TM_S + 64 * hf + 16 * blk, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; i += 4)
                *reinterpret_cast<float4*>(dst + 16 * blk + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// [rows, H*128] bf16, box 64 x 64, 128-byte swizzle
static bool make_map(CUtensorMap* m, const void* base, int64_t rows, int H) {
    EncodeTiledFn enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)H * 128, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)H * 128 * 2};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tc

template <bool kCtaStatus>
static cudaError_t launch_tc_t(const void* q, const void* k, const void* v, const void* alpha,
                               const void* beta, const float* S0, const int32_t* cu, int nseq,
                               void* out, float* S_final, int64_t rows, int64_t T, int H,
                               int* status, cudaStream_t stream) {
    CUtensorMap mq, mk, ma, mv;
    if (!tc::make_map(&mq, q, rows, H) || !tc::make_map(&mk, k, rows, H) ||
        !tc::make_map(&ma, alpha, rows, H) || !tc::make_map(&mv, v, rows, H))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(tc::kda_chunk_tc_kernel<kCtaStatus>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)tc::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    dim3 grid(1, H, nseq);
    tc::kda_chunk_tc_kernel<kCtaStatus><<<grid, tc::NT, tc::SMEM_BYTES, stream>>>(
        mq, mk, ma, mv, (const __nv_bfloat16*)beta, S0, cu, (__nv_bfloat16*)out, S_final, T, H,
        status);
    return cudaGetLastError();
}

cudaError_t launch_chunk_tc(const void* q, const void* k, const void* v, const void* alpha,
                            const void* beta, const float* S0, const int32_t* cu, int nseq,
                            void* out, float* S_final, int64_t rows, int64_t T, int H, int* status,
                            cudaStream_t stream) {
    return launch_tc_t<false>(q, k, v, alpha, beta, S0, cu, nseq, out, S_final, rows, T, H,
                              status, stream);
}

// Same kernel, one status word per (sequence, head) CTA at status[n * H + h].
cudaError_t launch_chunk_tc_cta_status(const void* q, const void* k, const void* v,
                                       const void* alpha, const void* beta, const float* S0,
                                       const int32_t* cu, int nseq, void* out, float* S_final,
                                       int64_t rows, int64_t T, int H, int* status,
                                       cudaStream_t stream) {
    return launch_tc_t<true>(q, k, v, alpha, beta, S0, cu, nseq, out, S_final, rows, T, H,
                             status, stream);
}

}  // namespace kda
