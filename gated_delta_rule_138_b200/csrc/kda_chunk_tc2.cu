// KDA chunked forward on the sm_100a tensor cores, pipelined: the work of a chunk
// that does not depend on the state runs one chunk ahead of the state chain, on
// its own warps, and the state lives transposed in tensor memory so that every
// state-dependent product takes its A operand from TMEM.
// bf16 q, k, v, alpha, beta; fp32 state; d_k = d_v = 128; chunk C = 64.
//
// The worldcybernews article "Kimi K3 Open Model Surpasses Closed GPT and
// Anthropic Systems on Independent Benchmarks": paragraph 2 gives the state S
// (d_k x d_v), the delta-rule update with write strength beta and forget gate
// alpha in [e^-5, 1]; paragraph 3 processes the tokens of a chunk in parallel
// and carries the sequential state across chunks.  Per chunk, with start state S
// and a = clamp(alpha), D(r, j) = prod_{s=j+1..r} a_s, gamma_r = prod_{s<=r} a_s,
// eta_j = prod_{s>j} a_s:
//
//   A[r,j] = beta_r sum_c k_rc k_jc D(r,j)_c (j < r),  P[r,j] = sum_c q_rc k_jc D(r,j)_c (j <= r)
//   Tb = (I + A)^-1 diag(beta)
//   Z = (k*gamma) S,   U = Tb (V - Z),   O = (q*gamma) S + P U,   S <- Diag(gamma_C) S + (k*eta)^T U
//
// Transposed, with S^T in TMEM (lane n = value column, columns = key channels), and
// with gamma_r = lam_r Gamma_I for the tokens r of 32-token sub-chunk I (lam_r the
// in-sub-chunk factor of the gate phase below, Gamma_I = gamma at the sub-chunk's
// reference token, one value per key channel):
//
//   Z^T[:, I] = (S^T Diag(Gamma_I)) (k*lam)_I^T     M=128 (n), N=32 (j), K=128 (c)
//   O^T[:, I] = (S^T Diag(Gamma_I)) (q*lam)_I^T     M=128, N=32 (r), K=128
//   U^T = V^T Tb^T - Z^T Tb^T                       M=128, N=64, K=64 (j'); V^T from shared memory
//   S^T <- S^T Diag(gamma_C) + U^T (k*eta)          M=128, N=128 (c), K=64
//   O^T += U^T P^T                                  M=128, N=64, K=64
//
// with every other A operand in TMEM: the two scaled bf16 copies of S^T, Z^T and U^T.
// The chain that carries the state from chunk to chunk moves no operand of its own
// through shared memory; its B operands are the chunk's state-independent products,
// prepared one chunk ahead: k*lam and q*lam (also the left operands of [A/beta ; P],
// written over k and q), Tb, P and k*eta = (k*rho^1) Diag(gamma_C / Gamma_1) (written
// over alpha as k*rho^1, the right operand of [A/beta ; P], then rescaled).
//
// Warp roles (512 threads = four warpgroups, one CTA per SM):
//   warps 0-7   prep: gate products, the bf16 operands, [A/beta ; P] (one tcgen05
//               MMA), the triangular solve, Tb, k*eta; one of its threads issues its
//               MMAs.  Works on chunk c+1 while the state chain runs chunk c.
//   warps 8-11  the state chain, warp 8+q owning TMEM lane quarter q: the scaled bf16
//               copies and the decay of S^T, Z and U to bf16, and O^T out to global memory
//               (transposed in registers by 8 x 8 shuffles, 16-byte stores).
//   warp 12     one thread: every TMA load (k, q, alpha one stage per chunk parity;
//               v) and the state chain's MMAs, in chunk order (warps 13-15 idle).
// Registers are rebalanced per warpgroup (setmaxnreg): 168 for prep, 104 for the
// state chain, 72 for the issuing warpgroup (8 x 168 + 4 x 104 + 4 x 72 = 16 x 128,
// the launch's share).
//
// The decays use running products of the clamped gates with 32-token sub-chunk
// references (D(r, j) = lam_r rho^{I(r)}_j), exactly as the gate phase below
// describes; nothing evaluates exp or log (except the optional transforms of the
// fused variant).  Every wait is bounded (2 s): a role whose wait gives up stops,
// the others leave at their next wait, in-flight copies and MMAs are drained, the
// tensor memory is freed and the status word set.
#include <cuda.h>

#include "kda_common.cuh"
#include "kda_sm100.cuh"
#include "kda_tc_maps.cuh"

// Optional event hook for timing builds: (slot, chunk, event); slots 0-7 are the prep
// warps, 8 the state chain, 9 the issuing thread (no-op in the library).
#ifndef KDA_TC2_MARK
#define KDA_TC2_MARK(role, chunk, event)
#endif

namespace kda {
using namespace sm100;

namespace tc2 {

constexpr int C = 64;
constexpr int DK = 128;
constexpr int DV = 128;
constexpr int NPREP = 256;                     // warps 0-7
constexpr int NSTATE = 128;                    // warps 8-11
constexpr int NTHREADS = NPREP + NSTATE + 128; // + warpgroup 3 (warp 12 issues, 13-15 idle)
constexpr uint32_t REG_PREP = 168, REG_STATE = 104, REG_CTL = 72;
static_assert(8 * REG_PREP + 4 * REG_STATE + 4 * REG_CTL == 16 * 128, "register split");
constexpr int WARP_STATE = 8;
constexpr int WARP_CTL = 12;
constexpr uint64_t kWaitNs = 2000000000ull;    // 2 s per wait, then report a timeout

// shared-memory map (bytes from the 1024-aligned base)
// A stage (one per chunk parity) holds the chunk's k, q and alpha tiles as TMA
// delivers them, in the atoms the MMAs read afterwards:
//   kq: per 64-channel atom a, rows 0-63 k then rows 64-127 q ([128][64] bf16, 16 KB
//       at a * 16 KB): k*lam and q*lam in place, the M=128 left operand of [A/beta ; P]
//   ar: per atom a, rows 0-31 k*rho^0, rows 32-95 alpha -> k*rho^1 -> k*eta
//       ([96][64] bf16, 12 KB at a * 12 KB): the N=96 right operand of [A/beta ; P]
constexpr uint32_t KQ_STAGE = 32768;
constexpr uint32_t AR_STAGE = 24576;
constexpr uint32_t OFF_KQ = 0;                 // 2 stages
constexpr uint32_t OFF_AR = 65536;             // 2 stages
constexpr uint32_t OFF_V = 114688;             // v tile [64 j][128 n] (two [64][64] atoms)
constexpr uint32_t OFF_X = 131072;             // solve work region, 56 KB (below)
constexpr uint32_t OFF_P = 188416;             // P [64 r][64 j] x 2 stages
constexpr uint32_t OFF_TB = 204800;            // Tb [64 j][64 j'] x 2 stages
constexpr uint32_t OFF_MISC = 221184;
constexpr uint32_t MISC_PI = 0;                // float [8][128] octant gate products
constexpr uint32_t MISC_GAM = 4096;            // float [2 stages][4][128]: Gamma_0, Gamma_1, gamma_C, gamma_C/Gamma_1
constexpr uint32_t MISC_BETA = 8192;           // float [2][64] beta per stage
constexpr uint32_t MISC_BAR = 8704;            // mbarriers (enum below)
constexpr uint32_t MISC_TMEM = 8832;
constexpr uint32_t MISC_FLAG = 8836;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 9216 + 1024;   // + alignment slack

// solve work region
constexpr int AS = 68;             // row stride (floats) of the fp32 A and Tinv tiles
constexpr uint32_t X_AM = 0;       // float A    [64][68]
constexpr uint32_t X_TM = 17408;   // float Tinv [64][68]
constexpr uint32_t X_XS = 34816;   // float scratch [32][36]
constexpr uint32_t X_T0T = 40960;  // Tinv[0:32, 0:32]^T, fp32 K-major [64 rows (32 used)][32]
constexpr uint32_t X_T1 = 49152;   // Tinv[32:64, 32:64], fp32 K-major [32][32]
constexpr uint32_t X_A10 = 53248;  // A[32:64, 0:32], fp32 K-major [32][32]

enum Bar {
    B_FULL = 0,       // [2] k, q, alpha of a stage landed (TMA)
    B_EMPTY = 2,      // [2] the state chain is done with a stage (MMA commit)
    B_READY = 4,      // [2] prep has filled a stage's operands
    B_VFULL = 6,      // v landed (TMA)
    B_PMMA = 7,       // prep's MMA groups
    B_RZ = 8,         // state -> issuer: S^T copied, issue Z^T
    B_RQ = 9,         //                 previous O^T read out, issue O^T
    B_RU = 10,        //                 Z^T (bf16) written, issue U^T
    B_R3 = 11,        //                 U^T written, issue the state update and O^T += U^T P^T
    B_BZ = 12,        // issuer -> state: Z^T done
    B_BU = 13,        //                  U^T done
    B_BS = 14,        //                  state update and O^T done
    NBAR = 15
};

// TMEM columns
constexpr uint32_t TS = 0;      // S^T fp32 [128 n][128 c]
constexpr uint32_t TSB0 = 128;  // S^T Diag(Gamma_0) bf16 pairs (64 columns)
constexpr uint32_t TSB1 = 192;  // S^T Diag(Gamma_1) bf16 pairs (64 columns)
constexpr uint32_t TZ = 256;    // Z^T, then U^T, fp32 (64 columns)
constexpr uint32_t TO = 320;    // O^T fp32 (64 columns)
constexpr uint32_t TVU = 384;   // Z^T, then U^T, bf16 pairs (32 columns)
constexpr uint32_t TP = 416;    // prep: [A/beta ; P] (96 columns), then the tf32 solve products

__device__ __forceinline__ uint32_t swz(uint32_t row, uint32_t chunk) {
    return row * 128u + (((chunk ^ row) & 7u) << 4);
}
// byte offset of fp32 element (r, k) in a K-major 128B-swizzled tile with 32 floats per row
__device__ __forceinline__ uint32_t f32_off(uint32_t r, uint32_t k) {
    return r * 128u + ((((k >> 2) ^ r) & 7u) << 4) + ((k & 3u) << 2);
}
__device__ __forceinline__ void unpack4_bf16(uint2 raw, float (&v)[4]) {
    const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
    const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
    v[0] = lo.x; v[1] = lo.y; v[2] = hi.x; v[3] = hi.y;
}
__device__ __forceinline__ void st4_bf16(uint8_t* p, const float (&v)[4]) {
    *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
}
__device__ __forceinline__ uint4 pack8(const float* v) {
    return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                      pack_bf16x2(v[6], v[7]));
}
__device__ __forceinline__ float u2f(uint32_t x) { return __uint_as_float(x); }

// the prep warps' and the state warps' own barriers (the others are not held up)
__device__ __forceinline__ void prep_bar() { named_bar_sync(1, NPREP); }
__device__ __forceinline__ void state_bar() { named_bar_sync(2, NSTATE); }

// Time segments and state slots: as the first tensor-core kernel (kda_chunk_tc.cu).
struct Segments {
    int nseg;             // segments per sequence (1: whole sequences)
    int per_seq;          // segment CTAs per sequence in this launch
    const float* start;   // nseg > 1: start states [nseq * nseg, H, DK, DV]
    const int32_t* slots; // whole sequences only: S0 / S_final at slot slots[n] (null: n)
    int num_slots;
};

// kCtaStatus = false: a timed-out wait sets the shared word *status to 1.
// kCtaStatus = true:  every CTA writes its own word status[n * H + h] (0 or 1).
// kFused = true: alpha and beta arrive as logits (alpha = 1/(1+e^x), beta =
// sigmoid(x)) and q, k unnormalised (L2-normalised per token and head here).
template <bool kCtaStatus, bool kFused>
__global__ void __launch_bounds__(NTHREADS, 1)
kda_chunk_tc2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmV,
                     const __nv_bfloat16* __restrict__ beta, const float* S0,
                     const int32_t* __restrict__ cu_seqlens, __nv_bfloat16* __restrict__ out,
                     float* S_final, int64_t T, int H, int* status, const Segments seg) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    uint8_t* sKQ = sm + OFF_KQ;
    uint8_t* sAR = sm + OFF_AR;
    uint8_t* sV = sm + OFF_V;
    uint8_t* sX = sm + OFF_X;
    uint8_t* sP = sm + OFF_P;
    uint8_t* sTB = sm + OFF_TB;
    float* sPi = reinterpret_cast<float*>(sm + OFF_MISC + MISC_PI);
    float* sGam = reinterpret_cast<float*>(sm + OFF_MISC + MISC_GAM);
    float* sBeta = reinterpret_cast<float*>(sm + OFF_MISC + MISC_BETA);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_MISC + MISC_BAR);
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + OFF_MISC + MISC_TMEM);
    volatile int* sFlag = reinterpret_cast<volatile int*>(sm + OFF_MISC + MISC_FLAG);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool is_prep = warp < WARP_STATE;
    const bool ctl = warp == WARP_CTL && lane == 0;
    const int q4 = warp & 3;            // TMEM lane quarter this warp may touch
    const int h = blockIdx.y;
    const int per_seq = seg.per_seq, gseg = (int)blockIdx.z % per_seq;
    __shared__ int s_seq;
    if (threadIdx.x < 32) {
        const int sq = longest_first_seq(cu_seqlens, (int)gridDim.z / per_seq,
                                         (int)blockIdx.z / per_seq, T);
        if (threadIdx.x == 0) s_seq = sq;
    }
    __syncthreads();
    const int n = s_seq;
    int64_t bos, len;
    seq_range(cu_seqlens, n, T, bos, len);
    if (seg.nseg > 1) {   // this CTA's segment of the sequence
        const int64_t nch = (len + C - 1) / C, cps = (nch + seg.nseg - 1) / seg.nseg;
        const int64_t c0 = min((int64_t)gseg * cps, nch), c1 = min((int64_t)(gseg + 1) * cps, nch);
        const int64_t t0 = min(c0 * C, len), t1 = min(c1 * C, len);
        bos += t0;
        len = t1 - t0;
    }
    const int nchunks = (int)((len + C - 1) / C);
    const bool last_seg = gseg == seg.nseg - 1;
    const int slot = seg.slots ? seg.slots[n] : n;
    const bool slot_ok = !seg.slots || (slot >= 0 && slot < seg.num_slots);

    if (tid == 0) {
        for (int i = 0; i < NBAR; ++i) mbar_init(bar + i, 1);
        mbar_fence_init();
        *sFlag = 0;
    }
    if (warp == 0) tmem_alloc(sTmem, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *sTmem;
    const uint32_t tlane = (uint32_t)(32 * q4) << 16;

    bool ok = true;   // this thread has seen every one of its waits complete
    // bounded wait; a thread that gives up (or finds the flag set) records it and stops waiting
    auto wait_bar = [&](int b, uint32_t parity) -> bool {
        if (!ok) return false;
        if (*sFlag) { ok = false; return false; }
        if (!mbar_wait_ns(bar + b, parity, kWaitNs)) {
            ok = false;
            *sFlag = 1;
            return false;
        }
        return true;
    };

    auto chunk_len = [&](int c) -> int {
        const int64_t rest = len - (int64_t)c * C;
        return (int)(rest < C ? rest : C);
    };

    // =====================================================================================
    // warp 12: TMA loads and the state chain's MMAs, in chunk order
    // =====================================================================================
    if (warp >= WARP_CTL) {
    warpgroup_reg_dealloc<REG_CTL>();
    if (ctl) {
        int issued_full[2] = {0, 0}, issued_v = 0;
        int last_commit = -1;          // the barrier of the last committed MMA group
        uint32_t last_commit_ph = 0;
        auto issue_stage = [&](int c) {
            const int s = c & 1;
            const int row0 = (int)(bos + (int64_t)c * C);
            mbar_arrive_expect_tx(bar + B_FULL + s, 3 * 16384);
#pragma unroll
            for (int a = 0; a < 2; ++a) {
                uint8_t* kq = sKQ + s * KQ_STAGE + a * 16384;
                tma_load_2d(kq, &tmK, bar + B_FULL + s, h * DK + 64 * a, row0);
                tma_load_2d(kq + 8192, &tmQ, bar + B_FULL + s, h * DK + 64 * a, row0);
                tma_load_2d(sAR + s * AR_STAGE + a * 12288 + 4096, &tmA, bar + B_FULL + s, h * DK + 64 * a, row0);
            }
            ++issued_full[s];
        };
        auto issue_v = [&](int c) {
            const int row0 = (int)(bos + (int64_t)c * C);
            mbar_arrive_expect_tx(bar + B_VFULL, 16384);
#pragma unroll
            for (int a = 0; a < 2; ++a)
                tma_load_2d(sV + a * 8192, &tmV, bar + B_VFULL, h * DV + 64 * a, row0);
            ++issued_v;
        };
        auto commit = [&](int b, uint32_t ph) {
            mma_commit(bar + b);
            last_commit = b;
            last_commit_ph = ph;
        };
        constexpr uint32_t id32 = idesc_bf16(128, 32);                  // both operands K-major
        constexpr uint32_t id64 = idesc_bf16(128, 64);
        constexpr uint32_t id128mn = idesc_bf16(128, 128, false, true);  // B MN-major
        if (nchunks > 0) {
            issue_stage(0);
            issue_v(0);
        }
        if (nchunks > 1) issue_stage(1);
        for (int c = 0; c < nchunks; ++c) {
            const int s = c & 1;
            const uint32_t ph = (uint32_t)c & 1u;
            // Z^T = S^T (k*gamma)^T
            if (!wait_bar(B_RZ, ph)) break;
            tc_fence_after();
            KDA_TC2_MARK(9, c, 0);
            {   // sub-chunk I: Z^T columns j in [32 I, 32 I + 32) from k*lam rows 32 I ..
                const uint32_t kq = smem_u32(sKQ + s * KQ_STAGE);
#pragma unroll
                for (int I = 0; I < 2; ++I)
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_bf16_ts(tmem + TZ + 32 * I, tmem + (I ? TSB1 : TSB0) + 8 * ks,
                                    sdesc_sw128(kq + (ks >> 2) * 16384 + I * 4096 + (ks & 3) * 32), id32,
                                    ks > 0);
                commit(B_BZ, ph);
            }
            // O^T = S^T (q*gamma)^T, once the previous chunk's O^T is read out
            if (!wait_bar(B_RQ, ph)) break;
            tc_fence_after();
            KDA_TC2_MARK(9, c, 1);
            {   // from q*lam rows 32 I .. (the q half of each kq atom)
                const uint32_t qg = smem_u32(sKQ + s * KQ_STAGE) + 8192;
#pragma unroll
                for (int I = 0; I < 2; ++I)
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_bf16_ts(tmem + TO + 32 * I, tmem + (I ? TSB1 : TSB0) + 8 * ks,
                                    sdesc_sw128(qg + (ks >> 2) * 16384 + I * 4096 + (ks & 3) * 32), id32,
                                    ks > 0);
            }
            // U^T = V^T Tb^T - Z^T Tb^T: the v tile as the MN-major A operand (M = 128 value
            // columns, K = 64 tokens) from shared memory, then bf16(Z)^T from TMEM, negated
            if (!wait_bar(B_RU, ph)) break;
            tc_fence_after();
            KDA_TC2_MARK(9, c, 2);
            {
                constexpr uint32_t idv = idesc_bf16(128, 64, true, false);
                constexpr uint32_t idneg = idesc_bf16(128, 64, false, false, true);
                const uint32_t tb = smem_u32(sTB + s * 8192), v0 = smem_u32(sV);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + TZ, sdesc_sw128(v0 + ks * 2048, 1024, 8192), sdesc_sw128(tb + ks * 32), idv,
                             ks > 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ts(tmem + TZ, tmem + TVU + 8 * ks, sdesc_sw128(tb + ks * 32), idneg, 1);
                commit(B_BU, ph);
            }
            // S^T += U^T (k*eta) (S^T already decayed) and O^T += U^T P^T
            if (!wait_bar(B_R3, ph)) break;
            tc_fence_after();
            KDA_TC2_MARK(9, c, 3);
            if (c + 1 < nchunks) issue_v(c + 1);   // U^T is done (the state waited for it): v is free
            {
                // k*eta: rows 32..95 of the ar atoms, the MN-major B operand (N = 128 channels
                // in two atoms 12 KB apart, K = 64 tokens)
                const uint32_t kh = smem_u32(sAR + s * AR_STAGE) + 4096, p0 = smem_u32(sP + s * 8192);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ts(tmem + TS, tmem + TVU + 8 * ks, sdesc_sw128(kh + ks * 2048, 1024, 12288),
                                id128mn, 1);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ts(tmem + TO, tmem + TVU + 8 * ks, sdesc_sw128(p0 + ks * 32), id64, 1);
                commit(B_EMPTY + s, (uint32_t)(c >> 1) & 1u);
                commit(B_BS, ph);
            }
            // the stage is free once these MMAs complete: load chunk c + 2 into it
            if (c + 2 < nchunks) {
                if (!wait_bar(B_EMPTY + s, (uint32_t)(c >> 1) & 1u)) break;
                KDA_TC2_MARK(9, c, 4);
                issue_stage(c + 2);
            }
        }
        if (!ok) {
            // let this thread's copies and MMAs in flight finish (bounded) before the
            // shared and tensor memory are released; a barrier's last issued phase
            // has parity (issued - 1) & 1
            *sFlag = 1;
            for (int s = 0; s < 2; ++s)
                if (issued_full[s]) mbar_wait_ns(bar + B_FULL + s, (uint32_t)(issued_full[s] - 1) & 1u, kWaitNs);
            if (issued_v) mbar_wait_ns(bar + B_VFULL, (uint32_t)(issued_v - 1) & 1u, kWaitNs);
            if (last_commit >= 0) mbar_wait_ns(bar + last_commit, last_commit_ph, kWaitNs);
        }
    }
    }

    // =====================================================================================
    // warps 0-7: the state-independent work of each chunk, one chunk ahead
    // =====================================================================================
    else if (is_prep) {
        warpgroup_reg_alloc<REG_PREP>();
        constexpr bool fused = kFused;
        auto load_beta = [&](int64_t token) {   // token index in the segment, < len
            const float x = __bfloat162float(beta[(size_t)(bos + token) * H + h]);
            return fused ? sigmoid_f(x) : x;
        };
        float beta_next = (tid < C && tid < len) ? load_beta(tid) : 0.0f;
        uint32_t ph_p = 0;
        bool pmma_out = false;   // (thread 0) a prep MMA group committed, not yet waited for
        uint32_t pmma_ph = 0;
        const int hf = warp >> 2;   // which half of the columns this warp handles
        for (int c = 0; c < nchunks; ++c) {
            const int s = c & 1;
            const int Lc = chunk_len(c);
            uint8_t* sKQc = sKQ + s * KQ_STAGE;
            uint8_t* sARc = sAR + s * AR_STAGE;
            float* sBeta_s = sBeta + 64 * s;
            float* sGam_s = sGam + 512 * s;
            if (tid < C) sBeta_s[tid] = beta_next;
            if (lane == 0) KDA_TC2_MARK(warp, c, 0);
            wait_bar(B_FULL + s, (uint32_t)(c >> 1) & 1u);
            if (lane == 0) KDA_TC2_MARK(warp, c, 1);

            // ================= gate products and bf16 operands
            {
                // thread = (channels c0..c0+3) x (8-token octant O).  Quarter Q = O/2 holds 16
                // tokens, sub-chunk I = Q/2 holds 32; the reference token of I is ref_I = 32I + 15.
                // With phi / psi the in-quarter forward (inclusive) / backward (exclusive) gate
                // products and pi_Q the quarter product:
                //   left  lam_t   = e^{g_t - g_ref}  = phi_t * (Q even ? 1/pi_Q : 1)
                //   right rho^I_j = e^{g_ref - g_j}  = psi_j * c_I(Q(j))
                //   c_0 = {1, 1/pi_1},  c_1 = {pi_1 pi_2, pi_2, 1, 1/pi_3}
                // so that lam_r rho^I_j = prod_{s=j+1..r} a_s for j <= r, every factor within
                // [e^-80, e^80] except right factors that underflow where the product is negligible.
                // In-quarter products come from in-octant ones phi8, psi8 and the octant products
                // pi8: phi = phi8 * (O odd ? pi8_{O-1} : 1), psi = psi8 * (O even ? pi8_{O+1} : 1);
                // those octant factors are folded into the per-thread scales below.
                // Every tile touched here is row-major with 128-byte swizzled rows; a warp covers
                // one token row of all 128 channels (8 bytes per thread).  Outputs: k*lam over
                // k, q*lam over q, k*rho^1 over alpha, k*rho^0 in the rows before it.
                const int cq = tid & 31, O = tid >> 5, Q = O >> 1, c0 = 4 * cq;
                const uint32_t chk = (uint32_t)((c0 & 63) >> 3), inner = (uint32_t)((c0 & 7) << 1);
                const uint32_t a64 = (uint32_t)(c0 >> 6);
                auto sw_of = [&](int r) {
                    return (uint32_t)r * 128u + (((chk ^ (uint32_t)r) & 7u) << 4) + inner;
                };
                uint8_t* kbase = sKQc + a64 * 16384u;           // k rows; q rows at + 8192
                uint8_t* abase = sARc + a64 * 12288u;           // k*rho^0 rows; alpha rows at + 4096
                float phi[8][4], psi[8][4];   // psi holds the clamped gates until the backward pass
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = 8 * O + i;
                    float a[4];
                    unpack4_bf16(*reinterpret_cast<const uint2*>(abase + 4096 + sw_of(r)), a);
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        const float g = clamp_gate(fused ? gate_from_logit(a[cc]) : a[cc]);
                        psi[i][cc] = (Lc == C || r < Lc) ? g : 1.0f;
                    }
                }
                {
                    float p[4] = {1.f, 1.f, 1.f, 1.f}, b[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll
                    for (int i = 0; i < 8; ++i)
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) { p[cc] *= psi[i][cc]; phi[i][cc] = p[cc]; }
#pragma unroll
                    for (int i = 7; i >= 0; --i)
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) { const float a = psi[i][cc]; psi[i][cc] = b[cc]; b[cc] *= a; }
                    *reinterpret_cast<float4*>(&sPi[O * DK + c0]) = make_float4(p[0], p[1], p[2], p[3]);
                }
                if (lane == 0) KDA_TC2_MARK(warp, c, 2);
                prep_bar();
                if (lane == 0) KDA_TC2_MARK(warp, c, 3);
                // per-thread scales: quarter products; the sub-chunk reference products
                // Gamma_0 = gamma_15, Gamma_1 = gamma_47, gamma_C and gamma_C / Gamma_1 per channel
                float dlf[4], r0g[4], r1g[4];
                {
                    float pq[4][4];   // [quarter][channel]
#pragma unroll
                    for (int M = 0; M < 4; ++M) {
                        const float4 u = *reinterpret_cast<const float4*>(&sPi[(2 * M) * DK + c0]);
                        const float4 v = *reinterpret_cast<const float4*>(&sPi[(2 * M + 1) * DK + c0]);
                        pq[M][0] = u.x * v.x; pq[M][1] = u.y * v.y; pq[M][2] = u.z * v.z; pq[M][3] = u.w * v.w;
                    }
                    // the partner octant of this quarter: phi8 -> phi (O odd), psi8 -> psi (O even)
                    const float4 po = *reinterpret_cast<const float4*>(&sPi[(O ^ 1) * DK + c0]);
                    const float pov[4] = {po.x, po.y, po.z, po.w};
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        float bef = 1.f, aft = 1.f, own = 1.f;
#pragma unroll
                        for (int M = 0; M < 4; ++M) {
                            if (M < Q) bef *= pq[M][cc];
                            if (M > Q) aft *= pq[M][cc];
                            if (M == Q) own = pq[M][cc];
                        }
                        if (O == 0) {
                            const float g1 = pq[0][cc] * pq[1][cc] * pq[2][cc];
                            sGam_s[c0 + cc] = pq[0][cc];
                            sGam_s[128 + c0 + cc] = g1;
                            sGam_s[256 + c0 + cc] = g1 * pq[3][cc];
                            sGam_s[384 + c0 + cc] = pq[3][cc];
                        }
                        const float fO = (O & 1) ? pov[cc] : 1.0f;
                        const float gO = (O & 1) ? 1.0f : pov[cc];
                        const float dl = (Q & 1) ? 1.0f : __frcp_rn(own);
                        const float r0 = Q == 1 ? __frcp_rn(own) : 1.0f;
                        const float r1 = Q == 0 ? pq[1][cc] * pq[2][cc]
                                                : (Q == 1 ? pq[2][cc] : (Q == 2 ? 1.0f : __frcp_rn(own)));
                        dlf[cc] = dl * fO;
                        r0g[cc] = r0 * gO;
                        r1g[cc] = r1 * gO;
                        (void)bef;
                        (void)aft;
                    }
                }
                // fused inputs: k and q rows L2-normalised in place (bf16), before any
                // operand is formed.  A warp holds all 128 channels of its eight rows, four
                // per lane, and each thread rewrites only the elements it reads again below.
                if constexpr (kFused) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int r = 8 * O + i;
                        const uint32_t in_off = sw_of(r);
                        float k[4], q[4];
                        unpack4_bf16(*reinterpret_cast<const uint2*>(kbase + in_off), k);
                        unpack4_bf16(*reinterpret_cast<const uint2*>(kbase + 8192 + in_off), q);
                        float sk = k[0] * k[0] + k[1] * k[1] + k[2] * k[2] + k[3] * k[3];
                        float sq = q[0] * q[0] + q[1] * q[1] + q[2] * q[2] + q[3] * q[3];
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) {
                            sk += __shfl_xor_sync(0xffffffffu, sk, o);
                            sq += __shfl_xor_sync(0xffffffffu, sq, o);
                        }
                        const float ik = rsqrtf(fmaxf(sk, 1e-12f)), iq = rsqrtf(fmaxf(sq, 1e-12f));
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) { k[cc] *= ik; q[cc] *= iq; }
                        st4_bf16(kbase + in_off, k);
                        st4_bf16(kbase + 8192 + in_off, q);
                    }
                }
                // each row's k and q are read before the previous row's stores: k*lam and q*lam
                // are written in place, so a load placed after a store could not be moved above it
                uint2 kn = *reinterpret_cast<const uint2*>(kbase + sw_of(8 * O));
                uint2 qn = *reinterpret_cast<const uint2*>(kbase + 8192 + sw_of(8 * O));
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = 8 * O + i;
                    const uint32_t sw = sw_of(r);
                    float k[4], q[4];
                    unpack4_bf16(kn, k);
                    unpack4_bf16(qn, q);
                    if (i < 7) {
                        kn = *reinterpret_cast<const uint2*>(kbase + sw_of(r + 1));
                        qn = *reinterpret_cast<const uint2*>(kbase + 8192 + sw_of(r + 1));
                    }
                    if (r >= Lc) {
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) { k[cc] = 0.0f; q[cc] = 0.0f; }
                    }
                    float lam[4], w[4];
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) lam[cc] = phi[i][cc] * dlf[cc];
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) w[cc] = k[cc] * lam[cc];
                    st4_bf16(kbase + sw, w);                                  // k*lam over k, row r
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) w[cc] = q[cc] * lam[cc];
                    st4_bf16(kbase + 8192 + sw, w);                           // q*lam over q, row 64 + r
                    if (O < 4) {
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) w[cc] = k[cc] * (psi[i][cc] * r0g[cc]);
                        st4_bf16(abase + sw, w);                              // k*rho^0, row r < 32
                    }
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) w[cc] = k[cc] * (psi[i][cc] * r1g[cc]);
                    st4_bf16(abase + 4096 + sw, w);                           // k*rho^1 over alpha, row 32 + r
                }
                if (lane == 0) KDA_TC2_MARK(warp, c, 4);
            }
            fence_async_smem();
            tc_fence_before();
            prep_bar();
            tc_fence_after();
            if (lane == 0) KDA_TC2_MARK(warp, c, 5);

            // ================= [A/beta ; P] = [k*lam ; q*lam] [k*rho^0 ; k*rho^1]^T   (M=128, N=96, K=128)
            //   rows 0..63 are A/beta rows r, rows 64..127 are P rows r.  Columns [0, 32) hold
            //   rho^0 (j < 32, valid for r < 32), columns [32, 96) hold rho^1 (j < 64, valid for r >= 32).
            if (tid == 0 && ok) {
                const uint32_t l0 = smem_u32(sKQc), r0 = smem_u32(sARc);
                constexpr uint32_t idesc = idesc_bf16(128, 96);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16(tmem + TP, sdesc_sw128(l0 + (ks >> 2) * 16384u + (ks & 3) * 32u),
                             sdesc_sw128(r0 + (ks >> 2) * 12288u + (ks & 3) * 32u), idesc, ks > 0);
                mma_commit(bar + B_PMMA);
                pmma_out = true;
                pmma_ph = ph_p;
            }
            if (wait_bar(B_PMMA, ph_p) && tid == 0) pmma_out = false;
            ph_p ^= 1u;
            tc_fence_after();
            if (lane == 0) KDA_TC2_MARK(warp, c, 6);

            // ================= A (fp32, times beta_r, j < r) and P (bf16 K-major, j <= r)
            {
                // lane = row R of the accumulator: R < 64 is A row r = R, R >= 64 is P row r = R - 64;
                // this warp's column half covers j in [32 hf, 32 hf + 32)
                const int R = 32 * q4 + lane, r = R & 63, j0 = 32 * hf;
                const bool lower = (q4 & 1) == 0;          // r < 32: group 1 columns
                const bool zero = lower && hf == 1;        // j >= 32 > r: all zero
                float v[32];
                if (!zero) {
                    const uint32_t col = lower ? 0u : 32u + 32u * hf;
                    tmem_ld16(tmem + tlane + TP + col, *reinterpret_cast<float(*)[16]>(&v[0]));
                    tmem_ld16(tmem + tlane + TP + col + 16, *reinterpret_cast<float(*)[16]>(&v[16]));
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = 0.0f;
                }
                if (lane == 0) KDA_TC2_MARK(warp, c, 7);
                if (q4 < 2) {
                    float* Am = reinterpret_cast<float*>(sX + X_AM);
                    const float b = sBeta_s[r];
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        float4 f;
                        f.x = (j0 + i + 0 < r) ? b * v[i + 0] : 0.0f;
                        f.y = (j0 + i + 1 < r) ? b * v[i + 1] : 0.0f;
                        f.z = (j0 + i + 2 < r) ? b * v[i + 2] : 0.0f;
                        f.w = (j0 + i + 3 < r) ? b * v[i + 3] : 0.0f;
                        *reinterpret_cast<float4*>(&Am[r * AS + j0 + i]) = f;
                    }
                } else {
                    uint8_t* sPc = sP + s * 8192;
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8) {
                        float w[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) w[i] = (j0 + 8 * c8 + i <= r) ? v[8 * c8 + i] : 0.0f;
                        *reinterpret_cast<uint4*>(sPc + swz(r, (j0 >> 3) + c8)) = pack8(w);
                    }
                }
            }
            if (lane == 0) KDA_TC2_MARK(warp, c, 8);
            // beta of the next chunk, while the solve runs
            if (tid < C) {
                const int64_t nxt = (int64_t)(c + 1) * C + tid;   // token index in the segment
                beta_next = (c + 1 < nchunks && nxt < len) ? load_beta(nxt) : 0.0f;
            }
            // (no proxy fence here: P is read by an MMA only in the state chain, after the
            // fence that precedes the stage hand-over; A is read by the CUDA cores)
            tc_fence_before();
            prep_bar();
            tc_fence_after();

            // ================= Tinv = (I + A)^-1 by doubling: 16x16 blocks, then 32, then 64
            //   inv([[X, 0], [Y, Z]]) = [[X^-1, 0], [-Z^-1 Y X^-1, Z^-1]]
            {
                if (lane == 0) KDA_TC2_MARK(warp, c, 9);
                const float* Am = reinterpret_cast<const float*>(sX + X_AM);
                float* Tm = reinterpret_cast<float*>(sX + X_TM);
                float* Xs = reinterpret_cast<float*>(sX + X_XS);
                if (warp < 4) {
                    // diagonal 16x16 blocks by forward substitution: warp I, lane m < 16 owns column m
                    const int I = warp, m = lane & 15, o = 16 * I;
                    float col[16];
#pragma unroll
                    for (int r = 0; r < 16; ++r) {
                        float arow[16];
#pragma unroll
                        for (int jj = 0; jj < 16; jj += 4)
                            if (jj < r) *reinterpret_cast<float4*>(&arow[jj]) =
                                *reinterpret_cast<const float4*>(&Am[(o + r) * AS + o + jj]);
                        float s0 = 0.0f, s1 = 0.0f, s2 = 0.0f, s3 = 0.0f;
#pragma unroll
                        for (int jj = 0; jj < r; ++jj) {
                            if ((jj & 3) == 0) s0 = fmaf(arow[jj], col[jj], s0);
                            else if ((jj & 3) == 1) s1 = fmaf(arow[jj], col[jj], s1);
                            else if ((jj & 3) == 2) s2 = fmaf(arow[jj], col[jj], s2);
                            else s3 = fmaf(arow[jj], col[jj], s3);
                        }
                        col[r] = r < m ? 0.0f : (r == m ? 1.0f : -((s0 + s1) + (s2 + s3)));
                    }
                    if (lane < 16) {
#pragma unroll
                        for (int r = 0; r < 16; ++r) Tm[(o + r) * AS + o + m] = col[r];
                    }
                } else {
                    // zeros above the diagonal blocks that the doubling steps read
                    const int t = tid - 128;                       // 0..127
                    const int r = t >> 2, cq = (t & 3) * 4;        // rows 0..31, 4 columns each
                    const int rb = r < 16 ? r : 16 + r;            // rows 0-15 and 32-47
                    const int cb = r < 16 ? 16 + cq : 48 + cq;     // columns 16-31 and 48-63
                    *reinterpret_cast<float4*>(&Tm[rb * AS + cb]) = make_float4(0.f, 0.f, 0.f, 0.f);
                    const int r2 = t >> 2;                         // rows 0..31, columns 32..63
#pragma unroll
                    for (int c4 = 0; c4 < 2; ++c4)
                        *reinterpret_cast<float4*>(&Tm[r2 * AS + 32 + 16 * c4 + cq]) =
                            make_float4(0.f, 0.f, 0.f, 0.f);
                    // k*eta = (k*rho^1) Diag(gamma_C / Gamma_1), in place (the [A/beta ; P] MMA
                    // that read k*rho^1 is done).  Thread: atom, 16-byte chunk (8 channels), 8 rows.
                    const int at = t >> 6, ch = t & 7, rg = (t >> 3) & 7;
                    const float* ef = sGam_s + 384 + 64 * at + 8 * ch;
                    const float4 e0 = *reinterpret_cast<const float4*>(ef);
                    const float4 e1 = *reinterpret_cast<const float4*>(ef + 4);
                    const float ev[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
                    uint8_t* kr = sARc + at * 12288 + 4096;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const uint32_t row = (uint32_t)(8 * rg + i);
                        uint4* pr = reinterpret_cast<uint4*>(kr + row * 128u + ((((uint32_t)ch ^ row) & 7u) << 4));
                        const uint4 raw = *pr;
                        float x[8];
                        unpack4_bf16(make_uint2(raw.x, raw.y), *reinterpret_cast<float(*)[4]>(&x[0]));
                        unpack4_bf16(make_uint2(raw.z, raw.w), *reinterpret_cast<float(*)[4]>(&x[4]));
#pragma unroll
                        for (int e = 0; e < 8; ++e) x[e] *= ev[e];
                        *pr = pack8(x);
                    }
                }
                prep_bar();
                if (lane == 0) KDA_TC2_MARK(warp, c, 10);
                // 16 -> 32: blocks (1,0) and (3,2).  thread: block b, row r, columns m2, m2+1
                {
                    const int b = tid >> 7, r = (tid >> 3) & 15, m2 = (tid & 7) * 2;
                    const int o0 = 32 * b, o1 = o0 + 16;
                    float arow[16];
#pragma unroll
                    for (int j = 0; j < 16; j += 4)
                        *reinterpret_cast<float4*>(&arow[j]) = *reinterpret_cast<const float4*>(&Am[(o1 + r) * AS + o0 + j]);
                    float x0 = 0.f, x1 = 0.f, x2 = 0.f, x3 = 0.f;
#pragma unroll
                    for (int j = 0; j < 16; j += 2) {
                        const float2 t2 = *reinterpret_cast<const float2*>(&Tm[(o0 + j) * AS + o0 + m2]);
                        const float2 t3 = *reinterpret_cast<const float2*>(&Tm[(o0 + j + 1) * AS + o0 + m2]);
                        x0 = fmaf(arow[j], t2.x, x0); x1 = fmaf(arow[j], t2.y, x1);
                        x2 = fmaf(arow[j + 1], t3.x, x2); x3 = fmaf(arow[j + 1], t3.y, x3);
                    }
                    x0 += x2; x1 += x3;
                    *reinterpret_cast<float2*>(&Xs[(16 * b + r) * 36 + m2]) = make_float2(x0, x1);
                    prep_bar();
                    float y0 = 0.f, y1 = 0.f;
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) {
                        const float tz = Tm[(o1 + r) * AS + o1 + jj];
                        const float2 xx = *reinterpret_cast<const float2*>(&Xs[(16 * b + jj) * 36 + m2]);
                        y0 = fmaf(tz, xx.x, y0); y1 = fmaf(tz, xx.y, y1);
                    }
                    *reinterpret_cast<float2*>(&Tm[(o1 + r) * AS + o0 + m2]) = make_float2(-y0, -y1);
                }
                prep_bar();
                if (lane == 0) KDA_TC2_MARK(warp, c, 11);
                // 32 -> 64 on the tensor cores (tf32): X^T = T0^T A10^T, then Y^T = X^T T1^T with
                // X^T read back from TMEM by the second MMA; Tinv[32:64, 0:32] = -Y.  Operands:
                // fp32 K-major tiles written here (T1 serves as the second product's B).
                {
                    uint8_t* t0t = sX + X_T0T;
                    uint8_t* t1 = sX + X_T1;
                    const int rw = tid >> 3, k4 = (tid & 7) * 4;       // row 0..31, 4 columns
                    float4 c4;
                    c4.x = Tm[(k4 + 0) * AS + rw]; c4.y = Tm[(k4 + 1) * AS + rw];
                    c4.z = Tm[(k4 + 2) * AS + rw]; c4.w = Tm[(k4 + 3) * AS + rw];
                    *reinterpret_cast<float4*>(t0t + f32_off(rw, k4)) = c4;                 // T0^T[m][j]
                    *reinterpret_cast<float4*>(t1 + f32_off(rw, k4)) =
                        *reinterpret_cast<const float4*>(&Tm[(32 + rw) * AS + 32 + k4]);  // T1[r][jj]
                    *reinterpret_cast<float4*>(sX + X_A10 + f32_off(rw, k4)) =
                        *reinterpret_cast<const float4*>(&Am[(32 + rw) * AS + k4]);       // A10[r][j]
                }
                fence_async_smem();
                tc_fence_before();
                prep_bar();
                tc_fence_after();
                if (tid == 0 && ok) {
                    constexpr uint32_t idesc = idesc_tf32(64, 32);
                    const uint32_t a0 = smem_u32(sX + X_T0T), b0 = smem_u32(sX + X_A10);
                    const uint32_t b1 = smem_u32(sX + X_T1);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_tf32(tmem + TP, sdesc_sw128(a0 + ks * 32), sdesc_sw128(b0 + ks * 32), idesc, ks > 0);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_tf32_ts(tmem + TP + 32, tmem + TP + 8 * ks, sdesc_sw128(b1 + ks * 32), idesc,
                                    ks > 0);
                    mma_commit(bar + B_PMMA);
                    pmma_out = true;
                    pmma_ph = ph_p;
                }
                if (wait_bar(B_PMMA, ph_p) && tid == 0) pmma_out = false;
                ph_p ^= 1u;
                tc_fence_after();
                if (lane == 0) KDA_TC2_MARK(warp, c, 12);
                // both products are done: Y^T = X^T T1^T is in TMEM (M=64 rows c = 16 q4 + lane,
                // columns r'); Tinv[32 + r', c] = -Y[r', c]
                if (q4 < 2) {
                    float v[32];
                    tmem_ld16(tmem + tlane + TP + 32, *reinterpret_cast<float(*)[16]>(&v[0]));
                    tmem_ld16(tmem + tlane + TP + 48, *reinterpret_cast<float(*)[16]>(&v[16]));
                    tmem_wait_ld();
                    if (hf == 0 && lane < 16) {
                        const int cc = 16 * q4 + lane;
#pragma unroll
                        for (int r = 0; r < 32; ++r) Tm[(32 + r) * AS + cc] = -v[r];
                    }
                }
                tc_fence_before();
                prep_bar();
                if (lane == 0) KDA_TC2_MARK(warp, c, 13);
                // Tb = Tinv diag(beta): the K-major B operand [64 j][64 j'] of U^T; zero above
                // the diagonal
                uint8_t* sTBc = sTB + s * 8192;
#pragma unroll
                for (int rep = 0; rep < 2; ++rep) {
                    const int e = tid + NPREP * rep;
                    const int jr = e & 63, ch = e >> 6;
                    float v[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int m = 8 * ch + i;
                        v[i] = (jr >= m) ? Tm[jr * AS + m] * sBeta_s[m] : 0.0f;
                    }
                    *reinterpret_cast<uint4*>(sTBc + swz(jr, ch)) = pack8(v);
                }
            }
            // the stage's operands are complete: hand them to the state chain
            fence_async_smem();
            tc_fence_before();
            const bool stop = named_bar_or(1, NPREP, !ok || *sFlag != 0);
            if (stop) break;
            if (lane == 0) KDA_TC2_MARK(warp, c, 14);
            if (tid == 0) mbar_arrive(bar + B_READY + s);
        }
        if (tid == 0 && pmma_out) mbar_wait_ns(bar + B_PMMA, pmma_ph, kWaitNs);
        if (!ok) *sFlag = 1;
    }

    // =====================================================================================
    // warps 8-11: the state chain.  Thread = TMEM lane n = value column n of S^T.
    // =====================================================================================
    else {
        warpgroup_reg_dealloc<REG_STATE>();
        const int nn = 32 * q4 + lane;         // value column owned by this thread
        const bool elected = warp == WARP_STATE && lane == 0;
        // ---- initial state S^T (column n of S0, or of the segment's start state)
        {
            const float* base = seg.nseg > 1
                                    ? seg.start + (((size_t)n * seg.nseg + gseg) * H + h) * DK * DV
                                    : (S0 && slot_ok ? S0 + ((size_t)slot * H + h) * DK * DV : nullptr);
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                uint32_t r[32];
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    r[i] = base ? __float_as_uint(base[(size_t)(32 * p + i) * DV + nn]) : 0u;
                tmem_st32(tmem + tlane + TS + 32 * p, r);
            }
            tmem_wait_st();
        }
        // O^T of chunk c from TMEM to out[row0 + r][h][n].  Thread n holds column n of O for
        // the 64 rows; each 8 x 8 block (8 rows x 8 consecutive columns of 8 lanes) is
        // transposed by three xor-butterfly rounds of shuffles (rounds 4 and 2 swap whole
        // bf16 pairs, round 1 swaps halves), after which lane i of the group holds 8
        // consecutive columns of row i: one 16-byte store.  Rows past the chunk's length
        // are not stored.
        auto store_o = [&](int c) {
            const int Lc = chunk_len(c);
            const int64_t row0 = bos + (int64_t)c * C;
            const int gi = lane & 7;
            const bool b4 = (gi >> 2) & 1, b2 = (gi >> 1) & 1, b1 = gi & 1;
            __nv_bfloat16* obase = out + ((size_t)row0 * H + h) * DV + (32 * q4 + (lane & ~7));
            const size_t rs = (size_t)H * DV;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t f[32];
                tmem_ld32(tmem + tlane + TO + 32 * half, f);
                tmem_wait_ld();
#pragma unroll
                for (int blk = 0; blk < 4; ++blk) {
                    uint32_t p[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) p[u] = pack_bf16x2(u2f(f[8 * blk + 2 * u]), u2f(f[8 * blk + 2 * u + 1]));
                    {   // rows 4..7 <-> lanes 4..7
                        const uint32_t x0 = b4 ? p[0] : p[2], x1 = b4 ? p[1] : p[3];
                        const uint32_t y0 = __shfl_xor_sync(0xffffffffu, x0, 4);
                        const uint32_t y1 = __shfl_xor_sync(0xffffffffu, x1, 4);
                        if (b4) { p[0] = y0; p[1] = y1; } else { p[2] = y0; p[3] = y1; }
                    }
                    {   // rows 2,3 <-> lanes 2,3 (within each half)
                        const uint32_t x0 = b2 ? p[0] : p[1], x1 = b2 ? p[2] : p[3];
                        const uint32_t y0 = __shfl_xor_sync(0xffffffffu, x0, 2);
                        const uint32_t y1 = __shfl_xor_sync(0xffffffffu, x1, 2);
                        if (b2) { p[0] = y0; p[2] = y1; } else { p[1] = y0; p[3] = y1; }
                    }
                    {   // odd rows <-> odd lanes: 16-bit halves
                        const uint32_t x0 = b1 ? __byte_perm(p[0], p[1], 0x5410) : __byte_perm(p[0], p[1], 0x7632);
                        const uint32_t x1 = b1 ? __byte_perm(p[2], p[3], 0x5410) : __byte_perm(p[2], p[3], 0x7632);
                        const uint32_t y0 = __shfl_xor_sync(0xffffffffu, x0, 1);
                        const uint32_t y1 = __shfl_xor_sync(0xffffffffu, x1, 1);
                        if (b1) {
                            p[0] = __byte_perm(y0, p[0], 0x7610); p[1] = __byte_perm(y0, p[1], 0x7632);
                            p[2] = __byte_perm(y1, p[2], 0x7610); p[3] = __byte_perm(y1, p[3], 0x7632);
                        } else {
                            p[0] = __byte_perm(p[0], y0, 0x5410); p[1] = __byte_perm(p[1], y0, 0x7610);
                            p[2] = __byte_perm(p[2], y1, 0x5410); p[3] = __byte_perm(p[3], y1, 0x7610);
                        }
                    }
                    const int row = 32 * half + 8 * blk + gi;
                    if (row < Lc)
                        *reinterpret_cast<uint4*>(obase + (size_t)row * rs) = make_uint4(p[0], p[1], p[2], p[3]);
                }
            }
        };
        bool broke = false;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c & 1;
            const uint32_t ph = (uint32_t)c & 1u;
            wait_bar(B_READY + s, (uint32_t)(c >> 1) & 1u);
            if (c > 0) wait_bar(B_BS, ph ^ 1u);
            ok = __all_sync(0xffffffffu, ok);   // the TMEM loads and stores below are warp-wide
            tc_fence_after();
            if (elected) KDA_TC2_MARK(8, c, 0);
            // ---- S^T Diag(Gamma_0) and S^T Diag(Gamma_1) to bf16 (the A operands of this chunk's
            //      products), and S^T <- S^T Diag(gamma_C)
            if (ok) {
                const float* g0 = sGam + 512 * s;
                const float* g1 = g0 + 128;
                const float* gc = g0 + 256;
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    uint32_t r[32];
                    tmem_ld32(tmem + tlane + TS + 32 * p, r);
                    tmem_wait_ld();
                    uint32_t b0[16], b1[16];
#pragma unroll
                    for (int i = 0; i < 16; i += 2) {
                        const float4 a0 = *reinterpret_cast<const float4*>(g0 + 32 * p + 2 * i);
                        const float4 a1 = *reinterpret_cast<const float4*>(g1 + 32 * p + 2 * i);
                        const float x0 = u2f(r[2 * i]), x1 = u2f(r[2 * i + 1]);
                        const float x2 = u2f(r[2 * i + 2]), x3 = u2f(r[2 * i + 3]);
                        b0[i] = pack_bf16x2(x0 * a0.x, x1 * a0.y);
                        b0[i + 1] = pack_bf16x2(x2 * a0.z, x3 * a0.w);
                        b1[i] = pack_bf16x2(x0 * a1.x, x1 * a1.y);
                        b1[i + 1] = pack_bf16x2(x2 * a1.z, x3 * a1.w);
                    }
                    tmem_st16u(tmem + tlane + TSB0 + 16 * p, b0);
                    tmem_st16u(tmem + tlane + TSB1 + 16 * p, b1);
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        const float4 gg = *reinterpret_cast<const float4*>(gc + 32 * p + i);
                        r[i] = __float_as_uint(u2f(r[i]) * gg.x);
                        r[i + 1] = __float_as_uint(u2f(r[i + 1]) * gg.y);
                        r[i + 2] = __float_as_uint(u2f(r[i + 2]) * gg.z);
                        r[i + 3] = __float_as_uint(u2f(r[i + 3]) * gg.w);
                    }
                    tmem_st32(tmem + tlane + TS + 32 * p, r);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            if (named_bar_or(2, NSTATE, !ok || *sFlag != 0)) { broke = true; break; }
            if (elected) mbar_arrive(bar + B_RZ);
            if (elected) KDA_TC2_MARK(8, c, 1);
            // ---- the previous chunk's O^T leaves while Z^T is computed
            if (c > 0) store_o(c - 1);
            tc_fence_before();
            state_bar();
            if (elected) mbar_arrive(bar + B_RQ);
            if (elected) KDA_TC2_MARK(8, c, 2);
            // ---- (V - Z)^T: column n of the v tile minus row n of Z^T, as bf16 pairs
            wait_bar(B_VFULL, ph);
            wait_bar(B_BZ, ph);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
            if (elected) KDA_TC2_MARK(8, c, 3);
            if (ok) {   // Z^T to bf16 pairs, the A operand of the second U^T product
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t z[32];
                    tmem_ld32(tmem + tlane + TZ + 32 * half, z);
                    tmem_wait_ld();
                    uint32_t b[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) b[i] = pack_bf16x2(u2f(z[2 * i]), u2f(z[2 * i + 1]));
                    tmem_st16u(tmem + tlane + TVU + 16 * half, b);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            state_bar();
            if (elected) mbar_arrive(bar + B_RU);
            if (elected) KDA_TC2_MARK(8, c, 4);
            // ---- U^T as bf16 pairs
            wait_bar(B_BU, ph);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
            if (elected) KDA_TC2_MARK(8, c, 5);
            if (ok) {
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t u[32];
                    tmem_ld32(tmem + tlane + TZ + 32 * half, u);
                    tmem_wait_ld();
                    uint32_t b[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) b[i] = pack_bf16x2(u2f(u[2 * i]), u2f(u[2 * i + 1]));
                    tmem_st16u(tmem + tlane + TVU + 16 * half, b);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            if (named_bar_or(2, NSTATE, !ok || *sFlag != 0)) { broke = true; break; }
            if (elected) mbar_arrive(bar + B_R3);
            if (elected) KDA_TC2_MARK(8, c, 6);
        }
        // ---- the last chunk's O^T, then S_final (column n of S^T)
        if (!broke && nchunks > 0) {
            wait_bar(B_BS, (uint32_t)(nchunks - 1) & 1u);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
            if (ok) store_o(nchunks - 1);
        }
        if (!broke && ok && S_final && last_seg && slot_ok) {
            float* dst = S_final + ((size_t)slot * H + h) * DK * DV + nn;
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                uint32_t r[32];
                tmem_ld32(tmem + tlane + TS + 32 * p, r);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) dst[(size_t)(32 * p + i) * DV] = u2f(r[i]);
            }
        }
        if (!ok || broke) *sFlag = 1;
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const int failed = *sFlag;
    if (kCtaStatus && tid == 0) status[(size_t)n * H + h] = failed;
    if (!kCtaStatus && failed && tid == 0) atomicExch(status, 1);
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace tc2

template <bool kCtaStatus, bool kFused>
static cudaError_t launch_tc2_t(const TcMaps& m, const void* beta, const float* S0, const int32_t* cu,
                                int nseq, void* out, float* S_final, int64_t T, int H, int* status,
                                const tc2::Segments& seg, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(tc2::kda_chunk_tc2_kernel<kCtaStatus, kFused>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)tc2::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    dim3 grid(1, H, nseq * seg.per_seq);
    tc2::kda_chunk_tc2_kernel<kCtaStatus, kFused><<<grid, tc2::NTHREADS, tc2::SMEM_BYTES, stream>>>(
        m.q, m.k, m.a, m.v, (const __nv_bfloat16*)beta, S0, cu, (__nv_bfloat16*)out, S_final, T, H,
        status, seg);
    return cudaGetLastError();
}

// Whole sequences (optionally from and into pooled state slots).
cudaError_t launch_chunk_tc2(const void* q, const void* k, const void* v, const void* alpha,
                             const void* beta, const float* S0, const int32_t* cu, int nseq,
                             void* out, float* S_final, int64_t rows, int64_t T, int H, int* status,
                             cudaStream_t stream, const int32_t* slots, int num_slots, int fused) {
    TcMaps m;
    if (!make_tc_maps(&m, q, k, v, alpha, out, rows, H)) return cudaErrorInvalidValue;
    const tc2::Segments whole{1, 1, nullptr, slots, num_slots};
    return fused ? launch_tc2_t<false, true>(m, beta, S0, cu, nseq, out, S_final, T, H, status, whole,
                                             stream)
                 : launch_tc2_t<false, false>(m, beta, S0, cu, nseq, out, S_final, T, H, status, whole,
                                              stream);
}

// The forward of every time segment from its start state (start: [nseq * nseg, H, DK, DV]).
cudaError_t launch_chunk_tc2_segments(const void* q, const void* k, const void* v, const void* alpha,
                                      const void* beta, const float* start, const int32_t* cu,
                                      int nseq, void* out, float* S_final, int64_t rows, int64_t T,
                                      int H, int nseg, int* status, cudaStream_t stream, int fused) {
    TcMaps m;
    if (!make_tc_maps(&m, q, k, v, alpha, out, rows, H)) return cudaErrorInvalidValue;
    const tc2::Segments fwd{nseg, nseg, start, nullptr, 0};
    return fused ? launch_tc2_t<false, true>(m, beta, nullptr, cu, nseq, out, S_final, T, H, status,
                                             fwd, stream)
                 : launch_tc2_t<false, false>(m, beta, nullptr, cu, nseq, out, S_final, T, H, status,
                                              fwd, stream);
}

// Whole sequences, one status word per (sequence, head) CTA at status[n * H + h].
cudaError_t launch_chunk_tc2_cta_status(const void* q, const void* k, const void* v,
                                        const void* alpha, const void* beta, const float* S0,
                                        const int32_t* cu, int nseq, void* out, float* S_final,
                                        int64_t rows, int64_t T, int H, int* status,
                                        cudaStream_t stream) {
    TcMaps m;
    if (!make_tc_maps(&m, q, k, v, alpha, out, rows, H)) return cudaErrorInvalidValue;
    const tc2::Segments whole{1, 1, nullptr, nullptr, 0};
    return launch_tc2_t<true, false>(m, beta, S0, cu, nseq, out, S_final, T, H, status, whole, stream);
}

}  // namespace kda
