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
// Transposed, with S^T in TMEM (lane n = value column, columns = key channels):
//
//   Z^T = S^T (k*gamma)^T            M=128 (n), N=64 (j), K=128 (c)   A: S^T bf16 (TMEM)
//   O^T = S^T (q*gamma)^T            M=128, N=64 (r), K=128            A: S^T bf16 (TMEM)
//   U^T = (V - Z)^T Tb^T             M=128, N=64, K=64 (j')            A: (V - Z)^T bf16 (TMEM)
//   S^T <- S^T Diag(gamma_C) + U^T (k*eta)    M=128, N=128 (c), K=64   A: U^T bf16 (TMEM)
//   O^T += U^T P^T                   M=128, N=64, K=64                 A: U^T bf16 (TMEM)
//
// so the chain that carries the state from chunk to chunk moves no operand of its
// own through shared memory: the B operands (k*gamma, q*gamma, Tb, k*eta, P) are
// the state-independent products of the chunk, prepared one chunk ahead.
//
// Warp roles (512 threads = four warpgroups, one CTA per SM):
//   warps 0-7   prep: gate products, the seven bf16 operands, [A/beta ; P] (one
//               tcgen05 MMA), the triangular solve, Tb; one of its threads issues
//               its MMAs.  Works on chunk c+1 while the state chain runs chunk c.
//   warps 8-11  the state chain, warp 8+q owning TMEM lane quarter q: the bf16 copy
//               and decay of S^T, V - Z, U, and O^T out to global memory (through a
//               staging tile and TMA stores; a partial last chunk row by row).
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

// Optional event hook for timing builds: (role, chunk, event) by one thread of the
// role (no-op in the library).
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
constexpr uint32_t STAGE = 16384;              // per-parity stride of the k, q, alpha stages
constexpr uint32_t OFF_K = 0;                  // k tile [64 j][128 c] x 2 stages -> k*gamma in place
constexpr uint32_t OFF_Q = 32768;              // q tile x 2 stages -> q*gamma in place
constexpr uint32_t OFF_A = 65536;              // alpha tile x 2 stages -> k*eta in place
constexpr uint32_t OFF_V = 98304;              // v tile [64 j][128 n]
constexpr uint32_t OFF_X = 114688;             // prep work region, 56 KB (below)
constexpr uint32_t OFF_P = 172032;             // P [64 r][64 j] x 2 stages
constexpr uint32_t OFF_TB = 188416;            // Tb [64 j][64 j'] x 2 stages
constexpr uint32_t OFF_OST = 204800;           // O staging tile [64 r][128 n] (TMA store box layout)
constexpr uint32_t OFF_MISC = 221184;
constexpr uint32_t MISC_PI = 0;                // float [8][128] octant gate products
constexpr uint32_t MISC_GC = 4096;             // float [2][128] gamma_C per stage
constexpr uint32_t MISC_BETA = 5120;           // float [2][64] beta per stage
constexpr uint32_t MISC_BAR = 5632;            // mbarriers (enum below)
constexpr uint32_t MISC_TMEM = 5760;
constexpr uint32_t MISC_FLAG = 5764;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 5888 + 1024;   // + alignment slack

// prep work region: the operands of [A/beta ; P], then (after that MMA) the solve
constexpr uint32_t X_L = 0;        // [k*lam ; q*lam] [128][128] (two [128][64] atoms)
constexpr uint32_t X_R = 32768;    // [k*rho^0 (32 rows) ; k*rho^1 (64 rows)] (two [96][64] atoms)
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
    B_RU = 10,        //                 (V - Z)^T written, issue U^T
    B_R3 = 11,        //                 U^T written, issue the state update and O^T += U^T P^T
    B_BZ = 12,        // issuer -> state: Z^T done
    B_BU = 13,        //                  U^T done
    B_BS = 14,        //                  state update and O^T done
    NBAR = 15
};

// TMEM columns
constexpr uint32_t TS = 0;      // S^T fp32 [128 n][128 c]
constexpr uint32_t TSB = 128;   // S^T bf16 pairs (64 columns)
constexpr uint32_t TZ = 192;    // Z^T, then U^T, fp32 (64 columns)
constexpr uint32_t TO = 256;    // O^T fp32 (64 columns)
constexpr uint32_t TVB = 320;   // (V - Z)^T bf16 pairs (32 columns)
constexpr uint32_t TUB = 352;   // U^T bf16 pairs (32 columns)
constexpr uint32_t TP = 384;    // prep: [A/beta ; P] (96 columns), then the tf32 solve products

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
                     const __grid_constant__ CUtensorMap tmO, const __nv_bfloat16* __restrict__ beta, const float* S0,
                     const int32_t* __restrict__ cu_seqlens, __nv_bfloat16* __restrict__ out,
                     float* S_final, int64_t T, int H, int* status, const Segments seg) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    uint8_t* sK = sm + OFF_K;
    uint8_t* sQ = sm + OFF_Q;
    uint8_t* sAl = sm + OFF_A;
    uint8_t* sV = sm + OFF_V;
    uint8_t* sX = sm + OFF_X;
    uint8_t* sP = sm + OFF_P;
    uint8_t* sTB = sm + OFF_TB;
    uint8_t* sOst = sm + OFF_OST;
    float* sPi = reinterpret_cast<float*>(sm + OFF_MISC + MISC_PI);
    float* sGC = reinterpret_cast<float*>(sm + OFF_MISC + MISC_GC);
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
                tma_load_2d(sK + s * STAGE + a * 8192, &tmK, bar + B_FULL + s, h * DK + 64 * a, row0);
                tma_load_2d(sQ + s * STAGE + a * 8192, &tmQ, bar + B_FULL + s, h * DK + 64 * a, row0);
                tma_load_2d(sAl + s * STAGE + a * 8192, &tmA, bar + B_FULL + s, h * DK + 64 * a, row0);
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
        constexpr uint32_t id64 = idesc_bf16(128, 64);                  // both operands K-major
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
            KDA_TC2_MARK(2, c, 0);
            {
                const uint32_t kg = smem_u32(sK + s * STAGE);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16_ts(tmem + TZ, tmem + TSB + 8 * ks,
                                sdesc_sw128(kg + (ks >> 2) * 8192 + (ks & 3) * 32), id64, ks > 0);
                commit(B_BZ, ph);
            }
            // O^T = S^T (q*gamma)^T, once the previous chunk's O^T is read out
            if (!wait_bar(B_RQ, ph)) break;
            tc_fence_after();
            KDA_TC2_MARK(2, c, 1);
            {
                const uint32_t qg = smem_u32(sQ + s * STAGE);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16_ts(tmem + TO, tmem + TSB + 8 * ks,
                                sdesc_sw128(qg + (ks >> 2) * 8192 + (ks & 3) * 32), id64, ks > 0);
            }
            // U^T = (V - Z)^T Tb^T; the v tile is free again
            if (!wait_bar(B_RU, ph)) break;
            tc_fence_after();
            KDA_TC2_MARK(2, c, 2);
            {
                const uint32_t tb = smem_u32(sTB + s * 8192);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ts(tmem + TZ, tmem + TVB + 8 * ks, sdesc_sw128(tb + ks * 32), id64, ks > 0);
                commit(B_BU, ph);
            }
            if (c + 1 < nchunks) issue_v(c + 1);
            // S^T += U^T (k*eta) (S^T already decayed) and O^T += U^T P^T
            if (!wait_bar(B_R3, ph)) break;
            tc_fence_after();
            KDA_TC2_MARK(2, c, 3);
            {
                const uint32_t kh = smem_u32(sAl + s * STAGE), p0 = smem_u32(sP + s * 8192);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ts(tmem + TS, tmem + TUB + 8 * ks, sdesc_sw128(kh + ks * 2048, 1024, 8192),
                                id128mn, 1);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ts(tmem + TO, tmem + TUB + 8 * ks, sdesc_sw128(p0 + ks * 32), id64, 1);
                commit(B_EMPTY + s, (uint32_t)(c >> 1) & 1u);
                commit(B_BS, ph);
            }
            // the stage is free once these MMAs complete: load chunk c + 2 into it
            if (c + 2 < nchunks) {
                if (!wait_bar(B_EMPTY + s, (uint32_t)(c >> 1) & 1u)) break;
                KDA_TC2_MARK(2, c, 4);
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
            uint8_t* sKc = sK + s * STAGE;
            uint8_t* sQc = sQ + s * STAGE;
            uint8_t* sAc = sAl + s * STAGE;
            float* sBeta_s = sBeta + 64 * s;
            float* sGC_s = sGC + 128 * s;
            if (tid < C) sBeta_s[tid] = beta_next;
            if (tid == 0) KDA_TC2_MARK(0, c, 0);
            wait_bar(B_FULL + s, (uint32_t)(c >> 1) & 1u);
            if (tid == 0) KDA_TC2_MARK(0, c, 1);

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
                // one token row of all 128 channels (8 bytes per thread).
                const int cq = tid & 31, O = tid >> 5, Q = O >> 1, c0 = 4 * cq;
                const uint32_t chk = (uint32_t)((c0 & 63) >> 3), inner = (uint32_t)((c0 & 7) << 1);
                const uint32_t a64 = (uint32_t)(c0 >> 6);
                auto in_off_of = [&](int r) {
                    return a64 * 8192u + (uint32_t)r * 128u + (((chk ^ (uint32_t)r) & 7u) << 4) + inner;
                };
                float phi[8][4], psi[8][4];   // psi holds the clamped gates until the backward pass
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = 8 * O + i;
                    float a[4];
                    unpack4_bf16(*reinterpret_cast<const uint2*>(sAc + in_off_of(r)), a);
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc)
                        psi[i][cc] = r < Lc ? clamp_gate(fused ? gate_from_logit(a[cc]) : a[cc]) : 1.0f;
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
                if (tid == 0) KDA_TC2_MARK(0, c, 2);
                prep_bar();
                if (tid == 0) KDA_TC2_MARK(0, c, 3);
                // per-thread scales: quarter products, gamma before / eta after this quarter
                float dlf[4], bf[4], r0g[4], r1g[4], ag[4];
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
                        if (O == 0) sGC_s[c0 + cc] = pq[0][cc] * pq[1][cc] * pq[2][cc] * pq[3][cc];
                        const float fO = (O & 1) ? pov[cc] : 1.0f;
                        const float gO = (O & 1) ? 1.0f : pov[cc];
                        const float dl = (Q & 1) ? 1.0f : __frcp_rn(own);
                        const float r0 = Q == 1 ? __frcp_rn(own) : 1.0f;
                        const float r1 = Q == 0 ? pq[1][cc] * pq[2][cc]
                                                : (Q == 1 ? pq[2][cc] : (Q == 2 ? 1.0f : __frcp_rn(own)));
                        dlf[cc] = dl * fO;
                        bf[cc] = bef * fO;
                        r0g[cc] = r0 * gO;
                        r1g[cc] = r1 * gO;
                        ag[cc] = aft * gO;
                    }
                }
                // fused inputs: k and q rows L2-normalised in place (bf16), before any
                // operand is formed.  A warp holds all 128 channels of its eight rows, four
                // per lane, and each thread rewrites only the elements it reads again below.
                if constexpr (kFused) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int r = 8 * O + i;
                        const uint32_t in_off = in_off_of(r);
                        float k[4], q[4];
                        unpack4_bf16(*reinterpret_cast<const uint2*>(sKc + in_off), k);
                        unpack4_bf16(*reinterpret_cast<const uint2*>(sQc + in_off), q);
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
                        st4_bf16(sKc + in_off, k);
                        st4_bf16(sQc + in_off, q);
                    }
                }
                // each row's k and q are read before the previous row's stores: k*gamma,
                // q*gamma and k*eta are written in place, so a load placed after a store
                // could not be moved above it
                uint2 kn = *reinterpret_cast<const uint2*>(sKc + in_off_of(8 * O));
                uint2 qn = *reinterpret_cast<const uint2*>(sQc + in_off_of(8 * O));
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = 8 * O + i;
                    const uint32_t sw = (uint32_t)r * 128u + (((chk ^ (uint32_t)r) & 7u) << 4) + inner;
                    const uint32_t in_off = a64 * 8192u + sw;    // 64-row tiles: q, k, alpha
                    float k[4], q[4];
                    unpack4_bf16(kn, k);
                    unpack4_bf16(qn, q);
                    if (i < 7) {
                        kn = *reinterpret_cast<const uint2*>(sKc + in_off_of(r + 1));
                        qn = *reinterpret_cast<const uint2*>(sQc + in_off_of(r + 1));
                    }
                    if (r >= Lc) {
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) { k[cc] = 0.0f; q[cc] = 0.0f; }
                    }
                    float kp[4], qp[4], ks[4], w[4];
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        kp[cc] = k[cc] * phi[i][cc];
                        qp[cc] = q[cc] * phi[i][cc];
                        ks[cc] = k[cc] * psi[i][cc];
                    }
                    uint8_t* lrow = sX + X_L + a64 * 16384u + sw;             // 128-row atoms
                    uint8_t* rrow = sX + X_R + a64 * 12288u + sw;             // 96-row atoms
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) w[cc] = kp[cc] * dlf[cc];
                    st4_bf16(lrow, w);                                        // k*lam, row r
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) w[cc] = qp[cc] * dlf[cc];
                    st4_bf16(lrow + 64 * 128, w);                             // q*lam, row 64 + r
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) w[cc] = qp[cc] * bf[cc];
                    st4_bf16(sQc + in_off, w);                                // q*gamma in place
                    if (O < 4) {
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) w[cc] = ks[cc] * r0g[cc];
                        st4_bf16(rrow, w);                                    // k*rho^0, row r < 32
                    }
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) w[cc] = ks[cc] * r1g[cc];
                    st4_bf16(rrow + 32 * 128, w);                             // k*rho^1, row 32 + r
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) w[cc] = kp[cc] * bf[cc];
                    st4_bf16(sKc + in_off, w);                                // k*gamma in place
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) w[cc] = ks[cc] * ag[cc];
                    st4_bf16(sAc + in_off, w);                                // k*eta over alpha
                }
                if (tid == 0) KDA_TC2_MARK(0, c, 4);
            }
            fence_async_smem();
            tc_fence_before();
            prep_bar();
            tc_fence_after();
            if (tid == 0) KDA_TC2_MARK(0, c, 5);

            // ================= [A/beta ; P] = [k*lam ; q*lam] [k*rho^0 ; k*rho^1]^T   (M=128, N=96, K=128)
            //   rows 0..63 are A/beta rows r, rows 64..127 are P rows r.  Columns [0, 32) hold
            //   rho^0 (j < 32, valid for r < 32), columns [32, 96) hold rho^1 (j < 64, valid for r >= 32).
            if (tid == 0 && ok) {
                const uint32_t l0 = smem_u32(sX + X_L), r0 = smem_u32(sX + X_R);
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
            if (tid == 0) KDA_TC2_MARK(0, c, 6);

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
                if (tid == 0) KDA_TC2_MARK(0, c, 7);
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
            if (tid == 0) KDA_TC2_MARK(0, c, 8);
            // beta of the next chunk, while the solve runs
            if (tid < C) {
                const int64_t nxt = (int64_t)(c + 1) * C + tid;   // token index in the segment
                beta_next = (c + 1 < nchunks && nxt < len) ? load_beta(nxt) : 0.0f;
            }
            fence_async_smem();
            tc_fence_before();
            prep_bar();
            tc_fence_after();

            // ================= Tinv = (I + A)^-1 by doubling: 16x16 blocks, then 32, then 64
            //   inv([[X, 0], [Y, Z]]) = [[X^-1, 0], [-Z^-1 Y X^-1, Z^-1]]
            {
                if (tid == 0) KDA_TC2_MARK(0, c, 9);
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
                }
                prep_bar();
                if (tid == 0) KDA_TC2_MARK(0, c, 10);
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
                if (tid == 0) KDA_TC2_MARK(0, c, 11);
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
                if (tid == 0) KDA_TC2_MARK(0, c, 12);
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
                if (tid == 0) KDA_TC2_MARK(0, c, 13);
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
            if (tid == 0) KDA_TC2_MARK(0, c, 14);
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
        // O^T of chunk c from TMEM to out[row0 + r][h][n].  A full chunk goes through the
        // staging tile (thread n writes column n of the row-major, 128-byte swizzled box;
        // a warp's 32 columns of one row are 64 contiguous bytes) and two TMA stores
        // issued by the elected thread; a partial last chunk is stored row by row.
        bool ost_pending = false;   // (elected) a TMA store may still be reading the tile
        auto store_o = [&](int c) {
            const int Lc = chunk_len(c);
            const int64_t row0 = bos + (int64_t)c * C;
            if (Lc == C) {
                // the previous store has read the tile (elected waits, the barrier publishes)
                if (elected && ost_pending) bulk_wait_read_all();
                state_bar();
                const uint32_t ocol = (uint32_t)(nn >> 6) * 8192u + (uint32_t)(nn & 7) * 2u;
                const uint32_t ochk = (uint32_t)((nn & 63) >> 3);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t r[32];
                    tmem_ld32(tmem + tlane + TO + 32 * half, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const uint32_t rr = (uint32_t)(32 * half + i);
                        *reinterpret_cast<__nv_bfloat16*>(sOst + ocol + rr * 128u + (((ochk ^ rr) & 7u) << 4)) =
                            __float2bfloat16_rn(u2f(r[i]));
                    }
                }
                fence_async_smem();
                state_bar();
                if (elected) {
#pragma unroll
                    for (int a = 0; a < 2; ++a) tma_store_2d(&tmO, sOst + a * 8192, h * DV + 64 * a, (int)row0);
                    bulk_commit_group();
                    ost_pending = true;
                }
            } else {
                __nv_bfloat16* dst = out + ((size_t)row0 * H + h) * DV + nn;
                const size_t rs = (size_t)H * DV;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t r[32];
                    tmem_ld32(tmem + tlane + TO + 32 * half, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (32 * half + i < Lc) dst[(size_t)(32 * half + i) * rs] = __float2bfloat16_rn(u2f(r[i]));
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
            if (elected) KDA_TC2_MARK(1, c, 0);
            // ---- S^T to bf16 (the A operand of this chunk's products), and S^T <- S^T Diag(gamma_C)
            if (ok) {
                const float* g = sGC + 128 * s;
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    uint32_t r[32];
                    tmem_ld32(tmem + tlane + TS + 32 * p, r);
                    tmem_wait_ld();
                    uint32_t b[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) b[i] = pack_bf16x2(u2f(r[2 * i]), u2f(r[2 * i + 1]));
                    tmem_st16u(tmem + tlane + TSB + 16 * p, b);
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        const float4 gg = *reinterpret_cast<const float4*>(g + 32 * p + i);
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
            if (elected) KDA_TC2_MARK(1, c, 1);
            // ---- the previous chunk's O^T leaves while Z^T is computed
            if (c > 0) store_o(c - 1);
            tc_fence_before();
            state_bar();
            if (elected) mbar_arrive(bar + B_RQ);
            if (elected) KDA_TC2_MARK(1, c, 2);
            // ---- (V - Z)^T: column n of the v tile minus row n of Z^T, as bf16 pairs
            wait_bar(B_VFULL, ph);
            wait_bar(B_BZ, ph);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
            if (elected) KDA_TC2_MARK(1, c, 3);
            if (ok) {
                const uint32_t vcol = (uint32_t)(nn >> 6) * 8192u + (uint32_t)(nn & 7) * 2u;
                const uint32_t vchk = (uint32_t)((nn & 63) >> 3);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t z[32];
                    tmem_ld32(tmem + tlane + TZ + 32 * half, z);
                    tmem_wait_ld();
                    uint32_t b[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const uint32_t j0 = (uint32_t)(32 * half + 2 * i), j1 = j0 + 1;
                        const float v0 = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                            sV + vcol + j0 * 128u + (((vchk ^ j0) & 7u) << 4)));
                        const float v1 = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                            sV + vcol + j1 * 128u + (((vchk ^ j1) & 7u) << 4)));
                        b[i] = pack_bf16x2(v0 - u2f(z[2 * i]), v1 - u2f(z[2 * i + 1]));
                    }
                    tmem_st16u(tmem + tlane + TVB + 16 * half, b);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            state_bar();
            if (elected) mbar_arrive(bar + B_RU);
            if (elected) KDA_TC2_MARK(1, c, 4);
            // ---- U^T as bf16 pairs
            wait_bar(B_BU, ph);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
            if (elected) KDA_TC2_MARK(1, c, 5);
            if (ok) {
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t u[32];
                    tmem_ld32(tmem + tlane + TZ + 32 * half, u);
                    tmem_wait_ld();
                    uint32_t b[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) b[i] = pack_bf16x2(u2f(u[2 * i]), u2f(u[2 * i + 1]));
                    tmem_st16u(tmem + tlane + TUB + 16 * half, b);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            if (named_bar_or(2, NSTATE, !ok || *sFlag != 0)) { broke = true; break; }
            if (elected) mbar_arrive(bar + B_R3);
            if (elected) KDA_TC2_MARK(1, c, 6);
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
        if (elected && ost_pending) bulk_wait_all();   // every O store has completed
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
        m.q, m.k, m.a, m.v, m.o, (const __nv_bfloat16*)beta, S0, cu, (__nv_bfloat16*)out, S_final, T, H,
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
